// Wave-round block-causal attention: every active (chunk, level) node of one
// round in ONE persistent kernel launch on sm_100a.
//
// What it computes (Wave Forcing page, "Key Findings"; design-space paper,
// Table 1 / Figure 1; Wan-Streamer v0.2 page, glossary "block-causal
// attention"): for node (c, l) and head h,
//   O[q, h] = softmax_k(Q[q, h] . K[k, h] / sqrt(d)) V[k, h]
// over the tokens of the node's key list (prefix, history E(c-r, phi(l, r)),
// own E(c, l)) -- full attention inside every listed chunk, nothing else.
//
// How (B200 design, not the pages'): one CTA per SM, each claiming work items
// (node, head, pair of 128-query tiles) longest key list first from a global
// counter; query tiles of one head are adjacent, so concurrent CTAs share that
// head's K/V pages in L2. Per CTA (384 threads):
//   warp 0   TMA producer: both Q tiles once per item, then each 128-token K
//            and V page of the key list, gathered by page id (the tensor-map
//            row coordinate), into a 5-slot (d = 64: 10-slot) shared ring.
//   warps 1, 3  tcgen05 issuers, one per query tile w: S = Q_w K^T (both
//            operands in shared memory, 128-byte swizzle, K-major) into the
//            one TMEM S buffer, then O_w += P_w V with P_w read from TMEM
//            (bf16, its own 64 columns) and V from shared memory (MN-major).
//            Pipe order per page t: S_0(t), PV_0(t-1), S_1(t), PV_1(t-1): the
//            S buffer is reloaded while the P.V behind it runs, and a tile's
//            P(t) is needed only after the next page's S. Two issuing threads
//            keep the tensor pipe's short queue fed while either one waits;
//            they do nothing but wait for S_FREE / P_FULL, issue and commit
//            (a tcgen05.mma call returns only about when the pipe takes it,
//            so every other step on these threads delays the pipe).
//   warps 4-11  softmax, one warpgroup per query tile, one row per thread:
//            tcgen05.ld of the S row (then S is handed back), padding keys of
//            a partial page masked, max in the log2 domain, exp2, bf16 P
//            written to P_w with tcgen05.st. O is rescaled only when the
//            running max grows by more than 8 (log2 units); otherwise the
//            stale max is kept, exact after the final division as P <= 2^8
//            stays inside fp32/bf16. Epilogue: O / l, bf16, stored straight
//            from registers (only rows that belong to the node).
//   warp 2   ring watcher: takes part in every S_FREE and P_FULL phase,
//            arriving once the pages the MMAs behind it read have landed
//            (K(t+1) for the S_FREE that lets S_0(t+1) go, V(t) for P_FULL),
//            and gives each K slot back once the page's last S has been
//            loaded (V slots go back by a commit behind each P.V), so neither
//            the issuers nor the softmax do any ring work.
// A node's last pair of query tiles may hold one tile. Thread 1 skips such a
// single-tile item while its S tiles advance S_FREE_0; an mbarrier parity wait
// is only sound for the phase right after the last one its waiter saw, so
// before its next S thread 1 waits (bounded) until the watcher's count of
// pages whose last S has been loaded covers the skipped pages.
// Every wait is bounded (by default 2 s; wave_kv_set_wait_limit); on timeout
// the kernel records a status word, every role stops, and TMEM is freed
// before exit.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <numeric>
#include <vector>

#include "exp2_poly.h"
#include "ptx.cuh"
#include "wave_internal.h"
#include "wave_sync.cuh"

using namespace wptx;

namespace wavei {

namespace {

constexpr int kThreads = 384;  // warp 0 TMA, 1 and 3 MMA, 2 ring watcher, 4..11 softmax
// Register split after start-up (setmaxnreg): warps 0..3 (the TMA producer,
// the two MMA issuers and the ring watcher; one per SM sub-partition) drop to
// kRegsLow, the two softmax warpgroups (two
// warps per sub-partition) rise to kRegsHigh, so each softmax thread can hold
// a full 128-column S row without spilling. Per sub-partition
// kRegsLow + 2 kRegsHigh <= 504 registers per lane, i.e. at most what the
// launch holds at 168 per thread; the host refuses to launch a build compiled
// with fewer.
#ifndef WAVE_REGS_LOW
#define WAVE_REGS_LOW 72
#endif
#ifndef WAVE_REGS_HIGH
#define WAVE_REGS_HIGH 216
#endif
constexpr uint32_t kRegsLow = WAVE_REGS_LOW, kRegsHigh = WAVE_REGS_HIGH, kRegsLaunch = 168;
static_assert(128 * kRegsLow + 256 * kRegsHigh <= kThreads * kRegsLaunch, "register split");
constexpr uint32_t kPageMask = (1u << 25) - 1;  // page id bits of a page word
constexpr int64_t kCounterOffset = 128;         // work-queue counter in the pool header

struct AttnNode {
  int32_t q_row0;    // first row of this node in Q / O
  int32_t page0;     // first page word
  int32_t n_pages;   // key pages
  int32_t item0;     // first work item
  int32_t n_pairs;   // ceil(n_qtiles / 2): pairs of 128-row query tiles
  int32_t n_qtiles;  // ceil(T / 128)
  int32_t n_splits;  // key ranges per (head, pair); > 1: partial results
};

struct AttnParams {
  CUtensorMap tm_q;   // Q as [rows][H][d]
  CUtensorMap tm_kv;  // pool page region as rows of d
  uint16_t* out;      // O, bf16 [rows][H][d]
  int32_t* status;    // device status word (pool header)
  int32_t* counter;   // work-queue counter, zero at launch (pool header)
  int64_t* clock_out; // CTA 0's SM cycles and nanoseconds (pool header)
  float* part_o;      // split key ranges: unnormalised O per (item, tile, row), fp32
  float* part_ml;     // ... and the row's (running max, sum), fp32
  uint64_t wait_ns;   // bound on one barrier wait
  float scale_log2;   // log2(e) / sqrt(d)
  int32_t heads;
  int32_t n_nodes;
  int32_t n_items;
  int32_t q_rows;     // T: query rows per node
  int32_t pad;
  AttnNode nodes[WAVE_MAX_NODES];
  uint32_t pages[WAVE_MAX_PAGES_PER_ROUND];  // page id | (valid - 1) << 25
};
static_assert(sizeof(AttnParams) <= 32760, "kernel parameter space is 32 KB");

// Softmax columns (of each 32) whose exp2 runs on the FMA pipe (polynomial)
// instead of the special-function unit; even, 0..32. Two: measured against
// 0, 4, 6 and 8, it took the fewest cycles per launch (8 about 4 % more).
#ifndef WAVE_EMU_PER_CHUNK
#define WAVE_EMU_PER_CHUNK 2
#endif
constexpr int kEmuPerChunk = WAVE_EMU_PER_CHUNK;
// 1: scale/shift of S and the row sum use packed fp32x2 FMA/ADD.
#ifndef WAVE_PACKED_FMA
#define WAVE_PACKED_FMA 1
#endif
static_assert(kEmuPerChunk % 2 == 0 && kEmuPerChunk >= 0 && kEmuPerChunk <= 32, "emulated share");

template <int D>
struct Cfg {
  static constexpr int kPanels = D / 64;           // 64-column, 128-byte-wide panels
  static constexpr int kPanelBytes = 128 * 128;    // 128 rows x 128 bytes
  static constexpr int kTileBytes = 128 * D * 2;   // one Q, K or V tile
  static constexpr int kSlots = D == 128 ? 5 : 10; // K/V ring slots (K and V alternate)
  static constexpr int kQOff = 0;                  // Q0, then Q1
  static constexpr int kRingOff = 2 * kTileBytes;
  static constexpr int kBarOff = kRingOff + kSlots * kTileBytes;
  static constexpr int kSmemBytes = kBarOff + 512 + 1024;  // + barriers + alignment slack
  // TMEM columns: one S buffer (fp32, 128 keys) that the two query tiles
  // take in turn, P_w (bf16x2, 64 columns) at 128 + 64 w, O_w at 256 + 128 w.
  // S is free again as soon as its softmax warpgroup has loaded it, so the next
  // S = Q K^T need not wait for the previous P.V: the softmax of a tile has a
  // whole page period of MMAs (both tiles' S and P.V) to hide in.
  static constexpr uint32_t kColS = 0, kColP = 128, kColO = 256, kCols = 512;
  // Instruction descriptors (kind::f16): fp32 accumulate, bf16 A and B, M = 128.
  static constexpr uint32_t kIdescS = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) |
                                      ((128u >> 4) << 24);
  static constexpr uint32_t kIdescO = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                      ((uint32_t(D) >> 3) << 17) | ((128u >> 4) << 24);
};

// Barrier slots (8 bytes each) after the tiles.
enum : int {
  B_Q_FULL = 0,
  B_Q_EMPTY,
  B_S_FULL,                  // 2: S = Q_w K^T computed into the S buffer
  B_S_FREE = B_S_FULL + 2,   // 2: softmax w has loaded S (4 warp arrivals + the watcher)
  B_P_FULL = B_S_FREE + 2,   // 2: P_w written (4 warp arrivals + the watcher)
  B_P_FREE = B_P_FULL + 2,   // 2: the P.V that read P_w is done
  B_O_FULL = B_P_FREE + 2,   // 2: last P.V of an item done
  B_O_EMPTY = B_O_FULL + 2,  // 2: epilogue has read O_w (128 arrivals)
  B_DRAIN = B_O_EMPTY + 2,   // 2: every MMA of MMA thread w done (while stopping)
  B_ITEM_FULL = B_DRAIN + 2, // 2: next work item published by the producer
  B_ITEM_EMPTY = B_ITEM_FULL + 2,  // 2: item read by 2 MMA threads, the watcher, 8 softmax warps
  B_RING_FULL = B_ITEM_EMPTY + 2,  // kSlots each from here
};
constexpr int kItemSlots = 2;
constexpr int kItemWords = 8;  // an Item as published in the shared-memory queue

template <int D>
struct Bars {
  static constexpr int kS = Cfg<D>::kSlots;
  static constexpr int RING_FULL = B_RING_FULL, RING_EMPTY = RING_FULL + kS,
                       COUNT = RING_EMPTY + kS;
  static_assert(COUNT * 8 + 16 + 4 * kItemWords * kItemSlots + 4 <= 448, "barrier area");  // 448..: clock
};

// A work item: (node, head, pair of 128-row query tiles, key range). The
// producer decodes it once and publishes these fields to the other roles.
struct Item {
  int id, node, head, pair, two, page_begin, n_pages, split;
};

__device__ __forceinline__ Item decode_item(const AttnParams& p, int item) {
  int n = 0;
  while (n + 1 < p.n_nodes && item >= p.nodes[n + 1].item0) ++n;
  const AttnNode& nd = p.nodes[n];
  const int j = item - nd.item0;
  const int ns = nd.n_splits;
  const int split = j % ns, hp = j / ns;  // key ranges of one (head, pair) are adjacent
  const int pair = hp % nd.n_pairs;
  const int base = nd.n_pages / ns, extra = nd.n_pages % ns;
  return Item{item, n, hp / nd.n_pairs, pair, 2 * pair + 1 < nd.n_qtiles ? 1 : 0,
              split * base + min(split, extra), base + (split < extra ? 1 : 0), split};
}

// 2^x for a pair of x <= 8 on the FMA pipe: x = j + f, j = round(x),
// |f| <= 1/2, 2^f from the minimax cubic of exp2_poly.h, 2^j added to the
// exponent field. Inputs below -126 (including -inf) are clamped there, giving
// at most 2^-126 -- negligible against a row sum >= 1.
__device__ __forceinline__ void exp2_poly2(float x0, float x1, float& y0, float& y1) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23: adding it rounds to an integer
  x0 = fmaxf(x0, -126.f);
  x1 = fmaxf(x1, -126.f);
  const uint64_t x = f2_pack(x0, x1);
  const uint64_t t = f2_add(x, f2_pack(kRound, kRound));
  const uint64_t jf = f2_add(t, f2_pack(-kRound, -kRound));
  const uint64_t f = f2_fma(jf, f2_pack(-1.f, -1.f), x);
  uint64_t p = f2_fma(f2_pack(WAVE_EXP2_C3, WAVE_EXP2_C3), f, f2_pack(WAVE_EXP2_C2, WAVE_EXP2_C2));
  p = f2_fma(p, f, f2_pack(WAVE_EXP2_C1, WAVE_EXP2_C1));
  p = f2_fma(p, f, f2_pack(WAVE_EXP2_C0, WAVE_EXP2_C0));
  float p0, p1, t0, t1;
  f2_unpack(p, p0, p1);
  f2_unpack(t, t0, t1);
  // The low mantissa bits of t hold j (two's complement); shifting them into
  // the exponent field scales p by 2^j.
  y0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
  y1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    round_attn_kernel(const __grid_constant__ AttnParams p) {
  using C = Cfg<D>;
  using BR = Bars<D>;
  constexpr int S = C::kSlots;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_addr(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + C::kBarOff + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kBarOff + 8 * BR::COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kBarOff + 8 * BR::COUNT + 4);
  volatile int* item_q = reinterpret_cast<volatile int*>(smem + C::kBarOff + 8 * BR::COUNT + 8);
  // Pages whose last S has been loaded, as the watcher saw them (monotonic).
  volatile uint32_t* s_done = reinterpret_cast<volatile uint32_t*>(
      smem + C::kBarOff + 8 * BR::COUNT + 8 + 4 * kItemWords * kItemSlots);
  const Ctl ctl{abort_flag, p.status, p.wait_ns};

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // CTA 0 times itself in SM cycles and in nanoseconds (start kept in shared
  // memory): their ratio is the SM clock the launch actually ran at.
  volatile int64_t* clock_start = reinterpret_cast<volatile int64_t*>(smem + C::kBarOff + 448);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    clock_start[0] = clock64();
    clock_start[1] = (int64_t)globaltimer_ns();
  }

  if (threadIdx.x == 0) {
    mbar_init(bar(B_Q_FULL), 1);
    mbar_init(bar(B_Q_EMPTY), 1);
    for (int w = 0; w < 2; ++w) {
      mbar_init(bar(B_S_FULL + w), 1);
      mbar_init(bar(B_S_FREE + w), 5);  // the warpgroup's 4 warps + the ring watcher
      mbar_init(bar(B_P_FULL + w), 5);
      mbar_init(bar(B_P_FREE + w), 1);
      mbar_init(bar(B_O_FULL + w), 1);
      mbar_init(bar(B_O_EMPTY + w), 128);
    }
    for (int k = 0; k < kItemSlots; ++k) {
      mbar_init(bar(B_ITEM_FULL + k), 1);
      mbar_init(bar(B_ITEM_EMPTY + k), 3 + 8);  // MMA threads, watcher, one lane per softmax warp
    }
    mbar_init(bar(B_DRAIN), 1);
    mbar_init(bar(B_DRAIN + 1), 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(bar(BR::RING_FULL + s), 1);
      mbar_init(bar(BR::RING_EMPTY + s), 2);  // K: one arrival of 2; V: a commit per tile
    }
    *abort_flag = 0;
    *s_done = 0;
    fence_mbar_init();
    prefetch_tmap(&p.tm_q);
    prefetch_tmap(&p.tm_kv);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), C::kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int H = p.heads;

  // Work items, longest key list first, are handed out dynamically: the
  // producer claims the next one (the CTA's first is blockIdx.x, later ones
  // come from a global counter) and publishes it to the other roles through a
  // two-slot queue in shared memory. An id >= n_items tells every role to stop.
  auto next_item = [&](uint32_t k, int code, Item& w) -> bool {  // consumer side
    if (!wait_bar(bar(B_ITEM_FULL + (k % kItemSlots)), (k / kItemSlots) & 1, ctl, code))
      return false;
    const volatile int* q = item_q + kItemWords * (k % kItemSlots);
    w = Item{q[0], q[1], q[2], q[3], q[4], q[5], q[6], q[7]};
    return true;
  };

  if (warp < 4) {
    regs_dec<kRegsLow>();
    if (warp == 0) {
      // ---------------------------------------------------------- TMA producer
      if (lane == 0) {
        uint32_t r = 0, it = 0;  // ring sequence (K(g) = 2g, V(g) = 2g + 1), item count
        // Phase of the newest copy issued on each full barrier (-1: none yet),
        // so that an early stop can wait for copies still in flight.
        int q_last = -1, ring_last[S];
        for (int s = 0; s < S; ++s) ring_last[s] = -1;
        bool ok = true;
        for (uint32_t k = 0; ok; ++k) {
          const int slot = k % kItemSlots;
          if (k >= (uint32_t)kItemSlots &&
              !wait_bar(bar(B_ITEM_EMPTY + slot), ((k / kItemSlots) & 1) ^ 1, ctl, 0x100)) {
            ok = false;
            break;
          }
          const int item = k == 0 ? (int)blockIdx.x : (int)gridDim.x + atomicAdd(p.counter, 1);
          Item w{item, 0, 0, 0, 0, 0, 0, 0};
          if (item < p.n_items) w = decode_item(p, item);
          volatile int* q = item_q + kItemWords * slot;
          q[0] = w.id; q[1] = w.node; q[2] = w.head; q[3] = w.pair;
          q[4] = w.two; q[5] = w.page_begin; q[6] = w.n_pages; q[7] = w.split;
          mbar_arrive(bar(B_ITEM_FULL + slot));
          if (item >= p.n_items) break;
          const AttnNode& nd = p.nodes[w.node];
          if (it > 0 && !wait_bar(bar(B_Q_EMPTY), (it - 1) & 1, ctl, 0x101)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(B_Q_FULL), (w.two ? 2 : 1) * C::kTileBytes);
          for (int q = 0; q < (w.two ? 2 : 1); ++q)
            for (int pn = 0; pn < C::kPanels; ++pn)
              tma_load_3d(sbase + C::kQOff + q * C::kTileBytes + pn * C::kPanelBytes, &p.tm_q,
                          pn * 64, w.head, nd.q_row0 + (2 * w.pair + q) * 128, bar(B_Q_FULL));
          q_last = it & 1;
          ++it;
          for (int t = 0; ok && t < w.n_pages; ++t) {
            const uint32_t page = p.pages[nd.page0 + w.page_begin + t] & kPageMask;
            const int32_t yk = (int32_t)(((int64_t)page * 2 * H + w.head) * 128);
            for (int kv = 0; kv < 2; ++kv, ++r) {
              const int s = r % S;
              const uint32_t ph = (r / S) & 1;
              if (r >= (uint32_t)S && !wait_bar(bar(BR::RING_EMPTY + s), ph ^ 1, ctl, 0x102)) {
                ok = false;
                break;
              }
              mbar_arrive_expect_tx(bar(BR::RING_FULL + s), C::kTileBytes);
              for (int pn = 0; pn < C::kPanels; ++pn)
                tma_load_2d(sbase + C::kRingOff + s * C::kTileBytes + pn * C::kPanelBytes,
                            &p.tm_kv, pn * 64, yk + kv * H * 128, bar(BR::RING_FULL + s));
              ring_last[s] = (int)ph;
            }
          }
        }
        if (!ok) {
          // Stopping early: let the copies already issued land before the
          // CTA's shared memory is released.
          if (q_last >= 0) drain_wait(bar(B_Q_FULL), (uint32_t)q_last);
          for (int s = 0; s < S; ++s)
            if (ring_last[s] >= 0) drain_wait(bar(BR::RING_FULL + s), (uint32_t)ring_last[s]);
        }
      }
    } else if (warp == 2) {
      // ---------------------------------------------------------- ring watcher
      // Takes part in every S_FREE and P_FULL phase, in order, arriving only
      // once the ring slots the MMAs behind that phase read have landed:
      // K(t+1) for an S_FREE that lets S_0(t+1) go, V(t) for a P_FULL. It
      // arrives on a barrier's next phase only after the previous one
      // completed, so it is never two phases ahead. Once page t's last S has
      // been loaded (its S_FREE phase complete), both S MMAs are done with
      // K(t) and the watcher gives that slot back (both expected arrivals),
      // and counts the page in s_done (read by MMA thread 1 after a skip).
      if (lane == 0) {
        uint32_t g = 0, sf[2] = {0, 0}, pf[2] = {0, 0};
        bool ok = true;
        auto landed = [&](uint32_t r) -> bool {
          return wait_bar(bar(BR::RING_FULL + r % S), (r / S) & 1, ctl, 0x12a);
        };
        auto next_phase = [&](int base, int w, uint32_t& n) -> bool {
          if (n > 0 && !wait_bar(bar(base + w), (n - 1) & 1, ctl, 0x12b)) return false;
          mbar_arrive(bar(base + w));
          ++n;
          return true;
        };
        for (uint32_t k = 0; ok; ++k) {
          Item w;
          if (!next_item(k, 0x12c, w)) break;
          mbar_arrive(bar(B_ITEM_EMPTY + (k % kItemSlots)));
          if (w.id >= p.n_items) break;
          const int nq = w.two ? 2 : 1;
          for (int t = 0; ok && t < w.n_pages; ++t, ++g) {
            for (int q = 0; ok && q < nq; ++q) {
              // S_FREE_q(t): if it lets S_0(t+1) go, K(t+1) must be in.
              if (q == nq - 1 && t + 1 < w.n_pages && !landed(2 * g + 2)) { ok = false; break; }
              ok = next_phase(B_S_FREE, q, sf[q]);
            }
            // Page t's last S was loaded once that S_FREE completes: K(t) goes back.
            if (ok) ok = wait_bar(bar(B_S_FREE + nq - 1), (sf[nq - 1] - 1) & 1, ctl, 0x12d);
            if (ok) *s_done = g + 1;
            if (ok) mbar_arrive_cnt(bar(BR::RING_EMPTY + (2 * g) % S), 2);
            if (!ok || !landed(2 * g + 1)) { ok = false; break; }
            for (int q = 0; ok && q < nq; ++q) ok = next_phase(B_P_FULL, q, pf[q]);
          }
        }
      }
    } else if (warp == 1 || warp == 3) {
      // ---------------------------------------------------------- tcgen05 issuers
      // Two threads issue MMAs: warp 1 for query tile 0, warp 3 for tile 1.
      // While one waits on a barrier the other keeps the tensor pipe's short
      // queue fed. Both walk the same items and pages and follow the S
      // buffer's owners in the same global order (S_0(t), S_1(t) per page), so
      // each knows whose S_FREE to wait for; only data dependencies order the
      // two threads' MMAs.
      if (lane == 0) {
        const int mw = warp == 1 ? 0 : 1;  // the query tile this thread issues for
        // g: pages walked; pv: P.V MMAs issued (P_mw buffers consumed);
        // sc[b]: S MMAs issued so far (by either thread) whose load signals
        // S_FREE_b; itw: items done by tile mw; s_last: that barrier for the
        // S the buffer holds.
        uint32_t g = 0, it = 0, pv = 0, sc[2] = {0, 0}, itw = 0;
        bool resync = false;  // thread 1 skipped an item since its last S
        int s_last = -1;
        bool ok = true;
        auto ring_wait = [&](uint32_t r, int code) -> bool {
          return wait_bar(bar(BR::RING_FULL + r % S), (r / S) & 1, ctl, code);
        };
        auto slot_addr = [&](uint32_t r) -> uint32_t {
          return sbase + C::kRingOff + (r % S) * C::kTileBytes;
        };
        // Shared-memory descriptors split into a per-address low word and a
        // constant high word (stride 1024 B between 8-row groups, sm_100
        // version bit, 128-byte swizzle); K-steps add constants to the low word.
        constexpr uint32_t kDescHi = (1024u >> 4) | (1u << 14) | (2u << 29);
        auto lo_k = [](uint32_t addr) { return ((addr & 0x3FFFFu) >> 4) | (1u << 16); };
        auto lo_mn = [](uint32_t addr) { return ((addr & 0x3FFFFu) >> 4) | ((16384u >> 4) << 16); };
        // An S (ours or the other thread's) takes the buffer; w names the
        // S_FREE barrier its load signals (2: tile 0 of a single-tile item).
        auto take_s = [&](int w) {
          ++sc[w];
          s_last = w;
        };
        // S = Q_mw K(t)^T into the S buffer, once the buffer's previous owner
        // has loaded it.
        auto issue_s = [&](uint32_t t) -> bool {
          if (s_last >= 0 &&
              !wait_bar(bar(B_S_FREE + s_last), (sc[s_last] - 1) & 1, ctl, 0x119 + s_last))
            return false;
          tc_fence_after();
          const uint32_t qaddr = sbase + C::kQOff + mw * C::kTileBytes;
          const uint32_t kaddr = slot_addr(2 * t);
          if constexpr (D == 128) {
            mma_ss_k128<2, C::kPanelBytes / 16, 2, C::kPanelBytes / 16>(
                tmem + C::kColS, lo_k(qaddr), kDescHi, lo_k(kaddr), kDescHi, C::kIdescS, 0u);
          } else {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk / 4) * C::kPanelBytes + (kk % 4) * 32;
              mma_ss(tmem + C::kColS, desc_k(qaddr + off), desc_k(kaddr + off), C::kIdescS,
                     kk > 0 ? 1u : 0u);
            }
          }
          tc_commit(bar(B_S_FULL + mw));
          take_s(mw);
          return true;
        };
        // O_mw (+)= P_mw V(t), once softmax mw has written P_mw (and, for an
        // item's first P.V, once its epilogue has read O_mw) and V(t) is in.
        // The commit on P_FREE_mw hands P_mw (and O_mw) back to the softmax.
        auto issue_pv = [&](uint32_t t, bool accumulate) -> bool {
          if (!wait_bar(bar(B_P_FULL + mw), pv & 1, ctl, 0x112 + mw)) return false;
          if (!accumulate && itw > 0 &&
              !wait_bar(bar(B_O_EMPTY + mw), (itw - 1) & 1, ctl, 0x114 + mw))
            return false;
          // P_FULL implies V(t) has landed: the watcher joins it only then.
          tc_fence_after();
          const uint32_t vaddr = slot_addr(2 * t + 1);
          mma_ts_k128<2048 / 16>(tmem + C::kColO + 128 * mw, tmem + C::kColP + 64 * mw,
                                 lo_mn(vaddr), kDescHi, C::kIdescO, accumulate ? 1u : 0u);
          tc_commit(bar(B_P_FREE + mw));
          ++pv;
          return true;
        };
        // V(t) goes back to the producer by one commit behind each tile's P.V
        // (two from thread 0 with a single tile); K(t) by the watcher once the
        // page's last S has been loaded.
        auto release_v = [&](uint32_t t, int nq) {
          tc_commit(bar(BR::RING_EMPTY + (2 * t + 1) % S));
          if (nq == 1) tc_commit(bar(BR::RING_EMPTY + (2 * t + 1) % S));
        };
        // Pipe order per page t: S_0(t), PV_0(t-1) from thread 0 and S_1(t),
        // PV_1(t-1) from thread 1. A tile's P(t) is consumed after S of page
        // t+1, so its softmax has a whole page period; the S buffer is reloaded
        // while the P.V behind it runs.
        for (uint32_t k = 0; ok; ++k) {
          Item w;
          if (!next_item(k, 0x118, w)) { ok = false; break; }
          mbar_arrive(bar(B_ITEM_EMPTY + (k % kItemSlots)));
          if (w.id >= p.n_items) break;
          const int n = w.n_pages;
          const int nq = w.two ? 2 : 1;
          const uint32_t qit = it++;
          if (mw >= nq) {
            // The item has no tile for this thread: its S tiles advance
            // S_FREE_0 without this thread's waits, so before its next S it
            // lets the watcher's page count catch up (a parity wait is only
            // sound for the phase right after the last one its waiter saw).
            for (int j = 0; j < n; ++j) take_s(0);
            g += n;
            resync = true;
            continue;
          }
          // Thread 0 waits for both Q tiles; thread 1's first S waits for the
          // S_FREE_0 of thread 0's, so it needs no Q_FULL wait of its own (it
          // skips single-tile items, whose Q_FULL phases it would not see).
          if (mw == 0 && !wait_bar(bar(B_Q_FULL), qit & 1, ctl, 0x110)) { ok = false; break; }
          if (resync) {  // every S before this item's has been loaded
            const uint64_t t0 = globaltimer_ns();
            while (ok && *s_done < g) {
              __nanosleep(64);
              if (*abort_flag) ok = false;
              else if (globaltimer_ns() - t0 > ctl.timeout_ns) {
                *abort_flag = 1;
                atomicCAS(p.status, 0, 0x11c);
                ok = false;
              }
            }
            if (!ok) break;
            resync = false;
          }
          for (int j = 0; j < n && ok; ++j, ++g) {
            if (mw == 1) take_s(0);  // thread 0's S_0(t) went first
            // K(t) has landed: for an item's first page this thread checks;
            // later, the S_FREE it waits for implies it (the watcher joins the
            // S_FREE that lets S_0(t) go only once K(t) is in, and thread 1's
            // S follows S_0(t)).
            if (mw == 0 && j == 0 && !ring_wait(2 * g, 0x111)) { ok = false; break; }
            if (!issue_s(g)) { ok = false; break; }
            if (mw == nq - 1 && j == n - 1) tc_commit(bar(B_Q_EMPTY));  // the item's last S
            if (mw == 0 && nq == 2) take_s(1);  // thread 1's S_1(t) follows
            if (j > 0) {
              if (!issue_pv(g - 1, j > 1)) { ok = false; break; }
              release_v(g - 1, nq);
            }
          }
          if (!ok) break;
          // The item's last page: this tile's P.V, then its O is complete.
          if (!issue_pv(g - 1, n > 1)) { ok = false; break; }
          tc_commit(bar(B_O_FULL + mw));
          release_v(g - 1, nq);
          ++itw;
        }
        // Wait (bounded) until every MMA issued by this thread has finished.
        tc_commit(bar(B_DRAIN + mw));
        drain_wait(bar(B_DRAIN + mw), 0);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    regs_inc<kRegsHigh>();
    const int wq = (warp - 4) >> 2;  // query tile of this warpgroup
    const int quarter = warp & 3;    // TMEM lanes this warp may access
    const int row = quarter * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t tS = trow + C::kColS;
    const uint32_t tP = trow + C::kColP + 64 * wq;
    const uint32_t tO = trow + C::kColO + 128 * wq;
    const float sl2 = p.scale_log2;
    // g: S tiles loaded, pw: P_w written (each one read by a P.V that commits
    // P_FREE_w), it: items finished by this warpgroup, gp: pages of every
    // item so far, both tiles' (the ring holds K(gp) at 2 gp, V(gp) at 2 gp + 1).
    uint32_t g = 0, pw = 0, it = 0, gp = 0;
    for (uint32_t k = 0;; ++k) {
      Item w;
      bool ok = __all_sync(0xffffffffu, next_item(k, 0x124 + wq, w));
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_ITEM_EMPTY + (k % kItemSlots)));
      if (w.id >= p.n_items) break;
      if (wq == 1 && !w.two) {  // the pair's second tile lies past the node
        gp += w.n_pages;
        continue;
      }
      const AttnNode& nd = p.nodes[w.node];
      float m_run = -INFINITY, l_run = 0.f;
      for (int t = 0; t < w.n_pages; ++t, ++g, ++gp) {
        ok = __all_sync(0xffffffffu, wait_bar(bar(B_S_FULL + wq), g & 1, ctl, 0x120 + wq));
        if (!ok) break;
        tc_fence_after();

        const int valid = (int)(p.pages[nd.page0 + w.page_begin + t] >> 25) + 1;
        // The whole S row in one TMEM round trip; then the S buffer goes back
        // to the MMA thread for the other tile's (or the next page's) S.
        float sv[128];
        tmem_ld128_wait(tS, *reinterpret_cast<uint32_t(*)[128]>(sv));
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_S_FREE + wq));
        if (valid < 128) {  // partial last page of an entry: drop the padding keys
#pragma unroll
          for (int i = 0; i < 128; ++i) sv[i] = i < valid ? sv[i] : -INFINITY;
        }
        float mx[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mx[i] = fmax3(sv[i], sv[8 + i], sv[16 + i]);
#pragma unroll
        for (int k = 24; k < 120; k += 16)
#pragma unroll
          for (int i = 0; i < 8; ++i) mx[i] = fmax3(mx[i], sv[k + i], sv[k + 8 + i]);
#pragma unroll
        for (int i = 0; i < 8; ++i) mx[i] = fmaxf(mx[i], sv[120 + i]);
        const float mrow = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]),
                                 fmaxf(mx[6], mx[7]));
        const float m_new = fmaxf(m_run, mrow * sl2);
        const bool grow = __any_sync(0xffffffffu, t > 0 && m_new > m_run + 8.f);
        // P_w and O_w are ours again once the P.V that read the previous P_w
        // has finished (it was issued right after this page's S).
        bool p_free = pw == 0;
        if (t == 0) {
          m_run = m_new;
        } else if (grow) {
          ok = __all_sync(0xffffffffu, wait_bar(bar(B_P_FREE + wq), (pw - 1) & 1, ctl, 0x126 + wq));
          if (!ok) break;
          tc_fence_after();
          p_free = true;
          // Bring O up to the new max (O holds every P.V up to the previous page).
          const float alpha = ex2_approx(m_run - m_new);
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32_wait(tO + c * 32, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tO + c * 32, o);
          }
          l_run *= alpha;
          m_run = m_new;
        }
        // P = 2^(S log2e/sqrt(d) - m), packed to bf16 in registers, then stored
        // to P_w in two 32-column pieces.
        const float negm = -m_run;
#if WAVE_PACKED_FMA
        const uint64_t scale2 = f2_pack(sl2, sl2), negm2 = f2_pack(negm, negm);
        uint64_t acc2[2] = {0, 0};
#else
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#endif
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // 64 columns of S -> 32 columns of P
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int c = 64 * h + 2 * i;
            float x0, x1;
#if WAVE_PACKED_FMA
            f2_unpack(f2_fma(f2_pack(sv[c], sv[c + 1]), scale2, negm2), x0, x1);
#else
            x0 = fmaf(sv[c], sl2, negm);
            x1 = fmaf(sv[c + 1], sl2, negm);
#endif
            float y0, y1;
            if ((c & 31) < kEmuPerChunk) {
              exp2_poly2(x0, x1, y0, y1);
            } else {
              y0 = ex2_approx(x0);
              y1 = ex2_approx(x1);
            }
#if WAVE_PACKED_FMA
            acc2[i & 1] = f2_add(acc2[i & 1], f2_pack(y0, y1));
#else
            acc[i & 3] += y0 + y1;
#endif
            pk[i] = pack_bf16x2(y0, y1);
          }
          if (h == 0 && !p_free) {
            ok = __all_sync(0xffffffffu,
                            wait_bar(bar(B_P_FREE + wq), (pw - 1) & 1, ctl, 0x126 + wq));
            if (!ok) break;
            tc_fence_after();
          }
          tmem_st32(tP + 32 * h, pk);
        }
        if (!ok) break;
#if WAVE_PACKED_FMA
        float acc[4];
        f2_unpack(acc2[0], acc[0], acc[1]);
        f2_unpack(acc2[1], acc[2], acc[3]);
#endif
        l_run += (acc[0] + acc[1]) + (acc[2] + acc[3]);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_P_FULL + wq));
        ++pw;
      }
      if (!ok) break;
      ok = __all_sync(0xffffffffu, wait_bar(bar(B_O_FULL + wq), it & 1, ctl, 0x122 + wq));
      if (!ok) break;
      tc_fence_after();
      if (nd.n_splits > 1) {
        // One key range of several: the unnormalised O row and its (running
        // max, sum), both relative to the same max, for the combine kernel.
        const int64_t slot = ((int64_t)w.id * 2 + wq) * 128 + row;
        float4* po = reinterpret_cast<float4*>(p.part_o + slot * D);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32_wait(tO + c * 32, o);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            po[c * 8 + v] = make_float4(__uint_as_float(o[4 * v]), __uint_as_float(o[4 * v + 1]),
                                        __uint_as_float(o[4 * v + 2]), __uint_as_float(o[4 * v + 3]));
        }
        reinterpret_cast<float2*>(p.part_ml)[slot] = make_float2(m_run, l_run);
        tc_fence_before();
        mbar_arrive(bar(B_O_EMPTY + wq));
        ++it;
        continue;
      }
      const float inv = 1.f / l_run;
      const int q_local = (2 * w.pair + wq) * 128 + row;
      const bool store = q_local < p.q_rows;
      uint4* orow = reinterpret_cast<uint4*>(
          p.out + ((int64_t)(nd.q_row0 + q_local) * H + w.head) * D);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32_wait(tO + c * 32, o);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
        if (store) {
#pragma unroll
          for (int v = 0; v < 4; ++v)
            orow[c * 4 + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
        __syncwarp();  // rows past the node skip the store: reconverge before the next tcgen05.ld
      }
      tc_fence_before();
      mbar_arrive(bar(B_O_EMPTY + wq));
      ++it;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kCols);
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    p.clock_out[0] = clock64() - clock_start[0];
    p.clock_out[1] = (int64_t)globaltimer_ns() - clock_start[1];
  }
}

// Combine of split key ranges: for each query row of a node whose key list
// was cut into S ranges, O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s
// with M = max_s m_s (the m_s are the ranges' running maxima in the log2
// domain; each O_s and l_s is relative to its own m_s). One warp per query
// row (eight rows per CTA, kCombineRowsPerCta), so thousands of rows' loads
// are in flight at once; lane s holds range s's (m, l), and lanes split the d
// values of O.
struct CombineParams {
  const float* part_o;
  const float* part_ml;
  uint16_t* out;
  int32_t heads;
  int32_t q_rows;
  int32_t n_nodes;
  int32_t pad;
  AttnNode nodes[WAVE_MAX_NODES];
  int32_t block0[WAVE_MAX_NODES + 1];  // first CTA of each node (nodes without ranges: none)
};
constexpr int kCombineRowsPerCta = 8;

template <int D>
__global__ void __launch_bounds__(32 * kCombineRowsPerCta)
    attn_combine_kernel(const __grid_constant__ CombineParams p) {
  constexpr int V = D / 32;  // O values per lane
  constexpr int kCtasPerTile = 128 / kCombineRowsPerCta;
  int n = 0;
  while (n + 1 < p.n_nodes && (int)blockIdx.x >= p.block0[n + 1]) ++n;
  const AttnNode& nd = p.nodes[n];
  const int j = (blockIdx.x - p.block0[n]) / kCtasPerTile;
  const int head = j / nd.n_qtiles, qt = j - head * nd.n_qtiles;
  const int pair = qt >> 1, w = qt & 1, S = nd.n_splits;
  const int64_t item_base = nd.item0 + (int64_t)(head * nd.n_pairs + pair) * S;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  {
    const int r = ((blockIdx.x - p.block0[n]) % kCtasPerTile) * kCombineRowsPerCta + warp;
    const int q_local = qt * 128 + r;
    if (q_local >= p.q_rows) return;
    float m = -INFINITY, l = 0.f;
    if (lane < S) {
      const float2 ml = reinterpret_cast<const float2*>(p.part_ml)[((item_base + lane) * 2 + w) * 128 + r];
      m = ml.x;
      l = ml.y;
    }
    float mx = m;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float e = lane < S ? exp2f(m - mx) : 0.f;
    float den = e * l;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    float acc[V];
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = 0.f;
#pragma unroll 8
    for (int sp = 0; sp < S; ++sp) {
      const float es = __shfl_sync(0xffffffffu, e, sp);
      const float* po = p.part_o + (((item_base + sp) * 2 + w) * 128 + r) * D + lane * V;
      if constexpr (V == 4) {
        const float4 v = *reinterpret_cast<const float4*>(po);
        acc[0] += es * v.x; acc[1] += es * v.y; acc[2] += es * v.z; acc[3] += es * v.w;
      } else {
        const float2 v = *reinterpret_cast<const float2*>(po);
        acc[0] += es * v.x; acc[1] += es * v.y;
      }
    }
    const float inv = 1.f / den;
    uint16_t* dst = p.out + ((int64_t)(nd.q_row0 + q_local) * p.heads + head) * D + lane * V;
    if constexpr (V == 4) {
      *reinterpret_cast<uint2*>(dst) =
          make_uint2(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv));
    } else {
      *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    }
  }
}

template <int D>
int launch(const AttnParams& prm, int grid, cudaStream_t stream) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  static int num_regs = 0;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(round_attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    Cfg<D>::kSmemBytes);
    cudaFuncAttributes fa;
    if (attr_err == cudaSuccess) attr_err = cudaFuncGetAttributes(&fa, round_attn_kernel<D>);
    if (attr_err == cudaSuccess) num_regs = fa.numRegs;
  });
  if (attr_err != cudaSuccess)
    return fail(WAVE_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(attr_err));
  // setmaxnreg.inc waits until registers are free: with fewer registers per
  // thread at launch than the split assumes it would never return.
  if ((uint32_t)num_regs < kRegsLaunch)
    return fail(WAVE_ERR_UNSUPPORTED, "round_attn_kernel compiled with %d registers per thread; "
                "its warpgroup register split needs %u", num_regs, kRegsLaunch);
  round_attn_kernel<D><<<grid, kThreads, Cfg<D>::kSmemBytes, stream>>>(prm);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(WAVE_ERR_CUDA, "round_attn_kernel launch: %s", cudaGetErrorString(e));
  return WAVE_OK;
}

}  // namespace

}  // namespace wavei

using namespace wavei;

namespace wavei {
namespace {

// One round of attention with the work-queue counter at `counter` (a device
// int32 that this call sets to zero on `stream` before the launch).
// Key ranges per (node, head, pair) for a call: `splits` >= 1 as asked; 0 =
// none when the round already has a wave of items for the SMs (the dynamic
// longest-first queue balances those), else the fewest ranges whose items
// fill their last wave of SMs to at least 90 % (the best fill found if none
// does); at most the node's pages and kMaxSplits.
constexpr int kMaxSplits = 32;
int choose_splits(const wave_kv* kv, int32_t n_active, int32_t splits) {
  if (splits > 0) return std::min(splits, kMaxSplits);
  const int T = kv->cfg.tokens_per_chunk, H = kv->cfg.heads;
  const int64_t items = (int64_t)n_active * H * (((T + 127) / 128 + 1) / 2);
  if (items >= kv->num_sms) return 1;
  int best = 1;
  double best_fill = 0.0;
  for (int s = 2; s <= kMaxSplits; ++s) {
    const int64_t n = items * s;
    const int64_t waves = (n + kv->num_sms - 1) / kv->num_sms;
    const double fill = (double)n / (double)(waves * kv->num_sms);
    if (fill >= 0.9) return s;
    if (fill > best_fill) best_fill = fill, best = s;
  }
  return best;
}

// Bytes of workspace a split call needs: per work item and query tile, 128
// rows of d fp32 O values and an fp32 (max, sum) pair.
uint64_t split_workspace_bytes(const wave_kv* kv, int64_t n_items) {
  return (uint64_t)n_items * 2 * 128 * ((uint64_t)kv->cfg.head_dim + 2) * sizeof(float);
}

int round_attn_impl(wave_kv* kv, const wave_node* active, int32_t n_active, int32_t policy,
                    const void* Q, void* O, void* stream, int32_t* counter, int32_t splits = 1,
                    void* workspace = nullptr, uint64_t workspace_bytes = 0,
                    uint64_t* bytes_needed = nullptr) {
  if (!kv) return fail(WAVE_ERR_ARG, "NULL handle");
  if (!kv->on_device) return fail(WAVE_ERR_ARG, "host-only handle (pool == NULL)");
  if (int rc = check_current_device(kv)) return rc;
  if (!valid_policy(policy)) return fail(WAVE_ERR_ARG, "unknown policy %d", policy);
  if (n_active < 0 || (n_active > 0 && !active)) return fail(WAVE_ERR_ARG, "bad active list");
  if (n_active == 0) return WAVE_OK;
  if (n_active > WAVE_MAX_NODES)
    return fail(WAVE_ERR_CAPACITY, "%d active nodes exceed %d", n_active, WAVE_MAX_NODES);
  if (!bytes_needed &&
      (!Q || !O || ((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(O)) & 15)))
    return fail(WAVE_ERR_ARG, "Q and O must be non-NULL and 16-byte aligned");
  std::vector<int32_t> rows, offs;
  int rc = build_rows(kv, active, n_active, policy, rows, offs);
  if (rc) return rc;
  const int64_t n_rows = (int64_t)rows.size() / 2;
  if (n_rows > WAVE_MAX_PAGES_PER_ROUND)
    return fail(WAVE_ERR_CAPACITY, "%lld key pages exceed %d per call", (long long)n_rows,
                WAVE_MAX_PAGES_PER_ROUND);
  const int T = kv->cfg.tokens_per_chunk, H = kv->cfg.heads, D = kv->cfg.head_dim;
  if ((int64_t)n_active * T >= (1LL << 31) / H)
    return fail(WAVE_ERR_ARG, "too many query rows");

  static thread_local AttnParams prm;
  std::memset(&prm, 0, offsetof(AttnParams, pages));
  // Nodes in longest-key-list-first order, each with its key ranges.
  const int n_qtiles = (T + 127) / 128;
  const int n_pairs = (n_qtiles + 1) / 2;
  std::vector<int> order(n_active);
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) {
    return offs[a + 1] - offs[a] > offs[b + 1] - offs[b];
  });
  int64_t n_items = 0;
  bool any_split = false;
  for (int k = 0; k < n_active; ++k) {
    const int i = order[k];
    const int ns = std::max(1, std::min<int>(splits, offs[i + 1] - offs[i]));
    any_split |= ns > 1;
    n_items += (int64_t)H * n_pairs * ns;
  }
  if (n_items >= (1LL << 30)) return fail(WAVE_ERR_CAPACITY, "too many work items");
  // FP8 pools: the round's distinct pages are expanded to bf16 staging pages
  // (slot = order of first use) at the start of the workspace.
  std::vector<int32_t> slot_page;
  std::map<int32_t, int32_t> slot_of;
  if (kv->fp8) {
    for (int64_t rr = 0; rr < n_rows; ++rr)
      if (slot_of.emplace(rows[2 * rr], (int32_t)slot_page.size()).second)
        slot_page.push_back(rows[2 * rr]);
  }
  const uint64_t staging = ((uint64_t)slot_page.size() * bf16_page_bytes(kv) + 255) / 256 * 256;
  const uint64_t need = staging + (any_split ? split_workspace_bytes(kv, n_items) : 0);
  if (bytes_needed) {
    *bytes_needed = need;
    return WAVE_OK;
  }
  if (need > 0 && (!workspace || workspace_bytes < need ||
                   (reinterpret_cast<uintptr_t>(workspace) & 255)))
    return fail(WAVE_ERR_ARG, "%s need a 256-byte aligned workspace of %llu bytes (got %llu; "
                "use wave_round_attn_split)", kv->fp8 ? "FP8 pages" : "split key ranges",
                (unsigned long long)need, (unsigned long long)workspace_bytes);
  auto encode = tensor_map_encoder();
  if (!encode) return fail(WAVE_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)n_active * T};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
  cuuint32_t box[3] = {64, 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = encode(&prm.tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(Q), dims,
                      strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(WAVE_ERR_CUDA, "cuTensorMapEncodeTiled(Q) failed: %d", (int)r);
  if (kv->fp8) {
    cuuint64_t sd[2] = {(cuuint64_t)D, (cuuint64_t)slot_page.size() * 2 * H * kPageTokens};
    cuuint64_t ss[1] = {(cuuint64_t)D * 2};
    cuuint32_t sb[2] = {64, 128};
    cuuint32_t se[2] = {1, 1};
    r = encode(&prm.tm_kv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, workspace, sd, ss, sb, se,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
      return fail(WAVE_ERR_CUDA, "cuTensorMapEncodeTiled(staging) failed: %d", (int)r);
  } else {
    prm.tm_kv = kv->tm_kv;
  }
  prm.out = static_cast<uint16_t*>(O);
  prm.status = static_cast<int32_t*>(kv->cfg.pool);
  prm.counter = counter;
  prm.clock_out = reinterpret_cast<int64_t*>(static_cast<char*>(kv->cfg.pool) + 256);
  prm.wait_ns = wait_limit_ns(kv);
  prm.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  prm.heads = H;
  prm.q_rows = T;
  prm.n_nodes = n_active;

  // Longest key list first (ties keep list order): a static round-robin of
  // items over persistent CTAs then approximates longest-processing-time order.
  int32_t item0 = 0, w = 0;
  for (int k = 0; k < n_active; ++k) {
    const int i = order[k];
    AttnNode& nd = prm.nodes[k];
    nd.q_row0 = i * T;
    nd.page0 = w;
    nd.n_pages = offs[i + 1] - offs[i];
    nd.item0 = item0;
    nd.n_pairs = n_pairs;
    nd.n_qtiles = n_qtiles;
    nd.n_splits = std::max(1, std::min<int>(splits, nd.n_pages));
    for (int32_t rr = offs[i]; rr < offs[i + 1]; ++rr) {
      const int32_t pg = kv->fp8 ? slot_of[rows[2 * rr]] : rows[2 * rr];
      prm.pages[w++] = (uint32_t)pg | ((uint32_t)(rows[2 * rr + 1] - 1) << 25);
    }
    item0 += H * n_pairs * nd.n_splits;
  }
  prm.n_items = item0;
  if (any_split) {
    prm.part_o = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + staging);
    prm.part_ml = prm.part_o + (int64_t)item0 * 2 * 128 * D;
  }
  const int grid = std::min(prm.n_items, kv->num_sms);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (kv->fp8) {
    rc = launch_fp8_expand(kv, (int32_t)slot_page.size(), slot_page.data(), workspace, s);
    if (rc) return rc;
  }
  cudaError_t e = cudaMemsetAsync(prm.counter, 0, sizeof(int32_t), s);
  if (e != cudaSuccess) return fail(WAVE_ERR_CUDA, "cudaMemsetAsync(work counter): %s", cudaGetErrorString(e));
  rc = D == 128 ? launch<128>(prm, grid, s) : launch<64>(prm, grid, s);
  if (rc || !any_split) return rc;
  // Combine the key ranges of every split node into O.
  static thread_local CombineParams cp;
  std::memset(&cp, 0, sizeof(cp));
  cp.part_o = prm.part_o;
  cp.part_ml = prm.part_ml;
  cp.out = prm.out;
  cp.heads = H;
  cp.q_rows = T;
  cp.n_nodes = n_active;
  int32_t blocks = 0;
  for (int k = 0; k < n_active; ++k) {
    cp.nodes[k] = prm.nodes[k];
    cp.block0[k] = blocks;
    if (prm.nodes[k].n_splits > 1) blocks += H * n_qtiles * (128 / kCombineRowsPerCta);
  }
  cp.block0[n_active] = blocks;
  if (D == 128)
    attn_combine_kernel<128><<<blocks, 32 * kCombineRowsPerCta, 0, s>>>(cp);
  else
    attn_combine_kernel<64><<<blocks, 32 * kCombineRowsPerCta, 0, s>>>(cp);
  e = cudaGetLastError();
  if (e != cudaSuccess) return fail(WAVE_ERR_CUDA, "attn_combine_kernel launch: %s", cudaGetErrorString(e));
  return WAVE_OK;
}

}  // namespace
}  // namespace wavei

extern "C" int wave_round_attn(wave_kv* kv, const wave_node* active, int32_t n_active,
                               int32_t policy, const void* Q, void* O, void* stream) {
  clear_error();
  if (!kv) return fail(WAVE_ERR_ARG, "NULL handle");
  if (!kv->on_device) return fail(WAVE_ERR_ARG, "host-only handle (pool == NULL)");
  int32_t* counter =
      reinterpret_cast<int32_t*>(static_cast<uint8_t*>(kv->cfg.pool) + kCounterOffset);
  return round_attn_impl(kv, active, n_active, policy, Q, O, stream, counter);
}

extern "C" int wave_round_attn_split_workspace(wave_kv* kv, const wave_node* active,
                                               int32_t n_active, int32_t policy, int32_t splits,
                                               uint64_t* bytes, int32_t* splits_used) {
  clear_error();
  if (!kv || !bytes) return fail(WAVE_ERR_ARG, "NULL argument");
  if (!kv->on_device) return fail(WAVE_ERR_ARG, "host-only handle (pool == NULL)");
  if (splits < 0) return fail(WAVE_ERR_ARG, "splits must be >= 0, got %d", splits);
  const int ns = choose_splits(kv, n_active, splits);
  if (splits_used) *splits_used = ns;
  int32_t* counter = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(kv->cfg.pool) + kCounterOffset);
  return round_attn_impl(kv, active, n_active, policy, nullptr, nullptr, nullptr, counter, ns,
                         nullptr, 0, bytes);
}

extern "C" int wave_round_attn_split(wave_kv* kv, const wave_node* active, int32_t n_active,
                                     int32_t policy, int32_t splits, const void* Q, void* O,
                                     void* workspace, uint64_t workspace_bytes, void* stream) {
  clear_error();
  if (!kv) return fail(WAVE_ERR_ARG, "NULL handle");
  if (!kv->on_device) return fail(WAVE_ERR_ARG, "host-only handle (pool == NULL)");
  if (splits < 0) return fail(WAVE_ERR_ARG, "splits must be >= 0, got %d", splits);
  int32_t* counter =
      reinterpret_cast<int32_t*>(static_cast<uint8_t*>(kv->cfg.pool) + kCounterOffset);
  return round_attn_impl(kv, active, n_active, policy, Q, O, stream, counter,
                         choose_splits(kv, n_active, splits), workspace, workspace_bytes);
}

// ----------------------------------------------------------------------------
// Static-scratch variant of wave_round_attn.
//
// wave_round_attn keeps its one piece of per-call device scratch -- the
// work-queue counter that the persistent CTAs draw work items from -- in the
// header of the caller's pool. This variant keeps it in the array below
// instead, a file-scope device array of a fixed 256 bytes that exists on every
// GPU that loads the library, until the process exits. Nothing is allocated
// per call. Host code must not hand the array's name to a kernel (on the host
// it is only a stand-in, not a device address); its device address is looked
// up with cudaGetSymbolAddress on the first call made with that device current
// (again after a device reset, which gives the device a new context), and
// cached.
namespace wavei {
namespace {
constexpr int kStaticScratchWords = 64;    // 256 bytes per device
constexpr int kStaticScratchNeeded = 1;    // words used: the work-queue counter
constexpr int kMaxDevices = 64;
static_assert(kStaticScratchNeeded <= kStaticScratchWords, "static scratch too small");
std::mutex g_scratch_mu;
int32_t* g_scratch_addr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};  // the context each address was looked up in

// The calling thread's current context, from the driver (reached through the
// runtime's entry-point query; null if unavailable).
CUcontext current_context() {
  using Fn = CUresult (*)(CUcontext*);
  static Fn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<Fn>(f);
  });
  CUcontext ctx = nullptr;
  if (fn) fn(&ctx);
  return ctx;
}
}  // namespace
}  // namespace wavei

static __device__ __align__(256) int32_t g_round_attn_scratch[wavei::kStaticScratchWords];

extern "C" int wave_round_attn_static_scratch(wave_kv* kv, const wave_node* active,
                                              int32_t n_active, int32_t policy, const void* Q,
                                              void* O, void* stream) {
  clear_error();
  if (!kv) return fail(WAVE_ERR_ARG, "NULL handle");
  if (!kv->on_device) return fail(WAVE_ERR_ARG, "host-only handle (pool == NULL)");
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(WAVE_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev != kv->device)
    return fail(WAVE_ERR_ARG, "current device %d is not the pool's device %d", dev, kv->device);
  if (dev < 0 || dev >= kMaxDevices)
    return fail(WAVE_ERR_UNSUPPORTED, "device index %d beyond %d", dev, kMaxDevices - 1);
  // The scratch need does not grow with the round (one counter), so the only
  // size limits are those wave_round_attn enforces: at most WAVE_MAX_NODES
  // nodes and WAVE_MAX_PAGES_PER_ROUND key pages (WAVE_ERR_CAPACITY beyond).
  // Looked up once per device and context: a device reset makes a new
  // context, in which the array lives at a new address.
  int32_t* scratch = nullptr;
  {
    const CUcontext ctx = current_context();
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev] || g_scratch_ctx[dev] != ctx) {
      void* ptr = nullptr;
      e = cudaGetSymbolAddress(&ptr, g_round_attn_scratch);
      if (e != cudaSuccess || !ptr)
        return fail(WAVE_ERR_CUDA, "cudaGetSymbolAddress(static scratch): %s",
                    cudaGetErrorString(e));
      g_scratch_addr[dev] = static_cast<int32_t*>(ptr);
      g_scratch_ctx[dev] = ctx;
    }
    scratch = g_scratch_addr[dev];
  }
  // round_attn_impl zeroes the counter (word 0) on `stream` before launching.
  return round_attn_impl(kv, active, n_active, policy, Q, O, stream, scratch);
}
