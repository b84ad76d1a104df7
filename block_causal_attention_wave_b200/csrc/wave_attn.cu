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
// How (B200 design, not the pages'): one CTA per SM, each looping over work
// items (node, head, 128-query tile) ordered longest key list first, query
// tiles of one head adjacent so concurrent CTAs share that head's K/V pages in
// L2. Per CTA:
//   warp 0   TMA producer: Q tile once per item, then each 128-token K and V
//            page of the key list, gathered by page id (the page id is the
//            tensor-map row coordinate), into a 3-stage shared-memory ring.
//   warp 1   tcgen05 issuer: S = Q K^T (both operands in shared memory,
//            128-byte swizzle, K-major) into one of two TMEM S buffers, then
//            O += P V with P read from TMEM (bf16) and V from shared memory
//            (MN-major). O accumulates in TMEM in fp32.
//   warps 2-5  softmax: one query row per thread. tcgen05.ld of the S row,
//            padding keys of a partial page masked, online max in the log2
//            domain, exp2, bf16 P written back to TMEM with tcgen05.st. O is
//            rescaled only when the running max grows by more than 8 (log2
//            units); otherwise the stale max is kept, which is exact after the
//            final division because P <= 2^8 stays well inside fp32/bf16 range.
//            Epilogue: O / l, bf16, stored straight from registers (only rows
//            that belong to the node).
// Every wait is bounded (2 s); on timeout the kernel records a status word,
// every role stops, and TMEM is freed before exit.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <numeric>
#include <vector>

#include "ptx.cuh"
#include "wave_internal.h"

using namespace wptx;

namespace wavei {

namespace {

constexpr int kThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2..5 softmax
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr uint64_t kDrainNs = 200000000ull;
constexpr uint32_t kPageMask = (1u << 25) - 1;  // page id bits of a page word

struct AttnNode {
  int32_t q_row0;    // first row of this node in Q / O
  int32_t page0;     // first page word
  int32_t n_pages;   // key pages
  int32_t item0;     // first work item
  int32_t n_qtiles;  // ceil(T / 128)
  int32_t pad;
};

struct AttnParams {
  CUtensorMap tm_q;   // Q as [rows][H][d]
  CUtensorMap tm_kv;  // pool page region as rows of d
  uint16_t* out;      // O, bf16 [rows][H][d]
  int32_t* status;    // device status word (pool header)
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

template <int D>
struct Cfg {
  static constexpr int kPanels = D / 64;           // 64-column, 128-byte-wide panels
  static constexpr int kPanelBytes = 128 * 128;    // 128 rows x 128 bytes
  static constexpr int kTileBytes = 128 * D * 2;   // one Q, K or V tile
  static constexpr int kStages = D == 128 ? 3 : 4;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kTileBytes;
  static constexpr int kVOff = kKOff + kStages * kTileBytes;
  static constexpr int kBarOff = kVOff + kStages * kTileBytes;
  static constexpr int kSmemBytes = kBarOff + 256 + 1024;  // + barriers + alignment slack
  // TMEM columns: S0, S1 (128 fp32 each), O (d fp32), P0, P1 (64 x bf16x2 each).
  static constexpr uint32_t kColS = 0, kColO = 256, kColP = 384, kCols = 512;
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
  B_S_FULL,        // 2
  B_P_FULL = B_S_FULL + 2,  // 2
  B_PV_DONE = B_P_FULL + 2,
  B_O_FULL,
  B_O_EMPTY,
  B_DRAIN,
  B_K_FULL,        // kStages each from here
};

template <int D>
struct Bars {
  static constexpr int kS = Cfg<D>::kStages;
  static constexpr int K_FULL = B_K_FULL, K_EMPTY = K_FULL + kS, V_FULL = K_EMPTY + kS,
                       V_EMPTY = V_FULL + kS, COUNT = V_EMPTY + kS;
  static_assert(COUNT * 8 + 16 <= 256, "barrier area");
};

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version field.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// K-major operand (Q, K): rows of 128 bytes, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_k(uint32_t addr) { return smem_desc(addr, 16, 1024); }
// MN-major operand (V as [key][d]): 64-column groups one panel (16 KB) apart,
// 8-key groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_mn(uint32_t addr) { return smem_desc(addr, 16384, 1024); }

struct Ctl {
  volatile int* abort_flag;
  int32_t* status;
};

// Bounded wait on an mbarrier phase. Returns false if this CTA is stopping.
__device__ __noinline__ bool wait_bar(uint32_t bar, uint32_t parity, const Ctl& ctl, int code) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  uint32_t spins = 0;
  while (!mbar_try_wait(bar, parity)) {
    if (*ctl.abort_flag) return false;
    if ((++spins & 31u) == 0 && globaltimer_ns() - t0 > kTimeoutNs) {
      *ctl.abort_flag = 1;
      atomicCAS(ctl.status, 0, code);
      return false;
    }
  }
  return true;
}

// Bounded wait that ignores the stop flag: used only while stopping, to let
// asynchronous copies or MMAs that were already issued complete.
__device__ __noinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > kDrainNs) return;
}

struct Item {
  int node, head, qtile;
};

__device__ __forceinline__ Item decode_item(const AttnParams& p, int item) {
  int n = 0;
  while (n + 1 < p.n_nodes && item >= p.nodes[n + 1].item0) ++n;
  const int j = item - p.nodes[n].item0;
  const int nq = p.nodes[n].n_qtiles;
  return Item{n, j / nq, j % nq};
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    round_attn_kernel(const __grid_constant__ AttnParams p) {
  using C = Cfg<D>;
  using BR = Bars<D>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_addr(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + C::kBarOff + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kBarOff + 8 * BR::COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kBarOff + 8 * BR::COUNT + 4);
  const Ctl ctl{abort_flag, p.status};

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar(B_Q_FULL), 1);
    mbar_init(bar(B_Q_EMPTY), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(B_S_FULL + b), 1);
      mbar_init(bar(B_P_FULL + b), 128);
    }
    mbar_init(bar(B_PV_DONE), 1);
    mbar_init(bar(B_O_FULL), 1);
    mbar_init(bar(B_O_EMPTY), 128);
    mbar_init(bar(B_DRAIN), 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(bar(BR::K_FULL + s), 1);
      mbar_init(bar(BR::K_EMPTY + s), 1);
      mbar_init(bar(BR::V_FULL + s), 1);
      mbar_init(bar(BR::V_EMPTY + s), 1);
    }
    *abort_flag = 0;
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

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t kv_it = 0, it = 0;
      // Phase of the newest copy issued on each full barrier (-1: none yet), so
      // that an early stop can wait for copies still in flight.
      int q_last = -1, k_last[S], v_last[S];
      for (int s = 0; s < S; ++s) k_last[s] = v_last[s] = -1;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x, ++it) {
        const Item w = decode_item(p, item);
        const AttnNode& nd = p.nodes[w.node];
        if (it > 0 && !wait_bar(bar(B_Q_EMPTY), (it - 1) & 1, ctl, 0x101)) { ok = false; break; }
        mbar_arrive_expect_tx(bar(B_Q_FULL), C::kTileBytes);
        for (int pn = 0; pn < C::kPanels; ++pn)
          tma_load_3d(sbase + C::kQOff + pn * C::kPanelBytes, &p.tm_q, pn * 64, w.head,
                      nd.q_row0 + w.qtile * 128, bar(B_Q_FULL));
        q_last = it & 1;
        for (int t = 0; t < nd.n_pages; ++t, ++kv_it) {
          const uint32_t page = p.pages[nd.page0 + t] & kPageMask;
          const int s = kv_it % S;
          const uint32_t ph = (kv_it / S) & 1;
          const int32_t yk = (int32_t)(((int64_t)page * 2 * H + w.head) * 128);
          const int32_t yv = yk + H * 128;
          if (kv_it >= (uint32_t)S && !wait_bar(bar(BR::K_EMPTY + s), ph ^ 1, ctl, 0x102)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(BR::K_FULL + s), C::kTileBytes);
          for (int pn = 0; pn < C::kPanels; ++pn)
            tma_load_2d(sbase + C::kKOff + s * C::kTileBytes + pn * C::kPanelBytes, &p.tm_kv,
                        pn * 64, yk, bar(BR::K_FULL + s));
          k_last[s] = (int)ph;
          if (kv_it >= (uint32_t)S && !wait_bar(bar(BR::V_EMPTY + s), ph ^ 1, ctl, 0x103)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(BR::V_FULL + s), C::kTileBytes);
          for (int pn = 0; pn < C::kPanels; ++pn)
            tma_load_2d(sbase + C::kVOff + s * C::kTileBytes + pn * C::kPanelBytes, &p.tm_kv,
                        pn * 64, yv, bar(BR::V_FULL + s));
          v_last[s] = (int)ph;
        }
      }
      if (!ok) {
        // Stopping early: let the copies already issued land before the CTA's
        // shared memory is released.
        if (q_last >= 0) drain_wait(bar(B_Q_FULL), (uint32_t)q_last);
        for (int s = 0; s < S; ++s) {
          if (k_last[s] >= 0) drain_wait(bar(BR::K_FULL + s), (uint32_t)k_last[s]);
          if (v_last[s] >= 0) drain_wait(bar(BR::V_FULL + s), (uint32_t)v_last[s]);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ tcgen05 issuer
    if (lane == 0) {
      uint32_t kv_it = 0, it = 0;
      bool ok = true;
      auto issue_pv = [&](uint32_t g, bool first) -> bool {
        const int s = g % S;
        const uint32_t b = g & 1;
        if (!wait_bar(bar(B_P_FULL + b), (g >> 1) & 1, ctl, 0x111)) return false;
        if (!wait_bar(bar(BR::V_FULL + s), (g / S) & 1, ctl, 0x112)) return false;
        if (first && it > 0 && !wait_bar(bar(B_O_EMPTY), (it - 1) & 1, ctl, 0x113)) return false;
        tc_fence_after();
        const uint32_t vaddr = sbase + C::kVOff + s * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + C::kColO, tmem + C::kColP + b * 64 + kk * 8, desc_mn(vaddr + kk * 2048),
                 C::kIdescO, (first && kk == 0) ? 0u : 1u);
        tc_commit(bar(B_PV_DONE));
        tc_commit(bar(BR::V_EMPTY + s));
        return true;
      };
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x, ++it) {
        const Item w = decode_item(p, item);
        const int n_pages = p.nodes[w.node].n_pages;
        if (!wait_bar(bar(B_Q_FULL), it & 1, ctl, 0x110)) { ok = false; break; }
        tc_fence_after();
        for (int t = 0; t < n_pages; ++t, ++kv_it) {
          const int s = kv_it % S;
          const uint32_t b = kv_it & 1;
          if (!wait_bar(bar(BR::K_FULL + s), (kv_it / S) & 1, ctl, 0x114)) { ok = false; break; }
          tc_fence_after();
          const uint32_t qaddr = sbase + C::kQOff;
          const uint32_t kaddr = sbase + C::kKOff + s * C::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk / 4) * C::kPanelBytes + (kk % 4) * 32;
            mma_ss(tmem + C::kColS + b * 128, desc_k(qaddr + off), desc_k(kaddr + off), C::kIdescS,
                   kk > 0 ? 1u : 0u);
          }
          tc_commit(bar(B_S_FULL + b));
          tc_commit(bar(BR::K_EMPTY + s));
          if (t == n_pages - 1) tc_commit(bar(B_Q_EMPTY));
          if (t > 0 && !issue_pv(kv_it - 1, t == 1)) { ok = false; break; }
        }
        if (!ok) break;
        if (!issue_pv(kv_it - 1, n_pages == 1)) { ok = false; break; }
        tc_commit(bar(B_O_FULL));
      }
      // Wait (bounded) until every MMA issued by this thread has finished.
      tc_commit(bar(B_DRAIN));
      drain_wait(bar(B_DRAIN), 0);
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int row = quarter * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
    const float sl2 = p.scale_log2;
    uint32_t kv_it = 0, it = 0;
    for (int item = blockIdx.x; item < p.n_items; item += gridDim.x, ++it) {
      const Item w = decode_item(p, item);
      const AttnNode& nd = p.nodes[w.node];
      float m_run = -INFINITY, l_run = 0.f;
      bool ok = true;
      for (int t = 0; t < nd.n_pages; ++t, ++kv_it) {
        const uint32_t b = kv_it & 1;
        ok = __all_sync(0xffffffffu, wait_bar(bar(B_S_FULL + b), (kv_it >> 1) & 1, ctl, 0x120));
        if (!ok) break;
        tc_fence_after();
        const int valid = (int)(p.pages[nd.page0 + t] >> 25) + 1;
        float sv[128];
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tmem_ld32(trow + C::kColS + b * 128 + c * 32,
                    *reinterpret_cast<uint32_t(*)[32]>(&sv[c * 32]));
        tmem_wait_ld();
        float mx = -INFINITY;
#pragma unroll
        for (int i = 0; i < 128; ++i) {
          sv[i] = i < valid ? sv[i] : -INFINITY;
          mx = fmaxf(mx, sv[i]);
        }
        const float m_new = fmaxf(m_run, mx * sl2);
        const bool grow = __any_sync(0xffffffffu, t > 0 && m_new > m_run + 8.f);
        if (t == 0) {
          m_run = m_new;
        } else if (grow) {
          // Bring O up to the new max: wait for the previous P.V, scale O in TMEM.
          ok = __all_sync(0xffffffffu, wait_bar(bar(B_PV_DONE), (kv_it - 1) & 1, ctl, 0x121));
          if (!ok) break;
          tc_fence_after();
          const float alpha = ex2_approx(m_run - m_new);
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(trow + C::kColO + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(trow + C::kColO + c * 32, o);
          }
          tmem_wait_st();
          l_run *= alpha;
          m_run = m_new;
        }
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float p0 = ex2_approx(fmaf(sv[c * 32 + 2 * i], sl2, -m_run));
            const float p1 = ex2_approx(fmaf(sv[c * 32 + 2 * i + 1], sl2, -m_run));
            sum += p0 + p1;
            pk[i] = pack_bf16x2(p0, p1);
          }
          tmem_st16(trow + C::kColP + b * 64 + c * 16, pk);
        }
        l_run += sum;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(B_P_FULL + b));
      }
      if (!ok) break;
      ok = __all_sync(0xffffffffu, wait_bar(bar(B_O_FULL), it & 1, ctl, 0x122));
      if (!ok) break;
      tc_fence_after();
      const float inv = 1.f / l_run;
      const int q_local = w.qtile * 128 + row;
      const bool store = q_local < p.q_rows;
      uint4* orow = reinterpret_cast<uint4*>(
          p.out + ((int64_t)(nd.q_row0 + q_local) * H + w.head) * D);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(trow + C::kColO + c * 32, o);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
        if (store) {
#pragma unroll
          for (int v = 0; v < 4; ++v)
            orow[c * 4 + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(bar(B_O_EMPTY));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

template <int D>
int launch(const AttnParams& prm, int grid, cudaStream_t stream) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(round_attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    Cfg<D>::kSmemBytes);
  });
  if (attr_err != cudaSuccess)
    return fail(WAVE_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(attr_err));
  round_attn_kernel<D><<<grid, kThreads, Cfg<D>::kSmemBytes, stream>>>(prm);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(WAVE_ERR_CUDA, "round_attn_kernel launch: %s", cudaGetErrorString(e));
  return WAVE_OK;
}

}  // namespace

}  // namespace wavei

using namespace wavei;

extern "C" int wave_round_attn(wave_kv* kv, const wave_node* active, int32_t n_active,
                               int32_t policy, const void* Q, void* O, void* stream) {
  clear_error();
  if (!kv) return fail(WAVE_ERR_ARG, "NULL handle");
  if (!kv->on_device) return fail(WAVE_ERR_ARG, "host-only handle (pool == NULL)");
  if (!valid_policy(policy)) return fail(WAVE_ERR_ARG, "unknown policy %d", policy);
  if (n_active < 0 || (n_active > 0 && !active)) return fail(WAVE_ERR_ARG, "bad active list");
  if (n_active == 0) return WAVE_OK;
  if (n_active > WAVE_MAX_NODES)
    return fail(WAVE_ERR_CAPACITY, "%d active nodes exceed %d", n_active, WAVE_MAX_NODES);
  if (!Q || !O || ((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(O)) & 15))
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
  prm.tm_kv = kv->tm_kv;
  prm.out = static_cast<uint16_t*>(O);
  prm.status = static_cast<int32_t*>(kv->cfg.pool);
  prm.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  prm.heads = H;
  prm.q_rows = T;
  prm.n_nodes = n_active;

  // Longest key list first (ties keep list order): a static round-robin of
  // items over persistent CTAs then approximates longest-processing-time order.
  std::vector<int> order(n_active);
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) {
    return offs[a + 1] - offs[a] > offs[b + 1] - offs[b];
  });
  const int n_qtiles = (T + 127) / 128;
  int32_t item0 = 0, w = 0;
  for (int k = 0; k < n_active; ++k) {
    const int i = order[k];
    AttnNode& nd = prm.nodes[k];
    nd.q_row0 = i * T;
    nd.page0 = w;
    nd.n_pages = offs[i + 1] - offs[i];
    nd.item0 = item0;
    nd.n_qtiles = n_qtiles;
    for (int32_t rr = offs[i]; rr < offs[i + 1]; ++rr)
      prm.pages[w++] = (uint32_t)rows[2 * rr] | ((uint32_t)(rows[2 * rr + 1] - 1) << 25);
    item0 += H * n_qtiles;
  }
  prm.n_items = item0;
  const int grid = std::min(prm.n_items, kv->num_sms);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return D == 128 ? launch<128>(prm, grid, s) : launch<64>(prm, grid, s);
}
