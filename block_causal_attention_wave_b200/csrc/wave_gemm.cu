// The dense matrix products of one transformer block of a wave round, on
// sm_100a: the QKV projection of all the round's nodes (rotary embedding of Q
// and K and the K/V append fused into the epilogue), the out-projection and
// the two MLP products (tanh-GELU or residual add fused into the epilogue).
//
// What it computes (Wave Forcing page, "Key Findings": one output chunk per
// concurrent forward round, early K/V delivery; design-space paper, abstract:
// several denoising nodes processed together). The pages give no formula for
// the block; the readings are those of the float64 oracle: [Q|K|V] = X Wqkv^T
// with Q and K turned by a 3-axis (frame, row, column) rotary embedding and K,
// V written into the nodes' new cache pages; Y = X + A Wo^T; Z = Y +
// GELU(Y W1^T) W2^T; bf16 storage between the products, fp32 accumulation.
//
// How (one kernel, B200 design): C = A B^T with A [M][K] and B [N][K] both
// K-major bf16, tiles of 128 rows x 256 columns, one persistent CTA per SM
// walking its tiles. Tiles run row-tile-major: concurrent CTAs share A row
// tiles, and B (the weights, at most a few tens of MB) stays in L2, so A -- the
// activations, up to hundreds of MB -- comes from DRAM once.
// 192 threads:
//   warp 0 lane 0  TMA producer: 64-column slices of the A and B tiles
//                  (128-byte swizzle) into a 4-stage shared-memory ring that
//                  runs across tiles;
//   warp 1 lane 0  tcgen05 issuer: four M128 x N256 x K16 MMAs per slice into
//                  one of two fp32 TMEM accumulators (256 columns each);
//   warps 2..5     epilogue: thread r owns row r of a tile, reads it from
//                  TMEM 32 columns at a time, applies the mode's elementwise
//                  step and stores bf16, while the MMAs of the next tile run
//                  into the other accumulator.
// A 128 x 256 tile moves 96 KB through shared memory per 512 tensor cycles
// (TMA in, MMAs out) -- the reason for the wide tile. Every wait is bounded;
// on timeout the status word records it and the kernel frees TMEM and
// returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "ptx.cuh"
#include "wave_internal.h"
#include "wave_sync.cuh"

using namespace wptx;

namespace wavei {

namespace {

constexpr int kGemmThreads = 192;
constexpr int kGemmStages = 4;
constexpr int kRopePairs = 64;  // d = 128

struct GemmCfg {
  static constexpr int kATile = 128 * 128;  // 128 rows x 64 bf16
  static constexpr int kBTile = 256 * 128;  // 256 rows x 64 bf16
  static constexpr int kStage = kATile + kBTile;
  static constexpr int kBarOff = kGemmStages * kStage;
  // FULL[s], EMPTY[s], ACC_FULL[2], ACC_EMPTY[2], DRAIN
  static constexpr int kFull = 0, kEmpty = kGemmStages, kAccFull = 2 * kGemmStages,
                       kAccEmpty = kAccFull + 2, kDrain = kAccEmpty + 2, kBars = kDrain + 1;
  static constexpr int kSmemBytes = kBarOff + 128 + 1024;
  static_assert(kBars * 8 + 8 <= 128, "barrier area");
  // kind::f16: fp32 accumulate, bf16 A and B, both K-major, N = 256, M = 128.
  static constexpr uint32_t kIdesc =
      (1u << 4) | (1u << 7) | (1u << 10) | ((256u >> 3) << 17) | ((128u >> 4) << 24);
};

enum : int32_t { MODE_QKV = 0, MODE_LINEAR = 1 };

struct GemmParams {
  CUtensorMap tm_a;  // A [rows][K] bf16, box 64 x 128
  CUtensorMap tm_b;  // B [N][K] bf16, box 64 x 256
  int32_t* status;   // device status word (pool header)
  uint64_t wait_ns;  // bound on one barrier wait
  int32_t mode;
  int32_t k_slices;  // K / 64
  int32_t n_mtiles;  // 128-row tiles
  int32_t n_ntiles;  // 256-column tiles
  int32_t n_tiles;   // n_mtiles * n_ntiles
  // MODE_LINEAR: Y [M][N] = act(A B^T) (+ R)
  int32_t M, N;
  int32_t act;             // 0 none, 1 tanh-GELU
  uint16_t* y;
  const uint16_t* resid;   // R [M][N] or null
  // MODE_QKV: node i's rows are A rows i T .. i T + T - 1; its m-tile j
  // (ceil(T / 128) per node) is page pages[i * mt_per_node + j].
  uint16_t* q;             // Q [n T][H][128]
  uint8_t* data;           // pool + data_offset
  int64_t page_bytes;
  int32_t heads;
  int32_t tokens;          // T
  int32_t mt_per_node;
  int32_t rope;            // 1: turn Q and K
  int32_t rope_frames, rope_rows, rope_cols;
  float rope_theta[kRopePairs];   // radians per position step of each pair
  int32_t rope_axis[kRopePairs];  // 0 frame, 1 row, 2 column
  int32_t node_chunk[WAVE_MAX_NODES];
  int32_t pages[WAVE_MAX_APPEND_PAGES];
};
static_assert(sizeof(GemmParams) <= 32760, "kernel parameter space is 32 KB");

// GELU, tanh form, through 0.5 (1 + tanh u) = 1 / (1 + e^(-2u)): one
// exponential and one division on the special-function unit, with relative
// accuracy everywhere (the tail where 1 + tanh u is tiny included).
__device__ __forceinline__ float gelu_tanh(float x) {
  const float u = 0.7978845608028654f * fmaf(0.044715f * x, x * x, x);
  return __fdividef(x, 1.f + __expf(-2.f * u));
}

// sin and cos of a rotary angle: reduced to [-pi, pi] by subtracting the
// nearest multiple of 2 pi (Cody-Waite: 2 pi split into 6.28125, exact in a
// few bits, plus the remainder, so k * 6.28125 is exact for the k that occur),
// then the special-function unit's sin/cos, accurate to ~4e-7 on [-pi, pi].
__device__ __forceinline__ void rope_sincos(float a, float* sn, float* cs) {
  const float k = rintf(a * 0.15915494309189535f);
  float r = fmaf(-k, 6.28125f, a);
  r = fmaf(-k, 1.9353071795864769e-3f, r);
  __sincosf(r, sn, cs);
}

__device__ __forceinline__ int64_t a_row0(const GemmParams& p, int mt) {
  if (p.mode == MODE_QKV) {
    const int node = mt / p.mt_per_node;
    return (int64_t)node * p.tokens + (int64_t)(mt - node * p.mt_per_node) * 128;
  }
  return (int64_t)mt * 128;
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_wide_kernel(const __grid_constant__ GemmParams p) {
  using C = GemmCfg;
  constexpr int S = kGemmStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_addr(smem);
  auto bar = [&](int i) -> uint32_t { return sb + C::kBarOff + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kBarOff + 8 * C::kBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kBarOff + 8 * C::kBars + 4);
  const Ctl ctl{abort_flag, p.status, p.wait_ns};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = p.k_slices, n_tiles = p.n_tiles, n_n = p.n_ntiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(bar(C::kFull + s), 1);
      mbar_init(bar(C::kEmpty + s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar(C::kAccFull + a), 1);
      mbar_init(bar(C::kAccEmpty + a), 128);
    }
    mbar_init(bar(C::kDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&p.tm_a);
    prefetch_tmap(&p.tm_b);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // Producer: slices of every tile of this CTA through one ring.
      uint32_t g = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        const int mt = t / n_n, nt = t - mt * n_n;
        const int32_t row0 = (int32_t)a_row0(p, mt);
        for (int k = 0; k < nk; ++k, ++g) {
          const uint32_t s = g % S;
          if (g >= (uint32_t)S && !wait_bar(bar(C::kEmpty + s), ((g / S) - 1) & 1, ctl, 0x301)) {
            ok = false;
            break;
          }
          const uint32_t a = sb + s * C::kStage;
          mbar_arrive_expect_tx(bar(C::kFull + s), C::kStage);
          tma_load_2d(a, &p.tm_a, k * 64, row0, bar(C::kFull + s));
          tma_load_2d(a + C::kATile, &p.tm_b, k * 64, nt * 256, bar(C::kFull + s));
        }
      }
      // Copies still in flight land before the CTA exits.
      for (uint32_t k = g > (uint32_t)S ? g - S : 0; k < g; ++k)
        drain_wait(bar(C::kFull + k % S), (k / S) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // MMA issuer: tile i of this CTA accumulates in TMEM columns 256 (i % 2).
      uint32_t g = 0, i = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++i) {
        const uint32_t acc = i & 1;
        if (i >= 2 && !wait_bar(bar(C::kAccEmpty + acc), ((i >> 1) - 1) & 1, ctl, 0x302)) break;
        tc_fence_after();
        for (int k = 0; k < nk; ++k, ++g) {
          const uint32_t s = g % S;
          if (!wait_bar(bar(C::kFull + s), (g / S) & 1, ctl, 0x303)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = sb + s * C::kStage;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tmem + 256 * acc, desc_k(a + kk * 32), desc_k(a + C::kATile + kk * 32),
                   C::kIdesc, (k | kk) != 0 ? 1u : 0u);
          tc_commit(bar(C::kEmpty + s));
        }
        if (ok) tc_commit(bar(C::kAccFull + acc));
      }
      // Every MMA issued above completes before TMEM is released.
      tc_commit(bar(C::kDrain));
      drain_wait(bar(C::kDrain), 0);
    }
  } else {
    // Epilogue: thread r of warps 2..5 owns row r of each tile (TMEM lane r;
    // warp w may read lanes 32 (w % 4) ..).
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
    uint32_t i = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
      const uint32_t acc = i & 1;
      const bool ok =
          __all_sync(0xffffffffu, wait_bar(bar(C::kAccFull + acc), (i >> 1) & 1, ctl, 0x304));
      if (!ok) break;
      tc_fence_after();
      const int mt = t / n_n, nt = t - mt * n_n;
      if (p.mode == MODE_LINEAR) {
        const int64_t r = (int64_t)mt * 128 + row;
        const bool in = r < p.M;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          const int64_t col0 = (int64_t)nt * 256 + 32 * c;
          uint32_t v[32];
          tmem_ld32_wait(trow + 256 * acc + 32 * c, v);
          float f[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) f[j] = __uint_as_float(v[j]);
          if (p.act == 1) {
#pragma unroll
            for (int j = 0; j < 32; ++j) f[j] = gelu_tanh(f[j]);
          }
          if (in) {
            if (p.resid) {
              const uint4* rp = reinterpret_cast<const uint4*>(p.resid + r * p.N + col0);
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const uint4 w4 = rp[j];
                const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  f[8 * j + 2 * e] += __uint_as_float(w[e] << 16);
                  f[8 * j + 2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
                }
              }
            }
            uint4* dst = reinterpret_cast<uint4*>(p.y + r * p.N + col0);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              dst[j] = make_uint4(pack_bf16x2(f[8 * j], f[8 * j + 1]),
                                  pack_bf16x2(f[8 * j + 2], f[8 * j + 3]),
                                  pack_bf16x2(f[8 * j + 4], f[8 * j + 5]),
                                  pack_bf16x2(f[8 * j + 6], f[8 * j + 7]));
          }
          __syncwarp();  // rows past M skip the store: reconverge before the next tcgen05.ld
        }
      } else {
        // QKV: the tile holds two head slices of 128 features each.
        const int node = mt / p.mt_per_node, m = mt - node * p.mt_per_node;
        const int token = m * 128 + row;  // within the node
        const bool in = token < p.tokens;
        const int page = p.pages[mt];
        float pos[3] = {0.f, 0.f, 0.f};
        if (p.rope) {
          const int rc = p.rope_rows * p.rope_cols;
          pos[0] = (float)(p.node_chunk[node] * p.rope_frames + token / rc);
          pos[1] = (float)((token / p.rope_cols) % p.rope_rows);
          pos[2] = (float)(token % p.rope_cols);
        }
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          const int n = 2 * nt + h;  // head slice: feature n * 128 ..
          const int which = n / p.heads, head = n - which * p.heads;
          const bool turn = p.rope && which < 2;
          uint4* dst;
          if (which == 0)
            dst = reinterpret_cast<uint4*>(p.q + (((int64_t)node * p.tokens + token) * p.heads + head) * 128);
          else
            dst = reinterpret_cast<uint4*>(p.data + (int64_t)page * p.page_bytes +
                                           ((((int64_t)(which - 1) * p.heads + head) * 128 + row) * 128) * 2);
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t v[32];
            tmem_ld32_wait(trow + 256 * acc + 128 * h + 32 * c, v);
            float f[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) f[j] = __uint_as_float(v[j]);
            if (turn) {
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const int pr = 16 * c + j;
                float sn, cs;
                rope_sincos(pos[p.rope_axis[pr]] * p.rope_theta[pr], &sn, &cs);
                const float a = f[2 * j], b = f[2 * j + 1];
                f[2 * j] = a * cs - b * sn;
                f[2 * j + 1] = a * sn + b * cs;
              }
            }
            if (!in) {  // rows past the node's tokens: zero page tail (K, V)
#pragma unroll
              for (int j = 0; j < 32; ++j) f[j] = 0.f;
            }
            if (which != 0 || in) {
#pragma unroll
              for (int j = 0; j < 4; ++j)
                dst[c * 4 + j] = make_uint4(pack_bf16x2(f[8 * j], f[8 * j + 1]),
                                            pack_bf16x2(f[8 * j + 2], f[8 * j + 3]),
                                            pack_bf16x2(f[8 * j + 4], f[8 * j + 5]),
                                            pack_bf16x2(f[8 * j + 6], f[8 * j + 7]));
            }
            __syncwarp();  // Q rows past the node skip the store: reconverge before the next tcgen05.ld
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar(C::kAccEmpty + acc));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

int launch_gemm(const GemmParams& prm, int grid, cudaStream_t stream) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(gemm_wide_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    GemmCfg::kSmemBytes);
  });
  if (attr_err != cudaSuccess)
    return fail(WAVE_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(attr_err));
  gemm_wide_kernel<<<grid, kGemmThreads, GemmCfg::kSmemBytes, stream>>>(prm);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(WAVE_ERR_CUDA, "gemm_wide_kernel launch: %s", cudaGetErrorString(e));
  return WAVE_OK;
}

// Tensor map over a K-major bf16 matrix [rows][k] with a box of 64 x box_rows.
int encode_kmajor(CUtensorMap* map, const void* base, int64_t rows, int64_t k, uint32_t box_rows,
                  const char* what) {
  auto encode = tensor_map_encoder();
  if (!encode) return fail(WAVE_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  cuuint64_t dims[2] = {(cuuint64_t)k, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)k * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                      strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(WAVE_ERR_CUDA, "cuTensorMapEncodeTiled(%s) failed: %d", what, (int)r);
  return WAVE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

bool qkv_wide_supported(const wave_kv* kv) {
  return kv->cfg.head_dim == 128 && (3 * kv->cfg.heads) % 2 == 0;
}

int qkv_wide_launch(wave_kv* kv, int32_t n, const wave_node* nodes, int32_t T, const void* X,
                    int32_t dim, const void* W, const wave_rope* rope, void* Q, void* stream) {
  static thread_local GemmParams prm;
  std::memset(&prm, 0, offsetof(GemmParams, pages));
  const int H = kv->cfg.heads;
  const int mt_per_node = (T + kPageTokens - 1) / kPageTokens;
  if ((int64_t)n * mt_per_node > WAVE_MAX_APPEND_PAGES)
    return fail(WAVE_ERR_CAPACITY, "%lld pages exceed %d per append call",
                (long long)n * mt_per_node, WAVE_MAX_APPEND_PAGES);
  if (int rc = encode_kmajor(&prm.tm_a, X, (int64_t)n * T, dim, 128, "X")) return rc;
  if (int rc = encode_kmajor(&prm.tm_b, W, (int64_t)3 * H * 128, dim, 256, "W")) return rc;
  prm.status = static_cast<int32_t*>(kv->cfg.pool);
  prm.wait_ns = wait_limit_ns(kv);
  prm.mode = MODE_QKV;
  prm.k_slices = dim / 64;
  prm.n_mtiles = n * mt_per_node;
  prm.n_ntiles = 3 * H / 2;
  prm.n_tiles = prm.n_mtiles * prm.n_ntiles;
  prm.q = static_cast<uint16_t*>(Q);
  prm.data = static_cast<uint8_t*>(kv->cfg.pool) + kv->data_offset;
  prm.page_bytes = kv->page_bytes;
  prm.heads = H;
  prm.tokens = T;
  prm.mt_per_node = mt_per_node;
  if (rope) {
    prm.rope = 1;
    prm.rope_frames = rope->frames;
    prm.rope_rows = rope->rows;
    prm.rope_cols = rope->cols;
    // Pairs 0 .. P - 2 (P // 3) - 1 turn with the frame, then P // 3 with the
    // row and P // 3 with the column; pair i of a group of n turns by
    // base^(-i / n) radians per position step (P = d / 2 = 64).
    const int n_hw = kRopePairs / 3, n_t = kRopePairs - 2 * n_hw;
    const int sizes[3] = {n_t, n_hw, n_hw};
    int p0 = 0;
    for (int axis = 0; axis < 3; ++axis) {
      for (int i = 0; i < sizes[axis]; ++i) {
        prm.rope_theta[p0 + i] = (float)std::pow((double)rope->base, -(double)i / sizes[axis]);
        prm.rope_axis[p0 + i] = axis;
      }
      p0 += sizes[axis];
    }
  }
  for (int32_t i = 0; i < n; ++i) {
    const wave_entry& ent = kv->entries.at(std::make_pair(nodes[i].chunk, nodes[i].level));
    prm.node_chunk[i] = nodes[i].chunk;
    std::memcpy(prm.pages + i * mt_per_node, ent.pages.data(), mt_per_node * sizeof(int32_t));
  }
  return launch_gemm(prm, std::min(prm.n_tiles, kv->num_sms), static_cast<cudaStream_t>(stream));
}

}  // namespace wavei

using namespace wavei;

extern "C" int wave_qkv_append_round(wave_kv* kv, const wave_node* nodes, int32_t n_nodes,
                                     const void* X, int32_t dim, const void* W,
                                     const wave_rope* rope, void* Q, void* stream) {
  clear_error();
  if (!kv) return fail(WAVE_ERR_ARG, "NULL handle");
  if (!kv->on_device) return fail(WAVE_ERR_ARG, "host-only handle (pool == NULL) cannot append");
  if (int rc = check_current_device(kv)) return rc;
  if (n_nodes < 1 || n_nodes > WAVE_MAX_NODES || !nodes)
    return fail(WAVE_ERR_ARG, "need 1..%d nodes, got %d", WAVE_MAX_NODES, n_nodes);
  if (!qkv_wide_supported(kv))
    return fail(WAVE_ERR_UNSUPPORTED, "the round projection needs head_dim 128 and 3 * heads even");
  if (kv->fp8) return fail(WAVE_ERR_UNSUPPORTED, "the fused projection writes bf16 pages; "
                           "append to an FP8 pool with wave_kv_append_batch");
  if (!X || !W || !Q || !aligned16(X) || !aligned16(W) || !aligned16(Q))
    return fail(WAVE_ERR_ARG, "X, W and Q must be non-NULL and 16-byte aligned");
  if (dim < 64 || dim % 64 != 0 || dim > (1 << 16))
    return fail(WAVE_ERR_ARG, "dim must be a positive multiple of 64 (at most 65536), got %d", dim);
  const int T = kv->cfg.tokens_per_chunk;
  if (rope) {
    if (rope->frames < 1 || rope->rows < 1 || rope->cols < 1 ||
        (int64_t)rope->frames * rope->rows * rope->cols != T || !(rope->base > 1.f))
      return fail(WAVE_ERR_ARG, "rope grid %d x %d x %d does not cover %d tokens (or base <= 1)",
                  rope->frames, rope->rows, rope->cols, T);
  }
  const int64_t need = (int64_t)n_nodes * ((T + kPageTokens - 1) / kPageTokens);
  if (need > WAVE_MAX_APPEND_PAGES)
    return fail(WAVE_ERR_CAPACITY, "%lld pages exceed %d per append call", (long long)need,
                WAVE_MAX_APPEND_PAGES);
  int32_t free_pages = 0;
  wave_kv_free_pages(kv, &free_pages);
  if (need > free_pages)
    return fail(WAVE_ERR_NO_PAGES, "need %lld pages, %d free", (long long)need, free_pages);
  // Take the pages in node order (as wave_kv_alloc calls in that order would);
  // on any error give back what was taken.
  int32_t taken = 0;
  int rc = WAVE_OK;
  for (; taken < n_nodes; ++taken) {
    rc = wave_kv_alloc(kv, nodes[taken].chunk, nodes[taken].level, T);
    if (rc) break;
  }
  if (!rc) rc = qkv_wide_launch(kv, n_nodes, nodes, T, X, dim, W, rope, Q, stream);
  if (rc) {
    std::string keep = wave_last_error_detail();
    for (int32_t i = 0; i < taken; ++i) wave_kv_release(kv, nodes[i].chunk, nodes[i].level);
    fail(rc, "%s", keep.c_str());
  }
  return rc;
}

extern "C" int wave_linear(wave_kv* kv, const void* A, int32_t M, int32_t K, const void* W,
                           int32_t N, const void* R, int32_t act, void* Y, void* stream) {
  clear_error();
  if (!kv) return fail(WAVE_ERR_ARG, "NULL handle");
  if (!kv->on_device) return fail(WAVE_ERR_ARG, "host-only handle (pool == NULL) cannot launch");
  if (int rc = check_current_device(kv)) return rc;
  if (M < 1 || K < 64 || K % 64 != 0 || K > (1 << 16) || N < 256 || N % 256 != 0 || N > (1 << 16))
    return fail(WAVE_ERR_ARG, "need M >= 1, K a multiple of 64 and N a multiple of 256 "
                "(K, N <= 65536); got M %d, K %d, N %d", M, K, N);
  if ((int64_t)M * N >= (1LL << 40)) return fail(WAVE_ERR_ARG, "M x N too large");
  if (act != WAVE_ACT_NONE && act != WAVE_ACT_GELU_TANH)
    return fail(WAVE_ERR_ARG, "unknown activation %d", act);
  if (!A || !W || !Y || !aligned16(A) || !aligned16(W) || !aligned16(Y) || (R && !aligned16(R)))
    return fail(WAVE_ERR_ARG, "A, W, Y (and R) must be non-NULL and 16-byte aligned");
  static thread_local GemmParams prm;
  std::memset(&prm, 0, offsetof(GemmParams, pages));
  if (int rc = encode_kmajor(&prm.tm_a, A, M, K, 128, "A")) return rc;
  if (int rc = encode_kmajor(&prm.tm_b, W, N, K, 256, "W")) return rc;
  prm.status = static_cast<int32_t*>(kv->cfg.pool);
  prm.wait_ns = wait_limit_ns(kv);
  prm.mode = MODE_LINEAR;
  prm.k_slices = K / 64;
  prm.n_mtiles = (M + 127) / 128;
  prm.n_ntiles = N / 256;
  prm.n_tiles = prm.n_mtiles * prm.n_ntiles;
  prm.M = M;
  prm.N = N;
  prm.act = act;
  prm.y = static_cast<uint16_t*>(Y);
  prm.resid = static_cast<const uint16_t*>(R);
  return launch_gemm(prm, std::min(prm.n_tiles, kv->num_sms), static_cast<cudaStream_t>(stream));
}
