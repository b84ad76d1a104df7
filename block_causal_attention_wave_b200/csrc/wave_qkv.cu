// QKV projection of one node's tokens with the K/V append fused into the
// epilogue, on sm_100a.
//
// What it computes: the node's Q, K, V = X W^T (X [T][C] hidden states, W
// [3 H d][C] a linear layer's weight, output feature (s H + h) d + j = Q, K or
// V (s = 0, 1, 2) of head h, component j), fp32 accumulation, bf16 results.
// Q goes to the caller's [T][H][d] buffer; K and V go straight into the pages
// of the node's new cache entry, in the layout wave_kv_append writes ([H][128]
// [d] of K, then of V, per page; rows past the T tokens zero). This is the
// producing side of the in-round K/V delivery of the Wave Forcing page ("Key
// Findings"): the K/V reach the round's cache without a separate copy.
//
// How. With d = 128 and 3 H even the projection runs on the persistent
// 128 x 256 GEMM of wave_gemm.cu (its QKV mode). Otherwise (d = 64, or 3 H
// odd) one CTA per output tile of 128 tokens x one head's d features of Q, K
// or V -- for K and V exactly one page tile. 128 threads:
//   warp 0 lane 0  TMA producer: 64-column slices of the X tile and the W tile
//                  (both K-major, 128-byte swizzle) into a 3-stage ring;
//   warp 1 lane 0  tcgen05 issuer: four M128 x Nd x K16 MMAs per slice into
//                  one fp32 TMEM accumulator; releases each stage by commit;
//   all 4 warps    epilogue: each thread reads its token row from TMEM,
//                  rounds to bf16 and stores it (Q row or page row).
// Token rows past T are loaded as zeros by TMA, so their K/V rows are zero.
// Two CTAs fit on an SM, so one's epilogue overlaps the other's main loop.
// Every wait is bounded; on timeout the status word records it and the kernel
// frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <string>

#include "ptx.cuh"
#include "wave_internal.h"
#include "wave_sync.cuh"

using namespace wptx;

namespace wavei {
namespace {

constexpr int kQkvThreads = 128;
constexpr int kQkvStages = 3;

template <int D>
struct QkvCfg {
  static constexpr int kATile = 128 * 128;  // 128 token rows x 64 bf16
  static constexpr int kBTile = D * 128;    // D weight rows x 64 bf16
  static constexpr int kStage = kATile + kBTile;
  static constexpr int kBarOff = kQkvStages * kStage;
  static constexpr int kBars = 2 * kQkvStages + 1;  // FULL[s], EMPTY[s], DONE
  static constexpr int kSmemBytes = kBarOff + 128 + 1024;  // + barriers/slots + alignment
  static_assert(kBars * 8 + 8 <= 128, "barrier area");
  // kind::f16 instruction descriptor: fp32 accumulate, bf16 A and B, both
  // K-major, N = D, M = 128.
  static constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                                     ((uint32_t(D) >> 3) << 17) | ((128u >> 4) << 24);
};

struct QkvParams {
  CUtensorMap tm_x;     // X [T][C] bf16, box 64 x 128
  CUtensorMap tm_w;     // W [3 H D][C] bf16, box 64 x D
  uint16_t* q;          // Q [T][H][D] bf16
  uint8_t* data;        // pool + data_offset
  int64_t page_bytes;
  int32_t* status;      // device status word (pool header)
  uint64_t wait_ns;     // bound on one barrier wait
  int32_t ntokens;
  int32_t heads;
  int32_t k_slices;     // C / 64
  int32_t n_mtiles;     // 128-token tiles = the entry's pages
  int32_t pad;
  int32_t pages[WAVE_MAX_APPEND_PAGES];  // the entry's pages, one per 128 tokens
};
static_assert(sizeof(QkvParams) <= 32760, "kernel parameter space is 32 KB");

template <int D>
__global__ void __launch_bounds__(kQkvThreads, 2) qkv_append_kernel(const __grid_constant__ QkvParams p) {
  using C = QkvCfg<D>;
  constexpr int S = kQkvStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_addr(smem);
  auto bar = [&](int i) -> uint32_t { return sb + C::kBarOff + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kBarOff + 8 * C::kBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kBarOff + 8 * C::kBars + 4);
  const Ctl ctl{abort_flag, p.status, p.wait_ns};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tile = blockIdx.x;          // 128-token tile = page of the entry
  const int which = blockIdx.y / p.heads;  // 0 Q, 1 K, 2 V
  const int head = blockIdx.y - which * p.heads;
  const int nk = p.k_slices;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(bar(s), 1);
      mbar_init(bar(S + s), 1);
    }
    mbar_init(bar(2 * S), 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&p.tm_x);
    prefetch_tmap(&p.tm_w);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // Producer. Slice k goes to stage k % S once the MMAs of slice k - S freed it.
    int issued = 0;
    for (int k = 0; k < nk; ++k) {
      const int s = k % S;
      if (k >= S && !wait_bar(bar(S + s), ((k / S) - 1) & 1, ctl, 0x201)) break;
      const uint32_t a = sb + s * C::kStage;
      mbar_arrive_expect_tx(bar(s), C::kStage);
      tma_load_2d(a, &p.tm_x, k * 64, m_tile * 128, bar(s));
      tma_load_2d(a + C::kATile, &p.tm_w, k * 64, blockIdx.y * D, bar(s));
      ++issued;
    }
    // Copies still in flight must land before the CTA exits (the last one per
    // stage; earlier ones completed before their stage was reused).
    for (int k = issued > S ? issued - S : 0; k < issued; ++k) drain_wait(bar(k % S), (k / S) & 1);
  } else if (warp == 1 && lane == 0) {
    // MMA issuer.
    for (int k = 0; k < nk; ++k) {
      const int s = k % S;
      if (!wait_bar(bar(s), (k / S) & 1, ctl, 0x202)) break;
      tc_fence_after();
      const uint32_t a = sb + s * C::kStage;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss(tmem, desc_k(a + kk * 32), desc_k(a + C::kATile + kk * 32), C::kIdesc,
               (k | kk) != 0 ? 1u : 0u);
      tc_commit(bar(S + s));
    }
    tc_commit(bar(2 * S));  // every MMA issued above is done
  }
  __syncwarp();

  // Epilogue: thread r of the CTA owns token row r of the tile (TMEM lane r).
  bool ok = wait_bar(bar(2 * S), 0, ctl, 0x203);
  if (!ok) drain_wait(bar(2 * S), 0);
  __syncwarp();
  tc_fence_after();
  ok = __all_sync(0xffffffffu, ok && !*abort_flag);
  if (ok) {
    const int row = warp * 32 + lane;
    const int token = m_tile * 128 + row;
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    uint4* dst;
    bool store;
    if (which == 0) {
      dst = reinterpret_cast<uint4*>(p.q + ((int64_t)token * p.heads + head) * D);
      store = token < p.ntokens;
    } else {
      dst = reinterpret_cast<uint4*>(p.data + (int64_t)p.pages[m_tile] * p.page_bytes +
                                     ((((int64_t)(which - 1) * p.heads + head) * 128 + row) * D) * 2);
      store = true;  // rows past the tokens hold zeros: the page tail
    }
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t v[32];
      tmem_ld32_wait(trow + 32 * c, v);
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
      if (store) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          dst[c * 4 + j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
      }
      __syncwarp();  // Q rows past the tokens skip the store: reconverge before the next tcgen05.ld
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

template <int D>
int launch_qkv(const QkvParams& prm, dim3 grid, cudaStream_t stream) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(qkv_append_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    QkvCfg<D>::kSmemBytes);
  });
  if (attr_err != cudaSuccess)
    return fail(WAVE_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(attr_err));
  qkv_append_kernel<D><<<grid, kQkvThreads, QkvCfg<D>::kSmemBytes, stream>>>(prm);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(WAVE_ERR_CUDA, "qkv_append_kernel launch: %s", cudaGetErrorString(e));
  return WAVE_OK;
}

int qkv_append_impl(wave_kv* kv, wave_node node, const wave_entry& ent, const void* X,
                    int32_t dim, const void* W, void* Q, void* stream) {
  const int H = kv->cfg.heads, D = kv->cfg.head_dim;
  // d = 128 with 3 H even: the persistent 128 x 256 GEMM of wave_gemm.cu.
  if (qkv_wide_supported(kv))
    return qkv_wide_launch(kv, 1, &node, ent.ntokens, X, dim, W, nullptr, Q, stream);
  static thread_local QkvParams prm;
  std::memset(&prm, 0, offsetof(QkvParams, pages));
  auto encode = tensor_map_encoder();
  if (!encode) return fail(WAVE_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  cuuint32_t estr[2] = {1, 1};
  {
    cuuint64_t dims[2] = {(cuuint64_t)dim, (cuuint64_t)ent.ntokens};
    cuuint64_t strides[1] = {(cuuint64_t)dim * 2};
    cuuint32_t box[2] = {64, 128};
    CUresult r = encode(&prm.tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(X), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(WAVE_ERR_CUDA, "cuTensorMapEncodeTiled(X) failed: %d", (int)r);
  }
  {
    cuuint64_t dims[2] = {(cuuint64_t)dim, (cuuint64_t)3 * H * D};
    cuuint64_t strides[1] = {(cuuint64_t)dim * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)D};
    CUresult r = encode(&prm.tm_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(W), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(WAVE_ERR_CUDA, "cuTensorMapEncodeTiled(W) failed: %d", (int)r);
  }
  prm.q = static_cast<uint16_t*>(Q);
  prm.data = static_cast<uint8_t*>(kv->cfg.pool) + kv->data_offset;
  prm.page_bytes = kv->page_bytes;
  prm.status = static_cast<int32_t*>(kv->cfg.pool);
  prm.wait_ns = wait_limit_ns(kv);
  prm.ntokens = ent.ntokens;
  prm.heads = H;
  prm.k_slices = dim / 64;
  const int n_pages = (int)ent.pages.size();
  std::memcpy(prm.pages, ent.pages.data(), n_pages * sizeof(int32_t));
  prm.n_mtiles = n_pages;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  dim3 grid((unsigned)n_pages, (unsigned)(3 * H));
  return D == 128 ? launch_qkv<128>(prm, grid, s) : launch_qkv<64>(prm, grid, s);
}

}  // namespace
}  // namespace wavei

using namespace wavei;

extern "C" int wave_qkv_append(wave_kv* kv, int32_t chunk, int32_t level, const void* X,
                               int32_t ntokens, int32_t dim, const void* W, void* Q, void* stream) {
  clear_error();
  if (!kv) return fail(WAVE_ERR_ARG, "NULL handle");
  if (!kv->on_device) return fail(WAVE_ERR_ARG, "host-only handle (pool == NULL) cannot append");
  if (int rc = check_current_device(kv)) return rc;
  if (kv->fp8) return fail(WAVE_ERR_UNSUPPORTED, "the fused projection writes bf16 pages; "
                           "append to an FP8 pool with wave_kv_append");
  if (!X || !W || !Q ||
      ((reinterpret_cast<uintptr_t>(X) | reinterpret_cast<uintptr_t>(W) | reinterpret_cast<uintptr_t>(Q)) & 15))
    return fail(WAVE_ERR_ARG, "X, W and Q must be non-NULL and 16-byte aligned");
  if (dim < 64 || dim % 64 != 0 || dim > (1 << 16))
    return fail(WAVE_ERR_ARG, "dim must be a positive multiple of 64 (at most 65536), got %d", dim);
  if (ntokens < 1) return fail(WAVE_ERR_ARG, "ntokens must be positive");
  const int64_t need = ((int64_t)ntokens + kPageTokens - 1) / kPageTokens;
  if (need > WAVE_MAX_APPEND_PAGES)
    return fail(WAVE_ERR_CAPACITY, "%lld pages exceed %d per append call", (long long)need,
                WAVE_MAX_APPEND_PAGES);
  int rc = wave_kv_alloc(kv, chunk, level, ntokens);
  if (rc) return rc;
  const wave_entry& e = kv->entries.at(std::make_pair(chunk, level));
  rc = qkv_append_impl(kv, wave_node{chunk, level}, e, X, dim, W, Q, stream);
  if (rc) {
    std::string keep = wave_last_error_detail();
    wave_kv_release(kv, chunk, level);
    fail(rc, "%s", keep.c_str());
  }
  return rc;
}
