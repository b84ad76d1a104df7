// Device set-up, the status word, and the paged K/V append kernel.
//
// The append is the in-round K/V delivery of the Wave Forcing page ("Key
// Findings": early K/V delivery) and the local cache write of the Wan-Streamer
// v0.2 page (glossary "pre-sharded": incoming K/V written into a local cache).
// It is a pure copy and therefore HBM-bound: every byte of K and V is read once
// and written once, plus zero fill for the unused tail of the entry's last page.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "wave_internal.h"
#include "wave_sync.cuh"

namespace wavei {

namespace {

// One launch copies every entry of an append call. The work unit is a tile:
// one page's 128 token rows of one head, of K or of V (16 KB at d = 64, 32 KB
// at d = 128), which is one contiguous run of the destination page. A block
// takes one tile: the tile's coordinates cost one search over at most 64
// entries and two small divisions per block, nothing per element.
struct AppendEntry {
  const uint4* k;    // [ntokens][H][d] bf16 as 16-byte vectors
  const uint4* v;
  int32_t ntokens;
  int32_t n_pages;
  int32_t page0;     // index of the entry's first page in `pages`
  int32_t tile0;     // index of the entry's first tile
};

struct AppendParams {
  uint8_t* data;        // pool + data_offset
  int64_t page_bytes;
  int32_t heads;
  int32_t vec_per_row;  // head_dim / 8 (16-byte vectors per token row): 8 or 16
  int32_t log2_vec;
  int32_t n_entries;
  int32_t n_tiles;
  int32_t pad;
  AppendEntry e[WAVE_MAX_APPEND_ENTRIES];
  int32_t pages[WAVE_MAX_APPEND_PAGES];
};
static_assert(sizeof(AppendParams) <= 32760, "kernel parameter space is 32 KB");

constexpr int kAppendThreads = 256;
constexpr int kAppendPer = WAVE_PAGE_TOKENS * 16 / kAppendThreads;  // vectors per thread, d = 128

// Thread t moves vectors t, t + 256, ... of the tile: every group of
// vec_per_row threads reads one 128/256-byte token row of the source (its
// head's slice), and the block's stores fill the tile's bytes in order. Loads
// are all issued before the stores. Rows past the entry's last token are
// written as zeros.
__global__ void __launch_bounds__(kAppendThreads) kv_append_kernel(
    const __grid_constant__ AppendParams p) {
  const int tile = blockIdx.x;
  if (tile >= p.n_tiles) return;
  int ei = 0;
  while (ei + 1 < p.n_entries && tile >= p.e[ei + 1].tile0) ++ei;
  const AppendEntry& en = p.e[ei];
  int local = tile - en.tile0;
  const int per_kv = en.n_pages * p.heads;
  const int kv = local >= per_kv;
  local -= kv * per_kv;
  const int pi = local / p.heads;
  const int h = local - pi * p.heads;
  const int per_tile = WAVE_PAGE_TOKENS * p.vec_per_row;
  const uint4* src = kv ? en.v : en.k;
  uint4* dst = reinterpret_cast<uint4*>(p.data + (int64_t)p.pages[en.page0 + pi] * p.page_bytes) +
               ((int64_t)kv * p.heads + h) * per_tile;
  const int token0 = pi * WAVE_PAGE_TOKENS;
  uint4 val[kAppendPer];
#pragma unroll
  for (int u = 0; u < kAppendPer; ++u) {
    const int i = threadIdx.x + u * kAppendThreads;
    val[u] = make_uint4(0, 0, 0, 0);
    const int token = token0 + (i >> p.log2_vec);
    if (i < per_tile && token < en.ntokens)
      val[u] = __ldg(src + ((int64_t)token * p.heads + h) * p.vec_per_row + (i & (p.vec_per_row - 1)));
  }
#pragma unroll
  for (int u = 0; u < kAppendPer; ++u) {
    const int i = threadIdx.x + u * kAppendThreads;
    if (i < per_tile) dst[i] = val[u];
  }
}

// FP8 pools: the same tiles, quantised. The block loads its tile (zeros past
// the entry's tokens), reduces amax over it, takes s = amax / 448 (1 if the
// tile is zero) with an IEEE float32 division, and stores E4M3(x / s) (IEEE
// division, round to nearest even, saturating) and s into the scale table.
__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__global__ void __launch_bounds__(kAppendThreads) kv_append_fp8_kernel(
    const __grid_constant__ AppendParams p, float* scales) {
  __shared__ float warp_max[kAppendThreads / 32];
  const int tile = blockIdx.x;
  if (tile >= p.n_tiles) return;
  int ei = 0;
  while (ei + 1 < p.n_entries && tile >= p.e[ei + 1].tile0) ++ei;
  const AppendEntry& en = p.e[ei];
  int local = tile - en.tile0;
  const int per_kv = en.n_pages * p.heads;
  const int kv = local >= per_kv;
  local -= kv * per_kv;
  const int pi = local / p.heads;
  const int h = local - pi * p.heads;
  const int per_tile = WAVE_PAGE_TOKENS * p.vec_per_row;  // 8-value vectors
  const uint4* src = kv ? en.v : en.k;
  const int page = p.pages[en.page0 + pi];
  uint2* dst = reinterpret_cast<uint2*>(p.data + (int64_t)page * p.page_bytes) +
               ((int64_t)kv * p.heads + h) * per_tile;
  const int token0 = pi * WAVE_PAGE_TOKENS;
  uint4 val[kAppendPer];
  float amax = 0.f;
#pragma unroll
  for (int u = 0; u < kAppendPer; ++u) {
    const int i = threadIdx.x + u * kAppendThreads;
    val[u] = make_uint4(0, 0, 0, 0);
    const int token = token0 + (i >> p.log2_vec);
    if (i < per_tile && token < en.ntokens)
      val[u] = __ldg(src + ((int64_t)token * p.heads + h) * p.vec_per_row + (i & (p.vec_per_row - 1)));
    const uint32_t w[4] = {val[u].x, val[u].y, val[u].z, val[u].w};
#pragma unroll
    for (int e = 0; e < 4; ++e)
      amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w[e] << 16)),
                               fabsf(__uint_as_float(w[e] & 0xFFFF0000u))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = warp_max[0];
#pragma unroll
  for (int w = 1; w < kAppendThreads / 32; ++w) amax = fmaxf(amax, warp_max[w]);
  const float sc = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  if (threadIdx.x == 0) scales[((int64_t)page * 2 + kv) * p.heads + h] = sc;
#pragma unroll
  for (int u = 0; u < kAppendPer; ++u) {
    const int i = threadIdx.x + u * kAppendThreads;
    if (i >= per_tile) continue;
    const uint32_t w[4] = {val[u].x, val[u].y, val[u].z, val[u].w};
    uint32_t q[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float a = __fdiv_rn(__uint_as_float(w[2 * e] << 16), sc);
      const float b = __fdiv_rn(__uint_as_float(w[2 * e] & 0xFFFF0000u), sc);
      const float c = __fdiv_rn(__uint_as_float(w[2 * e + 1] << 16), sc);
      const float d = __fdiv_rn(__uint_as_float(w[2 * e + 1] & 0xFFFF0000u), sc);
      q[e] = (uint32_t)e4m3x2(a, b) | ((uint32_t)e4m3x2(c, d) << 16);
    }
    dst[i] = make_uint2(q[0], q[1]);
  }
}

// FP8 pools, read side: expand page tiles into bf16 staging pages laid out as
// a bf16 pool (slot i = the i-th listed page): value bf16(code * s), the
// product in float32. One block per (slot, K/V, head) tile; each thread turns
// 8 codes into one 16-byte bf16 vector.
struct ExpandParams {
  const uint8_t* data;    // FP8 pages (pool + data_offset)
  const float* scales;    // [max_pages][2][H]
  uint4* staging;         // bf16 pages, slot by slot
  int64_t page_bytes;     // FP8 page bytes
  int32_t heads;
  int32_t vec_per_row;    // d / 8
  int32_t n_slots;
  int32_t pad;
  int32_t pages[WAVE_MAX_PAGES_PER_ROUND];
};
static_assert(sizeof(ExpandParams) <= 32760, "kernel parameter space is 32 KB");

__global__ void __launch_bounds__(kAppendThreads) kv_fp8_expand_kernel(
    const __grid_constant__ ExpandParams p) {
  const int tiles_per_slot = 2 * p.heads;
  const int slot = blockIdx.x / tiles_per_slot;
  const int t = blockIdx.x - slot * tiles_per_slot;  // kv * H + h
  if (slot >= p.n_slots) return;
  const int page = p.pages[slot];
  const int per_tile = WAVE_PAGE_TOKENS * p.vec_per_row;
  const uint2* src = reinterpret_cast<const uint2*>(p.data + (int64_t)page * p.page_bytes) +
                     (int64_t)t * per_tile;
  const float sc = p.scales[(int64_t)page * tiles_per_slot + t];
  uint4* dst = p.staging + ((int64_t)slot * tiles_per_slot + t) * per_tile;
  for (int i = threadIdx.x; i < per_tile; i += kAppendThreads) {
    const uint2 c = __ldg(src + i);
    const uint32_t w[2] = {c.x, c.y};
    uint32_t out[4];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t f16x2;
        const uint16_t pair = (uint16_t)(w[e] >> (16 * half));
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(f16x2) : "h"(pair));
        const float lo = __half2float(__ushort_as_half((unsigned short)(f16x2 & 0xFFFF))) * sc;
        const float hi = __half2float(__ushort_as_half((unsigned short)(f16x2 >> 16))) * sc;
        uint32_t b;
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(b) : "f"(hi), "f"(lo));
        out[2 * e + half] = b;
      }
    }
    dst[i] = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

}  // namespace

int launch_fp8_expand(wave_kv* kv, int32_t n, const int32_t* pages, void* staging, void* stream) {
  static thread_local ExpandParams p;
  if (n < 0 || n > WAVE_MAX_PAGES_PER_ROUND) return fail(WAVE_ERR_CAPACITY, "%d pages to expand", n);
  if (n == 0) return WAVE_OK;
  const uint8_t* pool = static_cast<const uint8_t*>(kv->cfg.pool);
  p.data = pool + kv->data_offset;
  p.scales = reinterpret_cast<const float*>(pool + kv->scale_offset);
  p.staging = static_cast<uint4*>(staging);
  p.page_bytes = kv->page_bytes;
  p.heads = kv->cfg.heads;
  p.vec_per_row = kv->cfg.head_dim / 8;
  p.n_slots = n;
  std::memcpy(p.pages, pages, n * sizeof(int32_t));
  kv_fp8_expand_kernel<<<(unsigned)(n * 2 * kv->cfg.heads), kAppendThreads, 0,
                         static_cast<cudaStream_t>(stream)>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return fail(WAVE_ERR_CUDA, "kv_fp8_expand_kernel launch: %s", cudaGetErrorString(e));
  return WAVE_OK;
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

static int cuda_fail(cudaError_t e, const char* what) {
  return fail(WAVE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int device_init(wave_kv* kv) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int major = 0, minor = 0, sms = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (major != 10 || minor != 0)
    return fail(WAVE_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a",
                dev, major, minor);
  cudaPointerAttributes pa;
  e = cudaPointerGetAttributes(&pa, kv->cfg.pool);
  if (e != cudaSuccess || pa.type != cudaMemoryTypeDevice || pa.device != dev) {
    cudaGetLastError();
    return fail(WAVE_ERR_ARG, "pool is not device memory of the current device %d", dev);
  }
  kv->device = dev;
  kv->num_sms = sms;
  e = cudaMemset(kv->cfg.pool, 0, kHeaderBytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemset(pool header)");
  e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");

  // Tensor map over the page region: rows of head_dim bf16, box 64 x 128 with
  // the 128-byte swizzle the tensor-core shared-memory descriptors expect.
  // (FP8 pools are read through bf16 staging pages; they need none.)
  if (kv->fp8) return WAVE_OK;
  auto encode = tensor_map_encoder();
  if (!encode) return fail(WAVE_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  const int d = kv->cfg.head_dim, H = kv->cfg.heads;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)kv->max_pages * 2 * H * kPageTokens};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  void* base = static_cast<uint8_t*>(kv->cfg.pool) + kv->data_offset;
  CUresult r = encode(&kv->tm_kv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box,
                      estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(WAVE_ERR_CUDA, "cuTensorMapEncodeTiled(pool) failed: %d", (int)r);
  return WAVE_OK;
}

int check_current_device(const wave_kv* kv) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev != kv->device)
    return fail(WAVE_ERR_ARG, "current device %d is not the pool's device %d", dev, kv->device);
  return WAVE_OK;
}

uint64_t wait_limit_ns(const wave_kv* kv) { return kv->wait_ns ? kv->wait_ns : kTimeoutNs; }

int launch_append(wave_kv* kv, int32_t n, const wave_entry* const* entries,
                  const void* const* K, const void* const* V, void* stream) {
  static thread_local AppendParams p;  // large: keep off the stack; launch copies it
  if (n < 1 || n > WAVE_MAX_APPEND_ENTRIES) return fail(WAVE_ERR_ARG, "bad entry count %d", n);
  p.data = static_cast<uint8_t*>(kv->cfg.pool) + kv->data_offset;
  p.page_bytes = kv->page_bytes;
  p.heads = kv->cfg.heads;
  p.vec_per_row = kv->cfg.head_dim / 8;
  p.log2_vec = p.vec_per_row == 16 ? 4 : 3;
  p.n_entries = n;
  int32_t pages = 0, tiles = 0;
  for (int32_t i = 0; i < n; ++i) {
    const wave_entry& ent = *entries[i];
    const int32_t np = (int32_t)ent.pages.size();
    if (pages + np > WAVE_MAX_APPEND_PAGES)
      return fail(WAVE_ERR_CAPACITY, "more than %d pages in one append", WAVE_MAX_APPEND_PAGES);
    p.e[i] = AppendEntry{static_cast<const uint4*>(K[i]), static_cast<const uint4*>(V[i]),
                         ent.ntokens, np, pages, tiles};
    std::memcpy(p.pages + pages, ent.pages.data(), np * sizeof(int32_t));
    pages += np;
    tiles += 2 * np * p.heads;
  }
  p.n_tiles = tiles;
  if (tiles == 0) return WAVE_OK;
  if (kv->fp8) {
    float* scales = reinterpret_cast<float*>(static_cast<uint8_t*>(kv->cfg.pool) + kv->scale_offset);
    kv_append_fp8_kernel<<<(unsigned)tiles, kAppendThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        p, scales);
  } else {
    kv_append_kernel<<<(unsigned)tiles, kAppendThreads, 0, static_cast<cudaStream_t>(stream)>>>(p);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "kv_append_kernel launch");
  return WAVE_OK;
}

}  // namespace wavei

extern "C" int wave_kv_last_launch_clock(wave_kv* kv, void* stream, int64_t* cycles,
                                         int64_t* ns) {
  using namespace wavei;
  clear_error();
  if (!kv || !cycles || !ns) return fail(WAVE_ERR_ARG, "NULL argument");
  *cycles = 0;
  *ns = 0;
  if (!kv->on_device) return WAVE_OK;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int64_t words[2] = {0, 0};
  e = cudaMemcpy(words, static_cast<char*>(kv->cfg.pool) + 256, sizeof words,
                 cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(clock words)");
  *cycles = words[0];
  *ns = words[1];
  return WAVE_OK;
}

extern "C" int wave_kv_status(wave_kv* kv, void* stream) {
  using namespace wavei;
  clear_error();
  if (!kv) return fail(WAVE_ERR_ARG, "NULL handle");
  if (!kv->on_device) return WAVE_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int32_t word = 0;
  e = cudaMemcpy(&word, kv->cfg.pool, sizeof word, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(status)");
  if (word != 0) {
    int32_t zero = 0;
    cudaMemcpy(kv->cfg.pool, &zero, sizeof zero, cudaMemcpyHostToDevice);
    return fail(WAVE_ERR_TIMEOUT, "a kernel gave up on a bounded wait (status word 0x%x)", word);
  }
  return WAVE_OK;
}
