// Device set-up, the status word, and the paged K/V append kernel.
//
// The append is the in-round K/V delivery of the Wave Forcing page ("Key
// Findings": early K/V delivery) and the local cache write of the Wan-Streamer
// v0.2 page (glossary "pre-sharded": incoming K/V written into a local cache).
// It is a pure copy and therefore HBM-bound: every byte of K and V is read once
// and written once, plus zero fill for the unused tail of the entry's last page.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "wave_internal.h"

namespace wavei {

namespace {

constexpr int kMaxEntryPages = 4096;  // 512K tokens per entry

struct AppendParams {
  const uint4* k;
  const uint4* v;
  uint8_t* data;        // pool + data_offset
  int64_t page_bytes;
  int32_t ntokens;
  int32_t heads;
  int32_t n_pages;
  int32_t vec_per_row;  // head_dim / 8 (16-byte vectors per token row)
  int32_t pages[kMaxEntryPages];
};

// One 16-byte vector per thread step. The linear index walks the DESTINATION in
// order (K then V; page; head; token-in-page; vector), so stores are fully
// contiguous; each group of vec_per_row threads reads one 128/256-byte token
// row of the source, which keeps loads sector-efficient as well.
__global__ void __launch_bounds__(256) kv_append_kernel(const __grid_constant__ AppendParams p) {
  const int64_t per_head = (int64_t)WAVE_PAGE_TOKENS * p.vec_per_row;
  const int64_t per_page = per_head * p.heads;
  const int64_t per_kv = per_page * p.n_pages;
  const int64_t total = 2 * per_kv;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  constexpr int kUnroll = 4;
  for (int64_t base = (int64_t)blockIdx.x * blockDim.x * kUnroll + threadIdx.x; base < total;
       base += stride * kUnroll) {
    uint4 val[kUnroll];
    uint4* dst[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      int64_t i = base + (int64_t)u * blockDim.x;
      dst[u] = nullptr;
      if (i >= total) continue;
      int kv = i >= per_kv;
      int64_t j = i - kv * per_kv;
      int pi = (int)(j / per_page);
      int64_t r = j - (int64_t)pi * per_page;
      int h = (int)(r / per_head);
      int64_t r2 = r - (int64_t)h * per_head;
      int t = (int)(r2 / p.vec_per_row);
      int c = (int)(r2 - (int64_t)t * p.vec_per_row);
      int token = pi * WAVE_PAGE_TOKENS + t;
      const uint4* src = kv ? p.v : p.k;
      val[u] = make_uint4(0, 0, 0, 0);
      if (token < p.ntokens) val[u] = __ldg(src + ((int64_t)token * p.heads + h) * p.vec_per_row + c);
      uint8_t* page = p.data + (int64_t)p.pages[pi] * p.page_bytes;
      dst[u] = reinterpret_cast<uint4*>(page) + ((int64_t)kv * p.heads + h) * per_head + r2;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (dst[u]) *dst[u] = val[u];
  }
}

}  // namespace

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
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
    return fail(WAVE_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  auto encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
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

int launch_append(wave_kv* kv, const wave_entry& ent, const void* K, const void* V,
                  int32_t ntokens, void* stream) {
  if ((int)ent.pages.size() > kMaxEntryPages)
    return fail(WAVE_ERR_CAPACITY, "entry of %d pages exceeds %d", (int)ent.pages.size(),
                kMaxEntryPages);
  static thread_local AppendParams p;  // large: keep off the stack; launch copies it
  p.k = static_cast<const uint4*>(K);
  p.v = static_cast<const uint4*>(V);
  p.data = static_cast<uint8_t*>(kv->cfg.pool) + kv->data_offset;
  p.page_bytes = kv->page_bytes;
  p.ntokens = ntokens;
  p.heads = kv->cfg.heads;
  p.n_pages = (int32_t)ent.pages.size();
  p.vec_per_row = kv->cfg.head_dim / 8;
  std::memcpy(p.pages, ent.pages.data(), ent.pages.size() * sizeof(int32_t));
  int64_t total = 2LL * p.n_pages * WAVE_PAGE_TOKENS * p.heads * p.vec_per_row;
  int64_t blocks = (total + 256 * 4 - 1) / (256 * 4);
  int64_t cap = (int64_t)kv->num_sms * 8;
  if (blocks > cap) blocks = cap;
  kv_append_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
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
