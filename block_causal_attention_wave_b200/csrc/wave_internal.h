// Internal declarations shared by the host (wave_host.cpp) and device (*.cu)
// halves of libwave.so. Not part of the ABI.
#pragma once

#include <cuda.h>  // CUtensorMap (type only; the driver is reached at run time)
#include <cudaTypedefs.h>  // PFN_cuTensorMapEncodeTiled (type only)

#include <cstdint>
#include <map>
#include <set>
#include <utility>
#include <vector>

#include "wave.h"

struct wave_entry {
  std::vector<int32_t> pages;  // page ids in token order
  int32_t ntokens = 0;
};

struct wave_kv {
  wave_kv_config cfg{};
  int64_t page_bytes = 0;   // 2 * H * 128 * d * sizeof(bf16)
  int64_t data_offset = 0;  // byte offset of page 0 inside the pool
  int32_t max_pages = 0;
  std::set<int32_t> free_pages;  // ordered: begin() is the lowest free id
  std::map<std::pair<int32_t, int32_t>, wave_entry> entries;
  bool on_device = false;  // pool != NULL
  int device = -1;
  int num_sms = 0;
  uint64_t wait_ns = 0;     // bound on one device wait; 0 = the default (2 s)
  bool fp8 = false;         // pages hold E4M3 codes with per-(page, head) scales
  int64_t scale_offset = 0; // FP8: byte offset of the scale table in the pool
  alignas(64) CUtensorMap tm_kv;  // rows of d bf16 over every page's K and V
};

namespace wavei {

constexpr int kPageTokens = WAVE_PAGE_TOKENS;
constexpr int64_t kHeaderBytes = 4096;  // device status word lives here

// Record a message for wave_last_error_detail() and return `code`.
int fail(int code, const char* fmt, ...);
void clear_error();

// phi(j, r) of the design-space paper, Table 1 (r >= 1).
int phi(int policy, int j, int r);
bool valid_policy(int policy);

// Ordered entries (chunk, level) of a node's key list: prefix, history by
// ascending chunk, own entry.
void key_entries(const wave_kv* kv, wave_node node, int policy,
                 std::vector<std::pair<int32_t, int32_t>>& out);

// Per active node, its (page, valid) rows; offsets has n + 1 entries.
int build_rows(const wave_kv* kv, const wave_node* active, int n, int policy,
               std::vector<int32_t>& rows, std::vector<int32_t>& offsets);

// Validate one query node against the handle's shape.
int check_query_node(const wave_kv* kv, wave_node node);

// Device halves (defined in .cu files).
int device_init(wave_kv* kv);
// WAVE_ERR_ARG unless the calling thread's current device is the pool's: the
// handle's tensor maps and pool pointer belong to that device.
int check_current_device(const wave_kv* kv);
// The handle's bound on one device wait, in nanoseconds.
uint64_t wait_limit_ns(const wave_kv* kv);
// The driver's tensor-map encoder, looked up once (nullptr if unavailable).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();
// The persistent 128 x 256 tcgen05 GEMM (wave_gemm.cu) in its QKV mode: the
// projection of n nodes of T tokens each (rows i T .. of X) into Q and the
// pages of their entries (already allocated), Q and K turned when rope is
// non-null. Needs head_dim 128 and 3 * heads even (qkv_wide_supported).
bool qkv_wide_supported(const wave_kv* kv);
int qkv_wide_launch(wave_kv* kv, int32_t n, const wave_node* nodes, int32_t T, const void* X,
                    int32_t dim, const void* W, const wave_rope* rope, void* Q, void* stream);
// bf16 bytes of one page (the layout the attention kernel reads).
inline int64_t bf16_page_bytes(const wave_kv* kv) {
  return 2LL * kv->cfg.heads * WAVE_PAGE_TOKENS * kv->cfg.head_dim * 2;
}
// FP8 pools: expand `n` pages (ids in `pages`) into bf16 pages at `staging`
// (slot i = pages[i]), the read-back bf16(code * scale), one launch.
int launch_fp8_expand(wave_kv* kv, int32_t n, const int32_t* pages, void* staging, void* stream);
// One kernel launch copying the K/V of n entries (already allocated) into
// their pages (quantising them for an FP8 pool).
int launch_append(wave_kv* kv, int32_t n, const wave_entry* const* entries,
                  const void* const* K, const void* const* V, void* stream);

}  // namespace wavei
