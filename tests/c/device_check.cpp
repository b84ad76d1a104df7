// White-box check of the device rule of wave.h: every call that launches a
// kernel (append, batched append, fused projection, attention, static-scratch
// attention) refuses to run unless the calling thread's current device is the
// pool's. The handle is created host-only (no pool, so no GPU is needed) and
// then marked, through the library's internal handle struct, as a device
// handle bound to a device id that no machine has. Each call must stop at the
// device check: no page taken, no launch, nothing read through the fake pool
// pointer. With a GPU present the check reports WAVE_ERR_ARG (current device 0
// is not the pool's); without one, cudaGetDevice itself fails (WAVE_ERR_CUDA).
// Usage: device_check <1 if a CUDA device is visible, else 0>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>

#include "wave.h"
#include "wave_internal.h"

static int g_fail = 0;

static void expect(int rc, int want, const char* what) {
  if (rc != want) {
    std::fprintf(stderr, "FAIL %s: rc %d, want %d (%s)\n", what, rc, want,
                 wave_last_error_detail());
    g_fail = 1;
  } else {
    std::printf("ok %s\n", what);
  }
}

int main(int argc, char** argv) {
  const bool gpu = argc > 1 && std::atoi(argv[1]) == 1;
  const int want = gpu ? WAVE_ERR_ARG : WAVE_ERR_CUDA;
  wave_kv_config cfg;
  std::memset(&cfg, 0, sizeof cfg);
  cfg.heads = 2;
  cfg.head_dim = 128;
  cfg.tokens_per_chunk = 256;
  cfg.num_levels = 2;
  cfg.pool = nullptr;
  cfg.pool_bytes = 4096 + 16ull * 2 * 2 * 128 * 128 * 2;
  wave_kv* kv = nullptr;
  if (wave_kv_create(&cfg, &kv) != WAVE_OK) {
    std::fprintf(stderr, "FAIL create: %s\n", wave_last_error_detail());
    return 1;
  }
  int32_t free0 = 0, free1 = 0;
  wave_kv_free_pages(kv, &free0);
  // Reserve one entry while the handle is still host-only, so the attention
  // calls get past their table checks if the device check were missing.
  expect(wave_kv_alloc(kv, 0, 2, 256), WAVE_OK, "host-only alloc of (0, 2)");
  kv->on_device = true;     // pretend: a device handle ...
  kv->device = 1 << 20;     // ... of a device that does not exist
  alignas(16) static uint16_t buf[256 * 2 * 128];
  const void* K = buf;
  const void* V = buf;
  const wave_node e{1, 2};
  const int32_t nt = 256;
  wave_kv_free_pages(kv, &free0);
  expect(wave_kv_append(kv, 1, 2, K, V, 256, nullptr), want, "append refused");
  expect(wave_kv_append_batch(kv, 1, &e, &K, &V, &nt, nullptr), want, "batched append refused");
  expect(wave_qkv_append(kv, 1, 2, buf, 256, 128, buf, buf, nullptr), want, "projection refused");
  const wave_node act{0, 2};
  expect(wave_round_attn(kv, &act, 1, WAVE_POLICY_PROGRESSIVE, buf, buf, nullptr), want,
         "attention refused");
  expect(wave_round_attn_static_scratch(kv, &act, 1, WAVE_POLICY_PROGRESSIVE, buf, buf, nullptr),
         want, "static-scratch attention refused");
  const std::string detail = wave_last_error_detail();  // before another call clears it
  wave_kv_free_pages(kv, &free1);
  expect(free1 == free0 ? WAVE_OK : WAVE_ERR_ARG, WAVE_OK, "no pages taken by refused calls");
  if (gpu && detail.find("device") == std::string::npos) {
    std::fprintf(stderr, "FAIL message names the device: %s\n", detail.c_str());
    g_fail = 1;
  }
  kv->on_device = false;
  wave_kv_destroy(kv);
  return g_fail;
}
