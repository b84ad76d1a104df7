// Host half of libwave.so: the round scheduler, the page allocator and the
// key-list tables. No device work happens here.
//
// Sources: design-space paper (arXiv 2609.22283 summary page), Table 1 and
// Figure 1 (context policies), Figure 2 (serial vs pipelined rounds); Wave
// Forcing page, "Key Findings" (cache refresh, in-round K/V delivery, one
// output chunk per round after the pipeline fills).
#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <set>
#include <string>
#include <tuple>

#include "wave_internal.h"

namespace wavei {

static thread_local std::string g_detail;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_detail = buf;
  return code;
}

void clear_error() { g_detail.clear(); }

bool valid_policy(int policy) {
  return policy == WAVE_POLICY_CLEAN || policy == WAVE_POLICY_SAME ||
         policy == WAVE_POLICY_PROGRESSIVE;
}

int phi(int policy, int j, int r) {
  switch (policy) {
    case WAVE_POLICY_CLEAN: return 0;
    case WAVE_POLICY_SAME: return j;
    default: return j > r ? j - r : 0;  // progressive: max(j - r, 0)
  }
}

static int history_span(int c, int window) { return window <= 0 ? c : std::min(c, window); }

void key_entries(const wave_kv* kv, wave_node node, int policy,
                 std::vector<std::pair<int32_t, int32_t>>& out) {
  out.clear();
  if (kv->cfg.prefix_tokens > 0) out.emplace_back(WAVE_PREFIX_CHUNK, 0);
  for (int r = history_span(node.chunk, kv->cfg.window); r >= 1; --r)
    out.emplace_back(node.chunk - r, phi(policy, node.level, r));
  out.emplace_back(node.chunk, node.level);
}

int check_query_node(const wave_kv* kv, wave_node node) {
  if (node.chunk < 0 || node.level < 0 || node.level > kv->cfg.num_levels)
    return fail(WAVE_ERR_ARG, "node (%d, %d) is not a query node (chunk >= 0, 0 <= level <= %d)",
                node.chunk, node.level, kv->cfg.num_levels);
  return WAVE_OK;
}

int build_rows(const wave_kv* kv, const wave_node* active, int n, int policy,
               std::vector<int32_t>& rows, std::vector<int32_t>& offsets) {
  rows.clear();
  offsets.assign(1, 0);
  std::vector<std::pair<int32_t, int32_t>> ents;
  for (int i = 0; i < n; ++i) {
    int rc = check_query_node(kv, active[i]);
    if (rc) return rc;
    key_entries(kv, active[i], policy, ents);
    for (auto& e : ents) {
      auto it = kv->entries.find(e);
      if (it == kv->entries.end())
        return fail(WAVE_ERR_MISSING_KV, "K/V of (%d, %d) read by node (%d, %d) is not cached",
                    e.first, e.second, active[i].chunk, active[i].level);
      const wave_entry& we = it->second;
      for (size_t p = 0; p < we.pages.size(); ++p) {
        int valid = std::min<int>(kPageTokens, we.ntokens - (int)p * kPageTokens);
        rows.push_back(we.pages[p]);
        rows.push_back(valid);
      }
    }
    offsets.push_back((int32_t)(rows.size() / 2));
  }
  return WAVE_OK;
}

}  // namespace wavei

using namespace wavei;

extern "C" {

const char* wave_strerror(int code) {
  switch (code) {
    case WAVE_OK: return "ok";
    case WAVE_ERR_ARG: return "invalid argument";
    case WAVE_ERR_MISSING_KV: return "K/V of a required (chunk, level) is not cached";
    case WAVE_ERR_NO_PAGES: return "K/V pool out of pages";
    case WAVE_ERR_CUDA: return "CUDA error";
    case WAVE_ERR_TIMEOUT: return "device wait timed out";
    case WAVE_ERR_EXISTS: return "(chunk, level) already cached";
    case WAVE_ERR_CAPACITY: return "request exceeds a table capacity";
    case WAVE_ERR_UNSUPPORTED: return "unsupported shape or device";
    default: return "unknown status";
  }
}

const char* wave_last_error_detail(void) { return g_detail.c_str(); }

int wave_kv_create(const wave_kv_config* cfg, wave_kv** out) {
  clear_error();
  if (!cfg || !out) return fail(WAVE_ERR_ARG, "cfg and out must be non-NULL");
  *out = nullptr;
  if (cfg->heads < 1 || cfg->tokens_per_chunk < 1 || cfg->num_levels < 1 || cfg->window < 0 ||
      cfg->prefix_tokens < 0)
    return fail(WAVE_ERR_ARG, "heads, tokens_per_chunk, num_levels must be >= 1; window, "
                              "prefix_tokens >= 0");
  if (cfg->head_dim != 64 && cfg->head_dim != 128)
    return fail(WAVE_ERR_UNSUPPORTED, "head_dim %d: only 64 and 128 are built", cfg->head_dim);
  if (cfg->pool && (reinterpret_cast<uintptr_t>(cfg->pool) & 255))
    return fail(WAVE_ERR_ARG, "pool must be 256-byte aligned");
  if (cfg->kv_format != WAVE_KV_BF16 && cfg->kv_format != WAVE_KV_FP8_E4M3)
    return fail(WAVE_ERR_ARG, "unknown kv_format %d", cfg->kv_format);
  wave_kv* kv = new wave_kv();
  kv->cfg = *cfg;
  kv->fp8 = cfg->kv_format == WAVE_KV_FP8_E4M3;
  kv->page_bytes = 2LL * cfg->heads * kPageTokens * cfg->head_dim * (kv->fp8 ? 1 : 2);
  kv->data_offset = kHeaderBytes;
  // An FP8 page also needs its 2 H float32 scales (table after the pages,
  // 256-byte aligned).
  const int64_t per_page = kv->page_bytes + (kv->fp8 ? 2LL * cfg->heads * 4 : 0);
  int64_t avail = (int64_t)cfg->pool_bytes - kv->data_offset - (kv->fp8 ? 256 : 0);
  int64_t pages = avail > 0 ? avail / per_page : 0;
  // Row coordinates of the pool's tensor map are int32: pages * 2H * 128 < 2^31.
  int64_t max_by_coord = ((int64_t)1 << 31) / (2LL * cfg->heads * kPageTokens) - 1;
  pages = std::min<int64_t>(pages, std::min<int64_t>(max_by_coord, (1 << 25) - 1));
  if (pages < 1) {
    delete kv;
    return fail(WAVE_ERR_ARG, "pool of %llu bytes holds no page of %lld bytes after the header",
                (unsigned long long)cfg->pool_bytes, (long long)(2LL * cfg->heads * kPageTokens *
                                                                  cfg->head_dim * 2));
  }
  kv->max_pages = (int32_t)pages;
  if (kv->fp8) kv->scale_offset = (kv->data_offset + pages * kv->page_bytes + 255) / 256 * 256;
  for (int32_t p = 0; p < kv->max_pages; ++p) kv->free_pages.insert(kv->free_pages.end(), p);
  kv->on_device = cfg->pool != nullptr;
  if (kv->on_device) {
    int rc = device_init(kv);
    if (rc) {
      delete kv;
      return rc;
    }
  }
  *out = kv;
  return WAVE_OK;
}

int wave_kv_destroy(wave_kv* kv) {
  delete kv;
  return WAVE_OK;
}

int wave_kv_pool_layout(const wave_kv* kv, int64_t* page_bytes, int64_t* data_offset,
                        int32_t* max_pages) {
  clear_error();
  if (!kv) return fail(WAVE_ERR_ARG, "NULL handle");
  if (page_bytes) *page_bytes = kv->page_bytes;
  if (data_offset) *data_offset = kv->data_offset;
  if (max_pages) *max_pages = kv->max_pages;
  return WAVE_OK;
}

namespace wavei {
// Shape and existence checks of wave_kv_alloc, without taking pages.
static int check_new_entry(const wave_kv* kv, int32_t chunk, int32_t level, int32_t ntokens) {
  if (chunk == WAVE_PREFIX_CHUNK) {
    if (level != 0 || ntokens != kv->cfg.prefix_tokens || ntokens < 1)
      return fail(WAVE_ERR_ARG, "prefix must be level 0 with prefix_tokens (%d) tokens",
                  kv->cfg.prefix_tokens);
  } else {
    if (chunk < 0 || level < 0 || level > kv->cfg.num_levels)
      return fail(WAVE_ERR_ARG, "bad entry (%d, %d)", chunk, level);
    if (ntokens != kv->cfg.tokens_per_chunk)
      return fail(WAVE_ERR_ARG, "entry needs tokens_per_chunk (%d) tokens, got %d",
                  kv->cfg.tokens_per_chunk, ntokens);
  }
  if (kv->entries.count(std::make_pair(chunk, level)))
    return fail(WAVE_ERR_EXISTS, "(%d, %d) already cached", chunk, level);
  return WAVE_OK;
}
}  // namespace wavei

int wave_kv_alloc(wave_kv* kv, int32_t chunk, int32_t level, int32_t ntokens) {
  clear_error();
  if (!kv) return fail(WAVE_ERR_ARG, "NULL handle");
  if (int rc = check_new_entry(kv, chunk, level, ntokens)) return rc;
  auto key = std::make_pair(chunk, level);
  int32_t need = (ntokens + kPageTokens - 1) / kPageTokens;
  if ((int64_t)need > (int64_t)kv->free_pages.size())
    return fail(WAVE_ERR_NO_PAGES, "need %d pages, %zu free", need, kv->free_pages.size());
  wave_entry e;
  e.ntokens = ntokens;
  e.pages.reserve(need);
  for (int32_t i = 0; i < need; ++i) {
    auto it = kv->free_pages.begin();
    e.pages.push_back(*it);
    kv->free_pages.erase(it);
  }
  kv->entries.emplace(key, std::move(e));
  return WAVE_OK;
}

int wave_kv_release(wave_kv* kv, int32_t chunk, int32_t level) {
  clear_error();
  if (!kv) return fail(WAVE_ERR_ARG, "NULL handle");
  auto it = kv->entries.find(std::make_pair(chunk, level));
  if (it == kv->entries.end())
    return fail(WAVE_ERR_MISSING_KV, "(%d, %d) is not cached", chunk, level);
  for (int32_t p : it->second.pages) kv->free_pages.insert(p);
  kv->entries.erase(it);
  return WAVE_OK;
}

int wave_kv_scale_offset(const wave_kv* kv, int64_t* offset) {
  clear_error();
  if (!kv || !offset) return fail(WAVE_ERR_ARG, "NULL argument");
  if (!kv->fp8) return fail(WAVE_ERR_ARG, "not an FP8 pool");
  *offset = kv->scale_offset;
  return WAVE_OK;
}

int wave_kv_entry_pages(const wave_kv* kv, int32_t chunk, int32_t level, int32_t* pages,
                        int32_t cap, int32_t* n) {
  clear_error();
  if (!kv || !n) return fail(WAVE_ERR_ARG, "NULL argument");
  auto it = kv->entries.find(std::make_pair(chunk, level));
  if (it == kv->entries.end())
    return fail(WAVE_ERR_MISSING_KV, "(%d, %d) holds no K/V", chunk, level);
  *n = (int32_t)it->second.pages.size();
  if (*n > cap || !pages) return fail(WAVE_ERR_CAPACITY, "entry has %d pages, capacity %d", *n, cap);
  std::memcpy(pages, it->second.pages.data(), *n * sizeof(int32_t));
  return WAVE_OK;
}

int wave_kv_set_wait_limit(wave_kv* kv, uint64_t ns) {
  clear_error();
  if (!kv) return fail(WAVE_ERR_ARG, "NULL handle");
  kv->wait_ns = ns;
  return WAVE_OK;
}

int wave_kv_free_pages(const wave_kv* kv, int32_t* n) {
  clear_error();
  if (!kv || !n) return fail(WAVE_ERR_ARG, "NULL argument");
  *n = (int32_t)kv->free_pages.size();
  return WAVE_OK;
}

int wave_kv_append(wave_kv* kv, int32_t chunk, int32_t level, const void* K, const void* V,
                   int32_t ntokens, void* stream) {
  const wave_node e{chunk, level};
  return wave_kv_append_batch(kv, 1, &e, &K, &V, &ntokens, stream);
}

int wave_kv_append_batch(wave_kv* kv, int32_t n_entries, const wave_node* entries,
                         const void* const* K, const void* const* V, const int32_t* ntokens,
                         void* stream) {
  clear_error();
  if (!kv) return fail(WAVE_ERR_ARG, "NULL handle");
  if (!kv->on_device) return fail(WAVE_ERR_ARG, "host-only handle (pool == NULL) cannot append");
  if (int rc = check_current_device(kv)) return rc;
  if (n_entries < 0 || (n_entries > 0 && (!entries || !K || !V || !ntokens)))
    return fail(WAVE_ERR_ARG, "bad arguments");
  if (n_entries > WAVE_MAX_APPEND_ENTRIES)
    return fail(WAVE_ERR_CAPACITY, "%d entries exceed %d per append call", n_entries,
                WAVE_MAX_APPEND_ENTRIES);
  // Check everything before taking any page.
  int64_t need = 0;
  std::set<std::pair<int32_t, int32_t>> seen;
  for (int32_t i = 0; i < n_entries; ++i) {
    if (!K[i] || !V[i] || ((reinterpret_cast<uintptr_t>(K[i]) | reinterpret_cast<uintptr_t>(V[i])) & 15))
      return fail(WAVE_ERR_ARG, "K and V of entry %d must be non-NULL and 16-byte aligned", i);
    if (int rc = check_new_entry(kv, entries[i].chunk, entries[i].level, ntokens[i])) return rc;
    if (!seen.insert(std::make_pair(entries[i].chunk, entries[i].level)).second)
      return fail(WAVE_ERR_ARG, "(%d, %d) named twice in one append call", entries[i].chunk,
                  entries[i].level);
    need += (ntokens[i] + kPageTokens - 1) / kPageTokens;
  }
  if (need > WAVE_MAX_APPEND_PAGES)
    return fail(WAVE_ERR_CAPACITY, "%lld pages exceed %d per append call", (long long)need,
                WAVE_MAX_APPEND_PAGES);
  if (need > (int64_t)kv->free_pages.size())
    return fail(WAVE_ERR_NO_PAGES, "need %lld pages, %zu free", (long long)need,
                kv->free_pages.size());
  std::vector<const wave_entry*> ents;
  ents.reserve(n_entries);
  for (int32_t i = 0; i < n_entries; ++i) {
    int rc = wave_kv_alloc(kv, entries[i].chunk, entries[i].level, ntokens[i]);
    if (rc) {  // cannot happen after the checks above; undo all the same
      std::string keep = g_detail;
      for (int32_t j = 0; j < i; ++j) wave_kv_release(kv, entries[j].chunk, entries[j].level);
      g_detail = keep;
      return rc;
    }
    ents.push_back(&kv->entries.at(std::make_pair(entries[i].chunk, entries[i].level)));
  }
  if (n_entries == 0) return WAVE_OK;
  int rc = launch_append(kv, n_entries, ents.data(), K, V, stream);
  if (rc) {
    std::string keep = g_detail;
    for (int32_t i = 0; i < n_entries; ++i)
      wave_kv_release(kv, entries[i].chunk, entries[i].level);
    g_detail = keep;
  }
  return rc;
}

int wave_gather_table(const wave_kv* kv, const wave_node* active, int32_t n_active,
                      int32_t policy, int32_t* rows, int32_t* node_offsets, int32_t cap,
                      int32_t* n_rows) {
  clear_error();
  if (!kv || (n_active > 0 && !active) || n_active < 0 || !n_rows)
    return fail(WAVE_ERR_ARG, "bad arguments");
  if (!valid_policy(policy)) return fail(WAVE_ERR_ARG, "unknown policy %d", policy);
  std::vector<int32_t> r, off;
  int rc = build_rows(kv, active, n_active, policy, r, off);
  if (rc) return rc;
  int32_t n = (int32_t)(r.size() / 2);
  *n_rows = n;
  if (n > cap || !rows || !node_offsets)
    return fail(WAVE_ERR_CAPACITY, "table needs %d rows, capacity %d", n, cap);
  std::memcpy(rows, r.data(), r.size() * sizeof(int32_t));
  std::memcpy(node_offsets, off.data(), off.size() * sizeof(int32_t));
  return WAVE_OK;
}

}  // extern "C"

namespace wavei {

// As-soon-as-possible round of every node; rnd[c * (K + 1) + l] = -1 if the
// node does not exist (refresh nodes nobody reads).
static int compute_rounds(int32_t B, int32_t K, int32_t policy, int32_t window,
                          std::vector<int32_t>& rnd, int32_t* n_nodes, int32_t* n_rounds) {
  if (B < 1 || K < 1 || window < 0)
    return fail(WAVE_ERR_ARG, "need B >= 1, K >= 1, window >= 0");
  if ((int64_t)B * (K + 1) > (1 << 24)) return fail(WAVE_ERR_ARG, "B * (K + 1) too large");
  if (!valid_policy(policy)) return fail(WAVE_ERR_ARG, "unknown policy %d", policy);
  auto span = [&](int c) { return window <= 0 ? c : std::min(c, window); };
  // Which chunks need a refresh node (c, 0): any node reading E(c, 0). A refresh
  // itself reads level-0 history (phi(0, r) = 0 for every policy), so sweep
  // chunks from last to first, marking what updates and needed refreshes read.
  std::vector<char> refresh(B, 0);
  for (int c = B - 1; c >= 0; --c) {
    for (int l = (refresh[c] ? 0 : 1); l <= K; ++l)
      for (int r = 1; r <= span(c); ++r)
        if (phi(policy, l, r) == 0) refresh[c - r] = 1;
  }
  // Chunk by chunk, level K down to 0: the least round meeting the state
  // chain, the admission rule and every read.
  rnd.assign((size_t)B * (K + 1), -1);
  auto at = [&](int c, int l) -> int32_t& { return rnd[(size_t)c * (K + 1) + l]; };
  int32_t last = 0, count = 0;
  for (int c = 0; c < B; ++c) {
    for (int l = K; l >= 0; --l) {
      if (l == 0 && !refresh[c]) break;
      int32_t t = (l == K) ? c : at(c, l + 1) + 1;
      for (int r = 1; r <= span(c); ++r) t = std::max(t, at(c - r, phi(policy, l, r)));
      at(c, l) = t;
      last = std::max(last, t);
      ++count;
    }
  }
  *n_nodes = count;
  *n_rounds = last + 1;
  return WAVE_OK;
}

}  // namespace wavei

extern "C" {

int wave_schedule(int32_t B, int32_t K, int32_t policy, int32_t window, wave_node* nodes,
                  int32_t nodes_cap, int32_t* round_offsets, int32_t rounds_cap,
                  int32_t* n_nodes, int32_t* n_rounds) {
  clear_error();
  if (!n_nodes || !n_rounds) return fail(WAVE_ERR_ARG, "NULL counts");
  std::vector<int32_t> rnd;
  int rc = compute_rounds(B, K, policy, window, rnd, n_nodes, n_rounds);
  if (rc) return rc;
  const int32_t count = *n_nodes, nr = *n_rounds;
  if (count > nodes_cap || nr + 1 > rounds_cap || !nodes || !round_offsets)
    return fail(WAVE_ERR_CAPACITY, "schedule needs %d nodes and %d round offsets", count, nr + 1);
  // Counting sort by round; chunks ascending inside a round.
  std::vector<int32_t> per(nr + 1, 0);
  for (int32_t v : rnd)
    if (v >= 0) per[v + 1]++;
  for (int t = 0; t < nr; ++t) per[t + 1] += per[t];
  std::memcpy(round_offsets, per.data(), (nr + 1) * sizeof(int32_t));
  for (int c = 0; c < B; ++c)
    for (int l = K; l >= 0; --l) {
      int32_t v = rnd[(size_t)c * (K + 1) + l];
      if (v >= 0) nodes[per[v]++] = wave_node{c, l};
    }
  return WAVE_OK;
}

int wave_schedule_last_read(int32_t B, int32_t K, int32_t policy, int32_t window,
                            const wave_node* nodes, int32_t n, int32_t* last_round) {
  clear_error();
  if (n < 0 || (n > 0 && (!nodes || !last_round))) return fail(WAVE_ERR_ARG, "bad arguments");
  std::vector<int32_t> rnd;
  int32_t nn = 0, nr = 0;
  int rc = compute_rounds(B, K, policy, window, rnd, &nn, &nr);
  if (rc) return rc;
  std::vector<int32_t> last(rnd);
  for (int c = 0; c < B; ++c)
    for (int l = 0; l <= K; ++l) {
      int32_t t = rnd[(size_t)c * (K + 1) + l];
      if (t < 0) continue;
      int span = window <= 0 ? c : std::min<int>(c, window);
      for (int r = 1; r <= span; ++r) {
        int32_t& e = last[(size_t)(c - r) * (K + 1) + phi(policy, l, r)];
        e = std::max(e, t);
      }
    }
  for (int32_t i = 0; i < n; ++i) {
    const wave_node& nd = nodes[i];
    if (nd.chunk < 0 || nd.chunk >= B || nd.level < 0 || nd.level > K ||
        rnd[(size_t)nd.chunk * (K + 1) + nd.level] < 0)
      return fail(WAVE_ERR_ARG, "(%d, %d) is not a node of this schedule", nd.chunk, nd.level);
    last_round[i] = last[(size_t)nd.chunk * (K + 1) + nd.level];
  }
  return WAVE_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Wave Parallelism (Wave Forcing page, "Key Findings"; "Wave Forcing Targets
// Near-Light-Speed Video Streaming Generation": one-way K/V communication
// between full-model replicas): node (c, l) runs on rank l mod N; the entry a
// node produces is pushed in its own round to every other rank that runs a
// node reading it.

extern "C" {

int wave_wp_transfers(int32_t B, int32_t K, int32_t policy, int32_t window, int32_t n_ranks,
                      int32_t round, wave_transfer* out, int32_t cap, int32_t* n) {
  using namespace wavei;
  clear_error();
  if (!n || n_ranks < 1) return fail(WAVE_ERR_ARG, "need n_ranks >= 1 and a count pointer");
  std::vector<int32_t> rnd;
  int32_t nn = 0, nr = 0;
  int rc = compute_rounds(B, K, policy, window, rnd, &nn, &nr);
  if (rc) return rc;
  if (round < 0 || round >= nr) return fail(WAVE_ERR_ARG, "round %d outside 0..%d", round, nr - 1);
  // Ranks reading each entry: the producer's own, plus those of its readers.
  std::vector<std::set<int32_t>> dst((size_t)B * (K + 1));
  for (int c = 0; c < B; ++c)
    for (int l = 0; l <= K; ++l) {
      if (rnd[(size_t)c * (K + 1) + l] < 0) continue;
      const int span = window <= 0 ? c : std::min<int>(c, window);
      for (int r = 1; r <= span; ++r)
        dst[(size_t)(c - r) * (K + 1) + phi(policy, l, r)].insert(l % n_ranks);
    }
  std::vector<wave_transfer> t;
  for (int c = 0; c < B; ++c)
    for (int l = 0; l <= K; ++l) {
      if (rnd[(size_t)c * (K + 1) + l] != round) continue;
      const int32_t src = l % n_ranks;
      for (int32_t d : dst[(size_t)c * (K + 1) + l])
        if (d != src) t.push_back(wave_transfer{c, l, src, d});
    }
  // Sorted by (chunk, level, src, dst): the order every rank walks them in.
  std::sort(t.begin(), t.end(), [](const wave_transfer& a, const wave_transfer& b) {
    return std::make_tuple(a.chunk, a.level, a.src, a.dst) <
           std::make_tuple(b.chunk, b.level, b.src, b.dst);
  });
  *n = (int32_t)t.size();
  if (*n > cap || (*n > 0 && !out))
    return fail(WAVE_ERR_CAPACITY, "round %d has %d transfers, capacity %d", round, *n, cap);
  if (*n > 0) std::memcpy(out, t.data(), t.size() * sizeof(wave_transfer));
  return WAVE_OK;
}

int wave_wp_rank_last_read(int32_t B, int32_t K, int32_t policy, int32_t window, int32_t n_ranks,
                           int32_t rank, const wave_node* entries, int32_t n,
                           int32_t* last_round) {
  using namespace wavei;
  clear_error();
  if (n_ranks < 1 || rank < 0 || rank >= n_ranks || n < 0 || (n > 0 && (!entries || !last_round)))
    return fail(WAVE_ERR_ARG, "bad arguments");
  std::vector<int32_t> rnd;
  int32_t nn = 0, nr = 0;
  int rc = compute_rounds(B, K, policy, window, rnd, &nn, &nr);
  if (rc) return rc;
  std::vector<int32_t> last((size_t)B * (K + 1), -1);
  for (int c = 0; c < B; ++c)
    for (int l = 0; l <= K; ++l) {
      const int32_t t = rnd[(size_t)c * (K + 1) + l];
      if (t < 0 || l % n_ranks != rank) continue;
      int32_t& own = last[(size_t)c * (K + 1) + l];
      own = std::max(own, t);
      const int span = window <= 0 ? c : std::min<int>(c, window);
      for (int r = 1; r <= span; ++r) {
        int32_t& e = last[(size_t)(c - r) * (K + 1) + phi(policy, l, r)];
        e = std::max(e, t);
      }
    }
  for (int32_t i = 0; i < n; ++i) {
    const wave_node& e = entries[i];
    if (e.chunk < 0 || e.chunk >= B || e.level < 0 || e.level > K ||
        last[(size_t)e.chunk * (K + 1) + e.level] < 0)
      return fail(WAVE_ERR_ARG, "rank %d holds no entry (%d, %d)", rank, e.chunk, e.level);
    last_round[i] = last[(size_t)e.chunk * (K + 1) + e.level];
  }
  return WAVE_OK;
}

}  // extern "C"
