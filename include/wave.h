/*
 * wave.h -- C ABI of the wave-round block-causal attention library (libwave.so).
 *
 * The method: pipelined streaming video diffusion. In one concurrent forward
 * round several chunks sit at staggered denoising levels; each attends to its
 * own tokens plus the K/V of earlier chunks at the levels a context policy
 * phi(j, r) picks (level 0 = clean). Sources, cited by page title and section:
 *   [WF]  "Wave Forcing: towards speed-of-light streaming video generation"
 *         (aiany.app), "Key Findings": one output chunk per concurrent round,
 *         chunk-wise causal attention over earlier cleaner chunks, cache
 *         refresh, early K/V delivery.
 *   [DS]  design-space paper (thelatestinai.com, arXiv 2609.22283 summary),
 *         Table 1 and Figure 1 (policies), Figure 2 (serial B*K vs pipelined
 *         B+K-1 rounds), Appendix Table 4 (7 chunks of 3 latent frames).
 *   [WS]  "Wan-Streamer v0.2: Higher Resolution, Same Latency", Figure 1 and
 *         glossary "block-causal attention", "K/V cache", "pre-sharded".
 *
 * Conventions for every call:
 *   - Returns WAVE_OK (0) or a negative WAVE_ERR_* code; nothing throws across
 *     the ABI. wave_strerror() names a code; wave_last_error_detail() gives a
 *     message for the last failure on the calling thread.
 *   - "stream" is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Device work is enqueued on it and is asynchronous; inputs must stay valid
 *     and unmodified until that work has run.
 *   - Device buffers are caller-owned. The library never calls cudaMalloc; the
 *     K/V pool is one caller-provided device buffer (see wave_kv_config).
 *   - Activations are bf16, token-major and contiguous: [tokens][heads][head_dim].
 *   - Calls that launch kernels (append, projection, attention) must be made
 *     with the pool's device current (the device current at wave_kv_create);
 *     otherwise they return WAVE_ERR_ARG before taking pages or launching.
 *   - No call is thread-safe on the same wave_kv handle.
 */
#ifndef WAVE_H_
#define WAVE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------- */
#define WAVE_OK               0
#define WAVE_ERR_ARG         (-1) /* bad argument, shape or alignment            */
#define WAVE_ERR_MISSING_KV  (-2) /* a (chunk, level) the policy reads is absent */
#define WAVE_ERR_NO_PAGES    (-3) /* the pool has too few free pages             */
#define WAVE_ERR_CUDA        (-4) /* a CUDA runtime/driver call failed           */
#define WAVE_ERR_TIMEOUT     (-5) /* a kernel's bounded wait ran out             */
#define WAVE_ERR_EXISTS      (-6) /* (chunk, level) already holds K/V            */
#define WAVE_ERR_CAPACITY    (-7) /* a round exceeds one launch's table limits   */
#define WAVE_ERR_UNSUPPORTED (-8) /* head_dim or device not supported            */

/* ---- context policies phi(j, r) ([DS] Table 1, Figure 1) ---------------- */
#define WAVE_POLICY_CLEAN       0 /* phi = 0                */
#define WAVE_POLICY_SAME        1 /* phi = j                */
#define WAVE_POLICY_PROGRESSIVE 2 /* phi = max(j - r, 0)    */

#define WAVE_PAGE_TOKENS   128   /* tokens per K/V page                       */
#define WAVE_PREFIX_CHUNK  (-1)  /* chunk id of the always-visible prefix     */
#define WAVE_MAX_NODES     64    /* active nodes per wave_round_attn call     */
#define WAVE_MAX_PAGES_PER_ROUND 7168 /* key pages summed over a call's nodes */
#define WAVE_MAX_APPEND_ENTRIES 64  /* entries per wave_kv_append_batch call  */
#define WAVE_MAX_APPEND_PAGES 7168   /* pages summed over one append call       */

typedef struct wave_kv wave_kv; /* opaque; owned by the library */

/* One (chunk, level) node. Level 0 = clean; an update at level j >= 1 turns the
 * level-j state into level j-1; a level-0 node is a cache refresh ([WF]). */
typedef struct {
  int32_t chunk;
  int32_t level;
} wave_node;

typedef struct {
  int32_t heads;            /* H (query heads = K/V heads)                        */
  int32_t head_dim;         /* d: 64 or 128                                       */
  int32_t tokens_per_chunk; /* T: tokens of one chunk / streaming unit            */
  int32_t num_levels;       /* K: update levels K..1                               */
  int32_t window;           /* W: history chunks visible; 0 = unbounded           */
  int32_t prefix_tokens;    /* conditioning prefix length; 0 = none               */
  void*    pool;            /* caller-owned device buffer, 256-byte aligned, or
                               NULL for a host-only handle (tables, no kernels)   */
  uint64_t pool_bytes;      /* size of pool (for a host-only handle: the size the
                               page count is derived from)                       */
  int32_t kv_format;        /* WAVE_KV_BF16 (0) or WAVE_KV_FP8_E4M3              */
} wave_kv_config;

/* Page formats. BF16: K and V as bf16. FP8_E4M3: K and V as E4M3 codes (1
 * sign, 4 exponent bits with bias 7, 3 mantissa bits; largest finite 448),
 * each (page, head) tile of K and of V with one float32 scale: s = amax / 448
 * over the tile's 128 token rows (1 if amax = 0), code = E4M3(x / s) with
 * round to nearest even and saturation; the attention reads bf16(code * s).
 * This halves the bytes of every cached entry -- the pages leave K/V cache
 * growth open ([WS], limitations), and the same-level policy keeps K levels of
 * history alive ([DS] Table 1). */
#define WAVE_KV_BF16     0
#define WAVE_KV_FP8_E4M3 1

/* Create a paged (chunk, level) K/V cache over cfg->pool ([WF] history cache,
 * [WS] "K/V cache"). The pool holds a 4096-byte header (the device status
 * word at byte 0, the attention kernel's work-queue counter at byte 128, the
 * last attention launch's clock words at bytes 256..271) and
 * then pages of 2*H*128*d values (bf16, or E4M3 codes for WAVE_KV_FP8_E4M3):
 * K as [H][128][d], then V as [H][128][d]. Page p starts at pool +
 * data_offset + p * page_bytes. FP8 pools hold after the last page (at
 * wave_kv_scale_offset) the scales, float32 [max_pages][2 (K, V)][H]. With a
 * non-NULL pool this call clears the header synchronously and needs a CUDA
 * device with sm_100. *out receives the handle; destroy it with
 * wave_kv_destroy. Errors: ARG (bad sizes, misaligned pool, pool too small),
 * UNSUPPORTED (head_dim not 64/128, or a device other than sm_100), CUDA. */
int wave_kv_create(const wave_kv_config* cfg, wave_kv** out);

/* Destroy a handle (the pool stays the caller's). NULL is accepted. */
int wave_kv_destroy(wave_kv* kv);

/* Report the pool layout: bytes per page, byte offset of page 0, page count. */
int wave_kv_pool_layout(const wave_kv* kv, int64_t* page_bytes, int64_t* data_offset,
                        int32_t* max_pages);

/* Byte offset (from the pool's start) of an FP8 pool's scale table,
 * float32 [max_pages][2][H]. Errors: ARG (not an FP8 handle). */
int wave_kv_scale_offset(const wave_kv* kv, int64_t* offset);

/* Reserve pages for entry (chunk, level) holding ntokens tokens without
 * writing them: ceil(ntokens/128) pages, each the lowest free page id, taken
 * in call order. chunk = WAVE_PREFIX_CHUNK (level 0) names the prefix, whose
 * ntokens must equal prefix_tokens; any other chunk needs ntokens =
 * tokens_per_chunk and 0 <= level <= num_levels. Host only, no device work.
 * Errors: ARG, EXISTS, NO_PAGES (nothing is taken then). */
int wave_kv_alloc(wave_kv* kv, int32_t chunk, int32_t level, int32_t ntokens);

/* wave_kv_alloc, then copy K and V (device, bf16 [ntokens][H][d], contiguous,
 * 16-byte aligned, caller-owned) into the new pages with one kernel on stream;
 * the unused tail of the last page is zero-filled. This is the in-round K/V
 * delivery of [WF] and the local-cache write of [WS] "pre-sharded".
 * Errors: as wave_kv_alloc, plus ARG for misaligned K/V, CAPACITY for more
 * than WAVE_MAX_APPEND_PAGES pages, and CUDA; on any error no pages stay
 * taken. */
int wave_kv_append(wave_kv* kv, int32_t chunk, int32_t level, const void* K, const void* V,
                   int32_t ntokens, void* stream);

/* wave_kv_append for n_entries entries in ONE kernel launch (the round's
 * appends of [WF] in-round delivery, batched). Entry i is (entries[i].chunk,
 * entries[i].level) with K[i], V[i] (device, bf16 [ntokens[i]][H][d],
 * contiguous, 16-byte aligned, caller-owned); `entries`, `K`, `V` and
 * `ntokens` are host arrays of n_entries elements. Every entry is checked
 * first; then pages are taken in list order, exactly as n_entries
 * wave_kv_append calls in that order would take them, and the pages receive
 * the same bytes. Limits: n_entries <= WAVE_MAX_APPEND_ENTRIES and total pages
 * <= WAVE_MAX_APPEND_PAGES (else CAPACITY). Errors: ARG (including an entry
 * named twice), EXISTS, NO_PAGES, CAPACITY, CUDA; on any error no pages stay
 * taken. */
int wave_kv_append_batch(wave_kv* kv, int32_t n_entries, const wave_node* entries,
                         const void* const* K, const void* const* V, const int32_t* ntokens,
                         void* stream);

/* A node's QKV projection with its K/V append fused into the epilogue: one
 * kernel computes [Q | K | V] = X W^T (fp32 accumulation, bf16 results) for
 * the entry (chunk, level), writes Q to the caller's buffer, and writes K and
 * V straight into the entry's new pages -- the same pages and bytes that
 * wave_kv_alloc + wave_kv_append of those K and V would give. This is the
 * producing side of the in-round K/V delivery of [WF] ("Key Findings"); the
 * pages give no formula for the projection, so it is the plain linear map of
 * a multi-head attention layer: no bias, no positional or norm term.
 * X: device bf16 [ntokens][dim] (the node's hidden states), W: device bf16
 * [3*H*d][dim] (a linear layer's [out][in] weight; output feature
 * (s*H + h)*d + j is Q (s = 0), K (s = 1) or V (s = 2) of head h, component
 * j), Q: device bf16 [ntokens][H][d], written. All caller-owned, contiguous,
 * 16-byte aligned; dim a multiple of 64. Entry rules as wave_kv_alloc.
 * Errors: as wave_kv_alloc, plus ARG (pointers, alignment, dim), CAPACITY
 * (more than WAVE_MAX_APPEND_PAGES pages) and CUDA; on any error no pages stay
 * taken. A device-side timeout is reported by wave_kv_status. */
int wave_qkv_append(wave_kv* kv, int32_t chunk, int32_t level, const void* X, int32_t ntokens,
                    int32_t dim, const void* W, void* Q, void* stream);

/* Rotary position embedding of a chunk's tokens over three axes of the video
 * latent (frame, row, column): token t of chunk c sits at frame
 * c * frames + t / (rows * cols), row (t / cols) % rows, column t % cols. Of
 * the d/2 rotation pairs of a head (elements 2p, 2p+1) the first
 * d/2 - 2 (d/6) turn with the frame, the next d/6 with the row and the last
 * d/6 with the column (integer division); pair i of a group of n pairs turns
 * by position * base^(-i/n) radians: (a, b) -> (a cos - b sin, a sin + b cos).
 * The pages give no positional scheme; this is the reading of a rotary
 * embedding on the latent grid of the chunks they describe ([DS] Appendix
 * Table 4: 3 latent frames of 832x480 per chunk). */
typedef struct {
  int32_t frames; /* F: latent frames per chunk                        */
  int32_t rows;   /* R: token rows per frame                           */
  int32_t cols;   /* W: token columns per frame; F * R * W = T          */
  float base;     /* frequency base, > 1 (10000 in common use)         */
} wave_rope;

/* The QKV projection of ALL n_nodes nodes of a round in ONE kernel launch,
 * with the rotary embedding of Q and K and the K/V append fused into its
 * epilogue: for node i = nodes[i], [Q | K | V] = X_i W^T (fp32 accumulation),
 * Q and K turned by `rope` (NULL: no rotation), Q rounded to bf16 into the
 * caller's buffer, K and V rounded to bf16 straight into the node's new cache
 * entry (the pages and bytes wave_kv_alloc + wave_kv_append would give,
 * zero page tail). This is the producing side of the in-round K/V delivery of
 * [WF] ("Key Findings") for one transformer block of a round.
 * X: device bf16 [n_nodes * T][dim], node i's hidden states at rows i*T;
 * W: device bf16 [3*H*d][dim] (output feature (s*H + h)*d + j is Q (s = 0), K
 * (s = 1) or V (s = 2) of head h, component j); Q: device bf16
 * [n_nodes * T][H][d], written (node i at rows i*T, the layout
 * wave_round_attn reads). All caller-owned, contiguous, 16-byte aligned; dim a
 * multiple of 64; T = tokens_per_chunk. Needs head_dim 128 and 3*H even
 * (UNSUPPORTED otherwise). Pages are taken in node order, lowest free first.
 * Errors: ARG (pointers, dim, rope grid not covering T), EXISTS, NO_PAGES,
 * CAPACITY (more than WAVE_MAX_APPEND_PAGES pages or WAVE_MAX_NODES nodes),
 * UNSUPPORTED, CUDA; on any error no pages stay taken. A device-side timeout
 * is reported by wave_kv_status. */
int wave_qkv_append_round(wave_kv* kv, const wave_node* nodes, int32_t n_nodes, const void* X,
                          int32_t dim, const void* W, const wave_rope* rope, void* Q,
                          void* stream);

#define WAVE_ACT_NONE      0
#define WAVE_ACT_GELU_TANH 1 /* 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))) */

/* A dense layer of the round's transformer block on the tensor cores:
 * Y = act(A W^T) (+ R), fp32 accumulation, bf16 result -- the out-projection
 * (Y = X + attention W_o^T) and the two MLP products (U = GELU(Y W_1^T),
 * Z = Y + U W_2^T) of one concurrent forward round ([WF] "Key Findings"; the
 * pages give no formula for the block, these are the plain readings).
 * A: device bf16 [M][K]; W: device bf16 [N][K] (a linear layer's [out][in]
 * weight); R: device bf16 [M][N] residual or NULL (added after act); Y:
 * device bf16 [M][N], written (may be R itself). All caller-owned,
 * contiguous, 16-byte aligned. K a multiple of 64, N a multiple of 256,
 * K, N <= 65536. `kv` names the device handle whose status word records a
 * timeout (wave_kv_status) and whose device must be current; the pool itself
 * is not touched. Errors: ARG, CUDA. */
int wave_linear(wave_kv* kv, const void* A, int32_t M, int32_t K, const void* W, int32_t N,
                const void* R, int32_t act, void* Y, void* stream);

/* Return the pages of (chunk, level) to the free set. Host only; the caller
 * must not release an entry that queued device work still reads (all library
 * kernels read the pool in stream order, so releasing after enqueueing the
 * last reader on the same stream is safe when the next writer uses that
 * stream too). Errors: MISSING_KV. */
int wave_kv_release(wave_kv* kv, int32_t chunk, int32_t level);

/* Page ids of entry (chunk, level) in token order (page j holds tokens
 * 128 j .. 128 j + 127; rows past the entry's tokens are zero once written).
 * `cap` = capacity of pages; *n = the entry's page count. Host only.
 * Errors: ARG, MISSING_KV, CAPACITY (cap too small; *n = pages needed). */
int wave_kv_entry_pages(const wave_kv* kv, int32_t chunk, int32_t level, int32_t* pages,
                        int32_t cap, int32_t* n);

/* Number of free pages. */
int wave_kv_free_pages(const wave_kv* kv, int32_t* n);

/* The key list of each active node, as the attention kernel reads it: for node
 * i, rows node_offsets[i] .. node_offsets[i+1]-1 of `rows`, each row a pair
 * (page id, valid tokens) = rows[2*r], rows[2*r+1]. Key order: prefix, then
 * history E(c - r, phi(l, r)) for r = min(c, W)..1 (ascending chunk), then the
 * node's own E(c, l) ([DS] Table 1; [WF] "Key Findings"). `cap` = capacity of
 * rows in pairs; node_offsets holds n_active + 1 ints. Host only.
 * Errors: ARG, MISSING_KV, CAPACITY (cap too small; *n_rows = pairs needed). */
int wave_gather_table(const wave_kv* kv, const wave_node* active, int32_t n_active,
                      int32_t policy, int32_t* rows, int32_t* node_offsets, int32_t cap,
                      int32_t* n_rows);

/* One wave round of block-causal attention for all active nodes in ONE kernel
 * launch: for node i = (c, l) and head h,
 *   O_i[q, h] = softmax_k(Q_i[q, h] . K[k, h] / sqrt(d)) V[k, h]
 * over the tokens of the node's key list (see wave_gather_table); no mask
 * inside a chunk ([WS] "block-causal attention"; [DS] Figure 1).
 * Q and O: device bf16 [n_active * T][H][d], node i's rows at i*T, 16-byte
 * aligned, caller-owned; O is written, Q is read. Every entry the nodes read
 * must have been appended (on this stream or before it). Accumulation is fp32;
 * O is rounded to bf16 once. Limits: n_active <= WAVE_MAX_NODES, total key
 * pages <= WAVE_MAX_PAGES_PER_ROUND (else CAPACITY). A device-side timeout is
 * reported by the next wave_kv_status call. Errors: ARG, MISSING_KV, CAPACITY,
 * CUDA. */
int wave_round_attn(wave_kv* kv, const wave_node* active, int32_t n_active, int32_t policy,
                    const void* Q, void* O, void* stream);

/* wave_round_attn with each node's key list cut into key ranges (split-KV),
 * for rounds with too few (node, head, query-tile pair) work items to fill
 * the GPU -- short query blocks over long K/V, e.g. one Wan-Streamer unit of
 * 984 tokens over 32 units of history and a 512-token prefix ([WS] abstract,
 * glossary "K/V cache", "streaming unit"). Every (node, head, pair) item
 * becomes min(splits, node pages) items over consecutive page ranges; each
 * writes its unnormalised O rows and their (running max, sum) to
 * `workspace`, and a second kernel on `stream` combines them:
 * O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s, M = max_s m_s -- the same
 * softmax(Q K^T / sqrt(d)) V as wave_round_attn, up to rounding.
 * splits: >= 1 ranges per item (at most 32), or 0 = enough to give the GPU
 * about two waves of items (1 when the round already has a wave of them).
 * workspace: device buffer, 256-byte aligned, at least the bytes
 * wave_round_attn_split_workspace reports for the same arguments (none is
 * needed when no node is split); caller-owned, its contents are scratch.
 * For an FP8 pool the workspace also holds, first, the round's distinct pages
 * expanded to bf16 (one launch before the attention reads them), so an FP8
 * pool needs a workspace even with splits = 1; wave_round_attn and
 * wave_round_attn_static_scratch refuse FP8 pools (ARG).
 * Other arguments, layouts, limits and errors as wave_round_attn; ARG also
 * for a missing, misaligned (256 bytes) or too small workspace. */
int wave_round_attn_split(wave_kv* kv, const wave_node* active, int32_t n_active, int32_t policy,
                          int32_t splits, const void* Q, void* O, void* workspace,
                          uint64_t workspace_bytes, void* stream);

/* Workspace bytes wave_round_attn_split needs for these arguments (0 if no
 * node ends up split and the pool is bf16) and, in *splits_used (may be
 * NULL), the ranges per item
 * it will use (splits = 0 resolved). Host only. Errors: as wave_round_attn's
 * table checks (ARG, MISSING_KV, CAPACITY). */
int wave_round_attn_split_workspace(wave_kv* kv, const wave_node* active, int32_t n_active,
                                    int32_t policy, int32_t splits, uint64_t* bytes,
                                    int32_t* splits_used);

/* wave_round_attn without per-call scratch from the caller. The pages have no
 * counterpart to this call; it exists for callers that cannot allocate device
 * memory for the library while they run -- e.g. code inside CUDA stream
 * capture, where cudaMalloc is refused, or a host whose device memory is all
 * owned by another allocator. wave_round_attn keeps its per-call scratch (the
 * 4-byte work-queue counter its persistent kernel draws work from) in the
 * header of the caller's pool; this call keeps it in a 256-byte array that
 * the library holds in device memory on every GPU it is loaded on, until the
 * process exits. Arguments, results, layouts, limits (WAVE_MAX_NODES nodes,
 * WAVE_MAX_PAGES_PER_ROUND key pages, WAVE_ERR_CAPACITY beyond) and error
 * codes are those of wave_round_attn; timeouts are still reported by
 * wave_kv_status. It allocates nothing: no cudaMalloc/cudaFree, no library
 * allocator. The first call on a device, made with that device current (it
 * must be the pool's device), looks up the array's device address once and
 * caches it (per device and context: after a device reset, which gives the
 * device a new context, the next call looks it up again); make that first
 * call, and the first after a reset, before any stream capture. A reset also
 * ends every handle made before it. Each call zeroes
 * the counter on `stream` before its launch. All calls on a device share the
 * one array: calls whose kernels overlap on the GPU (e.g. on two streams
 * without ordering) race on it and give undefined results. */
int wave_round_attn_static_scratch(wave_kv* kv, const wave_node* active, int32_t n_active,
                                   int32_t policy, const void* Q, void* O, void* stream);

/* Synchronise `stream`, then read the clock words of the last attention
 * launch on this pool: *cycles = SM clock cycles and *ns = nanoseconds
 * (%globaltimer) between the start and the end of the launch's first CTA, as
 * int64 at bytes 256 and 264 of the pool header. *cycles / *ns (GHz) is the
 * SM clock the tensor-core kernel actually ran at; clock readings sampled by
 * the driver every few milliseconds miss short clock reductions. Both are 0
 * before the first launch and for a host-only handle. Errors: ARG, CUDA. */
int wave_kv_last_launch_clock(wave_kv* kv, void* stream, int64_t* cycles, int64_t* ns);

/* Bound on how long one wait inside a kernel launched on this handle may take
 * (attention and fused projection; the append kernel does not wait), in
 * nanoseconds; 0 restores the default of 2 s. A wait that runs out makes the
 * kernel stop every role, finish the copies and MMAs it has issued, free its
 * tensor memory and return; the launch's output is then undefined and the
 * next wave_kv_status reports WAVE_ERR_TIMEOUT. This is the failure-detection
 * path: a small bound lets a test make a wait run out without faulting the
 * GPU. Applies to launches made after the call. Host only. Errors: ARG. */
int wave_kv_set_wait_limit(wave_kv* kv, uint64_t ns);

/* Synchronise `stream`, then read and clear the pool's device status word.
 * Returns WAVE_OK, WAVE_ERR_TIMEOUT if a kernel gave up on a bounded wait
 * (its output is then undefined), or WAVE_ERR_CUDA. */
int wave_kv_status(wave_kv* kv, void* stream);

/* Round schedule for B chunks and K levels under `policy` and `window`
 * ([DS] Figure 2; [WF] "Key Findings"). Nodes: updates (c, j), j = K..1, and
 * refreshes (c, 0) where some node reads E(c, 0). Node (c, l) reads E(c, l)
 * and E(c - r, phi(l, r)) for r = 1..min(c, W). Each node runs in the least
 * round with round(c, l) >= round(c, l+1) + 1, round(c, K) >= c, and
 * round >= the round that writes each entry it reads (K/V written in a round
 * is visible in that round). Output: round t holds nodes
 * [round_offsets[t], round_offsets[t+1]) of `nodes`, ascending chunk.
 * Progressive and same-level give B+K-1 rounds, clean gives B*K.
 * Errors: ARG, CAPACITY (caps too small; *n_nodes, *n_rounds = sizes needed). */
int wave_schedule(int32_t B, int32_t K, int32_t policy, int32_t window, wave_node* nodes,
                  int32_t nodes_cap, int32_t* round_offsets, int32_t rounds_cap,
                  int32_t* n_nodes, int32_t* n_rounds);

/* Last round in which any node of the (B, K, policy, window) schedule reads
 * the entry E(c, l) of each given node (its own round at least). A rollout
 * driver releases E(c, l) after that round's attention. Host only.
 * Errors: ARG (bad sizes, or a node that is not in the schedule). */
int wave_schedule_last_read(int32_t B, int32_t K, int32_t policy, int32_t window,
                            const wave_node* nodes, int32_t n, int32_t* last_round);

/* ---- Wave Parallelism: one node per GPU, one-way K/V pushes ----------------
 * [WF] "Key Findings" (full-model replicas, early K/V delivery) and
 * "Wave Forcing Targets Near-Light-Speed Video Streaming Generation"
 * (aipulsen.com): Wave Parallelism with one-way key-value communication. The
 * pages give no placement or protocol; the reading implemented here: node
 * (c, l) runs on rank l mod n_ranks (with K + 1 ranks, one per denoising
 * level); the entry E(c, l) a node produces is pushed, in the node's own
 * round and before that round's attention, from its rank to every other rank
 * that runs a node reading it. Under the progressive policy pushes only go
 * from a cleaner level's rank to a noisier one; under same-level with a rank
 * per level there are none. Each rank keeps its own pool: per round it
 * appends the entries its nodes produce (node order), then takes pages for
 * the entries it receives (ascending (chunk, level)) and receives their page
 * bytes; it releases an entry after wave_wp_rank_last_read's round. */
typedef struct {
  int32_t chunk, level; /* the entry E(chunk, level)                           */
  int32_t src, dst;     /* producer's rank -> a reader's rank (src != dst)      */
} wave_transfer;

/* Pushes of `round` of the (B, K, policy, window) schedule on n_ranks ranks,
 * sorted by (chunk, level, src, dst). `cap` = capacity of out; *n = count.
 * Host only. Errors: ARG, CAPACITY (*n = entries needed). */
int wave_wp_transfers(int32_t B, int32_t K, int32_t policy, int32_t window, int32_t n_ranks,
                      int32_t round, wave_transfer* out, int32_t cap, int32_t* n);

/* For each entry, the last round in which a node that runs on `rank` reads it
 * (the round after which that rank releases it). Host only. Errors: ARG (an
 * entry the rank never holds). */
int wave_wp_rank_last_read(int32_t B, int32_t K, int32_t policy, int32_t window, int32_t n_ranks,
                           int32_t rank, const wave_node* entries, int32_t n,
                           int32_t* last_round);

/* Static name of a status code. */
const char* wave_strerror(int code);

/* Message describing the last failure on the calling thread ("" if none). */
const char* wave_last_error_detail(void);

#ifdef __cplusplus
}
#endif
#endif /* WAVE_H_ */
