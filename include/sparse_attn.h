/*
 * sparse_attn.h -- C ABI of libsparse_attn.so: query-aware block-sparse GQA
 * decode attention and the uncertainty router, hand-written CUDA for sm_100a.
 *
 * Sources (web pages, cited by title and section):
 *  [OFFLINE]  "Sparse Attention for Web Agents -- Offline Replay Records"
 *             (dataset card), section "The comparison": every method cuts the
 *             KV cache into chunks, scores each chunk against the current
 *             query, keeps the best ones and attends only to those; fixed
 *             16-token pages (Quest, BlockSparse) or 16-256-token
 *             structure-aligned chunks (TSA); envelope (per-dimension min/max
 *             upper bound) or centroid (mean key) scoring; the budget is
 *             page_size x top_k attended tokens.
 *  [WEBARENA] "WebArena 0-99 Sparse-Attention Method Comparison" (dataset
 *             card), section "Method configurations at a glance": kept blocks
 *             = max(topk_val + bos + eos, int(cached_block_len * topk_ratio))
 *             with forced first (bos) and last (eos) blocks.
 *  [ROUTER]   "Technische Samenvatting: Onzekerheidsgestuurde Selectie voor
 *             Blok-schaarse Aandacht", section "Methodologie", steps 1-5:
 *             per-tile block scores (max over the tile's rows), the margin
 *             sigma = (s_(k-1) - s_(k)) / (s_(0) - s_(k)), its mean over
 *             heads, a per-layer quantile trigger, and expansion to top-rho*k
 *             with sentinel padding so every tile's list has the same shape.
 *
 * Conventions shared by every call
 *  - All data pointers are DEVICE pointers (global memory of the current
 *    device) unless stated otherwise; descriptors and budgets are HOST structs
 *    read during the call only.  The caller owns all memory: the library never
 *    allocates, frees or synchronises (sparse_attn_get_device_status is the one
 *    call that waits on its stream).
 *  - Every compute call validates its arguments on the host first.  A bad
 *    argument returns SA_ERR_INVALID (or SA_ERR_UNSUPPORTED for a legal but
 *    unimplemented shape) and nothing is launched.  SA_OK means "enqueued on
 *    `stream`"; a failed launch returns SA_ERR_CUDA.  `stream` is a
 *    cudaStream_t (NULL = the legacy default stream).
 *  - Conditions found on the device (a page index out of range, a selection
 *    that overflows max_sel) are recorded in a status word inside the
 *    workspace `ws` and read with sparse_attn_get_device_status.  The offending
 *    entry is skipped; no kernel traps.
 *  - Tensors: q, K, V are bf16 with head_dim = 128 (the only supported value).
 *    K and V of one layer are [batch][n_kv_heads][cap_tokens][128], so a
 *    16-token page of one KV head is one contiguous 4 KiB block.  Several
 *    independent layers may be processed in one call by stacking them along
 *    the batch axis.
 *  - Metadata (`meta`) holds 512 bytes per (batch, KV head, page):
 *      SA_SCORE_ENVELOPE: bf16 kmin[128] followed by bf16 kmax[128];
 *      SA_SCORE_CENTROID: fp32 kmean[128].
 *    Layout [batch][n_kv_heads][max_pages][512 B].  One buffer serves one rule.
 *  - Grouped-query attention: query head h belongs to KV head h / G with
 *    G = n_q_heads / n_kv_heads, 1 <= G <= 8.  One page set is chosen per
 *    (sequence, KV head) and shared by its G query heads; the group score of a
 *    page is the maximum of its G per-head scores.
 *  - Ties: pages are ordered by group score descending, lower page index first
 *    on equal scores (-0.0 equals +0.0).  NaN or infinite inputs are undefined.
 */
#ifndef SPARSE_ATTN_H
#define SPARSE_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SA_OK = 0,
  SA_ERR_INVALID = 1,       /* bad argument (null/misaligned pointer, out-of-range size) */
  SA_ERR_UNSUPPORTED = 2,   /* legal but not implemented (head_dim != 128, G > 8, ...) */
  SA_ERR_WORKSPACE = 3,     /* ws is null, misaligned or smaller than required */
  SA_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed */
  SA_ERR_TIMEOUT = 5,       /* a bounded device-side wait gave up (re-init the workspace) */
  SA_ERR_DEVICE_CHECK = 6   /* a device-side range check failed (entry skipped) */
} sa_status;

typedef enum {
  SA_SCORE_ENVELOPE = 0,    /* sum_d max(q_d*kmin_d, q_d*kmax_d)  [OFFLINE] "The comparison" */
  SA_SCORE_CENTROID = 1     /* q . mean(K_page)                  [OFFLINE] "The comparison" */
} sa_score_rule;

typedef enum {
  SA_BUDGET_TOPK = 0,       /* keep min(top_k, P) pages                       [OFFLINE] */
  SA_BUDGET_RATIO = 1,      /* keep min(P, max(topk_val+bos+eos, floor(P*ratio))) incl. forced [WEBARENA] */
  SA_BUDGET_TOKENS = 2      /* longest rank-order prefix of chunks with <= token_budget tokens [OFFLINE] */
} sa_budget_kind;

/* View of one KV cache (one or more stacked layers). */
typedef struct {
  int32_t batch;            /* B >= 1: sequences (x stacked layers) */
  int32_t n_kv_heads;       /* Hkv >= 1 */
  int32_t head_dim;         /* must be 128 */
  int32_t page_size;        /* fixed pages: multiple of 16 in [16, 256]; 0 = variable chunks */
  int64_t cap_tokens;       /* token capacity per (b, kv head) */
  const void* k;            /* bf16 [B][Hkv][cap_tokens][128], 16-byte aligned */
  const void* v;            /* bf16 [B][Hkv][cap_tokens][128], 16-byte aligned */
  const int32_t* seq_len;   /* [B] tokens N_b in the cache, 1 <= N_b <= cap_tokens (includes the current token) */
  const int32_t* chunk_off; /* variable chunks only: [B][max_pages + 1] CSR token offsets, chunk c = [off[c], min(off[c+1], N_b)) */
  const int32_t* n_chunks;  /* variable chunks only: [B] chunk count C_b <= max_pages, off[C_b] = N_b */
  int32_t max_pages;        /* page/chunk capacity of the metadata axis; P_b = ceil(N_b / page_size) or C_b */
} sa_kv_desc;

/* Budget of one selection ([OFFLINE] "The comparison"; [WEBARENA]). */
typedef struct {
  sa_budget_kind kind;
  int32_t top_k;            /* TOPK: pages to keep, >= 1 */
  double topk_ratio;        /* RATIO: 0 < ratio <= 1, read as floor(P * ratio) */
  int32_t topk_val;         /* RATIO: floor term topk_val + bos + eos (1 on the WebArena card) */
  int32_t bos;              /* RATIO: first `bos` pages always kept */
  int32_t eos;              /* RATIO: last `eos` pages always kept (the newest token's page) */
  int32_t token_budget;     /* TOKENS: attended-token budget, >= 0 */
} sa_budget;

/* Bytes of workspace that every call below needs for this cache view, query
 * head count, query-row count (decode: B; router: rows) and selection width.
 * Returns 0 on invalid arguments.  The workspace must be 256-byte aligned and
 * zeroed once after allocation by sparse_attn_workspace_init; calls leave its
 * counters zeroed again, so one workspace serves any number of calls issued
 * in order on one stream (calls that may overlap need separate workspaces). */
size_t sparse_attn_workspace_size(const sa_kv_desc* kv, int32_t n_q_heads,
                                  int32_t n_q_rows, int32_t max_sel);

/* Zero the workspace (counters and status word).  Async on `stream`. */
sa_status sparse_attn_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* (a) Page metadata ([OFFLINE] "The comparison", scoring column).
 * For every (b, kv head), recompute the metadata of every page/chunk that
 * overlaps the token range [t0_b, N_b):
 *   first_token >= 0: t0_b = first_token            (0 = full build);
 *   first_token <  0: t0_b = max(0, N_b + first_token)  (-1 = the page of the
 *                     token just appended: the per-step incremental update).
 * Envelope: kmin/kmax per dimension, exact bf16.  Centroid: the mean of the
 * page's keys, accumulated in fp64 and stored as fp32.  Pages outside the
 * range are not touched.  meta: [B][Hkv][max_pages] x 512 B, 16-byte aligned. */
sa_status sparse_attn_build_meta(const sa_kv_desc* kv, sa_score_rule rule,
                                 int32_t first_token, void* meta, void* stream);

/* (b) Score + budgeted top-k ([OFFLINE] "The comparison"; [WEBARENA]).
 * q: bf16 [B][n_q_heads][128], the current query token of each sequence.
 * For each (b, kv head): group score of every page (max over the G query
 * heads), then the pages kept by `budget` under the order (score desc, index
 * asc).  Output: sel_idx[b][g][0 .. sel_count[b][g]) = the kept page indices
 * in ASCENDING page order (the set is what the budget defines; ascending
 * order is what the decode streams); entries past the count are untouched.
 * scores_out (nullable): [B][Hkv][max_pages] fp32 group score of every page.
 * max_sel bounds the kept count: TOPK needs top_k <= max_sel; RATIO needs
 * min(max_pages, max(topk_val+bos+eos, floor(max_pages*ratio))) <= max_sel;
 * TOKENS keeps at most max_sel chunks (overflow sets SA_ERR_DEVICE_CHECK). */
sa_status sparse_attn_select(const sa_kv_desc* kv, const void* meta, sa_score_rule rule,
                             const void* q, int32_t n_q_heads, const sa_budget* budget,
                             int32_t max_sel, int32_t* sel_idx, int32_t* sel_count,
                             float* scores_out, void* ws, size_t ws_bytes, void* stream);

/* (c) Sparse paged attention over the kept pages ([OFFLINE] "The comparison":
 * attend only to the kept chunks; exact softmax over their tokens).
 *  tile_rows == 1 (decode): q bf16 [B][n_q_heads][128]; n_q_rows == B; query
 *    head h of sequence b attends to every token of the pages idx[b][h/G][0 ..
 *    count[b][h/G]) (all tokens of the cache precede the current one).
 *  tile_rows > 1 (router tiles, [ROUTER] step 5): B == 1; q bf16
 *    [n_q_rows][n_q_heads][128] at positions q_pos0 + r; idx [T][Hkv][max_sel]
 *    with T = ceil(n_q_rows / tile_rows), -1 entries skipped; row r attends
 *    causally (token position <= q_pos0 + r) to the blocks of its tile.
 *    Blocks must be 64 tokens (page_size = 64); this path uses only the
 *    status word of ws (ws may be null: device checks are then not reported).
 * z = scale * q.k, softmax with fp32 accumulation.  out: fp32 [rows][Hq][128];
 * lse (nullable): fp32 [rows][Hq], natural-log sum of exp(z).  A row with no
 * visible token gets out = 0 and lse = -inf.  idx entries outside [0, P_b)
 * are skipped and flag SA_ERR_DEVICE_CHECK. */
sa_status sparse_attn_decode(const sa_kv_desc* kv, const void* q, int32_t n_q_heads,
                             int32_t n_q_rows, int32_t q_pos0, int32_t tile_rows, float scale,
                             const int32_t* idx, const int32_t* count, int32_t max_sel,
                             float* out, float* lse, void* ws, size_t ws_bytes, void* stream);

/* (e) One whole decode step in one launch ([OFFLINE] "The comparison": after
 * the new token's key is in the cache, score the chunks against the current
 * query, keep the best ones under the budget and attend only to them).
 * Computes exactly what this sequence computes, with the same arguments:
 *   sparse_attn_build_meta(kv, rule, -1, meta);          refresh the newest page
 *   sparse_attn_select(kv, meta, rule, q, n_q_heads, budget, max_sel,
 *                      sel_idx, sel_count, NULL, ...);
 *   sparse_attn_decode(kv, q, n_q_heads, B, 0, 1, scale, sel_idx, sel_count,
 *                      max_sel, out, lse, ...);
 * Results are bit-identical to that sequence, except under a token budget,
 * where the step divides the attention work by the budget (the separate decode
 * call does not know it and divides by max_sel): out and lse then agree to
 * rounding (the split partials merge in a different grouping), meta, sel_idx
 * and sel_count exactly.
 * meta is read and written (the metadata of the page or chunk holding token
 * N_b - 1 is rebuilt from K; every other page must be current).  sel_idx and
 * sel_count are written as by sparse_attn_select.  Work items of the three
 * stages share one persistent grid: the decode of a (sequence, KV head) starts
 * as soon as its selection is written, while other units are still being
 * scored; a decode item waits for its selection with a bounded wait (about a
 * second; SA_ERR_TIMEOUT when it runs out).  Needs B * n_kv_heads <= 32768 and
 * the workspace sized by sparse_attn_workspace_size.  out (and lse) may lie in
 * device memory or in pinned host memory, which the device addresses directly
 * under unified addressing: the result then crosses PCIe while the launch
 * runs, each unit's rows as its attention completes. */
sa_status sparse_attn_decode_step(const sa_kv_desc* kv, void* meta, sa_score_rule rule,
                                  const void* q, int32_t n_q_heads, const sa_budget* budget,
                                  int32_t max_sel, float scale, int32_t* sel_idx,
                                  int32_t* sel_count, float* out, float* lse, void* ws,
                                  size_t ws_bytes, void* stream);

/* Element type of the attention output of sparse_attn_decode_step_append. */
typedef enum {
  SA_OUT_F32 = 0,   /* fp32 [B][Hq][128] */
  SA_OUT_BF16 = 1   /* bf16 [B][Hq][128]: the fp32 result rounded to nearest even */
} sa_out_dtype;

/* (e') The decode step with the append of the newest token fused in
 * ([OFFLINE] "The comparison": the cache grows by one token per decode step,
 * and that token is scored and attended in the same step).  Same as
 * sparse_attn_decode_step, except that row N_b - 1 of the cache does not have
 * to hold the newest token yet: k_new and v_new (device, bf16
 * [B][n_kv_heads][128], 8-byte aligned, read only) are stored into the cache
 * at row N_b - 1 of every (sequence, KV head), so kv->k and kv->v must be
 * writable.  The newest page's metadata is rebuilt with k_new, and the
 * attention reads the appended row.  Results (meta, sel_idx, sel_count, out,
 * lse) and the cache contents afterwards are identical to storing the row
 * first and calling sparse_attn_decode_step.  out (16-byte aligned) holds
 * out_dtype elements: SA_OUT_F32 as in sparse_attn_decode_step, or SA_OUT_BF16,
 * the same fp32 values rounded to bf16 (half the bytes to read back; lse stays
 * fp32).  A (sequence, KV head) whose length is out of range is not appended
 * (SA_ERR_DEVICE_CHECK).  Null or misaligned k_new / v_new, or an unknown
 * out_dtype: SA_ERR_INVALID. */
sa_status sparse_attn_decode_step_append(const sa_kv_desc* kv, void* meta, sa_score_rule rule,
                                         const void* q, int32_t n_q_heads, const void* k_new,
                                         const void* v_new, const sa_budget* budget,
                                         int32_t max_sel, float scale, int32_t* sel_idx,
                                         int32_t* sel_count, void* out, sa_out_dtype out_dtype,
                                         float* lse, void* ws, size_t ws_bytes, void* stream);

/* (f) Per-query-head selection: every query head keeps its own page set,
 * the other reading of how GQA shares a selection ([OFFLINE] "The comparison"
 * scores chunks against the current query; here "the query" is one head
 * rather than the group of G heads that share a KV head).
 *   sparse_attn_select_per_head: as sparse_attn_select, except that the unit
 *     is (sequence, query head h): the score of a page is head h's own score
 *     (no group maximum) against the metadata of KV head h / G, and
 *     sel_idx is [B][n_q_heads][max_sel], sel_count [B][n_q_heads],
 *     scores_out [B][n_q_heads][max_pages].
 *   sparse_attn_decode_per_head: decode (one row per sequence) where query
 *     head h attends the pages listed for it in idx [B][n_q_heads][max_sel]
 *     (count [B][n_q_heads]), reading K/V of KV head h / G.  out and lse as
 *     in sparse_attn_decode.
 *   sparse_attn_decode_step_per_head: sparse_attn_decode_step with per-head
 *     units: one launch computes what build_meta(first_token = -1) ->
 *     sparse_attn_select_per_head -> sparse_attn_decode_per_head compute
 *     (the newest page's metadata is refreshed once per KV head); sel_idx,
 *     sel_count as in sparse_attn_select_per_head.  As with the shared step,
 *     token budgets may round differently from the separate calls (the
 *     attention splits follow the budget, not max_sel).
 * All take the workspace sized by sparse_attn_workspace_size_per_head (B *
 * n_q_heads <= 65536 units; the step needs 2 * B * n_q_heads <= 65536); other
 * checks and errors as in the shared calls.  K/V bytes read grow with the
 * number of distinct pages the G heads keep. */
size_t sparse_attn_workspace_size_per_head(const sa_kv_desc* kv, int32_t n_q_heads, int32_t max_sel);
sa_status sparse_attn_select_per_head(const sa_kv_desc* kv, const void* meta, sa_score_rule rule,
                                      const void* q, int32_t n_q_heads, const sa_budget* budget,
                                      int32_t max_sel, int32_t* sel_idx, int32_t* sel_count,
                                      float* scores_out, void* ws, size_t ws_bytes, void* stream);
sa_status sparse_attn_decode_per_head(const sa_kv_desc* kv, const void* q, int32_t n_q_heads,
                                      float scale, const int32_t* idx, const int32_t* count,
                                      int32_t max_sel, float* out, float* lse, void* ws,
                                      size_t ws_bytes, void* stream);
sa_status sparse_attn_decode_step_per_head(const sa_kv_desc* kv, void* meta, sa_score_rule rule,
                                           const void* q, int32_t n_q_heads, const sa_budget* budget,
                                           int32_t max_sel, float scale, int32_t* sel_idx,
                                           int32_t* sel_count, float* out, float* lse, void* ws,
                                           size_t ws_bytes, void* stream);

/* (d) Uncertainty router over query tiles ([ROUTER] "Methodologie" steps 2-5).
 * B == 1, fixed blocks (page_size = block size).  q bf16 [n_q_rows][n_q_heads][128]
 * at positions q_pos0 + r; tiles of tile_rows consecutive rows.  For tile t
 * and kv head g: the eligible blocks are those whose first token is not after
 * the tile's last row; the tile score of a block is the max over the tile's
 * rows and the group's G heads of the per-row score.  sigma[t][g] from the
 * descending scores (1 if at most k blocks are eligible, 0 if s_(0) = s_(k));
 * sigma_bar[t] = mean over kv heads; tau = the linear-interpolation quantile
 * `quantile` of sigma_bar over the tiles (or *tau if tau is non-null);
 * triggered[t] = sigma_bar[t] < tau.  kv_idx[t][g][0 .. rho*k) lists blocks in
 * RANK order: the first min(rho*k, E) if triggered else the first min(k, E),
 * padded with -1; kv_count[t][g] = number of valid entries.
 * tau_out (nullable): the threshold used. */
sa_status sparse_attn_route(const sa_kv_desc* kv, const void* meta, sa_score_rule rule,
                            const void* q, int32_t n_q_heads, int32_t n_q_rows,
                            int32_t q_pos0, int32_t tile_rows, int32_t k, int32_t rho,
                            float quantile, const float* tau, int32_t* kv_idx,
                            int32_t* kv_count, float* sigma, float* sigma_bar,
                            uint8_t* triggered, float* tau_out, void* ws, size_t ws_bytes,
                            void* stream);

/* (d') The router applied to decode ([ROUTER] "Methodologie" steps 2-5 with
 * tiles of one query row): every sequence b of the batch is a tile whose one
 * row sits at position N_b - 1, so all P_b = ceil(N_b / page_size) pages are
 * eligible, and its block score for KV head g is the decode group score
 * (max over the G heads of the envelope or centroid score, as in
 * sparse_attn_select).  sigma[b][g] from the descending scores (1 if P_b <= k,
 * 0 if s_(0) = s_(k)); sigma_bar[b] = mean over kv heads; tau = the
 * linear-interpolation quantile `quantile` of sigma_bar over the batch's
 * sequences (or *tau if tau is non-null); triggered[b] = sigma_bar[b] < tau.
 * kv_idx[b][g][0 .. rho*k) lists pages in RANK order (score descending, lower
 * index first): the first min(rho*k, P_b) if triggered else the first
 * min(k, P_b), padded with -1; kv_count[b][g] = number of valid entries, so
 * sparse_attn_decode(..., idx = kv_idx, count = kv_count, max_sel = rho*k)
 * attends exactly the listed pages.  Fixed pages only (page_size > 0), B <=
 * 1024, rho*k <= 1023; the workspace sized by sparse_attn_workspace_size with
 * max_sel >= rho*k.  tau_out (nullable): the threshold used.  Two launches. */
sa_status sparse_attn_route_decode(const sa_kv_desc* kv, const void* meta, sa_score_rule rule,
                                   const void* q, int32_t n_q_heads, int32_t k, int32_t rho,
                                   float quantile, const float* tau, int32_t* kv_idx,
                                   int32_t* kv_count, float* sigma, float* sigma_bar,
                                   uint8_t* triggered, float* tau_out, void* ws, size_t ws_bytes,
                                   void* stream);

/* Test of the step's bounded wait (failure detection without a GPU fault).
 * Runs sparse_attn_decode_step, except that the selection of unit
 * `held_unit` (= b * n_kv_heads + g) is never published: the decode items of
 * that unit poll its flag `flag_spin_limit` times (each poll a load and a
 * sleep of at most 256 ns), then record SA_ERR_TIMEOUT in the workspace
 * status word, and the CTA that waited stops taking work.  The launch still
 * ends, every other CTA finishes its items, and the last CTA out leaves the
 * workspace's counters and queue clean, so the next call on the same
 * workspace runs normally (read and clear the status first with
 * sparse_attn_get_device_status).  Outputs of this call are unspecified.
 * SA_ERR_INVALID: held_unit out of range or flag_spin_limit == 0; otherwise
 * the errors of sparse_attn_decode_step.  The pages have no counterpart: it
 * exists to test the error path. */
sa_status sparse_attn_decode_step_wait_test(const sa_kv_desc* kv, void* meta, sa_score_rule rule,
                                            const void* q, int32_t n_q_heads, const sa_budget* budget,
                                            int32_t max_sel, float scale, int32_t* sel_idx,
                                            int32_t* sel_count, float* out, float* lse,
                                            int32_t held_unit, uint32_t flag_spin_limit, void* ws,
                                            size_t ws_bytes, void* stream);

/* The router applied to decode and the decode over its lists, in ONE launch
 * ("Onzekerheidsgestuurde Selectie voor Blok-schaarse Aandacht",
 * "Methodologie" steps 1-5 on one-row tiles; what sparse_attn_route_decode
 * followed by sparse_attn_decode over kv_idx / kv_count computes, after the
 * newest page's metadata is refreshed as in sparse_attn_decode_step: the
 * lists, sigma, sigma_bar, tau and triggers exactly, out and lse up to
 * rounding, as the attention runs in a top-k and an expansion window merged
 * in two steps).  meta is read and its newest page rewritten.
 * Outputs: kv_idx / kv_count / sigma / sigma_bar / triggered / tau_out as
 * sparse_attn_route_decode (lists in rank order, -1 padded), out fp32
 * [B][Hq][128] and lse (nullable) as sparse_attn_decode.  Every unit's top k
 * pages are attended as soon as the unit is selected; the pages k .. rho*k-1
 * of the triggered sequences once the batch's triggers are known.  Fixed
 * pages only, B <= 1024, rho*k <= 1023; the workspace sized by
 * sparse_attn_workspace_size with max_sel >= rho*k. */
sa_status sparse_attn_route_decode_step(const sa_kv_desc* kv, void* meta, sa_score_rule rule,
                                        const void* q, int32_t n_q_heads, int32_t k, int32_t rho,
                                        float quantile, const float* tau, float scale, int32_t* kv_idx,
                                        int32_t* kv_count, float* sigma, float* sigma_bar,
                                        uint8_t* triggered, float* tau_out, float* out, float* lse,
                                        void* ws, size_t ws_bytes, void* stream);

/* Copy the workspace status word to *host_out (SA_OK if no device check
 * fired since the last init/clear) and clear it.  Synchronises `stream`. */
sa_status sparse_attn_get_device_status(void* ws, sa_status* host_out, void* stream);

/* (c') Sparse attention without a caller-provided workspace.
 * The pages have no counterpart for this call; it exists for deployment.
 * Some callers cannot allocate device memory at the point where they run the
 * attention: a plugin interface that hands an op only its input and output
 * pointers at enqueue time, or a latency-bound decode loop that must never
 * pay the device-wide synchronisation that cudaMalloc can cause.  For them
 * this call computes exactly what sparse_attn_decode computes (same arguments
 * minus ws/ws_bytes) using a scratch area built into the library: one
 * file-scope device array of 8 MiB, which every GPU that loads the library
 * holds until the process exits.
 *  - The first call on a device, with that device current, looks up the
 *    array's device address and caches it; make that first call before any
 *    stream capture.
 *  - Every call shares the one array and overwrites it.  Calls that may run at
 *    the same time on the GPU (different streams, overlapping graph launches,
 *    several host threads) race and corrupt each other's results: order them
 *    on one stream.  Each call clears the counters it uses before launching.
 *  - Limits: one-row decode only (tile_rows == 1; multi-row tile attention,
 *    tile_rows > 1, returns SA_ERR_UNSUPPORTED); at most 4096 (row, KV head)
 *    units per call, and the split partials of the call must fit the array;
 *    beyond either the call returns SA_ERR_WORKSPACE and launches nothing.
 *  - It allocates and frees no memory.
 *  - device_status (nullable): a device int32, zeroed by the caller, that
 *    receives the first device-side error code of the call (a range check or
 *    a bounded-wait timeout).  With device_status null such errors are NOT
 *    reported: they land in the array's own status word, which the next call
 *    clears before anyone could read it.  Pass one to see them. */
sa_status sparse_attn_decode_static(const sa_kv_desc* kv, const void* q, int32_t n_q_heads,
                                    int32_t n_q_rows, int32_t q_pos0, int32_t tile_rows,
                                    float scale, const int32_t* idx, const int32_t* count,
                                    int32_t max_sel, float* out, float* lse,
                                    int32_t* device_status, void* stream);

/* Static description of a status code (never null). */
const char* sparse_attn_status_string(sa_status s);

#ifdef __cplusplus
}
#endif
#endif /* SPARSE_ATTN_H */
