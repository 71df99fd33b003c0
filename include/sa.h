/*
 * sa.h — C ABI of the paged sparse-KV attention library (libsa.so, sm_100a).
 *
 * What the calls compute (sources are page titles and sections):
 *  - sa_select_pages: page scoring against per-page key summaries and top-k
 *    selection with forced sink and local pages ("Universal Attention Engine —
 *    Declarative Sparse Attention for Production", "The Product" for the
 *    sink/local/budget pattern and "Content-Dependent Dynamic Routing" for
 *    top_k_blocks(q @ mean(k_blocks))).
 *  - sa_select_pages_tiered: TileSparse's Critical/Ambient tiers ("TileSparse:
 *    Arithmetic-Intensity-Aware Sparse Attention for Compute-Bound LLM
 *    Decoding", "Motivation").
 *  - sa_sparse_decode: attention over per-head page lists read in place from a
 *    paged cache (UAE "Architecture": gather-based sparse KV decode over a
 *    PagedAttention-compatible layout; TileSparse "Two implementations": a
 *    per-head page-list Flash-decode kernel), split over the list.
 *  - sa_combine: the log-sum-exp merge of split partials (the merge step of a
 *    split-KV Flash-decode, TileSparse "Configuration", mode "full").
 *  - sa_block_union: CompactAttention's Block-Union KV Selection (abstract on
 *    the page titled "Causal Attention on CPU: ..."): Q-block union plus
 *    intra-group union into per-group KV block tables, used in place.
 *  - sa_build_page_summaries / sa_update_page_summaries: the per-page key
 *    means the router scores (all referenced pages / the pages an append
 *    changed)
 *    (UAE "Content-Dependent Dynamic Routing", mean(k_blocks)).
 *  - sa_sparse_attention / sa_sparse_step: decode + merge, and selection +
 *    decode + merge, in one call each.
 *  - sa_append_kv: new tokens written into their pages and those pages'
 *    summaries recomputed, in one launch.
 *  - sa_select_ambient_heads: the ambient head set by estimated attention-mass
 *    coverage (TileSparse's AutoTuner objective).
 *  - sa_sparse_decode_at / sa_sparse_attention_at: query tokens at explicit
 *    positions (a prompt chunk computed against a longer cache).
 *  - *_dir: the same calls over a two-level page map sized to the pages in
 *    use (SPIN's two-level metadata).
 *
 * Conventions for every call:
 *  - Pointers marked (dev) are caller-owned device memory on the current
 *    device; (host) pointers are read before the call returns.  The library
 *    allocates no memory in a call and carries no data from one call to the
 *    next (it caches only per-context launch set-up: shared-memory caps, SM
 *    count, occupancy; sa_select_pages_no_alloc's static array is described
 *    there); scratch space (workspace) is caller-owned device memory of the
 *    size a *_size call gives.
 *  - bf16 tensors are passed as uint16_t bit patterns.  Strides are in
 *    elements; the innermost (feature) stride must be 1, other strides of
 *    bf16 tensors multiples of 8 elements, base pointers 16-byte aligned.
 *  - Calls are asynchronous and ordered on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream).  Argument errors are found on the host
 *    before any launch and return SA_ERR_INVALID_ARG or SA_ERR_UNSUPPORTED
 *    with nothing launched.  Launch failures return SA_ERR_CUDA.
 *  - dev_error (dev, optional, may be NULL): an int32 word the kernels OR
 *    error bits into when data they read is out of range (a page id outside
 *    the sequence or the pool, a list count above its capacity).  The
 *    offending page is skipped; kernels never trap.  The caller zeroes it and
 *    reads it back when it wants to know.
 *
 * Page-count reading of a token budget (the pages give tokens, not pages):
 *   n_sink = ceil(sink/P), n_local = ceil(local/P), budget_pages = floor(budget/P),
 *   k_top = budget_pages - n_sink - n_local (must be >= 0).
 */
#ifndef SA_H_
#define SA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SA_API __attribute__((visibility("default")))
#else
#define SA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SA_OK = 0,
  SA_ERR_INVALID_ARG = 1,   /* a null pointer, a bad size, stride or alignment */
  SA_ERR_UNSUPPORTED = 2,   /* valid, but outside what the kernels implement   */
  SA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required      */
  SA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed            */
} sa_status;

/* Bits kernels OR into *dev_error. */
#define SA_DEVERR_PAGE_RANGE 1   /* logical page >= ceil(seq_len/P) or < 0      */
#define SA_DEVERR_POOL_RANGE 2   /* physical page id outside [0, P_pool)        */
#define SA_DEVERR_COUNT 4        /* list count < 0 or above its capacity        */
#define SA_DEVERR_TIMEOUT 8      /* a bounded wait on a copy gave up             */
#define SA_DEVERR_VALUE_RANGE 16 /* FP8 pages: a query value beyond +-65504      */

/* Human-readable name of a status code (static storage). */
SA_API const char* sa_status_string(int status);

/* ABI version: 100 * major + minor. */
SA_API int sa_abi_version(void);

/*
 * sa_select_pages — page scoring and top-k selection, GQA.
 *
 * For each (b, kv head g): every logical page p < N_b = ceil(seq_lens[b]/P)
 * of the sequence has the summary sigma = summaries[page_table[b,p], g, :].
 * Sink pages [0, n_sink) and local pages [N_b - n_local, N_b) are always
 * selected; of the remaining candidates the k_top with the largest score win,
 * ties to the lower logical page.  score_p = max over the group's query rows
 * (t < T, heads h with h / (Hq/Hkv) == g) of the dot product q[b,t,h,:].sigma,
 * unscaled and correctly rounded to float64 (so the selection equals the one
 * exact arithmetic gives).  If N_b <= budget_pages every page is selected.
 *
 *  q          (dev) [B,T,Hq,Dk] bf16, strides q_strides (elements)
 *  summaries  (dev) [P_pool,Hkv,Dk] bf16, contiguous
 *  page_table (dev) [B,max_pages] int32 physical page ids, contiguous
 *  seq_lens   (dev) [B] int32, 0 <= seq_lens[b] <= max_pages*P
 *  out_pages  (dev) [B,Hkv,budget_pages] int32: selected logical ids ascending,
 *                   then -1 padding
 *  out_counts (dev) [B,Hkv] int32
 *  workspace  (dev) sa_select_workspace_size(B, Hkv, max_pages) bytes (may be
 *                   NULL when k_top == 0); SA_ERR_WORKSPACE if missing or short
 * Supported: Dk in {64,128,256}, T*Hq/Hkv <= 16, max_pages <= 16384.
 * Two launches: a scoring pass over all candidate pages (every SM streams
 * summaries) and one selection block per (b, g).
 */
SA_API int sa_select_pages(const uint16_t* q, const int64_t q_strides[4],
                           const uint16_t* summaries, const int32_t* page_table,
                           const int32_t* seq_lens, int B, int T, int Hq, int Hkv, int Dk,
                           int page_size, int max_pages, int P_pool, int sink_tokens,
                           int local_tokens, int budget_tokens, int32_t* out_pages,
                           int32_t* out_counts, void* workspace, size_t workspace_bytes,
                           int32_t* dev_error, void* stream);

/* Bytes of device workspace sa_select_pages needs (16-byte aligned, no
 * initial contents; the call overwrites it): the float32 lower/upper score
 * bounds of every page, [B, Hkv, max_pages] x 8 bytes.  0 for bad sizes. */
SA_API size_t sa_select_workspace_size(int B, int Hkv, int max_pages);

/*
 * sa_select_pages_no_alloc — sa_select_pages for callers that cannot
 * allocate device memory at the call site: code running inside a CUDA-graph
 * capture, a serving loop whose memory pool is sealed after warm-up, or a host
 * framework that owns every allocation and passes only raw pointers.  (The
 * pages this library implements have no counterpart of this entry point; it
 * is a deployment convenience.)
 *
 * Same arguments, outputs and results as sa_select_pages, minus the
 * workspace: the score bounds go to a 16 MiB array of the library's own device
 * memory (2,097,152 pages x 8 bytes), which every GPU that loads the library
 * holds until the process exits.  Limit: B * Hkv * max_pages <= 2,097,152;
 * larger calls return SA_ERR_UNSUPPORTED and launch nothing.  The first call
 * on a device looks up the array's device address (cudaGetSymbolAddress) and
 * keeps it for that device's current context; the first call after the
 * context is created again (cudaDeviceReset, say) looks it up afresh.  Make
 * that first call before any stream capture.  All calls share the one array
 * (it needs no clearing: each call writes every entry it reads), so calls
 * whose kernels overlap on the GPU — on different streams, or from different
 * threads — race and must be serialised by the caller.
 */
SA_API int sa_select_pages_no_alloc(const uint16_t* q, const int64_t q_strides[4],
                                    const uint16_t* summaries, const int32_t* page_table,
                                    const int32_t* seq_lens, int B, int T, int Hq, int Hkv,
                                    int Dk, int page_size, int max_pages, int P_pool,
                                    int sink_tokens, int local_tokens, int budget_tokens,
                                    int32_t* out_pages, int32_t* out_counts, int32_t* dev_error,
                                    void* stream);

/*
 * sa_select_pages_tiered — Critical / Ambient tier selection for one shared
 * latent KV head (MLA; "TileSparse: Arithmetic-Intensity-Aware Sparse
 * Attention for Compute-Bound LLM Decoding", "Motivation": a Critical Tier of
 * alpha pages computed with all query heads, an Ambient Tier of beta pages
 * computed with h heads).
 *
 * Every logical page p < N_b of sequence b is a candidate, scored by the max
 * over all T x Hq query rows of q[b,t,h,:] . summaries[page_table[b,p],0,:]
 * (unscaled, correctly rounded to float64).  Ranked by (score desc, logical
 * page asc), the first alpha pages form the critical tier and the next beta
 * the ambient tier.  Output as two decode lists per sequence:
 *   lists[b,0,:] = critical pages ascending, lists[b,1,:] = critical + ambient
 *   pages ascending, each -1 padded to alpha+beta; list_counts[b,0..1].
 * Give sa_sparse_decode head_to_list[h] = 1 for the ambient heads, 0 for the
 * rest.
 *
 *  q          (dev) [B,T,Hq,Dk] bf16, strides q_strides
 *  summaries  (dev) [P_pool,1,Dk] bf16, contiguous
 *  page_table (dev) [B,max_pages] int32;  seq_lens (dev) [B] int32
 *  lists      (dev) [B,2,alpha+beta] int32;  list_counts (dev) [B,2] int32
 *  workspace  (dev) sa_select_tiered_workspace_size(B,T,Hq,max_pages) bytes
 * Supported: Dk % 8 == 0, Dk <= 880, max_pages <= 8192 (the choose pass keeps
 * 21 bytes per page in shared memory).
 */
SA_API int sa_select_pages_tiered(const uint16_t* q, const int64_t q_strides[4],
                                  const uint16_t* summaries, const int32_t* page_table,
                                  const int32_t* seq_lens, int B, int T, int Hq, int Dk,
                                  int page_size, int max_pages, int P_pool, int alpha, int beta,
                                  int32_t* lists, int32_t* list_counts, void* workspace,
                                  size_t workspace_bytes, int32_t* dev_error, void* stream);

/* Bytes of workspace sa_select_pages_tiered needs (16-byte aligned). */
SA_API size_t sa_select_tiered_workspace_size(int B, int T, int Hq, int max_pages);

/*
 * sa_select_ambient_heads — the h query heads that attend the ambient tier
 * ("TileSparse: Arithmetic-Intensity-Aware Sparse Attention for Compute-Bound
 * LLM Decoding", "Motivation": the Ambient Tier is computed with h heads;
 * "Configuration": an AutoTuner picks them per layer by estimated
 * attention-mass coverage).  This library's reading of that coverage: for
 * sequence b, query token t and head h, page p carries the estimated mass
 * n_p * exp(scale * (q[b,t,h] . sigma_p)) (n_p its valid tokens, sigma_p its
 * summary: each key replaced by the page's mean); the coverage is the share of
 * the sequence's estimated mass on its ambient pages (in lists[b,1] and not in
 * lists[b,0]); a head's score sums its coverages over every b and t.  The h
 * heads of largest score win, ties to the lower head.  A calibration call (once
 * per layer and traffic sample): pass the chosen heads to sa_sparse_decode as
 * head_to_list[h] = 1 for them, 0 for the others.
 *
 *  q, summaries, page_table, seq_lens   as sa_select_pages_tiered
 *  lists      (dev) [B,2,list_cap] int32, list_counts (dev) [B,2]: the output of
 *             sa_select_pages_tiered (critical pages; critical + ambient pages)
 *  scale      the attention scale (finite)
 *  out_heads  (dev) [h] int32: the chosen heads, ascending
 *  out_scores (dev, optional) [Hq] float64: every head's score
 *  workspace  (dev) sa_select_ambient_heads_workspace_size(B,T,Hq,max_pages)
 *             bytes, 8-byte aligned
 * Dot products in float64 from exact bf16 products, masses and scores in
 * float64.  Supported: Dk <= 768, Hq <= 1024.
 */
SA_API size_t sa_select_ambient_heads_workspace_size(int B, int T, int Hq, int max_pages);
SA_API int sa_select_ambient_heads(const uint16_t* q, const int64_t q_strides[4],
                                   const uint16_t* summaries, const int32_t* page_table,
                                   int max_pages, const int32_t* seq_lens, const int32_t* lists,
                                   const int32_t* list_counts, int list_cap, int B, int T, int Hq,
                                   int Dk, int page_size, int P_pool, float scale, int h,
                                   int32_t* out_heads, double* out_scores, void* workspace,
                                   size_t workspace_bytes, int32_t* dev_error, void* stream);

/*
 * sa_sparse_decode — split-KV attention over per-head page lists.
 *
 * Query row (b, t, h) attends the keys of list l = head_to_list[h] of
 * sequence b, read from kv head h / (Hq/Hkv): the tokens j of every logical
 * page p in lists[b,l,0:list_counts[b,l]] whose position p*P + j is below
 * seq_lens[b] and at most seq_lens[b] - T + t (query token t sits at that
 * position: causal MTP / chunked prefill).  s_j = scale * q.k_j; natural-log
 * LSE.  Split s takes the entries [s*c, (s+1)*c) of the list with
 * c = ceil(max_list/n_splits) (so a short list leaves its last splits empty;
 * the many-row kernel instead takes c = ceil(list_count/n_splits), an equal
 * share of each list's actual length) and writes its own normalised output
 * and LSE.  A split without a visible
 * key writes LSE = -inf; its O rows are 0 when n_splits == 1 and otherwise
 * unspecified (sa_combine gives such a split no weight).  With n_splits == 1
 * the partials are the final result; otherwise pass them to sa_combine.
 *
 *  q            (dev) [B,T,Hq,Dk] bf16, strides q_strides
 *  k_cache      (dev) [P_pool,Hkv,P,Dk] bf16, strides k_strides (vLLM's
 *                     [P_pool,P,Hkv,Dk] is the same tensor with other strides)
 *  v_cache      (dev) [P_pool,Hkv,P,Dv] bf16, strides v_strides; may alias
 *                     k_cache (MLA: V = first Dv columns of the latent K)
 *  page_table   (dev) [B,max_pages] int32;  seq_lens (dev) [B] int32
 *  lists        (dev) [B,n_lists,max_list] int32 logical page ids
 *  list_counts  (dev) [B,n_lists] int32
 *  head_to_list (host) [Hq] int32 in [0, n_lists)
 *  o_partial    (dev) [n_splits,B,T,Hq,Dv] float32
 *  lse_partial  (dev) [n_splits,B,T,Hq] float32
 * Kernels, chosen from the shapes (P a multiple of 16 up to 128 throughout):
 *  - at most 16 query rows (T x heads) per (list, kv head) pair, Dk == Dv in
 *    {64,128,256}: one warp per split, warp-level tensor-core MMAs;
 *  - more rows per pair (chunked prefill, long MTP), Dk == Dv in {64,128}:
 *    128-row tiles on tcgen05 with TMEM accumulators;
 *  - MLA, Dk == 576 with Dv == 512 and v_cache == k_cache (same strides: the
 *    values are the first 512 key columns): 64-row tiles on tcgen05.
 * Limits: Hq <= 256, at most 64 (list, kv head) pairs read by some head, at
 * most 128 heads per pair (SA_ERR_UNSUPPORTED beyond).
 * Pool rows past a sequence's end are read with the page but masked; they
 * must hold finite values (a NaN there could reach the output through 0*NaN).
 */
SA_API int sa_sparse_decode(const uint16_t* q, const int64_t q_strides[4], const uint16_t* k_cache,
                     const int64_t k_strides[4], const uint16_t* v_cache,
                     const int64_t v_strides[4], const int32_t* page_table, int max_pages,
                     const int32_t* seq_lens, const int32_t* lists, const int32_t* list_counts,
                     int n_lists, int max_list, const int32_t* head_to_list, int B, int T,
                     int Hq, int Hkv, int Dk, int Dv, int page_size, int P_pool, float scale,
                     int n_splits, float* o_partial, float* lse_partial, int32_t* dev_error,
                     void* stream);

/*
 * sa_sparse_decode_fp8 — sa_sparse_decode over K and V pages stored as FP8
 * E4M3 codes (1 sign, 4 exponent bits with bias 7, 3 fraction bits; the two
 * NaN codes must not occur) with one float32 scale per (physical page, kv
 * head): key j of a page is e4m3(k_codes[...]) * k_scale[page, kv head], and
 * likewise for values.  Source: "Universal Attention Engine — Declarative
 * Sparse Attention for Production", "Key Design Decisions" 2 (cache format:
 * paged, block-sparse, quantized) and "Roadmap" (quantized KV cache support);
 * the E4M3 format and the per-(page, kv head) scale are this library's
 * reading of "quantized".
 *
 *  k_codes, v_codes (dev) [P_pool,Hkv,P,D] uint8, strides k_strides/v_strides
 *                   (elements = bytes; unit feature stride, the others
 *                   multiples of 16; 16-byte aligned base)
 *  k_scale, v_scale (dev) [P_pool,Hkv] float32, contiguous, finite
 * Everything else (q, page table, lists, head_to_list, splits, partials,
 * device errors) as sa_sparse_decode.  Supported: D == 128 (keys and values),
 * page_size a multiple of 16 up to 128, at most 16 query rows (T x heads) per
 * (list, kv head) pair; other shapes return SA_ERR_UNSUPPORTED.
 */
SA_API int sa_sparse_decode_fp8(const uint16_t* q, const int64_t q_strides[4],
                                const uint8_t* k_codes, const int64_t k_strides[4],
                                const uint8_t* v_codes, const int64_t v_strides[4],
                                const float* k_scale, const float* v_scale,
                                const int32_t* page_table, int max_pages, const int32_t* seq_lens,
                                const int32_t* lists, const int32_t* list_counts, int n_lists,
                                int max_list, const int32_t* head_to_list, int B, int T, int Hq,
                                int Hkv, int D, int page_size, int P_pool, float scale,
                                int n_splits, float* o_partial, float* lse_partial,
                                int32_t* dev_error, void* stream);

/*
 * sa_sparse_decode_at / sa_sparse_attention_at — sa_sparse_decode and
 * sa_sparse_attention with the query positions given explicitly: query token t
 * of sequence b sits at position q_pos[b] + t and sees the listed keys at
 * positions below seq_lens[b] and at most its own.  (The other calls put the
 * queries at the end of the sequence, q_pos[b] = seq_lens[b] - T.)  For a chunk
 * of a prompt computed while the cache already holds tokens past it -- chunked
 * prefill over block tables used in place (CompactAttention abstract, on the
 * page titled "Causal Attention on CPU: A Cache-Aware and Load-Balanced
 * Scheduling Kernel for Prefill").  A token whose position is at or past
 * seq_lens[b] sees every listed key; one before every listed key sees none
 * (O = 0, LSE = -inf).
 *
 *  q_pos (dev) [B] int32 (required).  Every other argument as sa_sparse_decode
 *  (resp. sa_sparse_attention).
 */
SA_API int sa_sparse_decode_at(const uint16_t* q, const int64_t q_strides[4],
                               const uint16_t* k_cache, const int64_t k_strides[4],
                               const uint16_t* v_cache, const int64_t v_strides[4],
                               const int32_t* page_table, int max_pages, const int32_t* seq_lens,
                               const int32_t* q_pos, const int32_t* lists,
                               const int32_t* list_counts, int n_lists, int max_list,
                               const int32_t* head_to_list, int B, int T, int Hq, int Hkv, int Dk,
                               int Dv, int page_size, int P_pool, float scale, int n_splits,
                               float* o_partial, float* lse_partial, int32_t* dev_error,
                               void* stream);
SA_API int sa_sparse_attention_at(const uint16_t* q, const int64_t q_strides[4],
                                  const uint16_t* k_cache, const int64_t k_strides[4],
                                  const uint16_t* v_cache, const int64_t v_strides[4],
                                  const int32_t* page_table, int max_pages,
                                  const int32_t* seq_lens, const int32_t* q_pos,
                                  const int32_t* lists, const int32_t* list_counts, int n_lists,
                                  int max_list, const int32_t* head_to_list, int B, int T, int Hq,
                                  int Hkv, int Dk, int Dv, int page_size, int P_pool, float scale,
                                  int n_splits, float* o_out, uint16_t* o_out_bf16, float* lse_out,
                                  void* workspace, size_t workspace_bytes, int32_t* dev_error,
                                  void* stream);

/*
 * sa_combine — merge split partials: lse = log sum_s exp(lse_s),
 * O = sum_s exp(lse_s - lse) O_s; splits with lse_s = -inf weigh nothing
 * (their O rows are not used, whatever they hold);
 * rows whose splits are all empty give O = 0, lse = -inf.
 *
 *  o_partial  (dev) [n_splits,rows,Dv] float32;  lse_partial (dev) [n_splits,rows]
 *  o_out      (dev, optional) [rows,Dv] float32
 *  o_out_bf16 (dev, optional) [rows,Dv] bf16 (round to nearest even)
 *  lse_out    (dev, optional) [rows] float32
 * At least one output must be given.  Dv % 4 == 0.  Limits: n_splits <= 64
 * and rows * Dv / 4 < 2^32 (SA_ERR_UNSUPPORTED otherwise).
 */
SA_API int sa_combine(const float* o_partial, const float* lse_partial, int n_splits, int64_t rows,
               int Dv, float* o_out, uint16_t* o_out_bf16, float* lse_out, void* stream);

/*
 * sa_sparse_attention — sa_sparse_decode followed by the sa_combine merge, in
 * one call with final outputs: the decode launch writes the split partials
 * into the workspace, then the combine launch merges them.  (A merge inside
 * the decode kernel, by the last split of each pair to finish, was measured
 * slower than the separate merge launch: one warp's dependent L2 round trips
 * over the pair's partials cost more than the launch.)  Sources: as
 * sa_sparse_decode and sa_combine (the merge step of a split Flash-decode,
 * "TileSparse", "Configuration": mode full = fused Flash-decode).
 *
 *  q ... n_splits   as sa_sparse_decode
 *  o_out      (dev, optional) [B,T,Hq,Dv] float32, 16-byte aligned
 *  o_out_bf16 (dev, optional) [B,T,Hq,Dv] bf16, 8-byte aligned
 *  lse_out    (dev, optional) [B,T,Hq] float32
 *  workspace  (dev) sa_sparse_attention_workspace_size(B,T,Hq,Dv,n_splits)
 *             bytes, 16-byte aligned, owned by the caller (the partials; no
 *             initial contents needed).  Calls sharing a workspace must not
 *             overlap.
 * At least one output must be given.  Errors: as sa_sparse_decode and
 * sa_combine (n_splits <= 64); SA_ERR_WORKSPACE for a missing, misaligned or
 * short workspace.
 */
SA_API size_t sa_sparse_attention_workspace_size(int B, int T, int Hq, int Dv, int n_splits);
SA_API int sa_sparse_attention(const uint16_t* q, const int64_t q_strides[4],
                               const uint16_t* k_cache, const int64_t k_strides[4],
                               const uint16_t* v_cache, const int64_t v_strides[4],
                               const int32_t* page_table, int max_pages, const int32_t* seq_lens,
                               const int32_t* lists, const int32_t* list_counts, int n_lists,
                               int max_list, const int32_t* head_to_list, int B, int T, int Hq,
                               int Hkv, int Dk, int Dv, int page_size, int P_pool, float scale,
                               int n_splits, float* o_out, uint16_t* o_out_bf16, float* lse_out,
                               void* workspace, size_t workspace_bytes, int32_t* dev_error,
                               void* stream);

/*
 * sa_sparse_step — the whole GQA sparse-attention call in one entry point:
 * sa_select_pages (scoring against the page summaries, forced sink and local
 * pages, top-k) and then sa_sparse_attention over the selected lists, every
 * head h reading the list of its kv head h / (Hq/Hkv).  Sources: as
 * sa_select_pages ("Universal Attention Engine — Declarative Sparse Attention
 * for Production", "Content-Dependent Dynamic Routing": selected blocks get
 * full attention) and sa_sparse_attention.
 *
 *  q, summaries, page_table, seq_lens, budget arguments   as sa_select_pages
 *  k_cache, v_cache (dev) [P_pool,Hkv,P,D] bf16, strides as sa_sparse_decode
 *  scale      s in s_j = scale * q.k_j (finite)
 *  n_splits   decode splits per list; <= 0 picks the default for the current
 *             device (the splits that fill one wave of resident decode warps)
 *  out_pages  (dev) [B,Hkv,budget_pages] int32, out_counts (dev) [B,Hkv]: the
 *             selection, as sa_select_pages writes it
 *  o_out, o_out_bf16, lse_out   as sa_sparse_attention (at least one)
 *  workspace  (dev) sa_sparse_step_workspace_size(...) bytes, 16-byte aligned,
 *             caller-owned, no initial contents; calls sharing one must not
 *             overlap
 * Supported: D in {64,128,256}, T*Hq/Hkv <= 16, max_pages <= 16384, page_size
 * a multiple of 16 up to 128, Hq <= 256.  Every argument is checked before the
 * first launch; then four launches (score, choose, decode, merge).
 */
SA_API size_t sa_sparse_step_workspace_size(int B, int T, int Hq, int Hkv, int D, int page_size,
                                            int max_pages, int budget_tokens, int n_splits);
SA_API int sa_sparse_step(const uint16_t* q, const int64_t q_strides[4], const uint16_t* summaries,
                          const uint16_t* k_cache, const int64_t k_strides[4],
                          const uint16_t* v_cache, const int64_t v_strides[4],
                          const int32_t* page_table, int max_pages, const int32_t* seq_lens,
                          int B, int T, int Hq, int Hkv, int D, int page_size, int P_pool,
                          int sink_tokens, int local_tokens, int budget_tokens, float scale,
                          int n_splits, int32_t* out_pages, int32_t* out_counts, float* o_out,
                          uint16_t* o_out_bf16, float* lse_out, void* workspace,
                          size_t workspace_bytes, int32_t* dev_error, void* stream);

/*
 * sa_sparse_step_fp8 — sa_sparse_step over FP8 E4M3 pages: the selection
 * (bf16 queries against the bf16 summaries sa_build_page_summaries_fp8 gives),
 * then sa_sparse_attention_fp8 over the selected lists, in one call.  K and V
 * as sa_sparse_decode_fp8 (codes [P_pool,Hkv,P,D] with strides, scales
 * [P_pool,Hkv] float32), D == 128; every other argument, the workspace (sized
 * by sa_sparse_step_workspace_size) and the errors as sa_sparse_step.
 */
SA_API int sa_sparse_step_fp8(const uint16_t* q, const int64_t q_strides[4],
                              const uint16_t* summaries, const uint8_t* k_codes,
                              const int64_t k_strides[4], const uint8_t* v_codes,
                              const int64_t v_strides[4], const float* k_scale,
                              const float* v_scale, const int32_t* page_table, int max_pages,
                              const int32_t* seq_lens, int B, int T, int Hq, int Hkv, int D,
                              int page_size, int P_pool, int sink_tokens, int local_tokens,
                              int budget_tokens, float scale, int n_splits, int32_t* out_pages,
                              int32_t* out_counts, float* o_out, uint16_t* o_out_bf16,
                              float* lse_out, void* workspace, size_t workspace_bytes,
                              int32_t* dev_error, void* stream);

/*
 * sa_sparse_attention_fp8 — sa_sparse_decode_fp8 followed by the merge, in one
 * call.  Arguments as sa_sparse_decode_fp8 for the inputs and as
 * sa_sparse_attention for the outputs and the workspace (sized with Dv = D).
 */
SA_API int sa_sparse_attention_fp8(const uint16_t* q, const int64_t q_strides[4],
                                   const uint8_t* k_codes, const int64_t k_strides[4],
                                   const uint8_t* v_codes, const int64_t v_strides[4],
                                   const float* k_scale, const float* v_scale,
                                   const int32_t* page_table, int max_pages,
                                   const int32_t* seq_lens, const int32_t* lists,
                                   const int32_t* list_counts, int n_lists, int max_list,
                                   const int32_t* head_to_list, int B, int T, int Hq, int Hkv,
                                   int D, int page_size, int P_pool, float scale, int n_splits,
                                   float* o_out, uint16_t* o_out_bf16, float* lse_out,
                                   void* workspace, size_t workspace_bytes, int32_t* dev_error,
                                   void* stream);

/*
 * sa_build_page_summaries — sigma[page_table[b,p], g, :] for every logical
 * page p < ceil(seq_lens[b]/P): the mean of the page's valid keys
 * (positions < seq_lens[b]), computed as RNE_bf16(RN64(RN64(exact sum)/n)).
 * Rows of pages no sequence references are left untouched.
 *
 *  k_cache    (dev) [P_pool,Hkv,P,Dk] bf16, strides k_strides
 *  summaries  (dev) [P_pool,Hkv,Dk] bf16, contiguous (written)
 */
SA_API int sa_build_page_summaries(const uint16_t* k_cache, const int64_t k_strides[4],
                            const int32_t* page_table, int max_pages, const int32_t* seq_lens,
                            int B, int Hkv, int Dk, int page_size, int P_pool,
                            uint16_t* summaries, int32_t* dev_error, void* stream);

/*
 * sa_update_page_summaries — the same summaries, rewritten only for the pages
 * that hold the last n_new tokens of each sequence (positions
 * [seq_lens[b] - n_new, seq_lens[b]) clamped at 0): the pages an append of
 * n_new tokens per sequence changed (normally the one last page, two when the
 * append crosses a page boundary).  Call it after the new keys are in the
 * cache and seq_lens counts them; every other summary row stays as it was.
 * Arguments as for sa_build_page_summaries; n_new >= 1 (SA_ERR_INVALID_ARG
 * otherwise).
 */
SA_API int sa_update_page_summaries(const uint16_t* k_cache, const int64_t k_strides[4],
                             const int32_t* page_table, int max_pages, const int32_t* seq_lens,
                             int B, int Hkv, int Dk, int page_size, int P_pool, int n_new,
                             uint16_t* summaries, int32_t* dev_error, void* stream);

/*
 * sa_build_page_summaries_fp8 — sa_build_page_summaries for FP8 E4M3 key
 * pages with per-(page, kv head) scales (as sa_sparse_decode_fp8): the mean of
 * the dequantized valid keys, RNE_bf16(RN64(RN64(exact sum)/n)).
 *
 *  k_codes    (dev) [P_pool,Hkv,P,Dk] uint8, strides k_strides (elements)
 *  k_scale    (dev) [P_pool,Hkv] float32, contiguous
 *  summaries  (dev) [P_pool,Hkv,Dk] bf16, contiguous (written)
 * page_size <= 128.  Other arguments as sa_build_page_summaries.
 */
SA_API int sa_build_page_summaries_fp8(const uint8_t* k_codes, const int64_t k_strides[4],
                                       const float* k_scale, const int32_t* page_table,
                                       int max_pages, const int32_t* seq_lens, int B, int Hkv,
                                       int Dk, int page_size, int P_pool, uint16_t* summaries,
                                       int32_t* dev_error, void* stream);

/*
 * sa_append_kv — append tokens to the paged cache and refresh the summaries of
 * the pages they land in, in one launch ("Universal Attention Engine —
 * Declarative Sparse Attention for Production", "Content-Dependent Dynamic
 * Routing": the router scores mean(k_blocks), so a block's mean changes when
 * tokens land in it; "Architecture": a PagedAttention-compatible cache).
 *
 * Sequence b appends n_new[b] tokens: token i (i < n_new[b]) of k_new and v_new
 * goes to position seq_lens[b] + i, i.e. row (pos % P) of physical page
 * page_table[b, pos / P], every kv head.  Then, for every page those positions
 * fall in, summaries[page, g, :] becomes the mean of the page's keys at
 * positions below seq_lens[b] + n_new[b], computed as sa_build_page_summaries
 * does (RNE_bf16(RN64(RN64(exact sum)/n))).  No other cache row or summary row
 * changes.  The pages must already be in the page table (the caller allocates
 * them); positions past its row are dropped and flagged (SA_DEVERR_PAGE_RANGE).
 *
 *  k_new, v_new (dev) [B,max_new,Hkv,D] bf16, strides kn_strides/vn_strides
 *                     (unit feature stride, others multiples of 8, 16-byte base)
 *  n_new        (dev) [B] int32 in [0, max_new] (outside: clamped, SA_DEVERR_COUNT)
 *  k_cache, v_cache (dev) [P_pool,Hkv,P,D] bf16, written in place
 *  seq_lens     (dev) [B] int32: the lengths BEFORE the append
 *  out_seq_lens (dev, optional) [B] int32: receives seq_lens[b] + n_new[b]; must
 *                     not be seq_lens itself (every block reads it)
 *  summaries    (dev) [P_pool,Hkv,D] bf16, contiguous (the touched rows rewritten)
 * D % 8 == 0.  Appends that touch the same page from two sequences race.
 */
SA_API int sa_append_kv(const uint16_t* k_new, const int64_t kn_strides[4], const uint16_t* v_new,
                        const int64_t vn_strides[4], const int32_t* n_new, int max_new,
                        uint16_t* k_cache, const int64_t k_strides[4], uint16_t* v_cache,
                        const int64_t v_strides[4], const int32_t* page_table, int max_pages,
                        const int32_t* seq_lens, int32_t* out_seq_lens, int B, int Hkv, int D,
                        int page_size, int P_pool, uint16_t* summaries, int32_t* dev_error,
                        void* stream);

/*
 * Two-level page metadata (the *_dir entry points).  SPIN ("Vortex: Efficient
 * and Programmable Sparse Attention Serving for AI Agents", the SPIN abstract:
 * a two-level hierarchical metadata layout sized to the active working set
 * rather than the worst-case address space) keeps a batch's page map in two
 * levels instead of one [B, max_pages] table:
 *
 *  page_dir    (dev) [B,n_dir] int32: entry j of row b is the block holding
 *              logical pages [j << block_shift, (j + 1) << block_shift) of
 *              sequence b, or -1 where the sequence has no pages
 *  page_blocks (dev) [n_blocks, 1 << block_shift] int32: physical page ids
 *
 * Logical page p of sequence b is physical page
 *   page_blocks[page_dir[b, p >> block_shift], p & ((1 << block_shift) - 1)],
 * and the map holds n_dir << block_shift logical pages per sequence (the
 * capacity that stands for max_pages).  Blocks are allocated only for the
 * page ranges sequences use, so the metadata grows with the pages in use, not
 * with B x the longest sequence.  A directory entry outside [0, n_blocks) for
 * a page below ceil(seq_lens[b] / P) is reported as a physical id outside the
 * pool (SA_DEVERR_POOL_RANGE) and that page is skipped, as a bad id of a flat
 * table is.  0 <= block_shift <= 16, (n_dir << block_shift) <= 2^30.
 *
 * Every *_dir entry point computes exactly what its flat counterpart computes
 * on the table this map defines (same kernels, same bits): arguments and
 * errors as that counterpart, with (page_dir, n_dir, page_blocks, n_blocks,
 * block_shift) in place of (page_table, max_pages).  sa_sparse_step_dir takes
 * the workspace sa_sparse_step_workspace_size gives for max_pages = n_dir <<
 * block_shift.
 */
SA_API int sa_build_page_summaries_dir(const uint16_t* k_cache, const int64_t k_strides[4],
                                       const int32_t* page_dir, int n_dir,
                                       const int32_t* page_blocks, int n_blocks, int block_shift,
                                       const int32_t* seq_lens, int B, int Hkv, int Dk,
                                       int page_size, int P_pool, uint16_t* summaries,
                                       int32_t* dev_error, void* stream);
SA_API int sa_sparse_step_dir(const uint16_t* q, const int64_t q_strides[4],
                              const uint16_t* summaries, const uint16_t* k_cache,
                              const int64_t k_strides[4], const uint16_t* v_cache,
                              const int64_t v_strides[4], const int32_t* page_dir, int n_dir,
                              const int32_t* page_blocks, int n_blocks, int block_shift,
                              const int32_t* seq_lens, int B, int T, int Hq, int Hkv, int D,
                              int page_size, int P_pool, int sink_tokens, int local_tokens,
                              int budget_tokens, float scale, int n_splits, int32_t* out_pages,
                              int32_t* out_counts, float* o_out, uint16_t* o_out_bf16,
                              float* lse_out, void* workspace, size_t workspace_bytes,
                              int32_t* dev_error, void* stream);
SA_API int sa_append_kv_dir(const uint16_t* k_new, const int64_t kn_strides[4],
                            const uint16_t* v_new, const int64_t vn_strides[4],
                            const int32_t* n_new, int max_new, uint16_t* k_cache,
                            const int64_t k_strides[4], uint16_t* v_cache,
                            const int64_t v_strides[4], const int32_t* page_dir, int n_dir,
                            const int32_t* page_blocks, int n_blocks, int block_shift,
                            const int32_t* seq_lens, int32_t* out_seq_lens, int B, int Hkv,
                            int D, int page_size, int P_pool, uint16_t* summaries,
                            int32_t* dev_error, void* stream);

/*
 * sa_block_union — per-group KV block tables for chunked prefill.
 * For head h and Q-block j the block mask is the sink blocks [0, n_sink),
 * the diagonal block d = q_block_offset + j, and the top_k blocks of
 * [n_sink, d) by (score desc, index asc).  Table g = the ascending union of
 * the masks of every head of group g (h / (Hq/Hkv) == g) over all Q-blocks.
 *
 *  scores (dev) [Hq,NQB,NKB] float32 (finite)
 *  tables (dev) [Hkv,NKB] int32: ascending block ids, then -1 padding
 *  counts (dev) [Hkv] int32
 * Requires q_block_offset + NQB <= NKB.
 */
SA_API int sa_block_union(const float* scores, int Hq, int Hkv, int NQB, int NKB, int q_block_offset,
                   int top_k, int n_sink_blocks, int32_t* tables, int32_t* counts,
                   void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SA_H_ */
