/*
 * csa.h -- C ABI of libcsa.so: one decode step of combined sparse attention
 * (pinned prefix + sliding window + Quest-style top-k pages) for the
 * full-attention layers of hybrid LLMs, over a full-size paged bf16 GQA KV
 * cache, on NVIDIA B200 (sm_100a).
 *
 * What the operation is ("Accelerating Long-Context Decoding in Large-Scale
 * Hybrid LLMs Without Retraining", abstract; arxivlens analysis of the same
 * paper, "Methodology"; roboaidigest post, "The Move" and "Why It Matters"):
 * each query head of a full-attention layer attends to the union of
 *   - a pinned prefix: the first `prefix` tokens,
 *   - a sliding window: the last `window` tokens,
 *   - a fixed budget of the most relevant tokens, chosen query-aware as the
 *     top-k pages by the Quest upper-bound score
 *         s_h(p) = sum_i max(q_{h,i} * max_{p,i}, q_{h,i} * min_{p,i})
 *     where min/max are the per-page, per-channel key extremes,
 * and the KV cache itself stays full size, so any page can be selected.
 * Window and budget are per-layer arguments.
 *
 * Readings this library takes where the pages are silent:
 *   - page size is 16 tokens; k = floor(budget_tokens / 16) pages;
 *   - prefix and window are counted in tokens and applied token-exactly;
 *     a page is a top-k candidate unless all its valid tokens already lie in
 *     prefix or window; a selected page contributes all its valid tokens;
 *   - the score of a kv-head's page is the max over the G query heads of
 *     the group of the per-head bound (an upper bound for every head);
 *   - equal scores: the lower logical page index wins; the selected pages
 *     are returned in ascending page order;
 *   - softmax scale defaults to 1/sqrt(D); no soft-cap; q and k are taken
 *     after any positional encoding;
 *   - scores are unscaled (q.k, not q.k/sqrt(D)); the order is the same.
 *
 * ---------------------------------------------------------------- layouts
 * All tensors are row-major and contiguous; bf16 is IEEE bfloat16.
 *   q          bf16  [B][Hq][D]                 query of the step
 *   k_cache    bf16  [num_pages][Hkv][16][D]    keys, one page of one kv-head
 *   v_cache    bf16  [num_pages][Hkv][16][D]    is a contiguous 32*D-byte tile
 *   meta       bf16  [num_pages][Hkv][2][D]     row 0 = min, row 1 = max key
 *   page_table int32 [B][max_pages_per_seq]     logical page -> physical page
 *   seq_lens   int32 [B]                        valid tokens incl. this step's
 *   sel_pages  int32 [B][Hkv][max_sel]          selected logical pages
 *   n_sel      int32 [B][Hkv]
 *   out        bf16  [B][Hq][D]
 *   lse        fp32  [B][Hq]                    natural-log sum-exp of scale*q.k
 * Query head h reads kv-head h / (Hq/Hkv).  Token t of sequence b lives in
 * physical page page_table[b][t/16], slot t%16.
 *
 * ----------------------------------------------------------- conventions
 *  - Every pointer argument except the ones marked "host" is a DEVICE
 *    pointer owned by the caller; the library allocates no device memory.
 *  - Device pointers must be 16-byte aligned (CSA_ERR_INVALID_ARG if not).
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  All calls
 *    are asynchronous on it; the status code reports argument checks and
 *    launch errors only.  Calls sharing one workspace must not overlap.
 *  - Kernels are launched with programmatic dependent launch, so a kernel
 *    may start while the previous kernel on the stream finishes.  Each call
 *    waits for the preceding work before it reads anything, with two
 *    exceptions.  (1) csa_meta_update, csa_score_select and
 *    csa_sparse_attention read `page_table` and `seq_lens` early, and
 *    csa_decode / csa_decode_full read `page_table`, `seq_lens`, `sel_pages`
 *    and `n_sel` early (the dependency wait comes before the cache and the
 *    workspace): those inputs must not come from the kernel launched just
 *    before the call if that kernel releases its dependents early (a host
 *    copy, an event, a plain kernel or a call of this library is fine; the
 *    selections of csa_score_select and csa_select_scores count, see (2)).
 *    (2) When the previous call of this library on the same stream was
 *    csa_score_select or csa_select_scores, csa_decode / csa_decode_full
 *    stream the prefix and window pages while the selection kernel is still
 *    running and read the selection only after their wait: their `q`,
 *    `k_cache`, `v_cache`, `page_table` and `seq_lens` must not be written
 *    between the two calls.  The library remembers the last call per stream
 *    handle on the host; this is its only state outside the workspace.
 *  - Page ids that fall outside [0, num_pages), selected pages outside the
 *    candidate range, and a selection that is not strictly ascending are
 *    detected on the device: the page is skipped and a flag is latched in
 *    the workspace; csa_get_device_status() reports and clears it.  No
 *    kernel traps or spins without a bound.
 *  - Supported shapes: page_size == 16, D in {64, 128, 256},
 *    Hq/Hkv in {1, 2, 4, 8, 16}, B*Hkv <= 2048; else CSA_ERR_UNSUPPORTED.
 */
#ifndef CSA_H
#define CSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every entry point. */
enum {
    CSA_OK = 0,
    CSA_ERR_INVALID_ARG = -1, /* null/misaligned pointer, bad size or range  */
    CSA_ERR_UNSUPPORTED = -2, /* shape outside the supported set             */
    CSA_ERR_WORKSPACE = -3,   /* workspace missing or smaller than required  */
    CSA_ERR_CUDA = -4,        /* a CUDA runtime call or launch failed        */
    CSA_ERR_DEVICE_FLAG = -5  /* a kernel latched a device-side error flag   */
};

/* Bits of the device-side flag word (see csa_get_device_status). */
enum {
    CSA_DEVFLAG_BAD_PAGE_ID = 1,  /* page_table entry outside [0, num_pages)  */
    CSA_DEVFLAG_BAD_SELECTION = 2,/* sel_pages entry outside the candidates,
                                     not ascending, or n_sel out of range     */
    CSA_DEVFLAG_BAD_SEQ_LEN = 4,  /* seq_len < 0 or > 16 * max_pages_per_seq,
                                     or shorter than the appended chunk       */
    CSA_DEVFLAG_TIMEOUT = 8       /* a kernel's bounded wait for its own copies
                                     ran out (the fp8 scoring of 4 or 8
                                     kv-heads): that call's results are void */
};

/* Problem shape, passed by host pointer to every call. */
typedef struct csa_dims {
    int B;                 /* sequences in the batch                          */
    int Hq;                /* query heads                                     */
    int Hkv;               /* key/value heads (Hq % Hkv == 0)                 */
    int D;                 /* head dimension                                  */
    int page_size;         /* tokens per page; must be 16                     */
    int max_pages_per_seq; /* row length of page_table                        */
    int num_pages;         /* physical pages in k_cache / v_cache / meta      */
    int max_sel;           /* row length of sel_pages (>= budget_tokens / 16) */
} csa_dims;

/* Bytes of device workspace the calls below need for shape *d (host
 * pointer).  Returns 0 for an invalid or unsupported shape.  The workspace
 * holds the device flag word, per-(sequence, kv-head) bookkeeping, the fp32
 * page scores and the split-K partial results. */
size_t csa_workspace_size(const csa_dims *d);

/* Zero `bytes` of `workspace` on `stream`.  Required once before the first
 * call that uses a fresh workspace: the device flag word and the per-unit
 * key ranges that the scoring kernel merges with atomicMax must start at
 * zero (every selection leaves its ranges at zero again). */
int csa_workspace_init(void *workspace, size_t bytes, void *stream);

/*
 * Append tokens to the paged cache and keep the page metadata current
 * (the full-size cache of "Why It Matters"; the Quest per-page key min/max
 * used by the top-k selection of "Methodology").
 *
 * The last n_new tokens of each sequence, positions [seq_lens[b] - n_new,
 * seq_lens[b]), are the new ones.  new_k/new_v are bf16 [B][n_new][Hkv][D];
 * each new token is written to k_cache/v_cache at its page slot.  For every
 * page that holds a new token, meta is set to the elementwise min/max of
 * the page's valid keys: from the new keys alone when the page starts within
 * the new tokens, else from the stored min/max and the new keys (so the
 * stored metadata of the page's older tokens must be current).
 * new_k == NULL (and new_v == NULL) is the rebuild mode: nothing is
 * written to the cache, and meta is recomputed from k_cache for every page
 * that holds one of positions [max(0, seq_lens[b] - n_new), seq_lens[b]).
 * seq_lens already include the new tokens.  n_new >= 1 (in rebuild mode any
 * n_new >= max seq_len rebuilds everything).
 */
int csa_meta_update(const csa_dims *d, void *k_cache, void *v_cache, void *meta,
                    const int32_t *page_table, const int32_t *seq_lens,
                    const void *new_k, const void *new_v, int n_new,
                    void *workspace, size_t workspace_bytes, void *stream);

/*
 * Query-aware top-k page selection, Quest-style ("Methodology"; "The Move").
 *
 * For each (sequence b, kv-head g), with L = seq_lens[b], Pe = min(prefix, L)
 * and We = min(window, L), the candidates are the logical pages holding at
 * least one token of [Pe, L - We).  Each candidate gets the fp32 score
 *   s(p) = max over the G query heads h of group g of
 *          sum_i max(q_{h,i} * max_{p,i}, q_{h,i} * min_{p,i}),
 * reading only the page metadata.  The top k' = min(budget_tokens / 16,
 * #candidates) pages by (score descending, page ascending) are written to
 * sel_pages[b][g][0..k') in ascending page order and k' to n_sel[b][g].
 * scores_out (nullable) receives fp32 [B][Hkv][max_pages_per_seq] scores at
 * the candidate positions (other entries are left untouched).
 * budget_tokens / 16 must not exceed max_sel.
 */
int csa_score_select(const csa_dims *d, const void *q, const void *meta,
                     const int32_t *page_table, const int32_t *seq_lens,
                     int prefix, int window, int budget_tokens,
                     int32_t *sel_pages, int32_t *n_sel, float *scores_out,
                     void *workspace, size_t workspace_bytes, void *stream);

/*
 * Combined sparse attention decode ("Accelerating Long-Context Decoding ...",
 * abstract): for every query head h of sequence b (kv-head g = h / G),
 *   A = { t < L : t < Pe  or  t >= L - We  or  page t/16 in sel_pages[b][g] }
 *   out[b][h] = sum_{t in A} softmax_t(scale * q_h . k_t) v_t
 *   lse[b][h] = log sum_{t in A} exp(scale * q_h . k_t)
 * computed split-K across the GPU with an fp32 online softmax; the splits
 * are merged on the device.  An empty A gives out = 0 and lse = -inf.
 * sel_pages must be strictly ascending candidate pages (as csa_score_select
 * writes them).  scale <= 0 selects 1/sqrt(D).  lse is nullable.
 */
int csa_decode(const csa_dims *d, const void *q, const void *k_cache, const void *v_cache,
               const int32_t *page_table, const int32_t *seq_lens,
               const int32_t *sel_pages, const int32_t *n_sel, int prefix, int window,
               float scale, void *out, float *lse,
               void *workspace, size_t workspace_bytes, void *stream);

/*
 * Dense decode over every valid token: the unmodified full-attention layer
 * the pages compare against ("Results": every configuration is slower than
 * it at short context).  Same outputs and conventions as csa_decode with
 * A = { t < L }.
 */
int csa_decode_full(const csa_dims *d, const void *q, const void *k_cache,
                    const void *v_cache, const int32_t *page_table,
                    const int32_t *seq_lens, float scale, void *out, float *lse,
                    void *workspace, size_t workspace_bytes, void *stream);

/*
 * One call for the sparse part of a decode step: the Quest scoring and
 * top-k selection of csa_score_select followed by the attention of
 * csa_decode over the pages it selected (same arguments, meanings and
 * outputs: sel_pages and n_sel receive the selection, out and lse the
 * attention).  Up to 32 (sequence, kv-head) units with at least one page to
 * select run the selection and the decode of the selected pages in one
 * launch, the prefix and window pages being decoded meanwhile by other CTAs
 * of the same grid; other shapes run the separate kernels.  Reads
 * `page_table` and `seq_lens` early, like csa_score_select.
 */
int csa_sparse_attention(const csa_dims *d, const void *q, const void *k_cache,
                         const void *v_cache, const void *meta, const int32_t *page_table,
                         const int32_t *seq_lens, int prefix, int window, int budget_tokens,
                         float scale, int32_t *sel_pages, int32_t *n_sel, void *out,
                         float *lse, void *workspace, size_t workspace_bytes, void *stream);

/*
 * fp8 metadata (an option; the pages specify no metadata precision, and the
 * entry points above use the exact bf16 min/max).  meta8 is a lower-precision
 * copy of meta that the scoring reads instead, moving about half the bytes:
 *   meta8  uint8 [num_pages][Hkv][2*D + 16]
 * per (physical page, kv-head): D bytes of E4M3 (OCP FP8: bias 7, 3 mantissa
 * bits, largest value 448) for min * 2^-e rounded toward -inf, D bytes for
 * max * 2^-e rounded toward +inf, then a 16-byte trailer {int32 e, 0, 0, 0}.
 * e is the smallest integer with max |value| * 2^-e <= 448 over the two rows
 * (0 when they are all zero).  The decoded box [2^e min8, 2^e max8] contains
 * the exact one, so the Quest score from it is still an upper bound for every
 * head; it may be looser, so the selection can differ from the bf16 one.
 *
 * csa_meta_update_fp8: csa_meta_update, and the fp8 copy of every page whose
 *   metadata it writes (meta stays the exact master copy).
 * csa_score_select_fp8 / csa_sparse_attention_fp8: csa_score_select /
 *   csa_sparse_attention with the scores computed from meta8.
 */
int csa_meta_update_fp8(const csa_dims *d, void *k_cache, void *v_cache, void *meta,
                        void *meta8, const int32_t *page_table, const int32_t *seq_lens,
                        const void *new_k, const void *new_v, int n_new,
                        void *workspace, size_t workspace_bytes, void *stream);
int csa_score_select_fp8(const csa_dims *d, const void *q, const void *meta8,
                         const int32_t *page_table, const int32_t *seq_lens,
                         int prefix, int window, int budget_tokens,
                         int32_t *sel_pages, int32_t *n_sel, float *scores_out,
                         void *workspace, size_t workspace_bytes, void *stream);
int csa_sparse_attention_fp8(const csa_dims *d, const void *q, const void *k_cache,
                             const void *v_cache, const void *meta8,
                             const int32_t *page_table, const int32_t *seq_lens,
                             int prefix, int window, int budget_tokens, float scale,
                             int32_t *sel_pages, int32_t *n_sel, void *out, float *lse,
                             void *workspace, size_t workspace_bytes, void *stream);

/*
 * ------------------------------------------------- context parallelism
 * One layer's decode with every sequence's pages split over R ranks (each
 * rank holds the pages [page_lo, page_hi) of every sequence in its own
 * cache; rank 0 holds the prefix, the last rank the window), with one
 * exchange step: each rank scores its candidate pages (csa_score_select with
 * budget 0 and scores_out), the ranks all-gather the score arrays and
 * concatenate them along the page axis, every rank selects the global top-k
 * with csa_select_scores (the same pages csa_score_select would select on
 * one GPU), keeps its own pages with csa_shard_selection, attends over them
 * and its share of prefix/window with csa_decode, and the ranks all-gather
 * (out, lse) and merge them with csa_merge_attention.  The exact top-k of the
 * union is the top-k of the concatenated scores, and the attention over a
 * union of disjoint token sets is the log-sum-exp merge of the attentions
 * over the parts, so the result is the single-GPU one up to the bf16 rounding
 * of the parts' outputs.
 */

/*
 * Top-k page selection over caller-provided Quest scores: scores is fp32
 * [B][Hkv][max_pages_per_seq] (read only; entries outside each unit's
 * candidate range [c_lo, c_hi), as seq_lens, prefix and window define it,
 * are ignored), k = budget_tokens / 16, ties to the lower page, output
 * ascending, exactly as csa_score_select.  Uses the workspace of `d`.
 */
int csa_select_scores(const csa_dims *d, const float *scores, const int32_t *seq_lens,
                      int prefix, int window, int budget_tokens, int32_t *sel_pages,
                      int32_t *n_sel, void *workspace, size_t workspace_bytes, void *stream);

/*
 * The pages of a selection that fall in [page_lo, page_hi), as pages of the
 * shard: sel_local[b][g][j] = sel_pages[b][g][i] - page_lo for the selected
 * pages in range, in ascending order, and n_sel_local[b][g] their count.
 * sel_pages/n_sel as csa_score_select writes them for dims d (ascending,
 * n_sel <= d->max_sel); sel_local is int32 [B][Hkv][max_sel_local] with
 * max_sel_local >= d->max_sel (else CSA_ERR_INVALID_ARG).
 */
int csa_shard_selection(const csa_dims *d, const int32_t *sel_pages, const int32_t *n_sel,
                        int page_lo, int page_hi, int max_sel_local, int32_t *sel_local,
                        int32_t *n_sel_local, void *stream);

/*
 * Log-sum-exp merge of `parts` partial attention results over disjoint token
 * sets: out_parts bf16 [parts][batch][q_heads][head_dim], lse_parts fp32
 * [parts][batch][q_heads] (natural log; -inf for a part that attended no
 * token) -> out bf16 [batch][q_heads][head_dim] = sum_r e^(lse_r - lse)
 * out_r (fp32, rounded to nearest even) and lse fp32 [batch][q_heads] =
 * log sum_r e^(lse_r) (NULL to skip).  A head no part attended gets out 0 and
 * lse -inf.  head_dim is 64, 128 or 256; 1 <= parts <= 64.
 */
int csa_merge_attention(int parts, int batch, int q_heads, int head_dim, const void *out_parts,
                        const float *lse_parts, void *out, float *lse, void *stream);

/*
 * csa_decode for callers that cannot allocate device memory.  The paper has
 * no counterpart to this entry point; it exists for deployment: a plugin
 * hosted inside another runtime that owns every device buffer, or a server
 * that reserves all device memory at start-up and allows no allocation later,
 * has no way to provide the workspace csa_decode needs.
 *
 * Same arguments, results and conventions as csa_decode, minus the
 * workspace.  The split-K scratch lives in an 8 MiB __device__ array inside
 * the library (held on every GPU that loads it until the process exits).
 * The call allocates nothing (no cudaMalloc, cudaFree or allocating library
 * routine).  A shape whose scratch would exceed 8 MiB is rejected with
 * CSA_ERR_WORKSPACE; at D = 128, G = 8 on a 148-SM B200 that is about
 * 560 (sequence, kv-head) units while the decode grid stays at 444 CTAs.  The first call on a device looks up the
 * array's device address (make it before any stream capture).  The call
 * clears the array's flag word on `stream` before the kernels;
 * every call shares the array, so calls that overlap on the GPU race: keep
 * them on one stream or otherwise ordered.  Device-side flags of this call
 * are not reported (offending pages are still skipped).
 */
int csa_decode_noalloc(const csa_dims *d, const void *q, const void *k_cache,
                       const void *v_cache, const int32_t *page_table,
                       const int32_t *seq_lens, const int32_t *sel_pages,
                       const int32_t *n_sel, int prefix, int window, float scale,
                       void *out, float *lse, void *stream);

/*
 * Synchronise `stream`, read and clear the device flag word of `workspace`.
 * Returns CSA_OK when no flag was set, CSA_ERR_DEVICE_FLAG when one was (the
 * CSA_DEVFLAG_* bits go to *flags_out if it is not NULL), CSA_ERR_CUDA on a
 * CUDA error.
 */
int csa_get_device_status(void *workspace, void *stream, int *flags_out);

/* Static string for a status code (host). */
const char *csa_status_string(int status);

/* Library ABI version (major * 100 + minor): 102 (1.01 added the fp8-metadata
 * entry points, 1.02 the context-parallel ones). */
int csa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CSA_H */
