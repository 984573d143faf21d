/*
 * diffqkv.h -- C ABI of libdiffqkv.so: DiffQKV attention for NVIDIA B200 (sm_100a).
 *
 * DiffQKV attention ("Sigma: Differential Rescaling of Query, Key and Value
 * for Efficient Language Models", structured summary page, section 3.4
 * "DiffQKV Attention: Generalized Formulation") lets the K and V sides of a
 * KV cache have different head counts (n_k != n_v) and head dims
 * (d_k != d_v).  Under GroupSharing (same section, Step 3; and "FlexHeadFA
 * Kernel and Deployment Infrastructure", address calculation) query head h
 * reads K head h / (n_q / n_k) and V head h / (n_q / n_v).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors are dense, row-major, bf16 unless stated; pointers are DEVICE
 *    pointers unless stated and must be 16-byte aligned.
 *  - The caller owns every buffer.  The library never allocates or frees
 *    device memory and keeps no per-call state; the only library-wide state is
 *    cached device attributes, a per-device error word for the calls that have
 *    no word of their own (see below), and the built-in scratch array of
 *    diffqkv_decode_noalloc.
 *  - Every call is asynchronous on the caller's stream (NULL = legacy default
 *    stream) and never synchronises, except the two status reads
 *    (diffqkv_workspace_status, diffqkv_get_device_status).
 *  - Every call returns a diffqkv_status_t.  Argument errors are detected on
 *    the host before anything is launched or copied; nothing crosses the ABI
 *    as an exception.  Conditions only the device can see (a seq_len outside
 *    [0, t_max], a block-table entry outside the pool, a bounded wait that ran
 *    out) are recorded, first error wins, in the call's device error word:
 *      - calls that take a workspace (decode, its variants, top-v): the
 *        workspace's first 32-bit word, read and cleared by
 *        diffqkv_workspace_status;
 *      - diffqkv_prefill_causal_ex, diffqkv_prefill_causal_paged,
 *        diffqkv_augq_project: the word the caller passes (NULL: the
 *        per-device word);
 *      - every other call (prefill without a word, diffqkv_decode_noalloc,
 *        the wait self-test): the per-device word, read and cleared by
 *        diffqkv_get_device_status.
 *    So calls on different workspaces (different streams, different host
 *    threads) report independently, and reading one word clears no other.
 *  - Supported shapes: n_q % n_k == 0, n_q % n_v == 0 (else INVALID_ARG);
 *    n_q / n_k in {1, 2, 4, 8, 16} and d_k, d_v in {64, 128} (else
 *    UNSUPPORTED).
 */
#ifndef DIFFQKV_H_
#define DIFFQKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; NULL selects the legacy default stream. */
typedef struct CUstream_st *diffqkv_stream_t;

/* Attention shape.  scale multiplies q.k before the softmax (1/sqrt(d_k) in
 * the paper's Attend step, section 3.4 Step 4). */
typedef struct {
    int32_t batch; /* B >= 1 */
    int32_t n_q;   /* query heads */
    int32_t n_k;   /* K heads (n_q % n_k == 0) */
    int32_t n_v;   /* V heads (n_q % n_v == 0) */
    int32_t d_k;   /* K (and q) head dim */
    int32_t d_v;   /* V (and output) head dim */
    float scale;   /* > 0, finite */
} diffqkv_dims_t;

typedef enum {
    DIFFQKV_OK = 0,
    DIFFQKV_ERR_INVALID_ARG = 1,    /* bad dims, null pointer, bad size */
    DIFFQKV_ERR_UNSUPPORTED = 2,    /* legal shape this build has no kernel for */
    DIFFQKV_ERR_MISALIGNED = 3,     /* a pointer is not 16-byte aligned */
    DIFFQKV_ERR_WORKSPACE = 4,      /* workspace null or smaller than required */
    DIFFQKV_ERR_CUDA = 5,           /* a CUDA runtime call or launch failed */
    DIFFQKV_ERR_DEVICE_TIMEOUT = 6, /* a bounded device-side wait ran out */
    DIFFQKV_ERR_DEVICE_SEQLEN = 7,  /* a device seq_len was < 0 or > t_max (clamped) */
    DIFFQKV_ERR_NO_DEVICE = 8,      /* no CUDA device / driver */
    DIFFQKV_ERR_SCRATCH_LIMIT = 9,  /* shape needs more than the built-in scratch of diffqkv_decode_noalloc */
    DIFFQKV_ERR_DEVICE_PAGE = 10,   /* a block-table entry a paged call used was outside [0, num_pages) */
    DIFFQKV_ERR_DEVICE_BOUNDS = 11  /* a device-side index check failed (checked build only; the access
                                       was skipped) */
} diffqkv_status_t;

/* Human-readable name of a status code (static storage; never NULL). */
const char *diffqkv_status_string(int32_t status);

/* Library ABI version: major * 10000 + minor * 100 + patch. */
int32_t diffqkv_version(void);

/* ------------------------------------------------------------------------ */
/* Split/combine decode (FlexHeadFA's split kernel + combine kernel, section */
/* "FlexHeadFA Kernel and Deployment Infrastructure"; Steps 2-5 of 3.4).    */
/* ------------------------------------------------------------------------ */

/* Bytes of workspace diffqkv_decode needs for this shape (0 if dims are
 * invalid).  Depends only on the dims, not on the device or the lengths.
 * The workspace must be zero-filled before its FIRST use (cudaMemset, or
 * diffqkv_workspace_init); every call that completes leaves it zero-filled
 * again (its error word aside, which keeps the first device-side error until
 * diffqkv_workspace_status reads it), so it can be reused without clearing.
 * Two calls that may run concurrently must not share a workspace.  Layout: a
 * 256-byte header whose first 32-bit word is the error word, then one counter
 * per (batch, K head), then the split partials. */
size_t diffqkv_decode_workspace_size(const diffqkv_dims_t *dims);

/* Zero-fill a workspace on `stream` (cudaMemsetAsync). */
diffqkv_status_t diffqkv_workspace_init(void *workspace, size_t workspace_bytes,
                                        diffqkv_stream_t stream);

/*
 * Decode attention of one query token per sequence over a KV cache.
 *
 *   q        [B, n_q, d_k]          query (already projected and rotated)
 *   k_cache  [B, t_max, n_k, d_k]   K cache, token-major
 *   v_cache  [B, t_max, n_v, d_v]   V cache, token-major, separate from K
 *   seq_lens [B] int32 (device)     positions 0..seq_lens[b]-1 are attended
 *   out      [B, n_q, d_v]          bf16 output (written, never read)
 *
 * out[b,h] = sum_j softmax_j(scale * q[b,h].k_cache[b,j,h/(n_q/n_k)])
 *                   * v_cache[b,j,h/(n_q/n_v)],  j < seq_lens[b].
 * A row with seq_lens[b] == 0 is written as zeros.  seq_lens[b] < 0 or
 * > t_max is clamped into [0, t_max] and flagged DIFFQKV_ERR_DEVICE_SEQLEN in
 * the workspace's error word.
 * max_seq_len is a host-side upper bound of seq_lens (used only to size the
 * grid; a wrong hint costs speed, never correctness); pass t_max if unknown.
 * Each KV chunk produces (running max, sum of exp, unnormalised output)
 * partials and the combine merges them; both run in ONE kernel launch.
 */
diffqkv_status_t diffqkv_decode(const diffqkv_dims_t *dims, const void *q, const void *k_cache,
                                const void *v_cache, const int32_t *seq_lens, int32_t t_max,
                                int32_t max_seq_len, void *out, void *workspace,
                                size_t workspace_bytes, diffqkv_stream_t stream);

/*
 * Decode step with the KV-cache append fused in (the KV-cache store step of
 * the paper's deployment section, "FlexHeadFA Kernel and Deployment
 * Infrastructure", done inside the decode launch):
 *
 *   k_new    [B, n_k, d_k]   the step's new K rows (bf16, device, 16-byte aligned)
 *   v_new    [B, n_v, d_v]   the step's new V rows
 *   seq_lens [B] int32       cached positions BEFORE this step (p_b)
 *
 * Writes k_new[b] into k_cache[b, p_b] and v_new[b] into v_cache[b, p_b], and
 * out[b,h] = attention of q[b,h] over positions 0..p_b of the updated caches
 * (p_b + 1 positions).  seq_lens is not modified: the caller advances it.
 * Other arguments, layouts and the workspace are those of diffqkv_decode.  A
 * row with p_b >= t_max (no free slot) or p_b < 0 is flagged
 * DIFFQKV_ERR_DEVICE_SEQLEN; with p_b >= t_max nothing is written to its
 * caches and its output covers the t_max cached positions only.
 */
diffqkv_status_t diffqkv_decode_append(const diffqkv_dims_t *dims, const void *q, const void *k_new,
                                       const void *v_new, void *k_cache, void *v_cache,
                                       const int32_t *seq_lens, int32_t t_max, int32_t max_seq_len,
                                       void *out, void *workspace, size_t workspace_bytes,
                                       diffqkv_stream_t stream);

/*
 * Decode over PAGED K/V caches.  The pages compare DiffQKV with paged
 * attention, which manages K and V as one interchangeable cache ("Where
 * Existing Approaches Fall Short", system-level optimisations); here K and V
 * keep separate pools whose rows differ in size (n_k*d_k against n_v*d_v)
 * and share one block table:
 *
 *   k_pages     [num_pages, page_size, n_k, d_k]   K page pool (bf16, device)
 *   v_pages     [num_pages, page_size, n_v, d_v]   V page pool
 *   block_table [B, max_blocks] int32 (device)     pool page of each logical page
 *
 * Position j of sequence b is row j % page_size of pool page
 * block_table[b, j / page_size].  The logical capacity per sequence is
 * t_max = max_blocks * page_size (must fit in int32); seq_lens, q, out,
 * max_seq_len and the workspace are those of diffqkv_decode with that t_max
 * (the workspace size does not depend on t_max).  With k_new and v_new
 * NULL the call is diffqkv_decode over the paged caches; with both given it
 * is diffqkv_decode_append: position p_b = seq_lens[b] is written into its
 * page (block_table[b, p_b / page_size] must then name a pool page).
 * Only the entries of pages holding positions < seq_lens[b] (and p_b in
 * append mode) are read; others may hold anything.  A read entry outside
 * [0, num_pages) is flagged DIFFQKV_ERR_DEVICE_PAGE: pool page 0 is read in
 * its place and an append into it writes nothing.  Any page_size >= 1 is
 * accepted; a tile of the contiguous kernel is loaded as gcd(tile height,
 * page_size)-position pieces, so page sizes sharing a factor of 8 or 16 with
 * the tile height load fastest.  block_table must be 4-byte aligned, the
 * other pointers 16-byte aligned.  Pages may be shared between sequences
 * for reading; two sequences appending into one page row is a caller error.
 */
diffqkv_status_t diffqkv_decode_paged(const diffqkv_dims_t *dims, const void *q, const void *k_new,
                                      const void *v_new, void *k_pages, void *v_pages,
                                      const int32_t *block_table, int32_t max_blocks, int32_t page_size,
                                      int32_t num_pages, const int32_t *seq_lens, int32_t max_seq_len,
                                      void *out, void *workspace, size_t workspace_bytes,
                                      diffqkv_stream_t stream);

/*
 * Query and key of different widths (section 3.4 Step 4, the Attend
 * function): the pages bring each cached K row to the query width d_q with a
 * feed-forward layer, k_up = W k, before the dot product.  For a linear layer
 * without bias, <q, W k> = <W^T q, k>, so this call folds W into the query
 * instead and the attention entry points run unchanged on the result:
 *
 *   q_aug [dims->batch, n_q, d_q]     augmented query (bf16, device)
 *   w_up  [w_heads, d_q, d_k]         W of each K head (w_heads == n_k), or one
 *                                     W shared by all K heads (w_heads == 1)
 *   q_out [dims->batch, n_q, d_k]     q_out[b,h] = W[h/(n_q/n_k)]^T q_aug[b,h]
 *
 * Accumulation is fp32 and q_out is rounded to bf16 (nearest even).  Any
 * number of query rows works (a prefill's [B, S] rows pass as B*S batch
 * rows); the kernel runs on the CUDA cores and is sized for decode batches.
 * dims->scale, n_v and d_v are not used (they must still be valid dims);
 * the attention call that follows takes the scale of the d_q-wide dot product
 * (1/sqrt(d_q) for the pages' formula).  d_k in {64, 128}, d_q >= 8 and a
 * multiple of 8, w_heads in {1, n_k} (else DIFFQKV_ERR_INVALID_ARG /
 * DIFFQKV_ERR_UNSUPPORTED); pointers 16-byte aligned.  Asynchronous on
 * `stream`.
 */
diffqkv_status_t diffqkv_fold_query(const diffqkv_dims_t *dims, int32_t d_q, int32_t w_heads, const void *q_aug,
                                    const void *w_up, void *q_out, diffqkv_stream_t stream);

/*
 * Augmented query projection (section 3.2 "Big-Picture Architecture", item 4:
 * augmented Q with SwiGLU gating).  The query comes from a gated projection of
 * the hidden state whose parameters are never cached:
 *
 *   h = SiLU(x W_gate^T) * (x W_up^T)     SiLU(g) = g / (1 + e^-g), elementwise product
 *   q = h W_down^T
 *
 *   x      [tokens, d_model]     hidden states (bf16, device)
 *   w_gate [d_inter, d_model]    q_gate weights, one row per output feature
 *   w_up   [d_inter, d_model]    q_up weights
 *   w_down [d_out, d_inter]      q_down weights
 *   h_out  [tokens, d_inter]     the gated hidden state (written; bf16)
 *   q_out  [tokens, d_out]       the query (written; bf16), e.g. [tokens, n_q, d_q]
 *
 * Two tcgen05 GEMM launches on `stream`, fp32 accumulation; h is rounded to
 * bf16 (nearest even) before the second, q once at the end.  When the
 * attention uses query heads wider than the keys (diffqkv_fold_query), the
 * fold is linear and composes with q_down offline: per head, W_down's rows for
 * that head multiplied by W^T give a W_down of d_k-wide heads, and this call
 * then yields the folded query directly.
 * d_model a multiple of 64, d_inter a multiple of 128, d_out a multiple of 32
 * (else DIFFQKV_ERR_UNSUPPORTED); tokens >= 0 (0: nothing is launched, and
 * x, h_out and q_out may be NULL);
 * tokens * max(d_model, d_inter, d_out) < 2^31.  Pointers 16-byte aligned.
 * device_status_word as in diffqkv_prefill_causal_ex (NULL: the per-device
 * word); it receives DIFFQKV_ERR_DEVICE_TIMEOUT if a bounded wait runs out.
 */
diffqkv_status_t diffqkv_augq_project(const void *x, const void *w_gate, const void *w_up, const void *w_down,
                                      int32_t tokens, int32_t d_model, int32_t d_inter, int32_t d_out,
                                      void *h_out, void *q_out, int32_t *device_status_word,
                                      diffqkv_stream_t stream);

/* Optional launch controls for diffqkv_decode_ex (0 = library default). */
typedef struct {
    int32_t grid_ctas;   /* CTAs of the split kernel (>= 1); changes the split points */
    int32_t stages;      /* shared-memory pipeline depth (2..8) */
    int32_t ctas_per_sm; /* resident CTAs per SM the default grid assumes (1..4) */
} diffqkv_decode_tuning_t;

/* diffqkv_decode with explicit launch controls (tuning may be NULL).  The
 * result does not depend on the controls beyond fp32 rounding order. */
diffqkv_status_t diffqkv_decode_ex(const diffqkv_dims_t *dims, const void *q, const void *k_cache,
                                   const void *v_cache, const int32_t *seq_lens, int32_t t_max,
                                   int32_t max_seq_len, void *out, void *workspace,
                                   size_t workspace_bytes, const diffqkv_decode_tuning_t *tuning,
                                   diffqkv_stream_t stream);

/* Host-side launch plan of diffqkv_decode (no device needed; num_sms is the
 * SM count to plan for).  Returns INVALID_ARG / UNSUPPORTED like the call. */
typedef struct {
    int32_t tile_tokens;     /* cached positions per pipeline stage */
    int32_t stages;          /* pipeline depth */
    int32_t grid_ctas;       /* split-kernel CTAs */
    int32_t threads;         /* threads per CTA */
    int32_t v_heads_per_tile;/* V heads one K-head group reads */
    int64_t smem_bytes;      /* dynamic shared memory per CTA */
    int64_t workspace_bytes; /* == diffqkv_decode_workspace_size */
} diffqkv_decode_plan_t;

diffqkv_status_t diffqkv_decode_plan(const diffqkv_dims_t *dims, int32_t t_max, int32_t max_seq_len,
                                     int32_t num_sms, const diffqkv_decode_tuning_t *tuning,
                                     diffqkv_decode_plan_t *plan);

/*
 * End-to-end decode from HOST buffers: copies q, k_cache, v_cache and
 * seq_lens (host pointers, ideally pinned) into the caller's device buffers
 * with one cudaMemcpyAsync each, runs diffqkv_decode, and copies the bf16
 * output back into out_host, all on `stream`.  The caller synchronises the
 * stream before reading out_host.  Device buffers follow diffqkv_decode's
 * layouts; host buffers the same layouts.  Every check of diffqkv_decode
 * (dims, null or misaligned device pointers, the workspace) runs before the
 * first copy is enqueued: an argument error returns with nothing queued.
 */
diffqkv_status_t diffqkv_decode_from_host(const diffqkv_dims_t *dims, const void *q_host,
                                          const void *k_cache_host, const void *v_cache_host,
                                          const int32_t *seq_lens_host, int32_t t_max,
                                          int32_t max_seq_len, void *out_host, void *q_dev,
                                          void *k_cache_dev, void *v_cache_dev,
                                          int32_t *seq_lens_dev, void *out_dev, void *workspace,
                                          size_t workspace_bytes, diffqkv_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Selective V fetch decode ("Selective V Cache Fetching": only the V rows  */
/* of the top-k scoring positions are read; the softmax is renormalised    */
/* over them).                                                              */
/* ------------------------------------------------------------------------ */

/* Workspace bytes for diffqkv_decode_topv (0 if invalid).  Zero-fill it
 * before its first use (diffqkv_workspace_init); every call that completes
 * leaves it reusable without clearing (its error word aside, which keeps the
 * first device-side error until diffqkv_workspace_status reads it).  After a
 * call that reported DIFFQKV_ERR_DEVICE_TIMEOUT, zero-fill it again.  Layout,
 * with R = batch * n_q rows and U = batch * n_k (batch, K head) units, each
 * region starting on a 256-byte boundary:
 *   - a 256-byte header whose first 32-bit word is the error word;
 *   - the counters, kept zero between calls: U x 4 uint32, R x 4 uint32, and
 *     an R x 2048 uint32 histogram;
 *   - scratch written before it is read within a call.
 * Two calls that may run concurrently must not share a workspace. */
size_t diffqkv_decode_topv_workspace_size(const diffqkv_dims_t *dims, int32_t t_max, int32_t topk);

/*
 * Per (b, h): S = the topk positions j < seq_lens[b] with the largest EXACT
 * dot product q[b,h].k_cache[b,j,kh] (exact rational value, not a rounded
 * one), ties broken toward the lower j; all positions if topk >= seq_lens[b].
 *   out[b,h]     = sum_{j in S} e^{s_j - m} v[b,j,vh] / sum_{j in S} e^{s_j - m},
 *                  s_j = scale * q.k_j, m = max_{j in S} s_j   (bf16 [B,n_q,d_v])
 *   idx_out[b,h] = S in ascending order, padded with -1          (int32 [B,n_q,topk])
 * Only the selected V rows are read from v_cache.  Inputs and layouts as
 * diffqkv_decode.  topk >= 1 (any size; topk >= seq_lens[b] keeps every
 * position).  1 <= t_max <= 131072, else DIFFQKV_ERR_UNSUPPORTED (t_max >
 * 131072) or DIFFQKV_ERR_INVALID_ARG.  idx_out must be 4-byte aligned, the
 * other buffers and the workspace 16-byte aligned (DIFFQKV_ERR_MISALIGNED).
 * max_seq_len is accepted for symmetry with diffqkv_decode and ignored: the
 * kernels read the lengths from seq_lens on the device.  Lengths outside
 * [0, t_max] are clamped to that range and flagged
 * DIFFQKV_ERR_DEVICE_SEQLEN in the workspace's error word, as
 * diffqkv_decode does.  A row with length 0 gets a zero output and an all -1
 * index row.  One cooperative kernel launch on `stream` (its CTAs wait on
 * one another, with bounded waits, so the grid is sized to be resident at
 * once: one CTA per SM); returns once it is queued.
 */
diffqkv_status_t diffqkv_decode_topv(const diffqkv_dims_t *dims, const void *q, const void *k_cache,
                                     const void *v_cache, const int32_t *seq_lens, int32_t t_max,
                                     int32_t max_seq_len, int32_t topk, void *out,
                                     int32_t *idx_out, void *workspace, size_t workspace_bytes,
                                     diffqkv_stream_t stream);

/* Flags of diffqkv_decode_topv_ex. */
#define DIFFQKV_TOPV_FULL_SOFTMAX_WEIGHTS 1 /* weight the kept V rows by the full-softmax
                                               alpha_j of every cached position (the pages'
                                               formula: the others count as zero) instead of
                                               renormalising over the kept set */

/*
 * diffqkv_decode_topv with flags (0 = diffqkv_decode_topv).  With
 * DIFFQKV_TOPV_FULL_SOFTMAX_WEIGHTS:
 *   out[b,h] = sum_{j in S} e^{s_j - M} v[b,j,vh] / sum_{j < seq_lens[b]} e^{s_j - M},
 *   M = max over every cached position; S and idx_out are unchanged.
 * Other bits: DIFFQKV_ERR_INVALID_ARG.  Same workspace as diffqkv_decode_topv.
 */
diffqkv_status_t diffqkv_decode_topv_ex(const diffqkv_dims_t *dims, const void *q, const void *k_cache,
                                        const void *v_cache, const int32_t *seq_lens, int32_t t_max,
                                        int32_t max_seq_len, int32_t topk, int32_t flags, void *out,
                                        int32_t *idx_out, void *workspace, size_t workspace_bytes,
                                        diffqkv_stream_t stream);

/*
 * Selective V fetch over PAGED K/V caches: diffqkv_decode_topv_ex with the
 * K and V page pools and block table of diffqkv_decode_paged
 * ("Selective V Cache Fetching" over the separate per-position K and V
 * caches of section 3.4 Step 2, kept in pages):
 *
 *   k_pages     [num_pages, page_size, n_k, d_k]   K page pool (bf16, device)
 *   v_pages     [num_pages, page_size, n_v, d_v]   V page pool
 *   block_table [B, max_blocks] int32 (device)     pool page of each logical page
 *
 * Position j of sequence b is row j % page_size of pool page
 * block_table[b, j / page_size]; t_max = max_blocks * page_size <= 131072.
 * Selection, index output, weights (flags), lengths and the workspace
 * (diffqkv_decode_topv_workspace_size with that t_max) are those of
 * diffqkv_decode_topv_ex; for the same cached rows the results are those
 * of the contiguous call, bit for bit.  page_size must be a multiple of 8
 * (a K tile is loaded as gcd(120, page_size)-position pieces, each inside one
 * page, into 8-row swizzle atoms), else DIFFQKV_ERR_UNSUPPORTED.  Only the
 * entries of pages holding positions < seq_lens[b] are read; a read entry
 * outside [0, num_pages) is flagged DIFFQKV_ERR_DEVICE_PAGE and pool page 0
 * read in its place.  block_table must be 4-byte aligned.
 */
diffqkv_status_t diffqkv_decode_topv_paged(const diffqkv_dims_t *dims, const void *q, const void *k_pages,
                                           const void *v_pages, const int32_t *block_table, int32_t max_blocks,
                                           int32_t page_size, int32_t num_pages, const int32_t *seq_lens,
                                           int32_t max_seq_len, int32_t topk, int32_t flags, void *out,
                                           int32_t *idx_out, void *workspace, size_t workspace_bytes,
                                           diffqkv_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Causal prefill (the "prefix" phase the paper's efficiency study times)    */
/* ------------------------------------------------------------------------ */

/*
 *   q   [B, S, n_q, d_k], k [B, S, n_k, d_k], v [B, S, n_v, d_v]   bf16
 *   out [B, S, n_q, d_v]                                           bf16
 * out[b,i,h] = sum_{j<=i} softmax_j(scale * q[b,i,h].k[b,j,kh]) v[b,j,vh].
 * Runs on the tcgen05 tensor cores (TMEM accumulators, TMA-fed tiles).
 * Requires S >= 1; d_k = 64 or 128, d_v = 64 or 128.
 */
diffqkv_status_t diffqkv_prefill_causal(const diffqkv_dims_t *dims, const void *q, const void *k,
                                        const void *v, int32_t seq_len, void *out,
                                        diffqkv_stream_t stream);

/*
 * Causal prefill over an existing prefix (chunked prefill): the seq_len query
 * rows sit at positions prefix_len .. prefix_len + seq_len - 1 of a sequence
 * whose first prefix_len positions are already in k and v.
 *   q   [B, seq_len, n_q, d_k]                 the new rows' queries
 *   k   [B, prefix_len + seq_len, n_k, d_k]    prefix and new keys
 *   v   [B, prefix_len + seq_len, n_v, d_v]
 *   out [B, seq_len, n_q, d_v]
 * out[b,r,h] = sum_{j <= prefix_len + r} softmax_j(scale q[b,r,h].k[b,j,kh]) v[b,j,vh].
 * prefix_len >= 0 (0 is diffqkv_prefill_causal); other rules as there.
 */
diffqkv_status_t diffqkv_prefill_causal_prefix(const diffqkv_dims_t *dims, const void *q, const void *k,
                                               const void *v, int32_t prefix_len, int32_t seq_len, void *out,
                                               diffqkv_stream_t stream);

/*
 * diffqkv_prefill_causal_prefix with the call's own device error word:
 * device_status_word (int32, device memory, 4-byte aligned, zero before the
 * call) receives the first device-side error of this call (a bounded wait
 * that ran out) instead of the per-device word; NULL selects the per-device
 * word.  The caller reads it like any device memory after synchronising.
 */
diffqkv_status_t diffqkv_prefill_causal_ex(const diffqkv_dims_t *dims, const void *q, const void *k,
                                           const void *v, int32_t prefix_len, int32_t seq_len, void *out,
                                           int32_t *device_status_word, diffqkv_stream_t stream);

/*
 * diffqkv_prefill_causal_ex over paged K/V pools (chunked prefill whose prefix
 * sits in a paged cache, the layout of diffqkv_decode_paged):
 *   q        [B, seq_len, n_q, d_k]                  the new rows' queries
 *   k_pages  [num_pages, page_size, n_k, d_k]        K pool
 *   v_pages  [num_pages, page_size, n_v, d_v]        V pool
 *   block_table [B, max_blocks] int32 (device): position j of sequence b is
 *            row j % page_size of pool page block_table[b][j / page_size]
 *   out      [B, seq_len, n_q, d_v]
 * Every sequence holds prefix_len + seq_len positions, the new rows' k and v
 * included (written into their pages by the caller beforehand); query row r
 * sits at position prefix_len + r and attends to positions 0 .. prefix_len + r.
 * Only the first ceil((prefix_len + seq_len) / page_size) table entries of a
 * sequence are read; an entry outside [0, num_pages) is flagged
 * DIFFQKV_ERR_DEVICE_PAGE in the call's word and pool page 0 is read instead.
 * page_size a multiple of 8 (else DIFFQKV_ERR_UNSUPPORTED); max_blocks *
 * page_size >= prefix_len + seq_len (else DIFFQKV_ERR_INVALID_ARG); the table
 * 4-byte aligned.  The result equals diffqkv_prefill_causal_ex on contiguous
 * caches holding the same rows, bit for bit.  device_status_word as there.
 */
diffqkv_status_t diffqkv_prefill_causal_paged(const diffqkv_dims_t *dims, const void *q, const void *k_pages,
                                              const void *v_pages, const int32_t *block_table, int32_t max_blocks,
                                              int32_t page_size, int32_t num_pages, int32_t prefix_len,
                                              int32_t seq_len, void *out, int32_t *device_status_word,
                                              diffqkv_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Device error word                                                        */
/* ------------------------------------------------------------------------ */

/* Synchronises `stream`, returns (in *device_status) the first device-side
 * error recorded in the workspace's error word since the last read
 * (DIFFQKV_OK if none), and clears that word only.  For the workspaces of
 * diffqkv_decode (and its variants) and diffqkv_decode_topv; workspace_bytes
 * >= 256, 16-byte aligned.  The return value reports failures of the query. */
diffqkv_status_t diffqkv_workspace_status(void *workspace, size_t workspace_bytes, diffqkv_stream_t stream,
                                          int32_t *device_status);

/* Synchronises `stream`, returns (in *device_status) the first device-side
 * error recorded in the current device's word since the last read (DIFFQKV_OK
 * if none), and clears it.  Only calls without a word of their own report
 * there: diffqkv_prefill_causal / _prefix (and _ex given NULL),
 * diffqkv_decode_noalloc and diffqkv_selftest_wait_timeout.  The return value
 * reports failures of the query. */
diffqkv_status_t diffqkv_get_device_status(diffqkv_stream_t stream, int32_t *device_status);

/* Launches a kernel that waits on a barrier nothing ever signals, with a
 * bounded wait of `timeout_ns`, so callers can check that a wait that runs
 * out ends with DIFFQKV_ERR_DEVICE_TIMEOUT in the device error word instead
 * of a hang.  1e3 <= timeout_ns <= 5e9. */
diffqkv_status_t diffqkv_selftest_wait_timeout(int64_t timeout_ns, diffqkv_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Allocation-free decode (no counterpart in the paper)                      */
/* ------------------------------------------------------------------------ */

/* Size of the scratch buffer built into the library for diffqkv_decode_noalloc.
 * Every GPU that loads the library holds this much device memory until the
 * process exits. */
#define DIFFQKV_NOALLOC_SCRATCH_BYTES (8u << 20) /* 8 MiB */

/*
 * diffqkv_decode without a workspace argument, for callers that cannot hand
 * the library device memory: plugin interfaces whose enqueue step receives
 * only input and output buffers, and servers that forbid device allocation
 * after start-up (cudaMalloc synchronises the device and carves up a pool the
 * caller has already reserved).  The split partials and per-unit counters live
 * in a static device array of DIFFQKV_NOALLOC_SCRATCH_BYTES inside the
 * library instead; the call allocates and frees nothing.
 *
 * Arguments, layouts and results are those of diffqkv_decode.
 * - A shape whose scratch (split partials for batch * n_k units plus one
 *   per CTA, and batch * n_k counters) exceeds the array returns
 *   DIFFQKV_ERR_SCRATCH_LIMIT before anything is launched.  With the paper's
 *   decode shape (n_q 16, n_k 4, n_v 16, d_v 128) on a 148-SM B200 that
 *   allows batch <= 954.
 * - The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current) and caches it; make that
 *   first call before any stream capture on the device.
 * - Every call uses the same array, which keeps whatever the last call left
 *   there; each call clears the counters on `stream` before its kernel.
 *   Calls whose execution can overlap on the GPU (different streams, or
 *   concurrent host threads) race on the array and give wrong results:
 *   serialise them.
 */
diffqkv_status_t diffqkv_decode_noalloc(const diffqkv_dims_t *dims, const void *q, const void *k_cache,
                                        const void *v_cache, const int32_t *seq_lens, int32_t t_max,
                                        int32_t max_seq_len, void *out, diffqkv_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DIFFQKV_H_ */
