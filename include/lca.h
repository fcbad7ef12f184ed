/*
 * lca.h -- C ABI of liblca.so: the Latent-Condensed Attention (LCA) decode
 * step and the dense multi-head latent attention (MLA) decode it condenses,
 * on NVIDIA B200 (sm_100a).
 *
 * The operation is the one described in "Latent-Condensed Transformer for
 * Efficient Long Context Modeling" (gist.science summary of arXiv
 * 2604.12452), section 2 "Metodologia: Atencao Condensada Latente (LCA)",
 * "O Algoritmo LCA", steps 1-3.  For one query token per sequence b and
 * every head h, with scores s_t = q_c.c_t + q_r.k_t over the cached latents
 * c_t (C_KV) and RoPE keys k_t (K_R), t in [0, L):
 *
 *   step 1  n_G = floor((L - w) / g) groups G_j = [j g, (j+1) g) from token 0
 *           (0 when L <= w); the window W = [n_G g, L) -- the last w tokens
 *           plus the (L - w) mod g leftovers -- stays uncompressed;
 *   step 2  per group: pooling weights w_t = softmax_{t in G_j}(s_t) and the
 *           anchor a_j = the lowest index t in G_j with the largest s_t;
 *           the condensed entry is (c_bar_j = sum_t w_t c_t, k_{a_j});
 *   step 3  out = softmax attention of the query over [condensed || window]
 *           with value = latent:  logits S_j = q_c.c_bar_j + q_r.k_{a_j} and
 *           s_t (t in W); out = sum_e softmax(logit)_e value_e.
 *
 * No parameter is added (section 2, "Vantagens Teoricas"): there is no bias
 * and no internal scale; fold the softmax scale into q_c and q_r.  The
 * condensation is per head.  Dense MLA decode (section 1, "O Problema") is
 * out = sum_t softmax(s)_t c_t over all L tokens.
 *
 * All entry points are plain C: no exceptions cross them and none aborts.
 * Device entry points are asynchronous on the given stream; argument errors
 * are reported synchronously, before anything is launched or written.
 */
#ifndef LCA_H_
#define LCA_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LCA_OK = 0,
    LCA_ERR_INVALID_ARG = 1,     /* null pointer, g < 1, w < 0, L < 1, L > max_L, bad option */
    LCA_ERR_UNSUPPORTED = 2,     /* shape / dtype / group size with no kernel */
    LCA_ERR_ALIGNMENT = 3,       /* a device pointer not 16-byte aligned */
    LCA_ERR_CUDA = 4,            /* a CUDA runtime call or launch failed */
    LCA_ERR_DEVICE_TIMEOUT = 5,  /* a bounded wait inside a kernel ran out (see lca_get_device_error) */
    LCA_ERR_PLAN_MISMATCH = 6,   /* the plan was made for another shape / dtype / device */
    LCA_ERR_NO_MEMORY = 7,       /* device or host allocation failed */
    LCA_ERR_DEVICE_CHECK = 8,    /* debug build only: a kernel index failed its range check and the
                                    access was skipped (see lca_get_device_error) */
    LCA_ERR_DEVICE_INPUT = 9     /* lca_decode_paged: a length or block-table entry read on the
                                    device was out of range (see lca_get_device_error) */
} lca_status;

typedef enum { LCA_F32 = 0, LCA_BF16 = 1 } lca_dtype;

/* Opaque plan: shapes, kernel choice, split schedule and device workspace. */
typedef struct lca_plan lca_plan;

/*
 * Make a plan for batch B, H heads, latent width d_c, RoPE width d_r, element
 * type dt, and contexts up to max_L tokens, on the current CUDA device.
 * Allocates the plan's device workspace (split partials and the device
 * error word) once; no later call allocates device memory, except the first
 * lca_decode_host call (its staging buffers).
 * Kernels: bf16 with (d_c, d_r) = (512, 64) runs a tcgen05/TMA kernel -- the
 * two-CTA kernel when H is a multiple of 128 and g <= 64, else the 16-head
 * kernel when H is a multiple of 16; every other shape with d_c <= 1024,
 * d_r <= 256 and H <= 4096 runs the CUDA-core kernel (fp32 accumulation).
 * Errors: LCA_ERR_INVALID_ARG (null out_plan, non-positive sizes),
 * LCA_ERR_UNSUPPORTED, LCA_ERR_NO_MEMORY, LCA_ERR_CUDA.  *out_plan is
 * written only on LCA_OK; the caller frees it with lca_plan_destroy.
 */
lca_status lca_plan_create(int B, int H, int d_c, int d_r, lca_dtype dt, int64_t max_L,
                           lca_plan **out_plan);

/* Free a plan and its workspace.  NULL is accepted.  Call it only after every
 * launch that used the plan has finished. */
lca_status lca_plan_destroy(lca_plan *plan);

/* Plan options (lca_plan_set); values are int64. */
typedef enum {
    LCA_OPT_FORCE_SIMT = 1,        /* 1: use the CUDA-core kernel even where tcgen05 applies */
    LCA_OPT_NUM_CTAS = 2,          /* 1..SM count: CTAs of the tcgen05 kernel; 0: the SM count */
    LCA_OPT_WAIT_TIMEOUT_NS = 3,   /* bound of every in-kernel wait (default 2e9 ns) */
    LCA_OPT_DEBUG_SKIP_LOAD = 4,   /* 1: the tcgen05 producer skips its first load, so the
                                      consumer's bounded wait runs out (tests the timeout path) */
    LCA_OPT_KERNEL = 5             /* 0: automatic; else the lca_plan_kernel code to use
                                      (1 CUDA-core, 2 tcgen05, 3 tcgen05 two-CTA); a call whose
                                      shape that kernel cannot take returns LCA_ERR_UNSUPPORTED */
} lca_option;

lca_status lca_plan_set(lca_plan *plan, lca_option opt, int64_t value);

/*
 * LCA decode (steps 1-3 above) for all B sequences at context length L.
 *   q_c        [B][H][d_c]  device, plan dtype, row-major, 16-byte aligned
 *   q_r        [B][H][d_r]  device, plan dtype
 *   c_kv       [B][L][d_c]  device, plan dtype (the cache holds exactly L rows
 *                           per sequence: sequence b starts at b*L*d_c)
 *   k_r        [B][L][d_r]  device, plan dtype
 *   L          context length, 1 <= L <= max_L, the same for every sequence;
 *              the current token is the last cached row
 *   g, w       group size (>= 1) and window (>= 0); the tcgen05 kernel takes
 *              g in {1, 2, 4, ..., 128}, the CUDA-core kernel g <= 1024
 *   out        [B][H][d_c]  device float32, written
 *   anchor_idx [B][H][n_G]  device int32, absolute token positions in [0, L);
 *              may be NULL only when n_G == lca_num_groups(L, g, w) == 0
 *   stream     a cudaStream_t (NULL = legacy default stream)
 * The caller owns every buffer; nothing is retained after the call.  One
 * plan must not be used by two streams at once (the workspace is shared).
 * The tcgen05 path needs B * L < 2^31 cache rows (its TMA row coordinates
 * are 32-bit) and returns LCA_ERR_UNSUPPORTED otherwise.
 * The tcgen05 path launches two kernels, the main kernel and the split
 * combine, both as programmatic dependents of what precedes them in the
 * stream: each waits (griddepcontrol.wait) for the previous kernel to
 * complete before its first global-memory access, so only their prologues
 * overlap it.
 */
lca_status lca_decode(lca_plan *plan, const void *q_c, const void *q_r, const void *c_kv,
                      const void *k_r, int64_t L, int g, int w, float *out, int32_t *anchor_idx,
                      void *stream);

/*
 * Dense MLA decode: out[b][h] = sum_t softmax_t(q_c.c_t + q_r.k_t) c_t over all
 * L tokens (section 1 of the page: the cost LCA condenses).  Same layouts,
 * ownership and errors as lca_decode; no anchors.
 */
lca_status mla_decode(lca_plan *plan, const void *q_c, const void *q_r, const void *c_kv,
                      const void *k_r, int64_t L, float *out, void *stream);

/*
 * lca_decode with HOST buffers (same shapes): copies the inputs host->device
 * into plan-owned staging (allocated on the first call), runs lca_decode on
 * `stream`, copies out/anchor_idx back and synchronises the stream before
 * returning.  Pinned host memory gives full copy bandwidth.
 */
lca_status lca_decode_host(lca_plan *plan, const void *h_q_c, const void *h_q_r,
                           const void *h_c_kv, const void *h_k_r, int64_t L, int g, int w,
                           float *h_out, int32_t *h_anchor_idx, void *stream);

/*
 * Stored, head-shared condensed cache ("Latent-Condensed Transformer for
 * Efficient Long Context Modeling", section 4, "Eficiencia": the 128K KV cache
 * shrinks by ~90% and decode is faster because condensed groups are kept
 * instead of their tokens).  A group is condensed once, with the query of the
 * step that condenses it, and the entry serves every head.  The page does not
 * say how heads are combined; here the pooling weights and the anchor come
 * from the mean over heads of the scores (equal to the score of the mean
 * query):  s_bar_t = (1/H) sum_h (q_c^h . c_t + q_r^h . k_t),  w_t =
 * softmax over the group of s_bar_t,  a_j = the lowest index with the largest
 * s_bar_t,  entry j = (c_bar_j = sum w_t c_t, k_{a_j}).
 */

/*
 * Condense groups j0 .. j0+n-1 of every sequence (tokens [j g, j g + g), all
 * below L) with the head-mean score of q_c [B][H][d_c], q_r [B][H][d_r].
 *   c_kv [B][L][d_c], k_r [B][L][d_r]   device, plan dtype (the cache to condense)
 *   c_dst, k_dst  device, plan dtype: entry jj of sequence b is written to row
 *                 b * dst_rows + dst_row0 + jj of a [B][dst_rows][d_c] / [d_r] buffer
 *                 (c_bar_j rounded to the plan dtype; k_{a_j} copied as stored)
 *   anchor   [B][n] device int32: a_j, absolute positions (may be NULL when n == 0)
 * For condensing on eviction (a group leaving the window) or at prefill.
 * Errors: LCA_ERR_INVALID_ARG (null pointers, (j0 + n) g > L, L > max_L,
 * dst_row0 + n > dst_rows), LCA_ERR_PLAN_MISMATCH, LCA_ERR_CUDA.  Asynchronous
 * on `stream`; allocates nothing.
 */
lca_status lca_condense(lca_plan *plan, const void *q_c, const void *q_r, const void *c_kv,
                        const void *k_r, int64_t L, int g, int64_t j0, int64_t n, void *c_dst,
                        void *k_dst, int64_t dst_rows, int64_t dst_row0, int32_t *anchor,
                        void *stream);

/* Rows of the stored cache lca_build_stored writes for (L, g, w): n_G + (L - n_G g);
 * -1 if g < 1, w < 0 or L < 1. */
int64_t lca_stored_rows(int64_t L, int g, int w);

/*
 * Build the stored cache of every sequence from a full cache at context
 * length L (prefill): rows [0, n_G) of c_store [B][R][d_c] / k_store [B][R][d_r]
 * (R = lca_stored_rows(L, g, w)) are the condensed groups of section 2 step 1
 * (lca_condense with j0 = 0, n = n_G), rows [n_G, R) a copy of the window
 * tokens [n_G g, L).  anchor [B][n_G] int32 (NULL allowed when n_G == 0).
 * All pointers 16-byte aligned (else LCA_ERR_ALIGNMENT).  Asynchronous.
 */
lca_status lca_build_stored(lca_plan *plan, const void *q_c, const void *q_r, const void *c_kv,
                            const void *k_r, int64_t L, int g, int w, void *c_store,
                            void *k_store, int32_t *anchor, void *stream);

/*
 * Decode over a stored cache: softmax attention of every head of (q_c, q_r)
 * over the n_rows rows of c_store [B][n_rows][d_c] / k_store [B][n_rows][d_r]
 * (value = latent), with `bias` added to the logits of rows [0, n_cond) (the
 * condensed entries; log(g) counts an entry as the g tokens it stands for, 0
 * adds nothing -- the page names no bias).  out [B][H][d_c] float32.  The rows
 * may be in any order (attention is a sum over them); n_rows <= max_L.  Same
 * kernels, layouts and errors as mla_decode; reads (n_rows / L) of the bytes
 * a full-cache decode reads.
 */
lca_status lca_decode_stored(lca_plan *plan, const void *q_c, const void *q_r,
                             const void *c_store, const void *k_store, int64_t n_rows,
                             int64_t n_cond, float bias, float *out, void *stream);

/*
 * Context sharding.  The entries of one decode ([condensed groups || window]
 * over a context of L tokens) can be split by position among several holders
 * -- one slice of tokens [pos0, pos0 + n_tok) each (for example one GPU each),
 * cut on multiples of g inside the condensed part [0, n_G g) -- which compute
 * partial softmax sums over the entries they hold; the partials merge exactly
 * by the online-softmax merge (the merge of per-host softmax statistics of
 * "Pulsar Attention", Fase 2):  M = max_i M_i,
 *   out = sum_i e^{M_i - M} O_i / sum_i e^{M_i - M} Z_i.
 */

/* Condensed groups inside tokens [pos0, pos0 + n_tok) of a context of L tokens;
 * -1 if the slice cuts a group (or is out of range / g < 1 / w < 0). */
int64_t lca_slice_groups(int64_t L, int g, int w, int64_t pos0, int64_t n_tok);

/*
 * Partial decode over one slice:
 *   c_slice [B][n_tok][d_c], k_slice [B][n_tok][d_r]  device, plan dtype: tokens
 *            [pos0, pos0 + n_tok) of each sequence (n_tok <= max_L; 0 allowed)
 *   L, g, w  the whole context's length, group size and window
 *   part_mz  [B][H][2] float32, written: (M, Z) per head -- the largest logit of
 *            the slice's entries (-inf for an empty slice) and sum_e e^{logit_e - M}
 *   part_o   [B][H][d_c] float32, written: sum_e e^{logit_e - M} value_e
 *   anchor   [B][H][lca_slice_groups(...)] int32, absolute positions (NULL when 0)
 * Same kernels as lca_decode.  Errors: LCA_ERR_INVALID_ARG (a cut group among
 * them), LCA_ERR_UNSUPPORTED, LCA_ERR_ALIGNMENT, LCA_ERR_CUDA.  Asynchronous.
 */
lca_status lca_decode_partial(lca_plan *plan, const void *q_c, const void *q_r,
                              const void *c_slice, const void *k_slice, int64_t n_tok,
                              int64_t pos0, int64_t L, int g, int w, float *part_mz,
                              float *part_o, int32_t *anchor, void *stream);

/*
 * Merge n_parts partials stacked by part -- part_mz [n_parts][B][H][2],
 * part_o [n_parts][B][H][d_c] (device, float32, e.g. gathered from every
 * holder) -- into out [B][H][d_c] float32.  Asynchronous; allocates nothing.
 */
lca_status lca_merge_partials(lca_plan *plan, int n_parts, const float *part_mz,
                              const float *part_o, float *out, void *stream);

/* n_G for (L, g, w): floor((L - w) / g) when L > w, else 0; -1 if g < 1, w < 0 or L < 1. */
int64_t lca_num_groups(int64_t L, int g, int w);

/* Static text for a status code (never NULL). */
const char *lca_status_string(lca_status status);

/*
 * Synchronise `stream`, read and clear the plan's device error word.
 * Returns LCA_OK, LCA_ERR_DEVICE_CHECK when (in the range-checked debug build,
 * liblca_checked.so) a kernel index failed its check, LCA_ERR_DEVICE_TIMEOUT
 * when an in-kernel wait ran out (the kernel then skipped its remaining work
 * and left outputs undefined), LCA_ERR_DEVICE_INPUT when lca_decode_paged read
 * a length or block-table entry out of range, or LCA_ERR_CUDA when the
 * synchronisation itself failed.
 */
lca_status lca_get_device_error(lca_plan *plan, void *stream);

/*
 * The site of the last error that lca_get_device_error reported for this plan:
 * a code naming the wait that ran out (or, in the range-checked build, the
 * check that failed) inside the kernel, 0 if none was reported yet or for a
 * NULL plan.  Codes are fixed per wait site in the kernel sources (for
 * example 0x7xx for the O-MMA issuer of the two-CTA kernel).  Host only; no
 * CUDA call.
 */
int lca_get_device_error_site(const lca_plan *plan);

/*
 * Instrumentation for measuring the main kernel on its own: when `event` (a
 * cudaEvent_t) is non-NULL, each later lca_decode / mla_decode call records it
 * on the call's stream right after launching the main kernel and before
 * launching the split-combine kernel.  NULL turns it off.  The caller owns the
 * event.  Returns LCA_ERR_INVALID_ARG for a NULL plan.
 */
lca_status lca_plan_set_timing_event(lca_plan *plan, void *event);

/* Which kernel a plan runs for (L, g, w): 0 = none (invalid), 1 = CUDA-core, 2 = tcgen05
 * (16 heads per CTA), 3 = tcgen05 two-CTA (128 heads per cluster of two CTAs that split the
 * latent width; H a multiple of 128, g <= 64). */
int lca_plan_kernel(lca_plan *plan, int64_t L, int g, int w);

/*
 * LCA decode for grouped-query attention (GQA): one query token per sequence,
 * H query heads sharing n_kv_heads key/value heads (query head h reads KV head
 * h / (H / n_kv_heads)).  Section 2 ("Condensacao Dual-Path") pools the
 * semantic component and anchors the positional (RoPE) one; section 3, item 3
 * extends the method to GQA.  In a GQA cache the key carries the position and
 * the value the content, so per query head and per group G_j (the section-2
 * segmentation, n_G = floor((L - w) / g)):
 *   s_t = q . k_t;  w_t = softmax over G_j of s_t;  a_j = lowest-index argmax;
 *   condensed entry: key k_{a_j} (logit s_{a_j}), value sum_t w_t v_t;
 * window tokens stand for themselves; out = softmax attention over
 * [condensed || window].  This equals lca_decode's operation with q_c = 0,
 * C_KV = V and K_R = K per KV head.
 * The plan is made with B, H = query heads, d_c = d_v (value width) and
 * d_r = d_k (key width), max_L >= L.
 *   q        device [B][H][d_k]; k_cache device [B][L][n_kv_heads][d_k] (keys with
 *            RoPE applied); v_cache device [B][L][n_kv_heads][d_v]
 *   out      device fp32 [B][H][d_v];  anchor device int32 [B][H][n_G] (NULL allowed
 *            only when n_G = 0)
 * Runs a CUDA-core kernel with fp32 accumulation (one CTA per context split, KV
 * head and sequence, serving the KV head's query heads).  Needs
 * H / n_kv_heads <= 16, d_k <= 256, d_v a power of two in [32, 256], and g a
 * power of two <= 64 when there are groups (LCA_ERR_UNSUPPORTED otherwise).
 * Errors: LCA_ERR_INVALID_ARG (null pointers, L outside [1, max_L], g < 1, w < 0,
 * n_kv_heads < 1 or not dividing H, NULL anchor with groups), LCA_ERR_ALIGNMENT
 * (q, caches, out or anchor not 16-byte aligned), LCA_ERR_PLAN_MISMATCH,
 * LCA_ERR_UNSUPPORTED, LCA_ERR_CUDA.
 */
lca_status lca_decode_gqa(lca_plan *plan, const void *q, const void *k_cache, const void *v_cache,
                          int64_t L, int n_kv_heads, int g, int w, float *out, int32_t *anchor,
                          void *stream);

/*
 * LCA decode of a paged, variable-length batch: the caches of the B sequences
 * sit in pages of one pool, each sequence has its own length, and each is
 * decoded exactly as lca_decode decodes a contiguous cache of that length --
 * its own n_G(b) = floor((L_b - w) / g) groups (0 when L_b <= w) and its own
 * window (section 2, "O Algoritmo LCA", steps 1-3).  The page has no paged
 * layout: this is the serving form of the same step (several sequences of
 * different lengths in one call, caches grown a page at a time, pages shared
 * between sequences with a common prefix).
 *   q_c, q_r     device [B][H][d_c], [B][H][d_r] (the plan's B, H, dtype)
 *   c_pool       device [num_pages * page_size][d_c]; k_pool [.. ][d_r]
 *   page_size    rows per page, a positive multiple of 64
 *   block_table  device int32 [B][max_pages]: sequence b's token t is row
 *                block_table[b max_pages + t / page_size] page_size + t % page_size
 *                of the pools.  Entries past a sequence's last page are never read.
 *   seq_lens     device int32 [B]: L_b, 1 <= L_b <= min(max_L, max_pages page_size)
 *   out          device fp32 [B][H][d_c]
 *   anchor       device int32 [B][H][anchor_stride], a_j of (b, h) at
 *                (b H + h) anchor_stride + j for j < n_G(b); may be NULL only when no
 *                length up to min(max_L, max_pages page_size) has a group
 * Lengths and table entries stay on the device (no host synchronisation; the
 * call can be captured in a CUDA graph).  A length outside its range, or with
 * n_G(b) > anchor_stride, leaves that sequence's output NaN and its anchors
 * unwritten; a used table entry outside [0, num_pages) is read as page 0.
 * Either raises LCA_ERR_DEVICE_INPUT from the next lca_get_device_error.
 * Pool rows that hold no token of a sequence may hold anything, NaN included.
 * The kernels and their precision are lca_decode's for the plan's shape.
 * Errors (synchronous): LCA_ERR_INVALID_ARG (null pointers, page_size not a
 * positive multiple of 64, num_pages or max_pages < 1, g < 1, w < 0, a NULL
 * anchor where groups are possible), LCA_ERR_UNSUPPORTED (num_pages page_size
 * > 2^31 - 1, or no kernel), LCA_ERR_ALIGNMENT (q, pools, out, anchor not
 * 16-byte aligned; table or lengths not 4-byte aligned), LCA_ERR_PLAN_MISMATCH,
 * LCA_ERR_CUDA.
 */
lca_status lca_decode_paged(lca_plan *plan, const void *q_c, const void *q_r, const void *c_pool,
                            const void *k_pool, int64_t num_pages, int page_size,
                            const int32_t *block_table, int64_t max_pages, const int32_t *seq_lens,
                            int g, int w, float *out, int32_t *anchor, int64_t anchor_stride,
                            void *stream);

/*
 * LCA prefill of a chunk of queries of one sequence, each with per-query
 * condensation: the plan's B queries sit at positions pos0, pos0 + 1, ...,
 * pos0 + B - 1 of one sequence whose cache is paged through one block-table
 * row, and query i attends causally to tokens [0, pos0 + i] -- its own
 * n_G = floor((pos0 + i + 1 - w) / g) groups and its own window (section 2,
 * "O Algoritmo LCA", steps 1-3, applied at every position of the prompt; the
 * summary's prefill figures in section 4 speak of the same condensed
 * attention during the prefill).  The tokens of the chunk itself must already
 * be in the cache.  Query i's result is lca_decode_paged's for a sequence of
 * length pos0 + i + 1 with that block-table row, which is how it runs: the
 * same kernels, the lengths formed on the device from pos0, every query
 * reading the one row.
 *   q_c, q_r         device [B][H][d_c], [B][H][d_r]: query i of the chunk in row i
 *   c_pool, k_pool,
 *   num_pages,
 *   page_size        as for lca_decode_paged
 *   block_table_row  device int32 [max_pages]: the sequence's pages
 *   pos0             position of the chunk's first query; 0 <= pos0 and
 *                    pos0 + B <= min(max_L, max_pages page_size)
 *   out, anchor      as for lca_decode_paged ([B][H][d_c] and [B][H][anchor_stride])
 * Errors: LCA_ERR_INVALID_ARG (pos0 out of range, and as for lca_decode_paged);
 * the rest as for lca_decode_paged.
 */
lca_status lca_prefill_paged(lca_plan *plan, const void *q_c, const void *q_r, const void *c_pool,
                             const void *k_pool, int64_t num_pages, int page_size,
                             const int32_t *block_table_row, int64_t max_pages, int64_t pos0, int g,
                             int w, float *out, int32_t *anchor, int64_t anchor_stride, void *stream);

/*
 * lca_decode without a plan and without any allocation.  The page has no
 * counterpart: this is a deployment variant of lca_decode for callers that may
 * not allocate device memory when they decode (a server whose memory is all
 * reserved up front by its own pool, where a cudaMalloc would fail or
 * fragment it, and which cannot keep a plan per shape).
 * Arguments: B, H, d_c, d_r and dt as for lca_plan_create; the rest, their
 * layouts and ownership as for lca_decode (L has no max_L bound).  Same
 * kernels and results as lca_decode.
 * Scratch: the split partials live in one fixed file-scope device array of
 * 16 MiB of partial outputs plus 64 KiB of (max, sum) pairs, so the tile
 * ranges are capped to what both regions hold; shapes with
 * B * H * max(d_c, 512) > 4 Mi floats return LCA_ERR_UNSUPPORTED before
 * anything is launched.  The device error word in that array is cleared on
 * `stream` at the start of every call; a bounded in-kernel wait that runs out
 * leaves outputs undefined and is not reported by this call.
 * The first call on a device looks up the scratch's address there and sets
 * the kernels' shared-memory limit (thread-safe: concurrent first calls are
 * serialised); make that first call before any stream capture.  Every call on
 * a device shares the one scratch: calls that overlap on the GPU (two
 * streams, or two host threads) race and corrupt each other's results.
 * Errors: LCA_ERR_INVALID_ARG, LCA_ERR_UNSUPPORTED, LCA_ERR_ALIGNMENT,
 * LCA_ERR_CUDA.
 */
lca_status lca_decode_noalloc(int B, int H, int d_c, int d_r, lca_dtype dt, const void *q_c,
                              const void *q_r, const void *c_kv, const void *k_r, int64_t L, int g,
                              int w, float *out, int32_t *anchor_idx, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* LCA_H_ */
