/*
 * gqla.h -- C ABI of libgqla: GQLA (Group-Query Latent Attention) decode
 * attention on NVIDIA B200 (sm_100a).
 *
 * GQLA indexes the latent up-projections W_UK and W_UV by g groups instead of
 * by the h_q query heads, so one set of weights exposes two algebraically
 * equivalent decoding paths (GQLA, paperlayer.ai summary of arXiv:2605.15250v3,
 * sec. 2 "Algebraically equivalent decoding paths" and sec. 3 "Two equivalent
 * decoding paths"; gist.science technical summary, sec. 2 "Architektur"):
 *
 *   MQA-absorb path  gqla_absorb_query -> gqla_decode_absorb -> gqla_combine
 *       W_UK is folded into the query, every head attends over the 576-element
 *       latent row [c (512) | k^R (64)], the value is the 512-d latent itself,
 *       and W_UV is applied after the split combine.
 *   GQA path         gqla_expand_cache (once) -> gqla_decode_gqa -> gqla_combine
 *       the cache is expanded once per group into K_nope = c W_UK_g and
 *       V = c W_UV_g (128 each) beside the shared RoPE key; h_q/g query heads
 *       share each group (pwwt.cn article, sec. 3 and sec. 5: 16 heads per group).
 *
 * Conventions for every call:
 *  - All tensor arguments are DEVICE pointers owned by the caller, dense,
 *    row-major, 16-byte aligned.  Nothing is allocated, freed or copied to
 *    the host, and no call synchronises: work is enqueued on `stream`
 *    (NULL = the legacy default stream) and the call returns.
 *  - bf16 means IEEE bfloat16 (2 bytes).  "h" is dims->num_heads, "g" is
 *    dims->num_groups, G = h/g heads per group; head hd belongs to group hd/G.
 *  - Token t of sequence b lives at pool slot page_table[b][t/page_size] *
 *    page_size + t % page_size.  The s_q query tokens of a step are already
 *    the last s_q cached tokens: query s sees tokens t <= seqlen - s_q + s.
 *  - Return value: GQLA_OK, or a negative gqla_status.  Argument errors are
 *    detected before anything is launched.  Errors found on the device (a
 *    page index outside the pool, a sequence longer than its page-table row,
 *    a bounded wait that ran out) never trap: the kernel skips the bad work,
 *    records the first error in the workspace, and gqla_read_device_error()
 *    returns it.
 *  - Calls on the same workspace must not overlap on the GPU.
 *
 * Supported shapes: d_latent 512, d_rope 64, d_nope 128, d_v 128, page_size
 * 64, s_q in {1, 2}, h % g == 0 with (h/g) * s_q <= 32, batch <= 65535.
 * Anything else returns GQLA_ERR_UNSUPPORTED.
 */
#ifndef GQLA_H_
#define GQLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st *gqla_stream_t;

typedef enum {
    GQLA_OK = 0,
    GQLA_ERR_INVALID_ARG = -1,  /* null pointer, negative size, inconsistent dims */
    GQLA_ERR_UNSUPPORTED = -2,  /* valid but not one of the supported shapes      */
    GQLA_ERR_WORKSPACE = -3,    /* workspace missing or smaller than required    */
    GQLA_ERR_CUDA = -4,         /* a CUDA runtime/driver call or launch failed   */
    GQLA_ERR_DEVICE = -5,       /* device-side check failed (bad page index ...) */
    GQLA_ERR_TIMEOUT = -6       /* a bounded device-side wait ran out            */
} gqla_status;

/* Layer dimensions.  softmax_scale is applied to q.k before the softmax; the
 * pages do not state it, the MLA convention 1/sqrt(d_nope + d_rope) =
 * 1/sqrt(192) is the expected value. */
typedef struct {
    int num_heads;       /* h_q: e.g. 128 (DeepSeek-V3 shape) or 32 (LLaMA-3-8B) */
    int num_groups;      /* g: 8, or 4 (the (g, s_q) = (4, 1) point); G*s_q <= 32,
                            G a multiple of 4                                      */
    int d_latent;        /* r_kv: 512                                              */
    int d_rope;          /* d_R: 64                                                */
    int d_nope;          /* per-head no-RoPE key width: 128                        */
    int d_v;             /* per-head value width: 128                              */
    float softmax_scale; /* 1/sqrt(d_nope + d_rope)                                */
} gqla_dims;

/* Paged KV index shared by both decode paths and the combine. */
typedef struct {
    const int32_t *page_table; /* device int32 [batch][max_pages_per_seq]           */
    const int32_t *seqlens;    /* device int32 [batch], cached tokens incl. the s_q new ones */
    int batch;                 /* number of sequences, 1..65535                      */
    int max_pages_per_seq;     /* row length of page_table                           */
    int page_size;             /* tokens per page: 64                                */
    int num_pages;             /* pages in the pool; a page index outside [0, num_pages) is a device error */
} gqla_kv_index;

/*
 * One-shot cache expansion for the GQA path (deploy-time, not per step:
 * pwwt.cn article, sec. 3; paperlayer.ai sec. 3 "Two equivalent decoding
 * paths", the one-shot cache expansion).
 *   latent       bf16 [num_slots][576]   rows [c | k^R]
 *   w_uk, w_uv   bf16 [g][512][128]
 *   kv_expanded  bf16 [g][num_slots][256] out: [c W_UK_g | c W_UV_g]
 *   k_rope       bf16 [num_slots][64]    out: k^R copied
 * Rounding contract: each output is accumulated in fp32 from +0.0 by one
 * fused multiply-add per latent index 0..511 in ascending order, then
 * rounded once to bf16 (nearest, ties to even).  Results are therefore
 * bit-reproducible by any implementation of that order.
 */
int gqla_expand_cache(const gqla_dims *dims, const void *latent, int64_t num_slots,
                      const void *w_uk, const void *w_uv, void *kv_expanded, void *k_rope,
                      gqla_stream_t stream);

/*
 * The same expansion on the tensor cores (tcgen05): identical arguments,
 * layouts, ownership and errors as gqla_expand_cache; each output is the
 * fp32 tensor-core accumulation of the same 512 exact bf16 x bf16 products in
 * the hardware's own order, rounded once to bf16 (nearest, ties to even).
 * Not bit-reproducible against gqla_expand_cache: every output x satisfies
 * |x - exact| <= 2^-8 |exact| + 2^-15 sum_k |c_k w_k| (the bf16 rounding plus
 * the fp32 accumulation bound for 512 terms); k_rope is copied exactly.
 */
int gqla_expand_cache_tc(const gqla_dims *dims, const void *latent, int64_t num_slots,
                         const void *w_uk, const void *w_uv, void *kv_expanded, void *k_rope,
                         gqla_stream_t stream);

/*
 * Query absorption: W_UK folded into the query (paperlayer.ai summary, sec. 2).
 *   q           bf16 [batch][s_q][h][192]  (0..127 q^C, 128..191 q^R, RoPE applied)
 *   w_uk        bf16 [g][512][128]
 *   q_absorbed  bf16 [batch][s_q][h][576]  out: [W_UK_{g(h)} q^C ; q^R], fp32 accumulation
 * All pointers 16-byte aligned.  Runs on the tensor cores; its device-side
 * waits are bounded, and one that runs out (a fault elsewhere) leaves
 * q_absorbed unwritten, since this call has no workspace to report into.
 */
int gqla_absorb_query(const gqla_dims *dims, const void *q, int batch, int s_q,
                      const void *w_uk, void *q_absorbed, gqla_stream_t stream);

/*
 * Split-KV partial attention, MQA-absorb path: every head scores its absorbed
 * query against the latent row and accumulates the 512-d latent (paperlayer.ai
 * summary, sec. 2 "Algebraically equivalent decoding paths" and sec. 4
 * Roofline Analysis, "MQA-absorb path": one 576-element latent row per token
 * shared by all heads).
 *   q_absorbed    bf16 [batch][s_q][h][576]
 *   latent_cache  bf16 [num_pages][page_size][576]
 *   kv            page table / lengths (kv->batch is the batch)
 *   num_splits    C >= 1: the batch's pages, concatenated sequence after
 *                 sequence, are cut into C equal chunks, one per CTA; a chunk
 *                 that meets sequence b yields one partial in slot (b + chunk).
 *   o_part  fp32 [gqla_partial_slots(batch, C)][s_q][h][512]  out, normalised per partial
 *   lse_part fp32 [gqla_partial_slots(batch, C)][s_q][h]      out, natural-log LSE of the
 *                 scaled scores (-inf for an empty partial); unused slots are not written
 *   workspace  >= gqla_workspace_bytes() bytes of device memory, zeroed once
 *              before first use (holds the device error record)
 * Precision: bf16 operands, every score and the online softmax in fp32 (the
 * two 288-column halves of a score, computed on the two CTAs of a pair, are
 * exchanged and added in fp32), P in bf16, O accumulated in fp32.
 */
int gqla_decode_absorb(const gqla_dims *dims, const void *q_absorbed, int s_q,
                       const void *latent_cache, const gqla_kv_index *kv, int num_splits,
                       float *o_part, float *lse_part, void *workspace, size_t workspace_bytes,
                       gqla_stream_t stream);

/*
 * gqla_decode_absorb with a lead in the split plan: of the num_splits chunks,
 * the first `lead_splits` are lead_weight16 / 16 times as long as the others
 * (k = ceil(16 T / (lead_splits * lead_weight16 + 16 (num_splits - lead_splits)))
 * pages for the others, ceil(k * lead_weight16 / 16) for the lead ones, cut in
 * that order; the last chunks may come out short or empty).  The partials go
 * to the same slots (b + chunk) and must be merged by gqla_combine_lead with the
 * same three numbers.  lead_splits 0 (or lead_weight16 16) is gqla_decode_absorb.
 * This is for a step that runs the GQA path beside the absorb path on another
 * stream (gqla_plan_lead picks the numbers): the CTAs of the short chunks finish
 * early and leave their SMs to the GQA decode, while the lead chunks keep busy
 * the SMs that the GQA decode does not use.  Launched before the GQA decode, and
 * with a lead the decode does not let the combine be scheduled before its last
 * CTA is done, so nothing waits on the SMs it frees.
 *   lead_splits    0 .. num_splits;  lead_weight16  16 .. 1024
 * Otherwise as gqla_decode_absorb (GQLA_ERR_INVALID_ARG for a lead out of range).
 */
int gqla_decode_absorb_lead(const gqla_dims *dims, const void *q_absorbed, int s_q,
                            const void *latent_cache, const gqla_kv_index *kv, int num_splits,
                            int lead_splits, int lead_weight16, float *o_part, float *lse_part,
                            void *workspace, size_t workspace_bytes, gqla_stream_t stream);

/*
 * Split-KV partial attention, GQA path: the G*s_q query rows of each group
 * score [K_nope_g | k^R] (192) and accumulate V_g (128) (paperlayer.ai
 * summary, sec. 3 "Two equivalent decoding paths" and sec. 4, "GQA path";
 * pwwt.cn article, sec. 5: h_q/g query heads share a group).
 *   q            bf16 [batch][s_q][h][192]
 *   kv_expanded  bf16 [g][num_slots][256], k_rope bf16 [num_slots][64]
 *                (as written by gqla_expand_cache; num_slots = num_pages * page_size)
 *   o_part  fp32 [gqla_partial_slots(batch, C)][s_q][h][128], lse_part as above.
 * g must be 8, 4, 2 or 1 (GQLA_ERR_UNSUPPORTED otherwise; 2 and 1 are a
 * rank's share of the groups under group-axis tensor parallelism).  Precision:
 * bf16 operands, scores and softmax in fp32, P in bf16, O in fp32.
 */
int gqla_decode_gqa(const gqla_dims *dims, const void *q, int s_q, const void *kv_expanded,
                    const void *k_rope, int64_t num_slots, const gqla_kv_index *kv,
                    int num_splits, float *o_part, float *lse_part, void *workspace,
                    size_t workspace_bytes, gqla_stream_t stream);

/*
 * The GQA-path step in one call: gqla_decode_gqa, then gqla_combine (d_in =
 * 128) for the sequences that need it.  A sequence whose pages all fall in one
 * of the C chunks has a single partial, which is its result: the decode writes
 * it straight to `out` / `lse_out` in the combine's format, and the combine
 * leaves it alone.  With C = 1 every sequence is such a sequence and no combine
 * is launched at all (the single-split fusion: one kernel for the step).
 *   arguments as for gqla_decode_gqa and gqla_combine; o_part / lse_part may
 *   be NULL when num_splits == 1 (then nothing is written there); out bf16
 *   [batch][s_q][h][128] (required), lse_out fp32 [batch][s_q][h] or NULL.
 * A sequence with no token gets out = 0 and lse = -inf, as from gqla_combine.
 */
int gqla_decode_gqa_step(const gqla_dims *dims, const void *q, int s_q, const void *kv_expanded,
                         const void *k_rope, int64_t num_slots, const gqla_kv_index *kv,
                         int num_splits, float *o_part, float *lse_part, void *out, float *lse_out,
                         void *workspace, size_t workspace_bytes, gqla_stream_t stream);

/*
 * Sparse GQLA, GQA path (paperlayer.ai summary, sec. 2 "Sparse GQLA";
 * pwwt.cn article, sec. 5): each query token (b, s) attends only to its own
 * selected token positions, the same set for all heads.  This call gathers
 * them into a compact "selected" cache on which gqla_decode_gqa and
 * gqla_combine then run unchanged, as batch * s_q sequences of one query
 * token each (q and out keep their [batch][s_q][h][...] layout).
 *   kv_expanded, k_rope, num_slots, kv   the GQA-path cache, as for gqla_decode_gqa
 *   s_q          1 or 2
 *   topk_idx     int32 [batch][s_q][topk] device: token positions, distinct
 *                within a list; -1 marks an unused entry.  A position outside
 *                [0, L_b - s_q + s] or on a page outside the pool is reported
 *                (GQLA_ERR_DEVICE, info = b * s_q + s) and skipped.
 *   topk         1 .. 65536; cap = topk rounded up to a multiple of 64
 *   kv_sel       bf16 [g][batch * s_q * cap][256]   out (rows past each list's
 *   k_rope_sel   bf16 [batch * s_q * cap][64]        out  valid entries untouched)
 *   sel_page_table int32 [batch * s_q][cap / 64]     out (identity)
 *   sel_seqlens  int32 [batch * s_q]                 out: valid entries per list
 *   workspace    as for the decode calls (device error record)
 * Then: gqla_decode_gqa(dims, q, 1, kv_sel, k_rope_sel, batch * s_q * cap,
 * {sel_page_table, sel_seqlens, batch * s_q, cap / 64, 64, batch * s_q * cap / 64}, ...)
 * and gqla_combine with the same index and s_q = 1.
 */
int gqla_sparse_gather(const gqla_dims *dims, const void *kv_expanded, const void *k_rope,
                       int64_t num_slots, const gqla_kv_index *kv, int s_q, const int32_t *topk_idx,
                       int topk, void *kv_sel, void *k_rope_sel, int32_t *sel_page_table,
                       int32_t *sel_seqlens, void *workspace, size_t workspace_bytes,
                       gqla_stream_t stream);

/*
 * Sparse GQLA without the selected cache (the fused path): the same selection
 * as gqla_sparse_gather, but only each selected row's cache slot is written,
 *   sel_slot      int32 [batch * s_q * cap]  out: cache slot of selected row
 *                 r of query token v at [v * cap + r]; -1 past the list's
 *                 valid entries
 * with sel_page_table / sel_seqlens as there (kv_expanded and k_rope are not
 * read: pass NULL).  gqla_decode_gqa_sparse then gathers the rows itself.
 */
int gqla_sparse_select(const gqla_dims *dims, const gqla_kv_index *kv, int s_q, const int32_t *topk_idx,
                       int topk, int32_t *sel_slot, int32_t *sel_page_table, int32_t *sel_seqlens,
                       void *workspace, size_t workspace_bytes, gqla_stream_t stream);

/*
 * GQA-path decode over a selection written by gqla_sparse_select: the split
 * partials of batch * s_q one-token queries, each over its own selected rows,
 * which the kernel gathers from the cache four at a time (TMA tile::gather4)
 * instead of reading page tiles.
 *   q            bf16 [batch][s_q][h][192] (as for gqla_decode_gqa)
 *   kv_expanded, k_rope, num_slots   the cache, as for gqla_decode_gqa
 *   sel          {sel_page_table, sel_seqlens, batch * s_q, cap / 64, 64,
 *                 batch * s_q * cap / 64}
 *   sel_slot     as written by gqla_sparse_select
 *   o_part, lse_part, workspace   as for gqla_decode_gqa with sel's batch
 * Then gqla_combine(dims, sel, 1, num_splits, 128, ...).
 */
int gqla_decode_gqa_sparse(const gqla_dims *dims, const void *q, int s_q, const void *kv_expanded,
                           const void *k_rope, int64_t num_slots, const gqla_kv_index *sel,
                           const int32_t *sel_slot, int num_splits, float *o_part, float *lse_part,
                           void *workspace, size_t workspace_bytes, gqla_stream_t stream);

/*
 * Log-sum-exp merge of the partials of each sequence, then (absorb path,
 * d_in == 512) the per-group up-projection out = o~ W_UV_{g(h)}: W_UV folded into
 * the output (paperlayer.ai summary, sec. 2).
 *   o_part / lse_part as written by a decode call with the same kv and num_splits
 *   d_in      512 (absorb partials; w_uv required) or 128 (GQA partials; w_uv NULL)
 *   out       bf16 [batch][s_q][h][128]
 *   lse_out   fp32 [batch][s_q][h] or NULL
 * o_part, out and w_uv 16-byte aligned.  A row with no visible token gets
 * out = 0 and lse = -inf.  For d_in == 512 the merged latent row is rounded
 * to bf16 (the tensor-core operand type) before the product with W_UV, which
 * accumulates in fp32.  Like gqla_absorb_query this call has no workspace: a
 * bounded device-side wait that runs out leaves `out` unwritten.
 * Launched right after the decode call that wrote the partials, the combine
 * reads kv->seqlens (and W_UV) while that decode is still finishing: the
 * lengths must be the ones the decode call used.
 */
int gqla_combine(const gqla_dims *dims, const gqla_kv_index *kv, int s_q, int num_splits,
                 int d_in, const float *o_part, const float *lse_part, const void *w_uv,
                 void *out, float *lse_out, gqla_stream_t stream);

/* gqla_combine for partials written by gqla_decode_absorb_lead: the same
 * lead_splits and lead_weight16 locate each sequence's partial slots.  d_in
 * 512 only when the lead is not empty (no GQA decode writes such partials):
 * d_in 128 with lead_splits > 0 and lead_weight16 != 16 is GQLA_ERR_INVALID_ARG. */
int gqla_combine_lead(const gqla_dims *dims, const gqla_kv_index *kv, int s_q, int num_splits,
                      int lead_splits, int lead_weight16, int d_in, const float *o_part,
                      const float *lse_part, const void *w_uv, void *out, float *lse_out,
                      gqla_stream_t stream);

/*
 * GQA-path decode step that allocates nothing: gqla_decode_gqa followed by
 * gqla_combine, with the split partials, their LSEs and the device error
 * record kept in a file-scope device array owned by the library.  The pages
 * have no counterpart of this call: it exists for callers that cannot
 * allocate device memory -- code under an allocator that forbids cudaMalloc
 * once serving has started, plugins that are handed only their input and
 * output buffers, or threads that must not call into an allocator on the
 * decode path -- and so cannot supply o_part / lse_part / workspace.
 *
 *   Inputs and outputs are those of gqla_decode_gqa and gqla_combine (GQA
 *   partials, d_in = 128): q, kv_expanded, k_rope, num_slots, kv, num_splits
 *   as there; out bf16 [batch][s_q][h][128], lse_out fp32 [batch][s_q][h] or
 *   NULL; device_error: NULL, or a device int32[2] that receives {status,
 *   info} of the device-side checks of this call (what gqla_read_device_error
 *   would return for an ordinary workspace).
 *   Limit: the partials of (batch + num_splits) * s_q * h rows, 516 bytes
 *   each (rounded up), plus 256 bytes must fit in GQLA_NOALLOC_SCRATCH_BYTES
 *   (32 MiB); larger requests return GQLA_ERR_WORKSPACE before any launch.
 *   When the array is claimed: under CUDA's default lazy module loading the
 *   32 MiB are taken on a device when the first call there looks up the
 *   array's device address (cudaGetSymbolAddress, with that device current),
 *   not when the library is loaded; from then on the device holds them until
 *   the process exits.  On a device whose memory is nearly all claimed later
 *   (by a serving allocator), that first call could fail with GQLA_ERR_CUDA:
 *   make it at start-up, before serving begins and before any stream capture.
 *   Nothing is allocated or freed by the later calls, nor by any library they
 *   use.
 *   Sharing: every call on a device uses the same array, which keeps the last
 *   call's contents (the error record is cleared at the start of each call).
 *   Calls that overlap on the GPU -- on different streams, or from different
 *   threads -- race on it and give undefined results; serialise them.
 */
#define GQLA_NOALLOC_SCRATCH_BYTES (32u << 20)
int gqla_decode_gqa_noalloc(const gqla_dims *dims, const void *q, int s_q, const void *kv_expanded,
                            const void *k_rope, int64_t num_slots, const gqla_kv_index *kv,
                            int num_splits, void *out, float *lse_out, int32_t *device_error,
                            gqla_stream_t stream);

/* Number of partial slots the decode calls address: batch + num_splits. */
int gqla_partial_slots(int batch, int num_splits);

/* Workspace bytes the decode calls need. */
size_t gqla_workspace_bytes(void);

/* A split count that fills the current device with one wave: the GQA decode
 * runs one CTA per split, the absorb decode a 2-CTA cluster per split and per
 * 128 query rows of a sequence (s_q * num_heads rows).  path 0 = absorb,
 * 1 = GQA.  Returns < 0 on error. */
int gqla_num_splits_hint(int path, int num_heads, int s_q);

/* Host-side choice of a split count for known sequence lengths.  Both decode
 * calls cut the batch's pages, concatenated sequence after sequence (T pages
 * in all), into chunks of k = ceil(T / num_splits) pages, one chunk per split;
 * a chunk that holds the end of one sequence and the start of the next runs a
 * second "piece" (its own partial output, epilogue and query), which costs a
 * split more than a page.  Among num_splits = 1 .. max_splits this returns the
 * one whose heaviest chunk, counted as its pages plus `piece_cost_pages` for
 * every sequence that starts inside it after its first page, is lightest (the
 * smallest such count on a tie).  Host-only: touches no device.
 *   seqlens           host int32[batch], each >= 0
 *   batch             1 .. 65535
 *   max_splits        1 .. 65535 (e.g. gqla_num_splits_hint's value)
 *   piece_cost_pages  >= 0
 * Returns the split count, or GQLA_ERR_INVALID_ARG. */
int gqla_plan_splits(const int32_t *seqlens, int batch, int max_splits, int piece_cost_pages);

/* The lead of the absorb path's split plan (gqla_decode_absorb_lead) for a step
 * that runs both paths over one batch on two streams, the absorb decode
 * launched first.  From the times each call takes alone with equal chunks
 * (measured by the caller, µs): lead_splits = the absorb chunks whose CTAs
 * (2 per 128 query rows) fit on the SMs of a device with num_sms SMs that the
 * GQA decode (gqa_splits chunks, times its group split, the rule the GQA
 * decode applies on such a device) leaves idle, at most absorb_splits - 1;
 * lead_weight16 such that the lead chunks end the absorb combine's time before
 * the GQA decode does, with the total work unchanged:
 * W = 1 + (x / T_a) / (1 - x lead / (absorb_splits T_a)), x = gqa - combine,
 * T_a = absorb_decode_us, the denominator at least 0.05, W at most 64,
 * lead_weight16 = round(16 W).  lead 0 and weight 16 (equal chunks) when the
 * GQA decode fills the device or x <= 0.  Host-only: touches no device.
 * Returns GQLA_OK or GQLA_ERR_INVALID_ARG. */
int gqla_plan_lead(const gqla_dims *dims, int s_q, int num_sms, int absorb_splits, int gqa_splits,
                   float absorb_decode_us, float gqa_decode_us, float absorb_combine_us,
                   int *lead_splits, int *lead_weight16);

/* Reads (synchronising `stream`) and returns the first device-side error
 * recorded in `workspace` (GQLA_OK if none); `info`, if not NULL, receives
 * a code-specific detail (e.g. the sequence index).  Does not clear it. */
int gqla_read_device_error(const void *workspace, int *info, gqla_stream_t stream);

/* Clears the device error record (asynchronously, on `stream`). */
int gqla_clear_device_error(void *workspace, gqla_stream_t stream);

/* Diagnostic for testing the failure path: the next decode call made by this
 * host thread leaves out one load -- gqla_decode_gqa (or
 * gqla_decode_gqa_noalloc): the V load of work unit `unit` (units count
 * (page pair, group) in issue order within a CTA); gqla_decode_absorb: the
 * latent load of tile `unit` (64-token tiles in issue order within a CTA) --
 * so the wait for it runs out after about two seconds: that call then
 * records GQLA_ERR_TIMEOUT in its workspace, its outputs are unspecified, and
 * the context stays usable.  -1 cancels.  Returns GQLA_OK, or
 * GQLA_ERR_INVALID_ARG for unit < -1. */
int gqla_debug_drop_v_load(int unit);

/* Static description of a status code. */
const char *gqla_status_string(int status);

/* Description of the CUDA error behind the last GQLA_ERR_CUDA returned on the
 * calling thread ("no error" if none). */
const char *gqla_last_cuda_error(void);

/* Library ABI version: 1. */
int gqla_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GQLA_H_ */
