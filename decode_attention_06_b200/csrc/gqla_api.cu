// gqla_api.cu -- the extern "C" entry points of libgqla (declared in
// include/gqla.h): argument validation, then launches on the caller's stream.
#include <math.h>

#include <algorithm>
#include <vector>

#include "common.cuh"

namespace gqla {
cudaError_t launch_expand(const void *latent, int64_t num_slots, const void *w_uk,
                          const void *w_uv, void *kv, void *k_rope, int num_groups,
                          cudaStream_t stream);
cudaError_t launch_expand_tc(const void *latent, int64_t num_slots, const void *w_uk,
                             const void *w_uv, void *kv, void *k_rope, int num_groups,
                             cudaStream_t stream);
cudaError_t launch_sparse_gather(const void *kv, const void *k_rope, int64_t num_slots,
                                 const gqla_kv_index *idx, int s_q, const int32_t *topk_idx, int topk,
                                 int num_groups, void *kv_sel, void *k_rope_sel, int32_t *sel_page_table,
                                 int32_t *sel_seqlens, int32_t *sel_slot, void *ws, cudaStream_t stream);
cudaError_t launch_decode_gqa_sparse(const void *q, int heads, int num_groups, const void *kv,
                                     const void *k_rope, int64_t real_slots, const gqla_kv_index *sel,
                                     const int32_t *sel_slot, int num_splits, float scale, float *o_part,
                                     float *lse_part, void *ws, cudaStream_t stream);
cudaError_t launch_absorb_query(const void *q, int rows, int heads, int num_groups,
                                const void *w_uk, void *qa, cudaStream_t stream);
cudaError_t launch_decode_gqa(const void *q, int s_q, int heads, int num_groups, const void *kv,
                              const void *k_rope, int64_t num_slots, const gqla_kv_index *idx,
                              int num_splits, float scale, float *o_part, float *lse_part,
                              void *out, float *lse_out, void *ws, cudaStream_t stream);
cudaError_t launch_decode_absorb(const void *qa, int s_q, int heads, const void *cache,
                                 const gqla_kv_index *idx, int num_splits, int lead, int lead_w16,
                                 float scale, float *o_part, float *lse_part, void *ws,
                                 cudaStream_t stream);
cudaError_t launch_combine(const gqla_kv_index *kv, int s_q, int num_splits, int lead, int lead_w16,
                           int d_in, const float *o_part, const float *lse_part, const void *w_uv,
                           void *out, float *lse_out, int heads, int num_groups, bool skip_single,
                           cudaStream_t stream);
int group_splits_rule(int num_splits, int num_groups, int sms);
extern thread_local int g_drop_v_unit;
}  // namespace gqla

using namespace gqla;

namespace {

constexpr size_t kWorkspaceBytes = 256;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A lead of 0 .. num_splits chunks, each 1 to 64 times as long as the others (in 1/16).
bool lead_ok(int num_splits, int lead, int w16) {
    return lead >= 0 && lead <= num_splits && w16 >= 16 && w16 <= 1024;
}

int check_dims(const gqla_dims *d, int s_q) {
    if (!d) return GQLA_ERR_INVALID_ARG;
    if (d->num_heads <= 0 || d->num_groups <= 0 || d->num_heads % d->num_groups)
        return GQLA_ERR_INVALID_ARG;
    if (!(d->softmax_scale > 0.0f) || !isfinite(d->softmax_scale)) return GQLA_ERR_INVALID_ARG;
    if (!dims_supported(d)) return GQLA_ERR_UNSUPPORTED;
    const int G = d->num_heads / d->num_groups;
    if (s_q < 1 || s_q > 2) return s_q < 1 ? GQLA_ERR_INVALID_ARG : GQLA_ERR_UNSUPPORTED;
    if (G % 4 != 0 || G * s_q > 32) return GQLA_ERR_UNSUPPORTED;
    return GQLA_OK;
}

int check_index(const gqla_kv_index *kv) {
    if (!kv || !kv->page_table || !kv->seqlens) return GQLA_ERR_INVALID_ARG;
    if (kv->batch <= 0 || kv->max_pages_per_seq <= 0 || kv->num_pages <= 0)
        return GQLA_ERR_INVALID_ARG;
    if (kv->batch > 65535) return GQLA_ERR_UNSUPPORTED;
    if (kv->page_size != kPage) return GQLA_ERR_UNSUPPORTED;
    return GQLA_OK;
}

int check_workspace(const void *ws, size_t bytes) {
    if (!ws || bytes < kWorkspaceBytes || !aligned16(ws)) return GQLA_ERR_WORKSPACE;
    return GQLA_OK;
}

thread_local cudaError_t g_last_cuda_error = cudaSuccess;

int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return GQLA_OK;
    g_last_cuda_error = e;
    return GQLA_ERR_CUDA;
}

int check_expand_args(const gqla_dims *dims, const void *latent, int64_t num_slots, const void *w_uk,
                      const void *w_uv, void *kv_expanded, void *k_rope) {
    int st = check_dims(dims, 1);
    if (st == GQLA_ERR_UNSUPPORTED && dims && dims_supported(dims)) st = GQLA_OK;  // head split irrelevant here
    if (st != GQLA_OK) return st;
    if (num_slots < 0) return GQLA_ERR_INVALID_ARG;
    if (!latent || !w_uk || !w_uv || !kv_expanded || !k_rope) return GQLA_ERR_INVALID_ARG;
    if (!aligned16(latent) || !aligned16(w_uk) || !aligned16(w_uv) || !aligned16(kv_expanded) ||
        !aligned16(k_rope))
        return GQLA_ERR_INVALID_ARG;
    if (num_slots > ((int64_t)1 << 31) - 1) return GQLA_ERR_UNSUPPORTED;
    return GQLA_OK;
}

}  // namespace

extern "C" {

int gqla_version(void) { return 1; }

int gqla_debug_drop_v_load(int unit) {
    if (unit < -1) return GQLA_ERR_INVALID_ARG;
    g_drop_v_unit = unit;
    return GQLA_OK;
}

const char *gqla_last_cuda_error(void) { return cudaGetErrorString(g_last_cuda_error); }

const char *gqla_status_string(int status) {
    switch (status) {
        case GQLA_OK: return "ok";
        case GQLA_ERR_INVALID_ARG: return "invalid argument";
        case GQLA_ERR_UNSUPPORTED: return "unsupported shape";
        case GQLA_ERR_WORKSPACE: return "workspace missing or too small";
        case GQLA_ERR_CUDA: return "CUDA error";
        case GQLA_ERR_DEVICE: return "device-side check failed";
        case GQLA_ERR_TIMEOUT: return "device-side wait timed out";
        default: return "unknown status";
    }
}

size_t gqla_workspace_bytes(void) { return kWorkspaceBytes; }

int gqla_partial_slots(int batch, int num_splits) {
    if (batch <= 0 || num_splits <= 0) return GQLA_ERR_INVALID_ARG;
    return batch + num_splits;
}

int gqla_num_splits_hint(int path, int num_heads, int s_q) {
    if ((path != 0 && path != 1) || num_heads <= 0 || s_q <= 0) return GQLA_ERR_INVALID_ARG;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GQLA_ERR_CUDA;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return GQLA_ERR_CUDA;
    if (path == 1) return sms;
    const int row_blocks = (s_q * num_heads + 127) / 128;
    return sms / (2 * row_blocks) > 0 ? sms / (2 * row_blocks) : 1;
}

int gqla_plan_lead(const gqla_dims *dims, int s_q, int num_sms, int absorb_splits, int gqa_splits,
                   float absorb_decode_us, float gqa_decode_us, float absorb_combine_us,
                   int *lead_splits, int *lead_weight16) {
    int st = check_dims(dims, s_q);
    if (st != GQLA_OK) return st;
    if (num_sms <= 0 || absorb_splits <= 0 || absorb_splits > 65535 || gqa_splits <= 0 ||
        gqa_splits > 65535 || !lead_splits || !lead_weight16 || !(absorb_decode_us > 0.0f) ||
        !(gqa_decode_us >= 0.0f) || !(absorb_combine_us >= 0.0f))
        return GQLA_ERR_INVALID_ARG;
    *lead_splits = 0;
    *lead_weight16 = 16;
    const int sms = num_sms;
    // SMs the GQA decode leaves idle, in absorb chunks (2 CTAs per 128 query rows)
    const int row_blocks = (s_q * dims->num_heads + 127) / 128;
    const int gqa_ctas = gqa_splits * group_splits_rule(gqa_splits, dims->num_groups, sms);
    const int free_sms = sms - gqa_ctas;
    const int n = absorb_splits;
    int e = free_sms > 0 ? free_sms / (2 * row_blocks) : 0;
    if (e > n - 1) e = n - 1;
    // The short chunks' CTAs finish at T_s; the GQA decode then runs on their SMs for
    // gqa_decode_us, and the lead chunks should end the absorb combine's time before it
    // does: W T_s = T_s + x with x = gqa - combine.  The work is the same as with equal
    // chunks of time T_a: (e W + n - e) T_s = n T_a.  So W - 1 = (x / T_a) / (1 - x e / (n T_a)).
    const double x = (double)gqa_decode_us - (double)absorb_combine_us;
    if (e <= 0 || x <= 0.0) return GQLA_OK;
    const double ta = absorb_decode_us;
    double den = 1.0 - x * e / (n * ta);
    if (den < 0.05) den = 0.05;
    double w = 1.0 + (x / ta) / den;
    if (w > 64.0) w = 64.0;
    *lead_splits = e;
    *lead_weight16 = (int)lround(16.0 * w);
    return GQLA_OK;
}

int gqla_plan_splits(const int32_t *seqlens, int batch, int max_splits, int piece_cost_pages) {
    if (!seqlens || batch <= 0 || batch > 65535 || max_splits <= 0 || max_splits > 65535 ||
        piece_cost_pages < 0)
        return GQLA_ERR_INVALID_ARG;
    // first global page of every non-empty sequence after the first one
    std::vector<int64_t> starts;
    int64_t total = 0;
    for (int b = 0; b < batch; ++b) {
        if (seqlens[b] < 0) return GQLA_ERR_INVALID_ARG;
        const int64_t np = (seqlens[b] + kPage - 1) / kPage;
        if (np > 0 && total > 0) starts.push_back(total);
        total += np;
    }
    if (total == 0) return 1;
    // Every chunk but the last holds k pages, so the heaviest chunk is k pages (or the
    // whole batch when it fits one chunk) unless a chunk with sequence starts inside it
    // weighs more; the starts are ascending, so one pass groups them by chunk.
    // O(max_splits * batch) at most.
    int best = 1;
    int64_t best_cost = -1, prev_k = -1;
    for (int n = 1; n <= max_splits; ++n) {
        const int64_t k = (total + n - 1) / n;
        if (k == prev_k) continue;  // the same chunks as a smaller count
        prev_k = k;
        int64_t worst = std::min(k, total);
        for (size_t i = 0; i < starts.size();) {
            const int64_t c = starts[i] / k;
            int64_t inside = 0;
            for (; i < starts.size() && starts[i] / k == c; ++i) inside += starts[i] % k != 0;
            worst = std::max(worst, std::min(k, total - c * k) + inside * piece_cost_pages);
        }
        if (best_cost < 0 || worst < best_cost) {
            best_cost = worst;
            best = n;
        }
    }
    return best;
}

int gqla_read_device_error(const void *workspace, int *info, gqla_stream_t stream) {
    if (!workspace) return GQLA_ERR_INVALID_ARG;
    DeviceError e{0, 0};
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(&e, workspace, sizeof e, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return GQLA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return GQLA_ERR_CUDA;
    if (info) *info = e.info;
    return e.code;
}

int gqla_clear_device_error(void *workspace, gqla_stream_t stream) {
    if (!workspace) return GQLA_ERR_INVALID_ARG;
    return cuda_status(cudaMemsetAsync(workspace, 0, sizeof(DeviceError),
                                       reinterpret_cast<cudaStream_t>(stream)));
}

int gqla_expand_cache(const gqla_dims *dims, const void *latent, int64_t num_slots,
                      const void *w_uk, const void *w_uv, void *kv_expanded, void *k_rope,
                      gqla_stream_t stream) {
    const int st = check_expand_args(dims, latent, num_slots, w_uk, w_uv, kv_expanded, k_rope);
    if (st != GQLA_OK) return st;
    return cuda_status(launch_expand(latent, num_slots, w_uk, w_uv, kv_expanded, k_rope,
                                     dims->num_groups, reinterpret_cast<cudaStream_t>(stream)));
}

int gqla_expand_cache_tc(const gqla_dims *dims, const void *latent, int64_t num_slots,
                         const void *w_uk, const void *w_uv, void *kv_expanded, void *k_rope,
                         gqla_stream_t stream) {
    const int st = check_expand_args(dims, latent, num_slots, w_uk, w_uv, kv_expanded, k_rope);
    if (st != GQLA_OK) return st;
    return cuda_status(launch_expand_tc(latent, num_slots, w_uk, w_uv, kv_expanded, k_rope,
                                        dims->num_groups, reinterpret_cast<cudaStream_t>(stream)));
}

int gqla_absorb_query(const gqla_dims *dims, const void *q, int batch, int s_q,
                      const void *w_uk, void *q_absorbed, gqla_stream_t stream) {
    int st = check_dims(dims, s_q);
    if (st != GQLA_OK) return st;
    if (batch <= 0 || !q || !w_uk || !q_absorbed) return GQLA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(w_uk) || !aligned16(q_absorbed)) return GQLA_ERR_INVALID_ARG;
    const int rows = batch * s_q * dims->num_heads;
    return cuda_status(launch_absorb_query(q, rows, dims->num_heads, dims->num_groups, w_uk,
                                           q_absorbed, reinterpret_cast<cudaStream_t>(stream)));
}

int gqla_decode_absorb(const gqla_dims *dims, const void *q_absorbed, int s_q,
                       const void *latent_cache, const gqla_kv_index *kv, int num_splits,
                       float *o_part, float *lse_part, void *workspace, size_t workspace_bytes,
                       gqla_stream_t stream) {
    return gqla_decode_absorb_lead(dims, q_absorbed, s_q, latent_cache, kv, num_splits, 0, 16, o_part,
                                   lse_part, workspace, workspace_bytes, stream);
}

int gqla_decode_absorb_lead(const gqla_dims *dims, const void *q_absorbed, int s_q,
                            const void *latent_cache, const gqla_kv_index *kv, int num_splits,
                            int lead_splits, int lead_weight16, float *o_part, float *lse_part,
                            void *workspace, size_t workspace_bytes, gqla_stream_t stream) {
    int st = check_dims(dims, s_q);
    if (st != GQLA_OK) return st;
    if ((st = check_index(kv)) != GQLA_OK) return st;
    if ((st = check_workspace(workspace, workspace_bytes)) != GQLA_OK) return st;
    if (num_splits <= 0 || num_splits > 65535) return GQLA_ERR_INVALID_ARG;
    if (!lead_ok(num_splits, lead_splits, lead_weight16)) return GQLA_ERR_INVALID_ARG;
    if (!q_absorbed || !latent_cache || !o_part || !lse_part) return GQLA_ERR_INVALID_ARG;
    if (!aligned16(q_absorbed) || !aligned16(latent_cache) || !aligned16(o_part))
        return GQLA_ERR_INVALID_ARG;
    if ((s_q * dims->num_heads) % 32) return GQLA_ERR_UNSUPPORTED;
    if ((int64_t)num_splits * ((s_q * dims->num_heads + 127) / 128) * 2 > 65535 * 2)
        return GQLA_ERR_UNSUPPORTED;
    return cuda_status(launch_decode_absorb(q_absorbed, s_q, dims->num_heads, latent_cache, kv,
                                            num_splits, lead_splits, lead_weight16, dims->softmax_scale,
                                            o_part, lse_part, workspace,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

int gqla_decode_gqa(const gqla_dims *dims, const void *q, int s_q, const void *kv_expanded,
                    const void *k_rope, int64_t num_slots, const gqla_kv_index *kv,
                    int num_splits, float *o_part, float *lse_part, void *workspace,
                    size_t workspace_bytes, gqla_stream_t stream) {
    int st = check_dims(dims, s_q);
    if (st != GQLA_OK) return st;
    if ((st = check_index(kv)) != GQLA_OK) return st;
    if ((st = check_workspace(workspace, workspace_bytes)) != GQLA_OK) return st;
    if (num_splits <= 0 || num_splits > 65535) return GQLA_ERR_INVALID_ARG;
    if (!q || !kv_expanded || !k_rope || !o_part || !lse_part) return GQLA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(kv_expanded) || !aligned16(k_rope) || !aligned16(o_part))
        return GQLA_ERR_INVALID_ARG;
    if (num_slots != (int64_t)kv->num_pages * kv->page_size) return GQLA_ERR_INVALID_ARG;
    if (dims->num_groups != 8 && dims->num_groups != 4 && dims->num_groups != 2 && dims->num_groups != 1)
        return GQLA_ERR_UNSUPPORTED;
    return cuda_status(launch_decode_gqa(q, s_q, dims->num_heads, dims->num_groups, kv_expanded,
                                         k_rope, num_slots, kv, num_splits, dims->softmax_scale,
                                         o_part, lse_part, nullptr, nullptr, workspace,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

int gqla_decode_gqa_step(const gqla_dims *dims, const void *q, int s_q, const void *kv_expanded,
                         const void *k_rope, int64_t num_slots, const gqla_kv_index *kv,
                         int num_splits, float *o_part, float *lse_part, void *out, float *lse_out,
                         void *workspace, size_t workspace_bytes, gqla_stream_t stream) {
    int st = check_dims(dims, s_q);
    if (st != GQLA_OK) return st;
    if ((st = check_index(kv)) != GQLA_OK) return st;
    if ((st = check_workspace(workspace, workspace_bytes)) != GQLA_OK) return st;
    if (num_splits <= 0 || num_splits > 65535) return GQLA_ERR_INVALID_ARG;
    if (!q || !kv_expanded || !k_rope || !out) return GQLA_ERR_INVALID_ARG;
    if (num_splits > 1 && (!o_part || !lse_part)) return GQLA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(kv_expanded) || !aligned16(k_rope) || !aligned16(out) ||
        (o_part && !aligned16(o_part)))
        return GQLA_ERR_INVALID_ARG;
    if (num_slots != (int64_t)kv->num_pages * kv->page_size) return GQLA_ERR_INVALID_ARG;
    if (dims->num_groups != 8 && dims->num_groups != 4 && dims->num_groups != 2 && dims->num_groups != 1)
        return GQLA_ERR_UNSUPPORTED;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    st = cuda_status(launch_decode_gqa(q, s_q, dims->num_heads, dims->num_groups, kv_expanded, k_rope,
                                       num_slots, kv, num_splits, dims->softmax_scale, o_part, lse_part,
                                       out, lse_out, workspace, s));
    if (st != GQLA_OK || num_splits == 1) return st;  // one chunk: every sequence is final already
    return cuda_status(launch_combine(kv, s_q, num_splits, 0, 16, kDv, o_part, lse_part, nullptr, out,
                                      lse_out, dims->num_heads, dims->num_groups, true, s));
}

int gqla_sparse_gather(const gqla_dims *dims, const void *kv_expanded, const void *k_rope,
                       int64_t num_slots, const gqla_kv_index *kv, int s_q, const int32_t *topk_idx,
                       int topk, void *kv_sel, void *k_rope_sel, int32_t *sel_page_table,
                       int32_t *sel_seqlens, void *workspace, size_t workspace_bytes,
                       gqla_stream_t stream) {
    int st = check_dims(dims, s_q);
    if (st != GQLA_OK) return st;
    if ((st = check_index(kv)) != GQLA_OK) return st;
    if ((st = check_workspace(workspace, workspace_bytes)) != GQLA_OK) return st;
    if (topk <= 0 || topk > 65536) return GQLA_ERR_INVALID_ARG;
    if (!kv_expanded || !k_rope || !topk_idx || !kv_sel || !k_rope_sel || !sel_page_table || !sel_seqlens)
        return GQLA_ERR_INVALID_ARG;
    if (!aligned16(kv_expanded) || !aligned16(k_rope) || !aligned16(kv_sel) || !aligned16(k_rope_sel))
        return GQLA_ERR_INVALID_ARG;
    if (num_slots != (int64_t)kv->num_pages * kv->page_size) return GQLA_ERR_INVALID_ARG;
    if (dims->num_groups != 8 && dims->num_groups != 4) return GQLA_ERR_UNSUPPORTED;
    if ((int64_t)kv->batch * s_q > 65535) return GQLA_ERR_UNSUPPORTED;  // one grid row per query token
    const int64_t cap = (topk + 63) / 64 * 64;
    if ((int64_t)kv->batch * s_q * cap > ((int64_t)1 << 31) - 1) return GQLA_ERR_UNSUPPORTED;
    return cuda_status(launch_sparse_gather(kv_expanded, k_rope, num_slots, kv, s_q, topk_idx, topk,
                                            dims->num_groups, kv_sel, k_rope_sel, sel_page_table,
                                            sel_seqlens, nullptr, workspace, reinterpret_cast<cudaStream_t>(stream)));
}

int gqla_sparse_select(const gqla_dims *dims, const gqla_kv_index *kv, int s_q, const int32_t *topk_idx,
                       int topk, int32_t *sel_slot, int32_t *sel_page_table, int32_t *sel_seqlens,
                       void *workspace, size_t workspace_bytes, gqla_stream_t stream) {
    int st = check_dims(dims, s_q);
    if (st != GQLA_OK) return st;
    if ((st = check_index(kv)) != GQLA_OK) return st;
    if ((st = check_workspace(workspace, workspace_bytes)) != GQLA_OK) return st;
    if (topk <= 0 || topk > 65536) return GQLA_ERR_INVALID_ARG;
    if (!topk_idx || !sel_slot || !sel_page_table || !sel_seqlens || !aligned16(sel_slot))
        return GQLA_ERR_INVALID_ARG;
    if ((int64_t)kv->batch * s_q > 65535) return GQLA_ERR_UNSUPPORTED;
    const int64_t cap = (topk + 63) / 64 * 64;
    if ((int64_t)kv->batch * s_q * cap > ((int64_t)1 << 31) - 1) return GQLA_ERR_UNSUPPORTED;
    return cuda_status(launch_sparse_gather(nullptr, nullptr, 0, kv, s_q, topk_idx, topk, dims->num_groups,
                                            nullptr, nullptr, sel_page_table, sel_seqlens, sel_slot, workspace,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

int gqla_decode_gqa_sparse(const gqla_dims *dims, const void *q, int s_q, const void *kv_expanded,
                           const void *k_rope, int64_t num_slots, const gqla_kv_index *sel,
                           const int32_t *sel_slot, int num_splits, float *o_part, float *lse_part,
                           void *workspace, size_t workspace_bytes, gqla_stream_t stream) {
    int st = check_dims(dims, s_q);
    if (st != GQLA_OK) return st;
    if ((st = check_index(sel)) != GQLA_OK) return st;
    if ((st = check_workspace(workspace, workspace_bytes)) != GQLA_OK) return st;
    if (num_splits <= 0 || num_splits > 65535) return GQLA_ERR_INVALID_ARG;
    if (!q || !kv_expanded || !k_rope || !sel_slot || !o_part || !lse_part) return GQLA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(kv_expanded) || !aligned16(k_rope) || !aligned16(o_part) ||
        !aligned16(sel_slot))
        return GQLA_ERR_INVALID_ARG;
    if (sel->page_size != 64 || sel->batch % s_q != 0) return GQLA_ERR_INVALID_ARG;
    if (num_slots <= 0 || (int64_t)dims->num_groups * num_slots > ((int64_t)1 << 31) - 1)
        return GQLA_ERR_UNSUPPORTED;
    if (dims->num_groups != 8 && dims->num_groups != 4) return GQLA_ERR_UNSUPPORTED;
    return cuda_status(launch_decode_gqa_sparse(q, dims->num_heads, dims->num_groups, kv_expanded, k_rope,
                                                num_slots, sel, sel_slot, num_splits, dims->softmax_scale,
                                                o_part, lse_part, workspace,
                                                reinterpret_cast<cudaStream_t>(stream)));
}

int gqla_combine(const gqla_dims *dims, const gqla_kv_index *kv, int s_q, int num_splits,
                 int d_in, const float *o_part, const float *lse_part, const void *w_uv,
                 void *out, float *lse_out, gqla_stream_t stream) {
    return gqla_combine_lead(dims, kv, s_q, num_splits, 0, 16, d_in, o_part, lse_part, w_uv, out,
                             lse_out, stream);
}

int gqla_combine_lead(const gqla_dims *dims, const gqla_kv_index *kv, int s_q, int num_splits,
                      int lead_splits, int lead_weight16, int d_in, const float *o_part,
                      const float *lse_part, const void *w_uv, void *out, float *lse_out,
                      gqla_stream_t stream) {
    int st = check_dims(dims, s_q);
    if (st != GQLA_OK) return st;
    if ((st = check_index(kv)) != GQLA_OK) return st;
    if (num_splits <= 0 || num_splits > 65535) return GQLA_ERR_INVALID_ARG;
    if (!lead_ok(num_splits, lead_splits, lead_weight16)) return GQLA_ERR_INVALID_ARG;
    if (!o_part || !lse_part || !out) return GQLA_ERR_INVALID_ARG;
    if (!aligned16(o_part) || !aligned16(out) || (w_uv && !aligned16(w_uv)))
        return GQLA_ERR_INVALID_ARG;
    if (d_in == kLatent) {
        if (!w_uv) return GQLA_ERR_INVALID_ARG;
    } else if (d_in == kDv) {
        // no GQA decode writes partials on a plan with lead chunks
        if (w_uv || (lead_splits > 0 && lead_weight16 != 16)) return GQLA_ERR_INVALID_ARG;
    } else {
        return GQLA_ERR_INVALID_ARG;
    }
    return cuda_status(launch_combine(kv, s_q, num_splits, lead_splits, lead_weight16, d_in, o_part,
                                      lse_part, w_uv, out, lse_out, dims->num_heads, dims->num_groups,
                                      false, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
