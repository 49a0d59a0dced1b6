// sparse.cu -- the selection step of sparse GQLA on the GQA path (GQLA,
// paperlayer.ai summary, sec. 2 "Sparse GQLA"; pwwt.cn article, sec. 5: each
// new token attends to a small selected set of earlier tokens; with 16 query
// heads per KV group the GQA path keeps full tensor-core tiles).
//
// Every query token (b, s) brings its own list of selected token positions,
// shared by all heads.  This kernel compacts each list into a small dense
// cache: the selected rows of every group's expanded [K_nope | V] and of k^R,
// at rows [v * cap, v * cap + n_v) of a "selected" cache (v = b * s_q + s,
// cap = topk rounded up to a 64-token page, n_v = number of valid entries),
// plus the identity page table and lengths n_v of that cache.  The GQA decode
// then runs unchanged over the B * s_q selected sequences with s_q = 1
// (every selected token is visible to its query), and the usual combine
// merges the splits.
//
// One CTA per query token; 256 entries of the list at a time are checked
// (-1 marks an unused entry; any other position outside [0, L_b - s_q + s] or
// on a page outside the pool is a device error and is skipped), compacted by
// a block-wide prefix count, and copied with consecutive threads on
// consecutive 16-byte chunks of a row.
#include "common.cuh"

namespace gqla {

namespace {

constexpr int kSgThreads = 256;

struct SgParams {
    const __nv_bfloat16 *kv;      // [g][num_slots][256]
    const __nv_bfloat16 *k_rope;  // [num_slots][64]
    const int32_t *page_table;    // [batch][max_pages]
    const int32_t *seqlens;       // [batch]
    const int32_t *idx;           // [batch][s_q][topk]
    __nv_bfloat16 *kv_sel;        // [g][sel_slots][256]
    __nv_bfloat16 *k_rope_sel;    // [sel_slots][64]
    int32_t *sel_page_table;      // [batch * s_q][cap / 64]
    int32_t *sel_seqlens;         // [batch * s_q]
    void *ws;
    int64_t num_slots, sel_slots;
    int s_q, topk, cap, max_pages, num_pages, num_groups;
};

__global__ void __launch_bounds__(kSgThreads) sparse_gather_kernel(const SgParams p) {
    __shared__ int s_warp[kSgThreads / 32];
    __shared__ int s_slot[kSgThreads];
    __shared__ int s_dst[kSgThreads];
    const int v = blockIdx.x;
    const int b = v / p.s_q, s = v % p.s_q;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int L = p.seqlens[b];
    const int last = L - p.s_q + s;  // this query sees t <= last
    const int32_t *idx = p.idx + (int64_t)v * p.topk;
    const int32_t *prow = p.page_table + (int64_t)b * p.max_pages;
    const int chunks16 = p.num_groups * 32 + 8;  // 16-byte chunks per selected token
    int count = 0;
    for (int j0 = 0; j0 < p.topk; j0 += kSgThreads) {
        const int j = j0 + threadIdx.x;
        const int t = j < p.topk ? idx[j] : -1;
        int slot = -1;
        if (t >= 0 && t <= last && t / kPage < p.max_pages) {
            const int page = prow[t / kPage];
            if (page >= 0 && page < p.num_pages) slot = page * kPage + t % kPage;
        }
        if (slot < 0 && t != -1 && j < p.topk) report_error(p.ws, GQLA_ERR_DEVICE, v);
        // block-wide exclusive count of the valid entries before this one
        const unsigned m = __ballot_sync(0xffffffffu, slot >= 0);
        if (lane == 0) s_warp[warp] = __popc(m);
        __syncthreads();
        int before = 0, total = 0;
#pragma unroll
        for (int w = 0; w < kSgThreads / 32; ++w) {
            before += w < warp ? s_warp[w] : 0;
            total += s_warp[w];
        }
        if (slot >= 0) {
            const int k = before + __popc(m & ((1u << lane) - 1u));
            s_slot[k] = slot;
            s_dst[k] = v * p.cap + count + k;
        }
        __syncthreads();
        // copy the chunk's `total` rows: every group's 512-byte [K_nope | V] row, then k^R
        for (int e = threadIdx.x; e < total * chunks16; e += kSgThreads) {
            const int k = e / chunks16, part = e % chunks16;
            const int64_t src = s_slot[k], dst = s_dst[k];
            if (part < p.num_groups * 32) {
                const int g = part >> 5, c = part & 31;
                reinterpret_cast<uint4 *>(p.kv_sel + ((int64_t)g * p.sel_slots + dst) * kKv)[c] =
                    reinterpret_cast<const uint4 *>(p.kv + ((int64_t)g * p.num_slots + src) * kKv)[c];
            } else {
                const int c = part - p.num_groups * 32;
                reinterpret_cast<uint4 *>(p.k_rope_sel + dst * kRope)[c] =
                    reinterpret_cast<const uint4 *>(p.k_rope + src * kRope)[c];
            }
        }
        count += total;
        __syncthreads();  // s_slot / s_dst / s_warp are rewritten by the next chunk
    }
    const int pages = p.cap / kPage;
    for (int i = threadIdx.x; i < pages; i += kSgThreads) p.sel_page_table[(int64_t)v * pages + i] = v * pages + i;
    if (threadIdx.x == 0) p.sel_seqlens[v] = count;
}

}  // namespace

cudaError_t launch_sparse_gather(const void *kv, const void *k_rope, int64_t num_slots,
                                 const gqla_kv_index *idx, int s_q, const int32_t *topk_idx, int topk,
                                 int num_groups, void *kv_sel, void *k_rope_sel, int32_t *sel_page_table,
                                 int32_t *sel_seqlens, void *ws, cudaStream_t stream) {
    const int virt = idx->batch * s_q;
    SgParams p;
    p.kv = static_cast<const __nv_bfloat16 *>(kv);
    p.k_rope = static_cast<const __nv_bfloat16 *>(k_rope);
    p.page_table = idx->page_table;
    p.seqlens = idx->seqlens;
    p.idx = topk_idx;
    p.kv_sel = static_cast<__nv_bfloat16 *>(kv_sel);
    p.k_rope_sel = static_cast<__nv_bfloat16 *>(k_rope_sel);
    p.sel_page_table = sel_page_table;
    p.sel_seqlens = sel_seqlens;
    p.ws = ws;
    p.num_slots = num_slots;
    p.s_q = s_q;
    p.topk = topk;
    p.cap = (topk + kPage - 1) / kPage * kPage;
    p.sel_slots = (int64_t)virt * p.cap;
    p.max_pages = idx->max_pages_per_seq;
    p.num_pages = idx->num_pages;
    p.num_groups = num_groups;
    sparse_gather_kernel<<<virt, kSgThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace gqla
