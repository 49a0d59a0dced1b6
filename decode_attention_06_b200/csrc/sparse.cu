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
// With a slot list instead of a selected cache (the fused path), only each
// selected row's cache slot is written, and the GQA decode gathers the rows
// itself.
//
// One CTA per 32 entries of a list: it counts the valid entries before its
// own (-1 marks an unused entry; any other position outside [0, L_b - s_q + s]
// or on a page outside the pool is a device error and is skipped), compacts
// its entries with a warp ballot, and copies their rows with consecutive
// threads on consecutive 16-byte chunks of a row.
#include "common.cuh"

namespace gqla {

namespace {

constexpr int kSgThreads = 256;
constexpr int kSgChunk = 32;   // list entries per CTA (one warp compacts them)

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
    int32_t *sel_slot;            // [batch * s_q * cap]: the cache slot of each selected row, or null
    void *ws;
    int64_t num_slots, sel_slots;
    int s_q, topk, cap, max_pages, num_pages, num_groups;
};

// Cache slot of list entry t for a query that sees tokens [0, last], or -1.
__device__ __forceinline__ int entry_slot(const SgParams &p, const int32_t *prow, int t, int last) {
    if (t < 0 || t > last || t / kPage >= p.max_pages) return -1;
    const int page = prow[t / kPage];
    return page >= 0 && page < p.num_pages ? page * kPage + t % kPage : -1;
}

// grid (entries / kSgChunk, batch * s_q): CTA (c, v) compacts entries
// [c * kSgChunk, (c + 1) * kSgChunk) of list v, after counting the valid entries
// before them.
// With COPY the rows themselves go to the selected cache; without, only their
// cache slots go to sel_slot (the rows past a list's valid entries get -1).
template <bool COPY>
__global__ void __launch_bounds__(kSgThreads) sparse_gather_kernel(const SgParams p) {
    __shared__ int s_warp[kSgThreads / 32];
    __shared__ int s_slot[kSgChunk];
    __shared__ int s_dst[kSgChunk];
    const int v = blockIdx.y, j0 = blockIdx.x * kSgChunk;
    const int b = v / p.s_q, s = v % p.s_q;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int L = p.seqlens[b];
    const int last = L - p.s_q + s;  // this query sees t <= last
    const int32_t *idx = p.idx + (int64_t)v * p.topk;
    const int32_t *prow = p.page_table + (int64_t)b * p.max_pages;
    // valid entries before this chunk: eight list entries per thread are loaded first and
    // their page-table entries next, so a CTA late in a long list waits for two rounds of
    // loads per 2048 entries instead of two per 256
    int n = 0;
    constexpr int kU = 8;
    for (int jb = 0; jb < j0; jb += kSgThreads * kU) {
        int t[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int j = jb + u * kSgThreads + threadIdx.x;
            t[u] = j < j0 ? idx[j] : -1;
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) n += entry_slot(p, prow, t[u], last) >= 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
    if (lane == 0) s_warp[warp] = n;
    __syncthreads();
    int before = 0;
#pragma unroll
    for (int w = 0; w < kSgThreads / 32; ++w) before += s_warp[w];
    __syncthreads();  // s_warp is reused below
    // this chunk (warp 0): validity (errors reported here only), compaction by a ballot
    static_assert(kSgChunk == 32, "one warp compacts a chunk");
    int total = 0;
    if (warp < kSgChunk / 32) {
        const int j = j0 + threadIdx.x;
        const int t = j < p.topk ? idx[j] : -1;
        const int slot = j < p.topk ? entry_slot(p, prow, t, last) : -1;
        if (slot < 0 && t != -1) report_error(p.ws, GQLA_ERR_DEVICE, v);
        const unsigned m = __ballot_sync(0xffffffffu, slot >= 0);
        if (lane == 0) s_warp[warp] = __popc(m);
        const int k = __popc(m & ((1u << lane) - 1u));
        if (slot >= 0) {
            s_slot[k] = slot;
            s_dst[k] = v * p.cap + before + k;
        }
    }
    __syncthreads();
    total = s_warp[0];
    if constexpr (!COPY) {
        if (threadIdx.x < total) p.sel_slot[s_dst[threadIdx.x]] = s_slot[threadIdx.x];
        if (j0 + kSgChunk >= p.topk)  // the list's last chunk: rows past its valid entries
            for (int i = before + total + threadIdx.x; i < p.cap; i += kSgThreads) p.sel_slot[(int64_t)v * p.cap + i] = -1;
    }
    // copy the chunk's rows: every group's 512-byte [K_nope | V] row, then k^R;
    // consecutive threads take consecutive 16-byte chunks of a row
    const int chunks16 = p.num_groups * 32 + 8;
#pragma unroll 4
    for (int e = threadIdx.x; e < (COPY ? total * chunks16 : 0); e += kSgThreads) {
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
    if (j0 + kSgChunk >= p.topk && threadIdx.x == 0) p.sel_seqlens[v] = before + total;
    if (blockIdx.x == 0) {
        const int pages = p.cap / kPage;
        for (int i = threadIdx.x; i < pages; i += kSgThreads)
            p.sel_page_table[(int64_t)v * pages + i] = v * pages + i;
    }
}

}  // namespace

cudaError_t launch_sparse_gather(const void *kv, const void *k_rope, int64_t num_slots,
                                 const gqla_kv_index *idx, int s_q, const int32_t *topk_idx, int topk,
                                 int num_groups, void *kv_sel, void *k_rope_sel, int32_t *sel_page_table,
                                 int32_t *sel_seqlens, int32_t *sel_slot, void *ws, cudaStream_t stream) {
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
    p.sel_slot = sel_slot;
    p.ws = ws;
    p.num_slots = num_slots;
    p.s_q = s_q;
    p.topk = topk;
    p.cap = (topk + kPage - 1) / kPage * kPage;
    p.sel_slots = (int64_t)virt * p.cap;
    p.max_pages = idx->max_pages_per_seq;
    p.num_pages = idx->num_pages;
    p.num_groups = num_groups;
    const dim3 grid((unsigned)((topk + kSgChunk - 1) / kSgChunk), (unsigned)virt);
    if (sel_slot)
        sparse_gather_kernel<false><<<grid, kSgThreads, 0, stream>>>(p);
    else
        sparse_gather_kernel<true><<<grid, kSgThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace gqla
