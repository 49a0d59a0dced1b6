// decode_gqa.cu -- split-KV partial attention of the GQA path on the
// tcgen05 tensor cores (GQLA, paperlayer.ai summary, sec. 3 "Two equivalent
// decoding paths": the g K/V groups are materialised and decoding is standard
// grouped-query attention; pwwt.cn article, sec. 5: h_q/g = 16 query heads
// share one group).
//
// The path is HBM-bound (about 19 FLOP per cache byte at s_q = 1), so the
// design goal is to stream the 4224 bytes per token exactly once at full
// bandwidth and hide everything else behind it.
//
//  * Work unit = (128 tokens = two consecutive pages of one sequence, group).
//    The query rows of a group (G*s_q <= 32) are far below the MMA's minimum
//    M, so the products are transposed ("swap-AB"): the 128 tokens are the M
//    dimension and the group's query rows the N dimension (NQ = 16 or 32,
//    zero-padded):
//      S^T[128 tok][NQ]    = [K_nope_g | k^R] (128 x 192, K-major) x q_g^T
//      O^T_g[128 dv][NQ]  += V_g^T (MN-major) x P^T (MN-major, bf16)
//    With M = 128 every TMEM lane, and so every softmax thread, owns one
//    token.  O^T of all g (8 or 4) groups stays resident in TMEM for a whole piece.
//  * One CTA per chunk of the split plan (grid = SM count), 320 threads:
//      warp 0      TMA producer over three rings: q_g + K_nope_g (freed as
//                  soon as S^T is done), V_g (freed after O^T += ...), and
//                  per page pair the shared RoPE keys; each ring refills as
//                  soon as a slot frees, so loads run well ahead;
//      warp 1      TMEM owner; one thread issues the score MMAs;
//      warps 2-9   two softmax warpgroups (the even and the odd groups): each
//                  runs its online softmax, issues its own PV MMAs (one
//                  elected thread) and writes its epilogue.
//  * Online softmax in the base-2 domain with lazy rescaling: P is formed
//    against the running column maxima straight away, and one barrier-with-
//    OR over the warpgroup both publishes P and asks whether any score rose
//    more than 2^8 above its maximum.  Only then (and on a piece's first
//    tile) are the tile's column maxima reduced across warps, O^T in TMEM
//    rescaled and P recomputed.
//  * Every wait is bounded; a wait that runs out records GQLA_ERR_TIMEOUT
//    and the CTA drains and exits instead of hanging.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "sm100.cuh"

namespace gqla {

namespace {

using namespace sm100;

// warp 0 TMA, warp 1 score MMA, warp 2 PV MMA, warp 3 idle (warpgroup 0); warps 4-11 softmax
// (warpgroups 1 and 2)
constexpr int kThreads = 384;
// Register split by setmaxnreg: warpgroup 0 only issues copies and MMAs, the softmax
// warpgroups hold a unit's scores, probabilities and running maxima (3 x NQ values per
// thread).  The launch gives every thread kLaunchRegs (the count ptxas reports under
// these launch bounds, checked on the host before every launch); the split must not
// ask for more in all than the launch gave, or the increase would wait forever.
constexpr int kLaunchRegs = 168;
// The split (ptxas -v shows no spill in any instantiation with it): the issuing roles'
// loops need 72 registers, and the softmax fits in 216 once the running column maxima
// live in shared memory instead of NQ registers.
template <int NQ>
struct RegSplit {
    static constexpr int kIssue = 72;
    static constexpr int kSoftmax = 216;
    static_assert(128 * kIssue + 256 * kSoftmax <= kThreads * kLaunchRegs, "register split");
    static_assert(kIssue % 8 == 0 && kSoftmax % 8 == 0, "setmaxnreg takes multiples of 8");
};

template <int NQ>
__device__ __forceinline__ void regs_decrease() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(RegSplit<NQ>::kIssue));
}
template <int NQ>
__device__ __forceinline__ void regs_increase() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(RegSplit<NQ>::kSoftmax));
}
constexpr int kTok = 128;            // tokens per unit (two pages)
constexpr float kRescaleLog2 = 8.0f;
constexpr int kBox = 64 * 64 * 2;    // one 64-row x 64-column bf16 TMA box (8 KB)

template <int NQ>
struct GqaSmem {
    static constexpr int kKSlots = NQ == 16 ? 3 : 2;
    static constexpr int kVSlots = 2;
    static constexpr int kQBytes = 3 * NQ * 128;        // q_g: 3 column blocks x NQ rows x 128 B
    static constexpr int kKBytes = 4 * kBox;            // K lo | K hi, 128 rows each
    static constexpr int kKSlotBytes = kKBytes + ((kQBytes + 1023) / 1024) * 1024;
    static constexpr int kVBytes = 4 * kBox;            // V lo | V hi, 128 rows each
    static constexpr int kKrBytes = 2 * kBox;           // 128 rows x 64 RoPE dims
    static constexpr int kPBytes = kTok * NQ * 2;       // P^T [128 tokens][NQ] bf16
    static constexpr int oK = 0;
    static constexpr int oV = oK + kKSlots * kKSlotBytes;
    static constexpr int oKr = oV + kVSlots * kVBytes;
    static constexpr int oP = oKr + 2 * kKrBytes;            // one P^T buffer per warpgroup
    static constexpr int oRed = oP + 2 * kPBytes;            // float [2 wg][NQ][4 warps]
    static constexpr int oMrun = oRed + 2 * NQ * 4 * 4;      // float [8 groups][NQ]
    static constexpr int oLred = oMrun + 8 * NQ * 4;         // float [8 groups][NQ][4 warps]
    static constexpr int oBar = oLred + 8 * NQ * 4 * 4;
    // k_full/k_empty[KS], v_full/v_empty[VS], kr_full/kr_empty[2], s_full/s_free[4],
    // p_full/p_free[2], o_done[2], drain x2
    static constexpr int kNumBars = 2 * kKSlots + 2 * kVSlots + 4 + 8 + 6 + 2;
    static constexpr int oEpi = oBar + kNumBars * 8;   // float inv_l[2 wg][NQ], lse[2 wg][NQ]
    static constexpr int oMisc = oEpi + 4 * NQ * 4;  // tmem base, abort flag, plan[4]
    static constexpr int kBytes = oMisc + 32;
    static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024
};

struct GqaParams {
    const int32_t *page_table;
    const int32_t *seqlens;
    float *o_part;
    float *lse_part;
    void *ws;
    int batch, max_pages, num_pages, num_splits, s_q, heads, G;
    // KV groups of one CTA: the cache's g (8, 4 at the (g, s_q) = (4, 1) configuration's
    // 2176-byte tokens, 2 or 1 for a rank's share of 8 groups under group-axis tensor
    // parallelism), or g / gridDim.y when the groups are split over gridDim.y CTAs per
    // chunk (small batches); CTA (c, y) takes groups [y NG, y NG + NG)
    int NG;
    // final outputs for the sequences whose pages all fall in one chunk (their partial is
    // the result): out bf16 [batch][s_q][heads][128], lse_out fp32 (may be null); null out:
    // partials only
    __nv_bfloat16 *out;
    float *lse_out;
    float scale_log2;
    // sparse mode: the "pages" are those of a selection (identity page table, lengths =
    // selected rows per query token); row r of selected page P is cache slot sel_slot[64 P + r]
    // (-1: none), gathered from a cache of real_slots slots
    const int32_t *sel_slot;
    int real_slots;
    // diagnostic: the V load of this unit is never issued, so a bounded wait runs out
    // (-1: none)
    int drop_v_unit;
};

// Iterates the pieces (sequence b, pages [pb, pe)) of chunk `c`; identical in every role.
struct PieceIter {
    int b, P, r0, r1;
};

__device__ __forceinline__ bool next_piece(const GqaParams &p, PieceIter &it, int &b, int &L,
                                           int &pb, int &pe, bool &too_long) {
    while (it.b < p.batch && it.P < it.r1) {
        b = it.b++;
        L = p.seqlens[b];
        const int n = pages_of(L);
        if (n == 0) continue;
        pb = max(it.r0, it.P) - it.P;
        pe = min(it.r1, it.P + n) - it.P;
        it.P += n;
        too_long = L > p.max_pages * kPage;
        return true;
    }
    return false;
}

// Warpgroup w takes the units of the groups gi = w, w + 2, ...: with an even group count
// unit u (u = pair * NG + gi) belongs to warpgroup u % 2 and is its (u / 2)-th unit; with
// one group every unit is warpgroup 0's.
__device__ __forceinline__ uint32_t wg_unit(uint32_t u, int ng) { return ng == 1 ? u : u >> 1; }

// Groups of warpgroup wg: ceil(NG / 2) for warpgroup 0, floor(NG / 2) for warpgroup 1.
__device__ __forceinline__ int wg_groups(int ng, int wg) { return (ng + 1 - wg) >> 1; }

// The two pages of a unit and how many of their rows are real tokens.
struct PagePair {
    int page0, page1;  // -1: missing (past the piece) or outside the pool
    int rows0, rows1;  // valid token rows in each page
    bool bad;          // a page index outside the pool was met
};

__device__ __forceinline__ PagePair make_pair(const GqaParams &p, int L, int pg, int pe, int a0, int a1) {
    PagePair pp;
    const bool bad0 = a0 < 0 || a0 >= p.num_pages;
    const bool bad1 = pg + 1 < pe && (a1 < 0 || a1 >= p.num_pages);
    pp.bad = bad0 || bad1;
    pp.page0 = bad0 ? -1 : a0;
    pp.page1 = (pg + 1 < pe && !bad1) ? a1 : -1;
    pp.rows0 = bad0 ? 0 : min(kPage, L - pg * kPage);
    pp.rows1 = pp.page1 >= 0 ? min(kPage, L - (pg + 1) * kPage) : 0;
    return pp;
}

__device__ __forceinline__ PagePair load_pair(const GqaParams &p, int b, int L, int pg, int pe) {
    const int32_t *row = p.page_table + (int64_t)b * p.max_pages;
    return make_pair(p, L, pg, pe, row[pg], pg + 1 < pe ? row[pg + 1] : 0);
}

// Walks the units (sequence, page pair, group) of a chunk in pipeline order.
// The next pair's page indices are requested halfway through the current
// pair, so the page table is never waited for inside a piece.
struct UnitCursor {
    PieceIter it;
    int b, L, pg, pe, gi;
    int n0, n1;  // page indices of the pair after this one (valid from gi == (NG + 1) / 2)
    PagePair pp;
    bool valid;
    __device__ __forceinline__ bool next_valid_piece(const GqaParams &p) {
        int pb;
        bool too_long;
        while (next_piece(p, it, b, L, pb, pe, too_long)) {
            if (too_long) continue;
            pg = pb;
            gi = 0;
            pp = load_pair(p, b, L, pg, pe);
            return true;
        }
        return false;
    }
    __device__ __forceinline__ void start(const GqaParams &p, const PieceIter &it0) {
        it = it0;
        valid = next_valid_piece(p);
    }
    __device__ __forceinline__ void advance(const GqaParams &p) {
        ++gi;
        if (gi == (p.NG + 1) / 2 && pg + 2 < pe) {
            const int32_t *row = p.page_table + (int64_t)b * p.max_pages;
            n0 = row[pg + 2];
            n1 = pg + 3 < pe ? row[pg + 3] : 0;
        }
        if (gi < p.NG) return;
        gi = 0;
        pg += 2;
        if (pg < pe) { pp = make_pair(p, L, pg, pe, n0, n1); return; }
        valid = next_valid_piece(p);
    }
};

// Butterfly over the lanes of each NQ-lane group: each lane starts with NQ
// column values and ends holding column (lane % NQ) reduced over the group.
template <int NQ, bool MAX>
__device__ __forceinline__ float transpose_reduce(float (&v)[NQ], int lane) {
#pragma unroll
    for (int o = NQ / 2, c = NQ; o >= 1; o >>= 1, c >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < c / 2; ++i) {
            float send = upper ? v[i] : v[i + c / 2];
            float keep = upper ? v[i + c / 2] : v[i];
            float recv = __shfl_xor_sync(0xffffffffu, send, o);
            v[i] = MAX ? fmaxf(keep, recv) : keep + recv;
        }
    }
    return v[0];
}

// Column reduction over all 32 lanes; lane n (and n + 16 when NQ = 16) ends with column n.
template <int NQ, bool MAX>
__device__ __forceinline__ float column_reduce32(float (&v)[NQ], int lane) {
    float r = transpose_reduce<NQ, MAX>(v, lane);
    if constexpr (NQ == 16) {
        const float o = __shfl_xor_sync(0xffffffffu, r, 16);
        r = MAX ? fmaxf(r, o) : r + o;
    }
    return r;
}

// Barrier over the 128 threads of one softmax warpgroup (ids 1 and 2).
__device__ __forceinline__ void wg_bar(int wg) {
    asm volatile("bar.sync %0, 128;" ::"r"(1 + wg) : "memory");
}

// Same barrier, returning whether the predicate was true in any of the 128 threads.
__device__ __forceinline__ bool wg_bar_any(int wg, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(1 + wg)
        : "memory");
    return r != 0;
}

// Score of column n in log2 units, or -inf where the token is masked: not a
// real token, or (s_q = 2) the newest token hidden from the first query token,
// whose columns are n < G.
__device__ __forceinline__ float score_of(uint32_t raw, int n, bool tok_ok, bool hide_low, int G,
                                          float scale_log2) {
    return (tok_ok && !(hide_low && n < G)) ? __uint_as_float(raw) * scale_log2 : -INFINITY;
}

// P = 2^(score - m) in bf16 into this thread's P^T row (MN-major, 32B/64B-swizzled);
// ps receives the rounded probabilities.
template <int NQ>
__device__ __forceinline__ void write_p(const uint32_t (&sv)[NQ], const float *mrow,
                                        float (&ps)[NQ], bool tok_ok, bool hide_low, int G,
                                        float scale_log2, uint8_t *pbuf, int tok) {
#pragma unroll
    for (int n = 0; n < NQ; n += 8) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            const float x0 = score_of(sv[n + e], n + e, tok_ok, hide_low, G, scale_log2);
            const float x1 = score_of(sv[n + e + 1], n + e + 1, tok_ok, hide_low, G, scale_log2);
            // the column maxima are the same for every thread: broadcast shared-memory reads
            const float2 mm = *reinterpret_cast<const float2 *>(mrow + n + e);
            const float m0 = mm.x == -INFINITY ? 0.0f : mm.x;
            const float m1 = mm.y == -INFINITY ? 0.0f : mm.y;
            const float p0 = x0 == -INFINITY ? 0.0f : fast_exp2(x0 - m0);
            const float p1 = x1 == -INFINITY ? 0.0f : fast_exp2(x1 - m1);
            __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
            w[e / 2] = *reinterpret_cast<uint32_t *>(&h2);
            const float2 back = __bfloat1622float2(h2);
            ps[n + e] = back.x;
            ps[n + e + 1] = back.y;
        }
        *reinterpret_cast<uint4 *>(pbuf + swz(tok * NQ * 2 + n * 2, NQ * 2)) =
            make_uint4(w[0], w[1], w[2], w[3]);
    }
}

template <int NQ, bool SPARSE>
__global__ void __launch_bounds__(kThreads, 1)
    decode_gqa_tc_kernel(const __grid_constant__ CUtensorMap kv_map,
                         const __grid_constant__ CUtensorMap kr_map,
                         const __grid_constant__ CUtensorMap q_map,
                         const __grid_constant__ CUtensorMap kv_rows_map,
                         const __grid_constant__ CUtensorMap kr_rows_map, const GqaParams p) {
    using SM = GqaSmem<NQ>;
    constexpr int KS = SM::kKSlots, VS = SM::kVSlots;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::oBar);
    uint64_t *k_full = bars, *k_empty = bars + KS;
    uint64_t *v_full = bars + 2 * KS, *v_empty = v_full + VS;
    uint64_t *kr_full = v_empty + VS, *kr_empty = kr_full + 2;
    uint64_t *s_full = kr_empty + 2, *s_free = s_full + 4;
    uint64_t *p_full = s_free + 4, *p_free = p_full + 2, *o_done = p_free + 2;
    uint64_t *drain = o_done + 2;  // [0] score issuer, [1] PV issuer
    uint32_t *tmem_base_smem = reinterpret_cast<uint32_t *>(smem + SM::oMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + SM::oMisc + 4);
    int *plan = reinterpret_cast<int *>(smem + SM::oMisc + 8);
    GQLA_PROF_DECL;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x;
    const int gbase = blockIdx.y * p.NG;  // this CTA's first group
    const int real_cols = p.G * p.s_q;

    if (threadIdx.x == 0) {
        for (int i = 0; i < KS; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1); }
        for (int i = 0; i < VS; ++i) { mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1); }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&kr_full[i], 1); mbar_init(&kr_empty[i], 1);
            mbar_init(&p_full[i], 128); mbar_init(&p_free[i], 1); mbar_init(&o_done[i], 1);
            mbar_init(&drain[i], 1);
        }
        for (int i = 0; i < 4; ++i) { mbar_init(&s_full[i], 1); mbar_init(&s_free[i], 128); }
        *abort_flag = 0;
        fence_barrier_init();
    }
    griddep_wait();  // the previous kernel's results are visible from here on
    griddep_launch_dependents();
    if (warp == 0) {
        int total = warp_total_pages(p.seqlens, p.batch);
        int k = chunk_pages(total, p.num_splits);
        int r0 = c * k, r1 = min(total, r0 + k);
        int b = p.batch, start = 0;
        if (r0 < r1) warp_find_sequence(p.seqlens, p.batch, r0, &b, &start);
        if (lane == 0) {
            plan[0] = r0; plan[1] = r1; plan[2] = b; plan[3] = start;
            // the producer's first reads after the CTA's set-up: the descriptors and the
            // first pages' page-table entries, headed for L2 now
            prefetch_tensormap(SPARSE ? &kv_rows_map : &kv_map);
            prefetch_tensormap(SPARSE ? &kr_rows_map : &kr_map);
            prefetch_tensormap(&q_map);
            if (b < p.batch) prefetch_l2(p.page_table + (int64_t)b * p.max_pages + (r0 - start));
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_base_smem, 512);
        tmem_relinquish();
        tc_fence_before();
    }
    if (real_cols < NQ) {  // q rows past G*s_q are never written by TMA: zero them once
        const int pad = NQ - real_cols;
        for (int i = threadIdx.x; i < KS * 3 * pad * 8; i += kThreads) {
            const int slot = i / (3 * pad * 8), rem = i % (3 * pad * 8);
            const int blk = rem / (pad * 8), rr = rem % (pad * 8);
            *reinterpret_cast<uint4 *>(smem + SM::oK + slot * SM::kKSlotBytes + SM::kKBytes +
                                       blk * NQ * 128 + (real_cols + rr / 8) * 128 + (rr % 8) * 16) =
                make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_smem;
    const uint32_t t_s = tmem;            // S^T buffers: 4 x NQ columns, one token per lane
    const uint32_t t_o = tmem + 4 * NQ;   // O^T_g: NQ columns per group, one dv per lane
    const PieceIter it0{plan[2], plan[3], plan[0], plan[1]};

    const uint32_t sm_k = smem_u32(smem + SM::oK);
    const uint32_t sm_v = smem_u32(smem + SM::oV);
    const uint32_t sm_kr = smem_u32(smem + SM::oKr);
    const uint32_t sm_p = smem_u32(smem + SM::oP);

    // Register split: each warpgroup changes its register budget once, at the top of its
    // branch.  Warpgroup 0 gives registers up before it waits on anything, so the softmax
    // warpgroups' increase never waits on a warp that waits on them.
    if (warp < 4) {
        regs_decrease<NQ>();
        if (warp == 0 && SPARSE) {
            // ---------------------------------------------------------------- TMA producer, sparse
            // The same units and rings as below; the rows of a unit are gathered four at a
            // time (tile::gather4): lane l takes rows 4 (l % 16) .. + 3 of page l / 16 of the
            // unit's pair, for K_nope_g, V_g and the pair's RoPE keys.  Lane 0 waits for
            // the slots and sets each barrier's byte count before the warp issues.
            if (lane == 0) {
                prefetch_tensormap(&kv_rows_map);
                prefetch_tensormap(&kr_rows_map);
                prefetch_tensormap(&q_map);
            }
            const uint32_t q_bytes = 3u * 128u * (uint32_t)real_cols;
            const uint64_t stream_policy = l2_evict_first_policy();
            const int half = lane >> 4, r0 = 4 * (lane & 15);
            UnitCursor kc, vc;
            kc.start(p, it0);
            vc.start(p, it0);
            uint32_t kpos = 0, vpos = 0, pc = 0;
            int4 ksl = make_int4(-1, -1, -1, -1), vsl = ksl;  // this lane's four cache slots
            auto pair_slots = [&](const UnitCursor &cur) {
                const int page = half ? cur.pp.page1 : cur.pp.page0;
                return page < 0 ? make_int4(-1, -1, -1, -1)
                                : *reinterpret_cast<const int4 *>(p.sel_slot + (int64_t)page * kPage + r0);
            };
            auto row_of = [&](int slot, int gi) { return slot < 0 ? -1 : (gbase + gi) * p.real_slots + slot; };
            long long idle_since = clock64();
            while (kc.valid || vc.valid) {  // warp-uniform: every decision is lane 0's, broadcast
                bool progressed = false;
                const int aborted = __shfl_sync(0xffffffffu, (int)*abort_flag, 0);
                if (kc.valid && !aborted) {
                    const int ks = kpos % KS, kb = pc & 1;
                    const bool need_kr = kc.gi == 0;
                    int ready = 0;
                    if (lane == 0)
                        ready = (!need_kr || mbar_test_wait(&kr_empty[kb], ((pc >> 1) & 1) ^ 1)) &&
                                mbar_test_wait(&k_empty[ks], ((kpos / KS) & 1) ^ 1);
                    if (__shfl_sync(0xffffffffu, ready, 0)) {
                        if (need_kr) ksl = pair_slots(kc);  // the first unit of a pair
                        const PagePair &pp = kc.pp;
                        const int np = (pp.page0 >= 0) + (pp.page1 >= 0);
                        const bool mine = half ? pp.page1 >= 0 : pp.page0 >= 0;
                        if (need_kr) {
                            uint8_t *dst = smem + SM::oKr + kb * SM::kKrBytes;
                            if (lane == 0) {
                                if (np) mbar_arrive_expect_tx(&kr_full[kb], np * kBox);
                                else mbar_arrive(&kr_full[kb]);
                            }
                            __syncwarp();
                            if (mine)
                                tma_gather4_hint(dst + half * kBox + r0 * 128, &kr_rows_map, &kr_full[kb], 0,
                                                 ksl.x, ksl.y, ksl.z, ksl.w, stream_policy);
                            ++pc;
                        }
                        uint8_t *dst = smem + SM::oK + ks * SM::kKSlotBytes;
                        if (lane == 0) {
                            mbar_arrive_expect_tx(&k_full[ks], np * 2 * kBox + q_bytes);
#pragma unroll
                            for (int cb = 0; cb < 3; ++cb)  // q_g rows of this query token
                                tma_load_3d(dst + SM::kKBytes + cb * NQ * 128, &q_map, &k_full[ks], cb * 64,
                                            (gbase + kc.gi) * p.G, kc.b * p.s_q);
                        }
                        __syncwarp();
                        if (mine) {
#pragma unroll
                            for (int cb = 0; cb < 2; ++cb)  // K_nope lo / hi
                                tma_gather4_hint(dst + cb * 2 * kBox + half * kBox + r0 * 128, &kv_rows_map, &k_full[ks],
                                                 cb * 64, row_of(ksl.x, kc.gi), row_of(ksl.y, kc.gi),
                                                 row_of(ksl.z, kc.gi), row_of(ksl.w, kc.gi), stream_policy);
                        }
                        kc.advance(p);
                        ++kpos;
                        progressed = true;
                    }
                }
                if (vc.valid && vpos < kpos && !aborted) {
                    const int vs = vpos % VS;
                    int ready = 0;
                    if (lane == 0) ready = mbar_test_wait(&v_empty[vs], ((vpos / VS) & 1) ^ 1);
                    if (__shfl_sync(0xffffffffu, ready, 0)) {
                        if (vc.gi == 0) vsl = pair_slots(vc);
                        const PagePair &pp = vc.pp;
                        const int np = (pp.page0 >= 0) + (pp.page1 >= 0);
                        const bool mine = half ? pp.page1 >= 0 : pp.page0 >= 0;
                        uint8_t *dst = smem + SM::oV + vs * SM::kVBytes;
                        if (lane == 0) {
                            if (np) mbar_arrive_expect_tx(&v_full[vs], np * 2 * kBox);
                            else mbar_arrive(&v_full[vs]);
                        }
                        __syncwarp();
                        if (mine) {
#pragma unroll
                            for (int cb = 0; cb < 2; ++cb)  // V lo / hi
                                tma_gather4_hint(dst + cb * 2 * kBox + half * kBox + r0 * 128, &kv_rows_map, &v_full[vs],
                                                 128 + cb * 64, row_of(vsl.x, vc.gi), row_of(vsl.y, vc.gi),
                                                 row_of(vsl.z, vc.gi), row_of(vsl.w, vc.gi), stream_policy);
                        }
                        vc.advance(p);
                        ++vpos;
                        progressed = true;
                    }
                }
                int give_up = 0;
                if (lane == 0 && !progressed) give_up = aborted || clock64() - idle_since > kWaitCycles;
                if (progressed) {
                    idle_since = clock64();
                } else if (!__shfl_sync(0xffffffffu, give_up, 0)) {
                    __nanosleep(20);
                } else {
                    if (lane == 0) *abort_flag = 1;  // give up: the consumers stop waiting on us as well
                    break;
                }
            }
            // never leave with copies in flight: wait (bounded) for the last loads issued
            if (lane == 0) {
                int dummy = 0;
                volatile int *no_abort = reinterpret_cast<volatile int *>(&dummy);
                for (uint32_t u = (kpos > (uint32_t)KS ? kpos - KS : 0); u < kpos; ++u)
                    mbar_wait(&k_full[u % KS], (u / KS) & 1, no_abort);
                for (uint32_t u = (vpos > (uint32_t)VS ? vpos - VS : 0); u < vpos; ++u)
                    mbar_wait(&v_full[u % VS], (u / VS) & 1, no_abort);
                for (uint32_t u = (pc > 2u ? pc - 2 : 0); u < pc; ++u)
                    mbar_wait(&kr_full[u & 1], (u >> 1) & 1, no_abort);
            }
        } else if (warp == 0) {
            // ---------------------------------------------------------------- TMA producer
            if (lane == 0) {
                prefetch_tensormap(&kv_map);
                prefetch_tensormap(&kr_map);
                prefetch_tensormap(&q_map);
                {
                    PieceIter it = it0;
                    int b, L, pb, pe;
                    bool too_long;
                    while (next_piece(p, it, b, L, pb, pe, too_long))
                        if (too_long) report_error(p.ws, GQLA_ERR_DEVICE, b);
                }
                const uint32_t q_bytes = 3u * 128u * (uint32_t)real_cols;
                const uint64_t stream_policy = l2_evict_first_policy();  // the cache is read once
                UnitCursor kc, vc;
                kc.start(p, it0);
                vc.start(p, it0);
                uint32_t kpos = 0, vpos = 0, pc = 0;
                // Issue whichever load has a free slot: q_g + K_g as far ahead as their ring
                // allows (with the pair's RoPE keys before its first group), V_g never ahead of K_g.
                long long idle_since = clock64();
                while (kc.valid || vc.valid) {
                    bool progressed = false;
                    if (kc.valid && !*abort_flag) {
                        const int ks = kpos % KS, kb = pc & 1;
                        const bool need_kr = kc.gi == 0;
                        if ((!need_kr || mbar_test_wait(&kr_empty[kb], ((pc >> 1) & 1) ^ 1)) &&
                            mbar_test_wait(&k_empty[ks], ((kpos / KS) & 1) ^ 1)) {
                            const PagePair &pp = kc.pp;
                            const int np = (pp.page0 >= 0) + (pp.page1 >= 0);
                            if (need_kr) {
                                if (pp.bad) report_error(p.ws, GQLA_ERR_DEVICE, kc.b);
                                uint8_t *dst = smem + SM::oKr + kb * SM::kKrBytes;
                                if (np) {
                                    mbar_arrive_expect_tx(&kr_full[kb], np * kBox);
                                    if (pp.page0 >= 0)
                                        tma_load_2d_hint(dst, &kr_map, &kr_full[kb], 0, pp.page0 * kPage, stream_policy);
                                    if (pp.page1 >= 0)
                                        tma_load_2d_hint(dst + kBox, &kr_map, &kr_full[kb], 0, pp.page1 * kPage,
                                                         stream_policy);
                                } else {
                                    mbar_arrive(&kr_full[kb]);
                                }
                                ++pc;
                            }
                            uint8_t *dst = smem + SM::oK + ks * SM::kKSlotBytes;
                            mbar_arrive_expect_tx(&k_full[ks], np * 2 * kBox + q_bytes);
#pragma unroll
                            for (int cb = 0; cb < 3; ++cb)  // q_g rows (s, hg) of this sequence
                                tma_load_3d(dst + SM::kKBytes + cb * NQ * 128, &q_map, &k_full[ks], cb * 64,
                                            (gbase + kc.gi) * p.G, kc.b * p.s_q);
#pragma unroll
                            for (int cb = 0; cb < 2; ++cb) {  // K_nope lo / hi: page 0 rows, then page 1 rows
                                if (pp.page0 >= 0)
                                    tma_load_3d_hint(dst + cb * 2 * kBox, &kv_map, &k_full[ks], cb * 64,
                                                     pp.page0 * kPage, gbase + kc.gi, stream_policy);
                                if (pp.page1 >= 0)
                                    tma_load_3d_hint(dst + cb * 2 * kBox + kBox, &kv_map, &k_full[ks], cb * 64,
                                                     pp.page1 * kPage, gbase + kc.gi, stream_policy);
                            }
                            kc.advance(p);
                            ++kpos;
                            progressed = true;
                        }
                    }
                    if (vc.valid && vpos < kpos && !*abort_flag && (int)vpos == p.drop_v_unit) {
                        vc.advance(p);  // diagnostic: no load and no arrival for this unit
                        ++vpos;
                        progressed = true;
                    } else if (vc.valid && vpos < kpos && !*abort_flag) {
                        const int vs = vpos % VS;
                        if (mbar_test_wait(&v_empty[vs], ((vpos / VS) & 1) ^ 1)) {
                            const PagePair &pp = vc.pp;
                            const int np = (pp.page0 >= 0) + (pp.page1 >= 0);
                            uint8_t *dst = smem + SM::oV + vs * SM::kVBytes;
                            if (np) {
                                mbar_arrive_expect_tx(&v_full[vs], np * 2 * kBox);
#pragma unroll
                                for (int cb = 0; cb < 2; ++cb) {
                                    if (pp.page0 >= 0)
                                        tma_load_3d_hint(dst + cb * 2 * kBox, &kv_map, &v_full[vs], 128 + cb * 64,
                                                         pp.page0 * kPage, gbase + vc.gi, stream_policy);
                                    if (pp.page1 >= 0)
                                        tma_load_3d_hint(dst + cb * 2 * kBox + kBox, &kv_map, &v_full[vs],
                                                         128 + cb * 64, pp.page1 * kPage, gbase + vc.gi, stream_policy);
                                }
                            } else {
                                mbar_arrive(&v_full[vs]);
                            }
                            vc.advance(p);
                            ++vpos;
                            progressed = true;
                        }
                    }
                    if (progressed) {
                        idle_since = clock64();
                    } else if (!*abort_flag && clock64() - idle_since <= kWaitCycles) {
                        __nanosleep(20);
                    } else {
                        *abort_flag = 1;  // give up: the consumers stop waiting on us as well
                        break;
                    }
                }
                // never leave with copies in flight: wait (bounded) for the last loads issued
                int dummy = 0;
                volatile int *no_abort = reinterpret_cast<volatile int *>(&dummy);
                for (uint32_t u = (kpos > (uint32_t)KS ? kpos - KS : 0); u < kpos; ++u)
                    mbar_wait(&k_full[u % KS], (u / KS) & 1, no_abort);
                for (uint32_t u = (vpos > (uint32_t)VS ? vpos - VS : 0); u < vpos; ++u)
                    mbar_wait(&v_full[u % VS], (u / VS) & 1, no_abort);
                for (uint32_t u = (pc > 2u ? pc - 2 : 0); u < pc; ++u)
                    mbar_wait(&kr_full[u & 1], (u >> 1) & 1, no_abort);
            }
        } else if (warp == 1) {
            // ---------------------------------------------------------------- score MMA issuer
            if (lane == 0) {
                constexpr uint32_t idesc_s = idesc_bf16(kTok, NQ, 0, 0);
                PieceIter it = it0;
                int b, L, pb, pe;
                bool too_long;
                uint32_t u = 0, pc = 0;
                while (next_piece(p, it, b, L, pb, pe, too_long)) {
                    if (too_long) continue;
                    for (int pg = pb; pg < pe; pg += 2, ++pc) {
                        const int kb = pc & 1;
                        if (!GQLA_WAIT(2, &kr_full[kb], (pc >> 1) & 1, abort_flag)) *abort_flag = 1;
                        const uint32_t kr = sm_kr + kb * SM::kKrBytes;
                        for (int gi = 0; gi < p.NG; ++gi, ++u) {
                            // S^T(u) = [K_nope_g | k^R] q_g^T into S buffer u & 3
                            const int ks_ = u % KS, sb = u & 3;
                            if (!GQLA_WAIT(3, &k_full[ks_], (u / KS) & 1, abort_flag)) *abort_flag = 1;
                            if (!GQLA_WAIT(4, &s_free[sb], ((u >> 2) & 1) ^ 1, abort_flag)) *abort_flag = 1;
                            tc_fence_after();
                            // descriptors from the slot bases: each MMA only adds an offset
                            const uint64_t k_d = smem_desc(sm_k + ks_ * SM::kKSlotBytes, 16, 1024, kSw128);
                            const uint64_t q_d = desc_advance(k_d, SM::kKBytes);
                            const uint64_t kr_d = smem_desc(kr, 16, 1024, kSw128);
                            if (!*abort_flag) {
#pragma unroll
                                for (int ks = 0; ks < 12; ++ks) {
                                    const uint64_t ad = ks < 8 ? desc_advance(k_d, (ks >> 2) * 2 * kBox + (ks & 3) * 32)
                                                               : desc_advance(kr_d, (ks - 8) * 32);
                                    const uint64_t bd = desc_advance(q_d, (ks >> 2) * NQ * 128 + (ks & 3) * 32);
                                    mma_bf16(t_s + sb * NQ, ad, bd, idesc_s, ks > 0 ? 1u : 0u);
                                }
                            }
                            mma_commit(&s_full[sb]);
                            mma_commit(&k_empty[ks_]);
                            if (gi == p.NG - 1) mma_commit(&kr_empty[kb]);
                        }
                    }
                }
                // drain: nothing may still be running when TMEM is freed
                mma_commit(&drain[0]);
                int dummy = 0;
                mbar_wait(&drain[0], 0, reinterpret_cast<volatile int *>(&dummy));
            }
        } else if (warp == 2) {
            // ---------------------------------------------------------------- PV MMA issuer
            // O^T_g(u) (+)= V_g^T P^T(u), in unit order, as soon as the owning warpgroup
            // has published P^T(u) and V_g(u) has landed; no softmax warp waits for V.
            if (lane == 0) {
                constexpr uint32_t idesc_pv = idesc_bf16(128, NQ, 1, 1);
                constexpr uint32_t p_sw = NQ == 16 ? kSw32 : kSw64;
                constexpr uint32_t p_sbo = NQ == 16 ? 256 : 512;
                const uint64_t v_d0 = smem_desc(sm_v, 2 * kBox, 1024, kSw128);
                const uint64_t p_d0 = smem_desc(sm_p, SM::kPBytes, p_sbo, p_sw);
                PieceIter it = it0;
                int b, L, pb, pe;
                bool too_long;
                uint32_t u = 0;
                while (next_piece(p, it, b, L, pb, pe, too_long)) {
                    if (too_long) continue;
                    const int npairs = (pe - pb + 1) >> 1;
                    for (int ip = 0; ip < npairs; ++ip) {
                        for (int gi = 0; gi < p.NG; ++gi, ++u) {
                            const int w = gi & 1, vs = u % VS;
                            if (!GQLA_WAIT(5, &p_full[w], wg_unit(u, p.NG) & 1, abort_flag)) *abort_flag = 1;
                            if (!GQLA_WAIT(13, &v_full[vs], (u / VS) & 1, abort_flag)) *abort_flag = 1;
                            tc_fence_after();
                            const uint64_t v_d = desc_advance(v_d0, vs * SM::kVBytes);
                            const uint64_t p_d = desc_advance(p_d0, w * SM::kPBytes);
                            if (!*abort_flag) {
#pragma unroll
                                for (int ks = 0; ks < kTok / 16; ++ks)
                                    mma_bf16(t_o + gi * NQ, desc_advance(v_d, ks * 2048), desc_advance(p_d, ks * 16 * NQ * 2),
                                             idesc_pv, (ip == 0 && ks == 0) ? 0u : 1u);
                            }
                            mma_commit(&p_free[w]);
                            mma_commit(&v_empty[vs]);
                        }
                    }
                    mma_commit(&o_done[0]);
                    mma_commit(&o_done[1]);
                }
                mma_commit(&drain[1]);
                int dummy = 0;
                mbar_wait(&drain[1], 0, reinterpret_cast<volatile int *>(&dummy));
            }
        }
        // warp 3 is idle: it completes warpgroup 0 for the register split
    } else {
        regs_increase<NQ>();
        // ---------------------------------------------------------------- softmax, PV, epilogue
        // Warpgroup wg owns the groups gi = wg, wg + 2, ... (units of
        // one parity), so the two warpgroups never share a group.
        const int wg = (warp - 4) >> 2;        // 0 or 1
        const int wq = (warp - 4) & 3;         // warp within the warpgroup
        const int quad = warp & 3;             // TMEM lane quadrant of this warp
        const int wtid = (threadIdx.x - 128) & 127;
        const int tok = 32 * quad + lane;      // this thread's token row in a unit (and dv row of O^T)
        const uint32_t lane_off = static_cast<uint32_t>(32 * quad) << 16;
        float *red = reinterpret_cast<float *>(smem + SM::oRed) + wg * NQ * 4;
        float *mrun = reinterpret_cast<float *>(smem + SM::oMrun);
        float *lred = reinterpret_cast<float *>(smem + SM::oLred);
        uint8_t *pbuf = smem + SM::oP + wg * SM::kPBytes;
        float *inv_l = reinterpret_cast<float *>(smem + SM::oEpi) + wg * 2 * NQ;  // [NQ] 1/l, [NQ] lse
        PieceIter it = it0;
        int b, L, pb, pe;
        bool too_long;
        uint32_t j = 0, k = 0;
        while (next_piece(p, it, b, L, pb, pe, too_long)) {
            if (too_long) continue;
            const int npairs = (pe - pb + 1) >> 1;
            for (int ip = 0; ip < npairs; ++ip) {
                const int pg = pb + 2 * ip;
                const PagePair pp = load_pair(p, b, L, pg, pe);
                const bool tok_ok = tok < 64 ? tok < pp.rows0 : tok - 64 < pp.rows1;
                const bool partial = pp.rows0 < 64 || pp.rows1 < 64;
                // query s sees token t iff t <= L - s_q + s; columns are n = s*G + hg, so with
                // s_q <= 2 only the last token can be hidden, and only from columns n < G
                const bool hide_low = pg * kPage + tok - (L - p.s_q) > 0;
#pragma unroll 1
                for (int gl = 0; gl < wg_groups(p.NG, wg); ++gl) {
                    const int gi = 2 * gl + wg;
                    const uint32_t jj = j + ip * p.NG + gi;
                    // lane n (< NQ) keeps the column-n sum over this warp's tokens in shared memory
                    float *lw = lred + (gi * NQ + (lane & (NQ - 1))) * 4 + wq;
                    const int sb = jj & 3;
                    GQLA_SPAN_BEGIN(t_unit);
                    if (!GQLA_WAIT(6, &s_full[sb], (jj >> 2) & 1, abort_flag)) *abort_flag = 1;
                    tc_fence_after();
                    uint32_t sv[NQ];
                    GQLA_SPAN_BEGIN(t_ld);
                    tmem_ld16(t_s + lane_off + sb * NQ, sv);
                    if constexpr (NQ == 32) tmem_ld16(t_s + lane_off + sb * NQ + 16, sv + 16);
                    // the group's running column maxima stay in shared memory (read by every
                    // thread alike), not in NQ registers
                    const float *mrow = mrun + gi * NQ;
                    tmem_wait_ld();
                    GQLA_SPAN_END(11, t_ld);
                    tc_fence_before();
                    mbar_arrive(&s_free[sb]);
                    bool exceed = ip == 0;
#pragma unroll
                    for (int n = 0; n < NQ; ++n)
                        exceed |= score_of(sv[n], n, tok_ok, hide_low, p.G, p.scale_log2) > mrow[n] + kRescaleLog2;
                    // the P^T buffer (and O^T_g) are free once this warpgroup's previous PV completed
                    if (!GQLA_WAIT(7, &p_free[wg], (wg_unit(jj, p.NG) & 1) ^ 1, abort_flag)) *abort_flag = 1;
                    tc_fence_after();
                    float ps[NQ];
                    GQLA_SPAN_BEGIN(t_wp);
                    if (ip > 0)  // optimistic: P against the running maxima
                        write_p<NQ>(sv, mrow, ps, tok_ok, hide_low, p.G, p.scale_log2, pbuf, tok);
                    GQLA_SPAN_END(12, t_wp);
                    const int vs = jj % VS;
                    if (partial) {  // V rows that are not tokens (never written, maybe NaN) -> 0
                        if (!GQLA_WAIT(8, &v_full[vs], (jj / VS) & 1, abort_flag)) *abort_flag = 1;
                        uint8_t *vbase = smem + SM::oV + vs * SM::kVBytes;
                        const int n0 = 64 - pp.rows0, n1 = 64 - pp.rows1;
                        for (int i = wtid; i < 2 * (n0 + n1) * 8; i += 128) {
                            const int cb = i / ((n0 + n1) * 8), rem = i % ((n0 + n1) * 8);
                            const int r = rem / 8;
                            const int row = r < n0 ? pp.rows0 + r : 64 + pp.rows1 + (r - n0);
                            *reinterpret_cast<uint4 *>(vbase + cb * 2 * kBox + row * 128 + (rem % 8) * 16) =
                                make_uint4(0, 0, 0, 0);
                        }
                    }
                    GQLA_SPAN_BEGIN(t_fence);
                    fence_proxy_async_smem();
                    tc_fence_before();
                    GQLA_SPAN_END(15, t_fence);
                    GQLA_SPAN_BEGIN(t_vote);
                    const bool slow = wg_bar_any(wg, exceed);
                    GQLA_SPAN_END(9, t_vote);
                    if (slow) {  // uniform over the warpgroup: new column maxima for this tile
                        GQLA_SPAN_BEGIN(t_slow);
                        {
                            float t[NQ];
#pragma unroll
                            for (int n = 0; n < NQ; ++n) t[n] = score_of(sv[n], n, tok_ok, hide_low, p.G, p.scale_log2);
                            const float m = column_reduce32<NQ, true>(t, lane);
                            if (lane < NQ) red[lane * 4 + wq] = m;
                        }
                        wg_bar(wg);
                        // the new maxima, one column per thread, into mnew (the epilogue's
                        // scratch, free during the units); the barrier publishes them and
                        // tells every thread whether any column changed
                        float *mnew = inv_l;
                        bool changed = false;
                        if (wtid < NQ) {
                            const float4 r4 = *reinterpret_cast<const float4 *>(red + wtid * 4);
                            const float mt = fmaxf(fmaxf(r4.x, r4.y), fmaxf(r4.z, r4.w));
                            const float mold = mrow[wtid];
                            const float mn = ip == 0 ? mt : ((mt > mold + kRescaleLog2) ? mt : mold);
                            changed = ip > 0 && mn != mold;
                            mnew[wtid] = mn;
                        }
                        const bool need = wg_bar_any(wg, changed);
                        tc_fence_after();
                        if (need) {  // O^T_g columns *= 2^(m_old - m_new)
                            const uint32_t to = t_o + gi * NQ + lane_off;
#pragma unroll
                            for (int h16 = 0; h16 < NQ; h16 += 16) {
                                uint32_t r[16];
                                tmem_ld16(to + h16, r);
                                tmem_wait_ld();
#pragma unroll
                                for (int e = 0; e < 16; ++e) {
                                    const float mold = mrow[h16 + e], mn = mnew[h16 + e];
                                    const float a = mold == mn ? 1.0f : exp2f(mold - mn);
                                    r[e] = __float_as_uint(__uint_as_float(r[e]) * a);
                                }
                                tmem_st16(to + h16, r);
                            }
                            tmem_wait_st();
                        }
                        if (lane < NQ) {  // this lane's own column partial follows the same rescale
                            const float mold = mrow[lane], mn = mnew[lane];
                            *lw = ip == 0 ? 0.0f : (mn == mold ? *lw : *lw * exp2f(mold - mn));
                        }
                        write_p<NQ>(sv, mnew, ps, tok_ok, hide_low, p.G, p.scale_log2, pbuf, tok);
                        fence_proxy_async_smem();
                        tc_fence_before();
                        wg_bar(wg);  // P^T complete; everyone has read mrun / mnew / red
                        if (wtid < NQ) mrun[gi * NQ + wtid] = mnew[wtid];
                        GQLA_SPAN_END(17, t_slow);
                    }
                    mbar_arrive(&p_full[wg]);
                    // column sums of the rounded probabilities over this warp's tokens
                    GQLA_SPAN_BEGIN(t_sum);
                    {
                        const float l = column_reduce32<NQ, false>(ps, lane);
                        if (lane < NQ) *lw += l;
                    }
                    GQLA_SPAN_END(16, t_sum);
                    GQLA_SPAN_END(10, t_unit);
                }
            }
            j += npairs * p.NG;
            GQLA_SPAN_BEGIN(t_epi);
            // ---- epilogue: normalise O^T and write the partials of slot b + c
            if (!GQLA_WAIT(14, &o_done[wg], k & 1, abort_flag)) *abort_flag = 1;
            tc_fence_after();
            wg_bar(wg);  // all column partials of this warpgroup are in lred
            const int slot = b + c;
            const int dv = tok;
            // a piece that is its sequence's only one (all its pages in this chunk) is the
            // result itself: with final outputs given it goes there, in bf16, and no partial
            // is written (the combine then leaves the sequence alone)
            const bool final_out = p.out != nullptr && pb == 0 && pe == pages_of(L);
            // rows of the partial for columns n = s*G + hg: ((slot*s_q + s)*h + g*G + hg);
            // rows of the final output: ((b*s_q + s)*h + g*G + hg)
            const int64_t row_s0 = (int64_t)(final_out ? b : slot) * p.s_q * p.heads;
#pragma unroll 1
            for (int gl = 0; gl < wg_groups(p.NG, wg); ++gl) {
                const int gi = 2 * gl + wg;
                if (wtid < NQ) {  // per column: 1 / l and the natural-log LSE
                    const float4 l4 = *reinterpret_cast<const float4 *>(lred + (gi * NQ + wtid) * 4);
                    const float l = (l4.x + l4.y) + (l4.z + l4.w);
                    const float m = mrun[gi * NQ + wtid];
                    const bool ok = l > 0.0f && m != -INFINITY;
                    inv_l[wtid] = ok ? 1.0f / l : 0.0f;
                    inv_l[NQ + wtid] = ok ? (m + __log2f(l)) * 0.6931471805599453f : -INFINITY;
                    if (wtid < real_cols) {
                        const int s = wtid / p.G, hg = wtid - s * p.G;
                        float *lse_dst = final_out ? p.lse_out : p.lse_part;
                        if (lse_dst) lse_dst[row_s0 + (int64_t)s * p.heads + (gbase + gi) * p.G + hg] = inv_l[NQ + wtid];
                    }
                }
                wg_bar(wg);  // inv_l ready
                GQLA_SPAN_BEGIN(t_est);
                // O^T row dv of column n = s*G + hg goes to row (s*h + g*G + hg)
                const int64_t row_g = row_s0 + (int64_t)(gbase + gi) * p.G;
                if constexpr (NQ == 16) {
                    // 16 columns: straight from registers, one 4-byte store per column (the
                    // 32 lanes of a warp write 128 contiguous bytes of a row)
                    float *dst_p = p.o_part + row_g * kDv + dv;
                    __nv_bfloat16 *dst_o = final_out ? p.out + row_g * kDv + dv : nullptr;
                    int s = 0, hg = 0;
                    uint32_t r[16];
                    tmem_ld16(t_o + gi * NQ + lane_off, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        if (e < real_cols) {
                            const int64_t off = ((int64_t)s * p.heads + hg) * kDv;
                            const float v = __uint_as_float(r[e]) * inv_l[e];
                            if (dst_o) dst_o[off] = __float2bfloat16_rn(v);
                            else dst_p[off] = v;
                        }
                        if (++hg == p.G) { hg = 0; ++s; }
                    }
                } else {
                    // 32 columns: through the warpgroup's P^T buffer (free: all its PVs are
                    // done) 16 columns at a time: each thread writes its dv of every column
                    // there, then the warpgroup stores whole 16-byte pieces of the rows
                    // (coalesced, a quarter of the store count)
                    constexpr int kCC = SM::kPBytes / (kDv * 4);  // columns per round: 16
                    float *stg = reinterpret_cast<float *>(pbuf);  // [kCC][kDv] fp32
#pragma unroll 1
                    for (int h16 = 0; h16 < NQ; h16 += 16) {
                        uint32_t r[16];
                        tmem_ld16(t_o + gi * NQ + lane_off + h16, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int c0 = 0; c0 < 16; c0 += kCC) {
#pragma unroll
                            for (int e = 0; e < kCC; ++e)
                                stg[e * kDv + dv] = __uint_as_float(r[c0 + e]) * inv_l[h16 + c0 + e];
                            wg_bar(wg);
#pragma unroll
                            for (int i = wtid; i < kCC * (kDv / 4); i += 128) {
                                const int n = h16 + c0 + i / (kDv / 4), q4 = i % (kDv / 4);
                                if (n < real_cols) {
                                    const int sn = n / p.G, hn = n - sn * p.G;
                                    const int64_t row = row_g + (int64_t)sn * p.heads + hn;
                                    const float4 v = reinterpret_cast<const float4 *>(stg)[i];
                                    if (final_out)
                                        reinterpret_cast<uint2 *>(p.out + row * kDv)[q4] = pack_bf16x4(v.x, v.y, v.z, v.w);
                                    else
                                        reinterpret_cast<float4 *>(p.o_part + row * kDv)[q4] = v;
                                }
                            }
                            wg_bar(wg);  // the staging is rewritten by the next round
                        }
                    }
                }
                GQLA_SPAN_END(19, t_est);
                wg_bar(wg);  // inv_l is rewritten for the next group
            }
            tc_fence_before();
            GQLA_SPAN_BEGIN(t_ebar);
            wg_bar(wg);  // lred / mrun are reused by the next piece
            GQLA_SPAN_END(20, t_ebar);
            GQLA_SPAN_END(21, t_epi);
            ++k;
        }
        if (p.out != nullptr && c == 0) {
            // sequences with no token have no piece: with final outputs given, the CTAs of
            // chunk 0 write out = 0 and lse = -inf for their groups' heads (one thread per
            // sequence)
            const int hcols = p.NG * p.G;  // this CTA's heads
            for (int b2 = threadIdx.x - 128; b2 < p.batch; b2 += 256) {
                if (p.seqlens[b2] != 0) continue;
                for (int s = 0; s < p.s_q; ++s) {
                    const int64_t row0 = ((int64_t)b2 * p.s_q + s) * p.heads + (int64_t)gbase * p.G;
                    for (int i = 0; i < hcols * (kDv / 8); ++i)
                        *reinterpret_cast<uint4 *>(p.out + (row0 + i / (kDv / 8)) * kDv + (i % (kDv / 8)) * 8) =
                            make_uint4(0, 0, 0, 0);
                    if (p.lse_out)
                        for (int i = 0; i < hcols; ++i) p.lse_out[row0 + i] = -INFINITY;
                }
            }
        }
    }

    GQLA_PROF_FLUSH;
    __syncthreads();
    if (*abort_flag && threadIdx.x == 0) report_error(p.ws, GQLA_ERR_TIMEOUT, c);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------
// Host side: tensor maps (driver entry point obtained through the runtime, so
// the library does not link libcuda) and the launch.

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

bool make_map(CUtensorMap *map, const void *base, int rank, const cuuint64_t *dims,
              const cuuint64_t *strides_bytes, const cuuint32_t *box) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), dims,
                    strides_bytes, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int NQ, bool SPARSE>
cudaError_t launch_nq_mode(const CUtensorMap &kvm, const CUtensorMap &krm, const CUtensorMap &qm,
                           const CUtensorMap &kvrm, const CUtensorMap &krrm, const GqaParams &p,
                           int group_splits, cudaStream_t stream) {
    const int bytes = GqaSmem<NQ>::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(decode_gqa_tc_kernel<NQ, SPARSE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    // the register split asks for 128 x kIssue + 256 x kSoftmax registers: the
    // launch must give at least that many, or the kernel's increase would never return
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, decode_gqa_tc_kernel<NQ, SPARSE>);
    if (e != cudaSuccess) return e;
    if (128 * RegSplit<NQ>::kIssue + 256 * RegSplit<NQ>::kSoftmax > kThreads * fa.numRegs)
        return cudaErrorInvalidConfiguration;
    return launch_dependent(decode_gqa_tc_kernel<NQ, SPARSE>, dim3(p.num_splits, group_splits), dim3(kThreads),
                            bytes, stream, kvm, krm, qm, kvrm, krrm, p);
}

template <int NQ>
cudaError_t launch_nq(const CUtensorMap &kvm, const CUtensorMap &krm, const CUtensorMap &qm,
                      const GqaParams &p, int group_splits, cudaStream_t stream) {
    return launch_nq_mode<NQ, false>(kvm, krm, qm, kvm, krm, p, group_splits, stream);  // no row maps in dense mode
}

}  // namespace

// CTAs per chunk: a batch too small to fill the GPU with one CTA per chunk has its groups
// split over up to g CTAs per chunk (each reads the chunk's RoPE keys again: 128 of the
// 4224 bytes of a token per extra CTA), as long as two such grids still fit in one wave.
int group_splits_rule(int num_splits, int num_groups, int sms) {
    int gs = 1;
    while (gs < num_groups && (int64_t)num_splits * gs * 4 <= sms) gs *= 2;
    return gs;
}

int group_splits_for(int num_splits, int num_groups) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return group_splits_rule(num_splits, num_groups, sms);
}

// Set by gqla_debug_drop_v_load, consumed by the next GQA decode launch of the thread.
thread_local int g_drop_v_unit = -1;

cudaError_t launch_decode_gqa(const void *q, int s_q, int heads, int num_groups, const void *kv,
                              const void *k_rope, int64_t num_slots, const gqla_kv_index *idx,
                              int num_splits, float scale, float *o_part, float *lse_part,
                              void *out, float *lse_out, void *ws, cudaStream_t stream) {
    if (num_groups != 8 && num_groups != 4 && num_groups != 2 && num_groups != 1) return cudaErrorInvalidValue;
    const int G = heads / num_groups;
    CUtensorMap kvm, krm, qm;
    {
        cuuint64_t dims[3] = {256, (cuuint64_t)num_slots, (cuuint64_t)num_groups};
        cuuint64_t strides[2] = {256 * 2, (cuuint64_t)num_slots * 256 * 2};
        cuuint32_t box[3] = {64, 64, 1};
        if (!make_map(&kvm, kv, 3, dims, strides, box)) return cudaErrorInvalidValue;
    }
    {
        cuuint64_t dims[2] = {64, (cuuint64_t)num_slots};
        cuuint64_t strides[1] = {64 * 2};
        cuuint32_t box[2] = {64, 64};
        if (!make_map(&krm, k_rope, 2, dims, strides, box)) return cudaErrorInvalidValue;
    }
    {  // q [batch * s_q][heads][192]: a box is the G heads of one group for all s_q tokens
        cuuint64_t dims[3] = {(cuuint64_t)kQk, (cuuint64_t)heads, (cuuint64_t)idx->batch * s_q};
        cuuint64_t strides[2] = {(cuuint64_t)kQk * 2, (cuuint64_t)heads * kQk * 2};
        cuuint32_t box[3] = {64, (cuuint32_t)G, (cuuint32_t)s_q};
        if (!make_map(&qm, q, 3, dims, strides, box)) return cudaErrorInvalidValue;
    }
    GqaParams p;
    p.page_table = idx->page_table;
    p.seqlens = idx->seqlens;
    p.o_part = o_part;
    p.lse_part = lse_part;
    p.ws = ws;
    p.batch = idx->batch;
    p.max_pages = idx->max_pages_per_seq;
    p.num_pages = idx->num_pages;
    p.num_splits = num_splits;
    p.s_q = s_q;
    p.heads = heads;
    p.G = G;
    const int gs = group_splits_for(num_splits, num_groups);
    p.NG = num_groups / gs;
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.lse_out = lse_out;
    p.scale_log2 = scale * kLog2e;
    p.sel_slot = nullptr;
    p.real_slots = 0;
    p.drop_v_unit = g_drop_v_unit;
    g_drop_v_unit = -1;
    return G * s_q <= 16 ? launch_nq<16>(kvm, krm, qm, p, gs, stream)
                         : launch_nq<32>(kvm, krm, qm, p, gs, stream);
}

// Sparse GQLA: the decode over a selection (sel: batch * s_q one-token sequences over
// an identity page table), gathering each selected row straight from the cache.
cudaError_t launch_decode_gqa_sparse(const void *q, int heads, int num_groups, const void *kv,
                                     const void *k_rope, int64_t real_slots, const gqla_kv_index *sel,
                                     const int32_t *sel_slot, int num_splits, float scale, float *o_part,
                                     float *lse_part, void *ws, cudaStream_t stream) {
    if (num_groups != 8 && num_groups != 4) return cudaErrorInvalidValue;
    const int G = heads / num_groups;
    CUtensorMap kvr, krr, qm;
    {  // [g * real_slots][256]: one-row boxes for tile::gather4
        cuuint64_t dims[2] = {256, (cuuint64_t)num_groups * real_slots};
        cuuint64_t strides[1] = {256 * 2};
        cuuint32_t box[2] = {64, 1};
        if (!make_map(&kvr, kv, 2, dims, strides, box)) return cudaErrorInvalidValue;
    }
    {
        cuuint64_t dims[2] = {64, (cuuint64_t)real_slots};
        cuuint64_t strides[1] = {64 * 2};
        cuuint32_t box[2] = {64, 1};
        if (!make_map(&krr, k_rope, 2, dims, strides, box)) return cudaErrorInvalidValue;
    }
    {  // q [batch * s_q][heads][192]: one query token per selected sequence
        cuuint64_t dims[3] = {(cuuint64_t)kQk, (cuuint64_t)heads, (cuuint64_t)sel->batch};
        cuuint64_t strides[2] = {(cuuint64_t)kQk * 2, (cuuint64_t)heads * kQk * 2};
        cuuint32_t box[3] = {64, (cuuint32_t)G, 1};
        if (!make_map(&qm, q, 3, dims, strides, box)) return cudaErrorInvalidValue;
    }
    GqaParams p;
    p.page_table = sel->page_table;
    p.seqlens = sel->seqlens;
    p.o_part = o_part;
    p.lse_part = lse_part;
    p.ws = ws;
    p.batch = sel->batch;
    p.max_pages = sel->max_pages_per_seq;
    p.num_pages = sel->num_pages;
    p.num_splits = num_splits;
    p.s_q = 1;
    p.heads = heads;
    p.G = G;
    p.NG = num_groups;
    p.out = nullptr;
    p.lse_out = nullptr;
    p.scale_log2 = scale * kLog2e;
    p.sel_slot = sel_slot;
    p.real_slots = (int)real_slots;
    p.drop_v_unit = -1;
    // the dense tile maps are not used in sparse mode: the row maps stand in for them
    return G <= 16 ? launch_nq_mode<16, true>(kvr, krr, qm, kvr, krr, p, 1, stream)
                   : launch_nq_mode<32, true>(kvr, krr, qm, kvr, krr, p, 1, stream);
}

}  // namespace gqla
