// decode_gqa.cu -- split-KV partial attention of the GQA path on the
// tcgen05 tensor cores (GQLA, paperlayer.ai summary, sec. 3 "Two equivalent
// decoding paths": the g K/V groups are materialised and decoding is standard
// grouped-query attention; pwwt.cn article, sec. 5: h_q/g = 16 query heads
// share one group).
//
// The path is HBM-bound (about 19 FLOP per cache byte at s_q = 1), so the
// design goal is to stream the 4224 bytes per token exactly once at full
// bandwidth and hide everything else behind it:
//
//  * One CTA per chunk of the split plan (grid = SM count), 192 threads:
//      warp 0      TMA producer: per page, the shared RoPE keys (8 KB), then
//                  per group K_nope_g and V_g (4 boxes of 64 x 64 bf16,
//                  32 KB) into a 3-4 stage ring (128B-swizzled);
//      warp 1      TMEM owner and single-thread tcgen05.mma issuer;
//      warps 2-5   softmax, rescaling and the epilogue.
//  * The query rows of a group (G*s_q <= 32) are far below the 64/128-row
//    MMA minimum, so the products are transposed ("swap-AB"): the 64 tokens
//    of a page are the M dimension and the group's query rows the N
//    dimension.
//      S^T[64 tok][NQ]   = [K_nope_g | k^R] (64 x 192, K-major) x q_g^T
//      O^T_g[128 dv][NQ] += V_g^T (MN-major) x P^T (MN-major, bf16)
//    O^T of all 8 groups stays resident in TMEM for the whole piece.
//  * Online softmax in the base-2 domain with lazy rescaling: the running
//    maximum of a column moves only when a tile exceeds it by more than
//    2^8, so O^T in TMEM is rescaled rarely.  Column maxima and sums over
//    the 64 tokens are warp butterflies plus a 4-warp exchange.
//  * Every wait is bounded; a wait that runs out records GQLA_ERR_TIMEOUT
//    and the CTA drains and exits instead of hanging.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "sm100.cuh"

namespace gqla {

namespace {

using namespace sm100;

constexpr int kThreads = 192;
constexpr float kRescaleLog2 = 8.0f;
constexpr int kKvBox = 64 * 64 * 2;  // one 64-token x 64-column bf16 box

template <int NQ>
struct GqaSmem {
    static constexpr int kStages = NQ == 16 ? 4 : 3;
    static constexpr int kStageBytes = 4 * kKvBox;       // K lo | K hi | V lo | V hi
    static constexpr int kKrBytes = kKvBox;              // 64 tokens x 64 RoPE dims
    static constexpr int kQBlock = 8 * NQ * 128;         // 64 q dims x (8 groups x NQ rows)
    static constexpr int kPBytes = 64 * NQ * 2;          // P^T [64 tokens][NQ] bf16
    static constexpr int oStage = 0;
    static constexpr int oKr = oStage + kStages * kStageBytes;
    static constexpr int oQ = oKr + 2 * kKrBytes;
    static constexpr int oP = oQ + 3 * kQBlock;
    static constexpr int oRed = oP + 2 * ((kPBytes + 1023) / 1024) * 1024;  // float [NQ][4]
    static constexpr int oMrun = oRed + NQ * 4 * 4;                        // float [2][8][NQ]
    static constexpr int oLw = oMrun + 2 * 8 * NQ * 4;                     // float [4][8][NQ]
    static constexpr int oBar = oLw + 4 * 8 * NQ * 4;
    // barriers: full[S], empty[S], kr_full[2], kr_empty[2], s_full[2], s_free[2],
    //           p_full[2], p_free[2], q_full, o_done, drain
    static constexpr int kNumBars = 2 * kStages + 15;
    static constexpr int oMisc = oBar + kNumBars * 8;  // tmem base, abort flag, plan[4]
    static constexpr int kBytes = oMisc + 32;
    static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024
};

struct GqaParams {
    const __nv_bfloat16 *q;
    const int32_t *page_table;
    const int32_t *seqlens;
    float *o_part;
    float *lse_part;
    void *ws;
    int batch, max_pages, num_pages, num_splits, s_q, heads, G;
    float scale_log2;
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

__device__ __forceinline__ void named_bar_sync() {
    asm volatile("bar.sync 1, 128;" ::: "memory");
}

template <int NQ>
__global__ void __launch_bounds__(kThreads, 1)
    decode_gqa_tc_kernel(const __grid_constant__ CUtensorMap kv_map,
                         const __grid_constant__ CUtensorMap kr_map, const GqaParams p) {
    using SM = GqaSmem<NQ>;
    constexpr int S = SM::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::oBar);
    uint64_t *full = bars, *empty = bars + S;
    uint64_t *kr_full = bars + 2 * S, *kr_empty = kr_full + 2;
    uint64_t *s_full = kr_empty + 2, *s_free = s_full + 2;
    uint64_t *p_full = s_free + 2, *p_free = p_full + 2;
    uint64_t *q_full = p_free + 2, *o_done = q_full + 1, *drain = o_done + 1;
    uint32_t *tmem_base_smem = reinterpret_cast<uint32_t *>(smem + SM::oMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + SM::oMisc + 4);
    int *plan = reinterpret_cast<int *>(smem + SM::oMisc + 8);
    float *red = reinterpret_cast<float *>(smem + SM::oRed);
    float *mrun = reinterpret_cast<float *>(smem + SM::oMrun);
    float *lw = reinterpret_cast<float *>(smem + SM::oLw);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x;

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&kr_full[i], 1); mbar_init(&kr_empty[i], 1);
            mbar_init(&s_full[i], 1); mbar_init(&s_free[i], 128);
            mbar_init(&p_full[i], 128); mbar_init(&p_free[i], 1);
        }
        mbar_init(q_full, 128);
        mbar_init(o_done, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        int total = warp_total_pages(p.seqlens, p.batch);
        int k = chunk_pages(total, p.num_splits);
        int r0 = c * k, r1 = min(total, r0 + k);
        int b = p.batch, start = 0;
        if (r0 < r1) warp_find_sequence(p.seqlens, p.batch, r0, &b, &start);
        if (lane == 0) { plan[0] = r0; plan[1] = r1; plan[2] = b; plan[3] = start; }
    }
    if (warp == 1) {
        tmem_alloc(tmem_base_smem, 512);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_smem;
    const uint32_t t_s = tmem;            // S^T buffers: columns [0, 2 NQ), M = 64 layout
    const uint32_t t_o = tmem + 2 * NQ;   // O^T_g: columns [2 NQ + g NQ, ...), all 128 lanes
    PieceIter it0{plan[2], plan[3], plan[0], plan[1]};

    const uint32_t sm_stage = smem_u32(smem + SM::oStage);
    const uint32_t sm_kr = smem_u32(smem + SM::oKr);
    const uint32_t sm_q = smem_u32(smem + SM::oQ);
    const uint32_t sm_p = smem_u32(smem + SM::oP);
    constexpr int kPStride = ((SM::kPBytes + 1023) / 1024) * 1024;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            prefetch_tensormap(&kv_map);
            prefetch_tensormap(&kr_map);
            PieceIter it = it0;
            int b, L, pb, pe;
            bool too_long;
            uint32_t j = 0, pc = 0;
            while (next_piece(p, it, b, L, pb, pe, too_long)) {
                if (too_long) { report_error(p.ws, GQLA_ERR_DEVICE, b); continue; }
                for (int pg = pb; pg < pe; ++pg, ++pc) {
                    const int page = p.page_table[(int64_t)b * p.max_pages + pg];
                    const bool bad = page < 0 || page >= p.num_pages;
                    if (bad) report_error(p.ws, GQLA_ERR_DEVICE, b);
                    const int kb = pc & 1;
                    if (!mbar_wait(&kr_empty[kb], ((pc >> 1) & 1) ^ 1, abort_flag)) *abort_flag = 1;
                    if (!bad && !*abort_flag) {
                        mbar_arrive_expect_tx(&kr_full[kb], SM::kKrBytes);
                        tma_load_2d(smem + SM::oKr + kb * SM::kKrBytes, &kr_map, &kr_full[kb], 0, page * kPage);
                    } else {
                        mbar_arrive(&kr_full[kb]);
                    }
                    for (int gi = 0; gi < 8; ++gi, ++j) {
                        const int st = j % S;
                        if (!mbar_wait(&empty[st], ((j / S) & 1) ^ 1, abort_flag)) *abort_flag = 1;
                        uint8_t *dst = smem + SM::oStage + st * SM::kStageBytes;
                        if (!bad && !*abort_flag) {
                            mbar_arrive_expect_tx(&full[st], SM::kStageBytes);
#pragma unroll
                            for (int box = 0; box < 4; ++box)
                                tma_load_3d(dst + box * kKvBox, &kv_map, &full[st], box * 64, page * kPage, gi);
                        } else {
                            mbar_arrive(&full[st]);
                        }
                    }
                }
            }
            // never leave with copies in flight: wait (bounded) for the last loads issued
            for (uint32_t u = (j > (uint32_t)S ? j - S : 0); u < j; ++u) {
                int dummy = 0;
                mbar_wait(&full[u % S], (u / S) & 1, reinterpret_cast<volatile int *>(&dummy));
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16(64, NQ, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16(128, NQ, 1, 1);
            constexpr uint32_t p_sw = NQ == 16 ? kSw32 : kSw64;
            constexpr uint32_t p_sbo = NQ == 16 ? 256 : 512;
            PieceIter it = it0;
            int b, L, pb, pe;
            bool too_long;
            uint32_t j = 0, pc = 0, k = 0;
            auto issue_pv = [&](uint32_t u, bool first) {
                const int buf = u & 1;
                if (!mbar_wait(&p_full[buf], (u >> 1) & 1, abort_flag)) *abort_flag = 1;
                tc_fence_after();
                const int gi = u % 8;
                const uint32_t v_lo = sm_stage + (u % S) * SM::kStageBytes + 2 * kKvBox;
                const uint32_t pbuf = sm_p + buf * kPStride;
                if (!*abort_flag) {
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        uint64_t ad = smem_desc(v_lo + ks * 2048, kKvBox, 1024, kSw128);
                        uint64_t bd = smem_desc(pbuf + ks * 16 * NQ * 2, SM::kPBytes, p_sbo, p_sw);
                        mma_bf16(t_o + gi * NQ, ad, bd, idesc_pv, (first && ks == 0) ? 0u : 1u);
                    }
                }
                mma_commit(&p_free[buf]);
                mma_commit(&empty[u % S]);
            };
            while (next_piece(p, it, b, L, pb, pe, too_long)) {
                if (too_long) continue;
                if (!mbar_wait(q_full, k & 1, abort_flag)) *abort_flag = 1;
                tc_fence_after();
                const uint32_t j0 = j;
                for (int pg = pb; pg < pe; ++pg, ++pc) {
                    const int kb = pc & 1;
                    if (!mbar_wait(&kr_full[kb], (pc >> 1) & 1, abort_flag)) *abort_flag = 1;
                    const uint32_t kr = sm_kr + kb * SM::kKrBytes;
                    for (int gi = 0; gi < 8; ++gi, ++j) {
                        const int st = j % S, buf = j & 1;
                        if (!mbar_wait(&full[st], (j / S) & 1, abort_flag)) *abort_flag = 1;
                        if (!mbar_wait(&s_free[buf], ((j >> 1) & 1) ^ 1, abort_flag)) *abort_flag = 1;
                        tc_fence_after();
                        const uint32_t kst = sm_stage + st * SM::kStageBytes;
                        const uint32_t qg = sm_q + gi * NQ * 128;
                        if (!*abort_flag) {
#pragma unroll
                            for (int ks = 0; ks < 12; ++ks) {
                                const uint32_t a = ks < 8 ? kst + (ks >> 2) * kKvBox + (ks & 3) * 32
                                                          : kr + (ks - 8) * 32;
                                const uint32_t bq = qg + (ks >> 2) * SM::kQBlock + (ks & 3) * 32;
                                mma_bf16(t_s + buf * NQ, smem_desc(a, 16, 1024, kSw128),
                                         smem_desc(bq, 16, 1024, kSw128), idesc_s, ks > 0 ? 1u : 0u);
                            }
                        }
                        mma_commit(&s_full[buf]);
                        if (gi == 7) mma_commit(&kr_empty[kb]);
                        if (j > j0) issue_pv(j - 1, (j - 1 - j0) < 8);
                    }
                }
                issue_pv(j - 1, (j - 1 - j0) < 8);
                mma_commit(o_done);
                ++k;
            }
            // drain: nothing may still be running when TMEM is freed
            mma_commit(drain);
            int dummy = 0;
            mbar_wait(drain, 0, reinterpret_cast<volatile int *>(&dummy));
        }
    } else {
        // ---------------------------------------------------------------- softmax + epilogue
        const int quad = warp & 3;         // TMEM lane quadrant of this warp
        const int wq = warp - 2;           // 0..3 among the softmax warps
        const int stid = threadIdx.x - 64; // 0..127
        const bool has_tok = lane < 16;
        const int tok_in_tile = 16 * quad + lane;
        const int dv = 32 * quad + lane;
        const uint32_t lane_off = static_cast<uint32_t>(32 * quad) << 16;
        const int real_cols = p.G * p.s_q;
        uint8_t *qsm = smem + SM::oQ;
        PieceIter it = it0;
        int b, L, pb, pe;
        bool too_long;
        uint32_t j = 0, k = 0;
        while (next_piece(p, it, b, L, pb, pe, too_long)) {
            if (too_long) continue;
            // ---- q rows of all groups, 128B-swizzled K-major (rows gi*NQ + n), zero padding rows
            for (int i = stid; i < 8 * NQ * 24; i += 128) {
                const int R = i / 24, ch = i % 24;
                const int gi = R / NQ, n = R % NQ;
                uint4 v = make_uint4(0, 0, 0, 0);
                if (n < real_cols) {
                    const int s = n / p.G, hg = n % p.G;
                    v = *reinterpret_cast<const uint4 *>(
                        p.q + (((int64_t)b * p.s_q + s) * p.heads + gi * p.G + hg) * kQk + ch * 8);
                }
                *reinterpret_cast<uint4 *>(qsm + (ch >> 3) * SM::kQBlock + swz(R * 128 + (ch & 7) * 16, 128)) = v;
            }
            for (int i = lane; i < 8 * NQ; i += 32) lw[(wq * 8) * NQ + i] = 0.0f;
            fence_proxy_async_smem();
            mbar_arrive(q_full);

            const int np = pe - pb;
            for (int ip = 0; ip < np; ++ip) {
                const int pg = pb + ip;
                const int page = p.page_table[(int64_t)b * p.max_pages + pg];
                const bool bad = page < 0 || page >= p.num_pages;
                const int n_valid = bad ? 0 : min(kPage, L - pg * kPage);
                const int tok = pg * kPage + tok_in_tile;
                const bool tok_ok = has_tok && tok_in_tile < n_valid;
                const float *mold_row = mrun + ((ip & 1) ^ 1) * 8 * NQ;
                float *mnew_row = mrun + (ip & 1) * 8 * NQ;
                for (int gi = 0; gi < 8; ++gi, ++j) {
                    const int buf = j & 1;
                    // scores of this warp's 16 tokens
                    if (!mbar_wait(&s_full[buf], (j >> 1) & 1, abort_flag)) *abort_flag = 1;
                    tc_fence_after();
                    uint32_t sv[NQ];
                    tmem_ld16(t_s + lane_off + buf * NQ, sv);
                    if constexpr (NQ == 32) tmem_ld16(t_s + lane_off + buf * NQ + 16, sv + 16);
                    tmem_wait_ld();
                    tc_fence_before();
                    mbar_arrive(&s_free[buf]);
                    // query s sees token t iff t <= L - s_q + s; columns are n = s*G + hg,
                    // so with s_q <= 2 only the last token can be hidden, from columns n < G
                    float x[NQ];
                    const int s_min = tok - (L - p.s_q);
#pragma unroll
                    for (int n = 0; n < NQ; ++n) {
                        const bool vis = tok_ok && (s_min <= 0 || n >= p.G);
                        x[n] = vis ? __uint_as_float(sv[n]) * p.scale_log2 : -INFINITY;
                    }
                    // column maxima over the 64 tokens
                    {
                        float t[NQ];
#pragma unroll
                        for (int n = 0; n < NQ; ++n) t[n] = x[n];
                        const float m = transpose_reduce<NQ, true>(t, lane);
                        if (lane < NQ) red[lane * 4 + wq] = m;
                    }
                    named_bar_sync();
                    float mu[NQ], alpha[NQ];
                    bool need = false;
#pragma unroll
                    for (int n = 0; n < NQ; n += 4) {
                        float4 m_old4 = ip ? *reinterpret_cast<const float4 *>(mold_row + gi * NQ + n)
                                           : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
                        const float mo[4] = {m_old4.x, m_old4.y, m_old4.z, m_old4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float4 r4 = *reinterpret_cast<const float4 *>(red + (n + e) * 4);
                            const float mt = fmaxf(fmaxf(r4.x, r4.y), fmaxf(r4.z, r4.w));
                            const float mn = (mt > mo[e] + kRescaleLog2) ? mt : mo[e];
                            mu[n + e] = mn;
                            alpha[n + e] = (mn == mo[e]) ? 1.0f : exp2f(mo[e] - mn);
                            need |= (ip > 0) && (mn != mo[e]);
                        }
                    }
                    if (stid == 0) {
#pragma unroll
                        for (int n = 0; n < NQ; n += 4)
                            *reinterpret_cast<float4 *>(mnew_row + gi * NQ + n) =
                                make_float4(mu[n], mu[n + 1], mu[n + 2], mu[n + 3]);
                    }
                    // P^T buffer and O^T_g are free once PV(j - 2) has completed
                    if (!mbar_wait(&p_free[buf], ((j >> 1) & 1) ^ 1, abort_flag)) *abort_flag = 1;
                    tc_fence_after();
                    if (need) {  // uniform across the four warps
                        const uint32_t to = t_o + gi * NQ + lane_off;
#pragma unroll
                        for (int h16 = 0; h16 < NQ; h16 += 16) {
                            uint32_t r[16];
                            tmem_ld16(to + h16, r);
                            tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 16; ++e)
                                r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha[h16 + e]);
                            tmem_st16(to + h16, r);
                        }
                        tmem_wait_st();
                    }
                    // probabilities (bf16) into P^T, this warp's 16 token rows
                    float ps[NQ];
                    {
                        uint8_t *pbuf = smem + SM::oP + buf * kPStride;
#pragma unroll
                        for (int n = 0; n < NQ; n += 8) {
                            uint32_t w[4];
#pragma unroll
                            for (int e = 0; e < 8; e += 2) {
                                const float m0 = mu[n + e] == -INFINITY ? 0.0f : mu[n + e];
                                const float m1 = mu[n + e + 1] == -INFINITY ? 0.0f : mu[n + e + 1];
                                const float p0 = x[n + e] == -INFINITY ? 0.0f : exp2f(x[n + e] - m0);
                                const float p1 = x[n + e + 1] == -INFINITY ? 0.0f : exp2f(x[n + e + 1] - m1);
                                __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                                w[e / 2] = *reinterpret_cast<uint32_t *>(&h2);
                                const float2 back = __bfloat1622float2(h2);
                                ps[n + e] = back.x;
                                ps[n + e + 1] = back.y;
                            }
                            if (has_tok)
                                *reinterpret_cast<uint4 *>(pbuf + swz(tok_in_tile * NQ * 2 + n * 2, NQ * 2)) =
                                    make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                    // V rows of tokens past the sequence end (pool rows never written, maybe NaN) -> 0
                    if (n_valid < kPage) {
                        const int st = j % S;
                        if (!mbar_wait(&full[st], (j / S) & 1, abort_flag)) *abort_flag = 1;
                        uint8_t *vbase = smem + SM::oStage + st * SM::kStageBytes + 2 * kKvBox;
                        for (int i = stid; i < 2 * (kPage - n_valid) * 8; i += 128) {
                            const int half = i / ((kPage - n_valid) * 8);
                            const int rem = i % ((kPage - n_valid) * 8);
                            const int row = n_valid + rem / 8, ch = rem % 8;
                            *reinterpret_cast<uint4 *>(vbase + half * kKvBox + row * 128 + ch * 16) =
                                make_uint4(0, 0, 0, 0);
                        }
                    }
                    fence_proxy_async_smem();
                    tc_fence_before();
                    mbar_arrive(&p_full[buf]);
                    // column sums of the rounded probabilities, per warp (lane n holds column n)
                    {
                        const float l = transpose_reduce<NQ, false>(ps, lane);
                        if (lane < NQ) {
                            float *slot = lw + (wq * 8 + gi) * NQ + lane;
                            const float mo = ip ? mold_row[gi * NQ + lane] : -INFINITY;
                            const float4 r4 = *reinterpret_cast<const float4 *>(red + lane * 4);
                            const float mt = fmaxf(fmaxf(r4.x, r4.y), fmaxf(r4.z, r4.w));
                            const float mn = (mt > mo + kRescaleLog2) ? mt : mo;
                            const float a = (mn == mo || ip == 0) ? 1.0f : exp2f(mo - mn);
                            *slot = (ip ? *slot * a : 0.0f) + l;
                        }
                    }
                    named_bar_sync();  // red[] is rewritten by the next unit
                }
            }
            // ---- epilogue: normalise O^T and write the partials of slot b + c
            if (!mbar_wait(o_done, k & 1, abort_flag)) *abort_flag = 1;
            tc_fence_after();
            named_bar_sync();
            const float *mfin = mrun + ((np - 1) & 1) * 8 * NQ;
            const int slot = b + c;
            for (int gi = 0; gi < 8; ++gi) {
                uint32_t r[NQ];
                tmem_ld16(t_o + gi * NQ + lane_off, r);
                if constexpr (NQ == 32) tmem_ld16(t_o + gi * NQ + lane_off + 16, r + 16);
                tmem_wait_ld();
#pragma unroll
                for (int n = 0; n < NQ; ++n) {
                    if (n >= real_cols) break;
                    const float l = lw[(0 * 8 + gi) * NQ + n] + lw[(1 * 8 + gi) * NQ + n] +
                                    lw[(2 * 8 + gi) * NQ + n] + lw[(3 * 8 + gi) * NQ + n];
                    const int s = n / p.G, hg = n % p.G;
                    const int64_t row = ((int64_t)slot * p.s_q + s) * p.heads + gi * p.G + hg;
                    p.o_part[row * kDv + dv] = l > 0.0f ? __uint_as_float(r[n]) / l : 0.0f;
                    if (stid == 0) {
                        const float m = mfin[gi * NQ + n];
                        p.lse_part[row] = (l > 0.0f && m != -INFINITY)
                                              ? (m + __log2f(l)) * 0.6931471805599453f
                                              : -INFINITY;
                    }
                }
            }
            tc_fence_before();
            named_bar_sync();
            ++k;
        }
    }

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

template <int NQ>
cudaError_t launch_nq(const CUtensorMap &kvm, const CUtensorMap &krm, const GqaParams &p,
                      cudaStream_t stream) {
    const int bytes = GqaSmem<NQ>::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(decode_gqa_tc_kernel<NQ>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    decode_gqa_tc_kernel<NQ><<<p.num_splits, kThreads, bytes, stream>>>(kvm, krm, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_gqa(const void *q, int s_q, int heads, int num_groups, const void *kv,
                              const void *k_rope, int64_t num_slots, const gqla_kv_index *idx,
                              int num_splits, float scale, float *o_part, float *lse_part,
                              void *ws, cudaStream_t stream) {
    if (num_groups != 8) return cudaErrorInvalidValue;
    CUtensorMap kvm, krm;
    {
        cuuint64_t dims[3] = {256, (cuuint64_t)num_slots, 8};
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
    GqaParams p;
    p.q = static_cast<const __nv_bfloat16 *>(q);
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
    p.G = heads / num_groups;
    p.scale_log2 = scale * kLog2e;
    return p.G * s_q <= 16 ? launch_nq<16>(kvm, krm, p, stream) : launch_nq<32>(kvm, krm, p, stream);
}

}  // namespace gqla
