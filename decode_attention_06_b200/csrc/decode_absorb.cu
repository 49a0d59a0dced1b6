// decode_absorb.cu -- split-KV partial attention of the MQA-absorb path on the
// tcgen05 tensor cores (GQLA, paperlayer.ai summary, sec. 2 and sec. 3: W_UK is
// folded into the query and every head attends directly over the latent row
// [c (512) | k^R (64)]; the value is the 512-d latent itself).
//
// Per (sequence, block of up to 128 query rows) the products are
//   S = q~ C^T   (M = 128 rows, K = 576, N = tokens)
//   O += P C_lat (M = 128 rows, K = tokens, N = 512)
// The fp32 O alone (128 x 512) fills a whole SM's tensor memory, so the work
// is split over a 2-CTA cluster by latent column: CTA r owns the columns
// [256r, 256r + 256) of the latent and [32r, 32r + 32) of the RoPE key.  Each
// CTA streams only its 288 columns of every cache row (the pair reads each
// byte of the cache exactly once), computes a partial score tile over them,
// and the two partials are exchanged through distributed shared memory in
// fp16; both CTAs add the same two rounded partials, so their P and softmax
// statistics are bit-identical, and each accumulates its own 256 columns of O.
//
//  * Tile = one 64-token page.  An MMA instruction costs at least ~45 cycles
//    whatever its N, so the score tile is made 64 tokens wide.  Tensor memory
//    holds O (256 columns), a double-buffered S (2 x 64) and the latent half
//    of q~ (128 columns of bf16 pairs), so the score MMA reads q~ from TMEM;
//    P goes through shared memory, beside a 4-slot ring of cache tiles.
//    Roles, 19 warps:
//      warp 0      TMA producer: the RoPE columns of q~ (once per piece) and
//                  the ring (4 latent boxes 128B-swizzled + 1 RoPE box
//                  64B-swizzled, 36 KB per 64-token tile);
//      warp 1      TMEM owner, issues S = q~ C^T (latent part with A in TMEM);
//      warps 2-17  online softmax, four warps per TMEM lane quadrant, each
//                  taking 16 of the tile's 64 tokens: the fp16 partial
//                  scores go straight from registers into the peer CTA's
//                  receive buffer with st.async (completing on the peer's
//                  mbarrier), row maxima (lazy rescaling of O rows when a
//                  maximum rises by more than 2^8), P written to shared
//                  memory (bf16, 128B-swizzled, the PV MMA's A operand).  Tile
//                  i + 1's partial is sent before tile i is finished when its
//                  scores are already available;
//      warp 18     issues O += P C in tile order.
//  * The softmax warps copy each piece's latent half of q~ from global memory
//    into TMEM as soon as the previous piece's scores are done, and write
//    O / l with TMA stores staged in the (then idle) P buffers.
//  * Every wait is bounded and reports GQLA_ERR_TIMEOUT instead of hanging;
//    both CTAs of a cluster always execute the same sequence of steps.
#include <cudaTypedefs.h>

#include <cuda_fp16.h>

#include "common.cuh"
#include "sm100.cuh"
#include "tensor_map.cuh"

namespace gqla {

namespace {

using namespace sm100;

constexpr int kSmWarps = 16;                // softmax warps: kParts per TMEM lane quadrant
constexpr int kParts = kSmWarps / 4;
constexpr int kThreads = 32 * (3 + kSmWarps);
constexpr int kPvWarp = 2 + kSmWarps;       // warp issuing O += P C
constexpr int kRows = 128;           // MMA M: query rows of one row block (zero-padded)
constexpr int kT = 64;               // tokens per tile (one page)
constexpr int kRing = 4;
constexpr float kRescaleLog2 = 8.0f;
constexpr int kTokW = kT / kParts;          // tokens of a tile per softmax warp
constexpr int kSmThreads = 32 * kSmWarps;

struct AbsorbSmem {
    static constexpr int kQRope = kRows * 64;             // q~ RoPE columns [128 rows][32]
    static constexpr int kLatBox = kT * 128;              // [64 tokens][64 cols]
    static constexpr int kRopeBox = kT * 64;              // [64 tokens][32 cols]
    static constexpr int kSlot = 4 * kLatBox + kRopeBox;  // 36 KB
    static constexpr int kX = kRows * kT * 2;             // fp16 partial scores, [warps][32 rows][kTokW]
    static constexpr int kXw = kX / kSmWarps;             // one warp's block
    static constexpr int kP = kRows * kT * 2;             // P, [128 rows][64 tokens] bf16, 128B-swizzled
    static constexpr int oQ = 0;
    static constexpr int oP = oQ + kQRope;                // 2 buffers
    static constexpr int oRing = oP + 2 * kP;
    static constexpr int oX = oRing + kRing * kSlot;      // the peer's partials (2 buffers)
    static constexpr int oRm = oX + 2 * kX;               // float [2 tiles][kParts][128 rows]
    static constexpr int oL = oRm + 2 * kParts * kRows * 4;  // float [kParts][128 rows]
    static constexpr int oBar = oL + kParts * kRows * 4;
    // ring_full/empty[3], q_full, q_empty, s_full/s_free[2], p_full/p_free[2],
    // x_full/x_empty[2], o_done, drain[2]
    static constexpr int kNumBars = 2 * kRing + 2 + 4 + 4 + 4 + 1 + 2;
    static constexpr int oMisc = oBar + kNumBars * 8;     // tmem base, abort, plan[4]
    static constexpr int kBytes = oMisc + 32;
    static constexpr int kAlloc = kBytes + 1024;
};
static_assert(AbsorbSmem::kAlloc <= 227 * 1024, "shared memory");

struct AbsorbParams {
    const int32_t *page_table;
    const int32_t *seqlens;
    const __nv_bfloat16 *qa;
    float *o_part;
    float *lse_part;
    void *ws;
    int batch, max_pages, num_pages, num_splits, s_q, heads;
    int rows_total;   // s_q * heads: query rows of one sequence
    int row_blocks;   // ceil(rows_total / 128)
    float scale_log2;
};

struct PieceIter {
    int b, P, r0, r1;
};

__device__ __forceinline__ bool next_piece(const AbsorbParams &p, PieceIter &it, int &b, int &L,
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

__device__ __forceinline__ void quad_bar(int quad) {  // the softmax warps of one lane quadrant
    asm volatile("bar.sync %0, %1;" ::"r"(1 + quad), "n"(32 * kParts) : "memory");
}

__device__ __forceinline__ void softmax_bar() {  // all softmax warps
    asm volatile("bar.sync 5, %0;" ::"n"(kSmThreads) : "memory");
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    decode_absorb_tc_kernel(const __grid_constant__ CUtensorMap lat_map,
                            const __grid_constant__ CUtensorMap rope_map,
                            const __grid_constant__ CUtensorMap qrope_map,
                            const __grid_constant__ CUtensorMap o_map_wide,
                            const __grid_constant__ CUtensorMap o_map_narrow, const AbsorbParams p) {
    using SM = AbsorbSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::oBar);
    uint64_t *ring_full = bars, *ring_empty = bars + kRing;
    uint64_t *q_full = bars + 2 * kRing, *q_empty = q_full + 1;
    uint64_t *s_full = q_empty + 1, *s_free = s_full + 2;
    uint64_t *p_full = s_free + 2, *p_free = p_full + 2;
    uint64_t *x_full = p_free + 2, *x_empty = x_full + 2;
    uint64_t *o_done = x_empty + 2, *drain = o_done + 1;
    uint32_t *tmem_base_smem = reinterpret_cast<uint32_t *>(smem + SM::oMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + SM::oMisc + 4);
    int *plan = reinterpret_cast<int *>(smem + SM::oMisc + 8);
    GQLA_PROF_DECL;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const uint32_t peer = rank ^ 1u;
    const int cluster = blockIdx.x >> 1;
    const int c = cluster / p.row_blocks;   // chunk of the split plan
    const int rb = cluster % p.row_blocks;  // row block within the sequence's s_q * h rows
    const int rows_here = min(kRows, p.rows_total - rb * kRows);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kRing; ++i) { mbar_init(&ring_full[i], 1); mbar_init(&ring_empty[i], 1); }
        mbar_init(q_full, 1 + kSmWarps);  // RoPE TMA + the softmax warps' TMEM copies
        mbar_init(q_empty, kSmWarps);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1); mbar_init(&s_free[i], kSmThreads);
            mbar_init(&p_full[i], kSmThreads); mbar_init(&p_free[i], 1);
            mbar_init(&x_full[i], 1); mbar_init(&x_empty[i], kSmWarps);
            mbar_init(&drain[i], 1);
        }
        mbar_init(o_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    griddep_wait();  // the previous kernel's results are visible from here on
    griddep_launch_dependents();
    // first page indices of the first piece, loaded by the producer warp while the
    // CTA and the cluster synchronise (valid when pre_ok)
    int pre_page = 0;
    bool pre_ok = false;
    if (warp == 0) {
        if (lane == 0) {
            prefetch_tensormap(&lat_map);
            prefetch_tensormap(&rope_map);
            prefetch_tensormap(&qrope_map);
        }
        int total = warp_total_pages(p.seqlens, p.batch);
        int k = chunk_pages(total, p.num_splits);
        int r0 = c * k, r1 = min(total, r0 + k);
        int b = p.batch, start = 0;
        if (r0 < r1) warp_find_sequence(p.seqlens, p.batch, r0, &b, &start);
        if (lane == 0) { plan[0] = r0; plan[1] = r1; plan[2] = b; plan[3] = start; }
        if (b < p.batch) {
            const int n = pages_of(p.seqlens[b]);  // > 0: the search skips empty sequences
            if (n <= p.max_pages) {                 // not a sequence that is reported as too long
                const int pb0 = r0 - start, pe0 = min(r1 - start, n);
                pre_ok = true;
                if (lane < min(32, pe0 - pb0)) pre_page = p.page_table[(int64_t)b * p.max_pages + pb0 + lane];
            }
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_base_smem, 512);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    cluster_sync();  // the peer's barriers are initialised before any remote arrive
    tc_fence_after();
    const uint32_t tmem = *tmem_base_smem;
    const uint32_t t_o = tmem;             // O: columns [0, 256), this CTA's latent half
    const uint32_t t_s = tmem + 256;       // S: 2 x kT columns
    const uint32_t t_q = tmem + 384;       // q~ latent half (bf16 pairs): 128 columns
    const PieceIter it0{plan[2], plan[3], plan[0], plan[1]};
    const uint32_t sm_q = smem_u32(smem + SM::oQ);
    const uint32_t sm_ring = smem_u32(smem + SM::oRing);
    const uint32_t sm_p = smem_u32(smem + SM::oP);

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        // Lane 0 issues; the whole warp fetches the page indices 32 at a time so
        // that no page-table load sits between two tiles.
        const uint64_t stream_policy = l2_evict_first_policy();  // the cache is read once
        PieceIter it = it0;
        int b, L, pb, pe;
        bool too_long;
        uint32_t t = 0, k = 0;
        while (next_piece(p, it, b, L, pb, pe, too_long)) {
            if (too_long) {
                if (lane == 0 && rank == 0 && rb == 0) report_error(p.ws, GQLA_ERR_DEVICE, b);
                continue;
            }
            // RoPE columns of q~ for this row block; they wait for the previous piece's
            // scores, so up to kRing - 1 of this piece's tiles are issued first
            const int rope_at = min(pe - pb, kRing - 1);
            auto load_rope = [&]() {
                if (lane == 0) {
                    if (!GQLA_WAIT(1, q_empty, (k & 1) ^ 1, abort_flag)) *abort_flag = 1;
                    if (!*abort_flag) {
                        const int row0 = b * p.rows_total + rb * kRows;
                        mbar_arrive_expect_tx(q_full, SM::kQRope);
                        tma_load_2d(smem + SM::oQ, &qrope_map, q_full, 512 + 32 * rank, row0);
                    } else {
                        mbar_arrive(q_full);
                    }
                }
            };
            const int32_t *prow = p.page_table + (int64_t)b * p.max_pages;
            for (int i0 = pb; i0 < pe; i0 += 32) {
                const int n = min(32, pe - i0);
                // (the first piece is the one the early load above was for)
                const int my_page = pre_ok ? pre_page : (lane < n ? prow[i0 + lane] : 0);
                pre_ok = false;
                for (int j = 0; j < n; ++j, ++t) {
                    const int page = __shfl_sync(0xffffffffu, my_page, j);
                    if (i0 - pb + j == rope_at) load_rope();
                    if (lane == 0) {
                        const bool bad = page < 0 || page >= p.num_pages;
                        if (bad && rank == 0 && rb == 0) report_error(p.ws, GQLA_ERR_DEVICE, b);
                        const int slot = t % kRing;
                        if (!GQLA_WAIT(0, &ring_empty[slot], ((t / kRing) & 1) ^ 1, abort_flag)) *abort_flag = 1;
                        uint8_t *dst = smem + SM::oRing + slot * SM::kSlot;
                        if (!bad && !*abort_flag) {
                            mbar_arrive_expect_tx(&ring_full[slot], SM::kSlot);
#pragma unroll
                            for (int bx = 0; bx < 4; ++bx)
                                tma_load_2d_hint(dst + bx * SM::kLatBox, &lat_map, &ring_full[slot],
                                                 256 * rank + 64 * bx, page * kPage, stream_policy);
                            tma_load_2d_hint(dst + 4 * SM::kLatBox, &rope_map, &ring_full[slot], 512 + 32 * rank,
                                             page * kPage, stream_policy);
                        } else {
                            mbar_arrive(&ring_full[slot]);
                        }
                    }
                }
            }
            if (rope_at == pe - pb) load_rope();
            ++k;
        }
        if (lane == 0) {
            // no TMA may still be writing when the CTA exits
            int dummy = 0;
            volatile int *no_abort = reinterpret_cast<volatile int *>(&dummy);
            for (uint32_t u = (t > (uint32_t)kRing ? t - kRing : 0); u < t; ++u)
                mbar_wait(&ring_full[u % kRing], (u / kRing) & 1, no_abort);
            if (k) mbar_wait(q_full, (k - 1) & 1, no_abort);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- score MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16(kRows, kT, 0, 0);
            PieceIter it = it0;
            int b, L, pb, pe;
            bool too_long;
            uint32_t t = 0, k = 0;
            while (next_piece(p, it, b, L, pb, pe, too_long)) {
                if (too_long) continue;
                if (!GQLA_WAIT(2, q_full, k & 1, abort_flag)) *abort_flag = 1;
                for (int i = 0; i < pe - pb; ++i, ++t) {
                    const int slot = t % kRing, sb = t & 1;
                    if (!GQLA_WAIT(3, &ring_full[slot], (t / kRing) & 1, abort_flag)) *abort_flag = 1;
                    if (!GQLA_WAIT(4, &s_free[sb], ((t >> 1) & 1) ^ 1, abort_flag)) *abort_flag = 1;
                    tc_fence_after();
                    const uint32_t tile = sm_ring + slot * SM::kSlot;
                    if (!*abort_flag) {
#pragma unroll
                        for (int ks = 0; ks < 16; ++ks) {  // latent: A = q~ in TMEM, 16 dims = 8 columns
                            const uint64_t bd = smem_desc(tile + (ks >> 2) * SM::kLatBox + (ks & 3) * 32, 16, 1024, kSw128);
                            mma_bf16_ts(t_s + sb * kT, t_q + ks * 8, bd, idesc_s, ks > 0 ? 1u : 0u);
                        }
#pragma unroll
                        for (int ks = 0; ks < 2; ++ks) {  // RoPE: 32 columns, 64B-swizzled rows
                            const uint64_t ad = smem_desc(sm_q + ks * 32, 16, 512, kSw64);
                            const uint64_t bd = smem_desc(tile + 4 * SM::kLatBox + ks * 32, 16, 512, kSw64);
                            mma_bf16(t_s + sb * kT, ad, bd, idesc_s, 1u);
                        }
                    }
                    mma_commit(&s_full[sb]);
                }
                ++k;
            }
            mma_commit(&drain[0]);
            int dummy = 0;
            mbar_wait(&drain[0], 0, reinterpret_cast<volatile int *>(&dummy));
        }
    } else if (warp == kPvWarp) {
        // ---------------------------------------------------------------- PV MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_pv = idesc_bf16(kRows, 256, 0, 1);
            PieceIter it = it0;
            int b, L, pb, pe;
            bool too_long;
            uint32_t t = 0;
            while (next_piece(p, it, b, L, pb, pe, too_long)) {
                if (too_long) continue;
                for (int i = 0; i < pe - pb; ++i, ++t) {
                    const int slot = t % kRing, sb = t & 1;
                    if (!GQLA_WAIT(5, &p_full[sb], (t >> 1) & 1, abort_flag)) *abort_flag = 1;
                    tc_fence_after();
                    const uint32_t tile = sm_ring + slot * SM::kSlot;
                    if (!*abort_flag) {
#pragma unroll
                        for (int ks = 0; ks < kT / 16; ++ks) {
                            // B = C_lat[tokens][256 cols of this CTA]: MN-major, 4 atoms of 64 columns
                            const uint64_t bd = smem_desc(tile + ks * 2048, SM::kLatBox, 1024, kSw128);
                            // A = P[128 rows][64 tokens], K-major: 16 tokens = 32 bytes of a row
                            const uint64_t ad = smem_desc(sm_p + sb * SM::kP + ks * 32, 16, 1024, kSw128);
                            mma_bf16(t_o, ad, bd, idesc_pv, (i == 0 && ks == 0) ? 0u : 1u);
                        }
                    }
                    mma_commit(&p_free[sb]);
                    mma_commit(&ring_empty[slot]);
                }
                mma_commit(o_done);
            }
            mma_commit(&drain[1]);
            int dummy = 0;
            mbar_wait(&drain[1], 0, reinterpret_cast<volatile int *>(&dummy));
        }
    } else {
        // ---------------------------------------------------------------- softmax + epilogue
        constexpr int kPr = kTokW / 2;           // fp16 pairs of a warp's tokens
        const int quad = warp & 3;               // TMEM lane quadrant
        const int w = warp - 2;                  // softmax warp index: its block of a buffer
        const int part = w >> 2;                 // which kTokW tokens of the tile
        const int row = 32 * quad + lane;        // query row of the row block (= TMEM lane)
        const uint32_t lane_off = static_cast<uint32_t>(32 * quad) << 16;
        const int grow = rb * kRows + row;       // row within the sequence's s_q * h rows
        const int s_of_row = grow < p.rows_total ? grow / p.heads : p.s_q - 1;
        float *rm = reinterpret_cast<float *>(smem + SM::oRm);
        float *lsm = reinterpret_cast<float *>(smem + SM::oL);
        const uint8_t *xbuf = smem + SM::oX;
        const uint32_t x_remote =
            map_peer(smem_u32(smem + SM::oX), peer) + w * SM::kXw + lane * (kTokW * 2);
        const uint32_t xfull_remote = map_peer(smem_u32(x_full), peer);
        const uint32_t xempty_remote = map_peer(smem_u32(x_empty), peer);
        // ---- this warp's share of q~'s latent half (its 32 rows x 256/kParts columns)
        // into TMEM; the previous piece's scores, its last readers, are complete
        auto copy_q = [&](int bq) {
            constexpr int kQc = 256 / kParts;  // bf16 columns per warp
            const uint4 *src = reinterpret_cast<const uint4 *>(
                p.qa + ((int64_t)bq * p.rows_total + grow) * kRow + 256 * rank + part * kQc);
            const bool live = row < rows_here;
#pragma unroll
            for (int h = 0; h < kQc / 32; ++h) {
                uint32_t wv[16];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 v = live ? src[4 * h + j] : make_uint4(0, 0, 0, 0);
                    wv[4 * j] = v.x; wv[4 * j + 1] = v.y; wv[4 * j + 2] = v.z; wv[4 * j + 3] = v.w;
                }
                tmem_st16(t_q + lane_off + part * (kQc / 2) + 16 * h, wv);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(q_full);
        };
        const bool quad_live = 32 * quad < rows_here;  // rows_here is a multiple of 32
        bool q_loaded = false;                         // q~ of the coming piece already in TMEM
        PieceIter it = it0;
        int b, L, pb, pe;
        bool too_long;
        uint32_t t = 0, k = 0;
        while (next_piece(p, it, b, L, pb, pe, too_long)) {
            if (too_long) continue;
            float m_run = -INFINITY, l_run = 0.0f;  // this row, this warp's tokens of every tile
            const int32_t *prow = p.page_table + (int64_t)b * p.max_pages;
            // query s of this row sees tokens t <= L - s_q + s
            const int last_visible = L - p.s_q + s_of_row;
            const uint32_t t0 = t;
            const int nt = pe - pb;
            if (!q_loaded) copy_q(b);
            q_loaded = false;
            // stage A of tile i: this warp's partial scores -> fp16 -> the peer's receive buffer
            auto stage_a = [&](int i, uint32_t (&h2)[kPr]) {
                const uint32_t tt = t0 + i;
                const int sb = tt & 1;
                if (!GQLA_WAIT(6, &s_full[sb], (tt >> 1) & 1, abort_flag)) *abort_flag = 1;
                tc_fence_after();
                uint32_t sv[kTokW];
#pragma unroll
                for (int c16 = 0; c16 < kTokW; c16 += 16)
                    tmem_ld16(t_s + lane_off + sb * kT + part * kTokW + c16, sv + c16);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&s_free[sb]);
#pragma unroll
                for (int j = 0; j < kPr; ++j) {
                    __half2 v = __floats2half2_rn(__uint_as_float(sv[2 * j]), __uint_as_float(sv[2 * j + 1]));
                    h2[j] = *reinterpret_cast<uint32_t *>(&v);
                }
                if (w == 0 && lane == 0) mbar_arrive_expect_tx(&x_full[sb], SM::kX);
                // the peer's receive buffer sb is free once it has read tile tt - 2
                if (!GQLA_WAITC(7, &x_empty[sb], ((tt >> 1) & 1) ^ 1, abort_flag)) *abort_flag = 1;
#pragma unroll
                for (int j = 0; j < kPr / 4; ++j)
                    st_async_v4(x_remote + sb * SM::kX + 16 * j,
                                make_uint4(h2[4 * j], h2[4 * j + 1], h2[4 * j + 2], h2[4 * j + 3]),
                                xfull_remote + sb * 8);
            };
            uint32_t hc[kPr];
            stage_a(0, hc);
            bool have_next = false;  // stage A of tile i + 1 already done
            int page = prow[pb];
            for (int i = 0; i < nt; ++i) {
                // Tile i + 1's exchange is started early only when its scores are
                // already there: waiting for them here would tie the release of
                // tile i (and of its ring slot) to the arrival of the next tile.
                uint32_t hn[kPr];
                const bool next_ready =
                    i + 1 < nt && __shfl_sync(0xffffffffu,  // one decision per warp
                                              (int)mbar_test_wait(&s_full[(t0 + i + 1) & 1], ((t0 + i + 1) >> 1) & 1), 0);
                if (next_ready) {
                    stage_a(i + 1, hn);
                    have_next = true;
                }
                const int page_next = i + 1 < nt ? prow[pb + i + 1] : 0;  // in flight meanwhile
                const uint32_t tt = t0 + i;
                const int pg = pb + i;
                const int tok0 = pg * kPage;  // first token of this tile
                const int sb = tt & 1, slot = tt % kRing;
                const bool bad = page < 0 || page >= p.num_pages;
                const int n_valid = bad ? 0 : max(0, min(kT, L - tok0));
                GQLA_SPAN_BEGIN(t_tile);
                // ---- full raw scores = own + peer (the same rounded partials in both CTAs)
                if (!GQLA_WAITC(8, &x_full[sb], (tt >> 1) & 1, abort_flag)) *abort_flag = 1;
                __half2 x[kPr];
                GQLA_SPAN_BEGIN(b1);
                {
                    const uint4 *src =
                        reinterpret_cast<const uint4 *>(xbuf + sb * SM::kX + w * SM::kXw + lane * (kTokW * 2));
#pragma unroll
                    for (int j4 = 0; j4 < kPr / 4; ++j4) {
                        const uint4 pv = src[j4];
                        const uint32_t pw4[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            x[4 * j4 + e] = __hadd2(*reinterpret_cast<const __half2 *>(&hc[4 * j4 + e]),
                                                    *reinterpret_cast<const __half2 *>(&pw4[e]));
                    }
                }
                // the peer may refill our receive buffer sb (the values above are consumed)
                __syncwarp();
                if (lane == 0) mbar_arrive_remote_relaxed(xempty_remote + sb * 8);
                GQLA_SPAN_END(20, b1);
                GQLA_SPAN_BEGIN(b2);
                // ---- mask tokens past the sequence or past this query's causal limit
                const int lim = min(last_visible, tok0 + n_valid - 1) - (tok0 + part * kTokW);
                if (lim < kTokW - 1) {
                    const __half ninf = __ushort_as_half((unsigned short)0xFC00u);
#pragma unroll
                    for (int j = 0; j < kPr; ++j) {
                        if (2 * j > lim) x[j].x = ninf;
                        if (2 * j + 1 > lim) x[j].y = ninf;
                    }
                }
                // ---- row maximum over the 64 tokens (exchange among the quadrant's warps)
                __half2 hm;
                {
                    __half2 tr[kPr];
#pragma unroll
                    for (int j = 0; j < kPr; ++j) tr[j] = x[j];
#pragma unroll
                    for (int st = kPr / 2; st >= 1; st >>= 1)
#pragma unroll
                        for (int j = 0; j < st; ++j) tr[j] = __hmax2(tr[j], tr[j + st]);
                    hm = tr[0];
                }
                const float mx = fmaxf(__low2float(hm), __high2float(hm)) * p.scale_log2;  // log2 units
                rm[((tt & 1) * kParts + part) * kRows + row] = mx;
                quad_bar(quad);
                float mt = mx;
#pragma unroll
                for (int q = 0; q < kParts; ++q) mt = fmaxf(mt, rm[((tt & 1) * kParts + q) * kRows + row]);
                GQLA_SPAN_END(21, b2);
                const bool first = i == 0;
                float m_new = m_run;
                if (first || mt > m_run + kRescaleLog2) m_new = mt;
                const bool need = !first && m_new != m_run;
                const float alpha = need ? fast_exp2(m_run - m_new) : 1.0f;
                // P buffer sb is free once PV(tt - 2) completed
                if (!GQLA_WAIT(9, &p_free[sb], ((tt >> 1) & 1) ^ 1, abort_flag)) *abort_flag = 1;
                tc_fence_after();
                if (__any_sync(0xffffffffu, need)) {
                    // O rows are rescaled only after PV(tt - 1) has completed
                    if (!first)
                        if (!mbar_wait(&p_free[sb ^ 1], ((tt - 1) >> 1) & 1, abort_flag)) *abort_flag = 1;
                    tc_fence_after();
#pragma unroll 1
                    for (int c16 = 0; c16 < 256 / kParts; c16 += 16) {  // this warp's share of the O columns
                        uint32_t r[16];
                        const uint32_t ta = t_o + lane_off + part * (256 / kParts) + c16;
                        tmem_ld16(ta, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                        tmem_st16(ta, r);
                    }
                    tmem_wait_st();
                }
                l_run = first ? 0.0f : l_run * alpha;
                m_run = m_new;
                // ---- P = 2^(x scale - m) (fp32 ex2) in bf16 -- the top half of the fp32
                // value, rounded towards zero; the row sum adds the same truncated values,
                // so O / l stays unbiased -- into shared memory: bytes
                // [2 kTokW part, 2 kTokW (part + 1)) of the row
                GQLA_SPAN_BEGIN(b3);
                const float mu = m_run == -INFINITY ? 0.0f : m_run;
                uint32_t pw[kPr];
                float lsum = 0.0f;
#pragma unroll
                for (int j = 0; j < kPr; ++j) {
                    const float2 xf = __half22float2(x[j]);
                    const uint32_t p0 = __float_as_uint(fast_exp2(fmaf(xf.x, p.scale_log2, -mu)));
                    const uint32_t p1 = __float_as_uint(fast_exp2(fmaf(xf.y, p.scale_log2, -mu)));
                    pw[j] = __byte_perm(p0, p1, 0x7632);
                    lsum += __uint_as_float(p0 & 0xFFFF0000u) + __uint_as_float(p1 & 0xFFFF0000u);
                }
                l_run += lsum;
                GQLA_SPAN_END(22, b3);
                GQLA_SPAN_BEGIN(b4);
                {
                    uint8_t *prow_s = smem + SM::oP + sb * SM::kP + row * 128;
#pragma unroll
                    for (int j = 0; j < kPr / 4; ++j)
                        *reinterpret_cast<uint4 *>(prow_s + (((part * (kPr / 4) + j) ^ (row & 7)) << 4)) =
                            make_uint4(pw[4 * j], pw[4 * j + 1], pw[4 * j + 2], pw[4 * j + 3]);
                }
                // latent rows that are not tokens (never written, maybe NaN) -> 0
                if (n_valid < kT) {
                    if (!mbar_wait(&ring_full[slot], (tt / kRing) & 1, abort_flag)) *abort_flag = 1;
                    uint8_t *tile = smem + SM::oRing + slot * SM::kSlot;
                    const int nz = kT - n_valid;
                    for (int z = w * 32 + lane; z < 4 * nz * 8; z += kSmThreads) {
                        const int box = z / (nz * 8), rem = z % (nz * 8);
                        *reinterpret_cast<uint4 *>(tile + box * SM::kLatBox + (n_valid + rem / 8) * 128 +
                                                   (rem % 8) * 16) = make_uint4(0, 0, 0, 0);
                    }
                }
                fence_proxy_async_smem();  // P (and any zeroed rows) -> the PV MMA
                tc_fence_before();
                mbar_arrive(&p_full[sb]);
                GQLA_SPAN_END(23, b4);
                GQLA_SPAN_END(10, t_tile);
                if (i + 1 < nt && !have_next) stage_a(i + 1, hn);
                have_next = false;
                page = page_next;
#pragma unroll
                for (int j = 0; j < kPr; ++j) hc[j] = hn[j];
            }
            t = t0 + nt;
            // the last scores of the piece are read: the producer may load the next RoPE q~,
            // and the next piece's q~ goes into TMEM now, so that its scores overlap this epilogue
            __syncwarp();
            if (lane == 0) mbar_arrive(q_empty);
            bool more_pieces;
            {
                PieceIter nx = it;
                int b2, L2, pb2, pe2;
                bool tl2 = false;
                do {
                    more_pieces = next_piece(p, nx, b2, L2, pb2, pe2, tl2);
                } while (more_pieces && tl2);
                if (more_pieces) {
                    copy_q(b2);
                    q_loaded = true;
                }
            }
            // ---- epilogue: O / l for this CTA's 256 columns (this warp: 256 / kParts) through
            // TMA stores staged in shared memory.  After the last piece the ring is free
            // (every tile is consumed) and holds all of it: 8 KB per warp, two 128-byte-swizzled
            // boxes, one store round.  Between pieces the ring holds the next piece's tiles, so
            // each warp stages 2 KB at a time in the P buffers (free once the piece's last PV
            // is done).  LSE by rank 0.
            GQLA_SPAN_BEGIN(t_epi);
            if (!GQLA_WAIT(15, o_done, k & 1, abort_flag)) *abort_flag = 1;
            tc_fence_after();
            lsm[part * kRows + row] = l_run;
            quad_bar(quad);
            float l = 0.0f;
#pragma unroll
            for (int q = 0; q < kParts; ++q) l += lsm[q * kRows + row];
            const float inv = l > 0.0f ? 1.0f / l : 0.0f;
            const bool live = row < rows_here;
            const int64_t orow = (int64_t)(b + c) * p.rows_total + grow;  // slot b + c
            const int orow0 = (b + c) * p.rows_total + rb * kRows + 32 * quad;
            const int ocol0 = 256 * (int)rank + part * (256 / kParts);
            if (!more_pieces) {
                uint8_t *stg = smem + SM::oRing + w * 8192;  // [2 boxes][32 rows][128 B]
#pragma unroll
                for (int j = 0; j < 256 / kParts / 16; ++j) {
                    uint32_t r[16];
                    tmem_ld16(t_o + lane_off + part * (256 / kParts) + 16 * j, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {  // 128-byte swizzle: chunk ^= row % 8
                        const int chunk = (j & 1) * 4 + q4;
                        *reinterpret_cast<float4 *>(stg + (j >> 1) * 4096 + lane * 128 + ((chunk ^ (lane & 7)) << 4)) =
                            make_float4(__uint_as_float(r[4 * q4]) * inv, __uint_as_float(r[4 * q4 + 1]) * inv,
                                        __uint_as_float(r[4 * q4 + 2]) * inv, __uint_as_float(r[4 * q4 + 3]) * inv);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && quad_live && !*abort_flag) {
                    tma_store_2d(&o_map_wide, stg, ocol0, orow0);
                    tma_store_2d(&o_map_wide, stg + 4096, ocol0 + 32, orow0);
                    bulk_commit_group();
                }
            } else {
                uint8_t *stg = smem + SM::oP + w * 2048;  // [32 rows][16 fp32], 64-byte swizzle
#pragma unroll 1
                for (int j = 0; j < 256 / kParts / 16; ++j) {
                    if (j > 0) {
                        if (lane == 0) bulk_wait_group_read<0>();  // the previous chunk's store has read stg
                        __syncwarp();
                    }
                    uint32_t r[16];
                    tmem_ld16(t_o + lane_off + part * (256 / kParts) + 16 * j, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)  // 64-byte swizzle: chunk ^= (row / 2) % 4
                        *reinterpret_cast<float4 *>(stg + lane * 64 + ((q4 ^ ((lane >> 1) & 3)) << 4)) =
                            make_float4(__uint_as_float(r[4 * q4]) * inv, __uint_as_float(r[4 * q4 + 1]) * inv,
                                        __uint_as_float(r[4 * q4 + 2]) * inv, __uint_as_float(r[4 * q4 + 3]) * inv);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0 && quad_live && !*abort_flag) {
                        tma_store_2d(&o_map_narrow, stg, ocol0 + 16 * j, orow0);
                        bulk_commit_group();
                    }
                }
                if (lane == 0) bulk_wait_group_read<0>();
                // every warp's staging (spread over all the P rows) is read before any P is rewritten
                softmax_bar();
            }
            if (live && rank == 0 && part == 0)
                p.lse_part[orow] = (l > 0.0f && m_run != -INFINITY)
                                       ? (m_run + __log2f(l)) * 0.6931471805599453f
                                       : -INFINITY;
            tc_fence_before();
            GQLA_SPAN_END(16, t_epi);
            ++k;
        }
        if (lane == 0) bulk_wait_group<0>();  // the partials are written before the CTA exits
    }

    GQLA_PROF_FLUSH;
    __syncthreads();
    if (*abort_flag && threadIdx.x == 0) report_error(p.ws, GQLA_ERR_TIMEOUT, c);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    cluster_sync();  // no remote access may target a CTA that has exited
}

// 2D bf16 map over [rows][576] with a box of `box_cols` x `box_rows`.
bool make_row_map(CUtensorMap *map, const void *base, uint64_t rows, uint32_t box_cols,
                  uint32_t box_rows, CUtensorMapSwizzle swizzle) {
    const uint64_t dims[2] = {(uint64_t)kRow, rows};
    const uint64_t strides[1] = {(uint64_t)kRow * 2};
    const uint32_t box[2] = {box_cols, box_rows};
    return make_bf16_map(map, base, 2, dims, strides, box, swizzle);
}

}  // namespace

cudaError_t launch_decode_absorb(const void *qa, int s_q, int heads, const void *cache,
                                 const gqla_kv_index *idx, int num_splits, float scale,
                                 float *o_part, float *lse_part, void *ws, cudaStream_t stream) {
    CUtensorMap lat, rope, qrope, omap_w, omap_n;
    const uint64_t slots = (uint64_t)idx->num_pages * kPage;
    const uint64_t qrows = (uint64_t)idx->batch * s_q * heads;
    if (!make_row_map(&lat, cache, slots, 64, kT, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_row_map(&rope, cache, slots, 32, kT, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_row_map(&qrope, qa, qrows, 32, kRows, CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    {
        // partials fp32 [B + C][s_q][h][512]: 32 x 32 boxes (128-byte rows) for the last
        // piece's stores, 16 x 32 boxes for those between pieces
        const uint64_t orows = (uint64_t)(idx->batch + num_splits) * s_q * heads;
        const uint64_t dims[2] = {(uint64_t)kLatent, orows};
        const uint64_t strides[1] = {(uint64_t)kLatent * 4};
        const uint32_t box_w[2] = {32, 32}, box_n[2] = {16, 32};
        if (!make_map(&omap_w, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, o_part, 2, dims, strides, box_w,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map(&omap_n, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, o_part, 2, dims, strides, box_n,
                      CU_TENSOR_MAP_SWIZZLE_64B))
            return cudaErrorInvalidValue;
    }
    AbsorbParams p;
    p.page_table = idx->page_table;
    p.seqlens = idx->seqlens;
    p.qa = static_cast<const __nv_bfloat16 *>(qa);
    p.o_part = o_part;
    p.lse_part = lse_part;
    p.ws = ws;
    p.batch = idx->batch;
    p.max_pages = idx->max_pages_per_seq;
    p.num_pages = idx->num_pages;
    p.num_splits = num_splits;
    p.s_q = s_q;
    p.heads = heads;
    p.rows_total = s_q * heads;
    p.row_blocks = (p.rows_total + kRows - 1) / kRows;
    p.scale_log2 = scale * kLog2e;
    cudaError_t e = cudaFuncSetAttribute(decode_absorb_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, AbsorbSmem::kAlloc);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)num_splits * p.row_blocks * 2;
    return launch_dependent(decode_absorb_tc_kernel, dim3(grid), dim3(kThreads), AbsorbSmem::kAlloc,
                            stream, lat, rope, qrope, omap_w, omap_n, p);
}

}  // namespace gqla
