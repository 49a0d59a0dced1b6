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
// byte of the cache exactly once) and computes a partial score tile over
// them.  The softmax rows are split too: row i of the block belongs to rank
// (i / 16) % 2.  Each CTA sends the peer the fp32 partials of the peer's rows,
// adds the two partials of its own 64 rows, computes their P (bf16) and sends
// those P rows, with each row's O rescale factor, back; both CTAs then hold P
// for all 128 rows and each accumulates its own 256 columns of O.
//
//  * Tile = one 64-token page (an MMA instruction costs about the same at any
//    N up to 64).  Tensor memory holds O (256 columns), a double-buffered S
//    (2 x 64) and the latent half of q~ (128 columns of bf16 pairs: the score
//    MMA reads q~ from TMEM); P goes through shared memory, beside a 4-slot
//    ring of latent tiles and a 2-slot ring of RoPE tiles (the RoPE columns
//    are read by the score MMAs only, so their slot frees a whole PV earlier).
//  * Roles, 19 warps:
//      warp 0      TMA producer of the rings (4 latent boxes 128B-swizzled, 32 KB,
//                  and 1 RoPE box 64B-swizzled, 4 KB, per tile), cache tiles read
//                  with an L2 evict-first policy;
//      warp 1      TMEM owner, issues S = q~ C^T;
//      warps 2-9   score warps, two per TMEM lane quadrant, 32 tokens each.  Stage A
//                  of tile j: the fp32 partial scores of the CTA's own rows go to its
//                  local buffer, those of the peer's rows to a staging block that
//                  leaves as one 2 KB bulk copy per warp into the peer's receive buffer.
//                  Stage C of tile j - 1, only when the PV warp asks for it: O rows
//                  whose maximum rose are rescaled.  Also each piece's RoPE q~ (by
//                  TMA, as soon as the previous piece's scores are complete) and the
//                  epilogue;
//      warps 10-17 softmax warps of the CTA's 64 rows (stage B), four lanes per
//                  row: the two fp32 partials added, row maxima (lazy rescaling: a
//                  maximum has to rise by more than 2^8), P = 2^(s - m) written to
//                  both CTAs' P buffers (bulk copy of each warp's 8 rows, and one of
//                  their rescale factors); also the
//                  q~ copies into TMEM, each piece's next q~ prefetched into L2;
//      warp 18     waits for P of all 128 rows and issues O += P C in tile order; it
//                  zeroes the latent rows past a ragged sequence end and hands a tile to
//                  the score warps (stage C) only when some row's maximum rose.
//    The stages of consecutive tiles overlap: the score warps run A(j) while the
//    softmax warps run B(j - 1).  Every score is the fp32 sum of two fp32
//    partials: no precision is given up in the exchange.
//  * The epilogue writes O / l with TMA stores of 32 x 32 fp32 boxes staged in
//    shared memory: in the idle ring after the last piece, in the P buffers
//    between pieces.
//  * Every wait is bounded and reports GQLA_ERR_TIMEOUT instead of hanging;
//    both CTAs of a cluster always execute the same sequence of steps.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "sm100.cuh"
#include "tensor_map.cuh"

namespace gqla {

// Set by gqla_debug_drop_v_load, consumed by the next decode launch of the thread.
extern thread_local int g_drop_v_unit;

namespace {

using namespace sm100;

constexpr int kXWarps = 8;                  // score warps: two per TMEM lane quadrant
constexpr int kYWarps = 8;                  // softmax warps of the CTA's own rows
constexpr int kSmWarps = kXWarps + kYWarps;
constexpr int kThreads = 32 * (3 + kSmWarps);
constexpr int kPvWarp = 2 + kSmWarps;       // warp issuing O += P C
constexpr int kRows = 128;           // MMA M: query rows of one row block (zero-padded)
constexpr int kT = 64;               // tokens per tile (one page)
constexpr int kRing = 4;
constexpr float kRescaleLog2 = 8.0f;
constexpr int kXThreads = 32 * kXWarps;
constexpr int kXTok = kT / 2;               // tokens of a tile per score warp
constexpr int kXCols = 256 / 2;             // O columns per score warp
constexpr int kOwn = kRows / 2;             // rows whose softmax a CTA of the pair computes

struct AbsorbSmem {
    static constexpr int kQRope = kRows * 64;             // q~ RoPE columns [128 rows][32]
    static constexpr int kLatBox = kT * 128;              // [64 tokens][64 cols]
    static constexpr int kRopeBox = kT * 64;              // [64 tokens][32 cols]
    static constexpr int kSlot = 4 * kLatBox;             // latent ring slot, 32 KB
    static constexpr int kRopeRing = 2;
    // fp32 partial scores of this CTA's 64 rows in two token halves, [2][64 rows][32
    // tokens]: a half row is 128 bytes, eight 16-byte chunks stored at xoff(); the 16 rows
    // of one lane quadrant in one half are what one score warp computes, 2 KB in one piece,
    // so the peer's blocks arrive as whole bulk copies.  Read 16 tokens per lane (four
    // lanes per row).  One buffer for this CTA's partials and one for the peer's: the
    // softmax warps of both CTAs read tile j at the start of their stage B; the score warps
    // write tile j + 1 into the local buffer once this CTA's softmax warps have read it and
    // send it into the peer's once the peer's have.
    static constexpr int kX = kOwn * kT * 4;
    static constexpr int kXBlock = 16 * 32 * 4;           // one score warp's block, 2 KB
    static constexpr int kP = kRows * kT * 2;             // P, [128 rows][64 tokens] bf16, 128B-swizzled
    // the peer's 64 rows of P and their O rescale factors (bulk copies)
    static constexpr int kPRemote = kOwn * kT * 2 + kOwn * 4;
    static constexpr int oQ = 0;
    static constexpr int oP = oQ + kQRope;                // 2 buffers
    static constexpr int oRing = oP + 2 * kP;
    static constexpr int oRope = oRing + kRing * kSlot;   // kRopeRing RoPE tiles
    static constexpr int oXR = oRope + kRopeRing * kRopeBox;  // the peer's partials
    static constexpr int oXL = oXR + kX;                      // this CTA's partials
    static constexpr int oXStage = oXL + kX;              // [8 score warps] outgoing blocks
    static constexpr int oAlpha = oXStage + kXWarps * kXBlock;  // float [2 buffers][128 rows]
    static constexpr int oL = oAlpha + 2 * kRows * 4;     // float [128 rows]: row sums of a piece
    static constexpr int oBar = oL + kRows * 4;
    // ring_full/empty[kRing], rope_full/empty[kRopeRing], q_full, s_full/s_free[2],
    // x_full, x_empty_l, x_empty_r, p_full/p_empty[2], o_ready, c_dec[2], pv_done[2], l_full,
    // o_done, drain[2]
    static constexpr int kNumBars = 2 * kRing + 2 * kRopeRing + 1 + 4 + 3 + 4 + 3 + 2 + 1 + 1 + 2;
    static constexpr int oMisc = oBar + kNumBars * 8;     // tmem base, abort, plan[4], c_flag[2]
    static constexpr int kBytes = oMisc + 32;
    static constexpr int kAlloc = kBytes + 1024;
};
static_assert(AbsorbSmem::kAlloc <= 227 * 1024, "shared memory");
static_assert(AbsorbSmem::oRing % 1024 == 0 && AbsorbSmem::oRope % 512 == 0 && AbsorbSmem::oP % 1024 == 0,
              "swizzle atoms of the MMA operands");
// the last piece's epilogue stages every score warp's 32 x 128 fp32 block in the idle ring
static_assert(kXWarps * 32 * kXCols * 4 <= kRing * AbsorbSmem::kSlot, "epilogue staging");

// Byte offset of logical chunk c (tokens 4c .. 4c + 3, c < 16) of partial-score row r in a
// partial buffer: token half c / 8, then the row, then the chunk, XOR-swizzled so that both
// a lane writing the eight chunks of its half row (8 rows a phase, one chunk each) and four
// lanes reading four chunks of one row (two rows a phase) meet no bank conflict.
__device__ __forceinline__ int xoff(int r, int c) {
    const int x = c >> 3;
    return x * (kOwn * 128) + r * 128 + (((c & 7) ^ (r & 7) ^ (x << 1)) << 4);
}

struct AbsorbParams {
    const int32_t *page_table;
    const int32_t *seqlens;
    const __nv_bfloat16 *qa;
    float *o_part;
    float *lse_part;
    void *ws;
    int batch, max_pages, num_pages, num_splits, s_q, heads;
    int lead, lead_w16;  // the split plan's lead chunks and their length (x 1/16)
    int rows_total;   // s_q * heads: query rows of one sequence
    int row_blocks;   // ceil(rows_total / 128)
    float scale_log2;
    // diagnostic: the latent load of this tile (issue order within a CTA) is never issued,
    // so a bounded wait runs out (-1: none)
    int drop_tile;
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

// Is a piece that is not skipped still to come after `it`?  (`b2` its sequence.)
__device__ __forceinline__ bool another_piece(const AbsorbParams &p, PieceIter it, int &b2) {
    int L2, pb2, pe2;
    bool tl2 = false, more;
    do {
        more = next_piece(p, it, b2, L2, pb2, pe2, tl2);
    } while (more && tl2);
    return more;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    decode_absorb_tc_kernel(const __grid_constant__ CUtensorMap lat_map,
                            const __grid_constant__ CUtensorMap rope_map,
                            const __grid_constant__ CUtensorMap qrope_map,
                            const __grid_constant__ CUtensorMap o_map, const AbsorbParams p) {
    using SM = AbsorbSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::oBar);
    uint64_t *ring_full = bars, *ring_empty = bars + kRing;
    uint64_t *rope_full = bars + 2 * kRing, *rope_empty = rope_full + SM::kRopeRing;
    uint64_t *q_full = rope_empty + SM::kRopeRing;
    uint64_t *s_full = q_full + 1, *s_free = s_full + 2;
    uint64_t *x_full = s_free + 2, *x_empty_l = x_full + 1, *x_empty_r = x_empty_l + 1;
    uint64_t *p_full = x_empty_r + 1, *p_empty = p_full + 2;
    uint64_t *o_ready = p_empty + 2, *c_dec = o_ready + 1, *pv_done = c_dec + 2;
    uint64_t *l_full = pv_done + 2, *o_done = l_full + 1, *drain = o_done + 1;
    uint32_t *tmem_base_smem = reinterpret_cast<uint32_t *>(smem + SM::oMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + SM::oMisc + 4);
    int *plan = reinterpret_cast<int *>(smem + SM::oMisc + 8);
    // per P buffer: whether the score warps rescale O rows before that tile's PV
    volatile int *c_flag = reinterpret_cast<volatile int *>(smem + SM::oMisc + 24);
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
        for (int i = 0; i < SM::kRopeRing; ++i) { mbar_init(&rope_full[i], 1); mbar_init(&rope_empty[i], 1); }
        mbar_init(q_full, 1 + kYWarps);  // RoPE TMA + the softmax warps' TMEM copies
        mbar_init(x_full, 1 + kXWarps);  // expect_tx of the peer's partials + local score warps
        mbar_init(x_empty_l, kYWarps);   // this CTA's softmax warps have read both buffers
        mbar_init(x_empty_r, kYWarps);   // the peer's softmax warps have read both of theirs
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1); mbar_init(&s_free[i], kXThreads);
            mbar_init(&p_full[i], 1 + kYWarps);      // expect_tx of the peer's rows + local softmax warps
            mbar_init(&p_empty[i], 2);               // PV of both CTAs done with the buffer
            mbar_init(&c_dec[i], 1);
            mbar_init(&pv_done[i], 1);
            mbar_init(&drain[i], 1);
        }
        mbar_init(o_ready, kXWarps);  // only for tiles whose O rows the score warps rescale
        mbar_init(l_full, 1 + kYWarps);
        mbar_init(o_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    griddep_wait();  // the previous kernel's results are visible from here on
    // The combine may be scheduled as soon as every CTA has started: its set-up (split plan,
    // W_UV) then overlaps this kernel's tail.  Not with lead chunks: the SMs of the CTAs that
    // finish first belong to the GQA decode running beside this one, and a combine waiting
    // there for the last CTA would hold them.
    if (p.lead == 0) griddep_launch_dependents();
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
        int r0, r1;
        plan_chunk_range(total, SplitPlan{p.num_splits, p.lead, p.lead_w16}, c, &r0, &r1);
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
    // A thread whose wait runs out stops its CTA and the peer (both abort flags): every
    // role then leaves its loops at its next wait.  After a failed wait a role neither
    // arrives on a barrier nor sends anything -- an arrival for tile j + 1 on a barrier
    // whose phase j still waits for bytes would break the barrier's count -- so the
    // only traffic left is what was already in flight.
    const uint32_t abort_remote = map_peer(smem_u32(const_cast<int *>(abort_flag)), peer);
    auto give_up = [&]() {
        *abort_flag = 1;
        st_cluster_b32(abort_remote, 1u);
    };

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        // Lane 0 issues; the whole warp fetches the page indices 32 at a time so
        // that no page-table load sits between two tiles.
        const uint64_t stream_policy = l2_evict_first_policy();  // the cache is read once
        PieceIter it = it0;
        int b, L, pb, pe;
        bool too_long, quit = false;
        uint32_t t = 0, n_rope = 0;  // tiles whose latent / RoPE slot was armed (or skipped)
        while (!quit && next_piece(p, it, b, L, pb, pe, too_long)) {
            if (too_long) {
                if (lane == 0 && rank == 0 && rb == 0) report_error(p.ws, GQLA_ERR_DEVICE, b);
                continue;
            }
            const int32_t *prow = p.page_table + (int64_t)b * p.max_pages;
            for (int i0 = pb; i0 < pe && !quit; i0 += 32) {
                const int n = min(32, pe - i0);
                // (the first piece is the one the early load above was for)
                const int my_page = pre_ok ? pre_page : (lane < n ? prow[i0 + lane] : 0);
                pre_ok = false;
                for (int j = 0; j < n; ++j) {
                    const int page = __shfl_sync(0xffffffffu, my_page, j);
                    int ok = 1;
                    if (lane == 0) {
                        const bool bad = page < 0 || page >= p.num_pages;
                        if (bad && rank == 0 && rb == 0) report_error(p.ws, GQLA_ERR_DEVICE, b);
                        const int slot = t % kRing, rs = t % SM::kRopeRing;
                        if (!GQLA_WAIT(0, &ring_empty[slot], ((t / kRing) & 1) ^ 1, abort_flag)) {
                            give_up();
                            ok = 0;
                        } else {
                            uint8_t *dst = smem + SM::oRing + slot * SM::kSlot;
                            if ((int)t == p.drop_tile) {
                                // diagnostic: neither the load nor an arrival for this tile
                            } else if (!bad) {
                                mbar_arrive_expect_tx(&ring_full[slot], SM::kSlot);
#pragma unroll
                                for (int bx = 0; bx < 4; ++bx)
                                    tma_load_2d_hint(dst + bx * SM::kLatBox, &lat_map, &ring_full[slot],
                                                     256 * rank + 64 * bx, page * kPage, stream_policy);
                            } else {
                                mbar_arrive(&ring_full[slot]);
                            }
                            ++t;
                            // the RoPE slot frees once the score MMAs of tile t - kRopeRing are done
                            if (!GQLA_WAIT(1, &rope_empty[rs], ((n_rope / SM::kRopeRing) & 1) ^ 1, abort_flag)) {
                                give_up();
                                ok = 0;
                            } else {
                                if (!bad) {
                                    mbar_arrive_expect_tx(&rope_full[rs], SM::kRopeBox);
                                    tma_load_2d_hint(smem + SM::oRope + rs * SM::kRopeBox, &rope_map, &rope_full[rs],
                                                     512 + 32 * rank, page * kPage, stream_policy);
                                } else {
                                    mbar_arrive(&rope_full[rs]);
                                }
                                ++n_rope;
                            }
                        }
                    }
                    if (!__shfl_sync(0xffffffffu, ok, 0)) {
                        quit = true;
                        break;
                    }
                }
            }
        }
        if (lane == 0) {
            // no TMA may still be writing when the CTA exits: wait (bounded) for the last
            // loads of both rings (a slot left without its load, on purpose or by giving
            // up, just lets its wait run out)
            int dummy = 0;
            volatile int *no_abort = reinterpret_cast<volatile int *>(&dummy);
            for (uint32_t u = (t > (uint32_t)kRing ? t - kRing : 0); u < t; ++u)
                mbar_wait(&ring_full[u % kRing], (u / kRing) & 1, no_abort);
            for (uint32_t u = (n_rope > (uint32_t)SM::kRopeRing ? n_rope - SM::kRopeRing : 0); u < n_rope; ++u)
                mbar_wait(&rope_full[u % SM::kRopeRing], (u / SM::kRopeRing) & 1, no_abort);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- score MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16(kRows, kT, 0, 0);
            // descriptors of ring slot 0 and of the RoPE q~; a single issuing thread pays
            // for every instruction of a descriptor, so each MMA only adds an offset
            const uint64_t lat_d0 = smem_desc(sm_ring, 16, 1024, kSw128);
            const uint64_t rope_d0 = smem_desc(smem_u32(smem + SM::oRope), 16, 512, kSw64);
            const uint64_t q_d0 = smem_desc(sm_q, 16, 512, kSw64);
            PieceIter it = it0;
            int b, L, pb, pe;
            bool too_long;
            uint32_t t = 0, k = 0;
            bool quit = false;
            while (!quit && next_piece(p, it, b, L, pb, pe, too_long)) {
                if (too_long) continue;
                if (!GQLA_WAIT(2, q_full, k & 1, abort_flag)) {
                    give_up();
                    break;
                }
                for (int i = 0; i < pe - pb; ++i, ++t) {
                    const int slot = t % kRing, sb = t & 1, rs = t % SM::kRopeRing;
                    if (!GQLA_WAIT(3, &ring_full[slot], (t / kRing) & 1, abort_flag) ||
                        !GQLA_WAIT(3, &rope_full[rs], (t / SM::kRopeRing) & 1, abort_flag) ||
                        !GQLA_WAIT(4, &s_free[sb], ((t >> 1) & 1) ^ 1, abort_flag)) {
                        give_up();
                        quit = true;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t lat_d = desc_advance(lat_d0, slot * SM::kSlot);
                    const uint64_t rope_d = desc_advance(rope_d0, rs * SM::kRopeBox);
                    const uint32_t t_sb = t_s + sb * kT;
#pragma unroll
                    for (int ks = 0; ks < 16; ++ks)  // latent: A = q~ in TMEM, 16 dims = 8 columns
                        mma_bf16_ts(t_sb, t_q + ks * 8, desc_advance(lat_d, (ks >> 2) * SM::kLatBox + (ks & 3) * 32),
                                    idesc_s, ks > 0 ? 1u : 0u);
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks)  // RoPE: 32 columns, 64B-swizzled rows
                        mma_bf16(t_sb, desc_advance(q_d0, ks * 32), desc_advance(rope_d, ks * 32), idesc_s, 1u);
                    mma_commit(&s_full[sb]);
                    mma_commit(&rope_empty[rs]);
                }
                ++k;
            }
            mma_commit(&drain[0]);
            int dummy = 0;
            mbar_wait(&drain[0], 0, reinterpret_cast<volatile int *>(&dummy));
        }
    } else if (warp == kPvWarp) {
        // ---------------------------------------------------------------- PV MMA issuer
        // The whole warp waits for P of all 128 rows, checks their O rescale factors and
        // zeroes the latent rows of a ragged tile; lane 0 issues.  Only when some factor is
        // not 1 (a row maximum rose) does it hand the tile to the score warps (c_flag, c_dec)
        // and wait for their rescaling (o_ready) first; otherwise PV follows P at once.
        const float *alph = reinterpret_cast<const float *>(smem + SM::oAlpha);
        constexpr uint32_t idesc_pv = idesc_bf16(kRows, 256, 0, 1);
        const uint64_t v_d0 = smem_desc(sm_ring, SM::kLatBox, 1024, kSw128);
        const uint64_t p_d0 = smem_desc(sm_p, 16, 1024, kSw128);
        PieceIter it = it0;
        int b, L, pb, pe;
        bool too_long;
        uint32_t t = 0, n_c = 0;  // n_c: tiles handed to the score warps so far
        bool quit = false;
        while (!quit && next_piece(p, it, b, L, pb, pe, too_long)) {
            if (too_long) continue;
            const int32_t *prow = p.page_table + (int64_t)b * p.max_pages;
            for (int i = 0; i < pe - pb; ++i, ++t) {
                const int slot = t % kRing, sb = t & 1;
                const int page = prow[pb + i];
                if (!__all_sync(0xffffffffu, GQLA_WAITC(5, &p_full[sb], (t >> 1) & 1, abort_flag))) {
                    if (lane == 0) give_up();
                    quit = true;
                    break;
                }
                // P buffer sb takes tile t + 2's rows from the peer, which the peer sends only
                // after PV(t) below has freed the buffer in both CTAs
                if (lane == 0) mbar_arrive_expect_tx(&p_full[sb], SM::kPRemote);
                const float4 a4 = reinterpret_cast<const float4 *>(alph + sb * kRows)[lane];
                const bool need_c =
                    __any_sync(0xffffffffu, a4.x != 1.0f || a4.y != 1.0f || a4.z != 1.0f || a4.w != 1.0f);
                const bool bad = page < 0 || page >= p.num_pages;
                const int n_valid = bad ? 0 : max(0, min(kT, L - (pb + i) * kPage));
                if (n_valid < kT) {
                    // latent rows that are not tokens (never written, maybe NaN) -> 0, once the
                    // tile's load has landed
                    if (!__all_sync(0xffffffffu, mbar_wait(&ring_full[slot], (t / kRing) & 1, abort_flag))) {
                        if (lane == 0) give_up();
                        quit = true;
                        break;
                    }
                    uint8_t *tile = smem + SM::oRing + slot * SM::kSlot;
                    const int nz = kT - n_valid;
                    for (int z = lane; z < 4 * nz * 8; z += 32) {
                        const int box = z / (nz * 8), rem = z % (nz * 8);
                        *reinterpret_cast<uint4 *>(tile + box * SM::kLatBox + (n_valid + rem / 8) * 128 +
                                                   (rem % 8) * 16) = make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_smem();  // the zeros -> the PV MMAs (async proxy)
                }
                __syncwarp();
                if (lane == 0) {
                    c_flag[sb] = need_c ? 1 : 0;
                    mbar_arrive(&c_dec[sb]);
                }
                if (need_c) {
                    if (!__all_sync(0xffffffffu, GQLA_WAIT(10, o_ready, n_c & 1, abort_flag))) {
                        if (lane == 0) give_up();
                        quit = true;
                        break;
                    }
                    ++n_c;
                }
                if (lane == 0) {
                    tc_fence_after();
                    // B = C_lat[tokens][256 cols of this CTA]: MN-major, 4 atoms of 64 columns;
                    // A = P[128 rows][64 tokens], K-major: 16 tokens = 32 bytes of a row
                    const uint64_t v_d = desc_advance(v_d0, slot * SM::kSlot);
                    const uint64_t p_d = desc_advance(p_d0, sb * SM::kP);
#pragma unroll
                    for (int ks = 0; ks < kT / 16; ++ks)
                        mma_bf16(t_o, desc_advance(p_d, ks * 32), desc_advance(v_d, ks * 2048), idesc_pv,
                                 (i == 0 && ks == 0) ? 0u : 1u);
                    mma_commit_multicast(&p_empty[sb], 0x3);  // P buffer sb of both CTAs is free
                    mma_commit(&pv_done[sb]);
                    mma_commit(&ring_empty[slot]);
                }
                __syncwarp();
            }
            if (!quit && lane == 0) mma_commit(o_done);
        }
        if (lane == 0) {
            mma_commit(&drain[1]);
            int dummy = 0;
            mbar_wait(&drain[1], 0, reinterpret_cast<volatile int *>(&dummy));
        }
    } else if (warp < 2 + kXWarps) {
        // ---------------------------------------------------------------- score warps
        // Stage A of tile j: fp32 partial scores -> the owner of each row (row r of the
        // block belongs to rank (r / 16) % 2, so both CTAs use all four TMEM lane quadrants);
        // stage C of tile j - 1, when the PV warp found a rescale factor that is not 1: O
        // rows are rescaled where a row maximum rose and PV is released.  Also the q~
        // copies into TMEM and the epilogue.  Two warps per lane quadrant: warp half
        // `xpart` takes tokens [32 xpart, 32 xpart + 32) of a tile and O columns
        // [128 xpart, 128 xpart + 128).
        const int quad = warp & 3;
        const int xw = warp - 2;
        const int xpart = xw >> 2;
        const int row = 32 * quad + lane;        // TMEM row
        const uint32_t lane_off = static_cast<uint32_t>(32 * quad) << 16;
        const uint32_t a_owner = (lane >> 4) & 1;   // the owner of this row (stage A)
        const float *alph = reinterpret_cast<const float *>(smem + SM::oAlpha);
        const float *lsm = reinterpret_cast<const float *>(smem + SM::oL);
        const uint32_t x_remote = map_peer(smem_u32(smem + SM::oXR), peer);
        const uint32_t xfull_remote = map_peer(smem_u32(x_full), peer);
        // this lane's row among the owner's 64 rows, and its eight chunks (32 tokens)
        const int xrow = 16 * quad + (lane & 15);
        const bool quad_live = 32 * quad < rows_here;  // rows_here is a multiple of 32
        // the first two tiles' P buffers expect the peer's rows
        if (xw == 0 && lane == 0) {
            mbar_arrive_expect_tx(&p_full[0], SM::kPRemote);
            mbar_arrive_expect_tx(&p_full[1], SM::kPRemote);
        }
        // the RoPE columns of a piece's q~, by TMA: the first piece's at once, each next
        // piece's as soon as this piece's last scores are complete (one thread)
        auto load_rope = [&](int bq) {
            if (xw == 0 && lane == 0) {
                mbar_arrive_expect_tx(q_full, SM::kQRope);
                tma_load_2d(smem + SM::oQ, &qrope_map, q_full, 512 + 32 * rank, bq * p.rows_total + rb * kRows);
            }
        };
        bool rope_issued = false;
        PieceIter it = it0;
        int b, L, pb, pe;
        bool too_long;
        uint32_t t = 0, k = 0;
        while (next_piece(p, it, b, L, pb, pe, too_long)) {
            if (too_long) continue;
            if (!rope_issued) load_rope(b);
            int b_next = 0;
            const bool more_pieces = another_piece(p, it, b_next);  // its tiles then occupy the ring
            rope_issued = more_pieces;
            const uint32_t t0 = t;
            const int nt = pe - pb;
            // Each stage returns false when a wait failed (in any lane): the warp then stops.
            auto stage_a = [&](int i) -> bool {
                const uint32_t tt = t0 + i;
                const int sb = tt & 1;
                if (!__all_sync(0xffffffffu, GQLA_WAIT(6, &s_full[sb], (tt >> 1) & 1, abort_flag))) {
                    if (lane == 0) give_up();
                    return false;
                }
                GQLA_SPAN_BEGIN(t_a);
                tc_fence_after();
                uint32_t sv[kXTok];
                tmem_ld16(t_s + lane_off + sb * kT + kXTok * xpart, sv);
                tmem_ld16(t_s + lane_off + sb * kT + kXTok * xpart + 16, sv + 16);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&s_free[sb]);
                // this CTA's buffer is free once its softmax warps have read tile tt - 1
                if (!__all_sync(0xffffffffu, GQLA_WAIT(7, x_empty_l, (tt & 1) ^ 1, abort_flag))) {
                    if (lane == 0) give_up();
                    return false;
                }
                if (xw == 0 && lane == 0) mbar_arrive_expect_tx(x_full, SM::kX);
                // this lane's row, tokens 32 xpart .. 32 xpart + 31: the CTA's own rows into the
                // local buffer, the peer's rows into this warp's staging block (the peer's half
                // rows 16 quad .. 16 quad + 15), which leaves as one bulk copy
                if (tt > 0) {
                    // the previous tile's outgoing block has been read by its bulk copy
                    if (lane == 0) bulk_wait_group_read<0>();
                    __syncwarp();
                }
                // (the staging block holds the same 16 half rows as their place in the peer's
                // buffer, at the offset of row 16 quad of half xpart there)
                const int base = a_owner == rank ? SM::oXL
                                                 : SM::oXStage + xw * SM::kXBlock - xpart * (kOwn * 128) - 16 * quad * 128;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    *reinterpret_cast<uint4 *>(smem + base + xoff(xrow, 8 * xpart + j)) =
                        make_uint4(sv[4 * j], sv[4 * j + 1], sv[4 * j + 2], sv[4 * j + 3]);
                fence_proxy_async_smem();  // the staging block -> the bulk copy (async proxy)
                __syncwarp();
                if (lane == 0) mbar_arrive(x_full);  // this warp's local partials are in
                // the peer's receive buffer is free once the peer's softmax warps have read tile
                // tt - 1
                if (!__all_sync(0xffffffffu, GQLA_WAITC(7, x_empty_r, (tt & 1) ^ 1, abort_flag))) {
                    if (lane == 0) give_up();
                    return false;
                }
                if (lane == 0) {
                    bulk_copy_to_peer(x_remote + xpart * (kOwn * 128) + 16 * quad * 128,
                                      smem + SM::oXStage + xw * SM::kXBlock, SM::kXBlock, xfull_remote);
                    bulk_commit_group();
                }
                GQLA_SPAN_END(13, t_a);
                return true;
            };
            auto stage_c = [&](int i) -> bool {
                const uint32_t tt = t0 + i;
                const int sb = tt & 1;
                if (!__all_sync(0xffffffffu, GQLA_WAIT(11, &c_dec[sb], (tt >> 1) & 1, abort_flag))) {
                    if (lane == 0) give_up();
                    return false;
                }
                if (!c_flag[sb]) return true;  // no factor is not 1: PV(tt) needs nothing from here
                GQLA_SPAN_BEGIN(t_c);
                const float alpha = alph[sb * kRows + row];
                if (__any_sync(0xffffffffu, alpha != 1.0f)) {
                    // O rows are rescaled only after PV(tt - 1) has completed
                    if (i > 0 && !__all_sync(0xffffffffu, mbar_wait(&pv_done[(tt - 1) & 1], ((tt - 1) >> 1) & 1, abort_flag))) {
                        if (lane == 0) give_up();
                        return false;
                    }
                    tc_fence_after();
#pragma unroll 1
                    for (int c16 = 0; c16 < kXCols; c16 += 16) {
                        uint32_t r[16];
                        const uint32_t ta = t_o + lane_off + kXCols * xpart + c16;
                        tmem_ld16(ta, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                        tmem_st16(ta, r);
                    }
                    tmem_wait_st();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(o_ready);
                GQLA_SPAN_END(18, t_c);
                return true;
            };
            // The two stages run in whichever order their inputs arrive: lane 0 probes,
            // without blocking, the PV warp's decision for the oldest tile still waiting for
            // stage C (first: when it asks for rescaling, its PV holds up the ring) and then
            // the scores of the next tile with the peer's receive buffer free (stage A), and
            // the warp runs the first one that is ready.  Stage A runs at most one tile ahead
            // of stage C, so the PV warp's decision for tile j + 2 (same flag, same barrier)
            // cannot come before this warp has read the one for tile j.  With nothing ready
            // for kWaitCycles (or after an abort) the warp falls back to the stage's own
            // bounded wait, which then reports.
            int ia = 0, ic = 0;
            bool ok = true;
            long long idle_since = clock64();
            while (ok && ic < nt) {
                int act = 0;  // 1: stage A of tile ia, 2: stage C of tile ic
                if (lane == 0) {
                    const uint32_t ta = t0 + ia, tc = t0 + ic;
                    if (ic < ia && mbar_test_wait(&c_dec[tc & 1], (tc >> 1) & 1)) act = 2;
                    else if (ia < nt && ia <= ic + 1 && mbar_test_wait(&s_full[ta & 1], (ta >> 1) & 1) &&
                             mbar_test_wait(x_empty_l, (ta & 1) ^ 1)) act = 1;
                    else if (*abort_flag || clock64() - idle_since > kWaitCycles) act = ic < ia ? 2 : 1;
                }
                act = __shfl_sync(0xffffffffu, act, 0);
                if (act == 1) {
                    ok = stage_a(ia);
                    if (ok && ia == nt - 1 && more_pieces) load_rope(b_next);
                    ++ia;
                    idle_since = clock64();
                } else if (act == 2) {
                    ok = stage_c(ic);
                    ++ic;
                    idle_since = clock64();
                } else {
                    __nanosleep(32);
                }
            }
            if (!ok) break;
            t = t0 + nt;
            // ---- epilogue: O / l for this warp's 32 rows x 128 columns through TMA stores of
            // 32 x 32 fp32 boxes (128-byte swizzle) staged in shared memory.  After the last
            // piece the ring is free (every tile is consumed) and holds all of it, one store
            // round; between pieces the ring holds the next piece's tiles and each warp stages
            // one box at a time in the P buffers (free once the piece's last PV is done; P of
            // the next piece is written only after this warp's next scores).
            GQLA_SPAN_BEGIN(t_epi);
            if (!__all_sync(0xffffffffu, GQLA_WAIT(15, o_done, k & 1, abort_flag) &&
                                             GQLA_WAIT(12, l_full, k & 1, abort_flag))) {
                if (lane == 0) give_up();
                break;
            }
            tc_fence_after();
            const float l = lsm[row];
            const float inv = l > 0.0f ? 1.0f / l : 0.0f;
            const int orow0 = (b + c) * p.rows_total + rb * kRows + 32 * quad;
            const int ocol0 = 256 * (int)rank + kXCols * xpart;
            const bool last = !more_pieces;
            uint8_t *stg0 = last ? smem + SM::oRing + xw * (kXCols * 128) : smem + SM::oP + xw * 4096;
#pragma unroll 1
            for (int m = 0; m < kXCols / 32; ++m) {
                uint8_t *stg = last ? stg0 + m * 4096 : stg0;
                if (!last && m > 0) {
                    if (lane == 0) bulk_wait_group_read<0>();  // the previous box's store has read stg
                    __syncwarp();
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t r[16];
                    tmem_ld16(t_o + lane_off + kXCols * xpart + 32 * m + 16 * h, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)  // 128-byte swizzle: chunk ^= row % 8
                        *reinterpret_cast<float4 *>(stg + lane * 128 + (((4 * h + q4) ^ (lane & 7)) << 4)) =
                            make_float4(__uint_as_float(r[4 * q4]) * inv, __uint_as_float(r[4 * q4 + 1]) * inv,
                                        __uint_as_float(r[4 * q4 + 2]) * inv, __uint_as_float(r[4 * q4 + 3]) * inv);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && quad_live) {
                    tma_store_2d(&o_map, stg, ocol0 + 32 * m, orow0);
                    bulk_commit_group();
                }
            }
            if (lane == 0) bulk_wait_group_read<0>();  // staging read before the next tiles' P
            __syncwarp();
            tc_fence_before();
            GQLA_SPAN_END(16, t_epi);
            ++k;
        }
        if (lane == 0) bulk_wait_group<0>();  // the partials are written before the CTA exits
    } else {
        // ---------------------------------------------------------------- softmax warps
        // Stage B of every tile for this CTA's 64 rows: both partial scores added, row
        // maxima (lazy rescaling of O rows when a maximum rises by more than 2^8), P in
        // bf16 written here and bulk-copied to the same rows of the peer's buffer, with
        // each row's O rescale factor.  Four lanes per row, 16 tokens each.
        const int yw = warp - 2 - kXWarps;
        const int ob = 8 * yw + (lane >> 2);  // owned row index 0..63
        const int brow = 32 * (ob >> 4) + 16 * (int)rank + (ob & 15);
        const int bq4 = lane & 3;             // tokens [16 bq4, 16 bq4 + 16): chunks 2 bq4, 2 bq4 + 1
        const int bgrow = rb * kRows + brow;
        const int s_of_brow = bgrow < p.rows_total ? bgrow / p.heads : p.s_q - 1;
        const bool blive = brow < rows_here;
        // the q~ copies into TMEM: like the score warps, two warps per lane quadrant, warp
        // half `xpart` taking q~ columns [128 xpart, 128 xpart + 128) of the CTA's half
        const int quad = warp & 3, xpart = yw >> 2;
        const int row = 32 * quad + lane;
        const uint32_t lane_off = static_cast<uint32_t>(32 * quad) << 16;
        const int grow = rb * kRows + row;

        float *alph = reinterpret_cast<float *>(smem + SM::oAlpha);
        float *lsm = reinterpret_cast<float *>(smem + SM::oL);
        const uint32_t xempty_remote = map_peer(smem_u32(x_empty_r), peer);
        const uint32_t p_remote = map_peer(sm_p, peer);
        const uint32_t pfull_remote = map_peer(smem_u32(p_full), peer);
        const uint32_t alpha_remote = map_peer(smem_u32(alph), peer);
        const uint32_t l_remote = map_peer(smem_u32(lsm), peer);
        const uint32_t lfull_remote = map_peer(smem_u32(l_full), peer);
        // this warp's share of q~'s latent half (32 rows x 128 columns) into TMEM; the
        // previous piece's scores, its last readers, are complete (every tile's partials
        // are in, so every score MMA is done)
        auto q_row = [&](int bq) {
            return reinterpret_cast<const uint4 *>(p.qa + ((int64_t)bq * p.rows_total + grow) * kRow +
                                                   256 * rank + kXCols * xpart);
        };
        auto copy_q = [&](int bq) {
            const uint4 *src = q_row(bq);
            const bool live = row < rows_here;
            uint4 v[kXCols / 8];  // the whole 256-byte share in one round trip
#pragma unroll
            for (int j = 0; j < kXCols / 8; ++j) v[j] = live ? src[j] : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int h = 0; h < kXCols / 32; ++h) {
                uint32_t wv[16];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    wv[4 * j] = v[4 * h + j].x; wv[4 * j + 1] = v[4 * h + j].y;
                    wv[4 * j + 2] = v[4 * h + j].z; wv[4 * j + 3] = v[4 * h + j].w;
                }
                tmem_st16(t_q + lane_off + (kXCols / 2) * xpart + 16 * h, wv);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(q_full);
        };
        bool q_loaded = false;  // q~ of the coming piece already in TMEM
        PieceIter it = it0;
        int b, L, pb, pe;
        bool too_long;
        uint32_t t = 0;
        bool quit = false;
        while (!quit && next_piece(p, it, b, L, pb, pe, too_long)) {
            if (too_long) continue;
            if (!q_loaded) copy_q(b);
            q_loaded = false;
            // the next piece's q~ share heads for L2 now; its copy into TMEM at the end of this
            // piece then waits for L2, not for HBM
            PieceIter nx = it;
            int b2, L2, pb2, pe2;
            bool tl2 = false, more;
            do {
                more = next_piece(p, nx, b2, L2, pb2, pe2, tl2);
            } while (more && tl2);
            if (more && row < rows_here) {
                const uint4 *nq = q_row(b2);
                prefetch_l2(nq);
                prefetch_l2(nq + 8);
            }
            float m_run = -INFINITY, l_run = 0.0f;  // the owned row (4 lanes' tokens)
            const int32_t *prow = p.page_table + (int64_t)b * p.max_pages;
            const int last_visible = L - p.s_q + s_of_brow;  // this row's query sees t <= this
            const int nt = pe - pb;
            int page = prow[pb];
            for (int i = 0; i < nt; ++i, ++t) {
                const int page_next = i + 1 < nt ? prow[pb + i + 1] : 0;  // in flight meanwhile
                const uint32_t tt = t;
                const int sb = tt & 1;
                const int tok0 = (pb + i) * kPage;
                const bool bad = page < 0 || page >= p.num_pages;
                const int n_valid = bad ? 0 : max(0, min(kT, L - tok0));
                GQLA_SPAN_BEGIN(t_b0);
                if (!__all_sync(0xffffffffu, GQLA_WAITC(8, x_full, tt & 1, abort_flag))) {
                    if (lane == 0) give_up();
                    quit = true;
                    break;
                }
                GQLA_SPAN_BEGIN(t_b);
                // this row's tokens 16 bq4 .. 16 bq4 + 15 from both partials (fp32), added in fp32
                float x[16];
                {
                    const uint8_t *xl = smem + SM::oXL;
                    const uint8_t *xr = smem + SM::oXR;
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const int off = xoff(ob, 4 * bq4 + h);
                        const float4 a = *reinterpret_cast<const float4 *>(xl + off);
                        const float4 r = *reinterpret_cast<const float4 *>(xr + off);
                        x[4 * h] = a.x + r.x;
                        x[4 * h + 1] = a.y + r.y;
                        x[4 * h + 2] = a.z + r.z;
                        x[4 * h + 3] = a.w + r.w;
                    }
                }
                __syncwarp();
                // both CTAs' buffers may be refilled once every softmax warp of the pair has
                // read them
                if (lane == 0) {
                    mbar_arrive(x_empty_l);
                    mbar_arrive_remote_relaxed(xempty_remote);
                }
                // mask tokens past the sequence or past this query's causal limit
                const int lim = min(last_visible, tok0 + n_valid - 1) - (tok0 + 16 * bq4);
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    if (e > lim) x[e] = -INFINITY;
                float mx = x[0];
#pragma unroll
                for (int e = 1; e < 16; ++e) mx = fmaxf(mx, x[e]);
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                const float mt = mx * p.scale_log2;  // log2 units
                const bool first = i == 0;
                float m_new = m_run;
                if (first || mt > m_run + kRescaleLog2) m_new = mt;
                const float alpha = (!first && m_new != m_run) ? fast_exp2(m_run - m_new) : 1.0f;
                l_run = first ? 0.0f : l_run * alpha;
                m_run = m_new;
                // P = 2^(x scale - m) (fp32 ex2) in bf16 -- the top half of the fp32 value,
                // rounded towards zero; the row sum adds the same truncated values
                const float mu = m_run == -INFINITY ? 0.0f : m_run;
                uint32_t pw[8];
                float lsum = 0.0f;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint32_t p0 = __float_as_uint(fast_exp2(fmaf(x[2 * e], p.scale_log2, -mu)));
                    const uint32_t p1 = __float_as_uint(fast_exp2(fmaf(x[2 * e + 1], p.scale_log2, -mu)));
                    pw[e] = __byte_perm(p0, p1, 0x7632);
                    lsum += __uint_as_float(p0 & 0xFFFF0000u) + __uint_as_float(p1 & 0xFFFF0000u);
                }
                l_run += lsum;
                GQLA_SPAN_END(14, t_b);
                // P buffer sb of both CTAs is free once both PV(tt - 2) are done
                if (!__all_sync(0xffffffffu, GQLA_WAIT(9, &p_empty[sb], ((tt >> 1) & 1) ^ 1, abort_flag))) {
                    if (lane == 0) give_up();
                    quit = true;
                    break;
                }
                GQLA_SPAN_BEGIN(t_b2);
                uint8_t *prow_s = smem + SM::oP + sb * SM::kP + brow * 128;
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    *reinterpret_cast<uint4 *>(prow_s + (((2 * bq4 + h) ^ (brow & 7)) << 4)) =
                        make_uint4(pw[4 * h], pw[4 * h + 1], pw[4 * h + 2], pw[4 * h + 3]);
                if (bq4 == 0) alph[sb * kRows + brow] = alpha;
                fence_proxy_async_smem();  // P and the factors -> the PV MMAs and the bulk copies
                __syncwarp();
                if (lane == 0) {
                    // this warp's 8 rows of P are 1 KB of contiguous rows and their factors 32
                    // contiguous bytes: the same places in the peer's buffers
                    const uint32_t r0 = sb * SM::kP + brow * 128;
                    bulk_copy_to_peer(p_remote + r0, smem + SM::oP + r0, 8 * 128, pfull_remote + sb * 8);
                    const uint32_t a0 = (sb * kRows + brow) * 4;
                    bulk_copy_to_peer(alpha_remote + a0, smem + SM::oAlpha + a0, 8 * 4, pfull_remote + sb * 8);
                    mbar_arrive(&p_full[sb]);
                }
                GQLA_SPAN_END(17, t_b2);
                GQLA_SPAN_END(19, t_b0);
                page = page_next;
            }
            if (quit) break;
            // ---- the owned rows' sums and LSE; the sums of all 128 rows are gathered in
            // both CTAs' lsm for the score warps' epilogue.  They overwrite the previous
            // piece's sums: once PV of a tile of this piece is done in both CTAs, both CTAs'
            // score warps have sent that tile's partials, which they do only after the
            // previous piece's epilogue (which read the sums and waited for l_full's previous
            // phase), so the overwrite and the next arrivals on l_full are safe even for a
            // piece of a tile or two.  The tile is the piece's second-to-last
            // (its only one if it has one): no later tile on its P buffer has reached stage B,
            // so that buffer's barrier is at most one phase past it.
            const uint32_t t_pv = nt >= 2 ? t - 2 : t - 1;  // t is one past the piece's last tile
            if (!__all_sync(0xffffffffu, mbar_wait(&p_empty[t_pv & 1], (t_pv >> 1) & 1, abort_flag))) {
                if (lane == 0) give_up();
                break;
            }
            float l = l_run;
            l += __shfl_xor_sync(0xffffffffu, l, 1);
            l += __shfl_xor_sync(0xffffffffu, l, 2);
            if (yw == 0 && lane == 0) mbar_arrive_expect_tx(l_full, kOwn * 4);
            if (bq4 == 0) {
                lsm[brow] = l;
                st_async_b32(l_remote + brow * 4, __float_as_uint(l), lfull_remote);
                if (blive)
                    p.lse_part[(int64_t)(b + c) * p.rows_total + bgrow] =
                        (l > 0.0f && m_run != -INFINITY) ? (m_run + __log2f(l)) * 0.6931471805599453f : -INFINITY;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(l_full);
            // the next piece's q~ into TMEM, while the score warps write this piece's O
            if (more) {
                copy_q(b2);
                q_loaded = true;
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
    // Every step of the pair ran in both CTAs: if neither gave up, every byte either one
    // sent (partial scores, P rows, rescale factors, row sums) was waited for by the
    // other, so nothing is in flight here.  When one gave up (both flags are set then),
    // the copies sent before the roles stopped may still be in flight: after the first
    // barrier both CTAs wait about 100 us (those copies take microseconds) before the
    // second barrier lets either exit.
    cluster_sync();
    if (*abort_flag) {
        const long long t0 = clock64();
        while (clock64() - t0 < 200000) __nanosleep(1000);
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
                                 const gqla_kv_index *idx, int num_splits, int lead, int lead_w16, float scale,
                                 float *o_part, float *lse_part, void *ws, cudaStream_t stream) {
    CUtensorMap lat, rope, qrope, omap;
    const uint64_t slots = (uint64_t)idx->num_pages * kPage;
    const uint64_t qrows = (uint64_t)idx->batch * s_q * heads;
    if (!make_row_map(&lat, cache, slots, 64, kT, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_row_map(&rope, cache, slots, 32, kT, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_row_map(&qrope, qa, qrows, 32, kRows, CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    {
        // partials fp32 [B + C][s_q][h][512], stored in 32 x 32 boxes (128-byte rows)
        const uint64_t orows = (uint64_t)(idx->batch + num_splits) * s_q * heads;
        const uint64_t dims[2] = {(uint64_t)kLatent, orows};
        const uint64_t strides[1] = {(uint64_t)kLatent * 4};
        const uint32_t box[2] = {32, 32};
        if (!make_map(&omap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, o_part, 2, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B))
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
    p.lead = lead;
    p.lead_w16 = lead_w16;
    p.s_q = s_q;
    p.heads = heads;
    p.rows_total = s_q * heads;
    p.row_blocks = (p.rows_total + kRows - 1) / kRows;
    p.scale_log2 = scale * kLog2e;
    p.drop_tile = g_drop_v_unit;
    g_drop_v_unit = -1;
    cudaError_t e = cudaFuncSetAttribute(decode_absorb_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, AbsorbSmem::kAlloc);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)num_splits * p.row_blocks * 2;
    return launch_dependent(decode_absorb_tc_kernel, dim3(grid), dim3(kThreads), AbsorbSmem::kAlloc,
                            stream, lat, rope, qrope, omap, p);
}

}  // namespace gqla
