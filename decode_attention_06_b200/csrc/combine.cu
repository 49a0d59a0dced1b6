// combine.cu -- log-sum-exp merge of the split-KV partials, and for the
// MQA-absorb path the per-group up-projection out = o~ W_UV_g applied after
// the merge: W_UV folded into the output (GQLA, paperlayer.ai summary, sec. 2).
//
// Each partial o_i is normalised by its own softmax sum and carries
// lse_i = ln sum_t exp(s_t) over its tokens, so
//   out = sum_i exp(lse_i - M) o_i / sum_i exp(lse_i - M),  M = max_i lse_i,
//   lse = M + ln sum_i exp(lse_i - M).
// A row whose sequence saw no token (no partial, or every lse_i = -inf)
// gets out = 0 and lse = -inf.
//
// Both kernels spend most of their time on the read of the fp32 partials, on
// its latency more than on HBM bandwidth; they keep many independent 16-byte
// loads in flight per thread and compute the merge weights while the partials
// are on their way.  The absorb path's
// 512 -> 128 product runs on the tcgen05 tensor cores: in a pair of CTAs each
// merges half of the latent columns of a 64-row tile into bf16, the second CTA
// stores its half straight into the first CTA's shared memory, and that CTA
// runs the whole K = 512 product.
#include <cuda.h>

#include "common.cuh"
#include "sm100.cuh"
#include "tensor_map.cuh"

namespace gqla {

namespace {

using namespace sm100;

struct CombineParams {
    const float *o_part;
    const float *lse_part;
    const int32_t *seqlens;
    __nv_bfloat16 *out;
    float *lse_out;
    int batch;
    int num_splits;
    int lead, lead_w16;  // the decode's split plan: lead chunks and their length (x 1/16)
    int s_q;
    int heads;
    int G;         // heads per group
    int bs_total;  // batch * s_q
    // leave alone the sequences with exactly one partial: the decode wrote their final
    // output itself
    int skip_single;
};

// One full warp: chunk range [c0, c1) of the sequences of the (sequence,
// token) pairs bs_lo .. bs_lo + n - 1 (n <= 32; empty range past the end).
// Lane d looks at sequence b_first + d: the n pairs span at most 32
// sequences, so one warp-wide scan gives every pair its first page.
__device__ void plan_pairs(const CombineParams &p, int bs_lo, int n, int *c0, int *c1) {
    const int lane = threadIdx.x & 31;
    const int b_first = min(bs_lo / p.s_q, p.batch);
    const int bl = b_first + lane;
    const int np = bl < p.batch ? pages_of(p.seqlens[bl]) : 0;
    // one pass over the lengths: the batch's pages and the pages before b_first
    int total = 0, start = 0;
    for (int b = lane; b < p.batch; b += 32) {
        const int nb = pages_of(p.seqlens[b]);
        total += nb;
        start += b < b_first ? nb : 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        total += __shfl_xor_sync(0xffffffffu, total, o);
        start += __shfl_xor_sync(0xffffffffu, start, o);
    }
    const SplitPlan sp{p.num_splits, p.lead, p.lead_w16};
    const int excl = warp_incl_scan(np) - np;
    const int bs = bs_lo + lane;
    const int d = min(max(bs / p.s_q - b_first, 0), 31);
    const int np_d = __shfl_sync(0xffffffffu, np, d);
    const int st = start + __shfl_sync(0xffffffffu, excl, d);
    if (lane < n) {
        const bool any = bs < p.bs_total && np_d > 0;
        c0[lane] = any ? plan_chunk_of(total, sp, st) : 0;
        c1[lane] = any ? plan_chunk_of(total, sp, st + np_d - 1) + 1 : 0;
    }
}

__device__ __forceinline__ float4 ldg4(const float *p) {
    return __ldg(reinterpret_cast<const float4 *>(p));
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// ---------------------------------------------------------------------------
// GQA path (d_in = 128): one warp per quad of heads of one (sequence, token)
// pair, lane j owns columns 4j .. 4j+3; the first four partials are read with
// the LSEs (16 independent 16-byte loads in flight per lane), the rest four at a
// time.  Four rather than eight keeps the register count low enough for three
// blocks per SM: the common case (a sequence over one to four chunks) is one
// round trip either way.
// ---------------------------------------------------------------------------
constexpr int kQuadsPerBlock = 4;

__global__ void __launch_bounds__(32 * kQuadsPerBlock, 3) combine_v_kernel(CombineParams p) {
    __shared__ int s_c0[kQuadsPerBlock + 1], s_c1[kQuadsPerBlock + 1];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int quads_per_pair = p.heads / 4;
    const int q_first = blockIdx.x * kQuadsPerBlock;
    const int bs_lo = q_first / quads_per_pair;
    const int n_pairs = (q_first + kQuadsPerBlock - 1) / quads_per_pair - bs_lo + 1;
    // The split plan reads only the lengths, which the decode before this kernel read
    // itself after its own wait for its predecessor: it runs while the decode finishes.
    if (warp == 0) plan_pairs(p, bs_lo, n_pairs, s_c0, s_c1);
    griddep_wait();  // the decode's partials are visible from here on
    griddep_launch_dependents();
    __syncthreads();

    const int quad = q_first + warp;
    const int bs = quad / quads_per_pair;
    if (bs >= p.bs_total) return;
    const int h0 = (quad % quads_per_pair) * 4;
    const int b = bs / p.s_q, s = bs % p.s_q;
    const int c0 = s_c0[bs - bs_lo], nparts = s_c1[bs - bs_lo] - c0;
    if (p.skip_single && nparts == 1) return;
    // partial (b, c) row of head h: ((b + c) * s_q + s) * heads + h
    const int64_t row0 = ((int64_t)(b + c0) * p.s_q + s) * p.heads + h0;
    const int64_t part_stride = (int64_t)p.s_q * p.heads;

    // the first partials do not depend on the weights: their loads go out with the LSE
    // loads, so the common case (nparts <= kPre) makes one round trip to memory
    constexpr int kPre = 2;
    const float *base0 = p.o_part + row0 * kDv + lane * 4;
    float4 v0[kPre][4];
#pragma unroll
    for (int jj = 0; jj < kPre; ++jj)
#pragma unroll
        for (int i = 0; i < 4; ++i)
            v0[jj][i] = jj < nparts ? ldg4(base0 + ((int64_t)jj * part_stride + i) * kDv)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
    // LSE of partial c = lane (the first 32), kept for the weights of the first block
    float l0[4], M[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        l0[i] = lane < nparts ? __ldg(p.lse_part + row0 + lane * part_stride + i) : -INFINITY;
        M[i] = l0[i];
    }
    for (int c = lane + 32; c < nparts; c += 32)
#pragma unroll
        for (int i = 0; i < 4; ++i) M[i] = fmaxf(M[i], __ldg(p.lse_part + row0 + c * part_stride + i));
#pragma unroll
    for (int i = 0; i < 4; ++i) M[i] = warp_max(M[i]);

    float4 acc[4];
    float den[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        den[i] = 0.0f;
    }
    for (int cb = 0; cb < nparts; cb += 32) {
        float w[4];
        const int c = cb + lane;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float l = cb == 0 ? l0[i] : c < nparts ? __ldg(p.lse_part + row0 + c * part_stride + i) : -INFINITY;
            w[i] = l == -INFINITY ? 0.0f : __expf(l - M[i]);
            den[i] += w[i];
        }
        const int n = min(32, nparts - cb);
        const float *base = p.o_part + (row0 + (int64_t)cb * part_stride) * kDv + lane * 4;
        int j0 = 0;
        if (cb == 0) {  // the partials already in registers (zeros past nparts)
#pragma unroll
            for (int jj = 0; jj < kPre; ++jj)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float wj = __shfl_sync(0xffffffffu, w[i], jj);
                    acc[i].x = fmaf(wj, v0[jj][i].x, acc[i].x);
                    acc[i].y = fmaf(wj, v0[jj][i].y, acc[i].y);
                    acc[i].z = fmaf(wj, v0[jj][i].z, acc[i].z);
                    acc[i].w = fmaf(wj, v0[jj][i].w, acc[i].w);
                }
            j0 = kPre;
        }
        for (; j0 < n; j0 += 4) {
            float4 v[4][4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    v[jj][i] = j0 + jj < n ? ldg4(base + ((int64_t)(j0 + jj) * part_stride + i) * kDv)
                                           : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int jj = 0; jj < 4; ++jj)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float wj = __shfl_sync(0xffffffffu, w[i], (j0 + jj) & 31);
                    acc[i].x = fmaf(wj, v[jj][i].x, acc[i].x);
                    acc[i].y = fmaf(wj, v[jj][i].y, acc[i].y);
                    acc[i].z = fmaf(wj, v[jj][i].z, acc[i].z);
                    acc[i].w = fmaf(wj, v[jj][i].w, acc[i].w);
                }
        }
    }
    const int64_t orow = (int64_t)bs * p.heads + h0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float d = warp_sum(den[i]);
        const float inv = d > 0.0f ? 1.0f / d : 0.0f;
        *reinterpret_cast<uint2 *>(p.out + (orow + i) * kDv + lane * 4) =
            pack_bf16x4(acc[i].x * inv, acc[i].y * inv, acc[i].z * inv, acc[i].w * inv);
        if (p.lse_out && lane == 0)
            p.lse_out[orow + i] = d > 0.0f ? M[i] + __logf(d) : -INFINITY;
    }
}

// ---------------------------------------------------------------------------
// MQA-absorb path (d_in = 512).  A cluster of 2 CTAs takes tiles of up to 64 rows
// of one group (bst pairs x G heads), one after the other (as many per cluster as
// keep the grid within one wave).  CTA kq merges latent columns
// [256 kq, 256 kq + 256) of the tile's rows into bf16 (the MMA's A operand,
// K-major, 128-byte swizzle); CTA 1 sends its half into CTA 0's shared memory as
// one bulk copy, and CTA 0 runs the whole product
//   out[64 x 128] = A[64 x 512] * W_UV_g[512 x 128]   (tcgen05 M = 64, fp32 in TMEM)
// and writes the bf16 rows.
// ---------------------------------------------------------------------------
constexpr int kClThreads = 512;
constexpr int kClRows = 64;      // rows of a tile (MMA M)
constexpr int kClMaxPairs = 32;  // bst <= 64 / 4 = 16

struct ClSmem {
    static constexpr int kAHalf = kClRows * 256 * 2;       // one CTA's 4 K blocks of A
    static constexpr int oA = 0;                           // 8 K blocks x [64 rows][64] bf16
    static constexpr int oB = 2 * kAHalf;                  // W_UV_g: 2 N blocks x [512 k][64 n] bf16
    static constexpr int oStage = 0;                       // epilogue [64 rows][128] bf16, over A
    static constexpr int oRowM = oB + 512 * 128 * 2;       // [64 rows] max LSE
    static constexpr int oRowInv = oRowM + kClRows * 4;    // [64 rows] 1 / sum of weights
    static constexpr int oPlan = oRowInv + kClRows * 4;    // c0[32], c1[32]
    static constexpr int oBar = oPlan + 2 * kClMaxPairs * 4 + 16;
    static constexpr int kBytes = oBar + 40;
    static constexpr int kAlloc = kBytes + 1024;
};
static_assert(ClSmem::kAlloc <= 227 * 1024, "shared memory");

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kClThreads, 1)
    combine_latent_tc_kernel(const __grid_constant__ CUtensorMap wmap, CombineParams p, int bst,
                             int tiles_per_cluster, int num_tiles) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    float *sM = reinterpret_cast<float *>(smem + ClSmem::oRowM);
    float *sInv = reinterpret_cast<float *>(smem + ClSmem::oRowInv);
    int *s_c0 = reinterpret_cast<int *>(smem + ClSmem::oPlan);
    int *s_c1 = s_c0 + kClMaxPairs;
    uint64_t *a_full = reinterpret_cast<uint64_t *>(smem + ClSmem::oBar);
    uint64_t *b_full = a_full + 1;
    uint64_t *done = a_full + 2;
    uint64_t *a_free = a_full + 3;  // second CTA: the leader is done with A (its half may go)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(a_full + 4);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int kq = (int)cluster_rank();
    const bool leader = kq == 0;
    const int grp = blockIdx.z;
    // this cluster's tiles of group grp: [tile0, tile0 + n_tiles), one after the other, so
    // that W_UV_g, the barriers and the tensor memory are set up once for all of them
    const int tile0 = blockIdx.y * tiles_per_cluster;
    const int n_tiles = max(0, min(tiles_per_cluster, num_tiles - tile0));
    const int rows_in_tile = p.G * bst;
    const int64_t part_stride = (int64_t)p.s_q * p.heads;

    if (tid == 0) {
        mbar_init(a_full, 1);
        mbar_init(b_full, 1);
        mbar_init(done, 1);
        mbar_init(a_free, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    // W_UV_g and the first tile's split plan (from the lengths) do not depend on the decode
    // before this kernel, which read the same lengths after its own wait: both start while
    // the decode finishes (the barrier init above is ordered before the TMA by fence and sync)
    __syncthreads();
    if (tid == 0) {
        if (leader) {
            prefetch_tensormap(&wmap);
            mbar_arrive_expect_tx(b_full, 512 * 128 * 2);
            for (int nb = 0; nb < 2; ++nb)
                for (int kh = 0; kh < 2; ++kh)
                    tma_load_2d(smem + ClSmem::oB + nb * 65536 + kh * 32768, &wmap, b_full, nb * 64,
                                grp * kLatent + kh * 256);
        }
    }
    if (warp == 1 && leader) {
        tmem_alloc(tmem_slot, 128);
        tmem_relinquish();
    }
    if (warp == 2 && n_tiles > 0) {
        plan_pairs(p, tile0 * bst, bst, s_c0, s_c1);
    }
    griddep_wait();  // the decode's partials are visible from here on
    griddep_launch_dependents();
    tc_fence_before();
    cluster_sync();  // barriers of both CTAs initialised before any remote transfer
    tc_fence_after();
    const uint32_t tmem = leader ? *tmem_slot : 0u;
    bool ok = true;

#pragma unroll 1
    for (int k = 0; k < n_tiles && ok; ++k) {
        const int bs0 = (tile0 + k) * bst;
        if (k > 0) {
            // every warp is done with the previous tile's plan (and, in the leader, with the
            // staging over A; in the second CTA, the previous half has left its A): the next
            // plan replaces it
            if (!leader && tid == 0) bulk_wait_group_read<0>();
            __syncthreads();
            if (warp == 2) plan_pairs(p, bs0, bst, s_c0, s_c1);
            __syncthreads();
        }

    // ---- merge: warp w owns rows 4w .. 4w+3, four heads of one (sequence, token) pair
    // (the heads per group are a multiple of 4), and computes their weights itself (lane c
    // holds partial c of a 32-partial block); lane j covers columns 4j and 128 + 4j of
    // this CTA's 256 latent columns; two partials are read per step, the first two
    // right behind the LSEs (they do not depend on the weights)
    constexpr int kRw = kClRows / (kClThreads / 32);  // rows per warp
    static_assert(kRw == 4, "a warp's rows are one pair's heads");
    float4 acc[kRw][2];
#pragma unroll
    for (int i = 0; i < kRw; ++i) acc[i][0] = acc[i][1] = make_float4(0.f, 0.f, 0.f, 0.f);
    const int r0 = kRw * warp, j = r0 / p.G;
    const bool live = r0 < rows_in_tile && bs0 + j < p.bs_total;
    const int np_max = live ? s_c1[j] - s_c0[j] : 0;  // partials of the warp's rows
    // partial row of row r0's first partial: < (batch + splits) * s_q * heads < 2^27
    const int row0 = [&] {
        const int bs = bs0 + j, b = bs / p.s_q, s = bs % p.s_q;
        return ((b + (live ? s_c0[j] : 0)) * p.s_q + s) * p.heads + grp * p.G + r0 % p.G;
    }();
    const float *src = p.o_part + (int64_t)row0 * kLatent + kq * 256 + lane * 4;
    const float *lse0 = p.lse_part + row0;
    float4 v[2][kRw][2];
    auto load2 = [&](int c) {
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int i = 0; i < kRw; ++i) {
                const bool on = c + u < np_max;
                const float *q = src + ((int64_t)(c + u) * part_stride + i) * kLatent;
                v[u][i][0] = on ? ldg4(q) : make_float4(0.f, 0.f, 0.f, 0.f);
                v[u][i][1] = on ? ldg4(q + 128) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
    };
    // per row: M = max lse_i, d = sum exp(lse_i - M); the weights below are already
    // divided by d, and rows with more than 32 partials find M and 1/d in shared memory
    float l0[kRw];
#pragma unroll
    for (int i = 0; i < kRw; ++i) l0[i] = lane < np_max ? __ldg(lse0 + lane * part_stride + i) : -INFINITY;
    load2(0);
    float w[kRw];  // weight of partial cb + lane of the current 32-partial block
    float m[kRw], d[kRw];
    if (np_max <= 32) {
        // one block: the four rows' reductions interleave
#pragma unroll
        for (int i = 0; i < kRw; ++i) m[i] = l0[i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int i = 0; i < kRw; ++i) m[i] = fmaxf(m[i], __shfl_xor_sync(0xffffffffu, m[i], o));
#pragma unroll
        for (int i = 0; i < kRw; ++i) d[i] = w[i] = l0[i] == -INFINITY ? 0.0f : __expf(l0[i] - m[i]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int i = 0; i < kRw; ++i) d[i] += __shfl_xor_sync(0xffffffffu, d[i], o);
    } else {
#pragma unroll
        for (int i = 0; i < kRw; ++i) {
            float mi = l0[i];
            for (int c = lane + 32; c < np_max; c += 32) mi = fmaxf(mi, __ldg(lse0 + c * part_stride + i));
            m[i] = warp_max(mi);
        }
#pragma unroll
        for (int i = 0; i < kRw; ++i) {
            w[i] = l0[i] == -INFINITY ? 0.0f : __expf(l0[i] - m[i]);
            float di = w[i];
            for (int c = lane + 32; c < np_max; c += 32) {
                const float l = __ldg(lse0 + c * part_stride + i);
                di += l == -INFINITY ? 0.0f : __expf(l - m[i]);
            }
            d[i] = warp_sum(di);
        }
    }
#pragma unroll
    for (int i = 0; i < kRw; ++i) {
        const float inv = d[i] > 0.0f ? 1.0f / d[i] : 0.0f;
        w[i] *= inv;
        if (lane == 0) {
            sM[r0 + i] = m[i];
            sInv[r0 + i] = inv;
            if (leader && p.lse_out && live)
                p.lse_out[(int64_t)(bs0 + j) * p.heads + grp * p.G + (r0 + i) % p.G] =
                    d[i] > 0.0f ? m[i] + __logf(d[i]) : -INFINITY;
        }
    }
    __syncwarp();
    for (int cb = 0; cb < np_max; cb += 32) {
        if (cb > 0) {
#pragma unroll
            for (int i = 0; i < kRw; ++i) {
                const int c = cb + lane;
                const float l = c < np_max ? __ldg(lse0 + c * part_stride + i) : -INFINITY;
                w[i] = l == -INFINITY ? 0.0f : __expf(l - sM[r0 + i]) * sInv[r0 + i];
            }
        }
        const int n = min(32, np_max - cb);
#pragma unroll 1
        for (int j0 = 0; j0 < n; j0 += 2) {
            if (cb + j0 > 0) load2(cb + j0);
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int i = 0; i < kRw; ++i) {
                    // zero past the row's partials: its LSE there is -inf
                    const float wj = __shfl_sync(0xffffffffu, w[i], (j0 + u) & 31);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        acc[i][h].x = fmaf(wj, v[u][i][h].x, acc[i][h].x);
                        acc[i][h].y = fmaf(wj, v[u][i][h].y, acc[i][h].y);
                        acc[i][h].z = fmaf(wj, v[u][i][h].z, acc[i][h].z);
                        acc[i][h].w = fmaf(wj, v[u][i][h].w, acc[i][h].w);
                    }
                }
        }
    }

    // ---- merged rows -> this CTA's four K blocks of A (bf16, K-major, 128-byte swizzle),
    // at the place they take in the leader's A: the leader stores its own in place; the
    // second CTA stores its half at the same place of its own (otherwise unused) A and
    // sends it into the leader's as one 32 KB bulk copy counted on the leader's a_full
    {
        const int chunk = (lane & 15) >> 1, half8 = (lane & 1) * 8;
#pragma unroll
        for (int i = 0; i < kRw; ++i) {
            const int r = kRw * warp + i;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int kb = kq * 4 + 2 * h + (lane >> 4);
                const uint32_t off = kb * (kClRows * 128) + r * 128 + ((chunk ^ (r & 7)) << 4) + half8;
                *reinterpret_cast<uint2 *>(smem + ClSmem::oA + off) =
                    pack_bf16x4(acc[i][h].x, acc[i][h].y, acc[i][h].z, acc[i][h].w);
            }
        }
    }
    if (!leader) {
        fence_proxy_async_smem();  // the half -> the bulk copy (async proxy)
        // the leader is done with the previous tile's A
        if (!__syncthreads_and(k == 0 || mbar_wait(a_free, (k - 1) & 1, abort_flag))) {
            ok = false;  // the leader stopped (or never freed A): send nothing more
            break;
        }
        if (tid == 0) {
            bulk_copy_to_peer(map_peer(smem_u32(smem + ClSmem::oA + ClSmem::kAHalf), 0),
                              smem + ClSmem::oA + ClSmem::kAHalf, ClSmem::kAHalf,
                              map_peer(smem_u32(a_full), 0));
            bulk_commit_group();
        }
        continue;  // the second CTA goes on with its next tile's merge
    }
    fence_proxy_async_smem();
    __syncthreads();

    // ---- leader: the other half of A and W_UV_g in place -> 32 MMAs (M = 64, K = 512)
    if (tid == 0) {
        // this CTA's half of K first (its A blocks are in place), the peer's half once it lands
        mbar_arrive_expect_tx(a_full, ClSmem::kAHalf);
        constexpr uint32_t idesc = idesc_bf16(kClRows, 128, 0, 1);
        const uint64_t a_d = smem_desc(smem_u32(smem + ClSmem::oA), 16, 1024, kSw128);
        const uint64_t b_d = smem_desc(smem_u32(smem + ClSmem::oB), 65536, 1024, kSw128);
        bool got = k > 0 || mbar_wait(b_full, 0, abort_flag);
        if (got) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < kLatent / 32; ++kk)
                mma_bf16(tmem, desc_advance(a_d, (kk >> 2) * (kClRows * 128) + (kk & 3) * 32),
                         desc_advance(b_d, kk * 2048), idesc, kk > 0 ? 1u : 0u);
            got = mbar_wait_cluster(a_full, k & 1, abort_flag);
        }
        if (got) {
            tc_fence_after();
#pragma unroll
            for (int kk = kLatent / 32; kk < kLatent / 16; ++kk)
                mma_bf16(tmem, desc_advance(a_d, (kk >> 2) * (kClRows * 128) + (kk & 3) * 32),
                         desc_advance(b_d, kk * 2048), idesc, 1u);
        } else {
            *abort_flag = 1;
        }
        mma_commit(done);
    }
    ok = __syncthreads_and(mbar_wait(done, k & 1, abort_flag) && !*abort_flag);
    tc_fence_after();
    // ---- epilogue: TMEM (M = 64: row m in lane (m % 16) + 32 (m / 16)) -> bf16 rows in
    // shared memory (over A: the MMAs are done) -> coalesced 256-byte row stores
    if (ok) {
        constexpr int kCw = 128 / (kClThreads / 128);  // columns per warp
        const int q = warp & 3, cbase = (warp >> 2) * kCw;
        const int r = 16 * q + lane;  // valid for lanes 0..15
#pragma unroll
        for (int h = 0; h < kCw / 32; ++h) {
            uint32_t v[32];
            tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + cbase + 32 * h, v);
            tmem_wait_ld();
            if (lane < 16) {
                uint8_t *dst = smem + ClSmem::oStage + r * 256 + (cbase + 32 * h) * 2;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const uint2 lo = pack_bf16x4(__uint_as_float(v[8 * e]), __uint_as_float(v[8 * e + 1]),
                                                 __uint_as_float(v[8 * e + 2]), __uint_as_float(v[8 * e + 3]));
                    const uint2 hi = pack_bf16x4(__uint_as_float(v[8 * e + 4]), __uint_as_float(v[8 * e + 5]),
                                                 __uint_as_float(v[8 * e + 6]), __uint_as_float(v[8 * e + 7]));
                    reinterpret_cast<uint4 *>(dst)[e] = make_uint4(lo.x, lo.y, hi.x, hi.y);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (ok) {
        for (int i = tid; i < kClRows * 16; i += kClThreads) {
            const int r = i >> 4, part16 = i & 15;
            const int jr = r / p.G;
            if (r >= rows_in_tile || bs0 + jr >= p.bs_total) continue;
            const int64_t orow = (int64_t)(bs0 + jr) * p.heads + grp * p.G + r % p.G;
            reinterpret_cast<uint4 *>(p.out + orow * kDv)[part16] =
                reinterpret_cast<const uint4 *>(smem + ClSmem::oStage + r * 256)[part16];
        }
    }
    if (ok && k + 1 < n_tiles) {
        // the staging over A has been read: the second CTA may send its next half
        __syncthreads();
        if (tid == 0) mbar_arrive_remote(map_peer(smem_u32(a_free), 1));
    }
    }  // tiles

    // One cluster barrier operation per thread on every path: the second CTA waits until
    // the leader has consumed the last half it sent (the leader arrives once its MMAs are
    // done, or once it stopped), then both may exit.
    if (!leader) {
        if (tid == 0) bulk_wait_group<0>();  // its last half has landed in the leader
        cluster_sync();
        return;
    }
    tc_fence_before();
    __syncthreads();
    cluster_arrive_relaxed();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

}  // namespace

cudaError_t launch_combine(const gqla_kv_index *kv, int s_q, int num_splits, int lead, int lead_w16,
                           int d_in, const float *o_part, const float *lse_part, const void *w_uv,
                           void *out, float *lse_out, int heads, int num_groups, bool skip_single,
                           cudaStream_t stream) {
    CombineParams p{o_part, lse_part, kv->seqlens, static_cast<__nv_bfloat16 *>(out), lse_out,
                    kv->batch, num_splits, lead, lead_w16, s_q, heads, heads / num_groups,
                    kv->batch * s_q, skip_single ? 1 : 0};
    if (d_in == kDv) {
        const int64_t quads = (int64_t)p.bs_total * (heads / 4);
        return launch_dependent(combine_v_kernel,
                                dim3((unsigned)((quads + kQuadsPerBlock - 1) / kQuadsPerBlock)),
                                dim3(32 * kQuadsPerBlock), 0, stream, p);
    }
    const int bst = kClRows / p.G;
    // tiles of one group per cluster: as few as fill one wave of the SMs (a cluster takes
    // two), so that W_UV_g and the set-up are paid once per cluster, not once per tile
    const int num_tiles = (p.bs_total + bst - 1) / bst;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return cudaErrorInvalidValue;
    const int clusters_per_group = (sms / 2) / num_groups > 0 ? (sms / 2) / num_groups : 1;
    const int tpc = (num_tiles + clusters_per_group - 1) / clusters_per_group;
    CUtensorMap wmap;
    const uint64_t dims[2] = {(uint64_t)kDv, (uint64_t)num_groups * kLatent};
    const uint64_t strides[1] = {(uint64_t)kDv * 2};
    const uint32_t box[2] = {64, 256};
    if (!make_bf16_map(&wmap, w_uv, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(combine_latent_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, ClSmem::kAlloc);
    if (e != cudaSuccess) return e;
    dim3 grid(2, (unsigned)((num_tiles + tpc - 1) / tpc), (unsigned)num_groups);
    return launch_dependent(combine_latent_tc_kernel, grid, dim3(kClThreads), ClSmem::kAlloc, stream,
                            wmap, p, bst, tpc, num_tiles);
}

}  // namespace gqla
