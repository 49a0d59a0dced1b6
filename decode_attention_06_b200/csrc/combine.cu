// combine.cu -- log-sum-exp merge of the split-KV partials, and for the
// MQA-absorb path the per-group up-projection out = o~ W_UV_g applied after
// the merge ("folds W_UV into O": GQLA, paperlayer.ai summary, sec. 2).
//
// Each partial o_i is normalised by its own softmax sum and carries
// lse_i = ln sum_t exp(s_t) over its tokens, so
//   out = sum_i exp(lse_i - M) o_i / sum_i exp(lse_i - M),  M = max_i lse_i,
//   lse = M + ln sum_i exp(lse_i - M).
// A row whose sequence saw no token (no partial, or every lse_i = -inf)
// gets out = 0 and lse = -inf.
//
// Both kernels are bound by the read of the fp32 partials; they keep many
// independent 16-byte loads in flight per thread.  The absorb path's
// 512 -> 128 product runs on the tcgen05 tensor cores: a cluster of eight
// CTAs splits the 512-long contraction, each merging an eighth of the latent
// columns of its 128 rows, and the eight fp32 partial products are summed
// through distributed shared memory.
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
    int s_q;
    int heads;
    int G;         // heads per group
    int bs_total;  // batch * s_q
};

// One full warp: chunk range [c0, c1) of the sequences of the (sequence,
// token) pairs bs_lo .. bs_lo + n - 1 (n <= 32; empty range past the end).
// Lane d looks at sequence b_first + d: the n pairs span at most 32
// sequences, so one warp-wide scan gives every pair its first page.
__device__ void plan_pairs(const CombineParams &p, int bs_lo, int n, int *c0, int *c1) {
    const int lane = threadIdx.x & 31;
    const int total = warp_total_pages(p.seqlens, p.batch);
    const int k = chunk_pages(total, p.num_splits);
    const int b_first = min(bs_lo / p.s_q, p.batch);
    const int start = warp_sequence_start(p.seqlens, b_first);
    const int bl = b_first + lane;
    const int np = bl < p.batch ? pages_of(p.seqlens[bl]) : 0;
    const int excl = warp_incl_scan(np) - np;
    const int bs = bs_lo + lane;
    const int d = min(max(bs / p.s_q - b_first, 0), 31);
    const int np_d = __shfl_sync(0xffffffffu, np, d);
    const int st = start + __shfl_sync(0xffffffffu, excl, d);
    if (lane < n) {
        const bool any = bs < p.bs_total && np_d > 0;
        c0[lane] = any ? st / k : 0;
        c1[lane] = any ? (st + np_d - 1) / k + 1 : 0;
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

__device__ __forceinline__ uint2 pack_bf16x4(float a, float b, float c, float d) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
    return make_uint2(*reinterpret_cast<uint32_t *>(&lo), *reinterpret_cast<uint32_t *>(&hi));
}

// ---------------------------------------------------------------------------
// GQA path (d_in = 128): one warp per quad of heads of one (sequence, token)
// pair, lane j owns columns 4j .. 4j+3; the partials are read eight at a
// time so that one warp keeps 32 independent 16-byte loads in flight.
// ---------------------------------------------------------------------------
constexpr int kQuadsPerBlock = 4;

__global__ void __launch_bounds__(32 * kQuadsPerBlock) combine_v_kernel(CombineParams p) {
    __shared__ int s_c0[kQuadsPerBlock + 1], s_c1[kQuadsPerBlock + 1];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int quads_per_pair = p.heads / 4;
    const int q_first = blockIdx.x * kQuadsPerBlock;
    const int bs_lo = q_first / quads_per_pair;
    const int n_pairs = (q_first + kQuadsPerBlock - 1) / quads_per_pair - bs_lo + 1;
    if (warp == 0) plan_pairs(p, bs_lo, n_pairs, s_c0, s_c1);
    __syncthreads();

    const int quad = q_first + warp;
    const int bs = quad / quads_per_pair;
    if (bs >= p.bs_total) return;
    const int h0 = (quad % quads_per_pair) * 4;
    const int b = bs / p.s_q, s = bs % p.s_q;
    const int c0 = s_c0[bs - bs_lo], nparts = s_c1[bs - bs_lo] - c0;
    // partial (b, c) row of head h: ((b + c) * s_q + s) * heads + h
    const int64_t row0 = ((int64_t)(b + c0) * p.s_q + s) * p.heads + h0;
    const int64_t part_stride = (int64_t)p.s_q * p.heads;

    float M[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) M[i] = -INFINITY;
    for (int c = lane; c < nparts; c += 32)
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
            const float l = c < nparts ? __ldg(p.lse_part + row0 + c * part_stride + i) : -INFINITY;
            w[i] = l == -INFINITY ? 0.0f : __expf(l - M[i]);
            den[i] += w[i];
        }
        const int n = min(32, nparts - cb);
        const float *base = p.o_part + (row0 + (int64_t)cb * part_stride) * kDv + lane * 4;
        for (int j0 = 0; j0 < n; j0 += 8) {
            float4 v[8][4];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    v[jj][i] = j0 + jj < n ? ldg4(base + ((int64_t)(j0 + jj) * part_stride + i) * kDv)
                                           : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int jj = 0; jj < 8; ++jj)
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
// MQA-absorb path (d_in = 512).  A cluster of 8 CTAs per tile of up to 128
// rows of one group (bst pairs x G heads, as in the query absorption); CTA kq
// of the cluster merges latent columns [64 kq, 64 kq + 64) of the tile's rows
// and multiplies them by rows [64 kq, 64 kq + 64) of W_UV_g:
//   Y_kq[128 x 128] = A_kq[128 x 64] * B_kq[64 x 128]   (tcgen05, fp32 in TMEM)
// then CTA kq sums Y_0..Y_7 for rows [16 kq, 16 kq + 16) over DSMEM.
// ---------------------------------------------------------------------------
constexpr int kClCtas = 8;
constexpr int kClCols = kLatent / kClCtas;  // 64 latent columns per CTA
constexpr int kClThreads = 256;
constexpr int kClMaxPairs = 32;  // bst <= 128 / 4
constexpr int kClChunk = 32;     // partials whose weights are staged at a time
constexpr int kYStride = 132;    // fp32 row pitch of the partial product (bank spread)

struct ClSmem {
    static constexpr int oA = 0;                       // [128 rows][64] bf16, SW128 K-major
    static constexpr int oB = 16384;                   // 2 N blocks x [64 k][64 n] bf16, SW128
    static constexpr int oW = 32768;                   // [32 partials][128 rows] fp32 weights
    static constexpr int oY = 0;                       // [128][132] fp32, after the MMA
    static constexpr int oRowM = 69632;                // [128] fp32 max lse
    static constexpr int oRowInv = oRowM + 512;        // [128] fp32 1 / denominator
    static constexpr int oPlan = oRowInv + 512;        // c0[32], c1[32], max partials
    static constexpr int oBar = oPlan + 2 * kClMaxPairs * 4 + 16;
    static constexpr int kBytes = oBar + 32;
    static constexpr int kAlloc = kBytes + 1024;
};
static_assert(ClSmem::oW + 128 * kClChunk * 4 <= ClSmem::oRowM, "weights overlap");
static_assert(ClSmem::oY + 128 * kYStride * 4 <= ClSmem::oRowM, "Y overlaps the row data");

__global__ void __cluster_dims__(kClCtas, 1, 1) __launch_bounds__(kClThreads, 2)
    combine_latent_tc_kernel(const __grid_constant__ CUtensorMap wmap, CombineParams p, int bst) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    float *sW = reinterpret_cast<float *>(smem + ClSmem::oW);
    float *sInv = reinterpret_cast<float *>(smem + ClSmem::oRowInv);
    int *s_c0 = reinterpret_cast<int *>(smem + ClSmem::oPlan);
    int *s_c1 = s_c0 + kClMaxPairs;
    int *s_maxp = s_c1 + kClMaxPairs;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + ClSmem::oBar);
    uint64_t *done = full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(full + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int kq = (int)cluster_rank();
    const int tile = blockIdx.y, grp = blockIdx.z;
    const int bs0 = tile * bst;
    const int rows_in_tile = p.G * bst;
    const int64_t part_stride = (int64_t)p.s_q * p.heads;

    if (tid == 0) {
        prefetch_tensormap(&wmap);
        mbar_init(full, 1);
        mbar_init(done, 1);
        *abort_flag = 0;
        fence_barrier_init();
        mbar_arrive_expect_tx(full, 2 * kClCols * 128);
        for (int nb = 0; nb < 2; ++nb)
            tma_load_2d(smem + ClSmem::oB + nb * kClCols * 128, &wmap, full, nb * 64,
                        grp * kLatent + kq * kClCols);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 128);
        tmem_relinquish();
    }
    if (warp == 2) {
        plan_pairs(p, bs0, bst, s_c0, s_c1);
        if (lane == 0) {
            int m = 0;
            for (int j = 0; j < bst; ++j) m = max(m, s_c1[j] - s_c0[j]);
            *s_maxp = m;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // ---- threads 0..127: one row each -- max LSE, then weights per chunk
    float den = 0.0f, Mr = -INFINITY;
    const float *lse_row = p.lse_part;
    int np_r = 0;
    bool live_r = false;
    if (tid < 128) {
        const int j = tid / p.G;
        live_r = tid < rows_in_tile && bs0 + j < p.bs_total;
        if (live_r) {
            const int bs = bs0 + j, b = bs / p.s_q, s = bs % p.s_q;
            np_r = s_c1[j] - s_c0[j];
            lse_row = p.lse_part + ((int64_t)(b + s_c0[j]) * p.s_q + s) * p.heads + grp * p.G +
                      tid % p.G;
        }
        for (int c = 0; c < np_r; c += 8) {
            float l[8];
#pragma unroll
            for (int k = 0; k < 8; ++k)
                l[k] = c + k < np_r ? __ldg(lse_row + (c + k) * part_stride) : -INFINITY;
#pragma unroll
            for (int k = 0; k < 8; ++k) Mr = fmaxf(Mr, l[k]);
        }
    }

    // ---- merge: warp w owns rows 16w .. 16w+15 as 8 row pairs; lanes 0-15
    // take the first row of a pair, 16-31 the second, 4 columns each.
    const int sub = lane >> 4, c4 = (lane & 15) * 4;
    float4 acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    const float *src[8];
    int npq[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int r = 16 * warp + 2 * i;  // even row: both rows of the pair share the pair (bs)
        const int j = r / p.G;
        const bool live = r < rows_in_tile && bs0 + j < p.bs_total;
        npq[i] = live ? s_c1[j] - s_c0[j] : 0;
        const int bs = bs0 + j, b = bs / p.s_q, s = bs % p.s_q;
        src[i] = p.o_part +
                 (((int64_t)(b + (live ? s_c0[j] : 0)) * p.s_q + s) * p.heads + grp * p.G + r % p.G + sub) *
                     kLatent +
                 kq * kClCols + c4;
    }
    const int maxp = *s_maxp;
    for (int cb = 0; cb < maxp; cb += kClChunk) {
        __syncthreads();  // the previous chunk's weights are consumed
        if (tid < 128) {
            float l[kClChunk];
#pragma unroll
            for (int k = 0; k < kClChunk; ++k)
                l[k] = cb + k < np_r ? __ldg(lse_row + (cb + k) * part_stride) : -INFINITY;
#pragma unroll
            for (int k = 0; k < kClChunk; ++k) {
                const float w = l[k] == -INFINITY ? 0.0f : __expf(l[k] - Mr);
                den += w;
                sW[k * 128 + tid] = w;  // [partial][row]: conflict-free
            }
        }
        __syncthreads();
        const int n = min(kClChunk, maxp - cb);
        for (int j0 = 0; j0 < n; j0 += 2) {
            float4 v[2][8];
#pragma unroll
            for (int jj = 0; jj < 2; ++jj)
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    v[jj][i] = cb + j0 + jj < npq[i]
                                   ? ldg4(src[i] + (int64_t)(cb + j0 + jj) * part_stride * kLatent)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int jj = 0; jj < 2; ++jj)
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float wj = j0 + jj < n ? sW[(j0 + jj) * 128 + 16 * warp + 2 * i + sub] : 0.0f;
                    acc[i].x = fmaf(wj, v[jj][i].x, acc[i].x);
                    acc[i].y = fmaf(wj, v[jj][i].y, acc[i].y);
                    acc[i].z = fmaf(wj, v[jj][i].z, acc[i].z);
                    acc[i].w = fmaf(wj, v[jj][i].w, acc[i].w);
                }
        }
    }
    if (tid < 128) {
        sInv[tid] = den > 0.0f ? 1.0f / den : 0.0f;
        if (kq == 0 && p.lse_out && live_r)
            p.lse_out[(int64_t)(bs0 + tid / p.G) * p.heads + grp * p.G + tid % p.G] =
                den > 0.0f ? Mr + __logf(den) : -INFINITY;
    }
    __syncthreads();

    // ---- merged rows -> A (bf16, K-major, 128-byte swizzle)
    {
        const int chunk = (lane & 15) >> 1, half8 = (lane & 1) * 8;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int r = 16 * warp + 2 * i + sub;
            const float inv = sInv[r];
            *reinterpret_cast<uint2 *>(smem + ClSmem::oA + r * 128 + ((chunk ^ (r & 7)) << 4) + half8) =
                pack_bf16x4(acc[i].x * inv, acc[i].y * inv, acc[i].z * inv, acc[i].w * inv);
        }
    }
    fence_proxy_async_smem();
    __syncthreads();

    if (tid == 0) {
        if (mbar_wait(full, 0, abort_flag)) {
            tc_fence_after();
            constexpr uint32_t idesc = idesc_bf16(128, 128, 0, 1);
            const uint32_t a0 = smem_u32(smem + ClSmem::oA), b0 = smem_u32(smem + ClSmem::oB);
#pragma unroll
            for (int kk = 0; kk < kClCols / 16; ++kk) {
                const uint64_t ad = smem_desc(a0 + kk * 32, 16, 1024, kSw128);
                const uint64_t bd = smem_desc(b0 + kk * 2048, kClCols * 128, 1024, kSw128);
                mma_bf16(tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
            }
            mma_commit(done);
        } else {
            *abort_flag = 1;
        }
    }
    const bool ok = mbar_wait(done, 0, abort_flag);
    tc_fence_after();

    // ---- partial product -> Y (fp32) in this CTA's shared memory
    if (ok) {
        const int r = 32 * (warp & 3) + lane;
        const int cbase = (warp >> 2) * 64;
        float *y = reinterpret_cast<float *>(smem + ClSmem::oY) + r * kYStride + cbase;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t v[32];
            tmem_ld32(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + cbase + 32 * h, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 8; ++i)
                reinterpret_cast<float4 *>(y + 32 * h)[i] =
                    make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
        }
    }
    tc_fence_before();
    cluster_sync();  // all partial products written

    // ---- rows [16 kq, 16 kq + 16): sum the partial products, store bf16
    {
        const int r = 16 * kq + (tid >> 4);
        const int col = (tid & 15) * 8;
        const int j = r / p.G;
        const bool live = r < rows_in_tile && bs0 + j < p.bs_total;
        const uint32_t local = smem_u32(smem + ClSmem::oY) + (uint32_t)(r * kYStride + col) * 4;
        float4 v[2 * kClCtas];  // all remote loads issued before the first use
#pragma unroll
        for (int src_rank = 0; src_rank < kClCtas; ++src_rank) {
            const uint32_t a = map_peer(local, (uint32_t)src_rank);
            v[2 * src_rank] = ld_cluster_f4(a);
            v[2 * src_rank + 1] = ld_cluster_f4(a + 16);
        }
        float sum[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) sum[i] = 0.0f;
#pragma unroll
        for (int src_rank = 0; src_rank < kClCtas; ++src_rank)
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                sum[4 * i] += v[2 * src_rank + i].x;
                sum[4 * i + 1] += v[2 * src_rank + i].y;
                sum[4 * i + 2] += v[2 * src_rank + i].z;
                sum[4 * i + 3] += v[2 * src_rank + i].w;
            }
        if (live && !*abort_flag) {
            const uint2 lo = pack_bf16x4(sum[0], sum[1], sum[2], sum[3]);
            const uint2 hi = pack_bf16x4(sum[4], sum[5], sum[6], sum[7]);
            *reinterpret_cast<uint4 *>(p.out + ((int64_t)(bs0 + j) * p.heads + grp * p.G + r % p.G) * kDv +
                                       col) = make_uint4(lo.x, lo.y, hi.x, hi.y);
        }
    }
    cluster_sync();  // no CTA leaves while a peer may still read its partial product
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

}  // namespace

cudaError_t launch_combine(const gqla_kv_index *kv, int s_q, int num_splits, int d_in,
                           const float *o_part, const float *lse_part, const void *w_uv,
                           void *out, float *lse_out, int heads, int num_groups,
                           cudaStream_t stream) {
    CombineParams p{o_part, lse_part, kv->seqlens, static_cast<__nv_bfloat16 *>(out), lse_out,
                    kv->batch, num_splits, s_q, heads, heads / num_groups, kv->batch * s_q};
    if (d_in == kDv) {
        const int64_t quads = (int64_t)p.bs_total * (heads / 4);
        combine_v_kernel<<<(unsigned)((quads + kQuadsPerBlock - 1) / kQuadsPerBlock),
                           32 * kQuadsPerBlock, 0, stream>>>(p);
        return cudaGetLastError();
    }
    const int bst = 128 / p.G;
    CUtensorMap wmap;
    const uint64_t dims[2] = {(uint64_t)kDv, (uint64_t)num_groups * kLatent};
    const uint64_t strides[1] = {(uint64_t)kDv * 2};
    const uint32_t box[2] = {64, (uint32_t)kClCols};
    if (!make_bf16_map(&wmap, w_uv, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(combine_latent_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, ClSmem::kAlloc);
    if (e != cudaSuccess) return e;
    dim3 grid(kClCtas, (unsigned)((p.bs_total + bst - 1) / bst), (unsigned)num_groups);
    combine_latent_tc_kernel<<<grid, kClThreads, ClSmem::kAlloc, stream>>>(wmap, p, bst);
    return cudaGetLastError();
}

}  // namespace gqla
