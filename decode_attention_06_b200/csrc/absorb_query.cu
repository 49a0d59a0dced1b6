// absorb_query.cu -- query absorption for the MQA-absorb path on the tcgen05
// tensor cores: W_UK folded into the query (GQLA, paperlayer.ai summary, sec. 2;
// pwwt.cn article, sec. 3).
//
//   qa[r][0:512]   = W_UK_{g(r)} q_r^C      (q^C = the first 128 query dims)
//   qa[r][512:576] = q_r^R                  (RoPE part, copied)
//
// Rows of one group share W_UK_g, so a CTA owns a tile of up to 128 rows of
// one group -- `bst` consecutive (sequence, query token) pairs x the group's
// G heads -- and N = 128 or 256 columns of the latent output:
//   D[128 x N] = A[128 x 128] * B[128 x N],  A = q^C rows (K-major),
//   B^T = W_UK_g[columns] as stored ([latent][d_nope], K-major).
// Both operands arrive by TMA in the 128-byte swizzled layout; one thread
// issues 8 MMAs of K = 16 into an N-column TMEM accumulator; the four warps
// convert their 32 rows to bf16 into shared memory and write the tile out
// row by row, each row one contiguous segment.  N = 128 (3 CTAs per SM) splits
// a tile over four CTAs, for small batches; when that grid needs more than one
// wave, N = 256 (2 CTAs per SM) fits the work in one.
#include <cuda.h>

#include "common.cuh"
#include "sm100.cuh"
#include "tensor_map.cuh"

namespace gqla {

namespace {

using namespace sm100;

constexpr int kAqThreads = 128;
constexpr int kAqA = 128 * 128;        // one K block of A: 128 rows x 64 dims (bytes)

template <int N>  // latent columns per CTA
struct AqLayout {
    static constexpr int kB = N * 128;        // one K block of B: N latent rows x 64 dims
    static constexpr int kBar = 2 * kAqA + 2 * kB;
    static constexpr int kStage = 2 * N + 16;  // staging row pitch (bytes): N bf16 + bank skew
    static_assert(128 * kStage <= kBar, "staging tile overlaps the barriers");
    static constexpr int kSmem = kBar + 64 + 1024;  // + alignment slack
};

struct AqParams {
    const __nv_bfloat16 *q;
    __nv_bfloat16 *qa;
    int bs_total;  // batch * s_q
    int heads;
    int G;         // heads per group
    int bst;       // (sequence, token) pairs per tile: G * bst <= 128
};

template <int N>
__global__ void __launch_bounds__(kAqThreads, 2)
    absorb_query_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                           const __grid_constant__ CUtensorMap wmap, AqParams p) {
    constexpr int kAqN = N;
    constexpr int kAqB = AqLayout<N>::kB;
    constexpr int kAqBar = AqLayout<N>::kBar;
    constexpr int kAqStage = AqLayout<N>::kStage;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + 2 * kAqA;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kAqBar);
    uint64_t *done = full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(full + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(full + 3);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tile = blockIdx.x, grp = blockIdx.y, quarter = blockIdx.z;  // column block N * quarter
    const int bs0 = tile * p.bst;
    const int rows_in_tile = p.G * p.bst;

    if (threadIdx.x == 0) {
        prefetch_tensormap(&qmap);
        prefetch_tensormap(&wmap);
        mbar_init(full, 1);
        mbar_init(done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kAqN);
        tmem_relinquish();
    }
    griddep_wait();  // the previous kernel's results are visible from here on
    griddep_launch_dependents();
    if (threadIdx.x == 0) {
        const uint32_t a_bytes = (uint32_t)rows_in_tile * 128;
        mbar_arrive_expect_tx(full, 2 * a_bytes + 2 * kAqB);
        for (int kb = 0; kb < 2; ++kb) {
            tma_load_3d(sA + kb * kAqA, &qmap, full, kb * 64, grp * p.G, bs0);
            tma_load_2d(sB + kb * kAqB, &wmap, full, kb * 64, grp * kLatent + quarter * kAqN);
        }
    }
    // RoPE part of the query (quarter 0 only): loaded now, while the tiles are in
    // flight, and stored with the epilogue; 8 lanes per row, rows_in_tile * 8 <= 8 * kAqThreads
    constexpr int kRopeIt = 128 * 8 / kAqThreads;
    uint4 rope[kRopeIt];
    if (quarter == 0) {
#pragma unroll
        for (int j = 0; j < kRopeIt; ++j) {
            const int i = threadIdx.x + j * kAqThreads, r = i >> 3, part = i & 7;
            const int bs = bs0 + r / p.G;
            rope[j] = make_uint4(0, 0, 0, 0);
            if (r < rows_in_tile && bs < p.bs_total) {
                const int64_t row = (int64_t)bs * p.heads + grp * p.G + r % p.G;
                rope[j] = reinterpret_cast<const uint4 *>(p.q + row * kQk + kNope)[part];
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (threadIdx.x == 0) {
        if (mbar_wait(full, 0, abort_flag)) {
            tc_fence_after();
            constexpr uint32_t idesc = idesc_bf16(128, kAqN, 0, 0);
            const uint64_t a_d = smem_desc(smem_u32(sA), 16, 1024, kSw128);
            const uint64_t b_d = smem_desc(smem_u32(sB), 16, 1024, kSw128);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t off = (kk & 3) * 32;  // 16 dims = 32 bytes inside the swizzled row
                mma_bf16(tmem, desc_advance(a_d, (kk >> 2) * kAqA + off), desc_advance(b_d, (kk >> 2) * kAqB + off),
                         idesc, kk > 0 ? 1u : 0u);
            }
            mma_commit(done);
        } else {
            *abort_flag = 1;
        }
    }

    // Epilogue: each thread converts its row (TMEM lane) to bf16 into a
    // staging tile over A and B (the MMAs have completed), then
    // whole warps write rows out as contiguous 512-byte segments.
    const bool ok = mbar_wait(done, 0, abort_flag);
    tc_fence_after();
    uint8_t *stage = smem;  // [128 rows][kAqStage bytes]
    if (ok) {
        const int r = warp * 32 + lane;
#pragma unroll 1
        for (int c = 0; c < kAqN; c += 32) {
            uint32_t v[32];
            tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + c, v);
            tmem_wait_ld();
            uint4 st[4];
            uint32_t *w = reinterpret_cast<uint32_t *>(st);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                __nv_bfloat162 t = __floats2bfloat162_rn(__uint_as_float(v[2 * i]),
                                                         __uint_as_float(v[2 * i + 1]));
                w[i] = *reinterpret_cast<uint32_t *>(&t);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
                reinterpret_cast<uint4 *>(stage + r * kAqStage + c * 2)[i] = st[i];
        }
    }
    __syncthreads();
    if (ok) {
        // rows_in_tile rows of 2N bytes, 16 bytes a lane: a warp writes 32 / (N / 8) rows
        // at a time
        constexpr int kLanesPerRow = kAqN / 8, kRowsPerWarp = 32 / kLanesPerRow;
        for (int r0 = kRowsPerWarp * warp; r0 < rows_in_tile; r0 += 4 * kRowsPerWarp) {
            const int r = r0 + lane / kLanesPerRow, part = lane % kLanesPerRow;
            const int bs = bs0 + r / p.G;
            if (r < rows_in_tile && bs < p.bs_total) {
                const int64_t row = (int64_t)bs * p.heads + grp * p.G + r % p.G;
                reinterpret_cast<uint4 *>(p.qa + row * kRow + quarter * kAqN)[part] =
                    *reinterpret_cast<const uint4 *>(stage + r * kAqStage + part * 16);
            }
        }
        if (quarter == 0) {  // RoPE part: q[row][128:192] -> qa[row][512:576]
#pragma unroll
            for (int j = 0; j < kRopeIt; ++j) {
                const int i = threadIdx.x + j * kAqThreads, r = i >> 3, part = i & 7;
                const int bs = bs0 + r / p.G;
                if (r < rows_in_tile && bs < p.bs_total) {
                    const int64_t row = (int64_t)bs * p.heads + grp * p.G + r % p.G;
                    reinterpret_cast<uint4 *>(p.qa + row * kRow + kLatent)[part] = rope[j];
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kAqN);
    }
}

}  // namespace

cudaError_t launch_absorb_query(const void *q, int rows, int heads, int num_groups,
                                const void *w_uk, void *qa, cudaStream_t stream) {
    const int G = heads / num_groups;
    const int bs_total = rows / heads;
    if (bs_total == 0) return cudaSuccess;
    const int bst = 128 / G;
    CUtensorMap qmap, wmap;
    {
        const uint64_t dims[3] = {(uint64_t)kQk, (uint64_t)heads, (uint64_t)bs_total};
        const uint64_t strides[2] = {(uint64_t)kQk * 2, (uint64_t)heads * kQk * 2};
        const uint32_t box[3] = {64, (uint32_t)G, (uint32_t)bst};
        if (!make_bf16_map(&qmap, q, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    // N = 128 columns per CTA (a tile over four CTAs, 3 CTAs per SM) unless that grid
    // needs more than one wave; then N = 256 (2 CTAs per SM), which fits in one
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return cudaErrorInvalidValue;
    const int tiles = (bs_total + bst - 1) / bst;
    const bool wide = (int64_t)tiles * num_groups * (kLatent / 128) > 3LL * sms;
    const uint32_t n = wide ? 256 : 128;
    {
        const uint64_t dims[2] = {(uint64_t)kNope, (uint64_t)num_groups * kLatent};
        const uint64_t strides[1] = {(uint64_t)kNope * 2};
        const uint32_t box[2] = {64, n};
        if (!make_bf16_map(&wmap, w_uk, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    AqParams p{static_cast<const __nv_bfloat16 *>(q), static_cast<__nv_bfloat16 *>(qa), bs_total,
               heads, G, bst};
    dim3 grid((unsigned)tiles, (unsigned)num_groups, kLatent / n);
    if (wide) {
        cudaError_t e = cudaFuncSetAttribute(absorb_query_tc_kernel<256>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, AqLayout<256>::kSmem);
        if (e != cudaSuccess) return e;
        return launch_dependent(absorb_query_tc_kernel<256>, grid, dim3(kAqThreads), AqLayout<256>::kSmem,
                                stream, qmap, wmap, p);
    }
    cudaError_t e = cudaFuncSetAttribute(absorb_query_tc_kernel<128>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, AqLayout<128>::kSmem);
    if (e != cudaSuccess) return e;
    return launch_dependent(absorb_query_tc_kernel<128>, grid, dim3(kAqThreads), AqLayout<128>::kSmem, stream,
                            qmap, wmap, p);
}

}  // namespace gqla
