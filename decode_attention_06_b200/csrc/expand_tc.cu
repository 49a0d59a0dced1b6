// expand_tc.cu -- the one-shot per-group cache expansion for the GQA path on
// the tcgen05 tensor cores (GQLA, paperlayer.ai summary, sec. 3 "Two
// equivalent decoding paths"; pwwt.cn article, sec. 3):
//
//   kv[g][n][0:128] = c_n W_UK_g,  kv[g][n][128:256] = c_n W_UV_g,  k_rope[n] = k^R_n.
//
// The same product as expand.cu, accumulated in fp32 by the tensor cores in
// their own order and rounded once to bf16: results agree with the
// sequential-order expansion to within one bf16 rounding, not bit for bit.
//
// One CTA per tile of 128 cache slots, every group:
//   D_g[128 x 256] = A[128 x 512] * B_g[512 x 256],  B_g = [W_UK_g | W_UV_g]
// A (the tile's latent rows, K-major, 128 KB) stays in shared memory for all
// groups; B_g streams through a 4-stage ring of 32-row slabs (MN-major, the
// weights as stored); two 256-column TMEM accumulators let the epilogue of
// group g run while the MMAs of group g + 1 do.  Warp 0 issues the TMA loads
// (and stores the tile's RoPE columns straight from shared memory to k_rope),
// warp 1 the MMAs, warps 2-5 convert and store the output rows.
#include <cuda.h>

#include "common.cuh"
#include "sm100.cuh"
#include "tensor_map.cuh"

namespace gqla {

namespace {

using namespace sm100;

constexpr int kXtRows = 128;                 // slots per tile (MMA M)
constexpr int kXtThreads = 192;
constexpr int kXtBoxA = kXtRows * 128;       // [128 slots][64 latent cols] bf16
constexpr int kXtA = 8 * kXtBoxA;            // the tile's 512 latent columns
constexpr int kXtSlabRows = 32;              // K rows of B per ring stage
constexpr int kXtBoxB = kXtSlabRows * 128;   // [32 K rows][64 output cols] bf16
constexpr int kXtStage = 4 * kXtBoxB;        // 256 output columns: W_UK_g | W_UV_g
constexpr int kXtStages = 4;
constexpr int kXtSlabs = kLatent / kXtSlabRows;  // 16 per group

struct XtSmem {
    static constexpr int oA = 0;
    static constexpr int oRope = oA + kXtA;                 // [128 slots][64] bf16, 128B-swizzled
    static constexpr int oB = oRope + kXtBoxA;
    static constexpr int oBar = oB + kXtStages * kXtStage;
    // a_full, b_full/b_empty[kXtStages], acc_full/acc_empty[2], drain
    static constexpr int kNumBars = 1 + 2 * kXtStages + 4 + 1;
    static constexpr int oMisc = oBar + kNumBars * 8;       // tmem base, abort
    static constexpr int kAlloc = oMisc + 16 + 1024;
};
static_assert(XtSmem::kAlloc <= 227 * 1024, "shared memory");

__global__ void __launch_bounds__(kXtThreads, 1)
    expand_tc_kernel(const __grid_constant__ CUtensorMap lat_map,
                     const __grid_constant__ CUtensorMap wuk_map,
                     const __grid_constant__ CUtensorMap wuv_map,
                     const __grid_constant__ CUtensorMap rope_out_map, __nv_bfloat16 *kv,
                     int64_t num_slots, int num_groups) {
    using SM = XtSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::oBar);
    uint64_t *a_full = bars, *b_full = bars + 1, *b_empty = b_full + kXtStages;
    uint64_t *acc_full = b_empty + kXtStages, *acc_empty = acc_full + 2, *drain = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + SM::oMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + SM::oMisc + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t slot0 = (int64_t)blockIdx.x * kXtRows;

    if (threadIdx.x == 0) {
        mbar_init(a_full, 1);
        for (int i = 0; i < kXtStages; ++i) { mbar_init(&b_full[i], 1); mbar_init(&b_empty[i], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&acc_full[i], 1); mbar_init(&acc_empty[i], 4); }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            prefetch_tensormap(&lat_map);
            prefetch_tensormap(&wuk_map);
            prefetch_tensormap(&wuv_map);
            mbar_arrive_expect_tx(a_full, 9 * kXtBoxA);
            for (int bx = 0; bx < 9; ++bx)  // 8 latent boxes, then the RoPE box
                tma_load_2d(smem + SM::oA + bx * kXtBoxA, &lat_map, a_full, 64 * bx, (int)slot0);
            int u = 0;
            for (int g = 0; g < num_groups; ++g)
                for (int kb = 0; kb < kXtSlabs; ++kb, ++u) {
                    const int st = u % kXtStages;
                    if (!mbar_wait(&b_empty[st], ((u / kXtStages) & 1) ^ 1, abort_flag)) *abort_flag = 1;
                    if (*abort_flag) break;
                    uint8_t *dst = smem + SM::oB + st * kXtStage;
                    mbar_arrive_expect_tx(&b_full[st], kXtStage);
                    const int wrow = g * kLatent + kb * kXtSlabRows;
                    tma_load_2d(dst, &wuk_map, &b_full[st], 0, wrow);
                    tma_load_2d(dst + kXtBoxB, &wuk_map, &b_full[st], 64, wrow);
                    tma_load_2d(dst + 2 * kXtBoxB, &wuv_map, &b_full[st], 0, wrow);
                    tma_load_2d(dst + 3 * kXtBoxB, &wuv_map, &b_full[st], 64, wrow);
                }
            // k_rope rows of this tile, straight from the RoPE box (rows past the end
            // of the cache are dropped by the map)
            if (mbar_wait(a_full, 0, abort_flag)) {
                tma_store_2d(&rope_out_map, smem + SM::oRope, 0, (int)slot0);
                bulk_commit_group();
                bulk_wait_group<0>();
            } else {
                *abort_flag = 1;
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(kXtRows, 256, 0, 1);
            // A: K-major, 128B-swizzled 64-column boxes; B: MN-major, 4 atoms of 64 columns
            const uint64_t a_d0 = smem_desc(smem_u32(smem + SM::oA), 16, 1024, kSw128);
            const uint64_t b_d0 = smem_desc(smem_u32(smem + SM::oB), kXtBoxB, 1024, kSw128);
            if (!mbar_wait(a_full, 0, abort_flag)) *abort_flag = 1;
            tc_fence_after();
            int u = 0;
            for (int g = 0; g < num_groups && !*abort_flag; ++g) {
                const int ab = g & 1;
                // the epilogue has drained this accumulator (group g - 2)
                if (!mbar_wait(&acc_empty[ab], ((g >> 1) & 1) ^ 1, abort_flag)) *abort_flag = 1;
                tc_fence_after();
                for (int kb = 0; kb < kXtSlabs; ++kb, ++u) {
                    const int st = u % kXtStages;
                    if (!mbar_wait(&b_full[st], (u / kXtStages) & 1, abort_flag)) *abort_flag = 1;
                    tc_fence_after();
                    if (!*abort_flag) {
#pragma unroll
                        for (int ks = 0; ks < kXtSlabRows / 16; ++ks) {
                            const int k = kb * kXtSlabRows + ks * 16;  // latent index of this step
                            mma_bf16(tmem + 256 * ab,
                                     desc_advance(a_d0, (k >> 6) * kXtBoxA + ((k & 63) >> 3) * 16),
                                     desc_advance(b_d0, st * kXtStage + ks * 16 * 128), idesc,
                                     (kb > 0 || ks > 0) ? 1u : 0u);
                        }
                    }
                    mma_commit(&b_empty[st]);
                }
                mma_commit(&acc_full[ab]);
            }
            mma_commit(drain);
            int dummy = 0;
            mbar_wait(drain, 0, reinterpret_cast<volatile int *>(&dummy));
        }
    } else {
        // ---------------------------------------------------------------- epilogue warps
        // a thread per slot (its TMEM lane): 256 fp32 -> bf16, one contiguous 512-byte
        // row of kv[g] per slot
        const int quad = warp & 3;
        const int r = 32 * quad + lane;
        const int64_t slot = slot0 + r;
        const uint32_t lane_off = static_cast<uint32_t>(32 * quad) << 16;
        for (int g = 0; g < num_groups; ++g) {
            const int ab = g & 1;
            if (!mbar_wait(&acc_full[ab], (g >> 1) & 1, abort_flag)) *abort_flag = 1;
            tc_fence_after();
            uint4 *dst = reinterpret_cast<uint4 *>(kv + ((int64_t)g * num_slots + slot) * kKv);
#pragma unroll 1
            for (int c = 0; c < kKv; c += 32) {
                uint32_t v[32];
                tmem_ld32(tmem + 256 * ab + lane_off + c, v);
                tmem_wait_ld();
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    __nv_bfloat162 t = __floats2bfloat162_rn(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                    w[i] = *reinterpret_cast<uint32_t *>(&t);
                }
                if (slot < num_slots && !*abort_flag) {
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[c / 8 + i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[ab]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace

cudaError_t launch_expand_tc(const void *latent, int64_t num_slots, const void *w_uk,
                             const void *w_uv, void *kv, void *k_rope, int num_groups,
                             cudaStream_t stream) {
    if (num_slots == 0) return cudaSuccess;
    CUtensorMap lat, wuk, wuv, rope_out;
    {
        const uint64_t dims[2] = {(uint64_t)kRow, (uint64_t)num_slots};
        const uint64_t strides[1] = {(uint64_t)kRow * 2};
        const uint32_t box[2] = {64, (uint32_t)kXtRows};
        if (!make_bf16_map(&lat, latent, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    {
        const uint64_t dims[2] = {(uint64_t)kNope, (uint64_t)num_groups * kLatent};
        const uint64_t strides[1] = {(uint64_t)kNope * 2};
        const uint32_t box[2] = {64, (uint32_t)kXtSlabRows};
        if (!make_bf16_map(&wuk, w_uk, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_bf16_map(&wuv, w_uv, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    {
        const uint64_t dims[2] = {(uint64_t)kRope, (uint64_t)num_slots};
        const uint64_t strides[1] = {(uint64_t)kRope * 2};
        const uint32_t box[2] = {64, (uint32_t)kXtRows};
        if (!make_bf16_map(&rope_out, k_rope, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    cudaError_t e = cudaFuncSetAttribute(expand_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         XtSmem::kAlloc);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((num_slots + kXtRows - 1) / kXtRows);
    expand_tc_kernel<<<grid, kXtThreads, XtSmem::kAlloc, stream>>>(
        lat, wuk, wuv, rope_out, static_cast<__nv_bfloat16 *>(kv), num_slots, num_groups);
    return cudaGetLastError();
}

}  // namespace gqla
