// expand.cu -- one-shot per-group cache expansion for the GQA path (GQLA,
// paperlayer.ai summary, sec. 3 "Two equivalent decoding paths"; pwwt.cn
// article, sec. 3).
//
// Expansion: kv[g][n][0:128] = c_n W_UK_g, kv[g][n][128:256] = c_n W_UV_g,
// k_rope[n] = k^R_n.  The rounding order is part of the contract (fp32, one
// fused multiply-add per latent index in ascending order from +0.0, one RNE
// to bf16), so this runs on the FP32 pipes as a register-blocked SIMT GEMM:
// every output keeps its own accumulator and walks k = 0..511 in order.
// Because a bf16 x bf16 product is exact in fp32, fma(a, b, acc) equals
// round(acc + a*b), whichever the compiler picks.
#include "common.cuh"

namespace gqla {

namespace {

constexpr int EXP_BM = 128;  // slots per block
constexpr int EXP_BN = 128;  // output columns per block (one K or V half of a group)
constexpr int EXP_BK = 16;

__device__ __forceinline__ void unpack8(uint4 v, float *f) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 t = __bfloat1622float2(h[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}

// grid: x = slot tiles, y = 2 * g (group, K/V half).  256 threads, 8x8 outputs each.
__global__ void __launch_bounds__(256) expand_kernel(const __nv_bfloat16 *__restrict__ latent,
                                                     int64_t num_slots,
                                                     const __nv_bfloat16 *__restrict__ w_uk,
                                                     const __nv_bfloat16 *__restrict__ w_uv,
                                                     __nv_bfloat16 *__restrict__ kv) {
    __shared__ __align__(16) float As[EXP_BK][EXP_BM + 4];  // [k][slot]
    __shared__ __align__(16) float Bs[EXP_BK][EXP_BN];      // [k][col]
    const int tid = threadIdx.x;
    const int tx = tid % 16, ty = tid / 16;
    const int64_t row0 = (int64_t)blockIdx.x * EXP_BM;
    const int grp = blockIdx.y >> 1, part = blockIdx.y & 1;
    const __nv_bfloat16 *W = (part ? w_uv : w_uk) + (size_t)grp * kLatent * kNope;

    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;

    // A loader: slot = tid / 2, k-offset (tid % 2) * 8.  B loader: k = tid / 16, col = (tid % 16) * 8.
    const int a_row = tid >> 1, a_k = (tid & 1) * 8;
    const int64_t a_slot = row0 + a_row;
    const int b_k = tid >> 4, b_c = (tid & 15) * 8;

    for (int k0 = 0; k0 < kLatent; k0 += EXP_BK) {
        float fa[8], fb[8];
        if (a_slot < num_slots) {
            uint4 v = *reinterpret_cast<const uint4 *>(latent + a_slot * kRow + k0 + a_k);
            unpack8(v, fa);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) fa[i] = 0.0f;
        }
        {
            uint4 v = *reinterpret_cast<const uint4 *>(W + (size_t)(k0 + b_k) * kNope + b_c);
            unpack8(v, fb);
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < 8; ++i) As[a_k + i][a_row] = fa[i];
        *reinterpret_cast<float4 *>(&Bs[b_k][b_c]) = make_float4(fb[0], fb[1], fb[2], fb[3]);
        *reinterpret_cast<float4 *>(&Bs[b_k][b_c + 4]) = make_float4(fb[4], fb[5], fb[6], fb[7]);
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < EXP_BK; ++kk) {
            float a[8], b[8];
            float4 t0 = *reinterpret_cast<const float4 *>(&As[kk][ty * 4]);
            float4 t1 = *reinterpret_cast<const float4 *>(&As[kk][64 + ty * 4]);
            float4 u0 = *reinterpret_cast<const float4 *>(&Bs[kk][tx * 4]);
            float4 u1 = *reinterpret_cast<const float4 *>(&Bs[kk][64 + tx * 4]);
            a[0] = t0.x; a[1] = t0.y; a[2] = t0.z; a[3] = t0.w;
            a[4] = t1.x; a[5] = t1.y; a[6] = t1.z; a[7] = t1.w;
            b[0] = u0.x; b[1] = u0.y; b[2] = u0.z; b[3] = u0.w;
            b[4] = u1.x; b[5] = u1.y; b[6] = u1.z; b[7] = u1.w;
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = __fmaf_rn(a[i], b[j], acc[i][j]);
        }
    }

    __nv_bfloat16 *dst = kv + (size_t)grp * num_slots * kKv + part * kNope;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        int64_t slot = row0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
        if (slot >= num_slots) continue;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            int col = h ? 64 + tx * 4 : tx * 4;
            __nv_bfloat162 p0 = __floats2bfloat162_rn(acc[i][4 * h + 0], acc[i][4 * h + 1]);
            __nv_bfloat162 p1 = __floats2bfloat162_rn(acc[i][4 * h + 2], acc[i][4 * h + 3]);
            uint2 st;
            st.x = *reinterpret_cast<uint32_t *>(&p0);
            st.y = *reinterpret_cast<uint32_t *>(&p1);
            *reinterpret_cast<uint2 *>(dst + slot * kKv + col) = st;
        }
    }
}

// k_rope[n][0:64] = latent[n][512:576], 16 bytes per thread.
__global__ void copy_rope_kernel(const __nv_bfloat16 *__restrict__ latent, int64_t num_slots,
                                 __nv_bfloat16 *__restrict__ k_rope) {
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // one uint4 (8 elems)
    int64_t slot = i / 8;
    int part = (int)(i % 8);
    if (slot >= num_slots) return;
    uint4 v = *reinterpret_cast<const uint4 *>(latent + slot * kRow + kLatent + part * 8);
    *reinterpret_cast<uint4 *>(k_rope + slot * kRope + part * 8) = v;
}

}  // namespace

cudaError_t launch_expand(const void *latent, int64_t num_slots, const void *w_uk,
                          const void *w_uv, void *kv, void *k_rope, int num_groups,
                          cudaStream_t stream) {
    if (num_slots == 0) return cudaSuccess;
    dim3 grid((unsigned)((num_slots + EXP_BM - 1) / EXP_BM), 2 * num_groups);
    expand_kernel<<<grid, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(latent), num_slots,
        static_cast<const __nv_bfloat16 *>(w_uk), static_cast<const __nv_bfloat16 *>(w_uv),
        static_cast<__nv_bfloat16 *>(kv));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    int64_t vec = num_slots * 8;
    copy_rope_kernel<<<(unsigned)((vec + 255) / 256), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(latent), num_slots, static_cast<__nv_bfloat16 *>(k_rope));
    return cudaGetLastError();
}

}  // namespace gqla
