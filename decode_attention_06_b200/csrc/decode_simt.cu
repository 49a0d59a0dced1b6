// decode_simt.cu -- split-KV partial attention of the MQA-absorb path on the FP32 pipes.
//
// One CTA per (chunk of the split plan, 16 query rows).  Each page of 64 tokens is
// staged in shared memory, scores and the online softmax run in fp32 (base-2
// exponent with log2(e) folded into the scale), and the partial output is
// written normalised with its natural-log LSE.  This is the plain CUDA-core
// formulation of the decode; the tensor-core kernels compute the same
// quantities.
#include "common.cuh"

namespace gqla {

namespace {

__device__ __forceinline__ float bf(const __nv_bfloat16 &x) { return __bfloat162float(x); }

// ---------------------------------------------------------------------------
// MQA-absorb path.  grid (num_splits, s_q*h/16), 256 threads, 16 rows per CTA.
// Shared: q~ [16][576] fp32, page [64][576] bf16, P [16][64] fp32.
// Row i of the CTA is flat row rb*16 + i of [s_q][h].
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) decode_absorb_simt_kernel(
    const __nv_bfloat16 *__restrict__ qa, int s_q, int heads,
    const __nv_bfloat16 *__restrict__ cache, const int32_t *__restrict__ page_table,
    const int32_t *__restrict__ seqlens, int batch, int max_pages, int num_pages, int num_splits,
    float scale_log2, float *__restrict__ o_part, float *__restrict__ lse_part, void *ws) {
    constexpr int RB = 16;
    extern __shared__ __align__(16) float smem[];
    float *qs = smem;                                                        // [16][576]
    __nv_bfloat16 *Cs = reinterpret_cast<__nv_bfloat16 *>(qs + RB * kRow);  // [64][576]
    float *Ps = reinterpret_cast<float *>(Cs + kPage * kRow);                // [16][64]
    __shared__ float s_m[RB], s_l[RB], s_alpha[RB];
    __shared__ int s_plan[4];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c = blockIdx.x, rb = blockIdx.y;

    if (warp == 0) {
        int total = warp_total_pages(seqlens, batch);
        int k = chunk_pages(total, num_splits);
        int r0 = c * k, r1 = min(total, r0 + k);
        int b = batch, start = 0;
        if (r0 < r1) warp_find_sequence(seqlens, batch, r0, &b, &start);
        if (lane == 0) { s_plan[0] = r0; s_plan[1] = r1; s_plan[2] = b; s_plan[3] = start; }
    }
    __syncthreads();
    const int r0 = s_plan[0], r1 = s_plan[1];
    int b = s_plan[2], P = s_plan[3];

    for (; b < batch && P < r1; ++b) {
        const int L = seqlens[b];
        const int n = pages_of(L);
        if (n == 0) continue;
        const int p_begin = max(r0, P) - P, p_end = min(r1, P + n) - P;
        P += n;
        if (L > max_pages * kPage) {
            if (tid == 0) report_error(ws, GQLA_ERR_DEVICE, b);
            continue;
        }
        __syncthreads();
        for (int i = tid; i < RB * kRow; i += 256) {
            int row = rb * RB + i / kRow;  // flat (s, h)
            qs[i] = bf(qa[((int64_t)b * s_q * heads + row) * kRow + i % kRow]);
        }
        if (tid < RB) { s_m[tid] = -INFINITY; s_l[tid] = 0.0f; }
        float o[RB][2];
#pragma unroll
        for (int i = 0; i < RB; ++i) o[i][0] = o[i][1] = 0.0f;

        for (int p = p_begin; p < p_end; ++p) {
            const int page = page_table[(int64_t)b * max_pages + p];
            const bool bad = page < 0 || page >= num_pages;
            if (bad && tid == 0) report_error(ws, GQLA_ERR_DEVICE, b);
            __syncthreads();
            if (!bad) {
                const uint4 *src = reinterpret_cast<const uint4 *>(cache + (int64_t)page * kPage * kRow);
                uint4 *dst = reinterpret_cast<uint4 *>(Cs);
                for (int i = tid; i < kPage * kRow / 8; i += 256) dst[i] = src[i];
            }
            __syncthreads();
            for (int i = tid; i < RB * kPage; i += 256) {
                int row = i / kPage, t = i % kPage;
                int s = (rb * RB + row) / heads;
                int tok = p * kPage + t;
                float v = -INFINITY;
                if (!bad && tok <= L - s_q + s) {
                    float acc = 0.0f;
                    const float *qr = qs + row * kRow;
                    const __nv_bfloat162 *cr = reinterpret_cast<const __nv_bfloat162 *>(Cs + t * kRow);
                    for (int d = 0; d < kRow / 2; ++d) {
                        float2 cc = __bfloat1622float2(cr[d]);
                        acc = fmaf(qr[2 * d], cc.x, acc);
                        acc = fmaf(qr[2 * d + 1], cc.y, acc);
                    }
                    v = acc * scale_log2;
                }
                Ps[row * kPage + t] = v;
            }
            __syncthreads();
            for (int row = warp; row < RB; row += 8) {
                float a = Ps[row * kPage + lane], bb = Ps[row * kPage + lane + 32];
                float mx = fmaxf(a, bb);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                float m_old = s_m[row];
                float m_new = fmaxf(m_old, mx);
                float alpha = (m_new == -INFINITY) ? 1.0f : exp2f(m_old - m_new);
                float pa = (a == -INFINITY) ? 0.0f : exp2f(a - m_new);
                float pb = (bb == -INFINITY) ? 0.0f : exp2f(bb - m_new);
                Ps[row * kPage + lane] = pa;
                Ps[row * kPage + lane + 32] = pb;
                float sum = pa + pb;
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
                if (lane == 0) {
                    s_m[row] = m_new;
                    s_l[row] = s_l[row] * alpha + sum;
                    s_alpha[row] = alpha;
                }
            }
            __syncthreads();
            const int d0 = tid * 2;  // latent columns d0, d0+1
            const int t_end = bad ? 0 : min(kPage, L - p * kPage);  // pool rows past L are never read
#pragma unroll
            for (int i = 0; i < RB; ++i) {
                float a0 = o[i][0] * s_alpha[i], a1 = o[i][1] * s_alpha[i];
                const float *pr = Ps + i * kPage;
                for (int t = 0; t < t_end; ++t) {
                    float2 cc = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(Cs + t * kRow + d0));
                    a0 = fmaf(pr[t], cc.x, a0);
                    a1 = fmaf(pr[t], cc.y, a1);
                }
                o[i][0] = a0;
                o[i][1] = a1;
            }
        }
        __syncthreads();
        const int slot = b + c;
#pragma unroll
        for (int i = 0; i < RB; ++i) {
            float l = s_l[i];
            int64_t idx = (int64_t)slot * s_q * heads + rb * RB + i;
            float2 v = l > 0.0f ? make_float2(o[i][0] / l, o[i][1] / l) : make_float2(0.0f, 0.0f);
            *reinterpret_cast<float2 *>(o_part + idx * kLatent + tid * 2) = v;
            if (tid == 0)
                lse_part[idx] = l > 0.0f ? (s_m[i] + __log2f(l)) * 0.6931471805599453f : -INFINITY;
        }
    }
}

}  // namespace

cudaError_t launch_decode_absorb_simt(const void *qa, int s_q, int heads, const void *cache,
                                      const gqla_kv_index *idx, int num_splits, float scale,
                                      float *o_part, float *lse_part, void *ws,
                                      cudaStream_t stream) {
    size_t smem = sizeof(float) * 16 * kRow + sizeof(__nv_bfloat16) * kPage * kRow +
                  sizeof(float) * 16 * kPage;
    cudaFuncSetAttribute(decode_absorb_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    dim3 grid(num_splits, s_q * heads / 16);
    decode_absorb_simt_kernel<<<grid, 256, smem, stream>>>(
        static_cast<const __nv_bfloat16 *>(qa), s_q, heads, static_cast<const __nv_bfloat16 *>(cache),
        idx->page_table, idx->seqlens, idx->batch, idx->max_pages_per_seq, idx->num_pages,
        num_splits, scale * kLog2e, o_part, lse_part, ws);
    return cudaGetLastError();
}

}  // namespace gqla
