// combine.cu -- log-sum-exp merge of the split-KV partials, and for the
// MQA-absorb path the per-group up-projection out = o~ W_UV_g applied after
// the merge ("folds W_UV into O": GQLA, paperlayer.ai summary, sec. 2).
//
// Each partial o_i is normalised by its own softmax sum and carries
// lse_i = ln sum_t exp(s_t) over its tokens, so
//   out = sum_i exp(lse_i - M) o_i / sum_i exp(lse_i - M),  M = max_i lse_i,
//   lse = M + ln sum_i exp(lse_i - M).
#include "common.cuh"

namespace gqla {

namespace {

// One block per (sequence b, query token s, group of ROWS heads).  128 threads.
// For d_in = 512 the merged latent row is kept in shared memory and the
// 512 x 128 W_UV_g product is done by the block (thread j -> output j).
template <int DIN>
__global__ void __launch_bounds__(128) combine_kernel(const float *__restrict__ o_part,
                                                      const float *__restrict__ lse_part,
                                                      const int32_t *__restrict__ seqlens,
                                                      int batch, int num_splits, int s_q, int heads,
                                                      int heads_per_group,
                                                      const __nv_bfloat16 *__restrict__ w_uv,
                                                      __nv_bfloat16 *__restrict__ out,
                                                      float *__restrict__ lse_out) {
    constexpr int ROWS = 4;  // heads per block (same group: heads_per_group % 4 == 0 checked on host)
    __shared__ int s_plan[3];
    __shared__ float s_w[ROWS][64];
    __shared__ float s_lat[ROWS][DIN];
    const int tid = threadIdx.x;
    const int h0 = blockIdx.x * ROWS;
    const int s = blockIdx.y;
    const int b = blockIdx.z;

    if (tid < 32) {
        int total = warp_total_pages(seqlens, batch);
        int start = warp_sequence_start(seqlens, b);
        if (tid == 0) {
            int n = pages_of(seqlens[b]);
            int k = chunk_pages(total, num_splits);
            s_plan[0] = n > 0 ? start / k : 0;               // first chunk
            s_plan[1] = n > 0 ? (start + n - 1) / k + 1 : 0;  // one past the last chunk
        }
    }
    __syncthreads();
    const int c0 = s_plan[0], c1 = s_plan[1];
    const int nparts = c1 - c0;

    // per-row merge weights (nparts <= num_splits; up to 64 kept in shared memory at once)
    float M[ROWS], denom[ROWS];
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
        M[r] = -INFINITY;
        for (int c = c0; c < c1; ++c) {
            float v = lse_part[((int64_t)(b + c) * s_q + s) * heads + h0 + r];
            M[r] = fmaxf(M[r], v);
        }
        denom[r] = 0.0f;
    }
    float acc[ROWS][DIN / 128];
#pragma unroll
    for (int r = 0; r < ROWS; ++r)
#pragma unroll
        for (int j = 0; j < DIN / 128; ++j) acc[r][j] = 0.0f;

    for (int cb = c0; cb < c1; cb += 64) {
        int ce = min(c1, cb + 64);
        __syncthreads();
        for (int i = tid; i < ROWS * 64; i += 128) {
            int r = i / 64, c = cb + i % 64;
            float w = 0.0f;
            if (c < ce && M[r] != -INFINITY) {
                float v = lse_part[((int64_t)(b + c) * s_q + s) * heads + h0 + r];
                w = v == -INFINITY ? 0.0f : __expf(v - M[r]);
            }
            s_w[r][i % 64] = w;
        }
        __syncthreads();
        for (int c = cb; c < ce; ++c) {
#pragma unroll
            for (int r = 0; r < ROWS; ++r) {
                float w = s_w[r][c - cb];
                denom[r] += w;
                if (w == 0.0f) continue;
                const float *src = o_part + (((int64_t)(b + c) * s_q + s) * heads + h0 + r) * DIN;
#pragma unroll
                for (int j = 0; j < DIN / 128; ++j) acc[r][j] += w * src[tid + 128 * j];
            }
        }
    }

    if (DIN == kDv) {
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
            float v = denom[r] > 0.0f ? acc[r][0] / denom[r] : 0.0f;
            out[(((int64_t)b * s_q + s) * heads + h0 + r) * kDv + tid] = __float2bfloat16_rn(v);
        }
    } else {
#pragma unroll
        for (int r = 0; r < ROWS; ++r)
#pragma unroll
            for (int j = 0; j < DIN / 128; ++j)
                s_lat[r][tid + 128 * j] = denom[r] > 0.0f ? acc[r][j] / denom[r] : 0.0f;
        __syncthreads();
        const int grp = h0 / heads_per_group;
        const __nv_bfloat16 *W = w_uv + (size_t)grp * kLatent * kDv;
        float y[ROWS];
#pragma unroll
        for (int r = 0; r < ROWS; ++r) y[r] = 0.0f;
        for (int k = 0; k < kLatent; ++k) {
            float w = __bfloat162float(W[(size_t)k * kDv + tid]);
#pragma unroll
            for (int r = 0; r < ROWS; ++r) y[r] = fmaf(s_lat[r][k], w, y[r]);
        }
#pragma unroll
        for (int r = 0; r < ROWS; ++r)
            out[(((int64_t)b * s_q + s) * heads + h0 + r) * kDv + tid] = __float2bfloat16_rn(y[r]);
    }
    if (lse_out && tid < ROWS) {
        float l = (M[tid] == -INFINITY || denom[tid] <= 0.0f) ? -INFINITY : M[tid] + __logf(denom[tid]);
        lse_out[((int64_t)b * s_q + s) * heads + h0 + tid] = l;
    }
}

}  // namespace

cudaError_t launch_combine(const gqla_kv_index *kv, int s_q, int num_splits, int d_in,
                           const float *o_part, const float *lse_part, const void *w_uv,
                           void *out, float *lse_out, int heads, int num_groups,
                           cudaStream_t stream) {
    dim3 grid(heads / 4, s_q, kv->batch);
    const int G = heads / num_groups;
    if (d_in == kLatent) {
        combine_kernel<kLatent><<<grid, 128, 0, stream>>>(
            o_part, lse_part, kv->seqlens, kv->batch, num_splits, s_q, heads, G,
            static_cast<const __nv_bfloat16 *>(w_uv), static_cast<__nv_bfloat16 *>(out), lse_out);
    } else {
        combine_kernel<kDv><<<grid, 128, 0, stream>>>(
            o_part, lse_part, kv->seqlens, kv->batch, num_splits, s_q, heads, G, nullptr,
            static_cast<__nv_bfloat16 *>(out), lse_out);
    }
    return cudaGetLastError();
}

}  // namespace gqla
