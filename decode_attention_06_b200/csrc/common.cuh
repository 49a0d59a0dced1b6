// common.cuh -- shared device helpers of libgqla: fixed layer widths, the
// split-KV work plan, and the device error record.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gqla.h"

namespace gqla {

constexpr int kLatent = 512;             // r_kv
constexpr int kRope = 64;                // d_R
constexpr int kNope = 128;               // d_nope
constexpr int kDv = 128;                 // d_v
constexpr int kQk = kNope + kRope;       // 192: GQA-path key width
constexpr int kRow = kLatent + kRope;    // 576: latent cache row
constexpr int kKv = kNope + kDv;         // 256: one group's expanded row [K_nope | V]
constexpr int kPage = 64;                // tokens per page
constexpr float kLog2e = 1.4426950408889634f;

// Device error record at the start of the workspace: first error wins.
struct DeviceError {
    int code;
    int info;
};

// Four floats rounded to bf16 (round to nearest even), packed for one 8-byte store.
__device__ __forceinline__ uint2 pack_bf16x4(float a, float b, float c, float d) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
    return make_uint2(*reinterpret_cast<uint32_t *>(&lo), *reinterpret_cast<uint32_t *>(&hi));
}

__device__ __forceinline__ void report_error(void *ws, int code, int info) {
    if (!ws) return;
    DeviceError *e = reinterpret_cast<DeviceError *>(ws);
    if (atomicCAS(&e->code, 0, code) == 0) atomicExch(&e->info, info);
}

// ---------------------------------------------------------------------------
// Split-KV plan.
//
// The pages of the batch are concatenated sequence after sequence (sequence b
// owns global pages [P_b, P_b + n_b), n_b = ceil(L_b / 64)) and cut into
// `num_splits` chunks of ceil(T / num_splits) pages, T = sum_b n_b.  Chunk c
// meets sequence b in at most one contiguous page range, its "piece", whose
// partial result goes to slot b + c.  Distinct pieces get distinct slots
// (a later chunk can only meet later sequences), so batch + num_splits slots
// always suffice.  Every CTA and the combine derive the same plan from the
// device-resident lengths; nothing is precomputed on the host.
// ---------------------------------------------------------------------------

__device__ __forceinline__ int pages_of(int len) { return len > 0 ? (len + kPage - 1) / kPage : 0; }

__device__ __forceinline__ int warp_incl_scan(int v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    return v;
}

// One full warp: total pages T of the batch.
__device__ __forceinline__ int warp_total_pages(const int32_t *seqlens, int batch) {
    int acc = 0;
    for (int b = threadIdx.x & 31; b < batch; b += 32) acc += pages_of(seqlens[b]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    return acc;
}

// One full warp: the first sequence b whose page range ends after global page
// `pos` (skipping empty sequences), and its first global page P_b.  Returns
// b = batch if none.
__device__ __forceinline__ void warp_find_sequence(const int32_t *seqlens, int batch, int pos,
                                                   int *b_out, int *start_out) {
    const int lane = threadIdx.x & 31;
    int base = 0;
    for (int b0 = 0; b0 < batch; b0 += 32) {
        int b = b0 + lane;
        int n = b < batch ? pages_of(seqlens[b]) : 0;
        int incl = warp_incl_scan(n);
        bool hit = b < batch && n > 0 && base + incl > pos;
        unsigned m = __ballot_sync(0xffffffffu, hit);
        if (m) {
            int src = __ffs(m) - 1;
            int excl = __shfl_sync(0xffffffffu, incl - n, src);
            *b_out = b0 + src;
            *start_out = base + excl;
            return;
        }
        base += __shfl_sync(0xffffffffu, incl, 31);
    }
    *b_out = batch;
    *start_out = base;
}

// One full warp: first global page P_b of sequence b.
__device__ __forceinline__ int warp_sequence_start(const int32_t *seqlens, int b) {
    int acc = 0;
    for (int i = threadIdx.x & 31; i < b; i += 32) acc += pages_of(seqlens[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    return acc;
}

__device__ __forceinline__ int chunk_pages(int total_pages, int num_splits) {
    return (total_pages + num_splits - 1) / num_splits;
}

// A split plan with a lead: the batch's pages, concatenated sequence after sequence, are
// cut into num_splits chunks of which the first `lead` are lead_w16 / 16 times as long as
// the rest (whole pages, rounded up, the last chunks possibly short or empty).  With
// lead = 0 this is the equal cut of chunk_pages().  The longer chunks exist for a step that
// runs the GQA decode beside the absorb decode: the absorb decode's CTAs on the short
// chunks finish early and leave their SMs to the GQA decode, while those on the long
// chunks keep the SMs the GQA decode does not use busy.
struct SplitPlan {
    int num_splits, lead, lead_w16;
};

__device__ __forceinline__ void plan_chunk_lengths(int total, const SplitPlan &sp, int *k_lead, int *k_rest) {
    const long long units = (long long)sp.lead * sp.lead_w16 + (long long)(sp.num_splits - sp.lead) * 16;
    const long long k = ((long long)total * 16 + units - 1) / units;
    *k_rest = (int)k;
    *k_lead = (int)((k * sp.lead_w16 + 15) / 16);
}

// Pages [r0, r1) of chunk c (empty past the end).
__device__ __forceinline__ void plan_chunk_range(int total, const SplitPlan &sp, int c, int *r0, int *r1) {
    int kl, kr;
    plan_chunk_lengths(total, sp, &kl, &kr);
    const long long a = c < sp.lead ? (long long)c * kl : (long long)sp.lead * kl + (long long)(c - sp.lead) * kr;
    const long long e = a + (c < sp.lead ? kl : kr);
    *r0 = (int)(a < total ? a : total);
    *r1 = (int)(e < total ? e : total);
}

// The chunk that holds global page `page` (0 <= page < total).
__device__ __forceinline__ int plan_chunk_of(int total, const SplitPlan &sp, int page) {
    int kl, kr;
    plan_chunk_lengths(total, sp, &kl, &kr);
    const long long head = (long long)sp.lead * kl;
    const int c = page < head ? page / kl : sp.lead + (int)((page - head) / kr);
    return c < sp.num_splits - 1 ? c : sp.num_splits - 1;
}

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous kernel of the stream finishes, and waits for it with
// griddepcontrol.wait before touching global memory.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                    cudaStream_t stream, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...);
}

// Host-side argument checks shared by the entry points.
inline bool dims_supported(const gqla_dims *d) {
    return d->d_latent == kLatent && d->d_rope == kRope && d->d_nope == kNope && d->d_v == kDv;
}

}  // namespace gqla
