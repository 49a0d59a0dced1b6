// static_scratch.cu -- gqla_decode_gqa_noalloc: a GQA-path decode step whose
// scratch memory lives in a fixed, library-owned device array, for callers
// that cannot allocate device memory themselves.
//
// The ordinary path (gqla_decode_gqa + gqla_combine) needs three scratch
// buffers from the caller: the split partials, their LSEs and the workspace
// with the device error record.  Some callers have no way to provide them:
// code running under a memory manager that forbids cudaMalloc after start-up,
// plugins handed only their input/output tensors, or hosts whose allocator
// cannot be called from the decode thread.  This entry point takes the same
// inputs and the final outputs only; the scratch is the file-scope array
// below.  Under CUDA's lazy module loading (the default) a device claims the
// array when the first call there resolves its address, and holds it until the
// process exits: that first call belongs at start-up, before serving and
// before any stream capture.
#include <mutex>

#include "common.cuh"

using namespace gqla;

namespace {

constexpr size_t kHeaderBytes = 256;  // workspace (device error record), padded to the alignment
static_assert(GQLA_NOALLOC_SCRATCH_BYTES % 256 == 0, "scratch size must be a multiple of 256");

// The scratch.  In host code this name is only a host-side stand-in for the
// symbol: its device address must be obtained with cudaGetSymbolAddress on
// each device before it is handed to a kernel.
static __device__ __align__(256) unsigned char g_scratch[GQLA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_scratch on the current device (looked up once per device).
int scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GQLA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return GQLA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return GQLA_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return GQLA_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

extern "C" int gqla_decode_gqa_noalloc(const gqla_dims *dims, const void *q, int s_q,
                                       const void *kv_expanded, const void *k_rope,
                                       int64_t num_slots, const gqla_kv_index *kv, int num_splits,
                                       void *out, float *lse_out, int32_t *device_error,
                                       gqla_stream_t stream) {
    // the same argument rules as gqla_decode_gqa, checked before anything is enqueued
    if (!dims || !kv || !out || !q || !kv_expanded || !k_rope || !kv->page_table || !kv->seqlens)
        return GQLA_ERR_INVALID_ARG;
    if (dims->num_heads <= 0 || dims->num_groups <= 0 || dims->num_heads % dims->num_groups ||
        !(dims->softmax_scale > 0.0f) || kv->batch <= 0 || kv->max_pages_per_seq <= 0 ||
        kv->num_pages <= 0 || num_splits <= 0 || num_splits > 65535 || s_q <= 0)
        return GQLA_ERR_INVALID_ARG;
    if (!dims_supported(dims) || s_q > 2 || kv->page_size != kPage || kv->batch > 65535 ||
        (dims->num_heads / dims->num_groups) % 4 || (dims->num_heads / dims->num_groups) * s_q > 32)
        return GQLA_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(kv_expanded) |
         reinterpret_cast<uintptr_t>(k_rope) | reinterpret_cast<uintptr_t>(out)) & 15u)
        return GQLA_ERR_INVALID_ARG;
    if (num_slots != (int64_t)kv->num_pages * kv->page_size) return GQLA_ERR_INVALID_ARG;
    const size_t rows = (size_t)(kv->batch + (size_t)num_splits) * s_q * dims->num_heads;
    const size_t o_bytes = align256(rows * kDv * sizeof(float));
    const size_t lse_bytes = align256(rows * sizeof(float));
    if (kHeaderBytes + o_bytes + lse_bytes > GQLA_NOALLOC_SCRATCH_BYTES) return GQLA_ERR_WORKSPACE;

    void *base = nullptr;
    int st = scratch_address(&base);
    if (st != GQLA_OK) return st;
    unsigned char *b = static_cast<unsigned char *>(base);
    float *o_part = reinterpret_cast<float *>(b + kHeaderBytes);
    float *lse_part = reinterpret_cast<float *>(b + kHeaderBytes + o_bytes);

    // the array keeps the previous call's contents: the error record must start at zero
    st = gqla_clear_device_error(b, stream);
    if (st != GQLA_OK) return st;
    st = gqla_decode_gqa(dims, q, s_q, kv_expanded, k_rope, num_slots, kv, num_splits, o_part,
                         lse_part, b, kHeaderBytes, stream);
    if (st != GQLA_OK) return st;
    st = gqla_combine(dims, kv, s_q, num_splits, kDv, o_part, lse_part, nullptr, out, lse_out,
                      stream);
    if (st != GQLA_OK) return st;
    if (device_error &&
        cudaMemcpyAsync(device_error, b, sizeof(DeviceError), cudaMemcpyDeviceToDevice,
                        reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return GQLA_ERR_CUDA;
    return GQLA_OK;
}
