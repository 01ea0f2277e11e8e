// mla_block_gather_decode_noalloc: the block step for callers that cannot
// allocate device memory.
//
// Some callers have no way to obtain scratch memory at the point where they
// run the step: a serving engine or plugin host that owns every byte of device
// memory through its own pool and hands out only the tensors it manages, or
// code that must not touch the CUDA allocator in the middle of a stream it is
// building. For them this entry point takes the same inputs and output as
// mla_block_gather_decode() but no workspace: its scratch is one file-scope
// device array of MLA_NOALLOC_SCRATCH_BYTES, which every GPU that loads this
// library holds until the process exits. Nothing here calls cudaMalloc,
// cudaFree or any allocating routine.
//
// The array's host-side name is only a stand-in for the device symbol, so its
// device address is looked up with cudaGetSymbolAddress on the first call made
// on each device (with that device current) and cached. That first call may
// load the module, so it should be made before any stream capture.
//
// Every call shares the one array and leaves its contents behind; the step
// clears the parts that must start at zero (its status word) itself. Two calls
// that overlap on the GPU (different streams, or different host threads on the
// same device) race on the array and must be serialised by the caller. The
// status word of the last call (the array's first bytes, where the workspace
// plan puts it) is read back by mla_block_gather_decode_noalloc_status.
#include <mutex>

#include "common.cuh"

namespace {

static_assert(MLA_NOALLOC_SCRATCH_BYTES % 256 == 0, "scratch size must keep 256-byte alignment");

__device__ __align__(256) unsigned char g_noalloc_scratch[MLA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up once).
int scratch_for_current_device(void** addr) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MLA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return MLA_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *addr = g_scratch_addr[dev];
    return MLA_OK;
}

}  // namespace

extern "C" int mla_block_gather_decode_noalloc(
    const void* hidden_states, const float* input_norm_w,
    const void* wq_a, const float* q_norm_w, const void* wq_b,
    const void* wkv_a, const float* kv_norm_w,
    const void* q_absorb_w, const void* out_absorb_w, const void* o_proj_w,
    const float* cos_t, const float* sin_t,
    void* kv_cache, const int32_t* slot_mapping,
    const int32_t* block_table, const int32_t* positions,
    const int32_t* gather_indices,
    void* out,
    const mla_dims* dims, float softmax_scale, float norm_eps, void* stream) {
    const int dc = mla_block_check_dims(dims);
    if (dc != MLA_OK) return dc;
    if (mla_block_workspace_bytes(dims) > (size_t)MLA_NOALLOC_SCRATCH_BYTES)
        return MLA_ERR_WORKSPACE_TOO_SMALL;
    void* scratch = nullptr;
    if (dims->n_tokens > 0) {
        const int rc = scratch_for_current_device(&scratch);
        if (rc != MLA_OK) return rc;
    }
    return mla_block_gather_decode(hidden_states, input_norm_w, wq_a, q_norm_w, wq_b, wkv_a, kv_norm_w,
                                   q_absorb_w, out_absorb_w, o_proj_w, cos_t, sin_t, kv_cache,
                                   slot_mapping, block_table, positions, gather_indices, out, dims,
                                   softmax_scale, norm_eps, scratch, (size_t)MLA_NOALLOC_SCRATCH_BYTES,
                                   stream);
}

extern "C" int mla_block_gather_decode_noalloc_status(void* stream, int32_t* status) {
    if (!status) return MLA_ERR_NULL_POINTER;
    void* scratch = nullptr;
    const int rc = scratch_for_current_device(&scratch);
    if (rc != MLA_OK) return rc;
    return mla_get_device_status(scratch, stream, status);
}
