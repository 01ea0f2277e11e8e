// Shared device helpers of the sparse MLA gather-decode kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sparse_mla_decode.h"

namespace mla {

typedef __nv_bfloat16 bf16;

// Problem dims as the kernels see them (copied from mla_dims).
struct Dims {
    int T, H, Lq, L, dn, dr, dv, h, bs, n_blocks, max_blocks, P;
    __host__ __device__ int R() const { return L + dr; }          // kv_row_dim
    __host__ __device__ int qk() const { return dn + dr; }        // per-head q width
    __host__ __device__ int n_rows() const { return n_blocks * bs; }
};

__device__ __forceinline__ float bf2f(bf16 v) { return __bfloat162float(v); }
__device__ __forceinline__ double bf2d(bf16 v) { return (double)__bfloat162float(v); }

__device__ __forceinline__ void set_status(int32_t* status, int32_t bits) {
    atomicOr(status, bits);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Programmatic dependent launch. Every kernel of the block is launched with
// launch_pdl(): it may begin while the previous kernel of the stream finishes, so
// it lets its own dependents start (griddep_launch) and waits (griddep_wait)
// before its first access to global memory another kernel writes or reads.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Block-wide sum for blockDim.x a multiple of 32 (<= 1024); `red` holds >= 32 slots.
template <typename T>
__device__ T block_sum(T v, T* red) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    v = warp_sum(v);
    __syncthreads();
    if (lane == 0) red[wid] = v;
    __syncthreads();
    T r = (threadIdx.x < nw) ? red[threadIdx.x] : T(0);
    if (wid == 0) r = warp_sum(r);
    if (threadIdx.x == 0) red[0] = r;
    __syncthreads();
    r = red[0];
    __syncthreads();
    return r;
}

#ifndef __CUDACC_RTC__
// Host: launch `kernel` with programmatic stream serialization allowed (see griddep_wait)
// on a live stream. Under stream capture the launch is plain unless `in_graphs`: measured
// on B200, a graph of this chain replays faster with ordinary edges than with programmatic
// ones for kernels that wait at their start, while stream-launched steps gain from the
// overlap. The projection GEMMs and the query chain pass `in_graphs` (they load their first
// weight tiles before they wait), and so do the attention core and its merge (the core sets up
// its barriers and TMEM first). Without the attribute griddep_wait and griddep_launch do nothing.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_mode(bool in_graphs, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                   cudaStream_t s, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cap) != cudaSuccess) cap = cudaStreamCaptureStatusNone;
    cfg.attrs = attr;
    cfg.numAttrs = (cap == cudaStreamCaptureStatusNone || in_graphs) ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args&&... args) {
    return launch_pdl_mode(false, kernel, grid, block, smem, s, static_cast<Args&&>(args)...);
}
#endif

}  // namespace mla
