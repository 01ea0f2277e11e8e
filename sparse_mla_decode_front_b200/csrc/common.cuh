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

}  // namespace mla
