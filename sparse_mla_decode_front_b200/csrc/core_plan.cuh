// Work plan of the attention core: the first 64-key tile of every work item and
// the merge plan of the items split between cluster runs. Shared by the plan
// kernel (core_tc.cu) and the extra plan block of the q / kv fold (fold_tc.cu).
#pragma once

#include "common.cuh"

namespace mla {
namespace core {

constexpr int KT = 64;                    // keys per tile (N of the score UMMA)
constexpr int kMinTilesPerCluster = 2;    // fewer tiles per cluster run: fewer clusters

__host__ __device__ __forceinline__ int clusters_for(int U, int max_clusters) {
    const int c = U / kMinTilesPerCluster;
    return c < 1 ? 1 : (c > max_clusters ? max_clusters : c);
}

// First unit of cluster run c of C over U units (U * C < 2^31: checked on the host).
__device__ __forceinline__ int run_start(int U, int c, int C) { return (int)((unsigned)U * (unsigned)c / (unsigned)C); }
// The run holding unit u.
__device__ __forceinline__ int run_of(int U, int u, int C) {
    int c = (int)((unsigned)C * (unsigned)u / (unsigned)U);
    while (c + 1 < C && run_start(U, c + 1, C) <= u) ++c;
    while (c > 0 && run_start(U, c, C) > u) --c;
    return c;
}

// First tile of every work item (tiles = ceil(kept rows / KT)): block-wide scan.
// Then the merge plan of the partial contexts: an item is split when a run
// boundary falls strictly inside it; desc[cb] of the first such boundary holds
// (item, number of runs holding parts, whether the first part is its run's second
// slot), every other desc entry -1.
// Block-wide (blockDim.x a multiple of 32, at most 1024). base: [T * HG + 1];
// desc: [max_clusters + 1].
static __device__ __noinline__ void plan_items(const int32_t* __restrict__ n_valid, int T, int HG, int max_clusters,
                                               int32_t* __restrict__ base, int4* __restrict__ desc) {
    __shared__ int warp_tot[32];
    __shared__ int carry;
    const int W = T * HG;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    for (int w0 = 0; w0 < W; w0 += blockDim.x) {
        const int w = w0 + threadIdx.x;
        const int n = w < W ? (n_valid[w / HG] + KT - 1) / KT : 0;
        int incl = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) warp_tot[wid] = incl;
        __syncthreads();
        if (wid == 0) {
            const int nw = (int)blockDim.x >> 5;
            const int x = lane < nw ? warp_tot[lane] : 0;
            int xi = x;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, xi, o);
                if (lane >= o) xi += v;
            }
            if (lane < nw) warp_tot[lane] = xi - x;
        }
        __syncthreads();
        const int excl = carry + warp_tot[wid] + incl - n;
        if (w < W) base[w] = excl;
        __syncthreads();
        if (threadIdx.x == blockDim.x - 1) carry = excl + n;
        __syncthreads();
    }
    const int U = carry;
    if (threadIdx.x == 0) base[W] = U;
    for (int cb = threadIdx.x; cb <= max_clusters; cb += blockDim.x) desc[cb] = make_int4(-1, 0, 0, 0);
    __syncthreads();   // the block's writes of base and desc are ordered before what follows
    if (U == 0) return;
    const int C = clusters_for(U, max_clusters);
    for (int w = threadIdx.x; w < W; w += blockDim.x) {
        const int b0 = base[w], b1 = base[w + 1];
        if (b1 <= b0) continue;
        const int cf = run_of(U, b0, C);
        if (cf + 1 >= C || run_start(U, cf + 1, C) >= b1) continue;   // one run holds the whole item
        const int cl = run_of(U, b1 - 1, C);
        desc[cf + 1] = make_int4(w, cl - cf + 1, run_start(U, cf, C) < b0 ? 1 : 0, 0);
    }
}

}  // namespace core
}  // namespace mla
