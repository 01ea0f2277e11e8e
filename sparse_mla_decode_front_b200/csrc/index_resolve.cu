// Index resolve: selected absolute positions -> physical cache rows, with the
// causal mask (page "MLA Attention Block Gather Decode Kernel API Reference",
// :param gather_indices, positions, block_table; "Notes": the index build is
// issued first, ahead of the front-fold that does not consume it).
//
// For token t and entry j: p = gather_indices[t, j] is kept iff
// 0 <= p <= positions[t]; a kept p resolves to
// block_table[t, p / bs] * bs + p % bs. Kept rows are compacted, in their
// original order, into rows[t, 0 .. n_valid[t]); the softmax is over a set, so
// dropping masked entries and keeping order changes no value. Entries that
// would read outside the block table or the cache are dropped and flagged.
#include "common.cuh"
#include "launch.h"

namespace mla {

namespace {

constexpr int kResolveThreads = 1024;

__global__ void __launch_bounds__(kResolveThreads)
k_index_resolve(const int32_t* __restrict__ gather_indices, const int32_t* __restrict__ block_table,
                const int32_t* __restrict__ positions, Dims d, int32_t* __restrict__ rows,
                int32_t* __restrict__ n_valid, int32_t* __restrict__ status) {
    griddep_launch();   // dependents may start; they wait for this kernel
    griddep_wait();     // the previous kernel of the stream has completed
    __shared__ int32_t warp_tot[32];
    const int t = blockIdx.x;
    const int P = d.P;
    const int32_t pos = positions[t];
    const int32_t* gi = gather_indices + (size_t)t * P;
    const int32_t* bt = block_table + (size_t)t * d.max_blocks;
    int32_t* out = rows + (size_t)t * P;

    // Each thread owns a contiguous run of entries so compaction keeps order.
    const int per = (P + kResolveThreads - 1) / kResolveThreads;
    const int j0 = min(P, (int)threadIdx.x * per), j1 = min(P, j0 + per);
    int cnt = 0;
    int32_t bad = 0;
    for (int j = j0; j < j1; ++j) {
        const int32_t p = gi[j];
        if (p < 0 || p > pos) continue;
        const int32_t lb = p / d.bs;
        if (lb >= d.max_blocks) { bad |= MLA_DEV_BAD_LOGICAL_BLOCK; continue; }
        const int32_t blk = bt[lb];
        if (blk < 0 || blk >= d.n_blocks) { bad |= MLA_DEV_BAD_BLOCK_ID; continue; }
        ++cnt;
    }
    // Exclusive scan of cnt across the block.
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) warp_tot[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        int w = warp_tot[lane];
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += v;
        }
        warp_tot[lane] = wi - w;  // exclusive prefix of warp totals
        if (lane == 31) n_valid[t] = wi;
    }
    __syncthreads();
    int k = warp_tot[wid] + incl - cnt;
    for (int j = j0; j < j1; ++j) {
        const int32_t p = gi[j];
        if (p < 0 || p > pos) continue;
        const int32_t lb = p / d.bs;
        if (lb >= d.max_blocks) continue;
        const int32_t blk = bt[lb];
        if (blk < 0 || blk >= d.n_blocks) continue;
        out[k++] = blk * d.bs + p % d.bs;
    }
    if (bad) set_status(status, bad);
}

}  // namespace

cudaError_t launch_index_resolve(const int32_t* gather_indices, const int32_t* block_table,
                                 const int32_t* positions, const Dims& d, int32_t* rows,
                                 int32_t* n_valid, int32_t* status, cudaStream_t s) {
    return launch_pdl(k_index_resolve, dim3(d.T), dim3(kResolveThreads), 0, s, gather_indices, block_table, positions, d,
                      rows, n_valid, status);
}

}  // namespace mla
