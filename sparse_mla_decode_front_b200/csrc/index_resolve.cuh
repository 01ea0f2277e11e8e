// Index resolve of one token by one block (page "MLA Attention Block Gather
// Decode Kernel API Reference", :param gather_indices, positions, block_table).
//
// For token t and entry j: p = gather_indices[t, j] is kept iff
// 0 <= p <= positions[t]; a kept p resolves to
// block_table[t, p / bs] * bs + p % bs. Kept rows are compacted, in their
// original order, into rows[t, 0 .. n_valid[t]); the softmax is over a set, so
// dropping masked entries and keeping order changes no value. Entries that
// would read outside the block table or the cache are dropped and flagged.
#pragma once

#include "common.cuh"

namespace mla {

// blockDim.x: a multiple of 32, at most 1024. `warp_tot`: 32 shared ints.
__device__ __forceinline__ void resolve_token(const int32_t* __restrict__ gather_indices,
                                              const int32_t* __restrict__ block_table,
                                              const int32_t* __restrict__ positions, const Dims& d, int t,
                                              int32_t* __restrict__ rows, int32_t* __restrict__ n_valid,
                                              int32_t* __restrict__ status, int32_t* warp_tot) {
    const int P = d.P;
    const int32_t pos = positions[t];
    const int32_t* gi = gather_indices + (size_t)t * P;
    const int32_t* bt = block_table + (size_t)t * d.max_blocks;
    int32_t* out = rows + (size_t)t * P;

    // Each thread owns a contiguous run of entries so compaction keeps order.
    const int per = (P + (int)blockDim.x - 1) / (int)blockDim.x;
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
        const int nw = (int)blockDim.x >> 5;
        int w = lane < nw ? warp_tot[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += v;
        }
        if (lane < nw) warp_tot[lane] = wi - w;  // exclusive prefix of warp totals
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

}  // namespace mla
