// Index resolve kernel: one block per token (body in index_resolve.cuh; the
// page "MLA Attention Block Gather Decode Kernel API Reference", "Notes": the index
// build is issued first, ahead of the front-fold that does not consume it).
#include "common.cuh"
#include "index_resolve.cuh"
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
    resolve_token(gather_indices, block_table, positions, d, blockIdx.x, rows, n_valid, status, warp_tot);
}

}  // namespace

cudaError_t launch_index_resolve(const int32_t* gather_indices, const int32_t* block_table,
                                 const int32_t* positions, const Dims& d, int32_t* rows,
                                 int32_t* n_valid, int32_t* status, cudaStream_t s) {
    return launch_pdl(k_index_resolve, dim3(d.T), dim3(kResolveThreads), 0, s, gather_indices, block_table, positions, d,
                      rows, n_valid, status);
}

}  // namespace mla
