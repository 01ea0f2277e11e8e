// Internal launchers of the stage kernels (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace mla {

cudaError_t launch_index_resolve(const int32_t* gather_indices, const int32_t* block_table,
                                 const int32_t* positions, const Dims& d, int32_t* rows,
                                 int32_t* n_valid, int32_t* status, cudaStream_t s);

cudaError_t launch_fold_prep(const bf16* x, const float* gamma, const Dims& d, float eps,
                             double* r_in, float* xn, cudaStream_t s);
cudaError_t launch_kv_down_f64(const bf16* x, const float* gamma, const bf16* wkv_a,
                               const double* r_in, const Dims& d, double* kv, cudaStream_t s);
cudaError_t launch_fold_norm(const float* q_a, const float* q_norm_w, const double* kv,
                             const float* kv_norm_w, const float* cos_t, const float* sin_t,
                             const int32_t* slot_mapping, const Dims& d, float eps, float* q_an,
                             bf16* kv_cache, int32_t* status, cudaStream_t s);
cudaError_t launch_q_absorb_rope(const float* q, const bf16* q_absorb_w, const float* cos_t,
                                 const float* sin_t, const Dims& d, bf16* qtile, cudaStream_t s);

cudaError_t launch_gemm_simt_f32(const float* A, int lda, const bf16* W, int ldw, float* C, int ldc,
                                 int T, int N, int K, cudaStream_t s);
cudaError_t launch_gemm_simt_bf16(const float* A, int lda, const bf16* W, int ldw, bf16* C, int ldc,
                                  int T, int N, int K, cudaStream_t s);

size_t core_simt_smem(const Dims& d);
bool core_simt_supports(const Dims& d);
cudaError_t launch_core_simt(const bf16* qtile, const bf16* kv_cache, const int32_t* rows,
                             const int32_t* n_valid, const Dims& d, float scale, float* ctx,
                             cudaStream_t s);

cudaError_t launch_out_absorb_simt(const float* ctx, const bf16* out_absorb_w, const Dims& d, float* o,
                                   cudaStream_t s);

}  // namespace mla
