// Token-batch x weight product on CUDA cores: C[t, n] = sum_k A[t, k] W[k, n].
// A is fp32 [T, K] (row stride lda), W bf16 [K, N] row-major (the page stores
// every projection as [in, out]), C fp32 or bf16 [T, N] (row stride ldc).
// Used for the projections until the tensor-core GEMM covers a shape.
#include "common.cuh"
#include "launch.h"

namespace mla {

namespace {

constexpr int kCols = 256, kTok = 16, kK = 32;

template <typename OutT>
__global__ void __launch_bounds__(kCols)
k_gemm_simt(const float* __restrict__ A, int lda, const bf16* __restrict__ W, int ldw,
            OutT* __restrict__ C, int ldc, int T, int N, int K) {
    __shared__ float as[kTok][kK];
    const int n = blockIdx.x * kCols + threadIdx.x;
    const int t0 = blockIdx.y * kTok;
    float acc[kTok];
#pragma unroll
    for (int i = 0; i < kTok; ++i) acc[i] = 0.f;
    for (int k0 = 0; k0 < K; k0 += kK) {
        __syncthreads();
        for (int e = threadIdx.x; e < kTok * kK; e += blockDim.x) {
            const int i = e / kK, k = k0 + e % kK, t = t0 + i;
            as[i][e % kK] = (t < T && k < K) ? A[(size_t)t * lda + k] : 0.f;
        }
        __syncthreads();
        if (n < N) {
            const int kn = min(kK, K - k0);
#pragma unroll 4
            for (int kk = 0; kk < kn; ++kk) {
                const float w = bf2f(W[(size_t)(k0 + kk) * ldw + n]);
#pragma unroll
                for (int i = 0; i < kTok; ++i) acc[i] = fmaf(as[i][kk], w, acc[i]);
            }
        }
    }
    if (n < N) {
#pragma unroll
        for (int i = 0; i < kTok; ++i) {
            if (t0 + i >= T) break;
            if constexpr (sizeof(OutT) == 4) C[(size_t)(t0 + i) * ldc + n] = acc[i];
            else C[(size_t)(t0 + i) * ldc + n] = __float2bfloat16(acc[i]);
        }
    }
}

}  // namespace

cudaError_t launch_gemm_simt_f32(const float* A, int lda, const bf16* W, int ldw, float* C, int ldc,
                                 int T, int N, int K, cudaStream_t s) {
    dim3 grid((N + kCols - 1) / kCols, (T + kTok - 1) / kTok);
    k_gemm_simt<float><<<grid, kCols, 0, s>>>(A, lda, W, ldw, C, ldc, T, N, K);
    return cudaGetLastError();
}

cudaError_t launch_gemm_simt_bf16(const float* A, int lda, const bf16* W, int ldw, bf16* C, int ldc,
                                  int T, int N, int K, cudaStream_t s) {
    dim3 grid((N + kCols - 1) / kCols, (T + kTok - 1) / kTok);
    k_gemm_simt<bf16><<<grid, kCols, 0, s>>>(A, lda, W, ldw, C, ldc, T, N, K);
    return cudaGetLastError();
}

}  // namespace mla
