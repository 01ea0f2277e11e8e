// Front-fold element-wise stages and the exact cache-row path (CUDA cores).
//
// Page "MLA Attention Block Gather Decode Kernel API Reference": :param
// input_norm_w (RMSNorm folded into the front-fold), wkv_a (one cache row per
// token), kv_norm_w (RMSNorm of the latent part), cos/sin (interleaved RoPE),
// kv_cache + slot_mapping (the row is written in place), q_norm_w, q_absorb_w.
//
// The cache row is computed in fp64 from the exact inputs (bf16 x, fp32 gamma,
// bf16 weights) and rounded once to bf16, so it lands within one bf16 ulp of
// the exactly rounded row -- a single fp32 rounding of x*gamma before a 7168-
// long dot product already breaks that bar for small-magnitude elements.
#include "common.cuh"
#include "launch.h"

namespace mla {

namespace {

// r[t] = 1/sqrt(mean(x^2) + eps) (fp64) and xn[t] = x * r * gamma (fp32).
__global__ void __launch_bounds__(256)
k_fold_prep(const bf16* __restrict__ x, const float* __restrict__ gamma, Dims d, float eps,
            double* __restrict__ r_in, float* __restrict__ xn) {
    __shared__ double red[32];
    const int t = blockIdx.x;
    const bf16* xr = x + (size_t)t * d.H;
    double ss = 0.0;
    for (int k = threadIdx.x; k < d.H; k += blockDim.x) {
        const double v = bf2d(xr[k]);
        ss += v * v;
    }
    ss = block_sum(ss, red);
    const double r = 1.0 / sqrt(ss / d.H + (double)eps);
    if (threadIdx.x == 0) r_in[t] = r;
    for (int k = threadIdx.x; k < d.H; k += blockDim.x)
        xn[(size_t)t * d.H + k] = (float)(bf2d(xr[k]) * r * (double)gamma[k]);
}

// kv[t, n] = r[t] * sum_k (x[t,k] * gamma[k]) * wkv_a[k, n] in fp64 (products exact).
constexpr int kKvCols = 128, kKvTok = 8, kKvK = 128;

__global__ void __launch_bounds__(kKvCols)
k_kv_down_f64(const bf16* __restrict__ x, const float* __restrict__ gamma,
              const bf16* __restrict__ wkv_a, const double* __restrict__ r_in, Dims d,
              double* __restrict__ kv) {
    __shared__ double xs[kKvTok][kKvK];
    const int R = d.R();
    const int n = blockIdx.x * kKvCols + threadIdx.x;
    const int t0 = blockIdx.y * kKvTok;
    double acc[kKvTok];
#pragma unroll
    for (int i = 0; i < kKvTok; ++i) acc[i] = 0.0;
    for (int k0 = 0; k0 < d.H; k0 += kKvK) {
        __syncthreads();
        for (int e = threadIdx.x; e < kKvTok * kKvK; e += blockDim.x) {
            const int i = e / kKvK, k = k0 + e % kKvK, t = t0 + i;
            xs[i][e % kKvK] = (t < d.T && k < d.H) ? bf2d(x[(size_t)t * d.H + k]) * (double)gamma[k] : 0.0;
        }
        __syncthreads();
        if (n < R) {
            const int kn = min(kKvK, d.H - k0);
            for (int kk = 0; kk < kn; ++kk) {
                const double w = bf2d(wkv_a[(size_t)(k0 + kk) * R + n]);
#pragma unroll
                for (int i = 0; i < kKvTok; ++i) acc[i] = fma(xs[i][kk], w, acc[i]);
            }
        }
    }
    if (n < R) {
#pragma unroll
        for (int i = 0; i < kKvTok; ++i)
            if (t0 + i < d.T) kv[(size_t)(t0 + i) * R + n] = acc[i] * r_in[t0 + i];
    }
}

// Per token: q RMSNorm (fp32) and the cache row (fp64 -> one bf16 rounding).
__global__ void __launch_bounds__(256)
k_fold_norm(const float* __restrict__ q_a, const float* __restrict__ q_norm_w,
            const double* __restrict__ kv, const float* __restrict__ kv_norm_w,
            const float* __restrict__ cos_t, const float* __restrict__ sin_t,
            const int32_t* __restrict__ slot_mapping, Dims d, float eps,
            float* __restrict__ q_an, bf16* __restrict__ kv_cache, int32_t* __restrict__ status) {
    __shared__ double redd[32];
    __shared__ float redf[32];
    const int t = blockIdx.x;
    const int R = d.R(), L = d.L;
    // q latent RMSNorm
    const float* qa = q_a + (size_t)t * d.Lq;
    float ssq = 0.f;
    for (int i = threadIdx.x; i < d.Lq; i += blockDim.x) ssq += qa[i] * qa[i];
    ssq = block_sum(ssq, redf);
    const float rq = rsqrtf(ssq / d.Lq + eps);
    for (int i = threadIdx.x; i < d.Lq; i += blockDim.x)
        q_an[(size_t)t * d.Lq + i] = qa[i] * rq * q_norm_w[i];
    // kv latent RMSNorm + k_pe RoPE, fp64
    const double* kr = kv + (size_t)t * R;
    double ssk = 0.0;
    for (int i = threadIdx.x; i < L; i += blockDim.x) ssk += kr[i] * kr[i];
    ssk = block_sum(ssk, redd);
    const double rk = 1.0 / sqrt(ssk / L + (double)eps);
    const int32_t slot = slot_mapping[t];
    if (slot < 0 || slot >= d.n_rows()) {
        if (threadIdx.x == 0) set_status(status, MLA_DEV_BAD_SLOT);
        return;
    }
    bf16* row = kv_cache + (size_t)slot * R;
    for (int i = threadIdx.x; i < L; i += blockDim.x)
        row[i] = __double2bfloat16(kr[i] * rk * (double)kv_norm_w[i]);
    const int half = d.dr / 2;
    for (int i = threadIdx.x; i < half; i += blockDim.x) {
        const double a = kr[L + 2 * i], b = kr[L + 2 * i + 1];
        const double c = cos_t[(size_t)t * half + i], s = sin_t[(size_t)t * half + i];
        row[L + 2 * i] = __double2bfloat16(a * c - b * s);
        row[L + 2 * i + 1] = __double2bfloat16(a * s + b * c);
    }
}

// Query tile: qtile[t, h, 0:L] = q_nope[t,h] @ q_absorb_w[h]; qtile[t, h, L:R] = rope(q_pe).
constexpr int kAbsCols = 128, kAbsTok = 16;

__global__ void __launch_bounds__(kAbsCols)
k_q_absorb_rope(const float* __restrict__ q, const bf16* __restrict__ q_absorb_w,
                const float* __restrict__ cos_t, const float* __restrict__ sin_t, Dims d,
                bf16* __restrict__ qtile) {
    extern __shared__ float qs[];  // [kAbsTok][dn]
    const int hh = blockIdx.x;
    const int l = blockIdx.y * kAbsCols + threadIdx.x;
    const int R = d.R(), qk = d.qk();
    const bf16* A = q_absorb_w + (size_t)hh * d.dn * d.L;
    for (int t0 = 0; t0 < d.T; t0 += kAbsTok) {
        __syncthreads();
        for (int e = threadIdx.x; e < kAbsTok * d.dn; e += blockDim.x) {
            const int i = e / d.dn, j = e % d.dn, t = t0 + i;
            qs[e] = (t < d.T) ? q[(size_t)t * d.h * qk + (size_t)hh * qk + j] : 0.f;
        }
        __syncthreads();
        if (l < d.L) {
            float acc[kAbsTok];
#pragma unroll
            for (int i = 0; i < kAbsTok; ++i) acc[i] = 0.f;
            for (int j = 0; j < d.dn; ++j) {
                const float w = bf2f(A[(size_t)j * d.L + l]);
#pragma unroll
                for (int i = 0; i < kAbsTok; ++i) acc[i] = fmaf(qs[i * d.dn + j], w, acc[i]);
            }
#pragma unroll
            for (int i = 0; i < kAbsTok; ++i)
                if (t0 + i < d.T) qtile[((size_t)(t0 + i) * d.h + hh) * R + l] = __float2bfloat16(acc[i]);
        }
    }
    if (blockIdx.y == 0) {
        const int half = d.dr / 2;
        for (int e = threadIdx.x; e < d.T * half; e += blockDim.x) {
            const int t = e / half, i = e % half;
            const float* qp = q + (size_t)t * d.h * qk + (size_t)hh * qk + d.dn;
            const float a = qp[2 * i], b = qp[2 * i + 1];
            const float c = cos_t[(size_t)t * half + i], s = sin_t[(size_t)t * half + i];
            bf16* o = qtile + ((size_t)t * d.h + hh) * R + d.L;
            o[2 * i] = __float2bfloat16(a * c - b * s);
            o[2 * i + 1] = __float2bfloat16(a * s + b * c);
        }
    }
}

}  // namespace

cudaError_t launch_fold_prep(const bf16* x, const float* gamma, const Dims& d, float eps,
                             double* r_in, float* xn, cudaStream_t s) {
    k_fold_prep<<<d.T, 256, 0, s>>>(x, gamma, d, eps, r_in, xn);
    return cudaGetLastError();
}

cudaError_t launch_kv_down_f64(const bf16* x, const float* gamma, const bf16* wkv_a,
                               const double* r_in, const Dims& d, double* kv, cudaStream_t s) {
    dim3 grid((d.R() + kKvCols - 1) / kKvCols, (d.T + kKvTok - 1) / kKvTok);
    k_kv_down_f64<<<grid, kKvCols, 0, s>>>(x, gamma, wkv_a, r_in, d, kv);
    return cudaGetLastError();
}

cudaError_t launch_fold_norm(const float* q_a, const float* q_norm_w, const double* kv,
                             const float* kv_norm_w, const float* cos_t, const float* sin_t,
                             const int32_t* slot_mapping, const Dims& d, float eps, float* q_an,
                             bf16* kv_cache, int32_t* status, cudaStream_t s) {
    k_fold_norm<<<d.T, 256, 0, s>>>(q_a, q_norm_w, kv, kv_norm_w, cos_t, sin_t, slot_mapping, d, eps,
                                    q_an, kv_cache, status);
    return cudaGetLastError();
}

cudaError_t launch_q_absorb_rope(const float* q, const bf16* q_absorb_w, const float* cos_t,
                                 const float* sin_t, const Dims& d, bf16* qtile, cudaStream_t s) {
    dim3 grid(d.h, (d.L + kAbsCols - 1) / kAbsCols);
    const size_t smem = sizeof(float) * kAbsTok * d.dn;
    k_q_absorb_rope<<<grid, kAbsCols, smem, s>>>(q, q_absorb_w, cos_t, sin_t, d, qtile);
    return cudaGetLastError();
}

}  // namespace mla
