// Front-fold element-wise stages around the tensor-core projections.
//
// Page "MLA Attention Block Gather Decode Kernel API Reference": :param
// input_norm_w (the input RMSNorm is folded into the front-fold), wkv_a (one
// cache row per token), kv_norm_w, cos/sin (interleaved RoPE), kv_cache and
// slot_mapping (the row is written in place), q_norm_w.
//
// RMSNorm(x) W = r * ((x * gamma) W) with r = 1/sqrt(mean(x^2) + eps), so the
// projections run on x * gamma and the per-token r is applied afterwards.
//
// Cache-row precision. The row is held to one bf16 ulp of the exactly rounded
// row. x * gamma (fp32) is split into three bf16 slices hi + mid + lo that
// represent it exactly, and the KV projection runs on all three (3T token
// rows), so the only error left is fp32 accumulation, of order 2^-21 of the
// dot product's natural scale S. An element whose magnitude is within 2^-8 S
// of zero (where that error could reach an ulp) is recomputed exactly in fp64
// from x, gamma and the weight column; all other elements carry a relative
// error below 2^-10, under a bf16 ulp (>= 2^-8 relative).
#include "common.cuh"
#include "launch.h"

namespace mla {

namespace {

constexpr float kFixTau = 0.00390625f;   // 2^-8: recompute elements smaller than this x row RMS
constexpr int kFixGroup = 8;             // flagged elements recomputed together

// Per token: r (fp64), the three bf16 slices of x * gamma, and zeroed
// accumulation rows for the reducing GEMMs of this step.
__global__ void __launch_bounds__(256)
k_fold_prep_tc(const bf16* __restrict__ x, const float* __restrict__ gamma, Dims d, float eps,
               double* __restrict__ r_in, bf16* __restrict__ xg3, float* __restrict__ qacc,
               float* __restrict__ kacc, float* __restrict__ y32) {
    __shared__ double red[32];
    const int t = blockIdx.x;
    const bf16* xr = x + (size_t)t * d.H;
    double ss = 0.0;
    for (int k = threadIdx.x; k < d.H; k += blockDim.x) {
        const double v = bf2d(xr[k]);
        ss += v * v;
    }
    ss = block_sum(ss, red);
    if (threadIdx.x == 0) r_in[t] = 1.0 / sqrt(ss / d.H + (double)eps);
    bf16* hi = xg3 + (size_t)t * d.H;
    bf16* mid = xg3 + (size_t)(d.T + t) * d.H;
    bf16* lo = xg3 + (size_t)(2 * d.T + t) * d.H;
    for (int k = threadIdx.x; k < d.H; k += blockDim.x) {
        const float v = __fmul_rn(bf2f(xr[k]), gamma[k]);
        const bf16 a = __float2bfloat16_rn(v);
        const float r1 = v - __bfloat162float(a);          // exact
        const bf16 b = __float2bfloat16_rn(r1);
        const float r2 = r1 - __bfloat162float(b);         // exact
        hi[k] = a;
        mid[k] = b;
        lo[k] = __float2bfloat16_rn(r2);
    }
    for (int i = threadIdx.x; i < d.Lq; i += blockDim.x) qacc[(size_t)t * d.Lq + i] = 0.f;
    for (int s = 0; s < 3; ++s)
        for (int i = threadIdx.x; i < d.R(); i += blockDim.x) kacc[((size_t)s * d.T + t) * d.R() + i] = 0.f;
    for (int i = threadIdx.x; i < d.H; i += blockDim.x) y32[(size_t)t * d.H + i] = 0.f;
}

// Per token: q-latent RMSNorm -> q_an (bf16), and the cache row.
__global__ void __launch_bounds__(256)
k_fold_norm_tc(const bf16* __restrict__ x, const float* __restrict__ gamma_in, const bf16* __restrict__ wkv_a,
               const double* __restrict__ r_in, const float* __restrict__ qacc, const float* __restrict__ kacc,
               const float* __restrict__ q_norm_w, const float* __restrict__ kv_norm_w,
               const float* __restrict__ cos_t, const float* __restrict__ sin_t,
               const int32_t* __restrict__ slot_mapping, Dims d, float eps, bf16* __restrict__ q_an,
               bf16* __restrict__ kv_cache, int32_t* __restrict__ status) {
    extern __shared__ __align__(16) unsigned char sm[];
    const int R = d.R(), L = d.L, half = d.dr / 2;
    float* kvf = reinterpret_cast<float*>(sm);                      // [R]
    double* kvd = reinterpret_cast<double*>(sm + sizeof(float) * ((R + 1) & ~1));   // [R]
    int* flag_list = reinterpret_cast<int*>(kvd + R);               // [R]
    unsigned char* flagged = reinterpret_cast<unsigned char*>(flag_list + R);   // [R]
    __shared__ float redf[32];
    __shared__ double redd[32];
    __shared__ int n_flag;
    __shared__ double fix_red[8 * kFixGroup];
    const int t = blockIdx.x;
    const double r = r_in[t];
    const float rf = (float)r;

    // q latent RMSNorm
    const float* qa = qacc + (size_t)t * d.Lq;
    float ssq = 0.f;
    for (int i = threadIdx.x; i < d.Lq; i += blockDim.x) {
        const float v = qa[i] * rf;
        ssq += v * v;
    }
    ssq = block_sum(ssq, redf);
    const float rq = rsqrtf(ssq / d.Lq + eps);
    for (int i = threadIdx.x; i < d.Lq; i += blockDim.x)
        q_an[(size_t)t * d.Lq + i] = __float2bfloat16(qa[i] * rf * rq * q_norm_w[i]);

    // kv row from the three slices
    const size_t plane = (size_t)d.T * R;
    for (int j = threadIdx.x; j < R; j += blockDim.x) {
        const size_t o = (size_t)t * R + j;
        kvf[j] = rf * ((kacc[o] + kacc[plane + o]) + kacc[2 * plane + o]);
    }
    if (threadIdx.x == 0) n_flag = 0;
    for (int j = threadIdx.x; j < R; j += blockDim.x) flagged[j] = 0;
    __syncthreads();
    float sl = 0.f, sr = 0.f;
    for (int j = threadIdx.x; j < R; j += blockDim.x) {
        if (j < L) sl += kvf[j] * kvf[j];
        else sr += kvf[j] * kvf[j];
    }
    sl = block_sum(sl, redf);
    sr = block_sum(sr, redf);
    const float tau_l = kFixTau * sqrtf(sl / L), tau_r = kFixTau * sqrtf(sr / d.dr);
    for (int j = threadIdx.x; j < L; j += blockDim.x)
        if (fabsf(kvf[j]) < tau_l) flag_list[atomicAdd(&n_flag, 1)] = j;
    for (int i = threadIdx.x; i < half; i += blockDim.x) {
        const float a = kvf[L + 2 * i], b = kvf[L + 2 * i + 1];
        const float c = cos_t[(size_t)t * half + i], s = sin_t[(size_t)t * half + i];
        if (fminf(fabsf(a * c - b * s), fabsf(a * s + b * c)) < tau_r) {
            const int k = atomicAdd(&n_flag, 2);
            flag_list[k] = L + 2 * i;
            flag_list[k + 1] = L + 2 * i + 1;
        }
    }
    __syncthreads();
    const int nf = n_flag;
    // Exact recompute of flagged elements, r * sum_k (x_k gamma_k) wkv_a[k, j] in fp64,
    // up to kFixGroup elements at a time so the strided weight loads overlap.
    const bf16* xr = x + (size_t)t * d.H;
    for (int f0 = 0; f0 < nf; f0 += kFixGroup) {
        const int ng = min(kFixGroup, nf - f0);
        int jj[kFixGroup];
        double acc[kFixGroup];
#pragma unroll
        for (int q = 0; q < kFixGroup; ++q) {
            jj[q] = q < ng ? flag_list[f0 + q] : flag_list[f0];
            acc[q] = 0.0;
        }
#pragma unroll 4
        for (int k = threadIdx.x; k < d.H; k += blockDim.x) {
            const double xg = bf2d(xr[k]) * (double)gamma_in[k];
            const bf16* wrow = wkv_a + (size_t)k * R;
#pragma unroll
            for (int q = 0; q < kFixGroup; ++q) acc[q] = fma(xg, bf2d(wrow[jj[q]]), acc[q]);
        }
#pragma unroll
        for (int q = 0; q < kFixGroup; ++q) acc[q] = warp_sum(acc[q]);
        __syncthreads();
        if ((threadIdx.x & 31) == 0)
            for (int q = 0; q < kFixGroup; ++q) fix_red[(threadIdx.x >> 5) * kFixGroup + q] = acc[q];
        __syncthreads();
        if (threadIdx.x < ng) {
            double v = 0.0;
            for (int w = 0; w < (int)(blockDim.x >> 5); ++w) v += fix_red[w * kFixGroup + threadIdx.x];
            const int j = jj[threadIdx.x];
            kvd[j] = v * r;
            kvf[j] = (float)(v * r);
            flagged[j] = 1;
        }
        __syncthreads();
    }

    const int32_t slot = slot_mapping[t];
    if (slot < 0 || slot >= d.n_rows()) {
        if (threadIdx.x == 0) set_status(status, MLA_DEV_BAD_SLOT);
        return;
    }
    // kv-latent RMSNorm over the (corrected) latent part, fp64 sum
    double ssk = 0.0;
    for (int j = threadIdx.x; j < L; j += blockDim.x) ssk += (double)kvf[j] * (double)kvf[j];
    ssk = block_sum(ssk, redd);
    const double rk = 1.0 / sqrt(ssk / L + (double)eps);
    const float rkf = (float)rk;
    bf16* row = kv_cache + (size_t)slot * R;
    for (int j = threadIdx.x; j < L; j += blockDim.x)
        row[j] = flagged[j] ? __double2bfloat16(kvd[j] * (double)kv_norm_w[j] * rk)
                            : __float2bfloat16_rn(kvf[j] * kv_norm_w[j] * rkf);
    for (int i = threadIdx.x; i < half; i += blockDim.x) {
        const bool fl = flagged[L + 2 * i];
        const float c = cos_t[(size_t)t * half + i], s = sin_t[(size_t)t * half + i];
        if (fl) {
            const double a = kvd[L + 2 * i], b = kvd[L + 2 * i + 1];
            row[L + 2 * i] = __double2bfloat16(a * c - b * s);
            row[L + 2 * i + 1] = __double2bfloat16(a * s + b * c);
        } else {
            const float a = kvf[L + 2 * i], b = kvf[L + 2 * i + 1];
            row[L + 2 * i] = __float2bfloat16_rn(a * c - b * s);
            row[L + 2 * i + 1] = __float2bfloat16_rn(a * s + b * c);
        }
    }
}

__global__ void k_f32_to_bf16(const float* __restrict__ in, bf16* __restrict__ out, size_t n) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        out[i] = __float2bfloat16(in[i]);
}

}  // namespace

cudaError_t launch_fold_prep_tc(const bf16* x, const float* gamma, const Dims& d, float eps, double* r_in,
                                bf16* xg3, float* qacc, float* kacc, float* y32, cudaStream_t s) {
    k_fold_prep_tc<<<d.T, 256, 0, s>>>(x, gamma, d, eps, r_in, xg3, qacc, kacc, y32);
    return cudaGetLastError();
}

size_t fold_norm_tc_smem(const Dims& d) {
    const int R = d.R();
    return sizeof(float) * ((R + 1) & ~1) + sizeof(double) * R + sizeof(int) * R + R;
}

cudaError_t launch_fold_norm_tc(const bf16* x, const float* gamma_in, const bf16* wkv_a, const double* r_in,
                                const float* qacc, const float* kacc, const float* q_norm_w,
                                const float* kv_norm_w, const float* cos_t, const float* sin_t,
                                const int32_t* slot_mapping, const Dims& d, float eps, bf16* q_an,
                                bf16* kv_cache, int32_t* status, cudaStream_t s) {
    k_fold_norm_tc<<<d.T, 256, fold_norm_tc_smem(d), s>>>(x, gamma_in, wkv_a, r_in, qacc, kacc, q_norm_w,
                                                          kv_norm_w, cos_t, sin_t, slot_mapping, d, eps, q_an,
                                                          kv_cache, status);
    return cudaGetLastError();
}

cudaError_t launch_f32_to_bf16(const float* in, bf16* out, size_t n, cudaStream_t s) {
    const int block = 256;
    const int grid = (int)((n + block - 1) / block < 1184 ? (n + block - 1) / block : 1184);
    k_f32_to_bf16<<<grid, block, 0, s>>>(in, out, n);
    return cudaGetLastError();
}

}  // namespace mla
