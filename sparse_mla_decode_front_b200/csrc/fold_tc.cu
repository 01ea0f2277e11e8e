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
constexpr int kFixGroup = 4;             // flagged elements recomputed together

// The three bf16 slices of x * gamma (4 CTAs per token, 8 elements per thread
// per step) and zeroed accumulation rows for the reducing GEMMs of this step.
constexpr int kPrepSplit = 4;

__global__ void __launch_bounds__(256)
k_fold_prep_tc(const bf16* __restrict__ x, const float* __restrict__ gamma, Dims d, bf16* __restrict__ xg3,
               float* __restrict__ qacc, float* __restrict__ kacc, float* __restrict__ y32) {
    const int t = blockIdx.x / kPrepSplit, part = blockIdx.x % kPrepSplit;
    const int nvec = d.H / 8;                       // 8 bf16 per 16-byte vector
    const int v0 = nvec * part / kPrepSplit, v1 = nvec * (part + 1) / kPrepSplit;
    const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)t * d.H);
    uint4* hi = reinterpret_cast<uint4*>(xg3 + (size_t)t * d.H);
    uint4* mid = reinterpret_cast<uint4*>(xg3 + (size_t)(d.T + t) * d.H);
    uint4* lo = reinterpret_cast<uint4*>(xg3 + (size_t)(2 * d.T + t) * d.H);
    for (int v = v0 + threadIdx.x; v < v1; v += blockDim.x) {
        const uint4 xv = xr[v];
        const float4 g0 = reinterpret_cast<const float4*>(gamma)[2 * v];
        const float4 g1 = reinterpret_cast<const float4*>(gamma)[2 * v + 1];
        const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
        const bf16* xb = reinterpret_cast<const bf16*>(&xv);
        uint4 oh, om, ol;
        bf16* ph = reinterpret_cast<bf16*>(&oh);
        bf16* pm = reinterpret_cast<bf16*>(&om);
        bf16* pl = reinterpret_cast<bf16*>(&ol);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float val = __fmul_rn(bf2f(xb[e]), gg[e]);
            const bf16 a = __float2bfloat16_rn(val);
            const float r1 = val - __bfloat162float(a);   // exact
            const bf16 b = __float2bfloat16_rn(r1);
            const float r2 = r1 - __bfloat162float(b);    // exact
            ph[e] = a;
            pm[e] = b;
            pl[e] = __float2bfloat16_rn(r2);
        }
        hi[v] = oh;
        mid[v] = om;
        lo[v] = ol;
    }
    // zero this token's accumulation rows (quarter each)
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    auto zero = [&](float* row, int n) {
        const int n4 = n / 4;
        const int a = n4 * part / kPrepSplit, b = n4 * (part + 1) / kPrepSplit;
        for (int i = a + threadIdx.x; i < b; i += blockDim.x) reinterpret_cast<float4*>(row)[i] = z;
    };
    zero(qacc + (size_t)t * d.Lq, d.Lq);
    for (int sl = 0; sl < 3; ++sl) zero(kacc + ((size_t)sl * d.T + t) * d.R(), d.R());
    zero(y32 + (size_t)t * d.H, d.H);
}

// Per token: q-latent RMSNorm -> q_an (bf16), and the cache row.
__global__ void __launch_bounds__(512)
k_fold_norm_tc(const bf16* __restrict__ x, const float* __restrict__ gamma_in, const bf16* __restrict__ wkv_a,
               double* __restrict__ r_in, const float* __restrict__ qacc, const float* __restrict__ kacc,
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
    __shared__ double fix_red[16 * kFixGroup];
    const int t = blockIdx.x;
    // input RMSNorm scale r = 1/sqrt(mean(x^2) + eps), fp64
    double ssx = 0.0;
    {
        const uint4* xr4 = reinterpret_cast<const uint4*>(x + (size_t)t * d.H);
        for (int v = threadIdx.x; v < d.H / 8; v += blockDim.x) {
            const uint4 xv = xr4[v];
            const bf16* xb = reinterpret_cast<const bf16*>(&xv);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const double f = bf2d(xb[e]);
                ssx += f * f;
            }
        }
    }
    ssx = block_sum(ssx, redd);
    const double r = 1.0 / sqrt(ssx / d.H + (double)eps);
    if (threadIdx.x == 0) r_in[t] = r;
    const float rf = (float)r;

    // q latent RMSNorm
    const float4* qa4 = reinterpret_cast<const float4*>(qacc + (size_t)t * d.Lq);
    float ssq = 0.f;
    for (int i = threadIdx.x; i < d.Lq / 4; i += blockDim.x) {
        const float4 v = qa4[i];
        ssq += (v.x * v.x + v.y * v.y) + (v.z * v.z + v.w * v.w);
    }
    ssq = block_sum(ssq, redf) * rf * rf;
    const float rq = rsqrtf(ssq / d.Lq + eps) * rf;
    for (int i = threadIdx.x; i < d.Lq / 4; i += blockDim.x) {
        const float4 v = qa4[i];
        const float4 g = reinterpret_cast<const float4*>(q_norm_w)[i];
        __nv_bfloat162* o = reinterpret_cast<__nv_bfloat162*>(q_an + (size_t)t * d.Lq) + 2 * i;
        o[0] = __floats2bfloat162_rn(v.x * rq * g.x, v.y * rq * g.y);
        o[1] = __floats2bfloat162_rn(v.z * rq * g.z, v.w * rq * g.w);
    }

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
#pragma unroll 7
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

cudaError_t launch_fold_prep_tc(const bf16* x, const float* gamma, const Dims& d, bf16* xg3, float* qacc,
                                float* kacc, float* y32, cudaStream_t s) {
    k_fold_prep_tc<<<d.T * kPrepSplit, 256, 0, s>>>(x, gamma, d, xg3, qacc, kacc, y32);
    return cudaGetLastError();
}

size_t fold_norm_tc_smem(const Dims& d) {
    const int R = d.R();
    return sizeof(float) * ((R + 1) & ~1) + sizeof(double) * R + sizeof(int) * R + R;
}

cudaError_t launch_fold_norm_tc(const bf16* x, const float* gamma_in, const bf16* wkv_a, double* r_in,
                                const float* qacc, const float* kacc, const float* q_norm_w,
                                const float* kv_norm_w, const float* cos_t, const float* sin_t,
                                const int32_t* slot_mapping, const Dims& d, float eps, bf16* q_an,
                                bf16* kv_cache, int32_t* status, cudaStream_t s) {
    k_fold_norm_tc<<<d.T, 512, fold_norm_tc_smem(d), s>>>(x, gamma_in, wkv_a, r_in, qacc, kacc, q_norm_w,
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
