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
#include "core_plan.cuh"
#include "index_resolve.cuh"
#include "launch.h"

namespace mla {

namespace {

constexpr float kFixTau = 0.00390625f;   // 2^-8: recompute elements smaller than this x row RMS

// The three bf16 slices of x * gamma (4 CTAs per token, 8 elements per thread
// per step) and zeroed accumulation rows for the reducing GEMMs of this step.
constexpr int kPrepSplit = 4;

// Part `part` of `parts` of token t's prep work, by one block.
__device__ __forceinline__ void prep_token(const bf16* __restrict__ x, const float* __restrict__ gamma, const Dims& d,
                                           bf16* __restrict__ xg3, float* __restrict__ qacc, float* __restrict__ kacc,
                                           float* __restrict__ y32, double* __restrict__ fix,
                                           int32_t* __restrict__ flag_count, int t, int part, int parts) {
    const int nvec = d.H / 8;                       // 8 bf16 per 16-byte vector
    const int v0 = nvec * part / parts, v1 = nvec * (part + 1) / parts;
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
        const int a = n4 * part / parts, b = n4 * (part + 1) / parts;
        for (int i = a + threadIdx.x; i < b; i += blockDim.x) reinterpret_cast<float4*>(row)[i] = z;
    };
    zero(qacc + (size_t)t * d.Lq, d.Lq);
    for (int sl = 0; sl < 3; ++sl) zero(kacc + ((size_t)sl * d.T + t) * d.R(), d.R());
    zero(y32 + (size_t)t * d.H, d.H);
    double* fr = fix + (size_t)t * d.R();
    for (int i = d.R() * part / parts + threadIdx.x; i < d.R() * (part + 1) / parts; i += blockDim.x)
        fr[i] = 0.0;
    if (t == 0 && part == 0 && threadIdx.x == 0) *flag_count = 0;
}

__global__ void __launch_bounds__(256)
k_fold_prep_tc(const bf16* __restrict__ x, const float* __restrict__ gamma, Dims d, bf16* __restrict__ xg3,
               float* __restrict__ qacc, float* __restrict__ kacc, float* __restrict__ y32,
               double* __restrict__ fix, int32_t* __restrict__ flag_count) {
    griddep_launch();   // dependents may start; they wait for this kernel
    griddep_wait();     // the previous kernel of the stream has completed
    prep_token(x, gamma, d, xg3, qacc, kacc, y32, fix, flag_count, blockIdx.x / kPrepSplit,
               blockIdx.x % kPrepSplit, kPrepSplit);
}

// The step's first launch: blocks [0, T) resolve the indices of token t, blocks
// [T, 2T) the prep work of token t - T (the two are independent).
constexpr int kStartThreads = 512;
__global__ void __launch_bounds__(kStartThreads)
k_step_start(const int32_t* __restrict__ gather_indices, const int32_t* __restrict__ block_table,
             const int32_t* __restrict__ positions, int32_t* __restrict__ rows, int32_t* __restrict__ n_valid,
             int32_t* __restrict__ status, const bf16* __restrict__ x, const float* __restrict__ gamma, Dims d,
             bf16* __restrict__ xg3, float* __restrict__ qacc, float* __restrict__ kacc,
             float* __restrict__ y32, double* __restrict__ fix, int32_t* __restrict__ flag_count) {
    griddep_launch();   // dependents may start; they wait for this kernel
    griddep_wait();     // the previous kernel of the stream has completed
    __shared__ int32_t warp_tot[32];
    if ((int)blockIdx.x < d.T)
        resolve_token(gather_indices, block_table, positions, d, blockIdx.x, rows, n_valid, status, warp_tot);
    else
        prep_token(x, gamma, d, xg3, qacc, kacc, y32, fix, flag_count, blockIdx.x - d.T, 0, 1);
}

// Elements of the kv row that the exact fp64 path recomputes: latent elements
// smaller than kFixTau x the latent RMS, and both elements of a RoPE pair whose
// rotated value is smaller than kFixTau x the rope-part RMS. Evaluated the same
// way (same fp32 inputs) by the flagging and the row kernels.
__device__ __forceinline__ bool kv_flag(const float* kvf, int j, int L, float tau_l, float tau_r, float c, float s) {
    if (j < L) return fabsf(kvf[j]) < tau_l;
    const int base = L + ((j - L) & ~1);
    const float a = kvf[base], b = kvf[base + 1];
    return fminf(fabsf(a * c - b * s), fabsf(a * s + b * c)) < tau_r;
}

// Per token: input RMS scale r, q-latent RMSNorm -> q_an (bf16), the fp32 kv row
// (sum of the three slice accumulators, times r) and the list of its flagged elements.
// Every global load of the token is issued before the first reduction, so the block
// waits for memory once (the hidden row beyond kQkvX vectors per thread and the q
// row beyond kQkvQ go through a second round).
constexpr int kQkvThreads = 256;
constexpr int kQkvX = 4;   // 16-byte vectors of x per thread in the first round (hidden <= 8192)
constexpr int kQkvQ = 2;   // float4 of the q row per thread in the first round (q_lora_rank <= 2048)
constexpr int kQkvK = 3;   // kv-row elements per thread (kv_row_dim <= 768)

__global__ void __launch_bounds__(kQkvThreads)
k_fold_q_kv(const bf16* __restrict__ x, const float* __restrict__ qacc, const float* __restrict__ kacc,
            const float* __restrict__ q_norm_w, const float* __restrict__ cos_t, const float* __restrict__ sin_t,
            Dims d, float eps, double* __restrict__ r_in, bf16* __restrict__ q_an, float* __restrict__ kv_f32,
            int32_t* __restrict__ flag_count, int32_t* __restrict__ flag_list, CorePlanArgs plan) {
    griddep_launch();   // dependents may start; they wait for this kernel
    griddep_wait();     // the previous kernel of the stream has completed
    if ((int)blockIdx.x == d.T) {   // the extra block: the core's work plan (n_valid is final)
        core::plan_items(plan.n_valid, d.T, plan.HG, plan.max_clusters, plan.item_base, plan.merge_desc);
        return;
    }
    __shared__ float redf[32];
    __shared__ double redd[32];
    extern __shared__ __align__(16) float kvs[];   // [R]
    const int t = blockIdx.x, tid = threadIdx.x;
    const int R = d.R(), L = d.L, half = d.dr / 2;
    const int nx = d.H / 8, nq = d.Lq / 4;
    const uint4* xr4 = reinterpret_cast<const uint4*>(x + (size_t)t * d.H);
    const float4* qa4 = reinterpret_cast<const float4*>(qacc + (size_t)t * d.Lq);
    const float4* qw4 = reinterpret_cast<const float4*>(q_norm_w);
    const size_t plane = (size_t)d.T * R;

    uint4 xv[kQkvX];
    float4 qv[kQkvQ], gv[kQkvQ];
    float ka[kQkvK], kb[kQkvK], kc[kQkvK], cs[kQkvK], sn[kQkvK];
#pragma unroll
    for (int u = 0; u < kQkvX; ++u) {
        const int v = tid + u * kQkvThreads;
        xv[u] = v < nx ? xr4[v] : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kQkvQ; ++u) {
        const int i = tid + u * kQkvThreads;
        if (i < nq) { qv[u] = qa4[i]; gv[u] = qw4[i]; }
    }
#pragma unroll
    for (int u = 0; u < kQkvK; ++u) {
        const int j = tid + u * kQkvThreads;
        cs[u] = 0.f;
        sn[u] = 0.f;
        if (j < R) {
            const size_t o = (size_t)t * R + j;
            ka[u] = kacc[o];
            kb[u] = kacc[plane + o];
            kc[u] = kacc[2 * plane + o];
            if (j >= L) {
                const int pi = (j - L) >> 1;
                cs[u] = cos_t[(size_t)t * half + pi];
                sn[u] = sin_t[(size_t)t * half + pi];
            }
        }
    }

    // input RMS
    double ssx = 0.0;
    auto add_sq = [&](const uint4& w) {
        const bf16* xb = reinterpret_cast<const bf16*>(&w);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const double f = bf2d(xb[e]);
            ssx += f * f;
        }
    };
#pragma unroll
    for (int u = 0; u < kQkvX; ++u) add_sq(xv[u]);
    for (int v = tid + kQkvX * kQkvThreads; v < nx; v += kQkvThreads) add_sq(xr4[v]);
    ssx = block_sum(ssx, redd);
    const double r = 1.0 / sqrt(ssx / d.H + (double)eps);
    if (tid == 0) r_in[t] = r;
    const float rf = (float)r;
    // q latent RMSNorm
    float ssq = 0.f;
    auto sq4 = [](const float4& v) { return (v.x * v.x + v.y * v.y) + (v.z * v.z + v.w * v.w); };
#pragma unroll
    for (int u = 0; u < kQkvQ; ++u)
        if (tid + u * kQkvThreads < nq) ssq += sq4(qv[u]);
    for (int i = tid + kQkvQ * kQkvThreads; i < nq; i += kQkvThreads) ssq += sq4(qa4[i]);
    ssq = block_sum(ssq, redf) * rf * rf;
    const float rq = rsqrtf(ssq / d.Lq + eps) * rf;
    auto put_q = [&](int i, const float4& v, const float4& g) {
        __nv_bfloat162* o = reinterpret_cast<__nv_bfloat162*>(q_an + (size_t)t * d.Lq) + 2 * i;
        o[0] = __floats2bfloat162_rn(v.x * rq * g.x, v.y * rq * g.y);
        o[1] = __floats2bfloat162_rn(v.z * rq * g.z, v.w * rq * g.w);
    };
#pragma unroll
    for (int u = 0; u < kQkvQ; ++u)
        if (tid + u * kQkvThreads < nq) put_q(tid + u * kQkvThreads, qv[u], gv[u]);
    for (int i = tid + kQkvQ * kQkvThreads; i < nq; i += kQkvThreads) put_q(i, qa4[i], qw4[i]);
    // kv row
    float sl = 0.f, sr = 0.f;
#pragma unroll
    for (int u = 0; u < kQkvK; ++u) {
        const int j = tid + u * kQkvThreads;
        if (j < R) {
            const float v = rf * ((ka[u] + kb[u]) + kc[u]);
            kvs[j] = v;
            kv_f32[(size_t)t * R + j] = v;
            if (j < L) sl += v * v;
            else sr += v * v;
        }
    }
    sl = block_sum(sl, redf);   // its barriers also publish kvs
    sr = block_sum(sr, redf);
    const float tau_l = kFixTau * sqrtf(sl / L), tau_r = kFixTau * sqrtf(sr / d.dr);
#pragma unroll
    for (int u = 0; u < kQkvK; ++u) {
        const int j = tid + u * kQkvThreads;
        if (j < R && kv_flag(kvs, j, L, tau_l, tau_r, cs[u], sn[u])) {
            const int k = atomicAdd(flag_count, 1);
            if (k < d.T * R) flag_list[k] = t * R + j;
        }
    }
}

// Exact fp64 dots of the flagged elements, split over 16-row slices of wkv_a:
//   fix[t, j] += sum_{k in slice} (x[t, k] gamma[k]) wkv_a[k, j]   (fix zeroed by the prep kernel)
// The hidden size is a multiple of 16, so every slice is full. The slice is
// staged with all of a thread's loads in flight at once (one memory latency,
// not one per load); each flagged element then costs two 16-byte loads of x.
constexpr int kFixRows = 16;
constexpr int kFixThreads = 128;
constexpr int kFixMaxR = 576;                                            // widest supported kv row
constexpr int kFixVecs = (kFixRows * kFixMaxR / 8 + kFixThreads - 1) / kFixThreads;   // uint4 per thread

__global__ void __launch_bounds__(kFixThreads)
k_kv_fix(const bf16* __restrict__ x, const float* __restrict__ gamma_in, const bf16* __restrict__ wkv_a, Dims d,
         const int32_t* __restrict__ flag_count, const int32_t* __restrict__ flag_list, double* __restrict__ fix) {
    griddep_launch();   // dependents may start; they wait for this kernel
    griddep_wait();     // the previous kernel of the stream has completed
    __shared__ __align__(16) bf16 wsm[kFixRows * kFixMaxR];
    __shared__ double gsm[kFixRows];
    const int R = d.R();
    const int k0 = blockIdx.x * kFixRows;
    const int n = min(*flag_count, d.T * R);
    if (n == 0) return;
    const int nv = kFixRows * R / 8;
    const uint4* src = reinterpret_cast<const uint4*>(wkv_a + (size_t)k0 * R);
    uint4 v[kFixVecs];
#pragma unroll
    for (int u = 0; u < kFixVecs; ++u) {
        const int i = threadIdx.x + u * kFixThreads;
        if (i < nv) v[u] = src[i];
    }
#pragma unroll
    for (int u = 0; u < kFixVecs; ++u) {
        const int i = threadIdx.x + u * kFixThreads;
        if (i < nv) reinterpret_cast<uint4*>(wsm)[i] = v[u];
    }
    if (threadIdx.x < kFixRows) gsm[threadIdx.x] = (double)gamma_in[k0 + threadIdx.x];
    __syncthreads();
    for (int f = threadIdx.x; f < n; f += blockDim.x) {
        const int e = flag_list[f];
        const int t = e / R, j = e - t * R;
        const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)t * d.H + k0);
        const uint4 xa = xr[0], xb = xr[1];
        const bf16* xa_h = reinterpret_cast<const bf16*>(&xa);
        const bf16* xb_h = reinterpret_cast<const bf16*>(&xb);
        double acc = 0.0;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) acc = fma(bf2d(xa_h[kk]) * gsm[kk], bf2d(wsm[kk * R + j]), acc);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) acc = fma(bf2d(xb_h[kk]) * gsm[8 + kk], bf2d(wsm[(8 + kk) * R + j]), acc);
        atomicAdd(fix + e, acc);
    }
}

// Per token: the cache row. Flagged elements take r * fix (exact, fp64), the
// others the fp32 row; kv-latent RMSNorm over the latent part, RoPE on k_pe,
// one bf16 rounding, written at slot_mapping[t]. All of the token's loads are
// issued before the first reduction (one memory latency for the block).
constexpr int kRowThreads = 256;
constexpr int kRowK = 3;   // kv-row elements per thread (kv_row_dim <= 768)

__global__ void __launch_bounds__(kRowThreads)
k_kv_row(const float* __restrict__ kv_f32, const double* __restrict__ fix, const double* __restrict__ r_in,
         const float* __restrict__ kv_norm_w, const float* __restrict__ cos_t, const float* __restrict__ sin_t,
         const int32_t* __restrict__ slot_mapping, Dims d, float eps, bf16* __restrict__ kv_cache,
         int32_t* __restrict__ status) {
    griddep_launch();   // dependents may start; they wait for this kernel
    griddep_wait();     // the previous kernel of the stream has completed
    __shared__ float redf[32];
    __shared__ double redd[32];
    extern __shared__ __align__(16) unsigned char sm2[];
    const int t = blockIdx.x, tid = threadIdx.x;
    const int R = d.R(), L = d.L, half = d.dr / 2;
    float* kvf = reinterpret_cast<float*>(sm2);                                      // [R]
    double* kvd = reinterpret_cast<double*>(sm2 + sizeof(float) * ((R + 1) & ~1));  // [R]
    float v[kRowK], w[kRowK], cs[kRowK], sn[kRowK];
    double fx[kRowK];
#pragma unroll
    for (int u = 0; u < kRowK; ++u) {
        const int j = tid + u * kRowThreads;
        cs[u] = 0.f;
        sn[u] = 0.f;
        if (j < R) {
            v[u] = kv_f32[(size_t)t * R + j];
            fx[u] = fix[(size_t)t * R + j];
            w[u] = j < L ? kv_norm_w[j] : 0.f;
            if (j >= L) {
                const int pi = (j - L) >> 1;
                cs[u] = cos_t[(size_t)t * half + pi];
                sn[u] = sin_t[(size_t)t * half + pi];
            }
        }
    }
    const double r = r_in[t];
    const int32_t slot = slot_mapping[t];
    float sl = 0.f, sr = 0.f;
#pragma unroll
    for (int u = 0; u < kRowK; ++u) {
        const int j = tid + u * kRowThreads;
        if (j < R) {
            kvf[j] = v[u];
            if (j < L) sl += v[u] * v[u];
            else sr += v[u] * v[u];
        }
    }
    sl = block_sum(sl, redf);   // its barriers also publish kvf
    sr = block_sum(sr, redf);
    const float tau_l = kFixTau * sqrtf(sl / L), tau_r = kFixTau * sqrtf(sr / d.dr);
    bool flg[kRowK];
#pragma unroll
    for (int u = 0; u < kRowK; ++u) {
        const int j = tid + u * kRowThreads;
        flg[u] = j < R && kv_flag(kvf, j, L, tau_l, tau_r, cs[u], sn[u]);
    }
    __syncthreads();   // every flag decision has read the fp32 row
#pragma unroll
    for (int u = 0; u < kRowK; ++u) {
        const int j = tid + u * kRowThreads;
        if (flg[u]) {
            kvd[j] = fx[u] * r;
            kvf[j] = (float)kvd[j];
        }
    }
    if (slot < 0 || slot >= d.n_rows()) {   // uniform over the block
        if (tid == 0) set_status(status, MLA_DEV_BAD_SLOT);
        return;
    }
    double ssk = 0.0;
#pragma unroll
    for (int u = 0; u < kRowK; ++u) {
        const int j = tid + u * kRowThreads;
        if (j < L) ssk += (double)kvf[j] * (double)kvf[j];
    }
    ssk = block_sum(ssk, redd);   // its barriers also publish the fixed elements
    const double rk = 1.0 / sqrt(ssk / L + (double)eps);
    const float rkf = (float)rk;
    bf16* row = kv_cache + (size_t)slot * R;
#pragma unroll
    for (int u = 0; u < kRowK; ++u) {
        const int j = tid + u * kRowThreads;
        if (j < L) {
            row[j] = flg[u] ? __double2bfloat16(kvd[j] * (double)w[u] * rk) : __float2bfloat16_rn(kvf[j] * w[u] * rkf);
        } else if (j < R) {
            // RoPE: element j of the pair (base, base + 1); both elements share the pair's flag
            const int base = L + ((j - L) & ~1);
            const bool odd = ((j - L) & 1) != 0;
            const float c = cs[u], s = sn[u];
            if (flg[u]) {
                const double a = kvd[base], b = kvd[base + 1];
                row[j] = __double2bfloat16(odd ? a * s + b * c : a * c - b * s);
            } else {
                const float a = kvf[base], b = kvf[base + 1];
                row[j] = __float2bfloat16_rn(odd ? a * s + b * c : a * c - b * s);
            }
        }
    }
}

// out = bf16(in), eight elements per thread (n a multiple of 8; both pointers 16-byte aligned).
__global__ void __launch_bounds__(256) k_f32_to_bf16(const float* __restrict__ in, bf16* __restrict__ out, size_t n) {
    griddep_launch();   // dependents may start; they wait for this kernel
    griddep_wait();     // the previous kernel of the stream has completed
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n / 8; i += (size_t)gridDim.x * blockDim.x) {
        const float4 a = reinterpret_cast<const float4*>(in)[2 * i], b = reinterpret_cast<const float4*>(in)[2 * i + 1];
        const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 pr = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
            w[e] = *reinterpret_cast<const uint32_t*>(&pr);
        }
        reinterpret_cast<uint4*>(out)[i] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

}  // namespace

cudaError_t launch_fold_prep_tc(const bf16* x, const float* gamma, const Dims& d, bf16* xg3, float* qacc,
                                float* kacc, float* y32, double* fix, int32_t* flag_count, cudaStream_t s) {
    return launch_pdl(k_fold_prep_tc, dim3(d.T * kPrepSplit), dim3(256), 0, s, x, gamma, d, xg3, qacc, kacc, y32,
                      fix, flag_count);
}

cudaError_t launch_step_start(const int32_t* gather_indices, const int32_t* block_table, const int32_t* positions,
                              int32_t* rows, int32_t* n_valid, int32_t* status, const bf16* x, const float* gamma,
                              const Dims& d, bf16* xg3, float* qacc, float* kacc, float* y32, double* fix,
                              int32_t* flag_count, cudaStream_t s) {
    return launch_pdl(k_step_start, dim3(2 * d.T), dim3(kStartThreads), 0, s, gather_indices, block_table, positions,
                      rows, n_valid, status, x, gamma, d, xg3, qacc, kacc, y32, fix, flag_count);
}

cudaError_t launch_fold_q_kv(const bf16* x, const float* qacc, const float* kacc, const float* q_norm_w,
                             const float* cos_t, const float* sin_t, const Dims& d, float eps, double* r_in,
                             bf16* q_an, float* kv_f32, int32_t* flag_count, int32_t* flag_list,
                             const CorePlanArgs* plan, cudaStream_t s) {
    const int R = d.R();
    if (R > kQkvK * kQkvThreads) return cudaErrorInvalidValue;
    const CorePlanArgs pl = plan ? *plan : CorePlanArgs{};
    return launch_pdl(k_fold_q_kv, dim3(d.T + (plan ? 1 : 0)), dim3(kQkvThreads), sizeof(float) * R, s, x, qacc,
                      kacc, q_norm_w, cos_t, sin_t, d, eps, r_in, q_an, kv_f32, flag_count, flag_list, pl);
}

cudaError_t launch_kv_fix_row(const bf16* x, const float* gamma_in, const bf16* wkv_a, const float* kv_norm_w,
                              const float* cos_t, const float* sin_t, const int32_t* slot_mapping, const Dims& d,
                              float eps, const double* r_in, const float* kv_f32, const int32_t* flag_count,
                              const int32_t* flag_list, double* fix, bf16* kv_cache, int32_t* status,
                              cudaStream_t s) {
    const int R = d.R();
    if (R > kFixMaxR || d.H % kFixRows || R > kRowK * kRowThreads) return cudaErrorInvalidValue;
    cudaError_t e = launch_pdl(k_kv_fix, dim3(d.H / kFixRows), dim3(kFixThreads), 0, s, x, gamma_in, wkv_a, d,
                               flag_count, flag_list, fix);
    if (e != cudaSuccess) return e;
    const size_t smem = sizeof(float) * ((R + 1) & ~1) + sizeof(double) * R;
    return launch_pdl(k_kv_row, dim3(d.T), dim3(kRowThreads), smem, s, kv_f32, fix, r_in, kv_norm_w, cos_t, sin_t,
                      slot_mapping, d, eps, kv_cache, status);
}

cudaError_t launch_f32_to_bf16(const float* in, bf16* out, size_t n, cudaStream_t s) {
    if (n % 8) return cudaErrorInvalidValue;
    const size_t n8 = n / 8, block = 256;
    const int grid = (int)((n8 + block - 1) / block < 2368 ? (n8 + block - 1) / block : 2368);
    return launch_pdl(k_f32_to_bf16, dim3(grid > 0 ? grid : 1), dim3(block), 0, s, in, out, n);
}

}  // namespace mla
