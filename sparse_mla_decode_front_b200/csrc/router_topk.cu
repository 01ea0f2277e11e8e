// Fused RMSNorm + router top-K of a MoE decoder layer (page "RMSNorm Router Top-K
// A2AV Kernel API Reference": :param hidden_states, gamma, router_weights,
// router_bias, eps, top_k, router_act_fn; :return norm, top-K indices, masked
// affinities; Notes: top-K on raw logits, activation on the selected experts).
//
// RMSNorm(x) W = r ((x * gamma) W) with r = 1/sqrt(mean(x^2) + eps), so the router
// projection runs on x * gamma and the per-token r is applied to the logit sums.
// x * gamma (two bf16 factors) is exact in fp32 and splits exactly into hi + lo
// bf16 slices; the tensor-core GEMM runs on both (2T token rows), so the logits
// carry only fp32 accumulation error and the top-K follows the exact logits except
// between logits closer than that error.
//
// Three launches: prep (one block per token: RMS, the bf16 norm row, the slices,
// zeroed sums), the projection (k_gemm_tc, split-K, fp32 reductions), finish (one
// block per token: logits, top-K by warp arg-max rounds, activation, masked
// affinities).
#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace mla {

namespace {

constexpr int kRouterThreads = 256;
constexpr int kRouterMaxExperts = 1024;   // 32 logits per lane in the top-K warp

// Per token (one block): the RMS scale r (fp64 sum of squares), the normalised row
// (x gamma) r with one bf16 rounding, x * gamma as hi + lo bf16 slices, zeroed logit
// sums. Every load of the row is issued before the reduction (kPrepVecs 16-byte
// vectors of x and gamma per thread; wider rows take a second round).
constexpr int kPrepVecs = 4;   // hidden <= 8192 in one round

__global__ void __launch_bounds__(kRouterThreads)
k_router_prep(const bf16* __restrict__ x, const bf16* __restrict__ gamma, int T, int H, int E, float eps,
              bf16* __restrict__ norm_out, bf16* __restrict__ xg2, float* __restrict__ acc, float* __restrict__ r_out) {
    griddep_launch();   // dependents may start; they wait for this kernel
    griddep_wait();     // the previous kernel of the stream has completed
    __shared__ double redd[32];
    const int t = blockIdx.x, nv = H / 8;
    const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)t * H);
    const uint4* gr = reinterpret_cast<const uint4*>(gamma);
    uint4 xv[kPrepVecs], gv[kPrepVecs];
#pragma unroll
    for (int u = 0; u < kPrepVecs; ++u) {
        const int v = threadIdx.x + u * kRouterThreads;
        if (v < nv) {
            xv[u] = xr[v];
            gv[u] = gr[v];
        }
    }
    double ss = 0.0;
    auto add_sq = [&](const uint4& w) {
        const bf16* b = reinterpret_cast<const bf16*>(&w);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const double f = bf2d(b[e]);
            ss += f * f;
        }
    };
#pragma unroll
    for (int u = 0; u < kPrepVecs; ++u)
        if (threadIdx.x + u * kRouterThreads < nv) add_sq(xv[u]);
    for (int v = threadIdx.x + kPrepVecs * kRouterThreads; v < nv; v += kRouterThreads) add_sq(xr[v]);
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i = threadIdx.x; i < E / 4; i += blockDim.x) {   // (stores need no wait)
        reinterpret_cast<float4*>(acc + (size_t)t * E)[i] = z;
        reinterpret_cast<float4*>(acc + (size_t)(T + t) * E)[i] = z;
    }
    ss = block_sum(ss, redd);
    const double r = 1.0 / sqrt(ss / H + (double)eps);
    if (threadIdx.x == 0) r_out[t] = (float)r;
    uint4* nr = reinterpret_cast<uint4*>(norm_out + (size_t)t * H);
    uint4* hi = reinterpret_cast<uint4*>(xg2 + (size_t)t * H);
    uint4* lo = reinterpret_cast<uint4*>(xg2 + (size_t)(T + t) * H);
    auto emit = [&](int v, const uint4& xw, const uint4& gw) {
        const bf16* xb = reinterpret_cast<const bf16*>(&xw);
        const bf16* gb = reinterpret_cast<const bf16*>(&gw);
        uint4 on, oh, ol;
        bf16* pn = reinterpret_cast<bf16*>(&on);
        bf16* ph = reinterpret_cast<bf16*>(&oh);
        bf16* pl = reinterpret_cast<bf16*>(&ol);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float p = bf2f(xb[e]) * bf2f(gb[e]);        // exact: 8 x 8 significant bits
            pn[e] = __double2bfloat16((double)p * r);          // the norm, one rounding
            const bf16 a = __float2bfloat16_rn(p);
            ph[e] = a;
            pl[e] = __float2bfloat16_rn(p - __bfloat162float(a));   // exact remainder
        }
        nr[v] = on;
        hi[v] = oh;
        lo[v] = ol;
    };
#pragma unroll
    for (int u = 0; u < kPrepVecs; ++u) {
        const int v = threadIdx.x + u * kRouterThreads;
        if (v < nv) emit(v, xv[u], gv[u]);
    }
    for (int v = threadIdx.x + kPrepVecs * kRouterThreads; v < nv; v += kRouterThreads) emit(v, xr[v], gr[v]);
}

// (value, index) order of the top-K: larger value first, equal values by smaller index.
__device__ __forceinline__ bool ahead(float v, int e, float bv, int be) { return v > bv || (v == bv && e < be); }

// Per token (one block): logits = r (hi + lo sums) + bias, top-K on the raw logits
// by K rounds of a warp arg-max, the activation of the selected, masked affinities.
// kC: logits per lane of the top-K warp (E <= 32 kC).
template <int kC>
__global__ void __launch_bounds__(kRouterThreads)
k_router_finish(const bf16* __restrict__ bias, const float* __restrict__ acc, const float* __restrict__ r_in, int T,
                int E, int K, int act, int32_t* __restrict__ idx_out, bf16* __restrict__ aff_out) {
    griddep_launch();   // dependents may start; they wait for this kernel
    griddep_wait();     // the previous kernel of the stream has completed
    __shared__ float lg[kRouterMaxExperts];
    __shared__ float af[kRouterMaxExperts];
    const int t = blockIdx.x, lane = threadIdx.x & 31;
    const float rf = r_in[t];
    // raw logits
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        lg[e] = rf * (acc[(size_t)t * E + e] + acc[(size_t)(T + t) * E + e]) + (bias ? bf2f(bias[e]) : 0.f);
        af[e] = 0.f;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        // top-K on the raw logits: K rounds of a warp arg-max over the untaken experts
        // (lane l holds experts l, l + 32, ...), then the activation of the selected
        float v[kC];
#pragma unroll
        for (int i = 0; i < kC; ++i) {
            const int e = lane + 32 * i;
            v[i] = e < E ? lg[e] : -INFINITY;
        }
        uint32_t taken = 0;
        float sel_v = -INFINITY;
        int sel_e = -1;   // lanes past the selected count keep -1
        for (int k = 0; k < K; ++k) {
            float bv = -INFINITY;
            int be = 0x7fffffff;
#pragma unroll
            for (int i = 0; i < kC; ++i) {
                const int e = lane + 32 * i;
                if (e < E && !((taken >> i) & 1u) && ahead(v[i], e, bv, be)) {
                    bv = v[i];
                    be = e;
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                const int oe = __shfl_xor_sync(0xffffffffu, be, o);
                if (ahead(ov, oe, bv, be)) {
                    bv = ov;
                    be = oe;
                }
            }
            if (be >= E) break;   // no candidate left (non-finite logits): the rest stays unselected
            if (lane == (be & 31)) taken |= 1u << (be >> 5);
            if (lane == k) {
                sel_v = bv;
                sel_e = be;
            }
        }
        // lane k < K holds the k-th selected expert (largest first)
        float a = 0.f;
        if (act == 1) {   // softmax over the K selected logits
            const float m = __shfl_sync(0xffffffffu, sel_v, 0);
            const float ex = lane < K ? expf(sel_v - m) : 0.f;
            float sum = ex;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            a = ex / sum;
        } else {          // sigmoid of each selected logit
            a = 1.f / (1.f + expf(-sel_v));
        }
        if (lane < K) {
            if (sel_e >= 0) af[sel_e] = a;
            idx_out[(size_t)t * K + lane] = sel_e;
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) aff_out[(size_t)t * E + e] = __float2bfloat16_rn(af[e]);
}

}  // namespace

bool router_dims_ok(int T, int H, int E, int K) {
    return T >= 0 && H >= 16 && H % 16 == 0 && E >= 64 && E <= kRouterMaxExperts && E % 16 == 0 && K >= 1 &&
           K <= E && K <= 32;
}

size_t router_workspace_bytes(int T, int H, int E) {
    auto up = [](size_t v) { return (v + 255) / 256 * 256; };
    return up(256) + up(sizeof(bf16) * 2 * (size_t)T * H) + up(sizeof(float) * 2 * (size_t)T * E) +
           up(sizeof(float) * (size_t)T);
}

cudaError_t launch_router_topk(const bf16* x, const bf16* gamma, const bf16* w, const bf16* bias, int T, int H, int E,
                               int K, float eps, int act, bf16* norm_out, int32_t* idx_out, bf16* aff_out,
                               void* workspace, cudaStream_t s, int* n_launches) {
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    auto up = [](size_t v) { return (v + 255) / 256 * 256; };
    int32_t* status = reinterpret_cast<int32_t*>(ws);
    bf16* xg2 = reinterpret_cast<bf16*>(ws + up(256));
    float* acc = reinterpret_cast<float*>(ws + up(256) + up(sizeof(bf16) * 2 * (size_t)T * H));
    float* r = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(acc) + up(sizeof(float) * 2 * (size_t)T * E));
    cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int32_t), s);
    if (e != cudaSuccess) return e;
    e = launch_pdl(k_router_prep, dim3(T), dim3(kRouterThreads), 0, s, x, gamma, T, H, E, eps, norm_out, xg2, acc, r);
    if (e != cudaSuccess) return e;
    GemmSpec g{};
    g.a = w; g.a_rows = H; g.a_cols = E; g.a_mn_major = true;
    g.b = xg2; g.b_cols = H; g.b_ld = H; g.b_rows_alloc = 2 * T; g.n_rows = 2 * T;
    g.m_total = E; g.k_total = H; g.groups = 1; g.accumulate = 1; g.status = status;
    // A few tiles over a long K: split-K over about half the SMs, each slice reducing one tile
    // (stream-K over all SMs would reduce a whole tile per CTA for one or two K blocks each).
    const int tiles = ((E + 127) / 128) * ((2 * T + gemm_bn_for(2 * T) - 1) / gemm_bn_for(2 * T));
    const int k_blocks = (H + 63) / 64;
    g.splits = std::max(1, std::min(k_blocks, 64 / std::max(1, tiles)));
    e = launch_gemm_reduce_f32(g, acc, E, 0, s);
    if (e != cudaSuccess) return e;
    *n_launches = 3;
    auto fin = E <= 64 ? k_router_finish<2> : E <= 128 ? k_router_finish<4> : E <= 256 ? k_router_finish<8>
             : E <= 512 ? k_router_finish<16> : k_router_finish<32>;
    return launch_pdl(fin, dim3(T), dim3(kRouterThreads), 0, s, bias, acc, r, T, E, K, act, idx_out, aff_out);
}

}  // namespace mla
