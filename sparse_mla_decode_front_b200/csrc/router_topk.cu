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
// One cooperative launch where the shapes allow (up to 256 experts, a slice of at
// most four 64-deep K blocks per CTA on the device's SMs; k_router_fused), three
// otherwise: prep (one block per token: RMS, the bf16 norm row, the slices,
// zeroed sums), the projection (k_gemm_tc, split-K, fp32 reductions), finish (one
// block per token: logits, top-K by warp arg-max rounds, activation, masked
// affinities).
#include <algorithm>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

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

// Warp 0 of a block, one token: top-K on the raw logits lg[0, E) by K rounds of a warp
// arg-max over the untaken experts (lane l holds experts l, l + 32, ...), the activation of
// the selected into af[] (zero elsewhere, set by the caller), their indices (largest first)
// into idx_row[0, K). kC: logits per lane (E <= 32 kC).
template <int kC>
__device__ __forceinline__ void select_topk(const float* lg, float* af, int E, int K, int act, int32_t* idx_row) {
    const int lane = threadIdx.x & 31;
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
        idx_row[lane] = sel_e;
    }
}

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
    const int t = blockIdx.x;
    const float rf = r_in[t];
    // raw logits
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        lg[e] = rf * (acc[(size_t)t * E + e] + acc[(size_t)(T + t) * E + e]) + (bias ? bf2f(bias[e]) : 0.f);
        af[e] = 0.f;
    }
    __syncthreads();
    if (threadIdx.x < 32) select_topk<kC>(lg, af, E, K, act, idx_out + (size_t)t * K);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) aff_out[(size_t)t * E + e] = __float2bfloat16_rn(af[e]);
}


// ---------------------------------------------------------------- single launch
// k_router_fused: CTA b = (K slice ks, expert group eg) of a grid of nK x nE CTAs, all
// resident (cooperative launch). Phase 1, per tile of 128 tokens: the slice of x by TMA in
// the 128-byte-swizzled K-major layout of the UMMA's A operand, turned in place into x *
// gamma as exact hi + lo bf16 tiles, the slice's [K x 64 experts] weights by TMA (MN-major
// B, loaded once), the
// partial logits D[128 tokens x 64 experts] = hi W + lo W in TMEM, written to part[ks];
// the slice's sums of x^2 per token (fp64) to ss[ks]. A grid barrier (bounded wait). Phase
// 2: CTA b finishes tokens b, b + G, ...: r = 1/sqrt(sum ss / H + eps), logits = r (sum over
// slices in slice order) + bias; the top-K by rank (each thread counts the experts ahead of
// its own: larger logit, or equal logit and smaller index, the order k_router_finish
// selects in), the activation of the selected, and the token's norm row (x gamma) r, bf16.
namespace rfused {
constexpr int kThreads = 256;
constexpr int BT = 128;                          // tokens per tile (UMMA M)
constexpr int EG = 64;                           // experts per CTA (UMMA N)
constexpr int kMaxKb = 4;                        // 64-deep K blocks per slice
constexpr int kMaxGroups = 4;                    // expert groups (E <= 256)
constexpr int kABytes = BT * 64 * 2;             // one K block of a token tile (16 KB)
constexpr int kWBytes = 64 * EG * 2;             // one K block of the group's weights (8 KB)
constexpr int kSmem = 2 * kMaxKb * kABytes + kMaxKb * kWBytes + 1024;
constexpr uint32_t kTmemCols = 64;
constexpr int kSizedSms = 148;                   // workspaces are sized for at most this many CTAs

// K slices and expert groups of the single launch with one CTA on each of `sms` SMs, or 0
// when a slice would not fit the shared-memory tiles (or E needs more than four groups).
int fused_grid_for(int H, int E, int sms, int* nK, int* nE) {
    const int ne = (E + EG - 1) / EG;
    const int nkb = (H + 63) / 64;
    sms = std::min(sms, kSizedSms);
    if (ne > kMaxGroups || sms < ne) return 0;
    const int nk = std::min(nkb, sms / ne);
    if ((nkb + nk - 1) / nk > kMaxKb) return 0;
    *nK = nk;
    *nE = ne;
    return nk * ne;
}

struct Params {
    const bf16* x;        // [T, H]
    const bf16* gamma;    // [H]
    const bf16* bias;     // [E] or null
    int T, H, E, K, act, nK, nE, nKB;
    float eps;
    float* part;          // [nK][T][nE * EG] partial logits
    double* ss;           // [nK][T] partial sums of x^2
    uint32_t* arrive;     // grid barrier count (zeroed by the call)
    int32_t* status;
    bf16* norm_out;       // [T, H]
    int32_t* idx_out;     // [T, K]
    bf16* aff_out;        // [T, E]
};

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// 1 / sqrt(sum_ks ss[ks][t] / H + eps) by warp 0 (fixed summation order); into *r.
__device__ __forceinline__ void token_scale(const Params& p, int t, double* r) {
    const int lane = threadIdx.x & 31;
    double a = 0.0;
    for (int ks = lane; ks < p.nK; ks += 32) a += __ldcg(p.ss + (size_t)ks * p.T + t);
    a = warp_sum(a);
    if (lane == 0) *r = 1.0 / sqrt(a / p.H + (double)p.eps);
}

__global__ void __launch_bounds__(kThreads, 1)
k_router_fused(const __grid_constant__ CUtensorMap tma_w, const __grid_constant__ CUtensorMap tma_x, Params p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t w_full, x_full, d_full;
    __shared__ uint32_t tmem_slot;
    __shared__ __align__(16) float lg[kMaxGroups * EG];   // read as float4 by the ranking
    __shared__ __align__(16) float cand_v[kMaxGroups * EG / 32 * 32];   // per warp: its K best
    __shared__ int cand_e[kMaxGroups * EG / 32 * 32];
    __shared__ int n_cand[kThreads / 32];
    __shared__ float bias_sh[kMaxGroups * EG];
    __shared__ float sel_v[32];
    __shared__ uint4 gsh[kMaxKb * 8];   // gamma of the slice, 8-element chunks
    __shared__ double r_sh;
    __shared__ int go;
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char* hi = smem;
    unsigned char* lo = smem + kMaxKb * kABytes;   // the TMA lands x here; converted in place
    unsigned char* wsm = smem + 2 * kMaxKb * kABytes;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ks = blockIdx.x / p.nE, eg = blockIdx.x % p.nE;
    const int kb0 = ks * p.nKB / p.nK, nkb = (ks + 1) * p.nKB / p.nK - kb0;
    const int ep = p.nE * EG;
    const int ntt = (p.T + BT - 1) / BT;

    if (tid == 0) {
        ptx::mbar_init(&w_full, 1);
        ptx::mbar_init(&x_full, 1);
        ptx::mbar_init(&d_full, 1);
        ptx::fence_mbar_init();
        ptx::tma_prefetch_desc(&tma_w);
        ptx::tma_prefetch_desc(&tma_x);
        // the slice's weights and the first token tile's x (past H, E or T: zero)
        ptx::mbar_arrive_expect_tx(&w_full, nkb * kWBytes);
        for (int j = 0; j < nkb; ++j) ptx::tma_load_2d(wsm + j * kWBytes, &tma_w, &w_full, eg * EG, (kb0 + j) * 64);
        ptx::mbar_arrive_expect_tx(&x_full, nkb * kABytes);
        for (int j = 0; j < nkb; ++j) ptx::tma_load_2d(lo + j * kABytes, &tma_x, &x_full, (kb0 + j) * 64, 0);
    }
    if (tid < nkb * 8) {
        const int k = (kb0 + tid / 8) * 64 + (tid % 8) * 8;
        gsh[tid] = k < p.H ? *reinterpret_cast<const uint4*>(p.gamma + k) : make_uint4(0, 0, 0, 0);
    }
    for (int e = tid; e < p.E; e += kThreads) bias_sh[e] = p.bias ? bf2f(p.bias[e]) : 0.f;
    // the rows this CTA finishes after the grid barrier, and gamma, into L2 meanwhile
    for (int t = blockIdx.x; t < p.T; t += gridDim.x)
        for (int c = tid; c < p.H / 64; c += kThreads) {
            asm volatile("prefetch.global.L2 [%0];" ::"l"(p.x + (size_t)t * p.H + 64 * c));
            asm volatile("prefetch.global.L2 [%0];" ::"l"(p.gamma + 64 * c));
        }
    if (warp == 1) {
        ptx::tmem_alloc(&tmem_slot, kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = tmem_slot;
    bool ok = true;

    // ---- phase 1: partial logits of the slice, tile by tile
    const int r = tid >> 1, half = tid & 1;   // token row of the tile; half of the slice's chunks
    const int nch = nkb * 4;                  // 8-element chunks per thread
    for (int tt = 0; tt < ntt && ok; ++tt) {
        const int t = tt * BT + r;
        ok = __syncthreads_and(ptx::mbar_wait(&x_full, tt & 1, p.status));
        if (!ok) break;
        // x * gamma -> hi + lo bf16, in place: hi = x gamma rounded once (packed bf16 multiply),
        // lo = x gamma - hi by a fused multiply-add, exact (the product of two bf16 values has at
        // most 16 significant bits, hi holds the top 8); x^2 summed in fp32 (two accumulators)
        float ssa = 0.f, ssb = 0.f;
#pragma unroll
        for (int u = 0; u < kMaxKb * 4; ++u) {
            if (u >= nch) break;
            const int c = half * nch + u;   // chunk of the slice: block c / 8, 16-byte column group c % 8
            const int off = (c / 8) * kABytes + (r >> 3) * 1024 + (r & 7) * 128 + (((c % 8) ^ (r & 7)) << 4);
            const uint4 xw = *reinterpret_cast<const uint4*>(lo + off);
            const uint4 gw = gsh[c];
            const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&xw);
            const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gw);
            uint32_t wh[4], wl[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const __nv_bfloat162 h2 = __hmul2(x2[e], g2[e]);
                const __nv_bfloat162 l2 = __hfma2(x2[e], g2[e], __hneg2(h2));
                wh[e] = *reinterpret_cast<const uint32_t*>(&h2);
                wl[e] = *reinterpret_cast<const uint32_t*>(&l2);
                const float2 xf = __bfloat1622float2(x2[e]);
                ssa = fmaf(xf.x, xf.x, ssa);
                ssb = fmaf(xf.y, xf.y, ssb);
            }
            *reinterpret_cast<uint4*>(hi + off) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
            *reinterpret_cast<uint4*>(lo + off) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
        }
        double ssp = (double)ssa + (double)ssb;
        ssp += __shfl_xor_sync(0xffffffffu, ssp, 1);
        if (half == 0 && eg == 0 && t < p.T) p.ss[(size_t)ks * p.T + t] = ssp;
        ptx::fence_proxy_async_smem();   // generic stores -> the UMMA's reads (and the next x load)
        ptx::tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            if (tt == 0) ok = ptx::mbar_wait(&w_full, 0, p.status);
            if (ok) {
                ptx::tc_fence_after();
                const uint32_t idesc = ptx::idesc_bf16(BT, EG, false, true);
                const uint32_t ha = ptx::smem_u32(hi), la = ptx::smem_u32(lo), wa = ptx::smem_u32(wsm);
                // A (tokens) K-major: 128-byte rows, 8-row groups 1 KB apart, K=16 slice 32 B on.
                // B (weights) MN-major: one 64-column atom, 8-row K groups 1 KB apart, K=16 slice
                // 16 rows (2 KB) on.
                for (int j = 0; j < nkb; ++j)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        ptx::umma_bf16(tmem, ptx::sdesc_sw128(ha + j * kABytes + kk * 32, 16, 1024),
                                       ptx::sdesc_sw128(wa + j * kWBytes + kk * 2048, kWBytes, 1024), idesc,
                                       (j | kk) ? 1u : 0u);
                for (int j = 0; j < nkb; ++j)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        ptx::umma_bf16(tmem, ptx::sdesc_sw128(la + j * kABytes + kk * 32, 16, 1024),
                                       ptx::sdesc_sw128(wa + j * kWBytes + kk * 2048, kWBytes, 1024), idesc, 1u);
                ptx::umma_commit(&d_full);
            }
            go = ok ? 1 : 0;
        }
        __syncthreads();
        ok = go != 0;
        if (!ok) break;
        ok = __syncthreads_and(ptx::mbar_wait(&d_full, tt & 1, p.status));
        if (!ok) break;
        ptx::tc_fence_after();
        if (tid == 0 && tt + 1 < ntt) {   // the slices are free: the next tile's x
            ptx::mbar_arrive_expect_tx(&x_full, nkb * kABytes);
            for (int j = 0; j < nkb; ++j)
                ptx::tma_load_2d(lo + j * kABytes, &tma_x, &x_full, (kb0 + j) * 64, (tt + 1) * BT);
        }
        if (warp < 4) {
            // thread = token row of TMEM lane quarter `warp`; the group's 64 partial logits
            const int row = 32 * warp + lane, tr = tt * BT + row;
            const uint32_t t_row = tmem + ((uint32_t)(32 * warp) << 16);
            uint32_t v[4][16];
#pragma unroll
            for (int c = 0; c < 4; ++c) ptx::tmem_ld16_nowait(t_row + 16 * c, v[c]);
            ptx::tmem_wait_ld();
            if (tr < p.T) {
                float4* dst = reinterpret_cast<float4*>(p.part + ((size_t)ks * p.T + tr) * ep + eg * EG);
#pragma unroll
                for (int c = 0; c < 16; ++c)
                    dst[c] = make_float4(__uint_as_float(v[c / 4][4 * (c % 4)]), __uint_as_float(v[c / 4][4 * (c % 4) + 1]),
                                         __uint_as_float(v[c / 4][4 * (c % 4) + 2]),
                                         __uint_as_float(v[c / 4][4 * (c % 4) + 3]));
            }
        }
        ptx::tc_fence_before();
        __syncthreads();   // TMEM is reused by the next tile
    }

    // ---- grid barrier: every CTA's partials written (bounded wait)
    ok = __syncthreads_and(ok);
    if (ok) {
        if (tid == 0) {
            __threadfence();
            asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(p.arrive) : "memory");
            const uint64_t t0 = ptx::globaltimer();
            bool done = false;
            while (!(done = ld_acquire_gpu(p.arrive) >= gridDim.x)) {
                __nanosleep(32);
                if (ptx::globaltimer() - t0 > ptx::kWaitTimeoutNs) {
                    atomicOr(p.status, MLA_DEV_WAIT_TIMEOUT);
                    break;
                }
            }
            go = done ? 1 : 0;
        }
        __syncthreads();
        ok = go != 0;
    }

    // ---- phase 2: tokens blockIdx.x, + gridDim.x, ...: logits, top-K, activation, norm row
    // tpe threads per expert each sum a contiguous run of slices (in slice order), the runs
    // are added in order: a fixed summation order, all of a thread's loads in flight at once
    const int tpe = p.E <= 64 ? 4 : (p.E <= 128 ? 2 : 1);
    const int ex = tid / tpe, sub = tid % tpe;
    const int s0 = sub * p.nK / tpe, s1 = (sub + 1) * p.nK / tpe;
    const int cpr = p.H / 8;
    constexpr int kNormVecs = 4;   // norm-row chunks per thread held in registers (H <= 8192)
    for (int t = blockIdx.x; ok && t < p.T; t += gridDim.x) {
        // the norm row's inputs first: their latency overlaps everything below
        uint4 xw[kNormVecs], gw[kNormVecs];
#pragma unroll
        for (int u = 0; u < kNormVecs; ++u) {
            const int c = tid + u * kThreads;
            xw[u] = c < cpr ? *reinterpret_cast<const uint4*>(p.x + (size_t)t * p.H + 8 * c) : make_uint4(0, 0, 0, 0);
            gw[u] = c < cpr ? *reinterpret_cast<const uint4*>(p.gamma + 8 * c) : make_uint4(0, 0, 0, 0);
        }
        float part_sum = 0.f;
        if (ex < p.E) {
            const float* col = p.part + (size_t)t * ep + ex;
            for (int k0 = s0; k0 < s1; k0 += 40) {
                float v[40];
#pragma unroll
                for (int i = 0; i < 40; ++i) v[i] = k0 + i < s1 ? __ldcg(col + (size_t)(k0 + i) * p.T * ep) : 0.f;
                if (k0 == s0 && warp == 0) token_scale(p, t, &r_sh);   // its loads overlap these
#pragma unroll
                for (int i = 0; i < 40; ++i) part_sum += v[i];
            }
        } else if (warp == 0) {
            token_scale(p, t, &r_sh);
        }
        if (tid < p.K) p.idx_out[(size_t)t * p.K + tid] = -1;   // slots no finite logit fills
        lg[tid] = part_sum;   // [ex * tpe + sub]
        __syncthreads();
        const double rr = r_sh;
        float v = 0.f;
        if (tid < p.E) {
            float sum = 0.f;
            for (int i = 0; i < tpe; ++i) sum += lg[tid * tpe + i];
            v = (float)rr * sum + bias_sh[tid];
        }
        __syncthreads();
        lg[tid] = tid < p.E ? v : __int_as_float(0x7fc00000);   // past E: NaN, never ahead
        const int n_fin = __syncthreads_count(tid < p.E && !isnan(v));   // lg complete
        // Rank among the experts: larger logit first, equal logits by smaller index (NaN:
        // never). In two steps: the rank within the warp's 32 experts (an expert not among its
        // warp's K best is not among all K best), then among the warps' candidates.
        const bool fin = tid < p.E && !isnan(v);
        int wrank = 32;
        if (fin) {
            int c0 = 0, c1 = 0;
            const float4* l4 = reinterpret_cast<const float4*>(lg + 32 * warp);
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
                const float4 u = l4[j4];
                const int j = 32 * warp + 4 * j4;
                c0 += ((u.x > v) || (u.x == v && j < tid)) + ((u.y > v) || (u.y == v && j + 1 < tid));
                c1 += ((u.z > v) || (u.z == v && j + 2 < tid)) + ((u.w > v) || (u.w == v && j + 3 < tid));
            }
            wrank = c0 + c1;
        }
        const bool cand = fin && wrank < p.K;
        const uint32_t cb = __ballot_sync(0xffffffffu, cand);
        if (cand) {
            const int slot = 32 * warp + __popc(cb & ((1u << lane) - 1));
            cand_v[slot] = v;
            cand_e[slot] = tid;
        }
        if (lane == 0) n_cand[warp] = __popc(cb);
        __syncthreads();
        int rank = p.E;
        if (cand) {
            int c = 0;
            for (int w2 = 0; w2 < kThreads / 32; ++w2)
                for (int i = 0; i < n_cand[w2]; ++i) {
                    const float u = cand_v[32 * w2 + i];
                    const int j = cand_e[32 * w2 + i];
                    c += (u > v) || (u == v && j < tid);
                }
            rank = c;
        }
        if (rank < p.K) {
            sel_v[rank] = v;
            p.idx_out[(size_t)t * p.K + rank] = tid;
        }
        __syncthreads();
        // activation of the selected: sigmoid each, or softmax over the selected
        float a = 0.f;
        if (rank < p.K) {
            if (p.act == 1) {
                const int nsel = min(p.K, n_fin);
                const float m = sel_v[0];
                float den = 0.f;
                for (int k = 0; k < nsel; ++k) den += expf(sel_v[k] - m);
                a = expf(v - m) / den;
            } else {
                a = 1.f / (1.f + expf(-v));
            }
        }
        if (tid < p.E) p.aff_out[(size_t)t * p.E + tid] = __float2bfloat16_rn(a);
        // the norm row (x gamma) r, one rounding
#pragma unroll
        for (int u = 0; u < kNormVecs; ++u) {
            const int c = tid + u * kThreads;
            if (c >= cpr) break;
            const bf16* xb = reinterpret_cast<const bf16*>(&xw[u]);
            const bf16* gb = reinterpret_cast<const bf16*>(&gw[u]);
            uint4 on;
            bf16* pn = reinterpret_cast<bf16*>(&on);
#pragma unroll
            for (int e = 0; e < 8; ++e) pn[e] = __double2bfloat16((double)(bf2f(xb[e]) * bf2f(gb[e])) * rr);
            *reinterpret_cast<uint4*>(p.norm_out + (size_t)t * p.H + 8 * c) = on;
        }
        for (int c = tid + kNormVecs * kThreads; c < cpr; c += kThreads) {   // wider rows
            const uint4 xv = *reinterpret_cast<const uint4*>(p.x + (size_t)t * p.H + 8 * c);
            const uint4 gv = *reinterpret_cast<const uint4*>(p.gamma + 8 * c);
            const bf16* xb = reinterpret_cast<const bf16*>(&xv);
            const bf16* gb = reinterpret_cast<const bf16*>(&gv);
            uint4 on;
            bf16* pn = reinterpret_cast<bf16*>(&on);
#pragma unroll
            for (int e = 0; e < 8; ++e) pn[e] = __double2bfloat16((double)(bf2f(xb[e]) * bf2f(gb[e])) * rr);
            *reinterpret_cast<uint4*>(p.norm_out + (size_t)t * p.H + 8 * c) = on;
        }
        __syncthreads();   // lg, sel_v and r_sh are reused by the next token
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

// Grid of the single launch on this device, or 0 when the shapes need the three launches.
// Sets nK (K slices) and nE (expert groups).
int fused_grid(int H, int E, int* nK, int* nE) {
    int dev = 0, sms = 0, coop = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess || !coop)
        return 0;
    return fused_grid_for(H, E, sms, nK, nE);
}
}  // namespace rfused
}  // namespace

bool router_dims_ok(int T, int H, int E, int K) {
    return T >= 0 && H >= 16 && H % 16 == 0 && E >= 64 && E <= kRouterMaxExperts && E % 16 == 0 && K >= 1 &&
           K <= E && K <= 32;
}

int router_launches(int H, int E) {
    int nK = 0, nE = 0;
    return rfused::fused_grid(H, E, &nK, &nE) > 0 ? 1 : 3;
}

size_t router_workspace_bytes(int T, int H, int E) {
    auto up = [](size_t v) { return (v + 255) / 256 * 256; };
    const size_t three = up(256) + up(sizeof(bf16) * 2 * (size_t)T * H) + up(sizeof(float) * 2 * (size_t)T * E) +
                         up(sizeof(float) * (size_t)T);
    int nK = 0, nE = 0;
    if (!rfused::fused_grid_for(H, E, rfused::kSizedSms, &nK, &nE)) return three;
    const size_t one = up(256) + up(sizeof(float) * (size_t)nK * T * nE * rfused::EG) + up(sizeof(double) * (size_t)nK * T);
    return std::max(three, one);
}

cudaError_t launch_router_topk(const bf16* x, const bf16* gamma, const bf16* w, const bf16* bias, int T, int H, int E,
                               int K, float eps, int act, bf16* norm_out, int32_t* idx_out, bf16* aff_out,
                               void* workspace, cudaStream_t s, int* n_launches) {
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    auto up = [](size_t v) { return (v + 255) / 256 * 256; };
    int32_t* status = reinterpret_cast<int32_t*>(ws);
    int nK = 0, nE = 0;
    const int G = rfused::fused_grid(H, E, &nK, &nE);
    if (G > 0) {
        // one cooperative launch; the status word and the grid barrier's count start at zero
        cudaError_t e = cudaMemsetAsync(ws, 0, 8, s);
        if (e != cudaSuccess) return e;
        CUtensorMap tw, tx;
        // router_weights [H, E]: boxes of 64 K rows x 64 experts; hidden [T, H]: boxes of
        // 128 tokens x 64 columns (past H, E or T: zero)
        if (!make_tma_2d(&tw, w, (uint64_t)E, (uint64_t)H, (uint64_t)E * 2, 64, 64) ||
            !make_tma_2d(&tx, x, (uint64_t)H, (uint64_t)T, (uint64_t)H * 2, 64, rfused::BT))
            return cudaErrorInvalidValue;
        rfused::Params p;
        p.x = x;
        p.gamma = gamma;
        p.bias = bias;
        p.T = T;
        p.H = H;
        p.E = E;
        p.K = K;
        p.act = act;
        p.nK = nK;
        p.nE = nE;
        p.nKB = (H + 63) / 64;
        p.eps = eps;
        p.part = reinterpret_cast<float*>(ws + up(256));
        p.ss = reinterpret_cast<double*>(ws + up(256) + up(sizeof(float) * (size_t)nK * T * nE * rfused::EG));
        p.arrive = reinterpret_cast<uint32_t*>(ws + 4);
        p.status = status;
        p.norm_out = norm_out;
        p.idx_out = idx_out;
        p.aff_out = aff_out;
        {
            constexpr int kMaxDevices = 64;
            static bool attr_set[kMaxDevices] = {};   // function attributes are per device
            int dev = 0;
            cudaGetDevice(&dev);
            if (dev < 0 || dev >= kMaxDevices || !attr_set[dev]) {
                e = cudaFuncSetAttribute(rfused::k_router_fused, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         rfused::kSmem);
                if (e != cudaSuccess) return e;
                if (dev >= 0 && dev < kMaxDevices) attr_set[dev] = true;
            }
        }
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(G);
        cfg.blockDim = dim3(rfused::kThreads);
        cfg.dynamicSmemBytes = rfused::kSmem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;   // every CTA resident: they meet at a grid barrier
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        *n_launches = 1;
        return cudaLaunchKernelEx(&cfg, rfused::k_router_fused, tw, tx, p);
    }
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
