// Sparse latent attention core on CUDA cores (page "MLA Attention Block
// Gather Decode Kernel API Reference": :param gather_indices, kv_cache,
// softmax_scale, out_absorb_w -- the latent part of each selected row is the
// value). One CTA per (token, group of 8 heads): every head of the group
// shares the gathered rows, staged once in shared memory per chunk of keys.
// fp32 online softmax; ctx[t, h, :] = sum_j softmax(s)_j row_j[:L].
#include "common.cuh"
#include "launch.h"

namespace mla {

namespace {

constexpr int kHG = 8;        // heads per CTA (one warp each)
constexpr int kKC = 32;       // keys per chunk (one lane each for the scores)
constexpr int kMaxLat = 16;   // L / 32 accumulators per lane (L <= 512)

__global__ void __launch_bounds__(kHG * 32)
k_core_simt(const bf16* __restrict__ qtile, const bf16* __restrict__ kv_cache,
            const int32_t* __restrict__ rows, const int32_t* __restrict__ n_valid, Dims d,
            float scale, bf16* __restrict__ ctx) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int R = d.R(), L = d.L, RP = R + 8;
    float* qs = reinterpret_cast<float*>(smem);                       // [kHG][R]
    float* ps = qs + kHG * R;                                         // [kHG][kKC]
    bf16* rs = reinterpret_cast<bf16*>(ps + kHG * kKC);               // [kKC][RP]
    const int t = blockIdx.x, hg = blockIdx.y;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int head = hg * kHG + w;
    const bool active = head < d.h;
    for (int e = threadIdx.x; e < kHG * R; e += blockDim.x) {
        const int hh = hg * kHG + e / R;
        qs[e] = hh < d.h ? bf2f(qtile[((size_t)t * d.h + hh) * R + e % R]) : 0.f;
    }
    const int nv = n_valid[t];
    const int32_t* rw = rows + (size_t)t * d.P;
    const int nl = L / 32;
    float acc[kMaxLat];
#pragma unroll
    for (int i = 0; i < kMaxLat; ++i) acc[i] = 0.f;
    float m = -INFINITY, lsum = 0.f;
    const int vec_per_row = R / 8;
    for (int j0 = 0; j0 < nv; j0 += kKC) {
        const int n = min(kKC, nv - j0);
        __syncthreads();
        for (int e = threadIdx.x; e < n * vec_per_row; e += blockDim.x) {
            const int k = e / vec_per_row, c = e % vec_per_row;
            const uint4 v = reinterpret_cast<const uint4*>(kv_cache + (size_t)rw[j0 + k] * R)[c];
            *reinterpret_cast<uint4*>(rs + k * RP + c * 8) = v;
        }
        __syncthreads();
        if (active) {
            float s = -INFINITY;
            if (lane < n) {
                const float* q = qs + w * R;
                const bf16* r = rs + lane * RP;
                float a = 0.f;
                for (int c = 0; c < vec_per_row; ++c) {
                    const uint4 v = *reinterpret_cast<const uint4*>(r + c * 8);
                    const bf16* b = reinterpret_cast<const bf16*>(&v);
#pragma unroll
                    for (int u = 0; u < 8; ++u) a = fmaf(q[c * 8 + u], bf2f(b[u]), a);
                }
                s = a * scale;
            }
            const float m_new = fmaxf(m, warp_max(s));
            const float alpha = expf(m - m_new);
            const float p = (lane < n) ? expf(s - m_new) : 0.f;
            lsum = lsum * alpha + warp_sum(p);
            m = m_new;
            ps[w * kKC + lane] = p;
            __syncwarp();
#pragma unroll
            for (int i = 0; i < kMaxLat; ++i) {
                if (i >= nl) break;
                float a = acc[i] * alpha;
                for (int k = 0; k < n; ++k) a = fmaf(ps[w * kKC + k], bf2f(rs[k * RP + lane + 32 * i]), a);
                acc[i] = a;
            }
            __syncwarp();
        }
    }
    if (active) {
        const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
        bf16* o = ctx + ((size_t)t * d.h + head) * L;
#pragma unroll
        for (int i = 0; i < kMaxLat; ++i)
            if (i < nl) o[lane + 32 * i] = __float2bfloat16(acc[i] * inv);
    }
}

}  // namespace

size_t core_simt_smem(const Dims& d) {
    return sizeof(float) * (kHG * d.R() + kHG * kKC) + sizeof(bf16) * kKC * (d.R() + 8);
}

bool core_simt_supports(const Dims& d) { return d.R() % 8 == 0 && d.L % 32 == 0 && d.L <= 32 * kMaxLat; }

cudaError_t launch_core_simt(const bf16* qtile, const bf16* kv_cache, const int32_t* rows,
                             const int32_t* n_valid, const Dims& d, float scale, bf16* ctx,
                             cudaStream_t s) {
    const size_t smem = core_simt_smem(d);
    cudaError_t e = cudaFuncSetAttribute(k_core_simt, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(d.T, (d.h + kHG - 1) / kHG);
    k_core_simt<<<grid, kHG * 32, smem, s>>>(qtile, kv_cache, rows, n_valid, d, scale, ctx);
    return cudaGetLastError();
}

}  // namespace mla
