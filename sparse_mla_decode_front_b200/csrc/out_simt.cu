// Value absorption on CUDA cores (page "MLA Attention Block Gather Decode
// Kernel API Reference", :param out_absorb_w [n_heads, v_head_dim,
// kv_lora_rank] -- the value half of wkv_b, which maps a head's latent
// attention output back to its value width): o[t, h*dv + v] = out_absorb_w[h, v, :] . ctx[t, h, :].
#include "common.cuh"
#include "launch.h"

namespace mla {

namespace {

constexpr int kWarps = 8, kTok = 8;

__global__ void __launch_bounds__(kWarps * 32)
k_out_absorb_simt(const float* __restrict__ ctx, const bf16* __restrict__ out_absorb_w, Dims d,
                  float* __restrict__ o) {
    extern __shared__ float cs[];  // [kTok][L]
    const int hh = blockIdx.x, t0 = blockIdx.y * kTok;
    const int L = d.L;
    for (int e = threadIdx.x; e < kTok * L; e += blockDim.x) {
        const int i = e / L, t = t0 + i;
        cs[e] = t < d.T ? ctx[((size_t)t * d.h + hh) * L + e % L] : 0.f;
    }
    __syncthreads();
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bf16* B = out_absorb_w + (size_t)hh * d.dv * L;
    for (int v = w; v < d.dv; v += kWarps) {
        float acc[kTok];
#pragma unroll
        for (int i = 0; i < kTok; ++i) acc[i] = 0.f;
        for (int l = lane; l < L; l += 32) {
            const float b = bf2f(B[(size_t)v * L + l]);
#pragma unroll
            for (int i = 0; i < kTok; ++i) acc[i] = fmaf(b, cs[i * L + l], acc[i]);
        }
#pragma unroll
        for (int i = 0; i < kTok; ++i) {
            const float r = warp_sum(acc[i]);
            if (lane == 0 && t0 + i < d.T) o[(size_t)(t0 + i) * d.h * d.dv + (size_t)hh * d.dv + v] = r;
        }
    }
}

}  // namespace

cudaError_t launch_out_absorb_simt(const float* ctx, const bf16* out_absorb_w, const Dims& d, float* o,
                                   cudaStream_t s) {
    dim3 grid(d.h, (d.T + kTok - 1) / kTok);
    const size_t smem = sizeof(float) * kTok * d.L;
    k_out_absorb_simt<<<grid, kWarps * 32, smem, s>>>(ctx, out_absorb_w, d, o);
    return cudaGetLastError();
}

}  // namespace mla
