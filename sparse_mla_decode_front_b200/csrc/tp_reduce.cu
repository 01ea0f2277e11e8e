// Tensor parallelism over heads: the second half of the fused o-projection
// reduction. The page "MLA Attention Block Gather Decode Kernel API Reference"
// (introduction, :param o_proj_w) returns a rank's attention-block output; with the
// heads split over ranks the block output is the sum of the ranks' o-projection
// partials. The projection (k_gemm_tc with EpiReducePeers) has already reduced
// every tile into the accumulator of the rank owning its columns and counted its
// K blocks at every owner; this kernel, per rank:
//   1. waits (bounded) until all ranks' K blocks have arrived at its counter 0,
//   2. rounds its columns once to bf16, writes them into every rank's output and
//      zeroes its accumulator for the next step,
//   3. counts itself at every rank's counter 1 and waits (bounded) until every
//      rank's columns have arrived in its own output.
// Counters only grow; a step waits for epoch x (arrivals per step), compared
// modulo 2^32.
#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace mla {
namespace {

constexpr int kTpFinishThreads = 256;
constexpr int kTpFinishVecs = 2;       // 8-column groups in flight per thread
constexpr int kTpFinishMaxCtas = 128;  // CTAs of all the ranks a launch serves (co-resident)

// CTAs per rank: enough to cover the rank's columns in about one pass, at most
// kTpFinishMaxCtas / world. A function of the dims alone, so every rank agrees on it.
int tp_finish_ctas(int T, int H, int world) {
    const long long groups = (long long)T * (H / world) / 8;
    const long long want = (groups + kTpFinishThreads * kTpFinishVecs - 1) / (kTpFinishThreads * kTpFinishVecs);
    const int cap = kTpFinishMaxCtas / world;
    return (int)(want < 1 ? 1 : want > cap ? cap : want);
}

__device__ __forceinline__ uint32_t ld_acquire_sys(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Spin until *ctr has reached target (modulo 2^32), at most ptx::kWaitTimeoutNs.
__device__ bool wait_count_sys(const uint32_t* ctr, uint32_t target, int32_t* status) {
    const uint64_t t0 = ptx::globaltimer();
    while (true) {
        if ((int32_t)(ld_acquire_sys(ctr) - target) >= 0) return true;
        if (ptx::globaltimer() - t0 > ptx::kWaitTimeoutNs) {
            atomicOr(status, MLA_DEV_WAIT_TIMEOUT);
            return false;
        }
        __nanosleep(100);
    }
}

__global__ void __launch_bounds__(kTpFinishThreads) k_tp_finish(TpTable t, int rank0, int T, int H, int ctas,
                                                                uint32_t want_sums, uint32_t want_shards,
                                                                int32_t* status) {
    const int c = rank0 + (int)blockIdx.x / ctas;
    const int j = (int)blockIdx.x % ctas;
    const int shard = H / t.world;
    if (threadIdx.x == 0) wait_count_sys(t.flags[c], want_sums, status);
    __syncthreads();

    float* acc = t.acc[c];
    const long long n8 = (long long)T * shard / 8;   // shard % 32 == 0: 8-column groups stay in a row
    const long long stride = (long long)ctas * kTpFinishThreads;
    for (long long i0 = (long long)j * kTpFinishThreads * kTpFinishVecs + threadIdx.x; i0 < n8;
         i0 += stride * kTpFinishVecs) {
        float4 v[kTpFinishVecs][2];
#pragma unroll
        for (int u = 0; u < kTpFinishVecs; ++u) {   // all loads first (peers' sums live in L2 / HBM)
            const long long i = i0 + (long long)u * kTpFinishThreads;
            if (i < n8) {
                const float4* a = reinterpret_cast<const float4*>(acc + i * 8);
                v[u][0] = __ldcg(a);
                v[u][1] = __ldcg(a + 1);
            }
        }
#pragma unroll
        for (int u = 0; u < kTpFinishVecs; ++u) {
            const long long i = i0 + (long long)u * kTpFinishThreads;
            if (i >= n8) break;
            const long long e = i * 8;
            const int row = (int)(e / shard), col = (int)(e % shard);
            float4* a = reinterpret_cast<float4*>(acc + e);
            const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
            __stcg(a, z);
            __stcg(a + 1, z);
            uint4 packed;
            __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&packed);
            h[0] = __floats2bfloat162_rn(v[u][0].x, v[u][0].y);
            h[1] = __floats2bfloat162_rn(v[u][0].z, v[u][0].w);
            h[2] = __floats2bfloat162_rn(v[u][1].x, v[u][1].y);
            h[3] = __floats2bfloat162_rn(v[u][1].z, v[u][1].w);
            const size_t dst = (size_t)row * H + (size_t)c * shard + col;
            for (int r = 0; r < t.world; ++r) *reinterpret_cast<uint4*>(t.out[r] + dst) = packed;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence_system();   // the zeroes and the output stores, before the count
        for (int r = 0; r < t.world; ++r)
            asm volatile("red.relaxed.sys.global.add.u32 [%0], 1;" ::"l"(t.flags[r] + 1) : "memory");
        wait_count_sys(t.flags[c] + 1, want_shards, status);
    }
}

}  // namespace

cudaError_t launch_tp_finish(const TpTable& t, int rank0, int n_local, int T, int H, uint32_t epoch,
                             uint32_t units_per_rank, int32_t* status, cudaStream_t s) {
    if (t.world < 1 || t.world > kTpMaxRanks || n_local < 1 || rank0 < 0 || rank0 + n_local > t.world ||
        H % (32 * t.world) || T < 1)
        return cudaErrorInvalidValue;
    const int ctas = tp_finish_ctas(T, H, t.world);
    const uint32_t want_sums = epoch * (uint32_t)t.world * units_per_rank;
    const uint32_t want_shards = epoch * (uint32_t)t.world * (uint32_t)ctas;
    // Every CTA waits for the others' counts: a cooperative launch keeps them all resident.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(n_local * ctas);
    cfg.blockDim = dim3(kTpFinishThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_tp_finish, t, rank0, T, H, ctas, want_sums, want_shards, status);
}

}  // namespace mla
