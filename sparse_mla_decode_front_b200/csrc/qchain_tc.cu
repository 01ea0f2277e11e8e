// Query chain of the front-fold on tcgen05 (page "MLA Attention Block Gather
// Decode Kernel API Reference": :param wq_b, q_absorb_w, cos, sin; the two
// query tiles the block hands to its attention core).
//
// One CTA per (head h, tile of up to 128 tokens) runs both products of the
// head back to back, so its up-projection never leaves the SM:
//   q[t, :]     = q_an[t] . wq_b[:, h (dn + dr) .. (h + 1)(dn + dr))   fp32 in TMEM
//   q_pe        = rope(q[t, dn:])  -> bf16 -> query tile columns [L, L + dr)
//   q_nope      = bf16(q[t, :dn])  -> shared memory (A operand of the next product)
//   q_lat[t, :] = q_nope[t] . q_absorb_w[h]                           fp32 in TMEM
//               -> bf16 -> query tile columns [0, L)
// Both products have the token tile as the UMMA A operand (M = 128 tokens) and
// the head's weight slice as B (MN-major: the page's weights are [in, out]).
// The weight bytes stream through one ring of shared-memory stages: first the
// K blocks of wq_b's slice (with the matching K block of q_an), then the
// q_absorb_w slice in chunks of up to 256 output columns.
//
// Warps: 0 TMA producer, 1 UMMA issuer (allocates TMEM), 2-5 epilogue (TMEM
// lane quarter = warp % 4, one token row per thread). TMEM: the up-projection
// in columns [0, dn + dr); after the epilogue has read it out, the absorbed
// query in columns [0, L).
#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace mla {
namespace qchain {

constexpr int kThreads = 192;
constexpr int BT = 128;                      // tokens per CTA tile (UMMA M)
constexpr int BK = 64;                       // K per stage (one 128-byte swizzle atom of bf16)
constexpr int kABytes = BT * BK * 2;         // token tile of one K block
constexpr int kBoxBytes = 64 * BK * 2;       // one [64 K rows x 64 columns] weight box
constexpr int kMaxBoxes = 4;                 // weight boxes per stage (up to 256 columns)
constexpr int kStageBytes = kABytes + kMaxBoxes * kBoxBytes;   // 48 KB
constexpr int kStages = 4;
constexpr int kQnBytes = 2 * kABytes;        // q_nope A operand: up to 128 columns (two K blocks)
constexpr int kSmem = kStages * kStageBytes + kQnBytes + 1024;
constexpr int kMaxHalf = 32;                 // rope pairs per head (qk_rope_head_dim <= 64)

struct Params {
    int T, h, Lq, dn, dr, L, R;
    const float* cos_t;   // [T, dr / 2]
    const float* sin_t;
    bf16* qtile;          // [T, h, R]
    int32_t* status;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

__global__ void __launch_bounds__(kThreads, 1)
k_q_chain(const __grid_constant__ CUtensorMap tma_q, const __grid_constant__ CUtensorMap tma_wqb,
          const __grid_constant__ CUtensorMap tma_abs, Params p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    griddep_launch();
    __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages], d1_full, qn_ready, d2_full[2], mma_done;
    __shared__ uint32_t tmem_slot;
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char* qn = smem + kStages * kStageBytes;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int head = blockIdx.x % p.h, tt = blockIdx.x / p.h;
    const int qk = p.dn + p.dr;
    const int nb1 = (qk + 63) / 64;                 // weight boxes of an up-projection stage
    const int kb1 = (p.Lq + BK - 1) / BK;           // up-projection K blocks
    const int kb2 = (p.dn + BK - 1) / BK;           // absorption K blocks
    const int nch = (p.L + 255) / 256;              // absorption output chunks of <= 256 columns
    constexpr uint32_t kTmemCols = 512;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            ptx::mbar_init(&full_bar[i], 1);
            ptx::mbar_init(&empty_bar[i], 1);
        }
        ptx::mbar_init(&d1_full, 1);
        ptx::mbar_init(&qn_ready, 4);
        ptx::mbar_init(&d2_full[0], 1);
        ptx::mbar_init(&d2_full[1], 1);
        ptx::mbar_init(&mma_done, 1);
        ptx::fence_mbar_init();
        ptx::tma_prefetch_desc(&tma_q);
        ptx::tma_prefetch_desc(&tma_wqb);
        ptx::tma_prefetch_desc(&tma_abs);
    }
    if (warp == 1) {
        ptx::tmem_alloc(&tmem_slot, kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = tmem_slot;
    // The producer waits for the previous kernel only after it has started loading the first
    // stages' weight boxes (weights are never written by the block's kernels); every other
    // warp waits here, before its first access to memory another kernel writes.
    if (warp != 0) griddep_wait();

    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer: up-projection stages, then absorption chunks
        const uint64_t pol = ptx::policy_evict_first();   // weights are read once
        int stage = 0, n_issued = 0;
        uint32_t ph = 0;
        bool ok = true;
        auto load_w = [&](int kb, int st_i) {   // the stage's wq_b boxes; its barrier expects A too
            unsigned char* st = smem + st_i * kStageBytes;
            ptx::mbar_arrive_expect_tx(&full_bar[st_i], kABytes + nb1 * kBoxBytes);
            for (int bx = 0; bx < nb1; ++bx)
                ptx::tma_load_2d_hint(st + kABytes + bx * kBoxBytes, &tma_wqb, &full_bar[st_i], head * qk + 64 * bx,
                                      kb * BK, pol);
        };
        const int n_pre = kb1 < kStages ? kb1 : kStages;   // all stages are free at first
        for (int kb = 0; kb < n_pre; ++kb) load_w(kb, kb);
        griddep_wait();   // the token tiles (q_an) are the previous kernel's output
        for (int kb = 0; ok && kb < kb1; ++kb) {
            if (kb >= n_pre) {
                if (!(ok = ptx::mbar_wait(&empty_bar[stage], ph ^ 1, p.status))) break;
                load_w(kb, stage);
            }
            ptx::tma_load_2d(smem + stage * kStageBytes, &tma_q, &full_bar[stage], kb * BK, tt * BT);
            ++n_issued;
            if (++stage == kStages) { stage = 0; ph ^= 1; }
        }
        for (int n = 0; ok && n < nch; ++n)
            for (int k2 = 0; ok && k2 < kb2; ++k2) {
                if (!(ok = ptx::mbar_wait(&empty_bar[stage], ph ^ 1, p.status))) break;
                unsigned char* st = smem + stage * kStageBytes;
                const int nbox = (min(p.L, 256 * (n + 1)) - 256 * n) / 64;
                ptx::mbar_arrive_expect_tx(&full_bar[stage], nbox * kBoxBytes);
                for (int i = 0; i < nbox; ++i)
                    ptx::tma_load_2d_hint(st + i * kBoxBytes, &tma_abs, &full_bar[stage], 256 * n + 64 * i,
                                          head * p.dn + k2 * BK, pol);
                ++n_issued;
                if (++stage == kStages) { stage = 0; ph ^= 1; }
            }
        // every load issued lands before shared memory is released
        for (int i = 0; i < kStages && i < n_issued; ++i) {
            if (--stage < 0) { stage = kStages - 1; ph ^= 1; }
            ptx::mbar_wait(&full_bar[stage], ph, nullptr);
        }
    } else if (warp == 1 && lane == 0) {
        // ---------------- UMMA issuer
        const uint32_t sbase = ptx::smem_u32(smem);
        const uint32_t qbase = ptx::smem_u32(qn);
        int stage = 0;
        uint32_t ph = 0;
        bool ok = true;
        const uint32_t idesc1 = ptx::idesc_bf16(BT, qk, false, true);
        for (int kb = 0; ok && kb < kb1; ++kb) {
            if (!(ok = ptx::mbar_wait(&full_bar[stage], ph, p.status))) break;
            ptx::tc_fence_after();
            const uint32_t st = sbase + stage * kStageBytes;
            const int nkk = min(BK / 16, (p.Lq - kb * BK) / 16);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
                if (kk >= nkk) break;
                // A (tokens) K-major: 128-byte rows, 8-row groups 1 KB apart, K=16 slice 32 B on.
                // B (weight) MN-major: 64-column atoms one box (8 KB) apart, 8-row K groups 1 KB
                // apart, K=16 slice 16 rows (2 KB) on.
                ptx::umma_bf16(tmem, ptx::sdesc_sw128(st + kk * 32, 16, 1024),
                               ptx::sdesc_sw128(st + kABytes + kk * 2048, kBoxBytes, 1024), idesc1,
                               (kb > 0 || kk > 0) ? 1u : 0u);
            }
            ptx::umma_commit(&empty_bar[stage]);
            if (++stage == kStages) { stage = 0; ph ^= 1; }
        }
        if (ok) ptx::umma_commit(&d1_full);
        // the epilogue has read the up-projection out and written q_nope
        if (ok) ok = ptx::mbar_wait(&qn_ready, 0, p.status);
        ptx::tc_fence_after();
        // chunk by chunk, each committed on its own: the epilogue drains chunk 0 while chunk 1's
        // weights stream in
        for (int n = 0; ok && n < nch; ++n) {
            for (int k2 = 0; ok && k2 < kb2; ++k2) {
                if (!(ok = ptx::mbar_wait(&full_bar[stage], ph, p.status))) break;
                ptx::tc_fence_after();
                const uint32_t st = sbase + stage * kStageBytes;
                const int ncols = min(p.L, 256 * (n + 1)) - 256 * n;
                const uint32_t idesc2 = ptx::idesc_bf16(BT, ncols, false, true);
                const int nkk = min(BK / 16, (p.dn - k2 * BK) / 16);
                for (int kk = 0; kk < nkk; ++kk)
                    ptx::umma_bf16(tmem + 256 * n, ptx::sdesc_sw128(qbase + k2 * kABytes + kk * 32, 16, 1024),
                                   ptx::sdesc_sw128(st + kk * 2048, kBoxBytes, 1024), idesc2,
                                   (k2 > 0 || kk > 0) ? 1u : 0u);
                ptx::umma_commit(&empty_bar[stage]);
                if (++stage == kStages) { stage = 0; ph ^= 1; }
            }
            if (ok) ptx::umma_commit(&d2_full[n]);
        }
        // every UMMA of this CTA completes before TMEM is released
        ptx::umma_commit(&mma_done);
        ptx::mbar_wait(&mma_done, 0, p.status);
    } else if (warp >= 2) {
        // ---------------- epilogue: thread = token row of TMEM lane quarter (warp % 4)
        const int quarter = warp & 3;
        const int r = 32 * quarter + lane;
        const int t = tt * BT + r;
        const bool tok = t < p.T;
        const uint32_t t_row = tmem + ((uint32_t)(32 * quarter) << 16);
        bf16* dst = p.qtile + ((size_t)(tok ? t : 0) * p.h + head) * p.R;
        const int half = p.dr / 2;
        // The token's RoPE factors, loaded while the up-projection streams (these warps are idle
        // until it completes); kMaxHalf pairs at most, indexed statically below.
        float cs[kMaxHalf], sn[kMaxHalf];
#pragma unroll
        for (int i = 0; i < kMaxHalf; ++i) {
            cs[i] = (tok && i < half) ? p.cos_t[(size_t)t * half + i] : 0.f;
            sn[i] = (tok && i < half) ? p.sin_t[(size_t)t * half + i] : 0.f;
        }
        bool ok = __all_sync(0xffffffffu, ptx::mbar_wait(&d1_full, 0, p.status));
        if (ok) {
            ptx::tc_fence_after();
            // rope part: interleaved pairs (2i, 2i + 1) rotated by (cos_i, sin_i) of the token;
            // all of its TMEM loads in flight before one wait
            {
                const int nr = p.dr / 16;
                uint32_t rv[kMaxHalf / 8][16];
#pragma unroll
                for (int c = 0; c < kMaxHalf / 8; ++c)
                    if (c < nr) ptx::tmem_ld16_nowait(t_row + p.dn + 16 * c, rv[c]);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < kMaxHalf / 8; ++c) {
                    if (c >= nr) break;
                    uint32_t w[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float a = __uint_as_float(rv[c][2 * i]), b = __uint_as_float(rv[c][2 * i + 1]);
                        w[i] = pack_bf16x2(a * cs[8 * c + i] - b * sn[8 * c + i], a * sn[8 * c + i] + b * cs[8 * c + i]);
                    }
                    if (tok) {
                        uint4* d4 = reinterpret_cast<uint4*>(dst + p.L + 16 * c);
                        d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
                        d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
                    }
                }
            }
            // q_nope -> bf16 into the absorption's A operand (K-major, 128-byte swizzle), four
            // TMEM loads in flight per wait
            for (int c0 = 0; c0 < p.dn; c0 += 64) {
                uint32_t nv[4][16];
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if (c0 + 16 * c < p.dn) ptx::tmem_ld16_nowait(t_row + c0 + 16 * c, nv[c]);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int c16 = c0 + 16 * c;
                    if (c16 >= p.dn) break;
                    uint32_t w[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        w[i] = pack_bf16x2(__uint_as_float(nv[c][2 * i]), __uint_as_float(nv[c][2 * i + 1]));
                    unsigned char* blk = qn + (c16 / BK) * kABytes + (r >> 3) * 1024 + (r & 7) * 128;
                    const int ch = (c16 % BK) / 8;   // first 16-byte chunk of the 16 columns
                    *reinterpret_cast<uint4*>(blk + ((ch ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
                    *reinterpret_cast<uint4*>(blk + (((ch + 1) ^ (r & 7)) << 4)) = make_uint4(w[4], w[5], w[6], w[7]);
                }
            }
            ptx::fence_proxy_async_smem();   // generic stores -> the UMMA's reads
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&qn_ready);
        }
        if (ok) {
            for (int col = 0; ok && col < p.L; col += 32) {
                if (col % 256 == 0) {   // the chunk's absorption has completed
                    ok = __all_sync(0xffffffffu, ptx::mbar_wait(&d2_full[col / 256], 0, p.status));
                    if (!ok) break;
                    ptx::tc_fence_after();
                }
                uint32_t r0[16], r1[16];
                ptx::tmem_ld16_nowait(t_row + col, r0);
                ptx::tmem_ld16_nowait(t_row + col + 16, r1);
                ptx::tmem_wait_ld();
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    w[i] = pack_bf16x2(__uint_as_float(r0[2 * i]), __uint_as_float(r0[2 * i + 1]));
                    w[8 + i] = pack_bf16x2(__uint_as_float(r1[2 * i]), __uint_as_float(r1[2 * i + 1]));
                }
                if (tok) {
                    uint4* d4 = reinterpret_cast<uint4*>(dst + col);
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4)
                        d4[v4] = make_uint4(w[4 * v4], w[4 * v4 + 1], w[4 * v4 + 2], w[4 * v4 + 3]);
                }
            }
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace qchain

bool q_chain_supports(const Dims& d) {
    const int qk = d.qk();
    return qk % 16 == 0 && qk <= 256 && d.dn % 16 == 0 && d.dn <= 2 * qchain::BK && d.L % 64 == 0 && d.L <= 512 &&
           d.dr % 16 == 0 && d.dr <= 2 * qchain::kMaxHalf;
}

cudaError_t launch_q_chain(const bf16* q_an, const void* wq_b, const void* q_absorb_w, const float* cos_t,
                           const float* sin_t, const Dims& d, bf16* qtile, int32_t* status, cudaStream_t s) {
    using namespace qchain;
    if (!q_chain_supports(d)) return cudaErrorInvalidValue;
    CUtensorMap tq, tw, ta;
    // q_an [T, Lq]: token tiles of 128 rows (rows past T read as zero)
    if (!make_tma_2d(&tq, q_an, (uint64_t)d.Lq, (uint64_t)d.T, (uint64_t)d.Lq * 2, BK, BT) ||
        // wq_b [Lq, h (dn + dr)]: boxes of 64 K rows x 64 output columns
        !make_tma_2d(&tw, wq_b, (uint64_t)d.h * d.qk(), (uint64_t)d.Lq, (uint64_t)d.h * d.qk() * 2, 64, BK) ||
        // q_absorb_w [h, dn, L] as [h dn, L]: boxes of 64 K rows x 64 output columns
        !make_tma_2d(&ta, q_absorb_w, (uint64_t)d.L, (uint64_t)d.h * d.dn, (uint64_t)d.L * 2, 64, BK))
        return cudaErrorInvalidValue;
    Params p;
    p.T = d.T;
    p.h = d.h;
    p.Lq = d.Lq;
    p.dn = d.dn;
    p.dr = d.dr;
    p.L = d.L;
    p.R = d.R();
    p.cos_t = cos_t;
    p.sin_t = sin_t;
    p.qtile = qtile;
    p.status = status;
    {
        constexpr int kMaxDevices = 64;
        static bool attr_set[kMaxDevices] = {};   // function attributes are per device
        int dev = 0;
        cudaGetDevice(&dev);
        if (dev < 0 || dev >= kMaxDevices || !attr_set[dev]) {
            const cudaError_t e = cudaFuncSetAttribute(k_q_chain, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
            if (e != cudaSuccess) return e;
            if (dev >= 0 && dev < kMaxDevices) attr_set[dev] = true;
        }
    }
    const int tiles = (d.T + BT - 1) / BT;
    // programmatic launch in graphs too: the first weight boxes load while the previous kernel finishes
    return launch_pdl_mode(true, k_q_chain, dim3(d.h * tiles), dim3(kThreads), kSmem, s, tq, tw, ta, p);
}

}  // namespace mla
