// Weight-streaming tensor-core GEMM for the block's projections (sm_100a).
//
// Every projection of the page's block is "activations [T, K] x weight" with
// a weight far larger than the activations (T <= a few hundred decode tokens),
// so each is computed swapped: D[M = output features, N = tokens] =
// A[M, K] (weight tile, streamed by TMA) x B[N, K]^T (token tile). The
// accumulator lives in TMEM with lane = output feature and column = token, so
// epilogue warps write each token's features with coalesced stores.
//
// A is read either MN-major (weights stored [in, out], the page's layout for
// wq_a, wkv_a, wq_b, q_absorb_w, o_proj_w) or K-major (out_absorb_w is
// [heads, v_head_dim, kv_lora_rank], i.e. [M, K]). Both use 128-byte swizzled
// TMA boxes of 64 elements along the contiguous dimension.
//
// Work split: a "unit" is one 64-deep K block of one output tile. With an
// accumulating epilogue (fp32 reductions into a zeroed buffer) each CTA takes a
// contiguous run of units (stream-K: several partial tiles per CTA, balanced to
// +-1 unit), or, when the host picks split-K, items of (tile, K slice) round-robin;
// with a storing epilogue each CTA takes whole tiles round-robin.
// Warp 0 issues TMA, warp 1 issues UMMA (one thread) and owns TMEM, warps 2-5
// drain accumulators. Two TMEM accumulators let the next tile's UMMA overlap
// the previous tile's drain. With MP = 2 a CTA tile is two consecutive
// 128-feature tiles: each stage holds both weight tiles and one token tile, and
// the two UMMAs of a K step read the same token operand.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "ptx.cuh"

namespace mla {
namespace gemm {

constexpr int BM = 128;           // UMMA M (output features per tile)
constexpr int BK = 64;            // K per stage (one 128-byte swizzle atom of bf16)
constexpr int kThreads = 192;     // 6 warps
constexpr int kABytes = BM * BK * 2;

// MP: output-feature tiles per CTA tile. With MP = 2 a stage holds two weight tiles
// and one token tile, and both UMMAs read that token tile (half the token bytes).
template <int BN, int MP = 1>
struct Cfg {
    static constexpr int kBBytes = BN * BK * 2;
    static constexpr int kStageBytes = MP * kABytes + kBBytes;
    static constexpr int kStages = (196608 / kStageBytes) < 8 ? (196608 / kStageBytes) : 8;
    static constexpr int kEpiBuf = 16 * 32 * 4;   // per epilogue warp: [16 tokens][32 features] fp32
    static constexpr int kSmem = kStages * kStageBytes + 4 * kEpiBuf + 1024;
    static constexpr uint32_t kTmemCols = (2 * MP * BN) < 32 ? 32 : 2 * MP * BN;   // two accumulators
};

// Problem description (all sizes in elements).
struct Problem {
    int m_total;        // output features (rows of D)
    int n_rows;         // valid tokens (columns of D); rows of B beyond it are zero-filled
    int k_total;        // K per group (multiple of 16; the last block may be partial)
    int m_tiles, n_tiles, k_blocks, groups;
    int a_group_rows;   // A row offset per group (K rows if MN-major, M rows if K-major)
    int b_group_cols;   // B column (K) offset per group
    int accumulate;     // 1: stream-K units + reducing epilogue; 0: whole tiles + storing epilogue
    int32_t* status;
    // Optional second problem in the same launch (same K, B and epilogue type; one group,
    // its own A map and epilogue): tiles from groups * m_tiles * n_tiles on belong to it.
    int m_tiles1, n_tiles1;   // 0 when absent
    int a_evict_first;        // A loads carry an evict-first L2 policy
    int splits;               // accumulate mode: > 0 selects split-K with this many K slices per tile
};

// ------------------------------------------------------------------ epilogues
// Each epilogue warp owns 32 consecutive output features (TMEM lanes). For
// every 16-token chunk it stages D[32 features x 16 tokens] transposed into
// its shared buffer buf[token][feature] (fp32), then the functor writes it out
// token-row by token-row with 16-byte vectors. m_base is the warp's first
// feature; all 32 lanes call the functor (uniform control flow).

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}
// The same add at system scope: several GPUs add into one owner's accumulator over NVLink.
__device__ __forceinline__ void red_add_v4_sys(float* addr, float a, float b, float c, float d) {
    asm volatile("red.relaxed.sys.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}
__device__ __forceinline__ uint4 pack8_bf16(const float* v) {
    uint4 o;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    return o;
}

// out[n * ldo + g * group_off + m] += v  (fp32 reduction; out zeroed by the caller)
struct EpiReduceF32 {
    float* out;
    int ldo, group_off, m_total, n_rows;
    static constexpr bool kSignals = false;
    __device__ void operator()(int g, int m_base, int n0, const float* buf, int lane) const {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int k = lane + 32 * i, c = k >> 3, m = m_base + 4 * (k & 7);
            if (n0 + c >= n_rows || m >= m_total) continue;
            const float4 v = *reinterpret_cast<const float4*>(buf + c * 32 + 4 * (k & 7));
            red_add_v4(out + (size_t)(n0 + c) * ldo + (size_t)g * group_off + m, v.x, v.y, v.z, v.w);
        }
    }
};

// out[n * ldo + g * group_off + m] = bf16(v)
struct EpiStoreBF16 {
    bf16* out;
    int ldo, group_off, m_total, n_rows;
    static constexpr bool kSignals = false;
    __device__ void operator()(int g, int m_base, int n0, const float* buf, int lane) const {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int k = lane + 32 * i, c = k >> 2, m = m_base + 8 * (k & 3);
            if (n0 + c >= n_rows || m >= m_total) continue;
            *reinterpret_cast<uint4*>(out + (size_t)(n0 + c) * ldo + (size_t)g * group_off + m) =
                pack8_bf16(buf + c * 32 + 8 * (k & 3));
        }
    }
};

// Head-split o-projection (tensor parallelism over heads): output columns
// [r * shard, (r + 1) * shard) belong to rank r, and each 32-feature block is
// reduced straight into its owner's accumulator acc[r] ([n_rows, shard] fp32),
// another GPU's memory (over NVLink) when the owner is a peer. Every group of
// the launch (one per rank the launch serves) adds into the same owners. After
// its last tile each CTA adds the K blocks it processed to every owner's
// arrival counter (signal), so an owner knows when all ranks' sums are in. The adds are
// system-scope atomics, since adds from different GPUs meet in one accumulator.
constexpr int kTpMaxWorld = 8;
struct EpiReducePeers {
    float* acc[kTpMaxWorld];
    uint32_t* arrive[kTpMaxWorld];
    int world, shard, m_total, n_rows;
    static constexpr bool kSignals = true;
    __device__ void operator()(int, int m_base, int n0, const float* buf, int lane) const {
        if (m_base >= m_total) return;      // past the last column (uniform over the warp)
        const int owner = m_base / shard;   // shard is a multiple of 32: one owner per warp block
        float* out = acc[owner];
        const int m_loc = m_base - owner * shard;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int k = lane + 32 * i, c = k >> 3, dm = 4 * (k & 7);
            if (n0 + c >= n_rows || m_base + dm >= m_total) continue;
            const float4 v = *reinterpret_cast<const float4*>(buf + c * 32 + dm);
            red_add_v4_sys(out + (size_t)(n0 + c) * shard + m_loc + dm, v.x, v.y, v.z, v.w);
        }
    }
    // One thread, after every epilogue store of the CTA (a CTA barrier): release the
    // CTA's reductions to the whole system, then count them at every owner.
    __device__ void signal(int units) const {
        __threadfence_system();
        for (int r = 0; r < world; ++r)
            asm volatile("red.relaxed.sys.global.add.u32 [%0], %1;" ::"l"(arrive[r]), "r"((uint32_t)units)
                         : "memory");
    }
};

// ------------------------------------------------------------------ schedule
struct Seg {
    int tile, kb0, kb1;
};

// Sequence of (tile, k-range) segments of this CTA. Identical in every role.
struct Schedule {
    int total_units, u, u_end;     // accumulate mode, stream-K (units = tile * k_blocks + kb)
    int tile, tiles;               // store mode
    int splits, item, items;       // accumulate mode, split-K: item = tile * splits + slice
    bool acc;
    int k_blocks;
    __device__ Schedule(const Problem& p) {
        acc = p.accumulate != 0;
        k_blocks = p.k_blocks;
        tiles = p.groups * p.m_tiles * p.n_tiles + p.m_tiles1 * p.n_tiles1;
        splits = acc ? p.splits : 0;
        if (splits > 0) {
            item = blockIdx.x;
            items = tiles * splits;
        } else if (acc) {
            total_units = tiles * p.k_blocks;
            u = (int)((long long)total_units * blockIdx.x / gridDim.x);
            u_end = (int)((long long)total_units * (blockIdx.x + 1) / gridDim.x);
        } else {
            tile = blockIdx.x;
        }
    }
    __device__ bool next(Seg& s) {
        if (splits > 0) {   // items round-robin: CTAs running together read the same K rows
            if (item >= items) return false;
            s.tile = item / splits;
            const int sl = item - s.tile * splits;
            s.kb0 = k_blocks * sl / splits;
            s.kb1 = k_blocks * (sl + 1) / splits;
            item += gridDim.x;
            return true;
        }
        if (acc) {
            if (u >= u_end) return false;
            s.tile = u / k_blocks;
            s.kb0 = u - s.tile * k_blocks;
            s.kb1 = min(k_blocks, s.kb0 + (u_end - u));
            u += s.kb1 - s.kb0;
            return true;
        }
        if (tile >= tiles) return false;
        s.tile = tile;
        s.kb0 = 0;
        s.kb1 = k_blocks;
        tile += gridDim.x;
        return true;
    }
};

// tile -> (problem, group, m tile, n tile); n innermost so the n tiles of one
// weight tile run back to back and share it through L2.
__device__ __forceinline__ int split_tile(const Problem& p, int tile, int& g, int& mt, int& nt) {
    const int tiles0 = p.groups * p.m_tiles * p.n_tiles;
    if (tile >= tiles0) {
        tile -= tiles0;
        nt = tile % p.n_tiles1;
        mt = tile / p.n_tiles1;
        g = 0;
        return 1;
    }
    nt = tile % p.n_tiles;
    const int r = tile / p.n_tiles;
    mt = r % p.m_tiles;
    g = r / p.m_tiles;
    return 0;
}

// ------------------------------------------------------------------ kernel
template <int BN, bool A_MN, class Epi, int MP = 1>
__global__ void __launch_bounds__(kThreads, 1)
k_gemm_tc(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b, Problem p,
          Epi epi, const __grid_constant__ CUtensorMap tma_a1, Epi epi1) {
    static_assert(MP == 1 || MP == 2, "one or two feature tiles per CTA tile");
    static_assert(2 * MP * BN <= 512, "two accumulators must fit TMEM");
    using C = Cfg<BN, MP>;
    constexpr int S = C::kStages;
    griddep_launch();
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[S], empty_bar[S], acc_full[2], acc_empty[2], mma_done;
    __shared__ uint32_t tmem_base_slot;
    __shared__ int abort_flag;

    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            ptx::mbar_init(&full_bar[i], 1);
            ptx::mbar_init(&empty_bar[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&acc_full[i], 1);
            ptx::mbar_init(&acc_empty[i], 4);
        }
        ptx::mbar_init(&mma_done, 1);
        abort_flag = 0;
        ptx::fence_mbar_init();
        ptx::tma_prefetch_desc(&tma_a);
        ptx::tma_prefetch_desc(&tma_b);
        if (p.m_tiles1 > 0) ptx::tma_prefetch_desc(&tma_a1);
    }
    if (warp == 1) {
        ptx::tmem_alloc(&tmem_base_slot, C::kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = tmem_base_slot;
    // The producer waits for the previous kernel only after it has started loading the first
    // stages' weight tiles (weights are never written by the block's kernels); every other
    // warp waits here, before its first access to memory another kernel writes.
    if (warp != 0) griddep_wait();
    int units_issued = 0;   // K blocks this CTA loaded (thread 0)

    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer
        const uint64_t pol = ptx::policy_evict_first();
        // A (weight) loads of the K block at stage `stage`; its full barrier expects the whole
        // stage (A and B).
        auto load_a = [&](const CUtensorMap* ta, int g, int m0, int kb, int stage) {
            unsigned char* a_s0 = smem + stage * C::kStageBytes;
            ptx::mbar_arrive_expect_tx(&full_bar[stage], C::kStageBytes);
            const int k0 = kb * BK;
#pragma unroll
            for (int i = 0; i < MP; ++i) {   // a feature tile past the last row is zero-filled
                unsigned char* a_s = a_s0 + i * kABytes;
                const int mi = m0 + i * BM;
                if (p.a_evict_first) {
                    if (A_MN) {
                        ptx::tma_load_2d_hint(a_s, ta, &full_bar[stage], mi, g * p.a_group_rows + k0, pol);
                        ptx::tma_load_2d_hint(a_s + kABytes / 2, ta, &full_bar[stage], mi + 64,
                                              g * p.a_group_rows + k0, pol);
                    } else {
                        ptx::tma_load_2d_hint(a_s, ta, &full_bar[stage], k0, g * p.a_group_rows + mi, pol);
                    }
                } else if (A_MN) {
                    ptx::tma_load_2d(a_s, ta, &full_bar[stage], mi, g * p.a_group_rows + k0);
                    ptx::tma_load_2d(a_s + kABytes / 2, ta, &full_bar[stage], mi + 64, g * p.a_group_rows + k0);
                } else {
                    ptx::tma_load_2d(a_s, ta, &full_bar[stage], k0, g * p.a_group_rows + mi);
                }
            }
        };
        // Weight tiles of the first S K blocks (the stages are all free), then the wait for
        // the previous kernel, whose data the token tiles are.
        int n_pre = 0;
        {
            Schedule pre(p);
            Seg sg;
            while (n_pre < S && pre.next(sg)) {
                int g, mt, nt;
                const CUtensorMap* ta = split_tile(p, sg.tile, g, mt, nt) ? &tma_a1 : &tma_a;
                for (int kb = sg.kb0; kb < sg.kb1 && n_pre < S; ++kb, ++n_pre) load_a(ta, g, mt * BM * MP, kb, n_pre);
            }
        }
        griddep_wait();
        Schedule sch(p);
        Seg sg;
        int stage = 0, n_issued = 0;
        uint32_t phase = 0;
        while (sch.next(sg)) {
            int g, mt, nt;
            const CUtensorMap* ta = split_tile(p, sg.tile, g, mt, nt) ? &tma_a1 : &tma_a;
            const int m0 = mt * BM * MP, n0 = nt * BN;
            for (int kb = sg.kb0; kb < sg.kb1; ++kb) {
                if (n_issued >= n_pre) {   // past the prefetched stages: the usual wait and weight loads
                    if (!ptx::mbar_wait(&empty_bar[stage], phase ^ 1, p.status)) { abort_flag = 1; goto producer_done; }
                    if (*(volatile int*)&abort_flag) goto producer_done;
                    load_a(ta, g, m0, kb, stage);
                }
                unsigned char* b_s = smem + stage * C::kStageBytes + MP * kABytes;
                ptx::tma_load_2d(b_s, &tma_b, &full_bar[stage], g * p.b_group_cols + kb * BK, n0);
                ++n_issued;
                if (++stage == S) { stage = 0; phase ^= 1; }
            }
        }
    producer_done:
        units_issued = n_issued;
        // Every load this CTA issued must land before its shared memory is
        // released: wait (bounded) for the last phase of each stage used.
        for (int i = 0; i < S && i < n_issued; ++i) {
            if (--stage < 0) { stage = S - 1; phase ^= 1; }
            ptx::mbar_wait(&full_bar[stage], phase, p.status);
        }
    } else if (warp == 1 && lane == 0) {
        // ---------------- UMMA issuer
        constexpr uint32_t idesc = ptx::idesc_bf16(BM, BN, A_MN, false);
        Schedule sch(p);
        Seg sg;
        int stage = 0, seg = 0;
        uint32_t phase = 0, acc_phase[2] = {0, 0};
        while (sch.next(sg)) {
            const int buf = seg & 1;
            if (!ptx::mbar_wait(&acc_empty[buf], acc_phase[buf] ^ 1, p.status)) { abort_flag = 1; break; }
            acc_phase[buf] ^= 1;
            ptx::tc_fence_after();
            const uint32_t d_tmem = tmem_base + buf * (MP * BN);
            bool ok = true;
            for (int kb = sg.kb0; kb < sg.kb1; ++kb) {
                if (!ptx::mbar_wait(&full_bar[stage], phase, p.status)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t a_addr0 = ptx::smem_u32(smem + stage * C::kStageBytes);
                const uint32_t b_addr = a_addr0 + MP * kABytes;
                const int n_kk = min(BK / 16, (p.k_total - kb * BK) / 16);   // partial last block
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
                    if (kk >= n_kk) break;
                    // A MN-major: 64-element atoms along M at +8 KB (LBO), 8-row K groups at +1 KB (SBO);
                    //   a K=16 slice starts 16 rows (2 KB) further.
                    // A / B K-major: rows of 128 B, 8-row groups at +1 KB (SBO); a K=16 slice starts 32 B further.
                    const uint64_t bdesc = ptx::sdesc_sw128(b_addr + kk * 32, 16, 1024);
#pragma unroll
                    for (int i = 0; i < MP; ++i) {
                        const uint32_t a_addr = a_addr0 + i * kABytes;
                        const uint64_t adesc = A_MN ? ptx::sdesc_sw128(a_addr + kk * 2048, kABytes / 2, 1024)
                                                    : ptx::sdesc_sw128(a_addr + kk * 32, 16, 1024);
                        ptx::umma_bf16(d_tmem + i * BN, adesc, bdesc, idesc, (kb > sg.kb0 || kk > 0) ? 1u : 0u);
                    }
                }
                ptx::umma_commit(&empty_bar[stage]);
                if (++stage == S) { stage = 0; phase ^= 1; }
            }
            if (!ok) { abort_flag = 1; break; }
            ptx::umma_commit(&acc_full[buf]);
            ++seg;
        }
        // All UMMAs of this CTA complete before TMEM is released.
        ptx::umma_commit(&mma_done);
        ptx::mbar_wait(&mma_done, 0, p.status);
    } else if (warp >= 2) {
        // ---------------- epilogue (warps 2..5 -> TMEM lane quarters 2,3,0,1)
        const int quarter = warp & 3;
        Schedule sch(p);
        Seg sg;
        int seg = 0;
        uint32_t acc_phase[2] = {0, 0};
        while (sch.next(sg)) {
            const int buf = seg & 1;
            if (!ptx::mbar_wait(&acc_full[buf], acc_phase[buf], p.status)) break;
            acc_phase[buf] ^= 1;
            ptx::tc_fence_after();
            int g, mt, nt;
            const Epi& ep = split_tile(p, sg.tile, g, mt, nt) ? epi1 : epi;
            float* ebuf = reinterpret_cast<float*>(smem + S * C::kStageBytes + (warp - 2) * C::kEpiBuf);
#pragma unroll 1
            for (int mi = 0; mi < MP; ++mi) {
                const int m_base = (mt * MP + mi) * BM + quarter * 32;
                const uint32_t t_addr = tmem_base + ((uint32_t)(quarter * 32) << 16) + buf * (MP * BN) + mi * BN;
#pragma unroll 1
                for (int c = 0; c < BN; c += 16) {
                    float v[16];
                    ptx::tmem_ld16(t_addr + c, v);
#pragma unroll
                    for (int i = 0; i < 16; ++i) ebuf[i * 32 + lane] = v[i];
                    __syncwarp();
                    ep(g, m_base, nt * BN + c, ebuf, lane);
                    __syncwarp();
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&acc_empty[buf]);
            ++seg;
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if constexpr (Epi::kSignals) {
        if (threadIdx.x == 0 && units_issued > 0) epi.signal(units_issued);
    }
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

}  // namespace gemm
}  // namespace mla
