// Sparse latent attention core on tcgen05 (page "MLA Attention Block Gather
// Decode Kernel API Reference": :param gather_indices, kv_cache, positions,
// softmax_scale; "attending over only the prior keys the indexer selected").
//
// Per work item (token t, group of up to 128 heads) over its kept rows
// (resolved and compacted by the index stage):
//     s_j = softmax_scale * (q_lat . c_j + q_pe . kpe_j)   for all heads at once:
//         S [128 heads x keys] = Qtile [128 x R] . rows [keys x R]^T
//     ctx = softmax_j(s) . rows[:, :L]                      (latent part is the value)
// Every head shares the same gathered rows, so both products are dense
// tensor-core GEMMs with M = 128 heads.
//
// Column split over a 2-CTA cluster. The latent context of 128 heads
// (128 x 512 fp32) fills one SM's TMEM, and every kept row is needed by both
// products, so each CTA of the pair takes a share of every row's COLUMNS and
// each row is gathered from HBM exactly once:
//   CTA r gathers latent columns [r L/2, (r+1) L/2) and half of the rope part
//   (or, when the halves cannot be even, the whole rope part goes to the CTA
//   with fewer latent blocks).
// Per tile of 64 kept keys:
//   1. each CTA: partial scores S_r = Q[:, cols_r] . K[:, cols_r]^T (TMEM);
//   2. CTA r owns the softmax of heads [64r, 64r+64); it ships its partial
//      scores of the other 64 heads into the peer's shared memory (st.async);
//   3. each CTA, for its own heads: S = S_r + S_peer, fp32 online softmax (one
//      thread per head, base-2 exponent, lazy rescale: the running max only
//      moves when a tile exceeds it by 2^8); bf16 P rows go to the P buffers
//      of both CTAs, with the rescale factor of every head;
//   4. each CTA: O_r += P . V_r into its 256 latent columns of the context of
//      all 128 heads (TMEM), O rows rescaled in TMEM on the rare tiles that
//      moved a head's max.
// Rows are gathered by TMA (tile::gather4, four rows per instruction) straight
// into the swizzled layout the UMMA reads; four producer warps per CTA issue
// them so that enough bytes are in flight.
//
// TMEM of each CTA (512 columns): O_r [0, 256) | Q latent share [256, 384) |
// S buffers [384, 448) and [448, 512). The Q rope share is the score product's
// A operand from shared memory.
//
// Work split: tiles of 64 kept keys; all (item, tile) pairs are laid out item
// by item and each cluster takes a contiguous run (stream-K). An item fully
// inside one run is finished in place; an item split between runs leaves
// bf16 partial contexts with their (max, sum), merged by k_core_combine.
#include <type_traits>

#include "common.cuh"
#include "core_plan.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace mla {
namespace core {

constexpr int MH = 128;           // heads per work item (UMMA M)
constexpr int HALF = MH / 2;      // heads whose softmax one CTA owns
// Warps: 0-3, 8-11 row warps (TMEM lane quarter = warp % 4) | 4-7 producers | 12 score UMMA issuer
// (allocates TMEM) | 13 P.V UMMA issuer. A warp's gather issue is slow (each instruction issues its
// lanes' gathers one after another), so four producer warps share each tile's rows.
constexpr int kProducers = 4;
constexpr int kProdWarp0 = 4, kScoreWarp = 12, kPvWarp = 13;
constexpr int kWarps = 14;
constexpr int kThreads = 32 * kWarps;
constexpr int kMaxStages = 8;
constexpr int NP = 2;             // P buffers
constexpr int NX = 2;             // partial-score exchange buffers
constexpr float kRescaleLog2 = 8.f;
constexpr int kBlockBytes = KT * 128;             // [KT keys x 64 columns], 128-byte rows
constexpr int kPBytes = (KT / 64) * MH * 128;     // P [128 heads x KT keys] bf16, K-major 128-byte swizzle
constexpr int kXsBytes = HALF * KT * 4;           // partial scores of 64 heads, fp32, [KT/4][64][4]
constexpr int kExtraBytes = 4 * MH * 4 + 64;      // per head {rescale factor, max, sum of key half 0, of half 1},
                                                  // then one "some head of this warp rescales" word per own warp
constexpr int kPHalfBytes = HALF * KT * 2;        // P rows of one CTA's heads
constexpr int kFlagOff = 4 * MH * 4;              // offset of the four rescale flags in an extras buffer
constexpr int kPMsgBytes = kPHalfBytes + HALF * 16 + 16;   // what the peer's st.async deliver per tile
constexpr int kPOff = 0;                          // shared-memory offsets (identical in both CTAs)
constexpr int kXsOff = kPOff + NP * kPBytes;
constexpr int kExtraOff = kXsOff + NX * kXsBytes;
constexpr int kQrOff = (kExtraOff + NP * kExtraBytes + 1023) / 1024 * 1024;   // rope share of Q
constexpr int kOCol = 0, kQCol = 256, kSCol = 384;  // TMEM columns; S buffer b at kSCol + KT b
constexpr int kSmemPerBlock = 232448;             // opt-in shared memory per block on sm_100
static_assert(KT == 64 && kSCol + 2 * KT <= 512, "two S buffers after O and the Q latent share");

// The columns one CTA of the pair gathers (host-computed from the dims).
struct Share {
    int nl;            // latent 64-column blocks
    int lcol0;         // first latent column (also this CTA's first context column)
    int rope_x;        // first rope column gathered (when rope_w > 0)
    int rope_w;        // rope columns gathered: 0, 32 (64-byte swizzle) or 64 (128-byte swizzle)
    int qr_bytes;      // shared-memory bytes of the Q rope share (1 KB multiple; 0 without rope)
    int stage_off;     // offset of the first tile stage (after the Q rope share)
    int stage_bytes;   // shared-memory bytes of one tile stage (1 KB multiple)
    int stage_tx;      // bytes the TMA delivers per stage
    int ns;            // stages
};

struct Params {
    const int32_t* rows;        // [T, P] kept rows, compacted
    const int32_t* n_valid;     // [T]
    const int32_t* item_base;   // [W + 1] first tile of each item
    const bf16* qtile;          // [T * h, R]
    int T, h, HG, P, L, R, W, max_clusters;
    float scale_log2;           // softmax_scale * log2(e)
    Share share[2];
    bf16* ctx;                  // [T, h, L]
    bf16* part_o;               // [2 * max_clusters, 128, L]
    float* part_ml;             // [2 * max_clusters, 2, 128]  (max in log2 units, sum)
    int4* merge_desc;           // [max_clusters + 1] merge plan per run boundary (see k_core_plan)
    int32_t* status;
};

struct Seg {
    int w, j0, j1, n_w;
    bool run_start;   // segment begins this cluster's run
};

struct SegIter {
    const int32_t* base;
    int W, u, u0, u1, w;
    __device__ void init(const Params& p, int c, int C) {
        base = p.item_base;
        W = p.W;
        const int U = base[W];
        u0 = u = (int)((long long)U * c / C);
        u1 = (int)((long long)U * (c + 1) / C);
        int lo = 0, hi = W - 1;   // largest w with base[w] <= u
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (base[mid] <= u) lo = mid;
            else hi = mid - 1;
        }
        w = lo;
    }
    __device__ bool next(Seg& s) {
        if (u >= u1) return false;
        while (base[w + 1] <= u) ++w;
        s.w = w;
        s.n_w = base[w + 1] - base[w];
        s.j0 = u - base[w];
        s.j1 = min(u1, base[w + 1]) - base[w];
        s.run_start = (u == u0);
        u = base[w] + s.j1;
        return true;
    }
};


__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
    uint32_t u[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) u[i] = __float_as_uint(v[i]);
    ptx::tmem_st16_u32(taddr, u);
}

// 2^x by the SFU's approximate base-2 exponential (PTX ex2.approx.ftz.f32).
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);   // .x = lo (low 16 bits), .y = hi
    return *reinterpret_cast<const uint32_t*>(&v);
}

// Score product of one tile, latent columns: 4 NL K-steps, fully unrolled (a
// single issuing thread keeps the tensor core fed only when it does little
// else between issues). Q comes from TMEM; bd0 describes latent block 0 of the
// tile's stage, blocks kBlockBytes apart.
template <int NL>
__device__ __forceinline__ void issue_scores_latent(uint32_t d_s, uint32_t a_q, uint64_t bd0, uint32_t idesc) {
#pragma unroll
    for (int u = 0; u < 2 * NL; ++u)
#pragma unroll
        for (int k2 = 0; k2 < 2; ++k2)
            ptx::umma_bf16_ts(d_s, a_q + 16 * u + 8 * k2,
                              bd0 + (uint64_t)(((u >> 1) * kBlockBytes + (u & 1) * 64 + k2 * 32) >> 4), idesc,
                              (u | k2) ? 1u : 0u);
}

// Kept-row id number k (clamped to the last kept row) of item token t.
__device__ __forceinline__ int kept_row(const Params& p, int t, int nv, int k) {
    return p.rows[(size_t)t * p.P + min(k, nv - 1)];
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
k_core_tc(const __grid_constant__ CUtensorMap tma_w128, const __grid_constant__ CUtensorMap tma_w64, Params p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    griddep_launch();
    // Barriers sit at identical offsets in both ranks (remote arrivals rely on it).
    __shared__ __align__(8) uint64_t kf[kMaxStages], ke[kMaxStages];
    __shared__ __align__(8) uint64_t s_full[2], s_free[2], q_full, q_empty, o_free, mma_done, mma_done_p, corr_done;
    __shared__ __align__(8) uint64_t xs_full[NX];
    __shared__ __align__(8) uint64_t p_full[NP], p_ready[NP], pf_mine[NP], pf_peer[NP];
    __shared__ __align__(8) uint64_t l_sync[2], m_sync[2];
    __shared__ float l_x[2][2][2][32];   // [segment parity][own quarter][key half][lane]
    __shared__ float m_x[2][2][2][32];   // [tile parity][own quarter][key half][lane]
    __shared__ uint32_t tmem_slot;

    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t rank = ptx::cluster_ctarank();
    const uint32_t peer = rank ^ 1u;
    const Share sh = p.share[rank];
    const int c = (int)ptx::cluster_id_x();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr uint32_t kTmemCols = 512;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kMaxStages; ++i) { ptx::mbar_init(&kf[i], 1); ptx::mbar_init(&ke[i], 1); }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&s_full[i], 1);   // UMMA commit
            ptx::mbar_init(&s_free[i], 8);   // the 8 row warps have read S buffer i
        }
        ptx::mbar_init(&q_full, 8);
        ptx::mbar_init(&q_empty, 1);
        ptx::mbar_init(&o_free, 8);
        ptx::mbar_init(&mma_done, 1);
        ptx::mbar_init(&mma_done_p, 1);
        ptx::mbar_init(&corr_done, 4);       // the peer-head warps rescaled O (only on flagged tiles)
        // With two exchange buffers, buffer reuse needs no signal of its own: the peer's
        // P rows of tile g - 2, which the shipping warps wait for before shipping tile g,
        // are sent only after the peer has read that tile's partial scores.
        static_assert(NX == 2, "exchange-buffer reuse is ordered through the P of tile g - 2");
        for (int i = 0; i < NX; ++i) ptx::mbar_init(&xs_full[i], 1);   // local expect_tx + the peer's st.async bytes
        for (int i = 0; i < NP; ++i) {
            ptx::mbar_init(&p_full[i], 1);     // local expect_tx + the peer's st.async P rows and factors
            ptx::mbar_init(&p_ready[i], 4);    // this CTA's own P rows written, their O rows rescaled
            ptx::mbar_init(&pf_mine[i], 1);    // this CTA's P . V on buffer i has completed
            ptx::mbar_init(&pf_peer[i], 1);    // the peer's P . V on buffer i has completed
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&l_sync[i], 2);    // the two warps of an own quarter (lane 0 of each,
            ptx::mbar_init(&m_sync[i], 2);    // after the warp's shared-memory writes)
        }
        ptx::fence_mbar_init();
        ptx::tma_prefetch_desc(&tma_w128);
        ptx::tma_prefetch_desc(&tma_w64);
    }
    if (warp == kScoreWarp) {
        ptx::tmem_alloc(&tmem_slot, kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync_all();   // peer barriers initialised before any remote arrival
    ptx::tc_fence_after();
    const uint32_t tmem = tmem_slot;
    griddep_wait();   // barriers and TMEM were set up beside the previous kernel; now its data
    const int U = p.item_base[p.W];
    const int C = clusters_for(U, p.max_clusters);
    const bool active = c < C;

    if (active && warp >= kProdWarp0 && warp < kProdWarp0 + kProducers) {
        // ---------------- producers: this CTA's columns of each tile's 64 rows
        // Warp pw owns the tile's rows [16 pw, 16 pw + 16): lanes 0-15 hold their ids (loaded
        // before the wait for the stage, so the load overlaps it); lane l issues the four rows
        // of group l % 4 in column block l / 4 (latent blocks, then the rope block), taking
        // the group's ids from its neighbours.
        constexpr int RW = KT / kProducers, GW = RW / 4;
        static_assert(RW * kProducers == KT && GW * 4 == RW && 32 / GW >= 8, "producer row split");
        const int pw = warp - kProdWarp0;
        const int nblk = sh.nl + (sh.rope_w > 0 ? 1 : 0);
        const int gl = lane % GW, bA = lane / GW;
        const int gi = GW * pw + gl;   // four-row group within the tile
        const int rope_pitch = sh.rope_w * 2;
        const CUtensorMap* rope_map = sh.rope_w == 32 ? &tma_w64 : &tma_w128;
        // Cache rows are read once: their lines are the first to leave L2, so the step's
        // small working set (query tiles, row lists, partial contexts) stays.
        const uint64_t pol = ptx::policy_evict_first();
        auto gather = [&](unsigned char* st, int b, uint64_t* bar, int r0, int r1, int r2, int r3) {
            if (b < sh.nl)
                ptx::tma_gather4_hint(st + b * kBlockBytes + 4 * gi * 128, &tma_w128, bar, sh.lcol0 + 64 * b, r0, r1, r2,
                                      r3, pol);
            else
                ptx::tma_gather4_hint(st + sh.nl * kBlockBytes + 4 * gi * rope_pitch, rope_map, bar, sh.rope_x, r0, r1,
                                      r2, r3, pol);
        };

        SegIter it;
        it.init(p, c, C);
        Seg sg;
        int stage = 0, n_issued = 0;
        uint32_t ph = 0;
        bool ok = true;
        while (ok && it.next(sg)) {
            const int t = sg.w / p.HG;
            const int nv = p.n_valid[t];
            for (int j = sg.j0; ok && j < sg.j1; ++j) {
                const int my_row = kept_row(p, t, nv, j * KT + RW * pw + lane % RW);
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(&ke[stage], ph ^ 1, p.status));
                if (!ok) break;
                const int r0 = __shfl_sync(0xffffffffu, my_row, 4 * gl + 0);
                const int r1 = __shfl_sync(0xffffffffu, my_row, 4 * gl + 1);
                const int r2 = __shfl_sync(0xffffffffu, my_row, 4 * gl + 2);
                const int r3 = __shfl_sync(0xffffffffu, my_row, 4 * gl + 3);
                if (pw == 0 && lane == 0) ptx::mbar_arrive_expect_tx(&kf[stage], sh.stage_tx);
                unsigned char* st = smem + sh.stage_off + stage * sh.stage_bytes;
                if (bA < nblk) gather(st, bA, &kf[stage], r0, r1, r2, r3);
                ++n_issued;
                if (++stage == sh.ns) { stage = 0; ph ^= 1; }
            }
        }
        // loads already issued land before shared memory is released
        if (lane == 0)
            for (int i = 0; i < sh.ns && i < n_issued; ++i) {
                if (--stage < 0) { stage = sh.ns - 1; ph ^= 1; }
                ptx::mbar_wait(&kf[stage], ph, nullptr);
            }
    } else if (active && warp == kScoreWarp) {
        // ---------------- score UMMA issue: S(g) = Q_r K_r^T, tile by tile
        if (lane == 0) {
            const uint32_t idesc_s = ptx::idesc_bf16(MH, KT, false, false);
            const uint32_t sbase = ptx::smem_u32(smem + sh.stage_off);
            const uint32_t qr = ptx::smem_u32(smem + kQrOff);
            const int rope_valid = sh.rope_w > 0 ? min(sh.rope_w, p.R - sh.rope_x) : 0;
            const int n_rope = (rope_valid + 15) / 16;   // rope K-steps; step y is 32 y bytes into the rows
            SegIter it;
            it.init(p, c, C);
            Seg sg;
            int g = 0, si = 0, stage = 0;
            uint32_t ph = 0;
            bool ok = true;
            while (ok && it.next(sg)) {
                ok = ptx::mbar_wait(&q_full, si & 1, p.status);
                for (int j = sg.j0; ok && j < sg.j1; ++j, ++g) {
                    const int b = g & 1;   // S buffer
                    ok = ptx::mbar_wait(&s_free[b], ((g >> 1) & 1) ^ 1, p.status) &&
                         ptx::mbar_wait(&kf[stage], ph, p.status);
                    if (!ok) break;
                    ptx::tc_fence_after();
                    const uint32_t st = sbase + stage * sh.stage_bytes;
                    const uint32_t d_s = tmem + kSCol + KT * b;
                    const uint64_t bd0 = ptx::sdesc_sw128(st, 16, 1024);
                    switch (sh.nl) {
                        case 1: issue_scores_latent<1>(d_s, tmem + kQCol, bd0, idesc_s); break;
                        case 2: issue_scores_latent<2>(d_s, tmem + kQCol, bd0, idesc_s); break;
                        case 3: issue_scores_latent<3>(d_s, tmem + kQCol, bd0, idesc_s); break;
                        case 4: issue_scores_latent<4>(d_s, tmem + kQCol, bd0, idesc_s); break;
                        default: break;
                    }
                    if (n_rope > 0) {   // rope columns: Q's rope share from shared memory
                        const uint32_t rb = st + sh.nl * kBlockBytes;
                        const bool w64 = sh.rope_w == 32;
                        const uint64_t ad0 = w64 ? ptx::sdesc_sw64(qr, 16, 512) : ptx::sdesc_sw128(qr, 16, 1024);
                        const uint64_t rd0 = w64 ? ptx::sdesc_sw64(rb, 16, 512) : ptx::sdesc_sw128(rb, 16, 1024);
#pragma unroll
                        for (int y = 0; y < 4; ++y)
                            if (y < n_rope)
                                ptx::umma_bf16(d_s, ad0 + 2 * y, rd0 + 2 * y, idesc_s, (sh.nl > 0 || y > 0) ? 1u : 0u);
                    }
                    ptx::umma_commit(&s_full[b]);
                    if (j == sg.j1 - 1) ptx::umma_commit(&q_empty);
                    if (++stage == sh.ns) { stage = 0; ph ^= 1; }
                }
                ++si;
            }
            ptx::umma_commit(&mma_done);
            ptx::mbar_wait(&mma_done, 0, p.status);
        }
    } else if (active && warp == kPvWarp) {
        // ---------------- P . V UMMA issue: O += P(g) V_r(g), tile by tile
        // Tile g needs this CTA's own P rows (p_ready), the peer's P rows and rescale
        // factors (p_full, whose byte count this thread posts) and, when the peer flagged
        // a rescale of some head, the peer-head warps' rescale of this CTA's O rows.
        if (lane == 0) {
            const uint32_t idesc_o = ptx::idesc_bf16(MH, sh.nl > 0 ? 64 * sh.nl : 64, false, true);
            const uint32_t pbase = ptx::smem_u32(smem + kPOff);
            const uint32_t sbase = ptx::smem_u32(smem + sh.stage_off);
            SegIter it;
            it.init(p, c, C);
            Seg sg;
            int g = 0, si = 0, stage = 0, n_corr = 0;
            bool ok = true;
            while (ok && it.next(sg)) {
                if (si > 0) ok = ptx::mbar_wait(&o_free, (si - 1) & 1, p.status);   // previous context read out
                for (int j = sg.j0; ok && j < sg.j1; ++j, ++g) {
                    const bool first = j == sg.j0;
                    const int pb = g % NP;
                    ptx::mbar_arrive_expect_tx(&p_full[pb], kPMsgBytes);
                    ok = ptx::mbar_wait(&p_ready[pb], (g / NP) & 1, p.status) &&
                         ptx::mbar_wait_cluster(&p_full[pb], (g / NP) & 1, p.status);
                    if (!ok) break;
                    ptx::fence_proxy_async_smem();   // the peer's st.async P rows -> this CTA's UMMA
                    const uint4 fl = *reinterpret_cast<const uint4*>(smem + kExtraOff + pb * kExtraBytes + kFlagOff);
                    if (!first && (fl.x | fl.y | fl.z | fl.w)) {
                        ok = ptx::mbar_wait(&corr_done, n_corr & 1, p.status);
                        ++n_corr;
                        if (!ok) break;
                    }
                    ptx::tc_fence_after();
                    if (sh.nl > 0) {
                        // P (K-major, 128-byte swizzle): 32 bytes per 16 keys. V (MN-major): 64-column
                        // atoms kBlockBytes apart (LBO), 8-key groups 1 KB apart (SBO); a K=16 slice
                        // is 16 keys (2 KB) further.
                        const uint64_t ad0 = ptx::sdesc_sw128(pbase + pb * kPBytes, 16, 1024);
                        const uint64_t bd0 = ptx::sdesc_sw128(sbase + stage * sh.stage_bytes, kBlockBytes, 1024);
#pragma unroll
                        for (int kk = 0; kk < KT / 16; ++kk)
                            ptx::umma_bf16(tmem + kOCol, ad0 + 2 * kk, bd0 + 128 * kk, idesc_o,
                                           (first && kk == 0) ? 0u : 1u);
                    }
                    ptx::umma_commit(&ke[stage]);   // the tile's stage is free
                    ptx::umma_commit(&pf_mine[pb]);
                    ptx::umma_commit_multicast(&pf_peer[pb], (uint16_t)(1u << peer));
                    if (++stage == sh.ns) stage = 0;
                }
                ++si;
            }
            ptx::umma_commit(&mma_done_p);
            ptx::mbar_wait(&mma_done_p, 0, p.status);
        }
    } else if (active && (warp < 4 || (warp >= 8 && warp <= 11))) {
        // ---------------- row warps: thread = head row of TMEM lane quarter q; warps q and q+8
        // split the tile's keys (and the O columns) in halves. Quarters 2r, 2r+1 are this
        // CTA's own heads (softmax); the other two quarters ship partial scores to the peer
        // and apply the peer's rescale factors to this CTA's O rows.
        const int q = warp & 3, hk = warp >> 3;
        const bool own = (q >> 1) == (int)rank;
        const int row = 32 * q + lane;
        const int lr = 32 * (q & 1) + lane;   // row within the owner's 64 heads
        const uint32_t t_row = tmem + ((uint32_t)(32 * q) << 16);
        const int ow = 32 * sh.nl;            // O columns each warp of the quarter handles
        const int oc0 = hk * ow;
        const uint32_t peer_p = ptx::mapa_shared(ptx::smem_u32(smem + kPOff), peer);
        const uint32_t peer_xs = ptx::mapa_shared(ptx::smem_u32(smem + kXsOff), peer);
        const uint32_t peer_ext = ptx::mapa_shared(ptx::smem_u32(smem + kExtraOff), peer);
        const uint32_t peer_xs_full = ptx::mapa_shared(ptx::smem_u32(&xs_full[0]), peer);
        const uint32_t peer_p_full = ptx::mapa_shared(ptx::smem_u32(&p_full[0]), peer);

        // P . V of tile gg has completed, observed through this CTA's P-buffer-free barrier.
        auto wait_pv = [&](int gg) -> bool {
            if (!__all_sync(0xffffffffu, ptx::mbar_wait(&pf_mine[gg % NP], (gg / NP) & 1, p.status))) return false;
            ptx::tc_fence_after();
            return true;
        };
        auto rescale = [&](float al) {
            for (int col = oc0; col < oc0 + ow; col += 16) {
                float v[16];
                ptx::tmem_ld16(t_row + kOCol + col, v);
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] *= al;
                tmem_st16(t_row + kOCol + col, v);
            }
            ptx::tmem_wait_st();
        };
        // Q share of segment number si: the latent units into TMEM columns [kQCol, kQCol + 32 nl),
        // the rope share into shared memory (the score product's A operand for the rope columns).
        auto load_q = [&](const Seg& s, int si) -> bool {
            if (si > 0 && !__all_sync(0xffffffffu, ptx::mbar_wait(&q_empty, (si - 1) & 1, p.status))) return false;
            ptx::tc_fence_after();
            const int t = s.w / p.HG, hg = s.w % p.HG;
            const bool have = hg * MH + row < p.h;
            const uint4* src = reinterpret_cast<const uint4*>(p.qtile + ((size_t)t * p.h + (have ? hg * MH + row : 0)) * p.R);
            for (int u = hk; u < 2 * sh.nl; u += 2) {
                const int gc = sh.lcol0 + 32 * u;
                uint32_t w[16];
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const uint4 x = have ? src[(gc >> 3) + v] : make_uint4(0, 0, 0, 0);
                    w[4 * v] = x.x; w[4 * v + 1] = x.y; w[4 * v + 2] = x.z; w[4 * v + 3] = x.w;
                }
                ptx::tmem_st16_u32(t_row + kQCol + 16 * u, w);
            }
            if (sh.rope_w > 0 && hk == 0) {
                // rows of 2 rope_w bytes in 8-row atoms; 16-byte chunk k of row r sits at chunk
                // k ^ (r / 2 % 4) (64-byte swizzle) or k ^ (r % 8) (128-byte swizzle)
                const int pitch = 2 * sh.rope_w;
                const int sw = sh.rope_w == 32 ? ((row >> 1) & 3) : (row & 7);
                unsigned char* qr = smem + kQrOff + (row >> 3) * (8 * pitch) + (row & 7) * pitch;
                for (int k = 0; k < pitch / 16; ++k) {
                    const int c8 = sh.rope_x + 8 * k;
                    const uint4 x = (have && c8 + 8 <= p.R) ? src[c8 >> 3] : make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4*>(qr + ((k ^ sw) << 4)) = x;
                }
                ptx::fence_proxy_async_smem();   // generic stores -> the score UMMA
            }
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&q_full);
            return true;
        };
        // Context (or partial context) of this warp's rows and O columns.
        auto epilogue = [&](const Seg& s, int g_last, float m_fin, float l_fin) -> bool {
            if (!wait_pv(g_last)) return false;
            const int t = s.w / p.HG, hg = s.w % p.HG;
            const int rows_valid = min(MH, p.h - hg * MH);
            const bool full = (s.j0 == 0 && s.j1 == s.n_w);
            if (full) {
                const float inv = l_fin > 0.f ? 1.f / l_fin : 0.f;
                bf16* dst = p.ctx + ((size_t)t * p.h + hg * MH + row) * p.L + sh.lcol0;
                for (int col = oc0; col < oc0 + ow; col += 16) {
                    float v[16];
                    ptx::tmem_ld16(t_row + kOCol + col, v);
                    uint32_t w[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) w[i] = pack_bf16x2(v[2 * i] * inv, v[2 * i + 1] * inv);
                    if (row < rows_valid) {
                        uint4* d4 = reinterpret_cast<uint4*>(dst + col);
                        d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
                        d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
                    }
                }
            } else {
                const int slot_id = 2 * c + (s.run_start ? 0 : 1);
                bf16* dst = p.part_o + ((size_t)slot_id * MH + row) * p.L + sh.lcol0;
                for (int col = oc0; col < oc0 + ow; col += 16) {
                    float v[16];
                    ptx::tmem_ld16(t_row + kOCol + col, v);
                    uint32_t w[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) w[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
                    uint4* d4 = reinterpret_cast<uint4*>(dst + col);
                    d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
                    d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
                }
                if (own && hk == 0) {
                    p.part_ml[((size_t)slot_id * 2 + 0) * MH + row] = m_fin;
                    p.part_ml[((size_t)slot_id * 2 + 1) * MH + row] = l_fin;
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&o_free);
            return true;
        };

        SegIter it;
        it.init(p, c, C);
        Seg sg;
        bool have = it.next(sg);
        int g = 0, si = 0;
        bool ok = have ? load_q(sg, 0) : true;
        if (own) {
            // ======== softmax of this CTA's heads
            const bool posts_tx = (q == 2 * (int)rank) && hk == 0 && lane == 0;
            while (ok && have) {
                const int t = sg.w / p.HG;
                const int nv = p.n_valid[t];
                float m_used = -INFINITY, lsum = 0.f, l_fin = 0.f;
                for (int j = sg.j0; ok && j < sg.j1; ++j, ++g) {
                    const int pb = g % NP, xb = g % NX;
                    const int cnt = min(KT, nv - j * KT);
                    const bool first = j == sg.j0, last = j == sg.j1 - 1;
                    // this CTA's partial scores of the row, this warp's half of the keys
                    ok = __all_sync(0xffffffffu, ptx::mbar_wait(&s_full[g & 1], (g >> 1) & 1, p.status));
                    if (!ok) break;
                    ptx::tc_fence_after();
                    float sv[KT / 2];
                    {
                        uint32_t raw[KT / 32][16];
#pragma unroll
                        for (int c16 = 0; c16 < KT / 2; c16 += 16)
                            ptx::tmem_ld16_nowait(t_row + kSCol + KT * (g & 1) + hk * (KT / 2) + c16, raw[c16 / 16]);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int k = 0; k < KT / 2; ++k) sv[k] = __uint_as_float(raw[k / 16][k % 16]);
                    }
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&s_free[g & 1]);
                    // + the peer's partial scores
                    if (posts_tx) ptx::mbar_arrive_expect_tx(&xs_full[xb], kXsBytes);
                    ok = __all_sync(0xffffffffu, ptx::mbar_wait_cluster(&xs_full[xb], (g / NX) & 1, p.status));
                    if (!ok) break;
                    const float4* xs = reinterpret_cast<const float4*>(smem + kXsOff + xb * kXsBytes);
#pragma unroll
                    for (int k4 = 0; k4 < KT / 8; ++k4) {
                        const float4 v = xs[(hk * (KT / 8) + k4) * HALF + lr];
                        sv[4 * k4] += v.x; sv[4 * k4 + 1] += v.y; sv[4 * k4 + 2] += v.z; sv[4 * k4 + 3] += v.w;
                    }
                    // tile max over the kept keys (base-2 units): this half's, then both halves'
                    // through shared memory, so that both warps of the quarter agree
                    float mh = -INFINITY;
#pragma unroll
                    for (int k = 0; k < KT / 2; ++k) {
                        sv[k] *= p.scale_log2;
                        if (hk * (KT / 2) + k < cnt) mh = fmaxf(mh, sv[k]);
                    }
                    m_x[g & 1][q & 1][hk][lane] = mh;
                    __syncwarp();   // the warp's writes precede lane 0's (release) arrival
                    if (lane == 0) ptx::mbar_arrive(&m_sync[q & 1]);
                    ok = __all_sync(0xffffffffu, ptx::mbar_wait(&m_sync[q & 1], g & 1, p.status));
                    if (!ok) break;
                    const float mt = fmaxf(mh, m_x[g & 1][q & 1][hk ^ 1][lane]);
                    float alpha = 1.f;   // factor applied to this head's running context
                    if (mt > m_used + kRescaleLog2) {
                        alpha = m_used != -INFINITY ? fast_exp2(m_used - mt) : 0.f;
                        m_used = mt;
                    }
                    const bool resc = __any_sync(0xffffffffu, alpha != 1.f);   // some head of this warp rescales
                    // P buffer pb free in both CTAs (their P . V of tile g - NP has completed)
                    const uint32_t fpar = ((g / NP) & 1) ^ 1;
                    ok = __all_sync(0xffffffffu, ptx::mbar_wait(&pf_mine[pb], fpar, p.status) &&
                                                     ptx::mbar_wait_cluster(&pf_peer[pb], fpar, p.status));
                    if (!ok) break;
                    // P = 2^(s - m) for this warp's half of the keys, bf16, K-major 128-byte swizzle,
                    // written to this CTA's buffer first (the local P . V needs only that and the
                    // peer's rows), then to the peer's
                    unsigned char* pl = smem + kPOff + pb * kPBytes;
                    const uint32_t pr = peer_p + pb * kPBytes;
                    const uint32_t pbar = peer_p_full + pb * 8;
                    uint32_t w[KT / 4];   // this warp's KT / 2 probabilities, two per word
                    float ps0 = 0.f, ps1 = 0.f;
                    auto exps = [&](auto full) {
#pragma unroll
                        for (int i = 0; i < KT / 2; i += 2) {
                            const int kk = hk * (KT / 2) + i;   // key within the tile
                            const float e0 = (decltype(full)::value || kk < cnt) ? fast_exp2(sv[i] - m_used) : 0.f;
                            const float e1 = (decltype(full)::value || kk + 1 < cnt) ? fast_exp2(sv[i + 1] - m_used) : 0.f;
                            ps0 += e0;
                            ps1 += e1;
                            w[i / 2] = pack_bf16x2(e0, e1);
                        }
                    };
                    if (cnt == KT) exps(std::true_type{});   // uniform: only an item's last tile is partial
                    else exps(std::false_type{});
                    const float psum = ps0 + ps1;
                    auto p_off = [&](int h8) {   // 16-byte chunk h8 (8 keys) of this warp's half of the row
                        const int key = hk * (KT / 2) + 8 * h8;
                        return (key >> 6) * (MH * 128) + row * 128 + ((((key & 63) >> 3) ^ (row & 7)) << 4);
                    };
#pragma unroll
                    for (int h8 = 0; h8 < KT / 16; ++h8)
                        *reinterpret_cast<uint4*>(pl + p_off(h8)) = make_uint4(w[4 * h8], w[4 * h8 + 1], w[4 * h8 + 2], w[4 * h8 + 3]);
                    lsum = lsum * alpha + psum;
                    ptx::fence_proxy_async_smem();       // local P rows -> this CTA's UMMA
                    // Rescale this CTA's O rows of these heads once the previous P . V is done.
                    // These warps learn of P . V completions through pf_mine, which they
                    // wait on for every tile in order (here early, for tile g - 1, only when a
                    // rescale is due; the wait for the buffer's reuse two tiles on then
                    // finds that phase complete).
                    if (!first && resc) {
                        ok = wait_pv(g - 1);
                        if (!ok) break;
                        rescale(alpha);
                    }
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&p_ready[pb]);
                    // the peer's copy of the rows and {alpha, m, l0, l1} of the head (16 bytes per head)
#pragma unroll
                    for (int h8 = 0; h8 < KT / 16; ++h8)
                        ptx::st_async_v4(pr + p_off(h8), w[4 * h8], w[4 * h8 + 1], w[4 * h8 + 2], w[4 * h8 + 3], pbar);
                    const uint32_t pe = peer_ext + pb * kExtraBytes + row * 16;
                    if (hk == 0) {
                        ptx::st_async_v2(pe, __float_as_uint(alpha), __float_as_uint(m_used), pbar);
                        ptx::st_async_u32(pe + 8, __float_as_uint(lsum), pbar);
                    } else {
                        ptx::st_async_u32(pe + 12, __float_as_uint(lsum), pbar);
                    }
                    if (lane == 0)
                        ptx::st_async_u32(peer_ext + pb * kExtraBytes + kFlagOff + 4 * (2 * (q & 1) + hk), resc ? 1u : 0u,
                                          pbar);
                    if (last) {   // the two warps of the quarter add up their key halves
                        l_x[si & 1][q & 1][hk][lane] = lsum;
                        __syncwarp();
                        if (lane == 0) ptx::mbar_arrive(&l_sync[q & 1]);
                        ok = __all_sync(0xffffffffu, ptx::mbar_wait(&l_sync[q & 1], si & 1, p.status));
                        if (!ok) break;
                        l_fin = lsum + l_x[si & 1][q & 1][hk ^ 1][lane];
                    }
                }
                if (!ok) break;
                Seg nsg;
                const bool nh = it.next(nsg);
                if (nh) {
                    ok = load_q(nsg, si + 1);
                    if (!ok) break;
                }
                ok = epilogue(sg, g - 1, m_used, l_fin);
                sg = nsg;
                have = nh;
                ++si;
            }
        } else {
            // ======== the peer's heads: ship partial scores, take the peer's rescale factors.
            // The factors of tile g are taken after the scores of tile g + 1 have gone out.
            auto ship = [&](int gg) -> bool {
                const int xb = gg % NX;
                if (!__all_sync(0xffffffffu, ptx::mbar_wait(&s_full[gg & 1], (gg >> 1) & 1, p.status))) return false;
                ptx::tc_fence_after();
                float sv[KT / 2];
                {
                    uint32_t raw[KT / 32][16];
#pragma unroll
                    for (int c16 = 0; c16 < KT / 2; c16 += 16)
                        ptx::tmem_ld16_nowait(t_row + kSCol + KT * (gg & 1) + hk * (KT / 2) + c16, raw[c16 / 16]);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < KT / 2; ++k) sv[k] = __uint_as_float(raw[k / 16][k % 16]);
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&s_free[gg & 1]);
                const uint32_t dst = peer_xs + xb * kXsBytes;
                const uint32_t bar = peer_xs_full + xb * 8;
#pragma unroll
                for (int k4 = 0; k4 < KT / 8; ++k4) {
                    const int key4 = hk * (KT / 8) + k4;
                    ptx::st_async_v4(dst + (key4 * HALF + lr) * 16, __float_as_uint(sv[4 * k4]),
                                     __float_as_uint(sv[4 * k4 + 1]), __float_as_uint(sv[4 * k4 + 2]),
                                     __float_as_uint(sv[4 * k4 + 3]), bar);
                }
                return true;
            };
            // Tile gg's P rows and factors from the peer: keep the head's final (max, sum) and,
            // when the peer flagged a rescale, rescale this CTA's O rows of these heads after
            // P . V of tile gg - 1 and report it (the P . V issuer waits for that only then).
            auto finish = [&](int gg, bool first, bool last, float& m_fin, float& l_fin) -> bool {
                const int pb = gg % NP;
                if (!__all_sync(0xffffffffu, ptx::mbar_wait_cluster(&p_full[pb], (gg / NP) & 1, p.status)))
                    return false;
                const unsigned char* ext = smem + kExtraOff + pb * kExtraBytes;
                const float4 ex = *reinterpret_cast<const float4*>(ext + row * 16);
                const uint4 fl = *reinterpret_cast<const uint4*>(ext + kFlagOff);
                if (last) {
                    m_fin = ex.y;
                    l_fin = ex.z + ex.w;
                }
                // P . V completions are observed tile by tile, in order
                if (gg > 0 && !wait_pv(gg - 1)) return false;
                if (!first && (fl.x | fl.y | fl.z | fl.w)) {
                    rescale(ex.x);
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&corr_done);
                }
                return true;
            };
            bool have_prev = false, prev_first = false, prev_last = false;
            int g_prev = 0;
            Seg s_prev = sg;
            float m_prev = 0.f, l_prev = 0.f;
            while (ok && have) {
                for (int j = sg.j0; ok && j < sg.j1; ++j, ++g) {
                    ok = ship(g);
                    if (!ok) break;
                    if (have_prev) {
                        ok = finish(g_prev, prev_first, prev_last, m_prev, l_prev);
                        if (ok && prev_last) ok = epilogue(s_prev, g_prev, m_prev, l_prev);
                        if (!ok) break;
                    }
                    have_prev = true;
                    g_prev = g;
                    s_prev = sg;
                    prev_first = j == sg.j0;
                    prev_last = j == sg.j1 - 1;
                }
                if (!ok) break;
                Seg nsg;
                const bool nh = it.next(nsg);
                if (nh) ok = load_q(nsg, si + 1);
                sg = nsg;
                have = nh;
                ++si;
            }
            if (ok && have_prev) {
                ok = finish(g_prev, prev_first, prev_last, m_prev, l_prev);
                if (ok) ok = epilogue(s_prev, g_prev, m_prev, l_prev);
            }
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync_all();   // no remote store or arrival may target an exited peer
    if (warp == kScoreWarp) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}


// Work plan as its own kernel (the separate attention entry point; the fused step
// computes it in an extra block of the q / kv fold).
__global__ void __launch_bounds__(1024)
k_core_plan(const int32_t* __restrict__ n_valid, int T, int HG, int max_clusters, int32_t* __restrict__ base,
            int4* __restrict__ desc) {
    griddep_launch();   // dependents may start; they wait for this kernel
    griddep_wait();     // the previous kernel of the stream has completed
    plan_items(n_valid, T, HG, max_clusters, base, desc);
}

// Merge the partial contexts of items split between cluster runs; zero-fill
// items with no kept key. Items finished in place are left alone.
//   ctx[r] = sum_c 2^(m_c[r] - M[r]) O_c[r] / sum_c 2^(m_c[r] - M[r]) l_c[r],  M = max_c m_c
// Blocks are indexed by run boundary, not by item: run cb starts at unit
// floor(U cb / C), and an item is split exactly when a boundary falls strictly
// inside it, so at most C - 1 items need a merge. The first boundary inside an
// item merges it (kSlices blocks of kCombineRows head rows each); every block
// also zero-fills the empty items of its stride.
constexpr int kMaxParts = 80;
constexpr int kCombineRows = 8;                      // head rows per combine block: one warp per row
constexpr int kCombineThreads = 32 * kCombineRows;
constexpr int kCombineVecs = 512 / 8 / 32;           // 8-element vectors per lane (L <= 512)

__global__ void __launch_bounds__(kCombineThreads)
k_core_combine(Params p) {
    griddep_launch();   // dependents may start; they wait for this kernel
    griddep_wait();     // the previous kernel of the stream has completed
    __shared__ float scale[kMaxParts][kCombineRows];
    __shared__ float lsum[kMaxParts][kCombineRows];
    __shared__ int sid[kMaxParts];
    constexpr int kSlices = MH / kCombineRows;
    const int tid = threadIdx.x, lane = tid & 31, rr = tid >> 5;   // warp rr owns head row r0 + rr
    const int cb = blockIdx.x / kSlices + 1;                         // boundary between runs cb - 1 and cb
    const int r0 = (blockIdx.x % kSlices) * kCombineRows;
    const int vec_per_row = p.L / 8;
    // this boundary's merge plan (item, parts, first slot) from the plan kernel
    const int4 ds = p.merge_desc[cb];
    const int w = ds.x;
    const int hg = w >= 0 ? w % p.HG : 0;
    const int rows = min(kCombineRows, min(MH, p.h - hg * MH) - r0);
    if (w >= 0 && rows > 0) {
        bf16* ctx = p.ctx + ((size_t)(w / p.HG) * p.h + hg * MH + r0 + rr) * p.L;
        const int cf = cb - 1, np = ds.y;   // runs cf .. cf + np - 1 hold the item's parts
        for (int k = tid; k < np; k += blockDim.x) sid[k] = 2 * (cf + k) + (k == 0 ? ds.z : 0);
        __syncthreads();
        const bool row_ok = rr < rows;
        auto load_part = [&](int k, uint4 (&v)[kCombineVecs]) {
            const uint4* src = reinterpret_cast<const uint4*>(p.part_o + ((size_t)sid[k] * MH + r0 + rr) * p.L);
#pragma unroll
            for (int u = 0; u < kCombineVecs; ++u) {
                const int cv = lane + 32 * u;
                if (row_ok && cv < vec_per_row) v[u] = src[cv];
            }
        };
        // contexts of the first two parts and every part's (m, l) in one round of loads
        uint4 va[kCombineVecs], vb[kCombineVecs];
        load_part(0, va);
        load_part(1, vb);
        for (int q = tid; q < np * kCombineRows; q += blockDim.x) {
            const int k = q / kCombineRows, r = q % kCombineRows;
            if (r < rows) {
                const float* ml = p.part_ml + (size_t)sid[k] * 2 * MH + r0 + r;
                scale[k][r] = ml[0];
                lsum[k][r] = ml[MH];
            }
        }
        __syncthreads();
        if (tid < rows) {
            float m = -INFINITY;
            for (int k = 0; k < np; ++k) m = fmaxf(m, scale[k][tid]);
            float l = 0.f;
            for (int k = 0; k < np; ++k) {
                const float e = exp2f(scale[k][tid] - m);
                scale[k][tid] = e;
                l += e * lsum[k][tid];
            }
            const float inv = l > 0.f ? 1.f / l : 0.f;
            for (int k = 0; k < np; ++k) scale[k][tid] *= inv;
        }
        __syncthreads();
        if (row_ok) {
            float acc[kCombineVecs][8];
#pragma unroll
            for (int u = 0; u < kCombineVecs; ++u)
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[u][e] = 0.f;
            auto add_part = [&](int k, const uint4 (&v)[kCombineVecs]) {
                const float sc = scale[k][rr];
#pragma unroll
                for (int u = 0; u < kCombineVecs; ++u) {
                    if (lane + 32 * u >= vec_per_row) continue;
                    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v[u]);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(h2[e]);
                        acc[u][2 * e] += sc * f.x;
                        acc[u][2 * e + 1] += sc * f.y;
                    }
                }
            };
            add_part(0, va);
            add_part(1, vb);
            for (int k = 2; k < np; k += 2) {   // items spread over more than two runs
                load_part(k, va);
                if (k + 1 < np) load_part(k + 1, vb);
                add_part(k, va);
                if (k + 1 < np) add_part(k + 1, vb);
            }
            uint4* dst = reinterpret_cast<uint4*>(ctx);
#pragma unroll
            for (int u = 0; u < kCombineVecs; ++u) {
                const int cv = lane + 32 * u;
                if (cv >= vec_per_row) continue;
                uint4 o;
                uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                for (int e = 0; e < 4; ++e) ow[e] = pack_bf16x2(acc[u][2 * e], acc[u][2 * e + 1]);
                dst[cv] = o;
            }
        }
    }
    // empty items (no kept key) of this block's stride: zero context rows
    for (int we = cb - 1; we < p.W; we += p.max_clusters) {
        if (p.item_base[we] != p.item_base[we + 1]) continue;
        const int hge = we % p.HG;
        if (rr >= min(kCombineRows, min(MH, p.h - hge * MH) - r0)) continue;
        uint4* dst = reinterpret_cast<uint4*>(p.ctx + ((size_t)(we / p.HG) * p.h + hge * MH + r0 + rr) * p.L);
        for (int cv = lane; cv < vec_per_row; cv += 32) dst[cv] = make_uint4(0, 0, 0, 0);
    }
}

}  // namespace core

int core_tc_head_groups(const Dims& d) { return d.h <= core::MH ? 1 : d.h / core::MH; }

bool core_tc_supports(const Dims& d) {
    return d.L % 64 == 0 && d.L >= 64 && d.L <= 512 && d.dr % 16 == 0 && d.dr >= 16 && d.dr <= 64 &&
           (d.h <= core::MH || d.h % core::MH == 0);
}

namespace {

// Dynamic shared memory a block may request (the opt-in limit less the kernel's static part).
int core_dyn_smem_limit() {
    static int cached = -1;
    if (cached > 0) return cached;
    cudaFuncAttributes a = {};
    int lim = core::kSmemPerBlock - 2048;
    if (cudaFuncGetAttributes(&a, core::k_core_tc) == cudaSuccess) lim = core::kSmemPerBlock - (int)a.sharedSizeBytes;
    cached = lim;
    return lim;
}

// Column shares of the two CTAs and their stage rings.
void make_shares(const Dims& d, core::Share* sh) {
    using namespace core;
    const int nv = d.L / 64;
    sh[0].nl = (nv + 1) / 2;
    sh[1].nl = nv - sh[0].nl;
    sh[0].lcol0 = 0;
    sh[1].lcol0 = 64 * sh[0].nl;
    if (d.dr == 64 && sh[0].nl == sh[1].nl) {   // rope halves, 64-byte rows
        for (int r = 0; r < 2; ++r) {
            sh[r].rope_x = d.L + 32 * r;
            sh[r].rope_w = 32;
        }
    } else {                                    // whole rope part (one 64-column box) to the lighter CTA
        const int rr = sh[1].nl < sh[0].nl ? 1 : 0;
        sh[rr].rope_x = d.L;
        sh[rr].rope_w = 64;
        sh[1 - rr].rope_x = 0;
        sh[1 - rr].rope_w = 0;
    }
    // both CTAs place their stages after the larger rope share (identical offsets in the pair)
    const int qr_bytes = (MH * 2 * (sh[0].rope_w > sh[1].rope_w ? sh[0].rope_w : sh[1].rope_w) + 1023) / 1024 * 1024;
    const int budget = core_dyn_smem_limit() - 1024 - kQrOff - qr_bytes;
    for (int r = 0; r < 2; ++r) {
        sh[r].qr_bytes = qr_bytes;
        sh[r].stage_off = kQrOff + qr_bytes;
        sh[r].stage_tx = sh[r].nl * kBlockBytes + KT * sh[r].rope_w * 2;
        sh[r].stage_bytes = (sh[r].stage_tx + 1023) / 1024 * 1024;
        int ns = budget / sh[r].stage_bytes;
        sh[r].ns = ns > kMaxStages ? kMaxStages : ns;
    }
}

int core_dyn_smem_bytes(const core::Share* sh) {
    int m = 0;
    for (int r = 0; r < 2; ++r) {
        const int b = sh[r].ns * sh[r].stage_bytes;
        if (b > m) m = b;
    }
    return 1024 + sh[0].stage_off + m;
}

}  // namespace

int core_tc_max_clusters() {
    static int cached = -1;
    if (cached > 0) return cached;
    const int smem = core_dyn_smem_limit();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * 148, 1, 1);
    cfg.blockDim = dim3(core::kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    int n = 0;
    if (cudaFuncSetAttribute(core::k_core_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
        cudaOccupancyMaxActiveClusters(&n, core::k_core_tc, &cfg) != cudaSuccess || n <= 0) {
        int dev = 0, sms = 148;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        n = sms / 2;
    }
    cached = n;
    return n;
}

int core_tc_cluster_bound(const Dims& d) {
    const long long hg = d.h <= core::MH ? 1 : d.h / core::MH;
    const long long u_max = (long long)d.T * hg * ((d.P + core::KT - 1) / core::KT);
    long long c = u_max / core::kMinTilesPerCluster;
    if (c < 1) c = 1;
    if (c > kCoreMaxClusters) c = kCoreMaxClusters;   // <= core::kMaxParts
    return (int)c;
}

size_t core_tc_partial_bytes(const Dims& d, int max_clusters) {
    return (size_t)2 * max_clusters * core::MH * d.L * sizeof(bf16);
}
int4* core_tc_merge_desc(float* part_ml, int max_clusters) {
    return reinterpret_cast<int4*>(part_ml + (size_t)2 * max_clusters * 2 * core::MH);
}

size_t core_tc_ml_bytes(int max_clusters) {   // (m, l) of the partials, then the merge plan
    return (size_t)2 * max_clusters * 2 * core::MH * sizeof(float) + (size_t)(max_clusters + 1) * sizeof(int4);
}

cudaError_t launch_core_tc(const bf16* qtile, const bf16* kv_cache, const int32_t* rows, const int32_t* n_valid,
                           int32_t* item_base, const Dims& d, float scale, bf16* ctx, bf16* part_o, float* part_ml,
                           int max_clusters, bool plan_done, int32_t* status, cudaStream_t s) {
    using namespace core;
    const int HG = d.h <= MH ? 1 : d.h / MH;
    const int W = d.T * HG;
    // the plan evaluates run starts U * c / C in 32 bits
    if ((long long)W * ((d.P + KT - 1) / KT) * max_clusters >= (1LL << 31)) return cudaErrorInvalidValue;
    int4* merge_desc = core_tc_merge_desc(part_ml, max_clusters);
    cudaError_t e = cudaSuccess;
    if (!plan_done) {
        e = launch_pdl(k_core_plan, dim3(1), dim3(1024), 0, s, n_valid, d.T, HG, max_clusters, item_base, merge_desc);
        if (e != cudaSuccess) return e;
    }
    Params p;
    p.rows = rows;
    p.n_valid = n_valid;
    p.item_base = item_base;
    p.qtile = qtile;
    p.T = d.T;
    p.h = d.h;
    p.HG = HG;
    p.P = d.P;
    p.L = d.L;
    p.R = d.R();
    p.W = W;
    p.max_clusters = max_clusters;
    p.scale_log2 = scale * 1.4426950408889634f;
    make_shares(d, p.share);
    if (p.share[0].ns < 2 || p.share[1].ns < 2) return cudaErrorInvalidConfiguration;
    p.ctx = ctx;
    p.part_o = part_o;
    p.part_ml = part_ml;
    p.merge_desc = merge_desc;
    p.status = status;
    CUtensorMap t128, t64;
    if (!make_tma_2d(&t128, kv_cache, (uint64_t)d.R(), (uint64_t)d.n_rows(), (uint64_t)d.R() * 2, 64, 1, 128) ||
        !make_tma_2d(&t64, kv_cache, (uint64_t)d.R(), (uint64_t)d.n_rows(), (uint64_t)d.R() * 2, 32, 1, 64))
        return cudaErrorInvalidValue;
    const int smem = core_dyn_smem_bytes(p.share);
    {
        constexpr int kMaxDevices = 64;
        static bool attr_set[kMaxDevices] = {};   // function attributes are per device
        int dev = 0;
        cudaGetDevice(&dev);
        if (dev < 0 || dev >= kMaxDevices || !attr_set[dev]) {
            e = cudaFuncSetAttribute(k_core_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, core_dyn_smem_limit());
            if (e != cudaSuccess) return e;
            if (dev >= 0 && dev < kMaxDevices) attr_set[dev] = true;
        }
    }
    // Programmatic launch in graphs too: the clusters set up their barriers and TMEM on the SMs
    // the query chain leaves idle, and the merge's blocks are ready when the clusters finish
    // (measured on B200: 2-4 us per step on gather128; kernels that only wait at their start
    // gain nothing from it).
    e = launch_pdl_mode(true, k_core_tc, dim3(2 * max_clusters), dim3(kThreads), smem, s, t128, t64, p);
    if (e != cudaSuccess) return e;
    return launch_pdl_mode(true, k_core_combine, dim3(max_clusters * (MH / kCombineRows)), dim3(kCombineThreads), 0, s, p);
}

}  // namespace mla
