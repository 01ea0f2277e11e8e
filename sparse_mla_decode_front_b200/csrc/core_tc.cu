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
// TMEM holds 512 fp32 columns per SM; the latent context of 128 heads is
// 128 x 512 fp32 and fills it. So each work unit runs on a 2-CTA cluster:
//   rank 0 (S-CTA): Q in TMEM (loaded once per work item), key rows gathered
//       into shared memory 64 columns at a time (8 stages), S = Q K^T for 128
//       keys per tile into TMEM, fp32 online softmax (one thread per head,
//       base-2 exponent, lazy rescale: the running max only moves when a tile
//       exceeds it by 2^8), bf16 P staged in shared memory and shipped to the
//       O-CTA with one bulk DSMEM copy per tile;
//   rank 1 (O-CTA): the latent part of the same rows gathered 32 keys at a
//       time (4 stages), O += P V into the 512-column TMEM accumulator, O
//       rescaled in TMEM on the rare tiles that moved the max, O written out.
// Rows are gathered by TMA (tile::gather4, four rows x 64 columns per
// instruction) straight into the 128-byte-swizzled layout the UMMA reads;
// four producer warps per CTA issue them concurrently (one warp alone cannot
// keep the gather rate up). The O-CTA runs ahead and pulls the rows from HBM;
// the S-CTA reads the same rows back from L2.
//
// Work split: tiles of 128 kept keys; all (item, tile) pairs are laid out item
// by item and each cluster takes a contiguous run (stream-K). An item fully
// inside one run is finished in place; an item split between runs leaves
// bf16 partial contexts with their (max, sum), merged by k_core_combine.
#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace mla {
namespace core {

constexpr int KT = 128;           // keys per tile (N of S = Q K^T)
constexpr int MH = 128;           // heads per work item (UMMA M)
constexpr int kWarps = 14;        // 0-3 (+8-11 in the S-CTA) softmax | correction+epilogue,
                                  // 4 UMMA + TMEM, 5-7 and 12 producers, 13 P copy
constexpr int kThreads = 32 * kWarps;
constexpr int NSK = 8;            // S-CTA key stages: [128 keys x 64 columns]
constexpr int NSV = 4;            // O-CTA value stages: [128 keys x 128 latent columns]
constexpr int NP = 2;             // P buffers (staging in the S-CTA, slots in the O-CTA)
constexpr int kMinTilesPerCluster = 2;
constexpr float kRescaleLog2 = 8.f;
constexpr int kKStageBytes = KT * 128;              // 16 KB
constexpr int kPBytes = MH * KT * 2;                // 32 KB: two [128 rows x 128 B] blocks, 128-byte swizzle
constexpr int kPExtra = 4 * MH * 4;                 // alpha, final max, final sum of each key half
constexpr int kPBufBytes = kPBytes + kPExtra;       // bytes of one bulk copy
constexpr int kPBufStride = (kPBufBytes + 1023) / 1024 * 1024;
constexpr int kSCol = 384;                          // S tile columns in the S-CTA's TMEM (Q uses [0, R/2))

struct Params {
    const int32_t* rows;        // [T, P] kept rows, compacted
    const int32_t* n_valid;     // [T]
    const int32_t* item_base;   // [W + 1] first tile of each item
    const bf16* kv_cache;       // [n_rows, R]
    const bf16* qtile;          // [T * h, R]
    int T, h, HG, P, L, R, n_kblk, n_vblk, W, max_clusters;
    float scale_log2;           // softmax_scale * log2(e)
    bf16* ctx;                  // [T, h, L]
    bf16* part_o;               // [2 * max_clusters, 128, L]
    float* part_ml;             // [2 * max_clusters, 2, 128]  (max in log2 units, sum)
    int32_t* status;
};

// Dynamic shared-memory layout (offsets from a 1024-aligned base). Both ranks
// put their P buffers at the same offset so the S-CTA's staging buffer b maps
// onto the O-CTA's slot b.
struct Layout {
    int stages, pbuf, total;
    __host__ __device__ Layout(int n_kblk, int n_vblk) {
        const int s_stage = NSK * kKStageBytes;
        const int o_stage = NSV * 2 * kKStageBytes;
        stages = 0;
        pbuf = s_stage > o_stage ? s_stage : o_stage;
        total = pbuf + NP * kPBufStride + 1024;
        (void)n_kblk;
    }
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

__host__ __device__ __forceinline__ int clusters_for(int U, int max_clusters) {
    const int c = U / kMinTilesPerCluster;
    return c < 1 ? 1 : (c > max_clusters ? max_clusters : c);
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
    uint32_t u[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) u[i] = __float_as_uint(v[i]);
    ptx::tmem_st16_u32(taddr, u);
    ptx::tmem_wait_st();
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

// Kept-row id number k (clamped to the last kept row) of item token t.
__device__ __forceinline__ int kept_row(const Params& p, int t, int nv, int k) {
    return p.rows[(size_t)t * p.P + min(k, nv - 1)];
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
k_core_tc(const __grid_constant__ CUtensorMap tma_kv, Params p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // Barriers sit at identical offsets in both ranks (remote arrivals rely on it).
    __shared__ __align__(8) uint64_t kf[NSK], ke[NSK], s_full, s_empty, q_full, q_empty, stg_ready[NP], stg_free[NP];
    __shared__ __align__(8) uint64_t vf[NSV], ve[NSV], p_full[NP], p_empty[NP], p_ready[NP];
    __shared__ __align__(8) uint64_t o_done[2], o_free, mma_done;
    __shared__ uint32_t tmem_slot;

    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const Layout lay(p.n_kblk, p.n_vblk);
    const uint32_t rank = ptx::cluster_ctarank();
    const int c = (int)ptx::cluster_id_x();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int U = p.item_base[p.W];
    const int C = clusters_for(U, p.max_clusters);
    const bool active = c < C;
    constexpr uint32_t kTmemCols = 512;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NSK; ++i) { ptx::mbar_init(&kf[i], 1); ptx::mbar_init(&ke[i], 1); }
        ptx::mbar_init(&s_full, 1);
        ptx::mbar_init(&s_empty, 8);
        ptx::mbar_init(&q_full, 8);
        ptx::mbar_init(&q_empty, 1);
        for (int i = 0; i < NP; ++i) {
            ptx::mbar_init(&stg_ready[i], 8);
            ptx::mbar_init(&stg_free[i], 1);
            ptx::mbar_init(&p_full[i], 1);     // remote arrive.expect_tx + the bulk copy's bytes
            ptx::mbar_init(&p_empty[i], 1);    // O-CTA UMMA commit (multicast into the S-CTA)
            ptx::mbar_init(&p_ready[i], 4);    // O-CTA correction warps
        }
        for (int i = 0; i < NSV; ++i) { ptx::mbar_init(&vf[i], 1); ptx::mbar_init(&ve[i], 1); }
        for (int i = 0; i < 2; ++i) ptx::mbar_init(&o_done[i], 1);
        ptx::mbar_init(&o_free, 4);
        ptx::mbar_init(&mma_done, 1);
        ptx::fence_mbar_init();
        ptx::tma_prefetch_desc(&tma_kv);
    }
    if (warp == 4) {
        ptx::tmem_alloc(&tmem_slot, kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync_all();   // peer barriers initialised before any remote arrival
    ptx::tc_fence_after();
    const uint32_t tmem = tmem_slot;

    if (active && rank == 0) {
        // =========================== S-CTA ===========================
        if ((warp >= 5 && warp <= 7) || warp == 12) {
            // ---- producers: key rows, 64 columns per stage; warp pw gathers rows 32pw..32pw+31
            const int pw = warp == 12 ? 3 : warp - 5;
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
                    const int my_row = kept_row(p, t, nv, j * KT + pw * 32 + lane);
                    const int r0 = __shfl_sync(0xffffffffu, my_row, (lane & 7) * 4 + 0);
                    const int r1 = __shfl_sync(0xffffffffu, my_row, (lane & 7) * 4 + 1);
                    const int r2 = __shfl_sync(0xffffffffu, my_row, (lane & 7) * 4 + 2);
                    const int r3 = __shfl_sync(0xffffffffu, my_row, (lane & 7) * 4 + 3);
                    for (int cb = 0; cb < p.n_kblk; ++cb) {
                        ok = __all_sync(0xffffffffu, ptx::mbar_wait(&ke[stage], ph ^ 1, p.status));
                        if (!ok) break;
                        if (pw == 0 && lane == 0) ptx::mbar_arrive_expect_tx(&kf[stage], kKStageBytes);
                        if (lane < 8)
                            ptx::tma_gather4(smem + lay.stages + stage * kKStageBytes + (pw * 32 + lane * 4) * 128,
                                             &tma_kv, &kf[stage], 64 * cb, r0, r1, r2, r3);
                        ++n_issued;
                        if (++stage == NSK) { stage = 0; ph ^= 1; }
                    }
                }
            }
            // loads already issued land before shared memory is released
            if (lane == 0)
                for (int i = 0; i < NSK && i < n_issued; ++i) {
                    if (--stage < 0) { stage = NSK - 1; ph ^= 1; }
                    ptx::mbar_wait(&kf[stage], ph, nullptr);
                }
        } else if (warp == 4) {
            // ---- UMMA: S = Q K^T with Q in TMEM
            if (lane == 0) {
                constexpr uint32_t idesc = ptx::idesc_bf16(MH, KT, false, false);
                const int ksteps = p.R / 16;
                SegIter it;
                it.init(p, c, C);
                Seg sg;
                int stage = 0;
                uint32_t ph = 0, qf_ph = 0, se_ph = 0;
                bool ok = true;
                while (ok && it.next(sg)) {
                    ok = ptx::mbar_wait(&q_full, qf_ph, p.status);
                    qf_ph ^= 1;
                    ptx::tc_fence_after();
                    for (int j = sg.j0; ok && j < sg.j1; ++j) {
                        ok = ptx::mbar_wait(&s_empty, se_ph ^ 1, p.status);
                        se_ph ^= 1;
                        ptx::tc_fence_after();
                        for (int cb = 0; ok && cb < p.n_kblk; ++cb) {
                            ok = ptx::mbar_wait(&kf[stage], ph, p.status);
                            if (!ok) break;
                            ptx::tc_fence_after();
                            const uint32_t k_addr = ptx::smem_u32(smem + lay.stages + stage * kKStageBytes);
                            for (int kk = 0; kk < 4; ++kk) {
                                const int ks = cb * 4 + kk;
                                if (ks >= ksteps) break;
                                const uint64_t bd = ptx::sdesc_sw128(k_addr + kk * 32, 16, 1024);
                                ptx::umma_bf16_ts(tmem + kSCol, tmem + ks * 8, bd, idesc, ks > 0 ? 1u : 0u);
                            }
                            ptx::umma_commit(&ke[stage]);
                            if (++stage == NSK) { stage = 0; ph ^= 1; }
                        }
                        if (ok) ptx::umma_commit(&s_full);
                    }
                    ptx::umma_commit(&q_empty);
                }
                ptx::umma_commit(&mma_done);
                ptx::mbar_wait(&mma_done, 0, p.status);
            }
        } else if (warp == 13) {
            // ---- P copy: staging buffer b -> O-CTA slot b, one bulk copy per tile
            if (lane == 0) {
                const uint32_t peer_pbuf = ptx::mapa_shared(ptx::smem_u32(smem + lay.pbuf), 1);
                const uint32_t peer_pfull = ptx::mapa_shared(ptx::smem_u32(&p_full[0]), 1);
                SegIter it;
                it.init(p, c, C);
                Seg sg;
                int g = 0;
                uint32_t sr_ph[NP] = {0, 0}, pe_ph[NP] = {0, 0};
                bool ok = true;
                while (ok && it.next(sg)) {
                    for (int j = sg.j0; ok && j < sg.j1; ++j, ++g) {
                        const int b = g & 1;
                        ok = ptx::mbar_wait(&stg_ready[b], sr_ph[b], p.status);
                        sr_ph[b] ^= 1;
                        if (ok) ok = ptx::mbar_wait_cluster(&p_empty[b], pe_ph[b] ^ 1, p.status);
                        pe_ph[b] ^= 1;
                        if (!ok) break;
                        ptx::mbar_arrive_expect_tx_remote(peer_pfull + b * 8, kPBufBytes);
                        ptx::bulk_copy_to_peer(peer_pbuf + b * kPBufStride, smem + lay.pbuf + b * kPBufStride,
                                               kPBufBytes, peer_pfull + b * 8);
                        ptx::bulk_commit_group();
                        if (g > 0) {   // the previous tile's copy has finished reading its staging buffer
                            ptx::bulk_wait_group_read<1>();
                            ptx::mbar_arrive(&stg_free[b ^ 1]);
                        }
                    }
                }
                ptx::bulk_wait_group_read<0>();
            }
        } else if (warp < 4 || (warp >= 8 && warp <= 11)) {
            // ---- softmax: thread = head row r; warps w and w+8 share the rows of TMEM
            //      quarter w and exponentiate keys [0, 64) and [64, 128) respectively.
            const int quarter = warp & 3, half = warp >= 8 ? 1 : 0;
            const int r = quarter * 32 + lane;
            const uint32_t t_row = tmem + ((uint32_t)(quarter * 32) << 16);
            SegIter it;
            it.init(p, c, C);
            Seg sg;
            uint32_t sf_ph = 0, qe_ph = 0, sfree_ph[NP] = {0, 0};
            int g = 0;
            bool ok = true;
            while (ok && it.next(sg)) {
                const int t = sg.w / p.HG, hg = sg.w % p.HG;
                const int nv = p.n_valid[t];
                // Q rows of this item into TMEM columns [0, R/2) (two bf16 per column, low half first);
                // each of the two warps of a quarter loads half of the columns.
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(&q_empty, qe_ph ^ 1, p.status));
                qe_ph ^= 1;
                if (!ok) break;
                ptx::tc_fence_after();
                {
                    const long long qrow = (long long)t * p.h + hg * MH + r;
                    const bool have = qrow < (long long)p.T * p.h;
                    const uint4* src = reinterpret_cast<const uint4*>(p.qtile + (have ? qrow : 0) * p.R);
                    for (int col = half * 16; col < p.R / 2; col += 32) {
                        uint32_t w[16];
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            const int vi = (col >> 2) + v;   // 16-byte piece of the row (R / 8 of them)
                            const uint4 x = (have && vi < p.R / 8) ? src[vi] : make_uint4(0, 0, 0, 0);
                            w[4 * v] = x.x; w[4 * v + 1] = x.y; w[4 * v + 2] = x.z; w[4 * v + 3] = x.w;
                        }
                        ptx::tmem_st16_u32(t_row + col, w);
                    }
                    ptx::tmem_wait_st();
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&q_full);
                float m_used = -INFINITY, lsum = 0.f;
                for (int j = sg.j0; j < sg.j1; ++j, ++g) {
                    const int b = g & 1;
                    ok = __all_sync(0xffffffffu, ptx::mbar_wait(&s_full, sf_ph, p.status));
                    sf_ph ^= 1;
                    if (!ok) break;
                    ptx::tc_fence_after();
                    const int cnt = min(KT, nv - j * KT);
                    // tile max over all 128 keys (base-2 units); both warps of a quarter agree
                    float mt = -INFINITY;
                    for (int col = 0; col < KT; col += 16) {
                        float v[16];
                        ptx::tmem_ld16(t_row + kSCol + col, v);
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (col + i < cnt) mt = fmaxf(mt, v[i] * p.scale_log2);
                    }
                    float alpha = 1.f;   // factor the O-CTA applies to this head's running context
                    if (mt > m_used + kRescaleLog2) {
                        alpha = m_used != -INFINITY ? fast_exp2(m_used - mt) : 0.f;
                        m_used = mt;
                    }
                    // staging buffer b free (its previous copy has read it)
                    ok = __all_sync(0xffffffffu, ptx::mbar_wait(&stg_free[b], sfree_ph[b] ^ 1, p.status));
                    sfree_ph[b] ^= 1;
                    if (!ok) break;
                    unsigned char* stg = smem + lay.pbuf + b * kPBufStride;
                    // P = 2^(s - m) for this warp's 64 keys, packed bf16, K-major 128-byte swizzle
                    float psum = 0.f;
                    for (int col = half * 64; col < half * 64 + 64; col += 16) {
                        float v[16];
                        ptx::tmem_ld16(t_row + kSCol + col, v);
                        uint32_t w[8];
#pragma unroll
                        for (int i = 0; i < 16; i += 2) {
                            const float e0 = (col + i < cnt) ? fast_exp2(v[i] * p.scale_log2 - m_used) : 0.f;
                            const float e1 = (col + i + 1 < cnt) ? fast_exp2(v[i + 1] * p.scale_log2 - m_used) : 0.f;
                            psum += e0 + e1;
                            w[i / 2] = pack_bf16x2(e0, e1);
                        }
#pragma unroll
                        for (int h2 = 0; h2 < 2; ++h2) {
                            const int q = ((col & 63) >> 3) + h2;
                            uint4* d = reinterpret_cast<uint4*>(stg + half * (MH * 128) + r * 128 + ((q ^ (r & 7)) << 4));
                            *d = make_uint4(w[4 * h2], w[4 * h2 + 1], w[4 * h2 + 2], w[4 * h2 + 3]);
                        }
                    }
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&s_empty);   // S may be overwritten by the next tile
                    lsum = lsum * alpha + psum;
                    float* extra = reinterpret_cast<float*>(stg + kPBytes);
                    if (half == 0) extra[r] = alpha;
                    if (j == sg.j1 - 1) {
                        if (half == 0) extra[MH + r] = m_used;
                        extra[(2 + half) * MH + r] = lsum;
                    }
                    ptx::fence_proxy_async_smem();   // staging writes -> the bulk copy (async proxy)
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&stg_ready[b]);
                }
            }
        }
    } else if (active) {
        // =========================== O-CTA ===========================
        if ((warp >= 5 && warp <= 7) || warp == 12) {
            // ---- producers: latent columns of the same rows, [128 keys x 128 columns] per stage
            const int pw = warp == 12 ? 3 : warp - 5;
            const int n_chunk = (p.L + 127) / 128;
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
                    const int my_row = kept_row(p, t, nv, j * KT + pw * 32 + lane);
                    // lane l < 16 issues rows 4*(l&7).. of this warp's 32, 64-column block (l >> 3)
                    const int r0 = __shfl_sync(0xffffffffu, my_row, (lane & 7) * 4 + 0);
                    const int r1 = __shfl_sync(0xffffffffu, my_row, (lane & 7) * 4 + 1);
                    const int r2 = __shfl_sync(0xffffffffu, my_row, (lane & 7) * 4 + 2);
                    const int r3 = __shfl_sync(0xffffffffu, my_row, (lane & 7) * 4 + 3);
                    for (int cc = 0; cc < n_chunk; ++cc) {
                        ok = __all_sync(0xffffffffu, ptx::mbar_wait(&ve[stage], ph ^ 1, p.status));
                        if (!ok) break;
                        const int nb = min(2, p.n_vblk - 2 * cc);   // 64-column blocks in this chunk
                        if (pw == 0 && lane == 0) ptx::mbar_arrive_expect_tx(&vf[stage], nb * kKStageBytes);
                        const int blk = lane >> 3;
                        if (lane < 8 * nb)
                            ptx::tma_gather4(smem + lay.stages + stage * 2 * kKStageBytes + blk * kKStageBytes +
                                                 (pw * 32 + (lane & 7) * 4) * 128,
                                             &tma_kv, &vf[stage], 64 * (2 * cc + blk), r0, r1, r2, r3);
                        ++n_issued;
                        if (++stage == NSV) { stage = 0; ph ^= 1; }
                    }
                }
            }
            if (lane == 0)
                for (int i = 0; i < NSV && i < n_issued; ++i) {
                    if (--stage < 0) { stage = NSV - 1; ph ^= 1; }
                    ptx::mbar_wait(&vf[stage], ph, nullptr);
                }
        } else if (warp == 4) {
            // ---- UMMA: O += P V, one 128-column latent chunk per value stage
            if (lane == 0) {
                const int n_chunk = (p.L + 127) / 128;
                SegIter it;
                it.init(p, c, C);
                Seg sg;
                int stage = 0, g = 0;
                uint32_t ph = 0, of_ph = 0, pr_ph[NP] = {0, 0};
                bool ok = true;
                const uint32_t p_addr = ptx::smem_u32(smem + lay.pbuf);
                while (ok && it.next(sg)) {
                    ok = ptx::mbar_wait(&o_free, of_ph ^ 1, p.status);
                    of_ph ^= 1;
                    ptx::tc_fence_after();
                    for (int j = sg.j0; ok && j < sg.j1; ++j, ++g) {
                        const int b = g & 1;
                        ok = ptx::mbar_wait(&p_ready[b], pr_ph[b], p.status);
                        pr_ph[b] ^= 1;
                        if (!ok) break;
                        ptx::tc_fence_after();
                        for (int cc = 0; ok && cc < n_chunk; ++cc) {
                            ok = ptx::mbar_wait(&vf[stage], ph, p.status);
                            if (!ok) break;
                            ptx::tc_fence_after();
                            const int nN = min(128, p.L - 128 * cc);
                            const uint32_t idesc = ptx::idesc_bf16(MH, nN, false, true);
                            const uint32_t v_addr = ptx::smem_u32(smem + lay.stages + stage * 2 * kKStageBytes);
                            for (int kk = 0; kk < KT / 16; ++kk) {
                                // P (K-major, 128-byte swizzle): keys 64*blk.. in block blk, 32 B per 16 keys.
                                const uint64_t ad = ptx::sdesc_sw128(
                                    p_addr + b * kPBufStride + (kk >> 2) * (MH * 128) + (kk & 3) * 32, 16, 1024);
                                // V (MN-major): 64-column atoms kKStageBytes apart (LBO), 8-key groups at 1 KB (SBO),
                                // a K=16 slice is 16 keys (2 KB) further.
                                const uint64_t bd = ptx::sdesc_sw128(v_addr + kk * 2048, kKStageBytes, 1024);
                                ptx::umma_bf16(tmem + cc * 128, ad, bd, idesc, (j > sg.j0 || kk > 0) ? 1u : 0u);
                            }
                            ptx::umma_commit(&ve[stage]);
                            if (++stage == NSV) { stage = 0; ph ^= 1; }
                        }
                        if (!ok) break;
                        ptx::umma_commit_multicast(&p_empty[b], (uint16_t)0x1);
                        ptx::umma_commit(&o_done[g & 1]);
                    }
                }
                ptx::umma_commit(&mma_done);
                ptx::mbar_wait(&mma_done, 0, p.status);
            }
        } else if (warp < 4) {
            // ---- correction + epilogue: thread = head row r
            const int r = warp * 32 + lane;
            const uint32_t t_row = tmem + ((uint32_t)(warp * 32) << 16);
            SegIter it;
            it.init(p, c, C);
            Seg sg;
            uint32_t pf_ph[NP] = {0, 0}, od_ph[2] = {0, 0};
            int g = 0;
            bool ok = true;
            while (ok && it.next(sg)) {
                float m_fin = 0.f, l_fin = 0.f;
                for (int j = sg.j0; j < sg.j1; ++j, ++g) {
                    const int b = g & 1;
                    const bool first = (j == sg.j0);
                    ok = __all_sync(0xffffffffu, ptx::mbar_wait_cluster(&p_full[b], pf_ph[b], p.status));
                    pf_ph[b] ^= 1;
                    if (!ok) break;
                    const float* extra = reinterpret_cast<const float*>(smem + lay.pbuf + b * kPBufStride + kPBytes);
                    const float al = extra[r];
                    if (j == sg.j1 - 1) {
                        m_fin = extra[MH + r];
                        l_fin = extra[2 * MH + r] + extra[3 * MH + r];
                    }
                    // This warp's rows are rescaled in TMEM before the tile's PV is released,
                    // once the previous tile's PV has completed.
                    bool waited = false;
                    if (!first && __any_sync(0xffffffffu, al != 1.f)) {
                        const int pb = (g - 1) & 1;
                        ok = __all_sync(0xffffffffu, ptx::mbar_wait(&o_done[pb], od_ph[pb], p.status));
                        od_ph[pb] ^= 1;
                        waited = true;
                        if (!ok) break;
                        ptx::tc_fence_after();
                        for (int col = 0; col < p.L; col += 16) {
                            float v[16];
                            ptx::tmem_ld16(t_row + col, v);
#pragma unroll
                            for (int i = 0; i < 16; ++i) v[i] *= al;
                            tmem_st16(t_row + col, v);
                        }
                    }
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&p_ready[b]);
                    if (!first && !waited) {
                        const int pb = (g - 1) & 1;
                        ok = __all_sync(0xffffffffu, ptx::mbar_wait(&o_done[pb], od_ph[pb], p.status));
                        od_ph[pb] ^= 1;
                        if (!ok) break;
                    }
                }
                if (!ok) break;
                // segment end: the last tile's PV must be complete
                {
                    const int pb = (g - 1) & 1;
                    ok = __all_sync(0xffffffffu, ptx::mbar_wait(&o_done[pb], od_ph[pb], p.status));
                    od_ph[pb] ^= 1;
                    if (!ok) break;
                }
                ptx::tc_fence_after();
                const int t = sg.w / p.HG, hg = sg.w % p.HG;
                const int rows_valid = min(MH, p.h - hg * MH);
                const bool full = (sg.j0 == 0 && sg.j1 == sg.n_w);
                const bool keep = r < rows_valid;
                if (full) {
                    const float inv = l_fin > 0.f ? 1.f / l_fin : 0.f;
                    bf16* dst = p.ctx + ((size_t)t * p.h + hg * MH + r) * p.L;
                    for (int col = 0; col < p.L; col += 16) {
                        float v[16];
                        ptx::tmem_ld16(t_row + col, v);
                        uint32_t w[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) w[i] = pack_bf16x2(v[2 * i] * inv, v[2 * i + 1] * inv);
                        if (keep) {
                            uint4* d4 = reinterpret_cast<uint4*>(dst + col);
                            d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
                            d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
                        }
                    }
                } else {
                    const int slot_id = 2 * c + (sg.run_start ? 0 : 1);
                    bf16* dst = p.part_o + ((size_t)slot_id * MH + r) * p.L;
                    for (int col = 0; col < p.L; col += 16) {
                        float v[16];
                        ptx::tmem_ld16(t_row + col, v);
                        uint32_t w[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) w[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
                        uint4* d4 = reinterpret_cast<uint4*>(dst + col);
                        d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
                        d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
                    }
                    p.part_ml[((size_t)slot_id * 2 + 0) * MH + r] = m_fin;
                    p.part_ml[((size_t)slot_id * 2 + 1) * MH + r] = l_fin;
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&o_free);
            }
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync_all();   // no remote copy or arrival may target an exited peer
    if (warp == 4) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

// First tile of every work item (tiles = ceil(kept rows / 32)): block-wide scan.
__global__ void __launch_bounds__(1024)
k_core_plan(const int32_t* __restrict__ n_valid, int T, int HG, int32_t* __restrict__ base) {
    __shared__ int warp_tot[32];
    __shared__ int carry;
    const int W = T * HG;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    for (int w0 = 0; w0 < W; w0 += blockDim.x) {
        const int w = w0 + threadIdx.x;
        const int n = w < W ? (n_valid[w / HG] + KT - 1) / KT : 0;
        int incl = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) warp_tot[wid] = incl;
        __syncthreads();
        if (wid == 0) {
            const int x = warp_tot[lane];
            int xi = x;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, xi, o);
                if (lane >= o) xi += v;
            }
            warp_tot[lane] = xi - x;
        }
        __syncthreads();
        const int excl = carry + warp_tot[wid] + incl - n;
        if (w < W) base[w] = excl;
        __syncthreads();
        if (threadIdx.x == blockDim.x - 1) carry = excl + n;
        __syncthreads();
    }
    if (threadIdx.x == 0) base[W] = carry;
}

// Merge the partial contexts of items split between cluster runs; zero-fill
// items with no kept key. Items finished in place are left alone.
//   ctx[r] = sum_c 2^(m_c[r] - M[r]) O_c[r] / sum_c 2^(m_c[r] - M[r]) l_c[r],  M = max_c m_c
constexpr int kMaxParts = 80;
__global__ void __launch_bounds__(256)
k_core_combine(Params p) {
    __shared__ float scale[kMaxParts][MH];
    __shared__ int sid[kMaxParts];
    __shared__ int c_first, c_last;
    const int w = blockIdx.x;
    const int t = w / p.HG, hg = w % p.HG;
    const int rows_valid = min(MH, p.h - hg * MH);
    const int b0 = p.item_base[w], b1 = p.item_base[w + 1];
    bf16* ctx = p.ctx + ((size_t)t * p.h + hg * MH) * p.L;
    const int vec_per_row = p.L / 8;
    if (b1 == b0) {
        for (int i = threadIdx.x; i < rows_valid * vec_per_row; i += blockDim.x)
            reinterpret_cast<uint4*>(ctx)[i] = make_uint4(0, 0, 0, 0);
        return;
    }
    const int U = p.item_base[p.W];
    const int C = clusters_for(U, p.max_clusters);
    if (threadIdx.x == 0) {
        int cf = 0, cl = 0;
        for (int cc = 0; cc < C; ++cc) {
            const int u0 = (int)((long long)U * cc / C), u1 = (int)((long long)U * (cc + 1) / C);
            if (u0 <= b0 && b0 < u1) cf = cc;
            if (u0 <= b1 - 1 && b1 - 1 < u1) cl = cc;
        }
        c_first = cf;
        c_last = cl;
    }
    __syncthreads();
    const int cf = c_first, np = c_last - c_first + 1;
    if (np == 1) return;   // one run covered the item: already written
    for (int k = threadIdx.x; k < np; k += blockDim.x) {
        const int cc = cf + k;
        const int u0 = (int)((long long)U * cc / C);
        sid[k] = 2 * cc + (u0 < b0 ? 1 : 0);
    }
    __syncthreads();
    auto sid_of = [&](int k) { return sid[k]; };
    if (threadIdx.x < MH) {
        const int r = threadIdx.x;
        float m = -INFINITY;
        for (int k = 0; k < np; ++k) m = fmaxf(m, p.part_ml[((size_t)sid_of(k) * 2) * MH + r]);
        float l = 0.f;
        for (int k = 0; k < np; ++k) {
            const float e = exp2f(p.part_ml[((size_t)sid_of(k) * 2) * MH + r] - m);
            scale[k][r] = e;
            l += e * p.part_ml[((size_t)sid_of(k) * 2 + 1) * MH + r];
        }
        const float inv = l > 0.f ? 1.f / l : 0.f;
        for (int k = 0; k < np; ++k) scale[k][r] *= inv;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < rows_valid * vec_per_row; i += blockDim.x) {
        const int r = i / vec_per_row, cv = i - r * vec_per_row;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int k = 0; k < np; ++k) {
            const float sc = scale[k][r];
            const uint4 v = reinterpret_cast<const uint4*>(p.part_o + ((size_t)sid_of(k) * MH + r) * p.L)[cv];
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(h2[e]);
                acc[2 * e] += sc * f.x;
                acc[2 * e + 1] += sc * f.y;
            }
        }
        uint4 o;
        uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
        for (int e = 0; e < 4; ++e) ow[e] = pack_bf16x2(acc[2 * e], acc[2 * e + 1]);
        reinterpret_cast<uint4*>(ctx)[(size_t)r * vec_per_row + cv] = o;
    }
}

}  // namespace core

bool core_tc_supports(const Dims& d) {
    return d.L % 64 == 0 && d.L <= 512 && d.R() % 16 == 0 && d.R() / 2 <= core::kSCol &&
           (d.h <= core::MH || d.h % core::MH == 0);
}

int core_tc_max_clusters() {
    static int cached = -1;
    if (cached > 0) return cached;
    const core::Layout lay(9, 8);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * 148, 1, 1);
    cfg.blockDim = dim3(core::kThreads, 1, 1);
    cfg.dynamicSmemBytes = lay.total;
    int n = 0;
    if (cudaFuncSetAttribute(core::k_core_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, lay.total) != cudaSuccess ||
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
size_t core_tc_ml_bytes(int max_clusters) { return (size_t)2 * max_clusters * 2 * core::MH * sizeof(float); }

cudaError_t launch_core_tc(const bf16* qtile, const bf16* kv_cache, const int32_t* rows, const int32_t* n_valid,
                           int32_t* item_base, const Dims& d, float scale, bf16* ctx, bf16* part_o, float* part_ml,
                           int max_clusters, int32_t* status, cudaStream_t s) {
    using namespace core;
    const int HG = d.h <= MH ? 1 : d.h / MH;
    const int W = d.T * HG;
    k_core_plan<<<1, 1024, 0, s>>>(n_valid, d.T, HG, item_base);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    Params p;
    p.kv_cache = kv_cache;
    p.qtile = qtile;
    p.rows = rows;
    p.n_valid = n_valid;
    p.item_base = item_base;
    p.T = d.T;
    p.h = d.h;
    p.HG = HG;
    p.P = d.P;
    p.L = d.L;
    p.R = d.R();
    p.n_kblk = (d.R() + 63) / 64;
    p.n_vblk = d.L / 64;
    p.W = W;
    p.max_clusters = max_clusters;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.ctx = ctx;
    p.part_o = part_o;
    p.part_ml = part_ml;
    p.status = status;
    CUtensorMap tkv;
    if (!make_tma_2d(&tkv, kv_cache, (uint64_t)d.R(), (uint64_t)d.n_rows(), (uint64_t)d.R() * 2, 64, 1))
        return cudaErrorInvalidValue;
    const Layout lay(p.n_kblk, p.n_vblk);
    e = cudaFuncSetAttribute(k_core_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, lay.total);
    if (e != cudaSuccess) return e;
    k_core_tc<<<2 * max_clusters, kThreads, lay.total, s>>>(tkv, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    k_core_combine<<<W, 256, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace mla
