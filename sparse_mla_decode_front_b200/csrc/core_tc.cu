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
//   rank 0 (S-CTA): Q in shared memory, key tiles gathered by TMA, S = Q K^T
//       into TMEM (two 32-column buffers), fp32 online softmax (one thread per
//       head, base-2 exponent, lazy rescale: the running max only moves when a
//       tile exceeds it by 2^8), bf16 P written into the O-CTA's shared memory;
//   rank 1 (O-CTA): value tiles (latent part of the same rows) gathered by
//       TMA, O += P V into the 512-column TMEM accumulator, O rescaled in TMEM
//       on the rare tiles that moved the max, O written out at the end.
// The O-CTA pulls the rows from HBM first and runs up to NS_O tiles ahead; the
// S-CTA reads the same rows back from L2, so HBM sees each row once.
//
// Work split: tiles of 32 kept keys; all (item, tile) pairs are laid out item
// by item and each cluster takes a contiguous run (stream-K). An item fully
// inside one run is finished in place; an item split between runs leaves
// bf16 partial contexts with their (max, sum), merged by k_core_combine.
#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace mla {
namespace core {

constexpr int KT = 32;            // keys per tile
constexpr int MH = 128;           // heads per work item (UMMA M)
constexpr int kThreads = 192;     // 6 warps: 0 TMA, 1 UMMA/TMEM, 2..5 softmax | correction+epilogue
constexpr int NS_S = 2;           // key stages in the S-CTA
constexpr int NS_O = 4;           // value stages in the O-CTA
constexpr int NP = 4;             // P slots (S-CTA -> O-CTA)
constexpr int kMinTilesPerCluster = 8;
constexpr float kRescaleLog2 = 8.f;
constexpr int kBlockBytes = KT * 128;       // one 64-column block of a tile (32 rows x 128 B)
constexpr int kPBytes = MH * KT * 2;        // one P slot, K-major, 64-byte swizzle

struct Params {
    const int32_t* rows;        // [T, P] kept rows, compacted
    const int32_t* n_valid;     // [T]
    const int32_t* item_base;   // [W + 1] first tile of each item
    int T, h, HG, P, L, R, n_kblk, n_vblk, W, max_clusters;
    float scale_log2;           // softmax_scale * log2(e)
    bf16* ctx;                  // [T, h, L]
    bf16* part_o;               // [2 * max_clusters, 128, L]
    float* part_ml;             // [2 * max_clusters, 2, 128]  (max in log2 units, sum)
    int32_t* status;
};

// Dynamic shared-memory layout (offsets from a 1024-aligned base), the same in both ranks.
struct Layout {
    int q, k, v, p, alpha, fin, total;
    __host__ __device__ Layout(int n_kblk, int n_vblk) {
        q = 0;                                       // S-CTA: n_kblk x [128 rows x 128 B]
        k = q + n_kblk * MH * 128;                   // S-CTA: NS_S stages x n_kblk blocks
        const int s_end = k + NS_S * n_kblk * kBlockBytes;
        v = 0;                                       // O-CTA: NS_O stages x n_vblk blocks
        p = v + NS_O * n_vblk * kBlockBytes;         // O-CTA: NP P slots
        alpha = p + NP * kPBytes;                    // O-CTA: NP x 128 fp32
        fin = alpha + NP * MH * 4;                   // O-CTA: NP x 2 x 128 fp32
        const int o_end = fin + NP * 2 * MH * 4;
        total = (s_end > o_end ? s_end : o_end) + 1024;
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

__device__ __forceinline__ int clusters_for(int U, int max_clusters) {
    const int c = U / kMinTilesPerCluster;
    return c < 1 ? 1 : (c > max_clusters ? max_clusters : c);
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
        "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
        "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
        "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
        "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15]))
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);   // .x = lo (low 16 bits), .y = hi
    return *reinterpret_cast<const uint32_t*>(&v);
}

// Load the 32 kept-row ids of tile j of item (t) into lane i; the tail repeats the last row.
__device__ __forceinline__ int tile_row(const Params& p, int t, int j, int lane) {
    const int nv = p.n_valid[t];
    const int k = min(j * KT + lane, nv - 1);
    return p.rows[(size_t)t * p.P + k];
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
k_core_tc(const __grid_constant__ CUtensorMap tma_q, const __grid_constant__ CUtensorMap tma_kv, Params p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // Barriers sit at identical offsets in both ranks (remote arrivals rely on it).
    __shared__ __align__(8) uint64_t k_full[NS_S], k_empty[NS_S], s_full[2], s_empty[2], q_full, q_empty;
    __shared__ __align__(8) uint64_t v_full[NS_O], v_empty[NS_O], p_full[NP], p_empty[NP], p_ready[NP];
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
    const uint32_t tmem_cols = rank == 0 ? 2 * KT : 512;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NS_S; ++i) { ptx::mbar_init(&k_full[i], 1); ptx::mbar_init(&k_empty[i], 1); }
        for (int i = 0; i < 2; ++i) { ptx::mbar_init(&s_full[i], 1); ptx::mbar_init(&s_empty[i], 4); }
        ptx::mbar_init(&q_full, 1);
        ptx::mbar_init(&q_empty, 1);
        for (int i = 0; i < NS_O; ++i) { ptx::mbar_init(&v_full[i], 1); ptx::mbar_init(&v_empty[i], 1); }
        for (int i = 0; i < NP; ++i) {
            ptx::mbar_init(&p_full[i], MH);    // every S-CTA softmax thread arrives
            ptx::mbar_init(&p_empty[i], 1);    // O-CTA UMMA commit (multicast)
            ptx::mbar_init(&p_ready[i], 4);    // O-CTA correction warps
        }
        for (int i = 0; i < 2; ++i) ptx::mbar_init(&o_done[i], 1);
        ptx::mbar_init(&o_free, 4);
        ptx::mbar_init(&mma_done, 1);
        ptx::fence_mbar_init();
        ptx::tma_prefetch_desc(&tma_q);
        ptx::tma_prefetch_desc(&tma_kv);
    }
    if (warp == 1) {
        ptx::tmem_alloc(&tmem_slot, tmem_cols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync_all();   // peer barriers initialised before any remote arrival
    ptx::tc_fence_after();
    const uint32_t tmem = tmem_slot;

    if (active && rank == 0) {
        // =========================== S-CTA ===========================
        if (warp == 0) {
            // ---- TMA: Q once per segment, key tiles (all R columns)
            SegIter it;
            it.init(p, c, C);
            Seg sg;
            int stage = 0, n_issued = 0, q_issued = 0;
            uint32_t k_ph = 0, q_ph = 0;
            bool ok = true;
            while (ok && it.next(sg)) {
                const int t = sg.w / p.HG, hg = sg.w % p.HG;
                if (lane == 0) {
                    ok = ptx::mbar_wait(&q_empty, q_ph ^ 1, p.status);
                    q_ph ^= 1;
                    if (ok) {
                        ++q_issued;
                        ptx::mbar_arrive_expect_tx(&q_full, p.n_kblk * MH * 128);
                        for (int b = 0; b < p.n_kblk; ++b)
                            ptx::tma_load_2d(smem + lay.q + b * MH * 128, &tma_q, &q_full, 64 * b, t * p.h + hg * MH);
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                for (int j = sg.j0; ok && j < sg.j1; ++j) {
                    const int row = tile_row(p, t, j, lane);
                    if (lane == 0) {
                        ok = ptx::mbar_wait(&k_empty[stage], k_ph ^ 1, p.status);
                        if (ok) ptx::mbar_arrive_expect_tx(&k_full[stage], p.n_kblk * kBlockBytes);
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    const int r0 = __shfl_sync(0xffffffffu, row, (lane & 7) * 4 + 0);
                    const int r1 = __shfl_sync(0xffffffffu, row, (lane & 7) * 4 + 1);
                    const int r2 = __shfl_sync(0xffffffffu, row, (lane & 7) * 4 + 2);
                    const int r3 = __shfl_sync(0xffffffffu, row, (lane & 7) * 4 + 3);
                    if (lane < 8) {
                        unsigned char* dst = smem + lay.k + stage * p.n_kblk * kBlockBytes + lane * 4 * 128;
                        for (int b = 0; b < p.n_kblk; ++b)
                            ptx::tma_gather4(dst + b * kBlockBytes, &tma_kv, &k_full[stage], 64 * b, r0, r1, r2, r3);
                    }
                    ++n_issued;
                    if (++stage == NS_S) { stage = 0; k_ph ^= 1; }
                }
            }
            // drain: loads already issued must land before shared memory is released
            if (lane == 0) {
                for (int i = 0; i < NS_S && i < n_issued; ++i) {
                    if (--stage < 0) { stage = NS_S - 1; k_ph ^= 1; }
                    ptx::mbar_wait(&k_full[stage], k_ph, nullptr);
                }
                if (q_issued) ptx::mbar_wait(&q_full, (uint32_t)(q_issued - 1) & 1u, nullptr);
            }
        } else if (warp == 1) {
            // ---- UMMA: S[b] = Q . K^T
            if (lane == 0) {
                constexpr uint32_t idesc = ptx::idesc_bf16(MH, KT, false, false);
                const int ksteps = p.R / 16;
                SegIter it;
                it.init(p, c, C);
                Seg sg;
                int stage = 0;
                uint32_t k_ph = 0, qf_ph = 0, se_ph[2] = {0, 0};
                int g = 0;
                bool ok = true;
                const uint32_t q_addr = ptx::smem_u32(smem + lay.q);
                while (ok && it.next(sg)) {
                    ok = ptx::mbar_wait(&q_full, qf_ph, p.status);
                    qf_ph ^= 1;
                    ptx::tc_fence_after();
                    for (int j = sg.j0; ok && j < sg.j1; ++j, ++g) {
                        const int b = g & 1;
                        ok = ptx::mbar_wait(&s_empty[b], se_ph[b] ^ 1, p.status);
                        se_ph[b] ^= 1;
                        if (ok) ok = ptx::mbar_wait(&k_full[stage], k_ph, p.status);
                        if (!ok) break;
                        ptx::tc_fence_after();
                        const uint32_t k_addr = ptx::smem_u32(smem + lay.k + stage * p.n_kblk * kBlockBytes);
                        for (int ks = 0; ks < ksteps; ++ks) {
                            const int blk = ks >> 2, kk = ks & 3;
                            const uint64_t ad = ptx::sdesc_sw128(q_addr + blk * MH * 128 + kk * 32, 16, 1024);
                            const uint64_t bd = ptx::sdesc_sw128(k_addr + blk * kBlockBytes + kk * 32, 16, 1024);
                            ptx::umma_bf16(tmem + b * KT, ad, bd, idesc, ks > 0 ? 1u : 0u);
                        }
                        ptx::umma_commit(&k_empty[stage]);
                        ptx::umma_commit(&s_full[b]);
                        if (++stage == NS_S) { stage = 0; k_ph ^= 1; }
                    }
                    ptx::umma_commit(&q_empty);
                }
                ptx::umma_commit(&mma_done);
                ptx::mbar_wait(&mma_done, 0, p.status);
            }
        } else {
            // ---- softmax: thread = head row r
            const int quarter = warp & 3;
            const int r = quarter * 32 + lane;
            const uint32_t t_row = tmem + ((uint32_t)(quarter * 32) << 16);
            const uint32_t peer_p = ptx::mapa_shared(ptx::smem_u32(smem + lay.p), 1);
            const uint32_t peer_alpha = ptx::mapa_shared(ptx::smem_u32(smem + lay.alpha), 1);
            const uint32_t peer_fin = ptx::mapa_shared(ptx::smem_u32(smem + lay.fin), 1);
            const uint32_t peer_pfull = ptx::mapa_shared(ptx::smem_u32(&p_full[0]), 1);
            SegIter it;
            it.init(p, c, C);
            Seg sg;
            uint32_t sf_ph[2] = {0, 0}, pe_ph[NP] = {0, 0, 0, 0};
            int g = 0;
            bool ok = true;
            while (ok && it.next(sg)) {
                const int t = sg.w / p.HG;
                const int nv = p.n_valid[t];
                float m_used = -INFINITY, lsum = 0.f;
                for (int j = sg.j0; j < sg.j1; ++j, ++g) {
                    const int b = g & 1, slot = g % NP;
                    ok = ptx::mbar_wait(&s_full[b], sf_ph[b], p.status);
                    sf_ph[b] ^= 1;
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    ptx::tc_fence_after();
                    float s[KT];
                    {
                        float a[16], bb[16];
                        ptx::tmem_ld16(t_row + b * KT, a);
                        ptx::tmem_ld16(t_row + b * KT + 16, bb);
#pragma unroll
                        for (int i = 0; i < 16; ++i) { s[i] = a[i]; s[16 + i] = bb[i]; }
                    }
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&s_empty[b]);
                    const int cnt = min(KT, nv - j * KT);
                    float mt = -INFINITY;
#pragma unroll
                    for (int i = 0; i < KT; ++i) {
                        s[i] = i < cnt ? s[i] * p.scale_log2 : -INFINITY;
                        mt = fmaxf(mt, s[i]);
                    }
                    float alpha = 1.f;   // factor the O-CTA applies to this head's running context
                    if (mt > m_used + kRescaleLog2) {
                        alpha = m_used != -INFINITY ? exp2f(m_used - mt) : 0.f;
                        m_used = mt;
                    }
                    uint32_t pk[KT / 2];
                    float psum = 0.f;
#pragma unroll
                    for (int i = 0; i < KT; i += 2) {
                        const float e0 = exp2f(s[i] - m_used), e1 = exp2f(s[i + 1] - m_used);
                        psum += e0 + e1;
                        pk[i / 2] = pack_bf16x2(e0, e1);
                    }
                    lsum = lsum * alpha + psum;
                    const bool last = (j == sg.j1 - 1);
                    ok = __all_sync(0xffffffffu, ptx::mbar_wait_cluster(&p_empty[slot], pe_ph[slot] ^ 1, p.status));
                    pe_ph[slot] ^= 1;
                    if (!ok) break;
                    // P row r: 64 bytes, K-major with 64-byte swizzle (16-byte chunk c at c ^ ((r >> 1) & 3)).
                    const uint32_t prow = peer_p + slot * kPBytes + r * 64;
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        ptx::st_cluster_v4(prow + ((q ^ ((r >> 1) & 3)) << 4), pk[4 * q], pk[4 * q + 1],
                                           pk[4 * q + 2], pk[4 * q + 3]);
                    ptx::st_cluster_f32(peer_alpha + (slot * MH + r) * 4, alpha);
                    if (last) {
                        ptx::st_cluster_f32(peer_fin + (slot * 2 * MH + r) * 4, m_used);
                        ptx::st_cluster_f32(peer_fin + (slot * 2 * MH + MH + r) * 4, lsum);
                    }
                    ptx::fence_proxy_async_cluster();
                    ptx::mbar_arrive_remote(peer_pfull + slot * 8);
                }
            }
        }
    } else if (active) {
        // =========================== O-CTA ===========================
        if (warp == 0) {
            // ---- TMA: value tiles (latent columns of the same rows)
            SegIter it;
            it.init(p, c, C);
            Seg sg;
            int stage = 0, n_issued = 0;
            uint32_t v_ph = 0;
            bool ok = true;
            while (ok && it.next(sg)) {
                const int t = sg.w / p.HG;
                for (int j = sg.j0; ok && j < sg.j1; ++j) {
                    const int row = tile_row(p, t, j, lane);
                    if (lane == 0) {
                        ok = ptx::mbar_wait(&v_empty[stage], v_ph ^ 1, p.status);
                        if (ok) ptx::mbar_arrive_expect_tx(&v_full[stage], p.n_vblk * kBlockBytes);
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    const int r0 = __shfl_sync(0xffffffffu, row, (lane & 7) * 4 + 0);
                    const int r1 = __shfl_sync(0xffffffffu, row, (lane & 7) * 4 + 1);
                    const int r2 = __shfl_sync(0xffffffffu, row, (lane & 7) * 4 + 2);
                    const int r3 = __shfl_sync(0xffffffffu, row, (lane & 7) * 4 + 3);
                    if (lane < 8) {
                        unsigned char* dst = smem + lay.v + stage * p.n_vblk * kBlockBytes + lane * 4 * 128;
                        for (int b = 0; b < p.n_vblk; ++b)
                            ptx::tma_gather4(dst + b * kBlockBytes, &tma_kv, &v_full[stage], 64 * b, r0, r1, r2, r3);
                    }
                    ++n_issued;
                    if (++stage == NS_O) { stage = 0; v_ph ^= 1; }
                }
            }
            if (lane == 0) {
                for (int i = 0; i < NS_O && i < n_issued; ++i) {
                    if (--stage < 0) { stage = NS_O - 1; v_ph ^= 1; }
                    ptx::mbar_wait(&v_full[stage], v_ph, nullptr);
                }
            }
        } else if (warp == 1) {
            // ---- UMMA: O += P . V
            if (lane == 0) {
                const int n_half = (p.L + 255) / 256;
                const int nN = p.L < 256 ? p.L : 256;
                const uint32_t idesc = ptx::idesc_bf16(MH, nN, false, true);
                SegIter it;
                it.init(p, c, C);
                Seg sg;
                int stage = 0, g = 0;
                uint32_t v_ph = 0, of_ph = 0, pr_ph[NP] = {0, 0, 0, 0};
                bool ok = true;
                const uint32_t p_addr = ptx::smem_u32(smem + lay.p);
                while (ok && it.next(sg)) {
                    ok = ptx::mbar_wait(&o_free, of_ph ^ 1, p.status);
                    of_ph ^= 1;
                    ptx::tc_fence_after();
                    for (int j = sg.j0; ok && j < sg.j1; ++j, ++g) {
                        const int slot = g % NP;
                        ok = ptx::mbar_wait(&p_ready[slot], pr_ph[slot], p.status);
                        pr_ph[slot] ^= 1;
                        if (ok) ok = ptx::mbar_wait(&v_full[stage], v_ph, p.status);
                        if (!ok) break;
                        ptx::tc_fence_after();
                        const uint32_t v_addr = ptx::smem_u32(smem + lay.v + stage * p.n_vblk * kBlockBytes);
                        for (int kk = 0; kk < KT / 16; ++kk) {
                            // P: 64-byte rows, 8-row groups at 512 B; a K=16 slice is 32 B further.
                            const uint64_t ad = ptx::sdesc_sw64(p_addr + slot * kPBytes + kk * 32, 16, 512);
                            for (int nh = 0; nh < n_half; ++nh) {
                                // V (MN-major): 64-column atoms at kBlockBytes (LBO), 8-key groups at 1 KB (SBO);
                                // a K=16 slice is 16 keys (2 KB) further.
                                const uint64_t bd =
                                    ptx::sdesc_sw128(v_addr + nh * 4 * kBlockBytes + kk * 2048, kBlockBytes, 1024);
                                ptx::umma_bf16(tmem + nh * 256, ad, bd, idesc, (j > sg.j0 || kk > 0) ? 1u : 0u);
                            }
                        }
                        ptx::umma_commit(&v_empty[stage]);
                        ptx::umma_commit_multicast(&p_empty[slot], (uint16_t)0x1);
                        ptx::umma_commit(&o_done[g & 1]);
                        if (++stage == NS_O) { stage = 0; v_ph ^= 1; }
                    }
                }
                ptx::umma_commit(&mma_done);
                ptx::mbar_wait(&mma_done, 0, p.status);
            }
        } else {
            // ---- correction + epilogue: thread = head row r
            const int quarter = warp & 3;
            const int r = quarter * 32 + lane;
            const uint32_t t_row = tmem + ((uint32_t)(quarter * 32) << 16);
            const float* alpha_s = reinterpret_cast<const float*>(smem + lay.alpha);
            const float* fin_s = reinterpret_cast<const float*>(smem + lay.fin);
            SegIter it;
            it.init(p, c, C);
            Seg sg;
            uint32_t pf_ph[NP] = {0, 0, 0, 0}, od_ph[2] = {0, 0};
            int g = 0;
            bool ok = true;
            while (ok && it.next(sg)) {
                float m_fin = 0.f, l_fin = 0.f;
                for (int j = sg.j0; j < sg.j1; ++j, ++g) {
                    const int slot = g % NP;
                    const bool first = (j == sg.j0);
                    ok = ptx::mbar_wait_cluster(&p_full[slot], pf_ph[slot], p.status);
                    pf_ph[slot] ^= 1;
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    const float al = alpha_s[slot * MH + r];
                    if (j == sg.j1 - 1) {
                        m_fin = fin_s[slot * 2 * MH + r];
                        l_fin = fin_s[slot * 2 * MH + MH + r];
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
                    ptx::fence_proxy_async_smem();
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&p_ready[slot]);
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
    ptx::cluster_sync_all();   // no remote write or arrival may target an exited peer
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, tmem_cols);
    }
}

// First tile of every work item (tiles = ceil(kept rows / 32)), one thread.
__global__ void k_core_plan(const int32_t* __restrict__ n_valid, int T, int HG, int32_t* __restrict__ base) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    int acc = 0;
    for (int w = 0; w < T * HG; ++w) {
        base[w] = acc;
        acc += (n_valid[w / HG] + KT - 1) / KT;
    }
    base[T * HG] = acc;
}

// Merge the partial contexts of items split between cluster runs; zero-fill
// items with no kept key. Items finished in place are left alone.
__global__ void __launch_bounds__(256)
k_core_combine(Params p) {
    __shared__ float wgt[MH], inv_l[MH];
    __shared__ int c_first, c_last;
    const int w = blockIdx.x;
    const int t = w / p.HG, hg = w % p.HG;
    const int rows_valid = min(MH, p.h - hg * MH);
    const int b0 = p.item_base[w], b1 = p.item_base[w + 1];
    bf16* ctx = p.ctx + ((size_t)t * p.h + hg * MH) * p.L;
    if (b1 == b0) {
        for (int i = threadIdx.x; i < rows_valid * p.L; i += blockDim.x) ctx[i] = __float2bfloat16(0.f);
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
    if (c_first == c_last) return;   // one run covered the item: already written
    if (threadIdx.x < MH) {
        const int r = threadIdx.x;
        float m = -INFINITY;
        for (int cc = c_first; cc <= c_last; ++cc) {
            const int u0 = (int)((long long)U * cc / C);
            const int sid = 2 * cc + (u0 < b0 ? 1 : 0);
            m = fmaxf(m, p.part_ml[((size_t)sid * 2) * MH + r]);
        }
        float l = 0.f;
        for (int cc = c_first; cc <= c_last; ++cc) {
            const int u0 = (int)((long long)U * cc / C);
            const int sid = 2 * cc + (u0 < b0 ? 1 : 0);
            l += exp2f(p.part_ml[((size_t)sid * 2) * MH + r] - m) * p.part_ml[((size_t)sid * 2 + 1) * MH + r];
        }
        wgt[r] = m;
        inv_l[r] = l > 0.f ? 1.f / l : 0.f;
    }
    __syncthreads();
    for (int r = 0; r < rows_valid; ++r) {
        for (int col = threadIdx.x; col < p.L; col += blockDim.x) {
            float acc = 0.f;
            for (int cc = c_first; cc <= c_last; ++cc) {
                const int u0 = (int)((long long)U * cc / C);
                const int sid = 2 * cc + (u0 < b0 ? 1 : 0);
                const float sc = exp2f(p.part_ml[((size_t)sid * 2) * MH + r] - wgt[r]);
                acc += sc * __bfloat162float(p.part_o[((size_t)sid * MH + r) * p.L + col]);
            }
            ctx[(size_t)r * p.L + col] = __float2bfloat16(acc * inv_l[r]);
        }
    }
}

}  // namespace core

bool core_tc_supports(const Dims& d) {
    return d.L % 64 == 0 && d.L <= 512 && d.R() % 16 == 0 && (d.h <= core::MH || d.h % core::MH == 0);
}

int core_tc_max_clusters() {
    static int cached = -1;
    if (cached > 0) return cached;
    const core::Layout lay((576 + 63) / 64, 8);
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
    if (c > kCoreMaxClusters) c = kCoreMaxClusters;
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
    k_core_plan<<<1, 32, 0, s>>>(n_valid, d.T, HG, item_base);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    CUtensorMap tq, tkv;
    if (!make_tma_2d(&tq, qtile, (uint64_t)d.R(), (uint64_t)d.T * d.h, (uint64_t)d.R() * 2, 64, MH))
        return cudaErrorInvalidValue;
    if (!make_tma_2d(&tkv, kv_cache, (uint64_t)d.R(), (uint64_t)d.n_rows(), (uint64_t)d.R() * 2, 64, 1))
        return cudaErrorInvalidValue;
    Params p;
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
    const Layout lay(p.n_kblk, p.n_vblk);
    e = cudaFuncSetAttribute(k_core_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, lay.total);
    if (e != cudaSuccess) return e;
    k_core_tc<<<2 * max_clusters, kThreads, lay.total, s>>>(tq, tkv, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    k_core_combine<<<W, 256, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace mla
