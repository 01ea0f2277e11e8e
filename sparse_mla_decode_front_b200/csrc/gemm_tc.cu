// Host side of the tensor-core projection GEMM: TMA descriptors and launches.
#include <mutex>

#include "gemm_tc.cuh"
#include "launch.h"

namespace mla {

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

constexpr int kMaxDevices = 64;

int num_sms() {
    static int cached[kMaxDevices] = {};
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < kMaxDevices && cached[dev] > 0) return cached[dev];
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    n = n > 0 ? n : 148;
    if (dev >= 0 && dev < kMaxDevices) cached[dev] = n;
    return n;
}

constexpr bool kSplitK = true;   // reducing projections: round-robin split-K where it balances

// Split-K slices per tile for `tiles` tiles of `k_blocks` K blocks on `grid` CTAs,
// a CTA taking items blockIdx.x, + grid, ... (item = tile x slices + slice). Modelled
// cost: rounds of items x (K blocks per slice + kItemCost); stream-K's: the even share
// plus kItemCost per segment. Split-K is taken when its best count costs at most
// kSplitSlack times stream-K: it trades some balance for DRAM locality (the CTAs of a
// round read the same K rows of neighbouring tiles). 0: stream-K.
constexpr double kItemCost = 2.0;     // epilogue and pipeline refill per item, in K blocks
constexpr double kSplitSlack = 1.03;
int choose_splits(long long tiles, int k_blocks, int grid) {
    const double stream_k = (double)tiles * k_blocks / grid + kItemCost * (1 + (tiles + grid - 1) / grid);
    int best = 0;
    double best_cost = kSplitSlack * stream_k;
    for (int sl = 1; sl <= k_blocks; ++sl) {
        const long long rounds = (tiles * sl + grid - 1) / grid;
        const double cost = (double)rounds * ((k_blocks + sl - 1) / sl + kItemCost);
        if (cost < best_cost - 1e-9) {
            best_cost = cost;
            best = sl;
        }
    }
    return best;
}

template <int BN, bool A_MN, class Epi, int MP = 1>
cudaError_t launch_bn(const CUtensorMap& ta, const CUtensorMap& tb, const gemm::Problem& p, const Epi& e,
                      cudaStream_t s, const CUtensorMap& ta1, const Epi& e1) {
    using C = gemm::Cfg<BN, MP>;
    auto kern = gemm::k_gemm_tc<BN, A_MN, Epi, MP>;
    static bool attr_set[kMaxDevices] = {};   // per instantiation and device (attributes are per device)
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= kMaxDevices || !attr_set[dev]) {
        cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
        if (err != cudaSuccess) return err;
        if (dev >= 0 && dev < kMaxDevices) attr_set[dev] = true;
    }
    gemm::Problem q = p;
    const long long tiles = (long long)q.groups * q.m_tiles * q.n_tiles + (long long)q.m_tiles1 * q.n_tiles1;
    if (q.accumulate && q.splits < 0) q.splits = choose_splits(tiles, q.k_blocks, num_sms());
    const long long work = !q.accumulate ? tiles : q.splits > 0 ? tiles * q.splits : tiles * q.k_blocks;
    const int grid = (int)(work < num_sms() ? work : num_sms());
    if (grid <= 0) return cudaSuccess;
    // programmatic launch in graphs too: the weight tiles of the first stages load while the
    // previous kernel finishes
    return launch_pdl_mode(true, kern, dim3(grid), dim3(gemm::kThreads), C::kSmem, s, ta, tb, q, e, ta1, e1);
}

// Two feature tiles per CTA tile sharing one token tile (MN-major A, token tiles of at
// most 128 rows); p.m_tiles (and p.m_tiles1) already count pairs. ta1 / e1: the second
// problem's A map and epilogue (ignored when p.m_tiles1 == 0).
template <class Epi>
cudaError_t launch_pair_dispatch(int bn, const CUtensorMap& ta, const CUtensorMap& tb, const gemm::Problem& p,
                                 const Epi& e, cudaStream_t s, const CUtensorMap& ta1, const Epi& e1) {
    switch (bn) {
        case 16: return launch_bn<16, true, Epi, 2>(ta, tb, p, e, s, ta1, e1);
        case 32: return launch_bn<32, true, Epi, 2>(ta, tb, p, e, s, ta1, e1);
        case 64: return launch_bn<64, true, Epi, 2>(ta, tb, p, e, s, ta1, e1);
        default: return launch_bn<128, true, Epi, 2>(ta, tb, p, e, s, ta1, e1);
    }
}

// ta1 / e1: the second problem's A map and epilogue (ignored when p.m_tiles1 == 0).
template <bool A_MN, class Epi>
cudaError_t launch_dispatch(int bn, const CUtensorMap& ta, const CUtensorMap& tb, const gemm::Problem& p,
                            const Epi& e, cudaStream_t s, const CUtensorMap& ta1, const Epi& e1) {
    switch (bn) {
        case 16: return launch_bn<16, A_MN>(ta, tb, p, e, s, ta1, e1);
        case 32: return launch_bn<32, A_MN>(ta, tb, p, e, s, ta1, e1);
        case 64: return launch_bn<64, A_MN>(ta, tb, p, e, s, ta1, e1);
        case 128: return launch_bn<128, A_MN>(ta, tb, p, e, s, ta1, e1);
        default: return launch_bn<256, A_MN>(ta, tb, p, e, s, ta1, e1);
    }
}

}  // namespace

int gemm_bn_for(int rows) {
    if (rows <= 16) return 16;
    if (rows <= 32) return 32;
    if (rows <= 64) return 64;
    if (rows <= 128) return 128;
    return 256;
}

namespace {

// Encoded maps of recent calls: a step encodes the same weight and workspace maps every
// time, and encoding costs host time on every launch. A map is a pure function of its
// arguments (the address is a unified virtual address), so equal keys give equal maps.
struct MapKey {
    const void* base;
    uint64_t inner, outer, row_bytes;
    uint32_t box_inner, box_outer;
    int swizzle;
    bool operator==(const MapKey& o) const {
        return base == o.base && inner == o.inner && outer == o.outer && row_bytes == o.row_bytes &&
               box_inner == o.box_inner && box_outer == o.box_outer && swizzle == o.swizzle;
    }
};
constexpr int kMapCache = 64;
struct MapCache {
    std::mutex mu;
    MapKey key[kMapCache];
    CUtensorMap map[kMapCache];
    int used = 0, next = 0;
};
MapCache& map_cache() {
    static MapCache c;
    return c;
}

}  // namespace

bool make_tma_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                 uint32_t box_inner, uint32_t box_outer, int swizzle_bytes) {
    const MapKey k{base, inner, outer, row_bytes, box_inner, box_outer, swizzle_bytes};
    MapCache& c = map_cache();
    {
        std::lock_guard<std::mutex> lock(c.mu);
        for (int i = 0; i < c.used; ++i)
            if (c.key[i] == k) {
                *map = c.map[i];
                return true;
            }
    }
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t gdim[2] = {inner, outer};
    const cuuint64_t gstride[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estride[2] = {1, 1};
    if (fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride, box, estride,
           CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    std::lock_guard<std::mutex> lock(c.mu);
    const int slot = c.used < kMapCache ? c.used++ : (c.next++ % kMapCache);
    c.key[slot] = k;
    c.map[slot] = *map;
    return true;
}

// Fill a Problem and the two TMA maps for D[M, N] = A x B^T with A either
// MN-major (weight [K rows, M cols] per group, groups stacked along rows) or
// K-major (weight [M rows, K cols] per group, groups stacked along rows) and B
// [N rows, K cols per group] with groups side by side along columns.
// Whether a problem runs with two feature tiles per CTA tile.
bool use_pairs(GemmSpec const& g) { return g.m_pair && g.a_mn_major && gemm_bn_for(g.n_rows) <= 128; }

cudaError_t gemm_setup(GemmSpec const& g, CUtensorMap* ta, CUtensorMap* tb, gemm::Problem* p) {
    const int bn = gemm_bn_for(g.n_rows);
    if (g.a_mn_major) {
        if (!make_tma_2d(ta, g.a, (uint64_t)g.a_cols, (uint64_t)g.a_rows, (uint64_t)g.a_cols * 2, 64, 64))
            return cudaErrorInvalidValue;
    } else {
        if (!make_tma_2d(ta, g.a, (uint64_t)g.a_cols, (uint64_t)g.a_rows, (uint64_t)g.a_cols * 2, 64, gemm::BM))
            return cudaErrorInvalidValue;
    }
    if (!make_tma_2d(tb, g.b, (uint64_t)g.b_cols, (uint64_t)g.b_rows_alloc, (uint64_t)g.b_ld * 2, 64, bn))
        return cudaErrorInvalidValue;
    p->m_total = g.m_total;
    p->n_rows = g.n_rows;
    p->k_total = g.k_total;
    p->m_tiles = (g.m_total + gemm::BM - 1) / gemm::BM;
    if (use_pairs(g)) p->m_tiles = (p->m_tiles + 1) / 2;   // CTA tiles of two feature tiles
    p->n_tiles = (g.n_rows + bn - 1) / bn;
    p->k_blocks = (g.k_total + gemm::BK - 1) / gemm::BK;
    p->groups = g.groups;
    p->a_group_rows = g.a_group_rows;
    p->b_group_cols = g.b_group_cols;
    p->accumulate = g.accumulate;
    p->status = g.status;
    p->m_tiles1 = 0;
    p->n_tiles1 = 0;
    p->a_evict_first = g.a_evict_first;
    p->splits = g.splits > 0 ? g.splits : kSplitK ? -1 : 0;   // -1: chosen at launch
    return cudaSuccess;
}

cudaError_t launch_gemm_reduce_f32(GemmSpec const& g, float* out, int ldo, int group_off, cudaStream_t s) {
    CUtensorMap ta, tb;
    gemm::Problem p;
    cudaError_t e = gemm_setup(g, &ta, &tb, &p);
    if (e != cudaSuccess) return e;
    gemm::EpiReduceF32 epi{out, ldo, group_off, g.m_total, g.n_rows};
    const int bn = gemm_bn_for(g.n_rows);
    if (use_pairs(g)) return launch_pair_dispatch(bn, ta, tb, p, epi, s, ta, epi);
    return g.a_mn_major ? launch_dispatch<true>(bn, ta, tb, p, epi, s, ta, epi)
                        : launch_dispatch<false>(bn, ta, tb, p, epi, s, ta, epi);
}

cudaError_t launch_gemm_store_bf16(GemmSpec const& g, bf16* out, int ldo, int group_off, cudaStream_t s) {
    CUtensorMap ta, tb;
    gemm::Problem p;
    cudaError_t e = gemm_setup(g, &ta, &tb, &p);
    if (e != cudaSuccess) return e;
    gemm::EpiStoreBF16 epi{out, ldo, group_off, g.m_total, g.n_rows};
    const int bn = gemm_bn_for(g.n_rows);
    return g.a_mn_major ? launch_dispatch<true>(bn, ta, tb, p, epi, s, ta, epi)
                        : launch_dispatch<false>(bn, ta, tb, p, epi, s, ta, epi);
}

static_assert(gemm::kTpMaxWorld == kTpMaxRanks, "peer table sizes differ");
cudaError_t launch_gemm_reduce_peers(GemmSpec const& g0, const TpTable& t, int hidden, cudaStream_t s) {
    // MN-major weights only, in CTA tiles of two feature tiles whenever the token tile is at
    // most 128 rows: the tiling whose K blocks tp_gemm_units counts
    if (t.world < 1 || t.world > gemm::kTpMaxWorld || hidden % (32 * t.world) || g0.m_total != hidden ||
        !g0.a_mn_major)
        return cudaErrorInvalidValue;
    GemmSpec g = g0;
    g.m_pair = 1;
    CUtensorMap ta, tb;
    gemm::Problem p;
    cudaError_t e = gemm_setup(g, &ta, &tb, &p);
    if (e != cudaSuccess) return e;
    gemm::EpiReducePeers epi{};
    for (int r = 0; r < t.world; ++r) {
        epi.acc[r] = t.acc[r];
        epi.arrive[r] = t.flags[r];
    }
    epi.world = t.world;
    epi.shard = hidden / t.world;
    epi.m_total = g.m_total;
    epi.n_rows = g.n_rows;
    const int bn = gemm_bn_for(g.n_rows);
    if (use_pairs(g)) return launch_pair_dispatch(bn, ta, tb, p, epi, s, ta, epi);
    return launch_dispatch<true>(bn, ta, tb, p, epi, s, ta, epi);
}

// K blocks of CTA tiles one rank's share of the head split's o-projection issues (what its
// CTAs count in at every owner): CTA tiles of two 128-feature tiles when the token tile is at
// most 128 rows (the launch pairs them then), of one otherwise.
long long tp_gemm_units(int n_tokens, int k_rank, int hidden) {
    const int bn = gemm_bn_for(n_tokens);
    const long long m_tiles = (hidden + gemm::BM - 1) / gemm::BM;
    const long long cta_m_tiles = bn <= 128 ? (m_tiles + 1) / 2 : m_tiles;
    return cta_m_tiles * ((n_tokens + bn - 1) / bn) * ((k_rank + gemm::BK - 1) / gemm::BK);
}

// Two reducing projections in one launch: D0 = A0 x B^T and D1 = A1 x B^T over the
// same B rows and K (a stream-K split over the tiles of both), each reduced into its
// own fp32 target. Each problem uses the first n_rows rows of B.
cudaError_t launch_gemm_reduce_f32_pair(GemmSpec const& g0, float* out0, int ldo0, GemmSpec const& g1, float* out1,
                                        int ldo1, cudaStream_t s) {
    if (!g0.a_mn_major || !g1.a_mn_major || g0.groups != 1 || g1.groups != 1 || !g0.accumulate || !g1.accumulate ||
        g0.k_total != g1.k_total || g0.b != g1.b || g0.b_ld != g1.b_ld || g0.b_cols != g1.b_cols)
        return cudaErrorInvalidValue;
    GemmSpec gb = g0;   // one B map: the tile width of the smaller token count, rows of the larger
    gb.n_rows = g0.n_rows < g1.n_rows ? g0.n_rows : g1.n_rows;
    gb.b_rows_alloc = g0.b_rows_alloc > g1.b_rows_alloc ? g0.b_rows_alloc : g1.b_rows_alloc;
    const int bn = gemm_bn_for(gb.n_rows);
    // both problems in CTA tiles of two feature tiles, or neither
    gb.m_pair = g0.m_pair && g1.m_pair && use_pairs(gb);
    const int mp = gb.m_pair ? 2 : 1;
    CUtensorMap ta0, ta1, tb;
    gemm::Problem p;
    cudaError_t e = gemm_setup(gb, &ta0, &tb, &p);   // tiling of both problems is set below
    if (e != cudaSuccess) return e;
    if (!make_tma_2d(&ta1, g1.a, (uint64_t)g1.a_cols, (uint64_t)g1.a_rows, (uint64_t)g1.a_cols * 2, 64, 64))
        return cudaErrorInvalidValue;
    p.n_rows = g0.n_rows;
    p.n_tiles = (g0.n_rows + bn - 1) / bn;
    p.m_tiles1 = ((g1.m_total + gemm::BM - 1) / gemm::BM + mp - 1) / mp;
    p.n_tiles1 = (g1.n_rows + bn - 1) / bn;
    gemm::EpiReduceF32 e0{out0, ldo0, 0, g0.m_total, g0.n_rows};
    gemm::EpiReduceF32 e1{out1, ldo1, 0, g1.m_total, g1.n_rows};
    if (gb.m_pair) return launch_pair_dispatch(bn, ta0, tb, p, e0, s, ta1, e1);
    return launch_dispatch<true>(bn, ta0, tb, p, e0, s, ta1, e1);
}

}  // namespace mla
