// C ABI of the sparse MLA gather-decode block: validation, workspace plan and
// the launch chain on the caller's stream. The operation is the one of the
// page "MLA Attention Block Gather Decode Kernel API Reference"
// (mla_attention_block_gather_decode, section "API Reference"); every argument
// is documented in include/sparse_mla_decode.h.
#include <cmath>
#include <cstring>

#include <cstdio>
#include <initializer_list>

#include "common.cuh"
#include "launch.h"
#include "mla_tp.h"
#include "moe_router.h"

namespace mla {
namespace {

thread_local cudaError_t g_last_cuda_error = cudaSuccess;

// Record a failed CUDA call of this host thread and map it to MLA_ERR_CUDA.
inline bool cuda_failed(cudaError_t e) {
    if (e == cudaSuccess) return false;
    g_last_cuda_error = e;
    return true;
}


constexpr size_t kAlign = 256;

inline size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

// Workspace regions, in order. Offsets are multiples of kAlign.
struct Plan {
    size_t status, rows, n_valid, r_in, xg3, qacc, kacc, kv_f32, fix, flag_list, q_an, qtile, ctx, o, y32,
        item_base, part_o, part_ml, total;
    int clusters;
};

Plan make_plan(const Dims& d) {
    Plan p;
    size_t off = 0;
    auto take = [&](size_t bytes) { const size_t at = off; off += align_up(bytes); return at; };
    const size_t T = d.T;
    p.status = take(kAlign);
    p.rows = take(sizeof(int32_t) * T * d.P);
    p.n_valid = take(sizeof(int32_t) * T);
    p.r_in = take(sizeof(double) * T);
    p.xg3 = take(sizeof(bf16) * 3 * T * d.H);          // hi / mid / lo slices of x * gamma
    p.qacc = take(sizeof(float) * T * d.Lq);            // fp32 reduction targets
    p.kacc = take(sizeof(float) * 3 * T * d.R());
    p.kv_f32 = take(sizeof(float) * T * d.R());           // kv rows before the exact fix-up
    p.fix = take(sizeof(double) * T * d.R());             // exact dots of flagged elements
    p.flag_list = take(sizeof(int32_t) * (T * d.R() + 1)); // [0] = count, then flagged (t, j)
    p.q_an = take(sizeof(bf16) * T * d.Lq);
    p.qtile = take(sizeof(bf16) * T * d.h * d.R());     // [q_lat | rotated q_pe] per head
    p.ctx = take(sizeof(bf16) * T * d.h * d.L);
    p.o = take(sizeof(bf16) * T * d.h * d.dv);
    p.y32 = take(sizeof(float) * T * d.H);
    const int hg = d.h <= 128 ? 1 : d.h / 128;
    p.clusters = core_tc_cluster_bound(d);
    p.item_base = take(sizeof(int32_t) * (T * hg + 1));   // attention work plan
    p.part_o = take(core_tc_partial_bytes(d, p.clusters)); // contexts of items split between clusters
    p.part_ml = take(core_tc_ml_bytes(p.clusters));
    p.total = off;
    return p;
}

Dims to_dims(const mla_dims& a) {
    Dims d;
    d.T = a.n_tokens; d.H = a.hidden; d.Lq = a.q_lora_rank; d.L = a.kv_lora_rank;
    d.dn = a.qk_nope_head_dim; d.dr = a.qk_rope_head_dim; d.dv = a.v_head_dim; d.h = a.n_heads;
    d.bs = a.block_size; d.n_blocks = a.n_blocks; d.max_blocks = a.max_blocks_per_seq; d.P = a.n_prior;
    return d;
}

int check_dims(const mla_dims* a) {
    if (!a) return MLA_ERR_NULL_POINTER;
    const Dims d = to_dims(*a);
    if (d.T < 0 || d.P < 0) return MLA_ERR_BAD_DIMS;
    if (d.H <= 0 || d.Lq <= 0 || d.L <= 0 || d.dn <= 0 || d.dr <= 0 || d.dv <= 0 || d.h <= 0 ||
        d.bs <= 0 || d.n_blocks <= 0 || d.max_blocks <= 0)
        return MLA_ERR_BAD_DIMS;
    if (d.dr % 2) return MLA_ERR_BAD_DIMS;
    if ((long long)d.n_blocks * d.bs > INT32_MAX) return MLA_ERR_UNSUPPORTED_DIMS;
    if ((long long)d.max_blocks * d.bs > INT32_MAX) return MLA_ERR_UNSUPPORTED_DIMS;
    if (!core_tc_supports(d) || !q_chain_supports(d)) return MLA_ERR_UNSUPPORTED_DIMS;
    {   // the work plan evaluates (total tiles) x (clusters) in 32 bits
        const long long hg = d.h <= 128 ? 1 : d.h / 128;
        if ((long long)d.T * hg * ((d.P + 63) / 64) * kCoreMaxClusters >= (1LL << 31)) return MLA_ERR_UNSUPPORTED_DIMS;
    }
    // Tensor-core projections: K extents are multiples of 16 (UMMA K step) and
    // every row handed to TMA is a multiple of 16 bytes.
    if (d.H % 16 || d.Lq % 16 || d.dn % 16 || d.L % 16 || (d.h * d.dv) % 16) return MLA_ERR_UNSUPPORTED_DIMS;
    if (d.R() % 8 || d.dr % 8 || d.dv % 8) return MLA_ERR_UNSUPPORTED_DIMS;   // 16-byte vector epilogues
    if (d.R() % 8 || (d.h * d.qk()) % 8) return MLA_ERR_UNSUPPORTED_DIMS;
    return MLA_OK;
}

inline bool misaligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

// Base of the device allocation holding p (driver entry point; the library links
// only the CUDA runtime). False if p is not a device pointer.
bool allocation_base(const void* p, CUdeviceptr* base) {
    typedef CUresult (*RangeFn)(CUdeviceptr*, size_t*, CUdeviceptr);
    static RangeFn fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            f = nullptr;
        return reinterpret_cast<RangeFn>(f);
    }();
    size_t size = 0;
    return fn && fn(base, &size, reinterpret_cast<CUdeviceptr>(p)) == CUDA_SUCCESS;
}

// Validate a head-split peer table for `hidden` columns and ranks [rank, rank + n_local),
// and copy it into the kernels' form.
int tp_table_of(const mla_tp_peers* tp, int hidden, int n_local, TpTable* t) {
    static_assert(MLA_TP_MAX_WORLD == kTpMaxRanks, "peer table sizes differ");
    if (!tp) return MLA_ERR_NULL_POINTER;
    if (tp->world < 1 || tp->world > MLA_TP_MAX_WORLD || tp->rank < 0 || n_local < 1 ||
        tp->world % n_local || tp->rank % n_local || tp->rank + n_local > tp->world || tp->epoch == 0)
        return MLA_ERR_BAD_ARGUMENT;
    if (hidden % (32 * tp->world)) return MLA_ERR_UNSUPPORTED_DIMS;
    *t = TpTable{};
    t->world = tp->world;
    for (int r = 0; r < tp->world; ++r) {
        if (!tp->acc[r] || !tp->out[r] || !tp->flags[r]) return MLA_ERR_NULL_POINTER;
        if (misaligned(tp->acc[r]) || misaligned(tp->out[r]) || misaligned(tp->flags[r])) return MLA_ERR_MISALIGNED;
        t->acc[r] = tp->acc[r];
        t->out[r] = static_cast<bf16*>(tp->out[r]);
        t->flags[r] = tp->flags[r];
    }
    return MLA_OK;
}

}  // namespace
}  // namespace mla

using namespace mla;

extern "C" {

int32_t mla_abi_version(void) { return (1 << 16) | 4; }

const char* mla_status_string(int code) {
    switch (code) {
        case MLA_OK: return "ok";
        case MLA_ERR_NULL_POINTER: return "a required pointer is NULL";
        case MLA_ERR_BAD_DIMS: return "a dimension is non-positive or inconsistent";
        case MLA_ERR_UNSUPPORTED_DIMS: return "dimensions are valid but not supported by the kernels";
        case MLA_ERR_MISALIGNED: return "a pointer is not 16-byte aligned";
        case MLA_ERR_WORKSPACE_TOO_SMALL: return "workspace is smaller than mla_block_workspace_bytes()";
        case MLA_ERR_CUDA: return "a CUDA runtime call or kernel launch failed";
        case MLA_ERR_BAD_ARGUMENT: return "a scalar argument is out of range";
        default: return "unknown status code";
    }
}

const char* mla_last_cuda_error_string(void) {
    static thread_local char buf[160];
    if (g_last_cuda_error == cudaSuccess) return "no error";
    snprintf(buf, sizeof(buf), "%s: %s", cudaGetErrorName(g_last_cuda_error), cudaGetErrorString(g_last_cuda_error));
    return buf;
}

int mla_block_check_dims(const mla_dims* dims) { return check_dims(dims); }

size_t mla_block_workspace_bytes(const mla_dims* dims) {
    if (check_dims(dims) != MLA_OK) return 0;
    return make_plan(to_dims(*dims)).total;
}

int mla_get_device_status(const void* workspace, void* stream, int32_t* status) {
    if (!workspace || !status) return MLA_ERR_NULL_POINTER;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int32_t v = 0;
    if (cuda_failed(cudaMemcpyAsync(&v, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost, s)))
        return MLA_ERR_CUDA;
    if (cuda_failed(cudaStreamSynchronize(s))) return MLA_ERR_CUDA;
    *status = v;
    return MLA_OK;
}

}  // extern "C"

namespace {

// A side stream and its fork / join events, one set per host thread and device (created on
// first use, kept until the process exits).
struct SideStream {
    cudaStream_t s = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};
constexpr int kMaxSideDevices = 64;
SideStream* side_stream() {
    thread_local SideStream ss[kMaxSideDevices];
    int dev = 0;
    if (cuda_failed(cudaGetDevice(&dev)) || dev < 0 || dev >= kMaxSideDevices) return nullptr;
    SideStream& x = ss[dev];
    if (!x.s) {
        SideStream n;
        if (cuda_failed(cudaStreamCreateWithFlags(&n.s, cudaStreamNonBlocking))) return nullptr;
        if (cuda_failed(cudaEventCreateWithFlags(&n.fork, cudaEventDisableTiming)) ||
            cuda_failed(cudaEventCreateWithFlags(&n.join, cudaEventDisableTiming))) {
            if (n.fork) cudaEventDestroy(n.fork);
            cudaStreamDestroy(n.s);
            return nullptr;
        }
        x = n;
    }
    return &x;
}

// Workspace regions of one call, as pointers.
struct Bufs {
    int32_t *status, *rows, *n_valid, *flag_count, *flag_list, *item_base;
    double *r_in, *fix;
    bf16 *xg3, *q_an, *qtile, *ctx, *o, *part_o;
    float *qacc, *kacc, *kv_f32, *y32, *part_ml;
    int clusters;
};

Bufs bufs_of(const Plan& pl, void* workspace) {
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    Bufs b;
    b.status = reinterpret_cast<int32_t*>(ws + pl.status);
    b.rows = reinterpret_cast<int32_t*>(ws + pl.rows);
    b.n_valid = reinterpret_cast<int32_t*>(ws + pl.n_valid);
    b.r_in = reinterpret_cast<double*>(ws + pl.r_in);
    b.xg3 = reinterpret_cast<bf16*>(ws + pl.xg3);
    b.qacc = reinterpret_cast<float*>(ws + pl.qacc);
    b.kacc = reinterpret_cast<float*>(ws + pl.kacc);
    b.kv_f32 = reinterpret_cast<float*>(ws + pl.kv_f32);
    b.fix = reinterpret_cast<double*>(ws + pl.fix);
    b.flag_count = reinterpret_cast<int32_t*>(ws + pl.flag_list);
    b.flag_list = b.flag_count + 1;
    b.q_an = reinterpret_cast<bf16*>(ws + pl.q_an);
    b.qtile = reinterpret_cast<bf16*>(ws + pl.qtile);
    b.ctx = reinterpret_cast<bf16*>(ws + pl.ctx);
    b.o = reinterpret_cast<bf16*>(ws + pl.o);
    b.y32 = reinterpret_cast<float*>(ws + pl.y32);
    b.item_base = reinterpret_cast<int32_t*>(ws + pl.item_base);
    b.part_o = reinterpret_cast<bf16*>(ws + pl.part_o);
    b.part_ml = reinterpret_cast<float*>(ws + pl.part_ml);
    b.clusters = pl.clusters;
    return b;
}

// Clusters the core launches with (the plan and the core must agree on it).
int core_clusters(const Bufs& b) {
    const int occ = core_tc_max_clusters();
    return b.clusters < occ ? b.clusters : occ;
}

// Common checks of the workspace; MLA_OK or the code to return.
int check_workspace(const Plan& pl, const void* workspace, size_t workspace_bytes) {
    if (!workspace) return MLA_ERR_NULL_POINTER;
    if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return MLA_ERR_MISALIGNED;
    if (workspace_bytes < pl.total) return MLA_ERR_WORKSPACE_TOO_SMALL;
    return MLA_OK;
}

int check_ptrs(std::initializer_list<const void*> ptrs) {
    for (const void* p : ptrs)
        if (!p) return MLA_ERR_NULL_POINTER;
    for (const void* p : ptrs)
        if (misaligned(p)) return MLA_ERR_MISALIGNED;
    return MLA_OK;
}

#define MLA_TRY(expr)                                  \
    do {                                               \
        if (cuda_failed(expr)) return MLA_ERR_CUDA;    \
    } while (0)
#define MLA_LAUNCH(expr) \
    do {                 \
        MLA_TRY(expr);   \
        ++n_launches;    \
    } while (0)

// Front-fold (page "MLA Attention Block Gather Decode Kernel API Reference": :param
// input_norm_w .. q_absorb_w, cos, sin, kv_cache, slot_mapping): x*gamma slices,
// down-projections, norms + cache row, up-projection + RoPE, absorption into the
// query tiles qtile [T, h, R].
int enqueue_front(const Dims& d, const Bufs& b, const bf16* x, const float* input_norm_w, const void* wq_a,
                  const float* q_norm_w, const void* wq_b, const void* wkv_a, const float* kv_norm_w,
                  const void* q_absorb_w, const float* cos_t, const float* sin_t, void* kv_cache,
                  const int32_t* slot_mapping, float norm_eps, bf16* qtile, cudaStream_t s, int& n_launches,
                  bool prep_done, const CorePlanArgs* plan) {
    if (!prep_done)
        MLA_LAUNCH(launch_fold_prep_tc(x, input_norm_w, d, b.xg3, b.qacc, b.kacc, b.y32, b.fix, b.flag_count, s));
    {
        GemmSpec g{};
        g.a = wq_a; g.a_rows = d.H; g.a_cols = d.Lq; g.a_mn_major = true;
        g.b = b.xg3; g.b_cols = d.H; g.b_ld = d.H; g.b_rows_alloc = d.T; g.n_rows = d.T;
        g.m_total = d.Lq; g.k_total = d.H; g.groups = 1; g.accumulate = 1; g.status = b.status;
        g.m_pair = 1;      // two feature tiles share each token tile (the kv problem's are 3T rows)
        GemmSpec gk = g;   // the kv down-projection runs on all three slices (3T token rows)
        gk.a = wkv_a; gk.a_cols = d.R(); gk.m_total = d.R();
        gk.b_rows_alloc = 3 * d.T; gk.n_rows = 3 * d.T;
        g.b_rows_alloc = 3 * d.T;   // one B map over the slices; the q projection reads the first T rows
        // both down-projections in one stream-K launch over their tiles
        MLA_LAUNCH(launch_gemm_reduce_f32_pair(g, b.qacc, d.Lq, gk, b.kacc, d.R(), s));
    }
    MLA_LAUNCH(launch_fold_q_kv(x, b.qacc, b.kacc, q_norm_w, cos_t, sin_t, d, norm_eps, b.r_in, b.q_an, b.kv_f32,
                                b.flag_count, b.flag_list, plan, s));
    // The cache rows (fix-up, norm + RoPE, write) and the query chain depend only on the fold
    // above, not on each other: the rows go on a side stream, forked and joined with events
    // (edges of a captured graph as well), and run on the SMs the query chain leaves free.
    SideStream* side = side_stream();
    if (!side) return MLA_ERR_CUDA;
    MLA_TRY(cudaEventRecord(side->fork, s));
    MLA_TRY(cudaStreamWaitEvent(side->s, side->fork, 0));
    MLA_TRY(launch_kv_fix_row(x, input_norm_w, static_cast<const bf16*>(wkv_a), kv_norm_w, cos_t, sin_t,
                              slot_mapping, d, norm_eps, b.r_in, b.kv_f32, b.flag_count, b.flag_list, b.fix,
                              static_cast<bf16*>(kv_cache), b.status, side->s));
    n_launches += 2;
    MLA_TRY(cudaEventRecord(side->join, side->s));
    // per head: up-projection, q RoPE and absorption in one CTA (the up-projection stays on chip)
    MLA_LAUNCH(launch_q_chain(b.q_an, wq_b, q_absorb_w, cos_t, sin_t, d, qtile, b.status, s));
    MLA_TRY(cudaStreamWaitEvent(s, side->join, 0));   // every row of this step is in the cache
    return MLA_OK;
}

// Attention back half: core over the resolved rows (after every row of this step is
// in the cache: stream order), out absorption, o-projection into out [T, H].
// ev (optional): events recorded after the core and after the out absorption.
int enqueue_back(const Dims& d, const Bufs& b, const bf16* qtile, const void* kv_cache, const void* out_absorb_w,
                 const void* o_proj_w, void* out, float softmax_scale, cudaStream_t s, int& n_launches,
                 cudaEvent_t ev_core, cudaEvent_t ev_absorb, bool plan_done, const mla_tp_peers* tp = nullptr) {
    {
        MLA_TRY(launch_core_tc(qtile, static_cast<const bf16*>(kv_cache), b.rows, b.n_valid, b.item_base, d,
                               softmax_scale, b.ctx, b.part_o, b.part_ml, core_clusters(b), plan_done, b.status, s));
        n_launches += plan_done ? 2 : 3;   // (plan,) clusters, combine
    }
    if (ev_core) MLA_TRY(cudaEventRecord(ev_core, s));
    {
        GemmSpec g{};
        g.a = out_absorb_w; g.a_rows = d.h * d.dv; g.a_cols = d.L; g.a_mn_major = false;
        g.b = b.ctx; g.b_cols = d.h * d.L; g.b_ld = d.h * d.L; g.b_rows_alloc = d.T; g.n_rows = d.T;
        g.m_total = d.dv; g.k_total = d.L; g.groups = d.h; g.a_group_rows = d.dv; g.b_group_cols = d.L;
        g.accumulate = 0; g.status = b.status;
        MLA_LAUNCH(launch_gemm_store_bf16(g, b.o, d.h * d.dv, d.dv, s));
    }
    if (ev_absorb) MLA_TRY(cudaEventRecord(ev_absorb, s));
    GemmSpec g{};
    g.a = o_proj_w; g.a_rows = d.h * d.dv; g.a_cols = d.H; g.a_mn_major = true;
    g.b = b.o; g.b_cols = d.h * d.dv; g.b_ld = d.h * d.dv; g.b_rows_alloc = d.T; g.n_rows = d.T;
    g.m_total = d.H; g.k_total = d.h * d.dv; g.groups = 1; g.accumulate = 1; g.status = b.status;
    g.a_evict_first = 1;   // read once: these lines leave L2 first, the step's working set stays
    g.m_pair = 1;   // two feature tiles share each token tile: a quarter fewer bytes into every SM
    if (tp) {   // head split: tiles reduced into the owners' accumulators, then the shards exchanged
        TpTable t;
        const int rc = tp_table_of(tp, d.H, 1, &t);
        if (rc != MLA_OK) return rc;
        MLA_LAUNCH(launch_gemm_reduce_peers(g, t, d.H, s));
        MLA_LAUNCH(launch_tp_finish(t, tp->rank, 1, d.T, d.H, tp->epoch,
                                    (uint32_t)tp_gemm_units(d.T, d.h * d.dv, d.H), b.status, s));
        return MLA_OK;
    }
    MLA_LAUNCH(launch_gemm_reduce_f32(g, b.y32, d.H, 0, s));
    if (out) MLA_LAUNCH(launch_f32_to_bf16(b.y32, static_cast<bf16*>(out), (size_t)d.T * d.H, s));
    return MLA_OK;
}

}  // namespace

extern "C" {

int mla_block_gather_decode_ex(
    const void* hidden_states, const float* input_norm_w,
    const void* wq_a, const float* q_norm_w, const void* wq_b,
    const void* wkv_a, const float* kv_norm_w,
    const void* q_absorb_w, const void* out_absorb_w, const void* o_proj_w,
    const float* cos_t, const float* sin_t,
    void* kv_cache, const int32_t* slot_mapping,
    const int32_t* block_table, const int32_t* positions,
    const int32_t* gather_indices,
    void* out,
    const mla_dims* dims, float softmax_scale, float norm_eps,
    void* workspace, size_t workspace_bytes, void* stream, mla_launch_opts* opts) {
    if (opts) opts->n_launches = 0;
    const int dc = check_dims(dims);
    if (dc != MLA_OK) return dc;
    const Dims d = to_dims(*dims);
    if (!std::isfinite(softmax_scale) || !std::isfinite(norm_eps) || norm_eps < 0.f)
        return MLA_ERR_BAD_ARGUMENT;
    if (d.T == 0) return MLA_OK;
    float* out_f32 = opts ? opts->out_f32 : nullptr;
    const mla_tp_peers* tp = opts ? opts->tp : nullptr;
    if (tp) {   // the head split's output goes to tp->out[tp->rank]; out and out_f32 are not used
        if (out_f32) return MLA_ERR_BAD_ARGUMENT;
        TpTable t;
        const int rc_tp = tp_table_of(tp, d.H, 1, &t);
        if (rc_tp != MLA_OK) return rc_tp;
        out = tp->out[tp->rank];
    }
    int rc = check_ptrs({hidden_states, input_norm_w, wq_a, q_norm_w, wq_b, wkv_a, kv_norm_w, q_absorb_w,
                         out_absorb_w, o_proj_w, cos_t, sin_t, kv_cache, slot_mapping, block_table, positions,
                         out_f32 ? static_cast<const void*>(out_f32) : out});
    if (rc != MLA_OK) return rc;
    if (d.P > 0 && !gather_indices) return MLA_ERR_NULL_POINTER;
    if (d.P > 0 && misaligned(gather_indices)) return MLA_ERR_MISALIGNED;
    const Plan pl = make_plan(d);
    rc = check_workspace(pl, workspace, workspace_bytes);
    if (rc != MLA_OK) return rc;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    Bufs b = bufs_of(pl, workspace);
    if (out_f32) b.y32 = out_f32;   // the o-projection sums land in the caller's fp32 buffer
    int n_launches = 0;
    cudaEvent_t const* ev = opts && opts->stage_events
                                ? reinterpret_cast<cudaEvent_t const*>(opts->stage_events) : nullptr;
    if (ev) MLA_TRY(cudaEventRecord(ev[0], s));
    MLA_TRY(cudaMemsetAsync(b.status, 0, sizeof(int32_t), s));
    // Index build first, in one launch with the front-fold's prep (independent work).
    MLA_LAUNCH(launch_step_start(gather_indices, block_table, positions, b.rows, b.n_valid, b.status,
                                 static_cast<const bf16*>(hidden_states), input_norm_w, d, b.xg3, b.qacc, b.kacc,
                                 b.y32, b.fix, b.flag_count, s));
    if (ev) MLA_TRY(cudaEventRecord(ev[MLA_STAGE_INDEX_RESOLVE + 1], s));
    // The core's work plan rides on an extra block of the q / kv fold.
    const CorePlanArgs plan{b.n_valid, core_tc_head_groups(d), core_clusters(b), b.item_base,
                            core_tc_merge_desc(b.part_ml, core_clusters(b))};
    rc = enqueue_front(d, b, static_cast<const bf16*>(hidden_states), input_norm_w, wq_a, q_norm_w, wq_b, wkv_a,
                       kv_norm_w, q_absorb_w, cos_t, sin_t, kv_cache, slot_mapping, norm_eps, b.qtile, s, n_launches,
                       true, &plan);
    if (rc != MLA_OK) return rc;
    if (ev) MLA_TRY(cudaEventRecord(ev[MLA_STAGE_FRONT_FOLD + 1], s));
    rc = enqueue_back(d, b, b.qtile, kv_cache, out_absorb_w, o_proj_w, out_f32 ? nullptr : out, softmax_scale, s,
                      n_launches, ev ? ev[MLA_STAGE_CORE + 1] : nullptr, ev ? ev[MLA_STAGE_OUT_ABSORB + 1] : nullptr,
                      true, tp);
    if (rc != MLA_OK) return rc;
    if (ev) MLA_TRY(cudaEventRecord(ev[MLA_STAGE_O_PROJ + 1], s));
    if (opts) opts->n_launches = n_launches;
    return MLA_OK;
}

int mla_decode_qkv(const void* hidden_states, const float* input_norm_w, const void* wq_a, const float* q_norm_w,
                   const void* wq_b, const void* wkv_a, const float* kv_norm_w, const void* q_absorb_w,
                   const float* cos_t, const float* sin_t, void* kv_cache, const int32_t* slot_mapping,
                   void* q_tiles, const mla_dims* dims, float norm_eps, void* workspace, size_t workspace_bytes,
                   void* stream) {
    const int dc = check_dims(dims);
    if (dc != MLA_OK) return dc;
    const Dims d = to_dims(*dims);
    if (!std::isfinite(norm_eps) || norm_eps < 0.f) return MLA_ERR_BAD_ARGUMENT;
    if (d.T == 0) return MLA_OK;
    int rc = check_ptrs({hidden_states, input_norm_w, wq_a, q_norm_w, wq_b, wkv_a, kv_norm_w, q_absorb_w, cos_t,
                         sin_t, kv_cache, slot_mapping, q_tiles});
    if (rc != MLA_OK) return rc;
    const Plan pl = make_plan(d);
    rc = check_workspace(pl, workspace, workspace_bytes);
    if (rc != MLA_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const Bufs b = bufs_of(pl, workspace);
    int n_launches = 0;
    MLA_TRY(cudaMemsetAsync(b.status, 0, sizeof(int32_t), s));
    return enqueue_front(d, b, static_cast<const bf16*>(hidden_states), input_norm_w, wq_a, q_norm_w, wq_b, wkv_a,
                         kv_norm_w, q_absorb_w, cos_t, sin_t, kv_cache, slot_mapping, norm_eps,
                         static_cast<bf16*>(q_tiles), s, n_launches, false, nullptr);
}

int mla_decode_attention(const void* q_tiles, const void* kv_cache, const int32_t* block_table,
                         const int32_t* positions, const int32_t* gather_indices, const void* out_absorb_w,
                         const void* o_proj_w, void* out, const mla_dims* dims, float softmax_scale, void* workspace,
                         size_t workspace_bytes, void* stream) {
    const int dc = check_dims(dims);
    if (dc != MLA_OK) return dc;
    const Dims d = to_dims(*dims);
    if (!std::isfinite(softmax_scale)) return MLA_ERR_BAD_ARGUMENT;
    if (d.T == 0) return MLA_OK;
    int rc = check_ptrs({q_tiles, kv_cache, block_table, positions, out_absorb_w, o_proj_w, out});
    if (rc != MLA_OK) return rc;
    if (d.P > 0 && !gather_indices) return MLA_ERR_NULL_POINTER;
    if (d.P > 0 && misaligned(gather_indices)) return MLA_ERR_MISALIGNED;
    const Plan pl = make_plan(d);
    rc = check_workspace(pl, workspace, workspace_bytes);
    if (rc != MLA_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const Bufs b = bufs_of(pl, workspace);
    int n_launches = 0;
    MLA_TRY(cudaMemsetAsync(b.status, 0, sizeof(int32_t), s));
    MLA_TRY(cudaMemsetAsync(b.y32, 0, sizeof(float) * (size_t)d.T * d.H, s));   // o-projection target
    MLA_LAUNCH(launch_index_resolve(gather_indices, block_table, positions, d, b.rows, b.n_valid, b.status, s));
    return enqueue_back(d, b, static_cast<const bf16*>(q_tiles), kv_cache, out_absorb_w, o_proj_w, out,
                        softmax_scale, s, n_launches, nullptr, nullptr, false);
}

int mla_router_launches(int n_tokens, int hidden, int n_experts, int top_k) {
    if (!router_dims_ok(n_tokens, hidden, n_experts, top_k)) return 0;
    return router_launches(hidden, n_experts);
}

size_t mla_router_workspace_bytes(int n_tokens, int hidden, int n_experts, int top_k) {
    if (!router_dims_ok(n_tokens, hidden, n_experts, top_k)) return 0;
    return router_workspace_bytes(n_tokens, hidden, n_experts);
}

int mla_rmsnorm_router_topk(const void* hidden_states, const void* gamma, const void* router_weights,
                            const void* router_bias, int n_tokens, int hidden, int n_experts, int top_k,
                            float eps, int act, void* norm_out, int32_t* topk_idx, void* affinities,
                            void* workspace, size_t workspace_bytes, void* stream) {
    if (n_tokens < 0 || hidden <= 0 || n_experts <= 0 || top_k <= 0) return MLA_ERR_BAD_DIMS;
    if (!std::isfinite(eps) || eps < 0.f || (act != MLA_ROUTER_SIGMOID && act != MLA_ROUTER_SOFTMAX))
        return MLA_ERR_BAD_ARGUMENT;
    if (!router_dims_ok(n_tokens, hidden, n_experts, top_k)) return MLA_ERR_UNSUPPORTED_DIMS;
    if (n_tokens == 0) return MLA_OK;
    int rc = check_ptrs({hidden_states, gamma, router_weights, norm_out, topk_idx, affinities});
    if (rc != MLA_OK) return rc;
    if (router_bias && misaligned(router_bias)) return MLA_ERR_MISALIGNED;
    if (!workspace) return MLA_ERR_NULL_POINTER;
    if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return MLA_ERR_MISALIGNED;
    if (workspace_bytes < router_workspace_bytes(n_tokens, hidden, n_experts)) return MLA_ERR_WORKSPACE_TOO_SMALL;
    int nl = 0;
    MLA_TRY(launch_router_topk(static_cast<const bf16*>(hidden_states), static_cast<const bf16*>(gamma),
                               static_cast<const bf16*>(router_weights), static_cast<const bf16*>(router_bias),
                               n_tokens, hidden, n_experts, top_k, eps, act, static_cast<bf16*>(norm_out), topk_idx,
                               static_cast<bf16*>(affinities), workspace, reinterpret_cast<cudaStream_t>(stream),
                               &nl));
    return MLA_OK;
}

int mla_tp_o_proj_allreduce(const void* o, const void* o_proj_w, int n_tokens, int k_rank, int hidden,
                            const mla_tp_peers* tp, int n_local, void* workspace, void* stream) {
    if (n_tokens < 1 || k_rank < 1 || hidden < 1) return MLA_ERR_BAD_DIMS;
    if (k_rank % 16) return MLA_ERR_UNSUPPORTED_DIMS;
    TpTable t;
    int rc = tp_table_of(tp, hidden, n_local, &t);
    if (rc != MLA_OK) return rc;
    rc = check_ptrs({o, o_proj_w, workspace});
    if (rc != MLA_OK) return rc;
    if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return MLA_ERR_MISALIGNED;
    const long long units = tp_gemm_units(n_tokens, k_rank, hidden);
    if (units * tp->world >= (1LL << 31)) return MLA_ERR_UNSUPPORTED_DIMS;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int32_t* status = static_cast<int32_t*>(workspace);
    int n_launches = 0;
    MLA_TRY(cudaMemsetAsync(status, 0, sizeof(int32_t), s));
    GemmSpec g{};
    g.a = o_proj_w; g.a_rows = n_local * k_rank; g.a_cols = hidden; g.a_mn_major = true;
    g.b = o; g.b_cols = n_local * k_rank; g.b_ld = n_local * k_rank; g.b_rows_alloc = n_tokens; g.n_rows = n_tokens;
    g.m_total = hidden; g.k_total = k_rank; g.groups = n_local; g.a_group_rows = k_rank; g.b_group_cols = k_rank;
    g.accumulate = 1; g.status = status; g.a_evict_first = 1;
    MLA_LAUNCH(launch_gemm_reduce_peers(g, t, hidden, s));
    MLA_LAUNCH(launch_tp_finish(t, tp->rank, n_local, n_tokens, hidden, tp->epoch, (uint32_t)units, status, s));
    return MLA_OK;
}

int mla_ipc_export(const void* dev_ptr, mla_ipc_handle* handle) {
    if (!dev_ptr || !handle) return MLA_ERR_NULL_POINTER;
    CUdeviceptr base = 0;
    if (cuda_failed(cudaFree(nullptr))) return MLA_ERR_CUDA;   // a current context for the driver call
    if (!allocation_base(dev_ptr, &base)) {
        g_last_cuda_error = cudaErrorInvalidDevicePointer;
        return MLA_ERR_CUDA;
    }
    cudaIpcMemHandle_t h;
    MLA_TRY(cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)));
    static_assert(sizeof(h) == sizeof(handle->bytes), "IPC handle size");
    std::memcpy(handle->bytes, &h, sizeof(h));
    handle->offset = reinterpret_cast<CUdeviceptr>(dev_ptr) - base;
    return MLA_OK;
}

int mla_ipc_open(const mla_ipc_handle* handle, void** dev_ptr) {
    if (!handle || !dev_ptr) return MLA_ERR_NULL_POINTER;
    cudaIpcMemHandle_t h;
    std::memcpy(&h, handle->bytes, sizeof(h));
    void* base = nullptr;
    MLA_TRY(cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess));
    *dev_ptr = static_cast<char*>(base) + handle->offset;
    return MLA_OK;
}

int mla_ipc_close(void* dev_ptr) {
    if (!dev_ptr) return MLA_ERR_NULL_POINTER;
    CUdeviceptr base = 0;
    if (!allocation_base(dev_ptr, &base)) {
        g_last_cuda_error = cudaErrorInvalidDevicePointer;
        return MLA_ERR_CUDA;
    }
    MLA_TRY(cudaIpcCloseMemHandle(reinterpret_cast<void*>(base)));
    return MLA_OK;
}

#undef MLA_LAUNCH
#undef MLA_TRY

int mla_block_gather_decode(
    const void* hidden_states, const float* input_norm_w,
    const void* wq_a, const float* q_norm_w, const void* wq_b,
    const void* wkv_a, const float* kv_norm_w,
    const void* q_absorb_w, const void* out_absorb_w, const void* o_proj_w,
    const float* cos_t, const float* sin_t,
    void* kv_cache, const int32_t* slot_mapping,
    const int32_t* block_table, const int32_t* positions,
    const int32_t* gather_indices,
    void* out,
    const mla_dims* dims, float softmax_scale, float norm_eps,
    void* workspace, size_t workspace_bytes, void* stream) {
    return mla_block_gather_decode_ex(hidden_states, input_norm_w, wq_a, q_norm_w, wq_b, wkv_a, kv_norm_w,
                                      q_absorb_w, out_absorb_w, o_proj_w, cos_t, sin_t, kv_cache,
                                      slot_mapping, block_table, positions, gather_indices, out, dims,
                                      softmax_scale, norm_eps, workspace, workspace_bytes, stream, nullptr);
}

}  // extern "C"
