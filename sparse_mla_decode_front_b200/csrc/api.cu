// C ABI of the sparse MLA gather-decode block: validation, workspace plan and
// the launch chain on the caller's stream. The operation is the one of the
// page "MLA Attention Block Gather Decode Kernel API Reference"
// (mla_attention_block_gather_decode, section "API Reference"); every argument
// is documented in include/sparse_mla_decode.h.
#include <cmath>
#include <cstring>

#include "common.cuh"
#include "launch.h"

namespace mla {
namespace {

constexpr size_t kAlign = 256;

inline size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

// Workspace regions, in order. Offsets are multiples of kAlign.
struct Plan {
    size_t status, rows, n_valid, r_in, xn, q_a, kv, q_an, q, qtile, ctx, o, total;
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
    p.xn = take(sizeof(float) * T * d.H);
    p.q_a = take(sizeof(float) * T * d.Lq);
    p.kv = take(sizeof(double) * T * d.R());
    p.q_an = take(sizeof(float) * T * d.Lq);
    p.q = take(sizeof(float) * T * d.h * d.qk());
    p.qtile = take(sizeof(bf16) * T * d.h * d.R());
    p.ctx = take(sizeof(float) * T * d.h * d.L);
    p.o = take(sizeof(float) * T * d.h * d.dv);
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
    if (!core_simt_supports(d)) return MLA_ERR_UNSUPPORTED_DIMS;
    return MLA_OK;
}

inline bool misaligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

}  // namespace
}  // namespace mla

using namespace mla;

extern "C" {

int32_t mla_abi_version(void) { return (1 << 16) | 0; }

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

int mla_block_check_dims(const mla_dims* dims) { return check_dims(dims); }

size_t mla_block_workspace_bytes(const mla_dims* dims) {
    if (check_dims(dims) != MLA_OK) return 0;
    return make_plan(to_dims(*dims)).total;
}

int mla_get_device_status(const void* workspace, void* stream, int32_t* status) {
    if (!workspace || !status) return MLA_ERR_NULL_POINTER;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int32_t v = 0;
    if (cudaMemcpyAsync(&v, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return MLA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MLA_ERR_CUDA;
    *status = v;
    return MLA_OK;
}

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
    const void* need[] = {hidden_states, input_norm_w, wq_a, q_norm_w, wq_b, wkv_a, kv_norm_w,
                          q_absorb_w, out_absorb_w, o_proj_w, cos_t, sin_t, kv_cache,
                          slot_mapping, block_table, positions, out, workspace};
    for (const void* p : need)
        if (!p) return MLA_ERR_NULL_POINTER;
    if (d.P > 0 && !gather_indices) return MLA_ERR_NULL_POINTER;
    for (const void* p : need)
        if (misaligned(p)) return MLA_ERR_MISALIGNED;
    if (d.P > 0 && misaligned(gather_indices)) return MLA_ERR_MISALIGNED;
    if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return MLA_ERR_MISALIGNED;
    const Plan pl = make_plan(d);
    if (workspace_bytes < pl.total) return MLA_ERR_WORKSPACE_TOO_SMALL;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    int32_t* status = reinterpret_cast<int32_t*>(ws + pl.status);
    int32_t* rows = reinterpret_cast<int32_t*>(ws + pl.rows);
    int32_t* n_valid = reinterpret_cast<int32_t*>(ws + pl.n_valid);
    double* r_in = reinterpret_cast<double*>(ws + pl.r_in);
    float* xn = reinterpret_cast<float*>(ws + pl.xn);
    float* q_a = reinterpret_cast<float*>(ws + pl.q_a);
    double* kv = reinterpret_cast<double*>(ws + pl.kv);
    float* q_an = reinterpret_cast<float*>(ws + pl.q_an);
    float* q = reinterpret_cast<float*>(ws + pl.q);
    bf16* qtile = reinterpret_cast<bf16*>(ws + pl.qtile);
    float* ctx = reinterpret_cast<float*>(ws + pl.ctx);
    float* o = reinterpret_cast<float*>(ws + pl.o);

    const bf16* x = static_cast<const bf16*>(hidden_states);
    const int nq = d.h * d.qk();
    int n_launches = 0;
    cudaEvent_t const* ev = opts && opts->stage_events
                                ? reinterpret_cast<cudaEvent_t const*>(opts->stage_events) : nullptr;
#define MLA_TRY(expr)                                  \
    do {                                               \
        if ((expr) != cudaSuccess) return MLA_ERR_CUDA; \
    } while (0)
#define MLA_LAUNCH(expr) \
    do {                 \
        MLA_TRY(expr);   \
        ++n_launches;    \
    } while (0)
#define MLA_STAGE_DONE(i) \
    do {                  \
        if (ev) MLA_TRY(cudaEventRecord(ev[(i) + 1], s)); \
    } while (0)
    if (ev) MLA_TRY(cudaEventRecord(ev[0], s));
    MLA_TRY(cudaMemsetAsync(status, 0, sizeof(int32_t), s));
    // Index build first: it does not depend on the front-fold.
    MLA_LAUNCH(launch_index_resolve(gather_indices, block_table, positions, d, rows, n_valid, status, s));
    MLA_STAGE_DONE(MLA_STAGE_INDEX_RESOLVE);
    // Front-fold.
    MLA_LAUNCH(launch_fold_prep(x, input_norm_w, d, norm_eps, r_in, xn, s));
    MLA_LAUNCH(launch_gemm_simt_f32(xn, d.H, static_cast<const bf16*>(wq_a), d.Lq, q_a, d.Lq, d.T, d.Lq, d.H, s));
    MLA_LAUNCH(launch_kv_down_f64(x, input_norm_w, static_cast<const bf16*>(wkv_a), r_in, d, kv, s));
    MLA_LAUNCH(launch_fold_norm(q_a, q_norm_w, kv, kv_norm_w, cos_t, sin_t, slot_mapping, d, norm_eps, q_an,
                                static_cast<bf16*>(kv_cache), status, s));
    MLA_LAUNCH(launch_gemm_simt_f32(q_an, d.Lq, static_cast<const bf16*>(wq_b), nq, q, nq, d.T, nq, d.Lq, s));
    MLA_LAUNCH(launch_q_absorb_rope(q, static_cast<const bf16*>(q_absorb_w), cos_t, sin_t, d, qtile, s));
    MLA_STAGE_DONE(MLA_STAGE_FRONT_FOLD);
    // Core: after every row of this step is in the cache (stream order).
    MLA_LAUNCH(launch_core_simt(qtile, static_cast<const bf16*>(kv_cache), rows, n_valid, d, softmax_scale, ctx, s));
    MLA_STAGE_DONE(MLA_STAGE_CORE);
    MLA_LAUNCH(launch_out_absorb_simt(ctx, static_cast<const bf16*>(out_absorb_w), d, o, s));
    MLA_STAGE_DONE(MLA_STAGE_OUT_ABSORB);
    MLA_LAUNCH(launch_gemm_simt_bf16(o, d.h * d.dv, static_cast<const bf16*>(o_proj_w), d.H,
                                     static_cast<bf16*>(out), d.H, d.T, d.H, d.h * d.dv, s));
    MLA_STAGE_DONE(MLA_STAGE_O_PROJ);
#undef MLA_STAGE_DONE
#undef MLA_LAUNCH
#undef MLA_TRY
    if (opts) opts->n_launches = n_launches;
    return MLA_OK;
}

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
