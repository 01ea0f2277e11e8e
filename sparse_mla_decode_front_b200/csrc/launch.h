// Internal launchers of the stage kernels (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace mla {

cudaError_t launch_index_resolve(const int32_t* gather_indices, const int32_t* block_table,
                                 const int32_t* positions, const Dims& d, int32_t* rows,
                                 int32_t* n_valid, int32_t* status, cudaStream_t s);

// Tensor-core projection GEMM (see gemm_tc.cuh): D[M, N] = A x B^T per group.
struct GemmSpec {
    const void* a;          // A storage: a_rows x a_cols bf16, row-major
    int a_rows, a_cols;
    bool a_mn_major;        // true: rows are K (weight [in, out]); false: rows are M
    const void* b;          // B storage: rows of b_ld bf16, b_cols used, b_rows_alloc rows
    int b_cols, b_ld, b_rows_alloc;
    int n_rows;             // N (tokens)
    int m_total, k_total;   // per group
    int groups, a_group_rows, b_group_cols;
    int accumulate;         // 1: fp32 reduction epilogue with stream-K; 0: storing epilogue
    int32_t* status;
    int a_evict_first;      // 1: A's lines are the first to leave L2 (weights read once)
    int splits;             // accumulate: > 0 forces split-K with this many K slices; 0 chooses
    int m_pair;             // 1: two feature tiles per CTA tile share each token tile (MN-major A,
                            //    token tiles of at most 128 rows; a two-problem launch pairs both
                            //    problems or neither)
};
int gemm_bn_for(int rows);
cudaError_t launch_gemm_reduce_f32(GemmSpec const& g, float* out, int ldo, int group_off, cudaStream_t s);
cudaError_t launch_gemm_store_bf16(GemmSpec const& g, bf16* out, int ldo, int group_off, cudaStream_t s);
// Two MN-major, single-group reducing projections sharing B and K, in one launch.
cudaError_t launch_gemm_reduce_f32_pair(GemmSpec const& g0, float* out0, int ldo0, GemmSpec const& g1, float* out1,
                                        int ldo1, cudaStream_t s);
// Query chain (qchain_tc.cu): per head, the wq_b up-projection, q RoPE and the q_absorb_w
// absorption in one CTA, writing the query tile qtile [T, h, L + dr] = [q_lat | rotated q_pe].
bool q_chain_supports(const Dims& d);
cudaError_t launch_q_chain(const bf16* q_an, const void* wq_b, const void* q_absorb_w, const float* cos_t,
                           const float* sin_t, const Dims& d, bf16* qtile, int32_t* status, cudaStream_t s);

cudaError_t launch_fold_prep_tc(const bf16* x, const float* gamma, const Dims& d, bf16* xg3, float* qacc,
                                float* kacc, float* y32, double* fix, int32_t* flag_count, cudaStream_t s);
// The attention core's work plan (item first tiles, merge plan), computed by one extra
// block of the q / kv fold when given.
struct CorePlanArgs {
    const int32_t* n_valid;
    int HG, max_clusters;
    int32_t* item_base;
    int4* merge_desc;
};
// Per token: input RMS, q RMSNorm (q_an), the fp32 kv row and its flagged elements; an
// extra block computes the core's work plan when `plan` is given.
cudaError_t launch_fold_q_kv(const bf16* x, const float* qacc, const float* kacc, const float* q_norm_w,
                             const float* cos_t, const float* sin_t, const Dims& d, float eps, double* r_in,
                             bf16* q_an, float* kv_f32, int32_t* flag_count, int32_t* flag_list,
                             const CorePlanArgs* plan, cudaStream_t s);
// The cache rows: exact fp64 fix-up of the flagged elements, then kv RMSNorm + k RoPE and the
// row write at slot_mapping (two launches on `s`).
cudaError_t launch_kv_fix_row(const bf16* x, const float* gamma_in, const bf16* wkv_a, const float* kv_norm_w,
                              const float* cos_t, const float* sin_t, const int32_t* slot_mapping, const Dims& d,
                              float eps, const double* r_in, const float* kv_f32, const int32_t* flag_count,
                              const int32_t* flag_list, double* fix, bf16* kv_cache, int32_t* status,
                              cudaStream_t s);
// Index resolve (blocks [0, T)) and the front-fold prep (blocks [T, 2T)) in one launch.
cudaError_t launch_step_start(const int32_t* gather_indices, const int32_t* block_table, const int32_t* positions,
                              int32_t* rows, int32_t* n_valid, int32_t* status, const bf16* x, const float* gamma,
                              const Dims& d, bf16* xg3, float* qacc, float* kacc, float* y32, double* fix,
                              int32_t* flag_count, cudaStream_t s);
cudaError_t launch_f32_to_bf16(const float* in, bf16* out, size_t n, cudaStream_t s);

// Tensor parallelism over heads, o-projection reduced into the owners' accumulators
// (tp_reduce.cu; the table mirrors mla_tp_peers).
constexpr int kTpMaxRanks = 8;
struct TpTable {
    float* acc[kTpMaxRanks];
    bf16* out[kTpMaxRanks];
    uint32_t* flags[kTpMaxRanks];   // [0]: o-projection K blocks arrived, [1]: output shards arrived
    int world;
};
// o-projection over n_local groups (ranks), each tile reduced into its owner's acc. MN-major
// weights only; feature tiles paired whenever the token tile allows (what tp_gemm_units counts).
cudaError_t launch_gemm_reduce_peers(GemmSpec const& g, const TpTable& t, int hidden, cudaStream_t s);
// K blocks one rank's o-projection processes (its arrivals at every owner per step).
long long tp_gemm_units(int n_tokens, int k_rank, int hidden);
// Waits for every rank's sums, rounds ranks [rank0, rank0 + n_local)'s shards, writes
// them into every rank's output and waits until this GPU's outputs are complete.
cudaError_t launch_tp_finish(const TpTable& t, int rank0, int n_local, int T, int H, uint32_t epoch,
                             uint32_t units_per_rank, int32_t* status, cudaStream_t s);

// Fused RMSNorm + router top-K (router_topk.cu). act: 0 sigmoid, 1 softmax over the selected.
bool router_dims_ok(int T, int H, int E, int K);
size_t router_workspace_bytes(int T, int H, int E);
int router_launches(int H, int E);   // kernels launch_router_topk enqueues on the current device
cudaError_t launch_router_topk(const bf16* x, const bf16* gamma, const bf16* w, const bf16* bias, int T, int H, int E,
                               int K, float eps, int act, bf16* norm_out, int32_t* idx_out, bf16* aff_out,
                               void* workspace, cudaStream_t s, int* n_launches);

// 2-D bf16 tensor map with a 128-byte (default) or 64-byte swizzle.
bool make_tma_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                 uint32_t box_inner, uint32_t box_outer, int swizzle_bytes = 128);

// Tensor-core attention core (core_tc.cu).
constexpr int kCoreMaxClusters = 80;   // >= the 2-CTA clusters a B200 holds at once (148 SMs)
bool core_tc_supports(const Dims& d);
int core_tc_head_groups(const Dims& d);                       // work items per token
int core_tc_max_clusters();                                   // co-resident clusters on this device
int core_tc_cluster_bound(const Dims& d);                     // clusters the dims can use (host-only)
size_t core_tc_partial_bytes(const Dims& d, int max_clusters);
size_t core_tc_ml_bytes(int max_clusters);
// plan_done: the work plan was already written (the q / kv fold's plan block), else the
// plan kernel runs first. core_tc_merge_desc: where the merge plan lives in part_ml.
cudaError_t launch_core_tc(const bf16* qtile, const bf16* kv_cache, const int32_t* rows, const int32_t* n_valid,
                           int32_t* item_base, const Dims& d, float scale, bf16* ctx, bf16* part_o, float* part_ml,
                           int max_clusters, bool plan_done, int32_t* status, cudaStream_t s);
int4* core_tc_merge_desc(float* part_ml, int max_clusters);

}  // namespace mla
