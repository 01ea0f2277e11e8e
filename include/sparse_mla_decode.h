/*
 * sparse_mla_decode.h -- C ABI of the B200 (sm_100a) sparse MLA gather-decode block.
 *
 * One DeepSeek-V3.2 MLA decode step, from the residual stream to the
 * attention-block output, attending only over the prior keys an indexer
 * selected. The operation is the one defined by the page "MLA Attention Block
 * Gather Decode Kernel API Reference" (AWS Neuron NKI library,
 * mla_attention_block_gather_decode), section "API Reference": its signature
 * and one ":param" entry per argument, plus the "Notes" and "Dimensions"
 * sections. The page prints no equations; the computation, as read from the
 * parameter descriptions, is:
 *
 *   for every token t (one decode token per sequence):
 *     xn      = rmsnorm(hidden_states[t], input_norm_w)            (:param input_norm_w)
 *     q       = rmsnorm(xn @ wq_a, q_norm_w) @ wq_b, per head
 *               [q_nope (dn) | q_pe (dr)], head-major               (:param wq_a, q_norm_w, wq_b)
 *     kv      = xn @ wkv_a = [latent (L) | k_pe (dr)]               (:param wkv_a)
 *     row     = [rmsnorm(latent, kv_norm_w) | rope(k_pe)]           (:param kv_norm_w, cos, sin)
 *     kv_cache.flat[slot_mapping[t]] = bf16(row)                    (:param kv_cache, slot_mapping)
 *     q_lat[h]= q_nope[h] @ q_absorb_w[h]; q_pe[h] = rope(q_pe[h])  (:param q_absorb_w)
 *   after ALL rows are written, for every token t and head h:
 *     keys    = { p in gather_indices[t] : 0 <= p <= positions[t] } (:param gather_indices, positions)
 *     row_p   = kv_cache.flat[block_table[t, p / bs] * bs + p % bs] (:param block_table)
 *     s_p     = softmax_scale * (q_lat[h] . row_p[:L] + q_pe[h] . row_p[L:])
 *     ctx     = sum_p softmax(s)_p * row_p[:L]       (the latent part is the value)
 *     o[h]    = out_absorb_w[h] @ ctx                               (:param out_absorb_w)
 *   out[t] = concat_h(o[h]) @ o_proj_w                              (:param o_proj_w)
 *
 * RoPE is "interleaved": adjacent pairs (2i, 2i+1) rotate by the angle whose
 * cosine / sine are cos[t, i] / sin[t, i]. RMSNorm is v / sqrt(mean(v^2) + eps)
 * * gamma with one eps (norm_eps) for all three norms. A token with no kept key
 * gets o = 0. No residual is added: out is this rank's partial block output.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers to caller-owned, contiguous,
 *     row-major memory (e.g. a torch tensor's data_ptr()). The library keeps no
 *     reference to them after the call returns and allocates no device memory:
 *     all scratch lives in the caller's `workspace`.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Work is enqueued asynchronously; the call returns once it is
 *     enqueued. Buffers must stay valid until the stream reaches that point.
 *   - dtypes: bf16 = IEEE bfloat16 stored as 16-bit words; fp32 gammas and
 *     cos/sin; int32 indices.
 *   - Pointers must be 16-byte aligned (MLA_ERR_MISALIGNED otherwise).
 *   - Return value: MLA_OK (0) or a negative MLA_ERR_* code; on error nothing
 *     has been enqueued, except MLA_ERR_CUDA (a launch failed: the stream may
 *     hold part of the step). mla_status_string() names each code.
 *   - Index errors found on the device (a block id outside [0, n_blocks), a
 *     kept position beyond the block table, a slot outside the cache) do not
 *     fault: the key is treated as masked / the row is not written, and a bit
 *     is set in a status word inside the workspace (MLA_DEV_* below), readable
 *     with mla_get_device_status().
 */
#ifndef SPARSE_MLA_DECODE_H
#define SPARSE_MLA_DECODE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes. */
#define MLA_OK                       0
#define MLA_ERR_NULL_POINTER        -1  /* a required pointer is NULL                         */
#define MLA_ERR_BAD_DIMS            -2  /* a dimension is <= 0 or inconsistent                  */
#define MLA_ERR_UNSUPPORTED_DIMS    -3  /* valid, but outside what the kernels are built for    */
#define MLA_ERR_MISALIGNED          -4  /* a pointer is not 16-byte aligned                     */
#define MLA_ERR_WORKSPACE_TOO_SMALL -5  /* workspace_bytes < mla_block_workspace_bytes(dims)    */
#define MLA_ERR_CUDA                -6  /* a CUDA runtime call or kernel launch failed          */
#define MLA_ERR_BAD_ARGUMENT        -7  /* a scalar argument is out of range (e.g. eps < 0)     */

/* Bits of the device status word (sticky within one call; cleared at the start of each call). */
#define MLA_DEV_BAD_BLOCK_ID        0x1 /* block_table entry outside [0, n_blocks): key masked  */
#define MLA_DEV_BAD_LOGICAL_BLOCK   0x2 /* kept position p with p / block_size >= max_blocks    */
#define MLA_DEV_BAD_SLOT            0x4 /* slot_mapping outside [0, n_blocks*block_size): row
                                           not written                                         */
#define MLA_DEV_WAIT_TIMEOUT        0x8 /* a bounded on-device wait gave up (output invalid)    */

/*
 * Problem dimensions. Names follow the page's parameters and its "Dimensions"
 * section; the page infers most of them from tensor shapes, the C ABI takes
 * them explicitly.
 *   n_tokens            decode tokens in the batch, one per sequence (T)
 *   hidden              residual width (H)
 *   q_lora_rank         query latent width (Lq)
 *   kv_lora_rank        KV latent width = latent width of a cache row (L)
 *   qk_nope_head_dim    per-head query/key width RoPE does not rotate (dn)
 *   qk_rope_head_dim    per-head query/key width RoPE rotates (dr, even)
 *   v_head_dim          per-head value width (dv)
 *   n_heads             attention heads on this rank (h)
 *   block_size          cache rows per physical block (bs)
 *   n_blocks            physical blocks in kv_cache
 *   max_blocks_per_seq  columns of block_table
 *   n_prior             selected prior keys per token = columns of gather_indices (P)
 * kv_row_dim = kv_lora_rank + qk_rope_head_dim (R).
 */
typedef struct mla_dims {
    int32_t n_tokens;
    int32_t hidden;
    int32_t q_lora_rank;
    int32_t kv_lora_rank;
    int32_t qk_nope_head_dim;
    int32_t qk_rope_head_dim;
    int32_t v_head_dim;
    int32_t n_heads;
    int32_t block_size;
    int32_t n_blocks;
    int32_t max_blocks_per_seq;
    int32_t n_prior;
} mla_dims;

/*
 * Bytes of device scratch mla_block_gather_decode() needs for `dims`
 * (0 if dims are invalid or unsupported). Host-only; touches no GPU.
 */
size_t mla_block_workspace_bytes(const mla_dims* dims);

/*
 * Checks `dims` against what the kernels support. Returns MLA_OK,
 * MLA_ERR_BAD_DIMS or MLA_ERR_UNSUPPORTED_DIMS. Host-only; touches no GPU.
 */
int mla_block_check_dims(const mla_dims* dims);

/*
 * One decode step of the block (the page's mla_attention_block_gather_decode).
 *
 * Inputs (device, read-only):
 *   hidden_states  [T, H]                    bf16  this step's residual-stream hidden states
 *   input_norm_w   [H]        (page: [1,H])  fp32  RMSNorm gamma of the layer input
 *   wq_a           [H, Lq]                   bf16  query down-projection
 *   q_norm_w       [Lq]       (page: [1,Lq]) fp32  RMSNorm gamma of the query latent
 *   wq_b           [Lq, h*(dn+dr)]           bf16  query up-projection; column block
 *                                                   h*(dn+dr) .. holds head h's [q_nope | q_pe]
 *   wkv_a          [H, L+dr]                 bf16  KV down-projection: one cache row per token
 *   kv_norm_w      [L]        (page: [1,L])  fp32  RMSNorm gamma of the KV latent
 *   q_absorb_w     [h, dn, L]                bf16  nope half of wkv_b (nope query -> latent)
 *   out_absorb_w   [h, dv, L]                bf16  value half of wkv_b (latent -> value width)
 *   o_proj_w       [h*dv, H]                 bf16  this rank's shard of the o-projection
 *   cos, sin       [T, dr/2]                 fp32  interleaved-RoPE tables of each token
 *   slot_mapping   [T]                       int32 flat cache row each token's own key goes to
 *   block_table    [T, max_blocks_per_seq]   int32 logical -> physical block map per sequence
 *   positions      [T]                       int32 absolute position of each token
 *   gather_indices [T, P]                    int32 selected absolute prior positions, any order
 * In/out:
 *   kv_cache       [n_blocks, 1, bs, L+dr]   bf16  paged cache, MUTATED IN PLACE: row
 *                                                   slot_mapping[t] is overwritten with token t's
 *                                                   [rmsnorm(latent) | rope(k_pe)]; all T rows
 *                                                   are written before any selected row is read.
 *                                                   Two tokens with one slot: undefined.
 * Output:
 *   out            [T, H]                    bf16  attention-block output (no residual)
 * Scalars:
 *   softmax_scale  score scale (conventionally 1/sqrt(dn+dr)); finite
 *   norm_eps       epsilon of every RMSNorm (page default 1e-6); >= 0
 * Scratch:
 *   workspace      device buffer of >= mla_block_workspace_bytes(dims) bytes, 256-byte
 *                  aligned, owned by the caller, not shared by calls in flight at once.
 * Keys with p < 0 or p > positions[t] are masked and never dereferenced; a
 * duplicated index counts as two keys.
 */
int mla_block_gather_decode(
    const void* hidden_states, const float* input_norm_w,
    const void* wq_a, const float* q_norm_w, const void* wq_b,
    const void* wkv_a, const float* kv_norm_w,
    const void* q_absorb_w, const void* out_absorb_w, const void* o_proj_w,
    const float* cos, const float* sin,
    void* kv_cache, const int32_t* slot_mapping,
    const int32_t* block_table, const int32_t* positions,
    const int32_t* gather_indices,
    void* out,
    const mla_dims* dims, float softmax_scale, float norm_eps,
    void* workspace, size_t workspace_bytes, void* stream);

/*
 * Stage boundaries of one step, in launch order. mla_block_gather_decode_ex()
 * can record a caller-created cudaEvent_t after each stage so the caller can
 * time the stages live on its stream.
 */
#define MLA_STAGE_INDEX_RESOLVE  0  /* gather_indices -> cache rows, causal mask     */
#define MLA_STAGE_FRONT_FOLD     1  /* norms, projections, RoPE, cache write, q tile */
#define MLA_STAGE_CORE           2  /* gathered latent attention                      */
#define MLA_STAGE_OUT_ABSORB     3  /* out_absorb_w                                   */
#define MLA_STAGE_O_PROJ         4  /* o_proj_w -> out                                */
#define MLA_N_STAGES             5

/*
 * Launch options of mla_block_gather_decode_ex(). Zero-initialise unused fields.
 *   stage_events   NULL, or MLA_N_STAGES + 1 cudaEvent_t handles (as void*):
 *                  events[0] is recorded before the first stage and events[i+1]
 *                  after stage i. The caller creates and destroys them.
 *   n_launches     out: number of kernels this call enqueued (0 on error).
 *   out_f32        NULL, or [T, hidden] fp32 device memory (16-byte aligned,
 *                  caller-owned): the o-projection's fp32 sums are written there
 *                  and `out` is not written (it may then be NULL). With a head
 *                  shard of the weights this is the rank's partial output of a
 *                  tensor-parallel split over heads, summed across ranks before
 *                  one bf16 rounding (the page's "this rank" output, in fp32).
 *   tp             NULL, or the peer table of a head split (mla_tp.h): the
 *                  weights are rank tp->rank's head shard, the o-projection's
 *                  tiles are reduced into the owning ranks' accumulators and the
 *                  call returns when tp->out[tp->rank] holds the bf16 sum over
 *                  all ranks (`out` is not used; out_f32 must be NULL). Every
 *                  rank makes the call with the same dims and epoch.
 */
typedef struct mla_launch_opts {
    void* const* stage_events;
    int32_t n_launches;
    int32_t reserved;
    float* out_f32;
    const struct mla_tp_peers* tp;
} mla_launch_opts;

/* mla_block_gather_decode() with launch options (opts may be NULL). */
int mla_block_gather_decode_ex(
    const void* hidden_states, const float* input_norm_w,
    const void* wq_a, const float* q_norm_w, const void* wq_b,
    const void* wkv_a, const float* kv_norm_w,
    const void* q_absorb_w, const void* out_absorb_w, const void* o_proj_w,
    const float* cos, const float* sin,
    void* kv_cache, const int32_t* slot_mapping,
    const int32_t* block_table, const int32_t* positions,
    const int32_t* gather_indices,
    void* out,
    const mla_dims* dims, float softmax_scale, float norm_eps,
    void* workspace, size_t workspace_bytes, void* stream, mla_launch_opts* opts);

/*
 * Separate-kernel path, first half: the front-fold of the decode step on its own.
 * The page "MLA Attention Block Gather Decode Kernel API Reference" (introduction
 * and "Notes") sets the fused block against a separate QKV kernel and attention
 * kernel that hand the query tiles over through HBM; these two calls are that
 * separate path, built from the same kernels as mla_block_gather_decode().
 *
 * Computes the input RMSNorm, the down-projections, the q and kv RMSNorms, the
 * up-projection with RoPE and the absorption, writes this step's latent cache
 * rows (kv_cache at slot_mapping, as mla_block_gather_decode) and the query tiles
 *   q_tiles  [T, n_heads, kv_lora_rank + qk_rope_head_dim] bf16, row (t, head) =
 *            [q_lat (kv_lora_rank) | rotated q_pe (qk_rope_head_dim)],
 *            caller-owned device memory, 16-byte aligned, fully overwritten.
 * Other arguments as in mla_block_gather_decode() (dims->n_prior and the
 * indexing arrays are not used here). The workspace is sized by
 * mla_block_workspace_bytes() and may be the one mla_decode_attention() uses.
 * Clears the workspace's device status word at its start (read it with
 * mla_get_device_status()). Returns MLA_OK or a negative MLA_ERR_* code, with
 * nothing enqueued unless the code is MLA_ERR_CUDA.
 */
int mla_decode_qkv(const void* hidden_states, const float* input_norm_w, const void* wq_a, const float* q_norm_w,
                   const void* wq_b, const void* wkv_a, const float* kv_norm_w, const void* q_absorb_w,
                   const float* cos, const float* sin, void* kv_cache, const int32_t* slot_mapping,
                   void* q_tiles, const mla_dims* dims, float norm_eps, void* workspace, size_t workspace_bytes,
                   void* stream);

/*
 * Separate-kernel path, second half: index resolve (gather_indices, block_table,
 * positions), sparse latent attention of q_tiles (as written by mla_decode_qkv)
 * over the kept prior rows of kv_cache (read only), out absorption and
 * o-projection into out [T, hidden] bf16 (caller-owned, overwritten).
 * Enqueue it after mla_decode_qkv() of the same step, so that this step's cache
 * rows are in place. Arguments as in mla_block_gather_decode(); same return
 * codes; clears the workspace's device status word at its start.
 */
int mla_decode_attention(const void* q_tiles, const void* kv_cache, const int32_t* block_table,
                         const int32_t* positions, const int32_t* gather_indices, const void* out_absorb_w,
                         const void* o_proj_w, void* out, const mla_dims* dims, float softmax_scale, void* workspace,
                         size_t workspace_bytes, void* stream);

/*
 * Size of the built-in scratch array used by mla_block_gather_decode_noalloc():
 * 8 MiB, held on every GPU that loads this library until the process exits.
 */
#define MLA_NOALLOC_SCRATCH_BYTES (8u << 20)

/*
 * The block step without a workspace argument, for callers that cannot
 * allocate device memory (for example a plugin inside a serving engine that
 * owns all device memory through its own pool, or code that must not call
 * the CUDA allocator while it builds a stream). The page has no counterpart to
 * this entry point; it exists only for such callers.
 *
 * Arguments are those of mla_block_gather_decode() minus workspace and
 * workspace_bytes; inputs and the output are still the caller's. The scratch
 * is a fixed device array of MLA_NOALLOC_SCRATCH_BYTES inside the library:
 *   - dims whose mla_block_workspace_bytes() exceeds it are rejected with
 *     MLA_ERR_WORKSPACE_TOO_SMALL before anything is enqueued;
 *   - the first call on each device (with that device current) looks up the
 *     array's device address and may load the module: make that first call
 *     before any stream capture;
 *   - all calls share the array and it keeps the last call's contents; the
 *     step clears what must start at zero itself. Calls that overlap on the
 *     GPU race on it: the caller must serialise them;
 *   - the device status word (MLA_DEV_* bits of the step) sits inside that
 *     array; mla_block_gather_decode_noalloc_status() reads it.
 * Nothing in this call allocates device or pinned memory.
 */
int mla_block_gather_decode_noalloc(
    const void* hidden_states, const float* input_norm_w,
    const void* wq_a, const float* q_norm_w, const void* wq_b,
    const void* wkv_a, const float* kv_norm_w,
    const void* q_absorb_w, const void* out_absorb_w, const void* o_proj_w,
    const float* cos, const float* sin,
    void* kv_cache, const int32_t* slot_mapping,
    const int32_t* block_table, const int32_t* positions,
    const int32_t* gather_indices,
    void* out,
    const mla_dims* dims, float softmax_scale, float norm_eps, void* stream);

/*
 * Device status word of the most recent mla_block_gather_decode_noalloc() call
 * on the current device: waits for `stream` (the stream that call was made
 * on), then stores the OR of its MLA_DEV_* bits (0 = clean) in *status. Like
 * the step itself it allocates nothing; the page has no counterpart to it.
 * Returns MLA_OK, MLA_ERR_NULL_POINTER or MLA_ERR_CUDA.
 */
int mla_block_gather_decode_noalloc_status(void* stream, int32_t* status);

/*
 * Waits for `stream`, then stores the device status word of the last call
 * that used `workspace` (OR of MLA_DEV_* bits; 0 = clean) in *status.
 * Returns MLA_OK, MLA_ERR_NULL_POINTER or MLA_ERR_CUDA.
 */
int mla_get_device_status(const void* workspace, void* stream, int32_t* status);

/* Static, NUL-terminated description of an MLA_* return code. Never NULL. */
const char* mla_status_string(int code);

/*
 * Name and description of the CUDA runtime error behind the calling host
 * thread's most recent MLA_ERR_CUDA return ("no error" if none has occurred).
 * Static or runtime-owned storage; never NULL. Diagnostic only.
 */
const char* mla_last_cuda_error_string(void);

/* ABI version: (major << 16) | minor (1.4 adds mla_block_gather_decode_noalloc_status). */
int32_t mla_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SPARSE_MLA_DECODE_H */
