/* Fused RMSNorm + router top-K of a MoE decoder layer, on B200 (sm_100a).
 *
 * The operation of the page "RMSNorm Router Top-K A2AV Kernel API Reference"
 * (AWS Neuron NKI library, rmsnorm_router_topk_a2av), API Reference and Notes:
 * for each token row x of hidden_states,
 *   norm   = x / sqrt(mean(x^2) + eps) * gamma             (returned, bf16)
 *   logits = norm @ router_weights (+ router_bias)          (fp32, not returned)
 *   the top_k experts with the largest raw logits (largest first; equal logits by
 *   increasing expert index) -> topk_idx, and the activation of the selected
 *   logits only -> affinities (0 for every other expert): SIGMOID per selected
 *   logit, or SOFTMAX over the top_k selected logits.
 * The router reads the normalised states before their bf16 store.
 *
 * Same library and error codes as sparse_mla_decode.h (MLA_OK, MLA_ERR_*).
 */
#ifndef MOE_ROUTER_H
#define MOE_ROUTER_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { MLA_ROUTER_SIGMOID = 0, MLA_ROUTER_SOFTMAX = 1 };

/* Workspace bytes for n_tokens x hidden tokens and n_experts experts (status word,
 * the grid barrier's count and the fp32 partial logits of the single launch, or the
 * x*gamma slices and fp32 logit sums of the three-launch form: enough for either),
 * or 0 if the sizes are unsupported (mla_rmsnorm_router_topk's limits). Host only. */
size_t mla_router_workspace_bytes(int n_tokens, int hidden, int n_experts, int top_k);

/* Kernels mla_rmsnorm_router_topk enqueues for these sizes on the calling host
 * thread's current device: 1 when the experts fit four groups of 64 and the hidden
 * size fits the single cooperative launch's K slices on that device's SMs (the
 * partial logits, a grid barrier and the finish in one kernel), else 3 (prep,
 * projection, finish); 0 if the sizes are unsupported. Host only. */
int mla_router_launches(int n_tokens, int hidden, int n_experts, int top_k);

/* Enqueue the step on `stream` (a cudaStream_t; NULL = legacy default stream).
 *
 *   hidden_states   [n_tokens, hidden] bf16, row-major (device)
 *   gamma           [hidden] bf16 RMSNorm scale (device)
 *   router_weights  [hidden, n_experts] bf16, row-major (device)
 *   router_bias     [n_experts] bf16 (device), or NULL for none
 *   eps             RMSNorm epsilon (finite, >= 0)
 *   act             MLA_ROUTER_SIGMOID or MLA_ROUTER_SOFTMAX
 *   norm_out        [n_tokens, hidden] bf16 (device, written)
 *   topk_idx        [n_tokens, top_k] int32 (device, written), largest logit first
 *   affinities      [n_tokens, n_experts] bf16 (device, written), masked
 *   workspace       >= mla_router_workspace_bytes(...) bytes of device memory,
 *                   256-byte aligned, caller-owned; its first int32 is the device
 *                   status word (read it with mla_get_device_status)
 *
 * Limits: hidden a multiple of 16; 64 <= n_experts <= 1024, a multiple of 16;
 * 1 <= top_k <= min(n_experts, 32); n_tokens >= 0 (0: nothing to do). Device
 * pointers 16-byte aligned. Errors (nothing is enqueued): MLA_ERR_NULL_POINTER,
 * MLA_ERR_MISALIGNED, MLA_ERR_BAD_DIMS (negative sizes, eps or act out of range),
 * MLA_ERR_UNSUPPORTED_DIMS (outside the limits), MLA_ERR_WORKSPACE_TOO_SMALL;
 * MLA_ERR_CUDA if a launch fails. Asynchronous; the caller owns every buffer. */
int mla_rmsnorm_router_topk(const void* hidden_states, const void* gamma, const void* router_weights,
                            const void* router_bias, int n_tokens, int hidden, int n_experts, int top_k,
                            float eps, int act, void* norm_out, int32_t* topk_idx, void* affinities,
                            void* workspace, size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_ROUTER_H */
