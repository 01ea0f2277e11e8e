/* Tensor parallelism over heads with the o-projection's reduction fused into it,
 * on B200 (sm_100a) over NVLink peer memory.
 *
 * The page "MLA Attention Block Gather Decode Kernel API Reference" (introduction,
 * :param n_heads, o_proj_w) returns "this rank's" attention-block output: with the
 * heads split over ranks, each rank's o-projection covers its heads' rows of
 * o_proj_w and the block output is the sum of the ranks' partial outputs. Here
 * that sum is formed inside the projection: every output tile the o-projection
 * finishes is added in fp32 straight into the accumulator of the rank that owns
 * its columns (hidden / world columns per rank, over NVLink when that rank is
 * another GPU), so the transfer overlaps the rest of the projection. Then each
 * rank rounds its columns once to bf16 and writes them into every rank's output
 * (an all-gather by stores), and returns when its own output is complete.
 *
 * Ranks meet through two arrival counters per rank (device-scope atomics with
 * system-scope release / acquire), each wait bounded in time: a rank that never
 * arrives makes the others set MLA_DEV_WAIT_TIMEOUT in their status word and
 * return instead of hanging.
 *
 * Same library and error codes as sparse_mla_decode.h (MLA_OK, MLA_ERR_*).
 */
#ifndef MLA_TP_H
#define MLA_TP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MLA_TP_MAX_WORLD 8

/*
 * The buffers of every rank of a head split, as device pointers this GPU can
 * address (its own allocations, and the peers' mapped with mla_ipc_open()).
 * Every rank passes the same table, entries in rank order.
 *   world   ranks of the split, 1..MLA_TP_MAX_WORLD; hidden % (32 * world) == 0
 *   rank    the rank this call computes (its first rank, see n_local below)
 *   epoch   this step's number for these buffers: 1 for the first step, then
 *           +1 per step, the same on every rank (modulo 2^32). It is a kernel
 *           argument: a captured CUDA graph would replay one step's epoch, so
 *           enqueue these calls as stream launches.
 *   acc[r]  rank r's fp32 accumulator [n_tokens, hidden / world] (its columns
 *           [r * hidden / world, (r + 1) * hidden / world) of the output);
 *           zero before the first step, and left zero by every step
 *   out[r]  rank r's bf16 block output [n_tokens, hidden], row-major
 *   flags[r] rank r's two uint32 arrival counters; zero before the first step
 * All pointers 16-byte aligned. A rank must have consumed (or copied) its `out`
 * of one step before its next step's o-projection starts on its stream; this
 * holds when the next step is enqueued after the consumer on the same stream.
 * The zero fills must have completed before any rank's first step. After a step
 * that set MLA_DEV_WAIT_TIMEOUT on any rank the counters and accumulators no
 * longer agree: every rank zeroes them again (and restarts epoch at 1).
 */
typedef struct mla_tp_peers {
    int32_t world;
    int32_t rank;
    uint32_t epoch;
    int32_t reserved;
    float* acc[MLA_TP_MAX_WORLD];
    void* out[MLA_TP_MAX_WORLD];
    uint32_t* flags[MLA_TP_MAX_WORLD];
} mla_tp_peers;

/*
 * The fused o-projection + reduction of a head split on its own: for each rank
 * r in [tp->rank, tp->rank + n_local),
 *     partial_r = o_r @ o_proj_w_r                   (fp32 accumulation)
 *     out[*]    = bf16(sum over all world ranks of partial_r)
 *   o          [n_tokens, n_local * k_rank] bf16 (device): local rank i's rows of
 *              the per-head outputs (its heads * v_head_dim columns) in columns
 *              [i * k_rank, (i + 1) * k_rank)
 *   o_proj_w   [n_local * k_rank, hidden] bf16 (device): local rank i's rows of
 *              o_proj_w in rows [i * k_rank, (i + 1) * k_rank)
 *   workspace  >= 256 bytes of device memory, 256-byte aligned; its first int32
 *              is the device status word (cleared here; read it with
 *              mla_get_device_status)
 * n_local = 1 on a GPU per rank. n_local = world runs every rank on this GPU in
 * one launch of each kernel (world must be a multiple of n_local and each call
 * serves n_local consecutive ranks), so a whole split can be checked on one GPU.
 * Limits: n_tokens >= 1, k_rank a multiple of 16, hidden a multiple of
 * 32 * world. Errors (nothing enqueued): MLA_ERR_NULL_POINTER,
 * MLA_ERR_MISALIGNED, MLA_ERR_BAD_DIMS, MLA_ERR_BAD_ARGUMENT (world, rank,
 * n_local or epoch out of range), MLA_ERR_UNSUPPORTED_DIMS; MLA_ERR_CUDA if a
 * launch fails. Asynchronous on `stream`.
 */
int mla_tp_o_proj_allreduce(const void* o, const void* o_proj_w, int n_tokens, int k_rank, int hidden,
                            const mla_tp_peers* tp, int n_local, void* workspace, void* stream);

/*
 * CUDA IPC of a device allocation, for building an mla_tp_peers table across
 * processes. mla_ipc_export() describes the allocation holding `dev_ptr` (its
 * IPC handle and the pointer's offset inside it); mla_ipc_open() maps another
 * process's export into this process (peer access enabled as needed) and returns
 * the exported pointer's address here; mla_ipc_close() unmaps it. Opening an
 * export of the same process is an error (CUDA refuses it). Host only; the
 * allocation must stay alive while any process has it open.
 */
typedef struct mla_ipc_handle {
    unsigned char bytes[64];
    uint64_t offset;
} mla_ipc_handle;
int mla_ipc_export(const void* dev_ptr, mla_ipc_handle* handle);
int mla_ipc_open(const mla_ipc_handle* handle, void** dev_ptr);
int mla_ipc_close(void* dev_ptr);

#ifdef __cplusplus
}
#endif

#endif /* MLA_TP_H */
