/*
 * echo_rank.h -- one rank of an Echo group spread over P processes (one GPU
 * each), with the two exchange steps left to the caller's collective
 * library.
 *
 * The operation is the one echo.h defines (steps 1-7), for P real ranks
 * instead of P virtual ranks on one GPU: the pages' setting is a
 * tensor-parallel group of GPUs on NVLink whose all-reduce moves 4-bit
 * integers and sums them in high precision (ai4snews news summary,
 * "Interpretation", paragraph 1; arXiv abstract, "Abstract").  Such an
 * all-reduce is a reduce-scatter followed by an all-gather; here each half
 * moves the packed codes and scales, and everything else runs in this
 * rank's kernels:
 *
 *   echo_rank_entry    steps 1-3 on this rank's input: correction, group
 *                      quantization of every chunk, partial EMA update
 *   (caller)           all-to-all: chunk o of every rank's codes and scales
 *                      to rank o
 *   echo_rank_reduce   steps 4-5 for this rank's own chunk: dequantize the P
 *                      received chunks, sum in fp32 in ascending rank order,
 *                      requantize, e_req; and, by fix-up mode, step 7
 *   (caller)           all-gather of the P owners' reduced codes and scales
 *   echo_rank_exit     step 6: dequantize every owner's chunk to bf16
 *
 * Run by every rank of the group with the same echo_config (P = the group
 * size), the sequence gives every rank the output, codes and states that
 * echo_allreduce gives the P virtual ranks of one plan, bit for bit.
 * echo_rank_reduce_scatter replaces the last three steps for the
 * reduce-scatter of sequence parallelism (echo_reduce_scatter in echo.h).
 *
 * Exchange buffers are owned by the caller (any device memory the collective
 * library can use).  With C = N/P elements per chunk, cb = C*bits/8 code
 * bytes and cs = C/G scales per chunk (echo_rank_exchange_bytes):
 *   send codes  [P][cb] bytes, send scales  [P][cs] fp32: chunk o at o*cb / o*cs
 *   recv codes  [P][cb] bytes, recv scales  [P][cs] fp32: from rank r at r*cb / r*cs
 *   red codes   [cb] bytes,    red scales   [cs] fp32:    this rank's chunk
 *   all codes   [P][cb] bytes, all scales   [P][cs] fp32: owner o's at o*cb / o*cs
 * so the exchanges are an equal-split all-to-all of the send buffers into
 * the recv buffers and an all-gather of the red buffers into the all
 * buffers (for example torch.distributed all_to_all_single and
 * all_gather_into_tensor, or ncclSend/ncclRecv in a group and
 * ncclAllGather).  Within a chunk, codes and scales keep the layout of
 * echo.h (element 2j in the low nibble of byte j for 4-bit codes, one byte
 * each for 8-bit codes; one fp32 scale per group of G, in element order).
 * Code buffers, inputs and outputs must be 16-byte aligned; scale buffers
 * 4-byte aligned.
 *
 * Conventions as in echo.h: device pointers on the plan's device,
 * stream-ordered asynchronous calls, host-side checks that return a status
 * before any launch, no aborts, not thread-safe.  Nothing here waits on
 * another rank: ordering between ranks is the collective library's.
 */
#ifndef ECHO_RANK_H
#define ECHO_RANK_H

#include "echo.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct echo_rank_plan echo_rank_plan;

/* Bytes of one chunk's codes (C*bits/8) and scales (4*C/G) for *cfg.
 * Errors: the same checks as echo_plan_create (INVALID_ARG, UNSUPPORTED,
 * SHAPE). */
echo_status echo_rank_exchange_bytes(const echo_config *cfg, size_t *chunk_code_bytes,
                                     size_t *chunk_scale_bytes);

/* Bytes of device memory a rank plan allocates: this rank's EMA states
 * (2*N fp32) and e_req of its own chunk (C fp32), when compensating, each
 * 256-byte aligned; 0 for an invalid config. */
size_t echo_rank_workspace_bytes(const echo_config *cfg);

/* Plan of rank `rank` (0 <= rank < cfg->P) of a group of cfg->P ranks:
 * validates *cfg as echo_plan_create does, allocates the workspace on
 * cfg->device and zeroes the state.  Synchronizes the device.
 * Errors: INVALID_ARG (also rank out of range), UNSUPPORTED, SHAPE, OOM,
 * CUDA.  *out is NULL on error. */
echo_status echo_rank_plan_create(echo_rank_plan **out, const echo_config *cfg, int32_t rank);

/* Free the plan (after synchronizing its device); NULL is ignored. */
echo_status echo_rank_plan_destroy(echo_rank_plan *plan);

/* Steps 1-3 on this rank's input, writing the send buffers.  With
 * ECHO_FIXUP_DEFERRED the entry first applies the owner fix-up held in the
 * plan's e_req: the previous reduce's, or -0.0f (an exact no-op) when none
 * is pending (after plan creation, reset_state and set_state).
 *   x_device       : bf16, N elements of this rank (read)
 *   send_codes     : [P][cb] bytes (written)
 *   send_scales    : [P][cs] fp32 (written)
 * One kernel.  Errors: INVALID_ARG (null), ALIGNMENT, CUDA. */
echo_status echo_rank_entry(echo_rank_plan *plan, const void *x_device, void *send_codes_device,
                            float *send_scales_device, void *stream);

/* Steps 4-5 for this rank's chunk, from the received buffers, writing the
 * reduced codes and scales that the all-gather distributes.  Step 7 by the
 * plan's fix-up mode: EXIT applies it inside the reduce kernel, SIDE keeps
 * e_req and runs it in its own kernel on side_stream (NULL: on stream; the
 * plan's next call waits for it), DEFERRED keeps e_req for the next entry.
 *   recv_codes, recv_scales : [P][cb] bytes, [P][cs] fp32 (read)
 *   red_codes, red_scales   : [cb] bytes, [cs] fp32 (written)
 * Must follow an echo_rank_entry on the plan (a second reduce without a new
 * entry would apply the fix-up twice).  One kernel, two in SIDE mode.
 * Errors: INVALID_ARG (null, or no entry since the last reduce),
 * ALIGNMENT, CUDA. */
echo_status echo_rank_reduce(echo_rank_plan *plan, const void *recv_codes_device,
                             const float *recv_scales_device, void *red_codes_device,
                             float *red_scales_device, void *stream, void *side_stream);

/* Step 6: dequantize the P owners' reduced chunks to bf16.
 *   all_codes, all_scales : [P][cb] bytes, [P][cs] fp32 (read)
 *   out_device            : bf16, N elements (written); may be this rank's
 *                           input
 * One kernel.  Reads no plan state.  Errors: INVALID_ARG, ALIGNMENT, CUDA. */
echo_status echo_rank_exit(echo_rank_plan *plan, const void *all_codes_device,
                           const float *all_scales_device, void *out_device, void *stream);

/* The reduce-scatter of sequence parallelism, after echo_rank_entry and the
 * all-to-all: out_device (C bf16 elements) receives bf16(s) of this rank's
 * chunk, quantized once at entry; the output residual s - float(bf16(s))
 * enters this rank's EMAs by the fix-up mode, as in echo_rank_reduce.
 * One kernel, two in side-stream mode.  Errors as echo_rank_reduce. */
echo_status echo_rank_reduce_scatter(echo_rank_plan *plan, const void *recv_codes_device,
                                     const float *recv_scales_device, void *out_device,
                                     void *stream, void *side_stream);

/* Zero this rank's state and drop a pending fix-up (e_req = -0), on stream
 * (a no-op when compensate == 0). */
echo_status echo_rank_reset_state(echo_rank_plan *plan, void *stream);

/* Copy this rank's states ([N] fp32 each), with a pending fix-up applied,
 * into caller device buffers; the plan's state is unchanged.
 * Errors: INVALID_ARG (null, or compensate == 0), ALIGNMENT, CUDA. */
echo_status echo_rank_get_state(echo_rank_plan *plan, float *m_fast_device,
                                float *m_slow_device, void *stream);

/* Overwrite this rank's states from caller device buffers ([N] fp32 each)
 * and drop a pending fix-up (e_req = -0).  Errors as echo_rank_get_state.
 *
 * Stream capture: every call above only launches kernels, copies on the
 * device and (with a side stream) records and waits on events, so a whole
 * rank call -- stages and the caller's exchanges -- may be captured into a
 * CUDA graph, with the same rules as echo_allreduce (include/echo.h): a
 * reduce or reduce-scatter with a side-stream fix-up returns UNSUPPORTED
 * while stream is capturing.  The host-side order check of
 * echo_rank_reduce applies when the calls are captured, not when the graph
 * is replayed. */
echo_status echo_rank_set_state(echo_rank_plan *plan, const float *m_fast_device,
                                const float *m_slow_device, void *stream);

/* Code width of the following calls, as echo_plan_set_bits (4, or 8 when
 * cfg.bits == 8; one state for every width).  The chunk sizes of the
 * exchange buffers follow the width: cb = C*bits/8 with the width in force,
 * so buffers sized for cfg.bits hold any call, at the offsets of that call's
 * width.  Errors: INVALID_ARG (null), UNSUPPORTED. */
echo_status echo_rank_plan_set_bits(echo_rank_plan *plan, int32_t bits);

/* Kernels one all-reduce (entry + reduce + exit) launches with this plan:
 * 3, or 4 in SIDE mode (the fix-up as its own kernel). */
int32_t echo_rank_launches_per_call(const echo_rank_plan *plan);

/* ---------------------------------------------------------------------------
 * Fused transport over peer memory.
 *
 * The two exchanges become accesses of the stage kernels themselves to the
 * other ranks' memory (NVLink on a B200 node), so that the bytes cross while
 * the kernel quantizes or dequantizes:
 *
 *   echo_rank_entry_peers  steps 1-3, storing chunk o of the codes and
 *                          scales straight into part `rank` of rank o's
 *                          receive buffers (the all-to-all)
 *   (caller)               barrier: every rank's entry has completed
 *   echo_rank_reduce       unchanged, from this rank's receive buffers into
 *                          its reduced buffers
 *   (caller)               barrier: every rank's reduce has completed
 *   echo_rank_exit_peers   step 6, loading owner o's reduced chunk straight
 *                          from owner o's reduced buffers (the all-gather)
 *
 * The barrier is any stream-ordered operation that completes on a rank only
 * after the preceding work of every rank has completed, for example a
 * one-element all-reduce of the collective library on the same stream.  No
 * kernel waits on another rank.  Two barriers per call also order the next
 * call: a rank's next entry_peers writes receive buffers that every owner
 * has finished reading (its reduce came before the second barrier), and an
 * owner's next reduce writes reduced buffers that every rank has finished
 * reading (each rank's exit came before its next entry, hence before the
 * next call's first barrier).  For the reduce-scatter: entry_peers, a
 * barrier, echo_rank_reduce_scatter from this rank's receive buffers, and a
 * barrier (the next entry_peers must not write receive buffers an owner is
 * still reading).
 *
 * The receive and reduced buffers peers reach are this plan's window: one
 * device allocation (so that a single CUDA IPC handle maps it into another
 * process) with the layouts above, viewed at the code width in force.  Every
 * rank of a group must use the same width for a call.  Plain loads and
 * stores only: no TMA, no multicast.
 * ------------------------------------------------------------------------- */

typedef struct echo_rank_window_layout {
    void *base;          /* the allocation, on the plan's device */
    size_t bytes;        /* its size, guard zone included */
    size_t recv_codes;   /* byte offsets of the four buffers from base, */
    size_t recv_scales;  /* each 256-byte aligned: recv codes [P][cb_max], */
    size_t red_codes;    /* recv scales [P][cs] fp32, red codes [cb_max], */
    size_t red_scales;   /* red scales [cs] fp32; cb_max = C*cfg.bits/8 */
    size_t guard;        /* offset of a guard zone after them: guard_bytes */
    size_t guard_bytes;  /* bytes of 0xA5 that no kernel writes */
} echo_rank_window_layout;

/* The plan's window, allocated (and zeroed) on the first call; the plan
 * owns it and frees it in echo_rank_plan_destroy.
 * Errors: INVALID_ARG, OOM, CUDA. */
echo_status echo_rank_window(echo_rank_plan *plan, echo_rank_window_layout *out);

/* Steps 1-3 as echo_rank_entry, with chunk o's codes and scales stored to
 * recv_codes_peers[o] + rank*cb and recv_scales_peers[o] + rank*cs:
 *   recv_codes_peers[o]  : rank o's receive codes buffer ([P][cb] bytes),
 *                          as mapped in this process (16-byte aligned);
 *                          entry o == rank may be this plan's own
 *   recv_scales_peers[o] : rank o's receive scales ([P][cs] fp32, 4-byte
 *                          aligned)
 * Both are host arrays of P pointers.  One kernel.
 * Errors: INVALID_ARG (null), ALIGNMENT, CUDA. */
echo_status echo_rank_entry_peers(echo_rank_plan *plan, const void *x_device,
                                  void *const *recv_codes_peers, float *const *recv_scales_peers,
                                  void *stream);

/* Step 6 as echo_rank_exit, with owner o's reduced chunk loaded from
 * red_codes_peers[o] ([cb] bytes, 16-byte aligned) and red_scales_peers[o]
 * ([cs] fp32): owner o's reduced buffers as mapped in this process.
 * One kernel.  Reads no plan state.  Errors: INVALID_ARG, ALIGNMENT, CUDA. */
echo_status echo_rank_exit_peers(echo_rank_plan *plan, const void *const *red_codes_peers,
                                 const float *const *red_scales_peers, void *out_device,
                                 void *stream);

/* CUDA IPC of a window between the processes of a group (a thin layer over
 * cudaIpcGetMemHandle / cudaIpcOpenMemHandle / cudaIpcCloseMemHandle).
 * echo_ipc_handle_get: the handle of the allocation that holds device_ptr
 * (pass a window base).  echo_ipc_open: map another process's allocation
 * into this one on `device` (peer access enabled as needed); *out is its
 * base.  A process cannot open its own handles.  echo_ipc_close: unmap.
 * Errors: INVALID_ARG, CUDA. */
typedef struct echo_ipc_handle {
    uint8_t bytes[64];
} echo_ipc_handle;

echo_status echo_ipc_handle_get(const void *device_ptr, echo_ipc_handle *out);
echo_status echo_ipc_open(const echo_ipc_handle *handle, int32_t device, void **out);
echo_status echo_ipc_close(void *ptr, int32_t device);

#ifdef __cplusplus
}
#endif

#endif /* ECHO_RANK_H */
