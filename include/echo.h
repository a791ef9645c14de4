/*
 * echo.h -- C ABI of the B200 implementation of Echo, the error-compensated
 * 4-bit tensor-parallel all-reduce ("Echo: Error-Compensated 4-Bit
 * Tensor-Parallel Communication for LLM Training and Inference",
 * arXiv 2610.14277).
 *
 * What one call computes (sources, by page and section):
 *  - ai4snews news summary, "Interpretation", paragraph 1: the values cross
 *    between ranks as 4-bit integers and are added at high precision.
 *  - arXiv abstract (fugumt mirror), "Abstract": no value is rounded more
 *    than twice in a call whatever the number of ranks; the rounding error
 *    that the sum exposes is carried into the calls that follow.
 *  - ai4snews news summary, "Interpretation", paragraph 2: the compensator
 *    is a fast and a slow exponential moving average; a weighted mix of the
 *    two is added to each input before quantization, and both are updated
 *    from the residual of the output.
 *
 * Per call, for P ranks of N elements each, group size G:
 *   1. c_r  = alpha*m_fast_r + (1-alpha)*m_slow_r;  xt_r = float(x_r) + c_r
 *   2. per group of G: a = max|xt|, scale = a/L,
 *      k = clamp(rint_half_even(xt/scale), -L, L) with L = 7 for 4-bit
 *      codes (packed two per byte, element 2j in the low nibble) or
 *      L = 127 for 8-bit codes (one byte each); scales fp32
 *   3. e_in_r = xt_r - k*scale;  m <- beta*m + (1-beta)*e_in_r (both EMAs)
 *   4. reduce-scatter: the owner o of chunk [o*N/P, (o+1)*N/P) sums
 *      s = sum over r = 0..P-1 (ascending) of k_r*scale_r in fp32
 *   5. requantize s with step 2 -> (k2, scale2); y = bf16_rne(k2*scale2);
 *      e_req = s - float(y)
 *   6. all-gather: every rank receives y
 *   7. the owner's states only: m <- m + (1-beta)*e_req (both EMAs)
 * With the compensator off, c = 0 and no state is read or written.
 * The constants alpha, beta_fast, beta_slow are parameters: the pages do not
 * fix them (defaults 0.5, 0.5, 0.95).
 *
 * All P ranks live on one GPU; the "wire" between the stages is the packed
 * codes and scales in HBM.  Every quantity at element i depends only
 * on the G-element group column of i across the P ranks.
 *
 * Conventions for every entry point:
 *  - Pointers named *device* are CUDA device pointers on the plan's device;
 *    pointers named *host* are host pointers (pinned for asynchronous
 *    copies).  Streams are cudaStream_t handles passed as void*; NULL is the
 *    legacy default stream.
 *  - Calls are stream-ordered and asynchronous: nothing synchronizes the
 *    host except echo_plan_create, echo_plan_destroy and echo_profile_read.
 *  - All argument checks happen on the host before any launch and return a
 *    status; a CUDA error returns ECHO_ERR_CUDA.  Nothing aborts.
 *  - A plan is not thread-safe; calls on one plan must not overlap.
 */
#ifndef ECHO_H
#define ECHO_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ECHO_ABI_VERSION 5
#define ECHO_MAX_RANKS 8

typedef enum echo_status {
    ECHO_OK = 0,
    ECHO_ERR_INVALID_ARG = 1, /* null pointer, value out of range */
    ECHO_ERR_SHAPE = 2,       /* N <= 0 or N % (P*G) != 0 */
    ECHO_ERR_ALIGNMENT = 3,   /* a buffer not 16-byte aligned */
    ECHO_ERR_UNSUPPORTED = 4, /* P, G or bits outside the supported set */
    ECHO_ERR_OOM = 5,         /* device allocation failed */
    ECHO_ERR_CUDA = 6,        /* a CUDA runtime call failed */
    ECHO_ERR_TIMEOUT = 7      /* a kernel's bounded wait ran out (echo_device_error_get) */
} echo_status;

/* Where the owner's requantization error enters its EMA states (step 7).
 * All three give bit-identical states, outputs and codes. */
typedef enum echo_fixup_mode {
    /* inside the kernel that sums and requantizes (the reduce), before the
     * call returns; e_req is then consumed there and not stored */
    ECHO_FIXUP_EXIT = 0,
    /* in its own kernel on the side stream given to echo_allreduce, so it
     * can run beside the caller's next matrix multiplication (the pages'
     * arrangement: the update overlaps the next matrix multiplication); the next call on the plan
     * waits for it */
    ECHO_FIXUP_SIDE = 1,
    /* kept pending in e_req and folded into the next call's entry pass,
     * which reads the state anyway (fewest HBM bytes).  e_req holds -0.0f
     * whenever no fix-up is pending (after plan creation, echo_reset_state
     * and echo_set_state), and m + (1-beta)*(-0) = m exactly, so every
     * entry applies e_req: no host-side flag selects the kernels a call
     * launches, and a captured graph replays correctly (see "Stream
     * capture" below) */
    ECHO_FIXUP_DEFERRED = 2
} echo_fixup_mode;

typedef struct echo_config {
    int32_t P;          /* ranks, 1..ECHO_MAX_RANKS */
    int32_t G;          /* group size: 32, 64 or 128 */
    int64_t N;          /* elements per rank, N > 0, N % (P*G) == 0 */
    int32_t compensate; /* 1: dual-EMA compensator on, 0: off */
    float alpha;        /* weight of the fast EMA in the correction, [0,1] */
    float beta_fast;    /* decay of the fast EMA, [0,1] */
    float beta_slow;    /* decay of the slow EMA, [0,1] */
    int32_t device;     /* CUDA device ordinal the plan lives on */
    int32_t fixup;      /* echo_fixup_mode */
    int32_t bits;       /* code width: 4 (levels -7..7, two codes per byte) or
                         * 8 (levels -127..127, one code per byte; the
                         * pages' serving policy gives 8-bit codes to the
                         * earlier layers, half of them, ai4snews
                         * "Perspective").
                         * The widest width of the plan's calls: the
                         * transport is sized for it, and a plan with
                         * bits = 8 can run any call at 4 bits
                         * (echo_plan_set_bits) on the same state. */
} echo_config;

typedef struct echo_plan echo_plan;

/* Fill *cfg with the defaults: compensate = 1, alpha = 0.5,
 * beta_fast = 0.5, beta_slow = 0.95, device = 0, fixup = ECHO_FIXUP_EXIT,
 * bits = 4; P, G, N are set to 0 and must be filled in. */
void echo_config_default(echo_config *cfg);

/* Bytes of device memory a plan for *cfg allocates: the EMA states
 * (2*P*N fp32 when compensating), the entry transport (P*N*bits/8 code
 * bytes + P*N/G fp32 scales), the reduced transport (N*bits/8 + 4*N/G
 * bytes), e_req (N fp32 when compensating), each sub-buffer 256-byte
 * aligned, and a 4 KiB guard zone after them (filled with 0xA5 at plan
 * creation and written by no kernel; see echo_debug_view).
 * Returns 0 for an invalid config. */
size_t echo_workspace_bytes(const echo_config *cfg);

/* Validate *cfg, allocate the plan's device workspace on cfg->device and
 * zero the compensator state (m_0 = 0).  Synchronizes the device.
 * The plan owns its workspace; release it with echo_plan_destroy.
 * Errors: INVALID_ARG (null, constants outside [0,1], bad fixup mode),
 * UNSUPPORTED (P, G), SHAPE (N), OOM, CUDA.  *out is NULL on error. */
echo_status echo_plan_create(echo_plan **out, const echo_config *cfg);

/* Free everything the plan allocated (after synchronizing its device).
 * NULL is accepted and ignored. */
echo_status echo_plan_destroy(echo_plan *plan);

/* One compensated 4-bit all-reduce over the P ranks (steps 1-7 above).
 *   in_device[r]  : bf16, N contiguous elements of rank r (read)
 *   out_device[r] : bf16, N contiguous elements (written with y); may equal
 *                   in_device[r] (in-place)
 *   stream        : stream the entry and reduce kernels run on (on one
 *                   GPU the reduce writes the outputs: there is no exit
 *                   pass; the rank path's exit kernel is the all-gather)
 *   side_stream   : used with ECHO_FIXUP_SIDE only (the owner fix-up runs
 *                   there after an event on stream); NULL runs the fix-up
 *                   on stream.  Ignored by the other modes.
 * Both pointer arrays are host arrays of P device pointers, each 16-byte
 * aligned.  Buffers are owned by the caller and must stay valid until the
 * call completes on the stream.  Output buffers must not overlap each other
 * or another rank's input.
 * Errors: INVALID_ARG (null plan/arrays/pointers), ALIGNMENT, CUDA. */
echo_status echo_allreduce(echo_plan *plan, const void *const *in_device,
                           void *const *out_device, void *stream,
                           void *side_stream);

/* Stream capture.  echo_allreduce and echo_reduce_scatter only launch
 * kernels (and, with a side stream, record and wait on events); they
 * allocate nothing and never synchronize, so they may be captured into a
 * CUDA graph on stream.  A replay runs the captured kernels on the plan's
 * current state and buffers, exactly as the same eager calls would, in the
 * EXIT and DEFERRED modes, whatever calls, replays or state resets came
 * before it, and in ECHO_FIXUP_SIDE mode without a side stream.  A capture
 * fixes the buffers and the code width (echo_plan_set_bits).  Refused with
 * UNSUPPORTED while stream is capturing: a call with profiling on (its
 * events are kept per call on the host), a side-stream fix-up (it leaves in
 * the graph an event that the plan's next call would wait on), and
 * echo_allreduce_host (host copies on internal streams).  echo_reset_state,
 * echo_get_state and echo_set_state capture too (copies and kernels). */

/* One reduce-scatter over the P ranks: the reduce-scatter of sequence
 * parallelism, which the pages name as a next target for the same scheme
 * (ai4snews news summary, "Perspective").  Steps 1-4 as for
 * echo_allreduce, then the owner o of chunk [o*N/P, (o+1)*N/P) receives
 * bf16(s) of that chunk: each value is quantized once, at entry.  The
 * owner's output residual s - float(bf16(s)) is folded into its own EMAs
 * like e_req (in the second kernel, on side_stream, or deferred into the
 * next call's entry pass, by the plan's fix-up mode).
 *   in_device[r]  : bf16, N elements of rank r (read)
 *   out_device[r] : bf16, N/P elements: rank r's own chunk of the sum
 *                   (written); must not overlap each other
 * A plan's state is shared between its all-reduce and reduce-scatter
 * calls.  Two kernels per call (three in side-stream mode).
 * Errors: INVALID_ARG, ALIGNMENT, CUDA. */
echo_status echo_reduce_scatter(echo_plan *plan, const void *const *in_device,
                                void *const *out_device, void *stream,
                                void *side_stream);

/* The same call on host buffers, pipelined: the call is cut into up to 32
 * slabs (the same sub-range of every owner chunk); each slab's inputs are
 * copied host -> device, its kernels run, and its outputs are copied
 * device -> host, on three internal streams, so copies in both directions
 * overlap each other and the kernels.  The staging area (2*P*N*2 bytes) and
 * the internal streams and events are created on first use and kept until
 * echo_plan_destroy.  The work starts after everything already queued on
 * stream, and stream waits for its end: synchronize stream before reading
 * out_host.  in_host[r], out_host[r]: N bf16 elements each; out_host[r] may
 * equal in_host[r] (a slab's outputs are copied back only after its inputs
 * were copied in, and later slabs read other parts); pinned host memory
 * makes the copies asynchronous, pageable memory makes them synchronous.  Results, codes and states equal echo_allreduce's; with
 * ECHO_FIXUP_SIDE the fix-up runs in the reduce kernel here.
 * Errors: INVALID_ARG, OOM (staging), CUDA. */
echo_status echo_allreduce_host(echo_plan *plan, const void *const *in_host,
                                void *const *out_host, void *stream);

/* Zero the compensator state (m_fast = m_slow = 0) and drop any pending
 * deferred fix-up (e_req = -0), on stream.  A no-op (ECHO_OK) when
 * compensate == 0. */
echo_status echo_reset_state(echo_plan *plan, void *stream);

/* Copy the current states, with any pending deferred fix-up applied, into
 * caller device buffers m_fast_device, m_slow_device ([P][N] fp32, rank
 * major), on stream.  The plan's state is not changed.
 * Errors: INVALID_ARG (null, or compensate == 0), CUDA. */
echo_status echo_get_state(echo_plan *plan, float *m_fast_device,
                           float *m_slow_device, void *stream);

/* Overwrite the states from caller device buffers ([P][N] fp32) and drop
 * any pending fix-up (e_req = -0), on stream (checkpoint restore, tests).
 * Errors: INVALID_ARG (null, or compensate == 0), CUDA. */
echo_status echo_set_state(echo_plan *plan, const float *m_fast_device,
                           const float *m_slow_device, void *stream);

/* Device pointers into the plan's workspace, for inspection by tests.  The
 * contents are those left by the last call; with ECHO_FIXUP_DEFERRED the
 * states lack the pending fix-up (echo_get_state applies it). */
typedef struct echo_debug_view {
    float *m_fast;      /* [P][N] fp32, or NULL when not compensating */
    float *m_slow;      /* [P][N] fp32, or NULL */
    uint8_t *codes;     /* [P][N*bits/8] entry codes */
    float *scales;      /* [P][N/G] entry scales */
    uint8_t *rcodes;    /* [N*bits/8] requantized sum codes */
    float *rscales;     /* [N/G] requantization scales */
    float *e_req;       /* [N] requantization error, or NULL */
    int32_t fixup_pending; /* 1 if a deferred-mode call ran since the last
                              reset or restore (host view: graph replays
                              do not change it) */
    int32_t bits;       /* code width of the calls (echo_plan_set_bits) */
    uint8_t *guard;     /* the guard zone after the workspace: guard_bytes */
    int64_t guard_bytes;/* bytes, each 0xA5 unless something overran */
} echo_debug_view;

echo_status echo_debug_view_get(echo_plan *plan, echo_debug_view *view);

/* Per-kernel timing with CUDA events recorded on the stream each kernel is
 * launched on.  While enabled, every call records events around its
 * kernels; echo_profile_read synchronizes on them, adds the elapsed times
 * to the totals below and returns them; reset clears the totals. */
typedef struct echo_profile {
    int64_t calls;          /* calls recorded */
    double entry_ms;        /* total time of echo_entry launches */
    double reduce_ms;       /* total time of echo_reduce launches */
    double exit_ms;         /* total time of echo_exit launches: 0, since
                             * a plan's reduce writes the outputs (kept for
                             * the layout of this struct) */
    double fixup_ms;        /* total time of side-stream fix-up launches */
    int64_t launches;       /* kernels launched by the recorded calls */
} echo_profile;

echo_status echo_profile_enable(echo_plan *plan, int32_t on);
echo_status echo_profile_read(echo_plan *plan, echo_profile *out, int32_t reset);

/* Code width of the plan's following calls: 4, or 8 when cfg.bits == 8
 * (per-call promotion: the pages' serving policy runs the earlier half of the
 * layers at 8 bits, ai4snews news summary, "Perspective").  Every width
 * shares the plan's one compensator state and any pending fix-up: the
 * state and e_req are fp32 whatever the width.  Takes effect for calls made
 * after it; launches nothing.  A new plan runs at cfg.bits.
 * Errors: INVALID_ARG (null), UNSUPPORTED (not 4 or 8, or above cfg.bits). */
echo_status echo_plan_set_bits(echo_plan *plan, int32_t bits);

/* Kernels launched by one echo_allreduce call with this plan. */
int32_t echo_launches_per_call(const echo_plan *plan);

/* ------------------------------------------------------------------------
 * Allocation-free call.  The paper has no counterpart: this entry point
 * exists for callers that cannot allocate device memory on their call path,
 * for example a serving process whose memory manager reserves the whole GPU
 * up front and accounts for every byte (a library cudaMalloc would fail or
 * break that accounting), code that cannot afford the device-wide
 * synchronization that cudaMalloc and cudaFree imply, or a plugin host that
 * hands a library only its buffers and a stream.
 *
 * It computes exactly what echo_allreduce computes for a plan made from
 * *cfg with ECHO_FIXUP_EXIT (cfg->fixup is ignored), but without a plan:
 *   in_device[r], out_device[r] : as for echo_allreduce (P bf16 buffers of
 *                                 N elements, 16-byte aligned)
 *   m_fast_device, m_slow_device: the compensator state, owned by the
 *                                 caller: [P][N] fp32, rank major, zero
 *                                 before the first call, updated in place
 *                                 (ignored, may be NULL, when
 *                                 cfg->compensate == 0)
 *   stream                      : where the kernels run
 * The scratch the kernels hand each other (entry codes and scales, the
 * requantized codes and scales and, compensating, e_req) lives in one
 * file-scope device array of ECHO_NOALLOC_MAX_SCRATCH_BYTES, which every
 * GPU that loads this code holds until the process exits.  A call needs
 *   P*N/2 + 4*P*N/G + N/2 + 4*N/G (+ 4*N when compensating)
 * bytes, each part rounded up to 256; a call that needs more returns
 * ECHO_ERR_UNSUPPORTED before launching anything (80 MiB holds, e.g., 8
 * ranks of 2048 x 4096 bf16 activations with the compensator on).
 * Set-up: the first call in a CUDA context on a device looks up the
 * array's address with cudaGetSymbolAddress while that device is current
 * (this may load the library's device code into the context), and later
 * calls in the same context reuse it.  The address belongs to that context:
 * after cudaDeviceReset, or when the caller makes another context current
 * (driver-API users), the next call sees a context it has not seen and does
 * the set-up again.  Make the first call in each context before any stream
 * capture: a call whose set-up is still due returns ECHO_ERR_UNSUPPORTED,
 * launching nothing, while its stream is capturing.  All calls on a device share the one array and
 * it keeps the last call's contents: nothing in it needs to start at zero
 * (every byte a call reads was written earlier in the same call), but calls
 * that overlap on the GPU -- on streams not ordered with each other, or
 * from several host threads at once -- race on it and corrupt each other's
 * results.  Order them on one stream.
 * 4-bit codes only (cfg->bits must be 4).
 * Calls no cudaMalloc, cudaFree or host allocator.  Errors as for
 * echo_allreduce, plus UNSUPPORTED for the size limit. */
#define ECHO_NOALLOC_MAX_SCRATCH_BYTES ((size_t)80 << 20)

echo_status echo_allreduce_noalloc(const echo_config *cfg, const void *const *in_device,
                                   void *const *out_device, float *m_fast_device,
                                   float *m_slow_device, void *stream);

/* ------------------------------------------------------------------------
 * Device error word.  Two kernels here wait: the reduce and the
 * reduce-scatter kernel, when they stage their blocks' tiles in shared
 * memory with bulk copies (P = 8, N >= 2^23; the all-reduce only for
 * uncompensated calls at G = 128, the reduce-scatter at G = 64 and 128),
 * wait for those copies.  A wait
 * gives up after 1 s, sets ECHO_DEVERR_WAIT_TIMEOUT in this library's device
 * error word on its device, and the kernel writes none of its outputs; the
 * call that launched it has already returned ECHO_OK.  echo_device_error_get copies the word of
 * `device` into *flags (a synchronous copy: read it once the work to check
 * has finished), clears it when clear != 0, and returns ECHO_ERR_TIMEOUT
 * when the word has ECHO_DEVERR_WAIT_TIMEOUT set, ECHO_OK when it is clear.
 * Errors: INVALID_ARG (null flags, device < 0), CUDA. */
#define ECHO_DEVERR_WAIT_TIMEOUT 1

echo_status echo_device_error_get(int32_t device, int32_t *flags, int32_t clear);

/* Self-test of the bounded wait on `device`: one block of 32 threads waits
 * on a barrier that nothing completes; the wait gives up after its limit
 * (1 s) and sets ECHO_DEVERR_WAIT_TIMEOUT in the device error word.  Runs on
 * a stream of its own and blocks the host until the kernel has ended (about
 * one second).  Errors: INVALID_ARG (device < 0), CUDA. */
echo_status echo_selftest_wait_limit(int32_t device);

/* Static name of a status code. */
const char *echo_status_string(echo_status s);

int32_t echo_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ECHO_H */
