/*
 * zero_adam.h -- C ABI of the B200 (sm_100a) ZeRO-2/3 mixed-precision Adam
 * step, run on one GPU with R logical data-parallel ranks held as R gradient
 * buffers in that GPU's memory.
 *
 * The method (sources, cited by page title and section):
 *   "Deep dive: DeepSpeed" lesson --
 *     "Count state before choosing a stage": the 16-byte recipe (2-byte
 *        weight, 2-byte gradient, fp32 master and both Adam moments) and the
 *        per-rank state of each ZeRO stage;
 *     "Reduce first, then update the owned slice": contiguous ownership
 *        [floor(P*r/R), floor(P*(r+1)/R)), reduce the gradient across ranks
 *        first, then apply Adam once per owned element to the reduced
 *        gradient; the token-weighted mean for unequal token counts;
 *     "Communication volume isn't elapsed time": ZeRO-2 is a gradient
 *        reduce-scatter followed by an all-gather of the updated parameters.
 *   DeepSpeed documentation page "ZeRO" (zero3.rst) -- stages 1-3 and the
 *        AdamW optimizer configuration (lr, betas, eps, weight_decay) with
 *        fp16 enabled.
 *
 * One fused pass per element does, for each owned index i:
 *   g   = (sum_r c_r * grad_r[i]) / S       c_r = w_r / sum(w), S = loss scale
 *   m   = b1*m + (1-b1)*g ;  v = b2*v + (1-b2)*g^2
 *   w   = w - lr*( (m/(1-b1^t)) / (sqrt(v/(1-b2^t)) + eps) + wd*w )
 *   p16 = round-to-nearest-even(w)          (written into the replicated
 *                                             16-bit parameter buffer)
 * with t the 1-based count of applied steps.  With the overflow check on, a
 * step whose gradients hold any inf or NaN changes no weight or moment, keeps
 * t, and halves S.  The reduction is exact up to one final rounding; m, v
 * and w are updated in float32, the square root and the division of the
 * step term with the hardware's approximate forms (a few units in the last
 * place of a term of size about lr). 
 *
 * Conventions for every entry point:
 *   - Return 0 (ZERO_OK) or a negative ZERO_E* code; arguments are checked on
 *     the host before anything is launched, and a rejected call launches
 *     nothing.  No error is signalled from the device by trapping.
 *   - Device-side calls are asynchronous on the given stream (a NULL stream is
 *     the legacy default stream) unless stated otherwise.  Their kernels are
 *     launched with programmatic stream serialization: a kernel may start
 *     while the kernel before it in the stream finishes, but waits for that
 *     kernel's completion before it reads or writes any memory, so stream
 *     order is kept exactly as with a plain launch.
 *   - The step calls (zero_step_fused, zero_step_fused_list,
 *     zero_step_fused_noalloc, with their scan and restore kernels),
 *     zero_accumulate_grads and zero_gather_params[_list] only enqueue work
 *     on the stream, so stream capture can record them into a CUDA graph.
 *     Capture a call after one eager call of the same kind on the device (the
 *     first launch of each kernel on a device fills its launch-shape cache).
 *     A replay reuses the values the arguments had at capture time (pointers,
 *     sizes, hyperparameters, rank weights); the step count, loss scale and
 *     skip record live in the control block and advance on every replay.
 *   - The caller owns and allocates every buffer; the library allocates no
 *     device memory and keeps no state between calls apart from per-device
 *     launch-shape caches and the static scratch array behind
 *     zero_step_fused_noalloc.
 *   - "device pointer" means memory the current CUDA device can access: its
 *     own, or another GPU's mapped into this process (the multi-GPU fields
 *     of zero_step_args); sizes are in elements unless named *_bytes.
 */
#ifndef ZERO_ADAM_H
#define ZERO_ADAM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------ status codes */
#define ZERO_OK 0
#define ZERO_EINVAL (-1)    /* NULL pointer, unknown dtype, bad count or hyperparameter */
#define ZERO_EALIGN (-2)    /* a device pointer is not 16-byte aligned */
#define ZERO_EOVERFLOW (-3) /* a byte size does not fit in 64 bits */
#define ZERO_ERANGE (-4)    /* a count beyond a documented limit */
#define ZERO_ECUDA (-5)     /* a CUDA runtime call or launch failed (zero_last_cuda_error) */
#define ZERO_EIO (-6)       /* a checkpoint file could not be used (zero_checkpoint_error) */

/* ------------------------------------------------------------------ dtypes */
#define ZERO_F32 0  /* IEEE binary32 */
#define ZERO_BF16 1 /* bfloat16 */
#define ZERO_F16 2  /* IEEE binary16 */

/* Largest number of logical ranks one step call accepts. */
#define ZERO_MAX_RANKS 256

/* Largest parameter count P of a step or accumulation call (2^40, far beyond
 * one GPU's memory): beyond it the calls return ZERO_ERANGE, so the kernels'
 * 32-bit tile numbers cannot wrap. */
#define ZERO_MAX_ELEMENTS 1099511627776ull /* 2^40 */

/* Bytes of the scratch workspace every step call needs (see zero_step_args). */
#define ZERO_WORKSPACE_BYTES 256

/* Adam/AdamW hyperparameters ("ZeRO" documentation page, optimizer config:
 * lr, betas, eps, weight_decay).  weight_decay = 0 is plain Adam, as in the
 * scalar update of "Reduce first, then update the owned slice".
 * Valid: lr >= 0, 0 <= beta1 < 1, 0 <= beta2 < 1, eps >= 0, weight_decay >= 0,
 * all finite.  They are rounded to float32 for the per-element arithmetic;
 * the bias corrections 1 - beta^t are formed in float64 on the device. */
typedef struct zero_adam_hparams {
    double lr;
    double beta1;
    double beta2;
    double eps;
    double weight_decay;
} zero_adam_hparams;

/* Control block: the persistent scalar state of one optimizer, in DEVICE
 * memory (caller-allocated, zero_ctrl_bytes() bytes, 8-byte aligned).  Set it
 * with zero_ctrl_init / zero_ctrl_set; step calls read and update it in
 * stream order, so no host synchronisation is needed between steps.  Together
 * with master, exp_avg and exp_avg_sq it is everything a resumed run needs
 * ("Resume training and export weights separately"). */
typedef struct zero_ctrl {
    uint64_t step;            /* t: applied updates so far */
    uint64_t skipped;         /* steps skipped because of inf/NaN gradients */
    float loss_scale;         /* S: gradients are stored multiplied by S */
    uint32_t growth_tracker;  /* applied steps since S last changed (check on) */
    uint32_t parity;          /* two-set mode: index of the set holding the state */
    uint32_t last_skipped;    /* 1 if the most recent step call skipped */
    uint32_t device_error;    /* nonzero: a bounded device-side wait of some
                                 step gave up (sticky until reset with
                                 zero_ctrl_set).  That step counts as not
                                 applied: t, parity, S and the growth count
                                 stay and last_skipped is 1, so a two-set
                                 optimizer keeps its last complete set; in
                                 place, the elements the step did reach are
                                 updated and the rest are not.  Never
                                 expected in normal use. */
    uint32_t reserved;        /* zero */
} zero_ctrl;

/* Kernel paths of the step and of the accumulation (field `path`):
 *   ZERO_PATH_STAGED   one producer thread per CTA stages tiles of every
 *                      input array into shared memory with 1-D bulk copies
 *                      (cp.async.bulk, no tensor map, no multicast); an
 *                      instance is compiled for 1, 2, 4 and 8 gradient
 *                      buffers, and for 16 with 16-bit gradients; for any
 *                      other count the step streams each tile's ranks through
 *                      the stages eight at a time;
 *   ZERO_PATH_REGISTER every thread reads its gradients with plain 16-byte
 *                      global loads (ld.global) into registers; any count;
 *   ZERO_PATH_AUTO     the step: the staged kernel (the faster one at
 *                      nearly every size); the accumulation: see
 *                      zero_accumulate_grads.
 * Both give bitwise identical results.  Across GPUs the gradient buffers are
 * other GPUs' memory mapped into this process: ZERO_PATH_REGISTER then reads
 * them with ordinary peer loads instead of bulk copies. */
#define ZERO_PATH_AUTO 0
#define ZERO_PATH_REGISTER 1
#define ZERO_PATH_STAGED 2

/* Arguments of one step over a FLAT parameter vector of P elements.
 *
 * Layout: every array is indexed by the flat parameter index i in [0, P);
 * owner r's slice is [floor(P*r/R), floor(P*(r+1)/R)).  All device pointers
 * must be 16-byte aligned (ZERO_EALIGN).
 *
 * State sets: master/exp_avg/exp_avg_sq[0] hold the fp32 master weights and
 * moments.  If all three [1] pointers are NULL the step updates set 0 in
 * place.  If all three are given ("two-set mode"), the step reads set
 * ctrl.parity and writes set 1-ctrl.parity, and flips ctrl.parity only when
 * the step is applied; with the overflow check on, this lets the whole step
 * run as one pass over memory, because a skipped step leaves the old set
 * untouched.  Mixing NULL and non-NULL [1] pointers is ZERO_EINVAL. */
typedef struct zero_step_args {
    uint64_t P;                   /* parameters (elements); 0 is allowed */
    uint32_t R;                   /* logical ranks, 1..ZERO_MAX_RANKS */
    int32_t owner;                /* -1: every owner's slice (all of [0,P)) in
                                     this one call; 0..R-1: only that owner's
                                     slice, with that owner's own ctrl */
    int32_t grad_dtype;           /* ZERO_F32, ZERO_BF16 or ZERO_F16 */
    int32_t param_dtype;          /* ZERO_BF16 or ZERO_F16 */
    const void *const *grads;     /* HOST array of R device pointers (n_grads
                                     if set), rank r's gradient [P] of
                                     grad_dtype (flat call); NULL for the
                                     list call */
    const double *rank_weights;   /* HOST array of R (n_grads if set) weights
                                     w_r (token counts: finite, >= 0, sum >
                                     0), or NULL for the equal-weight mean
                                     w_r = 1; used in float64 as given */
    float *master[2];             /* device [P] fp32 master weights */
    float *exp_avg[2];            /* device [P] fp32 first moment m */
    float *exp_avg_sq[2];         /* device [P] fp32 second moment v */
    void *params16;               /* device [P] param_dtype: the replicated
                                     16-bit parameters (flat call); NULL for
                                     the list call */
    float *reduced_out;           /* optional device [P] fp32: receives the
                                     reduced, unscaled gradient g of every
                                     updated element (the ZeRO-2 retained
                                     gradient slice); NULL: not written */
    zero_adam_hparams hp;
    int32_t check_nonfinite;      /* 1: skip the step on any inf/NaN gradient;
                                     2: skip it if the workspace's inf/NaN
                                     word (ZERO_WORKSPACE_FOUND_OFFSET) is
                                     set, i.e. the decision was taken by
                                     zero_scan_nonfinite calls; the call
                                     clears the word */
    uint32_t growth_interval;     /* check on: S doubles after this many
                                     consecutive applied steps; 0: never */
    void *ctrl;                   /* device zero_ctrl */
    void *workspace;              /* device scratch of ZERO_WORKSPACE_BYTES,
                                     16-byte aligned, all zero before its
                                     first use (zero_workspace_init); every
                                     call leaves it all zero again.  Calls
                                     that may overlap on the GPU need separate
                                     workspaces. */
    /* Data-parallel across GPUs (flat call only; 0 / NULL otherwise): the
     * call updates one owner's slice [lo, hi) as above, and when every rank
     * makes the call for its own slice, with the ranks' gradient buffers as
     * grads and the other ranks' replicas as push targets, the calls
     * together are the ZeRO-2 step of "Communication volume isn't elapsed
     * time" (gradient reduce-scatter, local update, all-gather of the
     * updated parameters).  Then: */
    uint64_t state_offset;        /* master, exp_avg, exp_avg_sq and
                                     reduced_out hold elements from flat index
                                     state_offset on (element i at index
                                     i - state_offset), so a rank allocates
                                     only [state_offset, hi).  A multiple of 8,
                                     at most lo; 0 for arrays of P elements. */
    uint32_t n_push;              /* 0..ZERO_MAX_PUSH; nonzero needs
                                     owner >= 0 (ZERO_EINVAL otherwise) */
    uint32_t path;                /* which step kernel reads the gradients:
                                     ZERO_PATH_AUTO (0), ZERO_PATH_REGISTER or
                                     ZERO_PATH_STAGED (see below) */
    void *const *push_params16;   /* HOST array of n_push device pointers,
                                     each [P] of param_dtype: the other ranks'
                                     replicated 16-bit parameters (peer
                                     mappings).  Every updated 16-bit value is
                                     stored there as well as into params16:
                                     the parameter all-gather, fused into the
                                     step. */
    uint32_t n_grads;             /* 0: the R ranks' gradients; else this many
                                     gradient buffers are reduced (e.g. 1: an
                                     owner's already-reduced accumulation
                                     slice), with rank_weights of n_grads
                                     entries; R still sets the partition */
    uint32_t reserved2;           /* zero */
    uint64_t grad_offset;         /* the gradient buffers hold elements from
                                     flat index grad_offset on (element i at
                                     i - grad_offset): a multiple of 8, at
                                     most lo; then check_nonfinite may not be
                                     1 (scan with zero_scan_nonfinite and use
                                     2).  0 for buffers of P elements. */
} zero_step_args;

/* Most push targets of one call (an NVLink domain's GPUs). */
#define ZERO_MAX_PUSH 72

/* Byte offset of the inf/NaN word in a workspace: a uint32, nonzero once a
 * zero_scan_nonfinite call found an inf or NaN.  Between the scans and a
 * step with check_nonfinite = 2 the caller may combine the word across
 * processes (e.g. an all-reduce MAX of it), so that every rank takes the
 * same skip decision. */
#define ZERO_WORKSPACE_FOUND_OFFSET 8

/* Device-resident description of a TENSOR LIST: T parameter tensors whose
 * concatenation, in list order and without padding, is the flat vector the
 * master weights and moments are laid out over.  Built once by
 * zero_list_table_build (the per-step call then only passes this handle).
 * All fields are filled by the build call; do not modify them. */
typedef struct zero_tensor_list {
    void *table;              /* caller-owned device memory holding the table */
    uint64_t P;               /* sum of the tensors' element counts */
    uint32_t T;               /* tensors */
    uint32_t R;               /* ranks */
    int32_t grad_dtype;
    int32_t param_dtype;
    uint64_t table_bytes;
} zero_tensor_list;

/* ---------------------------------------------------------------- host-only */

/* Ownership bounds ("Reduce first, then update the owned slice"):
 * lo[r] = floor(P*r/R), hi[r] = floor(P*(r+1)/R) for r in [0,R), computed
 * exactly (128-bit intermediates).  Slices may be uneven, and empty when
 * R > P.  lo, hi: caller HOST arrays of R entries.  ZERO_EINVAL for R == 0 or
 * NULL arrays.  Pure host function; needs no GPU. */
int zero_partition_bounds(uint64_t P, uint32_t R, uint64_t *lo, uint64_t *hi);

/* Per-rank persistent state bytes ("Count state before choosing a stage"):
 * with param_b, grad_b, opt_b the bytes per parameter of the 16-bit weight,
 * the gradient and the optimizer state (master + moments), and S = P/R,
 *   DP     = P*(param_b + grad_b + opt_b)
 *   ZeRO-1 = P*(param_b + grad_b) + S*opt_b
 *   ZeRO-2 = P*param_b + S*(grad_b + opt_b)
 *   ZeRO-3 = S*(param_b + grad_b + opt_b).
 * The values can be fractional, so out_times_R[k] receives R times the bytes
 * of stage k (k = 0: DP, 1..3: ZeRO-1..3), exactly.  ZERO_EINVAL if any count
 * or width is 0 or out is NULL, ZERO_EOVERFLOW if a product exceeds 64 bits.
 * Pure host function. */
int zero_state_bytes(uint64_t P, uint32_t R, uint32_t param_b, uint32_t grad_b,
                     uint32_t opt_b, uint64_t out_times_R[4]);

/* Human-readable text of a status code (static storage). */
const char *zero_status_string(int status);

/* Text of the last CUDA error this thread saw inside the library
 * ("no error" if none); static storage, valid until the next call. */
const char *zero_last_cuda_error(void);

/* Sizes of the caller-allocated device blocks. */
size_t zero_ctrl_bytes(void);      /* sizeof(zero_ctrl) */
size_t zero_workspace_bytes(void); /* ZERO_WORKSPACE_BYTES */

/* Bytes of device memory a tensor-list table for T tensors and R ranks needs
 * (the tensors' description plus 16 bytes of scratch counters that
 * zero3_gather uses and leaves zero). */
size_t zero_list_table_bytes(uint32_t T, uint32_t R);

/* ---------------------------------------------------------- control block */

/* ctrl = {step 0, skipped 0, loss_scale, growth 0, parity 0, last_skipped 0}.
 * loss_scale must be finite and > 0 (1 when no loss scaling is used). */
int zero_ctrl_init(void *ctrl, float loss_scale, void *stream);

/* ctrl = *value (e.g. restoring a checkpoint); value is a HOST struct passed
 * by value to the device, so it may be freed as soon as the call returns. */
int zero_ctrl_set(void *ctrl, const zero_ctrl *value, void *stream);

/* Copy the device ctrl into *out (HOST) and wait for it: synchronises the
 * stream. */
int zero_ctrl_read(const void *ctrl, zero_ctrl *out, void *stream);

/* Lets kernels on the current device read and write memory of GPU
 * `peer_device` (cudaDeviceEnablePeerAccess from the current device).  A
 * step whose grads or push_params16 are another GPU's buffers mapped into
 * this process needs it for every such GPU before its first launch: a
 * buffer mapped by CUDA IPC with its owner's device current (as PyTorch
 * maps a shared CUDA tensor) is not otherwise reachable from this device.
 * ZERO_OK also when peer_device is the current device or access is already
 * enabled.  Host call, synchronous.  Errors: ZERO_EINVAL (peer_device < 0, or
 * the two GPUs cannot access each other), ZERO_ERANGE (no such device),
 * ZERO_ECUDA. */
int zero_enable_peer_access(int32_t peer_device);

/* Zero a workspace of ZERO_WORKSPACE_BYTES (cudaMemsetAsync). */
int zero_workspace_init(void *workspace, void *stream);

/* Overflow scan of one gradient buffer: the inf/NaN check of the step with
 * loss scaling (given at the top of this file; the pages describe no loss
 * scaling), taken ahead of a step with check_nonfinite = 2: sets the
 * workspace's inf/NaN word if any of grad[0, n) is inf or NaN, and otherwise
 * leaves it as it is, so several scans accumulate.  grad: device, 16-byte aligned, of
 * grad_dtype.  Asynchronous on `stream`.  Errors: ZERO_EINVAL, ZERO_EALIGN,
 * ZERO_EOVERFLOW, ZERO_ECUDA. */
int zero_scan_nonfinite(const void *grad, int32_t grad_dtype, uint64_t n, void *workspace, void *stream);

/* Health check of the device-side timeout path (the pages have no
 * counterpart): launches one block whose thread waits, through the same
 * bounded wait as the staged kernels, on a shared-memory barrier that nothing
 * arrives at.  The wait gives up after its limit (about 2 s of GPU time) and
 * the kernel records the outcome through the step epilogue's control-block
 * update, as a two-set step with the overflow check on and growth_interval 1
 * whose wait gave up: device_error = 1 and last_skipped = 1, with step,
 * skipped, parity, loss_scale and growth_tracker unchanged.  It then exits
 * normally: no trap, no fault, the context stays usable.  Asynchronous on
 * `stream`; read the result with zero_ctrl_read.  Errors: ZERO_EINVAL (NULL ctrl), ZERO_EALIGN
 * (ctrl not 8-byte aligned), ZERO_ECUDA. */
int zero_selftest_wait_timeout(void *ctrl, void *stream);

/* ------------------------------------------------------------- the step */

/* One fused ZeRO-2/3 optimizer step over a flat parameter vector:
 * in-HBM reduce-scatter of the R rank gradients into the owner slices, the
 * optional loss-scale undo and inf/NaN skip, Adam/AdamW with bias correction
 * on the fp32 masters and moments, and the round-to-nearest-even cast of the
 * updated masters written into the replicated 16-bit parameters (the
 * updated-parameter all-gather).  The reduction runs over ranks 0..R-1 in
 * that order as float64 fused multiply-adds of w_r times the gradient (both
 * exact in float64), is scaled by 1/(sum(w)*S) and rounded once to float32;
 * results are bitwise reproducible run to run.  Sources: "Reduce first, then
 * update the owned slice" and "Communication volume isn't elapsed time"
 * ("Deep dive: DeepSpeed"); the AdamW/fp16 configuration of the "ZeRO"
 * documentation page.
 *
 * Launches: one kernel, except (a) check on, in place, or check on with
 * owner >= 0: a scan kernel over all R gradients first (the skip decision
 * covers every rank's whole gradient, as a flag combined across ranks would);
 * (b) check on in two-set mode with owner == -1: one pass plus a restore
 * kernel that, only if the step was skipped, re-casts the 16-bit parameters
 * from the untouched master set.
 * The step kernel is the one args->path selects; an unknown path is
 * ZERO_EINVAL.
 * Errors: ZERO_EINVAL, ZERO_EALIGN, ZERO_ERANGE (R > ZERO_MAX_RANKS, or
 * P > ZERO_MAX_ELEMENTS), ZERO_EOVERFLOW (P*8 bytes overflow), ZERO_ECUDA. */
int zero_step_fused(const zero_step_args *args, void *stream);

/* The same step over a tensor list: args->grads and args->params16 must be
 * NULL (the list supplies them), args->P / R / grad_dtype / param_dtype must
 * equal the list's.  master/exp_avg/exp_avg_sq are flat [P] over the list's
 * concatenation.  Tensors whose flat start is not a multiple of 8, or whose
 * buffers are not 16-byte aligned, take a scalar path (correct, slower). */
int zero_step_fused_list(const zero_step_args *args, const zero_tensor_list *list,
                         void *stream);

/* Build a tensor-list table in caller-owned device memory `table`
 * (>= zero_list_table_bytes(T, R) bytes, 16-byte aligned) and fill *out.
 *   numel:    HOST array of T element counts (0 allowed)
 *   params16: HOST array of T device pointers (param_dtype; NULL if numel 0)
 *   grads:    HOST array of R*T device pointers, RANK-MAJOR: grads[r*T + j]
 *             is rank r's gradient of tensor j (grad_dtype; NULL if numel 0)
 * SYNCHRONOUS: copies the table to the device and waits for the stream.
 * Rebuild it whenever a buffer moves. */
int zero_list_table_build(uint32_t T, uint32_t R, const uint64_t *numel,
                          void *const *params16, const void *const *grads,
                          int32_t grad_dtype, int32_t param_dtype, void *table,
                          size_t table_bytes, zero_tensor_list *out, void *stream);

/* Bytes of the library-owned scratch array behind zero_step_fused_noalloc. */
#define ZERO_NOALLOC_SCRATCH_BYTES 256

/* The same flat step as zero_step_fused, for callers that cannot allocate
 * device memory: a plugin running inside another framework whose memory pool
 * already holds the device's memory and that hands it only the parameter,
 * gradient and optimizer-state buffers; a runtime that forbids allocation
 * after start-up; or a latency-critical loop that must not take the device
 * synchronisation cudaMalloc and cudaFree can imply.  The pages describe no
 * counterpart of this entry point: it exists only for such callers.
 *
 * args->workspace must be NULL.  Instead of a caller workspace the step uses
 * one library-owned array of ZERO_NOALLOC_SCRATCH_BYTES in device memory,
 * which every GPU that loads the library keeps until the process exits.  The
 * call allocates nothing: no cudaMalloc, no cudaFree, no allocating library
 * routine.  The first call on a device looks up that device's copy of the
 * array (cudaGetSymbolAddress, with the device current); make that first
 * call before any stream capture.  Each call clears the array on `stream`
 * before the step, and the array keeps the last call's contents afterwards.
 * All calls share the one array: calls that may overlap on the GPU (other
 * streams, other host threads) race on it and must be ordered by the caller.
 * The step needs ZERO_WORKSPACE_BYTES of scratch whatever P and R are; a
 * build whose step needed more than the array holds would be refused with
 * ZERO_ERANGE.  check_nonfinite may be 0 or 1 (1 runs the overflow scan into
 * the library's array itself); 2 is ZERO_EINVAL, because no
 * zero_scan_nonfinite call can write the inf/NaN word of an array the caller
 * has no address for.  All other arguments, limits and errors are those of
 * zero_step_fused. */
int zero_step_fused_noalloc(const zero_step_args *args, void *stream);

/* ------------------------------------------------- micro-step accumulation */

/* One micro-batch's contribution to the fp32 gradient accumulation array
 * ("Deep dive: DeepSpeed": "Let the engine own the microstep" -- one update
 * per gradient-accumulation window; "Communication volume isn't elapsed
 * time" -- ZeRO-2/3 reduce and partition the gradient on every backward call
 * and keep only the owned slice between calls; "Count state before choosing
 * a stage" -- a 4-byte accumulation array, the 18-byte recipe).
 * For every element i of the slice:
 *   accum[i] = (first ? 0 : accum[i]) + scale * (sum_r w_r grad_r[i]) / sum(w)
 * computed in float64 and rounded once to float32.  The loss scale is not
 * undone here: after the last micro-batch, call zero_step_fused with R = 1,
 * grad_dtype ZERO_F32 and grads = {accum}; the step unscales, checks for
 * inf/NaN (which the sums carry) and skips exactly as for raw gradients.
 * scale is typically 1/(micro-batches per update) when each micro-batch loss
 * is a mean that was not divided by that count. */
typedef struct zero_accum_args {
    uint64_t P;                  /* elements of the flat vector; 0 is allowed */
    uint32_t R;                  /* ranks, 1..ZERO_MAX_RANKS */
    int32_t owner;               /* -1: all of [0,P); 0..R-1: that owner's slice */
    int32_t grad_dtype;          /* ZERO_F32, ZERO_BF16 or ZERO_F16 */
    int32_t first;               /* 1: start the window (accum ignored on input) */
    const void *const *grads;    /* HOST array of R device pointers [P] */
    const double *rank_weights;  /* HOST array of R weights, or NULL (equal) */
    float *accum;                /* device [P] fp32 accumulation array */
    double scale;                /* finite */
    void *workspace;             /* NULL, or a device workspace as in
                                    zero_step_args (all zero on entry, left
                                    all zero; not shared with a launch that
                                    may overlap this one on the GPU) */
    void *ctrl;                  /* NULL iff workspace is NULL; else a device
                                    zero_ctrl whose device_error receives a
                                    device-side wait timeout (nothing else of
                                    it is read or written) */
    int32_t path;                /* ZERO_PATH_AUTO (0), ZERO_PATH_REGISTER or
                                    ZERO_PATH_STAGED (see below) */
    uint64_t accum_offset;       /* accum holds elements from flat index
                                    accum_offset on (element i at
                                    i - accum_offset), so an owner can keep
                                    only its slice: a multiple of 8, at most
                                    the slice's first element; 0 for [P] */
} zero_accum_args;

/* Launches one kernel; asynchronous on `stream`.  The staged kernel
 * (ZERO_PATH_STAGED above: the instance compiled for R, else the ranks
 * streamed eight at a time) hands its tiles out dynamically; here it needs a
 * workspace and ctrl.  The register kernel streams through registers and
 * touches neither workspace nor ctrl.  Both give bitwise identical sums.
 * ZERO_PATH_AUTO takes the staged kernel when a workspace is given and the
 * staged kernel is the faster one: an instance compiled for R, or the
 * chunked kernel from R = 6 on (16-bit gradients) or R = 9 on (fp32), which
 * pays a fixed cost per tile; else the register kernel.  Errors:
 * ZERO_EINVAL (also: exactly one of workspace and ctrl given; an unknown
 * path; ZERO_PATH_STAGED without a workspace),
 * ZERO_EALIGN (accum, grads and workspace must be 16-byte aligned, ctrl
 * 8-byte aligned), ZERO_ERANGE (R > ZERO_MAX_RANKS, P > ZERO_MAX_ELEMENTS),
 * ZERO_EOVERFLOW, ZERO_ECUDA. */
int zero_accumulate_grads(const zero_accum_args *args, void *stream);

/* ------------------------------------------------------------------ ZeRO-3 */

/* ZeRO-3 partitions the 16-bit parameters too ("ZeRO" documentation page,
 * stage 3; "Deep dive: DeepSpeed", "Stage 3 needs a live working set"): each
 * rank keeps of every tensor of n elements a shard of s = ceil(n/R) elements
 * -- rank r holding elements [r*s, min((r+1)*s, n)), the last shards padded --
 * and a module's full view is gathered into a separate padded buffer of R*s
 * elements before use (and may be released after).
 *
 * The optimizer step of one rank is zero_step_fused_list over that rank's
 * shard tensors: a list whose tensor j has hi-lo elements, whose 16-bit
 * parameters are the rank's shard buffer, and whose gradient pointer of rank
 * r' is r''s full gradient of tensor j advanced by lo elements (the in-HBM
 * reduce-scatter); master and moments are the rank's own flat shard state. */

/* Shard of rank r of a tensor of n elements: *shard = ceil(n/R), and the
 * rank holds elements [*lo, *hi) of the tensor (possibly empty).  Host only.
 * ZERO_EINVAL if R == 0, r >= R or a pointer is NULL. */
int zero3_shard_bounds(uint64_t n, uint32_t R, uint32_t r, uint64_t *lo, uint64_t *hi, uint64_t *shard);

/* Parameter storage of one rank in elements (the same section's model):
 * out[0] = resident shards (sum of ceil(n_j/R)), out[1] = gathered buffers
 * (sum over the live tensors of R*ceil(n_j/R)), out[2] = their sum.  sizes:
 * HOST array of T counts (all > 0); live: HOST array of n_live distinct
 * tensor indices.  Host only.  ZERO_EINVAL on bad arguments, ZERO_EOVERFLOW. */
int zero_parameter_storage(const uint64_t *sizes, uint32_t T, uint32_t R, const uint32_t *live,
                           uint32_t n_live, uint64_t out[3]);

/* Build a gather list (table as for zero_list_table_build, >=
 * zero_list_table_bytes(T, R) bytes): numel = the tensors' true sizes,
 * full = T device buffers of R*ceil(n_j/R) elements (the padded full views),
 * shards = R*T device pointers, rank-major (shards[r*T + j], ceil(n_j/R)
 * elements each), dtype ZERO_BF16 or ZERO_F16.  SYNCHRONOUS like the list
 * build. */
int zero3_gather_list_build(uint32_t T, uint32_t R, const uint64_t *numel, void *const *full,
                            const void *const *shards, int32_t dtype, void *table, size_t table_bytes,
                            zero_tensor_list *out, void *stream);

/* full_j[r*s_j + k] = shard_{r,j}[k] for every tensor, rank and k < s_j,
 * padding included: the module-level all-gather of ZeRO-3 on one GPU (2 bytes
 * read and 2 written per padded element).  One kernel, asynchronous; it hands
 * out work through the table's scratch counters, so calls that may overlap
 * on the GPU must not share a gather list.  ZERO_EOVERFLOW beyond 2^32 - 2^16
 * chunks of 32768 elements. */
int zero3_gather(const zero_tensor_list *gather_list, void *stream);

/* ------------------------------------------------------------ checkpoints */

/* Checkpoint files ("Deep dive: DeepSpeed", "Resume training and export
 * weights separately": resuming a run needs the weights, both Adam moments
 * and the step counter, and the next update must then agree with an
 * uninterrupted run; exporting a model needs only the consolidated weights).
 *
 * A shard file holds one owner's slice (args->owner = r, the slice
 * [floor(P*r/R), floor(P*(r+1)/R))) or, with owner = -1, the whole vector:
 * a 128-byte header (magic "ZADAMCK1", R, P, owner, slice bounds, the control
 * block with parity reset to 0), the slice of the fp32 master weights, first
 * and second moments, and a 64-bit FNV-1a checksum.  Each owner writes and
 * reads its own shard, as each data-parallel rank saves its partition.
 * These calls are SYNCHRONOUS (they stage through host memory and wait for
 * `stream`); they allocate host memory only.  Errors: ZERO_EINVAL, ZERO_EIO
 * (text from zero_checkpoint_error), ZERO_ECUDA. */

/* Write the current state set (ctrl.parity in two-set mode) of args->owner's
 * slice and its control block to `path`.  Uses P, R, owner, master,
 * exp_avg, exp_avg_sq and ctrl of args. */
int zero_checkpoint_save(const char *path, const zero_step_args *args, void *stream);

/* Restore a shard written for the same P, R and owner into state set 0 and
 * the control block (parity 0); if args->params16 is given (flat layout),
 * re-cast the 16-bit parameters of the slice from the restored masters. */
int zero_checkpoint_load(const char *path, const zero_step_args *args, void *stream);

/* Consolidate the fp32 master weights of shard files into HOST memory
 * `weights` [P] (the weights-only export): the shards must all be for this P
 * and their slices must tile [0, P) exactly; every checksum is verified. */
int zero_checkpoint_consolidate(const char *const *paths, uint32_t n_paths, float *weights, uint64_t P);

/* Text of the last checkpoint error of this thread. */
const char *zero_checkpoint_error(void);

/* --------------------------------------------------------------- gathers */

/* params16[i] = round-to-nearest-even(master[i]) for i in [0,P): the cast of
 * the fp32 masters into the replicated 16-bit buffer on its own (the
 * updated-parameter all-gather of "Communication volume isn't elapsed time",
 * on one GPU).  Also used to initialise params16 from fresh masters.
 * master, params16: device, 16-byte aligned. */
int zero_gather_params(const float *master, void *params16, int32_t param_dtype,
                       uint64_t P, void *stream);

/* The same over a tensor list's parameter tensors. */
int zero_gather_params_list(const float *master, const zero_tensor_list *list,
                            void *stream);

#ifdef __cplusplus
}
#endif

#endif /* ZERO_ADAM_H */
