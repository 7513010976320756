/*
 * adamw4.h -- C ABI of the fused 4-bit AdamW optimizer step (ZIP-SR / ZE-EDEN)
 * for NVIDIA B200 (sm_100a).
 *
 * The method: AdamW keeps a first moment m and a second moment v per weight;
 * both are stored in 4 bits with one fp32 scale per block of 128 values
 * (1.0625 bytes per parameter), m in NF4, v in one of two codes:
 *   - ZIP-SR: the zero-inclusive code {k/15 * s}, rounded stochastically so
 *     that the preconditioner h(v) = 1/(sqrt(v/(1-b2^t)) + eps) is unbiased;
 *   - ZE-EDEN: the zero-excluded code {(k+1)/16 * s}, rounded to nearest,
 *     with the block scale multiplied by ||x||^2 / max(<x,Q(x)>, 1e-12 s^2).
 * The LM-head first moment is rounded stochastically (in state space) over
 * the final 10% of training; normalisation-layer tensors and tensors under
 * 4096 elements keep fp32 state.
 *
 * Sources (page title -- section):
 *   "ZIP-SR / ZE-EDEN: 4-bit AdamW state quantization" (daiwk.github.io)
 *       -- Method flowchart (decode, update moments, update weights,
 *          quantise, pack), Core equation (h(v), the ZIP-SR probability, the
 *          ZE-EDEN scale, weights updated before the moments are quantised),
 *          Local reproduction notes (uint8 nibble packing, fp32 block scales,
 *          fp32 fallback below 4096 elements).
 *   "ZIP-SR 4-bit AdamW -- Preconditioner-space stochastic rounding -- What
 *    does it mean?" (learnaivisually.com)
 *       -- memory paragraph (128-value blocks with one fp32 scale, 1.0625
 *          B/param, normalisation-layer states in fp32), ZE-EDEN paragraph
 *          (NF4 for m, LM-head stochastic rounding in the final 10%).
 *   "A New Approach to 4-bit AdamW Optimizer Quantization: Rounding in
 *    Preconditioner Space" (kongchang.com)
 *       -- AdamW and optimizer states; Preconditioner; Two Complementary
 *          Technical Approaches.
 *
 * Conventions for every entry point:
 *   - Status codes are returned; nothing is thrown across the ABI.  On an
 *     error the handle's state is unchanged (except where stated) and
 *     adamw4_last_error() describes it.
 *   - Device pointers are raw CUDA device addresses on the handle's device.
 *     Host pointers are plain process memory.
 *   - A handle is not thread-safe; one thread at a time may use it.
 *   - Work is enqueued on the caller's CUDA stream (a cudaStream_t passed as
 *     void*; NULL is the legacy default stream).  A device-side failure of an
 *     earlier step surfaces as ADAMW4_ECUDA on a later call.
 */
#ifndef ADAMW4_H
#define ADAMW4_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ADAMW4_OK = 0,
    ADAMW4_EINVAL = -1,     /* bad argument, bad descriptor, unknown handle    */
    ADAMW4_EALIGN = -2,     /* a device pointer is not 16-byte aligned         */
    ADAMW4_ENOMEM = -3,     /* device or host allocation failed                */
    ADAMW4_ECUDA = -4,      /* a CUDA runtime call or kernel launch failed     */
    ADAMW4_ESTATE = -5,     /* state blob does not match this handle           */
    ADAMW4_ENONFINITE = -6, /* a step produced a non-finite weight (NaN or +-inf:
                               from a non-finite grad or weight, or an overflow);
                               reported by adamw4_sync, the step still ran      */
    ADAMW4_ETIMEOUT = -7,   /* a bounded wait inside the step kernel ran out   */
    ADAMW4_ECHECK = -8,     /* library built with ADAMW4_CHECKED: a unit's values or
                               state fell outside its tensor or the state arena */
    ADAMW4_ERANGE = -9      /* size above a stated maximum, or a buffer too small */
} adamw4_status;

/* Faults adamw4_inject_fault can arm (test hooks; no GPU fault is raised). */
enum {
    ADAMW4_FAULT_STALL_PIPELINE = 1  /* next step: stages marked pending, never filled */
};

/* Second-moment codes.  ZIPSR and ZEEDEN are the two methods; the other three
 * are the state-space quantisers the pages compare them with (the controlled
 * ablation's round-to-nearest and stochastic rounding on the zero-inclusive
 * code, and a zero-excluded code with a positive floor and no rescale). */
typedef enum {
    ADAMW4_V_ZIPSR = 0,     /* zero-inclusive code, preconditioner-space SR    */
    ADAMW4_V_ZEEDEN = 1,    /* zero-excluded code, EDEN block rescale          */
    ADAMW4_V_ZI_RTN = 2,    /* zero-inclusive code, state-space nearest        */
    ADAMW4_V_ZI_SR = 3,     /* zero-inclusive code, state-space SR             */
    ADAMW4_V_ZE_FLOOR = 4,  /* zero-excluded code, nearest, no rescale         */
    ADAMW4_V_ZIPSR_U32 = 5  /* ZIP-SR with the decision taken in binary64: lower
                               iff (word * 2^-32) * B < rhs in one binary64 multiply
                               (ZIP-SR itself rounds the word and the product to
                               binary32; both resolve the keep probability to
                               2^-32 near zero) */
} adamw4_vcode;

/* Per-tensor flags. */
enum {
    ADAMW4_T_NORM = 1u,       /* normalisation-layer tensor: fp32 state        */
    ADAMW4_T_LM_HEAD = 2u,    /* LM head: m rounded stochastically in the final 10% */
    ADAMW4_T_FP32_STATE = 4u, /* force fp32 state                              */
    ADAMW4_T_QUANT_STATE = 8u, /* force 4-bit state below 4096 elements: a piece of a
                                  larger 4-bit tensor (not with NORM / FP32_STATE) */
    ADAMW4_T_BF16_PARAM = 16u  /* the weights are bf16, not fp32 (see adamw4_tensor) */
};

/* Tensors below this many elements keep fp32 state. */
#define ADAMW4_MIN_QUANT_NUMEL 4096
/* Values per quantisation block (one fp32 scale per block per moment). */
#define ADAMW4_BLOCK 128

/* One parameter tensor, flattened row-major, or a piece of one.
 *   param      device, fp32, numel elements, 16-byte aligned; updated in place.
 *              With ADAMW4_T_BF16_PARAM it holds numel bf16 bit patterns
 *              instead (pass it cast to float*): the step reads them exactly,
 *              computes the update in binary32 as for fp32 weights, and stores
 *              the result rounded to the nearest bf16 (ties to even).  Updates
 *              below half a bf16 ulp of a weight are then lost; the pages keep
 *              no bf16 weights, this is a lower-memory option (2 B/param less
 *              read and written per step).
 *   grad_bf16  device, bf16 bit patterns, numel elements, 16-byte aligned; read
 *   tensor_id  unique within a handle; keys the random draws, so it must stay
 *              the same across a checkpoint and resume
 *   flags      ADAMW4_T_* bits (other bits: ADAMW4_EINVAL)
 *   weight_decay  decoupled weight decay of this tensor (w <- w (1 - lr wd))
 *   elem_offset   0 for a whole tensor.  For a piece of a larger (logical)
 *              tensor, the index of the piece's first element in it: a
 *              multiple of 128 in [0, 2^39).  Blocks and random draws are
 *              keyed by the logical index, so stepping the pieces of a tensor
 *              (in one handle each, on one device or on several) gives the
 *              same bits as stepping the whole tensor.  A piece under 4096
 *              elements of a 4-bit tensor needs ADAMW4_T_QUANT_STATE, and a
 *              piece of an fp32-state tensor ADAMW4_T_FP32_STATE, so that it is
 *              classified like the whole.  The pages describe single-device
 *              training; the pieces are this library's ZeRO-1 sharding.
 * Both buffers are borrowed: they stay owned by the caller, and must stay
 * allocated and at the same address until adamw4_destroy. */
typedef struct {
    float *param;
    const uint16_t *grad_bf16;
    int64_t numel;
    uint32_t tensor_id;
    uint32_t flags;
    float weight_decay;
    int64_t elem_offset;
} adamw4_tensor;

/* Optimizer configuration.
 *   lr            default learning rate (each step passes its own lr)
 *   beta1, beta2  in [0, 1); eps > 0
 *   vcode         an adamw4_vcode
 *   seed          key of the counter-based random draws
 *   total_steps   T for the final-10% LM-head phase (active when 10 t > 9 T);
 *                 0 means the phase never starts */
typedef struct {
    float lr, beta1, beta2, eps;
    int32_t vcode;
    uint64_t seed;
    int64_t total_steps;
} adamw4_config;

typedef struct adamw4_handle adamw4_handle;

/* Creates an optimizer over n tensors on CUDA device `device`.
 * State layout from "ZIP-SR 4-bit AdamW -- Preconditioner-space stochastic
 * rounding" (learnaivisually.com), memory paragraph (128-value blocks, one
 * fp32 scale each, norm layers in fp32), and "ZIP-SR / ZE-EDEN: 4-bit AdamW
 * state quantization" (daiwk.github.io), Local reproduction notes (uint8
 * nibble pairs, fp32 state below 4096 elements).
 * Validates every descriptor on the host (non-NULL pointers, 16-byte
 * alignment, numel > 0, unique tensor_id, known flags, elem_offset), classifies
 * each tensor (fp32 state when flagged NORM/FP32_STATE, or when numel < 4096
 * and not flagged QUANT_STATE; else 4-bit), allocates the
 * packed state (owned by the handle) and zeroes it, which is the all-zero
 * initial state m = v = 0.  The step counter starts at t = 0.
 * Returns ADAMW4_EINVAL / EALIGN for bad input, ENOMEM, ECUDA.
 * On success *out receives the handle. */
int adamw4_create(const adamw4_config *cfg, const adamw4_tensor *tensors, int n, int device,
                  adamw4_handle **out);

/* One optimizer step over every tensor: t <- t + 1, then for each weight
 * decode (m, v), m <- b1 m + (1-b1) g, v <- b2 v + (1-b2) g^2,
 * w <- w (1 - lr wd) - lr/(1-b1^t) * m / (sqrt(v)/sqrt(1-b2^t) + eps),
 * then requantise and pack m and v: m to NF4 (nearest, or state-space
 * stochastic rounding for the LM head in the final 10%), v by the handle's
 * vcode.  Implements "ZIP-SR / ZE-EDEN: 4-bit AdamW state quantization"
 * (daiwk.github.io), Method flowchart and Core equation (the weights use the
 * unquantised moments; the ZIP-SR probability and the ZE-EDEN scale), with
 * the AdamW form of "A New Approach to 4-bit AdamW Optimizer Quantization"
 * (kongchang.com), AdamW and optimizer states.  lr must be finite and >= 0
 * (else ADAMW4_EINVAL, nothing enqueued).  A single kernel launch on
 * `cuda_stream`; the call returns without waiting.  Reads the grads, updates
 * the params and the state in place; device-side failures (a timed-out wait,
 * a non-finite updated weight) are reported by adamw4_sync. */
int adamw4_step(adamw4_handle *h, float lr, void *cuda_stream);

/* The same step with host buffers: for each tensor i, copies grads_host[i]
 * (numel bf16) to the tensor's device grad buffer, runs the step, copies the
 * updated params back to params_host[i] (numel fp32; numel bf16 for a tensor
 * flagged ADAMW4_T_BF16_PARAM), and waits for `cuda_stream`.
 * The work is pipelined over pieces of about 64 Mi values (whole 128-value
 * units, cutting tensors where they fall): piece k's grads go up on a copy
 * stream of the handle, piece k steps on `cuda_stream` (one launch per piece,
 * all at the same t, so the result equals adamw4_step's), and its params come
 * down on a second copy stream while the next pieces go up and step.  The
 * copies start after the work already queued on `cuda_stream`.  Pinned host
 * memory lets the copies overlap; pageable memory works but serialises them.
 * Either array may be NULL to skip that direction.  A CUDA error part-way
 * leaves the step partly applied. */
int adamw4_step_host(adamw4_handle *h, float lr, const uint16_t *const *grads_host,
                     float *const *params_host, void *cuda_stream);

/* Waits for `cuda_stream` and reports whether the steps enqueued on it so far
 * completed.  The step kernel bounds every wait on its shared-memory pipeline
 * (about one second); when a wait runs out, the kernel records it in a device
 * status word and the waiting warp stops, leaving that step incomplete.  The
 * kernel also records an updated weight that is not finite (a NaN or infinite
 * grad or weight leads to one; the pages leave non-finite inputs undefined, so
 * the step itself goes on).  This call reads and clears the word:
 * ADAMW4_ETIMEOUT if a wait ran out, else ADAMW4_ENONFINITE if a weight was
 * not finite, ADAMW4_ECUDA on a CUDA error, else ADAMW4_OK.  The CUDA context
 * stays usable.
 * A library built with -DADAMW4_CHECKED (build.py --checked, a debugging aid
 * in place of a memory checker) also tests every unit's element and state
 * range on the device; a unit outside them is skipped and this call returns
 * ADAMW4_ECHECK. */
int adamw4_sync(adamw4_handle *h, void *cuda_stream);

/* Test hook: arms `fault` (ADAMW4_FAULT_STALL_PIPELINE, or 0 to disarm) for
 * the next adamw4_step only (with h = NULL: for the next adamw4_step_noalloc
 * call of this process instead).  With the stall armed the kernel marks its
 * pipeline stages as filled without issuing the copies, so every stage wait
 * runs out after its time limit and adamw4_sync then returns ADAMW4_ETIMEOUT.
 * Nothing faults; the handle's state after that step is unspecified. */
int adamw4_inject_fault(adamw4_handle *h, int fault);

/* Frees the state and the handle.  Unknown or already destroyed handles
 * return ADAMW4_EINVAL. */
int adamw4_destroy(adamw4_handle *h);

/* Step counter: the last completed step (0 before the first).  After
 * adamw4_set_step(h, 999) the next step runs at t = 1000. */
int adamw4_get_step(const adamw4_handle *h, int64_t *t);
int adamw4_set_step(adamw4_handle *h, int64_t t);

/* Persistent optimizer-state bytes: 136 per 128-value block of each 4-bit
 * tensor (64 + 64 code bytes, two fp32 scales) plus 8 per element of each fp32
 * tensor; 1.0625 bytes per quantised parameter when numel is a multiple of
 * 128.  Alignment padding inside the allocation (at most 508 bytes per fp32
 * tensor) is not counted.  Returns -1 for an unknown handle. */
int64_t adamw4_state_bytes(const adamw4_handle *h);

/* Checkpoint.  The blob (little-endian) is
 *   char magic[8] = "ADAMW4S1"; uint32 n_tensors; uint32 vcode; int64 t;
 *   uint64 seed; uint64 payload_bytes;                       (40 bytes)
 * then per tensor, in creation order:
 *   uint32 tensor_id; uint32 kind (0 = 4-bit, 1 = fp32); int64 numel;
 *   4-bit: m codes [nb*64] u8, v codes [nb*64] u8, m scales [nb] f32,
 *          v scales [nb] f32, nb = ceil(numel/128);
 *   fp32:  m [numel] f32, v [numel] f32.
 * adamw4_state_export writes it to host_buf (capacity cap bytes; *used gets
 * the size, also when cap is too small, which returns ADAMW4_ERANGE;
 * host_buf may be NULL to query).  adamw4_state_import reads such a blob into
 * a handle created over the same tensor list (same ids, kinds, numels,
 * vcode and seed, else ADAMW4_ESTATE) and sets t.  Both synchronise the device
 * and copy with the CUDA runtime.  The blob does not record elem_offset: a
 * handle over pieces of tensors must be re-created over the same pieces, or
 * the pieces' blobs merged into a whole-tensor blob and cut again for the new
 * pieces (the Python zero1 module does both). */
int adamw4_state_export(const adamw4_handle *h, void *host_buf, int64_t cap, int64_t *used);
int adamw4_state_import(adamw4_handle *h, const void *host_buf, int64_t len);

/* The state class the library gives one descriptor (host only; its pointers
 * are not looked at): 1 when it keeps fp32 m and v (flagged NORM or
 * FP32_STATE, or numel < ADAMW4_MIN_QUANT_NUMEL and not flagged
 * QUANT_STATE), 0 when it keeps 4-bit codes and block scales, ADAMW4_EINVAL
 * for a NULL pointer, numel <= 0, unknown flag bits, QUANT_STATE with NORM or
 * FP32_STATE, or a bad elem_offset.  The classification follows "ZIP-SR
 * 4-bit AdamW -- Preconditioner-space stochastic rounding" (learnaivisually.com),
 * memory paragraph (normalisation layers in fp32), and "ZIP-SR / ZE-EDEN:
 * 4-bit AdamW state quantization" (daiwk.github.io), Local reproduction
 * notes (tensors below 4096 elements in fp32). */
int adamw4_tensor_state_kind(const adamw4_tensor *t);

/* Launch geometry used by adamw4_step (filled at create): CUDA blocks, threads
 * per block, and 128-value work units (4-bit blocks plus fp32 chunks). */
int adamw4_launch_info(const adamw4_handle *h, int *grid, int *block, int64_t *units);

/* ---------------------------------------------------------------------------
 * Allocation-free step.  The paper has no counterpart: this entry point exists
 * for callers that must not allocate device memory.  Examples are programs
 * whose device memory belongs to a pooling allocator or a fixed arena sized at
 * start-up, which has to account for every byte, and tight training loops,
 * where cudaMalloc and cudaFree can synchronise the device and stall other
 * streams.
 *
 * It runs the same step as adamw4_step, without a handle.  The caller passes
 * the tensors, the packed state buffers below, the step number t (1-based)
 * and lr; nothing is allocated.  The step kernel's own scratch (its table of
 * tensor descriptors and the status word of its bounded waits) lives in one
 * static device array of 256 + 64 * ADAMW4_NOALLOC_MAX_TENSORS bytes (about
 * 64 KB) that every GPU which loads this library holds until the process exits.
 *   - More than ADAMW4_NOALLOC_MAX_TENSORS tensors: ADAMW4_ERANGE, nothing runs.
 *   - Bad arguments: ADAMW4_EINVAL / ADAMW4_EALIGN, checked on the host first.
 *     The status code is the whole report: this call records no message for
 *     adamw4_last_error.
 *   - The first call on a device looks up the array's device address and the
 *     launch geometry for that device.
 *   - All calls share the one array and each overwrites it: calls whose work
 *     overlaps on the GPU (different streams, or different host threads without
 *     ordering) race.  Calls on one stream are ordered and safe.
 *   - The descriptor table is copied from a host staging array of this library
 *     with a pageable cudaMemcpyAsync, which the call's return leaves free for
 *     the next call.
 *   - Device-side failures (a pipeline wait that ran out, which ends the kernel
 *     early like in adamw4_step, or a non-finite updated weight) go to the
 *     status word in the array; adamw4_noalloc_sync reads and clears it.  The
 *     call itself returns only host-side and launch errors.
 * Results equal adamw4_step's for the same inputs, state and t.
 * ------------------------------------------------------------------------- */
#define ADAMW4_NOALLOC_MAX_TENSORS 1024

/* Packed optimizer state in caller-owned device memory, in the order of the
 * tensor list.  4-bit tensors (see adamw4_create for the classification) own
 * ceil(numel/128) consecutive blocks each; fp32-state tensors own consecutive
 * ranges of m32/v32, each starting at a multiple of 128 elements.
 *   mcodes, vcodes  64 bytes per block (element 2i in the low nibble of byte
 *                   i), 16-byte aligned
 *   mscale, vscale  one float per block, 4-byte aligned
 *   m32, v32        floats, 16-byte aligned
 * All-zero buffers are the initial state m = v = 0. */
typedef struct {
    uint8_t *mcodes, *vcodes;
    float *mscale, *vscale;
    float *m32, *v32;
} adamw4_state_buffers;

int adamw4_step_noalloc(const adamw4_config *cfg, const adamw4_tensor *tensors, int n,
                        const adamw4_state_buffers *state, int64_t t, float lr, int device,
                        void *cuda_stream);

/* Waits for `cuda_stream` and reads and clears the allocation-free step's
 * status word on `device` (with cudaMemcpyFromSymbol / cudaMemcpyToSymbol, no
 * allocation): ADAMW4_ETIMEOUT if a stage wait of a call on that device ran
 * out, else ADAMW4_ENONFINITE if a call produced a non-finite weight,
 * ADAMW4_ECUDA on a CUDA error, else ADAMW4_OK.  The word is shared by every
 * call on the device, so it reports all of them since the last read.
 * ADAMW4_EINVAL for a device no call has used yet. */
int adamw4_noalloc_sync(int device, void *cuda_stream);

/* Message of the last failed call on this handle, or of the last failed call
 * on this thread when h is NULL.  Never NULL; valid until the next call. */
const char *adamw4_last_error(const adamw4_handle *h);

#ifdef __cplusplus
}
#endif

#endif /* ADAMW4_H */
