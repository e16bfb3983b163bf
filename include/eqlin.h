/*
 * eqlin.h -- C ABI of the B200 (sm_100a) EQ-Linear over the cyclic group C_G:
 * the forward pass and its backward (input, weight and bias gradients).
 *
 * The operation.  Page "Flash EQ-Linear: Accelerating Equivariant Linear Layers
 * via Group-wise Discrete Fourier Transform", section "Percepcion Central": an
 * EQ-Linear layer is a circular convolution along the group axis composed with a
 * linear map over channels; its weight matrix is group-circulant (one learnable
 * set, cyclically shifted and replicated).  Written out:
 *
 *     y[n,o,g] = bias[o] + sum_{i<Cin} sum_{h<G} w[o,i,(g-h) mod G] * x[n,i,h]
 *
 * Section "Enfoque Algoritmico": it is computed exactly as a real DFT over the
 * group axis, one complex [Cout x Cin] contraction per frequency on the
 * non-redundant half of the spectrum (k = 0..G/2; conjugate symmetry of real
 * data), and an inverse DFT -- here fused into one kernel (section
 * "Implementacion").  The bias term is this library's reading (the page shows
 * none); a NULL bias means zero.
 *
 * Conventions for every entry point:
 *   - Tensors are dense and C-contiguous with the group axis fastest:
 *       x [N, Cin, G], w [Cout, Cin, G], bias [Cout], y [N, Cout, G].
 *   - "device" pointers are CUDA global-memory addresses on the CURRENT device
 *     (the device the handle was prepared on); "host" pointers are ordinary host
 *     memory.  The caller owns every pointer it passes.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   - Every function returns an eqlin_status: 0 on success, a negative code on
 *     failure.  Arguments are validated on the host before anything is launched;
 *     a failed call launches nothing and changes nothing.  Nothing throws, aborts
 *     or prints.  eqlin_last_error() describes the latest failure of the
 *     calling thread.
 *   - Supported: G in {2, 4, 8, 16}; Cin, Cout >= 1; for 16-bit I/O (bf16 or fp16)
 *     Cin*G and Cout*G multiples of 8 (16-byte rows for the TMA engine).  io_dtype
 *     EQLIN_BF16 or EQLIN_F16 runs the fused tcgen05 (tensor-core) kernels with that
 *     operand type and fp32 accumulation; EQLIN_F32 runs a fused FFMA kernel in float64.
 *   - Requires a compute-capability 10.0 device (B200).
 */
#ifndef EQLIN_H
#define EQLIN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define EQLIN_API __attribute__((visibility("default")))
#else
#define EQLIN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct eqlin_handle eqlin_handle; /* opaque */

typedef enum {
    EQLIN_F32 = 0,  /* IEEE float32 */
    EQLIN_BF16 = 1, /* bfloat16 */
    EQLIN_F16 = 2   /* IEEE float16 (the page's FP16 kernels, section "Implementacion") */
} eqlin_dtype;

typedef enum {
    EQLIN_OK = 0,
    EQLIN_ERR_INVALID_ARG = -1, /* null pointer, bad size, dtype or handle */
    EQLIN_ERR_UNSUPPORTED = -2, /* valid but not implemented (G, shape, device) */
    EQLIN_ERR_MISALIGNED = -3,  /* a device pointer is not 16-byte aligned */
    EQLIN_ERR_CUDA = -4,        /* a CUDA runtime / driver call failed */
    EQLIN_ERR_OOM = -5,         /* device allocation failed */
    EQLIN_ERR_TIMEOUT = -6      /* a kernel wait ran out (reported by the device) */
} eqlin_status;

/*
 * eqlin_prepare_weights -- move the weights to the frequency domain, once per
 * weight update (section "Enfoque Algoritmico": the per-frequency products need
 * W^_k = sum_m w[o,i,m] exp(-2 pi i m k / G), k = 0..G/2).
 *
 *   w        device, [Cout, Cin, G] of w_dtype.  Read only.
 *   bias     device, [Cout] of w_dtype, or NULL (zero bias).  Read only.
 *   Cout, Cin, G   layer sizes (see "Supported" above).
 *   w_dtype  EQLIN_F32, EQLIN_BF16 or EQLIN_F16: element type of w and bias.
 *   io_dtype EQLIN_F32, EQLIN_BF16 or EQLIN_F16: element type of x and y in
 *            eqlin_forward (and of dy, dx in the backward calls).
 *   stream   stream the transform runs on; the call synchronises it before
 *            returning, so w and bias may be freed or changed afterwards.
 *   out      host; receives the new handle (set to NULL on failure).
 *
 * The handle owns device memory for the transformed weights (16-bit tensor-core
 * image and/or fp32 planes), an fp32 copy of the bias and a device status word.
 * Errors: INVALID_ARG (null w/out, non-positive sizes, unknown dtype),
 * UNSUPPORTED (G not in {2,4,8,16}, Cin*G or Cout*G not a multiple of 8 for 16-bit I/O,
 * not an sm_100 device, shape too large for shared memory), MISALIGNED (w or
 * bias not aligned to its element size), OOM, CUDA.
 */
EQLIN_API int eqlin_prepare_weights(const void* w, const void* bias, int64_t Cout, int64_t Cin, int64_t G,
                          int w_dtype, int io_dtype, void* stream, eqlin_handle** out);

/*
 * eqlin_forward -- y = EQ-Linear(x), the whole forward in one fused launch:
 * TMA-staged loads of x, the group DFT in registers, the per-frequency
 * contractions (tcgen05 tensor cores for bf16 / fp16), the inverse DFT plus bias
 * written straight to y (sections "Enfoque Algoritmico", "Implementacion").
 *
 *   h        handle from eqlin_prepare_weights.  Not modified; may be shared by
 *            concurrent forwards on any streams.
 *   x        device, [N, Cin, G] of the handle's io_dtype, 16-byte aligned.
 *   y        device, [N, Cout, G] of io_dtype, 16-byte aligned; must not overlap x.
 *   N        number of tokens (rows); N == 0 is a no-op returning EQLIN_OK.
 *            N < 2^31.
 *   stream   the launch is asynchronous on this stream; the call allocates
 *            nothing and does not synchronise (unless the environment variable
 *            EQLIN_SYNC_CHECK=1 was set when the handle was prepared, in which
 *            case it synchronises and returns the device status word).
 *
 * Errors: INVALID_ARG (null handle, N < 0, null x/y with N > 0, wrong current
 * device), MISALIGNED (x or y not 16-byte aligned), CUDA (launch failure).
 * A bounded wait that expires inside the kernel is not reported by this call
 * (it is asynchronous); it sets the handle's device status word to
 * EQLIN_ERR_TIMEOUT, read with eqlin_device_status().
 */
EQLIN_API int eqlin_forward(const eqlin_handle* h, const void* x, void* y, int64_t N, void* stream);

/*
 * eqlin_forward_host -- the same forward with x and y in HOST memory: the library
 * copies x in, runs the fused kernel and copies y back, chunk by chunk, so that the
 * host-to-device copy of one chunk, the kernel of another and the device-to-host copy
 * of a third overlap (three internal streams: copies in, kernels, copies out;
 * full-duplex copies).
 *
 *   h        handle from eqlin_prepare_weights.  The first call allocates the handle's
 *            staging buffers (four chunks of x and of y, about 64 MB) and three streams,
 *            freed by eqlin_destroy.  Calls on one handle are serialised by the
 *            library (a mutex for the host side, the internal streams for the GPU).
 *   x_host   host, [N, Cin, G] of the handle's io_dtype.  Pinned memory (cudaHostAlloc,
 *            cudaHostRegister, torch pin_memory) lets the copies overlap; pageable
 *            memory works but the copies then serialise with the host.
 *   y_host   host, [N, Cout, G] of io_dtype; must not overlap x_host.
 *   N        number of tokens; N == 0 is a no-op returning EQLIN_OK.  N < 2^31.
 *   stream   ordering: the work starts after everything already queued on `stream`,
 *            and `stream` waits for its completion.  Asynchronous: synchronise `stream`
 *            before reading y_host (or reusing x_host).
 *
 * Errors: INVALID_ARG (null handle, N < 0, null x_host/y_host with N > 0, wrong
 * current device), OOM (staging allocation), CUDA (copy or launch failure).  Device
 * timeouts are reported as for eqlin_forward.
 */
EQLIN_API int eqlin_forward_host(eqlin_handle* h, const void* x_host, void* y_host, int64_t N, void* stream);

/*
 * eqlin_destroy -- free the handle and its device memory.  The caller must
 * ensure no forward using it is still executing (e.g. synchronise the streams).
 * NULL is accepted and ignored.  Returns EQLIN_OK, or CUDA if a free failed.
 */
EQLIN_API int eqlin_destroy(eqlin_handle* h);

/*
 * eqlin_device_status -- synchronise the device, then read and clear the
 * handle's device status word: *status_out receives EQLIN_OK or the first
 * error a kernel recorded (EQLIN_ERR_TIMEOUT).  Errors: INVALID_ARG, CUDA.
 */
EQLIN_API int eqlin_device_status(eqlin_handle* h, int* status_out);

/*
 * eqlin_get_attr -- read one property of a prepared handle (host only, no GPU
 * work).  attr is one of EQLIN_ATTR_*; *value receives it.
 * Errors: INVALID_ARG (null handle/value, unknown attr).
 */
enum {
    EQLIN_ATTR_G = 0,
    EQLIN_ATTR_CIN = 1,
    EQLIN_ATTR_COUT = 2,
    EQLIN_ATTR_IO_DTYPE = 3,
    EQLIN_ATTR_PATH = 4,            /* kernel variant: 0/1 tcgen05 with tokens on the MMA N dimension,
                                       weights resident / streamed; 2 fp32 I/O (float64 arithmetic);
                                       3/4 tcgen05 with tokens on the MMA M dimension, resident / streamed;
                                       5 tcgen05 with tokens on N and the input spectrum resident
                                       across output chunks (Cout > 128 and at least 4 chunks
                                       of 32 input channels), weights streamed */
    EQLIN_ATTR_TOKENS_PER_TILE = 5, /* tokens per work item of the fused kernel */
    EQLIN_ATTR_STAGES = 6,          /* depth of the shared-memory ring */
    EQLIN_ATTR_SMEM_BYTES = 7,      /* dynamic shared memory per CTA */
    EQLIN_ATTR_MAX_GRID = 8,        /* CTAs launched for a large N (one per SM) */
    EQLIN_ATTR_WEIGHT_BYTES = 9,    /* bytes of the frequency-domain weights the kernel reads */
    EQLIN_ATTR_ACTIVATION = 10,     /* epilogue activation of the forward: 0 none, 1 GELU */
    EQLIN_ATTR_Y_STAGING = 11,      /* tokens-on-N kernels: y staging buffers per epilogue warp
                                       (1 or 2, TMA stores), 0 = direct stores from registers;
                                       -1 for the other kernels */
    EQLIN_ATTR_DW_TILE_ROWS = 12,   /* weight gradient (16-bit I/O): output rows of a unit */
    EQLIN_ATTR_DW_TILE_COLS = 13,   /* weight gradient: input columns of a unit */
    EQLIN_ATTR_DW_RAW_STAGES = 14,  /* weight gradient: depth of the raw dy / x ring */
    EQLIN_ATTR_DW_TOKENS = 15       /* weight gradient: tokens per chunk */
};
EQLIN_API int eqlin_get_attr(const eqlin_handle* h, int attr, int64_t* value);

/*
 * eqlin_query_plan -- the same properties (EQLIN_ATTR_PATH .. EQLIN_ATTR_DW_TOKENS,
 * except ACTIVATION) that eqlin_prepare_weights would give a handle of these sizes
 * without an activation (a GELU handle with Cout > 128 and G <= 8 takes the tokens-on-N
 * kernel with the input spectrum resident wherever it fits),
 * planned on the host for a B200 (227 KB of shared memory per CTA, 148 SMs) under the
 * current environment overrides.  Host only: no GPU, no allocation.  The weight-gradient
 * attributes are -1 where no tiling fits (or for fp32 I/O).
 * Errors: INVALID_ARG / UNSUPPORTED as eqlin_check_shape, INVALID_ARG for an unknown attr.
 */
EQLIN_API int eqlin_query_plan(int64_t Cout, int64_t Cin, int64_t G, int io_dtype, int attr, int64_t* value);

/*
 * eqlin_copy_freq_weights -- copy the fp32 frequency-domain weights to host
 * memory, for inspection and tests.  Layout [G][Cin][Cout] (output channel
 * fastest), planes in the order Re W^_0, Re W^_{G/2}, then Re W^_k, Im W^_k for
 * k = 1..G/2-1, with W^_k = sum_m w[o,i,m] exp(-2 pi i m k / G) scaled by 1/G
 * (planes 0, 1) or 2/G (the others).  dst: host, `count` floats, count must be
 * >= G*Cin*Cout.  Synchronous.  Errors: INVALID_ARG, CUDA.
 */
EQLIN_API int eqlin_copy_freq_weights(const eqlin_handle* h, float* dst, int64_t count);

/*
 * eqlin_check_shape -- would eqlin_prepare_weights accept these sizes and
 * dtypes?  Host only (no GPU needed).  Returns EQLIN_OK, INVALID_ARG or
 * UNSUPPORTED, exactly as prepare's host-side validation would.
 */
EQLIN_API int eqlin_check_shape(int64_t Cout, int64_t Cin, int64_t G, int w_dtype, int io_dtype);

/*
 * eqlin_forward_noalloc -- the same forward as eqlin_prepare_weights followed by
 * eqlin_forward, in one call that allocates no device memory.  (Not a step of the
 * method: the source page has no counterpart; it exists for callers that cannot
 * allocate.)
 *
 * It is meant for callers that must not call cudaMalloc: a framework whose device
 * memory is owned by its own pool (a stray driver allocation fragments the pool or is
 * refused outright), or a host loop that cannot take the device-wide synchronisation
 * and latency an allocation or free can imply.  The caller passes its inputs and its
 * output; the device status word and the frequency-domain weights (which the handle
 * API keeps in memory it allocates) live instead in one fixed array of
 * EQLIN_NOALLOC_SCRATCH_BYTES (4 MiB) that is part of the library image, so every GPU
 * that loads the library holds it until the process exits.
 *
 *   x, y     device, [N, Cin, G] / [N, Cout, G] of dtype, 16-byte aligned.
 *   w, bias  device, [Cout, Cin, G] / [Cout] of dtype (bias may be NULL).
 *   dtype    EQLIN_BF16, EQLIN_F16 or EQLIN_F32, for all four tensors.
 *   stream   every step (weight transform, forward) is enqueued on it; nothing is
 *            synchronised.
 *
 * Each call re-transforms the weights (a small kernel, O(Cout*Cin*G^2)).  Every call
 * on a device shares the one array and leaves its contents there; the status word is
 * cleared at the start of each call.  Calls whose work overlaps on the GPU (other
 * streams, other host threads) race on the array: serialise them.  The first call on
 * a device sets up (it looks up the array's device address and sets kernel
 * attributes) and must be made with that device current and before any stream
 * capture that will contain this call.
 *
 * Errors: as eqlin_prepare_weights / eqlin_forward; UNSUPPORTED also when the shape's
 * transformed weights do not fit in the array (the message gives the bytes needed).
 * Kernel-side wait timeouts are recorded in the array's status word and are not
 * reported to the caller.
 */
#define EQLIN_NOALLOC_SCRATCH_BYTES (4u * 1024u * 1024u)
EQLIN_API int eqlin_forward_noalloc(const void* x, const void* w, const void* bias, void* y, int64_t N,
                                    int64_t Cout, int64_t Cin, int64_t G, int dtype, void* stream);

/*
 * Backward pass.  The page's section "Implementacion" lists backward kernels beside the
 * forward; its results section ("Pasada Backward") reports their speed-ups.  By the chain
 * rule on the definition above, for a loss L and its upstream gradient dy = dL/dy
 * ([N, Cout, G]):
 *
 *     dx[n,i,h] = sum_{o<Cout} sum_{g<G} w[o,i,(g-h) mod G] * dy[n,o,g]
 *     dw[o,i,m] = sum_{n<N}    sum_{g<G} dy[n,o,g] * x[n,i,(g-m) mod G]
 *     dbias[o]  = sum_{n<N}    sum_{g<G} dy[n,o,g]
 *
 * Both gradients are circular correlations along the group axis.  In the frequency domain
 * (section "Enfoque Algoritmico") they become per-frequency products on the half
 * spectrum: dX_k = W^_k^H dY_k, and dW_k = sum_n dY_k conj(X_k).
 *   - dx is the forward of the adjoint operator: the channel axes are swapped and the
 *     filters reflected, f[i,o,m] = w[o,i,(-m) mod G], so the same fused kernels run it
 *     with weights prepared for it.
 *   - dw is a contraction over tokens: a [Cout x N] by [N x Cin] product per frequency,
 *     on tcgen05 for bf16 / fp16, then an inverse DFT over the group axis.
 */

/* eqlin_prepare_weights_ex flag: also prepare the input-gradient weights, so the
 * handle can run eqlin_backward_dx.  They are about the same size as the forward
 * weights. */
#define EQLIN_PREPARE_BACKWARD 1u

/* eqlin_prepare_weights_ex flag: the forward applies GELU after the bias,
 * y = GELU(bias + EQ-Linear(x)), GELU(v) = v * Phi(v) with Phi the standard normal
 * CDF (erf form), in the fused epilogue (fp32 for 16-bit I/O, float64 for fp32 I/O).
 * It is the first half of the equivariant MLP block L2(GELU(L1(x))) of the page's
 * network-level results (section "A Nivel de Red"); the block is a forward with a
 * GELU handle followed by a forward with a plain one.  The backward calls of such a
 * handle compute the gradients of the linear map (before the activation); the
 * activation's derivative GELU'(h) dy is the caller's. */
#define EQLIN_PREPARE_GELU 2u

/*
 * eqlin_prepare_weights_ex -- eqlin_prepare_weights with flags (0, or any of
 * EQLIN_PREPARE_BACKWARD | EQLIN_PREPARE_GELU).  eqlin_prepare_weights(...) is this
 * call with flags 0.  Errors: as eqlin_prepare_weights; INVALID_ARG for an unknown
 * flag bit.
 */
EQLIN_API int eqlin_prepare_weights_ex(const void* w, const void* bias, int64_t Cout, int64_t Cin, int64_t G,
                                       int w_dtype, int io_dtype, unsigned flags, void* stream,
                                       eqlin_handle** out);

/*
 * eqlin_backward_dx -- dx = dL/dx from dy, in one fused launch: the forward kernel on
 * the adjoint operator (the weights were transformed by eqlin_prepare_weights_ex with
 * EQLIN_PREPARE_BACKWARD).
 *
 *   h        handle prepared with EQLIN_PREPARE_BACKWARD.  Not modified.
 *   dy       device, [N, Cout, G] of the handle's io_dtype, 16-byte aligned.
 *   dx       device, [N, Cin, G] of io_dtype, 16-byte aligned; written, not
 *            accumulated; must not overlap dy.
 *   N        tokens; N == 0 is a no-op.  N < 2^31.
 *   stream   asynchronous on this stream; allocates nothing.
 *
 * Errors: INVALID_ARG (null handle/pointers, N < 0, handle prepared without the flag,
 * wrong current device), MISALIGNED, CUDA.  Kernel wait timeouts go to the device
 * status word, as for eqlin_forward.
 */
EQLIN_API int eqlin_backward_dx(const eqlin_handle* h, const void* dy, void* dx, int64_t N, void* stream);

/*
 * eqlin_backward_dw_workspace_size -- bytes of device workspace eqlin_backward_dw needs
 * for N tokens (0 for N == 0).  Host only.  Errors: INVALID_ARG, UNSUPPORTED (no
 * weight-gradient tiling fits shared memory for this shape).
 */
EQLIN_API int eqlin_backward_dw_workspace_size(const eqlin_handle* h, int64_t N, size_t* bytes);

/*
 * eqlin_backward_dw -- dw = dL/dw and dbias = dL/dbias from x and dy.
 *
 *   h          any handle (no flag needed); gives the shape and the io_dtype.
 *   x          device, [N, Cin, G] of io_dtype, 16-byte aligned (the forward's input).
 *   dy         device, [N, Cout, G] of io_dtype, 16-byte aligned.
 *   dw         device, [Cout, Cin, G] float32, written (not accumulated).
 *   dbias      device, [Cout] float32, written; or NULL (not computed).
 *   N          tokens; N == 0 writes zeros to dw (and dbias).  N < 2^31.
 *   workspace  device, at least eqlin_backward_dw_workspace_size(h, N) bytes,
 *              16-byte aligned, owned by the caller.  Its contents on entry do not
 *              matter and on exit are unspecified.  Two calls whose work overlaps on
 *              the GPU must not share it.
 *   stream     asynchronous on this stream: 2 launches for 16-bit I/O (the tcgen05
 *              contraction with a per-CTA partial sum, then a deterministic reduction
 *              of the partial sums fused with the inverse DFT); for fp32, a clear, a float64
 *              CUDA-core kernel and a conversion.  Allocates nothing.
 *
 * 16-bit I/O: the spectra are rounded to the I/O type for the tensor cores and
 * accumulated in fp32; the partial sums are reduced in float64 in a fixed order, so
 * repeated calls give identical results.  fp32: float64 arithmetic throughout (the order of the float64
 * additions across token slices may vary).
 * Errors: INVALID_ARG (null handle/dw, N < 0, null x/dy with N > 0, workspace missing or
 * too small, wrong device), MISALIGNED, UNSUPPORTED, CUDA.  Kernel wait timeouts go to
 * the device status word.
 */
EQLIN_API int eqlin_backward_dw(const eqlin_handle* h, const void* x, const void* dy, float* dw, float* dbias,
                                int64_t N, void* workspace, size_t workspace_bytes, void* stream);

/*
 * The equivariant MLP block y = L2(GELU(L1(x))) in ONE fused launch.  Page "Flash
 * EQ-Linear: ...", section "A Nivel de Red": the network-level gains come from networks
 * built of EQ-Linear layers; section "Implementacion": the Fourier fragments stay on chip
 * between the steps.  Here the hidden activation [N, H, G] never reaches global memory:
 * per token tile the kernel transforms x once, and for each 128-channel chunk of the hidden
 * layer runs the layer-1 contraction (tensor cores), bias, GELU (erf form, as
 * EQLIN_PREPARE_GELU) and the group DFT of the result in registers, then accumulates the
 * layer-2 contraction; the output epilogue adds b2 and writes y.  GELU acts pointwise in
 * the group domain, so the block is equivariant.
 *
 * eqlin_mlp_prepare -- transform both weight sets once per weight update.
 *   w1, b1   device, [H, Cin, G] and [H] (b1 may be NULL) of w_dtype.
 *   w2, b2   device, [Cout, H, G] and [Cout] (b2 may be NULL) of w_dtype.
 *   Cin, H, Cout, G   block sizes; the same "Supported" rules as one layer for each
 *            layer ([H x Cin] and [Cout x H]), and further, for 16-bit I/O, Cout <= 128
 *            (one output chunk) and Cin small enough that the input spectrum of a token
 *            tile stays in shared memory (Cin <= 256, less for large G; UNSUPPORTED
 *            otherwise).  For fp32 I/O: 8 * G * (Cin + H) doubles of shared memory.
 *   w_dtype, io_dtype, stream   as eqlin_prepare_weights (the call synchronises stream).
 *   out      host; receives the handle (NULL on failure).
 * The handle owns the two transformed weight sets, fp32 copies of the biases and a
 * device status word.  Errors: as eqlin_prepare_weights.
 *
 * eqlin_mlp_forward -- y [N, Cout, G] = L2(GELU(L1(x [N, Cin, G]))), one launch,
 * asynchronous on `stream`, allocates nothing.  x and y: device, io_dtype, 16-byte aligned,
 * not overlapping.  16-bit I/O: tcgen05 tensor cores with fp32 accumulation; the hidden
 * spectrum is rounded to the I/O type for the second contraction (the two-launch block
 * rounds the hidden activation instead).  fp32 I/O: float64 throughout, y rounded once.
 * N == 0 is a no-op; N < 2^31.  Errors: as eqlin_forward; kernel wait timeouts go to the
 * handle's device status word (eqlin_mlp_device_status).
 *
 * eqlin_mlp_query -- host only: EQLIN_OK if the fused block supports these sizes (and then
 * the weight-ring depth and the dynamic shared memory of its kernel on a B200), else the
 * status eqlin_mlp_prepare would return.  stages and smem_bytes may be NULL.
 */
typedef struct eqlin_mlp eqlin_mlp; /* opaque */

EQLIN_API int eqlin_mlp_prepare(const void* w1, const void* b1, const void* w2, const void* b2, int64_t Cin,
                                int64_t H, int64_t Cout, int64_t G, int w_dtype, int io_dtype, void* stream,
                                eqlin_mlp** out);
EQLIN_API int eqlin_mlp_forward(const eqlin_mlp* m, const void* x, void* y, int64_t N, void* stream);
/* Reads and clears the block's device status word (synchronises the device). */
EQLIN_API int eqlin_mlp_device_status(eqlin_mlp* m, int* status_out);
/* Frees the handle's device memory; no forward using it may still be in flight.  NULL is a no-op. */
EQLIN_API int eqlin_mlp_destroy(eqlin_mlp* m);
EQLIN_API int eqlin_mlp_query(int64_t Cin, int64_t H, int64_t Cout, int64_t G, int io_dtype, int64_t* stages,
                              int64_t* smem_bytes);

/* Static description of a status code ("ok", "invalid argument", ...). */
EQLIN_API const char* eqlin_status_string(int status);

/* Message for the calling thread's latest failed call ("" if none).  The
 * pointer stays valid until the thread's next call into this library. */
EQLIN_API const char* eqlin_last_error(void);

/* Library version, major*10000 + minor*100 + patch. */
EQLIN_API int eqlin_version(void);

#ifdef __cplusplus
}
#endif

#endif /* EQLIN_H */
