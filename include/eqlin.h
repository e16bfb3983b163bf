/*
 * eqlin.h -- C ABI of the B200 (sm_100a) EQ-Linear forward over the cyclic group C_G.
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
 *   - Supported: G in {2, 4, 8, 16}; Cin, Cout >= 1; for bf16 I/O Cin*G and
 *     Cout*G multiples of 8 (16-byte rows for the TMA engine).  io_dtype EQLIN_BF16 runs the fused
 *     tcgen05 (tensor-core) kernel; EQLIN_F32 runs a fused FFMA kernel.
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
    EQLIN_BF16 = 1  /* bfloat16 */
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
 *   w_dtype  EQLIN_F32 or EQLIN_BF16: element type of w and bias.
 *   io_dtype EQLIN_F32 or EQLIN_BF16: element type of x and y in eqlin_forward.
 *   stream   stream the transform runs on; the call synchronises it before
 *            returning, so w and bias may be freed or changed afterwards.
 *   out      host; receives the new handle (set to NULL on failure).
 *
 * The handle owns device memory for the transformed weights (bf16 tensor-core
 * image and/or fp32 planes), an fp32 copy of the bias and a device status word.
 * Errors: INVALID_ARG (null w/out, non-positive sizes, unknown dtype),
 * UNSUPPORTED (G not in {2,4,8,16}, Cin*G or Cout*G not a multiple of 8 for bf16 I/O,
 * not an sm_100 device, shape too large for shared memory), MISALIGNED (w or
 * bias not aligned to its element size), OOM, CUDA.
 */
EQLIN_API int eqlin_prepare_weights(const void* w, const void* bias, int64_t Cout, int64_t Cin, int64_t G,
                          int w_dtype, int io_dtype, void* stream, eqlin_handle** out);

/*
 * eqlin_forward -- y = EQ-Linear(x), the whole forward in one fused launch:
 * TMA-staged loads of x, the group DFT in registers, the per-frequency
 * contractions (tcgen05 tensor cores for bf16), the inverse DFT plus bias
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
                                       3/4 tcgen05 with tokens on the MMA M dimension, resident / streamed */
    EQLIN_ATTR_TOKENS_PER_TILE = 5, /* tokens per work item of the fused kernel */
    EQLIN_ATTR_STAGES = 6,          /* depth of the shared-memory ring */
    EQLIN_ATTR_SMEM_BYTES = 7,      /* dynamic shared memory per CTA */
    EQLIN_ATTR_MAX_GRID = 8,        /* CTAs launched for a large N (one per SM) */
    EQLIN_ATTR_WEIGHT_BYTES = 9     /* bytes of the frequency-domain weights the kernel reads */
};
EQLIN_API int eqlin_get_attr(const eqlin_handle* h, int attr, int64_t* value);

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
 *   dtype    EQLIN_BF16 or EQLIN_F32, for all four tensors.
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
