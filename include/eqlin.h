/*
 * eqlin.h -- C ABI of the Flash EQ-Linear library for NVIDIA B200 (sm_100a).
 *
 * The operation ("Flash EQ-Linear: Accelerating Equivariant Linear Layers via
 * Group-wise Discrete Fourier Transform", abstract; technical summary of the
 * same paper, section "Insight Central") is the equivariant linear layer whose
 * weight is a group-circulant matrix: a circular convolution along the group
 * axis composed with a linear map along channels.  With T the order of the
 * cyclic group (T = 4 is the rotation group p4), C' input and D' output
 * channels per group element:
 *
 *   y[n, d*T+s] = b[d] + sum_{c<C'} sum_{t<T} W[d, c, (s-t) mod T] * x[n, c*T+t]
 *
 * The library evaluates it the way the paper's section "Abordagem
 * Algoritmica" describes: a real DFT along t, channel GEMMs for each
 * frequency of the non-redundant half spectrum (six real GEMMs for p4,
 * section "Especializacao para o Grupo de Rotacao p4"), then an inverse DFT,
 * all inside its own CUDA kernels.
 *
 * Conventions shared by every call
 * --------------------------------
 * - Layouts are row-major and contiguous:
 *     x  [N, C'*T]  index c*T+t        y  [N, D'*T]  index d*T+s
 *     gy [N, D'*T]  (dL/dy)            dx [N, C'*T]  (dL/dx)
 *     W  [D', C', T]                   b  [D']
 *     dW [D', C', T] float32           db [D'] float32
 * - x, y, gy, dx, W and b have the handle's dtype; dW and db are float32.
 * - Every tensor pointer is a DEVICE pointer owned by the caller, on the
 *   device that was current when the handle was created.  It must be 16-byte
 *   aligned, and every row of x, y, gy and dx must be a multiple of 16 bytes
 *   (C'*T*elemsize and D'*T*elemsize), else EQLIN_ERR_MISALIGNED.
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *   stream).  Calls are stream-ordered and asynchronous: they enqueue kernels
 *   and return without synchronising.  Device-side failures (a bounded wait
 *   that ran out) are recorded in the handle and read with eqlin_get_error()
 *   after the caller has synchronised the stream.
 * - N = 0 is a no-op that returns EQLIN_OK (dW and db are then zeroed).
 * - Supported T: 1, 2, 3, 4, 6, 8.  Other values give EQLIN_ERR_UNSUPPORTED.
 *   The tensor-core kernels serve f16/bf16 for every supported T (T = 3 and 6
 *   with FP32 butterflies and the sqrt(3)/2 twiddles).  FP32 handles of
 *   order T = 1, 2, 4 run every pass on the tensor cores as 3xTF32 (each
 *   operand split into two TF32 terms, three TF32 products per real product,
 *   FP32 accumulation; an FP32-level result, within 1e-5 relative Frobenius
 *   error), and order 8 its forward and dx, except a forward or dx whose
 *   reduction would feed more than 256 MMAs into one accumulator (K = C' or
 *   D' above 680 for T = 1, 2, above 336 for T = 4, 8), which runs on the
 *   CUDA cores; the T = 8 weight gradient and FP32 handles of order 3, 6 run
 *   on the CUDA cores.  The stash forms (fused backward)
 *   take f16/bf16 and T = 1, 2, 4, 8.
 *   eqlin_backward_dw_noalloc takes T = 1, 2, 4, 8 only.
 * - Nothing is thrown across the ABI; every call returns a status.
 * - A handle may be used from one host thread at a time.
 */
#ifndef EQLIN_H
#define EQLIN_H

#include <stdint.h>

#if defined(__GNUC__)
#define EQLIN_API __attribute__((visibility("default")))
#else
#define EQLIN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    EQLIN_F32 = 0,   /* float32 in/out; FP32-level arithmetic (3xTF32 tensor cores or FFMA) */
    EQLIN_F16 = 1,   /* float16 in/out; tensor cores, FP32 accumulation */
    EQLIN_BF16 = 2   /* bfloat16 in/out; tensor cores, FP32 accumulation */
} eqlin_dtype_t;

typedef enum {
    EQLIN_OK = 0,
    EQLIN_ERR_INVALID_ARG = -1,  /* NULL handle/pointer, negative size, bad dtype */
    EQLIN_ERR_UNSUPPORTED = -2,  /* T not in {1,2,3,4,6,8}, or a size beyond the limits */
    EQLIN_ERR_MISALIGNED = -3,   /* pointer or row not 16-byte aligned */
    EQLIN_ERR_CUDA = -4,         /* a CUDA runtime/driver call failed */
    EQLIN_ERR_NO_WEIGHTS = -5,   /* forward/backward before eqlin_set_weights */
    EQLIN_ERR_TIMEOUT = -6,      /* a kernel's bounded wait ran out (device-side) */
    EQLIN_ERR_OOM = -7           /* device allocation failed */
} eqlin_status_t;

typedef enum {
    EQLIN_GROUP_CYCLIC = 0,     /* Z_T, rotations by multiples of 2 pi / T (p4: T = 4) */
    EQLIN_GROUP_DIHEDRAL = 1    /* D_m, rotations and reflections of a regular m-gon, order 2m */
} eqlin_group_t;

typedef struct eqlin_handle *eqlin_t;

/*
 * Create a layer handle for group order T, C' = Cp input and D' = Dp output
 * channels per group element, and the given dtype.  Allocates the handle's
 * device buffers (Fourier-domain weights, bias, the dW reduction workspace and
 * an error word) on the current device.  *out receives the handle.
 * Limits: 1 <= Cp, Dp <= 65536 and Cp*T, Dp*T rows 16-byte multiples.
 */
EQLIN_API eqlin_status_t eqlin_create(int T, int64_t Cp, int64_t Dp, eqlin_dtype_t dtype,
                            eqlin_t *out);

/*
 * A layer over another group: the group convolution
 *
 *   y[n, d*|G|+g] = b[d] + sum_c sum_h W[d, c, h^-1 g] * x[n, c*|G|+h]
 *
 * which for the cyclic group is the formula above ((s - t) mod T = h^-1 g).
 * The paper names reflection groups as future work (technical summary,
 * section "Limitacoes e Trabalho Futuro") without a formula; this is the
 * plainest reading.
 *   group = EQLIN_GROUP_CYCLIC, m = T: the same as eqlin_create(T, ...).
 *   group = EQLIN_GROUP_DIHEDRAL, m in {1, 2, 3, 4, 5, 6, 8}: D_m of order
 *     |G| = 2m, element r^a s^f (rotation by 2 pi a / m after f reflections)
 *     at group index g = f*m + a; products follow from s r = r^-1 s.
 *     Evaluated by the Fourier transform over D_m's real irreducible
 *     representations (12 real channel GEMMs for D_4 against 64), in FP32
 *     CUDA-core kernels for every dtype; the stash forms and
 *     eqlin_backward_dw_noalloc are for cyclic groups only.
 * Layouts and every other call are those of the cyclic layer with T = |G|:
 * x [N, C'*|G|], y [N, D'*|G|], W [D', C', |G|], dW [D', C', |G|] with
 *   dx[n, c*|G|+h] = sum_d sum_g W[d, c, h^-1 g] gy[n, d*|G|+g]
 *   dW[d, c, u]    = sum_n sum_h x[n, c*|G|+h] gy[n, d*|G| + h u]
 *   db[d]          = sum_n sum_g gy[n, d*|G|+g]
 */
EQLIN_API eqlin_status_t eqlin_create_group(eqlin_group_t group, int m, int64_t Cp, int64_t Dp,
                                            eqlin_dtype_t dtype, eqlin_t *out);

/*
 * Load weights: W [D', C', T] and b [D'] (b may be NULL: zero bias), device
 * pointers of the handle's dtype.  Enqueues the weight pre-transform (the DFT
 * of W along its group axis, the paper's Fourier-domain weights) on `stream`;
 * W and b may be freed or overwritten once that work has run.  Must be called
 * again after every weight update.
 */
EQLIN_API eqlin_status_t eqlin_set_weights(eqlin_t h, const void *W, const void *b, void *stream);

/* Forward: y = EQ-Linear(x) + b.  x [N, C'*T] -> y [N, D'*T]. */
EQLIN_API eqlin_status_t eqlin_forward(eqlin_t h, const void *x, void *y, int64_t N, void *stream);

/*
 * The forward with each complex frequency's product in three real GEMMs
 * instead of four (Gauss): with X = Xr + i Xi and W = Wr + i Wi,
 *   k1 = (Xr + Xi) Wr,  k2 = Xr (Wi - Wr),  k3 = Xi (Wr + Wi),
 *   Re(X W) = k1 - k3,  Im(X W) = k1 + k2,
 * five real GEMMs per p4 layer instead of the six the paper counts
 * (technical summary, section "Especializacao para o Grupo de Rotacao p4";
 * the method's general-T form, section "Abordagem Algoritmica", leaves the
 * complex product's evaluation open).  Same arguments and result as
 * eqlin_forward up to rounding: Xr + Xi, Wi - Wr and Wr + Wi are each rounded
 * to the dtype, and k1 - k3 and k1 + k2 cancel, so the error is somewhat
 * larger.  Provided for comparison; T = 4, f16/bf16 handles whose passes both
 * run on the tensor cores, else EQLIN_ERR_UNSUPPORTED.
 */
EQLIN_API eqlin_status_t eqlin_forward_gauss(eqlin_t h, const void *x, void *y, int64_t N, void *stream);

/*
 * Input gradient: dx[n, c*T+t] = sum_d sum_s W[d, c, (s-t) mod T] gy[n, d*T+s].
 * gy [N, D'*T] -> dx [N, C'*T]; dx is overwritten.
 */
EQLIN_API eqlin_status_t eqlin_backward_dx(eqlin_t h, const void *gy, void *dx, int64_t N,
                                 void *stream);

/*
 * Weight and bias gradients over the N tokens:
 *   dW[d, c, tau] = sum_n sum_s gy[n, d*T+s] x[n, c*T + (s-tau) mod T]
 *   db[d]         = sum_n sum_s gy[n, d*T+s]
 * dW [D', C', T] and db [D'] are float32 and OVERWRITTEN (not accumulated);
 * db may be NULL.  Uses the handle's workspace; the reduction is
 * deterministic (fixed order, no atomics).
 */
EQLIN_API eqlin_status_t eqlin_backward_dw(eqlin_t h, const void *x, const void *gy, float *dW,
                                 float *db, int64_t N, void *stream);

/*
 * The fused backward: spectra formed once, by the kernels that already form them
 * --------------------------------------------------------------------------------
 * The paper fuses the data flow so that the Fourier fragments are formed on
 * chip and no intermediate goes through global memory where it can be avoided
 * (technical summary, section "Implementacao"), and attributes the backward
 * pass's smaller speed-up to the gradient's extra memory traffic (section
 * "Resultados Experimentais", operator level).  In this library the forward
 * and the input gradient already form the group DFT of their inputs, X =
 * DFT(x) and G = DFT(gy), in shared memory as their GEMMs' operands.  Their
 * stash forms also write those spectra out, and the weight gradient is then
 * a plain per-frequency GEMM over them (no second DFT of x and gy):
 *
 *   dW_hat_k[d, c] = sum_n G_k[n, d] conj(X_k[n, c]),   db[d] = sum_n G_0[n, d]
 *
 * Spectra layout: T planes x channels x ld tokens of the handle's dtype,
 * tokens contiguous, ld = eqlin_spectra_ld(N) (N rounded up to a multiple of
 * 64); planes in the order Re V_0, Re V_{T/2} (even T), then Re V_k, Im V_k
 * for k = 1 .. ceil(T/2)-1 (p4: V_0, V_2, Re V_1, Im V_1), the unscaled DFT
 * V_k = sum_t v_t e^{-2 pi i k t / T}, rounded to the dtype.  X is
 * [T][C'][ld], G is [T][D'][ld]; columns past N are not written.  The caller
 * owns these buffers (16-byte aligned device memory).
 *
 * The stash forms take f16/bf16 handles whose pass runs on the tensor cores
 * (eqlin_backend_name shows "tcgen05" for it), else EQLIN_ERR_UNSUPPORTED.
 */

/* Row pitch, in elements, of a spectra buffer for N tokens (-1 if N < 0). */
EQLIN_API int64_t eqlin_spectra_ld(int64_t N);

/* eqlin_forward that also writes X = DFT(x) into xs [T][C'][ld]. */
EQLIN_API eqlin_status_t eqlin_forward_stash(eqlin_t h, const void *x, void *y, void *xs, int64_t N,
                                             void *stream);

/* eqlin_backward_dx that also writes G = DFT(gy) into gs [T][D'][ld]. */
EQLIN_API eqlin_status_t eqlin_backward_dx_stash(eqlin_t h, const void *gy, void *dx, void *gs,
                                                 int64_t N, void *stream);

/*
 * dW [D', C', T] and db [D'] (float32, overwritten; db may be NULL) from the
 * spectra xs and gs of the same N tokens, as eqlin_backward_dw computes them
 * from x and gy.  Uses the handle's workspace; deterministic.
 */
EQLIN_API eqlin_status_t eqlin_backward_dw_spectra(eqlin_t h, const void *xs, const void *gs, float *dW,
                                                   float *db, int64_t N, void *stream);

/*
 * The whole backward pass in one call, given the forward's stash xs:
 * dx from gy (writing G into gs), then dW and db from xs and gs.  gy is read
 * from memory once and transformed once.
 */
EQLIN_API eqlin_status_t eqlin_backward(eqlin_t h, const void *gy, const void *xs, void *dx, void *gs,
                                        float *dW, float *db, int64_t N, void *stream);

/*
 * dW and db without a handle and without any device allocation.
 *
 * For callers that cannot call cudaMalloc -- code that runs while another
 * allocator owns the device memory, runtimes that forbid allocation after
 * start-up, plug-ins inside a host that manages memory itself.  They cannot
 * create an eqlin_t, but the weight gradient needs no weights, so this call
 * takes the layer shape directly.  The paper has no counterpart; it is a
 * service of this library.
 *
 * Same arguments and results as eqlin_backward_dw (T, C' = Cp, D' = Dp and
 * the dtype describe the layer; x [N, C'*T], gy [N, D'*T] device pointers of
 * that dtype; dW [D', C', T] and db [D'] float32, overwritten; db may be
 * NULL), computed by the same tensor-core kernels.  f16 and bf16 only
 * (EQLIN_ERR_UNSUPPORTED for f32).
 *
 * Scratch: a fixed 64 MiB device array inside the library, held on a device
 * until the process exits.  A shape whose per-chunk partial sums would not fit
 * returns EQLIN_ERR_UNSUPPORTED (the need is splits * (T*C'*D' + D') * 4
 * bytes, with up to one token split per SM for a single 128 x 128 channel
 * tile; e.g. p4 with C' = D' = 1024 fits, C' = D' = 2048 does not).
 * - The CUDA runtime loads the library's device code on a device lazily, so
 *   the array is reserved by the FIRST call on each device (which also looks
 *   up its device address with cudaGetSymbolAddress).  Make that first call
 *   at start-up -- before the caller's own allocator takes the device's
 *   memory, and before any stream capture.  If the device has no room for the
 *   array then, that call returns EQLIN_ERR_OOM and computes nothing; a later
 *   call tries again.
 * - Every call on a device shares the array, so calls that may overlap on
 *   the GPU (different streams, or concurrent host threads) race and give
 *   wrong results: order them on one stream.
 * - A device-side wait that runs out (only if the GPU stalls for seconds)
 *   leaves dW and db undefined; there is no handle to report it through.
 * After that first call, the call allocates nothing and frees nothing.
 */
EQLIN_API eqlin_status_t eqlin_backward_dw_noalloc(int T, int64_t Cp, int64_t Dp,
                                                   eqlin_dtype_t dtype, const void *x,
                                                   const void *gy, float *dW, float *db,
                                                   int64_t N, void *stream);

/*
 * Read and clear the handle's device-side error word.  Call after
 * synchronising the streams the handle's kernels ran on.  Returns EQLIN_OK,
 * EQLIN_ERR_TIMEOUT (a kernel's bounded wait ran out and the kernel returned
 * early: its outputs are invalid) or EQLIN_ERR_CUDA.
 */
EQLIN_API eqlin_status_t eqlin_get_error(eqlin_t h);

/*
 * Where the last error that eqlin_get_error reported (other than EQLIN_OK)
 * came from, for diagnosis: detail[0] the device status (1 = timeout),
 * detail[1] the site of the first wait that ran out, (kernel << 8) |
 * (role << 4) | barrier (kernels: 1 forward/dx, 2 dW from x and gy, 3 dW from
 * spectra), detail[2] that CTA's index | (its stage or tile counter << 12),
 * detail[3] the polls it made | (milliseconds it waited << 20).  All zero if
 * no error has been read on this handle.
 */
EQLIN_API eqlin_status_t eqlin_error_detail(eqlin_t h, uint32_t detail[4]);

/*
 * Tail split of the f16/bf16 forward and dx (off by default; enable != 0
 * turns it on, 0 off).  The tensor-core kernel gives each SM whole tiles of
 * 128 tokens in turn.  When a call's last wave of tiles would occupy at most
 * half of the SMs, and its reduction (C' for the forward, D' for dx) spans 256
 * channels or more, each of those tiles then runs as two parts of the
 * reduction on two SMs; the part that finishes first hands its FP32
 * accumulator to the other through a workspace of the handle.  That shortens
 * a call that runs alone (the EQ-ViT-B fc1 dx and fc2 forward, 198 tiles:
 * 51-54 -> 49 us), but the hand-over is extra work: where other kernels, on
 * other streams, would use the idle SMs anyway, it lowers throughput.
 *
 * Turning it on allocates, for each such pass, SMs / 2 accumulators of
 * 128 x T x tile-width floats (at most 256 KB each) and a few flags;
 * turning it off frees them.  Both synchronize the device.  While it is on,
 * two calls of the same pass on one handle must not overlap on the GPU
 * (eqlin_forward, eqlin_forward_stash and eqlin_forward_gauss are one pass;
 * eqlin_backward_dx and eqlin_backward_dx_stash the other): order them on one
 * stream.  Results do not depend on which part finishes first; they may
 * differ from the unsplit call's in the last bit (two partial sums added).
 * FP32 and dihedral handles accept the call and do not split.
 */
EQLIN_API eqlin_status_t eqlin_set_tail_split(eqlin_t h, int enable);

/*
 * Cap, in polling iterations, on every wait inside this handle's kernels
 * (0 restores the default).  A wait that reaches the cap records
 * EQLIN_ERR_TIMEOUT and its kernel returns early instead of spinning.
 */
EQLIN_API eqlin_status_t eqlin_set_wait_limit(eqlin_t h, uint32_t iterations);

/*
 * Which kernel family serves each pass of this handle, as
 * "fwd=<k> dx=<k> dw=<k>", where <k> is "tcgen05" (the tensor-core kernels)
 * or "simt" (the FP32 CUDA-core kernels).  f32 handles run tcgen05 (3xTF32)
 * in every pass when T is 1, 2 or 4 and in the forward and dx when T is 8,
 * except a forward or dx past the reduction-length limit above, and simt
 * otherwise.
 * f16/bf16 handles run tcgen05 except where the shape rules it out:
 * a forward (dx) whose K = C' (D') is not a multiple of 8 -- the row pitch of
 * that pass's weight tiles would not be a TMA stride.  For logging and tests; the string lives as long as the handle.
 */
EQLIN_API const char *eqlin_backend_name(eqlin_t h);

/*
 * Number of CUDA kernels this library has enqueued in this process, over all
 * handles (a monotonically increasing counter, for accounting).
 */
EQLIN_API uint64_t eqlin_launch_count(void);

/* Static description of a status code. */
EQLIN_API const char *eqlin_status_string(eqlin_status_t s);

/* Free the handle and its device buffers (synchronises the device first).  NULL is a no-op. */
EQLIN_API void eqlin_destroy(eqlin_t h);

#ifdef __cplusplus
}
#endif

#endif /* EQLIN_H */
