/*
 * eqlinear.h -- C ABI of the B200 (sm_100a) Flash EQ-Linear library.
 *
 * The layer (Flash EQ-Linear technical summary, gist.science/ko/paper/2607.21271,
 * "Key insight" and "Algorithmic approach") is the group-equivariant linear map
 *
 *     Y[n, d*T+s] = bias[d] + sum_{c<C} sum_{t<T} W[d][c][(t-s) mod T] * X[n, c*T+t]
 *
 * over the cyclic group of order T.  Its weight matrix is group-circulant, so the
 * library computes it exactly through a DFT over the group axis: a real DFT of
 * every length-T group vector, one real GEMM per real frequency and four per
 * complex frequency (conjugate symmetry keeps only k = 0..floor(T/2)), then the
 * inverse DFT.  For the p4 group (T = 4) the transforms use only 0, +-1 and
 * +-1/2-type coefficients and the products are six real GEMMs ("Specialisation
 * for p4").
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Every tensor is a dense row-major array in DEVICE memory, owned by the
 *    caller, in the plan's dtype (EQL_F32: float, EQL_F16: IEEE binary16),
 *    accumulation is FP32.  The library never allocates device memory after
 *    eqlinear_plan_create and never frees caller memory.
 *  - Every device pointer must be 16-byte aligned, and rows must be a whole
 *    number of 16-byte units for the tensor-core path (the dispatcher falls
 *    back to the CUDA-core path when they are not); violations of the 16-byte
 *    pointer rule return EQL_ERR_ALIGNMENT before anything is launched.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  All calls are
 *    asynchronous on it and return once the work is enqueued; only
 *    eqlinear_get_status synchronises.
 *  - The plan is bound to the CUDA device current at eqlinear_plan_create;
 *    every call must be made with that device current.
 *  - A plan is immutable after creation except for eqlinear_plan_set_kernel;
 *    it may be shared by several streams provided each concurrent
 *    eqlinear_backward_weight call has its own workspace.
 *  - Argument errors are reported synchronously and nothing is launched.
 *    Launch failures return EQL_ERR_CUDA.  Device-side failures (a bounded
 *    wait that gave up) set a sticky status word in the plan, read by
 *    eqlinear_get_status.
 */
#ifndef EQLINEAR_H_
#define EQLINEAR_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define EQL_API __attribute__((visibility("default")))
#else
#define EQL_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct eqlinear_plan_s* eqlinear_plan_t;

typedef enum {
  EQL_OK = 0,
  EQL_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, bad enum      */
  EQL_ERR_UNSUPPORTED = 2, /* T or dtype with no instantiated kernel         */
  EQL_ERR_ALIGNMENT = 3,   /* device pointer not 16-byte aligned             */
  EQL_ERR_WORKSPACE = 4,   /* workspace missing or smaller than required     */
  EQL_ERR_CUDA = 5,        /* CUDA runtime error (launch, allocation, ...)   */
  EQL_ERR_TIMEOUT = 6      /* a device-side bounded wait gave up             */
} eqlinear_status_t;

typedef enum { EQL_F32 = 0, EQL_F16 = 1 } eqlinear_dtype_t;

/* Kernel family selection (testing and measurement; AUTO is the default). */
typedef enum {
  EQL_KERNEL_AUTO = 0,   /* tensor cores where the shape allows, else CUDA cores */
  EQL_KERNEL_SIMT = 1,   /* CUDA-core FP32 FMA kernels, any supported shape      */
  EQL_KERNEL_TCGEN05 = 2 /* tcgen05/TMEM tensor-core kernels; calls whose shape
                            they cannot take return EQL_ERR_UNSUPPORTED         */
} eqlinear_kernel_t;

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
EQL_API int eqlinear_version(void);

/* Human-readable name of a status code (static storage; never NULL). */
EQL_API const char* eqlinear_status_string(eqlinear_status_t status);

/*
 * Create a plan for group order T, C input channels and D output channels per
 * group element (input width C*T features, output width D*T), in `dtype`.
 * Supported T: 1..8.  The plan owns host metadata (DFT twiddles computed in
 * double on the host, rounded once to float) and a 4-byte device status word
 * allocated on the current device.  *out is written only on EQL_OK.
 */
EQL_API eqlinear_status_t eqlinear_plan_create(int T, int C, int D, eqlinear_dtype_t dtype,
                                       eqlinear_plan_t* out);

/*
 * A plan for the layer over the dihedral group D4 (p4m: quarter turns and a
 * mirror; the pages name reflection groups as the natural generalisation,
 * "Limitations and future work", without a formula).  Reading: the same
 * group-circulant weight structure with the group law in place of the cyclic
 * shift,
 *   Y[n, d*8+g] = bias[d] + sum_{c,h} W[d][c][g^-1 h] * X[n, c*8+h],
 * group element g = a + 4b for r^a m^b (m r m = r^-1).  D4 is not abelian: its
 * Fourier transform has four characters and one 2 x 2 representation (entries
 * 0, +-1, so the transforms are adds), and the per-frequency products are four
 * real GEMMs plus a 2 x 2 block product (eight), 12 real products per (row,
 * in-channel, out-channel) against the dense 64.
 * Supported: FP16, C and D multiples of 16:
 *   forward: eqlinear_forward and eqlinear_forward_act (fused one-CTA kernel), or
 *     eqlinear_group_dft + eqlinear_forward_tiled (the Fourier planes as a pass,
 *     then SM-pair tensor cores);
 *   dX: eqlinear_group_dft of dY + eqlinear_backward_input_tiled (the D4 layer of
 *     dY with W'[c][d][v] = W[d][c][v^-1]); eqlinear_backward_input returns
 *     EQL_ERR_UNSUPPORTED;
 *   dW and dbias: eqlinear_backward_weight(_f32) on CUDA cores (workspace from
 *     eqlinear_backward_weight_workspace_bytes; EQL_ERR_UNSUPPORTED when the plan
 *     is forced to the tensor cores).
 * For other plans of this kind eqlinear_prepared_weight_bytes is 0 and every
 * call returns EQL_ERR_UNSUPPORTED.  W [D][C][8], X [N][C*8], Y [N][D*8].  Free
 * with eqlinear_plan_destroy.
 */
EQL_API eqlinear_status_t eqlinear_plan_create_dihedral4(int C, int D, eqlinear_dtype_t dtype,
                                                        eqlinear_plan_t* out);

/* Free the plan and its status word.  NULL is ignored.  The caller must make
 * sure no call using the plan is still running on any stream. */
EQL_API void eqlinear_plan_destroy(eqlinear_plan_t plan);

/* Choose the kernel family used by later calls (not thread-safe with respect
 * to calls running concurrently on the same plan). */
EQL_API eqlinear_status_t eqlinear_plan_set_kernel(eqlinear_plan_t plan, eqlinear_kernel_t which);

/* Name of the kernel eqlinear_forward would launch for N rows with the
 * current selection ("simt", "tcgen05", or "unsupported"). */
EQL_API const char* eqlinear_forward_kernel_name(eqlinear_plan_t plan, int64_t N);

/* Same for eqlinear_backward_weight. */
EQL_API const char* eqlinear_backward_weight_kernel_name(eqlinear_plan_t plan, int64_t N);

/*
 * Size in bytes of the prepared (frequency-domain) weights W_hat.
 * W_hat layout, plane by plane, each plane a dense matrix in the plan dtype:
 *   forward planes  [P][D][C]  then  adjoint planes [P][C][D],  P = T + n_cplx,
 * where n_cplx = number of complex frequencies (T-1)/2 for odd T, T/2-1 for
 * even T.  Plane order inside each block: real frequency 0; real frequency T/2
 * (even T); Re and Im of each complex frequency k = 1..n_cplx; then -Im of each
 * complex frequency.  Forward planes hold conj(DFT(W)) (the correlation form of
 * the convolution theorem), adjoint planes hold DFT(W) transposed, used for dX.
 * Every plane is stored times 1/Tp, Tp the smallest power of two >= T (exact):
 * a DFT coefficient is at most T max|W| in magnitude, so a stored value never
 * exceeds max|W| and no finite FP16 weight overflows its plane.
 * For FP16 plans with T = 4 or 8 and C, D multiples of 16 two more blocks
 * follow: the forward and adjoint planes re-arranged as the tensor-core
 * kernel's operand tiles (one contiguous blob per out-channel tile and K stage:
 * 128 x 32 channels at T = 4, 64 x 16 at T = 8, in the kernel's swizzled
 * shared-memory order, the same values), so each pipeline stage is one copy.
 * At T = 4 two more follow: the same planes as the two-SM spectral kernel's
 * stages (forward, then adjoint; per 128 out-channels and 32 input channels,
 * each SM's 64 out-channels of the four planes X0, X2, Re, Im: 2 x 16 KB).
 */
EQL_API size_t eqlinear_prepared_weight_bytes(eqlinear_plan_t plan);

/*
 * One-time frequency-domain transform of the weights ("Implementation": the
 * layer replaces a naive EQ-Linear with no retraining; only the parameters are
 * re-expressed).  W is [D][C][T] in the plan dtype; W_hat receives
 * eqlinear_prepared_weight_bytes(plan) bytes.  The DFT runs in FP32 and is
 * rounded once to the plan dtype.
 */
EQL_API eqlinear_status_t eqlinear_prepare_weights(eqlinear_plan_t plan, const void* W, void* W_hat,
                                           void* stream);

/*
 * Forward pass ("Algorithmic approach" items 1-3; "Implementation": fused
 * dataflow with no intermediate global-memory writes).
 *   X     [N][C*T]  input, feature index c*T+t
 *   W_hat prepared weights of this plan
 *   bias  [D] in the plan dtype, or NULL for no bias
 *   Y     [N][D*T]  output, feature index d*T+s (must not overlap X)
 * N = 0 is a no-op returning EQL_OK.
 */
EQL_API eqlinear_status_t eqlinear_forward(eqlinear_plan_t plan, const void* X, int64_t N,
                                   const void* W_hat, const void* bias, void* Y, void* stream);

/* Output activation applied by eqlinear_forward_act. */
typedef enum {
  EQL_ACT_NONE = 0,
  EQL_ACT_GELU = 1  /* GELU(y) = y * Phi(y) = 0.5 y (1 + erf(y / sqrt 2)), exact erf form
                       (erf within 3e-7, Abramowitz & Stegun 7.1.28) */
} eqlinear_act_t;

/*
 * Forward pass with an elementwise activation fused into the epilogue, the
 * first half of an EQ-MLP block (the pages' network-level Flash EQ-ViT/Swin
 * models stack EQ-Linear layers in MLP blocks, "Results / network level"):
 *   Y[n, d*T+s] = act(bias[d] + sum_{c,t} W[d][c][(t-s) mod T] * X[n, c*T+t])
 * A pointwise function of each output feature commutes with the cyclic shift
 * of the group axis, so the block stays equivariant.  The activation runs in
 * FP32 on the accumulated value and is followed by the single rounding to the
 * plan dtype.  Same arguments, layouts and errors as eqlinear_forward, plus
 * EQL_ERR_INVALID_ARG for an unknown act.  eqlinear_forward is this call with
 * EQL_ACT_NONE.
 */
EQL_API eqlinear_status_t eqlinear_forward_act(eqlinear_plan_t plan, const void* X, int64_t N,
                                               const void* W_hat, const void* bias,
                                               eqlinear_act_t act, void* Y, void* stream);

/*
 * Two-layer EQ-MLP block with the intermediate kept in the frequency domain
 * ("Algorithmic approach": the layer is a per-frequency product between a
 * forward and an inverse group DFT; when one EQ-Linear feeds another, the
 * second layer's forward DFT can be taken by the first layer's epilogue).
 *
 * eqlinear_forward_to_spectral writes, instead of Y, the group DFT of
 * act(Y) as four FP16 planes Xhat[4][N][D], each value times 1/4 (plane 0: sum
 * over s, 1: alternating sum, 2: y0 - y2, 3: y3 - y1, then / 4; FP32 arithmetic,
 * one rounding; the factor keeps every plane within max|act(Y)|, so no finite
 * FP16 activation overflows), which is the input a following p4 layer
 * multiplies directly.  eqlinear_forward_from_spectral
 * is the forward of a layer whose input arrives as such planes Xhat[4][N][C]
 * (Y [N][D*T], optional bias and act as in eqlinear_forward_act).  Chaining the
 * two equals eqlinear_forward_act followed by eqlinear_forward up to rounding.
 *
 * Only FP16 plans with T = 4 and C, D multiples of 16 (the tensor-core path);
 * others return EQL_ERR_UNSUPPORTED, as does a plan forced to the CUDA-core
 * kernels.  Buffers: eqlinear_spectral_bytes(plan, N) = 4 * N * D * 2 bytes for
 * the output of eqlinear_forward_to_spectral (the same size as Y).
 */
EQL_API size_t eqlinear_spectral_bytes(eqlinear_plan_t plan, int64_t N);
EQL_API eqlinear_status_t eqlinear_forward_to_spectral(eqlinear_plan_t plan, const void* X,
                                                       int64_t N, const void* W_hat,
                                                       const void* bias, eqlinear_act_t act,
                                                       void* Xhat_next, void* stream);
EQL_API eqlinear_status_t eqlinear_forward_from_spectral(eqlinear_plan_t plan, const void* Xhat,
                                                         int64_t N, const void* W_hat,
                                                         const void* bias, eqlinear_act_t act,
                                                         void* Y, void* stream);

/*
 * The layer in the frequency domain, as separate steps ("Algorithmic approach"
 * items 1-3: forward group DFT, per-frequency products, inverse DFT): the
 * input's DFT is formed once by eqlinear_group_dft and kept in HBM as "tiled
 * planes"; the products and the inverse then run in a kernel that copies those
 * planes straight into the tensor cores' operand layout, two SMs per 256-row
 * tile (tcgen05 cta_group::2), and can write its output as the next layer's
 * tiled planes, so a chain of p4 layers stays in the frequency domain.
 *
 * Tiled planes of a [N][c*4] array: the four planes of eqlinear_forward_to_spectral
 * (X0, X2, Xr, Xi, each times 1/4) stored as the kernel's shared-memory image.
 * Rows are padded to Np = N rounded up to a multiple of 128; element (plane p,
 * row n, channel j) is the FP16 value at byte offset
 *   ((p * (c / 16) + j / 16) * Np + n) * 32 + 16 * (((j % 16) / 8) ^ ((n / 4) % 2))
 *   + 2 * (j % 8).
 * eqlinear_tiled_spectrum_bytes(plan, N, c) = 4 * Np * c * 2 bytes.
 *
 * eqlinear_group_dft: X [N][channels*4] -> tiled planes (rows N..Np-1 zero);
 *   channels is the plan's C (a layer input) or D (an upstream gradient).
 * eqlinear_forward_tiled: tiled planes of X [N][C*4] -> Y [N][D*4], bias and
 *   act as in eqlinear_forward_act.
 * eqlinear_forward_tiled_next: the same, written as the tiled planes of act(Y)
 *   (padding rows N..Np-1 hold values of no meaning).
 * eqlinear_backward_input_tiled: tiled planes of dY [N][D*4] -> dX [N][C*4].
 * Each equals eqlinear_forward_act / eqlinear_backward_input up to the rounding
 * of the planes.  Plans taken (else EQL_ERR_UNSUPPORTED; never a plan forced to
 * the CUDA cores):
 *   - p4 FP16, C and D multiples of 16: as above.
 *   - FP16 with T = 8, cyclic or D4 (eqlinear_plan_create_dihedral4), C and D
 *     multiples of 16. Eight planes, each times 1/8: cyclic V0, V4, Re/Im of
 *     V1, V2, V3 of the DFT; D4 the four characters (chi(r), chi(m)) = (+,+),
 *     (+,-), (-,+), (-,-), then the 2 x 2 representation's entries
 *     X[i][j] = sum_g x_g rho(g)_ij at plane 4 + 2i + j, with rho(r) =
 *     [[0,-1],[1,0]] and rho(m) = diag(1,-1). The same tiled layout with p < 8;
 *     tiled_spectrum_bytes = 8 * Np * c * 2. The _next form writes the planes of
 *     act(Y) rounded to FP16, as eqlinear_group_dft of eqlinear_forward_tiled's
 *     output (bitwise for D4; cyclic: up to one rounding of Y where the
 *     sqrt(2)/2 twiddle products round differently), with rows N..Np-1 zero.
 *   - p4 FP32, C and D multiples of 8 (3xTF32 on the tensor cores). Eight
 *     planes: the TF32 values hi = tf32(v) of X0, X2, Xr, Xi, then the
 *     residuals lo = tf32(v - hi). 8 FP32 channels per 32-byte row: element
 *     (q, n, j) at ((q * (c / 8) + j / 8) * Np + n) * 32 +
 *     16 * (((j % 8) / 4) ^ ((n / 4) % 2)) + 4 * (j % 4);
 *     tiled_spectrum_bytes = 8 * Np * c * 4. No _next form. The result is within
 *     the FP32 bar (products hi*hi + lo*hi + hi*lo, FP32 accumulation).
 * Channels not C or D: EQL_ERR_INVALID_ARG. All pointers must be 16-byte
 * aligned, and outputs must not overlap inputs. N = 0 is a no-op.
 */
EQL_API size_t eqlinear_tiled_spectrum_bytes(eqlinear_plan_t plan, int64_t N, int channels);
EQL_API eqlinear_status_t eqlinear_group_dft(eqlinear_plan_t plan, const void* X, int64_t N,
                                             int channels, void* Xt, void* stream);
EQL_API eqlinear_status_t eqlinear_forward_tiled(eqlinear_plan_t plan, const void* Xt,
                                                 int64_t N, const void* W_hat, const void* bias,
                                                 eqlinear_act_t act, void* Y, void* stream);
EQL_API eqlinear_status_t eqlinear_forward_tiled_next(eqlinear_plan_t plan, const void* Xt,
                                                      int64_t N, const void* W_hat,
                                                      const void* bias, eqlinear_act_t act,
                                                      void* Yt_next, void* stream);
EQL_API eqlinear_status_t eqlinear_backward_input_tiled(eqlinear_plan_t plan, const void* dYt,
                                                        int64_t N, const void* W_hat, void* dX,
                                                        void* stream);

/*
 * The weight gradient from tiled planes ("Implementation", bullet 1: the backward
 * is the same per-frequency product, transposed, summed over rows):
 * eqlinear_backward_weight_tiled(plan, Xt, dYt, N, dW, dbias, ...) gives
 * eqlinear_backward_weight of X [N][C*4] and dY [N][D*4] from their tiled
 * planes Xt and dYt (eqlinear_group_dft of each), so one transform of X serves
 * the forward and dW, and one of dY serves dX and dW.  dW [D][C][4], dbias [D]
 * (may be NULL), workspace as eqlinear_backward_weight
 * (eqlinear_backward_weight_workspace_bytes); _f32 writes FP32 dW and dbias as
 * eqlinear_backward_weight_f32.  dW's operands are the planes' FP16 values;
 * dbias sums dYt's plane 0 (rounded to FP16) times 4.  The padding rows of the
 * planes must be zero, as eqlinear_group_dft leaves them (the planes of
 * eqlinear_forward_tiled_next do not qualify).
 *
 * p4 FP16 plans with C and D multiples of 16, not forced to the CUDA cores;
 * otherwise EQL_ERR_UNSUPPORTED.  Pointers 16-byte aligned; N = 0 writes zeros.
 */
EQL_API eqlinear_status_t eqlinear_backward_weight_tiled(eqlinear_plan_t plan, const void* Xt,
                                                         const void* dYt, int64_t N, void* dW,
                                                         void* dbias, void* workspace,
                                                         size_t workspace_bytes, void* stream);
EQL_API eqlinear_status_t eqlinear_backward_weight_tiled_f32(eqlinear_plan_t plan,
                                                             const void* Xt, const void* dYt,
                                                             int64_t N, float* dW, float* dbias,
                                                             void* workspace,
                                                             size_t workspace_bytes,
                                                             void* stream);

/*
 * Two chained layers on tiled planes in one launch (the MLP pair of a Flash
 * EQ-ViT block, kept in the frequency domain between the layers):
 *   Ht = tiled planes of act1(first(X))   (as eqlinear_forward_tiled_next)
 *   Y  = second(H)                        (as eqlinear_forward_tiled), Y [N][D2*4]
 * from Xt, the tiled planes of X [N][C0*4] (eqlinear_group_dft).  Results are
 * bitwise those of the two separate calls; the tiles of both layers share one
 * queue, so neither layer's last partial wave leaves SMs idle.  Ht is the
 * caller's buffer (eqlinear_tiled_spectrum_bytes(first, N, first's D)).
 * workspace: eqlinear_chain_tiled_workspace_bytes(first, second, N) bytes of
 * int32 counters that must be zero before the first call; each call leaves
 * them zero (after a timeout reported by eqlinear_get_status, zero them again).
 * Plans: p4 FP16 with C, D multiples of 16, second's C = first's D, same device,
 * not forced to the CUDA cores (else EQL_ERR_UNSUPPORTED / EQL_ERR_INVALID_ARG);
 * EQL_ERR_WORKSPACE for a short workspace; pointers 16-byte aligned.
 */
EQL_API size_t eqlinear_chain_tiled_workspace_bytes(eqlinear_plan_t first, eqlinear_plan_t second,
                                                    int64_t N);
EQL_API eqlinear_status_t eqlinear_forward_chain_tiled(eqlinear_plan_t first,
                                                       eqlinear_plan_t second, const void* Xt,
                                                       int64_t N, const void* W1_hat,
                                                       const void* bias1, eqlinear_act_t act1,
                                                       const void* W2_hat, const void* bias2,
                                                       void* Ht, void* Y, void* workspace,
                                                       size_t workspace_bytes, void* stream);

/*
 * Two chained layers in one launch (the MLP pair of a Flash EQ-ViT block):
 *   H = act1(layer first (X))     H: [N][D1*T], or with spectral_intermediate = 1
 *                                    the planes [4][N][D1] of
 *                                    eqlinear_forward_to_spectral
 *   Y = layer second (H)          Y: [N][D2*T], no activation
 * first: C0 -> D1 channels, second: D1 -> D2 (second's C must equal first's D).
 * The results, H included, are bitwise those of the two separate calls
 * (eqlinear_forward_act then eqlinear_forward, or eqlinear_forward_to_spectral
 * then eqlinear_forward_from_spectral): every tile runs the same arithmetic.
 * What changes is the schedule: both layers' tiles form one queue that the
 * GPU's CTAs take from as they become free, and a second-layer tile starts as
 * soon as the first-layer tiles of its 128 rows are stored, so neither layer's
 * last partial wave leaves SMs idle.
 *
 * Both plans: T = 4, FP16, C and D multiples of 16, not forced to the CUDA
 * cores, on the same device; otherwise EQL_ERR_UNSUPPORTED (EQL_ERR_INVALID_ARG
 * for widths that do not chain).  W1_hat, W2_hat: the plans' prepared weights;
 * bias1, bias2: [D1], [D2] or NULL; act1: EQL_ACT_NONE or EQL_ACT_GELU.  All
 * pointers 16-byte aligned; H must not overlap X or Y.  workspace: at least
 * eqlinear_chain_workspace_bytes(first, second, N) bytes of device memory
 * (int32 counters: the task queue and one per 128 rows), owned by the caller,
 * ZERO-FILLED before its first use (e.g. cudaMemset) and not shared by calls
 * that may run at the same time.  Every call that completes leaves the counters
 * zero again, so the same workspace serves the next call (of any N up to its
 * size) with no clearing.  After a call that reports EQL_ERR_TIMEOUT through
 * eqlinear_get_status(first, ...), zero the workspace again before reusing it.
 * Asynchronous on `stream`.  N = 0 does nothing.
 */
EQL_API size_t eqlinear_chain_workspace_bytes(eqlinear_plan_t first, eqlinear_plan_t second,
                                              int64_t N);
EQL_API eqlinear_status_t eqlinear_forward_chain(eqlinear_plan_t first, eqlinear_plan_t second,
                                                 const void* X, int64_t N, const void* W1_hat,
                                                 const void* bias1, eqlinear_act_t act1,
                                                 const void* W2_hat, const void* bias2,
                                                 int spectral_intermediate, void* H, void* Y,
                                                 void* workspace, size_t workspace_bytes,
                                                 void* stream);

/*
 * Group-circulant convolution.  The pages name equivariant convolution as the
 * natural next operator for the per-frequency method ("Limitations and future
 * work") and give no formula; this library's reading is the layer's
 * group-circulant channel mixing at every tap of a KH x KW kernel, stride 1,
 * zero padding:
 *   Y[n][oy][ox][d*T+s] = act(bias[d] + sum_{i<KH, j<KW} sum_{c,t}
 *       Wc[i][j][d][c][(t-s) mod T] * X[n][oy+i-pad_h][ox+j-pad_w][c*T+t])
 * with X zero outside the H x W image; Ho = H + 2 pad_h - KH + 1,
 * Wo = W + 2 pad_w - KW + 1.  Like the layer it commutes with the cyclic shift
 * of every pixel's group axis, and with translations away from the border.
 *
 * Plans: T = 4, FP16, C and D multiples of 16, not forced to the CUDA cores
 * (otherwise EQL_ERR_UNSUPPORTED).  KH, KW in 1..15, 0 <= pad < kernel size.
 *   eqlinear_conv_prepared_weight_bytes(plan, KH, KW): size of Wc_hat.
 *   eqlinear_conv_prepare_weights: Wc [KH][KW][D][C][T] (tap-major; each tap a
 *     contiguous [D][C][T] block) -> Wc_hat, once per weight update (forward
 *     tiles, each tap's planes, then the adjoint tiles of the flipped taps that
 *     eqlinear_conv_backward_input reads).
 *   eqlinear_conv_workspace_bytes(plan, N, H, W): scratch of eqlinear_conv_forward
 *     (the group DFT of X times 1/4 as FP16 planes, 4 * N * H * W * C * 2 bytes).
 *   eqlinear_conv_forward: X [N][H][W][C*T] (feature index c*T+t, pixels
 *     row-major), Y [N][Ho][Wo][D*T], bias [D] or NULL, act as in
 *     eqlinear_forward_act.  All pointers 16-byte aligned; the caller owns every
 *     buffer.  Asynchronous on `stream`.  N = 0 does nothing.
 * A 1 x 1 kernel with no padding computes exactly eqlinear_forward on the N*H*W
 * pixels.
 */
EQL_API size_t eqlinear_conv_prepared_weight_bytes(eqlinear_plan_t plan, int KH, int KW);
EQL_API eqlinear_status_t eqlinear_conv_prepare_weights(eqlinear_plan_t plan, int KH, int KW,
                                                        const void* Wc, void* Wc_hat,
                                                        void* stream);
EQL_API size_t eqlinear_conv_workspace_bytes(eqlinear_plan_t plan, int64_t N, int H, int W);
EQL_API eqlinear_status_t eqlinear_conv_forward(eqlinear_plan_t plan, const void* X, int64_t N,
                                                int H, int W, int KH, int KW, int pad_h,
                                                int pad_w, const void* Wc_hat, const void* bias,
                                                eqlinear_act_t act, void* Y, void* workspace,
                                                size_t workspace_bytes, void* stream);

/*
 * Gradients of the group-circulant convolution (the definition above,
 * differentiated; "Implementation": forward and backward passes):
 *   dX[n][y][x][c*T+t] = sum_{i,j,d,s} Wc[i][j][d][c][(t-s) mod T]
 *                                      * dY[n][y-i+pad_h][x-j+pad_w][d*T+s]
 *   dWc[i][j][d][c][u] = sum_{n,oy,ox,s} dY[n][oy][ox][d*T+s]
 *                                       * X[n][oy+i-pad_h][ox+j-pad_w][c*T + (s+u) mod T]
 *   dbias[d]           = sum_{n,oy,ox,s} dY[n][oy][ox][d*T+s]
 * (terms whose pixel falls outside the image are zero).  dY [N][Ho][Wo][D*T].
 *   eqlinear_conv_backward_input: dX [N][H][W][C*T] is the convolution of dY with
 *     the spatially flipped kernel of adjoint taps and padding (KH-1-pad_h,
 *     KW-1-pad_w); it runs the forward's tensor-core kernel with the adjoint
 *     tiles that eqlinear_conv_prepare_weights also writes into Wc_hat.
 *   eqlinear_conv_backward_weight: dWc [KH][KW][D][C][T] and dbias [D] (or NULL)
 *     in the plan dtype. X and dY are copied once into the workspace on the
 *     padded pixel grid ((H + 2 pad_h) x (W + 2 pad_w) per image: X shifted by
 *     the padding, dY at the top left, zeros elsewhere); tap (i, j) is then the
 *     layer's weight gradient between dY's padded rows and X's padded rows
 *     offset by i (W + 2 pad_w) + j. With C and D multiples of 64 (and a plan
 *     not forced to the CUDA cores), the padded rows' group spectra are formed
 *     once and one tensor-core launch takes all taps; otherwise each tap runs
 *     the layer's weight-gradient kernel.
 *   eqlinear_conv_backward_workspace_bytes(plan, N, H, W, KH, KW, pad_h, pad_w):
 *     scratch of both calls.
 * Plans and limits as for eqlinear_conv_forward; all pointers 16-byte aligned;
 * EQL_ERR_WORKSPACE for a short workspace; N = 0 does nothing.
 */
EQL_API size_t eqlinear_conv_backward_workspace_bytes(eqlinear_plan_t plan, int64_t N, int H,
                                                      int W, int KH, int KW, int pad_h,
                                                      int pad_w);
EQL_API eqlinear_status_t eqlinear_conv_backward_input(eqlinear_plan_t plan, const void* dY,
                                                       int64_t N, int H, int W, int KH, int KW,
                                                       int pad_h, int pad_w, const void* Wc_hat,
                                                       void* dX, void* workspace,
                                                       size_t workspace_bytes, void* stream);
EQL_API eqlinear_status_t eqlinear_conv_backward_weight(eqlinear_plan_t plan, const void* X,
                                                        int64_t N, int H, int W, const void* dY,
                                                        int KH, int KW, int pad_h, int pad_w,
                                                        void* dWc, void* dbias, void* workspace,
                                                        size_t workspace_bytes, void* stream);

/*
 * Gradient with respect to the input ("Implementation": backward pass):
 *   dX[n, c*T+t] = sum_{d,s} dY[n, d*T+s] * W[d][c][(t-s) mod T]
 * which is the same group-circulant product with the transposed weights and the
 * opposite conjugation.  dY [N][D*T], dX [N][C*T] (must not overlap).
 */
EQL_API eqlinear_status_t eqlinear_backward_input(eqlinear_plan_t plan, const void* dY, int64_t N,
                                          const void* W_hat, void* dX, void* stream);

/* Workspace bytes eqlinear_backward_weight needs for N rows (FP32 partial
 * spectra of the split reduction over rows; large enough for either kernel). */
EQL_API size_t eqlinear_backward_weight_workspace_bytes(eqlinear_plan_t plan, int64_t N);

/*
 * Gradient with respect to the weights and the bias:
 *   dW[d][c][u] = sum_{n,s} dY[n, d*T+s] * X[n, c*T + (s+u) mod T]
 *   dbias[d]    = sum_{n,s} dY[n, d*T+s]
 * computed per frequency as a reduction over the N rows (FP32, fixed order, so
 * results are bitwise reproducible for a given N), then one inverse DFT.  FP16
 * plans with T = 4, C and D multiples of 16 and 16-byte aligned X and dY run on
 * the tensor cores (the group DFTs of X and dY rounded once to FP16, FP32
 * accumulation); other plans on CUDA cores in FP32.
 *   X [N][C*T], dY [N][D*T], dW [D][C][T] (plan dtype, overwritten),
 *   dbias [D] or NULL, workspace >= eqlinear_backward_weight_workspace_bytes.
 * N = 0 writes zeros to dW and dbias.
 */
EQL_API eqlinear_status_t eqlinear_backward_weight(eqlinear_plan_t plan, const void* X, const void* dY,
                                           int64_t N, void* dW, void* dbias, void* workspace,
                                           size_t workspace_bytes, void* stream);

/*
 * Data-parallel form of the weight gradient.  dW and dbias are sums over rows,
 * so a batch split by rows across ranks has dW = the sum over ranks of each
 * rank's dW.  To add the ranks' contributions in FP32 (one rounding to the plan
 * dtype at the end, as for a single rank), each rank calls
 * eqlinear_backward_weight_f32 on its rows, the ranks sum the FP32 results
 * (an all-reduce), and eqlinear_cast_from_f32 rounds the sum.  The page
 * describing the layer trains on one device and has no counterpart to these
 * two calls.
 *
 * eqlinear_backward_weight_f32: the same computation, kernels and arguments as
 * eqlinear_backward_weight, except that dW [D][C][T] and dbias [D] (or NULL)
 * are FP32 whatever the plan dtype: the fixed-order FP32 sums before the final
 * cast.  Rounding that output to the plan dtype gives exactly what
 * eqlinear_backward_weight writes.  dW must be 16-byte aligned.
 */
EQL_API eqlinear_status_t eqlinear_backward_weight_f32(eqlinear_plan_t plan, const void* X,
                                                       const void* dY, int64_t N, float* dW,
                                                       float* dbias, void* workspace,
                                                       size_t workspace_bytes, void* stream);

/*
 * Training with saved input spectra.  The weight gradient is a sum over rows
 * of per-frequency products of the group DFTs of X and dY ("Algorithmic
 * approach": the backward pass reuses the per-frequency structure); the
 * forward and the input-gradient kernels already form exactly those DFTs as
 * their tensor-core operands.  These calls keep them, so the weight gradient
 * multiplies them directly and runs no transform of its own:
 *
 * eqlinear_forward_save_spectrum: eqlinear_forward_act (Y bitwise the same),
 *   and also Xhat [4][N][C], the group DFT of X times 1/4 (plane 0:
 *   (x0+x1+x2+x3)/4, 1: (x0-x1+x2-x3)/4, 2: (x0-x2)/4, 3: (x3-x1)/4; FP32
 *   arithmetic, one rounding to FP16; no finite FP16 input overflows), the
 *   planes order and scale of eqlinear_forward_to_spectral.
 * eqlinear_backward_input_save_spectrum: eqlinear_backward_input (dX bitwise
 *   the same), and also dYhat [4][N][D], the group DFT of dY in that order.
 * eqlinear_backward_weight_from_spectra (and _f32, as eqlinear_backward_weight
 *   _f32): eqlinear_backward_weight from Xhat and dYhat instead of X and dY,
 *   with the same workspace (eqlinear_backward_weight_workspace_bytes).  dW's
 *   operands are the same FP16 values the transforming kernel forms; dbias sums
 *   dYhat's plane 0 (already rounded to FP16) times 4 instead of the FP32 sums.
 *   A layer whose input arrives as the planes of eqlinear_forward_to_spectral
 *   may pass them as its Xhat.
 *
 * Tensor cores only: FP16 plans with T = 4 and C, D multiples of 16 (the save
 * calls) or of 64 (the weight gradient), not forced to the CUDA cores;
 * otherwise EQL_ERR_UNSUPPORTED.  Xhat takes 4 * N * C * 2 bytes (as X),
 * dYhat 4 * N * D * 2 (as dY); all pointers 16-byte aligned; a spectrum must
 * not overlap the call's other buffers.  N = 0: the save calls do nothing and
 * the weight gradient writes zeros.
 */
EQL_API eqlinear_status_t eqlinear_forward_save_spectrum(eqlinear_plan_t plan, const void* X,
                                                         int64_t N, const void* W_hat,
                                                         const void* bias, eqlinear_act_t act,
                                                         void* Y, void* Xhat, void* stream);
EQL_API eqlinear_status_t eqlinear_backward_input_save_spectrum(eqlinear_plan_t plan,
                                                                const void* dY, int64_t N,
                                                                const void* W_hat, void* dX,
                                                                void* dYhat, void* stream);
EQL_API eqlinear_status_t eqlinear_backward_weight_from_spectra(eqlinear_plan_t plan,
                                                                const void* Xhat,
                                                                const void* dYhat, int64_t N,
                                                                void* dW, void* dbias,
                                                                void* workspace,
                                                                size_t workspace_bytes,
                                                                void* stream);
EQL_API eqlinear_status_t eqlinear_backward_weight_from_spectra_f32(
    eqlinear_plan_t plan, const void* Xhat, const void* dYhat, int64_t N, float* dW, float* dbias,
    void* workspace, size_t workspace_bytes, void* stream);

/*
 * dst[i] = src[i] rounded to nearest-even in the plan dtype, for i < count
 * (a copy for FP32 plans).  src: count FP32 values on the plan's device; dst:
 * count values of the plan dtype; the two must not overlap (an FP32 plan may
 * pass dst == src, which does nothing).  Asynchronous on `stream`.
 */
EQL_API eqlinear_status_t eqlinear_cast_from_f32(eqlinear_plan_t plan, const float* src,
                                                 int64_t count, void* dst, void* stream);

/*
 * Weight gradient for callers that cannot allocate device memory.  The page
 * describing the layer has no counterpart to this call; it exists for users of
 * this library whose device memory is all owned by another allocator or fixed
 * at start-up, or who must not call cudaMalloc/cudaFree (those calls can
 * synchronise the whole device) on a latency-critical path.
 *
 * Computes what eqlinear_backward_weight computes (same arguments minus the
 * workspace), always with the CUDA-core kernels (wgrad_simt + finalize), and
 * keeps the FP32 partial spectra of their split reduction over rows in a
 * scratch array that the library reserves statically: 16 MiB (4,194,304
 * floats) per GPU on which the library is loaded, held until the process exits.
 *   - Kernels: for FP16 plans with T = 4 the workspace entry runs the tensor
 *     cores, so the two can differ in rounding (both within the FP16 accuracy
 *     target) and in speed; a plan forced to EQL_KERNEL_TCGEN05 is rejected
 *     with EQL_ERR_UNSUPPORTED.
 *   - Size limit: one row split needs T*C*D + D floats; plans above 4,194,304
 *     floats are rejected with EQL_ERR_WORKSPACE before anything is launched.
 *     When the usual number of splits does not fit, fewer splits are used (at
 *     T = 4, C = 320, D = 1280 only 2 fit, so the row reduction runs on fewer,
 *     longer CTAs and is several times slower than the workspace entry).
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 *   - The first call in each CUDA context looks up the scratch array's device
 *     address (cudaGetSymbolAddress) in that context and remembers it; make that
 *     first call before any stream capture.
 *   - Every call on a GPU shares the one scratch array and leaves its contents
 *     behind; each call writes every scratch element before reading it, so no
 *     clearing is needed, but calls whose executions overlap on the GPU (other
 *     streams, other plans, other host threads) race on it: serialise them.
 */
EQL_API eqlinear_status_t eqlinear_backward_weight_noalloc(eqlinear_plan_t plan, const void* X,
                                                           const void* dY, int64_t N, void* dW,
                                                           void* dbias, void* stream);

/*
 * Synchronise `stream`, then read and clear the plan's device status word.
 * Returns EQL_OK, EQL_ERR_TIMEOUT if a kernel's bounded wait gave up since the
 * last call, or EQL_ERR_CUDA if the stream reports an error.
 */
EQL_API eqlinear_status_t eqlinear_get_status(eqlinear_plan_t plan, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* EQLINEAR_H_ */
