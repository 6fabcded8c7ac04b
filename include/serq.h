/*
 * libserq -- SERQ quantized linear layer for NVIDIA B200 (sm_100a).
 *
 *   Y = X^_q W^_q + X~_{s,q} Q(R)
 *
 * SERQ ("Saliency-Aware Low-Rank Error Reconstruction for LLM Quantization";
 * papernotes.org ICLR 2026 notes, core idea and key designs 1-3; gist.science
 * technical summaries, section 2) replaces a two-factor low-rank error
 * correction with one r x d_out compensator R on the r most salient rows of
 * the smoothed, permuted weight.  At inference the layer is a per-token 4-bit
 * (W4A4) or 8-bit (W4A8) activation quantizer followed by one integer GEMM
 * that accumulates the main product and the residual product separately.
 *
 * Conventions for every entry point
 *  - Return a serq_status.  Arguments are checked on the host before any
 *    launch; a rejected call launches nothing and leaves outputs untouched.
 *    serq_last_error_string() gives a human-readable reason (per host thread).
 *  - "device" pointers are CUDA global-memory pointers on the current device;
 *    "host" pointers are ordinary CPU memory.  The caller owns every buffer it
 *    passes; a serq_layer owns the device buffers it allocated.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Runtime calls only enqueue work on it; they never synchronise
 *    it.  serq_prepare* and the serq_layer_get_* copies are synchronous.
 *  - Matrices are row-major.  K = d_in, N = d_out, M = tokens, r = rank.
 *    K and N must be multiples of 32; 0 <= r <= K.
 *  - Packed INT4 (activations, weights, compensator): two's-complement
 *    nibbles; every run of 32 consecutive codes of a row is 16 bytes, byte j
 *    holding code j of the run in its low nibble and code j + 16 in its high
 *    nibble.  Activations: M rows of K/2 bytes (W4A4) or K bytes of int8 in
 *    natural order (W4A8).  Codes lie in [-7, 7] (INT4) or [-127, 127] (INT8).
 *  - Device pointers must be 16-byte aligned and leading dimensions must make
 *    every row start 16-byte aligned; otherwise SERQ_ERR_INVALID_ARG.
 */
#ifndef SERQ_H_
#define SERQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SERQ_OK = 0,
  SERQ_ERR_INVALID_ARG = 1,        /* null pointer, bad size, misalignment   */
  SERQ_ERR_UNSUPPORTED_SHAPE = 2,  /* K/N not multiples of 32, r > K, ...    */
  SERQ_ERR_UNSUPPORTED_DEVICE = 3, /* current device is not sm_100           */
  SERQ_ERR_ALLOC = 4,              /* cudaMalloc failed (prepare only)       */
  SERQ_ERR_CUDA = 5,               /* a CUDA call or kernel launch failed    */
  SERQ_ERR_TIMEOUT = 6,            /* a kernel gave up a bounded wait        */
  SERQ_ERR_NUMERIC = 7             /* GPTQ: a Cholesky pivot was not positive */
} serq_status;

typedef enum { SERQ_W4A4 = 0, SERQ_W4A8 = 1 } serq_mode;
typedef enum { SERQ_F32 = 0, SERQ_BF16 = 1 } serq_dtype;

/* Kernel choice for serq_linear_ex / serq_linear_accum / serq_linear_group.
 * AUTO picks DECODE for M <= serq_decode_max_m() and PREFILL otherwise;
 * DECODE accepts M <= 64 when asked for explicitly.  PREFILL picks CTA pairs
 * with 256 x 256 tiles when the call's tiles (all layers of a group
 * together) keep at least 90% of the SMs busy, else 128 x 128 tiles. */
typedef enum {
  SERQ_ALGO_AUTO = 0,
  SERQ_ALGO_PREFILL = 1,       /* tcgen05 kind::i8 GEMM, TMEM accumulators; the
                                  output tile width is chosen from the shape  */
  SERQ_ALGO_DECODE = 2,        /* memory-bound GEMV (mma.sync), M <= 64: the
                                  streaming kernel when every SM's share of the
                                  weights is >= 96 KB and it fits, else the
                                  item-ring kernel                             */
  SERQ_ALGO_PREFILL_N128 = 3,  /* PREFILL with 128 x 128 output tiles, one CTA  */
  SERQ_ALGO_PREFILL_N256 = 4,  /* PREFILL with 128 x 256 output tiles, one CTA  */
  SERQ_ALGO_PREFILL_PAIR_N256 = 5, /* PREFILL with 256 x 256 tiles on a CTA pair
                                      (tcgen05 cta_group::2)                    */
  SERQ_ALGO_PREFILL_PAIR_TMEM_A = 6, /* W4A4 only: 256 x 192 tiles on a CTA pair with
                                        the widened activations in tensor memory  */
  SERQ_ALGO_DECODE_TC = 7,     /* M <= 32: tcgen05 GEMV with the weight rows as the
                                  MMA's M, split-K partial sums in the layer's
                                  workspace (one stream per layer at a time)  */
  SERQ_ALGO_DECODE_ITEMS = 8,  /* M <= 64: the memory-bound GEMV over 16-channel
                                  items with a shared bulk-copy ring          */
  SERQ_ALGO_DECODE_STREAM = 9  /* M <= 64: the streaming GEMV (equal channel
                                  shares per SM, TMA rings per warp) where its
                                  shared memory fits (M <= 32), else the item
                                  ring                                         */
} serq_algo;

typedef struct serq_layer serq_layer;

/* ------------------------------------------------------------------------ */
/* Offline preparation (untimed)                                            */
/* ------------------------------------------------------------------------ */

/* Saliency metric of step 2 below (SERQ notes, key design 2: the salient
 * rows of the folded weight are identified by their scale). */
typedef enum {
  SERQ_SALIENCY_SCALE = 0,      /* by s_j (default; the pages' "scale")      */
  SERQ_SALIENCY_ROW_ABSMAX = 1  /* by the folded row's max |s_j W_jn|        */
} serq_saliency;

/* Quantizer of the main weight in step 3 below. */
typedef enum {
  SERQ_QUANT_RTN = 0,  /* round-to-nearest (default; the pages' RTN)          */
  SERQ_QUANT_GPTQ = 1  /* GPTQ past the r salient rows ("SERQ(GPTQ)")         */
} serq_quantizer;

/* Options of the offline stage.  Fill with serq_prepare_opts_init, then
 * change what differs. */
typedef struct {
  float alpha;                /* SmoothQuant migration strength in [0, 1];
                                 default 0.5 (the square-root form)          */
  int rank;                   /* r, 0 <= r <= K; default 128                 */
  serq_mode mode;             /* activation format; weights are INT4 in both;
                                 default SERQ_W4A4                           */
  int saliency;               /* serq_saliency; default SERQ_SALIENCY_SCALE  */
  const int32_t* out_perm;    /* serq_prepare only: nullable HOST int32[N],
                                 the NEXT layer's saliency order (step 5)    */
  const float* out_colscale;  /* serq_prepare only: nullable HOST float[N],
                                 the NEXT layer's smoothing scales, divided
                                 into the columns (step 5); needs out_perm   */
  int quantizer;              /* serq_quantizer; default SERQ_QUANT_RTN      */
} serq_prepare_opts;

/* Defaults: alpha 0.5, rank 128, SERQ_W4A4, SERQ_SALIENCY_SCALE, no fold,
 * SERQ_QUANT_RTN. */
void serq_prepare_opts_init(serq_prepare_opts* opts);

/*
 * serq_prepare -- SERQ's offline stage for one weight, from HOST arrays.
 * Allocates the layer, uploads W and X_calib (and the fold arrays) to the
 * current device, runs the steps below there and returns when they have
 * finished; the handle owns its device memory (release with
 * serq_layer_destroy).
 *
 * Steps (SERQ notes, "overall framework" and key designs 1-3):
 *  1. static activation flattening (key design 1, SmoothQuant's static
 *     scale): s_j = max_t|Xc_tj|^alpha / max_n|W_jn|^(1 - alpha), both maxima
 *     floored at 1e-5; at alpha = 0.5 this is sqrt / sqrt / divide in fp32,
 *     any other alpha is evaluated in fp64 and rounded to fp32 once;
 *  2. saliency order P: channels by descending key (opts->saliency), ties by
 *     channel index (key design 2);
 *  3. W^ = P diag(s) W, quantized per output channel to INT4:
 *     code = clamp(rint(W^ * (7/amax)), -7, 7), sw = amax/7;
 *     With opts->quantizer = SERQ_QUANT_GPTQ ("SERQ(GPTQ)" in the SERQ notes'
 *     main results; gist.science (de) 2B names RTN or GPTQ for the main
 *     weight), rows r.. are quantized by GPTQ instead: with U the upper
 *     Cholesky factor of the inverse of H = sum_t xh_t xh_t^T + 0.01 *
 *     mean(diag) * I over the flattened, permuted calibration activations
 *     xh (serq_gptq_factor), row by row in order, e_i = (w_i - code_i*sw) /
 *     u_ii (fp32, U rounded to fp32) and w_j -= u_ij * e_i for j > i; the
 *     salient rows 0..r-1 keep round-to-nearest and move nothing (R below
 *     corrects them); amax and sw are the column's before any update;
 *  4. R = W^[0:r] - code[0:r]*sw (the main path's own error on the r salient
 *     rows, key design 2 / core idea), quantized the same way -> Rq, sR;
 *  5. optionally, before all of the above, the NEXT layer's order and
 *     smoothing scales are folded into this weight's output columns:
 *     W'[:, i] = W[:, out_perm[i]] / out_colscale[out_perm[i]] (key design 3:
 *     down_proj's order propagates into the gate/up columns).
 * Every step but the general-alpha power is IEEE fp32 with one rounding per
 * operation.
 *
 *  W        HOST, K x N fp32, row-major (d_in x d_out; Y = X W); N a multiple
 *           of 32.
 *  X_calib  HOST, n_calib x K fp32 calibration activations (n_calib >= 1).
 *  opts     options (NULL = the defaults above).
 *  layer    receives the new handle (NULL on failure; nothing leaks).
 * Errors: SERQ_ERR_INVALID_ARG (null pointers, alpha outside [0, 1], bad mode,
 * metric or quantizer, out_colscale without out_perm),
 * SERQ_ERR_UNSUPPORTED_SHAPE (K or N not a multiple of 32, rank outside
 * [0, K]), SERQ_ERR_ALLOC, SERQ_ERR_CUDA, SERQ_ERR_UNSUPPORTED_DEVICE,
 * SERQ_ERR_NUMERIC (GPTQ only: the damped Hessian or its inverse was not
 * positive definite in floating point).  Synchronous.
 */
serq_status serq_prepare(const float* W, int K, int N, const float* X_calib, int n_calib,
                         const serq_prepare_opts* opts, serq_layer** layer);

/*
 * serq_prepare_shared -- serq_prepare for n_weights weights that read the
 * same activation (q/k/v share one input, gate/up share one): one smoothing
 * vector s, whose weight maximum runs over all n_weights weights, and one
 * order P, so one set of activation codes feeds every returned layer.
 *  W        HOST array of n_weights HOST K x N_i fp32 arrays.
 *  N        HOST array of n_weights output widths (multiples of 32).
 *  X_calib  HOST, n_calib x K fp32.
 *  opts     options; opts->out_perm and opts->out_colscale must be NULL (the
 *           folds are per weight here).
 *  out_perm, out_colscale  NULL, or HOST arrays of n_weights nullable HOST
 *           arrays of N_i entries (step 5 per weight).
 *  layers   HOST array receiving n_weights new handles (all NULL on failure).
 * Errors as serq_prepare.  Synchronous.
 */
serq_status serq_prepare_shared(int n_weights, const float* const* W, const int* N, int K,
                                const float* X_calib, int n_calib, const serq_prepare_opts* opts,
                                const int32_t* const* out_perm, const float* const* out_colscale,
                                serq_layer** layers);

/*
 * serq_prepare_group -- serq_prepare_shared with every array on the DEVICE:
 * W[i] (K x N_i fp32), X_calib (n_calib x K fp32), out_perm[i] (int32[N_i])
 * and out_colscale[i] (float[N_i]) are DEVICE pointers (the pointer arrays
 * and N themselves are host arrays).  For callers whose weights are already
 * resident, such as a model loaded onto the GPU; nothing is uploaded.
 * Errors as serq_prepare.  Synchronous.
 */
serq_status serq_prepare_group(int n_weights, const float* const* W, const int* N, int K,
                               const float* X_calib, int n_calib, const serq_prepare_opts* opts,
                               const int32_t* const* out_perm, const float* const* out_colscale,
                               serq_layer** layers);

/*
 * serq_gptq_factor -- the inverse-Hessian factor GPTQ uses (serq_prepare's
 * step 3 with SERQ_QUANT_GPTQ computes it internally; this call exposes it).
 *   H = sum_t xh_t xh_t^T over the n_calib rows of Xh, in token order (fp64),
 *   H_ii += 0.01 * (H_00 + ... + H_K-1,K-1) / K   (H = I if that sum is 0),
 *   H = L L^T (Cholesky), V = L^-1, H^-1 = V^T V = L2 L2^T, U = L2^T,
 * so H^-1 = U^T U with U upper triangular (GPTQ, Frantar et al. 2022).
 * Every fp64 entry receives its terms in the order of the textbook
 * unblocked loops (sums from +0 in increasing index; Cholesky and forward
 * substitution subtracting their products in increasing index), one
 * rounding per product, sum, difference, quotient and square root, so the
 * result does not depend on the blocking.
 *  Xh  DEVICE, n_calib x K fp32, row-major: the flattened, permuted
 *      calibration activations (X[:, P] / s[P]).
 *  U   DEVICE, K x K fp64, row-major; receives U (zeros below the diagonal).
 *  K a positive multiple of 32, n_calib >= 1.  Uses 2 K^2 fp64 of
 *  temporary device memory.
 * Errors: SERQ_ERR_INVALID_ARG, SERQ_ERR_UNSUPPORTED_SHAPE, SERQ_ERR_ALLOC,
 * SERQ_ERR_CUDA, SERQ_ERR_NUMERIC (a pivot that is not positive; U is then
 * not meaningful).  Synchronous.
 */
serq_status serq_gptq_factor(const float* Xh, int n_calib, int K, double* U);

/* Frees the handle's device memory.  NULL is accepted.  Synchronous. */
void serq_layer_destroy(serq_layer* layer);

/* Shape and configuration of a prepared layer (any pointer may be NULL). */
serq_status serq_layer_info(const serq_layer* layer, int* K, int* N, int* rank, int* mode);

/* Synchronous copies of the layer's saliency order P (int32[K]: position i
 * holds original channel P[i]) and smoothing scales s (float[K]) into HOST
 * buffers: what the previous layer's serq_prepare needs for its fold
 * (opts->out_perm / out_colscale) or a caller needs to produce X^. */
serq_status serq_layer_get_perm(const serq_layer* layer, int32_t* perm);
serq_status serq_layer_get_smooth(const serq_layer* layer, float* smooth);

/* DEVICE pointers to the layer's permutation (int32[K]) and smoothing scales
 * (float[K]); owned by the layer, valid until serq_layer_destroy.  Used by
 * the previous layer's serq_prepare_group (out_perm / out_colscale) or by
 * serq_flatten_permute. */
serq_status serq_layer_perm_smooth(const serq_layer* layer, const int32_t** perm,
                                   const float** smooth);

/* Synchronous copies of the prepared tensors to HOST buffers (any may be
 * NULL):  wq  N*K/2 bytes (N x K packed INT4),  rq  N*rpad/2 bytes where
 * rpad = r rounded up to a multiple of 32 (columns past r are zero),
 * sw, sr  float[N],  perm  int32[K],  smooth  float[K]. */
serq_status serq_layer_get_packed(const serq_layer* layer, uint8_t* wq, uint8_t* rq, float* sw,
                                  float* sr, int32_t* perm, float* smooth);

/* ------------------------------------------------------------------------ */
/* Inference path                                                           */
/* ------------------------------------------------------------------------ */

/*
 * serq_quantize_act -- per-token symmetric activation quantizer and packer
 * (the X^_q of key design 2; X~_{s,q} is its first r columns, so no second
 * quantization is needed).  For each row m:
 *   amax = max_k |X[m,k]|,  inv = Q/amax,  code = clamp(rint(X*inv), -Q, Q),
 *   sx[m] = amax/Q  (Q = 7 for W4A4, 127 for W4A8; a zero row gives codes 0
 *   and sx 0).  fp32 arithmetic, round-to-nearest-even.
 *  X     DEVICE, M x K, dtype f32 or bf16, row stride ldx elements.
 *  Xq    DEVICE output: W4A4 -> M x K/2 bytes packed; W4A8 -> M x K int8.
 *  sx    DEVICE output float[M].
 * M >= 1; K <= 32768 (bf16) or 16384 (fp32).  Asynchronous on `stream`.
 */
serq_status serq_quantize_act(const void* X, serq_dtype dtype, int M, int K, int ldx,
                              serq_mode mode, void* Xq, float* sx, void* stream);

/*
 * serq_linear -- Y = sx * (sw * (Xq Wq^T) + sR * (Xq[:, :r] Rq^T)), bf16 out.
 * Both products are exact int32 sums; the residual reuses the activation
 * codes already loaded for the first r columns (key design 2: one matmul on
 * the salient channels, no intermediate quantization).  Output columns are
 * in the layer's output order (the original order, or out_perm's order when
 * a fold was given at prepare).
 *  Xq, sx  DEVICE, from serq_quantize_act with the layer's mode and K.
 *  Y       DEVICE bf16 output, M x N, row stride ldy elements (ldy >= N).
 * Asynchronous.  Uses no memory beyond its arguments and the layer.
 */
serq_status serq_linear(const serq_layer* layer, const void* Xq, const float* sx, int M,
                        void* Y, int ldy, void* stream);

/* serq_linear with an explicit kernel choice (SERQ_ALGO_DECODE needs
 * M <= 64). */
serq_status serq_linear_ex(const serq_layer* layer, const void* Xq, const float* sx, int M,
                           void* Y, int ldy, serq_algo algo, void* stream);

/* Test hook: the same kernels with the epilogue replaced by a store of the
 * exact integer accumulators.  acc0, acc1: DEVICE int32 M x N row-major
 * (acc1 is all zero when r = 0). */
serq_status serq_linear_accum(const serq_layer* layer, const void* Xq, int M, int32_t* acc0,
                              int32_t* acc1, serq_algo algo, void* stream);

/*
 * serq_linear_group -- serq_linear (or, with acc0/acc1, the accumulator
 * hook) for n layers that read the same activation codes, such as a
 * block's q/k/v projections or its gate/up pair (key design 2, applied to
 * each layer; the pages run them as separate GEMMs).  With a prefill kernel
 * the n products run as one launch over the union of their output tiles, so
 * setup and the last partial wave are paid once; SERQ_ALGO_DECODE runs the
 * union of the layers' 16-channel items as one launch; SERQ_ALGO_DECODE_TC
 * and SERQ_ALGO_PREFILL_PAIR_TMEM_A run one launch per layer.  Results are
 * identical to n serq_linear_ex calls with the same kernel.
 *  n        1..4.
 *  layers   HOST array of n layers with equal K and mode and ranks that
 *           round up to the same multiple of 32 (N may differ).
 *  Xq, sx   DEVICE, as serq_linear; the codes are read in each layer's
 *           input order, so the layers normally come from one
 *           serq_prepare_group call (one smoothing vector and order).
 *  Y, ldy   HOST arrays of n DEVICE bf16 outputs (M x N_l, row stride
 *           ldy[l] >= N_l) and their strides; may be null when acc0/acc1
 *           are given.
 *  acc0, acc1  both null, or HOST arrays of n DEVICE int32 M x N_l outputs
 *           (exact accumulators; sx and Y are then not used).
 *  algo     as serq_linear_ex (AUTO picks by M and the group's total tiles).
 * Asynchronous.  Uses no memory beyond its arguments and the layers.
 * Errors: SERQ_ERR_INVALID_ARG for n out of range or layers that differ in
 * K, padded rank or mode, and every serq_linear_ex error of any member.
 */
serq_status serq_linear_group(int n, const serq_layer* const* layers, const void* Xq, const float* sx,
                              int M, void* const* Y, const int* ldy, int32_t* const* acc0,
                              int32_t* const* acc1, serq_algo algo, void* stream);

/*
 * serq_linear_group_act -- serq_quantize_act followed by serq_linear_group,
 * from the flattened, permuted activations X^ (the token rows the layers
 * consume).  For few tokens (the decode kernels chosen, bf16 input, M <= 8,
 * K <= 4096) it is ONE launch: every CTA of the streaming decode kernel
 * quantizes the M rows itself (the per-token symmetric quantizer of
 * serq_quantize_act, same arithmetic, same codes) into the shared-memory
 * rows its MMAs read, so the codes never go through HBM and the quantize
 * launch and its dependency on the step before leave the critical path.
 * Otherwise (where every CTA reading all M bf16 rows would cost more than
 * the launch it saves) it runs the two calls one after the other.
 *  X, dtype, ldx  DEVICE M x K activations (bf16 or fp32), row stride ldx,
 *           rows 16-byte aligned.
 *  Xq, sx   DEVICE scratch with the sizes serq_quantize_act writes (M x K/2
 *           bytes for W4A4, M x K for W4A8; M floats); written when the call
 *           quantizes in a launch of its own, contents unspecified after.
 *  the rest as serq_linear_group.
 * Asynchronous.  Errors: those of serq_quantize_act and serq_linear_group.
 */
serq_status serq_linear_group_act(int n, const serq_layer* const* layers, const void* X, serq_dtype dtype,
                                  int ldx, int M, void* Xq, float* sx, void* const* Y, const int* ldy,
                                  int32_t* const* acc0, int32_t* const* acc1, serq_algo algo, void* stream);

/*
 * serq_linear_decode_static -- serq_linear (or, with acc0/acc1, the
 * accumulator hook) through the tensor-core decode kernel
 * (SERQ_ALGO_DECODE_TC) with its split-K partial sums and tile counters in a
 * scratch area compiled into the library (a file-scope __device__ array of
 * 4 MB, one per device that loads the library, held until the process
 * exits) instead of the layer's workspace, so the call allocates nothing.
 * It is for callers that cannot call cudaMalloc on the decode path: a
 * serving loop whose device memory is reserved up front by another pool, a
 * caller running inside an allocator's own callbacks, or one that must not
 * take the allocator's lock or its implicit synchronisation between tokens.
 * The pages have no counterpart; this is a deployment variant of the same
 * arithmetic.
 *  Xq, sx, Y, ldy  as serq_linear; 1 <= M <= 32.
 *  acc0, acc1      both null (bf16 output in Y), or both DEVICE int32 M x N
 *                  (exact accumulators; sx and Y are then not used).
 *  N <= 16384 and M <= 32, else SERQ_ERR_UNSUPPORTED_SHAPE.
 * Set-up: the first call on a device (with that device current) looks up the
 * array's device address and clears the array with cudaMemsetAsync on
 * `stream`, ordered before the kernel; make that first call before any stream
 * capture.  Every completed call leaves the scratch zero.  After
 * serq_device_error has reported a timed-out wait, which can leave partial
 * sums behind, the next call on that device clears it again the same way.
 * Races: all calls on a device share the one scratch area and each call
 * relies on the previous one having finished, so calls that overlap on the
 * GPU race (use one stream, or order streams by events), across all layers.
 */
serq_status serq_linear_decode_static(const serq_layer* layer, const void* Xq, const float* sx, int M,
                                      void* Y, int ldy, int32_t* acc0, int32_t* acc1, void* stream);

/* ------------------------------------------------------------------------ */
/* Comparator: two-factor low-rank error reconstruction (L2QER)             */
/* ------------------------------------------------------------------------ */

/*
 * The method SERQ is measured against (SERQ notes, "field status", "pain
 * points" and "vs L2QER"; gist.science (ja) summary, "computation flow"):
 * the weight's quantization error is approximated by two low-rank factors,
 * L1 L2 ~ W^ - Q(W^), applied one after the other at inference with an
 * on-the-fly quantization of the intermediate:
 *     Y = X_q W_q + Q(X_q L1_q) L2_q.
 * Built on a prepared SERQ layer so that the main product X_q W_q is the
 * same; only the error path differs.  The factors are given (an offline
 * step, like calibration data; the pages extract them by a scaled SVD) and
 * quantized here per output channel to INT4 like W^ (the pages' L2QER keeps
 * them in 8 bits; 4 bits is the cheaper choice, so the comparison isolates
 * the serial structure).  W4A4 layers only.
 */
typedef struct serq_l2qer serq_l2qer;

/*
 * serq_l2qer_prepare -- quantizes and packs the factors.
 *  layer  prepared W4A4 layer (not owned; must outlive the comparator).
 *  L1     DEVICE, K x r fp32 row-major, rows in the layer's input order
 *         (the flattened, permuted X^ multiplies it).
 *  L2     DEVICE, r x N fp32 row-major.
 *  r      a positive multiple of 32, <= K.
 *  out    receives the handle (NULL on failure).  Synchronous.
 */
serq_status serq_l2qer_prepare(const serq_layer* layer, const float* L1, const float* L2, int r,
                               serq_l2qer** out);

/* Frees the comparator's device memory (not the layer).  NULL accepted. */
void serq_l2qer_destroy(serq_l2qer* q);

/* Synchronous copies to HOST buffers (any may be NULL): l1q r x K/2 bytes
 * (L1's codes, output channel major), s_l1 float[r], l2q N x r/2 bytes,
 * s_l2 float[N]. */
serq_status serq_l2qer_get_packed(const serq_l2qer* q, uint8_t* l1q, float* s_l1, uint8_t* l2q, float* s_l2);

/*
 * serq_l2qer_linear -- the comparator's inference path, three launches on
 * `stream`: Z = bf16(sx * (s_L1 * (X_q L1_q))) (the layer epilogue of a
 * rank-0 linear), per-token quantization of Z (as serq_quantize_act,
 * W4A4), then Y = sx * (sw * acc0) + sz * (s_L2 * acc2) with
 * acc0 = X_q W_q and acc2 = Z_q L2_q exact in int32.
 *  Xq, sx   DEVICE, from serq_quantize_act of the layer's X^.
 *  Z        DEVICE bf16 M x r (written), Zq DEVICE M x r/2 bytes (written),
 *           sz DEVICE float[M] (written): the intermediate, owned by the
 *           caller (the call allocates nothing).
 *  Y, ldy   DEVICE bf16 M x N output.
 *  algo     SERQ_ALGO_AUTO, DECODE (M <= 32), PREFILL, PREFILL_N128 or
 *           PREFILL_PAIR_N256.
 * Asynchronous.
 */
serq_status serq_l2qer_linear(const serq_l2qer* q, const void* Xq, const float* sx, int M, void* Z, void* Zq,
                              float* sz, void* Y, int ldy, serq_algo algo, void* stream);

/* Test hook: the final GEMM's exact accumulators acc0 = X_q W_q and
 * acc1 = Z_q L2_q (DEVICE int32 M x N) for given codes Xq and Zq. */
serq_status serq_l2qer_accum(const serq_l2qer* q, const void* Xq, const void* Zq, int M, int32_t* acc0,
                             int32_t* acc1, serq_algo algo, void* stream);

/*
 * serq_silu_mul_quantize -- MLP intermediate of a Llama block whose gate/up
 * were prepared with down_proj's fold: h = silu(G) * U in fp32 (silu(g) =
 * g / (1 + e^-g), e^x by Cody-Waite reduction and a degree-7 Taylor
 * polynomial, saturating beyond |x| > 88), then quantized per token exactly
 * as serq_quantize_act.  G and U arrive already in down_proj's saliency order
 * with U already divided by down_proj's smoothing scales (key design 3), so h
 * is down_proj's X^.
 *  G, U  DEVICE bf16, M x F (F <= 16384), row stride ld elements.
 *  Xq, sx as serq_quantize_act with K = F.
 */
serq_status serq_silu_mul_quantize(const void* G, const void* U, int M, int F, int ld,
                                   serq_mode mode, void* Xq, float* sx, void* stream);

/*
 * serq_flatten_permute -- X^ = X diag(s)^-1 P^-1 for a layer whose producer
 * was not folded (standalone layers, benchmarks):  X^[m, i] =
 * X[m, perm[i]] / s[perm[i]] in fp32, stored as out_dtype (bf16 by
 * round-to-nearest-even).  In a folded network this is done offline
 * (key design 3) and this call is not used.
 *  X     DEVICE M x K (ldx), dtype in_dtype.   Xh  DEVICE M x K (ldxh).
 */
serq_status serq_flatten_permute(const serq_layer* layer, const void* X, serq_dtype in_dtype,
                                 int M, int ldx, void* Xh, serq_dtype out_dtype, int ldxh,
                                 void* stream);

/* ------------------------------------------------------------------------ */
/* Diagnostics                                                              */
/* ------------------------------------------------------------------------ */

/* Largest M for which SERQ_ALGO_AUTO chooses the decode kernel. */
int serq_decode_max_m(void);

/* Thread-local description of the last failure ("" after success). */
const char* serq_last_error_string(void);

/* SERQ_OK when the current device is sm_100 (B200 class). */
serq_status serq_check_device(void);

/* Reads and clears the device-side status word that kernels set when a
 * bounded wait gives up (0 = none).  Synchronises the current device. */
serq_status serq_device_error(int* code);

/*
 * Test hook for failure detection (no GPU fault involved): runs the
 * streaming decode kernel (SERQ_ALGO_DECODE, M <= 32) with its activation
 * copies withheld and the bounded wait for them shortened to wait_us
 * microseconds (1 .. 10^6).  Every CTA gives up that wait, records the
 * timeout in the device status word (serq_device_error then reports 2),
 * lets its weight copies land and returns; Y is not written.  The next call
 * on the device runs normally.
 */
serq_status serq_test_decode_timeout(const serq_layer* layer, const void* Xq, const float* sx, int M, void* Y,
                                     int ldy, int wait_us, void* stream);

/* Library version string. */
const char* serq_version(void);

/*
 * ---------------------------------------------------------------------------
 * SERQ with MXFP4 codes.  The SERQ pages name MXFP4 beside INT4 as a data
 * format the method supports and quote their Blackwell latency on it
 * (gist.science (de) sections 3 "Kompatibilität" and 4 "Performance &
 * Latenz", about 1% over plain MXFP4; gist.science (ja) section 2: with R in
 * 4 bits the linear is 4-bit integer or MXFP4 arithmetic).  The format is
 * the OCP Microscaling (MX) one: blocks of 32 consecutive elements along K
 * share a power-of-two scale stored as an E8M0 byte (2^(byte - 127)), every
 * element is FP4 E2M1 (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6; sign in bit
 * 3).  A block's exponent is floor(log2(max|v|)) - 2 clamped to [-127, 127]
 * (-127 for an all-zero block); an element is v / 2^e rounded to the
 * nearest E2M1 value, ties to the even code, beyond 6 to 6, zero as +0.
 *
 * The steps of serq_prepare stay as they are (the smoothing scales s and
 * the saliency order P are taken from a prepared INT4 layer); W^, R and the
 * per-token activations are MXFP4 instead of INT4, and the GEMM multiplies
 * the codes on the tensor core with the block scales applied inside it, the
 * residual product X~_{s,q} Q(R) accumulating into the same fp32 sums:
 *     Y = deq(X_q) deq(W^_q) + deq(X_q[:, 0:r]) deq(R_q)     (rounded to bf16).
 *
 * Storage: codes two per byte in K order (element 2i in the low nibble),
 * rows of K/2 bytes.  Scales of the GEMM's operands are TILED: 1 KB tiles of
 * 128 rows x 8 blocks (256 elements of K), row-major over (row / 128,
 * block / 8), 8 bytes per row inside a tile; the byte of (row m, block b) is
 * at ((m / 128) * (K / 256) + b / 8) * 1024 + (m % 128) * 8 + b % 8.
 * Shapes: K a multiple of 256, N a multiple of 128, r a multiple of 32.
 * ---------------------------------------------------------------------------
 */
typedef struct serq_mx_layer serq_mx_layer;

/*
 * serq_mx_prepare -- the offline stage with MXFP4 codes.
 *  base  a prepared layer (not owned; may be destroyed afterwards) whose
 *        smoothing scales s, saliency order P and rank r are used; prepared
 *        without an output fold, from the same W.
 *  W     DEVICE, K x N fp32 row-major, the weight base was prepared from.
 *  out   receives the handle (NULL on failure; nothing leaks).
 * W^ = P diag(s) W (one fp32 multiply per element, as serq_prepare) is
 * quantized per output channel in blocks of 32 along K; R = W^[0:r] -
 * deq(W^_q)[0:r] (one fp32 subtraction, the dequantized value being exact)
 * is quantized the same way.
 * Errors: SERQ_ERR_INVALID_ARG (null pointers, layer of another device),
 * SERQ_ERR_UNSUPPORTED_SHAPE (K not a multiple of 256, N not of 128, r not
 * of 32), SERQ_ERR_ALLOC, SERQ_ERR_CUDA, SERQ_ERR_UNSUPPORTED_DEVICE.
 * Synchronous.
 */
serq_status serq_mx_prepare(const serq_layer* base, const float* W, serq_mx_layer** out);

/* Frees the layer's device memory.  NULL accepted. */
void serq_mx_destroy(serq_mx_layer* q);

/* Synchronous copies to HOST buffers (any may be NULL), scales UNTILED:
 * wq N x K/2 bytes, we N x K/32 E8M0 bytes, rq N x r/2 bytes, re N x r/32
 * E8M0 bytes (rq and re untouched when r = 0). */
serq_status serq_mx_get_packed(const serq_mx_layer* q, uint8_t* wq, uint8_t* we, uint8_t* rq, uint8_t* re);

/* Bytes of the tiled activation scales for M tokens of K channels:
 * ceil(M / 128) * 128 * K / 32 (rows past M hold zero bytes); 0 for an
 * invalid shape. */
size_t serq_mx_act_scale_bytes(int M, int K);

/*
 * serq_mx_quantize_act -- per-token MXFP4 of the flattened, permuted
 * activations X^ (serq_flatten_permute's output), blocks of 32 along K.
 *  Xh    DEVICE M x K (row stride ldxh elements, rows 16-byte aligned), bf16
 *        or fp32.
 *  Xq    DEVICE M x K/2 bytes (written).
 *  xe    DEVICE serq_mx_act_scale_bytes(M, K) bytes, tiled (written).
 * The residual product reads the first r/32 blocks of the same codes and
 * scales.  Inputs must be finite.  Errors: SERQ_ERR_INVALID_ARG (null or
 * misaligned pointers, bad dtype or M), SERQ_ERR_UNSUPPORTED_SHAPE (K not a
 * positive multiple of 256), SERQ_ERR_CUDA.  Asynchronous on `stream`.
 */
serq_status serq_mx_quantize_act(const void* Xh, serq_dtype dtype, int M, int K, int ldxh, void* Xq, void* xe,
                                 void* stream);

/*
 * serq_mx_linear -- Y = deq(X_q) deq(W^_q) + deq(X_q[:, 0:r]) deq(R_q) for
 * codes and tiled scales from serq_mx_quantize_act.  One launch: 128 x 128
 * output tiles, tcgen05.mma kind::mxf4 with E8M0 block scales, fp32
 * accumulation in tensor memory (summation order within the tensor core
 * unspecified), bf16 output by round-to-nearest-even.
 *  Y, ldy  DEVICE bf16 M x N output, row stride ldy elements (a multiple of
 *          8, >= N).
 * Errors: SERQ_ERR_INVALID_ARG (null or misaligned pointers, M outside
 * [1, 65535 * 128], bad ldy), SERQ_ERR_CUDA.  A wait that gives up is
 * reported by serq_device_error.  Asynchronous on `stream`.
 * Validation: the codes and scales of serq_mx_prepare and
 * serq_mx_quantize_act are bit-exact against the CPU oracle on a B200; this
 * product's parity with the replicated scale-word layout is not yet
 * confirmed on a B200.
 */
serq_status serq_mx_linear(const serq_mx_layer* q, const void* Xq, const void* xe, int M, void* Y, int ldy,
                           void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SERQ_H_ */
