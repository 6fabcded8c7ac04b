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
  SERQ_ERR_TIMEOUT = 6             /* a kernel gave up a bounded wait        */
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
  SERQ_ALGO_DECODE = 2,        /* memory-bound split-K tensor-core GEMV, M <= 64 */
  SERQ_ALGO_PREFILL_N128 = 3,  /* PREFILL with 128 x 128 output tiles, one CTA  */
  SERQ_ALGO_PREFILL_N256 = 4,  /* PREFILL with 128 x 256 output tiles, one CTA  */
  SERQ_ALGO_PREFILL_PAIR_N256 = 5, /* PREFILL with 256 x 256 tiles on a CTA pair
                                      (tcgen05 cta_group::2)                    */
  SERQ_ALGO_PREFILL_PAIR_TMEM_A = 6, /* W4A4 only: 256 x 192 tiles on a CTA pair with
                                        the widened activations in tensor memory  */
  SERQ_ALGO_DECODE_TC = 7      /* M <= 32: tcgen05 GEMV with the weight rows as the
                                  MMA's M, split-K partial sums in the layer's
                                  workspace (one stream per layer at a time)  */
} serq_algo;

typedef struct serq_layer serq_layer;

/* ------------------------------------------------------------------------ */
/* Offline preparation (untimed)                                            */
/* ------------------------------------------------------------------------ */

/*
 * serq_prepare_group -- SERQ's offline stage for n_weights weights that read
 * the same activation (q/k/v share one input, gate/up share one).
 *
 * Steps (SERQ notes, "overall framework" and key designs 1-3):
 *  1. static activation flattening: s_j = sqrt(max_t|Xc_tj|) / sqrt(max|W_j,:|)
 *     with both maxima floored at 1e-5 and the weight maximum taken over all
 *     n_weights weights (key design 1; SmoothQuant form with strength 1/2);
 *  2. saliency order P: channels by descending s_j, ties by channel index
 *     (key design 2: salient rows are identified by their scale);
 *  3. W^ = P diag(s) W, quantized per output channel to INT4:
 *     code = clamp(rint(W^ * (7/amax)), -7, 7), sw = amax/7;
 *  4. R = W^[0:r] - code[0:r]*sw (the main path's own error on the r salient
 *     rows, key design 2 / core idea), quantized the same way -> Rq, sR;
 *  5. optionally, before all of the above, the NEXT layer's permutation and
 *     smoothing divisor are folded into this weight's output columns:
 *     W'[:, i] = W[:, out_perm[i]] / out_div[out_perm[i]] (key design 3:
 *     down_proj's order propagates into the gate/up columns).
 * All arithmetic is IEEE fp32 with one rounding per operation.
 *
 *  W        host array of n_weights DEVICE pointers, each K x N_i fp32,
 *           row-major (d_in x d_out; Y = X W).
 *  N        host array of n_weights output widths (multiples of 32).
 *  X_calib  DEVICE, n_calib x K fp32 calibration activations (n_calib >= 1).
 *  rank     r, 0 <= r <= K.
 *  mode     SERQ_W4A4 or SERQ_W4A8 (weights are INT4 in both).
 *  out_perm host array of n_weights nullable DEVICE int32[N_i] pointers (or
 *           NULL for none).  out_div likewise with DEVICE float[N_i]; an
 *           out_div entry requires the matching out_perm entry.
 *  layers   host array receiving n_weights new handles.  On failure every
 *           entry is set to NULL and nothing is leaked.
 * Synchronous (returns after the device work has finished).
 */
serq_status serq_prepare_group(int n_weights, const float* const* W, const int* N, int K,
                               const float* X_calib, int n_calib, int rank, serq_mode mode,
                               const int32_t* const* out_perm, const float* const* out_div,
                               serq_layer** layers);

/* One weight: serq_prepare_group with n_weights = 1. */
serq_status serq_prepare(const float* W, int K, int N, const float* X_calib, int n_calib,
                         int rank, serq_mode mode, const int32_t* out_perm,
                         const float* out_div, serq_layer** layer);

/* Frees the handle's device memory.  NULL is accepted.  Synchronous. */
void serq_layer_destroy(serq_layer* layer);

/* Shape and configuration of a prepared layer (any pointer may be NULL). */
serq_status serq_layer_info(const serq_layer* layer, int* K, int* N, int* rank, int* mode);

/* DEVICE pointers to the layer's permutation (int32[K]) and smoothing scales
 * (float[K]); owned by the layer, valid until serq_layer_destroy.  Used by
 * the previous layer's prepare (out_perm / out_div) or by
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
 * serq_linear_decode_static -- serq_linear (or, with acc0/acc1, the
 * accumulator hook) through the tensor-core decode kernel
 * (SERQ_ALGO_DECODE_TC) with its split-K partial sums and tile counters in a
 * scratch area compiled into the library, one per device, instead of the
 * layer's workspace: the call allocates nothing.  The pages have no
 * counterpart; this is a deployment variant of the same arithmetic.
 *  Xq, sx, Y, ldy  as serq_linear; M <= 32.
 *  acc0, acc1      both null (bf16 output in Y), or both DEVICE int32 M x N
 *                  (exact accumulators; sx and Y are then not used).
 *  N <= 16384, else SERQ_ERR_UNSUPPORTED_SHAPE.
 * The scratch must start at zero: the first call on a device clears it (a
 * synchronous cudaMemset) and every completed call leaves it zero.
 * Races: all calls on a device share the one scratch area, so they must not
 * overlap in time (one stream, or streams ordered by events), across all
 * layers.  A wait that times out (serq_device_error) leaves it undefined.
 */
serq_status serq_linear_decode_static(const serq_layer* layer, const void* Xq, const float* sx, int M,
                                      void* Y, int ldy, int32_t* acc0, int32_t* acc1, void* stream);

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

/* Library version string. */
const char* serq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SERQ_H_ */
