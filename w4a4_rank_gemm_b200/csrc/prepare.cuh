// Offline SERQ preparation kernels (untimed): static activation flattening,
// saliency order, folding, per-output-channel INT4 quantization of W^ and of
// the compensator R, packing.
//
// Every floating-point step is one IEEE fp32 operation with round-to-nearest
// (explicit __f*_rn intrinsics, so no multiply-add contraction can change a
// rounding), because the resulting integer codes must be reproducible.
#pragma once
#include "common.cuh"

namespace serq {
namespace prep {

// A weight as seen after the optional fold of the next layer's order into
// its output columns (SERQ notes, key design 3):
//   W'[j, n] = W[j, perm[n]] / div[perm[n]]     (or W[j, n] without a fold).
struct WeightView {
  const float* W;
  int N;
  const int32_t* perm;  // nullable
  const float* div;     // nullable (only with perm)
  __device__ __forceinline__ float at(int j, int n) const {
    if (perm) {
      const int p = perm[n];
      const float v = W[(size_t)j * N + p];
      return div ? __fdiv_rn(v, div[p]) : v;
    }
    return W[(size_t)j * N + n];
  }
};

// Positive floats order like their bit patterns, so an integer atomicMax on
// the bits is a float max for values >= 0.
__device__ __forceinline__ void atomic_max_nonneg(float* addr, float v) {
  atomicMax(reinterpret_cast<int*>(addr), __float_as_int(v));
}

// out[c] = max_r |X[r, c]|   (activation maxima over the calibration tokens)
__global__ void k_colmax_abs(const float* __restrict__ X, int rows, int cols, float* __restrict__ out) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= cols) return;
  float m = 0.f;
  for (int r = 0; r < rows; ++r) m = fmaxf(m, fabsf(X[(size_t)r * cols + c]));
  out[c] = m;
}

// amax_w[j] = max(amax_w[j], max_n |W'[j, n]|)   (one block per row j)
__global__ void k_rowmax_abs(WeightView w, int K, float* __restrict__ amax_w) {
  const int j = blockIdx.x;
  if (j >= K) return;
  float m = 0.f;
  for (int n = threadIdx.x; n < w.N; n += blockDim.x) m = fmaxf(m, fabsf(w.at(j, n)));
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float red[32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < (int)(blockDim.x >> 5); ++i) m = fmaxf(m, red[i]);
    m = fmaxf(m, red[0]);
    atomic_max_nonneg(&amax_w[j], m);
  }
}

// s_j = max(amax_x, 1e-5)^alpha / max(amax_w, 1e-5)^(1 - alpha)  (SmoothQuant's
// static scale with migration strength alpha; SERQ notes key design 1).  At
// the default alpha = 1/2 it is sqrt / sqrt / divide, each one fp32 rounding;
// any other alpha is two fp64 powers and a division rounded to fp32 once.
// In place over amax_x.
__global__ void k_smooth(float* __restrict__ ax_to_s, const float* __restrict__ amax_w, int K, float alpha) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= K) return;
  const float floor_ = 1e-5f;
  const float ax = fmaxf(ax_to_s[j], floor_), aw = fmaxf(amax_w[j], floor_);
  if (alpha == 0.5f) {
    ax_to_s[j] = __fdiv_rn(__fsqrt_rn(ax), __fsqrt_rn(aw));
  } else {
    const double a = (double)alpha;
    ax_to_s[j] = __double2float_rn(__ddiv_rn(pow((double)ax, a), pow((double)aw, 1.0 - a)));
  }
}

// Saliency key of channel j: s_j (metric 0) or the folded row's absolute
// maximum s_j * max_n |W_jn| (metric 1, one fp32 multiply).
__global__ void k_saliency_key(const float* __restrict__ s, const float* __restrict__ amax_w, int K, int metric,
                               float* __restrict__ key) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= K) return;
  key[j] = (metric == 1) ? __fmul_rn(s[j], amax_w[j]) : s[j];
}

// Saliency order (SERQ notes key design 2): position of channel i is the
// number of channels with a larger scale plus the number of equal-scale
// channels before it; perm[position] = i.  O(K^2) comparisons, run once.
__global__ void k_rank_perm(const float* __restrict__ s, int K, int32_t* __restrict__ perm) {
  extern __shared__ float tile[];
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const float si = (i < K) ? s[i] : 0.f;
  int rank = 0;
  for (int base = 0; base < K; base += blockDim.x) {
    const int j = base + threadIdx.x;
    tile[threadIdx.x] = (j < K) ? s[j] : 0.f;
    __syncthreads();
    const int lim = min((int)blockDim.x, K - base);
    if (i < K) {
      for (int t = 0; t < lim; ++t) {
        const float sj = tile[t];
        const int jj = base + t;
        rank += (sj > si) || (sj == si && jj < i);
      }
    }
    __syncthreads();
  }
  if (i < K) perm[rank] = i;
}

// W^[i, n] = s[perm[i]] * W'[perm[i], n]
__device__ __forceinline__ float w_hat(const WeightView& w, const float* s, const int32_t* perm, int i,
                                       int n) {
  const int j = perm[i];
  return __fmul_rn(s[j], w.at(j, n));
}

// amax_col[n] = max over rows [i0, i0 + rows) of |W^[i, n]|
__global__ void k_colmax_what(WeightView w, const float* __restrict__ s, const int32_t* __restrict__ perm,
                              int K, int rows_per_block, float* __restrict__ amax_col) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= w.N) return;
  const int i0 = blockIdx.y * rows_per_block;
  const int i1 = min(K, i0 + rows_per_block);
  float m = 0.f;
  for (int i = i0; i < i1; ++i) m = fmaxf(m, fabsf(w_hat(w, s, perm, i, n)));
  atomic_max_nonneg(&amax_col[n], m);
}

// Symmetric INT4 code of v with the group maximum amax:
// clamp(rint(v * (7 / amax)), -7, 7); 0 when amax == 0.
__device__ __forceinline__ int code4(float v, float amax) {
  if (!(amax > 0.f)) return 0;
  const float inv = __fdiv_rn(7.f, amax);
  int q = __float2int_rn(__fmul_rn(v, inv));
  return max(-7, min(7, q));
}

// Packed storage: every run of 32 codes of a row is 16 bytes; byte j holds
// code j (low nibble) and code j + 16 (high nibble), two's complement.  The
// tensor-core kernels widen such a run to 32 int8 in natural order with three
// logic ops per 4 bytes.
__device__ __forceinline__ uint4 pack_run32(const int (&q)[32]) {
  uint32_t w[4] = {0, 0, 0, 0};
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const uint32_t b = (uint32_t)(q[j] & 0xF) | ((uint32_t)(q[j + 16] & 0xF) << 4);
    w[j >> 2] |= b << (8 * (j & 3));
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Quantize W^ per output channel and pack into wq (N x K/2 bytes).  One
// thread packs one 32-code run of one output channel.
__global__ void k_quant_pack_w(WeightView w, const float* __restrict__ s, const int32_t* __restrict__ perm,
                               int K, const float* __restrict__ amax_col, uint8_t* __restrict__ wq) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  const int i0 = blockIdx.y * 32;
  if (n >= w.N || i0 >= K) return;
  const float amax = amax_col[n];
  int q[32];
#pragma unroll
  for (int t = 0; t < 32; ++t) q[t] = code4(w_hat(w, s, perm, i0 + t, n), amax);
  *reinterpret_cast<uint4*>(wq + (size_t)n * (K / 2) + i0 / 2) = pack_run32(q);
}

// R[i, n] = W^[i, n] - code(W^[i, n]) * sw[n], sw = amax_col / 7 (the main
// path's own dequantized salient rows; SERQ notes core idea).
__device__ __forceinline__ float resid(const WeightView& w, const float* s, const int32_t* perm, int i, int n,
                                       float amax_col_n) {
  const float v = w_hat(w, s, perm, i, n);
  const float sw = __fdiv_rn(amax_col_n, 7.f);
  const float deq = __fmul_rn((float)code4(v, amax_col_n), sw);
  return __fsub_rn(v, deq);
}

__global__ void k_colmax_resid(WeightView w, const float* __restrict__ s, const int32_t* __restrict__ perm,
                               int r, const float* __restrict__ amax_col, float* __restrict__ amax_r) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= w.N) return;
  const float a = amax_col[n];
  float m = 0.f;
  for (int i = 0; i < r; ++i) m = fmaxf(m, fabsf(resid(w, s, perm, i, n, a)));
  amax_r[n] = m;
}

// Quantize R per output channel and pack into rq (N x rpad/2 bytes, codes
// past r are zero).  One thread per 32-code run.
__global__ void k_quant_pack_r(WeightView w, const float* __restrict__ s, const int32_t* __restrict__ perm,
                               int r, int rpad, const float* __restrict__ amax_col,
                               const float* __restrict__ amax_r, uint8_t* __restrict__ rq) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  const int i0 = blockIdx.y * 32;
  if (n >= w.N || i0 >= rpad) return;
  const float a = amax_col[n];
  const float ar = amax_r[n];
  int q[32];
#pragma unroll
  for (int t = 0; t < 32; ++t) {
    const int i = i0 + t;
    q[t] = (i < r) ? code4(resid(w, s, perm, i, n, a), ar) : 0;
  }
  *reinterpret_cast<uint4*>(rq + (size_t)n * (rpad / 2) + i0 / 2) = pack_run32(q);
}

// sw = amax_col / 7, sR = amax_r / 7 (in place)
__global__ void k_finalize_scales(float* __restrict__ amax_col_to_sw, float* __restrict__ amax_r_to_sr,
                                  int N, int has_r) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  amax_col_to_sw[n] = __fdiv_rn(amax_col_to_sw[n], 7.f);
  amax_r_to_sr[n] = has_r ? __fdiv_rn(amax_r_to_sr[n], 7.f) : 0.f;
}

}  // namespace prep
}  // namespace serq
