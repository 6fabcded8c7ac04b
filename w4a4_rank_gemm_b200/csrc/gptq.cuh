// GPTQ for SERQ's main weight (offline, untimed): the damped Hessian of the
// flattened, permuted calibration activations, the upper Cholesky factor U of
// its inverse, and the row-by-row quantization with error feedback past the
// r salient rows (GPTQ, Frantar et al. 2022, as "SERQ(GPTQ)" in the SERQ
// notes' main results table; gist.science (de) section 2B).
//
// Arithmetic order.  Every entry of every fp64 matrix receives its terms in
// the order of the textbook unblocked algorithms, one rounding per product
// and per sum or difference (explicit __d*_rn intrinsics, no contraction):
//   * a sum starts from +0 and adds its terms in increasing index (the Gram
//     matrix over tokens, H^-1 = V^T V over k);
//   * Cholesky (right-looking): T_ij loses L_ik L_jk for k = 0..j-1 in
//     order, then L_jj = sqrt(T_jj), L_ij = T_ij / L_jj;
//   * V = L^-1 (forward substitution on the identity): T_ik loses L_im V_mk
//     for m = 0..i-1 in order, then V_ik = T_ik / L_ii.
// The kernels below block these loops (32-column panels, 64 x 64 output
// tiles) without changing any entry's sequence, so the factor is the same
// bits as the unblocked loops.  Terms that the unblocked loops skip because
// one factor is a structural zero (above the diagonal of L or V) may be
// included here: their products are zeros, and subtracting or adding a
// zero leaves every value these loops can hold unchanged (no entry is ever
// -0: sums start at +0 and exact cancellations round to +0).
#pragma once
#include "common.cuh"
#include "prepare.cuh"

namespace serq {
namespace gptq {

constexpr int kTile = 64;   // output tile edge of k_tile
constexpr int kChunk = 32;  // k per shared-memory stage; also the panel width
constexpr int kPitch = kTile + 1;

// One tile pass  C[i][j] (op)= sum_k P(k, i) * Q(k, j)  over k in [kb, ke).
// P(k, i) is P[k * ldp + i] (k-major) or, with PT, P[i * ldp + k]; same for Q.
struct TileArgs {
  double* C;
  int ldc;
  int ci0, cj0;    // C coordinates of output (0, 0)
  int mi, mj;      // output extent
  const void* P;
  int ldp, pi0;    // P coordinates: output row i reads P(., pi0 + i)
  const void* Q;
  int ldq, qj0;
  int kb, ke;
  int kb_row_tile; // 1: a tile's k starts at max(kb, its first output row + kb_offset)
  int kb_offset;
  int lower;       // 1: only tiles with tj <= ti (square output), entries i >= j stored
  int ntj;         // column tiles (when !lower)
};

template <typename T>
__device__ __forceinline__ double ld_as_double(const void* p, size_t idx) {
  return (double)static_cast<const T*>(p)[idx];
}

// SUB: C -= sum (the matrix keeps its entry and loses the terms); else
// C = +0 + sum.
template <typename TP, bool PT, bool QT, bool SUB>
__global__ void __launch_bounds__(256) k_tile(TileArgs a) {
  __shared__ double Ps[kChunk][kPitch];
  __shared__ double Qs[kChunk][kPitch];
  int ti, tj;
  if (a.lower) {
    // blockIdx.x = ti (ti + 1) / 2 + tj, tj <= ti
    const int x = blockIdx.x;
    ti = (int)((sqrtf(8.f * (float)x + 1.f) - 1.f) * 0.5f);
    while ((ti + 1) * (ti + 2) / 2 <= x) ++ti;
    while (ti * (ti + 1) / 2 > x) --ti;
    tj = x - ti * (ti + 1) / 2;
  } else {
    ti = blockIdx.x / a.ntj;
    tj = blockIdx.x % a.ntj;
  }
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int r0 = ti * kTile, c0 = tj * kTile;
  double acc[4][4];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int i = r0 + ty + 16 * r, j = c0 + tx + 16 * c;
      acc[r][c] = (SUB && i < a.mi && j < a.mj) ? a.C[(size_t)(a.ci0 + i) * a.ldc + a.cj0 + j] : 0.0;
    }
  int kb = a.kb;
  if (a.kb_row_tile) kb = max(kb, r0 + a.kb_offset);
  for (int k0 = kb; k0 < a.ke; k0 += kChunk) {
    const int kn = min(kChunk, a.ke - k0);
#pragma unroll
    for (int s = 0; s < (kChunk * kTile) / 256; ++s) {
      const int e = threadIdx.x + 256 * s;
      int kk, ii;
      if (PT) { kk = e % kChunk; ii = e / kChunk; } else { kk = e / kTile; ii = e % kTile; }
      const int i = r0 + ii;
      double v = 0.0;
      if (kk < kn && i < a.mi) {
        const int k = k0 + kk;
        v = PT ? ld_as_double<TP>(a.P, (size_t)(a.pi0 + i) * a.ldp + k)
               : ld_as_double<TP>(a.P, (size_t)k * a.ldp + a.pi0 + i);
      }
      Ps[kk][ii] = v;
    }
#pragma unroll
    for (int s = 0; s < (kChunk * kTile) / 256; ++s) {
      const int e = threadIdx.x + 256 * s;
      int kk, jj;
      if (QT) { kk = e % kChunk; jj = e / kChunk; } else { kk = e / kTile; jj = e % kTile; }
      const int j = c0 + jj;
      double v = 0.0;
      if (kk < kn && j < a.mj) {
        const int k = k0 + kk;
        v = QT ? ld_as_double<TP>(a.Q, (size_t)(a.qj0 + j) * a.ldq + k)
               : ld_as_double<TP>(a.Q, (size_t)k * a.ldq + a.qj0 + j);
      }
      Qs[kk][jj] = v;
    }
    __syncthreads();
    for (int kk = 0; kk < kn; ++kk) {
      double p[4], q[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) p[r] = Ps[kk][ty + 16 * r];
#pragma unroll
      for (int c = 0; c < 4; ++c) q[c] = Qs[kk][tx + 16 * c];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const double t = __dmul_rn(p[r], q[c]);
          acc[r][c] = SUB ? __dsub_rn(acc[r][c], t) : __dadd_rn(acc[r][c], t);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int i = r0 + ty + 16 * r, j = c0 + tx + 16 * c;
      if (i < a.mi && j < a.mj && (!a.lower || i >= j)) a.C[(size_t)(a.ci0 + i) * a.ldc + a.cj0 + j] = acc[r][c];
    }
}

// Xh[t][i] = X[t][perm[i]] / s[perm[i]]  (one fp32 division; n x K)
__global__ void k_flatten(const float* __restrict__ X, const float* __restrict__ s, const int32_t* __restrict__ perm,
                          int n, int K, float* __restrict__ Xh) {
  const size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (size_t)n * K) return;
  const int t = (int)(e / K), i = (int)(e % K);
  const int p = perm[i];
  Xh[e] = __fdiv_rn(X[(size_t)t * K + p], s[p]);
}

// d = H_00 + H_11 + ... in order; H_ii += 0.01 * (d / K), or += 1 when d is
// not positive (all-zero calibration activations: H = I).
__global__ void k_damp(double* __restrict__ H, int K) {
  __shared__ double lam;
  if (threadIdx.x == 0) {
    double d = 0.0;
    for (int i = 0; i < K; ++i) d = __dadd_rn(d, H[(size_t)i * K + i]);
    lam = (d > 0.0) ? __dmul_rn(0.01, __ddiv_rn(d, (double)K)) : 1.0;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < K; i += blockDim.x) H[(size_t)i * K + i] = __dadd_rn(H[(size_t)i * K + i], lam);
}

// The 32 x 32 diagonal block of panel j0, unblocked (one warp; lane = row).
// A pivot that is not positive sets *status.
__global__ void k_chol_diag(double* __restrict__ A, int K, int j0, int* __restrict__ status) {
  __shared__ double T[32][33];
  const int l = threadIdx.x;
  for (int c = 0; c <= l; ++c) T[l][c] = A[(size_t)(j0 + l) * K + j0 + c];
  __syncwarp();
  for (int k = 0; k < 32; ++k) {
    if (l == k) {
      const double p = T[k][k];
      if (!(p > 0.0)) atomicOr(status, 1);
      T[k][k] = __dsqrt_rn(p);
    }
    __syncwarp();
    if (l > k) T[l][k] = __ddiv_rn(T[l][k], T[k][k]);
    __syncwarp();
    if (l > k)
      for (int j = k + 1; j <= l; ++j) T[l][j] = __dsub_rn(T[l][j], __dmul_rn(T[l][k], T[j][k]));
    __syncwarp();
  }
  for (int c = 0; c <= l; ++c) A[(size_t)(j0 + l) * K + j0 + c] = T[l][c];
}

// Rows below the diagonal block of panel j0 (one thread per row): the
// panel's columns in order, each divided by its pivot and then subtracted
// (times the block's column) from the row's later panel entries.
__global__ void __launch_bounds__(128) k_chol_trsm(double* __restrict__ A, int K, int j0) {
  __shared__ double D[32][33];
  for (int e = threadIdx.x; e < 32 * 32; e += blockDim.x) {
    const int r = e / 32, c = e % 32;
    D[r][c] = (c <= r) ? A[(size_t)(j0 + r) * K + j0 + c] : 0.0;
  }
  __syncthreads();
  const int i = j0 + 32 + blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= K) return;
  double* row = A + (size_t)i * K + j0;
  double t[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) t[c] = row[c];
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    const double x = __ddiv_rn(t[c], D[c][c]);
    t[c] = x;
#pragma unroll
    for (int c2 = c + 1; c2 < 32; ++c2) t[c2] = __dsub_rn(t[c2], __dmul_rn(x, D[c2][c]));
  }
#pragma unroll
  for (int c = 0; c < 32; ++c) row[c] = t[c];
}

// Forward substitution, panel of rows [i0, i0 + 32) of V (in place over the
// right-hand side B, which starts as the identity); one thread per column
// k < i0 + 32.
__global__ void __launch_bounds__(128) k_inv_panel(const double* __restrict__ L, double* __restrict__ B, int K,
                                                    int i0) {
  __shared__ double D[32][33];
  for (int e = threadIdx.x; e < 32 * 32; e += blockDim.x) {
    const int r = e / 32, c = e % 32;
    D[r][c] = (c <= r) ? L[(size_t)(i0 + r) * K + i0 + c] : 0.0;
  }
  __syncthreads();
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= i0 + 32) return;
  double t[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) t[c] = B[(size_t)(i0 + c) * K + k];
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    const double v = __ddiv_rn(t[c], D[c][c]);
    t[c] = v;
#pragma unroll
    for (int c2 = c + 1; c2 < 32; ++c2) t[c2] = __dsub_rn(t[c2], __dmul_rn(D[c2][c], v));
  }
#pragma unroll
  for (int c = 0; c < 32; ++c) B[(size_t)(i0 + c) * K + k] = t[c];
}

__global__ void k_identity(double* __restrict__ B, int K) {
  const size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (size_t)K * K) return;
  B[e] = (e / K == e % K) ? 1.0 : 0.0;
}

// U[i][j] = L2[j][i] for j >= i, else 0 (fp32 copy rounded once; fp64 copy
// optional).
__global__ void k_upper_from_lower(const double* __restrict__ L2, int K, float* __restrict__ U32,
                                   double* __restrict__ U64) {
  const size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (size_t)K * K) return;
  const int i = (int)(e / K), j = (int)(e % K);
  const double v = (j >= i) ? L2[(size_t)j * K + i] : 0.0;
  if (U32) U32[e] = __double2float_rn(v);
  if (U64) U64[e] = v;
}

constexpr int kUStage = 64;  // rows of U and E staged per shared-memory pass

// GPTQ on one weight.  A CTA owns 32 output channels; in each block of 32
// rows, thread (t, lane) holds row b0 + t of channel n = 32 * blockIdx.x +
// lane, starting from W^[b0 + t, n] as the round-to-nearest path computes it:
//   1. the errors of the earlier rows i = r .. b0 - 1, in order:
//      w -= u_{i, b0+t} * e_i (staged 64 rows at a time through shared
//      memory when U fits in L2: measured 2-3x faster at K = 4096, but 3x
//      slower at K = 11008, where U streams from DRAM);
//   2. the block's rows in order: row t2 takes its code
//      code = clamp(rint(w * (7 / amax)), -7, 7) and, when b0 + t2 >= r, its
//      scaled error e = (w - code * sw) / u_{t2, t2}; the later rows of the
//      block then lose u_{t2, t} * e;
//   3. the 32 codes of each channel are packed as in the RTN path.
// Each entry therefore receives its updates in increasing row order, every
// fp32 operation rounded once.  amax is the column's maximum before any
// update (sw = amax / 7).  E (K x N) keeps the scaled errors of rows >= r.
template <bool STAGE>
__global__ void __launch_bounds__(1024) k_gptq_pack_w(prep::WeightView w, const float* __restrict__ s,
                                                       const int32_t* __restrict__ perm, int K, int r,
                                                       const float* __restrict__ amax_col,
                                                       const float* __restrict__ U, float* __restrict__ E,
                                                       uint8_t* __restrict__ wq) {
  __shared__ float ub[32][33];  // U over the block's rows and columns
  __shared__ float es[32][33];  // the block's scaled errors [row][channel]
  __shared__ int qs[32][33];    // the block's codes [row][channel]
  __shared__ float us[kUStage][33];  // U rows i of a stage, the block's columns
  __shared__ float eh[kUStage][32];  // scaled errors of those rows, this CTA's channels
  const int t = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = blockIdx.x * 32 + lane;
  const bool live = n < w.N;
  const float amax = live ? amax_col[n] : 0.f;
  const float sw = __fdiv_rn(amax, 7.f);
  for (int b0 = 0; b0 < K; b0 += 32) {
    float x = live ? prep::w_hat(w, s, perm, b0 + t, n) : 0.f;
    // earlier rows' errors in order: staged kUStage rows at a time through
    // shared memory (STAGE, U in L2), else read directly, every warp on its
    // own (more loads in flight when U comes from DRAM)
    if (STAGE) {
      for (int i0 = r; i0 < b0; i0 += kUStage) {
        const int ni = min(kUStage, b0 - i0);
        __syncthreads();
        for (int e = threadIdx.x; e < kUStage * 32; e += blockDim.x) {
          const int ii = e >> 5, c = e & 31;
          const bool in = ii < ni;
          us[ii][c] = in ? U[(size_t)(i0 + ii) * K + b0 + c] : 0.f;
          eh[ii][c] = (in && blockIdx.x * 32 + c < w.N) ? E[(size_t)(i0 + ii) * w.N + blockIdx.x * 32 + c] : 0.f;
        }
        __syncthreads();
        for (int ii = 0; ii < ni; ++ii) x = __fsub_rn(x, __fmul_rn(us[ii][t], eh[ii][lane]));
      }
    } else if (live) {
      const float* ucol = U + b0 + t;  // u_{i, b0+t}: the same for the whole warp
#pragma unroll 8
      for (int i = r; i < b0; ++i) x = __fsub_rn(x, __fmul_rn(ucol[(size_t)i * K], E[(size_t)i * w.N + n]));
    }
    __syncthreads();
    ub[t][lane] = U[(size_t)(b0 + t) * K + b0 + lane];
    __syncthreads();
    for (int t2 = 0; t2 < 32; ++t2) {
      if (t == t2) {
        const int q = prep::code4(x, amax);
        qs[t][lane] = q;
        if (b0 + t >= r) {
          const float err = __fdiv_rn(__fsub_rn(x, __fmul_rn((float)q, sw)), ub[t][t]);
          es[t][lane] = err;
          if (live) E[(size_t)(b0 + t) * w.N + n] = err;
        }
      }
      __syncthreads();
      if (t > t2 && b0 + t2 >= r) x = __fsub_rn(x, __fmul_rn(ub[t2][t], es[t2][lane]));
    }
    if (t == 0 && live) {
      int q[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) q[k] = qs[k][lane];
      *reinterpret_cast<uint4*>(wq + (size_t)n * (K / 2) + b0 / 2) = prep::pack_run32(q);
    }
    __syncthreads();
  }
}

}  // namespace gptq
}  // namespace serq
