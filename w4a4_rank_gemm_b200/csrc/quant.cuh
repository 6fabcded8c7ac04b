// Per-token activation quantize-and-pack (the X^_q of SERQ's linear), the
// fused SiLU*mul + quantize of a folded MLP block, and the runtime
// flatten-and-permute helper for layers whose producer was not folded.
//
// One CTA per token row.  The row is held in registers between the absmax
// reduction and the quantization, so HBM sees one read of X and one write of
// the codes.  Arithmetic is fp32 with one rounding per operation.
#pragma once
#include "common.cuh"

namespace serq {
namespace quant {

constexpr int kMaxThreads = 256;
constexpr int kMaxChunks = 8;  // 8-element chunks held per thread (K <= 16384)

// ------------------------------------------------------------- row loaders
// Each loader returns 8 consecutive fp32 values of row m starting at k0.
struct LoadBF16 {
  const __nv_bfloat16* X;
  int ld;
  __device__ __forceinline__ void operator()(int m, int k0, float (&v)[8]) const {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(X + (size_t)m * ld + k0));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
};

struct LoadF32 {
  const float* X;
  int ld;
  __device__ __forceinline__ void operator()(int m, int k0, float (&v)[8]) const {
    const float4* p = reinterpret_cast<const float4*>(X + (size_t)m * ld + k0);
    const float4 a = __ldg(p), b = __ldg(p + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
};

// e^x in fp32: Cody & Waite argument reduction x = k ln2 + r with ln 2 split
// into a 9-bit head (so k * head is exact) and a tail, a degree-7 Taylor
// polynomial for e^r (|r| <= ln2/2, truncation error < 1e-8 relative) by
// Horner's rule with separate multiply and add, then an exact scaling by 2^k.
// Saturates to +inf above 88 and to 0 below -88.
__device__ __forceinline__ float exp_cw(float x) {
  if (x > 88.f) return __int_as_float(0x7f800000);
  if (x < -88.f) return 0.f;
  const float kLog2e = (float)1.44269504088896341;
  const float kLn2Hi = 0.693359375f;
  const float kLn2Lo = (float)(0.69314718055994530942 - 0.693359375);
  const float k = rintf(__fmul_rn(x, kLog2e));
  const float r = __fsub_rn(__fsub_rn(x, __fmul_rn(k, kLn2Hi)), __fmul_rn(k, kLn2Lo));
  float p = (float)(1.0 / 5040.0);
  p = __fadd_rn(__fmul_rn(p, r), (float)(1.0 / 720.0));
  p = __fadd_rn(__fmul_rn(p, r), (float)(1.0 / 120.0));
  p = __fadd_rn(__fmul_rn(p, r), (float)(1.0 / 24.0));
  p = __fadd_rn(__fmul_rn(p, r), (float)(1.0 / 6.0));
  p = __fadd_rn(__fmul_rn(p, r), 0.5f);
  p = __fadd_rn(__fmul_rn(p, r), 1.0f);
  p = __fadd_rn(__fmul_rn(p, r), 1.0f);
  return ldexpf(p, (int)k);
}

// h = silu(g) * u = g / (1 + e^-g) * u, fp32.
struct LoadSiluMul {
  const __nv_bfloat16* G;
  const __nv_bfloat16* U;
  int ld;
  __device__ __forceinline__ void operator()(int m, int k0, float (&v)[8]) const {
    float g[8], u[8];
    LoadBF16{G, ld}(m, k0, g);
    LoadBF16{U, ld}(m, k0, u);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float den = __fadd_rn(1.f, exp_cw(-g[i]));
      v[i] = __fmul_rn(__fdiv_rn(g[i], den), u[i]);
    }
  }
};

// ------------------------------------------------------- quantize one row
// Q = 7 (packed INT4 output, K/2 bytes per row) or 127 (int8, K bytes).
template <int Q, int CH, class Loader>
__global__ void __launch_bounds__(kMaxThreads) k_quant_rows(Loader load, int K, uint8_t* __restrict__ Xq,
                                                           float* __restrict__ sx) {
  const int m = blockIdx.x;
  const int nchunks = K >> 3;
  float v[CH][8];
  float amax = 0.f;
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    const int ch = threadIdx.x + c * blockDim.x;
    if (ch < nchunks) {
      load(m, ch * 8, v[c]);
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[c][i]));
    }
  }
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  __shared__ float red[kMaxThreads / 32];
  const int nw = blockDim.x >> 5;
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
  for (int i = 1; i < nw; ++i) amax = fmaxf(amax, red[i]);

  const float qf = (float)Q;
  const float inv = (amax > 0.f) ? __fdiv_rn(qf, amax) : 0.f;
  if (threadIdx.x == 0) sx[m] = __fdiv_rn(amax, qf);
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    const int ch = threadIdx.x + c * blockDim.x;
    if (ch < nchunks) {
      int q[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int t = __float2int_rn(__fmul_rn(v[c][i], inv));
        q[i] = max(-Q, min(Q, t));
      }
      if (Q == 7) {
        uint32_t w = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) w |= (uint32_t)(q[i] & 0xF) << (4 * i);
        *reinterpret_cast<uint32_t*>(Xq + (size_t)m * (K >> 1) + ch * 4) = w;
      } else {
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          lo |= (uint32_t)(q[i] & 0xFF) << (8 * i);
          hi |= (uint32_t)(q[i + 4] & 0xFF) << (8 * i);
        }
        *reinterpret_cast<uint2*>(Xq + (size_t)m * K + ch * 8) = make_uint2(lo, hi);
      }
    }
  }
}

// Launch helper: block size = min(256, chunks rounded up to a warp), CH =
// chunks per thread (1, 2, 4 or 8).
template <int Q, class Loader>
inline cudaError_t launch_quant_rows(const Loader& load, int M, int K, uint8_t* Xq, float* sx,
                                     cudaStream_t st) {
  const int nchunks = K / 8;
  int threads = ((nchunks + 31) / 32) * 32;
  if (threads > kMaxThreads) threads = kMaxThreads;
  const int ch = (nchunks + threads - 1) / threads;
  dim3 grid(M), block(threads);
  if (ch <= 1)
    k_quant_rows<Q, 1, Loader><<<grid, block, 0, st>>>(load, K, Xq, sx);
  else if (ch <= 2)
    k_quant_rows<Q, 2, Loader><<<grid, block, 0, st>>>(load, K, Xq, sx);
  else if (ch <= 4)
    k_quant_rows<Q, 4, Loader><<<grid, block, 0, st>>>(load, K, Xq, sx);
  else if (ch <= kMaxChunks)
    k_quant_rows<Q, 8, Loader><<<grid, block, 0, st>>>(load, K, Xq, sx);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

// --------------------------------------------------- flatten and permute
// Xh[m, i] = X[m, perm[i]] / s[perm[i]]  (fp32 divide, stored bf16 or fp32)
template <bool IN_BF16, bool OUT_BF16>
__global__ void k_flatten_permute(const void* __restrict__ X, int ldx, const int32_t* __restrict__ perm,
                                  const float* __restrict__ s, int M, int K, void* __restrict__ Xh, int ldxh) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const int m = blockIdx.y;
  if (i >= K || m >= M) return;
  const int j = perm[i];
  float x;
  if (IN_BF16)
    x = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(X)[(size_t)m * ldx + j]);
  else
    x = reinterpret_cast<const float*>(X)[(size_t)m * ldx + j];
  const float y = __fdiv_rn(x, s[j]);
  if (OUT_BF16)
    reinterpret_cast<__nv_bfloat16*>(Xh)[(size_t)m * ldxh + i] = __float2bfloat16_rn(y);
  else
    reinterpret_cast<float*>(Xh)[(size_t)m * ldxh + i] = y;
}

}  // namespace quant
}  // namespace serq
