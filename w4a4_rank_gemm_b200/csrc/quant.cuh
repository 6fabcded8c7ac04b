// Per-token activation quantize-and-pack (the X^_q of SERQ's linear), the
// fused SiLU*mul + quantize of a folded MLP block, and the runtime
// flatten-and-permute helper for layers whose producer was not folded.
//
// Arithmetic is fp32 with one rounding per operation, so the codes are
// reproducible bit for bit.
#pragma once
#include "common.cuh"

namespace serq {
namespace quant {


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
// One warp per token row, two passes: the first reads the row for its
// absolute maximum, the second reads it again (from L2, the row was just
// streamed) and writes the codes.  HBM sees X once; many rows are in flight
// per SM, so the loads of different rows overlap.
//
// Output, Q = 7: the packed INT4 format, every run of 32 codes is 16 bytes
// with byte j = code j (low nibble) | code j+16 (high nibble).  Q = 127: int8
// codes in natural order.
constexpr int kRowsPerCta = 8;

template <int Q, class Loader>
__global__ void __launch_bounds__(kRowsPerCta * 32) k_quant_rows(Loader load, int M, int K, uint8_t* __restrict__ Xq,
                                                                float* __restrict__ sx) {
  const int m = blockIdx.x * kRowsPerCta + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (m >= M) return;
  const int nrun = K >> 5;  // runs of 32

  float amax = 0.f;
  for (int b = lane; b < nrun; b += 32) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float v[8];
      load(m, b * 32 + c * 8, v);
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));

  const float qf = (float)Q;
  const float inv = (amax > 0.f) ? __fdiv_rn(qf, amax) : 0.f;
  if (lane == 0) sx[m] = __fdiv_rn(amax, qf);

  for (int b = lane; b < nrun; b += 32) {
    int q[32];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float v[8];
      load(m, b * 32 + c * 8, v);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int t = __float2int_rn(__fmul_rn(v[i], inv));
        q[c * 8 + i] = max(-Q, min(Q, t));
      }
    }
    if (Q == 7) {
      uint32_t w[4] = {0, 0, 0, 0};
#pragma unroll
      for (int j = 0; j < 16; ++j)
        w[j >> 2] |= ((uint32_t)(q[j] & 0xF) | ((uint32_t)(q[j + 16] & 0xF) << 4)) << (8 * (j & 3));
      *reinterpret_cast<uint4*>(Xq + (size_t)m * (K >> 1) + b * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    } else {
      uint32_t w[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        w[j] = (uint32_t)(q[4 * j] & 0xFF) | ((uint32_t)(q[4 * j + 1] & 0xFF) << 8) |
               ((uint32_t)(q[4 * j + 2] & 0xFF) << 16) | ((uint32_t)(q[4 * j + 3] & 0xFF) << 24);
      uint4* dst = reinterpret_cast<uint4*>(Xq + (size_t)m * K + b * 32);
      dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
      dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
  }
}

template <int Q, class Loader>
inline cudaError_t launch_quant_rows(const Loader& load, int M, int K, uint8_t* Xq, float* sx,
                                     cudaStream_t st) {
  const int ctas = (M + kRowsPerCta - 1) / kRowsPerCta;
  k_quant_rows<Q, Loader><<<ctas, kRowsPerCta * 32, 0, st>>>(load, M, K, Xq, sx);
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
