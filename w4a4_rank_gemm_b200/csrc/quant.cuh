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
// A loader fetches the raw bytes of 8 consecutive elements of row m at k0
// (`load`) and turns them into fp32 (`value`).  The raw form is what the
// quantizer keeps in registers between its two uses of the row.
struct LoadBF16 {
  static constexpr int kWords = 1;  // uint4 per 8 elements
  const __nv_bfloat16* X;
  int ld;
  __device__ __forceinline__ void load(int m, int k0, uint4 (&r)[kWords]) const {
    r[0] = __ldg(reinterpret_cast<const uint4*>(X + (size_t)m * ld + k0));
  }
  __device__ __forceinline__ static void bf16x8(const uint4& u, float (&v)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
  __device__ __forceinline__ void value(const uint4 (&r)[kWords], float (&v)[8]) const { bf16x8(r[0], v); }
  __device__ __forceinline__ void finalize(uint4 (&)[kWords]) const {}
};

struct LoadF32 {
  static constexpr int kWords = 2;
  const float* X;
  int ld;
  __device__ __forceinline__ void load(int m, int k0, uint4 (&r)[kWords]) const {
    const uint4* p = reinterpret_cast<const uint4*>(X + (size_t)m * ld + k0);
    r[0] = __ldg(p);
    r[1] = __ldg(p + 1);
  }
  __device__ __forceinline__ void value(const uint4 (&r)[kWords], float (&v)[8]) const {
    v[0] = __uint_as_float(r[0].x); v[1] = __uint_as_float(r[0].y);
    v[2] = __uint_as_float(r[0].z); v[3] = __uint_as_float(r[0].w);
    v[4] = __uint_as_float(r[1].x); v[5] = __uint_as_float(r[1].y);
    v[6] = __uint_as_float(r[1].z); v[7] = __uint_as_float(r[1].w);
  }
  __device__ __forceinline__ void finalize(uint4 (&)[kWords]) const {}
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
  // p * 2^k, correctly rounded: a power-of-two factor is exact while the
  // product stays normal; below that the last multiply rounds once.
  const int ki = (int)k;  // -127 .. 127
  if (ki >= -125) return __fmul_rn(p, __int_as_float((ki + 127) << 23));
  return __fmul_rn(__fmul_rn(p, __int_as_float((ki + 129) << 23)), 0.25f);
}

// h = silu(g) * u = g / (1 + e^-g) * u, fp32.  `finalize` replaces the raw
// (g, u) bf16 pairs by the 8 fp32 values of h in the same two words, so h is
// computed once per element.
struct LoadSiluMul {
  static constexpr int kWords = 2;
  const __nv_bfloat16* G;
  const __nv_bfloat16* U;
  int ld;
  __device__ __forceinline__ void load(int m, int k0, uint4 (&r)[kWords]) const {
    r[0] = __ldg(reinterpret_cast<const uint4*>(G + (size_t)m * ld + k0));
    r[1] = __ldg(reinterpret_cast<const uint4*>(U + (size_t)m * ld + k0));
  }
  __device__ __forceinline__ void finalize(uint4 (&r)[kWords]) const {
    float g[8], u[8], h[8];
    LoadBF16::bf16x8(r[0], g);
    LoadBF16::bf16x8(r[1], u);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float den = __fadd_rn(1.f, exp_cw(-g[i]));
      h[i] = __fmul_rn(__fdiv_rn(g[i], den), u[i]);
    }
    r[0] = make_uint4(__float_as_uint(h[0]), __float_as_uint(h[1]), __float_as_uint(h[2]), __float_as_uint(h[3]));
    r[1] = make_uint4(__float_as_uint(h[4]), __float_as_uint(h[5]), __float_as_uint(h[6]), __float_as_uint(h[7]));
  }
  __device__ __forceinline__ void value(const uint4 (&r)[kWords], float (&v)[8]) const {
    v[0] = __uint_as_float(r[0].x); v[1] = __uint_as_float(r[0].y);
    v[2] = __uint_as_float(r[0].z); v[3] = __uint_as_float(r[0].w);
    v[4] = __uint_as_float(r[1].x); v[5] = __uint_as_float(r[1].y);
    v[6] = __uint_as_float(r[1].z); v[7] = __uint_as_float(r[1].w);
  }
};

// ------------------------------------------------ codes of one 32-code run
// code = clamp(rint(x * inv), -Q, Q).  |x| <= amax and inv = RN(Q/amax)
// give |RN(x * inv)| <= Q (1 + 2^-23), which rounds to at most Q, so the
// clamp never binds.  Adding 1.5 * 2^23 rounds to the nearest integer
// (ties to even) exactly for |y| < 2^22, and the sum's low mantissa bits
// are then the code in two's complement: a nibble or byte is a mask away.
// (The product and the sum stay two roundings; a fused multiply-add would
// round differently at ties.)
//
// Output, Q = 7: the packed INT4 format, every run of 32 codes is 16 bytes
// (dst[0]) with byte j = code j (low nibble) | code j+16 (high nibble).
// Q = 127: int8 codes in natural order (dst[0], dst[1]).
template <int Q>
__device__ __forceinline__ void quantize_run(const float (&v)[32], float inv, uint4* dst) {
  const float kMagic = 12582912.0f;  // 1.5 * 2^23
  uint32_t t[32];
#pragma unroll
  for (int e = 0; e < 32; ++e) t[e] = __float_as_uint(__fadd_rn(__fmul_rn(v[e], inv), kMagic));
  if (Q == 7) {
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t x = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) x |= ((t[4 * k + j] & 0xFu) | ((t[4 * k + j + 16] & 0xFu) << 4)) << (8 * j);
      w[k] = x;
    }
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
  } else {
    uint32_t w[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      w[j] = __byte_perm(__byte_perm(t[4 * j], t[4 * j + 1], 0x0040), __byte_perm(t[4 * j + 2], t[4 * j + 3], 0x0040),
                         0x5410);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
}

// ------------------------------------------------------- quantize one row
// One CTA per token row; lane l of warp w owns the 32-code runs
// b = l + 32 (w + W i), i < RPL, and holds their raw input in registers, so
// HBM sees the row once: load everything, reduce the absolute maximum
// (shuffles, then shared memory across the W warps), quantize from registers.
//
// Codes as quantize_run writes them.
template <int Q, int RPL, class Loader>
__global__ void __launch_bounds__(512) k_quant_rows(Loader ld, int K, uint8_t* __restrict__ Xq,
                                                    float* __restrict__ sx, int early_launch) {
  constexpr int W = Loader::kWords;
  const int m = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int nrun = K >> 5;
  uint4 raw[RPL][4][W];
  float amax = 0.f;
  // Programmatic dependent launch: the input (written by the previous
  // kernel) is read only after that kernel completed.  A grid that is all
  // resident at once lets the next kernel in right away (its weight prefetch
  // overlaps this one); a larger grid only at its end, so the next kernel
  // does not take SMs from rows still to come.
  if (early_launch) grid_dep_launch();
  grid_dep_wait();
#pragma unroll
  for (int i = 0; i < RPL; ++i) {
    const int b = lane + 32 * (warp + nw * i);
    if (b < nrun) {
#pragma unroll
      for (int c = 0; c < 4; ++c) ld.load(m, b * 32 + c * 8, raw[i][c]);
    }
  }
#pragma unroll
  for (int i = 0; i < RPL; ++i) {
    const int b = lane + 32 * (warp + nw * i);
    if (b < nrun) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float v[8];
        ld.finalize(raw[i][c]);
        ld.value(raw[i][c], v);
#pragma unroll
        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[e]));
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (nw > 1) {
    __shared__ float red[16];
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    amax = red[0];
    for (int i = 1; i < nw; ++i) amax = fmaxf(amax, red[i]);
  }

  const float qf = (float)Q;
  const float inv = (amax > 0.f) ? __fdiv_rn(qf, amax) : 0.f;
  if (threadIdx.x == 0) sx[m] = __fdiv_rn(amax, qf);

#pragma unroll
  for (int i = 0; i < RPL; ++i) {
    const int b = lane + 32 * (warp + nw * i);
    if (b >= nrun) continue;
    float v[32];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float u[8];
      ld.value(raw[i][c], u);
#pragma unroll
      for (int e = 0; e < 8; ++e) v[c * 8 + e] = u[e];
    }
    uint8_t* dst = (Q == 7) ? Xq + (size_t)m * (K >> 1) + b * 16 : Xq + (size_t)m * K + b * 32;
    quantize_run<Q>(v, inv, reinterpret_cast<uint4*>(dst));
  }
  if (!early_launch) grid_dep_launch();
}

// Runs per lane held in registers: 2 for one-word inputs (bf16), 1 for
// two-word inputs (fp32, or the two bf16 inputs of silu*mul); warps per row
// = ceil(runs / (32 * RPL)) <= 16, so K <= 32768 (bf16) / 16384.  Fewer
// runs per lane mean fewer registers and more resident warps: measured on
// the B200, the silu*mul quantize of a 4096 x 11008 block takes 83 us with
// one run per lane against 120 us with two (it is bound by the exact fp32
// SiLU arithmetic, ~46 instructions per element, and needs the warps to
// hide its latency), and a 2048 x 11008 bf16 quantize 12.0 against 13.3 us
// with two runs against four.
#ifndef SERQ_Q_RPL1
#define SERQ_Q_RPL1 2
#endif
#ifndef SERQ_Q_RPL2
#define SERQ_Q_RPL2 1
#endif
template <int Q, class Loader>
inline cudaError_t launch_quant_rows(const Loader& ld, int M, int K, uint8_t* Xq, float* sx, cudaStream_t st) {
  constexpr int RPL = (Loader::kWords == 1) ? SERQ_Q_RPL1 : SERQ_Q_RPL2;
  const int nrun = K / 32;
  const int warps = (nrun + 32 * RPL - 1) / (32 * RPL);
  if (warps > 16) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(M);
  cfg.blockDim = dim3(warps * 32);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int sms = 148, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int early = (M <= 4 * sms) ? 1 : 0;  // the whole grid is resident at once
  return cudaLaunchKernelEx(&cfg, k_quant_rows<Q, RPL, Loader>, ld, K, Xq, sx, early);
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
