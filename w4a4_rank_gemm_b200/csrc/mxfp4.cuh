// SERQ with MXFP4 codes (sm_100a): the OCP Microscaling format -- blocks of
// 32 consecutive elements along K share one power-of-two scale stored as an
// E8M0 byte, every element an FP4 E2M1 number -- for the folded weight W^,
// the compensator R and the per-token activations.  The SERQ pages name
// MXFP4 as a format the method supports and quote their Blackwell latency on
// it (gist.science (de) sections 3 "Kompatibilität" and 4 "Performance &
// Latenz"; gist.science (ja) section 2, R in 4 bits so that the whole linear
// is 4-bit integer or MXFP4 arithmetic).
//
// Conversion of a block (OCP MX v1.0, section 6.3): e = floor(log2(amax)) - 2
// (2 = the exponent of E2M1's largest normal, 6), clamped to [-127, 127]
// (-127 for an all-zero block); element = v * 2^-e rounded to the nearest
// E2M1 value, ties to the even code, beyond 6 to 6; zero is stored as +0.
// The scaling by 2^-e is exact in fp32 wherever it can change a rounding
// decision, so the codes are reproducible bit for bit.
//
// The product Y = deq(X_q) deq(W_q) + deq(X_q[:, :r]) deq(R_q) runs on
// tcgen05.mma kind::mxf4 with block scaling: the scales are applied inside
// the tensor core, so the main and the residual products accumulate into
// one fp32 TMEM accumulator and the epilogue only rounds to bf16.
#pragma once
#include "common.cuh"
#include "prepare.cuh"

namespace serq {
namespace mx {

constexpr int kBlock = 32;          // elements per scale
constexpr int kTileK = 256;         // elements of K per pipeline stage (128 bytes)
constexpr int kTileRows = 128;      // rows of a scale tile (the GEMM's M and N tile)

// Tiled scale layout the GEMM reads with one bulk copy per stage: 1 KB tiles
// of 128 rows x 8 blocks (256 elements of K), row-major over (row / 128,
// block / 8); inside a tile 8 bytes per row.  n_blocks = K / 32 (multiple
// of 8).
__host__ __device__ __forceinline__ size_t scale_offset(int row, int blk, int n_blocks) {
  return ((size_t)(row / kTileRows) * (size_t)(n_blocks / 8) + (size_t)(blk / 8)) * 1024u +
         (size_t)(row % kTileRows) * 8u + (size_t)(blk % 8);
}

// 2^e in fp32 for e in [-149, 127] (subnormal below -126).
__device__ __forceinline__ float pow2f(int e) {
  return e >= -126 ? __int_as_float((e + 127) << 23) : __int_as_float(1 << (e + 149));
}

// floor(log2(a)) - 2 clamped to [-127, 127] for finite a >= 0; -127 for 0.
// Read from the exponent field (normal) or the leading mantissa bit
// (subnormal): exact, no log.
__device__ __forceinline__ int shared_exp(float a) {
  const uint32_t b = __float_as_uint(a);
  if (b == 0u) return -127;
  const int E = (int)(b >> 23);
  const int fl = (E > 0) ? E - 127 : (31 - __clz((int)(b & 0x7FFFFFu))) - 149;
  return max(-127, fl - 2);
}

// E2M1 code of t.  Magnitudes by code 0..7: 0, .5, 1, 1.5, 2, 3, 4, 6; the
// midpoints .25 .75 1.25 1.75 2.5 3.5 5 go to the even code, so the
// comparisons alternate between <= (even code below) and < (even code
// above).
__device__ __forceinline__ uint32_t e2m1_code(float t) {
  const float a = fabsf(t);
  const uint32_t c = (uint32_t)(a > 0.25f) + (uint32_t)(a >= 0.75f) + (uint32_t)(a > 1.25f) +
                     (uint32_t)(a >= 1.75f) + (uint32_t)(a > 2.5f) + (uint32_t)(a >= 3.5f) + (uint32_t)(a > 5.f);
  return (c != 0u && t < 0.f) ? (c | 8u) : c;
}

// E2M1 value of a code (twice the magnitudes 0 1 2 3 4 6 8 12 in nibbles).
__device__ __forceinline__ float e2m1_value(uint32_t c) {
  const float v = 0.5f * (float)((0xC8643210u >> (4u * (c & 7u))) & 0xFu);
  return (c & 8u) ? -v : v;
}

// One block of 32 values -> 16 bytes (element 2j in the low nibble of byte
// j) and the shared exponent.
__device__ __forceinline__ int quant_block(const float (&v)[kBlock], uint4& packed) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < kBlock; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int e = shared_exp(amax);
  const float inv = pow2f(-e);  // -e in [-125, 127]: a normal power of two
  uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int i = 0; i < kBlock; ++i) w[i >> 3] |= e2m1_code(__fmul_rn(v[i], inv)) << (4 * (i & 7));
  packed = make_uint4(w[0], w[1], w[2], w[3]);
  return e;
}

__device__ __forceinline__ uint32_t nibble(const uint4& p, int i) {
  const uint32_t w = (i < 8) ? p.x : (i < 16) ? p.y : (i < 24) ? p.z : p.w;
  return (w >> (4 * (i & 7))) & 0xFu;
}

// ------------------------------------------------------------------ offline
// W^ per output channel n (blocks of 32 along K) and, for the blocks of the
// first rpad rows, R = W^ - deq(code) on rows < r (one fp32 subtraction; the
// dequantized value is exact) quantized the same way; R's blocks past r are
// zero.  One thread per (channel, block).
__global__ void k_quant_w(prep::WeightView w, const float* __restrict__ s, const int32_t* __restrict__ perm, int K,
                          int r, int rpad, uint8_t* __restrict__ wq, uint8_t* __restrict__ we,
                          uint8_t* __restrict__ rq, uint8_t* __restrict__ re) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  const int b = blockIdx.y;
  if (n >= w.N) return;
  float v[kBlock];
#pragma unroll
  for (int t = 0; t < kBlock; ++t) v[t] = prep::w_hat(w, s, perm, b * kBlock + t, n);
  uint4 pk;
  const int e = quant_block(v, pk);
  *reinterpret_cast<uint4*>(wq + (size_t)n * (K / 2) + (size_t)b * 16) = pk;
  we[scale_offset(n, b, K / kBlock)] = (uint8_t)(e + 127);
  if (b * kBlock < rpad) {
    float rr[kBlock];
    const bool salient = b * kBlock < r;  // r is a multiple of 32
    const float sc = pow2f(e);
#pragma unroll
    for (int t = 0; t < kBlock; ++t)
      rr[t] = salient ? __fsub_rn(v[t], __fmul_rn(e2m1_value(nibble(pk, t)), sc)) : 0.f;
    uint4 pr;
    const int er = quant_block(rr, pr);
    *reinterpret_cast<uint4*>(rq + (size_t)n * (rpad / 2) + (size_t)b * 16) = pr;
    re[scale_offset(n, b, rpad / kBlock)] = (uint8_t)(er + 127);
  }
}

// ----------------------------------------------------------------- per token
// One thread per (token, block); rows M..Mpad-1 get the all-zero block's
// scale byte 0 (their codes are never read: the GEMM's loads fill rows past
// M with zeros).
template <typename T>
__global__ void k_quant_act(const T* __restrict__ X, int M, int K, int ld, int Mpad, uint8_t* __restrict__ Xq,
                            uint8_t* __restrict__ xe) {
  const int nb = K / kBlock;
  const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long)Mpad * nb) return;
  const int m = (int)(idx / nb), b = (int)(idx % nb);
  int e = -127;
  if (m < M) {
    float v[kBlock];
    const T* src = X + (size_t)m * ld + (size_t)b * kBlock;
    if constexpr (sizeof(T) == 2) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 u = reinterpret_cast<const uint4*>(src)[q];
        const uint32_t ws[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          v[8 * q + 2 * j] = __uint_as_float(ws[j] << 16);
          v[8 * q + 2 * j + 1] = __uint_as_float(ws[j] & 0xFFFF0000u);
        }
      }
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 f = reinterpret_cast<const float4*>(src)[q];
        v[4 * q] = f.x;
        v[4 * q + 1] = f.y;
        v[4 * q + 2] = f.z;
        v[4 * q + 3] = f.w;
      }
    }
    uint4 pk;
    e = quant_block(v, pk);
    *reinterpret_cast<uint4*>(Xq + (size_t)m * (K / 2) + (size_t)b * 16) = pk;
  }
  xe[scale_offset(m, b, nb)] = (uint8_t)(e + 127);
}

// --------------------------------------------------------------------- GEMM
// One 128 x 128 output tile per CTA.  Warp 0 issues the TMA loads (codes of
// X and of W or R, 128 x 128 bytes each, 128-byte swizzle; the two 1 KB
// scale tiles by bulk copy), warp 1 the MMAs, warps 2-5 write each stage's
// scales into tensor memory and then run the epilogue.  Steps 0..K/256-1
// multiply X by W; the following rpad/256 steps multiply the same first
// activation tiles by R into the same accumulator (SERQ's single residual
// product reusing the activation codes).
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kSfCol = 128;     // scale slots: 32 columns per stage after the accumulator
constexpr int kCodeTile = 128 * 128; // bytes
constexpr int kSfTile = 1024;
constexpr int oA = 0;
constexpr int oB = oA + kStages * kCodeTile;
constexpr int oSFA = oB + kStages * kCodeTile;
constexpr int oSFB = oSFA + kStages * kSfTile;
constexpr int oBar = oSFB + kStages * kSfTile;
constexpr int oMisc = oBar + 8 * (3 * kStages + 2);
constexpr int kSmemBytes = oMisc + 16 + 1024;  // + alignment slack
constexpr uint32_t kTxBytes = 2 * kCodeTile + 2 * kSfTile;

struct Args {
  const uint8_t* xe;  // activation scales (tiled, rows padded to 128)
  const uint8_t* we;  // W^ scales (tiled)
  const uint8_t* re;  // R scales (tiled)
  __nv_bfloat16* Y;
  int ldy, M, N, K, rpad;
};

// Instruction descriptor of kind::mxf4 (dense, K = 64 per instruction):
// A and B E2M1, K-major; UE8M0 scales; both scale-factor ids 0 (bytes 0-1
// of each scale word).
__host__ __device__ constexpr uint32_t idesc_mxf4(int M, int N) {
  return (1u << 7)                       // A: E2M1
         | (1u << 10)                    // B: E2M1
         | ((uint32_t)(N >> 3) << 17)    // N / 8
         | (1u << 23)                    // scale type UE8M0
         | ((uint32_t)(M >> 4) << 24);   // M / 16
}

__device__ __forceinline__ void umma_mxf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%4], [%5], p;\n\t}\n" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
      : "memory");
}

// Scale words of one stage for the 32 TMEM lanes of warp quarter q.  The
// block-scaled MMA's sub-partition q (output rows 32q..32q+31) reads its
// scale factors from its own lane quarter only.  B's row n is read, for
// every q, from lane 32q + n % 32 at column n / 32 of the operand's slot, so
// B's words are the same in every quarter: column c holds row lane + 32c.
// A's row m = 32q + lane is read from lane m, at the slot's column m / 32
// (or its first column): A's column 0 holds the lane's own row and column
// c >= 1 row lane + 32c, which serves both.  For MMA k (elements
// 64k..64k+63 of the stage) each operand has one 4-column slot; bytes 0-1 of
// a word are the row's scales of blocks 2k and 2k+1 (scale-factor id 0),
// repeated in bytes 2-3.
template <bool A_OPERAND>
__device__ __forceinline__ void stage_scale_words(const uint8_t* sf, int q, int lane, uint32_t* w) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int row = (A_OPERAND && c == 0) ? 32 * q + lane : lane + 32 * c;
      const uint32_t b = *reinterpret_cast<const uint16_t*>(sf + row * 8 + 2 * k);
      w[4 * k + c] = b | (b << 16);
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    k_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW,
           const __grid_constant__ CUtensorMap tmR, const Args p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + oBar);
  uint64_t* full = bar;                     // codes and scales of a stage landed (tx)
  uint64_t* sf_ready = bar + kStages;       // the stage's scales are in tensor memory
  uint64_t* empty = bar + 2 * kStages;      // the stage's MMAs completed
  uint64_t* acc_full = bar + 3 * kStages;   // every MMA of the tile completed
  uint64_t* drain = acc_full + 1;           // abort path: MMAs complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + oMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + oMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * 128, m0 = blockIdx.y * 128;
  const int nkt = p.K / kTileK, nsteps = nkt + p.rpad / kTileK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&sf_ready[s], 4);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc<1>(tmem_slot, kTmemCols);
    tmem_relinquish<1>();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmW);
      tma_prefetch_desc(&tmR);
      const int xtiles = p.K / kTileK;
      for (int g = 0; g < nsteps; ++g) {
        const int s = g % kStages;
        const uint32_t ph = (uint32_t)(g / kStages) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, kDevTimeoutProducer)) break;
        const bool res = g >= nkt;
        const int j = res ? g - nkt : g;
        mbar_arrive_expect_tx(&full[s], kTxBytes);
        tma_load_2d(smem + oA + s * kCodeTile, &tmA, &full[s], j * (kTileK / 2), m0);
        tma_load_2d(smem + oB + s * kCodeTile, res ? &tmR : &tmW, &full[s], j * (kTileK / 2), n0);
        bulk_load(smem + oSFA + s * kSfTile, p.xe + ((size_t)(m0 / 128) * xtiles + j) * kSfTile, kSfTile, &full[s]);
        const uint8_t* bsf = res ? p.re + ((size_t)(n0 / 128) * (p.rpad / kTileK) + j) * kSfTile
                                 : p.we + ((size_t)(n0 / 128) * xtiles + j) * kSfTile;
        bulk_load(smem + oSFB + s * kSfTile, bsf, kSfTile, &full[s]);
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issue
    constexpr uint32_t idesc = idesc_mxf4(128, 128);
    bool ok = true;
    for (int g = 0; g < nsteps; ++g) {
      const int s = g % kStages;
      const uint32_t ph = (uint32_t)(g / kStages) & 1u;
      bool w = mbar_wait(&sf_ready[s], ph, abort_flag, kDevTimeoutMma);
      w = w && mbar_wait(&full[s], ph, abort_flag, kDevTimeoutMma);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint64_t da = umma_desc_k_sw128(smem_u32(smem + oA + s * kCodeTile));
      const uint64_t db = umma_desc_k_sw128(smem_u32(smem + oB + s * kCodeTile));
      const uint32_t sf = tmem + kSfCol + 32u * (uint32_t)s;
      if (elect_one()) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_mxf4(tmem, da + (uint64_t)(2 * k), db + (uint64_t)(2 * k), idesc, sf + 4u * k, sf + 16u + 4u * k,
                    (g > 0 || k > 0) ? 1u : 0u);
        umma_commit<1>(&empty[s]);
        if (g == nsteps - 1) umma_commit<1>(acc_full);
      }
      __syncwarp();
    }
    if (!ok) {
      if (elect_one()) {
        umma_commit<1>(drain);
        mbar_wait(drain, 0, nullptr, kDevTimeoutMma);
      }
      __syncwarp();
    }
  } else {
    // -------------------------------------------- scales, then the epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    bool ok = true;
    for (int g = 0; g < nsteps; ++g) {
      const int s = g % kStages;
      const uint32_t ph = (uint32_t)(g / kStages) & 1u;
      // full[s] of this round follows the producer's wait on empty[s] of
      // the previous one, so the slot's previous MMAs have completed
      const bool w = mbar_wait(&full[s], ph, abort_flag, kDevTimeoutEpilogue);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t words[32];
      stage_scale_words<true>(smem + oSFA + s * kSfTile, q, lane, words);
      stage_scale_words<false>(smem + oSFB + s * kSfTile, q, lane, words + 16);
      tmem_st_32x32b_x32(tmem + lane_base + kSfCol + 32u * (uint32_t)s, words);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sf_ready[s]);
    }
    if (ok) {
      const bool w = mbar_wait(acc_full, 0, abort_flag, kDevTimeoutEpilogue);
      if (__all_sync(0xffffffffu, w)) {
        tc_fence_after();
        const int row = m0 + 32 * q + lane;
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tmem + lane_base + 32u * (uint32_t)cc, r);
          tmem_ld_wait_regs(r);
          if (row < p.M) {
            uint32_t h[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
              h[j] = *reinterpret_cast<const uint32_t*>(&b2);
            }
            uint4* dst = reinterpret_cast<uint4*>(p.Y + (size_t)row * p.ldy + n0 + 32 * cc);
#pragma unroll
            for (int j = 0; j < 4; ++j) dst[j] = make_uint4(h[4 * j], h[4 * j + 1], h[4 * j + 2], h[4 * j + 3]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag && warp == 0 && lane == 0) {
    // let copies already issued land before the shared memory is released
    const unsigned long long t0 = global_ns();
    while (global_ns() - t0 < 100000ull) {
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<1>(tmem, kTmemCols);
  }
}

}  // namespace mx
}  // namespace serq
