// Decode-regime SERQ linear (M <= 64 tokens): memory-bound, so the goal is
// to stream the packed INT4 weights from HBM once at full bandwidth.
//
// Each CTA owns 8 output channels; its 8 warps split K.  Every thread loads
// 16 bytes (32 nibbles) of one weight row per 128-k segment straight into
// registers, unpacks them (nibble -> int8 x16) and feeds them, with the
// matching activation codes, to m16n8k32 integer tensor-core MMAs: no shared
// memory for weights, no re-read.  The segments that cover the first r
// columns also load the same 16 bytes of the compensator R and accumulate
// X~_{s,q} Q(R) into a second accumulator from the activation fragments
// already in registers (SERQ notes key design 2: one matmul on the salient
// channels).  The 8 warps' partial sums are reduced in shared memory and the
// epilogue applies sx * (sw * acc0 + sR * acc1).
//
// k-order inside a segment: thread t of a quad covers the 32-code run
// k in [128 seg + 32 t, +32).  MMA step s takes word s of the run's 16
// packed bytes: its low nibbles (k = base + 4s + {0..3}) form the first
// K-half fragment and its high nibbles (k = base + 16 + 4s + {0..3}) the
// second.  Activations use the identical mapping, so every product pairs
// equal k.
#pragma once
#include "common.cuh"

namespace serq {
namespace decode {

constexpr int kWarps = 8;
constexpr int kMaxTiles = 4;  // 16-row tiles: M <= 64

struct Args {
  const uint8_t* Xq;
  const float* sx;
  int M, K, N, rpad;
  const uint8_t* Wq;
  const uint8_t* Rq;
  const float* sw;
  const float* sr;
  __nv_bfloat16* Y;
  int ldy;
  int32_t* acc0;
  int32_t* acc1;
};

__device__ __forceinline__ void mma_s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ld_stream(const uint8_t* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t lo_x16(uint32_t w) { return (w << 4) & 0xF0F0F0F0u; }
__device__ __forceinline__ uint32_t hi_x16(uint32_t w) { return w & 0xF0F0F0F0u; }

// Operands of one 128-k segment for this thread.
template <int MT, bool A8>
struct Seg {
  uint4 w, r;
  uint4 a[MT][2][A8 ? 2 : 1];  // [tile][row g / g+8][16-byte piece]
};

template <int MT, bool A8>
__device__ __forceinline__ void load_seg(const Args& p, int seg, int g, int t, int n0, bool with_r,
                                         Seg<MT, A8>& s) {
  const uint4 z = make_uint4(0, 0, 0, 0);
  const int wb = seg * 64 + t * 16;  // byte offset in a packed weight row
  s.w = (wb < (p.K >> 1)) ? ld_stream(p.Wq + (size_t)(n0 + g) * (p.K >> 1) + wb) : z;
  s.r = (with_r && wb < (p.rpad >> 1)) ? ld_stream(p.Rq + (size_t)(n0 + g) * (p.rpad >> 1) + wb) : z;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = mt * 16 + g + 8 * h;
      if (A8) {
        const int ab = seg * 128 + t * 32;
        const bool ok = row < p.M && ab < p.K;
        const uint8_t* src = p.Xq + (size_t)row * p.K + ab;
        s.a[mt][h][0] = ok ? __ldg(reinterpret_cast<const uint4*>(src)) : z;
        s.a[mt][h][A8 ? 1 : 0] = ok ? __ldg(reinterpret_cast<const uint4*>(src + 16)) : z;
      } else {
        const bool ok = row < p.M && wb < (p.K >> 1);
        s.a[mt][h][0] = ok ? __ldg(reinterpret_cast<const uint4*>(p.Xq + (size_t)row * (p.K >> 1) + wb)) : z;
      }
    }
  }
}

template <int MT, bool A8>
__device__ __forceinline__ void mma_seg(const Seg<MT, A8>& s, bool with_r, int (&acc0)[MT][4],
                                        int (&acc1)[MT][4]) {
  const uint32_t wv[4] = {s.w.x, s.w.y, s.w.z, s.w.w};
  const uint32_t rv[4] = {s.r.x, s.r.y, s.r.z, s.r.w};
#pragma unroll
  for (int st = 0; st < 4; ++st) {
    const uint32_t b0 = lo_x16(wv[st]), b1 = hi_x16(wv[st]);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      uint32_t a0, a1, a2, a3;
      if (A8) {
        // int8 codes: word st of the first 16 bytes is k = base + 4 st + {0..3},
        // word st of the second 16 bytes is k = base + 16 + 4 st + {0..3}
        a0 = (&s.a[mt][0][0].x)[st];
        a2 = (&s.a[mt][0][A8 ? 1 : 0].x)[st];
        a1 = (&s.a[mt][1][0].x)[st];
        a3 = (&s.a[mt][1][A8 ? 1 : 0].x)[st];
      } else {
        const uint32_t x = (&s.a[mt][0][0].x)[st];
        const uint32_t y = (&s.a[mt][1][0].x)[st];
        a0 = lo_x16(x);
        a2 = hi_x16(x);
        a1 = lo_x16(y);
        a3 = hi_x16(y);
      }
      mma_s8(acc0[mt], a0, a1, a2, a3, b0, b1);
      if (with_r) mma_s8(acc1[mt], a0, a1, a2, a3, lo_x16(rv[st]), hi_x16(rv[st]));
    }
  }
}

template <int MT, bool A8, bool ACC_OUT>
__global__ void __launch_bounds__(kWarps * 32) k_decode(Args p) {
  __shared__ int red[kWarps][MT][2][4][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int n0 = blockIdx.x * 8;

  const int nseg = (p.K + 127) >> 7;
  const int rseg = (p.rpad + 127) >> 7;
  const int per = nseg / kWarps, extra = nseg % kWarps;
  const int s0 = warp * per + min(warp, extra);
  const int s1 = s0 + per + (warp < extra ? 1 : 0);

  int acc0[MT][4], acc1[MT][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc0[mt][j] = acc1[mt][j] = 0;

  constexpr int U = (MT <= 2) ? 4 : 2;  // segments in flight per thread
  int seg = s0;
  for (; seg + U <= s1; seg += U) {
    Seg<MT, A8> sv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) load_seg<MT, A8>(p, seg + u, g, t, n0, seg + u < rseg, sv[u]);
#pragma unroll
    for (int u = 0; u < U; ++u) mma_seg<MT, A8>(sv[u], seg + u < rseg, acc0, acc1);
  }
  for (; seg < s1; ++seg) {
    Seg<MT, A8> sv;
    load_seg<MT, A8>(p, seg, g, t, n0, seg < rseg, sv);
    mma_seg<MT, A8>(sv, seg < rseg, acc0, acc1);
  }

#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      red[warp][mt][0][j][lane] = acc0[mt][j];
      red[warp][mt][1][j][lane] = acc1[mt][j];
    }
  __syncthreads();

  // Accumulators carry the x16 of each unpacked INT4 operand.
  constexpr int kShift = A8 ? 4 : 8;
  for (int idx = threadIdx.x; idx < MT * 128; idx += blockDim.x) {
    const int mt = idx >> 7, j = (idx >> 5) & 3, l = idx & 31;
    int s_0 = 0, s_1 = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      s_0 += red[w][mt][0][j][l];
      s_1 += red[w][mt][1][j][l];
    }
    const int row = mt * 16 + (l >> 2) + 8 * (j >> 1);
    const int col = n0 + 2 * (l & 3) + (j & 1);
    if (row >= p.M) continue;
    const int q0 = s_0 >> kShift, q1 = s_1 >> kShift;
    if (ACC_OUT) {
      p.acc0[(size_t)row * p.N + col] = q0;
      p.acc1[(size_t)row * p.N + col] = q1;
    } else {
      const float y = p.sx[row] * fmaf(p.sw[col], (float)q0, p.sr[col] * (float)q1);
      p.Y[(size_t)row * p.ldy + col] = __float2bfloat16_rn(y);
    }
  }
}

template <int MT, bool A8, bool ACC_OUT>
inline cudaError_t launch_mt(const Args& p, cudaStream_t st) {
  k_decode<MT, A8, ACC_OUT><<<p.N / 8, kWarps * 32, 0, st>>>(p);
  return cudaGetLastError();
}

template <bool A8, bool ACC_OUT>
inline cudaError_t launch(const Args& p, cudaStream_t st) {
  const int tiles = (p.M + 15) / 16;
  switch (tiles) {
    case 1: return launch_mt<1, A8, ACC_OUT>(p, st);
    case 2: return launch_mt<2, A8, ACC_OUT>(p, st);
    case 3: return launch_mt<3, A8, ACC_OUT>(p, st);
    case 4: return launch_mt<4, A8, ACC_OUT>(p, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace decode
}  // namespace serq
