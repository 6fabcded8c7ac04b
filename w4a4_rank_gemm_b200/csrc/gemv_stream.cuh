// Decode-regime SERQ linear, streaming form (M <= 32 tokens): the packed
// INT4 weights are read from HBM exactly once, spread evenly over every SM.
//
// Work split.  The output channels of the launch (the layers of a group
// concatenated) are cut into one contiguous range per CTA at a granularity
// of two channels, so every SM streams the same number of weight bytes
// (o_proj at 4096 channels: 27 or 28 channels per SM instead of one or two
// 16-channel items).  Inside a CTA the range is covered by 16-channel tiles
// (rows past the range are never read and never written) and every tile by
// "units" of 256 k: 16 rows x 128 bytes of packed weights (2 KB), first the
// residual's units (R, k < r) and then the main product's.  The CTA's units,
// tile by tile, are dealt round-robin to its warps.
//
// Each warp streams its own units through a private ring of kDepth slots
// with 16-byte cp.async copies (each lane copies exactly the 64 bytes it
// will read back, so a lane waits only for its own copies and no barrier is
// involved); the first kDepth units are requested before the kernel waits
// for the grid it depends on, since no earlier kernel writes the weights.
// The activation codes of all tokens are staged once per CTA (one bulk copy
// per token row, on an mbarrier) at a row pitch that makes every fragment
// load conflict-free.
//
// Arithmetic: mma.sync m16n8k32 s8 with the weight rows as the 16-row A
// operand and the tokens as the 8-column B operand (one n8 tile per eight
// tokens, so M <= 8 wastes nothing).  k-order inside a 128-k chunk: lane
// (g, t) holds run t of its rows (32 codes in 16 bytes, byte j = code j |
// code j + 16 << 4); MMA step i takes word i: its low nibbles are codes
// 4i..4i+3 and its high nibbles codes 16+4i..16+4i+3 of the run, and the
// activation fragment of the same lane and step covers the same codes, so
// every product pairs equal k.  Nibbles are widened to int8 x16 by two mask
// operations (INT8 activations are used as they are), hence the final
// shift by 8 (W4A4) or 4 (W4A8).  The residual units accumulate
// X~_{s,q} Q(R) into a second accumulator from the same activation codes
// (SERQ notes, key design 2: one matmul on the salient channels).
//
// A warp adds its partial sums of a tile into the tile's shared
// accumulators whenever it moves on to another tile, then adds the number
// of units it covered to the tile's counter; the warp that completes the
// count applies the epilogue sx * (sw * acc0 + sR * acc1) for the tile's
// channels and every token.  No warp waits for another.
#pragma once
#include "common.cuh"

namespace serq {
namespace gs {

constexpr int kDepth = 4;         // ring slots per warp
constexpr int kUnitK = 256;       // k per unit
constexpr int kUnitBytes = 2048;  // 16 rows x 128 bytes
constexpr int kMaxWarps = 16;
constexpr int kMaxGroup = 4;
constexpr int kMaxTokenTiles = 4;  // n8 tiles: M <= 32

struct Layer {
  const uint8_t* Wq;  // N x K/2 packed INT4
  const uint8_t* Rq;  // N x rpad/2 packed INT4 (null when rpad = 0)
  const float* sw;
  const float* sr;
  __nv_bfloat16* Y;
  int ldy;
  int32_t* acc0;
  int32_t* acc1;
  int N;
  int base;  // first channel of this layer in the launch's channel list
};

struct Args {
  const uint8_t* Xq;
  const float* sx;
  // Two-factor comparator: the residual units read these codes (M x rpad,
  // packed like Xq, W4A4) and scale their product by sxr; null for SERQ,
  // whose residual reuses the first r columns of Xq.
  const uint8_t* Xr;
  const float* sxr;
  int M, K, rpad;
  int C;     // channels of the launch (all layers)
  int nlayers;
  Layer lo[kMaxGroup];
};

// Computed on the host.
struct Plan {
  int warps;       // warps per CTA
  int grid;        // CTAs
  int xbytes;      // activation bytes per token row (K/2 or K)
  int xpitch;      // staged row pitch
  int xrows;       // staged rows (8 per token tile)
  int xrpitch;     // staged row pitch of Xr (0 without it)
  int units_main;  // 256-k units of W per tile
  int units_res;   // 256-k units of R per tile
  int tmax;        // most tiles one CTA covers
  int smem;        // dynamic shared memory bytes
  // Failure-detection test only (zero in every other launch): the activation
  // copies are not issued, so the bounded wait for them runs out after
  // wait_ns and the kernel takes its abort path.
  int withhold_x;
  unsigned long long wait_ns;
};

template <int NTT>
struct AccLayout {
  static constexpr int kInts = 2 * NTT * 4 * 32;  // [acc0 / acc1][token tile][fragment q][lane]
};

__host__ __device__ inline int chan_begin(int c, int C, int grid) {
  return 2 * (int)(((long long)c * (C >> 1)) / grid);
}

__device__ __forceinline__ void mma_s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                       uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t lo_x16(uint32_t w) { return (w << 4) & 0xF0F0F0F0u; }
__device__ __forceinline__ uint32_t hi_x16(uint32_t w) { return w & 0xF0F0F0F0u; }
__device__ __forceinline__ uint32_t word(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

__device__ __forceinline__ int layer_of(const Args& p, int ch) {
  int l = 0;
#pragma unroll
  for (int i = 1; i < kMaxGroup; ++i)
    if (i < p.nlayers && ch >= p.lo[i].base) l = i;
  return l;
}

// Requests unit v of this CTA into ring slot `slot` (this lane's 4 pieces).
__device__ __forceinline__ void issue_unit(const Args& p, const Plan& pl, uint8_t* slot_base, int c0, int c1,
                                           int v, int g, int t, int lane) {
  const int ut = pl.units_res + pl.units_main;
  const int tile = v / ut, ku = v - tile * ut;
  const bool res = ku < pl.units_res;
  const int kunit = res ? ku : ku - pl.units_res;
  const int rowbytes = res ? (p.rpad >> 1) : (p.K >> 1);
#pragma unroll
  for (int hs = 0; hs < 2; ++hs) {
    const int ch = c0 + tile * 16 + g + 8 * hs;
    const uint8_t* src = p.lo[0].Wq;
    bool row_ok = ch < c1;
    if (row_ok) {
      const Layer& lo = p.lo[layer_of(p, ch)];
      src = (res ? lo.Rq : lo.Wq) + (size_t)(ch - lo.base) * rowbytes;
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int kb = (kunit * 2 + h) * 64 + 16 * t;
      const bool ok = row_ok && kb < rowbytes;
      cp_async16_zfill(slot_base + (h * 2 + hs) * 512 + lane * 16, ok ? src + kb : p.lo[0].Wq, ok ? 16u : 0u);
    }
  }
}

// The MMAs of one unit: w = this lane's pieces [chunk h][row g / g + 8].
template <int NTT, bool A8>
__device__ __forceinline__ void unit_mma(const uint4 (&w)[4], const uint8_t* xs, int xpitch, int xc0, int nch,
                                         int g, int t, int (&acc)[NTT][4]) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    if (h < nch) {
      const int xc = xc0 + h;
      uint4 xa[NTT], xb[NTT];
#pragma unroll
      for (int nt = 0; nt < NTT; ++nt) {
        const uint8_t* row = xs + (nt * 8 + g) * xpitch;
        if (A8) {
          xa[nt] = *reinterpret_cast<const uint4*>(row + xc * 128 + 32 * t);
          xb[nt] = *reinterpret_cast<const uint4*>(row + xc * 128 + 32 * t + 16);
        } else {
          xa[nt] = *reinterpret_cast<const uint4*>(row + xc * 64 + 16 * t);
          xb[nt] = xa[nt];
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t u = word(w[h * 2 + 0], i), v = word(w[h * 2 + 1], i);
        const uint32_t a0 = lo_x16(u), a1 = lo_x16(v), a2 = hi_x16(u), a3 = hi_x16(v);
#pragma unroll
        for (int nt = 0; nt < NTT; ++nt) {
          uint32_t b0, b1;
          if (A8) {
            b0 = word(xa[nt], i);
            b1 = word(xb[nt], i);
          } else {
            b0 = lo_x16(word(xa[nt], i));
            b1 = hi_x16(word(xa[nt], i));
          }
          mma_s8(acc[nt], a0, a1, a2, a3, b0, b1);
        }
      }
    }
  }
}

// Epilogue of one tile by one warp: every (token, channel) of the tile.
// The scales come from shared memory: ssw / ssr hold sw and sR of the CTA's
// channels (staged at the start), ssx / ssxr the tokens' scales.
template <int NTT, bool A8, bool ACC>
__device__ __forceinline__ void tile_epilogue(const Args& p, const int* acc, int ch0, int c0, int c1,
                                              const float* ssw, const float* ssr, const float* ssx,
                                              const float* ssxr, int lane) {
  constexpr int kShift = A8 ? 4 : 8;
  const bool two = p.sxr != nullptr;
#pragma unroll 4
  for (int idx = lane; idx < p.M * 16; idx += 32) {
    const int m = idx >> 4, cl = idx & 15;
    const int ch = ch0 + cl;
    if (ch >= c1) continue;
    const int g = cl & 7, hi = cl >> 3, nt = m >> 3, t = (m & 7) >> 1, q = hi * 2 + (m & 1);
    const int ln = g * 4 + t;
    const int a0 = acc[((0 * NTT + nt) * 4 + q) * 32 + ln] >> kShift;
    const int a1 = acc[((1 * NTT + nt) * 4 + q) * 32 + ln] >> kShift;
    const Layer& lo = p.lo[layer_of(p, ch)];
    const int col = ch - lo.base;
    if (ACC) {
      lo.acc0[(size_t)m * lo.N + col] = a0;
      lo.acc1[(size_t)m * lo.N + col] = a1;
    } else {
      const float sw = ssw[ch - c0], sr = ssr[ch - c0], sx = ssx[m];
      const float y = two ? fmaf(sx * sw, (float)a0, ssxr[m] * (sr * (float)a1)) : sx * fmaf(sw, (float)a0, sr * (float)a1);
      lo.Y[(size_t)m * lo.ldy + col] = __float2bfloat16_rn(y);
    }
  }
}

template <int NTT, bool A8, bool ACC>
__global__ void __launch_bounds__(kMaxWarps * 32, 1) k_gemv(const __grid_constant__ Args p, const Plan pl) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  uint8_t* xs = sm;                                                  // [xrows][xpitch]
  uint8_t* xr = xs + pl.xrows * pl.xpitch;                           // [xrows][xrpitch] (comparator only)
  uint8_t* ring = xr + pl.xrows * pl.xrpitch;                        // [warp][slot][4 pieces][32 lanes][16 B]
  int* acc = reinterpret_cast<int*>(ring + pl.warps * kDepth * kUnitBytes);  // [tile][AccLayout]
  int* cnt = acc + pl.tmax * AccLayout<NTT>::kInts;                  // [tile] units added
  float* ssw = reinterpret_cast<float*>(cnt + ((pl.tmax + 1) & ~1));  // [tmax * 16] sw of the CTA's channels
  float* ssr = ssw + pl.tmax * 16;                                   // [tmax * 16] sR
  float* ssx = ssr + pl.tmax * 16;                                   // [xrows] sx
  float* ssxr = ssx + pl.xrows;                                      // [xrows] residual scale (comparator)
  uint64_t* xbar = reinterpret_cast<uint64_t*>(ssxr + pl.xrows);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(xbar + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int c0 = chan_begin(blockIdx.x, p.C, pl.grid), c1 = chan_begin(blockIdx.x + 1, p.C, pl.grid);
  const int tiles = (c1 - c0 + 15) >> 4;
  const int ut = pl.units_res + pl.units_main;
  const int units = tiles * ut;
  const int nw = (warp < units) ? (units - warp + pl.warps - 1) / pl.warps : 0;  // this warp's units
  uint8_t* my_ring = ring + warp * kDepth * kUnitBytes;

  // Weights first: no earlier kernel writes them.
#pragma unroll
  for (int s = 0; s < kDepth; ++s) {
    if (s < nw) issue_unit(p, pl, my_ring + s * kUnitBytes, c0, c1, warp + s * pl.warps, g, t, lane);
    cp_async_commit();
  }

  // Shared accumulators, counters, the activation rows' zero padding.
  for (int i = threadIdx.x; i < tiles * AccLayout<NTT>::kInts; i += blockDim.x) acc[i] = 0;
  for (int i = threadIdx.x; i < tiles; i += blockDim.x) cnt[i] = 0;
  if (!ACC) {
    // sw and sR of this CTA's channels (static data: read before the wait)
    for (int i = threadIdx.x; i < c1 - c0; i += blockDim.x) {
      const Layer& lo = p.lo[layer_of(p, c0 + i)];
      ssw[i] = __ldg(lo.sw + (c0 + i - lo.base));
      ssr[i] = __ldg(lo.sr + (c0 + i - lo.base));
    }
  }
  {
    const int tail = pl.xpitch - pl.xbytes;  // bytes after each copied row
    const int words_row = pl.xpitch >> 2;
    for (int i = threadIdx.x; i < pl.xrows * words_row; i += blockDim.x) {
      const int m = i / words_row, b = (i - m * words_row) * 4;
      if (m >= p.M || b >= pl.xpitch - tail) reinterpret_cast<uint32_t*>(xs)[i] = 0u;
    }
    const int rbytes = p.rpad >> 1, words_r = pl.xrpitch >> 2;
    for (int i = threadIdx.x; i < pl.xrows * words_r; i += blockDim.x) {
      const int m = i / words_r, b = (i - m * words_r) * 4;
      if (m >= p.M || b >= rbytes) reinterpret_cast<uint32_t*>(xr)[i] = 0u;
    }
  }
  if (threadIdx.x == 0) {
    mbar_init(xbar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  grid_dep_launch();  // the next kernel in the stream may be scheduled
  grid_dep_wait();    // activations, sx and the outputs come after the grid this one depends on
  if (threadIdx.x == 0 && !pl.withhold_x) {
    const uint32_t rbytes = (uint32_t)(p.rpad >> 1);
    mbar_arrive_expect_tx(xbar, (uint32_t)(p.M * pl.xbytes) + (pl.xrpitch ? (uint32_t)p.M * rbytes : 0u));
    for (int m = 0; m < p.M; ++m) bulk_load(xs + m * pl.xpitch, p.Xq + (size_t)m * pl.xbytes, pl.xbytes, xbar);
    if (pl.xrpitch)
      for (int m = 0; m < p.M; ++m) bulk_load(xr + m * pl.xrpitch, p.Xr + (size_t)m * rbytes, rbytes, xbar);
  }
  if (!ACC) {
    for (int i = threadIdx.x; i < p.M; i += blockDim.x) {
      ssx[i] = __ldg(p.sx + i);
      if (p.sxr) ssxr[i] = __ldg(p.sxr + i);
    }
  }
  __syncthreads();
  const bool ok = mbar_wait(xbar, 0, abort_flag, kDevTimeoutUnpack, pl.wait_ns ? pl.wait_ns : kWaitLimitNs);

  if (ok) {
    const int kl_main = p.K, kl_res = p.rpad;
    int acc0[NTT][4], acc1[NTT][4];
#pragma unroll
    for (int nt = 0; nt < NTT; ++nt)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc0[nt][q] = acc1[nt][q] = 0;
    int cur = -1, cur_units = 0;
    bool had0 = false, had1 = false;

    auto flush = [&]() {
      int* a = acc + cur * AccLayout<NTT>::kInts;
#pragma unroll
      for (int nt = 0; nt < NTT; ++nt)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (had0) atomicAdd(&a[((0 * NTT + nt) * 4 + q) * 32 + lane], acc0[nt][q]);
          if (had1) atomicAdd(&a[((1 * NTT + nt) * 4 + q) * 32 + lane], acc1[nt][q]);
          acc0[nt][q] = acc1[nt][q] = 0;
        }
      __syncwarp();
      int last = 0;
      if (lane == 0) {
        __threadfence_block();
        last = (atomicAdd(&cnt[cur], cur_units) + cur_units == ut);
      }
      last = __shfl_sync(0xffffffffu, last, 0);
      if (last) {
        __threadfence_block();
        tile_epilogue<NTT, A8, ACC>(p, a, c0 + cur * 16, c0, c1, ssw, ssr, ssx, ssxr, lane);
      }
      cur_units = 0;
      had0 = had1 = false;
    };

    for (int j = 0; j < nw; ++j) {
      const int v = warp + j * pl.warps;
      const int tile = v / ut, ku = v - tile * ut;
      if (tile != cur) {
        if (cur >= 0) flush();
        cur = tile;
      }
      cp_async_wait_group<kDepth - 1>();  // this lane's copies of unit j have landed
      const uint8_t* slot = my_ring + (j % kDepth) * kUnitBytes;
      uint4 w[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) w[q] = *reinterpret_cast<const uint4*>(slot + q * 512 + lane * 16);
      __syncwarp();  // orders this lane's reads of the slot before its refill
      if (j + kDepth < nw)
        issue_unit(p, pl, my_ring + (j % kDepth) * kUnitBytes, c0, c1, v + kDepth * pl.warps, g, t, lane);
      cp_async_commit();
      const bool res = ku < pl.units_res;
      const int kunit = res ? ku : ku - pl.units_res;
      const int left = (res ? kl_res : kl_main) - kunit * kUnitK;
      const int nch = left >= 256 ? 2 : (left + 127) >> 7;
      if (res) {
        if (pl.xrpitch)
          unit_mma<NTT, A8>(w, xr, pl.xrpitch, kunit * 2, nch, g, t, acc1);
        else
          unit_mma<NTT, A8>(w, xs, pl.xpitch, kunit * 2, nch, g, t, acc1);
        had1 = true;
      } else {
        unit_mma<NTT, A8>(w, xs, pl.xpitch, kunit * 2, nch, g, t, acc0);
        had0 = true;
      }
      ++cur_units;
    }
    if (cur >= 0) flush();
  }
  cp_async_wait_all();
  __syncthreads();
  if (*abort_flag) {
    if (threadIdx.x == 0) {
      // let the activation copies already issued land before shared memory is released
      const unsigned long long t0 = global_ns();
      while (global_ns() - t0 < 100000ull) {
      }
    }
  }
}

// Host plan: the largest warp count whose shared memory fits.  Returns false
// when even four warps do not fit (large K with many tokens).
template <int NTT, bool A8>
inline bool make_plan(const Args& p, int sms, int max_smem, Plan& pl) {
  pl.xbytes = A8 ? p.K : p.K / 2;
  pl.units_main = (p.K + kUnitK - 1) / kUnitK;
  pl.units_res = (p.rpad + kUnitK - 1) / kUnitK;
  const int xrow = pl.units_main * (A8 ? 256 : 128);  // whole units, zero past K
  pl.xpitch = xrow + (A8 ? 16 : 64);                   // rows g, g + 1 in opposite bank halves
  pl.xrows = 8 * NTT;
  // comparator's residual codes: whole units, rows g, g + 1 in opposite bank halves
  pl.xrpitch = (p.Xr && !A8) ? pl.units_res * 128 + 64 : 0;
  int grid = (p.C + 15) / 16;
  if (grid > sms) grid = sms;
  if (grid < 1) grid = 1;
  pl.grid = grid;
  int most = 0;
  for (int c = 0; c < grid; ++c) {
    const int n = chan_begin(c + 1, p.C, grid) - chan_begin(c, p.C, grid);
    if (n > most) most = n;
  }
  pl.tmax = (most + 15) / 16;
  const int fixed = 128 + pl.xrows * (pl.xpitch + pl.xrpitch) + pl.tmax * AccLayout<NTT>::kInts * 4 +
                    ((pl.tmax + 1) & ~1) * 4 + pl.tmax * 16 * 8 + pl.xrows * 8 + 16;
  for (int w = kMaxWarps; w >= 4; w -= 4) {
    const int bytes = fixed + w * kDepth * kUnitBytes;
    if (bytes <= max_smem) {
      pl.warps = w;
      pl.smem = bytes;
      return true;
    }
  }
  return false;
}

template <int NTT, bool A8, bool ACC>
inline cudaError_t launch_ntt(const Args& p, int sms, int max_smem, cudaStream_t st, unsigned long long fault_wait_ns) {
  Plan pl;
  if (!make_plan<NTT, A8>(p, sms, max_smem, pl)) return cudaErrorInvalidValue;
  pl.withhold_x = fault_wait_ns ? 1 : 0;
  pl.wait_ns = fault_wait_ns;
  auto kern = k_gemv<NTT, A8, ACC>;
  cudaError_t e = serq::smem_limit(reinterpret_cast<const void*>(kern), pl.smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)pl.grid);
  cfg.blockDim = dim3((unsigned)(pl.warps * 32));
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p, pl);
}

// Whether the streaming kernel takes this launch (else the caller uses the
// item-ring kernel).
template <bool A8>
inline bool fits(const Args& p, int sms, int max_smem) {
  Plan pl = {};
  const int ntt = (p.M + 7) / 8;
  if (ntt < 1 || ntt > kMaxTokenTiles) return false;
  switch (ntt) {
    case 1: return make_plan<1, A8>(p, sms, max_smem, pl);
    case 2: return make_plan<2, A8>(p, sms, max_smem, pl);
    default: return make_plan<4, A8>(p, sms, max_smem, pl);
  }
}

// fault_wait_ns: zero, or (failure-detection test) withhold the activation
// copies and give the wait for them this limit.
template <bool A8, bool ACC>
inline cudaError_t launch(const Args& p, int sms, int max_smem, cudaStream_t st, unsigned long long fault_wait_ns = 0) {
  const int ntt = (p.M + 7) / 8;
  switch (ntt) {
    case 1: return launch_ntt<1, A8, ACC>(p, sms, max_smem, st, fault_wait_ns);
    case 2: return launch_ntt<2, A8, ACC>(p, sms, max_smem, st, fault_wait_ns);
    case 3:
    case 4: return launch_ntt<4, A8, ACC>(p, sms, max_smem, st, fault_wait_ns);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace gs
}  // namespace serq
