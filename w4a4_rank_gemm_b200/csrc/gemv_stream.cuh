// Decode-regime SERQ linear, streaming form (M <= 32 tokens): the packed
// INT4 weights are read from HBM exactly once, spread evenly over every SM.
//
// Work split.  The output channels of the launch (the layers of a group
// concatenated) are cut into one contiguous range per CTA at a granularity
// of four channels, so every SM streams the same number of weight bytes
// (o_proj at 4096 channels: 24 or 28 channels per SM instead of one or two
// 16-channel items).  Inside a CTA the range is covered by 16-channel tiles
// and every tile by "units" of 512 k: 16 rows x 256 bytes of packed weights
// (4 KB), first the residual's units (R, k < r) and then the main
// product's.  (The copy engine streams 16 x 256-byte boxes at the full HBM
// rate but 16 x 128-byte boxes at about two thirds of it.)  The CTA's unit list, tile by tile, is cut into one contiguous
// run per warp, so a warp moves to another tile (and hands its partial sums
// over) at most a few times.
//
// Each warp streams its run through a private ring of kDepth slots: one
// lane issues a unit as one TMA box of 16 rows x 256 bytes, or as up to four
// boxes of 4 rows x 256 bytes where the tile leaves the CTA's range or a
// layer (boxes past the range are skipped; bytes past a row's end are
// zero-filled), completing on the slot's mbarrier, so the copy engine, not the load/store
// unit, carries the stream.  The first kDepth units are requested before
// the kernel waits for the grid it depends on, since no earlier kernel
// writes the weights.  The activation codes of all tokens and the CTA's
// sw / sR are staged once per CTA by bulk copies, the codes at a row pitch
// that makes every fragment load conflict-free.
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
// shift by 8 (W4A4) or 4 (W4A8).  Codes past K (or r) meet zero-filled
// weights, so the staged activation rows need no padding of their own.  The
// residual units accumulate X~_{s,q} Q(R) into a second accumulator from
// the same activation codes (SERQ notes, key design 2: one matmul on the
// salient channels).
//
// A warp adds its partial sums of a tile into the tile's shared
// accumulators when it moves on to another tile.  After the loop (one CTA
// barrier) the warps share the epilogues sx * (sw * acc0 + sR * acc1), a
// tile at a time, so that no warp's loop is lengthened by them.
#pragma once
#include "common.cuh"
#include "quant.cuh"

namespace serq {
namespace gs {

constexpr int kDepth = 2;         // ring slots per warp
constexpr int kUnitK = 512;       // k per unit
constexpr int kUnitRow = 256;     // bytes of one weight row in a unit (a TMA box's inner extent)
constexpr int kUnitBytes = 16 * kUnitRow;
constexpr int kBoxRows = 4;       // rows per TMA box (the channel granularity of the CTA ranges)
constexpr int kBoxBytes = kBoxRows * kUnitRow;
#ifndef SERQ_GS_WARPS
#define SERQ_GS_WARPS 16
#endif
constexpr int kMaxWarps = SERQ_GS_WARPS;  // warps per CTA when shared memory allows
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
  // Fused activation quantize (null: Xq and sx are given): the flattened,
  // permuted bf16 activations, M x K at row stride ldxh, quantized per token
  // by the CTA itself (every CTA, the same codes) into the staged rows; K <=
  // 4096 (one warp holds a row in registers).
  const __nv_bfloat16* Xh;
  int ldxh;
  int M, K, rpad;
  int C;     // channels of the launch (all layers)
  int nlayers;
  Layer lo[kMaxGroup];
};

// Per layer: the weight and the compensator as 2-D byte tensors (rows =
// output channels) read in 256-byte x 16-row boxes (a whole unit) and in
// 256-byte x 4-row boxes (the last, partial tile of a CTA's range, or a
// tile across a layer boundary).
struct Maps {
  CUtensorMap w[kMaxGroup];
  CUtensorMap r[kMaxGroup];
  CUtensorMap w16[kMaxGroup];
  CUtensorMap r16[kMaxGroup];
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
  int cmax;        // most channels one CTA covers
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

// c * (C / 4) stays below 2^31 for grid <= 1024 and C <= 2^21.
__host__ __device__ inline int chan_begin(int c, int C, int grid) {
  return kBoxRows * ((c * (C / kBoxRows)) / grid);
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

// Generic-proxy reads of shared memory before async-proxy (TMA) writes to it.
__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ int layer_of(const Args& p, int ch) {
  int l = 0;
#pragma unroll
  for (int i = 1; i < kMaxGroup; ++i)
    if (i < p.nlayers && ch >= p.lo[i].base) l = i;
  return l;
}

// A warp's position in its CTA's unit list (tile-major; within a tile the
// residual units come first).
struct Cursor {
  int tile, ku;
  __device__ __forceinline__ void next(int ut) {
    if (++ku == ut) {
      ku = 0;
      ++tile;
    }
  }
};

// Issues the unit at cursor c into `slot` (called by one lane), completing
// on bar: one 16-row box when the tile lies within the CTA's range and one
// layer, else 4-row boxes up to the end of the range.
__device__ __forceinline__ void issue_unit(const Args& p, const Maps& mp, const Plan& pl, uint8_t* slot,
                                           uint64_t* bar, const Cursor& c, int c0, int c1) {
  const bool res = c.ku < pl.units_res;
  const int x = (res ? c.ku : c.ku - pl.units_res) * kUnitRow;
  const int r0 = c0 + c.tile * 16;
  const int l0 = layer_of(p, r0);
  if (r0 + 16 <= c1 && r0 + 16 <= p.lo[l0].base + p.lo[l0].N) {
    mbar_arrive_expect_tx(bar, (uint32_t)kUnitBytes);
    tma_load_2d(slot, res ? &mp.r16[l0] : &mp.w16[l0], bar, x, r0 - p.lo[l0].base);
    return;
  }
  const int nbox = min(4, (c1 - r0) / kBoxRows);
  mbar_arrive_expect_tx(bar, (uint32_t)(nbox * kBoxBytes));
  for (int b = 0; b < nbox; ++b) {
    const int ch = r0 + b * kBoxRows;
    const int l = layer_of(p, ch);
    tma_load_2d(slot + b * kBoxBytes, res ? &mp.r[l] : &mp.w[l], bar, x, ch - p.lo[l].base);
  }
}

// Per-token quantize of one bf16 row by one warp into the staged layout
// (packed INT4 runs of 16 bytes, or INT8 codes), with the arithmetic of the
// standalone quantizer (quant::quantize_run): lane l owns the runs l, l + 32,
// l + 64, l + 96 (K <= 4096) and holds them in registers between the
// absolute maximum and the codes.
template <int Q>
__device__ __forceinline__ void quantize_row_warp(const __nv_bfloat16* row, int K, uint8_t* dst, float* sx_out,
                                                  int lane) {
  const int nrun = K >> 5;
  uint4 raw[4][4];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int b = lane + 32 * i;
    if (b < nrun)
#pragma unroll
      for (int c = 0; c < 4; ++c) raw[i][c] = __ldg(reinterpret_cast<const uint4*>(row + b * 32 + c * 8));
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int b = lane + 32 * i;
    if (b < nrun)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float v[8];
        quant::LoadBF16::bf16x8(raw[i][c], v);
#pragma unroll
        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[e]));
      }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float qf = (float)Q;
  const float inv = (amax > 0.f) ? __fdiv_rn(qf, amax) : 0.f;
  if (lane == 0) *sx_out = __fdiv_rn(amax, qf);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int b = lane + 32 * i;
    if (b < nrun) {
      float v[32];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float u[8];
        quant::LoadBF16::bf16x8(raw[i][c], u);
#pragma unroll
        for (int e = 0; e < 8; ++e) v[c * 8 + e] = u[e];
      }
      quant::quantize_run<Q>(v, inv, reinterpret_cast<uint4*>(dst + (Q == 7 ? 16 : 32) * b));
    }
  }
}

// The MMAs of one unit.  The slot holds 16 rows x 128 bytes; lane (g, t)
// reads rows g and g + 8 at run t of each 128-k chunk.
template <int NTT, bool A8>
__device__ __forceinline__ void unit_mma(const uint8_t* slot, const uint8_t* xs, int xpitch, int xc0, int nch, int g,
                                         int t, int (&acc)[NTT][4]) {
#pragma unroll
  for (int h = 0; h < kUnitRow / 64; ++h) {
    if (h < nch) {
      const int xc = xc0 + h;
      const uint4 wg = *reinterpret_cast<const uint4*>(slot + g * kUnitRow + h * 64 + 16 * t);
      const uint4 wg8 = *reinterpret_cast<const uint4*>(slot + (g + 8) * kUnitRow + h * 64 + 16 * t);
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
        const uint32_t u = word(wg, i), v = word(wg8, i);
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
// channels, ssx / ssxr the tokens' scales.
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

// 112 registers per thread (57 344 for 16 warps) leave room in the register
// file for the small CTAs of the next kernel in the stream (a per-token
// quantize), which then become resident during this grid's tail and wait
// there instead of being launched after it: measured, the 7B decode step
// at M = 16 went from 56.9 to 54.3 us with the loop's rate unchanged.
template <int NTT, bool A8, bool ACC>
__global__ void __maxnreg__(112)
    k_gemv(const __grid_constant__ Args p, const __grid_constant__ Maps mp, const Plan pl) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  uint8_t* ring = sm;                                                 // [warp][slot][16 rows][256 B]
  uint8_t* xs = ring + pl.warps * kDepth * kUnitBytes;                // [xrows][xpitch]
  uint8_t* xr = xs + pl.xrows * pl.xpitch;                            // [xrows][xrpitch] (comparator only)
  int* acc = reinterpret_cast<int*>(xr + pl.xrows * pl.xrpitch);      // [tile][AccLayout]
  float* ssw = reinterpret_cast<float*>(acc + pl.tmax * AccLayout<NTT>::kInts);  // [cmax] sw of the CTA's channels
  float* ssr = ssw + pl.cmax;                                         // [cmax] sR
  float* ssx = ssr + pl.cmax;                                         // [xrows] sx
  float* ssxr = ssx + pl.xrows;                                       // [xrows] residual scale (comparator)
  uint64_t* bars = reinterpret_cast<uint64_t*>(ssxr + pl.xrows);      // [warp][slot] unit landed
  uint64_t* xbar = bars + pl.warps * kDepth;                          // activations and scales landed
  volatile int* abort_flag = reinterpret_cast<volatile int*>(xbar + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int c0 = chan_begin(blockIdx.x, p.C, pl.grid), c1 = chan_begin(blockIdx.x + 1, p.C, pl.grid);
  const int tiles = (c1 - c0 + 15) >> 4;
  const int ut = pl.units_res + pl.units_main;
  const int units = tiles * ut;
  // this warp's contiguous run of the CTA's units
  const int u0 = (units * warp) / pl.warps;
  const int nw = (units * (warp + 1)) / pl.warps - u0;
  uint8_t* my_ring = ring + warp * kDepth * kUnitBytes;
  uint64_t* my_bars = bars + warp * kDepth;

  // (No prefetch.tensormap of the maps: measured, it delays warp 0 by about
  // 0.5 us and the launch by 0.3-0.7 us.)
  if (lane == 0) {
    for (int s = 0; s < kDepth; ++s) mbar_init(&my_bars[s], 1);
    if (warp == 0) {
      mbar_init(xbar, 1);
      *abort_flag = 0;
    }
    fence_mbar_init();
  }
  __syncwarp();
  // Weights first: no earlier kernel writes them.  The issue cursor runs
  // kDepth units ahead of the compute cursor.  One slot is requested before
  // the dependency wait and the rest after the activation copies, which
  // would otherwise queue behind every SM's whole prefetch (measured: up to
  // 0.8 us per launch).
  Cursor ic{u0 / ut, u0 % ut};
  if (lane == 0 && nw > 0) {
    issue_unit(p, mp, pl, my_ring, &my_bars[0], ic, c0, c1);
    ic.next(ut);
  }
  const uint32_t rbytes = (uint32_t)(p.rpad >> 1);
  if (threadIdx.x == 0 && !pl.withhold_x) {
    uint32_t tx = p.Xh ? 0u : (uint32_t)(p.M * pl.xbytes) + (pl.xrpitch ? (uint32_t)p.M * rbytes : 0u);
    if (!ACC) tx += 8u * (uint32_t)(c1 - c0);
    mbar_arrive_expect_tx(xbar, tx);
    if (!ACC) {
      // sw and sR of the CTA's channels (static: before the wait), one piece
      // per layer they touch (channel ranges and layer bases are multiples
      // of 4: 16-byte pieces)
      for (int l = 0; l < p.nlayers; ++l) {
        const int a = max(c0, p.lo[l].base), b = min(c1, p.lo[l].base + p.lo[l].N);
        if (a >= b) continue;
        bulk_load(ssw + (a - c0), p.lo[l].sw + (a - p.lo[l].base), 4u * (uint32_t)(b - a), xbar);
        bulk_load(ssr + (a - c0), p.lo[l].sr + (a - p.lo[l].base), 4u * (uint32_t)(b - a), xbar);
      }
    }
  }
  // Shared accumulators.
  for (int i = threadIdx.x; i < tiles * AccLayout<NTT>::kInts; i += blockDim.x) acc[i] = 0;
  __syncthreads();    // barriers initialised, accumulators zero
  grid_dep_launch();  // the next kernel in the stream may be scheduled
  grid_dep_wait();    // activations, sx and the outputs come after the grid this one depends on
  if (p.Xh) {
    // the CTA quantizes the tokens itself, one warp per row
    for (int m = warp; m < p.M; m += pl.warps)
      quantize_row_warp<A8 ? 127 : 7>(p.Xh + (size_t)m * p.ldxh, p.K, xs + m * pl.xpitch, ssx + m, lane);
  } else if (lane == 0 && !pl.withhold_x) {
    // one token row per warp, so the copies are issued side by side (the
    // expected byte count was registered before the barrier above)
    for (int m = warp; m < p.M; m += pl.warps) {
      bulk_load(xs + m * pl.xpitch, p.Xq + (size_t)m * pl.xbytes, pl.xbytes, xbar);
      if (pl.xrpitch) bulk_load(xr + m * pl.xrpitch, p.Xr + (size_t)m * rbytes, rbytes, xbar);
    }
  }
  if (lane == 0) {
    for (int s = 1; s < kDepth && s < nw; ++s) {
      issue_unit(p, mp, pl, my_ring + s * kUnitBytes, &my_bars[s], ic, c0, c1);
      ic.next(ut);
    }
  }
  if (!ACC && !p.Xh) {
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
    int cur = -1;
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
      had0 = had1 = false;
    };

    Cursor cc{u0 / ut, u0 % ut};
    bool live = true;
    for (int j = 0; j < nw; ++j, cc.next(ut)) {
      if (cc.tile != cur) {
        if (cur >= 0) flush();
        cur = cc.tile;
      }
      const int s = j % kDepth;
      if (!mbar_wait(&my_bars[s], (uint32_t)(j / kDepth) & 1u, abort_flag, kDevTimeoutUnpack)) {
        live = false;
        break;
      }
      const uint8_t* slot = my_ring + s * kUnitBytes;
      const bool res = cc.ku < pl.units_res;
      const int kunit = res ? cc.ku : cc.ku - pl.units_res;
      const int left = (res ? kl_res : kl_main) - kunit * kUnitK;
      const int nch = min(kUnitRow / 64, (left + 127) >> 7);  // 128-k chunks with codes
      if (res) {
        if (pl.xrpitch)
          unit_mma<NTT, A8>(slot, xr, pl.xrpitch, kunit * (kUnitK / 128), nch, g, t, acc1);
        else
          unit_mma<NTT, A8>(slot, xs, pl.xpitch, kunit * (kUnitK / 128), nch, g, t, acc1);
        had1 = true;
      } else {
        unit_mma<NTT, A8>(slot, xs, pl.xpitch, kunit * (kUnitK / 128), nch, g, t, acc0);
        had0 = true;
      }
      // refill this slot with the unit kDepth ahead once every lane has read it
      __syncwarp();
      if (j + kDepth < nw && lane == 0) {
        fence_proxy_async_shared();
        issue_unit(p, mp, pl, my_ring + s * kUnitBytes, &my_bars[s], ic, c0, c1);
        ic.next(ut);
      }
    }
    if (live && cur >= 0) flush();
  }
  __syncthreads();
  // Every tile's sums are complete: the warps share the epilogues (one tile
  // each in turn), so no warp's loop carries them.
  if (ok && !*abort_flag)
    for (int tile = warp; tile < tiles; tile += pl.warps)
      tile_epilogue<NTT, A8, ACC>(p, acc + tile * AccLayout<NTT>::kInts, c0 + tile * 16, c0, c1, ssw, ssr, ssx,
                                  ssxr, lane);
  if (*abort_flag && threadIdx.x == 0) {
    // let the copies already issued land before shared memory is released
    const unsigned long long t0 = global_ns();
    while (global_ns() - t0 < 100000ull) {
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
  const int xrow = pl.units_main * (A8 ? kUnitK : kUnitK / 2);  // whole units (bytes past K meet zero weights)
  pl.xpitch = xrow + (A8 ? 16 : 64);                   // rows g, g + 1 in opposite bank halves
  pl.xrows = 8 * NTT;
  // comparator's residual codes: whole units, rows g, g + 1 in opposite bank halves
  pl.xrpitch = (p.Xr && !A8) ? pl.units_res * (kUnitK / 2) + 64 : 0;
  if (p.C > (1 << 21)) return false;  // keeps chan_begin in 32-bit arithmetic
  int grid = (p.C + 15) / 16;
  if (grid > sms) grid = sms;
  if (grid < 1) grid = 1;
  pl.grid = grid;
  int most = 0;
  for (int c = 0; c < grid; ++c) {
    const int n = chan_begin(c + 1, p.C, grid) - chan_begin(c, p.C, grid);
    if (n > most) most = n;
  }
  pl.cmax = most;
  pl.tmax = (most + 15) / 16;
  const int fixed = 128 + pl.xrows * (pl.xpitch + pl.xrpitch) + pl.tmax * AccLayout<NTT>::kInts * 4 +
                    pl.cmax * 8 + pl.xrows * 8 + 8 + 16;
  for (int w = kMaxWarps; w >= 4; w -= 4) {
    const int bytes = fixed + w * (kDepth * kUnitBytes + kDepth * 8);
    if (bytes <= max_smem) {
      pl.warps = w;
      pl.smem = bytes;
      return true;
    }
  }
  return false;
}

template <int NTT, bool A8, bool ACC>
inline cudaError_t launch_ntt(const Args& p, const Maps& mp, int sms, int max_smem, cudaStream_t st,
                              unsigned long long fault_wait_ns) {
  Plan pl = {};
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
  return cudaLaunchKernelEx(&cfg, kern, p, mp, pl);
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
inline cudaError_t launch(const Args& p, const Maps& mp, int sms, int max_smem, cudaStream_t st,
                          unsigned long long fault_wait_ns = 0) {
  const int ntt = (p.M + 7) / 8;
  switch (ntt) {
    case 1: return launch_ntt<1, A8, ACC>(p, mp, sms, max_smem, st, fault_wait_ns);
    case 2: return launch_ntt<2, A8, ACC>(p, mp, sms, max_smem, st, fault_wait_ns);
    case 3:
    case 4: return launch_ntt<4, A8, ACC>(p, mp, sms, max_smem, st, fault_wait_ns);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace gs
}  // namespace serq
