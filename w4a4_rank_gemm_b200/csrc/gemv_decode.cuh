// Decode-regime SERQ linear (M <= 64 tokens): memory-bound, so the goal is
// to stream the packed INT4 weights from HBM once at full bandwidth.
//
// Work item = 16 consecutive output channels (two n8 MMA tiles, so every
// activation fragment feeds two MMAs) over all of K.
// The grid is persistent (items strided over the CTAs).  One producer warp
// keeps a ring of items in shared memory with two untiled bulk copies per
// item (its 8 weight rows and its 8 compensator rows are contiguous in HBM)
// plus the item's 8 sw and sR,
// and the ring is filled before the kernel waits for the grid it depends on:
// weights are not produced by any earlier kernel, so with programmatic
// dependent launch their streaming overlaps the previous kernel's tail.  The
// activation codes (loaded once per CTA into shared memory when they fit,
// else read from L2) and everything written come after that wait.
//
// Eight compute warps split K: each lane takes 16 bytes (32 nibbles) of one
// weight row per 128-k segment, widens them in registers (nibble -> int8
// x16) and feeds m16n8k32 integer MMAs with the matching activation codes;
// the segments that cover the first r columns also take the same 16 bytes of
// R and accumulate X~_{s,q} Q(R) into a second accumulator from the same
// activation fragments (SERQ notes key design 2: one matmul on the salient
// channels).  The warps' partial sums are added into shared accumulators of
// the item's stage and the last warp to finish applies the epilogue
// sx * (sw * acc0 + sR * acc1).
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

constexpr int kComputeWarps = 8;
constexpr int kThreads = 32 * (kComputeWarps + 1);  // + one producer warp
constexpr int kMaxTiles = 4;                        // 16-row tiles: M <= 64
constexpr int kNT = 2;                              // n8 MMA tiles per item
constexpr int kRows = 8 * kNT;                      // output channels per item
constexpr int kPad = 16;                            // bytes added to every staged activation row

// Up to four layers that read the same activation codes run as one launch;
// their items form one list (layer l's items start at item_base).
constexpr int kMaxGroup = 4;
struct LayerDec {
  const uint8_t* Wq;
  const uint8_t* Rq;
  const float* sw;
  const float* sr;
  __nv_bfloat16* Y;
  int ldy;
  int32_t* acc0;
  int32_t* acc1;
  int N, item_base;
};

struct Args {
  const uint8_t* Xq;
  const float* sx;
  int M, K, N, rpad;  // N: all layers' channels together
  int nlayers;
  LayerDec lo[kMaxGroup];
};

// Layer of list item `item` and the item's index within that layer.
__device__ __forceinline__ int layer_of(const Args& p, int item, int& li) {
  int l = 0;
#pragma unroll
  for (int i = 1; i < kMaxGroup; ++i)
    if (i < p.nlayers && item >= p.lo[i].item_base) l = i;
  li = item - p.lo[l].item_base;
  return l;
}

// Shared-memory plan, computed on the host.
struct Plan {
  int kb;           // activation bytes per token row (K/2 or K)
  int wrow, rrow;   // staged weight / compensator row bytes
  int act_pitch;    // staged activation row pitch (activations in smem)
  int act_bytes;    // M * act_pitch rounded up to 128, 0 when read from L2
  int stage_bytes;  // kRows * (wrow + rrow + 8) rounded up to 128
  int stages;
  int items;        // N / kRows
};

// Shared accumulators of one item: [nt][mt][acc0 / acc1][fragment q][lane].
template <int MT>
struct Red {
  static constexpr int kInts = kNT * MT * 2 * 4 * 32;
};

inline int smem_bytes(const Plan& pl, int mt) {
  return 128 + pl.act_bytes + pl.stages * pl.stage_bytes + pl.stages * (Red<1>::kInts * mt + 1) * 4 + 8 +
         (2 * pl.stages + 1) * 8 + 16;
}

__device__ __forceinline__ void mma_s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t lo_x16(uint32_t w) { return (w << 4) & 0xF0F0F0F0u; }
__device__ __forceinline__ uint32_t hi_x16(uint32_t w) { return w & 0xF0F0F0F0u; }

// Operands of one 128-k segment for this thread.
template <int MT, bool A8>
struct Seg {
  uint4 w[kNT], r[kNT];        // weight / compensator row g of each n8 tile
  uint4 a[MT][2][A8 ? 2 : 1];  // [tile][row g / g+8][16-byte piece]
};

template <int MT, bool A8, bool ACT_SMEM>
__device__ __forceinline__ void load_seg(const Args& p, const Plan& pl, const uint8_t* wst, const uint8_t* rst,
                                         const uint8_t* act, int seg, int g, int t, bool with_r, Seg<MT, A8>& s) {
  const uint4 z = make_uint4(0, 0, 0, 0);
  const int wb = seg * 64 + t * 16;  // byte offset in a packed weight row
#pragma unroll
  for (int nt = 0; nt < kNT; ++nt) {
    s.w[nt] = (wb < (p.K >> 1)) ? *reinterpret_cast<const uint4*>(wst + (8 * nt + g) * pl.wrow + wb) : z;
    s.r[nt] = (with_r && wb < (p.rpad >> 1)) ? *reinterpret_cast<const uint4*>(rst + (8 * nt + g) * pl.rrow + wb) : z;
  }
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = mt * 16 + g + 8 * h;
      const int ab = A8 ? seg * 128 + t * 32 : wb;
      const bool ok = row < p.M && ab < pl.kb;
#pragma unroll
      for (int c = 0; c < (A8 ? 2 : 1); ++c) {
        if (ACT_SMEM)
          s.a[mt][h][c] = ok ? *reinterpret_cast<const uint4*>(act + row * pl.act_pitch + ab + 16 * c) : z;
        else
          s.a[mt][h][c] = ok ? __ldg(reinterpret_cast<const uint4*>(p.Xq + (size_t)row * pl.kb + ab + 16 * c)) : z;
      }
    }
  }
}

// One 128-k segment: every activation fragment is widened once and used by
// the MMAs of both n8 tiles (two independent accumulator chains).
template <int MT, bool A8>
__device__ __forceinline__ void mma_seg(const Seg<MT, A8>& s, bool with_r, int (&acc0)[kNT][MT][4],
                                        int (&acc1)[kNT][MT][4]) {
#pragma unroll
  for (int st = 0; st < 4; ++st) {
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
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt) {
        const uint32_t w = (&s.w[nt].x)[st];
        mma_s8(acc0[nt][mt], a0, a1, a2, a3, lo_x16(w), hi_x16(w));
        if (with_r) {
          const uint32_t r = (&s.r[nt].x)[st];
          mma_s8(acc1[nt][mt], a0, a1, a2, a3, lo_x16(r), hi_x16(r));
        }
      }
    }
  }
}

template <int MT, bool A8, bool ACC_OUT, bool ACT_SMEM>
// Two CTAs per SM where the ring fits twice (W4A4 with one 16-token tile,
// at 96 registers a thread; the other variants would spill and keep one):
// the kernel is latency-bound, so more resident warps hide more of it.
__global__ void __launch_bounds__(kThreads, (!A8 && MT == 1) ? 2 : 1) k_decode(const Args p, const Plan pl) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  uint8_t* act = smem;                                          // [M][act_pitch]
  uint8_t* ring = smem + pl.act_bytes;                          // stages of [W rows | R rows]
  int* racc = reinterpret_cast<int*>(ring + pl.stages * pl.stage_bytes);  // [stage][mt][acc][q][lane]
  int* cnt = racc + pl.stages * Red<MT>::kInts;                 // [stage] warps done with the item
  uint64_t* bar = reinterpret_cast<uint64_t*>(cnt + ((pl.stages + 1) & ~1));
  uint64_t* full = bar;                       // item landed (tx)
  uint64_t* empty = bar + pl.stages;          // item read and its sums consumed
  uint64_t* act_full = bar + 2 * pl.stages;   // activations landed (tx)
  volatile int* abort_flag = reinterpret_cast<volatile int*>(act_full + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < pl.stages * (Red<MT>::kInts + 1); i += blockDim.x) racc[i] = 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < pl.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kComputeWarps);
    }
    mbar_init(act_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // the next kernel in the stream may be scheduled from here on
  grid_dep_launch();

  const uint32_t wbytes = (uint32_t)p.K >> 1, rbytes = (uint32_t)p.rpad >> 1;

  if (warp == kComputeWarps) {
    // ------------------------------------------------------------ producer
    bool ok = true;
    int item = blockIdx.x, j = 0;
    {
      auto issue = [&](int item, int j) -> bool {
        const int s = j % pl.stages;
        const uint32_t ph = (j / pl.stages) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, kDevTimeoutProducer)) return false;
        uint8_t* st = ring + s * pl.stage_bytes;
        int li;
        const LayerDec& lo = p.lo[layer_of(p, item, li)];
        const size_t n0 = (size_t)li * kRows;
        mbar_arrive_expect_tx(&full[s], kRows * (wbytes + rbytes + 8));
        bulk_load(st, lo.Wq + n0 * wbytes, kRows * wbytes, &full[s]);
        if (rbytes) bulk_load(st + kRows * pl.wrow, lo.Rq + n0 * rbytes, kRows * rbytes, &full[s]);
        uint8_t* sc = st + kRows * (pl.wrow + pl.rrow);  // sw, sR of the item's channels (16 each)
        bulk_load(sc, lo.sw + n0, kRows * 4, &full[s]);
        bulk_load(sc + kRows * 4, lo.sr + n0, kRows * 4, &full[s]);
        return true;
      };
      // weights first: no earlier kernel writes them.  One item before the
      // dependency wait, the rest after the activation copies, which would
      // otherwise queue behind every SM's whole prefetch.
      if (lane == 0)
        for (; ok && item < pl.items && j < 1; item += gridDim.x, ++j) ok = issue(item, j);
      grid_dep_wait();
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (ok && ACT_SMEM) {
        // the token rows' copies go out side by side, one lane each
        if (lane == 0) mbar_arrive_expect_tx(act_full, (uint32_t)(p.M * pl.kb));
        __syncwarp();
        for (int m = lane; m < p.M; m += 32)
          bulk_load(act + m * pl.act_pitch, p.Xq + (size_t)m * pl.kb, pl.kb, act_full);
      }
      if (lane == 0)
        for (; ok && item < pl.items; item += gridDim.x, ++j) ok = issue(item, j);
    }
  } else {
    // ------------------------------------------------------- compute warps
    // Each warp adds its partial sums of an item into the stage's shared
    // accumulators; the last of the eight to finish the item (stage counter)
    // applies the epilogue, clears the accumulators and releases the stage.
    // No warp waits for another.
    grid_dep_wait();  // sx and (from L2) the activation codes; Y after it
    const int g = lane >> 2, t = lane & 3;
    const int nseg = (p.K + 127) >> 7;
    const int rseg = (p.rpad + 127) >> 7;
    const int per = nseg / kComputeWarps, extra = nseg % kComputeWarps;
    const int s0 = warp * per + min(warp, extra);
    const int s1 = s0 + per + (warp < extra ? 1 : 0);
    constexpr int kShift = A8 ? 4 : 8;  // the x16 of each widened INT4 operand
    // Epilogue operands: sx in registers (loaded once), sw and sR of an
    // item's channels in its stage.  No global load is outstanding at the
    // shared-memory fences below, so they do not wait on HBM.
    float sxr[MT][2];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int row = mt * 16 + g + 8 * hh;
        sxr[mt][hh] = (!ACC_OUT && row < p.M) ? __ldg(p.sx + row) : 0.f;
      }
    bool ok = !ACT_SMEM || mbar_wait(act_full, 0, abort_flag, kDevTimeoutUnpack);
    int j = 0;
    for (int item = blockIdx.x; ok && item < pl.items; item += gridDim.x, ++j) {
      const int s = j % pl.stages;
      const uint32_t ph = (j / pl.stages) & 1;
      if (!mbar_wait(&full[s], ph, abort_flag, kDevTimeoutUnpack)) { ok = false; break; }
      const uint8_t* wst = ring + s * pl.stage_bytes;
      const uint8_t* rst = wst + kRows * pl.wrow;
      int acc0[kNT][MT][4], acc1[kNT][MT][4];
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
          for (int q = 0; q < 4; ++q) acc0[nt][mt][q] = acc1[nt][mt][q] = 0;
      int seg = s0;
      if (MT <= 2) {  // two segments' shared-memory loads in flight
        for (; seg + 2 <= s1; seg += 2) {
          Seg<MT, A8> sa, sb;
          load_seg<MT, A8, ACT_SMEM>(p, pl, wst, rst, act, seg, g, t, seg < rseg, sa);
          load_seg<MT, A8, ACT_SMEM>(p, pl, wst, rst, act, seg + 1, g, t, seg + 1 < rseg, sb);
          mma_seg<MT, A8>(sa, seg < rseg, acc0, acc1);
          mma_seg<MT, A8>(sb, seg + 1 < rseg, acc0, acc1);
        }
      }
      for (; seg < s1; ++seg) {
        Seg<MT, A8> sa;
        load_seg<MT, A8, ACT_SMEM>(p, pl, wst, rst, act, seg, g, t, seg < rseg, sa);
        mma_seg<MT, A8>(sa, seg < rseg, acc0, acc1);
      }
      int* ra = racc + s * Red<MT>::kInts;
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            atomicAdd(&ra[(((nt * MT + mt) * 2 + 0) * 4 + q) * 32 + lane], acc0[nt][mt][q]);
            atomicAdd(&ra[(((nt * MT + mt) * 2 + 1) * 4 + q) * 32 + lane], acc1[nt][mt][q]);
          }
      __syncwarp();
      int last = 0;
      if (lane == 0) {
        __threadfence_block();
        last = (atomicAdd(&cnt[s], 1) == kComputeWarps - 1);
      }
      last = __shfl_sync(0xffffffffu, last, 0);
      if (last) {
        __threadfence_block();
        const float* sc = reinterpret_cast<const float*>(wst + kRows * (pl.wrow + pl.rrow));
        int li;
        const LayerDec& lo = p.lo[layer_of(p, item, li)];
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) {
          const int col = li * kRows + 8 * nt + 2 * t;  // this lane's two output channels of its layer
          const float2 sw2 = *reinterpret_cast<const float2*>(sc + 8 * nt + 2 * t);
          const float2 sr2 = *reinterpret_cast<const float2*>(sc + kRows + 8 * nt + 2 * t);
#pragma unroll
          for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const int row = mt * 16 + g + 8 * hh;
              int* e0 = &ra[(((nt * MT + mt) * 2 + 0) * 4 + 2 * hh) * 32 + lane];
              int* e1 = &ra[(((nt * MT + mt) * 2 + 1) * 4 + 2 * hh) * 32 + lane];
              const int a00 = e0[0] >> kShift, a01 = e0[32] >> kShift;  // columns col, col + 1
              const int a10 = e1[0] >> kShift, a11 = e1[32] >> kShift;
              e0[0] = 0; e0[32] = 0; e1[0] = 0; e1[32] = 0;
              if (row >= p.M) continue;
              if (ACC_OUT) {
                *reinterpret_cast<int2*>(lo.acc0 + (size_t)row * lo.N + col) = make_int2(a00, a01);
                *reinterpret_cast<int2*>(lo.acc1 + (size_t)row * lo.N + col) = make_int2(a10, a11);
              } else {
                const float sxm = sxr[mt][hh];
                const float y0 = sxm * fmaf(sw2.x, (float)a00, sr2.x * (float)a10);
                const float y1 = sxm * fmaf(sw2.y, (float)a01, sr2.y * (float)a11);
                *reinterpret_cast<__nv_bfloat162*>(lo.Y + (size_t)row * lo.ldy + col) = __floats2bfloat162_rn(y0, y1);
              }
            }
        }
        if (lane == 0) cnt[s] = 0;
        __threadfence_block();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);  // the stage (weights and sums) may be refilled
    }
  }
  __syncthreads();
  if (*abort_flag && threadIdx.x == kComputeWarps * 32) {
    // let bulk copies already issued land before shared memory is released
    const unsigned long long t0 = global_ns();
    while (global_ns() - t0 < 100000ull) {
    }
  }
}

// Ring depth: two items, or one when two do not fit next to the activations
// (activations go to shared memory when that leaves 2 stages).  A deeper ring
// requests all of a CTA's items at once; they then land interleaved and the
// first is complete only near the end, so the compute cannot overlap the
// loads (measured at M = 16: gate_proj 11.2 us with 2 stages, 12.2 with 6).
inline bool make_plan(const Args& p, bool a8, int mt, int max_smem, Plan& pl) {
  pl.kb = a8 ? p.K : p.K / 2;
  pl.wrow = p.K / 2;
  pl.rrow = p.rpad / 2;
  pl.stage_bytes = (kRows * (pl.wrow + pl.rrow + 8) + 127) & ~127;  // + sw, sR of the item's channels
  pl.items = p.N / kRows;
  pl.act_pitch = pl.kb + kPad;
  const int per_stage = pl.stage_bytes + Red<1>::kInts * mt * 4 + 4 + 16;  // ring, sums, counter, 2 barriers
  const int fixed = 128 + 8 + 16 + 8;
  const int act = (p.M * pl.act_pitch + 127) & ~127;
  auto stages_for = [&](int a) { return (max_smem - fixed - a) / per_stage; };
  pl.act_bytes = (stages_for(act) >= 2) ? act : 0;
  pl.stages = stages_for(pl.act_bytes);
  if (pl.stages > 2) pl.stages = 2;
  return pl.stages >= 1;  // one stage (K >= 14336 at W4A8) still works, unoverlapped
}

template <int MT, bool A8, bool ACC_OUT, bool ACT_SMEM>
inline cudaError_t launch_mt(const Args& p, const Plan& pl, int sms, cudaStream_t st) {
  auto kern = k_decode<MT, A8, ACC_OUT, ACT_SMEM>;
  const int bytes = smem_bytes(pl, MT);
  cudaError_t e = serq::smem_limit(reinterpret_cast<const void*>(kern), bytes);
  if (e != cudaSuccess) return e;
  // persistent: as many CTAs as are resident at once (one or two per SM)
  int per_sm = 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, bytes) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  if (per_sm > 2) per_sm = 2;
  const int ctas = pl.items < sms * per_sm ? pl.items : sms * per_sm;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ctas);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = bytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p, pl);
}

template <int MT, bool A8, bool ACC_OUT>
inline cudaError_t launch_tiles(const Args& p, const Plan& pl, int sms, cudaStream_t st) {
  return pl.act_bytes ? launch_mt<MT, A8, ACC_OUT, true>(p, pl, sms, st)
                      : launch_mt<MT, A8, ACC_OUT, false>(p, pl, sms, st);
}

template <bool A8, bool ACC_OUT>
inline cudaError_t launch(const Args& p, int sms, int max_smem, cudaStream_t st) {
  const int tiles = (p.M + 15) / 16;
  Plan pl;
  if (tiles < 1 || tiles > kMaxTiles || !make_plan(p, A8, tiles, max_smem, pl)) return cudaErrorInvalidValue;
  switch (tiles) {
    case 1: return launch_tiles<1, A8, ACC_OUT>(p, pl, sms, st);
    case 2: return launch_tiles<2, A8, ACC_OUT>(p, pl, sms, st);
    case 3: return launch_tiles<3, A8, ACC_OUT>(p, pl, sms, st);
    default: return launch_tiles<4, A8, ACC_OUT>(p, pl, sms, st);
  }
}

}  // namespace decode
}  // namespace serq
