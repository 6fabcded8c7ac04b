// Prefill-regime SERQ linear on the 5th-generation tensor cores (sm_100a):
//
//   acc0 = Xq Wq^T            (all K columns)
//   acc1 = Xq[:, :r] Rq^T     (the r salient columns; SERQ notes key design 2)
//   Y    = sx * (sw * acc0 + sR * acc1)   -> bf16
//
// CG = 1: one CTA computes a 128 x BN output tile.
// CG = 2: a cluster of two CTAs computes a 256 x BN tile with
//   tcgen05.mma.cta_group::2 (M = 256): each CTA holds its 128 rows of X and
//   half (BN/2 rows) of W, and its 128 x BN slice of both accumulators in its
//   own TMEM.  Each SM then stages and widens half the weight tile, and the
//   tensor cores of both SMs share every weight byte they read from shared
//   memory (no TMA multicast is involved: each CTA loads its own halves).
//
// Warp roles (per CTA):
//   warp 0      TMA producer: packed INT4 tiles of X and W (or R) -> smem
//   warp 1      TMEM owner; in CTA 0 of the pair, one thread issues the MMAs
//   warps 2..9  unpackers: packed nibbles -> int8 (x16) in the 128-byte
//               swizzled K-major layout the MMA reads; after a tile's last
//               step the same warps run its epilogue out of this CTA's TMEM
//               (bf16 tile staged in shared memory, written by TMA stores).
// The k loop runs K/128 main steps into acc0 followed by ceil(r/128)
// residual steps into acc1; a residual step reloads the matching activation
// block and takes R in place of W, so both accumulators use one pipeline.
// Both accumulators stay in TMEM (int32, exact) until the epilogue applies
// the per-token, per-channel and compensator scales separately.
//
// INT4 has no tensor-core input kind of its own, and no FP4 kind represents
// the codes -7..7 exactly, so the codes are widened to int8 in shared memory
// and multiplied by kind::i8.  The widening keeps each nibble in the high
// half of its byte (value x16), three logic ops per four codes; the factor
// 16 per widened operand leaves the accumulator exactly and is removed by a
// shift.
//
// W4A8: X arrives as int8 and is loaded by TMA straight into the swizzled
// layout; only W / R are widened.
#pragma once
#include "common.cuh"

namespace serq {
namespace tc {

constexpr int BM = 128;            // rows of X per CTA
constexpr int BK = 128;            // k per pipeline step (int8 bytes per row)
constexpr int kUnpackWarps = 8;
constexpr int kThreads = (2 + kUnpackWarps) * 32;

struct Args {
  int M, K, N, rpad;
  int nkb, nrb;  // main and residual steps
  const float* sx;
  const float* sw;
  const float* sr;
  __nv_bfloat16* Y;
  int ldy;
  int32_t* acc0;
  int32_t* acc1;
  int tiles_m, tiles_n;  // output tiles (BM * cluster rows x BN columns)
};

// k_gemm runs one launch over the output tiles of up to kMaxGroup layers that
// read the same activation codes (q/k/v, gate/up): per layer its width, the
// first tile index, its scales and its output.
constexpr int kMaxGroup = 4;
struct LayerOut {
  int N, tile_base;
  const float* sw;
  const float* sr;
  __nv_bfloat16* Y;
  int ldy;
  int32_t* acc0;
  int32_t* acc1;
};
struct GroupArgs {
  int M, K, rpad;
  int nkb, nrb;
  const float* sx;
  const float* sxr;  // two-source variant: per-row scale of the residual's activation codes
  int tiles_m;
  int nlayers, ntiles;
  LayerOut lo[kMaxGroup];
};
// Per-layer tensor maps: weights and compensator (box rows BN / CG) and the
// bf16 output (32 x 64 boxes).
struct GroupMaps {
  CUtensorMap b[kMaxGroup];
  CUtensorMap r[kMaxGroup];
  CUtensorMap y[kMaxGroup];
  CUtensorMap ar;  // activation codes of the residual steps (SERQ: the same map as the main steps)
};

// Layer of tile t and its tile index within that layer.
__device__ __forceinline__ int layer_of(const GroupArgs& p, int t, int& tl) {
  int l = 0;
#pragma unroll
  for (int i = 1; i < kMaxGroup; ++i)
    if (i < p.nlayers && t >= p.lo[i].tile_base) l = i;
  tl = t - p.lo[l].tile_base;
  return l;
}

// Shared memory: PS packed stages [A | B] written by TMA, US widened stages
// [A | B] read by the MMAs (W4A8: A is consumed straight from the packed
// stage, already in the MMA layout), per-warp epilogue scales, barriers.
// Between the last MMA of a tile and the first widening of the next, the
// widened ring is idle; the epilogue stages the bf16 output tile there for
// the TMA store.
template <int BN, bool A8, int CG>
struct Layout {
  // Ring depths, as deep as shared memory allows.  The widening warps form
  // G groups that take turns on the pipeline steps (group g % G widens step
  // g), so G steps are widened at once and each step's shared-memory round
  // trip and proxy fence overlap the others'.
  //
  // Parity waits need the waiter to be at most one phase ahead of the
  // barrier.  A group owns fixed widened slots (G divides US), so it waits on
  // their phases in order.  Packed slots are shared between groups; a group
  // waits for its packed slot only after its widened slot is free, which
  // means the MMAs of step g - US, and so the widening of every step up to
  // g - US >= g - PS, are complete: the slot's previous phase is behind it.
  static constexpr bool kBig1 = (CG == 1 && BN == 256);
  static constexpr int PS = kBig1 ? 3 : ((CG == 2 && A8) ? 6 : 5);  // packed (TMA) stages
  static constexpr int US = kBig1 ? 3 : 4;                             // widened stages
  static constexpr int G = kBig1 ? 1 : 4;
  static constexpr int kGroupWarps = kUnpackWarps / G;
  static_assert(US % G == 0 && PS >= US && kUnpackWarps % G == 0, "group ring ownership");
  static constexpr int BNL = BN / CG;                      // weight rows held by this CTA
  static constexpr int kPkA = A8 ? BM * BK : BM * BK / 2;  // A part of a packed stage
  static constexpr int kPkB = BNL * BK / 2;                // B/R part (packed INT4)
  static constexpr int kPk = kPkA + kPkB;
  static constexpr int kUnA = A8 ? 0 : BM * BK;            // A part of a widened stage
  static constexpr int kUnB = BNL * BK;
  static constexpr int kUn = kUnA + kUnB;
  static constexpr int oUn = 0;
  static constexpr int oPk = oUn + US * kUn;
  // epilogue scales: each widening warp keeps sw and sr of its BN / 2 columns
  static constexpr int oScl = oPk + PS * kPk;
  static constexpr int kSclWarp = 2 * (BN / 2) * 4;
  static constexpr int oBar = oScl + kUnpackWarps * kSclWarp;
  static constexpr int nBar = 2 * PS + 2 * US + 4;
  static constexpr int oMisc = oBar + nBar * 8;
  static constexpr int kBytes = oMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;             // slack for 1024-B alignment
  static constexpr uint32_t kTxBytes = kPk;
  static constexpr uint32_t kTmemCols = (2 * BN <= 256) ? 256 : 512;
  // widening work: rows of 64 packed bytes per stage, four 16-byte pieces each
  static constexpr int kRows = (A8 ? 0 : BM) + BNL;
  static constexpr int kPiecesPerThread = kRows * 4 / (kGroupWarps * 32);
  // output staging: boxes of 32 rows x 64 bf16 (4 KB, 128-byte swizzle),
  // (BN / 64) per TMEM lane quadrant, packed into whole widened stages
  static constexpr int kBoxBytes = 32 * 128;
  static constexpr int kBoxes = 4 * (BN / 64);
  static constexpr int kBoxesPerStage = kUn / kBoxBytes;
  static constexpr int kStgStages = (kBoxes + kBoxesPerStage - 1) / kBoxesPerStage;
  static_assert(kRows * 4 % (kGroupWarps * 32) == 0, "pieces must divide evenly");
  static_assert(kPk % 1024 == 0 && kUn % 1024 == 0 && oPk % 1024 == 0, "tiles must stay 1024-aligned");
  static_assert(kUn % kBoxBytes == 0 && kStgStages <= US, "output staging must fit the widened ring");
  static_assert(kAlloc <= 232448, "shared memory budget");
};

// Widens one 16-byte packed run (32 codes) into 32 int8 (x16) in natural k
// order: byte j of the run holds code j low and code j + 16 high, so
// (w << 4) & 0xF0F0F0F0 gives codes 4i..4i+3 of word i and w & 0xF0F0F0F0
// gives codes 16+4i..16+4i+3.
__device__ __forceinline__ void widen_run(const uint4 v, uint4& lo, uint4& hi) {
  const uint32_t m = 0xF0F0F0F0u;
  lo = make_uint4((v.x << 4) & m, (v.y << 4) & m, (v.z << 4) & m, (v.w << 4) & m);
  hi = make_uint4(v.x & m, v.y & m, v.z & m, v.w & m);
}

template <int CG>
__device__ __forceinline__ void cta_sync() {
  if (CG == 1)
    __syncthreads();
  else
    cluster_sync_all();
}

// Persistent: the grid holds at most one CTA (pair) per SM (pair of SMs),
// and CTA (pair) c takes output tiles c, c + G, c + 2G, ... (G = number of
// CTAs or pairs), M-tile fastest so that concurrent tiles share weight tiles
// in L2.  The packed and widened rings run on across tile boundaries, so the
// next tile's operands stream in while the epilogue drains the accumulators.
//
// TMEM holds one tile's acc0 and acc1 (2 BN columns); the first MMA of the
// next tile waits on tmem_empty until every epilogue warp of the pair has
// finished its TMEM reads (tcgen05.wait::ld -> tcgen05.fence::before_thread_sync
// -> mbarrier arrive -> MMA warp wait -> tcgen05.fence::after_thread_sync).
//
// TWO (the two-factor comparator): the residual steps read their activation
// codes through mp.ar (a second, already quantized activation) and the
// epilogue scales the two products by their own per-row scales,
// y = sx * (sw * acc0) + sxr * (sR * acc1).  SERQ itself passes the main
// activation map as mp.ar (its residual reuses the first r columns of the
// same codes, key design 2) and TWO = false.
template <int BN, bool A8, bool ACC_OUT, int CG, bool TWO = false>
__global__ void __launch_bounds__(kThreads, 1)
    k_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ GroupMaps mp, const GroupArgs p) {
  using L = Layout<BN, A8, CG>;
  constexpr int PS = L::PS, US = L::US;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::oBar);
  uint64_t* full_pk = bar;              // TMA bytes landed            (tx)
  uint64_t* empty_pk = bar + PS;        // packed stage consumed
  uint64_t* full_un = bar + 2 * PS;     // widened stage written (both CTAs, on CTA 0)
  uint64_t* empty_un = full_un + US;    // widened stage read by the MMAs
  uint64_t* acc_full = empty_un + US;   // all MMAs of a tile complete
  uint64_t* drain = acc_full + 1;       // abort path: MMAs complete
  uint64_t* stg_done = drain + 1;       // output staging read by the TMA stores
  uint64_t* tmem_empty = stg_done + 1;  // (CTA 0) every epilogue warp of the pair read its TMEM
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::oMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::oMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = (CG == 2) ? cluster_ctarank() : 0u;
  const bool leader = (rank == 0);
  const int cta_tile = (int)blockIdx.x / CG;            // this CTA (pair)'s first tile
  const int tile_stride = (int)gridDim.x / CG;
  const int ntiles = p.ntiles;
  const int nsteps = p.nkb + p.nrb;

  if (threadIdx.x == 0) {
    // full_un (on CTA 0) collects one arrival per widening warp of the
    // step's group in every CTA of the pair.
    for (int s = 0; s < PS; ++s) {
      mbar_init(&full_pk[s], 1);
      mbar_init(&empty_pk[s], L::kGroupWarps + (A8 ? 1 : 0));
    }
    for (int s = 0; s < US; ++s) {
      mbar_init(&full_un[s], L::kGroupWarps * CG);
      mbar_init(&empty_un[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    mbar_init(stg_done, kUnpackWarps);
    mbar_init(tmem_empty, kUnpackWarps * CG);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&mp.ar);
    for (int l = 0; l < p.nlayers; ++l) {
      tma_prefetch_desc(&mp.b[l]);
      tma_prefetch_desc(&mp.r[l]);
      if (!ACC_OUT) tma_prefetch_desc(&mp.y[l]);
    }
  }
  if (warp == 1) {
    tmem_alloc<CG>(tmem_slot, L::kTmemCols);
    tmem_relinquish<CG>();
  }
  tc_fence_before();
  cta_sync<CG>();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dep_launch();  // the next kernel in the stream may be scheduled

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // Weight (or R) tiles of the first PS steps go out before the wait for
      // the grid this launch depends on (programmatic dependent launch):
      // no earlier kernel writes them.  Their stages are fresh, so no empty
      // wait; the A tiles follow once the activation codes are final.
      int npre = 0;
      for (int t = cta_tile, step = 0; npre < PS && t < ntiles; ++npre) {
        int tl;
        const int l = layer_of(p, t, tl);
        const int nb0 = (tl / p.tiles_m) * BN + (int)rank * L::BNL;
        const bool res = step >= p.nkb;
        const int j = res ? step - p.nkb : step;
        mbar_arrive_expect_tx(&full_pk[npre], L::kTxBytes);
        tma_load_2d(smem + L::oPk + npre * L::kPk + L::kPkA, res ? &mp.r[l] : &mp.b[l], &full_pk[npre], j * (BK / 2),
                    nb0);
        if (++step == nsteps) {
          step = 0;
          t += tile_stride;
        }
      }
      grid_dep_wait();
      int g = 0;  // pipeline step across tiles
      bool ok = true;
      for (int t = cta_tile; ok && t < ntiles; t += tile_stride) {
        int tl;
        const int l = layer_of(p, t, tl);
        const int m0 = ((tl % p.tiles_m) * CG + (int)rank) * BM;
        const int nb0 = (tl / p.tiles_m) * BN + (int)rank * L::BNL;
        for (int step = 0; step < nsteps; ++step, ++g) {
          const int s = g % PS;
          const uint32_t ph = (g / PS) & 1;
          const bool res = step >= p.nkb;
          const int j = res ? step - p.nkb : step;
          uint8_t* stage = smem + L::oPk + s * L::kPk;
          if (g >= npre) {
            if (!mbar_wait(&empty_pk[s], ph ^ 1, abort_flag, kDevTimeoutProducer)) { ok = false; break; }
            mbar_arrive_expect_tx(&full_pk[s], L::kTxBytes);
            tma_load_2d(stage + L::kPkA, res ? &mp.r[l] : &mp.b[l], &full_pk[s], j * (BK / 2), nb0);
          }
          tma_load_2d(stage, res ? &mp.ar : &tmA, &full_pk[s], j * (A8 ? BK : BK / 2), m0);
        }
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issue
    // The whole warp runs the loop and waits together; one elected lane
    // issues.  Descriptors are built once per stage and advanced by the
    // 32-byte k step (2 in the 16-byte address field).
    if (leader) {
      constexpr uint32_t idesc = umma_idesc_i8(BM * CG, BN);
      const uint32_t pk_base = smem_u32(smem + L::oPk);
      const uint32_t un_base = smem_u32(smem + L::oUn);
      bool ok = true;
      int g = 0;
      int it = 0;
      for (int t = cta_tile; ok && t < ntiles; t += tile_stride, ++it) {
        // the accumulators are rewritten only after the previous tile's
        // epilogue has read them in both CTAs
        if (it > 0 && !mbar_wait<CG == 2>(tmem_empty, (uint32_t)(it - 1) & 1u, abort_flag, kDevTimeoutMma)) {
          ok = false;
          break;
        }
        for (int step = 0; step < nsteps; ++step, ++g) {
          const int u = g % US;
          const uint32_t uph = (g / US) & 1;
          const int s = g % PS;
          const uint32_t ph = (g / PS) & 1;
          if (!mbar_wait(&full_un[u], uph, abort_flag, kDevTimeoutMma)) { ok = false; break; }
          if (A8 && !mbar_wait(&full_pk[s], ph, abort_flag, kDevTimeoutMma)) { ok = false; break; }
          tc_fence_after();
          const bool res = step >= p.nkb;
          const int j = res ? step - p.nkb : step;
          const uint32_t d = tmem + (res ? (uint32_t)BN : 0u);
          const uint64_t da = umma_desc_k_sw128(A8 ? pk_base + s * L::kPk : un_base + u * L::kUn);
          const uint64_t db = umma_desc_k_sw128(un_base + u * L::kUn + L::kUnA);
          const int nk = res ? min(BK / 32, (p.rpad - j * BK) / 32) : BK / 32;
          if (elect_one()) {
            if (nk == BK / 32) {
#pragma unroll
              for (int kk = 0; kk < BK / 32; ++kk)
                umma_i8<CG>(d, da + (uint64_t)(2 * kk), db + (uint64_t)(2 * kk), idesc,
                            (j > 0 || kk > 0) ? 1u : 0u);
            } else {
              for (int kk = 0; kk < nk; ++kk)
                umma_i8<CG>(d, da + (uint64_t)(2 * kk), db + (uint64_t)(2 * kk), idesc,
                            (j > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit<CG>(&empty_un[u]);
            if (A8) umma_commit<CG>(&empty_pk[s]);
            if (step == nsteps - 1) umma_commit<CG>(acc_full);
          }
          __syncwarp();
        }
      }
      if (!ok) {
        if (elect_one()) {
          umma_commit<1>(drain);
          mbar_wait(drain, 0, nullptr, kDevTimeoutMma);
        }
        __syncwarp();
      }
    }
  } else {
    // ------------------------------------------------- widening + epilogue
    // Group wg widens the steps g with g % G == wg.  Thread ut of
    // the group widens the same rows and pieces in each of its steps: piece
    // p = ut + 32 kGroupWarps i covers row p / 4 (A rows first, then B rows) and packed
    // bytes [16 (p % 4), +16); its 32 int8 land in chunks 2 (p % 4) and
    // 2 (p % 4) + 1 of the 128-byte row, swizzled by row % 8.  Four
    // consecutive threads cover one row, so a warp reads 512 contiguous
    // bytes and each quarter-warp store fills all 32 banks.
    constexpr int kGroupWarps = L::kGroupWarps;
    const int wg = (warp - 2) / kGroupWarps;
    const int ut = threadIdx.x - 64 - wg * kGroupWarps * 32;
    // Piece i of thread ut sits kRowStep rows below piece i - 1: same
    // 16-byte column q and the same swizzle phase (kRowStep % 8 == 0).
    constexpr int NP = L::kPiecesPerThread;
    constexpr int kRowStep = kGroupWarps * 32 / 4;
    static_assert(kRowStep % 8 == 0, "pieces of a thread share the swizzle phase");
    const int urow = ut >> 2, uq = ut & 3;
    const uint32_t src0 = (A8 ? L::kPkA : 0) + urow * (BK / 2) + uq * 16;
    const uint32_t dst0 = urow * BK + (((2 * uq) ^ (urow & 7)) << 4);
    // Epilogue geometry: this warp may read TMEM lanes 32 (warp % 4) .. +31
    // (rows of its quadrant) and takes half of the BN columns.
    const int eq = warp & 3;
    const int eh = (warp - 2) >> 2;
    constexpr int kHalf = BN / 2;
    constexpr int kCpl = kHalf / 32;  // scale columns prefetched per lane
    constexpr int kShift = A8 ? 4 : 8;
    float* scl = reinterpret_cast<float*>(smem + L::oScl + (warp - 2) * L::kSclWarp);  // [sw | sr]
    const bool has_r = p.nrb > 0;

    // Widened stages holding output boxes whose TMA stores may still read
    // them; every widening warp arrives on stg_done once its own stores have
    // read their sources.
    uint32_t stg_mask = 0;
    uint32_t stg_parity = 0;
    auto release_staging = [&]() -> bool {
      if (stg_mask == 0) return true;
      const bool r = mbar_wait(stg_done, stg_parity, abort_flag, kDevTimeoutEpilogue);
      stg_parity ^= 1u;
      stg_mask = 0;
      return r;
    };

    // Widens pipeline step gs (this group's) into its widened slot.
    auto widen_step = [&](int gs) -> bool {
      const int s = gs % PS;
      const uint32_t ph = (gs / PS) & 1;
      const int u = gs % US;
      const uint32_t uph = (gs / US) & 1;
      if ((stg_mask >> u) & 1u) {
        if (!release_staging()) return false;
      }
      // widened slot first: see the ring notes in Layout
      if (!mbar_wait(&empty_un[u], uph ^ 1, abort_flag, kDevTimeoutUnpack)) return false;
      if (!mbar_wait(&full_pk[s], ph, abort_flag, kDevTimeoutUnpack)) return false;
      const uint8_t* pk = smem + L::oPk + s * L::kPk;
      uint8_t* un = smem + L::oUn + u * L::kUn;
      constexpr int NB = NP < 8 ? NP : 8;  // pieces in registers at a time
      static_assert(NP % NB == 0, "pieces come in whole batches");
#pragma unroll
      for (int b = 0; b < NP; b += NB) {
        uint4 v[NB];
#pragma unroll
        for (int i = 0; i < NB; ++i)
          v[i] = *reinterpret_cast<const uint4*>(pk + src0 + (b + i) * kRowStep * (BK / 2));
#pragma unroll
        for (int i = 0; i < NB; ++i) {
          uint4 lo, hi;
          widen_run(v[i], lo, hi);
          const uint32_t d = dst0 + (b + i) * kRowStep * BK;
          *reinterpret_cast<uint4*>(un + d) = lo;
          *reinterpret_cast<uint4*>(un + (d ^ 16u)) = hi;
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&empty_pk[s]);
        if (leader)
          mbar_arrive(&full_un[u]);
        else
          mbar_arrive_remote(&full_un[u], 0);
      }
      return true;
    };

    grid_dep_wait();  // sx and, in the epilogue, Y belong to the dependency chain
    bool ok = true;
    int g = 0;
    int it = 0;
    int pre_end = 0;  // steps before this were widened ahead of their tile
    for (int t = cta_tile; ok && t < ntiles; t += tile_stride, ++it) {
      int tl;
      const int l = layer_of(p, t, tl);
      const LayerOut& lo = p.lo[l];
      const int m0 = ((tl % p.tiles_m) * CG + (int)rank) * BM;
      const int n0 = (tl / p.tiles_m) * BN;
      // prefetch this tile's epilogue scales (consumed after the k loop)
      float swv[kCpl], srv[kCpl], sxv = 0.f, sxrv = 0.f;
      if (!ACC_OUT) {
#pragma unroll
        for (int i = 0; i < kCpl; ++i) {
          const int n = n0 + eh * kHalf + kCpl * lane + i;
          swv[i] = (n < lo.N) ? __ldg(lo.sw + n) : 0.f;
          srv[i] = (n < lo.N) ? __ldg(lo.sr + n) : 0.f;
        }
        const int row = m0 + eq * 32 + lane;
        sxv = (row < p.M) ? __ldg(p.sx + row) : 0.f;
        if (TWO) sxrv = (row < p.M) ? __ldg(p.sxr + row) : 0.f;
      }

      for (int step = 0; step < nsteps; ++step, ++g) {
        if (g % L::G != wg || g < pre_end) continue;
        if (!widen_step(g)) { ok = false; break; }
      }
      if (!ok) break;
      // Widen ahead: this group's steps of the next tile that go to widened
      // slots the epilogue below does not stage into, so that the next
      // tile's first MMAs can issue as soon as TMEM is free.
      if (t + tile_stride < ntiles) {
        const int ahead = min(US - L::kStgStages, nsteps);
        for (int ga = g; ga < g + ahead; ++ga)
          if (ga % L::G == wg && !widen_step(ga)) { ok = false; break; }
        pre_end = g + ahead;
      }
      if (!ok) break;

      // ---------------------------------------------------------- epilogue
      if (!release_staging()) { ok = false; break; }
      if (!mbar_wait(acc_full, (uint32_t)it & 1u, abort_flag, kDevTimeoutEpilogue)) { ok = false; break; }
      tc_fence_after();
      const int row = m0 + eq * 32 + lane;
      const uint32_t tq = tmem + ((uint32_t)(eq * 32) << 16);
      if (ACC_OUT) {
        for (int c = eh * kHalf; c < (eh + 1) * kHalf; c += 32) {
          uint32_t r0[32], r1[32];
          tmem_ld_32x32b_x32(tq + (uint32_t)c, r0);
          if (has_r) tmem_ld_32x32b_x32(tq + (uint32_t)(BN + c), r1);
          tmem_ld_wait_regs(r0);
          tmem_ld_wait_regs(r1);
          if (!has_r) {
#pragma unroll
            for (int i = 0; i < 32; ++i) r1[i] = 0;
          }
          if (row < p.M && n0 + c < lo.N) {
            int32_t* o0 = lo.acc0 + (size_t)row * lo.N + n0 + c;
            int32_t* o1 = lo.acc1 + (size_t)row * lo.N + n0 + c;
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              *reinterpret_cast<int4*>(o0 + i) =
                  make_int4((int)r0[i] >> kShift, (int)r0[i + 1] >> kShift, (int)r0[i + 2] >> kShift,
                            (int)r0[i + 3] >> kShift);
              *reinterpret_cast<int4*>(o1 + i) =
                  make_int4((int)r1[i] >> kShift, (int)r1[i + 1] >> kShift, (int)r1[i + 2] >> kShift,
                            (int)r1[i + 3] >> kShift);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (leader)
            mbar_arrive(tmem_empty);
          else
            mbar_arrive_remote(tmem_empty, 0);
        }
      } else {
        // scales of this warp's columns -> its private smem copy, with the
        // widening factor 2^kShift folded in (exact: a power of two)
        constexpr float kUnscale = 1.f / (float)(1 << kShift);
#pragma unroll
        for (int i = 0; i < kCpl; ++i) {
          scl[kCpl * lane + i] = swv[i] * kUnscale;
          scl[kHalf + kCpl * lane + i] = srv[i] * kUnscale;
        }
        __syncwarp();
        // output staging: box b = 32 rows x 64 columns of the tile, stored
        // in widened stage (first stage of the next tile's ring order that
        // is left for last) + b / kBoxesPerStage
        const int g_next = g;  // first pipeline step of the next tile
        auto box_ptr = [&](int b) -> uint8_t* {
          const int su = (g_next + US - L::kStgStages + b / L::kBoxesPerStage) % US;
          return smem + L::oUn + su * L::kUn + (b % L::kBoxesPerStage) * L::kBoxBytes;
        };
        const float4* sw4 = reinterpret_cast<const float4*>(scl);
        const float4* sr4 = reinterpret_cast<const float4*>(scl + kHalf);
        // 16-column chunks, double-buffered: the TMEM loads of chunk k + 1 are
        // in flight while chunk k is converted and staged; TMEM is released
        // as soon as the last chunk's loads have completed.
        constexpr int kChunks = kHalf / 16;
        auto release_tmem = [&]() {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (leader)
              mbar_arrive(tmem_empty);
            else
              mbar_arrive_remote(tmem_empty, 0);
          }
        };
        auto load_chunk = [&](uint32_t(&d0)[16], uint32_t(&d1)[16], int cc) {
          const int c = eh * kHalf + cc;
          tmem_ld_32x32b_x16(tq + (uint32_t)c, d0);
          if (has_r) {
            tmem_ld_32x32b_x16(tq + (uint32_t)(BN + c), d1);
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) d1[i] = 0;
          }
        };
        // Scales of the next group of four columns are loaded while the
        // current group is converted (carried across chunks), so their
        // shared-memory latency stays off the conversion's dependency chain.
        float4 wn = sw4[0], rn = sr4[0];
        auto convert_chunk = [&](const uint32_t(&r0)[16], const uint32_t(&r1)[16], int cc) {
          const int c = eh * kHalf + cc;  // tile column of this 16-column chunk
          // 128-byte swizzle: 16-byte chunk k of row r sits at chunk k ^ (r % 8)
          uint8_t* bp = box_ptr(eq * (BN / 64) + (c >> 6)) + lane * 128;
          const int k0 = (c & 63) >> 3;  // first 16-byte chunk of these 16 columns
          const float2 sx2 = make_float2(sxv, sxv);
          const float2 sxr2 = make_float2(sxrv, sxrv);
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            uint32_t pk[4];
#pragma unroll
            for (int i = 0; i < 8; i += 4) {
              // y = sx * (sw' * acc0 + sR' * acc1) on column pairs, with the
              // accumulators converted as they come out of TMEM (x256 or x16;
              // the factor is in sw', sR')
              const int e = 8 * k + i;
              const float4 w = wn, rr = rn;
              const int nx = (cc + e + 4 < kHalf) ? (cc + e + 4) >> 2 : 0;  // next group (wraps at the end)
              wn = sw4[nx];
              rn = sr4[nx];
              const float2 f0a = make_float2((float)(int)r0[e], (float)(int)r0[e + 1]);
              const float2 f0b = make_float2((float)(int)r0[e + 2], (float)(int)r0[e + 3]);
              const float2 f1a = make_float2((float)(int)r1[e], (float)(int)r1[e + 1]);
              const float2 f1b = make_float2((float)(int)r1[e + 2], (float)(int)r1[e + 3]);
              float2 ya, yb;
              if (TWO) {
                ya = fma2(mul2(sx2, make_float2(w.x, w.y)), f0a, mul2(sxr2, mul2(make_float2(rr.x, rr.y), f1a)));
                yb = fma2(mul2(sx2, make_float2(w.z, w.w)), f0b, mul2(sxr2, mul2(make_float2(rr.z, rr.w), f1b)));
              } else {
                ya = mul2(sx2, fma2(make_float2(w.x, w.y), f0a, mul2(make_float2(rr.x, rr.y), f1a)));
                yb = mul2(sx2, fma2(make_float2(w.z, w.w), f0b, mul2(make_float2(rr.z, rr.w), f1b)));
              }
              const __nv_bfloat162 h0 = __floats2bfloat162_rn(ya.x, ya.y);
              const __nv_bfloat162 h1 = __floats2bfloat162_rn(yb.x, yb.y);
              pk[i >> 1] = *reinterpret_cast<const uint32_t*>(&h0);
              pk[(i >> 1) + 1] = *reinterpret_cast<const uint32_t*>(&h1);
            }
            *reinterpret_cast<uint4*>(bp + (((k0 + k) ^ (lane & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        };
        uint32_t ra0[16], ra1[16], rb0[16], rb1[16];
        load_chunk(ra0, ra1, 0);
        tmem_ld_wait_regs(ra0, ra1);
        if (kChunks == 1) release_tmem();
#pragma unroll
        for (int k = 0; k < kChunks; ++k) {
          if ((k & 1) == 0) {
            if (k + 1 < kChunks) load_chunk(rb0, rb1, 16 * (k + 1));
            convert_chunk(ra0, ra1, 16 * k);
            if (k + 1 < kChunks) tmem_ld_wait_regs(rb0, rb1);
          } else {
            if (k + 1 < kChunks) load_chunk(ra0, ra1, 16 * (k + 1));
            convert_chunk(rb0, rb1, 16 * k);
            if (k + 1 < kChunks) tmem_ld_wait_regs(ra0, ra1);
          }
          if (k + 2 == kChunks) release_tmem();  // the last chunk's loads are complete
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int y = m0 + eq * 32;
#pragma unroll
          for (int b = 0; b < kHalf / 64; ++b) {
            const int x = n0 + eh * kHalf + b * 64;
            if (x < lo.N && y < p.M) tma_store_2d(&mp.y[l], box_ptr(eq * (BN / 64) + eh * (kHalf / 64) + b), x, y);
          }
          bulk_commit_group();
          bulk_wait_read_all();
          mbar_arrive(stg_done);
        }
        for (int k = 0; k < L::kStgStages; ++k) stg_mask |= 1u << ((g_next + US - L::kStgStages + k) % US);
      }
    }
    if (!ACC_OUT && lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag && warp == 0 && lane == 0) {
    // Let TMA copies already issued land before the CTA's shared memory is
    // released (they complete in microseconds; bounded).
    const unsigned long long t0 = global_ns();
    while (global_ns() - t0 < 100000ull) {
    }
  }
  // Neither CTA of a pair leaves (or frees TMEM) while its peer may still
  // touch its barriers or shared memory.
  cta_sync<CG>();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<CG>(tmem, L::kTmemCols);
  }
}

}  // namespace tc
}  // namespace serq

namespace serq {
namespace tc {

// ---------------------------------------------------------------------------
// W4A4 prefill on CTA pairs with the activation operand in tensor memory.
//
// Each 128-k step of the pipeline above moves, per SM, the TMA writes, the
// widening loads and stores and the tensor-core operand reads through shared
// memory; with the widened activations written to TMEM instead (tcgen05.st
// straight from the widening registers, read by the MMA as its A operand)
// the activation half of the widened stores and of the operand reads leaves
// shared memory.  TMEM then holds acc0 (BN columns), acc1 (BN) and TS widened
// activation stages of 32 columns (128 int8 per lane, four per column), so
// BN = 192: 2 * 192 + 4 * 32 = 512 columns.
//
// Warps: 0 TMA, 1 TMEM owner / MMA issue (CTA 0), 2..9 widen in two groups
// of four that take alternate steps; in its steps a group widens the 128
// activation rows of this CTA into TMEM (warp w writes TMEM lanes
// 32 (w % 4) .. +31, one row per thread) and this CTA's BN/2 weight rows
// into shared memory.  All eight run the epilogue, which stages
// the bf16 tile in a shared-memory area of its own (freed by the activation
// stages' absence) and writes it with TMA stores.
// The packed activation tile arrives with the 64-byte TMA swizzle, so the
// per-thread row reads hit distinct banks.
template <int BN>
struct LayoutTA {
  static constexpr int CG = 2;
  static constexpr int BNL = BN / 2;                  // weight rows per CTA
  static constexpr int PS = 8;                        // packed stages
  static constexpr int US = 4;                        // widened stages (smem B + TMEM A)
  // two widening groups of four warps take alternate steps (see Layout)
  static constexpr int G = 2;
  static constexpr int kGroupWarps = kUnpackWarps / G;
  static constexpr int kPkA = BM * BK / 2;            // 8 KB, 64-byte swizzled
  static constexpr int kPkB = BNL * BK / 2;
  static constexpr int kPk = kPkA + kPkB;
  static constexpr int kUn = BNL * BK;                // widened weight rows
  // output staging: boxes of 32 rows x 32 bf16 (2 KB, 64-byte swizzle), BN / 32
  // per TMEM lane quadrant; each epilogue warp owns the boxes it writes
  static constexpr int kBoxBytes = 32 * 64;
  static constexpr int kBoxes = 4 * (BN / 32);
  static constexpr int oUn = 0;
  static constexpr int oPk = oUn + US * kUn;
  static constexpr int oStg = oPk + PS * kPk;
  static constexpr int oScl = oStg + kBoxes * kBoxBytes;
  static constexpr int kSclWarp = 2 * (BN / 2) * 4;  // sw and sr of a warp's BN / 2 columns
  static constexpr int oBar = oScl + kUnpackWarps * kSclWarp;
  static constexpr int nBar = 2 * PS + 2 * US + 3;
  static constexpr int oMisc = oBar + nBar * 8;
  static constexpr int kBytes = oMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;
  static constexpr uint32_t kTxBytes = kPk;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kTmemA = 2 * BN;          // first activation stage column
  static constexpr int kPiecesB = BNL * 4 / 128;      // per weight-widening thread
  static_assert(2 * BN + US * (BK / 4) <= 512, "TMEM budget");
  static_assert(US % G == 0 && PS >= US && kGroupWarps == 4, "group ring ownership, one warp per lane quadrant");
  static_assert(BNL * 4 % 128 == 0 && BN % 64 == 0, "weight pieces must divide evenly");
  static_assert(kPk % 1024 == 0 && kUn % 1024 == 0 && oStg % 1024 == 0, "tiles must stay 1024-aligned");
  static_assert(kAlloc <= 232448, "shared memory budget");
};

// Persistent like k_gemm: CTA pair c takes tiles c, c + G, ... (M-tile
// fastest), the rings run on across tiles, and the first MMA of a tile waits
// through the widened-stage barrier for the previous epilogue's TMEM reads.
template <int BN, bool ACC_OUT>
__global__ void __launch_bounds__(kThreads, 1)
    k_gemm_ta(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const __grid_constant__ CUtensorMap tmR, const __grid_constant__ CUtensorMap tmY, const Args p) {
  using L = LayoutTA<BN>;
  constexpr int PS = L::PS, US = L::US;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::oBar);
  uint64_t* full_pk = bar;
  uint64_t* empty_pk = bar + PS;
  uint64_t* full_un = bar + 2 * PS;     // on CTA 0: both CTAs' widening warps
  uint64_t* empty_un = full_un + US;
  uint64_t* acc_full = empty_un + US;
  uint64_t* drain = acc_full + 1;
  uint64_t* tmem_empty = drain + 1;     // (CTA 0) every epilogue warp of the pair read its TMEM
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::oMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::oMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);
  const int cta_tile = (int)blockIdx.x / 2;
  const int tile_stride = (int)gridDim.x / 2;
  const int ntiles = p.tiles_m * p.tiles_n;
  const int nsteps = p.nkb + p.nrb;

  if (threadIdx.x == 0) {
    for (int s = 0; s < PS; ++s) {
      mbar_init(&full_pk[s], 1);
      mbar_init(&empty_pk[s], L::kGroupWarps);
    }
    for (int s = 0; s < US; ++s) {
      mbar_init(&full_un[s], L::kGroupWarps * 2);
      mbar_init(&empty_un[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    mbar_init(tmem_empty, kUnpackWarps * 2);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmR);
    if (!ACC_OUT) tma_prefetch_desc(&tmY);
  }
  if (warp == 1) {
    tmem_alloc<2>(tmem_slot, L::kTmemCols);
    tmem_relinquish<2>();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int g = 0;
      bool ok = true;
      for (int t = cta_tile; ok && t < ntiles; t += tile_stride) {
        const int m0 = ((t % p.tiles_m) * 2 + (int)rank) * BM;
        const int nb0 = (t / p.tiles_m) * BN + (int)rank * L::BNL;
        for (int step = 0; step < nsteps; ++step, ++g) {
          const int s = g % PS;
          const uint32_t ph = (g / PS) & 1;
          if (!mbar_wait(&empty_pk[s], ph ^ 1, abort_flag, kDevTimeoutProducer)) { ok = false; break; }
          mbar_arrive_expect_tx(&full_pk[s], L::kTxBytes);
          const bool res = step >= p.nkb;
          const int j = res ? step - p.nkb : step;
          uint8_t* stage = smem + L::oPk + s * L::kPk;
          tma_load_2d(stage, &tmA, &full_pk[s], j * (BK / 2), m0);
          tma_load_2d(stage + L::kPkA, res ? &tmR : &tmB, &full_pk[s], j * (BK / 2), nb0);
        }
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issue
    if (leader) {
      constexpr uint32_t idesc = umma_idesc_i8(BM * 2, BN);
      const uint32_t un_base = smem_u32(smem + L::oUn);
      bool ok = true;
      int g = 0;
      int it = 0;
      for (int t = cta_tile; ok && t < ntiles; t += tile_stride, ++it) {
        if (it > 0 && !mbar_wait<true>(tmem_empty, (uint32_t)(it - 1) & 1u, abort_flag, kDevTimeoutMma)) {
          ok = false;
          break;
        }
        for (int step = 0; step < nsteps; ++step, ++g) {
          const int u = g % US;
          const uint32_t uph = (g / US) & 1;
          if (!mbar_wait(&full_un[u], uph, abort_flag, kDevTimeoutMma)) { ok = false; break; }
          tc_fence_after();
          const bool res = step >= p.nkb;
          const int j = res ? step - p.nkb : step;
          const uint32_t d = tmem + (res ? (uint32_t)BN : 0u);
          const uint32_t a = tmem + L::kTmemA + (uint32_t)(u * (BK / 4));
          const uint64_t db = umma_desc_k_sw128(un_base + u * L::kUn);
          const int nk = res ? min(BK / 32, (p.rpad - j * BK) / 32) : BK / 32;
          if (elect_one()) {
            if (nk == BK / 32) {
#pragma unroll
              for (int kk = 0; kk < BK / 32; ++kk)
                umma_i8_ts<2>(d, a + (uint32_t)(kk * 8), db + (uint64_t)(2 * kk), idesc,
                              (j > 0 || kk > 0) ? 1u : 0u);
            } else {
              for (int kk = 0; kk < nk; ++kk)
                umma_i8_ts<2>(d, a + (uint32_t)(kk * 8), db + (uint64_t)(2 * kk), idesc,
                              (j > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit<2>(&empty_un[u]);
            if (step == nsteps - 1) umma_commit<2>(acc_full);
          }
          __syncwarp();
        }
      }
      if (!ok) {
        if (elect_one()) {
          umma_commit<1>(drain);
          mbar_wait(drain, 0, nullptr, kDevTimeoutMma);
        }
        __syncwarp();
      }
    }
  } else {
    // ------------------------------------------------- widening + epilogue
    // Group wg = warps 2 + 4 wg .. 5 + 4 wg widens steps g with g % 2 == wg:
    // each thread widens one activation row of its warp's TMEM lane quadrant
    // and three 16-byte weight pieces.
    const int wg = (warp - 2) >> 2;
    const int q = warp & 3;                            // TMEM lane quadrant
    const int arow = q * 32 + lane;                    // activation row
    const int bt = ((warp - 2) & 3) * 32 + lane;       // 0..127 within the group
    uint32_t a_off[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) a_off[c] = arow * (BK / 2) + ((c ^ ((arow >> 1) & 3)) << 4);
    constexpr int NPB = L::kPiecesB;
    uint32_t src_off[NPB], dst_off[NPB];
#pragma unroll
    for (int i = 0; i < NPB; ++i) {
      const int pc = bt + i * 128;
      const int row = pc >> 2, c = pc & 3;
      src_off[i] = L::kPkA + row * (BK / 2) + c * 16;
      dst_off[i] = row * BK + (((2 * c) ^ (row & 7)) << 4);
    }
    // epilogue geometry: TMEM lanes of quadrant q, columns [eh BN/2, +BN/2)
    const int eh = (warp - 2) >> 2;
    constexpr int kHalf = BN / 2;
    constexpr int kCpl = kHalf / 32;
    constexpr int kShift = 8;
    float* scl = reinterpret_cast<float*>(smem + L::oScl + (warp - 2) * L::kSclWarp);  // [sw | sr]
    const bool has_r = p.nrb > 0;
    bool stores_pending = false;

    bool ok = true;
    int g = 0;
    int it = 0;
    for (int t = cta_tile; ok && t < ntiles; t += tile_stride, ++it) {
      const int m0 = ((t % p.tiles_m) * 2 + (int)rank) * BM;
      const int n0 = (t / p.tiles_m) * BN;
      float swv[kCpl], srv[kCpl], sxv = 0.f;
      if (!ACC_OUT) {
#pragma unroll
        for (int i = 0; i < kCpl; ++i) {
          const int n = n0 + eh * kHalf + 32 * i + lane;
          swv[i] = (n < p.N) ? __ldg(p.sw + n) : 0.f;
          srv[i] = (n < p.N) ? __ldg(p.sr + n) : 0.f;
        }
        const int row = m0 + q * 32 + lane;
        sxv = (row < p.M) ? __ldg(p.sx + row) : 0.f;
      }
      for (int step = 0; step < nsteps; ++step, ++g) {
        if ((g & 1) != wg) continue;
        const int s = g % PS;
        const uint32_t ph = (g / PS) & 1;
        const int u = g % US;
        const uint32_t uph = (g / US) & 1;
        // widened slot first (see Layout)
        if (!mbar_wait(&empty_un[u], uph ^ 1, abort_flag, kDevTimeoutUnpack)) { ok = false; break; }
        if (!mbar_wait(&full_pk[s], ph, abort_flag, kDevTimeoutUnpack)) { ok = false; break; }
        const uint8_t* pk = smem + L::oPk + s * L::kPk;
        {
          uint32_t r[32];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 v = *reinterpret_cast<const uint4*>(pk + a_off[c]);
            uint4 lo, hi;
            widen_run(v, lo, hi);
            r[8 * c + 0] = lo.x; r[8 * c + 1] = lo.y; r[8 * c + 2] = lo.z; r[8 * c + 3] = lo.w;
            r[8 * c + 4] = hi.x; r[8 * c + 5] = hi.y; r[8 * c + 6] = hi.z; r[8 * c + 7] = hi.w;
          }
          tmem_st_32x32b_x32(tmem + ((uint32_t)(q * 32) << 16) + L::kTmemA + (uint32_t)(u * (BK / 4)), r);
        }
        {
          uint8_t* un = smem + L::oUn + u * L::kUn;
          uint4 v[NPB];
#pragma unroll
          for (int i = 0; i < NPB; ++i) v[i] = *reinterpret_cast<const uint4*>(pk + src_off[i]);
#pragma unroll
          for (int i = 0; i < NPB; ++i) {
            uint4 lo, hi;
            widen_run(v[i], lo, hi);
            *reinterpret_cast<uint4*>(un + dst_off[i]) = lo;
            *reinterpret_cast<uint4*>(un + (dst_off[i] ^ 16u)) = hi;
          }
        }
        tmem_st_wait();
        tc_fence_before();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&empty_pk[s]);
          if (leader)
            mbar_arrive(&full_un[u]);
          else
            mbar_arrive_remote(&full_un[u], 0);
        }
      }
      if (!ok) break;

      // ---------------------------------------------------------- epilogue
      if (!mbar_wait(acc_full, (uint32_t)it & 1u, abort_flag, kDevTimeoutEpilogue)) { ok = false; break; }
      tc_fence_after();
      const int row = m0 + q * 32 + lane;
      const uint32_t tq = tmem + ((uint32_t)(q * 32) << 16);
      if (ACC_OUT) {
        for (int c = eh * kHalf; c < (eh + 1) * kHalf; c += 32) {
          uint32_t r0[32], r1[32];
          tmem_ld_32x32b_x32(tq + (uint32_t)c, r0);
          if (has_r) tmem_ld_32x32b_x32(tq + (uint32_t)(BN + c), r1);
          tmem_ld_wait_regs(r0);
          tmem_ld_wait_regs(r1);
          if (!has_r) {
#pragma unroll
            for (int i = 0; i < 32; ++i) r1[i] = 0;
          }
          if (row < p.M && n0 + c < p.N) {
            int32_t* o0 = p.acc0 + (size_t)row * p.N + n0 + c;
            int32_t* o1 = p.acc1 + (size_t)row * p.N + n0 + c;
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              *reinterpret_cast<int4*>(o0 + i) =
                  make_int4((int)r0[i] >> kShift, (int)r0[i + 1] >> kShift, (int)r0[i + 2] >> kShift,
                            (int)r0[i + 3] >> kShift);
              *reinterpret_cast<int4*>(o1 + i) =
                  make_int4((int)r1[i] >> kShift, (int)r1[i + 1] >> kShift, (int)r1[i + 2] >> kShift,
                            (int)r1[i + 3] >> kShift);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (leader)
            mbar_arrive(tmem_empty);
          else
            mbar_arrive_remote(tmem_empty, 0);
        }
      } else {
        // this warp's staging boxes were read by its previous TMA stores
        if (stores_pending) {
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
        }
#pragma unroll
        for (int i = 0; i < kCpl; ++i) {
          scl[32 * i + lane] = swv[i];
          scl[kHalf + 32 * i + lane] = srv[i];
        }
        __syncwarp();
        const float4* sw4 = reinterpret_cast<const float4*>(scl);
        const float4* sr4 = reinterpret_cast<const float4*>(scl + kHalf);
        for (int cc = 0; cc < kHalf; cc += 32) {
          const int c = eh * kHalf + cc;  // tile column of this chunk = one box
          uint32_t r0[32], r1[32];
          tmem_ld_32x32b_x32(tq + (uint32_t)c, r0);
          if (has_r) tmem_ld_32x32b_x32(tq + (uint32_t)(BN + c), r1);
          tmem_ld_wait_regs(r0);
          tmem_ld_wait_regs(r1);
          if (!has_r) {
#pragma unroll
            for (int i = 0; i < 32; ++i) r1[i] = 0;
          }
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            const float4 w = sw4[(cc + i) >> 2];
            const float4 rr = sr4[(cc + i) >> 2];
            const float y0 = sxv * fmaf(w.x, (float)((int)r0[i] >> kShift), rr.x * (float)((int)r1[i] >> kShift));
            const float y1 = sxv * fmaf(w.y, (float)((int)r0[i + 1] >> kShift), rr.y * (float)((int)r1[i + 1] >> kShift));
            const float y2 = sxv * fmaf(w.z, (float)((int)r0[i + 2] >> kShift), rr.z * (float)((int)r1[i + 2] >> kShift));
            const float y3 = sxv * fmaf(w.w, (float)((int)r0[i + 3] >> kShift), rr.w * (float)((int)r1[i + 3] >> kShift));
            const __nv_bfloat162 h0 = __floats2bfloat162_rn(y0, y1);
            const __nv_bfloat162 h1 = __floats2bfloat162_rn(y2, y3);
            pk[i >> 1] = *reinterpret_cast<const uint32_t*>(&h0);
            pk[(i >> 1) + 1] = *reinterpret_cast<const uint32_t*>(&h1);
          }
          // 64-byte swizzle: 16-byte chunk k of row r sits at chunk k ^ ((r / 2) % 4)
          uint8_t* bp = smem + L::oStg + (q * (BN / 32) + (c >> 5)) * L::kBoxBytes + lane * 64;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            *reinterpret_cast<uint4*>(bp + ((k ^ ((lane >> 1) & 3)) << 4)) =
                make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
        }
        tc_fence_before();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (leader)
            mbar_arrive(tmem_empty);
          else
            mbar_arrive_remote(tmem_empty, 0);
          const int y = m0 + q * 32;
#pragma unroll
          for (int b = 0; b < kCpl; ++b) {
            const int x = n0 + eh * kHalf + 32 * b;
            if (x < p.N && y < p.M)
              tma_store_2d(&tmY, smem + L::oStg + (q * (BN / 32) + eh * kCpl + b) * L::kBoxBytes, x, y);
          }
          bulk_commit_group();
        }
        stores_pending = true;
      }
    }
    if (!ACC_OUT && lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag && warp == 0 && lane == 0) {
    const unsigned long long t0 = global_ns();
    while (global_ns() - t0 < 100000ull) {
    }
  }
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<2>(tmem, L::kTmemCols);
  }
}

}  // namespace tc
}  // namespace serq
