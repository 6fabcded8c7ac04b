// Decode-regime SERQ linear on the 5th-generation tensor cores, operands
// swapped: Y^T = W X^T, so the weight rows fill the MMA's M = 128 and the
// few tokens (M <= 32, padded to MP = 16 or 32) are its N.
//
//   acc0^T = Wq Xq^T            acc1^T = Rq Xq[:, :r]^T
//   Y[m, n] = sx[m] * (sw[n] * acc0[m, n] + sR[n] * acc1[m, n])
//
// The path is HBM-bound: every packed weight byte is read once and the
// tensor core only has to keep up.  A unit of work is one 128-row weight
// tile over a contiguous range of its K steps (split-K, so that about two
// units per SM are in flight even for 4096-row weights); the residual step
// belongs to split 0.  Partial int32 sums of a tile meet in the layer's
// workspace by atomic adds; the unit that finishes its tile last (tile
// counter) applies the epilogue and clears the workspace rows.  With one
// split the epilogue runs straight out of TMEM.
//
// Warps: 0 TMA (packed W or R tile, packed activation block), 1 TMEM owner
// and MMA issue (tcgen05.mma.cta_group::1.kind::i8, M = 128, N = MP, K = 32),
// 2..5 widen nibbles to int8 (x16) into the 128-byte-swizzled K-major
// layout, in two groups of two warps on alternate steps, then run the
// epilogue (warp w reads TMEM lanes 32 (w % 4) .. +31 = 32 weight rows).
// The weight tiles of the first steps are requested before the kernel waits
// for the grid it depends on (programmatic dependent launch).
//
// A wait that times out leaves the layer's workspace undefined (the error is
// reported through the device status word; the layer must be prepared again).
#pragma once
#include "common.cuh"

namespace serq {
namespace dtc {

constexpr int BM = 128;           // weight rows per tile (MMA M)
constexpr int BK = 128;           // k per step
constexpr int kWidenWarps = 4;
constexpr int kGroups = 2;        // widening groups (alternate steps)
constexpr int kGroupWarps = kWidenWarps / kGroups;
constexpr int kThreads = (2 + kWidenWarps) * 32;
constexpr int PS = 6;             // packed stages
constexpr int US = 2;             // widened stages (one per group)
constexpr int kMaxM = 32;

struct Args {
  int M, K, N, rpad;
  int nkb, nrb;     // main and residual steps of the whole K
  int splits;       // units per weight tile
  const float* sx;
  const float* sw;
  const float* sr;
  __nv_bfloat16* Y;
  int ldy;
  int32_t* acc0;    // raw accumulators out (test hook) or null
  int32_t* acc1;
  int32_t* ws;      // [2][kMaxM][N] partial sums (lanes of a warp: consecutive n), zero between calls
  int32_t* cnt;     // [tiles] units done, zero between calls
};

template <int MP, bool A8>
struct Layout {
  static constexpr int kPkA = BM * BK / 2;                 // packed weight tile
  static constexpr int kPkB = A8 ? MP * BK : MP * BK / 2;  // activation block
  static constexpr int kPk = kPkA + kPkB;
  static constexpr int kUnA = BM * BK;                     // widened weight tile
  static constexpr int kUnB = A8 ? 0 : MP * BK;            // widened activations (W4A8: packed stage)
  static constexpr int kUn = kUnA + kUnB;
  static constexpr int oUn = 0;
  static constexpr int oPk = oUn + US * kUn;
  static constexpr int oBar = oPk + PS * kPk;
  static constexpr int nBar = 2 * PS + 2 * US + 2;
  static constexpr int oMisc = oBar + nBar * 8;
  static constexpr int kAlloc = oMisc + 16 + 1024;
  static constexpr uint32_t kTmemCols = (2 * MP < 32) ? 32 : 2 * MP;
  static constexpr int kRowsA = BM, kRowsB = A8 ? 0 : MP;
  static constexpr int kPieces = (kRowsA + kRowsB) * 4;    // 16-byte packed pieces per step
  static_assert(kPk % 1024 == 0 || (kPkA % 1024 == 0), "weight tile stays 1024-aligned");
  static_assert(kUnA % 1024 == 0 && kUn % 1024 == 0 && oPk % 1024 == 0, "stages stay 1024-aligned");
  static_assert(US % kGroups == 0 && PS >= US, "group ring ownership");
};

__device__ __forceinline__ void widen_run(const uint4 v, uint4& lo, uint4& hi) {
  const uint32_t m = 0xF0F0F0F0u;
  lo = make_uint4((v.x << 4) & m, (v.y << 4) & m, (v.z << 4) & m, (v.w << 4) & m);
  hi = make_uint4(v.x & m, v.y & m, v.z & m, v.w & m);
}

template <int MP, bool A8, bool ACC_OUT>
__global__ void __launch_bounds__(kThreads, 1)
    k_decode_tc(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmR,
                const __grid_constant__ CUtensorMap tmX, const Args p) {
  using L = Layout<MP, A8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::oBar);
  uint64_t* full_pk = bar;
  uint64_t* empty_pk = bar + PS;
  uint64_t* full_un = bar + 2 * PS;
  uint64_t* empty_un = full_un + US;
  uint64_t* acc_full = empty_un + US;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::oMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::oMisc + 4);
  volatile int* last_flag = reinterpret_cast<volatile int*>(smem + L::oMisc + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x / p.splits, split = blockIdx.x % p.splits;
  const int n0 = tile * BM;
  // this unit's main steps [k0, k1); split 0 also runs the residual steps
  const int k0 = (int)((long)p.nkb * split / p.splits);
  const int k1 = (int)((long)p.nkb * (split + 1) / p.splits);
  const int nres = (split == 0) ? p.nrb : 0;
  const int nsteps = (k1 - k0) + nres;

  if (threadIdx.x == 0) {
    for (int s = 0; s < PS; ++s) {
      mbar_init(&full_pk[s], 1);
      mbar_init(&empty_pk[s], kGroupWarps + (A8 ? 1 : 0));
    }
    for (int s = 0; s < US; ++s) {
      mbar_init(&full_un[s], kGroupWarps);
      mbar_init(&empty_un[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    *last_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmR);
    tma_prefetch_desc(&tmX);
  }
  if (warp == 1) {
    tmem_alloc<1>(tmem_slot, L::kTmemCols);
    tmem_relinquish<1>();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dep_launch();

  auto step_k = [&](int step, bool& res) -> int {  // k block of a unit step
    res = step >= (k1 - k0);
    return res ? step - (k1 - k0) : k0 + step;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const int npre = nsteps < PS ? nsteps : PS;
      for (int step = 0; step < npre; ++step) {  // weight tiles: no earlier kernel writes them
        bool res;
        const int j = step_k(step, res);
        mbar_arrive_expect_tx(&full_pk[step], L::kPk);
        tma_load_2d(smem + L::oPk + step * L::kPk, res ? &tmR : &tmW, &full_pk[step], j * (BK / 2), n0);
      }
      grid_dep_wait();
      for (int step = 0; step < nsteps; ++step) {
        const int s = step % PS;
        const uint32_t ph = (step / PS) & 1;
        bool res;
        const int j = step_k(step, res);
        uint8_t* stage = smem + L::oPk + s * L::kPk;
        if (step >= npre) {
          if (!mbar_wait(&empty_pk[s], ph ^ 1, abort_flag, kDevTimeoutProducer)) break;
          mbar_arrive_expect_tx(&full_pk[s], L::kPk);
          tma_load_2d(stage, res ? &tmR : &tmW, &full_pk[s], j * (BK / 2), n0);
        }
        tma_load_2d(stage + L::kPkA, &tmX, &full_pk[s], j * (A8 ? BK : BK / 2), 0);
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issue
    constexpr uint32_t idesc = umma_idesc_i8(BM, MP);
    const uint32_t pk_base = smem_u32(smem + L::oPk);
    const uint32_t un_base = smem_u32(smem + L::oUn);
    bool ok = true;
    int first_main = 1, first_res = 1;
    for (int step = 0; step < nsteps; ++step) {
      const int u = step % US;
      const uint32_t uph = (step / US) & 1;
      const int s = step % PS;
      const uint32_t ph = (step / PS) & 1;
      if (!mbar_wait(&full_un[u], uph, abort_flag, kDevTimeoutMma)) { ok = false; break; }
      if (A8 && !mbar_wait(&full_pk[s], ph, abort_flag, kDevTimeoutMma)) { ok = false; break; }
      tc_fence_after();
      bool res;
      const int j = step_k(step, res);
      const uint32_t d = tmem + (res ? (uint32_t)MP : 0u);
      const uint64_t da = umma_desc_k_sw128(un_base + u * L::kUn);
      const uint64_t db = umma_desc_k_sw128(A8 ? pk_base + s * L::kPk + L::kPkA : un_base + u * L::kUn + L::kUnA);
      const int nk = res ? min(BK / 32, (p.rpad - j * BK) / 32) : BK / 32;
      int& first = res ? first_res : first_main;
      if (elect_one()) {
        for (int kk = 0; kk < nk; ++kk)
          umma_i8<1>(d, da + (uint64_t)(2 * kk), db + (uint64_t)(2 * kk), idesc, (first && kk == 0) ? 0u : 1u);
        umma_commit<1>(&empty_un[u]);
        if (A8) umma_commit<1>(&empty_pk[s]);
        if (step == nsteps - 1) umma_commit<1>(acc_full);
      }
      first = 0;
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
    // ------------------------------------------------- widening + epilogue
    // Group wg (warps 2 + 2 wg, 3 + 2 wg) widens the steps with
    // step % 2 == wg: piece c = ut + 64 i of a step is row c / 4 (weight
    // rows first, then token rows) and packed bytes [16 (c % 4), +16).
    const int wg = (warp - 2) / kGroupWarps;
    const int ut = threadIdx.x - 64 - wg * kGroupWarps * 32;  // 0 .. 63
    bool ok = true;
    for (int step = wg; step < nsteps; step += kGroups) {
      const int s = step % PS;
      const uint32_t ph = (step / PS) & 1;
      const int u = step % US;
      const uint32_t uph = (step / US) & 1;
      // widened slot first (its previous phase is this group's own step)
      if (!mbar_wait(&empty_un[u], uph ^ 1, abort_flag, kDevTimeoutUnpack)) { ok = false; break; }
      if (!mbar_wait(&full_pk[s], ph, abort_flag, kDevTimeoutUnpack)) { ok = false; break; }
      const uint8_t* pk = smem + L::oPk + s * L::kPk;
      uint8_t* un = smem + L::oUn + u * L::kUn;
      for (int c = ut; c < L::kPieces; c += kGroupWarps * 32) {
        const int row = c >> 2, q = c & 3;
        // weight rows live at the start of both stages; token rows follow
        const uint32_t src = (row < BM) ? row * (BK / 2) + q * 16 : L::kPkA + (row - BM) * (BK / 2) + q * 16;
        const uint32_t dst = (row < BM) ? row * BK : L::kUnA + (row - BM) * BK;
        const uint32_t chunk = ((2 * q) ^ (row & 7)) << 4;
        uint4 lo, hi;
        widen_run(*reinterpret_cast<const uint4*>(pk + src), lo, hi);
        *reinterpret_cast<uint4*>(un + dst + chunk) = lo;
        *reinterpret_cast<uint4*>(un + dst + (chunk ^ 16u)) = hi;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&empty_pk[s]);
        mbar_arrive(&full_un[u]);
      }
    }

    // ---------------------------------------------------------- epilogue
    // TMEM lane = weight row n0 + 32 (warp % 4) + lane, columns = tokens.
    grid_dep_wait();
    const int q = warp & 3;
    const int n = n0 + q * 32 + lane;
    constexpr int kShift = A8 ? 4 : 8;
    if (ok && mbar_wait(acc_full, 0, abort_flag, kDevTimeoutEpilogue)) {
      tc_fence_after();
      uint32_t a0[MP], a1[MP];
      const uint32_t tq = tmem + ((uint32_t)(q * 32) << 16);
      if constexpr (MP == 16) {
        tmem_ld_32x32b_x16(tq, a0);
        if (nres > 0) tmem_ld_32x32b_x16(tq + MP, a1);
      } else {
        tmem_ld_32x32b_x32(tq, a0);
        if (nres > 0) tmem_ld_32x32b_x32(tq + MP, a1);
      }
      if constexpr (MP == 16) {
        tmem_ld_wait_regs(a0, a1);
      } else {
        tmem_ld_wait_regs(a0);
        tmem_ld_wait_regs(a1);
      }
      if (nres == 0) {
#pragma unroll
        for (int m = 0; m < MP; ++m) a1[m] = 0;
      }
      if (p.splits == 1) {
        if (n < p.N) {
          const float swn = ACC_OUT ? 0.f : p.sw[n], srn = ACC_OUT ? 0.f : p.sr[n];
          float sxr[MP];
#pragma unroll
          for (int m = 0; m < MP; ++m) sxr[m] = (!ACC_OUT && m < p.M) ? __ldg(p.sx + m) : 0.f;
#pragma unroll
          for (int m = 0; m < MP; ++m) {
            if (m >= p.M) break;
            const int q0 = (int)a0[m] >> kShift, q1 = (int)a1[m] >> kShift;
            if (ACC_OUT) {
              p.acc0[(size_t)m * p.N + n] = q0;
              p.acc1[(size_t)m * p.N + n] = q1;
            } else {
              p.Y[(size_t)m * p.ldy + n] = __float2bfloat16_rn(sxr[m] * fmaf(swn, (float)q0, srn * (float)q1));
            }
          }
        }
      } else if (n < p.N) {
#pragma unroll
        for (int m = 0; m < MP; ++m) {
          if (m >= p.M) break;
          atomicAdd(&p.ws[(size_t)m * p.N + n], (int)a0[m] >> kShift);
          if (nres) atomicAdd(&p.ws[((size_t)kMaxM + m) * p.N + n], (int)a1[m] >> kShift);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (p.splits > 1 && threadIdx.x == 0 && !*abort_flag) {
    // every unit of the tile has added its sums once the counter reaches splits
    __threadfence();
    *last_flag = (atomicAdd(&p.cnt[tile], 1) == p.splits - 1);
    __threadfence();
  }
  __syncthreads();
  if (*last_flag && warp >= 2) {
    const int n = n0 + (warp & 3) * 32 + lane;
    if (n < p.N) {
      const float swn = ACC_OUT ? 0.f : p.sw[n], srn = ACC_OUT ? 0.f : p.sr[n];
      // every sum first (loads in flight together), then the stores
      int s0[MP], s1[MP];
      float sxr[MP];
#pragma unroll
      for (int m = 0; m < MP; ++m) {
        sxr[m] = (!ACC_OUT && m < p.M) ? __ldg(p.sx + m) : 0.f;
        s0[m] = (m < p.M) ? __ldcg(p.ws + (size_t)m * p.N + n) : 0;
        s1[m] = (m < p.M) ? __ldcg(p.ws + ((size_t)kMaxM + m) * p.N + n) : 0;
      }
#pragma unroll
      for (int m = 0; m < MP; ++m) {
        if (m >= p.M) break;
        p.ws[(size_t)m * p.N + n] = 0;
        p.ws[((size_t)kMaxM + m) * p.N + n] = 0;
        if (ACC_OUT) {
          p.acc0[(size_t)m * p.N + n] = s0[m];
          p.acc1[(size_t)m * p.N + n] = s1[m];
        } else {
          p.Y[(size_t)m * p.ldy + n] = __float2bfloat16_rn(sxr[m] * fmaf(swn, (float)s0[m], srn * (float)s1[m]));
        }
      }
    }
    if (threadIdx.x == 64) p.cnt[tile] = 0;
  }
  if (*abort_flag && warp == 0 && lane == 0) {
    const unsigned long long t0 = global_ns();
    while (global_ns() - t0 < 100000ull) {
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<1>(tmem, L::kTmemCols);
  }
}

}  // namespace dtc
}  // namespace serq
