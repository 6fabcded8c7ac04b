// libserq C ABI: argument checking, the prepared-layer handle, tensor-map
// construction and kernel dispatch.  Kernels live in the included headers;
// everything is one translation unit so the device status word is shared.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include "../../include/serq.h"
#include "common.cuh"
#include "gemm_tc.cuh"
#include "gemv_decode.cuh"
#include "gemv_stream.cuh"
#include "gemv_tc.cuh"
#include "prepare.cuh"
#include "gptq.cuh"
#include "quant.cuh"
#include "mxfp4.cuh"

namespace {

thread_local std::string g_last_error;

serq_status fail(serq_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

serq_status ok() {
  g_last_error.clear();
  return SERQ_OK;
}

serq_status cuda_fail(cudaError_t e, const char* what) {
  return fail(SERQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

serq_status check_device() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  static int cached[64] = {0};  // 0 unknown, 1 ok, 2 bad
  if (dev >= 0 && dev < 64 && cached[dev] == 1) return SERQ_OK;
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0) {
    return fail(SERQ_ERR_UNSUPPORTED_DEVICE, "device %d is sm_%d%d; libserq needs sm_100 (B200)", dev,
                major, minor);
  }
  if (dev >= 0 && dev < 64) cached[dev] = 1;
  return SERQ_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D tensor [rows][inner] of `dtype` elements with row stride `stride`
// bytes (inner and box_inner in elements).
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t stride,
              uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw,
              CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_UINT8) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {stride};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

struct serq_layer {
  int K, N, rank, rpad, mode, device;
  void* block;
  uint8_t* wq;
  uint8_t* rq;
  float* sw;
  float* sr;
  int32_t* perm;
  float* smooth;
  CUtensorMap tmB[3];  // box rows 128, 256, 96
  CUtensorMap tmR[3];
  CUtensorMap tmW4, tmR4;    // 256-byte x 4-row boxes (streaming decode kernel)
  CUtensorMap tmW16, tmR16;  // 256-byte x 16-row boxes (streaming decode kernel)
  int32_t* ws;         // split-K partial sums of the tensor-core decode, zero between calls
  int32_t* cnt;        // per 128-row tile: units done
};

namespace {

serq_status alloc_layer(int K, int N, int rank, int mode, serq_layer** out) {
  serq_layer* L = new (std::nothrow) serq_layer();
  if (!L) return fail(SERQ_ERR_ALLOC, "host allocation failed");
  std::memset(L, 0, sizeof(*L));
  L->K = K;
  L->N = N;
  L->rank = rank;
  L->rpad = (rank + 31) / 32 * 32;
  L->mode = mode;
  cudaGetDevice(&L->device);
  const size_t s_wq = up256((size_t)N * K / 2);
  const size_t s_rq = up256((size_t)N * L->rpad / 2);
  const size_t s_n = up256((size_t)N * 4);
  const size_t s_k = up256((size_t)K * 4);
  const size_t s_ws = up256((size_t)2 * N * serq::dtc::kMaxM * 4);
  const size_t s_cnt = up256((size_t)((N + 127) / 128) * 4);
  const size_t total = s_wq + s_rq + 2 * s_n + 2 * s_k + s_ws + s_cnt;
  cudaError_t e = cudaMalloc(&L->block, total);
  if (e != cudaSuccess) {
    delete L;
    cudaGetLastError();
    return fail(SERQ_ERR_ALLOC, "cudaMalloc(%zu) failed: %s", total, cudaGetErrorString(e));
  }
  uint8_t* b = static_cast<uint8_t*>(L->block);
  L->wq = b;
  b += s_wq;
  L->rq = L->rpad ? b : nullptr;
  b += s_rq;
  L->sw = reinterpret_cast<float*>(b);
  b += s_n;
  L->sr = reinterpret_cast<float*>(b);
  b += s_n;
  L->perm = reinterpret_cast<int32_t*>(b);
  b += s_k;
  L->smooth = reinterpret_cast<float*>(b);
  b += s_k;
  L->ws = reinterpret_cast<int32_t*>(b);
  b += s_ws;
  L->cnt = reinterpret_cast<int32_t*>(b);
  e = cudaMemset(L->ws, 0, s_ws + s_cnt);
  if (e != cudaSuccess) {
    cudaFree(L->block);
    delete L;
    cudaGetLastError();
    return fail(SERQ_ERR_CUDA, "cudaMemset of the workspace failed: %s", cudaGetErrorString(e));
  }
  *out = L;
  return SERQ_OK;
}

void free_layer(serq_layer* L) {
  if (!L) return;
  if (L->block) cudaFree(L->block);
  delete L;
}

bool build_weight_maps(serq_layer* L) {
  const int boxes[3] = {128, 256, 96};
  for (int i = 0; i < 3; ++i) {
    if (!make_map(&L->tmB[i], L->wq, (uint64_t)L->K / 2, (uint64_t)L->N, (uint64_t)L->K / 2, 64, boxes[i],
                  CU_TENSOR_MAP_SWIZZLE_NONE))
      return false;
    if (L->rpad) {
      if (!make_map(&L->tmR[i], L->rq, (uint64_t)L->rpad / 2, (uint64_t)L->N, (uint64_t)L->rpad / 2, 64,
                    boxes[i], CU_TENSOR_MAP_SWIZZLE_NONE))
        return false;
    } else {
      L->tmR[i] = L->tmB[i];  // never read when r = 0
    }
  }
  if (!make_map(&L->tmW4, L->wq, (uint64_t)L->K / 2, (uint64_t)L->N, (uint64_t)L->K / 2, 256, 4,
                CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_map(&L->tmW16, L->wq, (uint64_t)L->K / 2, (uint64_t)L->N, (uint64_t)L->K / 2, 256, 16,
                CU_TENSOR_MAP_SWIZZLE_NONE))
    return false;
  if (L->rpad) {
    if (!make_map(&L->tmR4, L->rq, (uint64_t)L->rpad / 2, (uint64_t)L->N, (uint64_t)L->rpad / 2, 256, 4,
                  CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&L->tmR16, L->rq, (uint64_t)L->rpad / 2, (uint64_t)L->N, (uint64_t)L->rpad / 2, 256, 16,
                  CU_TENSOR_MAP_SWIZZLE_NONE))
      return false;
  } else {
    L->tmR4 = L->tmW4;  // never read when r = 0
    L->tmR16 = L->tmW16;
  }
  return true;
}

serq_status check_layer(const serq_layer* L) {
  if (!L) return fail(SERQ_ERR_INVALID_ARG, "null layer");
  int dev = -1;
  cudaGetDevice(&dev);
  if (dev != L->device)
    return fail(SERQ_ERR_INVALID_ARG, "layer was prepared on device %d, current device is %d", L->device, dev);
  return SERQ_OK;
}



int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && cached[dev]) return cached[dev];
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (dev < 64) cached[dev] = sms;
  return sms;
}

// Opt-in shared memory per block of the current device.
int max_smem() {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && cached[dev]) return cached[dev];
  int v = 232448;
  cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (dev < 64) cached[dev] = v;
  return v;
}

// ------------------------------------------------------------ GEMM launch
// Layers whose products one launch computes (they read the same activation
// codes), with their outputs.
struct LinearGroup {
  int n;
  const serq_layer* L[serq::tc::kMaxGroup];
  __nv_bfloat16* Y[serq::tc::kMaxGroup];
  int ldy[serq::tc::kMaxGroup];
  int32_t* acc0[serq::tc::kMaxGroup];
  int32_t* acc1[serq::tc::kMaxGroup];
};

// Xr / sxr: the two-factor comparator's second activation (codes M x rpad,
// packed like Xq, and its per-row scales) for the residual steps; null for
// SERQ, whose residual reads the first r columns of Xq.
template <int BN, bool A8, bool ACC, int CG, bool TWO = false>
cudaError_t launch_tc(const LinearGroup& G, const void* Xq, const float* sx, int M, cudaStream_t st,
                      const void* Xr = nullptr, const float* sxr = nullptr) {
  using Lay = serq::tc::Layout<BN, A8, CG>;
  const serq_layer* L0 = G.L[0];
  const int K = L0->K;
  CUtensorMap tmA;
  bool okm = A8 ? make_map(&tmA, Xq, (uint64_t)K, (uint64_t)M, (uint64_t)K, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B)
                : make_map(&tmA, Xq, (uint64_t)K / 2, (uint64_t)M, (uint64_t)K / 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!okm) return cudaErrorInvalidValue;
  // weight maps by box rows: [0] 128, [1] 256 (BN / CG rows per CTA)
  const int bi = (BN / CG == 256) ? 1 : 0;
  static_assert(BN / CG == 128 || BN / CG == 256, "weight box rows");
  serq::tc::GroupArgs ga = {};
  serq::tc::GroupMaps mp;
  ga.M = M;
  ga.K = K;
  ga.rpad = L0->rpad;
  ga.nkb = (K + serq::tc::BK - 1) / serq::tc::BK;
  ga.nrb = (L0->rpad + serq::tc::BK - 1) / serq::tc::BK;
  ga.sx = sx;
  ga.sxr = sxr;
  ga.tiles_m = (M + serq::tc::BM * CG - 1) / (serq::tc::BM * CG);
  mp.ar = tmA;
  if (Xr && !make_map(&mp.ar, Xr, (uint64_t)L0->rpad / 2, (uint64_t)M, (uint64_t)L0->rpad / 2, 64, 128,
                      CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  ga.nlayers = G.n;
  int base = 0;
  for (int l = 0; l < serq::tc::kMaxGroup; ++l) {
    const int li = (l < G.n) ? l : 0;  // unused slots repeat layer 0
    const serq_layer* Ll = G.L[li];
    mp.b[l] = Ll->tmB[bi];
    mp.r[l] = Ll->tmR[bi];
    mp.y[l] = tmA;
    // output: bf16 [M][N] with row stride ldy, boxes of 32 rows x 64 columns
    if (!ACC && !make_map(&mp.y[l], G.Y[li], (uint64_t)Ll->N, (uint64_t)M, (uint64_t)G.ldy[li] * 2, 64, 32,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16))
      return cudaErrorInvalidValue;
    ga.lo[l] = serq::tc::LayerOut{Ll->N, base, Ll->sw, Ll->sr, G.Y[li], G.ldy[li], G.acc0[li], G.acc1[li]};
    if (l < G.n) base += ga.tiles_m * ((Ll->N + BN - 1) / BN);
  }
  ga.ntiles = base;
  auto kern = serq::tc::k_gemm<BN, A8, ACC, CG, TWO>;
  {
    const cudaError_t ea = serq::smem_limit(reinterpret_cast<const void*>(kern), Lay::kAlloc);
    if (ea != cudaSuccess) return ea;
  }
  // persistent: one CTA (pair) per SM (pair of SMs), tiles strided over them
  const long slots = sm_count() / CG;
  dim3 grid((unsigned)((base < slots ? base : slots) * CG), 1);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(serq::tc::kThreads);
  cfg.dynamicSmemBytes = Lay::kAlloc;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CG;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see the producer's first steps
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, tmA, mp, ga);
}

// W4A4 on CTA pairs with the activations in tensor memory, 256 x 192 tiles.
template <bool ACC>
cudaError_t launch_tc_ta(const serq_layer* L, const void* Xq, const serq::tc::Args& a, cudaStream_t st) {
  constexpr int BN = 192;
  using Lay = serq::tc::LayoutTA<BN>;
  CUtensorMap tmA;
  if (!make_map(&tmA, Xq, (uint64_t)a.K / 2, (uint64_t)a.M, (uint64_t)a.K / 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  CUtensorMap tmY = tmA;
  if (!ACC && !make_map(&tmY, a.Y, (uint64_t)a.N, (uint64_t)a.M, (uint64_t)a.ldy * 2, 32, 32,
                        CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16))
    return cudaErrorInvalidValue;
  auto kern = serq::tc::k_gemm_ta<BN, ACC>;
  {
    const cudaError_t ea = serq::smem_limit(reinterpret_cast<const void*>(kern), Lay::kAlloc);
    if (ea != cudaSuccess) return ea;
  }
  serq::tc::Args ap = a;
  ap.tiles_m = (a.M + 255) / 256;
  ap.tiles_n = (a.N + BN - 1) / BN;
  const long ntiles = (long)ap.tiles_m * ap.tiles_n;
  const long slots = sm_count() / 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((ntiles < slots ? ntiles : slots) * 2), 1);
  cfg.blockDim = dim3(serq::tc::kThreads);
  cfg.dynamicSmemBytes = Lay::kAlloc;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tmA, L->tmB[2], L->tmR[2], tmY, ap);
}

// Tensor-core decode (weights as the MMA's M), split-K over about two units
// per SM.
template <int MP, bool A8, bool ACC>
cudaError_t launch_decode_tc(const serq_layer* L, const void* Xq, serq::dtc::Args a, cudaStream_t st) {
  using Lay = serq::dtc::Layout<MP, A8>;
  CUtensorMap tmX;
  bool okm = A8 ? make_map(&tmX, Xq, (uint64_t)a.K, (uint64_t)a.M, (uint64_t)a.K, 128, MP, CU_TENSOR_MAP_SWIZZLE_128B)
                : make_map(&tmX, Xq, (uint64_t)a.K / 2, (uint64_t)a.M, (uint64_t)a.K / 2, 64, MP, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!okm) return cudaErrorInvalidValue;
  auto kern = serq::dtc::k_decode_tc<MP, A8, ACC>;
  {
    const cudaError_t ea = serq::smem_limit(reinterpret_cast<const void*>(kern), Lay::kAlloc);
    if (ea != cudaSuccess) return ea;
  }
  const int tiles = (a.N + serq::dtc::BM - 1) / serq::dtc::BM;
  int splits = (2 * sm_count() + tiles / 2) / tiles;
  if (splits < 1) splits = 1;
  if (splits > a.nkb) splits = a.nkb;
  a.splits = splits;
  if (!a.ws) {  // the layer's workspace unless the caller brings one
    a.ws = L->ws;
    a.cnt = L->cnt;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(tiles * splits));
  cfg.blockDim = dim3(serq::dtc::kThreads);
  cfg.dynamicSmemBytes = Lay::kAlloc;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, L->tmB[0], L->tmR[0], tmX, a);
}

template <bool A8, bool ACC>
cudaError_t dispatch_decode_tc(const serq_layer* L, const void* Xq, const serq::dtc::Args& a, cudaStream_t st) {
  return (a.M <= 16) ? launch_decode_tc<16, A8, ACC>(L, Xq, a, st) : launch_decode_tc<32, A8, ACC>(L, Xq, a, st);
}

template <bool A8, bool ACC>
cudaError_t dispatch_tc(const LinearGroup& G, const void* Xq, const float* sx, int M, serq_algo algo,
                        cudaStream_t st) {
  switch (algo) {
    case SERQ_ALGO_PREFILL_N128: return launch_tc<128, A8, ACC, 1>(G, Xq, sx, M, st);
    case SERQ_ALGO_PREFILL_N256: return launch_tc<256, A8, ACC, 1>(G, Xq, sx, M, st);
    case SERQ_ALGO_PREFILL_PAIR_N256: return launch_tc<256, A8, ACC, 2>(G, Xq, sx, M, st);
    case SERQ_ALGO_PREFILL_PAIR_TMEM_A: {
      if (A8 || G.n != 1) return cudaErrorInvalidValue;
      const serq_layer* L = G.L[0];
      serq::tc::Args a{M, L->K, L->N, L->rpad, (L->K + serq::tc::BK - 1) / serq::tc::BK,
                       (L->rpad + serq::tc::BK - 1) / serq::tc::BK, sx, L->sw, L->sr, G.Y[0], G.ldy[0],
                       G.acc0[0], G.acc1[0]};
      return launch_tc_ta<ACC>(L, Xq, a, st);
    }
    default: break;
  }
  // CTA pairs with 256 x 256 tiles unless that leaves most SMs idle; then
  // single-CTA 128 x 128 tiles.
  long ctas_pair = 0;
  for (int l = 0; l < G.n; ++l) ctas_pair += (long)((G.L[l]->N + 255) / 256) * 2 * ((M + 255) / 256);
  if (ctas_pair * 10 >= (long)sm_count() * 9) return launch_tc<256, A8, ACC, 2>(G, Xq, sx, M, st);
  return launch_tc<128, A8, ACC, 1>(G, Xq, sx, M, st);
}

// The mma.sync decode kernels over a group of layers (one launch; one layer
// is a group of one).  kind: 0 = automatic (the streaming kernel when every
// SM's share of the weights is at least 96 KB and its shared memory fits,
// else the item ring: for a share of one or two 16-channel items per SM its
// simpler start-up is measured faster), 1 = item ring, 2 = streaming where
// it fits.  fault_wait_ns is zero except in the failure-detection test hook.
// Xh (bf16, K <= 4096, else null): the activations still to be quantized;
// the streaming kernel quantizes them itself, the item ring after a
// quantize launch into Xq / sx (then scratch the caller provided).
cudaError_t launch_decode_group(const LinearGroup& G, const void* Xq, const float* sx, int M, bool a8, bool accum,
                                int kind, cudaStream_t st, unsigned long long fault_wait_ns = 0,
                                const __nv_bfloat16* Xh = nullptr, int ldxh = 0) {
  if (Xh && kind == 0) {
    kind = 2;  // one launch: the quantize lives in the streaming kernel
  } else if (kind == 0) {
    double bytes = 0;
    for (int l = 0; l < G.n; ++l) bytes += (double)G.L[l]->N * (G.L[l]->K / 2 + G.L[l]->rpad / 2);
    kind = (bytes >= 96.0 * 1024 * sm_count() || fault_wait_ns) ? 2 : 1;
  }
  if (kind == 2) {
    serq::gs::Args g = {};
    serq::gs::Maps mp;
    g.Xq = static_cast<const uint8_t*>(Xq);
    g.sx = sx;
    g.Xh = Xh;
    g.ldxh = ldxh;
    g.M = M;
    g.K = G.L[0]->K;
    g.rpad = G.L[0]->rpad;
    g.nlayers = G.n;
    int base = 0;
    for (int l = 0; l < serq::gs::kMaxGroup; ++l) {
      const int li = (l < G.n) ? l : 0;
      const serq_layer* L = G.L[li];
      g.lo[l] = serq::gs::Layer{L->wq, L->rq, L->sw, L->sr, G.Y[li], G.ldy[li], G.acc0[li], G.acc1[li], L->N,
                                l < G.n ? base : 1 << 30};
      mp.w[l] = L->tmW4;
      mp.r[l] = L->tmR4;
      mp.w16[l] = L->tmW16;
      mp.r16[l] = L->tmR16;
      if (l < G.n) base += L->N;
    }
    g.C = base;
    const bool fit = a8 ? serq::gs::fits<true>(g, sm_count(), max_smem()) : serq::gs::fits<false>(g, sm_count(), max_smem());
    if (fit) {
      if (a8)
        return accum ? serq::gs::launch<true, true>(g, mp, sm_count(), max_smem(), st, fault_wait_ns)
                     : serq::gs::launch<true, false>(g, mp, sm_count(), max_smem(), st, fault_wait_ns);
      return accum ? serq::gs::launch<false, true>(g, mp, sm_count(), max_smem(), st, fault_wait_ns)
                   : serq::gs::launch<false, false>(g, mp, sm_count(), max_smem(), st, fault_wait_ns);
    }
    if (fault_wait_ns) return cudaErrorInvalidValue;
  }
  if (Xh) {
    const serq::quant::LoadBF16 ld{Xh, ldxh};
    uint8_t* q = static_cast<uint8_t*>(const_cast<void*>(Xq));
    float* sq = const_cast<float*>(sx);
    const cudaError_t e = a8 ? serq::quant::launch_quant_rows<127>(ld, M, G.L[0]->K, q, sq, st)
                             : serq::quant::launch_quant_rows<7>(ld, M, G.L[0]->K, q, sq, st);
    if (e != cudaSuccess) return e;
  }
  serq::decode::Args a = {};
  a.Xq = static_cast<const uint8_t*>(Xq);
  a.sx = sx;
  a.M = M;
  a.K = G.L[0]->K;
  a.rpad = G.L[0]->rpad;
  a.nlayers = G.n;
  int items_n = 0;
  for (int l = 0; l < serq::decode::kMaxGroup; ++l) {
    const int li = (l < G.n) ? l : 0;
    const serq_layer* L = G.L[li];
    a.lo[l] = serq::decode::LayerDec{L->wq, L->rq, L->sw, L->sr, G.Y[li], G.ldy[li], G.acc0[li], G.acc1[li], L->N, items_n};
    if (l < G.n) items_n += L->N / serq::decode::kRows;
  }
  a.N = items_n * serq::decode::kRows;
  if (a8)
    return accum ? serq::decode::launch<true, true>(a, sm_count(), max_smem(), st)
                 : serq::decode::launch<true, false>(a, sm_count(), max_smem(), st);
  return accum ? serq::decode::launch<false, true>(a, sm_count(), max_smem(), st)
               : serq::decode::launch<false, false>(a, sm_count(), max_smem(), st);
}

int decode_kind(serq_algo a) {
  return a == SERQ_ALGO_DECODE_ITEMS ? 1 : a == SERQ_ALGO_DECODE_STREAM ? 2 : 0;
}

// Argument checks shared by the single-layer and grouped calls; resolves AUTO.
serq_status check_linear(const serq_layer* L, const void* Xq, const float* sx, int M, const void* Y, int ldy,
                         const int32_t* acc0, const int32_t* acc1, serq_algo* algo_io) {
  serq_status s;
  serq_algo algo = *algo_io;
  if (!L) return fail(SERQ_ERR_INVALID_ARG, "null layer");
  const bool accum = (acc0 != nullptr);
  if (!Xq) return fail(SERQ_ERR_INVALID_ARG, "null Xq");
  if (M < 1 || M > 65535 * 128) return fail(SERQ_ERR_INVALID_ARG, "M = %d out of range", M);
  if (!aligned16(Xq)) return fail(SERQ_ERR_INVALID_ARG, "Xq must be 16-byte aligned");
  if (accum) {
    if (!acc1) return fail(SERQ_ERR_INVALID_ARG, "null acc1");
    if (!aligned16(acc0) || !aligned16(acc1)) return fail(SERQ_ERR_INVALID_ARG, "acc0/acc1 must be 16-byte aligned");
  } else {
    if (!sx || !Y) return fail(SERQ_ERR_INVALID_ARG, "null sx or Y");
    if (ldy < L->N) return fail(SERQ_ERR_INVALID_ARG, "ldy (%d) < N (%d)", ldy, L->N);
    if (!aligned16(Y) || (ldy % 8) != 0)
      return fail(SERQ_ERR_INVALID_ARG, "Y must be 16-byte aligned with ldy a multiple of 8");
  }
  if (algo == SERQ_ALGO_AUTO) algo = (M <= serq_decode_max_m()) ? SERQ_ALGO_DECODE : SERQ_ALGO_PREFILL;
  if ((algo == SERQ_ALGO_DECODE || algo == SERQ_ALGO_DECODE_ITEMS || algo == SERQ_ALGO_DECODE_STREAM) &&
      M > serq::decode::kMaxTiles * 16)
    return fail(SERQ_ERR_UNSUPPORTED_SHAPE, "decode kernel takes M <= %d (got %d)", serq::decode::kMaxTiles * 16, M);
  if (algo == SERQ_ALGO_DECODE_TC && M > serq::dtc::kMaxM)
    return fail(SERQ_ERR_UNSUPPORTED_SHAPE, "SERQ_ALGO_DECODE_TC takes M <= %d (got %d)", serq::dtc::kMaxM, M);
  if (algo < SERQ_ALGO_PREFILL || algo > SERQ_ALGO_DECODE_STREAM) return fail(SERQ_ERR_INVALID_ARG, "bad algo %d", (int)algo);
  if (algo == SERQ_ALGO_PREFILL_PAIR_TMEM_A && L->mode != SERQ_W4A4)
    return fail(SERQ_ERR_INVALID_ARG, "SERQ_ALGO_PREFILL_PAIR_TMEM_A takes W4A4 layers");
  if ((s = check_device())) return s;
  if ((s = check_layer(L))) return s;
  *algo_io = algo;
  return ok();
}

serq_status linear_impl(const serq_layer* L, const void* Xq, const float* sx, int M, void* Y, int ldy,
                        int32_t* acc0, int32_t* acc1, serq_algo algo, void* stream, int32_t* scratch = nullptr,
                        int32_t* scratch_cnt = nullptr) {
  serq_status s;
  if ((s = check_linear(L, Xq, sx, M, Y, ldy, acc0, acc1, &algo))) return s;
  const bool accum = (acc0 != nullptr);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool a8 = (L->mode == SERQ_W4A8);
  cudaError_t e;
  if (algo == SERQ_ALGO_DECODE_TC) {
    serq::dtc::Args a{M, L->K, L->N, L->rpad, (L->K + serq::dtc::BK - 1) / serq::dtc::BK,
                      (L->rpad + serq::dtc::BK - 1) / serq::dtc::BK, 1, sx, L->sw, L->sr,
                      static_cast<__nv_bfloat16*>(Y), ldy, acc0, acc1, scratch, scratch_cnt};
    if (a8)
      e = accum ? dispatch_decode_tc<true, true>(L, Xq, a, st) : dispatch_decode_tc<true, false>(L, Xq, a, st);
    else
      e = accum ? dispatch_decode_tc<false, true>(L, Xq, a, st) : dispatch_decode_tc<false, false>(L, Xq, a, st);
  } else if (algo == SERQ_ALGO_DECODE || algo == SERQ_ALGO_DECODE_ITEMS || algo == SERQ_ALGO_DECODE_STREAM) {
    LinearGroup G = {};
    G.n = 1;
    G.L[0] = L;
    G.Y[0] = static_cast<__nv_bfloat16*>(Y);
    G.ldy[0] = ldy;
    G.acc0[0] = acc0;
    G.acc1[0] = acc1;
    e = launch_decode_group(G, Xq, sx, M, a8, accum, decode_kind(algo), st);
  } else {
    LinearGroup G = {};
    G.n = 1;
    G.L[0] = L;
    G.Y[0] = static_cast<__nv_bfloat16*>(Y);
    G.ldy[0] = ldy;
    G.acc0[0] = acc0;
    G.acc1[0] = acc1;
    if (a8)
      e = accum ? dispatch_tc<true, true>(G, Xq, sx, M, algo, st) : dispatch_tc<true, false>(G, Xq, sx, M, algo, st);
    else
      e = accum ? dispatch_tc<false, true>(G, Xq, sx, M, algo, st) : dispatch_tc<false, false>(G, Xq, sx, M, algo, st);
  }
  if (e != cudaSuccess) return cuda_fail(e, "serq_linear launch");
  return ok();
}

// Several layers over the same activation codes: the prefill kernels and the
// mma.sync decode kernels run them as one launch (one tile or channel space,
// one pass of setup and tail); SERQ_ALGO_DECODE_TC and the TMEM-activation
// variant run them one launch per layer.
serq_status group_impl(int n, const serq_layer* const* Ls, const void* Xq, const float* sx, int M,
                       void* const* Y, const int* ldy, int32_t* const* acc0, int32_t* const* acc1, serq_algo algo,
                       void* stream, const __nv_bfloat16* Xh = nullptr, int ldxh = 0) {
  serq_status s;
  if (n < 1 || n > serq::tc::kMaxGroup)
    return fail(SERQ_ERR_INVALID_ARG, "group of %d layers (1..%d)", n, serq::tc::kMaxGroup);
  if (!Ls) return fail(SERQ_ERR_INVALID_ARG, "null layer list");
  if ((acc0 == nullptr) != (acc1 == nullptr)) return fail(SERQ_ERR_INVALID_ARG, "acc0 and acc1: both or neither");
  const bool accum = (acc0 != nullptr);
  if (!accum && (!Y || !ldy)) return fail(SERQ_ERR_INVALID_ARG, "null Y or ldy list");
  serq_algo resolved = algo;
  for (int l = 0; l < n; ++l) {
    if (!Ls[l]) return fail(SERQ_ERR_INVALID_ARG, "null layer %d", l);
    if (Ls[l]->K != Ls[0]->K || Ls[l]->rpad != Ls[0]->rpad || Ls[l]->mode != Ls[0]->mode)
      return fail(SERQ_ERR_INVALID_ARG, "layer %d differs from layer 0 in K, rank or mode", l);
    serq_algo a = algo;
    if ((s = check_linear(Ls[l], Xq, sx, M, accum ? nullptr : Y[l], accum ? 0 : ldy[l], accum ? acc0[l] : nullptr,
                          accum ? acc1[l] : nullptr, &a)))
      return s;
    resolved = a;
  }
  if (resolved == SERQ_ALGO_DECODE_TC || resolved == SERQ_ALGO_PREFILL_PAIR_TMEM_A) {
    for (int l = 0; l < n; ++l)
      if ((s = linear_impl(Ls[l], Xq, sx, M, accum ? nullptr : Y[l], accum ? 0 : ldy[l], accum ? acc0[l] : nullptr,
                           accum ? acc1[l] : nullptr, resolved, stream)))
        return s;
    return ok();
  }
  LinearGroup G = {};
  G.n = n;
  for (int l = 0; l < n; ++l) {
    G.L[l] = Ls[l];
    G.Y[l] = accum ? nullptr : static_cast<__nv_bfloat16*>(Y[l]);
    G.ldy[l] = accum ? 0 : ldy[l];
    G.acc0[l] = accum ? acc0[l] : nullptr;
    G.acc1[l] = accum ? acc1[l] : nullptr;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (resolved == SERQ_ALGO_DECODE || resolved == SERQ_ALGO_DECODE_ITEMS || resolved == SERQ_ALGO_DECODE_STREAM) {
    e = launch_decode_group(G, Xq, sx, M, Ls[0]->mode == SERQ_W4A8, accum, decode_kind(resolved), st, 0, Xh, ldxh);
    if (e != cudaSuccess) return cuda_fail(e, "serq_linear_group launch");
    return ok();
  }
  if (Ls[0]->mode == SERQ_W4A8)
    e = accum ? dispatch_tc<true, true>(G, Xq, sx, M, resolved, st)
              : dispatch_tc<true, false>(G, Xq, sx, M, resolved, st);
  else
    e = accum ? dispatch_tc<false, true>(G, Xq, sx, M, resolved, st)
              : dispatch_tc<false, false>(G, Xq, sx, M, resolved, st);
  if (e != cudaSuccess) return cuda_fail(e, "serq_linear_group launch");
  return ok();
}

serq_status check_rows(const void* X, int M, int K, int ld, int elem, const char* name) {
  if (!X) return fail(SERQ_ERR_INVALID_ARG, "null %s", name);
  if (M < 1 || M > 2147483647) return fail(SERQ_ERR_INVALID_ARG, "M = %d out of range", M);
  if (K < 32 || K % 32) return fail(SERQ_ERR_UNSUPPORTED_SHAPE, "K = %d must be a positive multiple of 32", K);
  if (ld < K) return fail(SERQ_ERR_INVALID_ARG, "leading dimension of %s (%d) < K (%d)", name, ld, K);
  if (!aligned16(X) || ((size_t)ld * elem) % 16)
    return fail(SERQ_ERR_INVALID_ARG, "%s rows must start 16-byte aligned", name);
  return SERQ_OK;
}

// Scratch of serq_linear_decode_static: split-K partial sums [2][32][N] and
// tile counters of the tensor-core decode kernel, compiled into the library
// (one copy per device), so that the call allocates nothing.
constexpr int kStaticMaxN = 16384;
constexpr size_t kStaticCntOffset = (size_t)2 * serq::dtc::kMaxM * kStaticMaxN;
constexpr size_t kStaticInts = kStaticCntOffset + kStaticMaxN / serq::dtc::BM;
static __device__ __align__(256) int32_t g_decode_scratch[kStaticInts];

// Device address of the scratch, looked up once per device with that device
// current.  The scratch must start at zero and every completed call leaves it
// zero, so it is cleared (on the call's own stream, ordered before the
// kernel) only on the first call on a device and after a kernel reported a
// timed-out wait, which can leave partial sums behind.
std::mutex g_static_mu;
int32_t* g_static_addr[64] = {nullptr};
bool g_static_dirty[64] = {false};

serq_status static_scratch(cudaStream_t st, int32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(SERQ_ERR_UNSUPPORTED_DEVICE, "device index %d", dev);
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (!g_static_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the static decode scratch");
    g_static_addr[dev] = static_cast<int32_t*>(p);
    g_static_dirty[dev] = true;
  }
  if (g_static_dirty[dev]) {
    e = cudaMemsetAsync(g_static_addr[dev], 0, kStaticInts * sizeof(int32_t), st);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the static decode scratch");
    g_static_dirty[dev] = false;
  }
  *out = g_static_addr[dev];
  return SERQ_OK;
}

// After a reported timeout on `dev`, the next static call clears the scratch.
void static_scratch_mark_dirty(int dev) {
  if (dev < 0 || dev >= 64) return;
  std::lock_guard<std::mutex> lock(g_static_mu);
  g_static_dirty[dev] = true;
}

}  // namespace

extern "C" {

const char* serq_version(void) { return "libserq 0.1 (sm_100a)"; }

const char* serq_last_error_string(void) { return g_last_error.c_str(); }

int serq_decode_max_m(void) { return 32; }

serq_status serq_check_device(void) {
  serq_status s = check_device();
  return s ? s : ok();
}

serq_status serq_device_error(int* code) {
  if (!code) return fail(SERQ_ERR_INVALID_ARG, "null code");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  int v = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&v, serq::g_device_status, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "read device status");
  e = cudaMemcpyToSymbol(serq::g_device_status, &zero, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "clear device status");
  if (v != 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) static_scratch_mark_dirty(dev);
  }
  *code = v;
  return ok();
}

void serq_prepare_opts_init(serq_prepare_opts* opts) {
  if (!opts) return;
  opts->alpha = 0.5f;
  opts->rank = 128;
  opts->mode = SERQ_W4A4;
  opts->saliency = SERQ_SALIENCY_SCALE;
  opts->out_perm = nullptr;
  opts->out_colscale = nullptr;
  opts->quantizer = SERQ_QUANT_RTN;
}

}  // extern "C"

namespace {

// Checks the options shared by every prepare entry point.
serq_status check_opts(const serq_prepare_opts* o, int K) {
  if (!o) return fail(SERQ_ERR_INVALID_ARG, "null options");
  if (!(o->alpha >= 0.f && o->alpha <= 1.f)) return fail(SERQ_ERR_INVALID_ARG, "alpha = %g not in [0, 1]", o->alpha);
  if (o->rank < 0 || o->rank > K) return fail(SERQ_ERR_UNSUPPORTED_SHAPE, "rank %d not in [0, K=%d]", o->rank, K);
  if (o->mode != SERQ_W4A4 && o->mode != SERQ_W4A8) return fail(SERQ_ERR_INVALID_ARG, "bad mode %d", (int)o->mode);
  if (o->saliency != SERQ_SALIENCY_SCALE && o->saliency != SERQ_SALIENCY_ROW_ABSMAX)
    return fail(SERQ_ERR_INVALID_ARG, "bad saliency metric %d", o->saliency);
  if (o->quantizer != SERQ_QUANT_RTN && o->quantizer != SERQ_QUANT_GPTQ)
    return fail(SERQ_ERR_INVALID_ARG, "bad quantizer %d", o->quantizer);
  return SERQ_OK;
}

// Device buffers of one call, freed when the owner goes out of scope.
struct Scratch {
  std::vector<void*> bufs;
  ~Scratch() {
    for (void* b : bufs) cudaFree(b);
  }
  template <class T>
  serq_status get(size_t count, T** out, const char* what) {
    *out = nullptr;
    void* d = nullptr;
    cudaError_t e = cudaMalloc(&d, std::max<size_t>(count, 1) * sizeof(T));
    if (e != cudaSuccess) {
      cudaGetLastError();
      return fail(SERQ_ERR_ALLOC, "cudaMalloc of %zu bytes for %s failed: %s", count * sizeof(T), what,
                  cudaGetErrorString(e));
    }
    bufs.push_back(d);
    *out = static_cast<T*>(d);
    return SERQ_OK;
  }
};

template <typename TP, bool PT, bool QT, bool SUB>
void launch_tile(const serq::gptq::TileArgs& a, cudaStream_t st) {
  using namespace serq::gptq;
  const int ti = (a.mi + kTile - 1) / kTile;
  const int blocks = a.lower ? ti * (ti + 1) / 2 : ti * a.ntj;
  if (blocks > 0) k_tile<TP, PT, QT, SUB><<<blocks, 256, 0, st>>>(a);
}

// In-place Cholesky of the lower triangle of A (K x K): 32-column panels,
// each the diagonal block, the rows below it, then the trailing update.
void chol_lower(double* A, int K, int* status, cudaStream_t st) {
  using namespace serq::gptq;
  for (int j0 = 0; j0 < K; j0 += kChunk) {
    k_chol_diag<<<1, 32, 0, st>>>(A, K, j0, status);
    const int rest = K - j0 - kChunk;
    if (rest <= 0) break;
    k_chol_trsm<<<(rest + 127) / 128, 128, 0, st>>>(A, K, j0);
    TileArgs t{};
    t.C = A; t.ldc = K; t.ci0 = t.cj0 = j0 + kChunk; t.mi = t.mj = rest;
    t.P = A; t.ldp = K; t.pi0 = j0 + kChunk;
    t.Q = A; t.ldq = K; t.qj0 = j0 + kChunk;
    t.kb = j0; t.ke = j0 + kChunk; t.lower = 1;
    launch_tile<double, true, true, true>(t, st);
  }
}

// U (K x K upper; fp32 and/or fp64) with H^-1 = U^T U for the damped
// Hessian of Xh (n x K fp32, device).  All pointers device.
serq_status gptq_factor(const float* Xh, int n, int K, float* U32, double* U64, cudaStream_t st) {
  using namespace serq::gptq;
  Scratch sc;
  double *A = nullptr, *B = nullptr;
  int* status = nullptr;
  serq_status s;
  const size_t kk = (size_t)K * K;
  if ((s = sc.get(kk, &A, "the GPTQ Hessian"))) return s;
  if ((s = sc.get(kk, &B, "the GPTQ inverse"))) return s;
  if ((s = sc.get(1, &status, "a status word"))) return s;
  cudaMemsetAsync(status, 0, sizeof(int), st);
  // H = Xh^T Xh (lower), damped
  TileArgs g{};
  g.C = A; g.ldc = K; g.mi = g.mj = K;
  g.P = Xh; g.ldp = K; g.Q = Xh; g.ldq = K;
  g.kb = 0; g.ke = n; g.lower = 1;
  launch_tile<float, false, false, false>(g, st);
  k_damp<<<1, 256, 0, st>>>(A, K);
  chol_lower(A, K, status, st);
  // V = L^-1 in B (forward substitution on the identity, 32-row panels)
  const unsigned eb = (unsigned)((kk + 255) / 256);
  k_identity<<<eb, 256, 0, st>>>(B, K);
  for (int i0 = 0; i0 < K; i0 += kChunk) {
    k_inv_panel<<<(i0 + kChunk + 127) / 128, 128, 0, st>>>(A, B, K, i0);
    const int rest = K - i0 - kChunk;
    if (rest <= 0) break;
    TileArgs t{};
    t.C = B; t.ldc = K; t.ci0 = i0 + kChunk; t.cj0 = 0; t.mi = rest; t.mj = i0 + kChunk;
    t.P = A; t.ldp = K; t.pi0 = i0 + kChunk;
    t.Q = B; t.ldq = K; t.qj0 = 0;
    t.kb = i0; t.ke = i0 + kChunk; t.lower = 0; t.ntj = (t.mj + kTile - 1) / kTile;
    launch_tile<double, true, false, true>(t, st);
  }
  // H^-1 = V^T V (lower; a tile's sum starts at its first row: V is lower)
  TileArgs h{};
  h.C = A; h.ldc = K; h.mi = h.mj = K;
  h.P = B; h.ldp = K; h.Q = B; h.ldq = K;
  h.kb = 0; h.ke = K; h.kb_row_tile = 1; h.lower = 1;
  launch_tile<double, false, false, false>(h, st);
  chol_lower(A, K, status, st);
  k_upper_from_lower<<<eb, 256, 0, st>>>(A, K, U32, U64);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "GPTQ factor launch");
  int flag = 0;
  e = cudaMemcpyAsync(&flag, status, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "GPTQ factor");
  if (flag) return fail(SERQ_ERR_NUMERIC, "GPTQ: a Cholesky pivot was not positive (K = %d, %d calibration rows)", K, n);
  return SERQ_OK;
}

// The offline stage on device-resident inputs (all pointers DEVICE).
serq_status prepare_impl(int n_weights, const float* const* W, const int* N, int K, const float* X_calib,
                         int n_calib, const serq_prepare_opts& o, const int32_t* const* out_perm,
                         const float* const* out_div, serq_layer** layers) {
  serq_status s;
  const int rank = o.rank;
  for (int i = 0; i < n_weights; ++i) {
    s = alloc_layer(K, N[i], rank, o.mode, &layers[i]);
    if (s) {
      for (int j = 0; j < i; ++j) {
        free_layer(layers[j]);
        layers[j] = nullptr;
      }
      return s;
    }
  }
  auto cleanup = [&](serq_status st) {
    for (int i = 0; i < n_weights; ++i) {
      free_layer(layers[i]);
      layers[i] = nullptr;
    }
    return st;
  };
  float* key = nullptr;
  cudaError_t e = cudaMalloc(&key, sizeof(float) * K);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cleanup(fail(SERQ_ERR_ALLOC, "cudaMalloc of the saliency keys failed: %s", cudaGetErrorString(e)));
  }
  cudaStream_t st;
  e = cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking);
  if (e != cudaSuccess) {
    cudaFree(key);
    return cleanup(cuda_fail(e, "cudaStreamCreate"));
  }
  using namespace serq::prep;
  serq_layer* L0 = layers[0];
  auto view = [&](int i) {
    return WeightView{W[i], N[i], out_perm ? out_perm[i] : nullptr, out_div ? out_div[i] : nullptr};
  };
  // 1. flattening scales: amax_x into L0->smooth, amax_w into L0->perm's bytes
  float* amax_w = reinterpret_cast<float*>(L0->perm);
  k_colmax_abs<<<(K + 255) / 256, 256, 0, st>>>(X_calib, n_calib, K, L0->smooth);
  cudaMemsetAsync(amax_w, 0, sizeof(float) * K, st);
  for (int i = 0; i < n_weights; ++i) k_rowmax_abs<<<K, 256, 0, st>>>(view(i), K, amax_w);
  k_smooth<<<(K + 255) / 256, 256, 0, st>>>(L0->smooth, amax_w, K, o.alpha);
  // 2. saliency order
  k_saliency_key<<<(K + 255) / 256, 256, 0, st>>>(L0->smooth, amax_w, K, o.saliency, key);
  k_rank_perm<<<(K + 255) / 256, 256, 256 * sizeof(float), st>>>(key, K, L0->perm);
  for (int i = 1; i < n_weights; ++i) {
    cudaMemcpyAsync(layers[i]->smooth, L0->smooth, sizeof(float) * K, cudaMemcpyDeviceToDevice, st);
    cudaMemcpyAsync(layers[i]->perm, L0->perm, sizeof(int32_t) * K, cudaMemcpyDeviceToDevice, st);
  }
  // 3 (GPTQ). the inverse-Hessian factor of the flattened, permuted
  // calibration activations, shared by every weight of the group
  Scratch gsc;
  float* U32 = nullptr;
  float* E = nullptr;
  if (o.quantizer == SERQ_QUANT_GPTQ) {
    int max_n = 0;
    for (int i = 0; i < n_weights; ++i) max_n = std::max(max_n, N[i]);
    float* Xh = nullptr;
    if (!(s = gsc.get((size_t)n_calib * K, &Xh, "the flattened calibration activations")) &&
        !(s = gsc.get((size_t)K * K, &U32, "the GPTQ factor")) &&
        !(s = gsc.get((size_t)K * max_n, &E, "the GPTQ errors"))) {
      const size_t ne = (size_t)n_calib * K;
      serq::gptq::k_flatten<<<(unsigned)((ne + 255) / 256), 256, 0, st>>>(X_calib, L0->smooth, L0->perm, n_calib,
                                                                        K, Xh);
      s = gptq_factor(Xh, n_calib, K, U32, nullptr, st);
    }
    if (s) {
      cudaStreamSynchronize(st);
      cudaStreamDestroy(st);
      cudaFree(key);
      return cleanup(s);
    }
  }
  // 3-4. per weight: quantize W^ per output channel, compensator R
  for (int i = 0; i < n_weights; ++i) {
    serq_layer* Li = layers[i];
    const WeightView v = view(i);
    const int Ni = N[i];
    const int rows_per_block = 64;
    cudaMemsetAsync(Li->sw, 0, sizeof(float) * Ni, st);
    k_colmax_what<<<dim3((Ni + 255) / 256, (K + rows_per_block - 1) / rows_per_block), 256, 0, st>>>(
        v, L0->smooth, L0->perm, K, rows_per_block, Li->sw);
    if (o.quantizer == SERQ_QUANT_GPTQ) {
      // U and E staged through shared memory when U (K x K fp32) stays in L2;
      // measured: 2-3x faster at K = 4096 (even with E at 180 MB), 3x slower
      // at K = 11008, where U streams from DRAM
      const bool stage = (size_t)K * K * sizeof(float) <= (size_t)64 << 20;
      if (stage)
        serq::gptq::k_gptq_pack_w<true><<<(Ni + 31) / 32, 1024, 0, st>>>(v, L0->smooth, L0->perm, K, rank, Li->sw,
                                                                          U32, E, Li->wq);
      else
        serq::gptq::k_gptq_pack_w<false><<<(Ni + 31) / 32, 1024, 0, st>>>(v, L0->smooth, L0->perm, K, rank, Li->sw,
                                                                           U32, E, Li->wq);
    } else {
      k_quant_pack_w<<<dim3((Ni + 127) / 128, K / 32), 128, 0, st>>>(v, L0->smooth, L0->perm, K, Li->sw, Li->wq);
    }
    if (rank > 0) {
      k_colmax_resid<<<(Ni + 127) / 128, 128, 0, st>>>(v, L0->smooth, L0->perm, rank, Li->sw, Li->sr);
      k_quant_pack_r<<<dim3((Ni + 127) / 128, Li->rpad / 32), 128, 0, st>>>(v, L0->smooth, L0->perm, rank,
                                                                          Li->rpad, Li->sw, Li->sr, Li->rq);
    }
    k_finalize_scales<<<(Ni + 255) / 256, 256, 0, st>>>(Li->sw, Li->sr, Ni, rank > 0);
  }
  e = cudaGetLastError();
  cudaError_t e2 = cudaStreamSynchronize(st);
  cudaStreamDestroy(st);
  cudaFree(key);
  if (e != cudaSuccess) return cleanup(cuda_fail(e, "serq_prepare launch"));
  if (e2 != cudaSuccess) return cleanup(cuda_fail(e2, "serq_prepare"));
  for (int i = 0; i < n_weights; ++i)
    if (!build_weight_maps(layers[i])) return cleanup(fail(SERQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for weights"));
  return ok();
}

// Argument checks of the group calls (host or device pointers alike).
serq_status check_group_args(int n_weights, const float* const* W, const int* N, int K, const float* X_calib,
                             int n_calib, const serq_prepare_opts* opts, const int32_t* const* out_perm,
                             const float* const* out_div, serq_layer** layers) {
  if (!layers) return fail(SERQ_ERR_INVALID_ARG, "null layers");
  if (n_weights < 1 || n_weights > 64) return fail(SERQ_ERR_INVALID_ARG, "n_weights = %d", n_weights);
  for (int i = 0; i < n_weights; ++i) layers[i] = nullptr;
  serq_status s;
  if (!W || !N || !X_calib) return fail(SERQ_ERR_INVALID_ARG, "null W, N or X_calib");
  if (K < 32 || K % 32) return fail(SERQ_ERR_UNSUPPORTED_SHAPE, "K = %d must be a positive multiple of 32", K);
  if (n_calib < 1) return fail(SERQ_ERR_INVALID_ARG, "n_calib = %d", n_calib);
  if ((s = check_opts(opts, K))) return s;
  if (opts->out_perm || opts->out_colscale)
    return fail(SERQ_ERR_INVALID_ARG, "group calls take the folds per weight (out_perm / out_colscale arrays), "
                                      "not in the options");
  for (int i = 0; i < n_weights; ++i) {
    if (!W[i]) return fail(SERQ_ERR_INVALID_ARG, "null W[%d]", i);
    if (N[i] < 32 || N[i] % 32) return fail(SERQ_ERR_UNSUPPORTED_SHAPE, "N[%d] = %d must be a positive multiple of 32", i, N[i]);
    if (out_div && out_div[i] && !(out_perm && out_perm[i]))
      return fail(SERQ_ERR_INVALID_ARG, "out_colscale[%d] given without out_perm[%d]", i, i);
  }
  return check_device();
}

// Device copies of host arrays for the host-pointer prepare calls; freed
// when the owner goes out of scope.
struct Uploads {
  std::vector<void*> bufs;
  ~Uploads() {
    for (void* b : bufs) cudaFree(b);
  }
  template <class T>
  serq_status put(const T* host, size_t count, const T** out) {
    *out = nullptr;
    if (!host) return SERQ_OK;
    void* d = nullptr;
    cudaError_t e = cudaMalloc(&d, count * sizeof(T));
    if (e != cudaSuccess) {
      cudaGetLastError();
      return fail(SERQ_ERR_ALLOC, "cudaMalloc(%zu) for an upload failed: %s", count * sizeof(T), cudaGetErrorString(e));
    }
    bufs.push_back(d);
    e = cudaMemcpy(d, host, count * sizeof(T), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy of a prepare input");
    *out = static_cast<const T*>(d);
    return SERQ_OK;
  }
};

serq_status prepare_shared_host(int n_weights, const float* const* W, const int* N, int K, const float* X_calib,
                                int n_calib, const serq_prepare_opts& o, const int32_t* const* out_perm,
                                const float* const* out_div, serq_layer** layers) {
  Uploads up;
  std::vector<const float*> dW(n_weights, nullptr), dDiv(n_weights, nullptr);
  std::vector<const int32_t*> dPerm(n_weights, nullptr);
  const float* dX = nullptr;
  serq_status s;
  for (int i = 0; i < n_weights; ++i) {
    if ((s = up.put(W[i], (size_t)K * N[i], &dW[i]))) return s;
    if (out_perm && (s = up.put(out_perm[i], (size_t)N[i], &dPerm[i]))) return s;
    if (out_div && (s = up.put(out_div[i], (size_t)N[i], &dDiv[i]))) return s;
  }
  if ((s = up.put(X_calib, (size_t)n_calib * K, &dX))) return s;
  return prepare_impl(n_weights, dW.data(), N, K, dX, n_calib, o, dPerm.data(), dDiv.data(), layers);
}

}  // namespace

extern "C" {

serq_status serq_prepare_group(int n_weights, const float* const* W, const int* N, int K, const float* X_calib,
                               int n_calib, const serq_prepare_opts* opts, const int32_t* const* out_perm,
                               const float* const* out_colscale, serq_layer** layers) {
  serq_status s = check_group_args(n_weights, W, N, K, X_calib, n_calib, opts, out_perm, out_colscale, layers);
  if (s) return s;
  return prepare_impl(n_weights, W, N, K, X_calib, n_calib, *opts, out_perm, out_colscale, layers);
}

serq_status serq_gptq_factor(const float* Xh, int n_calib, int K, double* U) {
  if (!Xh || !U) return fail(SERQ_ERR_INVALID_ARG, "null Xh or U");
  if (K < 32 || K % 32) return fail(SERQ_ERR_UNSUPPORTED_SHAPE, "K = %d must be a positive multiple of 32", K);
  if (n_calib < 1) return fail(SERQ_ERR_INVALID_ARG, "n_calib = %d", n_calib);
  serq_status s = check_device();
  if (s) return s;
  cudaStream_t st;
  cudaError_t e = cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamCreate");
  s = gptq_factor(Xh, n_calib, K, nullptr, U, st);
  cudaStreamSynchronize(st);
  cudaStreamDestroy(st);
  return s ? s : ok();
}

serq_status serq_prepare_shared(int n_weights, const float* const* W, const int* N, int K, const float* X_calib,
                                int n_calib, const serq_prepare_opts* opts, const int32_t* const* out_perm,
                                const float* const* out_colscale, serq_layer** layers) {
  serq_status s = check_group_args(n_weights, W, N, K, X_calib, n_calib, opts, out_perm, out_colscale, layers);
  if (s) return s;
  return prepare_shared_host(n_weights, W, N, K, X_calib, n_calib, *opts, out_perm, out_colscale, layers);
}

serq_status serq_prepare(const float* W, int K, int N, const float* X_calib, int n_calib,
                         const serq_prepare_opts* opts, serq_layer** layer) {
  serq_prepare_opts o;
  serq_prepare_opts_init(&o);
  if (opts) o = *opts;
  const float* Ws[1] = {W};
  const int Ns[1] = {N};
  const int32_t* ps[1] = {o.out_perm};
  const float* ds[1] = {o.out_colscale};
  o.out_perm = nullptr;
  o.out_colscale = nullptr;
  serq_status s = check_group_args(1, Ws, Ns, K, X_calib, n_calib, &o, ps, ds, layer);
  if (s) return s;
  return prepare_shared_host(1, Ws, Ns, K, X_calib, n_calib, o, ps, ds, layer);
}

serq_status serq_layer_get_perm(const serq_layer* L, int32_t* host_out) {
  if (!host_out) return fail(SERQ_ERR_INVALID_ARG, "null output");
  return serq_layer_get_packed(L, nullptr, nullptr, nullptr, nullptr, host_out, nullptr);
}

serq_status serq_layer_get_smooth(const serq_layer* L, float* host_out) {
  if (!host_out) return fail(SERQ_ERR_INVALID_ARG, "null output");
  return serq_layer_get_packed(L, nullptr, nullptr, nullptr, nullptr, nullptr, host_out);
}

void serq_layer_destroy(serq_layer* layer) { free_layer(layer); }

serq_status serq_layer_info(const serq_layer* L, int* K, int* N, int* rank, int* mode) {
  if (!L) return fail(SERQ_ERR_INVALID_ARG, "null layer");
  if (K) *K = L->K;
  if (N) *N = L->N;
  if (rank) *rank = L->rank;
  if (mode) *mode = L->mode;
  return ok();
}

serq_status serq_layer_perm_smooth(const serq_layer* L, const int32_t** perm, const float** smooth) {
  if (!L) return fail(SERQ_ERR_INVALID_ARG, "null layer");
  if (perm) *perm = L->perm;
  if (smooth) *smooth = L->smooth;
  return ok();
}

serq_status serq_layer_get_packed(const serq_layer* L, uint8_t* wq, uint8_t* rq, float* sw, float* sr,
                                  int32_t* perm, float* smooth) {
  serq_status s = check_layer(L);
  if (s) return s;
  cudaError_t e = cudaSuccess;
  auto cp = [&](void* dst, const void* src, size_t n) {
    if (dst && src && n && e == cudaSuccess) e = cudaMemcpy(dst, src, n, cudaMemcpyDeviceToHost);
  };
  cp(wq, L->wq, (size_t)L->N * L->K / 2);
  cp(rq, L->rq, (size_t)L->N * L->rpad / 2);
  cp(sw, L->sw, sizeof(float) * L->N);
  cp(sr, L->sr, sizeof(float) * L->N);
  cp(perm, L->perm, sizeof(int32_t) * L->K);
  cp(smooth, L->smooth, sizeof(float) * L->K);
  if (e != cudaSuccess) return cuda_fail(e, "serq_layer_get_packed");
  return ok();
}

serq_status serq_quantize_act(const void* X, serq_dtype dtype, int M, int K, int ldx, serq_mode mode, void* Xq,
                              float* sx, void* stream) {
  serq_status s;
  if (dtype != SERQ_F32 && dtype != SERQ_BF16) return fail(SERQ_ERR_INVALID_ARG, "bad dtype");
  if ((s = check_rows(X, M, K, ldx, dtype == SERQ_F32 ? 4 : 2, "X"))) return s;
  if (K > (dtype == SERQ_F32 ? 16384 : 32768))
    return fail(SERQ_ERR_UNSUPPORTED_SHAPE, "quantize takes K <= %d for this dtype (got %d)",
                dtype == SERQ_F32 ? 16384 : 32768, K);
  if (!Xq || !sx) return fail(SERQ_ERR_INVALID_ARG, "null Xq or sx");
  if (!aligned16(Xq)) return fail(SERQ_ERR_INVALID_ARG, "Xq must be 16-byte aligned");
  if (mode != SERQ_W4A4 && mode != SERQ_W4A8) return fail(SERQ_ERR_INVALID_ARG, "bad mode");
  if ((s = check_device())) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* q = static_cast<uint8_t*>(Xq);
  cudaError_t e;
  using namespace serq::quant;
  if (dtype == SERQ_BF16) {
    LoadBF16 ld{static_cast<const __nv_bfloat16*>(X), ldx};
    e = (mode == SERQ_W4A4) ? launch_quant_rows<7>(ld, M, K, q, sx, st) : launch_quant_rows<127>(ld, M, K, q, sx, st);
  } else {
    LoadF32 ld{static_cast<const float*>(X), ldx};
    e = (mode == SERQ_W4A4) ? launch_quant_rows<7>(ld, M, K, q, sx, st) : launch_quant_rows<127>(ld, M, K, q, sx, st);
  }
  if (e != cudaSuccess) return cuda_fail(e, "serq_quantize_act launch");
  return ok();
}

serq_status serq_silu_mul_quantize(const void* G, const void* U, int M, int F, int ld, serq_mode mode, void* Xq,
                                   float* sx, void* stream) {
  serq_status s;
  if ((s = check_rows(G, M, F, ld, 2, "G"))) return s;
  if ((s = check_rows(U, M, F, ld, 2, "U"))) return s;
  if (F > 16384) return fail(SERQ_ERR_UNSUPPORTED_SHAPE, "silu_mul_quantize takes F <= 16384 (got %d)", F);
  if (!Xq || !sx) return fail(SERQ_ERR_INVALID_ARG, "null Xq or sx");
  if (!aligned16(Xq)) return fail(SERQ_ERR_INVALID_ARG, "Xq must be 16-byte aligned");
  if (mode != SERQ_W4A4 && mode != SERQ_W4A8) return fail(SERQ_ERR_INVALID_ARG, "bad mode");
  if ((s = check_device())) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  serq::quant::LoadSiluMul ldr{static_cast<const __nv_bfloat16*>(G), static_cast<const __nv_bfloat16*>(U), ld};
  uint8_t* q = static_cast<uint8_t*>(Xq);
  cudaError_t e = (mode == SERQ_W4A4) ? serq::quant::launch_quant_rows<7>(ldr, M, F, q, sx, st)
                                      : serq::quant::launch_quant_rows<127>(ldr, M, F, q, sx, st);
  if (e != cudaSuccess) return cuda_fail(e, "serq_silu_mul_quantize launch");
  return ok();
}

serq_status serq_flatten_permute(const serq_layer* L, const void* X, serq_dtype in_dtype, int M, int ldx, void* Xh,
                                 serq_dtype out_dtype, int ldxh, void* stream) {
  serq_status s;
  if (!L) return fail(SERQ_ERR_INVALID_ARG, "null layer");
  if (!X || !Xh) return fail(SERQ_ERR_INVALID_ARG, "null X or Xh");
  if (M < 1 || M > 65535) return fail(SERQ_ERR_INVALID_ARG, "M = %d out of range (1..65535)", M);
  if (ldx < L->K || ldxh < L->K) return fail(SERQ_ERR_INVALID_ARG, "leading dimension < K");
  const bool ib = (in_dtype == SERQ_BF16), ob = (out_dtype == SERQ_BF16);
  if ((in_dtype != SERQ_F32 && !ib) || (out_dtype != SERQ_F32 && !ob)) return fail(SERQ_ERR_INVALID_ARG, "bad dtype");
  if ((s = check_device())) return s;
  if ((s = check_layer(L))) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  dim3 grid((L->K + 255) / 256, M);
  using namespace serq::quant;
  if (ib && ob) k_flatten_permute<true, true><<<grid, 256, 0, st>>>(X, ldx, L->perm, L->smooth, M, L->K, Xh, ldxh);
  else if (ib) k_flatten_permute<true, false><<<grid, 256, 0, st>>>(X, ldx, L->perm, L->smooth, M, L->K, Xh, ldxh);
  else if (ob) k_flatten_permute<false, true><<<grid, 256, 0, st>>>(X, ldx, L->perm, L->smooth, M, L->K, Xh, ldxh);
  else k_flatten_permute<false, false><<<grid, 256, 0, st>>>(X, ldx, L->perm, L->smooth, M, L->K, Xh, ldxh);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "serq_flatten_permute launch");
  return ok();
}

serq_status serq_linear(const serq_layer* layer, const void* Xq, const float* sx, int M, void* Y, int ldy,
                        void* stream) {
  return linear_impl(layer, Xq, sx, M, Y, ldy, nullptr, nullptr, SERQ_ALGO_AUTO, stream);
}

serq_status serq_linear_ex(const serq_layer* layer, const void* Xq, const float* sx, int M, void* Y, int ldy,
                           serq_algo algo, void* stream) {
  return linear_impl(layer, Xq, sx, M, Y, ldy, nullptr, nullptr, algo, stream);
}

serq_status serq_linear_accum(const serq_layer* layer, const void* Xq, int M, int32_t* acc0, int32_t* acc1,
                              serq_algo algo, void* stream) {
  if (!acc0 || !acc1) return fail(SERQ_ERR_INVALID_ARG, "null acc0 or acc1");
  return linear_impl(layer, Xq, nullptr, M, nullptr, 0, acc0, acc1, algo, stream);
}

serq_status serq_linear_group(int n, const serq_layer* const* layers, const void* Xq, const float* sx, int M,
                              void* const* Y, const int* ldy, int32_t* const* acc0, int32_t* const* acc1,
                              serq_algo algo, void* stream) {
  return group_impl(n, layers, Xq, sx, M, Y, ldy, acc0, acc1, algo, stream);
}

serq_status serq_linear_group_act(int n, const serq_layer* const* layers, const void* X, serq_dtype dtype, int ldx,
                                  int M, void* Xq, float* sx, void* const* Y, const int* ldy, int32_t* const* acc0,
                                  int32_t* const* acc1, serq_algo algo, void* stream) {
  serq_status s;
  if (n < 1 || n > serq::tc::kMaxGroup || !layers || !layers[0])
    return fail(SERQ_ERR_INVALID_ARG, "null layer list or a group of %d layers", n);
  if (dtype != SERQ_F32 && dtype != SERQ_BF16) return fail(SERQ_ERR_INVALID_ARG, "bad dtype");
  const int K = layers[0]->K;
  if ((s = check_rows(X, M, K, ldx, dtype == SERQ_F32 ? 4 : 2, "X"))) return s;
  if (!Xq || !sx) return fail(SERQ_ERR_INVALID_ARG, "null Xq or sx (scratch)");
  serq_algo a = algo;
  if (a == SERQ_ALGO_AUTO) a = (M <= serq_decode_max_m()) ? SERQ_ALGO_DECODE : SERQ_ALGO_PREFILL;
  const bool decode = a == SERQ_ALGO_DECODE || a == SERQ_ALGO_DECODE_STREAM || a == SERQ_ALGO_DECODE_ITEMS;
  // One launch pays off for few tokens: every CTA reads all M bf16 rows
  // (M x K x 2 bytes from L2) before its loop, which at M = 16 already costs
  // more than the quantize launch it saves (measured on the 7B decode step:
  // 1-3% faster for M <= 8, 2% slower at 16, 11% at 32).
  if (dtype == SERQ_BF16 && K <= 4096 && M <= 8 && decode)
    return group_impl(n, layers, Xq, sx, M, Y, ldy, acc0, acc1, algo, stream,
                      static_cast<const __nv_bfloat16*>(X), ldx);
  if ((s = serq_quantize_act(X, dtype, M, K, ldx, static_cast<serq_mode>(layers[0]->mode), Xq, sx, stream))) return s;
  return group_impl(n, layers, Xq, sx, M, Y, ldy, acc0, acc1, algo, stream);
}

serq_status serq_test_decode_timeout(const serq_layer* layer, const void* Xq, const float* sx, int M, void* Y,
                                     int ldy, int wait_us, void* stream) {
  if (wait_us < 1 || wait_us > 1000000) return fail(SERQ_ERR_INVALID_ARG, "wait_us = %d not in [1, 1e6]", wait_us);
  serq_algo algo = SERQ_ALGO_DECODE;
  serq_status s;
  if ((s = check_linear(layer, Xq, sx, M, Y, ldy, nullptr, nullptr, &algo))) return s;
  if (M > 32) return fail(SERQ_ERR_UNSUPPORTED_SHAPE, "the streaming decode kernel takes M <= 32");
  LinearGroup G = {};
  G.n = 1;
  G.L[0] = layer;
  G.Y[0] = static_cast<__nv_bfloat16*>(Y);
  G.ldy[0] = ldy;
  cudaError_t e = launch_decode_group(G, Xq, sx, M, layer->mode == SERQ_W4A8, false, 2,
                                      static_cast<cudaStream_t>(stream), (unsigned long long)wait_us * 1000ull);
  if (e != cudaSuccess) return cuda_fail(e, "serq_test_decode_timeout launch");
  return ok();
}

serq_status serq_linear_decode_static(const serq_layer* layer, const void* Xq, const float* sx, int M, void* Y,
                                      int ldy, int32_t* acc0, int32_t* acc1, void* stream) {
  if (!layer) return fail(SERQ_ERR_INVALID_ARG, "null layer");
  if ((acc0 == nullptr) != (acc1 == nullptr)) return fail(SERQ_ERR_INVALID_ARG, "acc0 and acc1 go together");
  if (M < 1 || M > serq::dtc::kMaxM)
    return fail(SERQ_ERR_UNSUPPORTED_SHAPE, "serq_linear_decode_static takes 1 <= M <= %d (got %d)", serq::dtc::kMaxM, M);
  if (layer->N > kStaticMaxN)
    return fail(SERQ_ERR_UNSUPPORTED_SHAPE, "serq_linear_decode_static takes N <= %d (got %d)", kStaticMaxN, layer->N);
  serq_status s = check_device();
  if (s) return s;
  int32_t* scratch = nullptr;
  if ((s = static_scratch(static_cast<cudaStream_t>(stream), &scratch))) return s;
  return linear_impl(layer, Xq, sx, M, Y, ldy, acc0, acc1, SERQ_ALGO_DECODE_TC, stream, scratch,
                     scratch + kStaticCntOffset);
}

}  // extern "C"

// ------------------------------------------------------------------------
// The two-factor comparator (L2QER): X_q W_q + Q(X_q L1_q) L2_q on the
// kernels above.  L1 runs as a layer of r output channels (rank 0), its bf16
// output is quantized per token by the activation quantizer, and the final
// GEMM reads those codes in its residual steps with L2 in place of R.
// ------------------------------------------------------------------------
struct serq_l2qer {
  int K, N, r;
  serq_layer* f1;    // L1: r x K/2 packed codes, per-channel scales (owned)
  serq_layer view;   // the base layer with R / sR replaced by L2's codes / scales
  void* block;       // L2's codes (N x r/2) and scales (N)
};

namespace {

// scale = amax / 7 in place (the symmetric INT4 scale, one fp32 division)
__global__ void k_amax_to_scale(float* a, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) a[i] = __fdiv_rn(a[i], 7.f);
}

// Per-column INT4 quantization and packing of a plain K x N fp32 matrix
// (no smoothing, identity order) into codes (N x K/2) and scales (N).
serq_status quantize_columns(const float* W, int K, int N, uint8_t* codes, float* scales, const float* ones,
                             const int32_t* ident, cudaStream_t st) {
  using namespace serq::prep;
  const WeightView v{W, N, nullptr, nullptr};
  const int rows_per_block = 64;
  cudaMemsetAsync(scales, 0, sizeof(float) * N, st);
  k_colmax_what<<<dim3((N + 255) / 256, (K + rows_per_block - 1) / rows_per_block), 256, 0, st>>>(
      v, ones, ident, K, rows_per_block, scales);
  k_quant_pack_w<<<dim3((N + 127) / 128, K / 32), 128, 0, st>>>(v, ones, ident, K, scales, codes);
  k_amax_to_scale<<<(N + 255) / 256, 256, 0, st>>>(scales, N);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SERQ_OK : cuda_fail(e, "quantizing a factor");
}

__global__ void k_fill_ones_iota(float* ones, int32_t* ident, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    ones[i] = 1.f;
    ident[i] = i;
  }
}

void free_l2qer(serq_l2qer* q) {
  if (!q) return;
  free_layer(q->f1);
  if (q->block) cudaFree(q->block);
  delete q;
}

template <bool ACC>
cudaError_t dispatch_two(const LinearGroup& G, const void* Xq, const float* sx, int M, serq_algo algo,
                         const void* Zq, const float* sz, cudaStream_t st) {
  if (algo == SERQ_ALGO_PREFILL_N128) return launch_tc<128, false, ACC, 1, !ACC>(G, Xq, sx, M, st, Zq, sz);
  if (algo == SERQ_ALGO_PREFILL_PAIR_N256) return launch_tc<256, false, ACC, 2, !ACC>(G, Xq, sx, M, st, Zq, sz);
  const long ctas_pair = (long)((G.L[0]->N + 255) / 256) * 2 * ((M + 255) / 256);
  if (ctas_pair * 10 >= (long)sm_count() * 9) return launch_tc<256, false, ACC, 2, !ACC>(G, Xq, sx, M, st, Zq, sz);
  return launch_tc<128, false, ACC, 1, !ACC>(G, Xq, sx, M, st, Zq, sz);
}

// Final GEMM of the comparator (main product + L2 on the intermediate codes).
serq_status l2qer_final(const serq_l2qer* q, const void* Xq, const float* sx, int M, const void* Zq, const float* sz,
                        void* Y, int ldy, int32_t* acc0, int32_t* acc1, serq_algo algo, cudaStream_t st) {
  const bool accum = acc0 != nullptr;
  if (!aligned16(Zq)) return fail(SERQ_ERR_INVALID_ARG, "Zq must be 16-byte aligned");
  if (!accum && !aligned16(sz)) return fail(SERQ_ERR_INVALID_ARG, "null or misaligned sz");
  cudaError_t e;
  if (algo == SERQ_ALGO_DECODE) {
    serq::gs::Args g = {};
    g.Xq = static_cast<const uint8_t*>(Xq);
    g.sx = sx;
    g.Xr = static_cast<const uint8_t*>(Zq);
    g.sxr = accum ? nullptr : sz;
    g.M = M;
    g.K = q->K;
    g.rpad = q->view.rpad;
    g.nlayers = 1;
    const serq_layer* L = &q->view;
    serq::gs::Maps mp;
    for (int l = 0; l < serq::gs::kMaxGroup; ++l) {
      g.lo[l] = serq::gs::Layer{L->wq, L->rq, L->sw, L->sr, static_cast<__nv_bfloat16*>(Y), ldy, acc0, acc1, L->N,
                                l == 0 ? 0 : 1 << 30};
      mp.w[l] = L->tmW4;
      mp.r[l] = L->tmR4;
      mp.w16[l] = L->tmW16;
      mp.r16[l] = L->tmR16;
    }
    g.C = L->N;
    if (!serq::gs::fits<false>(g, sm_count(), max_smem()))
      return fail(SERQ_ERR_UNSUPPORTED_SHAPE, "the comparator's decode GEMM does not fit shared memory at M = %d", M);
    e = accum ? serq::gs::launch<false, true>(g, mp, sm_count(), max_smem(), st)
              : serq::gs::launch<false, false>(g, mp, sm_count(), max_smem(), st);
  } else {
    LinearGroup G = {};
    G.n = 1;
    G.L[0] = &q->view;
    G.Y[0] = static_cast<__nv_bfloat16*>(Y);
    G.ldy[0] = ldy;
    G.acc0[0] = acc0;
    G.acc1[0] = acc1;
    e = accum ? dispatch_two<true>(G, Xq, sx, M, algo, Zq, nullptr, st) : dispatch_two<false>(G, Xq, sx, M, algo, Zq, sz, st);
  }
  if (e != cudaSuccess) return cuda_fail(e, "comparator GEMM launch");
  return ok();
}

serq_status check_two_algo(const serq_l2qer* q, int M, serq_algo* algo) {
  if (!q) return fail(SERQ_ERR_INVALID_ARG, "null comparator");
  if (M < 1 || M > 65535 * 128) return fail(SERQ_ERR_INVALID_ARG, "M = %d out of range", M);
  serq_algo a = *algo;
  if (a == SERQ_ALGO_AUTO) a = (M <= serq_decode_max_m()) ? SERQ_ALGO_DECODE : SERQ_ALGO_PREFILL;
  if (a != SERQ_ALGO_DECODE && a != SERQ_ALGO_PREFILL && a != SERQ_ALGO_PREFILL_N128 &&
      a != SERQ_ALGO_PREFILL_PAIR_N256)
    return fail(SERQ_ERR_INVALID_ARG, "the comparator runs SERQ_ALGO_AUTO, DECODE, PREFILL, PREFILL_N128 or "
                                      "PREFILL_PAIR_N256 (got %d)", (int)*algo);
  if (a == SERQ_ALGO_DECODE && M > 32) return fail(SERQ_ERR_UNSUPPORTED_SHAPE, "decode takes M <= 32 (got %d)", M);
  serq_status s;
  if ((s = check_device())) return s;
  if ((s = check_layer(q->f1))) return s;
  *algo = a;
  return SERQ_OK;
}

}  // namespace

extern "C" {

serq_status serq_l2qer_prepare(const serq_layer* layer, const float* L1, const float* L2, int r, serq_l2qer** out) {
  if (!out) return fail(SERQ_ERR_INVALID_ARG, "null out");
  *out = nullptr;
  if (!layer || !L1 || !L2) return fail(SERQ_ERR_INVALID_ARG, "null layer, L1 or L2");
  if (layer->mode != SERQ_W4A4) return fail(SERQ_ERR_INVALID_ARG, "the comparator takes W4A4 layers");
  if (r < 32 || r % 32 || r > layer->K)
    return fail(SERQ_ERR_UNSUPPORTED_SHAPE, "rank %d must be a positive multiple of 32 and <= K = %d", r, layer->K);
  serq_status s;
  if ((s = check_device())) return s;
  if ((s = check_layer(layer))) return s;
  serq_l2qer* q = new (std::nothrow) serq_l2qer();
  if (!q) return fail(SERQ_ERR_ALLOC, "host allocation failed");
  q->K = layer->K;
  q->N = layer->N;
  q->r = r;
  q->f1 = nullptr;
  q->block = nullptr;
  if ((s = alloc_layer(layer->K, r, 0, SERQ_W4A4, &q->f1))) {
    delete q;
    return s;
  }
  const size_t s_codes = up256((size_t)layer->N * r / 2), s_sc = up256((size_t)layer->N * 4);
  const int tmpn = layer->K > r ? layer->K : r;
  const size_t s_tmp = up256((size_t)tmpn * 4);
  cudaError_t e = cudaMalloc(&q->block, s_codes + s_sc + 2 * s_tmp);
  if (e != cudaSuccess) {
    cudaGetLastError();
    free_l2qer(q);
    return fail(SERQ_ERR_ALLOC, "cudaMalloc for the comparator failed: %s", cudaGetErrorString(e));
  }
  uint8_t* b = static_cast<uint8_t*>(q->block);
  uint8_t* l2q = b;
  float* s_l2 = reinterpret_cast<float*>(b + s_codes);
  float* ones = reinterpret_cast<float*>(b + s_codes + s_sc);
  int32_t* ident = reinterpret_cast<int32_t*>(b + s_codes + s_sc + s_tmp);
  cudaStream_t st;
  e = cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking);
  if (e != cudaSuccess) {
    free_l2qer(q);
    return cuda_fail(e, "cudaStreamCreate");
  }
  k_fill_ones_iota<<<(tmpn + 255) / 256, 256, 0, st>>>(ones, ident, tmpn);
  s = quantize_columns(L1, layer->K, r, q->f1->wq, q->f1->sw, ones, ident, st);
  if (!s) {
    cudaMemsetAsync(q->f1->sr, 0, sizeof(float) * r, st);
    s = quantize_columns(L2, r, layer->N, l2q, s_l2, ones, ident, st);
  }
  e = cudaStreamSynchronize(st);
  cudaStreamDestroy(st);
  if (!s && e != cudaSuccess) s = cuda_fail(e, "serq_l2qer_prepare");
  if (s) {
    free_l2qer(q);
    return s;
  }
  q->view = *layer;
  q->view.rank = r;
  q->view.rpad = r;
  q->view.rq = l2q;
  q->view.sr = s_l2;
  if (!build_weight_maps(q->f1) || !build_weight_maps(&q->view)) {
    free_l2qer(q);
    return fail(SERQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the comparator");
  }
  *out = q;
  return ok();
}

void serq_l2qer_destroy(serq_l2qer* q) { free_l2qer(q); }

serq_status serq_l2qer_get_packed(const serq_l2qer* q, uint8_t* l1q, float* s_l1, uint8_t* l2q, float* s_l2) {
  if (!q) return fail(SERQ_ERR_INVALID_ARG, "null comparator");
  serq_status s = check_layer(q->f1);
  if (s) return s;
  cudaError_t e = cudaSuccess;
  auto cp = [&](void* dst, const void* src, size_t n) {
    if (dst && e == cudaSuccess) e = cudaMemcpy(dst, src, n, cudaMemcpyDeviceToHost);
  };
  cp(l1q, q->f1->wq, (size_t)q->r * q->K / 2);
  cp(s_l1, q->f1->sw, sizeof(float) * q->r);
  cp(l2q, q->view.rq, (size_t)q->N * q->r / 2);
  cp(s_l2, q->view.sr, sizeof(float) * q->N);
  if (e != cudaSuccess) return cuda_fail(e, "serq_l2qer_get_packed");
  return ok();
}

serq_status serq_l2qer_linear(const serq_l2qer* q, const void* Xq, const float* sx, int M, void* Z, void* Zq,
                              float* sz, void* Y, int ldy, serq_algo algo, void* stream) {
  serq_status s;
  if ((s = check_two_algo(q, M, &algo))) return s;
  if (!Xq || !sx || !Z || !Zq || !sz || !Y) return fail(SERQ_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(Z) || !aligned16(Zq) || !aligned16(Y) || (ldy % 8) || ldy < q->N)
    return fail(SERQ_ERR_INVALID_ARG, "Z, Zq, Y must be 16-byte aligned, ldy >= N and a multiple of 8");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // 1. Z = X_q L1_q (bf16, M x r)
  const serq_algo a1 = (algo == SERQ_ALGO_DECODE) ? SERQ_ALGO_DECODE : SERQ_ALGO_PREFILL;
  if ((s = linear_impl(q->f1, Xq, sx, M, Z, q->r, nullptr, nullptr, a1, stream))) return s;
  // 2. on-the-fly quantization of the intermediate
  if ((s = serq_quantize_act(Z, SERQ_BF16, M, q->r, q->r, SERQ_W4A4, Zq, sz, stream))) return s;
  // 3. X_q W_q + Z_q L2_q
  return l2qer_final(q, Xq, sx, M, Zq, sz, Y, ldy, nullptr, nullptr, algo, st);
}

serq_status serq_l2qer_accum(const serq_l2qer* q, const void* Xq, const void* Zq, int M, int32_t* acc0,
                             int32_t* acc1, serq_algo algo, void* stream) {
  serq_status s;
  if ((s = check_two_algo(q, M, &algo))) return s;
  if (!Xq || !Zq || !acc0 || !acc1) return fail(SERQ_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(Xq) || !aligned16(acc0) || !aligned16(acc1))
    return fail(SERQ_ERR_INVALID_ARG, "Xq, acc0, acc1 must be 16-byte aligned");
  return l2qer_final(q, Xq, nullptr, M, Zq, nullptr, nullptr, 0, acc0, acc1, algo, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

// ------------------------------------------------------------------------
// SERQ with MXFP4 codes: the base layer's smoothing scales and saliency
// order, W^ and R in OCP MX blocks of 32 along K, the block-scaled
// tcgen05 GEMM (mxfp4.cuh).
// ------------------------------------------------------------------------
struct serq_mx_layer {
  int K, N, r, rpad, device;
  void* block;
  uint8_t* wq;  // N x K/2 codes
  uint8_t* we;  // tiled scales of W^ (N x K/32)
  uint8_t* rq;  // N x rpad/2 codes (zero past r)
  uint8_t* re;  // tiled scales of R (N x rpad/32)
  CUtensorMap tmW, tmR;
};

namespace {

void free_mx(serq_mx_layer* q) {
  if (!q) return;
  if (q->block) cudaFree(q->block);
  delete q;
}

serq_status check_mx(const serq_mx_layer* q) {
  if (!q) return fail(SERQ_ERR_INVALID_ARG, "null MXFP4 layer");
  int dev = -1;
  cudaGetDevice(&dev);
  if (dev != q->device)
    return fail(SERQ_ERR_INVALID_ARG, "layer was prepared on device %d, current device is %d", q->device, dev);
  return check_device();
}

// Tiled scales -> plain rows x n_blocks bytes on the host.
void untile_scales(const uint8_t* tiled, int rows, int n_blocks, uint8_t* out) {
  for (int i = 0; i < rows; ++i)
    for (int b = 0; b < n_blocks; ++b) out[(size_t)i * n_blocks + b] = tiled[serq::mx::scale_offset(i, b, n_blocks)];
}

}  // namespace

extern "C" {

serq_status serq_mx_prepare(const serq_layer* base, const float* W, serq_mx_layer** out) {
  if (!out) return fail(SERQ_ERR_INVALID_ARG, "null out");
  *out = nullptr;
  if (!base || !W) return fail(SERQ_ERR_INVALID_ARG, "null base layer or W");
  serq_status s;
  if ((s = check_device())) return s;
  if ((s = check_layer(base))) return s;
  const int K = base->K, N = base->N, r = base->rank;
  if (K % serq::mx::kTileK || N % 128)
    return fail(SERQ_ERR_UNSUPPORTED_SHAPE, "MXFP4 needs K a multiple of 256 and N of 128 (K = %d, N = %d)", K, N);
  if (r % serq::mx::kBlock)
    return fail(SERQ_ERR_UNSUPPORTED_SHAPE, "MXFP4 needs the rank to be a multiple of 32 (r = %d)", r);
  serq_mx_layer* q = new (std::nothrow) serq_mx_layer();
  if (!q) return fail(SERQ_ERR_ALLOC, "host allocation failed");
  std::memset(q, 0, sizeof(*q));
  q->K = K;
  q->N = N;
  q->r = r;
  q->rpad = (r + serq::mx::kTileK - 1) / serq::mx::kTileK * serq::mx::kTileK;
  q->device = base->device;
  const size_t s_wq = up256((size_t)N * K / 2), s_we = up256((size_t)N * K / 32);
  const size_t s_rq = up256((size_t)N * q->rpad / 2), s_re = up256((size_t)N * q->rpad / 32);
  cudaError_t e = cudaMalloc(&q->block, s_wq + s_we + s_rq + s_re + 256);
  if (e != cudaSuccess) {
    cudaGetLastError();
    free_mx(q);
    return fail(SERQ_ERR_ALLOC, "cudaMalloc for the MXFP4 layer failed: %s", cudaGetErrorString(e));
  }
  uint8_t* b = static_cast<uint8_t*>(q->block);
  q->wq = b;
  q->we = b + s_wq;
  q->rq = b + s_wq + s_we;
  q->re = b + s_wq + s_we + s_rq;
  cudaStream_t st;
  e = cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking);
  if (e != cudaSuccess) {
    free_mx(q);
    return cuda_fail(e, "cudaStreamCreate");
  }
  const serq::prep::WeightView v{W, N, nullptr, nullptr};
  serq::mx::k_quant_w<<<dim3(N / 128, K / serq::mx::kBlock), 128, 0, st>>>(v, base->smooth, base->perm, K, r, q->rpad,
                                                                          q->wq, q->we, q->rq, q->re);
  e = cudaGetLastError();
  const cudaError_t e2 = cudaStreamSynchronize(st);
  cudaStreamDestroy(st);
  if (e == cudaSuccess) e = e2;
  if (e != cudaSuccess) {
    free_mx(q);
    return cuda_fail(e, "serq_mx_prepare");
  }
  const bool okw = make_map(&q->tmW, q->wq, (uint64_t)K / 2, (uint64_t)N, (uint64_t)K / 2, 128, 128,
                            CU_TENSOR_MAP_SWIZZLE_128B);
  const bool okr = q->rpad == 0 ? true
                                : make_map(&q->tmR, q->rq, (uint64_t)q->rpad / 2, (uint64_t)N, (uint64_t)q->rpad / 2,
                                           128, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!okw || !okr) {
    free_mx(q);
    return fail(SERQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the MXFP4 layer");
  }
  if (q->rpad == 0) q->tmR = q->tmW;  // never read when r = 0
  *out = q;
  return ok();
}

void serq_mx_destroy(serq_mx_layer* q) { free_mx(q); }

serq_status serq_mx_get_packed(const serq_mx_layer* q, uint8_t* wq, uint8_t* we, uint8_t* rq, uint8_t* re) {
  serq_status s;
  if ((s = check_mx(q))) return s;
  const int nb = q->K / 32, nbr = q->rpad / 32;
  cudaError_t e = cudaSuccess;
  if (wq) e = cudaMemcpy(wq, q->wq, (size_t)q->N * q->K / 2, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && we) {
    std::vector<uint8_t> t((size_t)q->N * nb);
    e = cudaMemcpy(t.data(), q->we, t.size(), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) untile_scales(t.data(), q->N, nb, we);
  }
  if (e == cudaSuccess && q->r > 0 && (rq || re)) {
    std::vector<uint8_t> c((size_t)q->N * q->rpad / 2), t((size_t)q->N * nbr);
    e = cudaMemcpy(c.data(), q->rq, c.size(), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemcpy(t.data(), q->re, t.size(), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) {
      std::vector<uint8_t> plain((size_t)q->N * nbr);
      untile_scales(t.data(), q->N, nbr, plain.data());
      for (int n = 0; n < q->N; ++n) {
        if (rq) std::memcpy(rq + (size_t)n * q->r / 2, c.data() + (size_t)n * q->rpad / 2, (size_t)q->r / 2);
        if (re) std::memcpy(re + (size_t)n * q->r / 32, plain.data() + (size_t)n * nbr, (size_t)q->r / 32);
      }
    }
  }
  if (e != cudaSuccess) return cuda_fail(e, "serq_mx_get_packed");
  return ok();
}

size_t serq_mx_act_scale_bytes(int M, int K) {
  if (M < 1 || K < serq::mx::kTileK || K % serq::mx::kTileK) return 0;
  return (size_t)((M + 127) / 128 * 128) * (size_t)(K / 32);
}

serq_status serq_mx_quantize_act(const void* Xh, serq_dtype dtype, int M, int K, int ldxh, void* Xq, void* xe,
                                 void* stream) {
  if (!Xh || !Xq || !xe) return fail(SERQ_ERR_INVALID_ARG, "null pointer argument");
  if (dtype != SERQ_F32 && dtype != SERQ_BF16) return fail(SERQ_ERR_INVALID_ARG, "bad dtype %d", (int)dtype);
  if (M < 1 || M > 65535 * 128) return fail(SERQ_ERR_INVALID_ARG, "M = %d out of range", M);
  if (K < serq::mx::kTileK || K % serq::mx::kTileK)
    return fail(SERQ_ERR_UNSUPPORTED_SHAPE, "MXFP4 needs K a positive multiple of 256 (got %d)", K);
  const int esz = dtype == SERQ_F32 ? 4 : 2;
  if (ldxh < K || ((size_t)ldxh * esz) % 16 || !aligned16(Xh) || !aligned16(Xq) || !aligned16(xe))
    return fail(SERQ_ERR_INVALID_ARG, "Xh, Xq, xe must be 16-byte aligned and ldxh >= K with 16-byte rows");
  serq_status s;
  if ((s = check_device())) return s;
  const int Mpad = (M + 127) / 128 * 128;
  const long n = (long)Mpad * (K / 32);
  const int threads = 256;
  const unsigned blocks = (unsigned)((n + threads - 1) / threads);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == SERQ_BF16)
    serq::mx::k_quant_act<uint16_t><<<blocks, threads, 0, st>>>(static_cast<const uint16_t*>(Xh), M, K, ldxh, Mpad,
                                                                static_cast<uint8_t*>(Xq), static_cast<uint8_t*>(xe));
  else
    serq::mx::k_quant_act<float><<<blocks, threads, 0, st>>>(static_cast<const float*>(Xh), M, K, ldxh, Mpad,
                                                             static_cast<uint8_t*>(Xq), static_cast<uint8_t*>(xe));
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "serq_mx_quantize_act launch");
  return ok();
}

serq_status serq_mx_linear(const serq_mx_layer* q, const void* Xq, const void* xe, int M, void* Y, int ldy,
                           void* stream) {
  serq_status s;
  if ((s = check_mx(q))) return s;
  if (!Xq || !xe || !Y) return fail(SERQ_ERR_INVALID_ARG, "null pointer argument");
  if (M < 1 || M > 65535 * 128) return fail(SERQ_ERR_INVALID_ARG, "M = %d out of range", M);
  if (!aligned16(Xq) || !aligned16(xe) || !aligned16(Y) || ldy < q->N || ldy % 8)
    return fail(SERQ_ERR_INVALID_ARG, "Xq, xe, Y must be 16-byte aligned, ldy >= N and a multiple of 8");
  CUtensorMap tmA;
  if (!make_map(&tmA, Xq, (uint64_t)q->K / 2, (uint64_t)M, (uint64_t)q->K / 2, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B))
    return fail(SERQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for Xq");
  serq::mx::Args a;
  a.xe = static_cast<const uint8_t*>(xe);
  a.we = q->we;
  a.re = q->re;
  a.Y = static_cast<__nv_bfloat16*>(Y);
  a.ldy = ldy;
  a.M = M;
  a.N = q->N;
  a.K = q->K;
  a.rpad = q->rpad;
  cudaError_t e = serq::smem_limit(reinterpret_cast<const void*>(serq::mx::k_gemm), serq::mx::kSmemBytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (MXFP4 GEMM)");
  const dim3 grid(q->N / 128, (M + 127) / 128);
  serq::mx::k_gemm<<<grid, serq::mx::kThreads, serq::mx::kSmemBytes, static_cast<cudaStream_t>(stream)>>>(
      tmA, q->tmW, q->tmR, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "serq_mx_linear launch");
  return ok();
}

}  // extern "C"
