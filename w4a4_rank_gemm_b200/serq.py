"""Thin Python binding of libserq (ctypes).  Argument marshalling only: every
step runs in the library's CUDA kernels.  torch is used for device memory and
streams.  Importing this module fails loudly if libserq.so is missing."""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libserq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libserq.so not found at {LIB_PATH}; build it with "
        "`python -m w4a4_rank_gemm_b200.build` (there is no fallback path)")

lib = ctypes.CDLL(LIB_PATH)

# enums
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED_SHAPE, ERR_UNSUPPORTED_DEVICE, ERR_ALLOC, ERR_CUDA, ERR_TIMEOUT, ERR_NUMERIC = range(8)
W4A4, W4A8 = 0, 1
F32, BF16 = 0, 1
(ALGO_AUTO, ALGO_PREFILL, ALGO_DECODE, ALGO_PREFILL_N128, ALGO_PREFILL_N256, ALGO_PREFILL_PAIR_N256,
 ALGO_PREFILL_PAIR_TMEM_A, ALGO_DECODE_TC, ALGO_DECODE_ITEMS, ALGO_DECODE_STREAM) = 0, 1, 2, 3, 4, 5, 6, 7, 8, 9

_vp = ctypes.c_void_p
_i = ctypes.c_int
SALIENCY_SCALE, SALIENCY_ROW_ABSMAX = 0, 1
QUANT_RTN, QUANT_GPTQ = 0, 1


class PrepareOpts(ctypes.Structure):
    """serq_prepare_opts."""
    _fields_ = [("alpha", ctypes.c_float), ("rank", _i), ("mode", _i), ("saliency", _i),
                ("out_perm", _vp), ("out_colscale", _vp), ("quantizer", _i)]


EXPORTS = {
    "serq_prepare_opts_init": (None, [ctypes.POINTER(PrepareOpts)]),
    "serq_prepare_group": (_i, [_i, ctypes.POINTER(_vp), ctypes.POINTER(_i), _i, _vp, _i, ctypes.POINTER(PrepareOpts),
                                ctypes.POINTER(_vp), ctypes.POINTER(_vp), ctypes.POINTER(_vp)]),
    "serq_prepare_shared": (_i, [_i, ctypes.POINTER(_vp), ctypes.POINTER(_i), _i, _vp, _i,
                                 ctypes.POINTER(PrepareOpts), ctypes.POINTER(_vp), ctypes.POINTER(_vp),
                                 ctypes.POINTER(_vp)]),
    "serq_prepare": (_i, [_vp, _i, _i, _vp, _i, ctypes.POINTER(PrepareOpts), ctypes.POINTER(_vp)]),
    "serq_gptq_factor": (_i, [_vp, _i, _i, _vp]),
    "serq_layer_get_perm": (_i, [_vp, _vp]),
    "serq_layer_get_smooth": (_i, [_vp, _vp]),
    "serq_layer_destroy": (None, [_vp]),
    "serq_layer_info": (_i, [_vp, ctypes.POINTER(_i), ctypes.POINTER(_i), ctypes.POINTER(_i), ctypes.POINTER(_i)]),
    "serq_layer_perm_smooth": (_i, [_vp, ctypes.POINTER(_vp), ctypes.POINTER(_vp)]),
    "serq_layer_get_packed": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "serq_quantize_act": (_i, [_vp, _i, _i, _i, _i, _i, _vp, _vp, _vp]),
    "serq_linear": (_i, [_vp, _vp, _vp, _i, _vp, _i, _vp]),
    "serq_linear_ex": (_i, [_vp, _vp, _vp, _i, _vp, _i, _i, _vp]),
    "serq_linear_accum": (_i, [_vp, _vp, _i, _vp, _vp, _i, _vp]),
    "serq_linear_decode_static": (_i, [_vp, _vp, _vp, _i, _vp, _i, _vp, _vp, _vp]),
    "serq_linear_group": (_i, [_i, ctypes.POINTER(_vp), _vp, _vp, _i, ctypes.POINTER(_vp), ctypes.POINTER(_i),
                               ctypes.POINTER(_vp), ctypes.POINTER(_vp), _i, _vp]),
    "serq_linear_group_act": (_i, [_i, ctypes.POINTER(_vp), _vp, _i, _i, _i, _vp, _vp, ctypes.POINTER(_vp),
                                   ctypes.POINTER(_i), ctypes.POINTER(_vp), ctypes.POINTER(_vp), _i, _vp]),
    "serq_l2qer_prepare": (_i, [_vp, _vp, _vp, _i, ctypes.POINTER(_vp)]),
    "serq_l2qer_destroy": (None, [_vp]),
    "serq_l2qer_get_packed": (_i, [_vp, _vp, _vp, _vp, _vp]),
    "serq_l2qer_linear": (_i, [_vp, _vp, _vp, _i, _vp, _vp, _vp, _vp, _i, _i, _vp]),
    "serq_l2qer_accum": (_i, [_vp, _vp, _vp, _i, _vp, _vp, _i, _vp]),
    "serq_mx_prepare": (_i, [_vp, _vp, ctypes.POINTER(_vp)]),
    "serq_mx_destroy": (None, [_vp]),
    "serq_mx_get_packed": (_i, [_vp, _vp, _vp, _vp, _vp]),
    "serq_mx_act_scale_bytes": (ctypes.c_size_t, [_i, _i]),
    "serq_mx_quantize_act": (_i, [_vp, _i, _i, _i, _i, _vp, _vp, _vp]),
    "serq_mx_linear": (_i, [_vp, _vp, _vp, _i, _vp, _i, _vp]),
    "serq_silu_mul_quantize": (_i, [_vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp]),
    "serq_flatten_permute": (_i, [_vp, _vp, _i, _i, _i, _vp, _i, _i, _vp]),
    "serq_test_decode_timeout": (_i, [_vp, _vp, _vp, _i, _vp, _i, _i, _vp]),
    "serq_decode_max_m": (_i, []),
    "serq_last_error_string": (ctypes.c_char_p, []),
    "serq_check_device": (_i, []),
    "serq_device_error": (_i, [ctypes.POINTER(_i)]),
    "serq_version": (ctypes.c_char_p, []),
}

for _name, (_res, _args) in EXPORTS.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class SerqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib.serq_last_error_string().decode(errors="replace")
        super().__init__(f"{where}: status {status}: {msg}")


def _check(status: int, where: str):
    if status != OK:
        raise SerqError(status, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported activation dtype {t.dtype}")


def _mode_code(mode) -> int:
    if isinstance(mode, str):
        return {"w4a4": W4A4, "w4a8": W4A8}[mode.lower()]
    return int(mode)


def _cuda2d(t: torch.Tensor, name: str):
    if not t.is_cuda or t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be a 2-D CUDA tensor with unit column stride")


class Layer:
    """Owner of one prepared SERQ layer (device-resident packed weights)."""

    def __init__(self, handle: ctypes.c_void_p):
        self._h = handle
        K, N, r, m = _i(), _i(), _i(), _i()
        _check(lib.serq_layer_info(handle, ctypes.byref(K), ctypes.byref(N), ctypes.byref(r), ctypes.byref(m)),
               "serq_layer_info")
        self.K, self.N, self.rank, self.mode = K.value, N.value, r.value, m.value
        self.rpad = (self.rank + 31) // 32 * 32

    @property
    def handle(self):
        return self._h

    def close(self):
        if self._h:
            lib.serq_layer_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def perm_smooth_ptrs(self) -> Tuple[int, int]:
        p, s = _vp(), _vp()
        _check(lib.serq_layer_perm_smooth(self._h, ctypes.byref(p), ctypes.byref(s)), "serq_layer_perm_smooth")
        return p.value, s.value

    def perm_smooth(self) -> Tuple["np.ndarray", "np.ndarray"]:
        """Host copies of the saliency order (int32[K]) and scales (f32[K])
        (serq_layer_get_perm / serq_layer_get_smooth)."""
        import numpy as np
        perm = np.empty(self.K, np.int32)
        smooth = np.empty(self.K, np.float32)
        _check(lib.serq_layer_get_perm(self._h, perm.ctypes.data_as(_vp)), "serq_layer_get_perm")
        _check(lib.serq_layer_get_smooth(self._h, smooth.ctypes.data_as(_vp)), "serq_layer_get_smooth")
        return perm, smooth

    def get_packed(self) -> dict:
        """Host copies of everything prepare produced."""
        import numpy as np
        wq = np.empty(self.N * self.K // 2, np.uint8)
        rq = np.empty(max(1, self.N * self.rpad // 2), np.uint8)
        sw = np.empty(self.N, np.float32)
        sr = np.empty(self.N, np.float32)
        perm = np.empty(self.K, np.int32)
        smooth = np.empty(self.K, np.float32)
        c = lambda a: a.ctypes.data_as(_vp)
        _check(lib.serq_layer_get_packed(self._h, c(wq), c(rq) if self.rpad else None, c(sw), c(sr), c(perm),
                                         c(smooth)), "serq_layer_get_packed")
        return dict(wq=wq.reshape(self.N, self.K // 2),
                    rq=rq[: self.N * self.rpad // 2].reshape(self.N, self.rpad // 2),
                    sw=sw, sr=sr, perm=perm, smooth=smooth)


def _quantizer_code(q) -> int:
    if isinstance(q, str):
        return {"rtn": QUANT_RTN, "gptq": QUANT_GPTQ}[q.lower()]
    return int(q)


def prepare_opts(rank: int = 128, mode="w4a4", alpha: float = 0.5, saliency: int = SALIENCY_SCALE,
                 quantizer="rtn") -> PrepareOpts:
    o = PrepareOpts()
    lib.serq_prepare_opts_init(ctypes.byref(o))
    o.rank, o.mode, o.alpha, o.saliency = rank, _mode_code(mode), alpha, saliency
    o.quantizer = _quantizer_code(quantizer)
    return o


def prepare_group(weights: Sequence[torch.Tensor], X_calib: torch.Tensor, rank: int, mode="w4a4",
                  out_perm: Optional[Sequence[Optional[torch.Tensor]]] = None,
                  out_div: Optional[Sequence[Optional[torch.Tensor]]] = None,
                  alpha: float = 0.5, saliency: int = SALIENCY_SCALE, quantizer="rtn") -> List[Layer]:
    """serq_prepare_group: weights are CUDA fp32 K x N tensors sharing one
    input; out_perm / out_div are the next layer's order and smoothing scales
    per weight (CUDA tensors or None); quantizer "rtn" or "gptq"."""
    n = len(weights)
    K = weights[0].shape[0]
    for w in weights:
        _cuda2d(w, "W")
        if w.dtype != torch.float32 or not w.is_contiguous() or w.shape[0] != K:
            raise ValueError("weights must be contiguous fp32 K x N CUDA tensors with equal K")
    _cuda2d(X_calib, "X_calib")
    if X_calib.dtype != torch.float32 or not X_calib.is_contiguous():
        raise ValueError("X_calib must be contiguous fp32")
    Ws = (_vp * n)(*[w.data_ptr() for w in weights])
    Ns = (_i * n)(*[w.shape[1] for w in weights])
    ps = (_vp * n)(*[(p.data_ptr() if p is not None else None) for p in (out_perm or [None] * n)])
    ds = (_vp * n)(*[(d.data_ptr() if d is not None else None) for d in (out_div or [None] * n)])
    outs = (_vp * n)()
    o = prepare_opts(rank, mode, alpha, saliency, quantizer)
    _check(lib.serq_prepare_group(n, Ws, Ns, K, _ptr(X_calib), X_calib.shape[0], ctypes.byref(o), ps, ds, outs),
           "serq_prepare_group")
    return [Layer(_vp(outs[i])) for i in range(n)]


def prepare(W: torch.Tensor, X_calib: torch.Tensor, rank: int, mode="w4a4", out_perm=None,
            out_div=None, alpha: float = 0.5, saliency: int = SALIENCY_SCALE, quantizer="rtn") -> Layer:
    return prepare_group([W], X_calib, rank, mode, [out_perm], [out_div], alpha, saliency, quantizer)[0]


def gptq_factor(Xh: torch.Tensor) -> torch.Tensor:
    """serq_gptq_factor: Xh is the CUDA fp32 n x K flattened, permuted
    calibration activations; returns the K x K fp64 upper factor U with
    H^-1 = U^T U."""
    _cuda2d(Xh, "Xh")
    if Xh.dtype != torch.float32 or not Xh.is_contiguous():
        raise ValueError("Xh must be contiguous fp32")
    K = Xh.shape[1]
    U = torch.empty((K, K), dtype=torch.float64, device=Xh.device)
    _check(lib.serq_gptq_factor(_ptr(Xh), Xh.shape[0], K, _ptr(U)), "serq_gptq_factor")
    return U


def _host_f32(a, name):
    import numpy as np
    a = np.ascontiguousarray(a, dtype=np.float32)
    if a.ndim not in (1, 2):
        raise ValueError(f"{name} must be a 1-D or 2-D array")
    return a


def prepare_host(W, X_calib, rank: int = 128, mode="w4a4", alpha: float = 0.5,
                 saliency: int = SALIENCY_SCALE, out_perm=None, out_colscale=None, quantizer="rtn") -> Layer:
    """serq_prepare: W (K x N) and X_calib (n x K) are host (numpy) arrays;
    the library uploads them."""
    import numpy as np
    W = _host_f32(W, "W")
    Xc = _host_f32(X_calib, "X_calib")
    o = prepare_opts(rank, mode, alpha, saliency, quantizer)
    keep = []
    if out_perm is not None:
        keep.append(np.ascontiguousarray(out_perm, dtype=np.int32))
        o.out_perm = keep[-1].ctypes.data
    if out_colscale is not None:
        keep.append(np.ascontiguousarray(out_colscale, dtype=np.float32))
        o.out_colscale = keep[-1].ctypes.data
    out = _vp()
    _check(lib.serq_prepare(W.ctypes.data_as(_vp), W.shape[0], W.shape[1], Xc.ctypes.data_as(_vp), Xc.shape[0],
                            ctypes.byref(o), ctypes.byref(out)), "serq_prepare")
    return Layer(out)


def prepare_shared_host(weights, X_calib, rank: int = 128, mode="w4a4", alpha: float = 0.5,
                        saliency: int = SALIENCY_SCALE, out_perm=None, out_colscale=None,
                        quantizer="rtn") -> List[Layer]:
    """serq_prepare_shared: host (numpy) weights sharing one input."""
    import numpy as np
    Ws = [_host_f32(w, "W") for w in weights]
    n = len(Ws)
    Xc = _host_f32(X_calib, "X_calib")
    o = prepare_opts(rank, mode, alpha, saliency, quantizer)
    keep = list(Ws)
    def arr(seq, dt):
        if seq is None:
            return None
        ptrs = []
        for a in seq:
            if a is None:
                ptrs.append(None)
            else:
                keep.append(np.ascontiguousarray(a, dtype=dt))
                ptrs.append(keep[-1].ctypes.data)
        return (_vp * n)(*ptrs)
    outs = (_vp * n)()
    _check(lib.serq_prepare_shared(n, (_vp * n)(*[w.ctypes.data for w in Ws]), (_i * n)(*[w.shape[1] for w in Ws]),
                                   Ws[0].shape[0], Xc.ctypes.data_as(_vp), Xc.shape[0], ctypes.byref(o),
                                   arr(out_perm, np.int32), arr(out_colscale, np.float32), outs),
           "serq_prepare_shared")
    return [Layer(_vp(outs[i])) for i in range(n)]


def act_bytes_per_row(K: int, mode) -> int:
    return K // 2 if _mode_code(mode) == W4A4 else K


def quantize_act(X: torch.Tensor, mode="w4a4", Xq: Optional[torch.Tensor] = None,
                 sx: Optional[torch.Tensor] = None, stream=None):
    _cuda2d(X, "X")
    M, K = X.shape
    if Xq is None:
        Xq = torch.empty((M, act_bytes_per_row(K, mode)), dtype=torch.uint8, device=X.device)
    if sx is None:
        sx = torch.empty(M, dtype=torch.float32, device=X.device)
    _check(lib.serq_quantize_act(_ptr(X), _dtype_code(X), M, K, X.stride(0), _mode_code(mode), _ptr(Xq), _ptr(sx),
                                 _stream(stream)), "serq_quantize_act")
    return Xq, sx


def silu_mul_quantize(G: torch.Tensor, U: torch.Tensor, mode="w4a4", Xq=None, sx=None, stream=None):
    _cuda2d(G, "G")
    _cuda2d(U, "U")
    if G.shape != U.shape or G.stride(0) != U.stride(0) or G.dtype != torch.bfloat16 or U.dtype != torch.bfloat16:
        raise ValueError("G and U must be bf16 tensors of one shape and stride")
    M, F = G.shape
    if Xq is None:
        Xq = torch.empty((M, act_bytes_per_row(F, mode)), dtype=torch.uint8, device=G.device)
    if sx is None:
        sx = torch.empty(M, dtype=torch.float32, device=G.device)
    _check(lib.serq_silu_mul_quantize(_ptr(G), _ptr(U), M, F, G.stride(0), _mode_code(mode), _ptr(Xq), _ptr(sx),
                                      _stream(stream)), "serq_silu_mul_quantize")
    return Xq, sx


def flatten_permute(layer: Layer, X: torch.Tensor, out_dtype=torch.bfloat16, Xh=None, stream=None):
    _cuda2d(X, "X")
    M, K = X.shape
    if Xh is None:
        Xh = torch.empty((M, K), dtype=out_dtype, device=X.device)
    _check(lib.serq_flatten_permute(layer.handle, _ptr(X), _dtype_code(X), M, X.stride(0), _ptr(Xh),
                                    _dtype_code(Xh), Xh.stride(0), _stream(stream)), "serq_flatten_permute")
    return Xh


def linear(layer: Layer, Xq: torch.Tensor, sx: torch.Tensor, Y: Optional[torch.Tensor] = None,
           algo: int = ALGO_AUTO, stream=None) -> torch.Tensor:
    M = Xq.shape[0]
    if Y is None:
        Y = torch.empty((M, layer.N), dtype=torch.bfloat16, device=Xq.device)
    _check(lib.serq_linear_ex(layer.handle, _ptr(Xq), _ptr(sx), M, _ptr(Y), Y.stride(0), algo, _stream(stream)),
           "serq_linear")
    return Y


def linear_accum(layer: Layer, Xq: torch.Tensor, algo: int = ALGO_AUTO, stream=None):
    M = Xq.shape[0]
    acc0 = torch.empty((M, layer.N), dtype=torch.int32, device=Xq.device)
    acc1 = torch.empty((M, layer.N), dtype=torch.int32, device=Xq.device)
    _check(lib.serq_linear_accum(layer.handle, _ptr(Xq), M, _ptr(acc0), _ptr(acc1), algo, _stream(stream)),
           "serq_linear_accum")
    return acc0, acc1


def linear_group(layers, Xq: torch.Tensor, sx: Optional[torch.Tensor] = None, Ys=None,
                 algo: int = ALGO_AUTO, accum: bool = False, stream=None):
    """serq_linear_group: the products of up to four layers that share the
    activation codes Xq (equal K, rank and mode), as one prefill launch.
    Returns the list of bf16 outputs, or of (acc0, acc1) pairs when accum."""
    n = len(layers)
    M = Xq.shape[0]
    hl = (_vp * n)(*[L.handle for L in layers])
    if accum:
        accs = [(torch.empty((M, L.N), dtype=torch.int32, device=Xq.device),
                 torch.empty((M, L.N), dtype=torch.int32, device=Xq.device)) for L in layers]
        a0 = (_vp * n)(*[_ptr(a[0]) for a in accs])
        a1 = (_vp * n)(*[_ptr(a[1]) for a in accs])
        _check(lib.serq_linear_group(n, hl, _ptr(Xq), None, M, None, None, a0, a1, algo, _stream(stream)),
               "serq_linear_group")
        return accs
    if Ys is None:
        Ys = [torch.empty((M, L.N), dtype=torch.bfloat16, device=Xq.device) for L in layers]
    yp = (_vp * n)(*[_ptr(Y) for Y in Ys])
    ld = (_i * n)(*[Y.stride(0) for Y in Ys])
    _check(lib.serq_linear_group(n, hl, _ptr(Xq), _ptr(sx), M, yp, ld, None, None, algo, _stream(stream)),
           "serq_linear_group")
    return Ys


def linear_group_act(layers, X: torch.Tensor, Ys=None, Xq: Optional[torch.Tensor] = None,
                     sx: Optional[torch.Tensor] = None, algo: int = ALGO_AUTO, accum: bool = False, stream=None):
    """serq_linear_group_act: quantize the flattened activations X (bf16 or
    fp32, M x K) and run the group's products; one launch at decode sizes.
    Xq / sx are scratch (allocated here when not given).  Returns the bf16
    outputs, or (acc0, acc1) pairs when accum."""
    n = len(layers)
    M, K = X.shape
    if X.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("X must be bf16 or fp32")
    dt = BF16 if X.dtype == torch.bfloat16 else F32
    if Xq is None:
        Xq = torch.empty((M, K // 2 if layers[0].mode == W4A4 else K), dtype=torch.uint8, device=X.device)
    if sx is None:
        sx = torch.empty(M, dtype=torch.float32, device=X.device)
    hl = (_vp * n)(*[L.handle for L in layers])
    if accum:
        accs = [(torch.empty((M, L.N), dtype=torch.int32, device=X.device),
                 torch.empty((M, L.N), dtype=torch.int32, device=X.device)) for L in layers]
        a0 = (_vp * n)(*[_ptr(a[0]) for a in accs])
        a1 = (_vp * n)(*[_ptr(a[1]) for a in accs])
        _check(lib.serq_linear_group_act(n, hl, _ptr(X), dt, X.stride(0), M, _ptr(Xq), _ptr(sx), None, None, a0, a1,
                                         algo, _stream(stream)), "serq_linear_group_act")
        return accs
    if Ys is None:
        Ys = [torch.empty((M, L.N), dtype=torch.bfloat16, device=X.device) for L in layers]
    yp = (_vp * n)(*[_ptr(Y) for Y in Ys])
    ld = (_i * n)(*[Y.stride(0) for Y in Ys])
    _check(lib.serq_linear_group_act(n, hl, _ptr(X), dt, X.stride(0), M, _ptr(Xq), _ptr(sx), yp, ld, None, None,
                                     algo, _stream(stream)), "serq_linear_group_act")
    return Ys


def linear_decode_static(layer: Layer, Xq: torch.Tensor, sx: Optional[torch.Tensor] = None,
                         Y: Optional[torch.Tensor] = None, accum: bool = False, stream=None):
    """serq_linear_decode_static: the tensor-core decode kernel with its
    split-K scratch in the library's static per-device area (no allocation).
    Returns Y (bf16), or (acc0, acc1) when accum is True."""
    M = Xq.shape[0]
    if accum:
        acc0 = torch.empty((M, layer.N), dtype=torch.int32, device=Xq.device)
        acc1 = torch.empty((M, layer.N), dtype=torch.int32, device=Xq.device)
        _check(lib.serq_linear_decode_static(layer.handle, _ptr(Xq), None, M, None, 0, _ptr(acc0), _ptr(acc1),
                                             _stream(stream)), "serq_linear_decode_static")
        return acc0, acc1
    if Y is None:
        Y = torch.empty((M, layer.N), dtype=torch.bfloat16, device=Xq.device)
    _check(lib.serq_linear_decode_static(layer.handle, _ptr(Xq), _ptr(sx), M, _ptr(Y), Y.stride(0), None, None,
                                         _stream(stream)), "serq_linear_decode_static")
    return Y


class L2QER:
    """Owner of a two-factor comparator built on a prepared layer."""

    def __init__(self, layer: Layer, L1: torch.Tensor, L2: torch.Tensor):
        K, r = L1.shape
        if L2.shape != (r, layer.N) or K != layer.K:
            raise ValueError("L1 must be K x r and L2 r x N")
        for t, n in ((L1, "L1"), (L2, "L2")):
            if not t.is_cuda or t.dtype != torch.float32 or not t.is_contiguous():
                raise ValueError(f"{n} must be a contiguous fp32 CUDA tensor")
        self.layer, self.K, self.N, self.r = layer, K, layer.N, r
        h = _vp()
        _check(lib.serq_l2qer_prepare(layer.handle, _ptr(L1), _ptr(L2), r, ctypes.byref(h)), "serq_l2qer_prepare")
        self._h = h

    def close(self):
        if self._h:
            lib.serq_l2qer_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def get_packed(self) -> dict:
        import numpy as np
        l1q = np.empty(self.r * self.K // 2, np.uint8)
        s1 = np.empty(self.r, np.float32)
        l2q = np.empty(self.N * self.r // 2, np.uint8)
        s2 = np.empty(self.N, np.float32)
        c = lambda a: a.ctypes.data_as(_vp)
        _check(lib.serq_l2qer_get_packed(self._h, c(l1q), c(s1), c(l2q), c(s2)), "serq_l2qer_get_packed")
        return dict(l1q=l1q.reshape(self.r, self.K // 2), s_l1=s1, l2q=l2q.reshape(self.N, self.r // 2), s_l2=s2)

    def buffers(self, M: int, device):
        """Caller-owned intermediate buffers (Z bf16, Zq, sz) for M tokens."""
        return (torch.empty((M, self.r), dtype=torch.bfloat16, device=device),
                torch.empty((M, self.r // 2), dtype=torch.uint8, device=device),
                torch.empty(M, dtype=torch.float32, device=device))

    def linear(self, Xq: torch.Tensor, sx: torch.Tensor, Y=None, bufs=None, algo: int = ALGO_AUTO, stream=None):
        M = Xq.shape[0]
        if Y is None:
            Y = torch.empty((M, self.N), dtype=torch.bfloat16, device=Xq.device)
        Z, Zq, sz = bufs if bufs is not None else self.buffers(M, Xq.device)
        _check(lib.serq_l2qer_linear(self._h, _ptr(Xq), _ptr(sx), M, _ptr(Z), _ptr(Zq), _ptr(sz), _ptr(Y),
                                     Y.stride(0), algo, _stream(stream)), "serq_l2qer_linear")
        return Y, (Z, Zq, sz)

    def accum(self, Xq: torch.Tensor, Zq: torch.Tensor, algo: int = ALGO_AUTO, stream=None):
        M = Xq.shape[0]
        acc0 = torch.empty((M, self.N), dtype=torch.int32, device=Xq.device)
        acc1 = torch.empty((M, self.N), dtype=torch.int32, device=Xq.device)
        _check(lib.serq_l2qer_accum(self._h, _ptr(Xq), _ptr(Zq), M, _ptr(acc0), _ptr(acc1), algo, _stream(stream)),
               "serq_l2qer_accum")
        return acc0, acc1


class MXLayer:
    """Owner of a SERQ layer with MXFP4 codes (serq_mx_prepare): the smoothing
    scales, saliency order and rank of a prepared INT4 layer, W^ and R in OCP
    MX blocks of 32 along K."""

    def __init__(self, base: Layer, W: torch.Tensor):
        if not W.is_cuda or W.dtype != torch.float32 or not W.is_contiguous() or W.shape != (base.K, base.N):
            raise ValueError("W must be the base layer's contiguous K x N fp32 CUDA weight")
        self.K, self.N, self.r = base.K, base.N, base.rank
        h = _vp()
        _check(lib.serq_mx_prepare(base.handle, _ptr(W), ctypes.byref(h)), "serq_mx_prepare")
        self._h = h

    @property
    def handle(self):
        return self._h

    def close(self):
        if self._h:
            lib.serq_mx_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def get_packed(self) -> dict:
        """Codes (N x K/2, N x r/2 bytes) and untiled E8M0 scale bytes
        (N x K/32, N x r/32)."""
        import numpy as np
        wq = np.empty((self.N, self.K // 2), np.uint8)
        we = np.empty((self.N, self.K // 32), np.uint8)
        rq = np.empty((self.N, self.r // 2), np.uint8)
        re = np.empty((self.N, self.r // 32), np.uint8)
        c = lambda a: a.ctypes.data_as(_vp)
        _check(lib.serq_mx_get_packed(self._h, c(wq), c(we), c(rq), c(re)), "serq_mx_get_packed")
        return dict(wq=wq, we=we, rq=rq, re=re)


def mx_act_scale_bytes(M: int, K: int) -> int:
    return int(lib.serq_mx_act_scale_bytes(M, K))


def mx_quantize_act(Xh: torch.Tensor, Xq: Optional[torch.Tensor] = None, xe: Optional[torch.Tensor] = None,
                    stream=None):
    """Per-token MXFP4 codes (M x K/2 bytes) and tiled E8M0 scales."""
    _cuda2d(Xh, "Xh")
    M, K = Xh.shape
    if Xq is None:
        Xq = torch.empty((M, K // 2), dtype=torch.uint8, device=Xh.device)
    if xe is None:
        xe = torch.empty(max(1, mx_act_scale_bytes(M, K)), dtype=torch.uint8, device=Xh.device)
    _check(lib.serq_mx_quantize_act(_ptr(Xh), _dtype_code(Xh), M, K, Xh.stride(0), _ptr(Xq), _ptr(xe),
                                    _stream(stream)), "serq_mx_quantize_act")
    return Xq, xe


def mx_linear(layer: MXLayer, Xq: torch.Tensor, xe: torch.Tensor, Y: Optional[torch.Tensor] = None, stream=None):
    M = Xq.shape[0]
    if Y is None:
        Y = torch.empty((M, layer.N), dtype=torch.bfloat16, device=Xq.device)
    _check(lib.serq_mx_linear(layer.handle, _ptr(Xq), _ptr(xe), M, _ptr(Y), Y.stride(0), _stream(stream)),
           "serq_mx_linear")
    return Y


def device_error() -> int:
    c = _i()
    _check(lib.serq_device_error(ctypes.byref(c)), "serq_device_error")
    return c.value


def decode_max_m() -> int:
    return lib.serq_decode_max_m()


def version() -> str:
    return lib.serq_version().decode()
