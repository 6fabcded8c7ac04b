"""CPU checks of the C ABI: the library loads, exports every function that
include/serq.h declares, and rejects bad arguments on the host before it
touches a device."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "serq.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(serq_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from w4a4_rank_gemm_b200 import build
    build.build()
    from w4a4_rank_gemm_b200 import serq
    return serq


def test_header_declares_the_boundary():
    names = _declared()
    for must in ("serq_prepare_group", "serq_prepare", "serq_quantize_act", "serq_linear",
                 "serq_linear_accum", "serq_silu_mul_quantize", "serq_layer_destroy"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", lib.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\sT\s+(serq_\w+)$", out, flags=re.M))
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing
    # and the binding knows each of them
    assert set(_declared()) <= set(lib.EXPORTS)


def test_version_and_constants(lib):
    assert "sm_100a" in lib.version()
    assert lib.decode_max_m() == 32


def test_host_side_argument_rejection(lib):
    L = lib.lib
    # null layer / null pointers are rejected before any device call
    assert L.serq_linear(None, None, None, 16, None, 256, None) == lib.ERR_INVALID_ARG
    assert b"null" in L.serq_last_error_string()
    assert L.serq_quantize_act(None, lib.BF16, 4, 256, 256, lib.W4A4, None, None, None) == lib.ERR_INVALID_ARG
    # K not a multiple of 32 is an unsupported shape (checked before device)
    fake = ctypes.c_void_p(0x1000)
    assert L.serq_quantize_act(fake, lib.BF16, 4, 100, 128, lib.W4A4, fake, fake, None) == lib.ERR_UNSUPPORTED_SHAPE
    # misaligned row stride
    assert L.serq_quantize_act(fake, lib.BF16, 4, 256, 260, lib.W4A4, fake, fake, None) == lib.ERR_INVALID_ARG
    # K beyond what the quantizer holds in registers
    assert L.serq_quantize_act(fake, lib.BF16, 4, 65536, 65536, lib.W4A4, fake, fake, None) == lib.ERR_UNSUPPORTED_SHAPE
    # prepare: rank > K and bad N
    W = (ctypes.c_void_p * 1)(0x1000)
    N = (ctypes.c_int * 1)(256)
    out = (ctypes.c_void_p * 1)()
    o = lib.prepare_opts(rank=300)
    assert L.serq_prepare_group(1, W, N, 256, fake, 8, ctypes.byref(o), None, None, out) == lib.ERR_UNSUPPORTED_SHAPE
    N[0] = 100
    o = lib.prepare_opts(rank=16)
    assert L.serq_prepare_group(1, W, N, 256, fake, 8, ctypes.byref(o), None, None, out) == lib.ERR_UNSUPPORTED_SHAPE
    assert out[0] is None


def test_prepare_options_host_side_rejection(lib):
    """serq_prepare / serq_prepare_shared / serq_prepare_group check their
    options before touching a device."""
    import numpy as np
    L = lib.lib
    o = lib.PrepareOpts()
    L.serq_prepare_opts_init(ctypes.byref(o))
    assert (abs(o.alpha - 0.5) < 1e-9, o.rank, o.mode, o.saliency, o.out_perm, o.out_colscale, o.quantizer) == \
        (True, 128, lib.W4A4, lib.SALIENCY_SCALE, None, None, lib.QUANT_RTN)
    W = np.zeros((256, 64), np.float32)
    Xc = np.zeros((4, 256), np.float32)
    out = ctypes.c_void_p()
    wp, xp = W.ctypes.data_as(ctypes.c_void_p), Xc.ctypes.data_as(ctypes.c_void_p)
    for field, value, status, msg in (("alpha", 1.5, lib.ERR_INVALID_ARG, b"alpha"),
                                      ("alpha", float("nan"), lib.ERR_INVALID_ARG, b"alpha"),
                                      ("rank", 257, lib.ERR_UNSUPPORTED_SHAPE, b"rank"),
                                      ("mode", 7, lib.ERR_INVALID_ARG, b"mode"),
                                      ("saliency", 2, lib.ERR_INVALID_ARG, b"saliency"),
                                      ("quantizer", 2, lib.ERR_INVALID_ARG, b"quantizer")):
        o = lib.prepare_opts(rank=32)
        setattr(o, field, value)
        assert L.serq_prepare(wp, 256, 64, xp, 4, ctypes.byref(o), ctypes.byref(out)) == status
        assert msg in L.serq_last_error_string()
        assert out.value is None
    # a column scale without an order
    o = lib.prepare_opts(rank=32)
    d = np.ones(64, np.float32)
    o.out_colscale = d.ctypes.data
    assert L.serq_prepare(wp, 256, 64, xp, 4, ctypes.byref(o), ctypes.byref(out)) == lib.ERR_INVALID_ARG
    assert b"without out_perm" in L.serq_last_error_string()
    # group calls take the folds per weight, not in the options
    Ws = (ctypes.c_void_p * 1)(W.ctypes.data)
    Ns = (ctypes.c_int * 1)(64)
    outs = (ctypes.c_void_p * 1)()
    assert L.serq_prepare_shared(1, Ws, Ns, 256, xp, 4, ctypes.byref(o), None, None, outs) == lib.ERR_INVALID_ARG
    assert b"per weight" in L.serq_last_error_string()
    assert L.serq_prepare_shared(1, Ws, Ns, 256, xp, 4, None, None, None, outs) == lib.ERR_INVALID_ARG
    assert outs[0] is None
    # silu: null inputs
    assert L.serq_silu_mul_quantize(None, None, 4, 256, 256, lib.W4A4, None, None, None) == lib.ERR_INVALID_ARG
    # the GPTQ factor: null pointers, K not a multiple of 32, no calibration rows
    buf = ctypes.c_void_p(1 << 20)
    assert L.serq_gptq_factor(None, 4, 256, buf) == lib.ERR_INVALID_ARG
    assert L.serq_gptq_factor(buf, 4, 256, None) == lib.ERR_INVALID_ARG
    assert L.serq_gptq_factor(buf, 4, 100, buf) == lib.ERR_UNSUPPORTED_SHAPE
    assert L.serq_gptq_factor(buf, 0, 256, buf) == lib.ERR_INVALID_ARG


def test_group_call_host_side_rejection(lib):
    """serq_linear_group checks the group on the host before any device call."""
    L = lib.lib
    fake = ctypes.c_void_p(0x1000)
    layers = (ctypes.c_void_p * 5)(0x1000, 0x1000, 0x1000, 0x1000, 0x1000)
    ys = (ctypes.c_void_p * 5)(0x1000, 0x1000, 0x1000, 0x1000, 0x1000)
    ld = (ctypes.c_int * 5)(256, 256, 256, 256, 256)
    for n in (0, 5, -1):
        assert L.serq_linear_group(n, layers, fake, fake, 16, ys, ld, None, None, 0, None) == lib.ERR_INVALID_ARG
        assert b"group of" in L.serq_last_error_string()
    assert L.serq_linear_group(2, None, fake, fake, 16, ys, ld, None, None, 0, None) == lib.ERR_INVALID_ARG
    # accumulators: both or neither
    accs = (ctypes.c_void_p * 2)(0x1000, 0x1000)
    assert L.serq_linear_group(2, layers, fake, None, 16, None, None, accs, None, 0, None) == lib.ERR_INVALID_ARG
    assert b"both or neither" in L.serq_last_error_string()
    # outputs missing when no accumulators are given
    assert L.serq_linear_group(2, layers, fake, fake, 16, None, None, None, None, 0, None) == lib.ERR_INVALID_ARG
    # a null layer in the list (checked before the layer is read)
    layers[0] = None
    assert L.serq_linear_group(2, layers, fake, fake, 16, ys, ld, None, None, 0, None) == lib.ERR_INVALID_ARG
    assert b"null layer 0" in L.serq_last_error_string()
    # the quantize-and-linear call: group size, null list or first layer, dtype
    layers[0] = 0x1000
    for n in (0, 5):
        assert L.serq_linear_group_act(n, layers, fake, lib.BF16, 256, 8, fake, fake, ys, ld, None, None, 0,
                                       None) == lib.ERR_INVALID_ARG
    assert L.serq_linear_group_act(2, None, fake, lib.BF16, 256, 8, fake, fake, ys, ld, None, None, 0,
                                   None) == lib.ERR_INVALID_ARG
    layers[0] = None
    assert L.serq_linear_group_act(2, layers, fake, lib.BF16, 256, 8, fake, fake, ys, ld, None, None, 0,
                                   None) == lib.ERR_INVALID_ARG
    layers[0] = 0x1000
    assert L.serq_linear_group_act(2, layers, fake, 7, 256, 8, fake, fake, ys, ld, None, None, 0,
                                   None) == lib.ERR_INVALID_ARG
    assert b"bad dtype" in L.serq_last_error_string()


def test_binding_refuses_to_load_without_library(tmp_path, monkeypatch):
    """The product path fails loudly when the CUDA library is missing."""
    import importlib.util
    import shutil
    pkg = tmp_path / "w4a4_rank_gemm_b200"
    pkg.mkdir()
    shutil.copy(os.path.join(ROOT, "w4a4_rank_gemm_b200", "serq.py"), pkg / "serq.py")
    spec = importlib.util.spec_from_file_location("serq_nolib", pkg / "serq.py")
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError, match="libserq.so not found"):
        spec.loader.exec_module(mod)


def test_comparator_host_side_rejection(lib):
    """The two-factor comparator's calls check their arguments on the host."""
    L = lib.lib
    out = ctypes.c_void_p()
    fake = ctypes.c_void_p(0x1000)
    assert L.serq_l2qer_prepare(None, fake, fake, 32, ctypes.byref(out)) == lib.ERR_INVALID_ARG
    assert L.serq_l2qer_prepare(fake, None, fake, 32, ctypes.byref(out)) == lib.ERR_INVALID_ARG
    assert out.value is None
    assert L.serq_l2qer_linear(None, fake, fake, 4, fake, fake, fake, fake, 256, 0, None) == lib.ERR_INVALID_ARG
    assert b"null comparator" in L.serq_last_error_string()
    assert L.serq_l2qer_accum(None, fake, fake, 4, fake, fake, 0, None) == lib.ERR_INVALID_ARG
    L.serq_l2qer_destroy(None)


def test_mxfp4_host_side_rejection(lib):
    """The MXFP4 calls check their arguments on the host; the scale-size
    helper is pure host arithmetic."""
    L = lib.lib
    out = ctypes.c_void_p()
    fake = ctypes.c_void_p(0x1000)
    assert L.serq_mx_prepare(None, fake, ctypes.byref(out)) == lib.ERR_INVALID_ARG
    assert L.serq_mx_prepare(fake, None, ctypes.byref(out)) == lib.ERR_INVALID_ARG
    assert out.value is None
    assert L.serq_mx_linear(None, fake, fake, 4, fake, 256, None) == lib.ERR_INVALID_ARG
    assert b"null MXFP4 layer" in L.serq_last_error_string()
    assert L.serq_mx_get_packed(None, None, None, None, None) == lib.ERR_INVALID_ARG
    # K must be a positive multiple of 256; rows 16-byte aligned; M in range
    assert L.serq_mx_quantize_act(fake, lib.BF16, 4, 384, 384, fake, fake, None) == lib.ERR_UNSUPPORTED_SHAPE
    assert L.serq_mx_quantize_act(fake, lib.BF16, 4, 256, 260, fake, fake, None) == lib.ERR_INVALID_ARG
    assert L.serq_mx_quantize_act(fake, lib.F32, 0, 256, 256, fake, fake, None) == lib.ERR_INVALID_ARG
    assert L.serq_mx_quantize_act(None, lib.F32, 4, 256, 256, fake, fake, None) == lib.ERR_INVALID_ARG
    assert L.serq_mx_quantize_act(fake, 7, 4, 256, 256, fake, fake, None) == lib.ERR_INVALID_ARG
    # scales of M tokens: rows padded to 128, K / 32 bytes each
    assert lib.mx_act_scale_bytes(1, 256) == 128 * 8
    assert lib.mx_act_scale_bytes(130, 4096) == 256 * 128
    assert lib.mx_act_scale_bytes(4, 100) == 0 and lib.mx_act_scale_bytes(0, 256) == 0
    L.serq_mx_destroy(None)
