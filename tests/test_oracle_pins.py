"""Pins for the CPU oracle: each test checks the oracle against something other
than itself -- a hand-computed fixture, an algebraic identity the pages state,
a brute-force sum, a closed form or a library routine on a special case.
CPU only."""
import json
import math
import os

import numpy as np
import pytest

from oracle import serq_oracle as O
from w4a4_rank_gemm_b200 import synth

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "quantizer_cases.json")))
F32 = np.float32


# --------------------------------------------------------------------------
# Quantizer, packing, smoothing and ranking against hand-computed fixtures
# --------------------------------------------------------------------------
@pytest.mark.parametrize("case", GOLD["quantize"], ids=lambda c: c["why"][:20])
def test_quantizer_golden(case):
    x = np.array([case["x"]], dtype=F32)
    q, s = O.quantize_act(x, case["bits"])
    assert q[0].tolist() == case["codes"]
    assert float(s[0]) == pytest.approx(case["scale"], rel=1e-7, abs=0)


def test_pack_golden():
    g = GOLD["pack_int4"]
    codes = np.zeros((1, 32), np.int8)
    for k, v in g["codes"].items():
        codes[0, int(k)] = v
    b = O.pack_int4_rows(codes)[0]
    want = np.zeros(16, np.uint8)
    for k, v in g["bytes"].items():
        want[int(k)] = v
    assert b.tolist() == want.tolist()
    assert O.unpack_int4_rows(b[None])[0].tolist() == codes[0].tolist()


def test_pack_roundtrip_all_codes():
    rng = np.random.default_rng(0)
    codes = rng.integers(-8, 8, size=(7, 96)).astype(np.int8)
    codes[0, :16] = np.arange(-8, 8)
    codes[0, 16:32] = np.arange(7, -9, -1)
    assert np.array_equal(O.unpack_int4_rows(O.pack_int4_rows(codes)), codes)


def test_smooth_scales_golden():
    g = GOLD["smooth"]
    s = O.smooth_scales(np.array(g["X_calib"], F32), np.array(g["W"], F32))
    assert s.tolist() == g["s"]


def test_smooth_scales_group_uses_max_over_weights():
    rng = np.random.default_rng(0)
    Xc = rng.standard_normal((8, 6)).astype(F32)
    W1 = rng.standard_normal((6, 5)).astype(F32)
    W2 = (3 * rng.standard_normal((6, 7))).astype(F32)
    s = O.smooth_scales(Xc, [W1, W2])
    amax_w = np.maximum(np.abs(W1).max(1), np.abs(W2).max(1)).astype(np.float64)
    ref = np.sqrt(np.abs(Xc).max(0).astype(np.float64)) / np.sqrt(amax_w)
    np.testing.assert_allclose(s, ref, rtol=3e-7)


def test_saliency_golden():
    g = GOLD["saliency"]
    assert O.saliency_perm(np.array(g["s"], F32)).tolist() == g["perm"]


def test_quantizer_extremes_and_range():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((64, 100)).astype(F32)
    for bits in (4, 8):
        Q = O.QMAX[bits]
        q, s = O.quantize_act(x, bits)
        assert q.min() >= -Q and q.max() <= Q
        i = np.argmax(np.abs(x), axis=1)
        assert np.all(np.abs(q[np.arange(64), i]) == Q)       # +-amax -> +-Q
        # round-to-nearest: error at most half a step (plus fp32 slack)
        err = np.abs(q * s[:, None].astype(np.float64) - x)
        assert np.all(err <= 0.5 * s[:, None] * (1 + 1e-5) + 1e-12)


# --------------------------------------------------------------------------
# Flattening and permutation identities ([radio]: X diag(s^-1) P^-1 P diag(s) W
# = XW; [notes] key design 3: permutation costs nothing)
# --------------------------------------------------------------------------
def _layer(seed=0, M=24, K=96, N=40):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, K)).astype(F32)
    X[:, [3, 17, 50]] *= 40
    W = (0.02 * rng.standard_normal((K, N))).astype(F32)
    return X, W


def test_flatten_permute_identity():
    X, W = _layer()
    s = O.smooth_scales(X, W)
    pi = O.saliency_perm(s)
    y = O.flatten_permute(X, s, pi, False).astype(np.float64) @ O.fold_weight(W, s, pi).astype(np.float64)
    ref = X.astype(np.float64) @ W.astype(np.float64)
    assert np.max(np.abs(y - ref)) <= 1e-5 * np.max(np.abs(ref))


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_permutation_invariance(seed):
    X, W = _layer(seed)
    s = O.smooth_scales(X, W)
    perm = np.random.default_rng(seed).permutation(X.shape[1]).astype(np.int32)
    y1 = O.flatten_permute(X, s, perm, False).astype(np.float64) @ O.fold_weight(W, s, perm).astype(np.float64)
    y2 = O.flatten_permute(X, s, O.saliency_perm(s), False).astype(np.float64) @ \
        O.fold_weight(W, s, O.saliency_perm(s)).astype(np.float64)
    assert np.max(np.abs(y1 - y2)) <= 1e-5 * np.max(np.abs(y1))


def test_saliency_puts_outlier_channels_first():
    X, W = _layer()
    s = O.smooth_scales(X, W)
    pi = O.saliency_perm(s)
    assert set(pi[:3].tolist()) == {3, 17, 50}
    assert np.all(np.diff(s[pi].astype(np.float64)) <= 0)


# --------------------------------------------------------------------------
# Compensator ([notes] core idea: R = W~_s - Q(W~_s))
# --------------------------------------------------------------------------
@pytest.mark.parametrize("r", [1, 8, 32])
def test_compensator_reconstructs_salient_rows(r):
    X, W = _layer(4)
    L = O.prepare(W, X, r)
    deq = L.q_w.astype(np.float64) * L.s_w.astype(np.float64)[None, :]
    recon = deq[:r] + L.R.astype(np.float64)
    target = L.W_hat[:r].astype(np.float64)
    # exact up to two fp32 roundings: of code*scale and of the subtraction
    bound = 2.0 ** -24 * (np.abs(deq[:r]) + np.abs(target - deq[:r]))
    assert np.all(np.abs(recon - target) <= bound)
    # and far better than the main path alone
    assert np.abs(recon - target).max() < 1e-3 * np.abs(target - deq[:r]).max()
    assert L.R.shape == (r, W.shape[1])       # R is r x d_out
    # rows past r are untouched by the compensator
    assert L.q_r.shape == (r, W.shape[1])


def test_compensator_is_not_a_separate_quantization():
    # A plausible mistake is R = W~_s - Q_sep(W~_s) with W~_s quantized on its
    # own (scale from the r rows only); that does not cancel the main error.
    X, W = _layer(5)
    r = 8
    L = O.prepare(W, X, r)
    q_sep, s_sep = O.quantize_weight(L.W_hat[:r])
    R_wrong = L.W_hat[:r] - q_sep * s_sep[None, :]
    assert not np.allclose(R_wrong, L.R)
    eff = L.q_w[:r] * L.s_w.astype(np.float64) + L.R
    assert np.allclose(eff, L.W_hat[:r], atol=1e-7)


# --------------------------------------------------------------------------
# Integer GEMM and epilogue
# --------------------------------------------------------------------------
def test_int_matmul_bruteforce():
    rng = np.random.default_rng(6)
    a = rng.integers(-7, 8, size=(5, 13)).astype(np.int8)
    b = rng.integers(-7, 8, size=(13, 4)).astype(np.int8)
    got = O.int_matmul(a, b)
    for m in range(5):
        for n in range(4):
            assert got[m, n] == sum(int(a[m, k]) * int(b[k, n]) for k in range(13))


def test_int_matmul_large_is_exact():
    # W4A8 worst case: |acc| <= 127 * 7 * K stays exact
    K = 14336
    a = np.full((2, K), 127, np.int8); a[1] = -127
    b = np.full((K, 3), 7, np.int8)
    got = O.int_matmul(a, b)
    assert got[0, 0] == 127 * 7 * K and got[1, 2] == -127 * 7 * K


def test_linear_equals_dequantize_then_matmul():
    X, W = _layer(7, M=9, K=64, N=24)
    r = 16
    L = O.prepare(W, X, r)
    xh = O.flatten_permute(X, L.s, L.pi, False)
    y, xq, sx, acc0, acc1 = O.linear(xh, L, 4)
    # brute-force definition: Y[m,n] = sum_k deqX[m,k] * Weff[k,n]
    deqx = xq.astype(np.float64) * sx.astype(np.float64)[:, None]
    Weff = O.dequant_weight(L, True)
    ref = np.zeros((9, 24))
    for m in range(9):
        for n in range(24):
            ref[m, n] = math.fsum(deqx[m, k] * Weff[k, n] for k in range(64))
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)
    # residual uses only the first r code columns
    assert np.array_equal(acc1, O.int_matmul(xq[:, :r], L.q_r))


def test_w4a8_integer_activations_exact():
    rng = np.random.default_rng(8)
    xi = rng.integers(-127, 128, size=(4, 32)).astype(F32)
    xi[:, 0] = 127
    q, s = O.quantize_act(xi, 8)
    assert np.array_equal(q.astype(F32), xi) and np.all(s == 1)


def test_r0_reduces_to_smoothquant_rtn():
    X, W = _layer(9)
    L = O.prepare(W, X, 0)
    xh = O.flatten_permute(X, L.s, L.pi, False)
    y = O.linear(xh, L, 4)[0]
    # textbook fake-quant matmul: per-token and per-channel RTN in fp64
    qx, sx = O.quantize_act(xh, 4)
    qw, sw = O.quantize_weight(L.W_hat, 4)
    ref = (qx * sx[:, None].astype(np.float64)) @ (qw * sw[None, :].astype(np.float64))
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_r_equals_k_unquantized_leaves_only_activation_error():
    X, W = _layer(10, K=64)
    K = 64
    L = O.prepare(W, X, K)
    xh = O.flatten_permute(X, L.s, L.pi, False)
    qx, sx = O.quantize_act(xh, 4)
    deqx = qx * sx[:, None].astype(np.float64)
    Weff = L.q_w * L.s_w.astype(np.float64)[None, :] + L.R.astype(np.float64)
    np.testing.assert_allclose(Weff, L.W_hat, rtol=0, atol=1e-6 * np.abs(L.W_hat).max())
    y = deqx @ Weff
    np.testing.assert_allclose(y, deqx @ L.W_hat.astype(np.float64), rtol=1e-5, atol=1e-6)


def test_rank_trend_on_outlier_data():
    """Statistical (the rank ablation's trend: error falls as r grows)."""
    wl = synth.custom_layer(64, 512, 256, 0, act_dtype="f32", seed=11, n_outliers=8)
    X, W = wl.inputs["x"].X, wl.projections[0].W
    ref = X.astype(np.float64) @ W.astype(np.float64)
    errs = []
    for r in (0, 16, 128):
        L = O.prepare(W, wl.inputs["x"].X_calib, r)
        y = O.linear(O.flatten_permute(X, L.s, L.pi, False), L, 4)[0]
        errs.append(np.linalg.norm(y - ref) / np.linalg.norm(ref))
    assert errs[0] > errs[1] > errs[2]


# --------------------------------------------------------------------------
# fp32 exponential and SiLU (Cody-Waite + Taylor) against libm in fp64
# --------------------------------------------------------------------------
def test_exp_f32_accuracy():
    x = np.concatenate([np.linspace(-87.9, 87.9, 200001, dtype=F32),
                        np.array([0, -0.0, 1e-8, -1e-8, 0.3465, -0.3466, 1, -1], F32)])
    got = O.exp_f32(x).astype(np.float64)
    ref = np.exp(x.astype(np.float64))
    ulp = np.spacing(ref.astype(F32)).astype(np.float64)
    assert np.max(np.abs(got - ref) / ulp) <= 4.0
    assert O.exp_f32(np.array([0.0], F32))[0] == 1.0


def test_exp_f32_saturation():
    assert np.isinf(O.exp_f32(np.array([89.0, 200.0], F32))).all()
    assert (O.exp_f32(np.array([-89.0, -1e4], F32)) == 0).all()


def test_silu_mul_against_fp64():
    rng = np.random.default_rng(12)
    g = (4 * rng.standard_normal(5000)).astype(F32)
    u = rng.standard_normal(5000).astype(F32)
    got = O.silu_mul_f32(g, u).astype(np.float64)
    gd = g.astype(np.float64)
    ref = gd / (1 + np.exp(-gd)) * u.astype(np.float64)
    assert np.max(np.abs(got - ref) / np.maximum(np.abs(ref), 1e-30)) <= 1e-6
    # saturation: large negative gate -> exactly zero; large positive -> g*u
    assert O.silu_mul_f32(np.array([-100.0], F32), np.array([3.0], F32))[0] == 0
    assert O.silu_mul_f32(np.array([100.0], F32), np.array([3.0], F32))[0] == 300.0


# --------------------------------------------------------------------------
# MLP-block permutation propagation ([notes] key design 3)
# --------------------------------------------------------------------------
def _silu64(x):
    return x / (1 + np.exp(-x))


def test_mlp_fold_is_exact_without_quantization():
    rng = np.random.default_rng(13)
    M, K, F = 8, 32, 48
    X = rng.standard_normal((M, K)).astype(F32)
    Wg = (0.1 * rng.standard_normal((K, F))).astype(F32)
    Wu = (0.1 * rng.standard_normal((K, F))).astype(F32)
    Wd = (0.1 * rng.standard_normal((F, K))).astype(F32)
    Hc = (_silu64(X.astype(np.float64) @ Wg) * (X.astype(np.float64) @ Wu)).astype(F32)
    s4 = O.smooth_scales(Hc, Wd)
    pi4 = O.saliency_perm(s4)
    Wg_f = O.fold_output_columns(Wg, pi4, None)
    Wu_f = O.fold_output_columns(Wu, pi4, s4)
    s = O.smooth_scales(X, [Wg_f, Wu_f])
    pi = O.saliency_perm(s)
    xh = O.flatten_permute(X, s, pi, False).astype(np.float64)
    g = xh @ O.fold_weight(Wg_f, s, pi).astype(np.float64)
    u = xh @ O.fold_weight(Wu_f, s, pi).astype(np.float64)
    h = _silu64(g) * u                                # arrives already as X^_4
    y = h @ O.fold_weight(Wd, s4, pi4).astype(np.float64)
    Xd = X.astype(np.float64)
    ref = (_silu64(Xd @ Wg) * (Xd @ Wu)) @ Wd.astype(np.float64)
    assert np.max(np.abs(y - ref)) <= 1e-5 * np.max(np.abs(ref))
    # and the intermediate is exactly down_proj's flattened, permuted input
    h_direct = O.flatten_permute((_silu64(Xd @ Wg) * (Xd @ Wu)).astype(F32), s4, pi4, False)
    np.testing.assert_allclose(h, h_direct, rtol=1e-5, atol=1e-6)


def test_mlp_quantized_chain_tracks_full_precision():
    """Statistical: the W4A4 chain stays near the fp64 block (4-bit RTN on
    Gaussian data costs ~10-15% per layer) and a larger rank helps."""
    blk = synth.mlp_block(M=32, K=256, F=512, rank=32, seed=14, n_calib=64)
    Xd = blk.X.astype(np.float64)
    ref = (_silu64(Xd @ blk.Wg) * (Xd @ blk.Wu)) @ blk.Wd.astype(np.float64)
    rel = []
    for r in (0, 128):
        prep = O.prepare_mlp(blk.Wg, blk.Wu, blk.Wd, blk.X_calib, blk.H_calib, r)
        y = O.mlp_forward(blk.X, prep)["y"]
        rel.append(np.linalg.norm(y - ref) / np.linalg.norm(ref))
    assert rel[1] < rel[0] < 0.4, rel


# --------------------------------------------------------------------------
# bf16 storage rounding and the smoothing floor against hand-worked bits
# --------------------------------------------------------------------------
GOLD2 = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "bf16_and_floor_cases.json")))


def _u32(h):
    return np.array([int(h, 16)], dtype=np.uint32)


@pytest.mark.parametrize("case", GOLD2["bf16"]["cases"], ids=lambda c: c["in"])
def test_to_bf16_golden(case):
    x = _u32(case["in"]).view(F32)
    with np.errstate(over="ignore"):
        got = O.to_bf16(x).view(np.uint32)
    assert int(got[0]) == int(case["out"], 16), case["why"]


def test_to_bf16_keeps_representable_values_and_halves_the_error():
    """Every bf16 value is a fixed point, and the rounding error of any other
    finite value is at most half a bf16 ulp (ties to even), checked on all
    2^16 upper halves with random lower halves."""
    rng = np.random.default_rng(2)
    hi = np.arange(1 << 16, dtype=np.uint32)
    exact = (hi << 16).view(F32)
    finite = np.isfinite(exact)
    assert np.array_equal(O.to_bf16(exact[finite]).view(np.uint32), (hi << 16)[finite])
    lo = rng.integers(0, 1 << 16, size=hi.size, dtype=np.uint32)
    x = ((hi << 16) | lo).view(F32)
    ok = np.isfinite(x) & (np.abs(x) < F32(3.0e38))
    x = x[ok]
    y = O.to_bf16(x).astype(np.float64)
    xe = x.astype(np.float64)
    # ulp of the bf16 grid at |x|: 2^(exponent - 7), subnormals 2^-133
    e = np.floor(np.log2(np.maximum(np.abs(xe), 2.0 ** -126)))
    ulp = 2.0 ** (e - 7)
    assert np.all(np.abs(y - xe) <= ulp / 2)


def test_smooth_scales_floor_golden():
    g = GOLD2["smooth_floor"]
    s = O.smooth_scales(np.array(g["X_calib"], F32), np.array(g["W"], F32))
    got = [f"0x{int(b):08X}" for b in s.view(np.uint32)]
    assert got == g["s_bits"], list(zip(got, g["why"]))
    assert O.saliency_perm(s).tolist() == g["perm"]


# --------------------------------------------------------------------------
# The MLP fold (key design 3): prepare_mlp / mlp_forward against a chain
# built without any fold.  Moving down_proj's order P4 into the gate/up
# output columns is a pure column permutation, so every per-column step
# (row maxima, per-channel quantization, the compensator, the epilogue,
# silu * mul) must give the permuted values of the unfolded chain bit for
# bit, provided the unfolded up_proj has its columns divided by s4 (the
# smoothing divisor of down_proj, which passes through up only).
# --------------------------------------------------------------------------
def _mlp_blk():
    return synth.mlp_block(M=24, K=96, F=160, rank=32, seed=21, n_calib=48)


def _fold_mismatches(prep, blk, r):
    """Names of the checks on which `prep` differs from the unfolded chain."""
    bad = []
    s4, pi4, (down,) = O.prepare_group([blk.Wd], blk.H_calib, r)
    if not (np.array_equal(prep["pi4"], pi4) and np.array_equal(prep["s4"].view(np.uint32), s4.view(np.uint32))):
        bad.append("down order / scales")
    Wu_div = (blk.Wu / s4[None, :]).astype(F32)
    s_ref, pi_ref, (g_ref, u_ref) = O.prepare_group([blk.Wg, Wu_div], blk.X_calib, r)
    if not (np.array_equal(prep["s_gu"].view(np.uint32), s_ref.view(np.uint32))
            and np.array_equal(prep["pi_gu"], pi_ref)):
        bad.append("gate/up smoothing")
    for name, ref in (("gate", g_ref), ("up", u_ref)):
        L = prep[name]
        same = (np.array_equal(L.q_w, ref.q_w[:, pi4]) and np.array_equal(L.s_w, ref.s_w[pi4])
                and np.array_equal(L.q_r, ref.q_r[:, pi4]) and np.array_equal(L.s_r, ref.s_r[pi4]))
        if not same:
            bad.append(name + " codes")
    out = O.mlp_forward(blk.X, prep)
    xh = O.flatten_permute(blk.X, s_ref, pi_ref, out_bf16=True)
    g = O.to_bf16(O.linear(xh, g_ref)[0].astype(F32))[:, pi4]
    u = O.to_bf16(O.linear(xh, u_ref)[0].astype(F32))[:, pi4]
    if not (np.array_equal(out["g"], g) and np.array_equal(out["u"], u)):
        bad.append("gate/up outputs")
    h = O.silu_mul_f32(g, u)
    if not np.array_equal(out["h"].view(np.uint32), h.view(np.uint32)):
        bad.append("intermediate")
    y = O.linear(h, down)[0]
    if not np.array_equal(out["y"], y):
        bad.append("block output")
    return bad


def test_prepare_mlp_is_the_permuted_unfolded_chain():
    blk = _mlp_blk()
    prep = O.prepare_mlp(blk.Wg, blk.Wu, blk.Wd, blk.X_calib, blk.H_calib, 32)
    assert _fold_mismatches(prep, blk, 32) == []
    # the folded intermediate is down_proj's flattened input: h / s4 in P4 order
    # up to the rounding of the quantized layers (not a pin, a sanity bound)
    assert not np.array_equal(prep["pi4"], np.arange(blk.Wd.shape[0]))


@pytest.mark.parametrize("mistake", ["s4 also on gate", "P4 inverted", "s4 left out of up"])
def test_prepare_mlp_check_catches_misfolds(mistake):
    """The check above fails on plausible wrong folds (planted in a copy of
    the oracle's preparation, on the CPU)."""
    blk = _mlp_blk()
    r = 32
    s4, pi4, (down,) = O.prepare_group([blk.Wd], blk.H_calib, r)
    inv = np.argsort(pi4).astype(np.int32)
    assert not np.array_equal(inv, pi4)
    if mistake == "s4 also on gate":
        Wg_f, Wu_f = O.fold_output_columns(blk.Wg, pi4, s4), O.fold_output_columns(blk.Wu, pi4, s4)
    elif mistake == "P4 inverted":
        Wg_f, Wu_f = O.fold_output_columns(blk.Wg, inv, None), O.fold_output_columns(blk.Wu, inv, s4)
    else:
        Wg_f, Wu_f = O.fold_output_columns(blk.Wg, pi4, None), O.fold_output_columns(blk.Wu, pi4, None)
    s_gu, pi_gu, (gate, up) = O.prepare_group([Wg_f, Wu_f], blk.X_calib, r)
    bad = dict(s_gu=s_gu, pi_gu=pi_gu, gate=gate, up=up, s4=s4, pi4=pi4, down=down)
    assert _fold_mismatches(bad, blk, r) != []


# --------------------------------------------------------------------------
# Preparation options: SmoothQuant's migration strength alpha and the
# saliency metric (the reading by the folded row's absolute maximum)
# --------------------------------------------------------------------------
def test_smooth_scales_alpha_closed_forms():
    Xc = np.array([[16.0, -2.0, 0.0], [3.0, 1.0, 0.0]], F32)   # column maxima 16, 2, 0 (-> 1e-5)
    W = np.array([[0.25, 0.0], [-3.0, 1.0], [0.5, 0.0]], F32)    # row maxima 0.25, 3, 0.5
    # alpha = 3/4 by hand: 16^(3/4) / 0.25^(1/4) = 8 / 2^(-1/2) = 8 sqrt(2) = 11.3137085 -> 0x413504f3
    s = O.smooth_scales(Xc, W, alpha=0.75)
    assert f"0x{int(s.view(np.uint32)[0]):08x}" == "0x413504f3"
    # alpha = 1: s = the floored activation maximum itself; alpha = 0: s = 1 / weight maximum
    s1 = O.smooth_scales(Xc, W, alpha=1.0)
    assert s1.tolist() == [16.0, 2.0, float(F32(1e-5))]
    s0 = O.smooth_scales(Xc, W, alpha=0.0)
    assert s0.tolist() == [4.0, float(F32(1.0 / 3.0)), 2.0]
    # the general path agrees with the square-root path next to alpha = 1/2
    rng = np.random.default_rng(4)
    Xr = np.abs(rng.standard_normal((16, 64))).astype(F32) * F32(30)
    Wr = (0.02 * rng.standard_normal((64, 40))).astype(F32)
    near = O.smooth_scales(Xr, Wr, alpha=float(np.nextafter(F32(0.5), F32(1))))
    half = O.smooth_scales(Xr, Wr, alpha=0.5)
    np.testing.assert_allclose(near, half, rtol=1e-5)


def test_saliency_metric_row_absmax_golden():
    # column maxima 4, 4, 4 and row maxima 4, 1, 0.25: s = 2/2, 2/1, 2/0.5 = 1, 2, 4 (exact);
    # folded row maxima s * amax_w = 4, 2, 1
    Xc = np.array([[4.0, -4.0, 1.0], [0.5, 2.0, -4.0]], F32)
    W = np.array([[-4.0, 1.0], [0.5, 1.0], [0.25, -0.125]], F32)
    s = O.smooth_scales(Xc, W)
    assert s.tolist() == [1.0, 2.0, 4.0]
    assert O.saliency_perm(O.saliency_key(s, W, O.SALIENCY_SCALE)).tolist() == [2, 1, 0]
    assert O.saliency_perm(O.saliency_key(s, W, O.SALIENCY_ROW_ABSMAX)).tolist() == [0, 1, 2]
    # the folded weight's row maxima are what metric 1 ranks
    W_hat = O.fold_weight(W, s, np.arange(3))
    np.testing.assert_array_equal(np.abs(W_hat).max(1), O.saliency_key(s, W, O.SALIENCY_ROW_ABSMAX))
