"""Pins of the MXFP4 oracle (oracle/mxfp4_oracle.py) against what the OCP MX
specification and the mathematics fix, CPU only:

* the E2M1 values derived from the format's bit fields, and hand-worked
  roundings and 32-element blocks (tests/golden/mxfp4_blocks.json);
* the shared-exponent rule's invariant (amax / 2^e in [4, 8)) and the
  element error bound it implies;
* exactness: values already on the MXFP4 grid quantize to themselves and
  leave a zero compensator;
* the product against exact rational arithmetic on tiny inputs;
* the compensator shrinking the salient rows' error, and the storage layout
  (nibble order, E8M0 bytes, tiled scale offsets) against hand cases.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import mxfp4_oracle as X
from oracle import serq_oracle as O

G = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "mxfp4_blocks.json")))


def test_e2m1_values_from_the_bit_fields():
    # E2M1: sign | 2 exponent bits | 1 mantissa bit, bias 1; exponent field 0
    # is subnormal (0.m x 2^0), otherwise 1.m x 2^(e - 1)
    vals = []
    for code in range(16):
        s, e, m = code >> 3, (code >> 1) & 3, code & 1
        v = (m / 2.0) if e == 0 else (1 + m / 2.0) * 2.0 ** (e - 1)
        vals.append(-v if s else v)
    assert vals == G["e2m1_values_by_code"]
    assert np.array_equal(X.e2m1_value(np.arange(16)), np.array(vals))


def test_rounding_hand_cases():
    r = G["rounding"]
    assert np.array_equal(X.e2m1_code(r["t"]), np.array(r["code"], np.uint8))


@pytest.mark.parametrize("i", range(len(G["blocks"])))
def test_hand_worked_blocks(i):
    b = G["blocks"][i]
    if "values" in b:
        v, codes = np.array(b["values"]), b["codes"]
    else:
        v = np.ldexp(np.array(G["blocks"][b["like_block"]]["values"]), b["values_times_2pow"])
        codes = G["blocks"][b["codes_like_block"]]["codes"]
    c, e = X.mx_quantize(v[None, :])
    assert np.array_equal(c[0], np.array(codes, np.uint8))
    assert int(X.e8m0_bytes(e)[0, 0]) == b["scale_byte"]


def test_rounding_is_nearest_and_monotone():
    t = np.linspace(-8, 8, 64001)
    c = X.e2m1_code(t)
    v = X.e2m1_value(c)
    # nearest: no other E2M1 value is strictly closer (brute force over codes)
    d = np.abs(t - v)
    for code in range(16):
        assert np.all(d <= np.abs(t - X.e2m1_value(code)) + 0.0)
    assert np.all(np.diff(v) >= 0)                       # monotone
    assert np.array_equal(X.e2m1_value(X.e2m1_code(-t)), -X.e2m1_value(X.e2m1_code(t)) + 0.0)


def test_shared_exponent_hand_cases():
    cases = [(1.0, -2), (6.0, 0), (7.99, 0), (8.0, 1), (0.1, -6), (2.0 ** 100, 98), (0.0, -127),
             (2.0 ** -130, -127), (2.0 ** -124, -126), (float(np.finfo(np.float32).max), 125)]
    for a, e in cases:
        assert int(X.shared_exponent(a)) == e, a


def test_block_invariants_on_random_data():
    rng = np.random.default_rng(0)
    V = (rng.standard_normal((64, 256)) * np.exp(rng.uniform(-20, 20, (64, 1)))).astype(np.float32)
    V[3, 32:64] = 0.0
    c, e = X.mx_quantize(V.astype(np.float64))
    blk = np.abs(V.astype(np.float64)).reshape(64, 8, 32)
    amax = blk.max(axis=-1)
    nz = amax > 0
    ratio = amax[nz] / np.ldexp(1.0, e[nz])
    assert np.all((ratio >= 4) & (ratio < 8))            # the spec's exponent choice
    D = X.mx_dequantize(c, e)
    err = np.abs(D - V).reshape(64, 8, 32)
    # half of the widest gap (4 -> 6) below 6X, under 2X in the saturated band
    assert np.all(err <= np.ldexp(2.0, e)[..., None])
    inside = blk <= 6 * np.ldexp(1.0, e)[..., None]
    assert np.all(err[inside] <= np.broadcast_to(np.ldexp(1.0, e)[..., None], err.shape)[inside])
    assert np.all(c.reshape(64, 8, 32)[3, 1] == 0) and e[3, 1] == -127


def test_grid_values_are_fixed_points_and_leave_no_residual():
    rng = np.random.default_rng(1)
    K, N, r = 128, 48, 64
    # a folded weight that is already MXFP4: every block holds a 6 x 2^e
    # (so that e is its exponent) and grid values x 2^e elsewhere
    e = rng.integers(-8, 4, (N, K // 32))
    codes = rng.integers(0, 16, (N, K))
    codes[:, ::32] = 7
    What = X.mx_dequantize(codes, e)
    c2, e2 = X.mx_quantize(What)
    assert np.array_equal(e2, e)
    assert np.array_equal(X.e2m1_value(c2), X.e2m1_value(codes))
    # through prepare_from with s = 1 and the identity order: W^ = W, R = 0
    s = np.ones(K, np.float32)
    pi = np.arange(K, dtype=np.int32)
    L = X.prepare_from(s, pi, What.T.astype(np.float32), r)
    assert np.all(L.R == 0) and np.all(L.q_r == 0) and np.all(L.e_r == -127)
    assert np.array_equal(X.effective_weight(L), What.T)


def _exact_linear(xq, xe, L):
    """Sum over blocks of 2^(ex + ew) * sum of exact element products, in
    rationals; the residual product over the first r columns the same way."""
    M, K = xq.shape
    N = L.q_w.shape[0]
    val = [Fraction(v) for v in G["e2m1_values_by_code"]]

    def prod(xc, xs, wc, ws, m, n, nb):
        acc = Fraction(0)
        for b in range(nb):
            blk = sum(val[int(xc[m, 32 * b + j])] * val[int(wc[n, 32 * b + j])] for j in range(32))
            acc += blk * Fraction(2) ** int(xs[m, b] + ws[n, b])
        return acc

    Y = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            y = prod(xq, xe, L.q_w, L.e_w, m, n, K // 32)
            if L.r:
                y += prod(xq, xe, L.q_r, L.e_r, m, n, L.r // 32)
            Y[m, n] = float(y)
    return Y


@pytest.mark.parametrize("r", [0, 32, 64])
def test_product_against_exact_rationals(r):
    rng = np.random.default_rng(10 + r)
    K, N, M = 96, 5, 3
    W = rng.standard_normal((K, N)).astype(np.float32)
    Xc = rng.standard_normal((16, K)).astype(np.float32)
    Xc[:, 7] *= 30
    L = X.prepare(W, Xc, r)
    Xh = O.flatten_permute(rng.standard_normal((M, K)).astype(np.float32), L.s, L.pi, out_bf16=True)
    Y, xq, xe = X.linear(Xh, L)
    assert np.allclose(Y, _exact_linear(xq, xe, L), rtol=1e-13, atol=0)
    # a transposed or dropped operand fails this pin
    assert not np.allclose(Y, X.linear_codes(xq, xe, X.MXLayer(L.s, L.pi, L.W_hat, L.q_w, L.e_w, L.R,
                                                               np.zeros_like(L.q_r), L.e_r, r))) or r == 0


def test_compensator_shrinks_the_salient_rows_error():
    rng = np.random.default_rng(2)
    K, N, r = 256, 96, 64
    W = (0.02 * rng.standard_normal((K, N))).astype(np.float32)
    Xc = rng.standard_normal((64, K)).astype(np.float32)
    Xc[:, rng.choice(K, 6, replace=False)] *= 40
    L = X.prepare(W, Xc, r)
    What = L.W_hat.astype(np.float64)
    e0 = np.linalg.norm((What - X.effective_weight(L, with_residual=False))[:r])
    e1 = np.linalg.norm((What - X.effective_weight(L))[:r])
    assert e1 < 0.3 * e0
    # rows past r are untouched by the compensator
    assert np.array_equal(X.effective_weight(L)[r:], X.effective_weight(L, with_residual=False)[r:])
    # R is the main path's own error on the salient rows
    deq = X.mx_dequantize(L.q_w, L.e_w).T
    assert np.array_equal(L.R.T.astype(np.float64), (What[:r] - deq[:r]).astype(np.float32).astype(np.float64))


def test_prepare_keeps_the_int4_path_smoothing_and_order():
    rng = np.random.default_rng(3)
    K, N, r = 128, 64, 32
    W = rng.standard_normal((K, N)).astype(np.float32)
    Xc = rng.standard_normal((20, K)).astype(np.float32)
    L = X.prepare(W, Xc, r)
    Li = O.prepare(W, Xc, r)
    assert np.array_equal(L.s, Li.s) and np.array_equal(L.pi, Li.pi) and np.array_equal(L.W_hat, Li.W_hat)


def test_packing_and_scale_layout_hand_cases():
    assert np.array_equal(X.pack_fp4_rows(np.array([[1, 2, 15, 0, 7, 8]], np.uint8)),
                          np.array([[0x21, 0x0F, 0x87]], np.uint8))
    c = np.random.default_rng(4).integers(0, 16, (3, 64)).astype(np.uint8)
    assert np.array_equal(X.unpack_fp4_rows(X.pack_fp4_rows(c)), c)
    assert np.array_equal(X.e8m0_bytes(np.array([-127, 0, 1, 127])), np.array([0, 127, 128, 254], np.uint8))
    t = G["tile_offsets"]
    for row, blk, off in t["cases"]:
        assert int(X.scale_tile_offset(row, blk, t["n_blocks"])) == off
    e = np.arange(131 * 16).reshape(131, 16) % 200 - 100
    tiled = X.tile_scales(e)
    assert tiled.size == 256 * 16
    assert tiled[3089] == X.e8m0_bytes(e[130, 9])
    assert tiled[2627] == 0                  # row 200 (padding), block 3: tile 2, 72 * 8 + 3
