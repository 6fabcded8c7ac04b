"""Pins for the CPU oracle of the two-factor comparator (L2QER): each test
checks it against something other than itself -- the SVD's exact
reconstruction, the Eckart-Young optimum in the scaled norm, a
dequantize-then-matmul restatement of the integer path, the fp64 value of
the intermediate.  CPU only."""
import numpy as np
import pytest

from oracle import l2qer_oracle as LQ
from oracle import serq_oracle as O
from w4a4_rank_gemm_b200 import synth

F32 = np.float32


def _case(M=24, K=128, N=96, seed=0):
    wl = synth.custom_layer(M, K, N, 32, "w4a4", "f32", seed=seed, n_calib=48)
    inp, W = wl.inputs["x"], wl.projections[0].W
    ol = O.prepare(W, inp.X_calib, 0)
    xh = O.flatten_permute(inp.X, ol.s, ol.pi, out_bf16=False)
    xc = O.flatten_permute(inp.X_calib, ol.s, ol.pi, out_bf16=False)
    return ol, xh, xc


def test_full_rank_factors_reconstruct_the_error_exactly():
    ol, xh, xc = _case()
    E = ol.W_hat.astype(np.float64) - ol.q_w.astype(np.float64) * ol.s_w.astype(np.float64)[None, :]
    S = LQ.activation_scale(xc)
    L1, L2 = LQ.factors(E, S, min(E.shape))
    np.testing.assert_allclose(L1 @ L2, E, rtol=0, atol=1e-12 * np.abs(E).max())


@pytest.mark.parametrize("r", [1, 8, 32])
def test_factors_are_the_scaled_eckart_young_optimum(r):
    """||S (E - L1 L2)||_F^2 equals the energy of S E beyond its r largest
    singular values, the least any rank-r correction can leave in that norm;
    a random rank-r correction, or the plain (unscaled) SVD's, leaves more."""
    ol, xh, xc = _case(seed=r)
    E = ol.W_hat.astype(np.float64) - ol.q_w.astype(np.float64) * ol.s_w.astype(np.float64)[None, :]
    S = LQ.activation_scale(xc)
    L1, L2 = LQ.factors(E, S, r)
    sig = np.linalg.svd(S[:, None] * E, compute_uv=False)
    got = np.linalg.norm(S[:, None] * (E - L1 @ L2)) ** 2
    assert got == pytest.approx(np.sum(sig[r:] ** 2), rel=1e-9)
    assert np.linalg.matrix_rank(L1 @ L2) == r
    U, sg, Vt = np.linalg.svd(E, full_matrices=False)       # unscaled truncated SVD
    plain = (U[:, :r] * sg[:r]) @ Vt[:r]
    assert np.linalg.norm(S[:, None] * (E - plain)) ** 2 >= got * (1 - 1e-12)


def test_activation_scale_is_the_mean_magnitude():
    x = np.array([[1.0, -2.0, 0.0], [-3.0, 2.0, 0.0]], F32)
    np.testing.assert_array_equal(LQ.activation_scale(x), [2.0, 2.0, 1e-5])


def test_intermediate_within_one_bf16_step_of_its_fp64_value():
    ol, xh, xc = _case(seed=3)
    lay = LQ.prepare(ol.W_hat, xc, 16)
    xq, sx = O.quantize_act(xh, 4)
    z_acc, Z, zq, sz = LQ.intermediate(xq, sx, lay)
    z64 = sx.astype(np.float64)[:, None] * lay.s_l1.astype(np.float64)[None, :] * z_acc
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(z64), 1e-30))) - 7)
    assert np.all(np.abs(Z - z64) <= ulp)
    # the on-the-fly quantization is the activation quantizer on Z
    zq2, sz2 = O.quantize_act(Z, 4)
    assert np.array_equal(zq, zq2) and np.array_equal(sz, sz2)


def test_linear_equals_dequantize_then_matmul():
    ol, xh, xc = _case(seed=5)
    lay = LQ.prepare(ol.W_hat, xc, 16)
    Y, xq, sx, acc0, zq, sz, acc2 = LQ.linear(xh, lay)
    deq = lambda q, s, ax: q.astype(np.float64) * np.expand_dims(s.astype(np.float64), ax)
    ref = deq(xq, sx, 1) @ deq(lay.q_w, lay.s_w, 0) + deq(zq, sz, 1) @ deq(lay.q_l2, lay.s_l2, 0)
    np.testing.assert_allclose(Y, ref, rtol=1e-12, atol=1e-12)
    # the main product is SERQ's, bit for bit (same W^, same codes)
    assert np.array_equal(acc0, O.int_matmul(xq, ol.q_w))


def test_correction_helps_on_outlier_data():
    """Statistical (not a pin): the two-factor correction lowers the output
    error of the 4-bit main path, and more rank lowers it further."""
    ol, xh, xc = _case(M=64, K=256, N=128, seed=9)
    ref = xh.astype(np.float64) @ ol.W_hat.astype(np.float64)
    errs = []
    for r in (0, 8, 64):
        if r == 0:
            xq, sx = O.quantize_act(xh, 4)
            y = sx.astype(np.float64)[:, None] * (O.int_matmul(xq, ol.q_w) * ol.s_w.astype(np.float64)[None, :])
        else:
            y = LQ.linear(xh, LQ.prepare(ol.W_hat, xc, r))[0]
        errs.append(np.linalg.norm(y - ref) / np.linalg.norm(ref))
    assert errs[2] < errs[1] < errs[0], errs
