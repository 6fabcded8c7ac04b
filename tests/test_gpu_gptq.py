"""GPU parity of GPTQ in the offline stage ("SERQ(GPTQ)" in the SERQ notes'
main results; gist.science (de) section 2B) against the CPU oracle: the fp64
inverse-Hessian factor and the packed codes and scales bit for bit, and the
quantized linear on a GPTQ-prepared layer (int32 accumulators bit-exact,
bf16 output within |y - y_ref| <= 1e-2 * max(|y_ref|, 1e-3))."""
import numpy as np
import pytest
import torch

from oracle import gptq_oracle as G
from oracle import serq_oracle as O
from tests.gpu_support import assert_y_close, bits, dev, expected_packed

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from w4a4_rank_gemm_b200 import serq  # raises if libserq.so is missing
    assert serq.lib.serq_check_device() == serq.OK, serq.lib.serq_last_error_string()
    return serq


def _calib(rng, n, K, corr=0.6, outliers=4):
    X = rng.standard_normal((n, K)).astype(np.float32)
    X[:, 1:] += np.float32(corr) * X[:, :-1]
    X[:, rng.choice(K, outliers, replace=False)] *= np.float32(25.0)
    return X


def _check_prepared(layer, ol):
    got = layer.get_packed()
    wq, rq = expected_packed(ol)
    assert np.array_equal(got["perm"], ol.pi), "saliency order differs"
    assert np.array_equal(bits(got["smooth"]), bits(ol.s)), "smoothing scales differ"
    assert np.array_equal(bits(got["sw"]), bits(ol.s_w)), "weight scales differ"
    assert np.array_equal(got["wq"], wq), "packed GPTQ codes differ"
    if ol.r:
        assert np.array_equal(bits(got["sr"]), bits(ol.s_r)), "compensator scales differ"
        assert np.array_equal(got["rq"], rq), "packed compensator codes differ"


# K = 32: one panel; 480: a ragged 64-tile edge; n not a multiple of 32
@pytest.mark.parametrize("K,n", [(32, 40), (256, 128), (480, 300), (512, 77)])
def test_factor_bit_exact(S, K, n):
    rng = np.random.default_rng(K + n)
    Xh = _calib(rng, n, K)
    U = S.gptq_factor(dev(Xh)).cpu().numpy()
    U_ref = G.inverse_hessian_factor(Xh)
    assert np.array_equal(U, U_ref), f"{np.count_nonzero(U != U_ref)} entries differ"
    assert np.all(np.tril(U, -1) == 0)


def test_factor_of_rank_deficient_and_zero_inputs(S):
    # fewer tokens than channels (H singular before the damping) and
    # all-zero activations (H = I, U = I)
    rng = np.random.default_rng(3)
    Xh = _calib(rng, 8, 128)
    assert np.array_equal(S.gptq_factor(dev(Xh)).cpu().numpy(), G.inverse_hessian_factor(Xh))
    Z = np.zeros((5, 64), np.float32)
    assert np.array_equal(S.gptq_factor(dev(Z)).cpu().numpy(), np.eye(64))


def test_factor_reports_a_nan_pivot(S):
    Xh = np.ones((16, 64), np.float32)
    Xh[3, 5] = np.nan
    with pytest.raises(RuntimeError) as e:
        S.gptq_factor(dev(Xh))
    assert e.value.status == S.ERR_NUMERIC and "pivot" in str(e.value)
    assert S.lib.serq_check_device() == S.OK      # the context stays usable
    ok = _calib(np.random.default_rng(4), 40, 64)
    assert np.array_equal(S.gptq_factor(dev(ok)).cpu().numpy(), G.inverse_hessian_factor(ok))


@pytest.mark.parametrize("K,Ns,r,n", [(256, [96, 160], 32, 64), (512, [128], 0, 100), (288, [64], 288, 50),
                                      (1024, [256, 64], 128, 256)])
def test_prepare_gptq_bit_exact(S, K, Ns, r, n):
    rng = np.random.default_rng(K + r)
    Xc = _calib(rng, n, K)
    Ws = [(0.02 * rng.standard_normal((K, N))).astype(np.float32) for N in Ns]
    _, _, ols = G.prepare_group(Ws, Xc, r)
    Ld = S.prepare_group([dev(W) for W in Ws], dev(Xc), r, "w4a4", quantizer="gptq")
    for L, ol in zip(Ld, ols):
        _check_prepared(L, ol)
    # the same from host arrays, one weight and a group
    _check_prepared(S.prepare_host(Ws[0], Xc, rank=r, quantizer="gptq"), G.prepare(Ws[0], Xc, r))
    for L, ol in zip(S.prepare_shared_host(Ws, Xc, rank=r, quantizer="gptq"), ols):
        _check_prepared(L, ol)
    if r < K:
        rtn = O.prepare_group(Ws, Xc, r)[2][0]
        assert not np.array_equal(rtn.q_w[r:], ols[0].q_w[r:]), "GPTQ should move some codes"


def test_prepare_gptq_with_options(S):
    rng = np.random.default_rng(11)
    K, N, r = 256, 128, 64
    Xc = _calib(rng, 48, K)
    W = (0.02 * rng.standard_normal((K, N))).astype(np.float32)
    W[rng.choice(K, 3, replace=False)] *= 8
    L = S.prepare_host(W, Xc, rank=r, alpha=0.7, saliency=S.SALIENCY_ROW_ABSMAX, quantizer="gptq")
    _check_prepared(L, G.prepare(W, Xc, r, alpha=0.7, saliency=O.SALIENCY_ROW_ABSMAX))


@pytest.mark.parametrize("M", [16, 300])
@pytest.mark.parametrize("mode", ["w4a4", "w4a8"])
def test_linear_on_a_gptq_layer(S, M, mode):
    rng = np.random.default_rng(M)
    K, N, r = 512, 384, 64
    Xc = _calib(rng, 128, K)
    W = (0.02 * rng.standard_normal((K, N))).astype(np.float32)
    ol = G.prepare(W, Xc, r)
    (L,) = S.prepare_group([dev(W)], dev(Xc), r, mode, quantizer="gptq")
    _check_prepared(L, ol)
    X = O.to_bf16(_calib(rng, M, K)).astype(np.float32)      # bf16 activations
    bits_a = 4 if mode == "w4a4" else 8
    xh = O.flatten_permute(X, ol.s, ol.pi, out_bf16=True)
    xq, osx = O.quantize_act(xh, bits_a)
    Xh = S.flatten_permute(L, dev(X).to(torch.bfloat16), out_dtype=torch.bfloat16)
    Xq, sx = S.quantize_act(Xh, mode)
    acc0, acc1 = O.linear_accum(xq, ol)
    g0, g1 = S.linear_accum(L, Xq, S.ALGO_AUTO)
    torch.cuda.synchronize()
    assert np.array_equal(g0.cpu().numpy(), acc0) and np.array_equal(g1.cpu().numpy(), acc1)
    assert_y_close(S.linear(L, Xq, sx), O.linear_epilogue(acc0, acc1, osx, ol))
    assert S.device_error() == 0


def test_prepare_gptq_with_output_fold(S):
    # the next layer's order and smoothing scales folded into the output
    # columns (SERQ notes, key design 3) before GPTQ runs on the folded weight
    rng = np.random.default_rng(12)
    K, N, r = 256, 192, 32
    Xc = _calib(rng, 64, K)
    W = (0.05 * rng.standard_normal((K, N))).astype(np.float32)
    P = rng.permutation(N).astype(np.int32)
    d = rng.uniform(0.2, 5.0, N).astype(np.float32)
    L = S.prepare_host(W, Xc, rank=r, out_perm=P, out_colscale=d, quantizer="gptq")
    _check_prepared(L, G.prepare(O.fold_output_columns(W, P, d), Xc, r))
