"""GPU parity of the two-factor comparator (L2QER) against its CPU oracle on
the same seeded factors: packed factor codes and scales, the intermediate Z
(bf16), its codes and scales, and the final GEMM's accumulators bit for bit;
the output within the same tolerance as SERQ's."""
import numpy as np
import pytest
import torch

from oracle import l2qer_oracle as LQ
from oracle import serq_oracle as O
from w4a4_rank_gemm_b200 import synth
from tests.gpu_support import act_bytes, assert_y_close, bits, dev, dev_act

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from w4a4_rank_gemm_b200 import serq
    assert serq.lib.serq_check_device() == serq.OK, serq.lib.serq_last_error_string()
    return serq


def _case(S, M, K, N, r, seed):
    wl = synth.custom_layer(M, K, N, 128 if K >= 128 else 0, "w4a4", "bf16", seed=seed)
    inp, W = wl.inputs["x"], wl.projections[0].W
    rs = min(128, K)
    (L,) = S.prepare_group([dev(W)], dev(inp.X_calib), rs, "w4a4")
    ol = O.prepare(W, inp.X_calib, rs)
    L1, L2 = synth.factor_pair(K, N, r, seed=seed + 1)
    Q = S.L2QER(L, dev(L1), dev(L2))
    oq = LQ.prepare_from_factors(ol, L1, L2)
    Xh = S.flatten_permute(L, dev_act(inp.X, "bf16"))
    Xq, sx = S.quantize_act(Xh, "w4a4")
    xq, osx = O.quantize_act(O.flatten_permute(inp.X, ol.s, ol.pi, True), 4)
    assert np.array_equal(Xq.cpu().numpy(), act_bytes(xq, 4))
    return L, Q, oq, Xq, sx, xq, osx


def test_factor_codes_bit_exact(S):
    L, Q, oq, *_ = _case(S, 8, 512, 384, 64, seed=1)
    got = Q.get_packed()
    assert np.array_equal(got["l1q"], O.pack_int4_rows(np.ascontiguousarray(oq.q_l1.T)))
    assert np.array_equal(bits(got["s_l1"]), bits(oq.s_l1))
    assert np.array_equal(got["l2q"], O.pack_int4_rows(np.ascontiguousarray(oq.q_l2.T)))
    assert np.array_equal(bits(got["s_l2"]), bits(oq.s_l2))


CASES = [
    # M, K, N, r
    (1, 256, 128, 32),
    (16, 1024, 512, 128),
    (32, 512, 320, 64),
    (300, 1024, 512, 128),     # ragged M
    (600, 2048, 1280, 96),     # several tiles, ragged N
]


@pytest.mark.parametrize("M,K,N,r", CASES)
def test_comparator_path_bit_exact(S, M, K, N, r):
    L, Q, oq, Xq, sx, xq, osx = _case(S, M, K, N, r, seed=M + K + r)
    z_acc, Z, zq, sz = LQ.intermediate(xq, osx, oq)
    acc0 = O.int_matmul(xq, oq.q_w)
    acc2 = O.int_matmul(zq, oq.q_l2)
    y_ref = (osx.astype(np.float64)[:, None] * oq.s_w.astype(np.float64)[None, :] * acc0
             + sz.astype(np.float64)[:, None] * oq.s_l2.astype(np.float64)[None, :] * acc2)
    algos = [S.ALGO_AUTO, S.ALGO_PREFILL_N128, S.ALGO_PREFILL_PAIR_N256] + ([S.ALGO_DECODE] if M <= 32 else [])
    for algo in algos:
        Y, (Zg, Zqg, szg) = Q.linear(Xq, sx, algo=algo)
        a0, a1 = Q.accum(Xq, Zqg, algo=algo)
        torch.cuda.synchronize()
        assert np.array_equal(bits(Zg.float().cpu().numpy()), bits(Z)), f"intermediate differs (algo {algo})"
        assert np.array_equal(Zqg.cpu().numpy(), act_bytes(zq, 4)), f"intermediate codes differ (algo {algo})"
        assert np.array_equal(bits(szg.cpu().numpy()), bits(sz)), f"intermediate scales differ (algo {algo})"
        assert np.array_equal(a0.cpu().numpy(), acc0), f"acc0 differs (algo {algo})"
        assert np.array_equal(a1.cpu().numpy(), acc2), f"acc2 differs (algo {algo})"
        assert_y_close(Y, y_ref)
    assert S.device_error() == 0


def test_comparator_rejections(S):
    L, Q, oq, Xq, sx, xq, osx = _case(S, 40, 256, 128, 32, seed=3)
    with pytest.raises(S.SerqError, match="M <= 32"):
        Q.linear(Xq, sx, algo=S.ALGO_DECODE)
    with pytest.raises(S.SerqError, match="comparator runs"):
        Q.linear(Xq, sx, algo=S.ALGO_PREFILL_N256)
    L1, L2 = synth.factor_pair(256, 128, 48, seed=4)
    with pytest.raises(S.SerqError, match="multiple of 32"):
        S.L2QER(L, dev(L1), dev(L2))
