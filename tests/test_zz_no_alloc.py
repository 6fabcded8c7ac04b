"""serq_linear_decode_static: the tensor-core decode kernel with its split-K
scratch in the library's static per-device area instead of the layer's
workspace.  Collected last, so that the per-device scratch is first touched
after every other test has run.  Results must equal the oracle's exact
accumulators and the layer-workspace path bit for bit."""
import numpy as np
import pytest
import torch

from oracle import serq_oracle as O
from tests.gpu_support import assert_y_close
from tests.test_gpu_parity import S, _linear_case  # noqa: F401  (S is the module's device fixture)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,K,N,r,mode", [
    (1, 4096, 4096, 128, "w4a4"),
    (16, 4096, 1408, 128, "w4a4"),   # N % 128 != 0: a partial last tile
    (32, 1024, 512, 160, "w4a8"),
    (7, 256, 96, 16, "w4a4"),        # the tiny shape, r padded to 32
])
def test_static_scratch_matches_oracle(S, M, K, N, r, mode):
    L, ol, Xq, sx, xq, osx = _linear_case(S, M, K, N, r, mode, seed=11)
    acc0, acc1 = O.linear_accum(xq, ol)
    for _ in range(3):  # the scratch is left zero after every call
        g0, g1 = S.linear_decode_static(L, Xq, accum=True)
        Y = S.linear_decode_static(L, Xq, sx)
        torch.cuda.synchronize()
        assert np.array_equal(g0.cpu().numpy(), acc0) and np.array_equal(g1.cpu().numpy(), acc1)
        assert_y_close(Y, O.linear_epilogue(acc0, acc1, osx, ol))
    w0, w1 = S.linear_accum(L, Xq, S.ALGO_DECODE_TC)
    torch.cuda.synchronize()
    assert np.array_equal(w0.cpu().numpy(), acc0) and np.array_equal(w1.cpu().numpy(), acc1)
    assert S.device_error() == 0


def test_static_scratch_limits(S):
    L, ol, Xq, sx, xq, osx = _linear_case(S, 33, 256, 96, 16, "w4a4", seed=12)
    with pytest.raises(S.SerqError) as e:
        S.linear_decode_static(L, Xq, sx)
    assert e.value.status == 2  # SERQ_ERR_UNSUPPORTED_SHAPE: M > 32
    W = np.random.default_rng(0).normal(0, 0.02, (32, 16416)).astype(np.float32)
    Xc = np.random.default_rng(1).normal(0, 1, (8, 32)).astype(np.float32)
    big = S.prepare(torch.from_numpy(W).cuda(), torch.from_numpy(Xc).cuda(), 0, "w4a4")
    xq_big = torch.zeros((1, 16), dtype=torch.uint8, device="cuda")
    sx_big = torch.ones(1, dtype=torch.float32, device="cuda")
    with pytest.raises(S.SerqError) as e:
        S.linear_decode_static(big, xq_big, sx_big)
    assert e.value.status == 2  # N > 16384


def test_static_scratch_after_a_reported_timeout(S):
    """After serq_device_error has reported a timed-out wait, the next static
    call clears the scratch again (on its own stream) and is still exact."""
    L, ol, Xq, sx, xq, osx = _linear_case(S, 8, 1024, 512, 128, "w4a4", seed=13)
    acc0, acc1 = O.linear_accum(xq, ol)
    Y = torch.empty((8, 512), dtype=torch.bfloat16, device="cuda")
    assert S.lib.serq_test_decode_timeout(L.handle, S._ptr(Xq), S._ptr(sx), 8, S._ptr(Y), 512, 1000, None) == S.OK
    assert S.device_error() == 2
    for _ in range(2):
        g0, g1 = S.linear_decode_static(L, Xq, accum=True)
        torch.cuda.synchronize()
        assert np.array_equal(g0.cpu().numpy(), acc0) and np.array_equal(g1.cpu().numpy(), acc1)
    assert S.device_error() == 0
