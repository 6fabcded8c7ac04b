"""Failure detection without a GPU fault: a kernel whose bounded wait runs
out (here the streaming decode kernel with its activation copies withheld
by a test-only argument and a 2 ms limit) records the timeout in the device
status word, leaves its outputs alone and returns; the context stays usable
and the next call is bit-exact."""
import time

import numpy as np
import pytest
import torch

from oracle import serq_oracle as O
from tests.gpu_support import assert_y_close
from tests.test_gpu_parity import S, _linear_case  # noqa: F401  (S is the module's device fixture)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,mode", [(16, "w4a4"), (1, "w4a8")])
def test_decode_wait_runs_out_then_next_call_is_exact(S, M, mode):
    L, ol, Xq, sx, xq, osx = _linear_case(S, M, 1024, 512, 128, mode, seed=21)
    acc0, acc1 = O.linear_accum(xq, ol)
    assert S.device_error() == 0
    Y = torch.full((M, 512), 3.0, dtype=torch.bfloat16, device="cuda")
    t0 = time.perf_counter()
    st = S.lib.serq_test_decode_timeout(L.handle, S._ptr(Xq), S._ptr(sx), M, S._ptr(Y), 512, 2000, None)
    assert st == S.OK, S.lib.serq_last_error_string()
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 5.0
    assert S.device_error() == 2          # the wait for the activation copies gave up
    assert S.device_error() == 0          # reading cleared it
    assert torch.all(Y == 3.0), "a timed-out launch wrote its output"
    for algo in (S.ALGO_DECODE, S.ALGO_PREFILL_N128):
        g0, g1 = S.linear_accum(L, Xq, algo)
        Y2 = S.linear(L, Xq, sx, algo=algo)
        torch.cuda.synchronize()
        assert np.array_equal(g0.cpu().numpy(), acc0) and np.array_equal(g1.cpu().numpy(), acc1)
        assert_y_close(Y2, O.linear_epilogue(acc0, acc1, osx, ol))
    assert S.device_error() == 0


def test_timeout_hook_rejects_bad_limits(S):
    L, ol, Xq, sx, xq, osx = _linear_case(S, 4, 256, 128, 32, "w4a4", seed=22)
    Y = torch.empty((4, 128), dtype=torch.bfloat16, device="cuda")
    for us in (0, -5, 2000000):
        assert S.lib.serq_test_decode_timeout(L.handle, S._ptr(Xq), S._ptr(sx), 4, S._ptr(Y), 128, us, None) == \
            S.ERR_INVALID_ARG
