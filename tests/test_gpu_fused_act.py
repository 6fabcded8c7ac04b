"""GPU parity of serq_linear_group_act: the per-token activation quantize and
the group's products from the flattened bf16 activations.  At decode sizes
(M <= 8, K <= 4096, bf16) it is one launch whose CTAs quantize the tokens
themselves; elsewhere it runs serq_quantize_act and serq_linear_group.
Accumulators must equal the oracle's (fed the oracle's own codes of the same
activations) bit for bit, and the bf16 outputs must equal those of the two
separate calls on the same kernel bit for bit and satisfy the oracle
tolerance."""
import numpy as np
import pytest
import torch

from oracle import serq_oracle as O
from w4a4_rank_gemm_b200 import synth
from tests.gpu_support import assert_y_close, dev, dev_act

pytestmark = pytest.mark.gpu

BITS = {"w4a4": 4, "w4a8": 8}


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from w4a4_rank_gemm_b200 import serq
    assert serq.lib.serq_check_device() == serq.OK, serq.lib.serq_last_error_string()
    return serq


def _case(S, M, K, Ns, r, mode, seed, dtype=torch.bfloat16):
    wl = synth.custom_layer(M, K, Ns[0], r, mode, "bf16", seed=seed)
    inp = wl.inputs["x"]
    rng = np.random.default_rng(seed + 7)
    Ws = [wl.projections[0].W] + [synth.draw_weight(rng, K, N) for N in Ns[1:]]
    layers = S.prepare_group([dev(W) for W in Ws], dev(inp.X_calib), r, mode)
    _, _, ols = O.prepare_group(Ws, inp.X_calib, r)
    Xh = S.flatten_permute(layers[0], dev_act(inp.X, "bf16"), out_dtype=dtype)
    xh = O.flatten_permute(inp.X, ols[0].s, ols[0].pi, out_bf16=(dtype == torch.bfloat16))
    xq, osx = O.quantize_act(xh, BITS[mode])
    return layers, ols, Xh, xq, osx


# one launch: M <= 8, K <= 4096, bf16; K % 512 != 0, several layers, a
# ragged last tile, W4A8, r = 0
FUSED = [
    (8, 4096, [4096, 1024, 1024], 128, "w4a4"),
    (1, 4096, [11008, 11008], 128, "w4a4"),
    (5, 1152, [320, 96], 96, "w4a4"),
    (2, 2048, [2048], 64, "w4a4"),
    (8, 4096, [1024, 512], 128, "w4a8"),
    (3, 768, [256, 96, 160, 512], 0, "w4a8"),
]


@pytest.mark.parametrize("M,K,Ns,r,mode", FUSED)
def test_fused_decode_bit_exact(S, M, K, Ns, r, mode):
    layers, ols, Xh, xq, osx = _case(S, M, K, Ns, r, mode, seed=M + K + r)
    for algo in (S.ALGO_AUTO, S.ALGO_DECODE_STREAM):
        got = S.linear_group_act(layers, Xh, accum=True, algo=algo)
        torch.cuda.synchronize()
        for (g0, g1), ol in zip(got, ols):
            a0, a1 = O.linear_accum(xq, ol)
            assert np.array_equal(g0.cpu().numpy(), a0), f"acc0 differs (algo {algo})"
            assert np.array_equal(g1.cpu().numpy(), a1), f"acc1 differs (algo {algo})"
        Ys = S.linear_group_act(layers, Xh, algo=algo)
        Xq, sx = S.quantize_act(Xh, mode)
        Ys2 = S.linear_group(layers, Xq, sx, algo=S.ALGO_DECODE_STREAM)
        torch.cuda.synchronize()
        for Y, Y2, ol in zip(Ys, Ys2, ols):
            a0, a1 = O.linear_accum(xq, ol)
            assert torch.equal(Y, Y2), "one launch and two launches differ"
            assert_y_close(Y, O.linear_epilogue(a0, a1, osx, ol))
    assert S.device_error() == 0


# two launches: K > 4096, fp32 input, the item ring, prefill sizes
@pytest.mark.parametrize("M,K,Ns,r,mode,dtype,algo", [
    (16, 5120, [1024], 128, "w4a4", torch.bfloat16, "auto"),
    (16, 4096, [1024, 512], 128, "w4a4", torch.bfloat16, "auto"),
    (32, 2048, [2048], 64, "w4a8", torch.bfloat16, "auto"),
    (16, 1024, [512, 256], 64, "w4a4", torch.float32, "auto"),
    (8, 2048, [1024], 64, "w4a8", torch.bfloat16, "items"),
    (200, 1024, [512, 384], 64, "w4a4", torch.bfloat16, "auto"),
])
def test_two_launch_paths(S, M, K, Ns, r, mode, dtype, algo):
    layers, ols, Xh, xq, osx = _case(S, M, K, Ns, r, mode, seed=3 * M + K, dtype=dtype)
    a = {"auto": S.ALGO_AUTO, "items": S.ALGO_DECODE_ITEMS}[algo]
    Xq = torch.zeros((M, K // 2 if mode == "w4a4" else K), dtype=torch.uint8, device="cuda")
    sx = torch.zeros(M, dtype=torch.float32, device="cuda")
    got = S.linear_group_act(layers, Xh, Xq=Xq, sx=sx, accum=True, algo=a)
    torch.cuda.synchronize()
    for (g0, g1), ol in zip(got, ols):
        a0, a1 = O.linear_accum(xq, ol)
        assert np.array_equal(g0.cpu().numpy(), a0) and np.array_equal(g1.cpu().numpy(), a1)
    Ys = S.linear_group_act(layers, Xh, Xq=Xq, sx=sx, algo=a)
    torch.cuda.synchronize()
    for Y, ol in zip(Ys, ols):
        a0, a1 = O.linear_accum(xq, ol)
        assert_y_close(Y, O.linear_epilogue(a0, a1, osx, ol))
    assert S.device_error() == 0
