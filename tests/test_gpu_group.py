"""GPU parity of serq_linear_group: several layers prepared together (one
smoothing vector and saliency order, so one set of activation codes) run as
one launch.  Accumulators must equal the oracle's per layer bit for bit, the
bf16 outputs must equal those of separate serq_linear_ex calls with the same
kernel bit for bit, and satisfy the oracle tolerance."""
import numpy as np
import pytest
import torch

from oracle import serq_oracle as O
from w4a4_rank_gemm_b200 import synth
from tests.gpu_support import act_bytes, assert_y_close, dev, dev_act

pytestmark = pytest.mark.gpu

BITS = {"w4a4": 4, "w4a8": 8}


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from w4a4_rank_gemm_b200 import serq
    assert serq.lib.serq_check_device() == serq.OK, serq.lib.serq_last_error_string()
    return serq


def _group_case(S, M, K, Ns, r, mode, seed):
    wl = synth.custom_layer(M, K, Ns[0], r, mode, "bf16", seed=seed)
    inp = wl.inputs["x"]
    rng = np.random.default_rng(seed + 101)
    Ws = [wl.projections[0].W] + [synth.draw_weight(rng, K, N) for N in Ns[1:]]
    layers = S.prepare_group([dev(W) for W in Ws], dev(inp.X_calib), r, mode)
    _, _, olayers = O.prepare_group(Ws, inp.X_calib, r)
    ol0 = olayers[0]
    Xh = S.flatten_permute(layers[0], dev_act(inp.X, "bf16"), out_dtype=torch.bfloat16)
    Xq, sx = S.quantize_act(Xh, mode)
    xq, osx = O.quantize_act(O.flatten_permute(inp.X, ol0.s, ol0.pi, out_bf16=True), BITS[mode])
    assert np.array_equal(Xq.cpu().numpy(), act_bytes(xq, BITS[mode]))
    return layers, olayers, Xq, sx, xq, osx


GROUPS = [
    # M, K, Ns, r, mode
    (300, 512, [256, 128, 384], 64, "w4a4"),        # q/k/v-like, ragged M
    (130, 1152, [320, 96], 96, "w4a4"),             # ragged N in both layers, K % 256 != 0
    (2100, 384, [1024, 3200, 512, 256], 32, "w4a4"),  # four layers, several tiles per CTA
    (257, 640, [512, 384, 256], 128, "w4a8"),
    (700, 256, [1024, 1024], 0, "w4a8"),            # no residual
]


@pytest.mark.parametrize("M,K,Ns,r,mode", GROUPS)
def test_group_accum_bit_exact(S, M, K, Ns, r, mode):
    layers, olayers, Xq, sx, xq, osx = _group_case(S, M, K, Ns, r, mode, seed=M + K)
    want = [O.linear_accum(xq, ol) for ol in olayers]
    for algo in (S.ALGO_AUTO, S.ALGO_PREFILL_N128, S.ALGO_PREFILL_N256, S.ALGO_PREFILL_PAIR_N256):
        got = S.linear_group(layers, Xq, accum=True, algo=algo)
        torch.cuda.synchronize()
        for l, ((g0, g1), (a0, a1)) in enumerate(zip(got, want)):
            assert np.array_equal(g0.cpu().numpy(), a0), f"acc0 of layer {l} differs (algo {algo})"
            assert np.array_equal(g1.cpu().numpy(), a1), f"acc1 of layer {l} differs (algo {algo})"
    assert S.device_error() == 0


@pytest.mark.parametrize("M,K,Ns,r,mode", GROUPS)
def test_group_output_matches_single_calls(S, M, K, Ns, r, mode):
    layers, olayers, Xq, sx, xq, osx = _group_case(S, M, K, Ns, r, mode, seed=M + 2 * K)
    for algo in (S.ALGO_PREFILL_N128, S.ALGO_PREFILL_N256, S.ALGO_PREFILL_PAIR_N256):
        Ys = S.linear_group(layers, Xq, sx, algo=algo)
        singles = [S.linear(L, Xq, sx, algo=algo) for L in layers]
        torch.cuda.synchronize()
        for l, (Y, Y1, ol) in enumerate(zip(Ys, singles, olayers)):
            assert torch.equal(Y.view(torch.int16), Y1.view(torch.int16)), f"layer {l} differs (algo {algo})"
            assert_y_close(Y, O.linear_epilogue(*O.linear_accum(xq, ol), osx, ol))


def test_group_strided_outputs_into_one_buffer(S):
    """q/k/v written side by side into one M x (Nq+Nk+Nv) buffer."""
    M, K, Ns = 333, 512, [256, 128, 128]
    layers, olayers, Xq, sx, xq, osx = _group_case(S, M, K, Ns, 64, "w4a4", seed=11)
    big = torch.full((M, sum(Ns) + 16), 5.0, dtype=torch.bfloat16, device="cuda")
    offs = np.concatenate([[0], np.cumsum(Ns)])
    Ys = [big[:, offs[l]:offs[l + 1]] for l in range(len(Ns))]
    S.linear_group(layers, Xq, sx, Ys=Ys)
    torch.cuda.synchronize()
    for Y, ol in zip(Ys, olayers):
        assert_y_close(Y, O.linear_epilogue(*O.linear_accum(xq, ol), osx, ol))
    assert torch.all(big[:, sum(Ns):] == 5.0)


DECODE_GROUPS = [
    # M, K, Ns, r, mode
    (1, 1024, [512, 256, 256], 128, "w4a4"),
    (7, 1024, [512, 256, 256], 128, "w4a4"),
    (16, 1024, [512, 256, 256], 128, "w4a4"),
    (32, 1024, [512, 256, 256], 128, "w4a4"),
    (16, 768, [256, 96, 160, 512], 64, "w4a4"),   # four layers (the most a group takes)
    (1, 512, [384, 128], 0, "w4a4"),              # rank 0: no compensator is read
    (16, 512, [384, 128], 0, "w4a8"),
    (1, 1024, [512, 128, 128], 128, "w4a8"),
    (32, 640, [256, 128, 96, 64], 160, "w4a8"),   # four layers, rank padded to 192
]


@pytest.mark.parametrize("M,K,Ns,r,mode", DECODE_GROUPS)
def test_group_decode_sizes(S, M, K, Ns, r, mode):
    """Decode-sized groups: the mma.sync decode kernels run the whole group as
    one launch (streaming kernel and item ring), DECODE_TC one launch per
    layer; accumulators bit-exact, outputs within tolerance and equal to the
    single-layer calls of the same kernel."""
    layers, olayers, Xq, sx, xq, osx = _group_case(S, M, K, Ns, r, mode, seed=M + 3 * K + r)
    want = [O.linear_accum(xq, ol) for ol in olayers]
    for algo in (S.ALGO_AUTO, S.ALGO_DECODE, S.ALGO_DECODE_ITEMS, S.ALGO_DECODE_STREAM, S.ALGO_DECODE_TC):
        got = S.linear_group(layers, Xq, accum=True, algo=algo)
        Ys = S.linear_group(layers, Xq, sx, algo=algo)
        singles = [S.linear(L, Xq, sx, algo=algo) for L in layers]
        torch.cuda.synchronize()
        for l, ((g0, g1), Y, Y1, (a0, a1), ol) in enumerate(zip(got, Ys, singles, want, olayers)):
            assert np.array_equal(g0.cpu().numpy(), a0), f"acc0 of layer {l} differs (algo {algo})"
            assert np.array_equal(g1.cpu().numpy(), a1), f"acc1 of layer {l} differs (algo {algo})"
            assert torch.equal(Y.view(torch.int16), Y1.view(torch.int16)), f"layer {l} differs (algo {algo})"
            assert_y_close(Y, O.linear_epilogue(a0, a1, osx, ol))
    assert S.device_error() == 0


@pytest.mark.parametrize("M,mode", [(1, "w4a4"), (16, "w4a4"), (32, "w4a8")])
def test_group_decode_strided_outputs_into_one_buffer(S, M, mode):
    """Decode groups written side by side into one M x (sum N + 16) buffer:
    every layer writes its own columns at the shared row stride only."""
    Ns = [256, 128, 96]
    layers, olayers, Xq, sx, xq, osx = _group_case(S, M, 512, Ns, 64, mode, seed=40 + M)
    offs = np.concatenate([[0], np.cumsum(Ns)])
    for algo in (S.ALGO_DECODE, S.ALGO_DECODE_ITEMS, S.ALGO_DECODE_STREAM):
        big = torch.full((M, sum(Ns) + 16), 5.0, dtype=torch.bfloat16, device="cuda")
        Ys = [big[:, offs[l]:offs[l + 1]] for l in range(len(Ns))]
        S.linear_group(layers, Xq, sx, Ys=Ys, algo=algo)
        torch.cuda.synchronize()
        for Y, ol in zip(Ys, olayers):
            assert_y_close(Y, O.linear_epilogue(*O.linear_accum(xq, ol), osx, ol))
        assert torch.all(big[:, sum(Ns):] == 5.0), f"algo {algo} wrote past the last layer"


def test_llama2_7b_qkv_group_sampled(S):
    """The Llama-2-7B attention input's three projections at M = 2048 as one
    launch (the bench's call); oracle on sampled rows."""
    wl = synth.llama2_7b(only=["q_proj", "k_proj", "v_proj"])
    inp = wl.inputs["attn_in"]
    Ws = [p.W for p in wl.projections]
    layers = S.prepare_group([dev(W) for W in Ws], dev(inp.X_calib), wl.rank, "w4a4")
    _, _, olayers = O.prepare_group(Ws, inp.X_calib, wl.rank)
    Xh = S.flatten_permute(layers[0], dev_act(inp.X, "bf16"), out_dtype=torch.bfloat16)
    Xq, sx = S.quantize_act(Xh, "w4a4")
    Ys = S.linear_group(layers, Xq, sx)
    accs = S.linear_group(layers, Xq, accum=True)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([[0, 255, 256, 2047], np.random.default_rng(3).choice(2048, 20, replace=False)]))
    ol0 = olayers[0]
    xq, osx = O.quantize_act(O.flatten_permute(inp.X[rows], ol0.s, ol0.pi, True), 4)
    ridx = torch.from_numpy(rows).cuda()
    for Y, (g0, g1), ol in zip(Ys, accs, olayers):
        a0, a1 = O.linear_accum(xq, ol)
        assert np.array_equal(g0.cpu().numpy()[rows], a0) and np.array_equal(g1.cpu().numpy()[rows], a1)
        assert_y_close(Y[ridx], O.linear_epilogue(a0, a1, osx, ol))


def test_group_rejects_mismatched_layers(S):
    a = synth.custom_layer(8, 256, 128, 16, "w4a4", "bf16", seed=3)
    b = synth.custom_layer(8, 512, 128, 16, "w4a4", "bf16", seed=4)
    (La,) = S.prepare_group([dev(a.projections[0].W)], dev(a.inputs["x"].X_calib), 16, "w4a4")
    (Lb,) = S.prepare_group([dev(b.projections[0].W)], dev(b.inputs["x"].X_calib), 16, "w4a4")
    (Lc,) = S.prepare_group([dev(a.projections[0].W)], dev(a.inputs["x"].X_calib), 64, "w4a4")
    Xq = torch.zeros((300, 128), dtype=torch.uint8, device="cuda")
    sx = torch.ones(300, device="cuda")
    with pytest.raises(S.SerqError, match="differs from layer 0"):
        S.linear_group([La, Lb], Xq, sx)
    with pytest.raises(S.SerqError, match="differs from layer 0"):
        S.linear_group([La, Lc], Xq, sx)
    with pytest.raises(S.SerqError, match="group of 5 layers"):
        S.linear_group([La] * 5, Xq, sx)
    with pytest.raises(S.SerqError, match="group of 0 layers"):
        S.linear_group([], Xq, sx)
