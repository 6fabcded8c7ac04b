"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the
same seeded inputs.  Integer and byte results must be bit-exact (packed
weights, scales, permutation, activation codes, int32 accumulators); the bf16
output must satisfy |y - y_ref| <= 1e-2 * max(|y_ref|, 1e-3) against the
oracle's fp64 epilogue."""
import numpy as np
import pytest
import torch

from oracle import serq_oracle as O
from w4a4_rank_gemm_b200 import synth
from tests.gpu_support import (act_bytes, assert_y_close, bits, dev, dev_act, expected_packed)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from w4a4_rank_gemm_b200 import serq  # raises if libserq.so is missing
    assert serq.lib.serq_check_device() == serq.OK, serq.lib.serq_last_error_string()
    return serq


BITS = {"w4a4": 4, "w4a8": 8}


def _prepare_both(S, weights, Xc, r, mode):
    layers = S.prepare_group([dev(W) for W in weights], dev(Xc), r, mode)
    _, _, olayers = O.prepare_group(weights, Xc, r)
    return layers, olayers


def _check_prepared(layer, ol):
    got = layer.get_packed()
    wq, rq = expected_packed(ol)
    assert np.array_equal(got["perm"], ol.pi), "saliency order differs"
    assert np.array_equal(bits(got["smooth"]), bits(ol.s)), "smoothing scales differ"
    assert np.array_equal(bits(got["sw"]), bits(ol.s_w)), "weight scales differ"
    assert np.array_equal(got["wq"], wq), "packed weight codes differ"
    if ol.r:
        assert np.array_equal(bits(got["sr"]), bits(ol.s_r)), "compensator scales differ"
        assert np.array_equal(got["rq"], rq), "packed compensator codes differ"
    else:
        assert np.all(got["sr"] == 0)


def _gpu_act(S, layer, X, act_dtype, mode):
    Xd = dev_act(X, act_dtype)
    Xh = S.flatten_permute(layer, Xd, out_dtype=torch.bfloat16 if act_dtype == "bf16" else torch.float32)
    Xq, sx = S.quantize_act(Xh, mode)
    return Xh, Xq, sx


def _oracle_act(ol, X, act_dtype, mode):
    xh = O.flatten_permute(X, ol.s, ol.pi, out_bf16=(act_dtype == "bf16"))
    xq, sx = O.quantize_act(xh, BITS[mode])
    return xh, xq, sx


# ---------------------------------------------------------------- prepare
@pytest.mark.parametrize("K,Ns,r", [(256, [256], 16), (288, [96], 0), (512, [128, 384, 64], 128),
                                    (1024, [256], 160), (128, [64], 128)])
def test_prepare_bit_exact(S, K, Ns, r):
    rng = np.random.default_rng(K + r)
    Xc = rng.standard_normal((40, K)).astype(np.float32)
    Xc[:, rng.choice(K, 3, replace=False)] *= 30
    Ws = [(0.02 * rng.standard_normal((K, n))).astype(np.float32) for n in Ns]
    layers, olayers = _prepare_both(S, Ws, Xc, r, "w4a4")
    for L, ol in zip(layers, olayers):
        assert (L.K, L.N, L.rank) == (K, ol.N, r)
        _check_prepared(L, ol)


def test_prepare_with_output_fold(S):
    rng = np.random.default_rng(5)
    K, N = 256, 192
    W = (0.05 * rng.standard_normal((K, N))).astype(np.float32)
    Xc = rng.standard_normal((32, K)).astype(np.float32)
    P = rng.permutation(N).astype(np.int32)
    d = rng.uniform(0.2, 5.0, N).astype(np.float32)
    L = S.prepare(dev(W), dev(Xc), 32, "w4a4", out_perm=dev(P), out_div=dev(d))
    ol = O.prepare(O.fold_output_columns(W, P, d), Xc, 32)
    _check_prepared(L, ol)


@pytest.mark.parametrize("alpha,saliency", [(0.5, 0), (0.5, 1), (0.8, 0), (0.3, 1), (1.0, 0)])
def test_prepare_options_host_and_device_paths(S, alpha, saliency):
    """serq_prepare (host arrays, one weight), serq_prepare_shared (host
    arrays, a group) and serq_prepare_group (device arrays) with the same
    options all give the oracle's bytes and scales bit for bit."""
    rng = np.random.default_rng(int(alpha * 10) + 7 * saliency)
    K, Ns, r = 512, [256, 128], 64
    Xc = rng.standard_normal((40, K)).astype(np.float32)
    Xc[:, rng.choice(K, 5, replace=False)] *= 40
    Ws = [(0.02 * rng.standard_normal((K, n))).astype(np.float32) for n in Ns]
    Ws[0][rng.choice(K, 3, replace=False)] *= 8          # rows whose folded maximum stands out
    L1 = S.prepare_host(Ws[0], Xc, rank=r, alpha=alpha, saliency=saliency)
    _check_prepared(L1, O.prepare(Ws[0], Xc, r, alpha=alpha, saliency=saliency))
    _, _, ols = O.prepare_group(Ws, Xc, r, alpha=alpha, saliency=saliency)
    Lh = S.prepare_shared_host(Ws, Xc, rank=r, alpha=alpha, saliency=saliency)
    Ld = S.prepare_group([dev(W) for W in Ws], dev(Xc), r, "w4a4", alpha=alpha, saliency=saliency)
    for a, b, ol in zip(Lh, Ld, ols):
        _check_prepared(a, ol)
        _check_prepared(b, ol)
    perm, smooth = Lh[1].perm_smooth()
    assert np.array_equal(perm, ols[1].pi) and np.array_equal(bits(smooth), bits(ols[1].s))
    if saliency == 1:
        s_only = O.saliency_perm(ols[0].s)
        assert not np.array_equal(s_only, ols[0].pi), "the test data should tell the two metrics apart"


def test_prepare_host_with_output_fold(S):
    rng = np.random.default_rng(6)
    K, N = 256, 192
    W = (0.05 * rng.standard_normal((K, N))).astype(np.float32)
    Xc = rng.standard_normal((32, K)).astype(np.float32)
    P = rng.permutation(N).astype(np.int32)
    d = rng.uniform(0.2, 5.0, N).astype(np.float32)
    L = S.prepare_host(W, Xc, rank=32, out_perm=P, out_colscale=d)
    _check_prepared(L, O.prepare(O.fold_output_columns(W, P, d), Xc, 32))
    Ls = S.prepare_shared_host([W, W], Xc, rank=32, out_perm=[P, None], out_colscale=[d, None])
    _check_prepared(Ls[1], O.prepare_group([O.fold_output_columns(W, P, d), W], Xc, 32)[2][1])


# --------------------------------------------------- activations: quantize
@pytest.mark.parametrize("act_dtype", ["bf16", "f32"])
@pytest.mark.parametrize("mode", ["w4a4", "w4a8"])
@pytest.mark.parametrize("M,K", [(1, 256), (7, 288), (33, 1024), (130, 4096), (3, 14336)])
def test_flatten_quantize_bit_exact(S, act_dtype, mode, M, K):
    wl = synth.custom_layer(M, K, 64, 16, mode, act_dtype, seed=M * 7 + K)
    inp, W = wl.inputs["x"], wl.projections[0].W
    (L,), (ol,) = _prepare_both(S, [W], inp.X_calib, 16, mode)
    Xh, Xq, sx = _gpu_act(S, L, inp.X, act_dtype, mode)
    xh, xq, osx = _oracle_act(ol, inp.X, act_dtype, mode)
    assert np.array_equal(bits(Xh.float().cpu().numpy()), bits(xh)), "flattened activations differ"
    assert np.array_equal(Xq.cpu().numpy(), act_bytes(xq, BITS[mode])), "activation codes differ"
    assert np.array_equal(bits(sx.cpu().numpy()), bits(osx)), "activation scales differ"


def test_quantize_zero_rows_and_extremes(S):
    X = np.zeros((4, 64), np.float32)
    X[1, 5] = 3.0          # single nonzero -> +Q
    X[2] = -1.0            # constant row -> all -Q
    X[3, ::2] = 2.5
    X[3, 1::2] = -7.0
    for mode in ("w4a4", "w4a8"):
        Xq, sx = S.quantize_act(dev(X), mode)
        xq, osx = O.quantize_act(X, BITS[mode])
        assert np.array_equal(Xq.cpu().numpy(), act_bytes(xq, BITS[mode]))
        assert np.array_equal(bits(sx.cpu().numpy()), bits(osx))
        assert sx[0].item() == 0.0


# ---------------------------------------------------------------- linear
SHAPES = [
    # M, K, N, r
    (16, 256, 256, 16),     # the tiny configuration's shape
    (1, 256, 96, 16),
    (5, 288, 128, 0),
    (33, 512, 384, 128),
    (64, 1024, 256, 160),
    (128, 512, 256, 32),
    (130, 1024, 512, 128),  # ragged M tail, two N tiles
    (300, 1152, 320, 96),   # ragged M and N (N % 256 != 0), K % 128 != 0 ... K = 1152 = 9*128
    (257, 416, 256, 416),   # r = K (whole matrix compensated), K % 128 = 32
    (512, 2048, 1024, 128),
    (2100, 384, 3200, 32),  # more tiles than CTA pairs / SMs: each CTA runs several tiles
    (1100, 128, 5120, 0),   # one k step per tile, no residual, several tiles per CTA
]


def _linear_case(S, M, K, N, r, mode, act_dtype="bf16", seed=0):
    wl = synth.custom_layer(M, K, N, r, mode, act_dtype, seed=seed + M + 3 * K + 7 * N + r)
    inp, W = wl.inputs["x"], wl.projections[0].W
    (L,), (ol,) = _prepare_both(S, [W], inp.X_calib, r, mode)
    _, Xq, sx = _gpu_act(S, L, inp.X, act_dtype, mode)
    _, xq, osx = _oracle_act(ol, inp.X, act_dtype, mode)
    assert np.array_equal(Xq.cpu().numpy(), act_bytes(xq, BITS[mode]))
    return L, ol, Xq, sx, xq, osx


@pytest.mark.parametrize("mode", ["w4a4", "w4a8"])
@pytest.mark.parametrize("M,K,N,r", SHAPES)
def test_linear_accum_bit_exact(S, mode, M, K, N, r):
    L, ol, Xq, sx, xq, osx = _linear_case(S, M, K, N, r, mode)
    acc0, acc1 = O.linear_accum(xq, ol)
    algos = [S.ALGO_PREFILL_N128, S.ALGO_PREFILL_N256, S.ALGO_PREFILL_PAIR_N256] + \
        ([S.ALGO_PREFILL_PAIR_TMEM_A] if mode == "w4a4" else []) + ([S.ALGO_DECODE, S.ALGO_DECODE_ITEMS, S.ALGO_DECODE_STREAM] if M <= 64 else []) + ([S.ALGO_DECODE_TC] if M <= 32 else [])
    for algo in algos:
        g0, g1 = S.linear_accum(L, Xq, algo)
        torch.cuda.synchronize()
        assert np.array_equal(g0.cpu().numpy(), acc0), f"acc0 differs (algo {algo})"
        assert np.array_equal(g1.cpu().numpy(), acc1), f"acc1 differs (algo {algo})"
    assert S.device_error() == 0


@pytest.mark.parametrize("mode", ["w4a4", "w4a8"])
@pytest.mark.parametrize("M,K,N,r", SHAPES)
def test_linear_output_within_tolerance(S, mode, M, K, N, r):
    L, ol, Xq, sx, xq, osx = _linear_case(S, M, K, N, r, mode, seed=1)
    acc0, acc1 = O.linear_accum(xq, ol)
    y_ref = O.linear_epilogue(acc0, acc1, osx, ol)
    algos = [S.ALGO_AUTO, S.ALGO_PREFILL_N128, S.ALGO_PREFILL_N256, S.ALGO_PREFILL_PAIR_N256] + \
        ([S.ALGO_PREFILL_PAIR_TMEM_A] if mode == "w4a4" else []) + ([S.ALGO_DECODE, S.ALGO_DECODE_ITEMS, S.ALGO_DECODE_STREAM] if M <= 64 else []) + ([S.ALGO_DECODE_TC] if M <= 32 else [])
    for algo in algos:
        Y = S.linear(L, Xq, sx, algo=algo)
        torch.cuda.synchronize()
        assert_y_close(Y, y_ref)


def test_linear_strided_output(S):
    L, ol, Xq, sx, xq, osx = _linear_case(S, 40, 256, 128, 16, "w4a4")
    y_ref = O.linear_epilogue(*O.linear_accum(xq, ol), osx, ol)
    for algo in (S.ALGO_PREFILL, S.ALGO_DECODE, S.ALGO_DECODE_ITEMS, S.ALGO_DECODE_STREAM):
        big = torch.full((40, 200), 7.0, dtype=torch.bfloat16, device="cuda")
        S.linear(L, Xq, sx, Y=big[:, 8:136], algo=algo)
        torch.cuda.synchronize()
        assert_y_close(big[:, 8:136], y_ref)
        assert torch.all(big[:, :8] == 7.0) and torch.all(big[:, 136:] == 7.0)


def test_tiny_configuration_end_to_end(S):
    wl = synth.tiny()
    inp, W = wl.inputs["x"], wl.projections[0].W
    (L,), (ol,) = _prepare_both(S, [W], inp.X_calib, wl.rank, "w4a4")
    _check_prepared(L, ol)
    _, Xq, sx = _gpu_act(S, L, inp.X, "f32", "w4a4")
    y_ref, xq, osx, _, _ = O.linear(O.flatten_permute(inp.X, ol.s, ol.pi, False), ol, 4)
    assert np.array_equal(Xq.cpu().numpy(), act_bytes(xq, 4))
    for algo in (S.ALGO_AUTO, S.ALGO_PREFILL, S.ALGO_DECODE):
        Y = S.linear(L, Xq, sx, algo=algo)
        torch.cuda.synchronize()
        assert_y_close(Y, y_ref)


# -------------------------------------------------------- SiLU * mul + quant
@pytest.mark.parametrize("mode", ["w4a4", "w4a8"])
@pytest.mark.parametrize("M,F", [(3, 256), (17, 11008), (64, 14336)])
def test_silu_mul_quantize_bit_exact(S, mode, M, F):
    rng = np.random.default_rng(M + F)
    g = synth.round_to_bf16((6 * rng.standard_normal((M, F))).astype(np.float32))
    u = synth.round_to_bf16(rng.standard_normal((M, F)).astype(np.float32))
    g[0, :8] = [-100, -88.5, -87.9, 0, 88.5, 100, -20, 1e-3]   # saturation edges
    g = synth.round_to_bf16(g)
    Gd, Ud = dev_act(g, "bf16"), dev_act(u, "bf16")
    Xq, sx = S.silu_mul_quantize(Gd, Ud, mode)
    h = O.silu_mul_f32(g, u)
    xq, osx = O.quantize_act(h, BITS[mode])
    assert np.array_equal(bits(sx.cpu().numpy()), bits(osx))
    assert np.array_equal(Xq.cpu().numpy(), act_bytes(xq, BITS[mode]))


# ------------------------------------------------------------- MLP chain
def test_mlp_block_chain(S):
    """gate/up (with down_proj's order folded into their columns) -> silu*mul
    + quantize -> down, against the oracle's folded chain and against the
    oracle chain without any folding (explicit runtime permutation)."""
    blk = synth.mlp_block(M=256, K=512, F=1024, rank=64, seed=3, n_calib=128)
    r = blk.rank
    prep = O.prepare_mlp(blk.Wg, blk.Wu, blk.Wd, blk.X_calib, blk.H_calib, r)
    (Ld,) = S.prepare_group([dev(blk.Wd)], dev(blk.H_calib), r, "w4a4")
    _check_prepared(Ld, prep["down"])
    p4, s4 = Ld.perm_smooth()
    Lg, Lu = S.prepare_group([dev(blk.Wg), dev(blk.Wu)], dev(blk.X_calib), r, "w4a4",
                             out_perm=[dev(p4), dev(p4)], out_div=[None, dev(s4)])
    _check_prepared(Lg, prep["gate"])
    _check_prepared(Lu, prep["up"])
    Xh = S.flatten_permute(Lg, dev_act(blk.X, "bf16"))
    Xq, sx = S.quantize_act(Xh, "w4a4")
    G = S.linear(Lg, Xq, sx)
    U = S.linear(Lu, Xq, sx)
    Hq, hsx = S.silu_mul_quantize(G, U, "w4a4")
    Y = S.linear(Ld, Hq, hsx)
    d0, d1 = S.linear_accum(Ld, Hq)
    torch.cuda.synchronize()
    out = O.mlp_forward(blk.X, prep)
    # gate/up outputs within the bf16 tolerance
    assert_y_close(G, O.linear(out["xh"], prep["gate"])[0])
    assert_y_close(U, O.linear(out["xh"], prep["up"])[0])
    # the intermediate codes from the GPU's own g/u are bit-exact (the oracle
    # fed the same bf16 values)
    g16 = G.float().cpu().numpy()
    u16 = U.float().cpu().numpy()
    hq_own, hsx_own = O.quantize_act(O.silu_mul_f32(g16, u16), 4)
    hq = Hq.cpu().numpy()
    assert np.array_equal(hq, act_bytes(hq_own, 4))
    assert np.array_equal(bits(hsx.cpu().numpy()), bits(hsx_own))
    # down_proj on the GPU's own codes: accumulators bit-exact, the block
    # output element by element within the tolerance
    a0, a1 = O.linear_accum(hq_own, prep["down"])
    assert np.array_equal(d0.cpu().numpy(), a0) and np.array_equal(d1.cpu().numpy(), a1)
    assert_y_close(Y, O.linear_epilogue(a0, a1, hsx_own, prep["down"]))
    # against the oracle's own chain: g/u may round differently in the last
    # bf16 place (fp32 vs fp64 epilogue), which may move a few down_proj input
    # codes by one
    ref_hq = act_bytes(out["hq"], 4)
    codes_g = O.unpack_int4_rows(hq).astype(int)
    codes_o = O.unpack_int4_rows(ref_hq).astype(int)
    diff = np.abs(codes_g - codes_o)
    assert diff.max() <= 1 and diff.mean() < 1e-3
    y = Y.float().cpu().numpy().astype(np.float64)
    rel = np.linalg.norm(y - out["y"]) / np.linalg.norm(out["y"])
    assert rel < 1e-2, rel
    # against the unfolded chain (runtime permutation, no fold): same block up
    # to quantization differences
    Xd = blk.X.astype(np.float64)
    silu = lambda x: x / (1 + np.exp(-x))
    ref_fp = (silu(Xd @ blk.Wg) * (Xd @ blk.Wu)) @ blk.Wd.astype(np.float64)
    rel_fp = np.linalg.norm(y - ref_fp) / np.linalg.norm(ref_fp)
    rel_or = np.linalg.norm(out["y"] - ref_fp) / np.linalg.norm(ref_fp)
    assert abs(rel_fp - rel_or) < 0.02 and rel_fp < 0.4


# ------------------------------------------------------------ full sizes
@pytest.mark.parametrize("name", ["q_proj", "gate_proj", "down_proj"])
def test_llama2_7b_prefill_sampled(S, name):
    """Full Llama-2-7B projection at M = 2048 through serq_linear (the bench's
    call); oracle on sampled rows."""
    wl = synth.llama2_7b(only=[name])
    p = wl.projections[0]
    inp = wl.inputs[p.input]
    (L,), (ol,) = _prepare_both(S, [p.W], inp.X_calib, wl.rank, "w4a4")
    _check_prepared(L, ol)
    _, Xq, sx = _gpu_act(S, L, inp.X, "bf16", "w4a4")
    Y = S.linear(L, Xq, sx)
    acc0g, acc1g = S.linear_accum(L, Xq)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 2047], np.random.default_rng(0).choice(2048, 27, replace=False)]))
    xh = O.flatten_permute(inp.X[rows], ol.s, ol.pi, True)
    xq, osx = O.quantize_act(xh, 4)
    assert np.array_equal(Xq.cpu().numpy()[rows], act_bytes(xq, 4))
    acc0, acc1 = O.linear_accum(xq, ol)
    assert np.array_equal(acc0g.cpu().numpy()[rows], acc0)
    assert np.array_equal(acc1g.cpu().numpy()[rows], acc1)
    assert_y_close(Y[torch.from_numpy(rows).cuda()], O.linear_epilogue(acc0, acc1, osx, ol))


@pytest.mark.parametrize("names", [["gate_proj", "up_proj"], ["down_proj"], ["q_proj", "k_proj", "v_proj"]])
def test_llama3_8b_w4a8_sampled(S, names):
    """Full Llama-3-8B projections at W4A8, M = 4096, through the calls the
    bench makes (gate/up and q/k/v as one grouped launch): accumulators
    bit-exact and outputs within tolerance on sampled rows."""
    wl = synth.llama3_8b(M=4096, only=names)
    inp = wl.inputs[wl.projections[0].input]
    Ws = [p.W for p in wl.projections]
    layers, olayers = _prepare_both(S, Ws, inp.X_calib, wl.rank, "w4a8")
    for L, ol in zip(layers, olayers):
        _check_prepared(L, ol)
    _, Xq, sx = _gpu_act(S, layers[0], inp.X, "bf16", "w4a8")
    Ys = S.linear_group(layers, Xq, sx)
    accs = S.linear_group(layers, Xq, accum=True)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([[0, 255, 256, 4095], np.random.default_rng(4).choice(4096, 20, replace=False)]))
    ol0 = olayers[0]
    xq, osx = O.quantize_act(O.flatten_permute(inp.X[rows], ol0.s, ol0.pi, True), 8)
    assert np.array_equal(Xq.cpu().numpy()[rows], act_bytes(xq, 8))
    ridx = torch.from_numpy(rows).cuda()
    for Y, (g0, g1), ol in zip(Ys, accs, olayers):
        a0, a1 = O.linear_accum(xq, ol)
        assert np.array_equal(g0.cpu().numpy()[rows], a0) and np.array_equal(g1.cpu().numpy()[rows], a1)
        assert_y_close(Y[ridx], O.linear_epilogue(a0, a1, osx, ol))
    del accs, Ys


@pytest.mark.parametrize("M", [1, 4, 16])
def test_llama2_7b_decode(S, M):
    wl = synth.llama2_7b(M=M, only=["gate_proj"])
    p = wl.projections[0]
    inp = wl.inputs[p.input]
    (L,), (ol,) = _prepare_both(S, [p.W], inp.X_calib, wl.rank, "w4a4")
    _, Xq, sx = _gpu_act(S, L, inp.X, "bf16", "w4a4")
    y_ref, xq, osx, acc0, acc1 = O.linear(O.flatten_permute(inp.X, ol.s, ol.pi, True), ol, 4)
    for algo in (S.ALGO_AUTO, S.ALGO_DECODE, S.ALGO_DECODE_ITEMS, S.ALGO_DECODE_STREAM, S.ALGO_DECODE_TC):
        Y = S.linear(L, Xq, sx, algo=algo)
        g0, g1 = S.linear_accum(L, Xq, algo)
        torch.cuda.synchronize()
        assert np.array_equal(g0.cpu().numpy(), acc0) and np.array_equal(g1.cpu().numpy(), acc1), f"algo {algo}"
        assert_y_close(Y, y_ref)


@pytest.mark.parametrize("M,K,N,mode", [
    (16, 11008, 512, "w4a4"),   # item ring: activations read from L2; streaming: staged (89 KB)
    (8, 14336, 256, "w4a8"),    # item ring: a one-stage ring; streaming: 115 KB of staged activations
    (32, 11008, 256, "w4a4"),   # streaming: four token tiles next to 176 KB of activations (four warps)
    (32, 14336, 128, "w4a8"),   # too large for the streaming kernel: DECODE falls back to the item ring
    (64, 4096, 256, "w4a4"),    # four 16-token tiles
])
def test_decode_large_k(S, M, K, N, mode):
    L, ol, Xq, sx, xq, osx = _linear_case(S, M, K, N, 128, mode, seed=5)
    acc0, acc1 = O.linear_accum(xq, ol)
    for algo in [S.ALGO_DECODE, S.ALGO_DECODE_ITEMS, S.ALGO_DECODE_STREAM] + ([S.ALGO_DECODE_TC] if M <= 32 else []):
        g0, g1 = S.linear_accum(L, Xq, algo)
        Y = S.linear(L, Xq, sx, algo=algo)
        torch.cuda.synchronize()
        assert np.array_equal(g0.cpu().numpy(), acc0) and np.array_equal(g1.cpu().numpy(), acc1), f"algo {algo}"
        assert_y_close(Y, O.linear_epilogue(acc0, acc1, osx, ol))
    assert S.device_error() == 0


def test_llama3_8b_w4a8_kv_sampled(S):
    wl = synth.llama3_8b(M=4096, only=["k_proj"])
    p = wl.projections[0]
    inp = wl.inputs[p.input]
    (L,), (ol,) = _prepare_both(S, [p.W], inp.X_calib, wl.rank, "w4a8")
    _check_prepared(L, ol)
    _, Xq, sx = _gpu_act(S, L, inp.X, "bf16", "w4a8")
    Y = S.linear(L, Xq, sx)
    torch.cuda.synchronize()
    rows = np.random.default_rng(1).choice(4096, 24, replace=False)
    xq, osx = O.quantize_act(O.flatten_permute(inp.X[rows], ol.s, ol.pi, True), 8)
    acc0, acc1 = O.linear_accum(xq, ol)
    assert_y_close(Y[torch.from_numpy(rows).cuda()], O.linear_epilogue(acc0, acc1, osx, ol))


# ------------------------------------------------------------ error paths
def test_rejected_calls_launch_nothing(S):
    wl = synth.custom_layer(8, 256, 128, 16, "w4a4", "bf16", seed=9)
    (L,), _ = _prepare_both(S, [wl.projections[0].W], wl.inputs["x"].X_calib, 16, "w4a4")
    Xq = torch.zeros((100, 128), dtype=torch.uint8, device="cuda")
    sx = torch.ones(100, device="cuda")
    Y = torch.full((100, 128), 3.0, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(S.SerqError, match="decode kernel takes M"):
        S.linear(L, Xq, sx, Y=Y, algo=S.ALGO_DECODE)     # M = 100 > 64
    with pytest.raises(S.SerqError, match="16-byte aligned"):
        S.linear(L, Xq[:, 1:], sx, Y=Y)                  # misaligned activation pointer
    # ldy < N, through the raw C entry point (returns a status, raises nothing)
    assert S.lib.serq_linear(L.handle, S._ptr(Xq), S._ptr(sx), 100, S._ptr(Y), 64, None) == S.ERR_INVALID_ARG
    assert b"ldy" in S.lib.serq_last_error_string()
    torch.cuda.synchronize()
    assert torch.all(Y == 3.0)
    assert S.device_error() == 0
