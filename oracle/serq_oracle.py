"""CPU oracle for the SERQ quantized linear -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg may import this module.  The product path (libserq and its
Python binding) never calls it, and it shares no code with that path.

It restates, step by step and in plain numpy, what the SERQ pages say the
method computes:

* "SERQ: Saliency-Aware Low-Rank Error Reconstruction for LLM Quantization",
  papernotes.org ICLR 2026 notes (cited below as [notes]), sections
  "core idea", "method / overall framework", key designs 1-3;
* the gist.science (de) technical summary, section 2 "Methodik" A-C
  (cited as [gist-de]);
* the gist.science (ja) technical summary, section 2 "proposed method" and
  "computation flow" (cited as [gist-ja]);
* the AI Radio episode transcript on SERQ (cited as [radio]).

Where the pages leave a step open, the reading taken is stated beside it.

Precision.  Decisions that turn floats into integers (smoothing scales,
saliency order, quantization codes, the compensator) are taken in IEEE fp32
with one rounding per operation (numpy float32 arithmetic, no fused
multiply-add), because that is the precision of the device kernels and
identical decisions are required.  Everything after the integer GEMM (the
dequantizing epilogue) is computed in fp64.  Integer products are exact: the
matmul of small integer codes is done by BLAS in fp64, whose sums stay far
below 2^53 and are therefore exact integers.
"""
from __future__ import annotations

import numpy as np

F32 = np.float32
QMAX = {4: 7, 8: 127}   # symmetric ranges: int4 [-7, 7], int8 [-127, 127]
SMOOTH_FLOOR = F32(1e-5)


# ---------------------------------------------------------------------------
# bf16 rounding of an fp32 value (storage of the flattened activations)
# ---------------------------------------------------------------------------
def to_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp32 -> bf16 (nearest, ties to even) and return it as fp32."""
    x = np.ascontiguousarray(x, dtype=F32)
    bits = x.view(np.uint32).astype(np.uint64)
    lsb = (bits >> np.uint64(16)) & np.uint64(1)
    r = ((bits + np.uint64(0x7FFF) + lsb) >> np.uint64(16)) << np.uint64(16)
    return r.astype(np.uint32).view(F32)


# ---------------------------------------------------------------------------
# Step 1 -- static activation flattening  ([notes] key design 1; [gist-de] 2A;
# [radio]).  Y = X W = (X diag(s)^-1)(diag(s) W).  SmoothQuant's static
# per-input-channel scale with migration strength alpha:
#     s_j = max|X_:,j|^alpha / max|W_j,:|^(1 - alpha)
# Reading: the pages name SmoothQuant's static scale without a formula; the
# default alpha = 1/2 form (s_j = sqrt(max|X_j|) / sqrt(max|W_j|)) and a 1e-5
# floor on both maxima are taken.  At alpha = 1/2 the two square roots and
# the division are single fp32 operations; any other alpha is evaluated in
# fp64 (two powers and a division) and rounded to fp32 once.  The row maxima
# of W run over every weight that consumes the same activation (q/k/v share
# one input, gate/up share one), so one s serves the whole group.
# ---------------------------------------------------------------------------
def weight_row_amax(weights) -> np.ndarray:
    """max_n |W_jn| over every weight of a group (unfloored)."""
    if isinstance(weights, np.ndarray):
        weights = [weights]
    return np.max(np.stack([np.max(np.abs(np.asarray(W, dtype=F32)), axis=1)
                            for W in weights]), axis=0).astype(F32)


def smooth_scales(X_calib: np.ndarray, weights, alpha: float = 0.5) -> np.ndarray:
    amax_x = np.max(np.abs(np.asarray(X_calib, dtype=F32)), axis=0)
    amax_w = weight_row_amax(weights)
    ax = np.maximum(amax_x, SMOOTH_FLOOR)
    aw = np.maximum(amax_w, SMOOTH_FLOOR)
    a = float(F32(alpha))
    if a == 0.5:
        return (np.sqrt(ax) / np.sqrt(aw)).astype(F32)
    num = np.power(ax.astype(np.float64), a)
    den = np.power(aw.astype(np.float64), 1.0 - a)
    return (num / den).astype(F32)


# ---------------------------------------------------------------------------
# Step 2 -- saliency ranking ([notes] key design 2: after flattening, the
# salient rows of the folded weight are identified directly by their scale;
# [gist-de] 2B: by the activations' scale factors).  Reading: "scale" is s_j
# (metric 0, the default); metric 1 ranks by the folded row's absolute
# maximum s_j * max_n |W_jn| (one fp32 multiply), the other plain reading of
# "the salient rows of the folded weight".  Rows are ordered by descending
# key, ties kept in channel order (stable).  P maps position i -> original
# channel pi[i].
# ---------------------------------------------------------------------------
SALIENCY_SCALE, SALIENCY_ROW_ABSMAX = 0, 1


def saliency_key(s: np.ndarray, weights, metric: int = SALIENCY_SCALE) -> np.ndarray:
    s = np.asarray(s, dtype=F32)
    if metric == SALIENCY_SCALE:
        return s
    if metric == SALIENCY_ROW_ABSMAX:
        return (s * weight_row_amax(weights)).astype(F32)
    raise ValueError(f"unknown saliency metric {metric}")


def saliency_perm(s: np.ndarray) -> np.ndarray:
    return np.argsort(-np.asarray(s, dtype=np.float64), kind="stable").astype(np.int32)


# ---------------------------------------------------------------------------
# Step 3 -- fold and permute: W_hat = P diag(s) W = [W~_s ; W~_r]
# ([notes] key design 2; [radio] identity X diag(s^-1) P^-1 P diag(s) W).
# ---------------------------------------------------------------------------
def fold_weight(W: np.ndarray, s: np.ndarray, pi: np.ndarray) -> np.ndarray:
    W = np.asarray(W, dtype=F32)
    return (s[pi][:, None].astype(F32) * W[pi, :]).astype(F32)


def flatten_permute(X: np.ndarray, s: np.ndarray, pi: np.ndarray,
                    out_bf16: bool) -> np.ndarray:
    """X_hat = X diag(s^-1) P^-1: column i is X[:, pi[i]] / s[pi[i]] (fp32
    divide), stored as bf16 when the activations are bf16."""
    X = np.asarray(X, dtype=F32)
    xh = (X[:, pi] / s[pi][None, :].astype(F32)).astype(F32)
    return to_bf16(xh) if out_bf16 else xh


# ---------------------------------------------------------------------------
# Quantizer Q(.) -- symmetric round-to-nearest.  The pages fix only "INT4"
# (W4A4) / "INT8" activations for W4A8 ([notes] key design 2, main table;
# [gist-de] 2B "RTN").  Reading: scales are per output channel for weights and
# per token for activations; codes lie in [-Q, Q] (no -Q-1); the code is
# rint(x * (Q / amax)) with ties to even, clamped; the scale is amax / Q; an
# all-zero group gets scale 0 and codes 0.
# ---------------------------------------------------------------------------
def quantize_groups(X: np.ndarray, bits: int, axis: int):
    """Quantize along ``axis`` (each slice along the other axis is a group).

    Returns (codes int8, scale fp32)."""
    Q = F32(QMAX[bits])
    X = np.asarray(X, dtype=F32)
    amax = np.max(np.abs(X), axis=axis, keepdims=True).astype(F32)
    nz = amax > 0
    inv = np.where(nz, Q / np.where(nz, amax, F32(1)), F32(0)).astype(F32)
    prod = (X * inv).astype(F32)
    q = np.clip(np.rint(prod), -Q, Q).astype(np.int8)
    scale = (amax / Q).astype(F32)
    return q, np.squeeze(scale, axis=axis)


def quantize_weight(W_hat: np.ndarray, bits: int = 4):
    """Per-output-channel (column of the K x N weight) quantization."""
    return quantize_groups(W_hat, bits, axis=0)


def quantize_act(X_hat: np.ndarray, bits: int):
    """Per-token (row) quantization of the flattened, permuted activations.

    The residual input X~_{s,q} is the first r columns of the same codes with
    the same per-token scale ([notes] key design 2: no intermediate
    quantization; [gist-ja] computation flow X_q W_q + X_{s,q} R_q)."""
    return quantize_groups(X_hat, bits, axis=1)


# ---------------------------------------------------------------------------
# Compensator R = W~_s - Q(W~_s), r x d_out, itself quantized
# ([notes] core idea and key design 2; [radio] "R r by d").
# Reading: Q(W~_s) is the main path's own dequantized salient rows, so that
# Q(W_hat) + [R; 0] reconstructs W_hat exactly when R is kept in full
# precision.  The dequantized weight is code * scale in fp32 and the
# difference is one fp32 subtraction.
# ---------------------------------------------------------------------------
def compensator(W_hat: np.ndarray, q_w: np.ndarray, s_w: np.ndarray, r: int) -> np.ndarray:
    deq = (q_w[:r, :].astype(F32) * s_w[None, :].astype(F32)).astype(F32)
    return (np.asarray(W_hat[:r, :], dtype=F32) - deq).astype(F32)


# ---------------------------------------------------------------------------
# Packing (storage format, not part of the method: the pages fix only that
# codes are 4-bit).  Two's-complement nibbles; every run of 32 consecutive
# codes of a row occupies 16 bytes, byte j holding code j of the run in its
# low nibble and code j + 16 in its high nibble.  Rows are the N x K (output
# channel major) weight / compensator and the M x K activations.
# ---------------------------------------------------------------------------
def pack_int4_rows(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, dtype=np.int16)
    L = c.shape[-1]
    assert L % 32 == 0, "packed rows hold whole runs of 32 codes"
    blk = c.reshape(c.shape[:-1] + (L // 32, 2, 16))
    lo = (blk[..., 0, :] & 0xF).astype(np.uint8)
    hi = (blk[..., 1, :] & 0xF).astype(np.uint8)
    return (lo | (hi << 4)).reshape(c.shape[:-1] + (L // 2,)).astype(np.uint8)


def unpack_int4_rows(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    B = p.shape[-1]
    assert B % 16 == 0
    blk = p.reshape(p.shape[:-1] + (B // 16, 16))
    lo = (blk & 0xF).astype(np.int16)
    hi = (blk >> 4).astype(np.int16)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.stack([lo, hi], axis=-2)            # (..., B/16, 2, 16)
    return out.reshape(p.shape[:-1] + (B * 2,)).astype(np.int8)


# ---------------------------------------------------------------------------
# Offline preparation of one weight (or a group sharing one input).
# ---------------------------------------------------------------------------
class PreparedLayer:
    def __init__(self, s, pi, W_hat, q_w, s_w, R, q_r, s_r, r):
        self.s, self.pi, self.W_hat = s, pi, W_hat
        self.q_w, self.s_w = q_w, s_w          # K x N codes, N scales
        self.R, self.q_r, self.s_r = R, q_r, s_r   # r x N
        self.r = r

    @property
    def K(self):
        return self.q_w.shape[0]

    @property
    def N(self):
        return self.q_w.shape[1]


def fold_output_columns(W: np.ndarray, out_perm=None, out_div=None) -> np.ndarray:
    """Propagate the next layer's permutation (and, where the next layer's
    smoothing divisor can pass through, its scale) into this weight's output
    columns ([notes] key design 3: down_proj's P4 moves into the gate/up
    columns; [gist-de] 2C).  Column i of the result is W[:, P[i]] / d[P[i]]."""
    W = np.asarray(W, dtype=F32)
    N = W.shape[1]
    P = np.arange(N) if out_perm is None else np.asarray(out_perm, dtype=np.int64)
    out = W[:, P]
    if out_div is not None:
        out = (out / np.asarray(out_div, dtype=F32)[P][None, :]).astype(F32)
    return out.astype(F32)


def prepare_group(weights, X_calib, r: int, w_bits: int = 4, alpha: float = 0.5,
                  saliency: int = SALIENCY_SCALE):
    """SERQ offline stage for the weights that consume one activation.

    Returns (s, pi, [PreparedLayer per weight])."""
    if isinstance(weights, np.ndarray):
        weights = [weights]
    s = smooth_scales(X_calib, weights, alpha)
    pi = saliency_perm(saliency_key(s, weights, saliency))
    layers = []
    for W in weights:
        W_hat = fold_weight(W, s, pi)
        q_w, s_w = quantize_weight(W_hat, w_bits)
        if r > 0:
            R = compensator(W_hat, q_w, s_w, r)
            q_r, s_r = quantize_weight(R, w_bits)
        else:
            R = np.zeros((0, W.shape[1]), F32)
            q_r = np.zeros((0, W.shape[1]), np.int8)
            s_r = np.zeros(W.shape[1], F32)
        layers.append(PreparedLayer(s, pi, W_hat, q_w, s_w, R, q_r, s_r, r))
    return s, pi, layers


def prepare(W, X_calib, r: int, w_bits: int = 4, alpha: float = 0.5,
            saliency: int = SALIENCY_SCALE) -> PreparedLayer:
    return prepare_group([W], X_calib, r, w_bits, alpha, saliency)[2][0]


# ---------------------------------------------------------------------------
# The quantized linear  Y = X^_q W^_q + X~_{s,q} Q(R)
# ([notes] key design 2; [gist-de] 2B formula; [gist-ja] computation flow).
# acc0 = sum_k Xq[m,k] Wq[k,n] over all K; acc1 = sum_{k<r} Xq[m,k] Rq[k,n];
# Y = sx[m] * (sw[n] * acc0 + sR[n] * acc1).  P acts on the input dimension
# only, so the output columns keep their original order.
# ---------------------------------------------------------------------------
def int_matmul(a_codes: np.ndarray, b_codes: np.ndarray) -> np.ndarray:
    """Exact integer product of small-integer code matrices (a: M x K, b: K x N)."""
    prod = np.asarray(a_codes, np.float64) @ np.asarray(b_codes, np.float64)
    return np.rint(prod).astype(np.int64)


def linear_accum(xq: np.ndarray, layer: PreparedLayer):
    acc0 = int_matmul(xq, layer.q_w)
    if layer.r > 0:
        acc1 = int_matmul(xq[:, :layer.r], layer.q_r)
    else:
        acc1 = np.zeros_like(acc0)
    return acc0, acc1


def linear_epilogue(acc0, acc1, sx, layer: PreparedLayer) -> np.ndarray:
    sx = np.asarray(sx, np.float64)[:, None]
    sw = np.asarray(layer.s_w, np.float64)[None, :]
    sr = np.asarray(layer.s_r, np.float64)[None, :]
    return sx * (sw * np.asarray(acc0, np.float64) + sr * np.asarray(acc1, np.float64))


def linear(X_hat: np.ndarray, layer: PreparedLayer, a_bits: int = 4):
    """Quantize the activations, then the two-accumulator integer GEMM and
    its epilogue.  Returns (Y fp64, xq, sx, acc0, acc1)."""
    xq, sx = quantize_act(X_hat, a_bits)
    acc0, acc1 = linear_accum(xq, layer)
    return linear_epilogue(acc0, acc1, sx, layer), xq, sx, acc0, acc1


def dequant_weight(layer: PreparedLayer, with_residual: bool = True) -> np.ndarray:
    """fp64 effective weight Q(W_hat) + [Q(R); 0] (what the GEMM applies)."""
    Wd = layer.q_w.astype(np.float64) * layer.s_w.astype(np.float64)[None, :]
    if with_residual and layer.r > 0:
        Wd[:layer.r] += layer.q_r.astype(np.float64) * layer.s_r.astype(np.float64)[None, :]
    return Wd


# ---------------------------------------------------------------------------
# SiLU on fp32, written out so that its value is fixed bit for bit:
#   silu(g) = g / (1 + e^{-g})
# e^x follows Cody & Waite's argument reduction (x = k ln2 + r with ln2 split
# in two parts so that k*C1 is exact), a degree-7 Taylor polynomial for e^r on
# |r| <= ln2/2 evaluated by Horner's rule with separate fp32 multiply and add,
# and an exact scaling by 2^k.  Beyond |x| > 88 the result saturates to +inf
# (x > 88) or 0 (x < -88).
# ---------------------------------------------------------------------------
LN2_HI = F32(0.693359375)                 # 355/512: 9 significant bits
LN2_LO = F32(np.log(2.0) - 0.693359375)  # ln 2 - LN2_HI, rounded to fp32
LOG2E = F32(1.44269504088896341)
TAYLOR = [F32(1.0 / f) for f in (5040.0, 720.0, 120.0, 24.0, 6.0, 2.0, 1.0, 1.0)]


def exp_f32(x: np.ndarray) -> np.ndarray:
    x = np.asarray(x, dtype=F32)
    xc = np.clip(x, F32(-88.0), F32(88.0))
    k = np.rint((xc * LOG2E).astype(F32)).astype(F32)
    r = ((xc - (k * LN2_HI).astype(F32)).astype(F32) - (k * LN2_LO).astype(F32)).astype(F32)
    p = np.full_like(r, TAYLOR[0])
    for c in TAYLOR[1:]:
        p = ((p * r).astype(F32) + c).astype(F32)
    e = np.ldexp(p, k.astype(np.int32)).astype(F32)
    e = np.where(x > F32(88.0), F32(np.inf), e)
    e = np.where(x < F32(-88.0), F32(0.0), e)
    return e.astype(F32)


def silu_mul_f32(g: np.ndarray, u: np.ndarray) -> np.ndarray:
    """h = silu(g) * u in fp32 (g, u are the bf16 outputs of gate/up)."""
    g = np.asarray(g, F32)
    u = np.asarray(u, F32)
    den = (F32(1.0) + exp_f32(-g)).astype(F32)
    with np.errstate(over="ignore", invalid="ignore"):
        sg = (g / den).astype(F32)
    return (sg * u).astype(F32)


# ---------------------------------------------------------------------------
# MLP block with offline permutation propagation ([notes] key design 3:
# down_proj's order P4 is propagated into the gate/up weight columns so the
# intermediate arrives already permuted).  Reading: the down_proj smoothing
# divisor s4 is folded into up_proj's columns only (silu is not homogeneous,
# so it cannot pass through gate).
# ---------------------------------------------------------------------------
def prepare_mlp(Wg, Wu, Wd, X_calib, H_calib, r: int):
    s4, pi4, (down,) = prepare_group([Wd], H_calib, r)
    Wg_f = fold_output_columns(Wg, pi4, None)
    Wu_f = fold_output_columns(Wu, pi4, s4)
    s_gu, pi_gu, (gate, up) = prepare_group([Wg_f, Wu_f], X_calib, r)
    return dict(s_gu=s_gu, pi_gu=pi_gu, gate=gate, up=up, s4=s4, pi4=pi4, down=down)


def mlp_forward(X: np.ndarray, prep, a_bits: int = 4):
    """Folded chain: X -> X^ (gate/up order) -> gate, up (bf16 outputs, already
    in P4 order) -> h = silu(g) u -> quantize -> down.  Returns a dict with the
    intermediates."""
    xh = flatten_permute(X, prep["s_gu"], prep["pi_gu"], out_bf16=True)
    g, xq, sx, _, _ = linear(xh, prep["gate"], a_bits)
    u, _, _, _, _ = linear(xh, prep["up"], a_bits)
    g16 = to_bf16(g.astype(F32))
    u16 = to_bf16(u.astype(F32))
    h = silu_mul_f32(g16, u16)
    y, hq, hsx, acc0, acc1 = linear(h, prep["down"], a_bits)
    return dict(xh=xh, g=g16, u=u16, h=h, hq=hq, hsx=hsx, y=y)
