"""CPU oracle for SERQ with MXFP4 codes -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may
import this module; the product path never calls it and shares no code with
it.

The SERQ pages name two 4-bit data formats the method works with, INT4 and
MXFP4 (gist.science (de) section 3, "Kompatibilität"); their Blackwell
latency figures are MXFP4, the low-rank path costing about 1% over plain
MXFP4 (same page, section 4, "Performance & Latenz"); and with R also in 4
bits the whole linear runs in 4-bit integer or MXFP4 arithmetic
(gist.science (ja) section 2, "complete low precision").  None of them
defines MXFP4.  The format
is the OCP Microscaling (MX) specification's: blocks of 32 consecutive
elements share one power-of-two scale stored as an E8M0 byte, and every
element is an FP4 E2M1 number.  Reading taken (the plainest one the pages
support): SERQ's steps stay as they are -- static flattening, saliency order,
fold, the main path's own error on the r salient rows as the compensator R,
and the residual product reusing the first r activation codes ("SERQ notes"
key designs 1-2) -- with every quantizer Q(.) replaced by MXFP4:

* weights W^ (K x N) and R (r x N): blocks of 32 along K for each output
  channel;
* activations X^ (M x K): blocks of 32 along K for each token, so the
  residual input X~_{s,q} is exactly the first r/32 blocks of the same codes
  (r a multiple of 32);
* the product Y = deq(X_q) deq(W_q) + deq(X_q[:, :r]) deq(R_q), which with
  block scales applied inside the product needs no per-channel epilogue.

Conversion of one block (OCP MX v1.0, section 6.3, and the E2M1 element
format of section 5.3.3):
  shared exponent  e = floor(log2(max_i |v_i|)) - 2   (2 = the exponent of
                   E2M1's largest normal, 6 = 1.5 * 2^2), clamped to E8M0's
                   range [-127, 127]; an all-zero block takes e = -127;
  element          t_i = v_i / 2^e rounded to the nearest E2M1 value, ties to
                   the value whose code is even, magnitudes above 6 to 6 (the
                   nearest value; the spec's saturating conversion).
Readings where the spec leaves a choice: a zero element is stored as +0
(code 0) whatever its sign; inputs are finite (the spec's NaN scale is not
produced).  The division by 2^e is exact in fp64 and, for every value whose
E2M1 rounding it can affect, in fp32 too.

Everything here is fp64 (exact for the scaling, the dequantized values and
the E2M1 decisions); the product is one fp64 matmul.
"""
from __future__ import annotations

import numpy as np

from oracle import serq_oracle as O

F32 = np.float32
BLOCK = 32
E2M1_EMAX = 2                      # exponent of the largest normal, 6 = 1.5 * 2^2
E8M0_BIAS = 127
E8M0_MIN, E8M0_MAX = -127, 127
# E2M1 magnitudes by code 0..7 (sign in bit 3): 0, 0.5 (subnormal), 1, 1.5,
# 2, 3, 4, 6
E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


# ---------------------------------------------------------------------------
# one element: nearest E2M1 value, ties to the even code
# ---------------------------------------------------------------------------
def e2m1_code(t) -> np.ndarray:
    """4-bit E2M1 code of each value of t (fp64): the code whose magnitude is
    nearest to |t|; of two equally near, the one with the even code."""
    t = np.asarray(t, dtype=np.float64)
    a = np.abs(t)
    dist = np.abs(a[..., None] - E2M1_VALUES)             # (..., 8)
    best = np.min(dist, axis=-1, keepdims=True)
    cand = dist == best
    # among the nearest, prefer an even code; codes ascend with magnitude,
    # so two nearest codes are neighbours and exactly one of them is even
    even = cand & (np.arange(8) % 2 == 0)
    mag = np.where(even.any(axis=-1), np.argmax(even, axis=-1), np.argmax(cand, axis=-1))
    sign = (t < 0) & (mag != 0)
    return (mag | (sign.astype(np.int64) << 3)).astype(np.uint8)


def e2m1_value(code) -> np.ndarray:
    c = np.asarray(code, dtype=np.int64)
    v = E2M1_VALUES[c & 7]
    return np.where(c & 8, -v, v)


# ---------------------------------------------------------------------------
# one block of 32: shared exponent and codes
# ---------------------------------------------------------------------------
def shared_exponent(amax) -> np.ndarray:
    """floor(log2(amax)) - 2 clamped to [-127, 127]; -127 for amax = 0."""
    a = np.asarray(amax, dtype=np.float64)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))             # a = f 2^ex, f in [0.5, 1)
    e = np.where(a > 0, ex - 1 - E2M1_EMAX, E8M0_MIN)
    return np.clip(e, E8M0_MIN, E8M0_MAX).astype(np.int64)


def mx_quantize(V: np.ndarray):
    """MXFP4 along the last axis (its length a multiple of 32).

    Returns (codes uint8 0..15 of V's shape, exponents int64 of shape
    V.shape[:-1] + (L/32,))."""
    V = np.asarray(V, dtype=np.float64)
    L = V.shape[-1]
    assert L % BLOCK == 0, "MXFP4 blocks are 32 elements"
    blk = V.reshape(V.shape[:-1] + (L // BLOCK, BLOCK))
    e = shared_exponent(np.max(np.abs(blk), axis=-1))
    t = blk / np.ldexp(1.0, e)[..., None]
    return e2m1_code(t).reshape(V.shape), e


def mx_dequantize(codes: np.ndarray, e: np.ndarray) -> np.ndarray:
    c = np.asarray(codes)
    L = c.shape[-1]
    v = e2m1_value(c).reshape(c.shape[:-1] + (L // BLOCK, BLOCK))
    return (v * np.ldexp(1.0, np.asarray(e))[..., None]).reshape(c.shape)


# ---------------------------------------------------------------------------
# storage (not part of the method): two codes per byte in K order, element
# 2i in the low nibble; exponents as E8M0 bytes (e + 127)
# ---------------------------------------------------------------------------
def pack_fp4_rows(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)


def unpack_fp4_rows(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


def e8m0_bytes(e: np.ndarray) -> np.ndarray:
    return (np.asarray(e, np.int64) + E8M0_BIAS).astype(np.uint8)


def scale_tile_offset(row, blk, n_blocks: int):
    """Byte offset of the E8M0 scale of (row, block) in the tiled scale
    layout the GEMM reads: 1 KB tiles of 128 rows x 8 blocks (256 elements of
    K), tiles row-major over (row / 128, block / 8), inside a tile row-major
    (8 bytes per row).  n_blocks = K / 32, a multiple of 8."""
    row = np.asarray(row, np.int64)
    blk = np.asarray(blk, np.int64)
    return ((row // 128) * (n_blocks // 8) + blk // 8) * 1024 + (row % 128) * 8 + blk % 8


def tile_scales(e: np.ndarray) -> np.ndarray:
    """E8M0 bytes of a rows x n_blocks exponent matrix in the tiled layout,
    rows padded to a multiple of 128 with zero bytes."""
    e = np.asarray(e)
    rows, nb = e.shape
    rp = (rows + 127) // 128 * 128
    out = np.zeros(rp * nb, np.uint8)
    r, b = np.meshgrid(np.arange(rows), np.arange(nb), indexing="ij")
    out[scale_tile_offset(r, b, nb)] = e8m0_bytes(e)
    return out


# ---------------------------------------------------------------------------
# SERQ with MXFP4 codes
# ---------------------------------------------------------------------------
class MXLayer:
    def __init__(self, s, pi, W_hat, q_w, e_w, R, q_r, e_r, r):
        self.s, self.pi, self.W_hat = s, pi, W_hat
        self.q_w, self.e_w = q_w, e_w        # N x K codes, N x K/32 exponents
        self.R, self.q_r, self.e_r = R, q_r, e_r   # N x r codes, N x r/32 exponents
        self.r = r

    @property
    def K(self):
        return self.q_w.shape[1]

    @property
    def N(self):
        return self.q_w.shape[0]


def prepare_from(s: np.ndarray, pi: np.ndarray, W: np.ndarray, r: int) -> MXLayer:
    """The offline stage with MXFP4 codes for a weight whose smoothing scales
    s and saliency order pi are already fixed (steps 1-2 do not depend on the
    format).  W^ = P diag(s) W as the INT4 path folds it (fp32); R = W~_s -
    deq(Q(W~_s)) on the r salient rows (one fp32 subtraction; the dequantized
    code times its power-of-two scale is exact in fp32)."""
    assert r % BLOCK == 0, "the compensator spans whole 32-element blocks"
    W_hat = O.fold_weight(W, s, pi)                       # K x N fp32
    q_w, e_w = mx_quantize(W_hat.T.astype(np.float64))    # per output channel along K
    deq = mx_dequantize(q_w[:, :r], e_w[:, :r // BLOCK]).astype(F32)   # N x r, exact
    R = (W_hat[:r, :].T.astype(F32) - deq).astype(F32)   # N x r
    if r > 0:
        q_r, e_r = mx_quantize(R.astype(np.float64))
    else:
        q_r = np.zeros((W_hat.shape[1], 0), np.uint8)
        e_r = np.zeros((W_hat.shape[1], 0), np.int64)
    return MXLayer(s, pi, W_hat, q_w, e_w, R, q_r, e_r, r)


def prepare(W: np.ndarray, X_calib: np.ndarray, r: int, alpha: float = 0.5,
            saliency: int = O.SALIENCY_SCALE) -> MXLayer:
    s = O.smooth_scales(X_calib, [W], alpha)
    pi = O.saliency_perm(O.saliency_key(s, [W], saliency))
    return prepare_from(s, pi, W, r)


def quantize_act(X_hat: np.ndarray):
    """Per token, blocks of 32 along K: (codes M x K, exponents M x K/32)."""
    return mx_quantize(np.asarray(X_hat, dtype=np.float64))


def effective_weight(layer: MXLayer, with_residual: bool = True) -> np.ndarray:
    """K x N fp64: deq(W_q) + [deq(R_q); 0] (what the product applies)."""
    Wd = mx_dequantize(layer.q_w, layer.e_w).T.copy()
    if with_residual and layer.r > 0:
        Wd[:layer.r] += mx_dequantize(layer.q_r, layer.e_r).T
    return Wd


def linear_codes(xq: np.ndarray, xe: np.ndarray, layer: MXLayer) -> np.ndarray:
    """Y = deq(X_q) deq(W_q) + deq(X_q)[:, :r] deq(R_q), fp64."""
    Xd = mx_dequantize(xq, xe)
    Y = Xd @ mx_dequantize(layer.q_w, layer.e_w).T
    if layer.r > 0:
        Y += Xd[:, :layer.r] @ mx_dequantize(layer.q_r, layer.e_r).T
    return Y


def abs_products(xq: np.ndarray, xe: np.ndarray, layer: MXLayer) -> np.ndarray:
    """sum over the reduction of |x_k w_k| (both products), fp64: the scale
    of an accumulation-order error bound."""
    Xd = np.abs(mx_dequantize(xq, xe))
    S = Xd @ np.abs(mx_dequantize(layer.q_w, layer.e_w)).T
    if layer.r > 0:
        S += Xd[:, :layer.r] @ np.abs(mx_dequantize(layer.q_r, layer.e_r)).T
    return S


def linear(X_hat: np.ndarray, layer: MXLayer):
    """Quantize the activations, then the product.  Returns (Y, xq, xe)."""
    xq, xe = quantize_act(X_hat)
    return linear_codes(xq, xe, layer), xq, xe
