"""CPU oracle for the two-factor low-rank error reconstruction that SERQ is
compared against (L2QER) -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may
import this module; the product path never calls it.

What the pages say the comparator computes:

* the quantization error of the weight is approximated by a LoRA-style pair
  of low-rank factors, L1 L2 ~ W - Q(W) (papernotes.org ICLR 2026 notes on
  SERQ, "field status"), extracted by SVD (same notes, "vs L2QER": "uses SVD
  to extract two serial factors"), in a space scaled by a diagonal matrix S
  computed from the calibration activations (the SRR notes on the same site,
  "field status": truncated SVD of S W in the scaled space, as in LQER);
* at inference the two factors are applied one after the other, and the
  intermediate X_q L1 must be quantized on the fly before the second product
  (SERQ notes, "pain points"); the gist.science (ja) summary writes the flow
  as X_q W_q + Q(X_q L_{1,q}) L_{2,q} ("computation flow").

Readings taken where the pages are silent:

1. The comparator works on SERQ's own flattened, permuted weight W^ and
   activations X^ (same smoothing and order), so that its main product is
   bit-identical to SERQ's and only the error path differs.
2. S_j = mean_t |X^_tj| over the calibration tokens (the activation
   statistic of LQER's scaled SVD), floored at 1e-5; the SVD is of S E with
   E = W^ - Q(W^) (fp64); L1 = S^-1 U_r (K x r) and L2 = Sigma_r V_r^T
   (r x N).
3. L1 and L2 are quantized like SERQ's weights: per output channel
   (column) symmetric RTN with 4-bit codes.  The notes say L2QER keeps its
   factors in 8 bits; 4 bits is the cheaper choice for the comparator's
   latency and reuses the same 4-bit kernels, so the comparison isolates the
   serial structure.
4. The intermediate is produced the way the device produces a linear
   layer's output: Z = bf16(sx * (s_L1 * acc)) with each multiply one fp32
   rounding, then quantized per token exactly like the activations (4-bit
   codes, scale amax / 7).
5. Output: Y = sx sw acc0 + sz s_L2 acc2 (fp64 here).
"""
from __future__ import annotations

import numpy as np

from oracle import serq_oracle as O

F32 = np.float32
S_FLOOR = 1e-5


class L2QERLayer:
    def __init__(self, q_w, s_w, L1, L2, q_l1, s_l1, q_l2, s_l2, S, r):
        self.q_w, self.s_w = q_w, s_w          # K x N codes, N scales (main path, as SERQ)
        self.L1, self.L2 = L1, L2              # fp32 factors before quantization
        self.q_l1, self.s_l1 = q_l1, s_l1      # K x r codes, r scales
        self.q_l2, self.s_l2 = q_l2, s_l2      # r x N codes, N scales
        self.S, self.r = S, r

    @property
    def K(self):
        return self.q_w.shape[0]

    @property
    def N(self):
        return self.q_w.shape[1]


def activation_scale(Xh_calib: np.ndarray) -> np.ndarray:
    """Reading 2: S_j = mean |X^_:,j| over the calibration tokens (floored)."""
    S = np.mean(np.abs(np.asarray(Xh_calib, np.float64)), axis=0)
    return np.maximum(S, S_FLOOR)


def factors(E: np.ndarray, S: np.ndarray, r: int):
    """Rank-r factors of E in the S-scaled space: S E = U Sigma V^T,
    L1 = S^-1 U_r, L2 = Sigma_r V_r^T (fp64)."""
    U, sig, Vt = np.linalg.svd(S[:, None] * np.asarray(E, np.float64), full_matrices=False)
    L1 = U[:, :r] / S[:, None]
    L2 = sig[:r, None] * Vt[:r, :]
    return L1, L2


def prepare(W_hat: np.ndarray, Xh_calib: np.ndarray, r: int) -> L2QERLayer:
    """Offline: quantize W^ as SERQ does, take the rank-r scaled SVD of its
    quantization error, quantize both factors per output channel."""
    q_w, s_w = O.quantize_weight(W_hat, 4)
    E = np.asarray(W_hat, np.float64) - q_w.astype(np.float64) * s_w.astype(np.float64)[None, :]
    S = activation_scale(Xh_calib)
    L1, L2 = factors(E, S, r)
    L1 = L1.astype(F32)
    L2 = L2.astype(F32)
    q_l1, s_l1 = O.quantize_weight(L1, 4)
    q_l2, s_l2 = O.quantize_weight(L2, 4)
    return L2QERLayer(q_w, s_w, L1, L2, q_l1, s_l1, q_l2, s_l2, S, r)


def intermediate(xq: np.ndarray, sx: np.ndarray, layer: L2QERLayer):
    """First factor: Z = bf16(sx * (s_L1 * (X_q L1_q))) (reading 4) and its
    on-the-fly per-token quantization.  Returns (z_acc, Z, zq, sz)."""
    z_acc = O.int_matmul(xq, layer.q_l1)
    t = (layer.s_l1.astype(F32)[None, :] * z_acc.astype(F32)).astype(F32)
    z = (np.asarray(sx, F32)[:, None] * t).astype(F32)
    Z = O.to_bf16(z)
    zq, sz = O.quantize_act(Z, 4)
    return z_acc, Z, zq, sz


def linear(X_hat: np.ndarray, layer: L2QERLayer):
    """X_q W_q + Q(X_q L1_q) L2_q.  Returns (Y fp64, xq, sx, acc0, zq, sz, acc2)."""
    xq, sx = O.quantize_act(X_hat, 4)
    acc0 = O.int_matmul(xq, layer.q_w)
    _, _, zq, sz = intermediate(xq, sx, layer)
    acc2 = O.int_matmul(zq, layer.q_l2)
    Y = (np.asarray(sx, np.float64)[:, None] * layer.s_w.astype(np.float64)[None, :] * acc0
         + np.asarray(sz, np.float64)[:, None] * layer.s_l2.astype(np.float64)[None, :] * acc2)
    return Y, xq, sx, acc0, zq, sz, acc2


def prepare_from_factors(serq_layer, L1: np.ndarray, L2: np.ndarray) -> L2QERLayer:
    """The comparator on a prepared SERQ layer (its W^ codes and scales) with
    given fp32 factors L1 (K x r, rows in the layer's input order) and L2
    (r x N), each quantized per output channel with 4-bit codes."""
    L1 = np.asarray(L1, F32)
    L2 = np.asarray(L2, F32)
    q_l1, s_l1 = O.quantize_weight(L1, 4)
    q_l2, s_l2 = O.quantize_weight(L2, 4)
    return L2QERLayer(serq_layer.q_w, serq_layer.s_w, L1, L2, q_l1, s_l1, q_l2, s_l2, None, L1.shape[1])
