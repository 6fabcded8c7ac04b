"""CPU oracle for GPTQ as SERQ's main-weight quantizer ("SERQ(GPTQ)") --
TEST INFRASTRUCTURE ONLY.

Only the tests may import this module; the product path never calls it.

The pages name the variant and nothing more: the papernotes.org notes on
SERQ list "SERQ(GPTQ)" beside the round-to-nearest SERQ in their main results
table, and the gist.science (de) summary, section 2B, says the main weight is
quantized with RTN or GPTQ.  GPTQ itself (Frantar et al., 2022) quantizes the
rows of W (its input channels) one after another and moves each row's
quantization error onto the rows not yet quantized, weighted by the upper
Cholesky factor U of the inverse Hessian H^-1 = U^T U of the layer's
calibration inputs, H = sum_t x_t x_t^T.

Readings where the pages are silent:

1. GPTQ runs on SERQ's flattened, permuted weight W^ with the flattened,
   permuted calibration activations X^ (same smoothing and order), and keeps
   SERQ's quantizer: per output channel, symmetric INT4, the scale fixed
   from the column's maximum before any update, code = clamp(rint(w * (7 /
   amax)), -7, 7).
2. The r salient rows are quantized first (they lead the saliency order) and
   their error is NOT propagated: the compensator R = W^[0:r] - deq(q[0:r])
   reconstructs it, exactly as in round-to-nearest SERQ.  Rows r.. carry
   GPTQ's error propagation among themselves.
3. Damping: H_ii += 0.01 * mean(diag H) (GPTQ's usual 1%); H = I when the
   calibration activations are all zero (then GPTQ is round-to-nearest).
   H's overall scale (GPTQ writes 2 X X^T) does not change U's ratios and is
   left out.
4. Arithmetic order, so that every bit is fixed and the device can be
   compared exactly (the algebra is GPTQ's):
   * fp64 for H and its factors.  A sum starts from +0 and adds its terms in
     increasing index; a Cholesky or substitution entry starts from its
     matrix entry and subtracts its product terms in increasing index, each
     product and each difference rounded once (no fused multiply-add).
   * Cholesky is the textbook right-looking column sweep; L^-1 is forward
     substitution on the identity; H^-1 = L^-T L^-1 (terms k >= max(a, b),
     the others being structural zeros); U is the transpose of the lower
     Cholesky factor of H^-1.
   * The weight updates are fp32 with U rounded to fp32 once: the scaled
     error e = (w_i - q_i * s) / u_ii, then w_j -= u_ij * e for j > i, row i
     by row i.
   A non-positive pivot is an error.
"""
from __future__ import annotations

import numpy as np

from oracle import serq_oracle as O

F32 = np.float32
F64 = np.float64
DAMP = 0.01


def hessian(Xh_calib: np.ndarray) -> np.ndarray:
    """H = sum_t x_t x_t^T over the calibration tokens in order (fp64; each
    product of two fp32 values is exact) with the damping of reading 3."""
    X = np.asarray(Xh_calib, F32).astype(F64)
    n, K = X.shape
    H = np.zeros((K, K), F64)
    for t in range(n):
        H += np.outer(X[t], X[t])
    d = 0.0
    for i in range(K):
        d = d + H[i, i]
    lam = DAMP * (d / K) if d > 0 else 1.0
    H[np.diag_indices(K)] += lam
    return H


def cholesky_lower(A: np.ndarray) -> np.ndarray:
    """Right-looking Cholesky, A = L L^T: column k takes the square root of
    the pivot and divides the column below by it, then the trailing block
    loses the outer product of that column."""
    T = np.array(A, dtype=F64, copy=True)
    K = T.shape[0]
    L = np.zeros_like(T)
    for k in range(K):
        p = T[k, k]
        if not p > 0:
            raise ValueError(f"non-positive pivot {p!r} at {k}")
        d = np.sqrt(p)
        L[k, k] = d
        L[k + 1:, k] = T[k + 1:, k] / d
        T[k + 1:, k + 1:] -= np.outer(L[k + 1:, k], L[k + 1:, k])
    return L


def inverse_lower(L: np.ndarray) -> np.ndarray:
    """V = L^-1 by forward substitution on the identity: row m of V is the
    current right-hand side row over L_mm, then every later row loses L_im
    times it (columns past m are structural zeros and are not touched)."""
    K = L.shape[0]
    T = np.eye(K, dtype=F64)
    V = np.zeros((K, K), F64)
    for m in range(K):
        V[m, :m + 1] = T[m, :m + 1] / L[m, m]
        T[m + 1:, :m + 1] -= np.outer(L[m + 1:, m], V[m, :m + 1])
    return V


def inverse_from_lower_inverse(V: np.ndarray) -> np.ndarray:
    """H^-1 = V^T V for V = L^-1: entry (a, b) sums V_ka V_kb over
    k >= max(a, b) in increasing k."""
    K = V.shape[0]
    A = np.zeros((K, K), F64)
    for k in range(K):
        A[:k + 1, :k + 1] += np.outer(V[k, :k + 1], V[k, :k + 1])
    return A


def inverse_hessian_factor(Xh_calib: np.ndarray) -> np.ndarray:
    """U (upper, fp64) with H^-1 = U^T U."""
    L = cholesky_lower(hessian(Xh_calib))
    return cholesky_lower(inverse_from_lower_inverse(inverse_lower(L))).T


def gptq_codes(W_hat: np.ndarray, U: np.ndarray, r: int, return_updated: bool = False):
    """Quantize rows in order; rows >= r move their error onto the later rows.

    Returns (codes int8 K x N, scales fp32 N) and, with return_updated, the
    K x N values each row had when it was quantized."""
    W = np.array(W_hat, dtype=F32, copy=True)
    K, N = W.shape
    amax = np.max(np.abs(W), axis=0).astype(F32)
    nz = amax > 0
    inv = np.where(nz, F32(7) / np.where(nz, amax, F32(1)), F32(0)).astype(F32)
    sw = (amax / F32(7)).astype(F32)
    U32 = np.asarray(U, F64).astype(F32)
    q = np.zeros((K, N), np.int8)
    for i in range(K):
        qi = np.clip(np.rint((W[i] * inv).astype(F32)), -7, 7).astype(F32)
        q[i] = qi.astype(np.int8)
        if i >= r and i + 1 < K:
            err = ((W[i] - (qi * sw).astype(F32)).astype(F32) / U32[i, i]).astype(F32)
            W[i + 1:] = (W[i + 1:] - (U32[i, i + 1:, None] * err[None, :]).astype(F32)).astype(F32)
    return (q, sw, W) if return_updated else (q, sw)


def prepare_group(weights, X_calib, r: int, alpha: float = 0.5, saliency: int = O.SALIENCY_SCALE):
    """SERQ's offline stage with GPTQ for the main weight: smoothing and the
    saliency order as in round-to-nearest SERQ, one inverse-Hessian factor
    shared by the weights that consume the activation.  Returns (s, pi,
    [PreparedLayer per weight])."""
    if isinstance(weights, np.ndarray):
        weights = [weights]
    s = O.smooth_scales(X_calib, weights, alpha)
    pi = O.saliency_perm(O.saliency_key(s, weights, saliency))
    U = inverse_hessian_factor(O.flatten_permute(X_calib, s, pi, out_bf16=False))
    layers = []
    for W in weights:
        W_hat = O.fold_weight(W, s, pi)
        q_w, s_w = gptq_codes(W_hat, U, r)
        if r > 0:
            R = O.compensator(W_hat, q_w, s_w, r)
            q_r, s_r = O.quantize_weight(R, 4)
        else:
            R = np.zeros((0, W.shape[1]), F32)
            q_r = np.zeros((0, W.shape[1]), np.int8)
            s_r = np.zeros(W.shape[1], F32)
        layers.append(O.PreparedLayer(s, pi, W_hat, q_w, s_w, R, q_r, s_r, r))
    return s, pi, layers


def prepare(W, X_calib, r: int, alpha: float = 0.5, saliency: int = O.SALIENCY_SCALE):
    return prepare_group([W], X_calib, r, alpha, saliency)[2][0]
