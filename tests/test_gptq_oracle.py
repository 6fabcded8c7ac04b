"""Pins of the GPTQ oracle (CPU).

GPTQ (Frantar et al., 2022) as SERQ's main-weight quantizer: the papernotes.org
SERQ notes' main results table ("SERQ(GPTQ)") and the gist.science (de)
summary, section 2B.  Each test checks the oracle against something other
than itself: a textbook routine, a closed form, a hand-worked case, or the
optimal-brain-surgeon update written with explicit inverses.
"""
import numpy as np
import pytest

from oracle import gptq_oracle as G
from oracle import serq_oracle as O

F32 = np.float32


def _spd(K, seed, corr=0.6):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((4 * K, K))
    X[:, 1:] += corr * X[:, :-1]            # neighbouring channels correlate
    return X.T @ X + 0.1 * np.eye(K)


def test_cholesky_exact_integer_case():
    # [[4, 2, -2], [2, 10, 2], [-2, 2, 6]] = L L^T with L = [[2,0,0],[1,3,0],[-1,1,2]]
    # (every step exact in binary).
    H = np.array([[4, 2, -2], [2, 10, 2], [-2, 2, 6]], np.float64)
    L = G.cholesky_lower(H)
    assert np.array_equal(L, np.array([[2, 0, 0], [1, 3, 0], [-1, 1, 2]], np.float64))


def test_cholesky_against_textbook():
    H = _spd(40, 1)
    L = G.cholesky_lower(H)
    assert np.allclose(L, np.linalg.cholesky(H), rtol=1e-12, atol=1e-12)
    assert np.allclose(L @ L.T, H, rtol=1e-13, atol=1e-10)
    assert np.all(np.triu(L, 1) == 0)


def test_cholesky_rejects_an_indefinite_matrix():
    with pytest.raises(ValueError):
        G.cholesky_lower(np.array([[1.0, 2.0], [2.0, 1.0]]))


def test_inverse_lower_against_textbook():
    L = np.linalg.cholesky(_spd(33, 2))
    V = G.inverse_lower(L)
    assert np.all(np.triu(V, 1) == 0)
    assert np.allclose(L @ V, np.eye(33), atol=1e-12)
    assert np.allclose(V, np.linalg.inv(L), rtol=1e-10, atol=1e-12)


def test_inverse_from_lower_inverse_is_the_inverse():
    H = _spd(37, 3)
    V = np.linalg.inv(np.linalg.cholesky(H))
    A = G.inverse_from_lower_inverse(V)
    assert np.array_equal(A, A.T)
    assert np.allclose(A, np.linalg.inv(H), rtol=1e-10, atol=1e-12)


def test_hessian_exact_on_integer_inputs():
    rng = np.random.default_rng(4)
    X = rng.integers(-3, 4, size=(50, 12)).astype(F32)
    H = G.hessian(X)
    G0 = X.astype(np.float64).T @ X.astype(np.float64)   # exact: small integers
    lam = 0.01 * (np.trace(G0) / 12)
    assert np.array_equal(H, G0 + lam * np.eye(12))


def test_hessian_of_zero_inputs_is_identity():
    assert np.array_equal(G.hessian(np.zeros((5, 8), F32)), np.eye(8))


def test_inverse_hessian_factor():
    rng = np.random.default_rng(5)
    X = rng.standard_normal((96, 24)).astype(F32)
    X[:, 3] *= 20.0
    U = G.inverse_hessian_factor(X)
    H = G.hessian(X)
    Hinv = np.linalg.inv(H)
    assert np.all(np.tril(U, -1) == 0) and np.all(np.diag(U) > 0)
    assert np.allclose(U.T @ U, Hinv, rtol=1e-9, atol=1e-12)
    assert np.allclose(U, np.linalg.cholesky(Hinv).T, rtol=1e-9, atol=1e-12)


def test_gptq_hand_worked_three_rows():
    # Activations (already flattened and permuted): rows (1,1,0), (1,0,0),
    # (0,0,1), so X^T X = [[2,1,0],[1,1,0],[0,0,1]], mean diagonal 4/3 and
    # H = X^T X + (0.04/3) I.  One output channel W^ = (0.3, 0.17, 0.5):
    # amax 0.5, inv 14, scale 1/14.
    # Row 0: 0.3 * 14 = 4.2 -> code 4, error 0.3 - 4/14 = 1/70.
    # The OBS update of row 1 (row 2 is decoupled: H is block diagonal) is
    # w1 += (H01 / H11) * error = 0.17 + (1 / (1 + 0.04/3)) / 70 = 0.18410,
    # and 0.18410 * 14 = 2.577 -> code 3 (round-to-nearest gives 0.17 * 14 =
    # 2.38 -> 2).  Row 2: 0.5 * 14 = 7 -> 7.
    X = np.array([[1, 1, 0], [1, 0, 0], [0, 0, 1]], F32)
    W = np.array([[0.3], [0.17], [0.5]], F32)
    U = G.inverse_hessian_factor(X)
    q, sw, upd = G.gptq_codes(W, U, r=0, return_updated=True)
    assert q[:, 0].tolist() == [4, 3, 7]
    assert O.quantize_weight(W)[0][:, 0].tolist() == [4, 2, 7]
    assert sw[0] == F32(0.5) / F32(7)
    h11 = 1.0 + 0.04 / 3
    assert abs(float(upd[1, 0]) - (0.17 + (0.3 - 4 / 14) / h11)) < 1e-6
    assert upd[2, 0] == W[2, 0]
    # the salient rows (r = 2) keep round-to-nearest and propagate nothing
    q2, _ = G.gptq_codes(W, U, r=2)
    assert q2[:, 0].tolist() == [4, 2, 7]


def test_gptq_with_a_diagonal_factor_is_round_to_nearest():
    rng = np.random.default_rng(6)
    W = rng.standard_normal((64, 48)).astype(F32)
    q, sw = G.gptq_codes(W, np.diag(np.linspace(0.5, 2.0, 64)), r=0)
    qr, swr = O.quantize_weight(W)
    assert np.array_equal(q, qr) and np.array_equal(sw, swr)


def test_gptq_with_r_equal_K_is_round_to_nearest():
    rng = np.random.default_rng(7)
    X = rng.standard_normal((80, 32)).astype(F32)
    W = rng.standard_normal((32, 40)).astype(F32)
    q, sw = G.gptq_codes(W, G.inverse_hessian_factor(X), r=32)
    qr, swr = O.quantize_weight(W)
    assert np.array_equal(q, qr) and np.array_equal(sw, swr)


def test_gptq_equals_obs_with_explicit_inverses():
    # The optimal-brain-surgeon step of GPTQ: after quantizing row i, the rows
    # still free move by -[H_F^-1]_{:, i} / [H_F^-1]_{ii} * (w_i - q_i s), with
    # H_F the Hessian restricted to rows i.. (an explicit inverse per step,
    # no Cholesky).  With the oracle's codes fixed, the values each row has
    # when quantized must agree, and every code must be a nearest code.
    rng = np.random.default_rng(8)
    K, N, r = 24, 40, 5
    X = rng.standard_normal((120, K)).astype(F32)
    X[:, 1:] += F32(0.7) * X[:, :-1]
    W = rng.standard_normal((K, N)).astype(F32)
    q, sw, upd = G.gptq_codes(W, G.inverse_hessian_factor(X), r, return_updated=True)
    H = G.hessian(X)
    w = W.astype(np.float64)
    for i in range(K):
        if i >= r and i + 1 < K:
            Hf = np.linalg.inv(H[i:, i:])
            w[i + 1:] -= np.outer(Hf[1:, 0] / Hf[0, 0], w[i] - q[i].astype(np.float64) * sw)
    scale = np.max(np.abs(W), axis=0)
    assert np.max(np.abs(upd - w) / scale) < 1e-4
    t = w * (7.0 / scale)
    assert np.all(np.abs(np.clip(t, -7, 7) - q) <= 0.5 + 1e-3)
    assert np.any(q != O.quantize_weight(W)[0])       # the feedback did something


def test_gptq_lowers_the_layer_output_error():
    # GPTQ minimises ||X (W - W_q)||^2 row by row; on correlated inputs it
    # must beat round-to-nearest on the rows it touches.
    rng = np.random.default_rng(9)
    K, N, r = 64, 96, 8
    X = rng.standard_normal((256, K)).astype(F32)
    for j in range(1, K):
        X[:, j] += F32(0.8) * X[:, j - 1]
    W = rng.standard_normal((K, N)).astype(F32)
    q, sw = G.gptq_codes(W, G.inverse_hessian_factor(X), r)
    qr, _ = O.quantize_weight(W)
    Xd = X.astype(np.float64)
    D = W.astype(np.float64) - q.astype(np.float64) * sw
    Dr = W.astype(np.float64) - qr.astype(np.float64) * sw
    D[:r] = Dr[:r] = 0.0                            # rows r.. only
    assert np.sum((Xd @ D) ** 2) < 0.8 * np.sum((Xd @ Dr) ** 2)


def test_prepare_group_keeps_serq_order_and_salient_rows():
    rng = np.random.default_rng(10)
    K, r = 64, 16
    X = rng.standard_normal((48, K)).astype(F32)
    X[:, [3, 17, 40]] *= F32(30.0)
    Ws = [rng.standard_normal((K, 32)).astype(F32) for _ in range(2)]
    s, pi, layers = G.prepare_group(Ws, X, r)
    s0, pi0, rtn = O.prepare_group(Ws, X, r)
    assert np.array_equal(s, s0) and np.array_equal(pi, pi0)
    for a, b in zip(layers, rtn):
        assert np.array_equal(a.W_hat, b.W_hat) and np.array_equal(a.s_w, b.s_w)
        assert np.array_equal(a.q_w[:r], b.q_w[:r])
        assert np.array_equal(a.R, b.R) and np.array_equal(a.q_r, b.q_r) and np.array_equal(a.s_r, b.s_r)
        assert not np.array_equal(a.q_w[r:], b.q_w[r:])
