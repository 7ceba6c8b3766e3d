"""The chunked (WY / UT-transform) form of the gated delta rule, in fp64, against
the token-by-token oracle.

This pins the algebra the CUDA prefill uses before any kernel runs.  Derivation
(from the erase-then-write update of the write-up's 模块 A, 递归状态): with
u_i = beta_i (v_i - alpha_i S_{i-1}^T k_i) the update is S_i = alpha_i S_{i-1} + k_i u_i^T.
Inside a chunk with start state S, cumulative log-decay G_i = sum_{j<=i} log alpha_j:
    (I + L) U = diag(beta) (V - diag(e^G) K S),  L_ij = beta_i (k_i.k_j) e^{G_i - G_j}, j < i
    Y  = diag(e^G) Q S + (Q K^T * e^{G_i - G_j} * [j <= i]) U
    S' = e^{G_C} S + (diag(e^{G_C - G}) K)^T U
All decays are evaluated as exp of a non-positive difference of log sums.
"""
import numpy as np
import pytest

import oracle


def chunked_delta_rule(q, k, v, log_alpha, beta, S0, C):
    T, dk = q.shape
    S = S0.copy()
    Y = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, C):
        sl = slice(c0, min(c0 + C, T))
        Q, K, V, g, b = q[sl], k[sl], v[sl], log_alpha[sl], beta[sl]
        n = Q.shape[0]
        G = np.cumsum(g)
        D = G[:, None] - G[None, :]
        low = np.tril(np.ones((n, n)), -1)
        Gam = np.exp(np.where(low + np.eye(n) > 0, D, -np.inf))   # e^{G_i-G_j}, j <= i, else 0
        L = b[:, None] * (K @ K.T) * Gam * low
        Tm = np.linalg.inv(np.eye(n) + L)
        W = Tm @ (b[:, None] * np.exp(G)[:, None] * K)
        Up = Tm @ (b[:, None] * V)
        U = Up - W @ S
        Y[sl] = np.exp(G)[:, None] * (Q @ S) + ((Q @ K.T) * Gam) @ U
        S = np.exp(G[-1]) * S + (np.exp(G[-1] - G)[:, None] * K).T @ U
    return Y, S


@pytest.mark.parametrize("C", [1, 16, 64])
@pytest.mark.parametrize("T", [1, 63, 64, 150])
@pytest.mark.parametrize("memory", ["short", "long"])
def test_chunked_form_equals_recurrence(C, T, memory):
    rng = np.random.default_rng(100 + C + T)
    dk, dv = 32, 16
    q = rng.standard_normal((T, dk)); q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = rng.standard_normal((T, dk)); k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv))
    if memory == "short":       # the workloads' gates: log alpha about -7 on average
        log_alpha = -np.exp(np.log(rng.uniform(1, 16))) * np.logaddexp(0, rng.standard_normal(T))
    else:                       # alpha close to 1
        log_alpha = -rng.uniform(0.01, 0.1) * np.logaddexp(0, rng.standard_normal(T) - 2)
    beta = 1 / (1 + np.exp(-rng.standard_normal(T)))
    S0 = 0.14 * rng.standard_normal((dk, dv))
    y_ref, S_ref = oracle.delta_rule(q, k, v, np.exp(log_alpha), beta, S0)
    y, S = chunked_delta_rule(q, k, v, log_alpha, beta, S0, C)
    scale = max(np.abs(y_ref).max(), 1e-300)
    assert np.abs(y - y_ref).max() <= 1e-12 * scale
    assert np.abs(S - S_ref).max() <= 1e-12 * max(np.abs(S_ref).max(), 1e-300)


def test_chunked_form_survives_underflowing_decay():
    """Decays far below the double range (sum of log alpha < -745) stay finite
    because only differences G_i - G_j <= 0 are exponentiated."""
    rng = np.random.default_rng(7)
    T, dk, dv = 64, 8, 8
    q = rng.standard_normal((T, dk)); q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = rng.standard_normal((T, dk)); k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv))
    log_alpha = np.full(T, -40.0)
    beta = np.full(T, 0.5)
    y, S = chunked_delta_rule(q, k, v, log_alpha, beta, np.zeros((dk, dv)), 64)
    y_ref, S_ref = oracle.delta_rule(q, k, v, np.exp(log_alpha), beta, np.zeros((dk, dv)))
    assert np.isfinite(y).all() and np.isfinite(S).all()
    assert np.allclose(y, y_ref, rtol=1e-12, atol=1e-14)
    assert np.allclose(S, S_ref, rtol=1e-12, atol=1e-14)
