"""The reverse-mode derivative of the chunked (WY / UT-transform) gated delta rule,
in fp64, against torch autograd through the token-by-token recurrence.

This pins, before any kernel, the chunk-level backward algebra that a
tensor-core backward would run: per chunk, from the chunk's start state S and the
incoming gradients dY (outputs) and dS' (end state), every gradient is a product
of chunk-sized matrices. With the forward quantities of the chunked form (see
test_chunk_algebra.py):

    A = (Q K^T) * Gamma (j <= i),  Qt = diag(e^G) Q,  Kt = diag(e^{G_C - G}) K
    X1 = diag(beta) V,  X2 = diag(beta e^G) K,  T = (I + L)^-1,
    W = T X2,  U' = T X1,  U = U' - W S,  Y = Qt S + A U,  S' = e^{G_C} S + Kt^T U

the backward is

    dU  = A^T dY + Kt dS'            dA = (dY U^T) * [j <= i]
    dQt = dY S^T                     dKt = U dS'^T
    dW  = -dU S^T                    dT  = dU X1^T + dW X2^T
    dX1 = T^T dU                     dX2 = T^T dW
    dL  = -(T^T dT T^T) * [j < i]
    dS  = Qt^T dY + e^{G_C} dS' - W^T dU        (the gradient of the chunk's start state)

then V, beta, K, Q by the chain rule through X1, X2, L = diag(beta)(K K^T * Gamma),
A, Qt and Kt, and the log-decays through every e^{...} factor: a gradient dG_i of
the cumulative sums G_i = sum_{j <= i} log alpha_j becomes d log alpha_j =
sum_{i >= j} dG_i (a reverse cumulative sum).
"""
import numpy as np
import pytest
import torch

import oracle


def _chunk_forward(Q, K, V, g, b, S, mm=np.matmul):
    n = Q.shape[0]
    G = np.cumsum(g)
    incl = np.tril(np.ones((n, n)))
    SL = np.tril(np.ones((n, n)), -1)
    Gam = np.exp(np.where(incl > 0, G[:, None] - G[None, :], -np.inf))
    KK = mm(K, K.T)
    L = b[:, None] * KK * Gam * SL
    T = np.linalg.inv(np.eye(n) + L)
    eG = np.exp(G)
    X1 = b[:, None] * V
    X2 = (b * eG)[:, None] * K
    W = mm(T, X2)
    U = mm(T, X1) - mm(W, S)
    QK = mm(Q, K.T)
    A = QK * Gam
    Qt = eG[:, None] * Q
    r = np.exp(G[-1] - G)
    Kt = r[:, None] * K
    Y = mm(Qt, S) + mm(A, U)
    S_next = np.exp(G[-1]) * S + mm(Kt.T, U)
    return dict(G=G, incl=incl, SL=SL, Gam=Gam, KK=KK, T=T, eG=eG, X1=X1, X2=X2, W=W, U=U, QK=QK, A=A, Qt=Qt,
                Kt=Kt, r=r), Y, S_next


def chunked_delta_rule_backward(q, k, v, log_alpha, beta, S0, C, dY, dS_final, mm=np.matmul,
                                keep=lambda x: x):
    """Gradients (dq, dk, dv, dlog_alpha, dbeta, dS0) of <dY, Y> + <dS_final, S_T>.
    `mm` computes every matrix product (an emulation of reduced-precision operands
    may stand in); `keep` rounds the state and its gradient where a kernel would
    store them."""
    T_len = q.shape[0]
    starts = list(range(0, T_len, C))
    S_at = []                                   # the state at each chunk's start (checkpoints)
    S = S0.copy()
    for c0 in starts:
        sl = slice(c0, min(c0 + C, T_len))
        S_at.append(S)
        _, _, S = _chunk_forward(q[sl], k[sl], v[sl], log_alpha[sl], beta[sl], S, mm)
        S = keep(S)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dg, db = np.zeros_like(log_alpha), np.zeros_like(beta)
    dS = dS_final.copy()
    for c0, S in zip(reversed(starts), reversed(S_at)):
        sl = slice(c0, min(c0 + C, T_len))
        Q, K, V, b, dYc = q[sl], k[sl], v[sl], beta[sl], dY[sl]
        f, _, _ = _chunk_forward(Q, K, V, log_alpha[sl], b, S, mm)
        eGC = np.exp(f["G"][-1])
        # through Y = Qt S + A U and S' = e^{G_C} S + Kt^T U
        dU = mm(f["A"].T, dYc) + mm(f["Kt"], dS)
        dA = mm(dYc, f["U"].T) * f["incl"]
        dQt = mm(dYc, S.T)
        dKt = mm(f["U"], dS.T)
        dS_prev = mm(f["Qt"].T, dYc) + eGC * dS
        dGC = eGC * np.sum(dS * S)
        # through U = U' - W S, U' = T X1, W = T X2, T = (I + L)^-1
        dW = -mm(dU, S.T)
        dS_prev -= mm(f["W"].T, dU)
        dT = mm(dU, f["X1"].T) + mm(dW, f["X2"].T)
        dX1 = mm(f["T"].T, dU)
        dX2 = mm(f["T"].T, dW)
        dL = -mm(mm(f["T"].T, dT), f["T"].T) * f["SL"]
        # leaves: V, beta, K, Q
        dv[sl] = b[:, None] * dX1
        db[sl] = (np.sum(dX1 * V, 1) + np.sum(dX2 * f["eG"][:, None] * K, 1)
                  + np.sum(dL * f["KK"] * f["Gam"], 1))
        P = b[:, None] * dL                              # gradient of K K^T * Gamma (strict lower)
        dKK = P * f["Gam"]
        dQK = dA * f["Gam"]
        dk[sl] = ((b * f["eG"])[:, None] * dX2 + f["r"][:, None] * dKt + mm(dKK, K) + mm(dKK.T, K)
                  + mm(dQK.T, Q))
        dq[sl] = f["eG"][:, None] * dQt + mm(dQK, K)
        # log-decays: every factor e^{G_i - G_j}, e^{G_i}, e^{G_C - G_i}, e^{G_C}
        E = (P * f["KK"] + dA * f["QK"]) * f["Gam"]
        dG = E.sum(1) - E.sum(0)
        dG += np.sum(dQt * f["Qt"], 1) + np.sum(dX2 * f["X2"], 1) - np.sum(dKt * f["Kt"], 1)
        dG[-1] += np.sum(dKt * f["Kt"]) + dGC
        dg[sl] = np.cumsum(dG[::-1])[::-1]
        dS = keep(dS_prev)
    return dq, dk, dv, dg, db, dS


def _autograd_reference(q, k, v, log_alpha, beta, S0, dY, dS_final):
    """Token-by-token erase-then-write recurrence in torch fp64; torch derives the gradient."""
    t = {n: torch.tensor(x, dtype=torch.float64, requires_grad=True)
         for n, x in dict(q=q, k=k, v=v, g=log_alpha, b=beta, S0=S0).items()}
    S = t["S0"]
    ys = []
    for i in range(q.shape[0]):
        a = torch.exp(t["g"][i])
        ki = t["k"][i]
        S = a * S - t["b"][i] * torch.outer(ki, a * (S.T @ ki)) + t["b"][i] * torch.outer(ki, t["v"][i])
        ys.append(S.T @ t["q"][i])
    Y = torch.stack(ys)
    loss = (Y * torch.from_numpy(dY)).sum() + (S * torch.from_numpy(dS_final)).sum()
    loss.backward()
    return Y.detach().numpy(), S.detach().numpy(), [t[n].grad.numpy() for n in ("q", "k", "v", "g", "b", "S0")]


def _case(T, memory, seed, dk=16, dv=8):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, dk)); q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = rng.standard_normal((T, dk)); k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv))
    if memory == "short":
        log_alpha = -rng.uniform(1, 16) * np.logaddexp(0, rng.standard_normal(T))
    else:
        log_alpha = -rng.uniform(0.01, 0.1) * np.logaddexp(0, rng.standard_normal(T) - 2)
    beta = 1 / (1 + np.exp(-rng.standard_normal(T)))
    S0 = 0.14 * rng.standard_normal((dk, dv))
    dY = rng.standard_normal((T, dv))
    dS_final = rng.standard_normal((dk, dv))
    return q, k, v, log_alpha, beta, S0, dY, dS_final


@pytest.mark.parametrize("C", [1, 16, 64])
@pytest.mark.parametrize("T", [1, 37, 130])
@pytest.mark.parametrize("memory", ["short", "long"])
def test_chunked_backward_equals_autograd(C, T, memory):
    q, k, v, g, b, S0, dY, dS_final = _case(T, memory, 300 + C + T)
    Y_ref, S_ref, grads_ref = _autograd_reference(q, k, v, g, b, S0, dY, dS_final)
    # the autograd reference differentiates the oracle's function
    y_o, S_o = oracle.delta_rule(q, k, v, np.exp(g), b, S0)
    np.testing.assert_allclose(Y_ref, y_o, rtol=0, atol=1e-12 * np.abs(y_o).max())
    np.testing.assert_allclose(S_ref, S_o, rtol=0, atol=1e-12 * np.abs(S_o).max())
    grads = chunked_delta_rule_backward(q, k, v, g, b, S0, C, dY, dS_final)
    for name, got, want in zip(("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0"), grads, grads_ref):
        scale = max(np.abs(want).max(), 1e-300)
        assert np.abs(got - want).max() <= 1e-10 * scale, (name, np.abs(got - want).max() / scale)


def test_chunk_size_does_not_change_the_gradient():
    """The same gradient from chunks of 1 (the token-level adjoint), 8 and 64."""
    q, k, v, g, b, S0, dY, dS_final = _case(100, "long", 9)
    g1 = chunked_delta_rule_backward(q, k, v, g, b, S0, 1, dY, dS_final)
    for C in (8, 64):
        gC = chunked_delta_rule_backward(q, k, v, g, b, S0, C, dY, dS_final)
        for a, c in zip(g1, gC):
            assert np.abs(a - c).max() <= 1e-11 * max(np.abs(a).max(), 1e-300)


def test_state_gradient_only():
    """dY = 0: the gradient flows from dS_final alone; with beta = 0 the state is only
    decayed, so dS0 = (prod alpha) dS_final exactly and dlog_alpha_j = <dS_final, S_T>."""
    q, k, v, g, b, S0, _, dS_final = _case(40, "long", 11)
    b = np.zeros_like(b)
    dq, dk, dv, dg, db, dS0 = chunked_delta_rule_backward(q, k, v, g, b, S0, 16, np.zeros((40, 8)), dS_final)
    decay = np.exp(g.sum())
    np.testing.assert_allclose(dS0, decay * dS_final, rtol=1e-13)
    np.testing.assert_allclose(dg, np.full(40, decay * np.sum(S0 * dS_final)), rtol=1e-12)
    assert not np.any(dq) and not np.any(dk) and not np.any(dv)
