"""Pins of the fp64 backward oracle (CPU).

The backward oracle is the hand-derived adjoint of the forward oracle, so it is
pinned against something else: central finite differences of the forward oracle
(itself pinned by tests/test_oracle_pins.py).  For every input tensor X and a
random direction u, L(X) = <d_out, out(X)> + <d_S_final, S_final(X)> must change
by <dL/dX, X+ - X-> between X- = fl32(X - eps u) and X+ = fl32(X + eps u) (the
perturbed inputs are rounded to fp32 exactly as the oracle reads them, and the
perturbation that really happened is used), up to the truncation error, which is
O(eps^2) relative: checked at eps = 1e-4, and checked to shrink 100-fold from
eps = 1e-3 (a wrong gradient leaves an error that does not shrink).
Two sequences of a packed batch (one shorter than the conv window plus a few
tokens), long memory (alpha close to 1) so that the state carries across tokens,
a nonzero RMSNorm weight and an initial state make every term matter.
"""
import numpy as np
import pytest

import oracle

EPS = 1e-4


def _case(seed=0, lengths=(7, 5), H=2, dk=4, dv=3, K=4):
    rng = np.random.default_rng(seed)
    n_tok = sum(lengths)
    f = lambda *s, std=1.0, mean=0.0: (rng.standard_normal(s) * std + mean).astype(np.float32)
    x = {
        "q": f(n_tok, H, dk), "k": f(n_tok, H, dk), "v": f(n_tok, H, dv),
        "conv_w": f(H * (2 * dk + dv), K, std=0.5),
        "a_logit": f(n_tok, H, mean=-2.0), "b_logit": f(n_tok, H),
        "A": np.log(rng.uniform(0.05, 0.5, H)).astype(np.float32),
        "b_alpha": f(H, std=0.3), "z": f(n_tok, H, dv), "norm_w": f(dv, std=0.3),
        "S0": f(len(lengths), H, dk, dv, std=0.5),
    }
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    d_out = rng.standard_normal((n_tok, H, dv))
    d_S = rng.standard_normal((len(lengths), H, dk, dv))
    return x, cu, d_out, d_S


def _loss(x, cu, d_out, d_S):
    out, S = oracle.prefill(x["q"], x["k"], x["v"], x["conv_w"], x["a_logit"], x["b_logit"], x["A"],
                            x["b_alpha"], x["z"], x["norm_w"], S0=x["S0"], cu_seqlens=cu)
    return float(np.sum(d_out * out) + np.sum(d_S * S))


def _grads(x, cu, d_out, d_S):
    return oracle.backward(x["q"], x["k"], x["v"], x["conv_w"], x["a_logit"], x["b_logit"], x["A"],
                           x["b_alpha"], x["z"], x["norm_w"], d_out, S0=x["S0"], d_S_final=d_S,
                           cu_seqlens=cu)


GRAD_OF = {"q": "dq", "k": "dk", "v": "dv", "conv_w": "d_conv_w", "a_logit": "d_a_logit",
           "b_logit": "d_b_logit", "A": "d_A", "b_alpha": "d_b_alpha", "z": "d_z",
           "norm_w": "d_norm_w", "S0": "d_S0"}


def _fd_error(name, seed, eps):
    x, cu, d_out, d_S = _case(seed)
    g = _grads(x, cu, d_out, d_S)[GRAD_OF[name]]
    u = np.random.default_rng(100 + seed).standard_normal(x[name].shape)
    xp, xm = dict(x), dict(x)
    xp[name] = (x[name].astype(np.float64) + eps * u).astype(np.float32)
    xm[name] = (x[name].astype(np.float64) - eps * u).astype(np.float32)
    fd = _loss(xp, cu, d_out, d_S) - _loss(xm, cu, d_out, d_S)
    step = xp[name].astype(np.float64) - xm[name].astype(np.float64)
    want = float(np.sum(g * step))
    assert abs(want) > 1e-8, "the direction must move the loss"
    return abs(fd - want) / abs(want)


@pytest.mark.parametrize("seed", [0, 1])
@pytest.mark.parametrize("name", list(GRAD_OF))
def test_backward_matches_finite_differences(name, seed):
    e_small = _fd_error(name, seed, EPS)
    assert e_small <= 1e-4, (name, e_small)
    e_big = _fd_error(name, seed, 10 * EPS)
    # truncation error falls as eps^2; rounding-level agreement needs no ratio
    assert e_small <= 1e-9 or e_big / e_small > 30, (name, e_big, e_small)


def test_backward_single_elements():
    """Element by element for one input of each kind (brute force on a tiny case)."""
    x, cu, d_out, d_S = _case(3, lengths=(5,), H=1, dk=3, dv=2)
    g = _grads(x, cu, d_out, d_S)
    for name, idx in (("q", (2, 0, 1)), ("k", (4, 0, 2)), ("v", (0, 0, 1)), ("conv_w", (4, 3)),
                      ("conv_w", (0, 0)), ("a_logit", (3, 0)), ("b_logit", (1, 0)), ("A", (0,)),
                      ("z", (2, 0, 0)), ("norm_w", (1,)), ("S0", (0, 0, 2, 1))):
        xp, xm = dict(x), dict(x)
        xp[name], xm[name] = x[name].copy(), x[name].copy()
        xp[name][idx] = np.float32(float(x[name][idx]) + EPS)
        xm[name][idx] = np.float32(float(x[name][idx]) - EPS)
        fd = (_loss(xp, cu, d_out, d_S) - _loss(xm, cu, d_out, d_S)) / (float(xp[name][idx]) - float(xm[name][idx]))
        want = g[GRAD_OF[name]][idx]
        assert abs(fd - want) <= 1e-4 * abs(want) + 1e-8, (name, idx, fd, want)


def test_backward_without_final_state_gradient():
    """d_S_final = None equals d_S_final = 0; zero d_out and d_S_final give zero gradients."""
    x, cu, d_out, d_S = _case(4)
    a = oracle.backward(x["q"], x["k"], x["v"], x["conv_w"], x["a_logit"], x["b_logit"], x["A"],
                        x["b_alpha"], x["z"], x["norm_w"], d_out, S0=x["S0"], cu_seqlens=cu)
    b = _grads(x, cu, d_out, np.zeros_like(d_S))
    for key in a:
        np.testing.assert_array_equal(a[key], b[key])
    z = _grads(x, cu, np.zeros_like(d_out), np.zeros_like(d_S))
    for key in z:
        assert not np.any(z[key]), key
