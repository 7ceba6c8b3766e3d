"""Pins of the fp64 oracle to what the pages and the mathematics fix.

Sources: the paper.rainbus.top digest of "On the Design of Qwen3.8-Next
Architecture" (方法步骤详情, step (1): the compact update and the decay gate) and
the slinene.github.io write-up of the same report (模块 A — Gated DeltaNet:
递归状态 = erase-then-write update and readout, 参数化 = prelude and output).

Every check here compares the oracle with something other than itself: a
different but equivalent formula, an explicit product of transition matrices,
closed forms, library routines (numpy convolution, scipy's expit), exact
rational arithmetic, or hand-derived cases in tests/golden/.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
from scipy.special import expit

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "delta_rule_cases.json")


def _unit(rng, n, d):
    x = rng.standard_normal((n, d))
    return x / np.linalg.norm(x, axis=1, keepdims=True)


# ------------------------------------------------------------- the recurrence

def test_compact_form_equals_erase_then_write():
    """digest step (1): S_t = alpha (I - beta k k^T) S + beta k v^T equals the
    write-up's erase-then-write form, for arbitrary alpha, beta, k, v, S."""
    rng = np.random.default_rng(11)
    for dk, dv in ((4, 3), (16, 16), (64, 32)):
        for _ in range(20):
            S = rng.standard_normal((dk, dv))
            k = rng.standard_normal(dk)          # not even normalised: the identity is algebraic
            v = rng.standard_normal(dv)
            q = rng.standard_normal(dk)
            alpha, beta = rng.uniform(0.01, 1.0), rng.uniform(0.0, 1.0)
            compact = alpha * (np.eye(dk) - beta * np.outer(k, k)) @ S + beta * np.outer(k, v)
            y, S1 = oracle.delta_rule(q[None], k[None], v[None], [alpha], [beta], S)
            scale = np.abs(compact).max()
            assert np.abs(S1 - compact).max() <= 1e-14 * scale * dk
            assert np.allclose(y[0], compact.T @ q, rtol=1e-13, atol=1e-13 * scale)


def test_literal_second_compact_form_differs_when_alpha_below_one():
    """The write-up's "等价紧凑形式" prints (alpha I - beta k k^T) S + beta k v^T; it
    matches the erase-then-write form only when alpha = 1.  The oracle follows the
    digest's alpha (I - beta k k^T) form, which agrees with erase-then-write."""
    rng = np.random.default_rng(12)
    dk, dv = 8, 8
    S = rng.standard_normal((dk, dv))
    k = _unit(rng, 1, dk)[0]
    v = rng.standard_normal(dv)
    beta = 0.7
    for alpha in (0.3, 1.0):
        literal = (alpha * np.eye(dk) - beta * np.outer(k, k)) @ S + beta * np.outer(k, v)
        _, S1 = oracle.delta_rule(k[None], k[None], v[None], [alpha], [beta], S)
        if alpha == 1.0:
            assert np.allclose(S1, literal, rtol=1e-13, atol=1e-13)
        else:
            assert np.abs(S1 - literal).max() > 1e-3


def test_materialised_transition_product():
    """On tiny inputs the state equals the explicit product of transition matrices
    M_t = alpha_t (I - beta_t k_t k_t^T):  S_T = M_T..M_1 S_0 + sum_t M_T..M_{t+1} beta_t k_t v_t^T,
    and y_t = S_t^T q_t for the materialised S_t."""
    rng = np.random.default_rng(13)
    for T in (1, 2, 5, 8):
        for dk, dv in ((1, 1), (2, 3), (4, 4), (3, 2)):
            q, k = _unit(rng, T, dk), _unit(rng, T, dk)
            v = rng.standard_normal((T, dv))
            alpha, beta = rng.uniform(0.05, 1.0, T), rng.uniform(0.0, 1.0, T)
            S0 = rng.standard_normal((dk, dv))
            y, ST = oracle.delta_rule(q, k, v, alpha, beta, S0)
            M = [alpha[t] * (np.eye(dk) - beta[t] * np.outer(k[t], k[t])) for t in range(T)]
            for t_end in range(1, T + 1):
                P = np.eye(dk)
                for t in range(t_end):
                    P = M[t] @ P
                St = P @ S0
                for t in range(t_end):
                    Pt = np.eye(dk)
                    for s in range(t + 1, t_end):
                        Pt = M[s] @ Pt
                    St = St + Pt @ (beta[t] * np.outer(k[t], v[t]))
                assert np.abs(y[t_end - 1] - St.T @ q[t_end - 1]).max() <= 1e-13
            assert np.abs(ST - St).max() <= 1e-13


def test_exact_rational_recurrence():
    """Brute force in exact rational arithmetic (fractions) on a 3x2 state:
    the oracle's double result must equal the exact one to rounding."""
    rng = np.random.default_rng(14)
    T, dk, dv = 6, 3, 2
    # Pythagorean unit keys make |k| = 1 exactly representable as fractions
    keys = [(Fraction(3, 5), Fraction(4, 5), Fraction(0)), (Fraction(0), Fraction(1), Fraction(0)),
            (Fraction(2, 3), Fraction(1, 3), Fraction(2, 3)), (Fraction(1), Fraction(0), Fraction(0)),
            (Fraction(0), Fraction(3, 5), Fraction(-4, 5)), (Fraction(-2, 3), Fraction(2, 3), Fraction(1, 3))]
    qs = [keys[(t + 2) % T] for t in range(T)]
    vs = [(Fraction(int(a), 4), Fraction(int(b), 8)) for a, b in rng.integers(-9, 9, (T, 2))]
    al = [Fraction(int(x), 16) for x in rng.integers(1, 17, T)]
    be = [Fraction(int(x), 8) for x in rng.integers(0, 9, T)]
    S = [[Fraction(int(x), 2) for x in row] for row in rng.integers(-3, 4, (dk, dv))]
    S0 = np.array([[float(x) for x in row] for row in S])
    ys = []
    for t in range(T):
        k, v, q = keys[t], vs[t], qs[t]
        S = [[al[t] * S[i][j] for j in range(dv)] for i in range(dk)]
        e = [v[j] - sum(S[i][j] * k[i] for i in range(dk)) for j in range(dv)]
        S = [[S[i][j] + be[t] * k[i] * e[j] for j in range(dv)] for i in range(dk)]
        ys.append([sum(S[i][j] * q[i] for i in range(dk)) for j in range(dv)])
    f = lambda rows: np.array([[float(x) for x in r] for r in rows])
    y, ST = oracle.delta_rule(f(qs), f(keys), f(vs), [float(a) for a in al], [float(b) for b in be], S0)
    assert np.abs(ST - f(S)).max() <= 1e-14
    assert np.abs(y - f(ys)).max() <= 1e-14


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"][:40])
def test_golden_hand_derived_cases(case):
    y, S = oracle.delta_rule(np.array(case["q"], float), np.array(case["k"], float),
                             np.array(case["v"], float), case["alpha"], case["beta"],
                             np.array(case["S0"], float))
    assert np.allclose(y, case["y"], rtol=0, atol=1e-14)
    assert np.allclose(S, case["S_final"], rtol=0, atol=1e-14)


def test_alpha_one_beta_zero_leaves_state_bit_exact():
    rng = np.random.default_rng(15)
    S0 = rng.standard_normal((16, 8))
    q, k = _unit(rng, 10, 16), _unit(rng, 10, 16)
    v = rng.standard_normal((10, 8))
    _, S = oracle.delta_rule(q, k, v, np.ones(10), np.zeros(10), S0)
    assert np.array_equal(S, S0)


def test_full_write_reads_back_value_for_any_alpha():
    """beta = 1 and unit k give S_t^T k_t = v_t exactly (for alpha = 1 as the pages
    state, and in fact for any alpha under the erase-then-write form)."""
    rng = np.random.default_rng(16)
    dk, dv = 32, 16
    S = rng.standard_normal((dk, dv))
    for t in range(30):
        k = _unit(rng, 1, dk)
        v = rng.standard_normal((1, dv))
        alpha = 1.0 if t % 2 == 0 else rng.uniform(0.01, 1.0)
        _, S = oracle.delta_rule(k, k, v, [alpha], [1.0], S)
        assert np.abs(S.T @ k[0] - v[0]).max() <= 1e-13


def test_associative_memory_with_orthonormal_keys():
    """alpha = 1, beta = 1, S0 = 0 and orthonormal keys: S = sum_j k_j v_j^T and
    querying k_j returns v_j (the textbook linear associative memory)."""
    rng = np.random.default_rng(17)
    dk, dv, m = 16, 8, 12
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Qm[:, :m].T.copy()
    vals = rng.standard_normal((m, dv))
    y, S = oracle.delta_rule(keys, keys, vals, np.ones(m), np.ones(m), np.zeros((dk, dv)))
    assert np.allclose(S, keys.T @ vals, atol=1e-13)
    assert np.allclose(keys @ S, vals, atol=1e-13)
    assert np.allclose(y, vals, atol=1e-13)


def test_beta_zero_gives_product_of_decays_closed_form():
    """beta = 0 (b logit -> -inf): S_T = (prod_t alpha_t) S0, with
    alpha_t = exp(-e^A softplus(a_t + b_alpha)) = (1 + e^(a_t + b_alpha))^(-e^A)."""
    rng = np.random.default_rng(18)
    T, H, d = 12, 2, 8
    q = rng.standard_normal((T, H, d)).astype(np.float32)
    a = rng.standard_normal((T, H)).astype(np.float32)
    b = np.full((T, H), -1e30, np.float32)
    A = np.log(np.array([1.5, 0.25], np.float32))
    ba = np.array([0.1, -0.3], np.float32)
    S0 = rng.standard_normal((1, H, d, d)).astype(np.float32)
    conv_w = rng.standard_normal((H * 3 * d, 4)).astype(np.float32)
    _, SF = oracle.prefill(q, q, q, conv_w, a, b, A, ba, q, np.zeros(d, np.float32), S0=S0)
    for h in range(H):
        e_A = np.exp(np.float64(A[h]))
        alpha = (1.0 + np.exp(a[:, h].astype(np.float64) + np.float64(ba[h]))) ** (-e_A)
        assert np.allclose(SF[0, h], np.prod(alpha) * S0[0, h], rtol=1e-12, atol=0)


def test_prefill_with_identity_gates_keeps_state_bit_exact():
    rng = np.random.default_rng(19)
    T, H, d = 9, 3, 4
    x = rng.standard_normal((T, H, d)).astype(np.float32)
    huge = np.full((T, H), -1e30, np.float32)
    S0 = rng.standard_normal((1, H, d, d)).astype(np.float32)
    _, SF = oracle.prefill(x, x, x, rng.standard_normal((H * 3 * d, 4)).astype(np.float32),
                           huge, huge, np.zeros(H, np.float32), np.zeros(H, np.float32), x,
                           np.zeros(d, np.float32), S0=S0)
    assert np.array_equal(SF, S0.astype(np.float64))


# ------------------------------------------------------- prelude and output

def test_prelude_matches_library_convolution_and_closed_forms():
    rng = np.random.default_rng(20)
    T, H, dk, dv, K = 37, 3, 8, 6, 4
    q = rng.standard_normal((T, H, dk)).astype(np.float32)
    k = rng.standard_normal((T, H, dk)).astype(np.float32)
    v = rng.standard_normal((T, H, dv)).astype(np.float32)
    a = rng.standard_normal((T, H)).astype(np.float32)
    b = rng.standard_normal((T, H)).astype(np.float32)
    C = H * (2 * dk + dv)
    w = rng.standard_normal((C, K)).astype(np.float32)
    A = np.log(rng.uniform(1, 16, H)).astype(np.float32)
    ba = rng.standard_normal(H).astype(np.float32)
    silu = lambda u: u * expit(u)
    for h in range(H):
        qh, kh, vh, al, be = oracle.prelude(q, k, v, w, a, b, A, ba, h)
        chans = [(q, h * dk + np.arange(dk), qh, True), (k, H * dk + h * dk + np.arange(dk), kh, True),
                 (v, 2 * H * dk + h * dv + np.arange(dv), vh, False)]
        for src, ch, got, norm in chans:
            d = got.shape[1]
            ref = np.zeros((T, d))
            for i in range(d):
                x = src[:, h, i].astype(np.float64)
                ref[:, i] = np.convolve(x, w[ch[i]].astype(np.float64)[::-1])[:T]
            ref = silu(ref)
            if norm:
                ref = ref / np.sqrt((ref ** 2).sum(1, keepdims=True) + 1e-6)
            assert np.allclose(got, ref, rtol=1e-12, atol=1e-14)
        ref_alpha = np.exp(-np.exp(np.float64(A[h])) *
                           np.logaddexp(0.0, a[:, h].astype(np.float64) + np.float64(ba[h])))
        assert np.allclose(al, ref_alpha, rtol=1e-13, atol=0)
        assert np.allclose(be, expit(b[:, h].astype(np.float64)), rtol=1e-14, atol=0)


def test_decay_gate_special_values():
    """A = log 2, a = 0, b_alpha = 0: alpha = (1 + 1)^(-2) = 1/4; A = 0: alpha = 1/2."""
    T, H, d = 1, 2, 4
    z = np.zeros((T, H, d), np.float32)
    _, _, _, al0, be0 = oracle.prelude(z, z, z, np.zeros((H * 3 * d, 4), np.float32),
                                       np.zeros((T, H), np.float32), np.zeros((T, H), np.float32),
                                       np.array([np.log(2.0), 0.0], np.float32),
                                       np.zeros(H, np.float32), 0)
    _, _, _, al1, _ = oracle.prelude(z, z, z, np.zeros((H * 3 * d, 4), np.float32),
                                     np.zeros((T, H), np.float32), np.zeros((T, H), np.float32),
                                     np.array([np.log(2.0), 0.0], np.float32),
                                     np.zeros(H, np.float32), 1)
    assert abs(al0[0] - 0.25) < 1e-7          # A = log 2 held in fp32
    assert al1[0] == 0.5
    assert be0[0] == 0.5


def test_shortconv_shift_and_identity_taps():
    """Weights (0,0,0,1) pass the current token; (1,0,0,0) delay by K-1 = 3 with
    zeros before the sequence start."""
    rng = np.random.default_rng(21)
    T, H, d = 10, 1, 4
    x = rng.standard_normal((T, H, d)).astype(np.float32)
    zeros = np.zeros((T, H), np.float32)
    for taps, shift in (((0, 0, 0, 1), 0), ((1, 0, 0, 0), 3), ((0, 1, 0, 0), 2)):
        w = np.tile(np.array(taps, np.float32), (3 * d, 1))
        _, _, vh, _, _ = oracle.prelude(x, x, x, w, zeros, zeros, np.zeros(1, np.float32),
                                        np.zeros(1, np.float32), 0)
        src = np.zeros((T, d))
        src[shift:] = x[:T - shift, 0].astype(np.float64)
        assert np.allclose(vh, src * expit(src), rtol=1e-14, atol=0)


def test_l2norm_and_zero_vector():
    rng = np.random.default_rng(22)
    T, d = 5, 16
    x = rng.standard_normal((T, 1, d)).astype(np.float32)
    w = np.tile(np.array([0, 0, 0, 1], np.float32), (3 * d, 1))
    zeros = np.zeros((T, 1), np.float32)
    qh, _, vh, _, _ = oracle.prelude(x, x, x, w, zeros, zeros, np.zeros(1, np.float32),
                                     np.zeros(1, np.float32), 0)
    n2 = (vh ** 2).sum(1)
    assert np.allclose((qh ** 2).sum(1), n2 / (n2 + 1e-6), rtol=1e-13)
    cos = (qh * vh).sum(1) / np.sqrt((qh ** 2).sum(1) * n2)
    assert np.allclose(cos, 1.0, rtol=1e-13)
    z = np.zeros((2, 1, d), np.float32)
    qz, _, _, _, _ = oracle.prelude(z, z, z, w, zeros[:2], zeros[:2], np.zeros(1, np.float32),
                                    np.zeros(1, np.float32), 0)
    assert np.array_equal(qz, np.zeros_like(qz))


def test_gated_rmsnorm_closed_forms():
    rng = np.random.default_rng(23)
    n, dv = 7, 32
    y = rng.standard_normal((n, dv))
    big = np.full((n, dv), 60.0)              # sigmoid(60) == 1 in double to 1e-26
    o = oracle.gated_rmsnorm(y, big, np.zeros(dv, np.float32))
    ms = (y ** 2).mean(1)
    assert np.allclose(np.sqrt((o ** 2).mean(1)), np.sqrt(ms / (ms + 1e-6)), rtol=1e-13)
    w = rng.standard_normal(dv).astype(np.float32)
    z = rng.standard_normal((n, dv))
    o2 = oracle.gated_rmsnorm(y, z, w)
    ref = expit(z) * y / np.sqrt(ms + 1e-6)[:, None] * (1.0 + w.astype(np.float64))
    assert np.allclose(o2, ref, rtol=1e-13, atol=1e-15)
    e1 = np.zeros((1, dv)); e1[0, 3] = -2.0
    o3 = oracle.gated_rmsnorm(e1, np.full((1, dv), 60.0), np.zeros(dv, np.float32))
    assert np.isclose(o3[0, 3], -2.0 / np.sqrt(4.0 / dv + 1e-6), rtol=1e-14)


# -------------------------------------------------- composition and batching

def _rand_inputs(rng, T, H, dk, dv, dtype=np.float32):
    f = lambda *s: rng.standard_normal(s).astype(np.float32)
    return dict(q=f(T, H, dk), k=f(T, H, dk), v=f(T, H, dv), z=f(T, H, dv),
                conv_w=(0.5 * f(H * (2 * dk + dv), 4)), a_logit=f(T, H), b_logit=f(T, H),
                A=np.log(rng.uniform(1, 16, H)).astype(np.float32), b_alpha=0.3 * f(H),
                norm_w=0.1 * f(dv))


def test_prefill_is_prelude_then_recurrence_then_output():
    rng = np.random.default_rng(24)
    T, H, dk, dv = 23, 2, 8, 4
    d = _rand_inputs(rng, T, H, dk, dv)
    S0 = rng.standard_normal((1, H, dk, dv)).astype(np.float32)
    out, SF = oracle.prefill(**d, S0=S0)
    for h in range(H):
        qh, kh, vh, al, be = oracle.prelude(d["q"], d["k"], d["v"], d["conv_w"], d["a_logit"],
                                            d["b_logit"], d["A"], d["b_alpha"], h)
        y, S = oracle.delta_rule(qh, kh, vh, al, be, S0[0, h].astype(np.float64))
        o = oracle.gated_rmsnorm(y, d["z"][:, h].astype(np.float64), d["norm_w"])
        assert np.array_equal(out[:, h], o)
        assert np.array_equal(SF[0, h], S)


def test_packed_varlen_equals_sequences_run_alone():
    rng = np.random.default_rng(25)
    lens = [5, 1, 17, 3, 9]
    H, dk, dv = 2, 8, 8
    N = sum(lens)
    d = _rand_inputs(rng, N, H, dk, dv)
    S0 = rng.standard_normal((len(lens), H, dk, dv)).astype(np.float32)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    out, SF = oracle.prefill(**d, S0=S0, cu_seqlens=cu)
    for n in range(len(lens)):
        sl = slice(cu[n], cu[n + 1])
        dn = {key: (val[sl] if val.ndim >= 2 and val.shape[0] == N else val) for key, val in d.items()}
        o1, s1 = oracle.prefill(**dn, S0=S0[n:n + 1])
        assert np.array_equal(out[sl], o1)
        assert np.array_equal(SF[n], s1[0])


def test_bf16_inputs_are_widened_exactly():
    rng = np.random.default_rng(26)
    T, H, d = 11, 2, 8
    f32 = _rand_inputs(rng, T, H, d, d)
    def to_bf16_bits(x):
        u = x.astype(np.float32).view(np.uint32)
        return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    def from_bits(b):
        return (b.astype(np.uint32) << 16).view(np.float32)
    bits = {key: to_bf16_bits(f32[key]) for key in ("q", "k", "v", "z", "a_logit", "b_logit")}
    wid = {key: from_bits(val) for key, val in bits.items()}
    rest = {key: f32[key] for key in ("conv_w", "A", "b_alpha", "norm_w")}
    o_b, s_b = oracle.prefill(**bits, **rest)
    o_f, s_f = oracle.prefill(**wid, **rest)
    assert np.array_equal(o_b, o_f) and np.array_equal(s_b, s_f)


def test_decode_steps_equal_prefill():
    """T decode steps from an empty history equal a prefill of T tokens, and the
    history ends holding the last K-1 raw tokens, oldest first."""
    rng = np.random.default_rng(27)
    T, B, H, dk, dv, K = 9, 3, 2, 8, 4, 4
    C = H * (2 * dk + dv)
    seqs = [_rand_inputs(rng, T, H, dk, dv) for _ in range(B)]
    shared = {key: seqs[0][key] for key in ("conv_w", "A", "b_alpha", "norm_w")}
    for s in seqs:
        s.update(shared)
    S0 = rng.standard_normal((B, H, dk, dv)).astype(np.float32)
    hist = np.zeros((B, K - 1, C), np.float32)
    S = S0.astype(np.float64).copy()
    outs = []
    for t in range(T):
        g = lambda key: np.stack([s[key][t] for s in seqs])
        outs.append(oracle.decode_step(g("q"), g("k"), g("v"), shared["conv_w"], hist,
                                       g("a_logit"), g("b_logit"), shared["A"],
                                       shared["b_alpha"], g("z"), shared["norm_w"], S))
    for b in range(B):
        o_ref, s_ref = oracle.prefill(**seqs[b], S0=S0[b:b + 1])
        got = np.stack([outs[t][b] for t in range(T)])
        assert np.allclose(got, o_ref, rtol=1e-12, atol=1e-13)
        assert np.allclose(S[b], s_ref[0], rtol=1e-12, atol=1e-13)
        raw = np.concatenate([seqs[b]["q"].reshape(T, -1), seqs[b]["k"].reshape(T, -1),
                              seqs[b]["v"].reshape(T, -1)], axis=1)
        # channel order [q heads | k heads | v heads] matches the (T, H, d) reshapes
        for j in range(K - 1):
            assert np.array_equal(hist[b, j], raw[T - (K - 1) + j])
