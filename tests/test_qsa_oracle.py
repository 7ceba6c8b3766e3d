"""Pins of the QSA indexer oracle (CPU): closed forms of RMSNorm and partial
RoPE, the pool-then-rotate order, the block-causal mask, the selection against
a library sort and the tie rule, a constructed case with a known answer, and
the token expansion with its tail."""
import numpy as np
import pytest

from oracle import qsa


def test_rmsnorm_closed_form():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 128)) * 3.0
    y = qsa.rmsnorm(x, np.ones(128))
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-6)
    np.testing.assert_allclose(qsa.rmsnorm(7.0 * x, np.ones(128)), y, rtol=1e-6)
    w = rng.standard_normal(128)
    np.testing.assert_allclose(qsa.rmsnorm(x, w), y * w, rtol=1e-12)


def test_rmsnorm_epsilon():
    # mean(x^2) = eps exactly: the normalised vector has RMS sqrt(eps / (2 eps)) = 1 / sqrt(2)
    x = np.full(128, np.sqrt(qsa.EPS))
    y = qsa.rmsnorm(x, np.ones(128))
    np.testing.assert_allclose(np.sqrt(np.mean(y * y)), np.sqrt(0.5), rtol=1e-12)
    assert qsa.EPS == 1e-6


def test_prope_basis_vectors():
    # e_j (j < 32) at position p turns in the plane (j, j + 32) by p * 10000^(-j/32)
    for j, p in ((0, 5), (1, 3), (31, 1000)):
        x = np.zeros(128)
        x[j] = 1.0
        y = qsa.prope(x, p)
        th = p * 10000.0 ** (-j / 32.0)
        want = np.zeros(128)
        want[j], want[j + 32] = np.cos(th), np.sin(th)
        np.testing.assert_allclose(y, want, atol=1e-12)
    x = np.zeros(128)
    x[40] = 1.0      # second half of the rotated dims: (j + 32) -> -sin, cos
    th = 9 * 10000.0 ** (-8 / 32.0)
    want = np.zeros(128)
    want[8], want[40] = -np.sin(th), np.cos(th)
    np.testing.assert_allclose(qsa.prope(x, 9), want, atol=1e-12)


def test_prope_invariants():
    rng = np.random.default_rng(1)
    x, y = rng.standard_normal(128), rng.standard_normal(128)
    for p in (0, 17, 123456):
        np.testing.assert_allclose(np.linalg.norm(qsa.prope(x, p)), np.linalg.norm(x), rtol=1e-12)
        np.testing.assert_array_equal(qsa.prope(x, p)[64:], x[64:])   # dims 64..127 pass through
    np.testing.assert_allclose(qsa.prope(x, 0), x, atol=0)
    # a rotary product depends only on the position difference
    a = qsa.prope(x, 40) @ qsa.prope(y, 12)
    b = qsa.prope(x, 128) @ qsa.prope(y, 100)
    c = qsa.prope(x, 28) @ y
    np.testing.assert_allclose([a, b], [c, c], rtol=1e-10)


def test_keys_pool_then_rotate():
    rng = np.random.default_rng(2)
    r, nb = 4, 6
    c = rng.standard_normal((nb, 128))
    k = np.repeat(c, r, axis=0)                       # constant within each block
    w = rng.uniform(0.5, 1.5, 128)
    want = np.stack([qsa.prope(qsa.rmsnorm(c[b], w), r * b) for b in range(nb)])
    np.testing.assert_allclose(qsa.keys(k, w, r), want, rtol=1e-12)
    # with varying tokens the order matters: rotating each token, then pooling differs
    k2 = rng.standard_normal((nb * r, 128))
    pooled_first = qsa.keys(k2, np.ones(128), r)
    rot_first = np.stack([qsa.rmsnorm(np.mean([qsa.prope(k2[b * r + j], b * r + j) for j in range(r)], axis=0),
                                      np.ones(128)) for b in range(nb)])
    assert np.abs(pooled_first[1:, :64] - rot_first[1:, :64]).max() > 1e-2
    # a trailing partial block has no compressed key
    assert qsa.keys(rng.standard_normal((4 * 3 + 2, 128)), np.ones(128), 4).shape == (3, 128)


def test_block_causal_mask():
    rng = np.random.default_rng(3)
    n = 23
    I = qsa.scores(rng.standard_normal((n, 4, 128)), rng.standard_normal((n, 128)), np.ones(128), np.ones(128))
    assert I.shape == (n, n // 4)
    for i in range(n):
        for b in range(n // 4):
            assert np.isfinite(I[i, b]) == (4 * b + 3 <= i), (i, b)
    assert np.all(I[np.isfinite(I)] >= 0)                 # sums of ReLUs


def test_score_is_relu_sum_over_heads():
    rng = np.random.default_rng(4)
    n = 12
    q = rng.standard_normal((n, 4, 128))
    k = rng.standard_normal((n, 128))
    qr, kb = qsa.queries(q, np.ones(128)), qsa.keys(k, np.ones(128))
    I = qsa.scores(q, k, np.ones(128), np.ones(128))
    i, b = 11, 1
    dots = [qr[i, h] @ kb[b] for h in range(4)]
    assert I[i, b] == pytest.approx(sum(max(d, 0.0) for d in dots), rel=1e-12)


def test_selection_matches_a_library_sort():
    rng = np.random.default_rng(5)
    n, nb = 400, 100
    I = rng.standard_normal((n, nb))
    I[(np.arange(nb)[None, :] * 4 + 3) > np.arange(n)[:, None]] = -np.inf
    B = qsa.select(I, K=40, r=4)                          # K_B = 10
    for i in range(n):
        valid = np.flatnonzero(np.isfinite(I[i]))
        top = valid[np.argsort(-I[i, valid], kind="stable")][:10]
        want = np.sort(top)
        np.testing.assert_array_equal(B[i, :len(want)], want)
        assert np.all(B[i, len(want):] == -1)


def test_ties_go_to_the_smaller_block():
    n = 64
    q = np.zeros((n, 4, 128))                             # every score is ReLU(0) summed: 0
    B, I = qsa.indexer(q, np.ones((n, 128)), np.ones(128), np.ones(128), K=12, r=4)   # K_B = 3
    for i in range(n):
        n_valid = (i + 1) // 4
        want = list(range(min(3, n_valid)))
        assert B[i, :len(want)].tolist() == want and np.all(B[i, len(want):] == -1)


def test_constructed_winner():
    """Query 40 points at block 6's compressed key and away from every other block:
    with K_B = 1 it selects block 6."""
    rng = np.random.default_rng(6)
    n, r = 48, 4
    k = rng.standard_normal((n, 128))
    kb = qsa.keys(k, np.ones(128), r)
    i, target = 40, 6
    # un-rotate the target key to the query's position, so that <q_i, k_bar_6> = |k_bar_6|^2
    q_hat = qsa.prope(kb[target], -i)
    q = np.zeros((n, 4, 128))
    q[i, 0] = q_hat                                       # one head; RMSNorm only rescales it
    B, I = qsa.indexer(q, k, np.ones(128), np.ones(128), K=4, r=r)
    assert B[i, 0] == target
    assert np.argmax(np.where(np.isfinite(I[i]), I[i], -1)) == target
    # rotated at position i, the normalised query is k_bar_6 / sqrt(mean(k_bar_6^2) + eps),
    # so the score is |k_bar_6|^2 over that root (the other heads are zero: ReLU(0) = 0);
    # rotating the query at position i + 1 instead gives a value about 1% smaller (only
    # the fast pairs turn far), which the 1e-12 closed form tells apart
    kk = kb[target]
    assert I[i, target] == pytest.approx(kk @ kk / np.sqrt(np.mean(kk * kk) + qsa.EPS), rel=1e-12)
    off = qsa.prope(qsa.rmsnorm(q_hat, np.ones(128)), i + 1) @ kk
    assert off < (1 - 1e-3) * I[i, target]


def test_expand_with_tail():
    B = np.array([2, 4, -1])                              # complete blocks at i = 22 are 0 .. 4
    toks = qsa.expand(B, 22, K=8, r=4)
    assert toks == [8, 9, 10, 11, 16, 17, 18, 19, 20, 21, 22]   # two blocks and the tail 20 .. 22
    assert all(t <= 22 for t in toks)
    assert qsa.expand(np.array([0]), 3, K=8, r=4) == [0, 1, 2, 3]   # (i + 1) % r == 0: empty tail
    # at i = 7 block 1 (tokens 4 .. 7) is complete: unless selected it is not in the set
    assert qsa.expand(np.array([0, -1]), 7, K=8, r=4) == [0, 1, 2, 3]
    assert qsa.expand(np.array([0, -1]), 8, K=8, r=4) == [0, 1, 2, 3, 8]
