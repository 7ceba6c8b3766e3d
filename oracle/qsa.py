"""fp64 CPU oracle of the QSA compressed indexer -- TEST INFRASTRUCTURE.

Only the tests, the smoke check in the package entry file and bench.py's
CPU-baseline leg may import this module; it shares no code with the CUDA path.

What it follows (slinene.github.io write-up of "On the Design of Qwen3.8-Next
Architecture", 模块 B — Qwen Sparse Attention, "压缩轻量 indexer" and the block
selection paragraph):
  * queries: per indexer head h (H = 4, MQA), q_hat = RMSNorm(W_Q^h x_i); one
    shared key k_i = W_K x_i (the projections are the inputs here);
  * keys are cut into non-overlapping blocks of r tokens, averaged, then
    RMS-normalised: k_hat_b = RMSNorm(mean(k_{rb .. rb+r-1})), b < floor(n / r);
  * the positional rotation comes after the pooling: q = PRoPE(q_hat, i),
    k_bar_b = PRoPE(k_hat_b, r b) (the block's start position); partial RoPE
    rotates 64 of the 128 dims;
  * block score I_ib = sum_h ReLU(<q_i^h, k_bar_b>) for blocks already complete
    at i (r b + r - 1 <= i), -inf otherwise;
  * B_i = the K_B = ceil(K / r) highest-scoring blocks; the token set is the
    blocks expanded back to tokens plus the tail r floor((i + 1) / r) .. i.

Readings where the page is silent (listed in the design notes): RMSNorm is
x / sqrt(mean(x^2) + 1e-6) times a weight vector ([128], one for the queries
shared by the heads, one for the keys); PRoPE is the rotate-half rotation of
dims [0, 64) -- pairs (j, j + 32), angle p * 10000^(-j / 32) -- and dims
[64, 128) pass through; ties in the top-K_B are broken towards the smaller
block index; B_i is returned in ascending order, padded with -1 when fewer
than K_B blocks are complete.
"""
import numpy as np

EPS = 1e-6
ROPE_DIMS = 64
ROPE_BASE = 10000.0


def rmsnorm(x, w):
    """x / sqrt(mean(x^2) + eps) * w over the last axis."""
    x = np.asarray(x, np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + EPS) * np.asarray(w, np.float64)


def prope(x, pos, dims=ROPE_DIMS, base=ROPE_BASE):
    """Partial RoPE: rotate-half rotation of x[..., :dims] at positions `pos`
    (broadcast over the leading axes of x[..., 0]); the other dims unchanged."""
    x = np.array(x, np.float64)
    half = dims // 2
    inv = base ** (-np.arange(half, dtype=np.float64) / half)
    ang = np.asarray(pos, np.float64)[..., None] * inv
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., :half].copy(), x[..., half:dims].copy()
    x[..., :half] = a * c - b * s
    x[..., half:dims] = a * s + b * c
    return x


def keys(k_raw, w_k, r=4):
    """Compressed keys k_bar [floor(n / r), d]: pool, normalise, then rotate at r b."""
    k = np.asarray(k_raw, np.float64)
    nb = k.shape[0] // r
    pooled = k[:nb * r].reshape(nb, r, k.shape[1]).mean(axis=1)
    return prope(rmsnorm(pooled, w_k), np.arange(nb) * r)


def queries(q_raw, w_q):
    """Rotated queries [n, H, d]: normalise per head, rotate at the token position."""
    q = rmsnorm(q_raw, w_q)
    n = q.shape[0]
    return prope(q, np.arange(n)[:, None] * np.ones(q.shape[1]))


def scores(q_raw, k_raw, w_q, w_k, r=4):
    """I [n, floor(n / r)]: sum over heads of ReLU(<q_i^h, k_bar_b>); -inf where
    block b is not complete at token i."""
    q = queries(q_raw, w_q)
    kb = keys(k_raw, w_k, r)
    s = np.maximum(q @ kb.T, 0.0).sum(axis=1)            # [n, H, nb] -> [n, nb]
    n, nb = s.shape
    complete = (np.arange(nb)[None, :] * r + r - 1) <= np.arange(n)[:, None]
    return np.where(complete, s, -np.inf)


def select(I, K=2048, r=4):
    """B [n, ceil(K / r)] int32: per row the highest-scoring complete blocks, ties
    to the smaller index, in ascending order, padded with -1."""
    n, nb = I.shape
    kb = -(-K // r)
    out = np.full((n, kb), -1, np.int32)
    for i in range(n):
        valid = np.flatnonzero(np.isfinite(I[i]))
        order = sorted(valid.tolist(), key=lambda b: (-I[i, b], b))
        chosen = sorted(order[:kb])
        out[i, :len(chosen)] = chosen
    return out


def indexer(q_raw, k_raw, w_q, w_k, K=2048, r=4):
    """The whole indexer: returns (B [n, K_B] int32, I [n, floor(n / r)] float64)."""
    I = scores(q_raw, k_raw, w_q, w_k, r)
    return select(I, K, r), I


def expand(B_row, i, K=2048, r=4):
    """Token set of query i: the selected blocks expanded to tokens (at most K)
    and the tail r floor((i + 1) / r) .. i."""
    toks = [b * r + j for b in B_row if b >= 0 for j in range(r)][:K]
    tail = list(range(r * ((i + 1) // r), i + 1))
    return sorted(set(toks) | set(tail))
