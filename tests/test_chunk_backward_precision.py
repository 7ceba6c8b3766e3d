"""Which tensor-core operand precision a chunked backward can use (fp64 emulation,
CPU), at the head size of the workloads (d = 128, chunks of 64).

Every matrix product of the chunked backward algebra (test_chunk_backward_algebra.py)
runs with its operands rounded the way a `tcgen05.mma` would see them, the
result rounded to fp32 (the accumulator), and the state and its gradient kept in
fp32 between chunks. Two schemes are compared against fp64:
- one fp16 (or tf32) product per matrix product: about 5e-4 normwise, outside
  the 2e-5 that the SIMT backward holds;
- each operand scaled by a power of two (exact) and split into fp16 hi + lo, with
  three products hi*hi + hi*lo + lo*hi: about 2e-7, at the level of plain fp32
  arithmetic. The scale keeps small gradients, such as a state gradient that
  short-memory decays have shrunk far below fp16's range, from flushing.
"""
import numpy as np
import pytest

from test_chunk_backward_algebra import chunked_delta_rule_backward


def _f32(x):
    return np.asarray(x, np.float64).astype(np.float32).astype(np.float64)


def _f16(x):
    return np.asarray(x, np.float64).astype(np.float16).astype(np.float64)


def _tf32(x):
    u = np.ascontiguousarray(np.asarray(x, np.float64).astype(np.float32)).view(np.uint32).astype(np.uint64)
    u = ((u + 0xFFF + ((u >> 13) & 1)) >> 13) << 13               # 10 mantissa bits, ties to even
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def mm_single(rnd):
    return lambda a, b: _f32(rnd(a) @ rnd(b))


def mm_split16_scaled(a, b):
    ma, mb = np.abs(a).max(), np.abs(b).max()
    if ma == 0 or mb == 0:
        return np.zeros((a.shape[0], b.shape[1]))
    sa, sb = 2.0 ** -np.floor(np.log2(ma)), 2.0 ** -np.floor(np.log2(mb))
    a, b = a * sa, b * sb
    ah, bh = _f16(a), _f16(b)
    al, bl = _f16(a - ah), _f16(b - bh)
    return _f32(_f32(ah @ bh + ah @ bl + al @ bh) / (sa * sb))


def _case(T, memory, seed, d=128):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, d)); q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = rng.standard_normal((T, d)); k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, d))
    if memory == "short":      # the workloads' gates: A = log U[1, 16], logits N(0, 1)
        g = -rng.uniform(1, 16) * np.logaddexp(0, rng.standard_normal(T))
    else:                      # alpha about 0.99
        g = -rng.uniform(0.01, 0.1) * np.logaddexp(0, rng.standard_normal(T) - 2)
    beta = 1 / (1 + np.exp(-rng.standard_normal(T)))
    return (q, k, v, g, beta, np.sqrt(0.02) * rng.standard_normal((d, d)), 64,
            rng.standard_normal((T, d)), rng.standard_normal((d, d)))


def _worst(args, mm):
    ref = chunked_delta_rule_backward(*args)
    got = chunked_delta_rule_backward(*args, mm=mm, keep=_f32)
    return max(np.abs(g - r).max() / np.abs(r).max() for g, r in zip(got, ref))


@pytest.mark.parametrize("memory", ["short", "long"])
def test_split_fp16_products_hold_fp32_accuracy(memory):
    args = _case(256, memory, 5)
    assert _worst(args, mm_split16_scaled) <= 2e-6
    plain = _worst(args, mm_single(_f32))
    assert plain <= 1e-6          # fp32 operands: the floor the split should reach


@pytest.mark.parametrize("memory", ["short", "long"])
def test_single_products_do_not(memory):
    args = _case(256, memory, 5)
    for rnd in (_f16, _tf32):
        e = _worst(args, mm_single(rnd))
        assert 5e-5 < e < 5e-3, e
