"""fp64 CPU oracle of the Gated DeltaNet token mixer -- TEST INFRASTRUCTURE.

Only the tests, the smoke check in the package entry file and bench.py's
CPU-baseline leg may import this module.  It wraps ``gdn_oracle.c`` (plain C,
double precision, token by token) through ctypes and numpy; it shares no code
with the CUDA path and never imports it.

Array conventions: bf16 inputs are passed as ``np.uint16`` bit patterns, fp32
inputs as ``np.float32``; results come back as ``np.float64``.
"""
import ctypes
import os

import numpy as np

from . import build as _build

F32, BF16 = 0, 1
_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        _lib = ctypes.CDLL(path)
        vp, ip, dp, fp = ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p
        _lib.gdn_oracle_prefill.argtypes = [ip] * 7 + [vp] * 14 + [ip]
        _lib.gdn_oracle_prefill.restype = ip
        _lib.gdn_oracle_decode_step.argtypes = [ip] * 6 + [vp] * 13 + [ip]
        _lib.gdn_oracle_decode_step.restype = ip
        _lib.gdn_oracle_delta_rule.argtypes = [ip] * 3 + [dp] * 7
        _lib.gdn_oracle_delta_rule.restype = ip
        _lib.gdn_oracle_prelude.argtypes = [ip] * 6 + [vp] * 8 + [ip] + [dp] * 5
        _lib.gdn_oracle_prelude.restype = ip
        _lib.gdn_oracle_gated_rmsnorm.argtypes = [ip, ip, dp, dp, fp, dp]
        _lib.gdn_oracle_gated_rmsnorm.restype = ip
        _lib.gdn_oracle_backward.argtypes = [ip] * 7 + [vp] * 25 + [ip]
        _lib.gdn_oracle_backward.restype = ip
        _lib.gdn_oracle_threads.argtypes = [ip]
        _lib.gdn_oracle_threads.restype = ip
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dtype_code(a):
    if a.dtype == np.uint16:
        return BF16
    if a.dtype == np.float32:
        return F32
    raise TypeError(f"oracle inputs must be bf16 bits (uint16) or float32, got {a.dtype}")


def _c(a, dt=None):
    if a is None:
        return None
    a = np.asarray(a)
    return np.ascontiguousarray(a if dt is None else a.astype(dt, copy=False))


def threads(n_threads: int = 0) -> int:
    """OpenMP threads the oracle uses for a given request (0 = library default)."""
    return lib().gdn_oracle_threads(int(n_threads))


def prefill(q, k, v, conv_w, a_logit, b_logit, A, b_alpha, z, norm_w, S0=None,
            cu_seqlens=None, num_seqs=None, n_threads=0):
    """Token-by-token fp64 prefill.  q,k [N_tok,H,dk]; v,z [N_tok,H,dv]; a,b [N_tok,H].

    Returns (out [N_tok,H,dv] float64, S_final [N_seq,H,dk,dv] float64).
    """
    q, k, v, z, a_logit, b_logit = (_c(x) for x in (q, k, v, z, a_logit, b_logit))
    dt = _dtype_code(q)
    for x in (k, v, z, a_logit, b_logit):
        if _dtype_code(x) != dt:
            raise TypeError("all token inputs must share one dtype")
    n_tok, H, dk = q.shape
    dv = v.shape[2]
    conv_w = _c(conv_w, np.float32)
    K = conv_w.shape[1]
    A, b_alpha, norm_w = _c(A, np.float32), _c(b_alpha, np.float32), _c(norm_w, np.float32)
    if cu_seqlens is not None:
        cu_seqlens = _c(cu_seqlens, np.int32)
        n_seq = cu_seqlens.shape[0] - 1
    else:
        n_seq = 1 if num_seqs is None else int(num_seqs)
    S0 = _c(S0, np.float32)
    out = np.zeros((n_tok, H, dv), np.float64)
    S_final = np.zeros((n_seq, H, dk, dv), np.float64)
    rc = lib().gdn_oracle_prefill(n_seq, n_tok, H, dk, dv, K, dt, _ptr(q), _ptr(k), _ptr(v),
                                  _ptr(conv_w), _ptr(a_logit), _ptr(b_logit), _ptr(A),
                                  _ptr(b_alpha), _ptr(z), _ptr(norm_w), _ptr(S0),
                                  _ptr(cu_seqlens), _ptr(out), _ptr(S_final), int(n_threads))
    if rc != 0:
        raise ValueError("oracle prefill rejected its arguments")
    return out, S_final


def decode_step(q, k, v, conv_w, hist, a_logit, b_logit, A, b_alpha, z, norm_w, S,
                n_threads=0):
    """One fp64 decode step.  ``hist`` (raw conv history [B,K-1,C], oldest first,
    input dtype) and ``S`` (float64 [B,H,dk,dv]) are updated IN PLACE; returns
    out [B,H,dv]."""
    q, k, v, z, a_logit, b_logit = (_c(x) for x in (q, k, v, z, a_logit, b_logit))
    dt = _dtype_code(q)
    B, H, dk = q.shape
    dv = v.shape[2]
    conv_w = _c(conv_w, np.float32)
    K = conv_w.shape[1]
    for name, arr, want in (("hist", hist, q.dtype), ("S", S, np.float64)):
        if arr.dtype != want or not arr.flags["C_CONTIGUOUS"]:
            raise TypeError(f"{name} must be a C-contiguous {np.dtype(want)} array")
    A, b_alpha, norm_w = _c(A, np.float32), _c(b_alpha, np.float32), _c(norm_w, np.float32)
    out = np.zeros((B, H, dv), np.float64)
    rc = lib().gdn_oracle_decode_step(B, H, dk, dv, K, dt, _ptr(q), _ptr(k), _ptr(v),
                                      _ptr(conv_w), _ptr(hist), _ptr(a_logit),
                                      _ptr(b_logit), _ptr(A), _ptr(b_alpha), _ptr(z),
                                      _ptr(norm_w), _ptr(S), _ptr(out), int(n_threads))
    if rc != 0:
        raise ValueError("oracle decode rejected its arguments")
    return out


def delta_rule(q, k, v, alpha, beta, S0):
    """The recurrence alone on prepared fp64 vectors; returns (y [T,dv], S [dk,dv])."""
    q, k, v, alpha, beta = (_c(x, np.float64) for x in (q, k, v, alpha, beta))
    S = np.array(S0, dtype=np.float64, order="C", copy=True)
    T, dk = q.shape
    dv = v.shape[1]
    y = np.zeros((T, dv), np.float64)
    rc = lib().gdn_oracle_delta_rule(T, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                                     _ptr(beta), _ptr(S), _ptr(y))
    if rc != 0:
        raise ValueError("bad sizes")
    return y, S


def prelude(q, k, v, conv_w, a_logit, b_logit, A, b_alpha, h):
    """Prelude of head h for one sequence (all tokens of the given arrays).

    Returns (q_hat [T,dk], k_hat [T,dk], v_hat [T,dv], alpha [T], beta [T]) in fp64."""
    q, k, v, a_logit, b_logit = (_c(x) for x in (q, k, v, a_logit, b_logit))
    dt = _dtype_code(q)
    T, H, dk = q.shape
    dv = v.shape[2]
    conv_w = _c(conv_w, np.float32)
    K = conv_w.shape[1]
    A, b_alpha = _c(A, np.float32), _c(b_alpha, np.float32)
    qh, kh = np.zeros((T, dk)), np.zeros((T, dk))
    vh, al, be = np.zeros((T, dv)), np.zeros(T), np.zeros(T)
    rc = lib().gdn_oracle_prelude(T, H, dk, dv, K, dt, _ptr(q), _ptr(k), _ptr(v), _ptr(conv_w),
                                  _ptr(a_logit), _ptr(b_logit), _ptr(A), _ptr(b_alpha), int(h),
                                  _ptr(qh), _ptr(kh), _ptr(vh), _ptr(al), _ptr(be))
    if rc != 0:
        raise ValueError("bad sizes")
    return qh, kh, vh, al, be


def gated_rmsnorm(y, z, w):
    """Output stage alone on rows of dv: sigmoid(z) * RMSNorm(y) * (1 + w)."""
    y, z = _c(y, np.float64), _c(z, np.float64)
    w = _c(w, np.float32)
    n, dv = y.shape
    o = np.zeros_like(y)
    rc = lib().gdn_oracle_gated_rmsnorm(n, dv, _ptr(y), _ptr(z), _ptr(w), _ptr(o))
    if rc != 0:
        raise ValueError("bad sizes")
    return o


def backward(q, k, v, conv_w, a_logit, b_logit, A, b_alpha, z, norm_w, d_out, S0=None,
             d_S_final=None, cu_seqlens=None, num_seqs=None, n_threads=0):
    """Token-by-token fp64 gradients of <d_out, out> + <d_S_final, S_final> with
    respect to every prefill input (same layouts as :func:`prefill`).

    Returns a dict of float64 arrays: dq, dk, dv, d_conv_w, d_a_logit, d_b_logit,
    d_A, d_b_alpha, d_z, d_norm_w, d_S0."""
    q, k, v, z, a_logit, b_logit = (_c(x) for x in (q, k, v, z, a_logit, b_logit))
    dt = _dtype_code(q)
    for x in (k, v, z, a_logit, b_logit):
        if _dtype_code(x) != dt:
            raise TypeError("all token inputs must share one dtype")
    n_tok, H, dk = q.shape
    dv = v.shape[2]
    conv_w = _c(conv_w, np.float32)
    K = conv_w.shape[1]
    A, b_alpha, norm_w = _c(A, np.float32), _c(b_alpha, np.float32), _c(norm_w, np.float32)
    if cu_seqlens is not None:
        cu_seqlens = _c(cu_seqlens, np.int32)
        n_seq = cu_seqlens.shape[0] - 1
    else:
        n_seq = 1 if num_seqs is None else int(num_seqs)
    S0 = _c(S0, np.float32)
    d_out = _c(d_out, np.float64)
    d_S_final = _c(d_S_final, np.float64)
    g = {"dq": np.zeros((n_tok, H, dk)), "dk": np.zeros((n_tok, H, dk)), "dv": np.zeros((n_tok, H, dv)),
         "d_conv_w": np.zeros(conv_w.shape), "d_a_logit": np.zeros((n_tok, H)),
         "d_b_logit": np.zeros((n_tok, H)), "d_A": np.zeros(H), "d_b_alpha": np.zeros(H),
         "d_z": np.zeros((n_tok, H, dv)), "d_norm_w": np.zeros(dv), "d_S0": np.zeros((n_seq, H, dk, dv))}
    rc = lib().gdn_oracle_backward(
        n_seq, n_tok, H, dk, dv, K, dt, _ptr(q), _ptr(k), _ptr(v), _ptr(conv_w), _ptr(a_logit),
        _ptr(b_logit), _ptr(A), _ptr(b_alpha), _ptr(z), _ptr(norm_w), _ptr(S0), _ptr(cu_seqlens),
        _ptr(d_out), _ptr(d_S_final), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["d_conv_w"]),
        _ptr(g["d_a_logit"]), _ptr(g["d_b_logit"]), _ptr(g["d_A"]), _ptr(g["d_b_alpha"]), _ptr(g["d_z"]),
        _ptr(g["d_norm_w"]), _ptr(g["d_S0"]), int(n_threads))
    if rc != 0:
        raise ValueError("oracle backward rejected its arguments")
    return g
