"""Thin Python binding of the C ABI in include/gdn.h (argument marshalling only).

Every step of the mixer runs in the CUDA library ``libgdn.so`` built in-tree by
``build.py``; this module only checks tensor placement, allocates outputs with
PyTorch and passes raw device pointers and the current CUDA stream.  There is
no fallback: if the library is missing or a tensor is not on a CUDA device the
call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdn.so")

GDN_F32, GDN_BF16 = 0, 1
STATUS = {0: "GDN_OK", 1: "GDN_ERR_INVALID_ARG", 2: "GDN_ERR_UNSUPPORTED", 3: "GDN_ERR_ALIGNMENT",
          4: "GDN_ERR_CUDA", 5: "GDN_ERR_TIMEOUT"}

# Every function the header declares (checked by the tests).
EXPORTS = ("gdn_prefill", "gdn_prefill_workspace_size", "gdn_decode_step", "gdn_status_string",
           "gdn_set_timing_events", "gdn_selftest_umma", "gdn_prefill_noalloc",
           "gdn_set_kernel_events", "gdn_last_call_launches", "gdn_last_call_slots",
           "gdn_device_error_status",
           "gdn_selftest_wait_timeout", "gdn_decode_multi", "gdn_prefill_backward",
           "gdn_prefill_backward_workspace_size", "gdn_qsa_indexer", "gdn_qsa_indexer_workspace_size",
           "gdn_layer_forward", "gdn_layer_workspace_size", "gdn_prefill_ws", "gdn_prefill_conv_tail",
           "gdn_gemm_bf16")
ERRF_PREP, ERRF_CHAIN, ERRF_DECODE, ERRF_QSA, ERRF_GEMM = 1, 2, 4, 8, 16


class GdnError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}")
        self.status = status


class Dims(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int32), ("total_tokens", ctypes.c_int32),
                ("H", ctypes.c_int32), ("dk", ctypes.c_int32), ("dv", ctypes.c_int32),
                ("conv_k", ctypes.c_int32), ("in_dtype", ctypes.c_int32),
                ("out_dtype", ctypes.c_int32)]


_lib = None


def load() -> ctypes.CDLL:
    """Load libgdn.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing "
                               "(run linear_attention_token_shortconv_b200/build.py)")
        lib = ctypes.CDLL(LIB_PATH)
        P, D = ctypes.c_void_p, ctypes.POINTER(Dims)
        lib.gdn_prefill.argtypes = [D] + [P] * 15
        lib.gdn_prefill.restype = ctypes.c_int
        lib.gdn_prefill_workspace_size.argtypes = [D, ctypes.POINTER(ctypes.c_size_t)]
        lib.gdn_prefill_workspace_size.restype = ctypes.c_int
        lib.gdn_decode_step.argtypes = [D] + [P] * 14
        lib.gdn_decode_step.restype = ctypes.c_int
        lib.gdn_decode_multi.argtypes = [D, ctypes.c_int] + [P] * 15
        lib.gdn_decode_multi.restype = ctypes.c_int
        lib.gdn_prefill_backward.argtypes = [D] + [P] * 26
        lib.gdn_prefill_backward.restype = ctypes.c_int
        lib.gdn_prefill_backward_workspace_size.argtypes = [D, ctypes.POINTER(ctypes.c_size_t)]
        lib.gdn_prefill_backward_workspace_size.restype = ctypes.c_int
        lib.gdn_qsa_indexer.argtypes = [ctypes.c_int] * 6 + [P] * 7
        lib.gdn_qsa_indexer.restype = ctypes.c_int
        lib.gdn_qsa_indexer_workspace_size.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t)]
        lib.gdn_qsa_indexer_workspace_size.restype = ctypes.c_int
        lib.gdn_layer_forward.argtypes = [D, ctypes.c_int] + [P] * 12
        lib.gdn_layer_forward.restype = ctypes.c_int
        lib.gdn_layer_workspace_size.argtypes = [D, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t)]
        lib.gdn_layer_workspace_size.restype = ctypes.c_int
        lib.gdn_gemm_bf16.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, P, ctypes.c_int, P, ctypes.c_int, P,
                                      ctypes.c_int, P]
        lib.gdn_gemm_bf16.restype = ctypes.c_int
        lib.gdn_prefill_noalloc.argtypes = [D] + [P] * 15
        lib.gdn_prefill_noalloc.restype = ctypes.c_int
        lib.gdn_selftest_umma.argtypes = [ctypes.c_int] * 5 + [P] * 5
        lib.gdn_selftest_umma.restype = ctypes.c_int
        lib.gdn_set_timing_events.argtypes = [P, P]
        lib.gdn_set_timing_events.restype = ctypes.c_int
        lib.gdn_set_kernel_events.argtypes = [ctypes.POINTER(P), ctypes.POINTER(P), ctypes.c_int]
        lib.gdn_set_kernel_events.restype = ctypes.c_int
        lib.gdn_last_call_launches.argtypes = []
        lib.gdn_last_call_launches.restype = ctypes.c_int
        lib.gdn_last_call_slots.argtypes = []
        lib.gdn_last_call_slots.restype = ctypes.c_int
        lib.gdn_device_error_status.argtypes = [ctypes.POINTER(ctypes.c_uint), ctypes.c_int, P]
        lib.gdn_device_error_status.restype = ctypes.c_int
        lib.gdn_selftest_wait_timeout.argtypes = [ctypes.c_uint, ctypes.c_uint, P]
        lib.gdn_selftest_wait_timeout.restype = ctypes.c_int
        lib.gdn_status_string.argtypes = [ctypes.c_int]
        lib.gdn_status_string.restype = ctypes.c_char_p
        lib.gdn_prefill_ws.argtypes = [D] + [P] * 15 + [ctypes.c_size_t, P]
        lib.gdn_prefill_ws.restype = ctypes.c_int
        lib.gdn_prefill_conv_tail.argtypes = [D] + [P] * 6
        lib.gdn_prefill_conv_tail.restype = ctypes.c_int
        _lib = lib
    return _lib


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    if t.dtype == torch.float32:
        return GDN_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("all tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("all tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


F32, BF16, I32 = torch.float32, torch.bfloat16, torch.int32


def _expect(name, t, shape, dtypes):
    """Raises unless tensor `t` (None: absent, accepted) has this shape (None entries:
    any size) and one of these dtypes.  The library sees only raw pointers, so a
    mismatch here would otherwise be read as other bytes, or past the tensor."""
    if t is None:
        return
    dtypes = dtypes if isinstance(dtypes, tuple) else (dtypes,)
    if t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {' or '.join(str(d) for d in dtypes)}")
    if t.dim() != len(shape) or any(w is not None and n != w for n, w in zip(t.shape, shape)):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")


def _device(*ts):
    """The one CUDA device that every given tensor (None entries skipped) is on;
    the call runs there."""
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("all tensors must live on a CUDA device")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"tensors on {dev} and {t.device}: all must be on one device")
    return dev


def _check_mixer(q, k, v, conv_w, a_logit, b_logit, A, b_alpha, z, norm_w, S0, cu_seqlens, out, S_final,
                 n_seq, io=None, names=("out", "S_final")):
    """Shapes and dtypes of the mixer's arguments in the packed token layout
    (`names`: what the caller calls its out and S_final slots)."""
    if q.dim() != 3 or v.dim() != 3 or conv_w.dim() != 2:
        raise ValueError("q, k [N_tok, H, dk], v, z [N_tok, H, dv] and conv_w [C, K] expected")
    n_tok, H, dk = q.shape
    dv, K = v.shape[2], conv_w.shape[1]
    io = (BF16, F32) if io is None else io
    _expect("q", q, (n_tok, H, dk), io)
    for name, t, shape in (("k", k, (n_tok, H, dk)), ("v", v, (n_tok, H, dv)), ("z", z, (n_tok, H, dv)),
                           ("a_logit", a_logit, (n_tok, H)), ("b_logit", b_logit, (n_tok, H))):
        _expect(name, t, shape, q.dtype)
    _expect("conv_w", conv_w, (H * (2 * dk + dv), K), F32)
    _expect("A", A, (H,), F32)
    _expect("b_alpha", b_alpha, (H,), F32)
    _expect("norm_w", norm_w, (dv,), F32)
    _expect("S0", S0, (n_seq, H, dk, dv), F32)
    _expect("cu_seqlens", cu_seqlens, (n_seq + 1,), I32)
    _expect(names[0], out, (n_tok, H, dv), (F32, BF16))
    _expect(names[1], S_final, (n_seq, H, dk, dv), F32)


def _check(rc: int, where: str):
    if rc != 0:
        raise GdnError(rc, where)


def prefill(q, k, v, conv_w, a_logit, b_logit, A, b_alpha, z, norm_w, S0=None, cu_seqlens=None,
            *, num_seqs=None, out=None, S_final=None, out_dtype=torch.float32, want_state=True,
            stream=None):
    """gdn_prefill on torch tensors.  q,k [N_tok,H,dk]; v,z [N_tok,H,dv]; a,b [N_tok,H].

    Returns (out [N_tok,H,dv], S_final [N_seq,H,dk,dv] or None)."""
    n_tok, H, dk = q.shape
    dv = v.shape[2]
    if cu_seqlens is not None:
        n_seq = cu_seqlens.shape[0] - 1
    else:
        n_seq = num_seqs if num_seqs is not None else (S0.shape[0] if S0 is not None else 1)
    if out is None:
        out = torch.empty((n_tok, H, dv), dtype=out_dtype, device=q.device)
    if S_final is None and want_state:
        S_final = torch.empty((n_seq, H, dk, dv), dtype=torch.float32, device=q.device)
    _check_mixer(q, k, v, conv_w, a_logit, b_logit, A, b_alpha, z, norm_w, S0, cu_seqlens, out, S_final, n_seq)
    dims = Dims(n_seq, n_tok, H, dk, dv, conv_w.shape[1], _dt(q), _dt(out))
    with torch.cuda.device(_device(q, k, v, conv_w, a_logit, b_logit, A, b_alpha, z, norm_w, S0, cu_seqlens,
                                   out, S_final)):
        rc = load().gdn_prefill(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(conv_w),
                                _ptr(a_logit), _ptr(b_logit), _ptr(A), _ptr(b_alpha), _ptr(z),
                                _ptr(norm_w), _ptr(S0), _ptr(cu_seqlens), _ptr(out), _ptr(S_final),
                                _stream(stream))
    _check(rc, "gdn_prefill")
    return out, S_final


def prefill_backward(q, k, v, conv_w, a_logit, b_logit, A, b_alpha, z, norm_w, d_out, S0=None,
                     d_S_final=None, cu_seqlens=None, *, num_seqs=None, want_d_S0=True, stream=None):
    """gdn_prefill_backward on fp32 torch tensors (same layouts as `prefill`).

    Returns a dict of fp32 tensors: dq, dk, dv, d_conv_w, d_a_logit, d_b_logit,
    d_A, d_b_alpha, d_z, d_norm_w and d_S0 (None unless wanted)."""
    n_tok, H, dk = q.shape
    dv = v.shape[2]
    if cu_seqlens is not None:
        n_seq = cu_seqlens.shape[0] - 1
    else:
        n_seq = num_seqs if num_seqs is not None else (S0.shape[0] if S0 is not None else 1)
    dev, f32 = q.device, torch.float32
    g = {"dq": torch.empty_like(q), "dk": torch.empty_like(k), "dv": torch.empty_like(v),
         "d_conv_w": torch.empty_like(conv_w), "d_a_logit": torch.empty_like(a_logit),
         "d_b_logit": torch.empty_like(b_logit), "d_A": torch.empty_like(A),
         "d_b_alpha": torch.empty_like(b_alpha), "d_z": torch.empty_like(z),
         "d_norm_w": torch.empty_like(norm_w),
         "d_S0": torch.empty((n_seq, H, dk, dv), dtype=f32, device=dev) if want_d_S0 else None}
    _check_mixer(q, k, v, conv_w, a_logit, b_logit, A, b_alpha, z, norm_w, S0, cu_seqlens, d_out, d_S_final,
                 n_seq, names=("d_out", "d_S_final"))
    _expect("d_out", d_out, (n_tok, H, dv), q.dtype)
    dims = Dims(n_seq, n_tok, H, dk, dv, conv_w.shape[1], _dt(q), _dt(d_out))
    with torch.cuda.device(_device(q, k, v, conv_w, a_logit, b_logit, A, b_alpha, z, norm_w, S0, cu_seqlens,
                                   d_out, d_S_final)):
        rc = load().gdn_prefill_backward(
            ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(conv_w), _ptr(a_logit), _ptr(b_logit),
            _ptr(A), _ptr(b_alpha), _ptr(z), _ptr(norm_w), _ptr(S0), _ptr(cu_seqlens), _ptr(d_out),
            _ptr(d_S_final), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["d_conv_w"]),
            _ptr(g["d_a_logit"]), _ptr(g["d_b_logit"]), _ptr(g["d_A"]), _ptr(g["d_b_alpha"]), _ptr(g["d_z"]),
            _ptr(g["d_norm_w"]), _ptr(g["d_S0"]), _stream(stream))
    _check(rc, "gdn_prefill_backward")
    return g


def prefill_backward_workspace_size(n_seq, n_tok, H, dk, dv, conv_k=4) -> int:
    dims = Dims(n_seq, n_tok, H, dk, dv, conv_k, GDN_F32, GDN_F32)
    n = ctypes.c_size_t(0)
    _check(load().gdn_prefill_backward_workspace_size(ctypes.byref(dims), ctypes.byref(n)),
           "gdn_prefill_backward_workspace_size")
    return n.value


def qsa_indexer(q, k, w_q, w_k, budget=2048, *, sel=None, scores=None, want_scores=False, stream=None):
    """gdn_qsa_indexer on torch tensors: q [B, n, 4, 128] and k [B, n, 128] bf16
    (a leading batch dimension may be omitted), w_q, w_k [128] fp32.

    Returns (sel [B, n, budget / 4] int32, scores [B, n, n / 4] fp32 or None)."""
    squeeze = q.dim() == 3
    if squeeze:
        q, k = q.unsqueeze(0), k.unsqueeze(0)
    if q.dim() != 4:
        raise ValueError("q [B, n, heads, d] (or [n, heads, d]) expected")
    B, n, H, d = q.shape
    if sel is None:
        sel = torch.empty((B, n, budget // 4), dtype=torch.int32, device=q.device)
    if scores is None and want_scores:
        scores = torch.empty((B, n, n // 4), dtype=torch.float32, device=q.device)
    _expect("q", q, (B, n, H, d), BF16)
    _expect("k", k, (B, n, d), BF16)
    _expect("w_q", w_q, (d,), F32)
    _expect("w_k", w_k, (d,), F32)
    _expect("sel", sel, (B, n, budget // 4), I32)
    _expect("scores", scores, (B, n, n // 4), F32)
    with torch.cuda.device(_device(q, k, w_q, w_k, sel, scores)):
        rc = load().gdn_qsa_indexer(B, n, H, d, 4, budget, _ptr(q), _ptr(k), _ptr(w_q), _ptr(w_k), _ptr(sel),
                                    _ptr(scores), _stream(stream))
    _check(rc, "gdn_qsa_indexer")
    if squeeze:
        sel = sel[0]
        scores = None if scores is None else scores[0]
    return sel, scores


def gemm_bf16(a, b, *, out=None, stream=None):
    """gdn_gemm_bf16 on torch tensors: a [M, K], b [K, N] bf16 (row-major views
    whose last dimension is contiguous) -> out [M, N] bf16."""
    M, K = a.shape
    K2, N = b.shape
    if K2 != K:
        raise ValueError(f"gemm_bf16: inner dimensions {K} and {K2}")
    for name, t in (("a", a), ("b", b)):
        if t.dtype != BF16 or t.device.type != "cuda" or t.stride(1) != 1:
            raise ValueError(f"gemm_bf16: {name} must be a bf16 CUDA matrix with contiguous rows")
    if out is None:
        out = torch.empty((M, N), dtype=BF16, device=a.device)
    if out.shape != (M, N) or out.dtype != BF16 or out.stride(1) != 1:
        raise ValueError("gemm_bf16: out must be a bf16 [M, N] matrix with contiguous rows")
    def mat_ptr(t):   # a row-strided matrix: rows need not be adjacent
        return ctypes.c_void_p(t.data_ptr()) if t.numel() else None

    with torch.cuda.device(_device(a, b, out)):
        rc = load().gdn_gemm_bf16(M, N, K, mat_ptr(a), a.stride(0), mat_ptr(b), b.stride(0), mat_ptr(out),
                                  out.stride(0), _stream(stream))
    _check(rc, "gdn_gemm_bf16")
    return out


def layer_forward(x, w_in, conv_w, A, b_alpha, norm_w, w_o, H, dk, dv, S0=None, cu_seqlens=None, *,
                  num_seqs=None, y=None, S_final=None, want_state=True, stream=None):
    """gdn_layer_forward on torch tensors: x [N_tok, d_model], w_in [d_model,
    H(2dk + 2dv) + 2H], w_o [H dv, d_model], all bf16.

    Returns (y [N_tok, d_model] bf16, S_final [N_seq, H, dk, dv] fp32 or None)."""
    n_tok, d_model = x.shape
    if cu_seqlens is not None:
        n_seq = cu_seqlens.shape[0] - 1
    else:
        n_seq = num_seqs if num_seqs is not None else (S0.shape[0] if S0 is not None else 1)
    if y is None:
        y = torch.empty((n_tok, d_model), dtype=torch.bfloat16, device=x.device)
    if S_final is None and want_state:
        S_final = torch.empty((n_seq, H, dk, dv), dtype=torch.float32, device=x.device)
    _expect("x", x, (n_tok, d_model), BF16)
    _expect("w_in", w_in, (d_model, H * (2 * dk + 2 * dv) + 2 * H), BF16)
    _expect("w_o", w_o, (H * dv, d_model), BF16)
    _expect("conv_w", conv_w, (H * (2 * dk + dv), None), F32)
    _expect("A", A, (H,), F32)
    _expect("b_alpha", b_alpha, (H,), F32)
    _expect("norm_w", norm_w, (dv,), F32)
    _expect("S0", S0, (n_seq, H, dk, dv), F32)
    _expect("cu_seqlens", cu_seqlens, (n_seq + 1,), I32)
    _expect("y", y, (n_tok, d_model), BF16)
    _expect("S_final", S_final, (n_seq, H, dk, dv), F32)
    dims = Dims(n_seq, n_tok, H, dk, dv, conv_w.shape[1], GDN_BF16, GDN_BF16)
    with torch.cuda.device(_device(x, w_in, conv_w, A, b_alpha, norm_w, w_o, S0, cu_seqlens, y, S_final)):
        rc = load().gdn_layer_forward(ctypes.byref(dims), d_model, _ptr(x), _ptr(w_in), _ptr(conv_w), _ptr(A),
                                      _ptr(b_alpha), _ptr(norm_w), _ptr(w_o), _ptr(S0), _ptr(cu_seqlens),
                                      _ptr(y), _ptr(S_final), _stream(stream))
    _check(rc, "gdn_layer_forward")
    return y, S_final


def prefill_noalloc(q, k, v, conv_w, a_logit, b_logit, A, b_alpha, z, norm_w, S0=None,
                    cu_seqlens=None, *, num_seqs=None, out=None, S_final=None,
                    out_dtype=torch.float32, want_state=True, stream=None):
    """gdn_prefill_noalloc on torch tensors: the tensor-core prefill with its
    workspace in the library's fixed device array (for callers that cannot
    allocate while running the layer; the outputs here are still allocated by
    torch when not supplied).  Same arguments and results as `prefill`."""
    n_tok, H, dk = q.shape
    dv = v.shape[2]
    if cu_seqlens is not None:
        n_seq = cu_seqlens.shape[0] - 1
    else:
        n_seq = num_seqs if num_seqs is not None else (S0.shape[0] if S0 is not None else 1)
    if out is None:
        out = torch.empty((n_tok, H, dv), dtype=out_dtype, device=q.device)
    if S_final is None and want_state:
        S_final = torch.empty((n_seq, H, dk, dv), dtype=torch.float32, device=q.device)
    _check_mixer(q, k, v, conv_w, a_logit, b_logit, A, b_alpha, z, norm_w, S0, cu_seqlens, out, S_final, n_seq)
    dims = Dims(n_seq, n_tok, H, dk, dv, conv_w.shape[1], _dt(q), _dt(out))
    with torch.cuda.device(_device(q, k, v, conv_w, a_logit, b_logit, A, b_alpha, z, norm_w, S0, cu_seqlens,
                                   out, S_final)):
        rc = load().gdn_prefill_noalloc(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(conv_w),
                                        _ptr(a_logit), _ptr(b_logit), _ptr(A), _ptr(b_alpha), _ptr(z),
                                        _ptr(norm_w), _ptr(S0), _ptr(cu_seqlens), _ptr(out),
                                        _ptr(S_final), _stream(stream))
    _check(rc, "gdn_prefill_noalloc")
    return out, S_final


def prefill_ws(q, k, v, conv_w, a_logit, b_logit, A, b_alpha, z, norm_w, workspace, S0=None,
               cu_seqlens=None, *, num_seqs=None, out=None, S_final=None, out_dtype=torch.float32,
               want_state=True, stream=None):
    """gdn_prefill_ws on torch tensors: `prefill` with the workspace supplied as a
    uint8 CUDA tensor of at least prefill_workspace_size() bytes."""
    n_tok, H, dk = q.shape
    dv = v.shape[2]
    if cu_seqlens is not None:
        n_seq = cu_seqlens.shape[0] - 1
    else:
        n_seq = num_seqs if num_seqs is not None else (S0.shape[0] if S0 is not None else 1)
    if out is None:
        out = torch.empty((n_tok, H, dv), dtype=out_dtype, device=q.device)
    if S_final is None and want_state:
        S_final = torch.empty((n_seq, H, dk, dv), dtype=torch.float32, device=q.device)
    _check_mixer(q, k, v, conv_w, a_logit, b_logit, A, b_alpha, z, norm_w, S0, cu_seqlens, out, S_final, n_seq)
    if workspace.dtype != torch.uint8 or workspace.dim() != 1:
        raise ValueError("workspace: a 1-D uint8 tensor expected")
    dims = Dims(n_seq, n_tok, H, dk, dv, conv_w.shape[1], _dt(q), _dt(out))
    with torch.cuda.device(_device(q, k, v, conv_w, a_logit, b_logit, A, b_alpha, z, norm_w, S0, cu_seqlens,
                                   out, S_final, workspace)):
        rc = load().gdn_prefill_ws(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(conv_w),
                                   _ptr(a_logit), _ptr(b_logit), _ptr(A), _ptr(b_alpha), _ptr(z),
                                   _ptr(norm_w), _ptr(S0), _ptr(cu_seqlens), _ptr(out), _ptr(S_final),
                                   _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "gdn_prefill_ws")
    return out, S_final


def prefill_conv_tail(q, k, v, cu_seqlens=None, *, num_seqs=None, conv_hist=None, stream=None):
    """gdn_prefill_conv_tail on torch tensors: the decode conv history
    [N_seq, 3, H(2dk+dv)] (q.dtype) that continues each prefilled sequence."""
    n_tok, H, dk = q.shape
    dv = v.shape[2]
    n_seq = cu_seqlens.shape[0] - 1 if cu_seqlens is not None else (num_seqs or 1)
    _expect("k", k, (n_tok, H, dk), q.dtype)
    _expect("v", v, (n_tok, H, dv), q.dtype)
    _expect("cu_seqlens", cu_seqlens, (n_seq + 1,), I32)
    if conv_hist is None:
        conv_hist = torch.empty((n_seq, 3, H * (2 * dk + dv)), dtype=q.dtype, device=q.device)
    _expect("conv_hist", conv_hist, (n_seq, 3, H * (2 * dk + dv)), q.dtype)
    dims = Dims(n_seq, n_tok, H, dk, dv, 4, _dt(q), _dt(q))
    with torch.cuda.device(_device(q, k, v, cu_seqlens, conv_hist)):
        rc = load().gdn_prefill_conv_tail(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens),
                                          _ptr(conv_hist), _stream(stream))
    _check(rc, "gdn_prefill_conv_tail")
    return conv_hist


def prefill_workspace_size(n_seq, n_tok, H, dk, dv, conv_k=4, in_dtype=torch.bfloat16,
                           out_dtype=torch.float32) -> int:
    dims = Dims(n_seq, n_tok, H, dk, dv, conv_k,
                GDN_BF16 if in_dtype == torch.bfloat16 else GDN_F32,
                GDN_BF16 if out_dtype == torch.bfloat16 else GDN_F32)
    n = ctypes.c_size_t(0)
    _check(load().gdn_prefill_workspace_size(ctypes.byref(dims), ctypes.byref(n)),
           "gdn_prefill_workspace_size")
    return int(n.value)


def decode_step(q, k, v, conv_w, conv_hist, a_logit, b_logit, A, b_alpha, z, norm_w, S, *,
                out=None, out_dtype=torch.float32, stream=None):
    """gdn_decode_step on torch tensors; updates conv_hist and S in place, returns out."""
    B, H, dk = q.shape
    dv = v.shape[2]
    if out is None:
        out = torch.empty((B, H, dv), dtype=out_dtype, device=q.device)
    K = conv_w.shape[1]
    C = H * (2 * dk + dv)
    _expect("q", q, (B, H, dk), (BF16, F32))
    for name, t, shape in (("k", k, (B, H, dk)), ("v", v, (B, H, dv)), ("z", z, (B, H, dv)),
                           ("conv_hist", conv_hist, (B, K - 1, C)), ("a_logit", a_logit, (B, H)),
                           ("b_logit", b_logit, (B, H))):
        _expect(name, t, shape, q.dtype)
    _expect("conv_w", conv_w, (C, K), F32)
    _expect("A", A, (H,), F32)
    _expect("b_alpha", b_alpha, (H,), F32)
    _expect("norm_w", norm_w, (dv,), F32)
    _expect("S", S, (B, H, dk, dv), F32)
    _expect("out", out, (B, H, dv), (F32, BF16))
    dims = Dims(B, B, H, dk, dv, K, _dt(q), _dt(out))
    with torch.cuda.device(_device(q, k, v, conv_w, conv_hist, a_logit, b_logit, A, b_alpha, z, norm_w, S, out)):
        rc = load().gdn_decode_step(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(conv_w),
                                    _ptr(conv_hist), _ptr(a_logit), _ptr(b_logit), _ptr(A),
                                    _ptr(b_alpha), _ptr(z), _ptr(norm_w), _ptr(S), _ptr(out),
                                    _stream(stream))
    _check(rc, "gdn_decode_step")
    return out


def decode_multi(q, k, v, conv_w, conv_hist, a_logit, b_logit, A, b_alpha, z, norm_w, S, *,
                 n_keep=None, out=None, out_dtype=torch.float32, stream=None):
    """gdn_decode_multi on torch tensors: q, k [B, T, H, dk]; v, z [B, T, H, dv];
    a_logit, b_logit [B, T, H].  Returns out [B, T, H, dv]; conv_hist and S
    advance in place by n_keep[b] tokens (int32 [B] CUDA tensor; None = all T)."""
    B, T, H, dk = q.shape
    dv = v.shape[3]
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=out_dtype, device=q.device)
    K = conv_w.shape[1]
    C = H * (2 * dk + dv)
    _expect("q", q, (B, T, H, dk), (BF16, F32))
    for name, t, shape in (("k", k, (B, T, H, dk)), ("v", v, (B, T, H, dv)), ("z", z, (B, T, H, dv)),
                           ("conv_hist", conv_hist, (B, K - 1, C)), ("a_logit", a_logit, (B, T, H)),
                           ("b_logit", b_logit, (B, T, H))):
        _expect(name, t, shape, q.dtype)
    _expect("conv_w", conv_w, (C, K), F32)
    _expect("A", A, (H,), F32)
    _expect("b_alpha", b_alpha, (H,), F32)
    _expect("norm_w", norm_w, (dv,), F32)
    _expect("S", S, (B, H, dk, dv), F32)
    _expect("out", out, (B, T, H, dv), (F32, BF16))
    _expect("n_keep", n_keep, (B,), I32)
    dims = Dims(B, B * T, H, dk, dv, K, _dt(q), _dt(out))
    with torch.cuda.device(_device(q, k, v, conv_w, conv_hist, a_logit, b_logit, A, b_alpha, z, norm_w, S, out,
                                   n_keep)):
        rc = load().gdn_decode_multi(ctypes.byref(dims), T, _ptr(q), _ptr(k), _ptr(v), _ptr(conv_w),
                                     _ptr(conv_hist), _ptr(a_logit), _ptr(b_logit), _ptr(A), _ptr(b_alpha),
                                     _ptr(z), _ptr(norm_w), _ptr(S), _ptr(out), _ptr(n_keep),
                                     _stream(stream))
    _check(rc, "gdn_decode_multi")
    return out


def set_timing_events(begin=None, end=None):
    """Record torch.cuda.Event `begin`/`end` around the dominant kernel of each
    following call (None, None clears the hook)."""
    b = None if begin is None else ctypes.c_void_p(begin.cuda_event)
    e = None if end is None else ctypes.c_void_p(end.cuda_event)
    _check(load().gdn_set_timing_events(b, e), "gdn_set_timing_events")


def set_kernel_events(begins=(), ends=()):
    """Record torch.cuda.Event begins[i] / ends[i] around launch slot i of each
    following call (slot order: prep/chain per segment for a prefill, the
    kernel for a decode step); empty sequences clear the hook.  The events must
    have been recorded once so that their CUDA handles exist."""
    if len(begins) != len(ends):
        raise ValueError("begins and ends differ in length")
    n = len(begins)
    arr = ctypes.c_void_p * max(n, 1)
    b = arr(*[e.cuda_event for e in begins])
    e = arr(*[x.cuda_event for x in ends])
    _check(load().gdn_set_kernel_events(b, e, n), "gdn_set_kernel_events")


def last_call_launches() -> int:
    """Kernels launched by this thread's most recent prefill / decode call."""
    return int(load().gdn_last_call_launches())


def last_call_slots() -> int:
    """Launch slots (event-bracketed kernels or kernel groups) of the same call."""
    return int(load().gdn_last_call_slots())


def device_error_status(clear=False, stream=None):
    """(status, flags): the current device's error words as a GDN_ERRF_* mask
    after the work queued on `stream`; status is GDN_ERR_TIMEOUT (5) when any
    flag is set.  Clears the words when `clear`."""
    flags = ctypes.c_uint(0)
    st = load().gdn_device_error_status(ctypes.byref(flags), int(bool(clear)), _stream(stream))
    if st not in (0, 5):
        raise GdnError(st, "gdn_device_error_status")
    return st, flags.value


def selftest_wait_timeout(family, max_polls=1024, stream=None):
    """Launch one CTA whose bounded wait (kernel family `family`) runs out."""
    _check(load().gdn_selftest_wait_timeout(family, max_polls, _stream(stream)),
           "gdn_selftest_wait_timeout")


def selftest_umma(A, B, init=None, *, a_mn=False, b_mn=False, negate_a=False, stream=None):
    """D = init + (+/-A) B computed on the tensor cores with the given operand
    layouts (A [128,K], B [K,N] fp16 CUDA tensors): a_mn 0 / 1 = A K-major /
    MN-major in shared memory, 2 = A in tensor memory; b_mn likewise for B."""
    M, K = A.shape
    N = B.shape[1]
    if M != 128 or B.shape[0] != K or A.dtype != torch.float16 or B.dtype != torch.float16:
        raise ValueError("A must be [128, K] and B [K, N], both fp16")
    D = torch.empty((128, N), dtype=torch.float32, device=A.device)
    rc = load().gdn_selftest_umma(int(a_mn), int(b_mn), int(negate_a), N, K, _ptr(A), _ptr(B),
                                  _ptr(init), _ptr(D), _stream(stream))
    _check(rc, "gdn_selftest_umma")
    return D


def status_string(status: int) -> str:
    return load().gdn_status_string(int(status)).decode()
