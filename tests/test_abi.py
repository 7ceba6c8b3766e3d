"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/gdn.h declares, and rejects bad arguments before it
touches CUDA."""
import ctypes
import os
import re

import pytest

from linear_attention_token_shortconv_b200 import gdn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"GDN_API\s+[\w\s\*]*?\b(gdn_\w+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def lib():
    from linear_attention_token_shortconv_b200 import build
    build.build()
    return gdn.load()


def test_library_exports_every_declared_function(lib):
    names = declared_functions()
    assert {"gdn_prefill", "gdn_decode_step", "gdn_status_string"} <= names
    for n in names:
        assert hasattr(lib, n), n
    assert set(gdn.EXPORTS) == names, (set(gdn.EXPORTS) ^ names)


def test_status_strings(lib):
    for code, name in gdn.STATUS.items():
        assert gdn.status_string(code) == name
    assert gdn.status_string(99) == "GDN_ERR_UNKNOWN"


def _dims(**kw):
    base = dict(num_seqs=1, total_tokens=64, H=2, dk=128, dv=128, conv_k=4, in_dtype=1, out_dtype=0)
    base.update(kw)
    return gdn.Dims(**base)


def _prefill(lib, dims, ptrs):
    return lib.gdn_prefill(ctypes.byref(dims) if dims is not None else None, *ptrs)


FAKE = [ctypes.c_void_p(4096 * (i + 1)) for i in range(11)]   # aligned, never dereferenced


def _args(q=FAKE[0], S0=None, cu=None, S_final=None, out=FAKE[10]):
    return [q, FAKE[1], FAKE[2], FAKE[3], FAKE[4], FAKE[5], FAKE[6], FAKE[7], FAKE[8], FAKE[9],
            S0, cu, out, S_final, None]


def test_prefill_argument_validation(lib):
    assert _prefill(lib, None, _args()) == 1
    assert _prefill(lib, _dims(num_seqs=0), _args()) == 1
    assert _prefill(lib, _dims(total_tokens=-1), _args()) == 1
    assert _prefill(lib, _dims(in_dtype=7), _args()) == 1
    assert _prefill(lib, _dims(num_seqs=3, total_tokens=64), _args()) == 1   # not divisible, no cu
    assert _prefill(lib, _dims(dk=96), _args()) == 2
    assert _prefill(lib, _dims(dv=256), _args()) == 2
    assert _prefill(lib, _dims(conv_k=3), _args()) == 2
    assert _prefill(lib, _dims(), _args(q=None)) == 1
    assert _prefill(lib, _dims(), _args(out=None)) == 1
    assert _prefill(lib, _dims(), _args(q=ctypes.c_void_p(4104))) == 3
    assert _prefill(lib, _dims(), _args(S0=ctypes.c_void_p(4100))) == 3
    assert _prefill(lib, _dims(), _args(cu=ctypes.c_void_p(4098))) == 3
    args = _args()
    args[4] = ctypes.c_void_p(4099)   # a_logit: bf16 needs 2-byte alignment
    assert _prefill(lib, _dims(), args) == 3


def test_decode_argument_validation(lib):
    args = [FAKE[i] for i in range(11)] + [ctypes.c_void_p(8192), ctypes.c_void_p(12288), None]
    d = _dims(num_seqs=4, total_tokens=4)
    assert lib.gdn_decode_step(ctypes.byref(_dims(num_seqs=4, total_tokens=5)), *args) == 1
    assert lib.gdn_decode_step(ctypes.byref(_dims(num_seqs=4, total_tokens=4, dk=32)), *args) == 2
    bad = list(args)
    bad[4] = None   # conv history is required
    assert lib.gdn_decode_step(ctypes.byref(d), *bad) == 1
    bad = list(args)
    bad[11] = ctypes.c_void_p(8200)  # S misaligned
    assert lib.gdn_decode_step(ctypes.byref(d), *bad) == 3


def test_workspace_size_query(lib):
    n = gdn.prefill_workspace_size(2, 1000, 4, 128, 64)
    assert n >= 1000 * 4 * (128 + 128 + 64) * 2
    assert gdn.prefill_workspace_size(1, 0, 1, 64, 64) == 0
    with pytest.raises(gdn.GdnError):
        gdn.prefill_workspace_size(1, 10, 1, 48, 64)


def test_kernel_events_hook_validation(lib):
    P = ctypes.c_void_p
    two = (P * 2)(P(16), P(32))
    assert lib.gdn_set_kernel_events(two, two, -1) == 1
    assert lib.gdn_set_kernel_events(None, two, 1) == 1
    holes = (P * 2)(P(16), None)
    assert lib.gdn_set_kernel_events(two, holes, 2) == 1
    assert lib.gdn_set_kernel_events(None, None, 0) == 0     # clears the hook


def test_rejected_calls_launch_nothing(lib):
    assert _prefill(lib, _dims(dk=96), _args()) == 2
    assert lib.gdn_last_call_launches() == 0
    assert lib.gdn_last_call_slots() == 0
    args = [FAKE[i] for i in range(11)] + [ctypes.c_void_p(8192), ctypes.c_void_p(12288), None]
    assert lib.gdn_decode_step(ctypes.byref(_dims(num_seqs=4, total_tokens=5)), *args) == 1
    assert lib.gdn_last_call_launches() == 0


def test_wait_selftest_validation(lib):
    assert lib.gdn_selftest_wait_timeout(32, 16, None) == 1      # not a family bit
    assert lib.gdn_selftest_wait_timeout(3, 16, None) == 1       # two bits
    assert lib.gdn_selftest_wait_timeout(1, 0, None) == 1
    assert lib.gdn_selftest_wait_timeout(1, 65537, None) == 1


def test_decode_multi_argument_validation(lib):
    args = [FAKE[i] for i in range(11)] + [ctypes.c_void_p(8192), ctypes.c_void_p(12288), None, None]
    ok = _dims(num_seqs=4, total_tokens=8, in_dtype=1)               # B = 4, T = 2
    assert lib.gdn_decode_multi(ctypes.byref(ok), 0, *args) == 1      # T outside [1, 4]
    assert lib.gdn_decode_multi(ctypes.byref(ok), 5, *args) == 1
    assert lib.gdn_decode_multi(ctypes.byref(ok), 3, *args) == 1      # total_tokens != B * T
    assert lib.gdn_decode_multi(ctypes.byref(_dims(num_seqs=4, total_tokens=8, dv=64)), 2, *args) == 2
    assert lib.gdn_decode_multi(ctypes.byref(_dims(num_seqs=4, total_tokens=8, in_dtype=0)), 2, *args) == 2
    bad = list(args)
    bad[11] = ctypes.c_void_p(8200)                                   # S misaligned
    assert lib.gdn_decode_multi(ctypes.byref(ok), 2, *bad) == 3
    bad = list(args)
    bad[13] = ctypes.c_void_p(4098)                                   # n_keep misaligned
    assert lib.gdn_decode_multi(ctypes.byref(ok), 2, *bad) == 3
    assert lib.gdn_last_call_launches() == 0


def _bwd_args(**over):
    names = ["q", "k", "v", "conv_w", "a", "b", "A", "b_alpha", "z", "norm_w", "S0", "cu", "d_out", "d_S_final",
             "dq", "dk", "dv", "d_conv_w", "d_a", "d_b", "d_A", "d_b_alpha", "d_z", "d_norm_w", "d_S0", "stream"]
    vals = {n: ctypes.c_void_p(4096 * (i + 1)) for i, n in enumerate(names)}
    for n in ("S0", "cu", "d_S_final", "d_S0", "stream"):
        vals[n] = None
    vals.update(over)
    return [vals[n] for n in names]


def test_backward_argument_validation(lib):
    f32 = dict(in_dtype=0, out_dtype=0)
    bwd = lambda dims, **kw: lib.gdn_prefill_backward(ctypes.byref(dims), *_bwd_args(**kw))
    assert lib.gdn_prefill_backward(None, *_bwd_args()) == 1
    assert bwd(_dims(in_dtype=1, out_dtype=0)) == 2                 # bf16 inputs
    assert bwd(_dims(dk=128, dv=64, **f32)) == 2                     # dk != dv
    assert bwd(_dims(num_seqs=3, total_tokens=64, **f32)) == 1       # not divisible, no cu
    assert bwd(_dims(**f32), q=None) == 1
    assert bwd(_dims(**f32), dq=None) == 1
    assert bwd(_dims(**f32), d_conv_w=None) == 1
    assert bwd(_dims(**f32), d_out=ctypes.c_void_p(4104)) == 3
    assert bwd(_dims(**f32), d_a=ctypes.c_void_p(4098)) == 3
    assert bwd(_dims(**f32), d_S0=ctypes.c_void_p(4100)) == 3
    assert lib.gdn_last_call_launches() == 0


def test_backward_workspace_size_query(lib):
    n = gdn.prefill_backward_workspace_size(2, 1000, 4, 128, 128)
    # q, k, v and their gradients in fp32, plus one 64 KB checkpoint per 16 tokens
    assert n >= 6 * 1000 * 4 * 128 * 4 + (1000 // 16) * 4 * 128 * 128 * 4
    with pytest.raises(gdn.GdnError):
        gdn.prefill_backward_workspace_size(1, 10, 1, 128, 64)


def test_layer_argument_validation(lib):
    P = ctypes.c_void_p
    ptrs = [P(4096 * (i + 1)) for i in range(7)]                  # x, w_in, conv_w, A, b_alpha, norm_w, w_o
    ok = _dims(num_seqs=1, total_tokens=64, in_dtype=1, out_dtype=1)
    call = lambda dims, d_model, y=P(65536), x=ptrs[0]: lib.gdn_layer_forward(
        ctypes.byref(dims) if dims is not None else None, d_model, x, *ptrs[1:], None, None, y, None, None)
    assert call(None, 256) == 1
    assert call(_dims(in_dtype=0, out_dtype=1), 256) == 2            # fp32 activations
    assert call(_dims(in_dtype=1, out_dtype=0), 256) == 2            # fp32 output
    assert call(ok, 0) == 1
    assert call(ok, 260) == 2                                        # d_model not a multiple of 8
    assert call(ok, 256, y=None) == 1
    assert call(ok, 256, x=P(4100)) == 3
    assert lib.gdn_last_call_launches() == 0
    n = ctypes.c_size_t(0)
    assert lib.gdn_layer_workspace_size(ctypes.byref(ok), 256, ctypes.byref(n)) == 0 and n.value > 0


def test_qsa_argument_validation(lib):
    P = ctypes.c_void_p
    q, k, wq, wk, sel = (P(4096 * (i + 1)) for i in range(5))
    call = lambda *dims, q=q, sel=sel: lib.gdn_qsa_indexer(*dims, q, k, wq, wk, sel, None, None)
    assert call(0, 64, 4, 128, 4, 2048) == 1
    assert call(1, 64, 8, 128, 4, 2048) == 2                         # heads
    assert call(1, 64, 4, 64, 4, 2048) == 2                          # d
    assert call(1, 64, 4, 128, 4, 2046) == 2                         # budget not a multiple of the block
    assert call(1, 64, 4, 128, 4, 2048, q=P(4100)) == 3
    assert call(1, 64, 4, 128, 4, 2048, sel=None) == 1
    assert call(1, 0, 4, 128, 4, 2048, q=None, sel=None) == 0        # nothing to do


def test_prefill_ws_checks_its_workspace(lib):
    """Workspace NULL or short -> GDN_ERR_INVALID_ARG, misaligned -> GDN_ERR_ALIGNMENT,
    both before any CUDA call."""
    d = _dims()
    need = ctypes.c_size_t(0)
    assert lib.gdn_prefill_workspace_size(ctypes.byref(d), ctypes.byref(need)) == 0 and need.value > 0
    a = _args()
    ws_args = a[:-1]
    assert lib.gdn_prefill_ws(ctypes.byref(d), *ws_args, None, need.value, None) == 1
    assert lib.gdn_prefill_ws(ctypes.byref(d), *ws_args, ctypes.c_void_p(1 << 20), need.value - 1, None) == 1
    assert lib.gdn_prefill_ws(ctypes.byref(d), *ws_args, ctypes.c_void_p((1 << 20) + 16), need.value, None) == 3


def test_conv_tail_rejects_bad_arguments(lib):
    d = _dims()
    q, k, v = FAKE[0], FAKE[1], FAKE[2]
    assert lib.gdn_prefill_conv_tail(ctypes.byref(d), q, k, v, None, None, None) == 1
    assert lib.gdn_prefill_conv_tail(ctypes.byref(d), q, k, v, None, ctypes.c_void_p(4104), None) == 3
    bad = _dims(dk=96)
    assert lib.gdn_prefill_conv_tail(ctypes.byref(bad), q, k, v, None, FAKE[4], None) == 2


def test_gemm_argument_validation(lib):
    P = ctypes.c_void_p
    a, b, c = P(4096), P(8192), P(12288)
    assert lib.gdn_gemm_bf16(128, 256, 0, a, 64, b, 256, c, 256, None) == 1      # K = 0
    assert lib.gdn_gemm_bf16(128, 256, 60, a, 64, b, 256, c, 256, None) == 1     # K not a multiple of 8
    assert lib.gdn_gemm_bf16(128, 256, 64, a, 32, b, 256, c, 256, None) == 1     # lda < K
    assert lib.gdn_gemm_bf16(128, 256, 64, a, 64, b, 260, c, 256, None) == 1     # wide: ldb not a multiple of 8
    assert lib.gdn_gemm_bf16(128, 256, 64, P(4100), 64, b, 256, c, 256, None) == 3   # A misaligned
    assert lib.gdn_gemm_bf16(128, 256, 64, a, 64, b, 256, None, 256, None) == 1   # no C
    assert lib.gdn_gemm_bf16(0, 256, 64, None, 64, None, 256, None, 256, None) == 0   # nothing to do
    assert lib.gdn_last_call_launches() == 0
