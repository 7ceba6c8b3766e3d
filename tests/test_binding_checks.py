"""The Python binding's argument checks, on the CPU: the library sees raw pointers
only, so a tensor of the wrong dtype or shape must be refused before any call
(else its bytes would be read as something else, or past its end), and host
tensors must be refused too (no CPU fallback)."""
from dataclasses import replace

import pytest
import torch

from linear_attention_token_shortconv_b200 import gdn
from linear_attention_token_shortconv_b200.workloads import (DECODE, PRETRAIN, QSA, make_decode_inputs,
                                                             make_layer_inputs, make_prefill_inputs,
                                                             make_qsa_inputs, scaled)

CFG = scaled(PRETRAIN, lengths=(9, 5), H=2, varlen=True, s0_var=0.02)


def _prefill_args():
    inp = make_prefill_inputs(CFG, "cpu")
    return inp, dict(S0=inp["S0"], cu_seqlens=inp["cu_seqlens"])


def _call_prefill(inp, kw, fn=gdn.prefill):
    return fn(inp["q"], inp["k"], inp["v"], inp["conv_w"], inp["a_logit"], inp["b_logit"], inp["A"],
              inp["b_alpha"], inp["z"], inp["norm_w"], **kw)


def test_valid_host_tensors_reach_the_device_check():
    inp, kw = _prefill_args()
    with pytest.raises(ValueError, match="CUDA device"):
        _call_prefill(inp, kw)


@pytest.mark.parametrize("key,bad,err,word", [
    ("conv_w", lambda t: t.to(torch.bfloat16), TypeError, "conv_w"),
    ("A", lambda t: t.double(), TypeError, "A"),
    ("k", lambda t: t.float(), TypeError, "k"),
    ("v", lambda t: t[:, :, :64].contiguous(), ValueError, "z"),          # v sets d_v: z no longer matches
    ("z", lambda t: t[:-1].contiguous(), ValueError, "z"),
    ("a_logit", lambda t: t[:, :1].contiguous(), ValueError, "a_logit"),
    ("norm_w", lambda t: t[:64].contiguous(), ValueError, "norm_w"),
    ("conv_w", lambda t: t[:-1].contiguous(), ValueError, "conv_w"),
])
def test_prefill_refuses_bad_tensors(key, bad, err, word):
    inp, kw = _prefill_args()
    inp[key] = bad(inp[key])
    for fn in (gdn.prefill, gdn.prefill_noalloc):
        with pytest.raises(err, match=word):
            _call_prefill(inp, kw, fn)


def test_prefill_refuses_bad_state_and_lengths():
    inp, kw = _prefill_args()
    with pytest.raises(ValueError, match="S0"):
        _call_prefill(inp, dict(kw, S0=inp["S0"][:1].contiguous()))
    with pytest.raises(TypeError, match="cu_seqlens"):
        _call_prefill(inp, dict(kw, cu_seqlens=inp["cu_seqlens"].long()))
    with pytest.raises(TypeError, match="S_final"):
        _call_prefill(inp, dict(kw, S_final=torch.empty(inp["S0"].shape, dtype=torch.bfloat16)))
    with pytest.raises(TypeError, match="out"):
        _call_prefill(inp, dict(kw, out=torch.empty(inp["z"].shape, dtype=torch.float16)))


def test_backward_refuses_a_mismatched_output_gradient():
    cfg = replace(CFG, in_dtype=torch.float32)
    inp = make_prefill_inputs(cfg, "cpu")
    args = [inp[k] for k in ("q", "k", "v", "conv_w", "a_logit", "b_logit", "A", "b_alpha", "z", "norm_w")]
    d_out = torch.zeros(inp["z"].shape)
    with pytest.raises(TypeError, match="d_out"):
        gdn.prefill_backward(*args, d_out.to(torch.bfloat16), S0=inp["S0"], cu_seqlens=inp["cu_seqlens"])
    with pytest.raises(ValueError, match="d_S_final"):
        gdn.prefill_backward(*args, d_out, S0=inp["S0"], cu_seqlens=inp["cu_seqlens"],
                             d_S_final=torch.zeros(1, 2, 128, 128))
    with pytest.raises(ValueError, match="CUDA device"):
        gdn.prefill_backward(*args, d_out, S0=inp["S0"], cu_seqlens=inp["cu_seqlens"])


def test_decode_refuses_bad_tensors():
    d = make_decode_inputs(replace(DECODE, B=3, H=2, pool=2), "cpu")
    args = lambda hist, S: (d["q"][0], d["k"][0], d["v"][0], d["conv_w"], hist, d["a_logit"][0], d["b_logit"][0],
                            d["A"], d["b_alpha"], d["z"][0], d["norm_w"], S)
    with pytest.raises(ValueError, match="conv_hist"):
        gdn.decode_step(*args(d["ring"][:, :2].contiguous(), d["S"]))
    with pytest.raises(TypeError, match="S"):
        gdn.decode_step(*args(d["ring"], d["S"].to(torch.bfloat16)))
    with pytest.raises(ValueError, match="CUDA device"):
        gdn.decode_step(*args(d["ring"], d["S"]))
    m = {k: d[k][:2].transpose(0, 1).contiguous() for k in ("q", "k", "v", "z", "a_logit", "b_logit")}
    margs = (m["q"], m["k"], m["v"], d["conv_w"], d["ring"], m["a_logit"], m["b_logit"], d["A"], d["b_alpha"],
             m["z"], d["norm_w"], d["S"])
    with pytest.raises(TypeError, match="n_keep"):
        gdn.decode_multi(*margs, n_keep=torch.zeros(3, dtype=torch.int64))
    with pytest.raises(ValueError, match="n_keep"):
        gdn.decode_multi(*margs, n_keep=torch.zeros(2, dtype=torch.int32))
    with pytest.raises(ValueError, match="CUDA device"):
        gdn.decode_multi(*margs)


def test_qsa_and_layer_refuse_bad_tensors():
    inp = make_qsa_inputs(replace(QSA, n=64), "cpu")
    with pytest.raises(TypeError, match="k"):
        gdn.qsa_indexer(inp["q"], inp["k"].float(), inp["w_q"], inp["w_k"], budget=16)
    with pytest.raises(ValueError, match="w_q"):
        gdn.qsa_indexer(inp["q"], inp["k"], inp["w_q"][:64].contiguous(), inp["w_k"], budget=16)
    with pytest.raises(ValueError, match="CUDA device"):
        gdn.qsa_indexer(inp["q"], inp["k"], inp["w_q"], inp["w_k"], budget=16)
    cfg = scaled(PRETRAIN, lengths=(8,), H=2)
    L = make_layer_inputs(cfg, 64, "cpu")
    largs = lambda w_in: (L["x"], w_in, L["conv_w"], L["A"], L["b_alpha"], L["norm_w"], L["w_o"], 2, 128, 128)
    with pytest.raises(ValueError, match="w_in"):
        gdn.layer_forward(*largs(L["w_in"][:, :-1].contiguous()), num_seqs=1)
    with pytest.raises(ValueError, match="CUDA device"):
        gdn.layer_forward(*largs(L["w_in"]), num_seqs=1)
