"""Multi-token decode (gdn_decode_multi) against the fp64 oracle run token by
token: the outputs of all T tokens equal T successive decode steps; the state
and the conv history (bit-exact: it only moves input bits) end as after the
first n_keep[b] of those steps."""
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
from harness import TOL_BF16, normwise, to_device
from linear_attention_token_shortconv_b200 import gdn
from linear_attention_token_shortconv_b200.workloads import DECODE, make_decode_inputs, to_oracle_bits

pytestmark = pytest.mark.gpu


def _multi_inputs(cfg, T):
    """The decode workload's pool entries 0..T-1 as T consecutive tokens: [B, T, H, d]."""
    inp = make_decode_inputs(cfg, "cpu")
    multi = {key: inp[key][:T].transpose(0, 1).contiguous() for key in ("q", "k", "v", "z", "a_logit", "b_logit")}
    return inp, multi


def _oracle(inp, T, n_keep):
    S = to_oracle_bits(inp["S"]).astype(np.float64)
    h = to_oracle_bits(inp["ring"]).copy()
    snaps_S, snaps_h, outs = [S.copy()], [h.copy()], []
    for t in range(T):
        outs.append(oracle.decode_step(*(to_oracle_bits(inp[key][t]) for key in ("q", "k", "v")),
                                       to_oracle_bits(inp["conv_w"]), h, to_oracle_bits(inp["a_logit"][t]),
                                       to_oracle_bits(inp["b_logit"][t]), to_oracle_bits(inp["A"]),
                                       to_oracle_bits(inp["b_alpha"]), to_oracle_bits(inp["z"][t]),
                                       to_oracle_bits(inp["norm_w"]), S))
        snaps_S.append(S.copy())
        snaps_h.append(h.copy())
    out = np.stack(outs, axis=1)                                   # [B, T, H, dv]
    B = S.shape[0]
    keep = [T] * B if n_keep is None else list(n_keep)
    S_exp = np.stack([snaps_S[keep[b]][b] for b in range(B)])
    h_exp = np.stack([snaps_h[keep[b]][b] for b in range(B)])
    return out, S_exp, h_exp


@pytest.mark.parametrize("T,keep,out_dtype", [
    (1, None, torch.float32),
    (2, None, torch.float32),
    (4, None, torch.float32),
    (3, "zeros", torch.float32),
    (4, "mixed", torch.float32),
    (4, "mixed", torch.bfloat16),
    (1, "mixed", torch.float32),   # T = 1 through the multi-token kernel
])
def test_decode_multi_matches_token_by_token(cuda_device, T, keep, out_dtype):
    cfg = replace(DECODE, B=12, H=4, seed=11)
    inp, multi = _multi_inputs(cfg, T)
    B = cfg.B
    if keep is None:
        n_keep = None
    elif keep == "zeros":
        n_keep = [0] * B
    else:
        n_keep = [b % (T + 1) for b in range(B)]
    g = to_device(inp, cuda_device)
    m = to_device(multi, cuda_device)
    S, hist = g["S"].clone(), g["ring"].clone()
    nk = None if n_keep is None else torch.tensor(n_keep, dtype=torch.int32, device=cuda_device)
    out = gdn.decode_multi(m["q"], m["k"], m["v"], g["conv_w"], hist, m["a_logit"], m["b_logit"], g["A"],
                           g["b_alpha"], m["z"], g["norm_w"], S, n_keep=nk, out_dtype=out_dtype)
    torch.cuda.synchronize()
    o_ref, S_ref, h_ref = _oracle(inp, T, n_keep)
    e_o = normwise(out.float().cpu().numpy(), o_ref)
    e_s = normwise(S.cpu().numpy(), S_ref)
    tol = TOL_BF16 + (2.0 ** -9 if out_dtype == torch.bfloat16 else 0.0)
    print(f"T={T} keep={keep}: out {e_o:.1e} S {e_s:.1e}")
    assert e_o <= tol and e_s <= TOL_BF16
    assert np.array_equal(to_oracle_bits(hist), h_ref)


@pytest.mark.parametrize("T", [2, 4])
def test_decode_multi_long_memory(cuda_device, T):
    """alpha close to 1 (A = log U[0.01, 0.1], a ~ N(-2, 1)): every token's output
    depends on the carried state, not only on its own write."""
    cfg = replace(DECODE, B=12, H=4, seed=13, long_memory=True)
    inp, multi = _multi_inputs(cfg, T)
    n_keep = [b % (T + 1) for b in range(cfg.B)]
    g, m = to_device(inp, cuda_device), to_device(multi, cuda_device)
    S, hist = g["S"].clone(), g["ring"].clone()
    nk = torch.tensor(n_keep, dtype=torch.int32, device=cuda_device)
    out = gdn.decode_multi(m["q"], m["k"], m["v"], g["conv_w"], hist, m["a_logit"], m["b_logit"], g["A"],
                           g["b_alpha"], m["z"], g["norm_w"], S, n_keep=nk)
    torch.cuda.synchronize()
    o_ref, S_ref, h_ref = _oracle(inp, T, n_keep)
    e_o, e_s = normwise(out.cpu().numpy(), o_ref), normwise(S.cpu().numpy(), S_ref)
    print(f"long memory T={T}: out {e_o:.1e} S {e_s:.1e}")
    assert e_o <= TOL_BF16 and e_s <= TOL_BF16
    assert np.array_equal(to_oracle_bits(hist), h_ref)


def test_decode_multi_zero_keep_leaves_state_untouched(cuda_device):
    cfg = replace(DECODE, B=8, H=2, seed=12)
    inp, multi = _multi_inputs(cfg, 4)
    g, m = to_device(inp, cuda_device), to_device(multi, cuda_device)
    S, hist = g["S"].clone(), g["ring"].clone()
    nk = torch.zeros(cfg.B, dtype=torch.int32, device=cuda_device)
    gdn.decode_multi(m["q"], m["k"], m["v"], g["conv_w"], hist, m["a_logit"], m["b_logit"], g["A"], g["b_alpha"],
                     m["z"], g["norm_w"], S, n_keep=nk)
    torch.cuda.synchronize()
    assert torch.equal(S, g["S"]) and torch.equal(hist, g["ring"])


def test_decode_multi_full_size_sampled(cuda_device):
    """B = 256, H = 32, T = 4 (the decode workload's shape): every sequence's
    outputs and committed state against the oracle, n_keep mixed."""
    T = 4
    inp, multi = _multi_inputs(DECODE, T)
    n_keep = [(b * 7) % (T + 1) for b in range(DECODE.B)]
    g, m = to_device(inp, cuda_device), to_device(multi, cuda_device)
    S, hist = g["S"].clone(), g["ring"].clone()
    nk = torch.tensor(n_keep, dtype=torch.int32, device=cuda_device)
    out = gdn.decode_multi(m["q"], m["k"], m["v"], g["conv_w"], hist, m["a_logit"], m["b_logit"], g["A"],
                           g["b_alpha"], m["z"], g["norm_w"], S, n_keep=nk)
    torch.cuda.synchronize()
    o_ref, S_ref, h_ref = _oracle(inp, T, n_keep)
    e_o, e_s = normwise(out.cpu().numpy(), o_ref), normwise(S.cpu().numpy(), S_ref)
    print(f"full size: out {e_o:.1e} S {e_s:.1e}")
    assert e_o <= TOL_BF16 and e_s <= TOL_BF16
    assert np.array_equal(to_oracle_bits(hist), h_ref)
