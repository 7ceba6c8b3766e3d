"""GPU decode step vs the fp64 oracle, step by step: outputs, the in-place state
and the conv history (bit-exact: it only moves input bits)."""
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
from harness import TOL_BF16, TOL_F32, gpu_prefill, normwise, to_device
from linear_attention_token_shortconv_b200 import gdn
from linear_attention_token_shortconv_b200.workloads import (DECODE, PRETRAIN, make_decode_inputs,
                                                             make_prefill_inputs, scaled,
                                                             to_oracle_bits)

pytestmark = pytest.mark.gpu


def _run_steps(cfg, steps, device, tol, check_every=1):
    inp = make_decode_inputs(cfg, "cpu")
    g = to_device(inp, device)
    S = g["S"].clone()
    hist = g["ring"].clone()
    S_ref = to_oracle_bits(inp["S"]).astype(np.float64)
    h_ref = to_oracle_bits(inp["ring"]).copy()
    worst = 0.0
    for t in range(steps):
        p = t % cfg.pool
        out = gdn.decode_step(g["q"][p], g["k"][p], g["v"][p], g["conv_w"], hist, g["a_logit"][p],
                              g["b_logit"][p], g["A"], g["b_alpha"], g["z"][p], g["norm_w"], S)
        o_ref = oracle.decode_step(*(to_oracle_bits(inp[key][p]) for key in ("q", "k", "v")),
                                   to_oracle_bits(inp["conv_w"]), h_ref,
                                   to_oracle_bits(inp["a_logit"][p]), to_oracle_bits(inp["b_logit"][p]),
                                   to_oracle_bits(inp["A"]), to_oracle_bits(inp["b_alpha"]),
                                   to_oracle_bits(inp["z"][p]), to_oracle_bits(inp["norm_w"]), S_ref)
        if t % check_every == 0 or t == steps - 1:
            torch.cuda.synchronize()
            e_o = normwise(out.cpu().numpy(), o_ref)
            e_s = normwise(S.cpu().numpy(), S_ref)
            worst = max(worst, e_o, e_s)
            assert e_o <= tol and e_s <= tol, (t, e_o, e_s)
            assert np.array_equal(to_oracle_bits(hist), h_ref), t
    return worst


def test_decode_small_many_steps(cuda_device):
    cfg = replace(DECODE, B=5, H=3, pool=4)
    print("worst", _run_steps(cfg, 20, cuda_device, TOL_BF16))


def test_decode_small_long_memory(cuda_device):
    """alpha close to 1: the state carries over many steps, so an error in reading
    or writing S shows in every later step's output."""
    cfg = replace(DECODE, B=5, H=3, pool=4, long_memory=True)
    print("worst", _run_steps(cfg, 40, cuda_device, TOL_BF16))


@pytest.mark.parametrize("long_memory", [False, True], ids=["short-memory", "long-memory"])
def test_decode_trajectory_1000_steps(cuda_device, long_memory):
    """The decode workload's 1000 consecutive steps (its 8-entry input pool used
    cyclically, state N(0, 0.02)) on a slice of 8 sequences x 4 heads, against the
    oracle run step by step; compared every 100 steps and at the end."""
    cfg = replace(DECODE, B=8, H=4, long_memory=long_memory)
    print("worst", _run_steps(cfg, cfg.steps, cuda_device, TOL_BF16, check_every=100))


def test_decode_fp32(cuda_device):
    cfg = replace(DECODE, B=3, H=2, dk=64, dv=64, in_dtype=torch.float32, pool=3)
    print("worst", _run_steps(cfg, 12, cuda_device, TOL_F32))


@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 64)])
def test_decode_mixed_head_dims(cuda_device, dk, dv):
    cfg = replace(DECODE, B=4, H=2, dk=dk, dv=dv, pool=2)
    _run_steps(cfg, 6, cuda_device, TOL_BF16)


def test_decode_full_batch(cuda_device):
    """The full decode workload (256 sequences x 32 heads), first steps."""
    print("worst", _run_steps(DECODE, 3, cuda_device, TOL_BF16))


def test_prefill_then_decode_continues_the_sequence(cuda_device):
    """Prefill of T tokens, then decode steps fed the next tokens with the conv
    history taken from the last 3 raw tokens, equals one prefill of T + n tokens."""
    T, n = 150, 6
    cfg = scaled(PRETRAIN, lengths=(T + n,), H=2, s0_var=0.02)
    inp = to_device(make_prefill_inputs(cfg, "cpu"), cuda_device)
    out_all, S_all = gpu_prefill(inp, 1)
    head = {key: (val[:T].contiguous() if key in ("q", "k", "v", "z", "a_logit", "b_logit") else val)
            for key, val in inp.items()}
    _, S = gpu_prefill(head, 1)
    H, dk, dv = cfg.H, cfg.dk, cfg.dv
    raw = torch.cat([inp["q"].reshape(T + n, -1), inp["k"].reshape(T + n, -1),
                     inp["v"].reshape(T + n, -1)], dim=1)
    hist = raw[T - 3:T].unsqueeze(0).contiguous()
    outs = []
    for t in range(T, T + n):
        sl = lambda key: inp[key][t:t + 1].contiguous()
        outs.append(gdn.decode_step(sl("q"), sl("k"), sl("v"), inp["conv_w"], hist, sl("a_logit"),
                                    sl("b_logit"), inp["A"], inp["b_alpha"], sl("z"),
                                    inp["norm_w"], S))
    torch.cuda.synchronize()
    got = torch.cat(outs).cpu().numpy()
    assert normwise(got, out_all[T:].cpu().numpy()) <= TOL_BF16
    assert normwise(S.cpu().numpy(), S_all.cpu().numpy()) <= TOL_BF16


def test_prefill_conv_tail_hands_off_to_decode(cuda_device):
    """Three sequences (150, 2 and 67 tokens, then 5 more each): a prefill of the
    first part, gdn_prefill_conv_tail's history (checked bit-exact against the raw
    rows, zero rows before a short sequence's start) and S_final continue every
    sequence through decode steps as one prefill of the whole does."""
    T_list, n = [150, 2, 67], 5
    cfg = scaled(PRETRAIN, lengths=tuple(T + n for T in T_list), H=2, s0_var=0.02, varlen=True)
    inp = to_device(make_prefill_inputs(cfg, "cpu"), cuda_device)
    out_all, S_all = gpu_prefill(inp, 3)
    cu_all = inp["cu_seqlens"].cpu().tolist()
    idx = torch.cat([torch.arange(cu_all[s], cu_all[s] + T_list[s]) for s in range(3)]).to(cuda_device)
    tok_keys = ("q", "k", "v", "z", "a_logit", "b_logit")
    head = {key: (val.index_select(0, idx).contiguous() if key in tok_keys else val) for key, val in inp.items()}
    cu_head = [0, T_list[0], T_list[0] + T_list[1], sum(T_list)]
    head["cu_seqlens"] = torch.tensor(cu_head, dtype=torch.int32, device=cuda_device)
    _, S = gpu_prefill(head, 3)
    hist = gdn.prefill_conv_tail(head["q"], head["k"], head["v"], head["cu_seqlens"])
    torch.cuda.synchronize()
    N = sum(T_list)
    raw = torch.cat([head["q"].reshape(N, -1), head["k"].reshape(N, -1), head["v"].reshape(N, -1)], dim=1)
    for s in range(3):
        for j in range(3):
            t = cu_head[s + 1] - 3 + j
            want = raw[t] if t >= cu_head[s] else torch.zeros_like(raw[0])
            assert torch.equal(hist[s, j], want), (s, j)
    outs = []
    for step in range(n):
        rows = torch.tensor([cu_all[s] + T_list[s] + step for s in range(3)], device=cuda_device)
        sl = lambda key: inp[key].index_select(0, rows).contiguous()
        outs.append(gdn.decode_step(sl("q"), sl("k"), sl("v"), inp["conv_w"], hist, sl("a_logit"),
                                    sl("b_logit"), inp["A"], inp["b_alpha"], sl("z"), inp["norm_w"], S))
    torch.cuda.synchronize()
    got = torch.stack(outs, dim=1).cpu().numpy()
    want = torch.stack([out_all[cu_all[s] + T_list[s]:cu_all[s] + T_list[s] + n] for s in range(3)]).cpu().numpy()
    assert normwise(got, want) <= TOL_BF16
    assert normwise(S.cpu().numpy(), S_all.cpu().numpy()) <= TOL_BF16
