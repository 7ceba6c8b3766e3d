"""Small workloads for ncu captures (a few hundred MB on the device, inputs
larger than L2), run through the public binding:

    python -m linear_attention_token_shortconv_b200.profile_case prefill 8192
        long-prefill shape with T tokens, H = 32, d = 128, S0 ~ N(0, 0.02):
        two warm-up calls, then one call
    python -m linear_attention_token_shortconv_b200.profile_case decode 64
        decode step for B sequences x 32 heads, d = 128: three steps
    python -m linear_attention_token_shortconv_b200.profile_case backward 1024
        prefill backward, 4 sequences x T tokens, H = 16, d = 128, fp32: three calls
    python -m linear_attention_token_shortconv_b200.profile_case qsa 16384
        QSA indexer on one sequence of n tokens, K = 2048: three calls
"""
import sys
from dataclasses import replace

import torch

from linear_attention_token_shortconv_b200 import gdn
from linear_attention_token_shortconv_b200.workloads import (DECODE, LONG, PRETRAIN, QSA, make_decode_inputs,
                                                             make_prefill_inputs, make_qsa_inputs, scaled)


def prefill(T: int):
    cfg = scaled(LONG, lengths=(T,))
    inp = make_prefill_inputs(cfg, "cuda")
    out = torch.empty((T, cfg.H, cfg.dv), dtype=torch.bfloat16, device="cuda")
    S = torch.empty((1, cfg.H, cfg.dk, cfg.dv), device="cuda")
    for _ in range(3):
        gdn.prefill(inp["q"], inp["k"], inp["v"], inp["conv_w"], inp["a_logit"], inp["b_logit"], inp["A"],
                    inp["b_alpha"], inp["z"], inp["norm_w"], S0=inp["S0"], out=out, S_final=S)
    torch.cuda.synchronize()
    print("ok", float(out.float().abs().mean()))


def decode(B: int):
    cfg = replace(DECODE, B=B)
    d = make_decode_inputs(cfg, "cuda")
    out = torch.empty((cfg.B, cfg.H, cfg.dv), dtype=torch.bfloat16, device="cuda")
    for t in range(3):
        gdn.decode_step(d["q"][t], d["k"][t], d["v"][t], d["conv_w"], d["ring"], d["a_logit"][t],
                        d["b_logit"][t], d["A"], d["b_alpha"], d["z"][t], d["norm_w"], d["S"], out=out)
    torch.cuda.synchronize()
    print("ok", float(out.float().abs().mean()))


def backward(T: int):
    cfg = replace(PRETRAIN, lengths=(T,) * 4, in_dtype=torch.float32)
    inp = make_prefill_inputs(cfg, "cuda")
    g = torch.Generator(device="cuda")
    g.manual_seed(cfg.seed + 100)
    d_out = torch.randn((cfg.total_tokens, cfg.H, cfg.dv), generator=g, device="cuda")
    for _ in range(3):
        grads = gdn.prefill_backward(inp["q"], inp["k"], inp["v"], inp["conv_w"], inp["a_logit"], inp["b_logit"],
                                     inp["A"], inp["b_alpha"], inp["z"], inp["norm_w"], d_out, S0=inp.get("S0"),
                                     num_seqs=cfg.num_seqs)
    torch.cuda.synchronize()
    print("ok", float(grads["dq"].abs().mean()))


def qsa(n: int):
    cfg = replace(QSA, n=n)
    inp = make_qsa_inputs(cfg, "cuda")
    for _ in range(3):
        sel, _ = gdn.qsa_indexer(inp["q"], inp["k"], inp["w_q"], inp["w_k"], budget=cfg.budget)
    torch.cuda.synchronize()
    print("ok", int(sel[-1, -1, 0]))


if __name__ == "__main__":
    kind, size = sys.argv[1], int(sys.argv[2])
    {"prefill": prefill, "decode": decode, "backward": backward, "qsa": qsa}[kind](size)
