"""Parity harness shared by the GPU tests: slicing inputs for the oracle, running
the CUDA path, and the normwise error metric.

The error metric reads "max relative error" normwise per tensor:
max|gpu - ref| / max|ref|, taken separately over `out` and over `S_final`.
"""
import numpy as np
import torch

import oracle
from linear_attention_token_shortconv_b200 import gdn
from linear_attention_token_shortconv_b200.workloads import to_oracle_bits

TOL_BF16 = 2e-3   # bf16 inputs, fp32 accumulation, fp32 out
TOL_F32 = 1e-5    # fp32 inputs end to end


def normwise(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    denom = np.abs(ref).max() if ref.size else 0.0
    if denom == 0.0:
        return float(np.abs(got).max()) if got.size else 0.0
    return float(np.abs(got - ref).max() / denom)


def seq_bounds(inp, n_tok, n_seq):
    cu = inp.get("cu_seqlens")
    if cu is not None:
        cu = cu.detach().cpu().numpy().astype(np.int64)
    else:
        L = n_tok // n_seq
        cu = np.arange(n_seq + 1, dtype=np.int64) * L
    return cu


def slice_pair(inp, n, h, cu):
    """Inputs of one (sequence, head) chain as an H = 1, single-sequence problem."""
    t0, t1 = int(cu[n]), int(cu[n + 1])
    H, dk = inp["q"].shape[1], inp["q"].shape[2]
    dv = inp["v"].shape[2]
    cw = inp["conv_w"]
    rows = torch.cat([torch.arange(h * dk, (h + 1) * dk),
                      H * dk + torch.arange(h * dk, (h + 1) * dk),
                      2 * H * dk + torch.arange(h * dv, (h + 1) * dv)]).to(cw.device)
    d = {key: inp[key][t0:t1, h:h + 1].contiguous() for key in ("q", "k", "v", "z", "a_logit", "b_logit")}
    d["conv_w"] = cw.index_select(0, rows)
    d["A"] = inp["A"][h:h + 1]
    d["b_alpha"] = inp["b_alpha"][h:h + 1]
    d["norm_w"] = inp["norm_w"]
    d["S0"] = None if inp.get("S0") is None else inp["S0"][n:n + 1, h:h + 1]
    return d, t0, t1


def oracle_pair(inp, n, h, cu, n_threads=1):
    d, t0, t1 = slice_pair(inp, n, h, cu)
    bits = {key: (None if val is None else to_oracle_bits(val)) for key, val in d.items()}
    out, SF = oracle.prefill(bits["q"], bits["k"], bits["v"], bits["conv_w"], bits["a_logit"],
                             bits["b_logit"], bits["A"], bits["b_alpha"], bits["z"],
                             bits["norm_w"], S0=bits["S0"], n_threads=n_threads)
    return out[:, 0], SF[0, 0], t0, t1


def oracle_full(inp):
    bits = {key: (None if val is None else to_oracle_bits(val)) for key, val in inp.items()}
    n_seq = None
    if bits.get("cu_seqlens") is None:
        n_seq = 1 if bits.get("S0") is None else bits["S0"].shape[0]
    return oracle.prefill(bits["q"], bits["k"], bits["v"], bits["conv_w"], bits["a_logit"],
                          bits["b_logit"], bits["A"], bits["b_alpha"], bits["z"], bits["norm_w"],
                          S0=bits.get("S0"), cu_seqlens=bits.get("cu_seqlens"), num_seqs=n_seq)


def to_device(inp, device):
    return {key: (None if val is None else val.to(device)) for key, val in inp.items()}


def gpu_prefill(inp, num_seqs, out_dtype=torch.float32):
    out, SF = gdn.prefill(inp["q"], inp["k"], inp["v"], inp["conv_w"], inp["a_logit"],
                          inp["b_logit"], inp["A"], inp["b_alpha"], inp["z"], inp["norm_w"],
                          S0=inp.get("S0"), cu_seqlens=inp.get("cu_seqlens"), num_seqs=num_seqs,
                          out_dtype=out_dtype)
    torch.cuda.synchronize()
    return out, SF
