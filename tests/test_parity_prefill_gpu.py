"""GPU prefill vs the fp64 oracle, element by element (normwise per tensor).

Small cases span several 64-token chunks, ragged tails, empty and one-token
sequences; full-size workloads are checked on sampled (sequence, head) chains
that the oracle recomputes token by token."""
import math
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
from harness import (TOL_BF16, TOL_F32, gpu_prefill, normwise, oracle_full, seq_bounds,
                     to_device)
from linear_attention_token_shortconv_b200 import gdn
from linear_attention_token_shortconv_b200.workloads import (LONG, PRETRAIN, TINY_F32, VARLEN,
                                                             make_prefill_inputs, scaled,
                                                             to_oracle_bits)

pytestmark = pytest.mark.gpu

SMALL = [
    ("tiny-fp32", TINY_F32, TOL_F32),
    ("tiny-fp32-long-memory", replace(TINY_F32, long_memory=True, s0_var=0.02, lengths=(300, 77)), TOL_F32),
    ("pretrain-small", scaled(PRETRAIN, lengths=(300, 257), H=3), TOL_BF16),
    ("long-small-S0", scaled(LONG, lengths=(1000,), H=2), TOL_BF16),
    ("varlen-edges", scaled(VARLEN, lengths=(1, 63, 64, 65, 0, 200, 130, 2), H=2), TOL_BF16),
    ("long-memory", scaled(PRETRAIN, lengths=(700, 64), H=2, long_memory=True, s0_var=0.02), TOL_BF16),
    # 40 (sequence, head) chains: the segmented pipeline (two segments) instead of the fused kernel
    ("many-chains-segmented", scaled(PRETRAIN, lengths=(700, 129), H=20, s0_var=0.02), TOL_BF16),
    # equal lengths, more (sequence, head) items than a quarter of the SMs: the fused
    # kernel's chain CTAs take several items in turn
    ("many-chains-fused", scaled(PRETRAIN, lengths=(150,) * 6, H=10, s0_var=0.02), TOL_BF16),
    # equal lengths, more items than SMs: the segmented pipeline with segments cut
    # over one sequence's chunks
    ("many-chains-equal-segmented", scaled(PRETRAIN, lengths=(70,) * 4, H=40, s0_var=0.02), TOL_BF16),
    ("dk64-dv128", replace(scaled(PRETRAIN, lengths=(190,), H=2), dk=64, dv=128, s0_var=0.02), TOL_BF16),
    ("dk128-dv64", replace(scaled(PRETRAIN, lengths=(190, 3), H=2), dk=128, dv=64, s0_var=0.02), TOL_BF16),
]


@pytest.mark.parametrize("name,cfg,tol", SMALL, ids=[c[0] for c in SMALL])
def test_prefill_matches_oracle(cuda_device, name, cfg, tol):
    inp = make_prefill_inputs(cfg, "cpu")
    out, SF = gpu_prefill(to_device(inp, cuda_device), cfg.num_seqs)
    o_ref, s_ref = oracle_full(inp)
    e_out = normwise(out.cpu().numpy(), o_ref)
    e_s = normwise(SF.cpu().numpy(), s_ref)
    print(f"{name}: out {e_out:.2e}  S_final {e_s:.2e}")
    assert np.isfinite(out.cpu().numpy()).all()
    assert e_out <= tol and e_s <= tol


def test_bf16_output(cuda_device):
    """bf16 `out` adds one rounding (<= 2^-9 relative) to the fp32 result."""
    cfg = scaled(PRETRAIN, lengths=(200,), H=2)
    inp = make_prefill_inputs(cfg, "cpu")
    out, _ = gpu_prefill(to_device(inp, cuda_device), 1, out_dtype=torch.bfloat16)
    o_ref, _ = oracle_full(inp)
    assert out.dtype == torch.bfloat16
    assert normwise(out.float().cpu().numpy(), o_ref) <= TOL_BF16 + 2.0 ** -9


def test_overflowing_log_decay_gives_alpha_zero(cuda_device):
    """Decay logits near the top of the bf16 range make -e^A softplus(a) overflow
    to -inf in fp32.  The oracle (fp64) sees alpha = 0 there; the tensor-core path
    must stay finite and agree (its log-decay is clamped where e^g is already 0)."""
    cfg = scaled(PRETRAIN, lengths=(200, 70), H=2, s0_var=0.02)
    inp = make_prefill_inputs(cfg, "cpu")
    a = inp["a_logit"].float()
    a[[5, 63, 64, 100, 150, 199, 230], 0] = 3.0e38
    a[[0, 64, 128, 269], 1] = 3.0e38
    inp["a_logit"] = a.to(torch.bfloat16)
    inp["A"] = torch.full_like(inp["A"], math.log(16.0))
    out, SF = gpu_prefill(to_device(inp, cuda_device), cfg.num_seqs)
    o_ref, s_ref = oracle_full(inp)
    assert torch.isfinite(out).all() and torch.isfinite(SF).all()
    e_out, e_s = normwise(out.cpu().numpy(), o_ref), normwise(SF.cpu().numpy(), s_ref)
    print(f"out {e_out:.2e} S_final {e_s:.2e}")
    assert e_out <= TOL_BF16 and e_s <= TOL_BF16


@pytest.mark.parametrize("cfg", [scaled(LONG, lengths=(700,), H=2),
                                 scaled(PRETRAIN, lengths=(700, 129), H=20, s0_var=0.02)],
                         ids=["fused", "segmented"])
def test_prefill_ws_matches_prefill(cuda_device, cfg):
    """gdn_prefill_ws runs gdn_prefill's kernels on a workspace the caller owns:
    the results are bit-identical, and a workspace one byte short is rejected
    before anything runs."""
    inp = to_device(make_prefill_inputs(cfg, "cpu"), cuda_device)
    ref_out, ref_S = gpu_prefill(inp, cfg.num_seqs)
    nbytes = gdn.prefill_workspace_size(cfg.num_seqs, cfg.total_tokens, cfg.H, cfg.dk, cfg.dv)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=cuda_device)
    args = (inp["q"], inp["k"], inp["v"], inp["conv_w"], inp["a_logit"], inp["b_logit"], inp["A"],
            inp["b_alpha"], inp["z"], inp["norm_w"])
    kw = dict(S0=inp.get("S0"), cu_seqlens=inp.get("cu_seqlens"), num_seqs=cfg.num_seqs)
    out, S = gdn.prefill_ws(*args, ws, **kw)
    torch.cuda.synchronize()
    assert torch.equal(out, ref_out) and torch.equal(S, ref_S)
    with pytest.raises(gdn.GdnError) as ei:
        gdn.prefill_ws(*args, ws[:nbytes - 1], **kw)
    assert ei.value.status == 1   # GDN_ERR_INVALID_ARG


def test_empty_batch_returns_initial_state(cuda_device):
    cfg = scaled(PRETRAIN, lengths=(0, 0), H=2, s0_var=0.02, varlen=True)
    inp = to_device(make_prefill_inputs(cfg, "cpu"), cuda_device)
    out, SF = gpu_prefill(inp, 2)
    assert out.numel() == 0
    assert torch.equal(SF, inp["S0"])


def test_state_may_alias_initial_state(cuda_device):
    cfg = scaled(LONG, lengths=(150,), H=2)
    inp = to_device(make_prefill_inputs(cfg, "cpu"), cuda_device)
    out1, SF1 = gpu_prefill(inp, 1)
    S = inp["S0"].clone()
    out2, SF2 = gdn.prefill(inp["q"], inp["k"], inp["v"], inp["conv_w"], inp["a_logit"],
                            inp["b_logit"], inp["A"], inp["b_alpha"], inp["z"], inp["norm_w"],
                            S0=S, S_final=S)
    torch.cuda.synchronize()
    assert torch.equal(out1, out2) and torch.equal(SF1, S)


def test_deterministic(cuda_device):
    cfg = scaled(VARLEN, lengths=(100, 37, 300), H=2)
    inp = to_device(make_prefill_inputs(cfg, "cpu"), cuda_device)
    a = gpu_prefill(inp, 3)
    b = gpu_prefill(inp, 3)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_rejects_host_tensors():
    cfg = scaled(PRETRAIN, lengths=(8,), H=1)
    inp = make_prefill_inputs(cfg, "cpu")
    with pytest.raises(ValueError):
        gdn.prefill(inp["q"], inp["k"], inp["v"], inp["conv_w"], inp["a_logit"], inp["b_logit"],
                    inp["A"], inp["b_alpha"], inp["z"], inp["norm_w"])


# ------------------------------------------------ full-size, sampled chains

def _oracle_heads(inp, n, heads, cu):
    """Oracle for sequence n restricted to `heads` (one OpenMP thread per head)."""
    t0, t1 = int(cu[n]), int(cu[n + 1])
    H, dk = inp["q"].shape[1], inp["q"].shape[2]
    dv = inp["v"].shape[2]
    hs = torch.tensor(heads)
    take = lambda key: to_oracle_bits(inp[key][t0:t1].index_select(1, hs.to(inp[key].device)))
    # conv rows of the selected heads in the [q heads | k heads | v heads] order
    rows = torch.cat([torch.arange(h * dk, (h + 1) * dk) for h in heads] +
                     [H * dk + torch.arange(h * dk, (h + 1) * dk) for h in heads] +
                     [2 * H * dk + torch.arange(h * dv, (h + 1) * dv) for h in heads])
    cw = to_oracle_bits(inp["conv_w"].index_select(0, rows.to(inp["conv_w"].device)))
    S0 = None
    if inp.get("S0") is not None:
        S0 = to_oracle_bits(inp["S0"][n:n + 1].index_select(1, hs.to(inp["S0"].device)))
    out, SF = oracle.prefill(take("q"), take("k"), take("v"), cw, take("a_logit"), take("b_logit"),
                             to_oracle_bits(inp["A"][hs.to(inp["A"].device)]),
                             to_oracle_bits(inp["b_alpha"][hs.to(inp["b_alpha"].device)]),
                             take("z"), to_oracle_bits(inp["norm_w"]), S0=S0,
                             n_threads=len(heads))
    return out, SF[0], t0, t1


FULL = [("pretrain", PRETRAIN, [(0, [0, 15]), (3, [7])]),
        ("long", LONG, [(0, [0, 17, 31])]),
        # alpha close to 1 over all 512 chunks: the fp32 state carries across every
        # chunk, and its fp16 copy (the tensor-core operand) feeds every chunk's U
        ("long-memory", replace(LONG, long_memory=True), [(0, [0, 31])]),
        ("varlen", VARLEN, None)]


@pytest.mark.parametrize("name,cfg,samples", FULL, ids=[c[0] for c in FULL])
def test_full_size_sampled(cuda_device, name, cfg, samples):
    inp = make_prefill_inputs(cfg, cuda_device)
    out, SF = gpu_prefill(inp, cfg.num_seqs)
    assert torch.isfinite(out).all() and torch.isfinite(SF).all()
    cu = seq_bounds(inp, cfg.total_tokens, cfg.num_seqs)
    if samples is None:   # shortest and longest sequence
        lens = np.diff(cu)
        samples = [(int(np.argmin(lens)), [0, cfg.H - 1]), (int(np.argmax(lens)), [5])]
    for n, heads in samples:
        o_ref, s_ref, t0, t1 = _oracle_heads(inp, n, heads, cu)
        hs = torch.tensor(heads, device=cuda_device)
        got_o = out[t0:t1].index_select(1, hs).cpu().numpy()
        got_s = SF[n].index_select(0, hs).cpu().numpy()
        e_out, e_s = normwise(got_o, o_ref), normwise(got_s, s_ref)
        print(f"{name} seq {n} heads {heads}: out {e_out:.2e} S_final {e_s:.2e}")
        assert e_out <= TOL_BF16 and e_s <= TOL_BF16
