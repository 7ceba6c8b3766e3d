"""GPU prefill backward vs the fp64 backward oracle (normwise per gradient tensor).

The oracle's backward is pinned by finite differences (tests/test_backward_oracle.py).
Cases: packed varlen batches with ragged tails (lengths not multiples of the
16-token checkpoint interval), a sequence shorter than the conv window, equal
lengths without cu_seqlens, d = 64 and d = 128, short and long memory, with and
without an initial state and a final-state gradient, a nonzero norm weight, and
an empty batch.

Tolerance: fp32 arithmetic throughout, with sums of up to d terms per token step
and gradients carried over whole sequences: 2e-5 normwise (max |gpu - ref| /
max |ref| per tensor; the largest error seen on these cases was 3.2e-6, on the
short-memory d = 128 case); observed errors are printed.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
from harness import normwise
from linear_attention_token_shortconv_b200 import gdn
from linear_attention_token_shortconv_b200.workloads import TINY_F32, make_prefill_inputs, scaled

pytestmark = pytest.mark.gpu

TOL_BWD = 2e-5

CASES = [
    ("varlen-d64-long-memory", scaled(TINY_F32, lengths=(37, 2, 20, 64), H=2, long_memory=True, s0_var=0.02,
                                      varlen=True), True),
    ("d128-one-seq", replace(scaled(TINY_F32, lengths=(87,), H=2, s0_var=0.02), dk=128, dv=128), True),
    ("d128-short-memory-no-S0", replace(scaled(TINY_F32, lengths=(150, 33), H=3, varlen=True), dk=128, dv=128),
     False),
    ("d64-equal-lengths", scaled(TINY_F32, lengths=(48, 48), H=2, s0_var=0.02), True),
    ("d128-long-memory", replace(scaled(TINY_F32, lengths=(300,), H=2, long_memory=True, s0_var=0.02),
                                 dk=128, dv=128), True),
]

GRADS = ["dq", "dk", "dv", "d_conv_w", "d_a_logit", "d_b_logit", "d_A", "d_b_alpha", "d_z", "d_norm_w", "d_S0"]


def _run(cfg, with_final_grad, device):
    inp = make_prefill_inputs(cfg, "cpu")
    rng = np.random.default_rng(cfg.seed + 7)
    inp["norm_w"] = torch.from_numpy((0.3 * rng.standard_normal(cfg.dv)).astype(np.float32))
    d_out = rng.standard_normal((cfg.total_tokens, cfg.H, cfg.dv)).astype(np.float32)
    d_S = (rng.standard_normal((cfg.num_seqs, cfg.H, cfg.dk, cfg.dv)).astype(np.float32)
           if with_final_grad else None)
    cu = inp.get("cu_seqlens")
    ref = oracle.backward(*(inp[key].numpy() for key in ("q", "k", "v", "conv_w", "a_logit", "b_logit", "A",
                                                         "b_alpha", "z", "norm_w")),
                          d_out.astype(np.float64),
                          S0=None if inp.get("S0") is None else inp["S0"].numpy(),
                          d_S_final=None if d_S is None else d_S.astype(np.float64),
                          cu_seqlens=None if cu is None else cu.numpy(), num_seqs=cfg.num_seqs)
    dev = {key: (None if val is None else val.to(device)) for key, val in inp.items()}
    got = gdn.prefill_backward(dev["q"], dev["k"], dev["v"], dev["conv_w"], dev["a_logit"], dev["b_logit"],
                               dev["A"], dev["b_alpha"], dev["z"], dev["norm_w"],
                               torch.from_numpy(d_out).to(device), S0=dev.get("S0"),
                               d_S_final=None if d_S is None else torch.from_numpy(d_S).to(device),
                               cu_seqlens=dev.get("cu_seqlens"), num_seqs=cfg.num_seqs)
    torch.cuda.synchronize()
    return got, ref


@pytest.mark.parametrize("name,cfg,final_grad", CASES, ids=[c[0] for c in CASES])
def test_backward_matches_oracle(cuda_device, name, cfg, final_grad):
    got, ref = _run(cfg, final_grad, cuda_device)
    errs = {key: normwise(got[key].cpu().numpy(), ref[key]) for key in GRADS}
    print(name, " ".join(f"{key} {val:.1e}" for key, val in errs.items()))
    for key, val in errs.items():
        assert val <= TOL_BWD, (key, val)


def test_backward_empty_batch(cuda_device):
    """No tokens: d_S0 = d_S_final, every other gradient zero."""
    H, D = 2, 64
    f = lambda *s: torch.zeros(s, dtype=torch.float32, device=cuda_device)
    rng = np.random.default_rng(5)
    d_S = torch.from_numpy(rng.standard_normal((1, H, D, D)).astype(np.float32)).to(cuda_device)
    S0 = torch.from_numpy(rng.standard_normal((1, H, D, D)).astype(np.float32)).to(cuda_device)
    conv_w = torch.from_numpy(rng.standard_normal((3 * H * D, 4)).astype(np.float32)).to(cuda_device)
    got = gdn.prefill_backward(f(0, H, D), f(0, H, D), f(0, H, D), conv_w, f(0, H), f(0, H), f(H), f(H),
                               f(0, H, D), f(D), f(0, H, D), S0=S0, d_S_final=d_S, num_seqs=1)
    torch.cuda.synchronize()
    assert torch.equal(got["d_S0"], d_S)
    for key in ("d_conv_w", "d_norm_w", "d_A", "d_b_alpha"):
        assert not torch.any(got[key]), key


def test_backward_is_deterministic(cuda_device):
    cfg = CASES[0][1]
    a, _ = _run(cfg, True, cuda_device)
    b, _ = _run(cfg, True, cuda_device)
    for key in GRADS:
        assert torch.equal(a[key], b[key]), key
