"""gdn_prefill_noalloc: the tensor-core prefill for callers that cannot allocate
device memory (its workspace lives in a fixed array inside the library).

Checked through the C ABI against the fp64 oracle and against gdn_prefill on
the same inputs, on calls in a row with different shapes (so a stale workspace
from one call would show in the next), plus its size limit.  This file is collected last so a run
that stops at the first failure has run every other test first; it also passes
alone in a fresh process."""
import ctypes

import pytest
import torch

from harness import TOL_BF16, normwise, oracle_full
from linear_attention_token_shortconv_b200 import gdn
from linear_attention_token_shortconv_b200.workloads import PRETRAIN, VARLEN, make_prefill_inputs, scaled

pytestmark = pytest.mark.gpu


def _args(inp):
    return (inp["q"], inp["k"], inp["v"], inp["conv_w"], inp["a_logit"], inp["b_logit"], inp["A"],
            inp["b_alpha"], inp["z"], inp["norm_w"])


def test_noalloc_matches_prefill_and_oracle_on_two_calls(cuda_device):
    """Three calls in a row with different shapes (a stale workspace from one call
    would show in the next), the last with dv = 64.  Each is checked against the
    fp64 oracle at the bf16 tolerance and against gdn_prefill on the same inputs."""
    from dataclasses import replace
    cases = [scaled(PRETRAIN, lengths=(700, 129), H=4, s0_var=0.02),
             scaled(VARLEN, lengths=(65, 1, 300, 0, 64), H=3),
             replace(scaled(PRETRAIN, lengths=(190, 3), H=2, s0_var=0.02), dv=64)]
    for cfg in cases:
        inp_cpu = make_prefill_inputs(cfg, "cpu")
        inp = {k: (None if v is None else v.to(cuda_device)) for k, v in inp_cpu.items()}
        kw = dict(S0=inp["S0"], cu_seqlens=inp["cu_seqlens"], num_seqs=cfg.num_seqs)
        ref_out, ref_S = gdn.prefill(*_args(inp), **kw)
        out, S = gdn.prefill_noalloc(*_args(inp), **kw)
        torch.cuda.synchronize()
        o_ref, s_ref = oracle_full(inp_cpu)
        e_out = normwise(out.cpu().numpy(), o_ref)
        e_s = normwise(S.cpu().numpy(), s_ref)
        d_out = normwise(out.cpu().numpy(), ref_out.cpu().numpy())
        d_s = normwise(S.cpu().numpy(), ref_S.cpu().numpy())
        print(f"{cfg.lengths} dv={cfg.dv}: vs oracle out {e_out:.1e} S {e_s:.1e}; "
              f"vs gdn_prefill out {d_out:.1e} S {d_s:.1e}")
        assert e_out <= TOL_BF16 and e_s <= TOL_BF16
        assert d_out <= TOL_BF16 and d_s <= TOL_BF16


def test_noalloc_rejects_sizes_beyond_its_array(cuda_device):
    per = 3 * 128 * 2 + 128 * 2 + 64 * 2 + 4
    n_tok = (32 << 20) // per + 64          # just over the fixed workspace
    cfg = scaled(PRETRAIN, lengths=(n_tok,), H=1)
    inp = make_prefill_inputs(cfg, cuda_device)
    with pytest.raises(gdn.GdnError) as ei:
        gdn.prefill_noalloc(*_args(inp))
    assert ei.value.status == 1   # GDN_ERR_INVALID_ARG, nothing launched


def test_noalloc_rejects_the_fp32_path(cuda_device):
    cfg = scaled(PRETRAIN, lengths=(64,), H=1, in_dtype=torch.float32)
    inp = make_prefill_inputs(cfg, cuda_device)
    with pytest.raises(gdn.GdnError) as ei:
        gdn.prefill_noalloc(*_args(inp))
    assert ei.value.status == 2   # GDN_ERR_UNSUPPORTED
