"""Launch accounting through the C ABI: gdn_last_call_launches() counts the
kernels a call launched, gdn_last_call_slots() its launch slots, and
gdn_set_kernel_events() brackets each slot with the caller's events (the hooks bench.py uses for its per-kernel timing)."""
from dataclasses import replace

import pytest
import torch

from harness import gpu_prefill, to_device
from linear_attention_token_shortconv_b200 import gdn
from linear_attention_token_shortconv_b200.workloads import (DECODE, PRETRAIN, make_decode_inputs,
                                                             make_prefill_inputs, scaled)

pytestmark = pytest.mark.gpu


def _events(n):
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for e in ev:
        e.record()
    torch.cuda.synchronize()
    return ev


@pytest.mark.parametrize("lengths,H,dv,launches,slots", [
    ((1280,), 2, 128, 1, 1),         # few (sequence, head) chains: the fused persistent kernel
    ((320,), 40, 128, 1, 1),         # 40 equal-length chains, still one fused launch
    ((300, 150, 90), 4, 128, 2, 1),  # unequal lengths: task-list builder + fused kernel, one slot
    ((320,), 40, 64, 2, 2),          # d_v = 64: segmented pipeline, one segment (prep, chain)
    ((1280,), 40, 64, 6, 6),         # three segments of 8, 8 and 4 chunks
])
def test_prefill_launch_slots(cuda_device, lengths, H, dv, launches, slots):
    cfg = replace(scaled(PRETRAIN, lengths=lengths, H=H), dv=dv)
    inp = to_device(make_prefill_inputs(cfg, "cpu"), cuda_device)
    b, e = _events(slots + 2), _events(slots + 2)
    gdn.set_kernel_events(b, e)
    try:
        gpu_prefill(inp, 1)
    finally:
        gdn.set_kernel_events()
    assert gdn.last_call_launches() == launches
    assert gdn.last_call_slots() == slots
    torch.cuda.synchronize()
    for i in range(slots):
        assert b[i].elapsed_time(e[i]) > 0.0, i


def test_decode_launch_slot(cuda_device):
    cfg = replace(DECODE, B=4, H=2)
    g = to_device(make_decode_inputs(cfg, "cpu"), cuda_device)
    b, e = _events(1), _events(1)
    gdn.set_kernel_events(b, e)
    try:
        gdn.decode_step(g["q"][0], g["k"][0], g["v"][0], g["conv_w"], g["ring"], g["a_logit"][0],
                        g["b_logit"][0], g["A"], g["b_alpha"], g["z"][0], g["norm_w"], g["S"])
    finally:
        gdn.set_kernel_events()
    assert gdn.last_call_launches() == 1
    assert gdn.last_call_slots() == 1
    torch.cuda.synchronize()
    assert b[0].elapsed_time(e[0]) > 0.0
