"""Failure detection on the GPU without a fault: each kernel family's bounded
wait is made to run out (one CTA waits for an mbarrier phase that nothing
completes); the family's device error word must come back through
gdn_device_error_status, clear, and leave the context usable for a normal call."""
import pytest
import torch

from harness import TOL_BF16, gpu_prefill, normwise, oracle_full, to_device
from linear_attention_token_shortconv_b200 import gdn
from linear_attention_token_shortconv_b200.workloads import PRETRAIN, make_prefill_inputs, scaled

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("family", [gdn.ERRF_PREP, gdn.ERRF_CHAIN, gdn.ERRF_DECODE, gdn.ERRF_QSA, gdn.ERRF_GEMM])
def test_expired_wait_is_reported(cuda_device, family):
    gdn.device_error_status(clear=True)    # start clean
    assert gdn.device_error_status() == (0, 0)
    gdn.selftest_wait_timeout(family, max_polls=1024)
    st, flags = gdn.device_error_status(clear=True)
    assert st == 5 and flags == family
    assert gdn.device_error_status() == (0, 0)


def test_context_usable_after_expired_waits(cuda_device):
    for f in (gdn.ERRF_PREP, gdn.ERRF_CHAIN, gdn.ERRF_DECODE, gdn.ERRF_QSA, gdn.ERRF_GEMM):
        gdn.selftest_wait_timeout(f, max_polls=256)
    assert gdn.device_error_status(clear=True) == (5, 31)
    cfg = scaled(PRETRAIN, lengths=(200, 72), H=2)
    cpu = make_prefill_inputs(cfg, "cpu")
    out, SF = gpu_prefill(to_device(cpu, cuda_device), 2)
    o_ref, s_ref = oracle_full(cpu)
    assert normwise(out.cpu().numpy(), o_ref) < TOL_BF16
    assert normwise(SF.cpu().numpy(), s_ref) < TOL_BF16
    assert gdn.device_error_status() == (0, 0)
