"""tcgen05 operand layouts (K-major / MN-major, 128-byte swizzle; A also from
tensor memory), TMEM accumulation and A negation, checked against a plain
matmul of the same fp16 values.  The chunked prefill kernels stage their operands with the same helpers."""
import itertools

import pytest
import torch

from linear_attention_token_shortconv_b200 import gdn

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("a_mn,b_mn,N,K", list(itertools.product([0, 1, 2], [0, 1], [64, 128], [64, 128])))
def test_umma_layouts(cuda_device, a_mn, b_mn, N, K):
    g = torch.Generator(device="cpu").manual_seed(1000 * a_mn + 100 * b_mn + N + K)
    A = torch.randn(128, K, generator=g).half()
    B = torch.randn(K, N, generator=g).half()
    ref = A.float() @ B.float()
    D = gdn.selftest_umma(A.to(cuda_device), B.to(cuda_device), a_mn=a_mn, b_mn=b_mn)
    err = (D.cpu() - ref).abs().max().item()
    assert err <= 1e-4 * ref.abs().max().item(), err


@pytest.mark.parametrize("a_mn,b_mn", [(0, 1), (1, 1)])
def test_umma_accumulate_onto_tmem_init_and_negate(cuda_device, a_mn, b_mn):
    g = torch.Generator(device="cpu").manual_seed(7)
    A = torch.randn(128, 64, generator=g).half()
    B = torch.randn(64, 128, generator=g).half()
    init = torch.randn(128, 128, generator=g)
    ref = init - A.float() @ B.float()
    D = gdn.selftest_umma(A.to(cuda_device), B.to(cuda_device), init.to(cuda_device), a_mn=a_mn,
                          b_mn=b_mn, negate_a=True)
    err = (D.cpu() - ref).abs().max().item()
    assert err <= 1e-4 * ref.abs().max().item(), err


@pytest.mark.parametrize("b_mn,N", [(0, 64), (1, 128)])
def test_umma_tmem_a_accumulates_onto_tmem_init(cuda_device, b_mn, N):
    g = torch.Generator(device="cpu").manual_seed(11 + N)
    A = torch.randn(128, 128, generator=g).half()
    B = torch.randn(128, N, generator=g).half()
    init = torch.randn(128, N, generator=g)
    ref = init + A.float() @ B.float()
    D = gdn.selftest_umma(A.to(cuda_device), B.to(cuda_device), init.to(cuda_device), a_mn=2,
                          b_mn=b_mn)
    err = (D.cpu() - ref).abs().max().item()
    assert err <= 1e-4 * ref.abs().max().item(), err
