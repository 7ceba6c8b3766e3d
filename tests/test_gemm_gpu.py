"""The library's bf16 GEMM (gdn_gemm_bf16, the layer's projections) against a
plain fp32 PyTorch product of the same bf16 operands.

Tolerance: C is rounded to bf16 once (half a unit in the last place, 2^-9 of an
element), after an fp32 accumulation whose order differs from the reference's
(relative 1e-6 over K = 2048): every element within 2^-8 of the largest |C|.
The shapes cover both tile shapes (N >= 64 and the narrow N < 64), ragged M, N
and K (K = 200 is not a whole 64-wide block), leading dimensions wider than the
matrices, and the layer's full in-projection block.
"""
import pytest
import torch

from linear_attention_token_shortconv_b200 import gdn

pytestmark = pytest.mark.gpu

TOL = 2.0 ** -8

SHAPES = [
    (300, 256, 512),      # one column of tiles, ragged M
    (257, 2048, 200),     # K tail inside a 64-wide block
    (128, 320, 64),       # N not a multiple of the 256-wide tile
    (1000, 40, 1024),     # narrow shape (B transposed)
    (999, 16, 2048),      # narrow, one gate-logit block
]


def _check(a, b, c):
    ref = a.float() @ b.float()
    err = float((c.float() - ref).abs().max() / ref.abs().max())
    assert err <= TOL, err
    return err


@pytest.mark.parametrize("M,N,K", SHAPES, ids=[f"{m}x{n}x{k}" for m, n, k in SHAPES])
def test_gemm_matches_fp32_product(cuda_device, M, N, K):
    g = torch.Generator(device=cuda_device).manual_seed(M * 7 + N * 13 + K)
    a = torch.randn((M, K), generator=g, device=cuda_device).to(torch.bfloat16)
    b = (torch.randn((K, N), generator=g, device=cuda_device) / K ** 0.5).to(torch.bfloat16)
    c = gdn.gemm_bf16(a, b)
    torch.cuda.synchronize()
    _check(a, b, c)


def test_gemm_strided_operands(cuda_device):
    """Sub-matrices of wider buffers, as the layer's column blocks of W_in."""
    g = torch.Generator(device=cuda_device).manual_seed(5)
    A = torch.randn((400, 520), generator=g, device=cuda_device).to(torch.bfloat16)
    B = (torch.randn((512, 8224), generator=g, device=cuda_device) / 512 ** 0.5).to(torch.bfloat16)
    C = torch.zeros((400, 1040), dtype=torch.bfloat16, device=cuda_device)
    a, b = A[:, :512], B[:, 2048:4096]
    out = C[:, 16:16 + 2048 - 1024 - 16]                    # 1008 columns, leading dimension 1040
    b = b[:, :out.shape[1]]
    gdn.gemm_bf16(a, b, out=out)
    torch.cuda.synchronize()
    _check(a, b, out)
    assert torch.count_nonzero(C[:, :16]) == 0 and torch.count_nonzero(C[:, 16 + out.shape[1]:]) == 0


def test_gemm_full_in_projection_block(cuda_device):
    """The bench layer's q block: x [16384, 2048] times W_in[:, 0:2048] (ld 8224)."""
    g = torch.Generator(device=cuda_device).manual_seed(11)
    x = torch.randn((16384, 2048), generator=g, device=cuda_device).to(torch.bfloat16)
    w = (torch.randn((2048, 8224), generator=g, device=cuda_device) / 2048 ** 0.5).to(torch.bfloat16)
    c = gdn.gemm_bf16(x, w[:, :2048])
    torch.cuda.synchronize()
    rows = torch.tensor([0, 1, 127, 128, 4095, 8191, 12000, 16383], device=cuda_device)
    ref = x[rows].float() @ w[:, :2048].float()
    err = float((c[rows].float() - ref).abs().max() / ref.abs().max())
    assert err <= TOL, err


def test_gemm_empty(cuda_device):
    a = torch.empty((0, 64), dtype=torch.bfloat16, device=cuda_device)
    b = torch.randn((64, 128), device=cuda_device).to(torch.bfloat16)
    assert gdn.gemm_bf16(a, b).shape == (0, 128)
