"""The attention block's projection GEMM (tcgen05, 128 x 256 tiles) through
the C ABI, against a float64 product of the same bf16 inputs on the CPU.

The output is rounded to bf16 (relative step 2^-8), so elements are compared
with |C - R| <= 2^-8 |R| + 1e-3 max|R|, the second term covering fp32
accumulation over K <= 1536 terms of mixed sign.  Shapes: the block's two
projections at the full 1560-token size, plus ragged cases whose M, N and K
are not multiples of the tile sizes (128, 256, 64)."""
import numpy as np
import pytest
import torch

from hybrid_linear_attention_arl2_b200 import arl2, build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    arl2.load_library()


@pytest.mark.parametrize("M,N,K", [(1560, 4632, 1536), (1560, 1536, 1536), (1, 8, 64), (130, 264, 72),
                                   (300, 520, 200), (6240, 1536, 1536)])
def test_gemm_matches_float64_product(M, N, K):
    g = torch.Generator().manual_seed(M * 7 + N * 3 + K)
    a = (torch.randn(M, K, generator=g) / 4).to(torch.bfloat16)
    b = (torch.randn(K, N, generator=g) / K ** 0.5).to(torch.bfloat16)
    ref = a.double() @ b.double()
    c = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    arl2.arl2_gemm_bf16(a.cuda(), b.cuda(), c, M, N, K)
    torch.cuda.synchronize()
    got = c.cpu().double()
    assert torch.isfinite(got).all()
    bound = 2.0 ** -8 * ref.abs() + 1e-3 * ref.abs().max()
    bad = ((got - ref).abs() > bound).sum().item()
    assert bad == 0, f"{bad} elements out of bound; max err {(got - ref).abs().max().item():.3e}"


def test_gemm_with_row_pitch_writes_only_its_columns():
    """C as a column block of a wider matrix (ldc > N): the columns beside it
    keep their values."""
    M, N, K, ldc = 200, 264, 128, 512
    g = torch.Generator().manual_seed(5)
    a = torch.randn(M, K, generator=g).to(torch.bfloat16)
    b = (torch.randn(K, N, generator=g) / K ** 0.5).to(torch.bfloat16)
    c = torch.full((M, ldc), 7.0, dtype=torch.bfloat16, device="cuda")
    arl2.arl2_gemm_bf16(a.cuda(), b.cuda(), c, M, N, K, ldc=ldc)
    torch.cuda.synchronize()
    host = c.cpu()
    assert (host[:, N:] == 7.0).all()
    ref = a.double() @ b.double()
    assert ((host[:, :N].double() - ref).abs() <= 2.0 ** -8 * ref.abs() + 1e-3 * ref.abs().max()).all()
