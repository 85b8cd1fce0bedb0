"""The decoder layer's tensor-core GEMM (s2o_gemm_bf16, through the C ABI) against a plain PyTorch
fp32 product of the same bf16 operands: C = bf16(A·B) or bf16(C + A·B), with full tiles, ragged
edges in every dimension (m not a multiple of 128, n not of 256, k not of 64), and several tiles
per CTA. Both kernels behind the call are covered: the CTA pair (n and k up to 8192, at least two
256 × 256 tiles) and the single-CTA kernel (one tile, n above 8192, or k above 8192)."""
import pytest
import torch

import long_context_sparse_stripe_b200 as s2o

pytestmark = pytest.mark.gpu


def reference(a, b, c=None):
    out = a.float() @ b.float()
    if c is not None:
        out = out + c.float()
    return out


@pytest.mark.parametrize("m,n,k", [(128, 256, 64), (256, 512, 128), (300, 520, 72),
                                   (1000, 776, 200), (4096, 2048, 4096), (129, 8, 8),
                                   (520, 8200, 72), (300, 264, 8208)])
@pytest.mark.parametrize("accumulate", [False, True])
def test_gemm_matches_fp32_product(m, n, k, accumulate):
    g = torch.Generator(device="cuda").manual_seed(m * 7 + n * 3 + k)
    a = torch.randn(m, k, device="cuda", generator=g).to(torch.bfloat16)
    b = (torch.randn(k, n, device="cuda", generator=g) / k ** 0.5).to(torch.bfloat16)
    c0 = torch.randn(m, n, device="cuda", generator=g).to(torch.bfloat16)
    c = c0.clone()
    out = s2o.gemm_bf16(a, b, c if accumulate else None, accumulate=accumulate)
    torch.cuda.synchronize()
    assert s2o.check_device_status() == 0
    want = reference(a, b, c0 if accumulate else None)
    err = (out.float() - want).abs()
    # One bf16 rounding of the result (half an ulp: 2^-9 relative) plus fp32 summation order.
    bound = want.abs() * 2.0 ** -8 + 1e-3
    assert (err <= bound).all(), f"max error {err.max().item():.3g}"
