"""Tensor-core building blocks (tcgen05.mma, TMEM, TMA, 128-byte swizzle)
checked against a plain PyTorch fp32 product of the same bf16 operands."""
import pytest
import torch

from chunked_state_space_b200 import ssd

pytestmark = pytest.mark.gpu

CORRECT = ["A_K_B_K", "A_K_B_MN", "A_MN_B_MN", "TS_A_TMEM_B_MN", "TMA_A_K_B_MN"]


def _operands(variant, N, K, seed=0):
    g = torch.Generator().manual_seed(seed)
    A = torch.randn(128, K, generator=g).to(torch.bfloat16)
    B = torch.randn(K, N, generator=g).to(torch.bfloat16)
    ref = A.float() @ B.float()
    a_dev = A.t().contiguous() if variant.startswith("A_MN") else A
    b_dev = B.t().contiguous() if variant == "A_K_B_K" else B
    return a_dev.cuda(), b_dev.cuda(), ref


@pytest.mark.parametrize("N,K", [(64, 64), (64, 256), (128, 128), (128, 256)])
@pytest.mark.parametrize("variant", CORRECT)
def test_umma_layouts(variant, N, K):
    a, b, ref = _operands(variant, N, K)
    D = ssd.ssd_selftest_umma(variant, a, b, N, K)
    torch.cuda.synchronize()
    assert ssd.ssd_read_device_status() == 0
    err = (D.cpu() - ref).abs().max().item() / ref.abs().max().item()
    assert err < 1e-5, f"{variant} N={N} K={K}: rel err {err}"


def test_swapped_strides_differ():
    """With M = 128 an MN-major A spans two 64-wide blocks; exchanging the two
    descriptor strides must change the product (documents which field is which)."""
    a, b, ref = _operands("A_MN_B_MN_SWAPPED", 64, 128)
    D = ssd.ssd_selftest_umma("A_MN_B_MN_SWAPPED", a, b, 64, 128)
    torch.cuda.synchronize()
    assert ssd.ssd_read_device_status() == 0
    err = (D.cpu() - ref).abs().max().item() / ref.abs().max().item()
    assert err > 1e-2
