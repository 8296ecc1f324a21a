"""The two building blocks the attention kernels rest on, checked in
isolation on the GPU: one tensor-core tile in both operand forms, and the
bounded wait that gives up instead of hanging."""
import pytest
import torch

import exact_io_aware_65_b200 as fa
from helpers import has_gpu

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not has_gpu(), reason="needs a B200")]


@pytest.mark.parametrize("n", [64, 128])
@pytest.mark.parametrize("k", [64, 128])
def test_mma_tile_both_operands_in_smem(n, k):
    g = torch.Generator().manual_seed(n * 1000 + k)
    A = torch.randn(128, k, generator=g).to(torch.bfloat16)
    Bt = torch.randn(n, k, generator=g).to(torch.bfloat16)
    C = fa.selftest_mma_tile(A.cuda(), Bt.cuda(), n, k, mode=0)
    torch.cuda.synchronize()
    ref = A.double() @ Bt.double().T
    torch.testing.assert_close(C.cpu().double(), ref, atol=1e-3, rtol=1e-4)


@pytest.mark.parametrize("n", [64, 128])
@pytest.mark.parametrize("k", [64, 128])
def test_mma_tile_a_in_tensor_memory(n, k):
    g = torch.Generator().manual_seed(7 + n * 1000 + k)
    A = torch.randn(128, k, generator=g).to(torch.bfloat16)
    B = torch.randn(k, n, generator=g).to(torch.bfloat16)
    C = fa.selftest_mma_tile(A.cuda(), B.cuda(), n, k, mode=1)
    torch.cuda.synchronize()
    ref = A.double() @ B.double()
    torch.testing.assert_close(C.cpu().double(), ref, atol=1e-3, rtol=1e-4)


def test_bounded_wait_times_out_and_reports():
    assert fa.device_status() == 0
    fa.selftest_bounded_wait(50_000_000)  # 50 ms
    assert fa.device_status() == 5          # FA_ERR_TIMEOUT, then cleared
    assert fa.device_status() == 0
    # the context is still usable
    x = torch.ones(4, device="cuda")
    assert float(x.sum()) == 4.0
