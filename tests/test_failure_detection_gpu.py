"""Failure detection without a GPU fault: a kernel's bounded wait runs out (a
barrier nothing completes), the kernel records FP4_ERR_TIMEOUT and returns,
the host reads the status, and the context keeps working."""
import pytest
import torch

from block_scaled_fp4_05_b200 import fp4

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    assert fp4.fp4_get_device_status() == 0
    fp4.fp4_selftest_bounded_wait()
    assert fp4.fp4_get_device_status() == 5          # FP4_ERR_TIMEOUT, then cleared
    assert fp4.fp4_get_device_status() == 0
    # the context is usable: a GEMM with a closed-form result
    M, N, K = 256, 256, 512
    A = torch.full((M, K // 2), 0x22, dtype=torch.uint8, device="cuda")     # 1.0
    B = torch.full((N, K // 2), 0x11, dtype=torch.uint8, device="cuda")     # 0.5
    sA = torch.full((fp4.fp4_scale_bytes(fp4.MXFP4, M, K),), 127, dtype=torch.uint8, device="cuda")
    sB = torch.full((fp4.fp4_scale_bytes(fp4.MXFP4, N, K),), 127, dtype=torch.uint8, device="cuda")
    D = fp4.gemm(fp4.MXFP4, A, sA, B, sB, K)
    torch.cuda.synchronize()
    assert torch.all(D.float() == 0.5 * K)
    assert fp4.fp4_get_device_status() == 0
