"""The allocation-free decode entry point (fp4_gemm_decode_noalloc) against the
decode entry point that takes a caller workspace (fp4_gemm_with_kernel with
FP4_GEMM_DECODE), through the C ABI.

The no-alloc form exists for callers that cannot allocate device memory on
their hot path (a plug-in inside a framework that owns the GPU's memory pool,
or a latency-bound loop where cudaMalloc would synchronize the device); its
split-K partials live in a fixed array inside the library.  Calls in a row
on different shapes and formats check each result against the oracle and
that no call depends on what the previous one left in that shared array.

Kept in a file that sorts last, so that a run stopping at the first failure
has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

from block_scaled_fp4_05_b200 import fp4, synth
from gpu_util import assert_gemm_close, bf16_dev_to_f64

pytestmark = pytest.mark.gpu


def _noalloc():
    f = fp4.lib().fp4_gemm_decode_noalloc
    P, i64 = ctypes.c_void_p, ctypes.c_int64
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int, P, P, P, P, i64, i64, i64, P, P, i64, P]
    return f


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _operands(fmt, M, N, K, seed):
    A = synth.normal_bf16(M, K, seed=seed, outlier_factor=100.0)
    W = synth.normal_bf16(N, K, seed=seed, tensor_id=1, sigma=0.02)
    Ad = synth.bits_to_torch(A).cuda()
    Wd = synth.bits_to_torch(W).cuda()
    if fmt == fp4.NVFP4:
        gA, gW = fp4.global_scale(Ad), fp4.global_scale(Wd)
        alpha = torch.empty(1, dtype=torch.float32, device="cuda")
        fp4.fp4_alpha_from_global_scales(gA, gW, alpha)
    else:
        gA = gW = alpha = None
    pA, sA = fp4.quantize(Ad, fmt, fp4.ROWWISE, gA)
    pW, sW = fp4.quantize(Wd, fmt, fp4.ROWWISE, gW)
    return (A, W, gA, gW), (pA, sA, pW, sW, alpha)


def test_noalloc_decode_matches_oracle_and_workspace_decode_on_two_calls(orc):
    # three calls in a row on different shapes and both formats: the shared
    # scratch keeps what the previous call left there, and each result must
    # still match the oracle (within the GEMM tolerance) and the workspace
    # form of the same kernel bit for bit
    f = _noalloc()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for fmt, M, N, K, seed in [(fp4.NVFP4, 16, 2048, 4096, 51), (fp4.NVFP4, 3, 1152, 2048, 52),
                               (fp4.MXFP4, 4, 1536, 4096, 53)]:
        host, (pA, sA, pW, sW, alpha) = _operands(fmt, M, N, K, seed)
        D_ref = fp4.gemm(fmt, pA, sA, pW, sW, K, alpha=alpha, kernel=fp4.GEMM_DECODE)
        D_new = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = f(fmt, _p(pA), _p(sA), _p(pW), _p(sW), M, N, K, _p(alpha), _p(D_new), N, stream)
        assert st == 0, fp4.lib().fp4_last_error()
        torch.cuda.synchronize()
        assert fp4.fp4_get_device_status() == 0
        d_ref, d_new = bf16_dev_to_f64(D_ref), bf16_dev_to_f64(D_new)
        # the oracle's product of its own quantization of the same inputs
        A, W, gA, gW = host
        gsA = float(np.float32(gA.item())) if gA is not None else 1.0
        gsW = float(np.float32(gW.item())) if gW is not None else 1.0
        ofmt = orc.NVFP4 if fmt == fp4.NVFP4 else orc.MXFP4
        qA, qsA = orc.quantize(ofmt, orc.ROWWISE, A, gs=gsA)
        qW, qsW = orc.quantize(ofmt, orc.ROWWISE, W, gs=gsW)
        D_orc, S = orc.gemm(ofmt, qA, qsA, qW, qsW, alpha=float(np.float32(gsA) * np.float32(gsW)))
        assert_gemm_close(d_new, D_orc, S, "no-alloc decode vs oracle")
        # same kernels, fixed reduction order: identical bits
        assert np.array_equal(d_new, d_ref)


def test_noalloc_decode_rejects_unsupported_shapes():
    f = _noalloc()
    d = torch.zeros(64, dtype=torch.uint8, device="cuda")
    D = torch.zeros((16, 64), dtype=torch.bfloat16, device="cuda")
    # Only shapes that the validation rejects whatever the device get the
    # undersized buffers above.  (With the stream-K + whole-tile schedule a CTA
    # holds at most 3 partial slots, so on a 148-SM device every accepted
    # shape fits the 4 MiB scratch; that bound is checked without a launch.)
    for N, K in [(65536, 256), (524288, 8192), (28672, 8192), (1024, 64)]:
        assert 0 < fp4.fp4_gemm_workspace_bytes(fp4.NVFP4, 16, N, K) <= 4 << 20
    N = 1 << 20   # beyond the decode kernel's arrival counters
    st = f(fp4.NVFP4, _p(d), _p(d), _p(d), _p(d), 16, N, 8192, None, _p(D), N, None)
    assert st == 2
    assert b"arrival counters" in fp4.lib().fp4_last_error()
    st = f(fp4.NVFP4, _p(d), _p(d), _p(d), _p(d), 17, 64, 64, None, _p(D), 64, None)
    assert st == 2
