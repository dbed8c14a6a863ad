"""The allocation-free decode entry point (fp4_gemm_decode_noalloc) against the
decode entry point that takes a caller workspace (fp4_gemm_with_kernel with
FP4_GEMM_DECODE), through the C ABI.

The no-alloc form exists for callers that cannot allocate device memory on
their hot path (a plug-in inside a framework that owns the GPU's memory pool,
or a latency-bound loop where cudaMalloc would synchronize the device); its
split-K partials live in a fixed array inside the library.  Two calls in a
row on different shapes check that the second call does not depend on what
the first one left in that shared array.

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


def _operands(M, N, K, seed):
    A = synth.normal_bf16(M, K, seed=seed, outlier_factor=100.0)
    W = synth.normal_bf16(N, K, seed=seed, tensor_id=1, sigma=0.02)
    Ad = synth.bits_to_torch(A).cuda()
    Wd = synth.bits_to_torch(W).cuda()
    gA, gW = fp4.global_scale(Ad), fp4.global_scale(Wd)
    alpha = torch.empty(1, dtype=torch.float32, device="cuda")
    fp4.fp4_alpha_from_global_scales(gA, gW, alpha)
    pA, sA = fp4.quantize(Ad, fp4.NVFP4, fp4.ROWWISE, gA)
    pW, sW = fp4.quantize(Wd, fp4.NVFP4, fp4.ROWWISE, gW)
    return (A, W, gA, gW), (pA, sA, pW, sW, alpha)


def test_noalloc_decode_matches_workspace_decode_on_two_calls(orc):
    f = _noalloc()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for M, N, K, seed in [(16, 2048, 4096, 51), (3, 1152, 2048, 52)]:
        host, (pA, sA, pW, sW, alpha) = _operands(M, N, K, seed)
        D_ref = fp4.gemm(fp4.NVFP4, pA, sA, pW, sW, K, alpha=alpha, kernel=fp4.GEMM_DECODE)
        D_new = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = f(fp4.NVFP4, _p(pA), _p(sA), _p(pW), _p(sW), M, N, K, _p(alpha), _p(D_new), N, stream)
        assert st == 0, fp4.lib().fp4_last_error()
        torch.cuda.synchronize()
        assert fp4.fp4_get_device_status() == 0
        d_ref, d_new = bf16_dev_to_f64(D_ref), bf16_dev_to_f64(D_new)
        # tolerance of the GEMM parity tests, with S from the oracle
        A, W, gA, gW = host
        gsA, gsW = np.float32(gA.item()), np.float32(gW.item())
        qA, qsA = orc.quantize(orc.NVFP4, orc.ROWWISE, A, gs=float(gsA))
        qW, qsW = orc.quantize(orc.NVFP4, orc.ROWWISE, W, gs=float(gsW))
        _, S = orc.gemm(orc.NVFP4, qA, qsA, qW, qsW, alpha=float(gsA * gsW))
        assert_gemm_close(d_new, d_ref, S, "no-alloc vs workspace decode")
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
