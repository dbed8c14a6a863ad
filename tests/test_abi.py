"""The C-ABI library loads and exports every function include/fp4.h declares;
host-side checks and size helpers work without a GPU (no compute calls)."""
import ctypes

import pytest

from block_scaled_fp4_05_b200 import fp4


def test_library_exports_every_declared_symbol():
    L = fp4.lib()
    names = fp4.declared_symbols()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
    assert L.fp4_abi_version() == 4


def test_status_strings():
    for code, name in fp4.STATUS_NAMES.items():
        assert fp4.fp4_status_string(code) == name
    assert fp4.fp4_status_string(99) == "FP4_ERR_UNKNOWN"


def test_size_helpers_match_oracle_layout(orc):
    for fmt in (fp4.NVFP4, fp4.MXFP4):
        k = fp4.block_size(fmt)
        for rows, K in [(1, 512), (128, 4096), (129, 8192), (28672, 8192), (3, 128)]:
            assert fp4.fp4_packed_bytes(rows, K) == rows * K // 2
            assert fp4.fp4_scale_bytes(fmt, rows, K) == orc.scale_bytes(rows, K // k)
    assert fp4.fp4_scale_bytes(7, 128, 512) == 0
    assert fp4.fp4_packed_bytes(0, 512) == 0


P = ctypes.c_void_p
A16 = P(1 << 20)       # 16-byte aligned dummy address (never dereferenced)
A1 = P((1 << 20) + 1)  # misaligned


@pytest.mark.parametrize("args,want", [
    ((5, 0, A16, 128, 512, 512, A16, A16, A16, None), 1),      # bad format
    ((0, 3, A16, 128, 512, 512, A16, A16, A16, None), 1),      # bad axis
    ((0, 0, A16, 128, 512, 256, A16, A16, A16, None), 1),      # ld < cols
    ((0, 0, A16, 128, 512, 512, A16, A16, None, None), 1),     # NVFP4 without S_global
    ((0, 0, None, 128, 512, 512, A16, A16, A16, None), 1),     # NULL input
    ((0, 0, A16, 128, 480, 480, A16, A16, A16, None), 2),      # cols % 64
    ((1, 0, A16, 128, 192, 192, A16, A16, None, None), 2),     # cols % 128 (MX)
    ((1, 1, A16, 96, 64, 64, A16, A16, None, None), 2),        # colwise rows % 128 (MX)
    ((0, 0, A1, 128, 512, 512, A16, A16, A16, None), 3),       # misaligned input
    ((0, 0, A16, 128, 512, 516, A16, A16, A16, None), 3),      # ld % 8
    ((0, 0, A16, 0, 512, 512, None, None, None, None), 0),     # empty: no-op
    ((0, 0, A16, 128, 512, 512, A16, A16, A16, None), 6),      # valid, but no device here
])
def test_quantize_host_checks_without_gpu(args, want):
    import torch
    if torch.cuda.is_available() and want == 6:
        pytest.skip("a device is present")
    assert fp4.lib().fp4_quantize(*args) == want


def test_gemm_host_checks_without_gpu():
    import torch
    L = fp4.lib()
    g = L.fp4_gemm_with_kernel
    assert g(9, A16, A16, A16, A16, 16, 16, 64, None, A16, 16, None, 0, 0, None) == 1
    assert g(0, A16, A16, A16, A16, 16, 16, 64, None, A16, 16, None, 0, 7, None) == 1
    assert g(0, A16, A16, A16, A16, 16, 16, 96, None, A16, 16, None, 0, 0, None) == 2
    assert g(1, A16, A16, A16, A16, 16, 16, 64, None, A16, 16, None, 0, 0, None) == 2
    assert g(0, A16, A16, A16, A16, 16, 12, 64, None, A16, 16, None, 0, 0, None) == 2
    assert g(0, A16, A16, A16, A16, 16, 16, 64, None, A1, 16, None, 0, 0, None) == 3
    assert g(0, A16, A16, A16, A16, 16, 16, 64, None, A16, 8, None, 0, 0, None) == 1
    assert g(0, A16, A16, A16, A16, 0, 16, 64, None, A16, 16, None, 0, 0, None) == 0
    if not torch.cuda.is_available():
        assert g(0, A16, A16, A16, A16, 16, 16, 64, None, A16, 16, None, 0, 0, None) == 6
        assert L.fp4_compute_global_scale(A16, 4, 8, 8, A16, None) == 6
    assert L.fp4_compute_global_scale(A16, 4, 12, 12, A16, None) == 2
    assert L.fp4_alpha_from_global_scales(None, A16, A16, None) == 1


def test_quantize_batch_host_checks_without_gpu():
    import torch
    L = fp4.lib()
    D = fp4.QuantizeDesc

    def call(fmt, descs):
        arr = (D * max(1, len(descs)))(*descs)
        return L.fp4_quantize_batch(fmt, len(descs), ctypes.cast(arr, P), None)

    good = D(1 << 20, 128, 512, 512, 1 << 20, 1 << 20, 1 << 20)
    assert call(5, [good]) == 1                                          # bad format
    assert L.fp4_quantize_batch(0, -1, None, None) == 1                  # negative count
    assert L.fp4_quantize_batch(0, 2, None, None) == 1                   # NULL array
    assert call(0, [good, D(1 << 20, 128, 480, 480, 1 << 20, 1 << 20, 1 << 20)]) == 2   # cols % 64
    assert call(1, [D(1 << 20, 128, 192, 192, 1 << 20, 1 << 20, None)]) == 2           # cols % 128 (MX)
    assert call(0, [D(1 << 20, 128, 512, 512, 1 << 20, 1 << 20, None)]) == 1           # NV without S_global
    assert call(0, [D((1 << 20) + 2, 128, 512, 512, 1 << 20, 1 << 20, 1 << 20)]) == 3  # misaligned
    assert call(0, [D(0, 0, 512, 512, 0, 0, 0)]) == 0                                   # empty only: no-op
    assert L.fp4_quantize_batch(0, 0, None, None) == 0
    if not torch.cuda.is_available():
        assert call(0, [good]) == 6                                      # valid, but no device here


def test_p1e8_host_checks(orc):
    # 16-element blocks: the same sizes and K rule as NVFP4; S_global is
    # required by the quantizer; the GEMM accepts the format
    import torch
    L = fp4.lib()
    for rows, K in [(1, 512), (129, 8192)]:
        assert fp4.fp4_scale_bytes(fp4.P1E8, rows, K) == orc.scale_bytes(rows, K // 16)
    assert L.fp4_quantize(2, 0, A16, 128, 512, 512, A16, A16, None, None) == 1
    assert L.fp4_quantize(2, 0, A16, 128, 480, 480, A16, A16, A16, None) == 2
    g = L.fp4_gemm_with_kernel
    assert g(2, A16, A16, A16, A16, 16, 16, 96, None, A16, 16, None, 0, 0, None) == 2   # K % 64
    assert g(2, A16, A16, A16, A16, 16, 12, 64, None, A16, 16, None, 0, 0, None) == 2   # N % 8
    if not torch.cuda.is_available():
        assert g(2, A16, A16, A16, A16, 16, 16, 64, None, A16, 16, None, 0, 0, None) == 6


def test_gemm_grouped_host_checks_without_gpu():
    import torch
    L = fp4.lib()
    G = fp4.GemmProblem

    def call(fmt, probs):
        arr = (G * max(1, len(probs)))(*probs)
        return L.fp4_gemm_grouped(fmt, len(probs), ctypes.cast(arr, P), None)

    a = 1 << 20
    good = G(a, a, a, a, 16, 16, 64, None, a, 16)
    assert call(9, [good]) == 1                                         # bad format
    assert L.fp4_gemm_grouped(0, -1, None, None) == 1
    assert call(0, [good, G(a, a, a, a, 16, 16, 96, None, a, 16)]) == 2  # K % 64
    assert call(0, [good, G(a, a, a, a, 16, 12, 64, None, a, 16)]) == 2  # N % 8
    assert call(0, [G(a + 1, a, a, a, 16, 16, 64, None, a, 16)]) == 3    # misaligned A
    assert call(0, [G(0, 0, 0, 0, 0, 16, 64, None, 0, 16)]) == 0         # empty only: no-op
    if not torch.cuda.is_available():
        assert call(0, [good]) == 6


def test_dequantize_and_dynamic_host_checks_without_gpu():
    import torch
    L = fp4.lib()
    dq = L.fp4_dequantize
    assert dq(7, A16, A16, A16, 16, 512, A16, 512, None) == 1          # bad format
    assert dq(0, A16, A16, None, 16, 512, A16, 512, None) == 1         # NVFP4 without S_global
    assert dq(0, A16, A16, A16, 16, 512, A16, 256, None) == 1          # ld < k
    assert dq(0, A16, A16, A16, 16, 480, A16, 480, None) == 2          # k % 64
    assert dq(1, A16, A16, None, 16, 192, A16, 192, None) == 2         # k % 128 (MX)
    assert dq(0, A1, A16, A16, 16, 512, A16, 512, None) == 3           # misaligned packed
    assert dq(0, A16, A16, A16, 16, 512, A16, 516, None) == 3          # ld % 8
    assert dq(0, A16, A16, A16, 0, 512, A16, 512, None) == 0           # empty: no-op
    dyn = L.fp4_quantize_dynamic
    assert dyn(1, A16, 4, 128, 128, A16, A16, A16, None, None, None) == 1      # MXFP4: no S_global
    assert dyn(0, A16, 4, 128, 128, A16, A16, None, None, None, None) == 1     # no gs_out
    assert dyn(0, A16, 4, 128, 128, A16, A16, A16, None, A16, None) == 1       # alpha without other
    assert dyn(0, A16, 4, 96, 96, A16, A16, A16, None, None, None) == 2        # cols % 64
    assert dyn(0, A1, 4, 128, 128, A16, A16, A16, None, None, None) == 3       # misaligned input
    if not torch.cuda.is_available():
        assert dq(0, A16, A16, A16, 16, 512, A16, 512, None) == 6
        assert dyn(0, A16, 4, 128, 128, A16, A16, A16, None, None, None) == 6


def test_global_scale_alpha_host_checks_without_gpu():
    import torch
    L = fp4.lib()
    f = L.fp4_compute_global_scale_alpha
    assert f(A16, 4, 8, 8, A16, None, A16, None) == 1        # no other_gs
    assert f(A16, 4, 8, 8, A16, A16, None, None) == 1        # no alpha_out
    assert f(A16, 4, 8, 8, None, A16, A16, None) == 1        # no gs_out
    assert f(A16, 4, 8, 4, A16, A16, A16, None) == 1         # ld < cols
    assert f(A16, 4, 12, 12, A16, A16, A16, None) == 2       # cols % 8
    assert f(A1, 4, 8, 8, A16, A16, A16, None) == 3          # misaligned input
    assert f(A16, 4, 8, 8, A16, A16, P((1 << 20) + 2), None) == 3   # misaligned alpha
    if not torch.cuda.is_available():
        assert f(A16, 4, 8, 8, A16, A16, A16, None) == 6


def test_global_scales_pair_host_checks_without_gpu():
    import torch
    L = fp4.lib()
    f = L.fp4_compute_global_scales_pair
    # (a, rows_a, cols_a, ld_a, b, rows_b, cols_b, ld_b, gs_a, gs_b, alpha, stream)
    assert f(A16, 4, 8, 8, A16, 4, 8, 8, None, A16, A16, None) == 1      # no gs_a_out
    assert f(A16, 4, 8, 8, A16, 4, 8, 8, A16, None, A16, None) == 1      # no gs_b_out
    assert f(A16, 4, 8, 8, None, 4, 8, 8, A16, A16, A16, None) == 1      # no b
    assert f(A16, 4, 8, 8, A16, 4, 8, 4, A16, A16, A16, None) == 1       # ld_b < cols_b
    assert f(A16, 4, 12, 12, A16, 4, 8, 8, A16, A16, A16, None) == 2     # cols_a % 8
    assert f(A16, 4, 8, 8, A1, 4, 8, 8, A16, A16, A16, None) == 3        # misaligned b
    assert f(A16, 4, 8, 8, A16, 4, 8, 8, A16, A16, P((1 << 20) + 2), None) == 3   # misaligned alpha
    if not torch.cuda.is_available():
        assert f(A16, 4, 8, 8, A16, 4, 8, 8, A16, A16, None, None) == 6


def test_decode_dynamic_host_checks_without_gpu():
    import torch
    L = fp4.lib()
    f = L.fp4_gemm_decode_dynamic
    ws = P(1 << 24)
    # (act, lda, W, sW, gsW, M, N, K, D, ldd, gs_out, alpha_out, ws, ws_bytes, stream)
    assert f(A16, 64, A16, A16, None, 4, 16, 64, A16, 16, A16, A16, ws, 1 << 20, None) == 1   # no gsW
    assert f(A16, 64, A16, A16, A16, 17, 16, 64, A16, 16, A16, A16, ws, 1 << 20, None) == 2   # M > 16
    assert f(A16, 96, A16, A16, A16, 4, 16, 96, A16, 16, A16, A16, ws, 1 << 20, None) == 2    # K % 64
    assert f(None, 64, A16, A16, A16, 4, 16, 64, A16, 16, A16, A16, ws, 1 << 20, None) == 1   # no activation
    assert f(A16, 32, A16, A16, A16, 4, 16, 64, A16, 16, A16, A16, ws, 1 << 20, None) == 1    # lda < K
    assert f(A1, 64, A16, A16, A16, 4, 16, 64, A16, 16, A16, A16, ws, 1 << 20, None) == 3     # misaligned
    assert f(A16, 64, A16, A16, A16, 0, 16, 64, A16, 16, A16, A16, ws, 1 << 20, None) == 0    # M == 0: no-op
    if not torch.cuda.is_available():
        assert f(A16, 64, A16, A16, A16, 4, 16, 64, A16, 16, A16, A16, ws, 1 << 20, None) == 6
