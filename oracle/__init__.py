"""CPU oracle for microscaling FP4 quantization and the block-scaled GEMM.

TEST INFRASTRUCTURE ONLY: the test suite, the entry module's smoke check and
the benchmark's CPU-baseline leg are the only callers.  The product path
(the CUDA library and its binding) never imports this package; the two share
no code.  The arithmetic lives in ``oracle.c`` (plain C, one IEEE rounding per
operation); this module only marshals numpy arrays through ctypes.

Formats: ``NVFP4`` (16-element blocks, unsigned E4M3 block scale under an FP32
per-tensor scale), ``MXFP4`` (32-element blocks, E8M0 scale) and ``P1E8``
(16-element blocks with E8M0 scales under a per-tensor scale, the dual-level
formula exactly as "NVFP4 Architecture: Microscaling & 4-Bit LLMs on
Blackwell", "1. The Dual-Level Mathematical Formulation" prints it).
"""
import ctypes
import os

import numpy as np

from . import build as _build

NVFP4, MXFP4, P1E8 = 0, 1, 2
ROWWISE, COLWISE = 0, 1

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        c = ctypes
        P = c.c_void_p
        i64 = c.c_int64
        L.orc_e2m1_decode.restype = c.c_double
        L.orc_e2m1_decode.argtypes = [c.c_uint8]
        L.orc_e2m1_encode.restype = c.c_uint8
        L.orc_e2m1_encode.argtypes = [c.c_float]
        L.orc_e2m1_encode_first_index_tie.restype = c.c_uint8
        L.orc_e2m1_encode_first_index_tie.argtypes = [c.c_float]
        L.orc_e8m0_decode.restype = c.c_double
        L.orc_e8m0_decode.argtypes = [c.c_uint8]
        L.orc_mx_exponent.restype = c.c_int
        L.orc_mx_exponent.argtypes = [c.c_float]
        L.orc_e8m0_encode_block.restype = c.c_uint8
        L.orc_e8m0_encode_block.argtypes = [c.c_float]
        L.orc_e4m3_decode.restype = c.c_double
        L.orc_e4m3_decode.argtypes = [c.c_uint8]
        L.orc_e4m3_encode_unsigned.restype = c.c_uint8
        L.orc_e4m3_encode_unsigned.argtypes = [c.c_float]
        L.orc_amax_bf16.restype = c.c_float
        L.orc_amax_bf16.argtypes = [P, i64]
        L.orc_global_scale_from_amax.restype = c.c_float
        L.orc_global_scale_from_amax.argtypes = [c.c_float]
        L.orc_global_scale.restype = c.c_float
        L.orc_global_scale.argtypes = [P, i64, i64, i64]
        L.orc_block_size.restype = c.c_int
        L.orc_block_size.argtypes = [c.c_int]
        L.orc_scale_offset.restype = i64
        L.orc_scale_offset.argtypes = [i64, i64, i64]
        L.orc_scale_bytes.restype = i64
        L.orc_scale_bytes.argtypes = [i64, i64]
        L.orc_quantize.restype = c.c_int
        L.orc_quantize.argtypes = [c.c_int, c.c_int, P, i64, i64, i64, c.c_float, P, P, P]
        L.orc_dequantize.restype = None
        L.orc_dequantize.argtypes = [c.c_int, P, P, i64, i64, c.c_double, P]
        L.orc_gemm_pairs.restype = None
        L.orc_gemm_pairs.argtypes = [c.c_int, P, P, P, P, i64, c.c_double, P, P, i64, P, P]
        L.orc_gemm.restype = None
        L.orc_gemm.argtypes = [c.c_int, P, P, P, P, i64, i64, i64, c.c_double, P, P, P, P]
        L.orc_naive_per_tensor.restype = None
        L.orc_naive_per_tensor.argtypes = [P, i64, P]
        L.orc_block_pow2_roundtrip.restype = None
        L.orc_block_pow2_roundtrip.argtypes = [P, i64, c.c_int, c.c_int, P]
        for name in ("orc_e2m1_encode_n", "orc_e4m3_encode_unsigned_n", "orc_mx_exponent_n"):
            getattr(L, name).restype = None
            getattr(L, name).argtypes = [P, i64, P]
        L.orc_num_threads.restype = c.c_int
        L.orc_num_threads.argtypes = []
        _lib = L
    return _lib


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _bits(x):
    """bf16 input as a C-contiguous uint16 array of bit patterns."""
    x = np.asarray(x)
    if x.dtype != np.uint16:
        raise TypeError("oracle inputs are bf16 bit patterns (uint16)")
    return np.ascontiguousarray(x)


def block_size(fmt):
    return lib().orc_block_size(fmt)


def e2m1_decode(nib):
    return lib().orc_e2m1_decode(int(nib))


def e2m1_encode(v):
    return lib().orc_e2m1_encode(float(v))


def e2m1_encode_first_index_tie(v):
    return lib().orc_e2m1_encode_first_index_tie(float(v))


def e8m0_decode(b):
    return lib().orc_e8m0_decode(int(b))


def mx_exponent(amax):
    return lib().orc_mx_exponent(float(amax))


def e8m0_encode_block(amax):
    return lib().orc_e8m0_encode_block(float(amax))


def e4m3_decode(b):
    return lib().orc_e4m3_decode(int(b))


def e4m3_encode_unsigned(t):
    return lib().orc_e4m3_encode_unsigned(float(t))


def scale_offset(row, col, n_scale_cols):
    return lib().orc_scale_offset(int(row), int(col), int(n_scale_cols))


def scale_bytes(rows, n_scale_cols):
    return lib().orc_scale_bytes(int(rows), int(n_scale_cols))


def global_scale_from_amax(amax):
    return lib().orc_global_scale_from_amax(float(amax))


def global_scale(x_bits):
    """S_global = amax / 2688 in FP32 (1.0 for an all-zero tensor)."""
    x = _bits(x_bits)
    if x.ndim == 1:
        x = x.reshape(1, -1)
    return lib().orc_global_scale(_ptr(x), x.shape[0], x.shape[1], x.shape[1])


def quantize(fmt, axis, x_bits, gs=1.0, with_rowmajor_scales=False):
    """Quantize a bf16 matrix (uint16 bits, [rows x cols]).

    Returns (packed [out_rows x K/2] uint8, scales tiled uint8 1-D,
    optional row-major scales [out_rows x K/k]).
    """
    x = _bits(x_bits)
    rows, cols = x.shape
    k = block_size(fmt)
    out_rows, K = (rows, cols) if axis == ROWWISE else (cols, rows)
    packed = np.zeros((out_rows, K // 2), dtype=np.uint8)
    scales = np.zeros(scale_bytes(out_rows, K // k), dtype=np.uint8)
    rm = np.zeros((out_rows, K // k), dtype=np.uint8) if with_rowmajor_scales else None
    rc = lib().orc_quantize(fmt, axis, _ptr(x), rows, cols, cols, float(gs),
                            _ptr(packed), _ptr(scales),
                            _ptr(rm) if rm is not None else None)
    if rc != 0:
        raise ValueError("oracle quantize: blocked length must be a multiple of the block size")
    if with_rowmajor_scales:
        return packed, scales, rm
    return packed, scales


def dequantize(fmt, packed, scales, gs=0.0):
    """x_hat = q * S_block (* S_global if gs != 0), FP64 [rows x K]."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, kh = packed.shape
    out = np.zeros((rows, 2 * kh), dtype=np.float64)
    lib().orc_dequantize(fmt, _ptr(packed), _ptr(scales), rows, 2 * kh, float(gs), _ptr(out))
    return out


def gemm(fmt, A, sA, B, sB, alpha=1.0):
    """Full D = alpha * A_hat @ B_hat^T and S = |alpha| * |A_hat| @ |B_hat|^T (FP64)."""
    A = np.ascontiguousarray(A, dtype=np.uint8)
    B = np.ascontiguousarray(B, dtype=np.uint8)
    sA = np.ascontiguousarray(sA, dtype=np.uint8)
    sB = np.ascontiguousarray(sB, dtype=np.uint8)
    M, N, K = A.shape[0], B.shape[0], 2 * A.shape[1]
    assert B.shape[1] * 2 == K
    Adq = np.zeros((M, K)); Bdq = np.zeros((N, K))
    D = np.zeros((M, N)); S = np.zeros((M, N))
    lib().orc_gemm(fmt, _ptr(A), _ptr(sA), _ptr(B), _ptr(sB), M, N, K, float(alpha),
                   _ptr(Adq), _ptr(Bdq), _ptr(D), _ptr(S))
    return D, S


def gemm_pairs(fmt, A, sA, B, sB, ms, ns, alpha=1.0):
    """D and S at the listed (m, n) pairs only."""
    A = np.ascontiguousarray(A, dtype=np.uint8)
    B = np.ascontiguousarray(B, dtype=np.uint8)
    sA = np.ascontiguousarray(sA, dtype=np.uint8)
    sB = np.ascontiguousarray(sB, dtype=np.uint8)
    ms = np.ascontiguousarray(ms, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    K = 2 * A.shape[1]
    D = np.zeros(len(ms)); S = np.zeros(len(ms))
    lib().orc_gemm_pairs(fmt, _ptr(A), _ptr(sA), _ptr(B), _ptr(sB), K, float(alpha),
                         _ptr(ms), _ptr(ns), len(ms), _ptr(D), _ptr(S))
    return D, S


def naive_per_tensor(x):
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.zeros(x.size)
    lib().orc_naive_per_tensor(_ptr(x), x.size, _ptr(out))
    return out


def block_pow2_roundtrip(x, k, page_tie=False):
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.zeros(x.size)
    lib().orc_block_pow2_roundtrip(_ptr(x), x.size, int(k), int(bool(page_tie)), _ptr(out))
    return out


def e2m1_encode_array(v):
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.zeros(v.shape, dtype=np.uint8)
    lib().orc_e2m1_encode_n(_ptr(v), v.size, _ptr(out))
    return out


def e4m3_encode_unsigned_array(t):
    t = np.ascontiguousarray(t, dtype=np.float32)
    out = np.zeros(t.shape, dtype=np.uint8)
    lib().orc_e4m3_encode_unsigned_n(_ptr(t), t.size, _ptr(out))
    return out


def mx_exponent_array(a):
    a = np.ascontiguousarray(a, dtype=np.float32)
    out = np.zeros(a.shape, dtype=np.int32)
    lib().orc_mx_exponent_n(_ptr(a), a.size, _ptr(out))
    return out


def num_threads():
    return lib().orc_num_threads()
