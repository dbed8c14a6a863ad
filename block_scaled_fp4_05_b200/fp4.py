"""Python binding of libfp4 (include/fp4.h): argument marshalling only.

Every function here passes device pointers of torch CUDA tensors and the
current torch stream to the C ABI; all arithmetic runs in the library's CUDA
kernels.  There is no fallback: if ``libfp4.so`` is missing or a call fails,
an exception is raised.
"""
import ctypes
import os
import re

import torch

NVFP4, MXFP4, P1E8 = 0, 1, 2   # P1E8: 16-element blocks, E8M0 scale under S_global (quantizer only)
ROWWISE, COLWISE = 0, 1
GEMM_AUTO, GEMM_PREFILL, GEMM_DECODE = 0, 1, 2
GEMM_B_STATIC = 0x100   # flag: B / sB not written by a kernel still running on the stream

FP4_OK = 0
STATUS_NAMES = {
    0: "FP4_OK", 1: "FP4_ERR_INVALID_ARG", 2: "FP4_ERR_UNSUPPORTED_SHAPE",
    3: "FP4_ERR_MISALIGNED", 4: "FP4_ERR_CUDA", 5: "FP4_ERR_TIMEOUT", 6: "FP4_ERR_NO_DEVICE",
    7: "FP4_ERR_WORKSPACE",
}

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfp4.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "fp4.h")


class Fp4Error(RuntimeError):
    def __init__(self, status, what=""):
        self.status = status
        super().__init__("%s%s" % (STATUS_NAMES.get(status, "status %d" % status),
                                   (": " + what) if what else ""))


_lib = None


def lib():
    """Load libfp4.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libfp4.so is missing; build it with "
                               "`python -m block_scaled_fp4_05_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        c = ctypes
        P, i64, sz, st = c.c_void_p, c.c_int64, c.c_size_t, c.c_void_p
        L.fp4_abi_version.restype = c.c_int
        L.fp4_abi_version.argtypes = []
        L.fp4_status_string.restype = c.c_char_p
        L.fp4_status_string.argtypes = [c.c_int]
        L.fp4_last_error.restype = c.c_char_p
        L.fp4_last_error.argtypes = []
        L.fp4_packed_bytes.restype = sz
        L.fp4_packed_bytes.argtypes = [i64, i64]
        L.fp4_scale_bytes.restype = sz
        L.fp4_scale_bytes.argtypes = [c.c_int, i64, i64]
        L.fp4_compute_global_scale.restype = c.c_int
        L.fp4_compute_global_scale.argtypes = [P, i64, i64, i64, P, st]
        L.fp4_compute_global_scale_alpha.restype = c.c_int
        L.fp4_compute_global_scale_alpha.argtypes = [P, i64, i64, i64, P, P, P, st]
        L.fp4_compute_global_scales_pair.restype = c.c_int
        L.fp4_compute_global_scales_pair.argtypes = [P, i64, i64, i64, P, i64, i64, i64, P, P, P, st]
        L.fp4_quantize.restype = c.c_int
        L.fp4_quantize.argtypes = [c.c_int, c.c_int, P, i64, i64, i64, P, P, P, st]
        L.fp4_gemm_grouped.restype = c.c_int
        L.fp4_gemm_grouped.argtypes = [c.c_int, c.c_int, P, st]
        L.fp4_dequantize.restype = c.c_int
        L.fp4_dequantize.argtypes = [c.c_int, P, P, P, i64, i64, P, i64, st]
        L.fp4_quantize_batch.restype = c.c_int
        L.fp4_quantize_batch.argtypes = [c.c_int, c.c_int, P, st]
        L.fp4_quantize_dynamic.restype = c.c_int
        L.fp4_quantize_dynamic.argtypes = [c.c_int, P, i64, i64, i64, P, P, P, P, P, st]
        L.fp4_alpha_from_global_scales.restype = c.c_int
        L.fp4_alpha_from_global_scales.argtypes = [P, P, P, st]
        L.fp4_gemm.restype = c.c_int
        L.fp4_gemm.argtypes = [c.c_int, P, P, P, P, i64, i64, i64, P, P, i64, P, sz, st]
        L.fp4_gemm_with_kernel.restype = c.c_int
        L.fp4_gemm_with_kernel.argtypes = [c.c_int, P, P, P, P, i64, i64, i64, P, P, i64, P, sz,
                                           c.c_int, st]
        L.fp4_gemm_workspace_bytes.restype = sz
        L.fp4_gemm_workspace_bytes.argtypes = [c.c_int, i64, i64, i64]
        L.fp4_get_device_status.restype = c.c_int
        L.fp4_get_device_status.argtypes = [st]
        L.fp4_selftest_bounded_wait.restype = c.c_int
        L.fp4_selftest_bounded_wait.argtypes = [st]
        L.fp4_gemm_decode_dynamic.restype = c.c_int
        L.fp4_gemm_decode_dynamic.argtypes = [P, i64, P, P, P, i64, i64, i64, P, i64, P, P, P, sz, st]
        L.fp4_gemm_decode_noalloc.restype = c.c_int
        L.fp4_gemm_decode_noalloc.argtypes = [c.c_int, P, P, P, P, i64, i64, i64, P, P, i64, st]
        _lib = L
    return _lib


def declared_symbols():
    """Names of the functions declared in include/fp4.h."""
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:[A-Za-z_][\w\s\*]*?)\b(fp4_\w+)\s*\(", text, re.M)))


def _check(status, what=""):
    if status != FP4_OK:
        detail = lib().fp4_last_error().decode()
        raise Fp4Error(status, what + (" (%s)" % detail if detail else ""))


def _stream(stream=None):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _dptr(t, what):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("%s must be a CUDA tensor" % what)
    return ctypes.c_void_p(t.data_ptr())


def _ld(t):
    if t.dim() == 2 and t.numel() == 0:
        return t.shape[1]            # an empty matrix: any stride torch reports
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("expected a 2-D tensor with unit column stride")
    return t.stride(0)


def block_size(fmt):
    return 32 if fmt == MXFP4 else 16


def fp4_status_string(status):
    return lib().fp4_status_string(int(status)).decode()


def fp4_packed_bytes(rows, k):
    return lib().fp4_packed_bytes(int(rows), int(k))


def fp4_scale_bytes(fmt, rows, k):
    return lib().fp4_scale_bytes(int(fmt), int(rows), int(k))


def fp4_compute_global_scale(x, gs_out, stream=None):
    """S_global of bf16 matrix x into gs_out (float32 CUDA tensor, 1 element)."""
    assert x.dtype == torch.bfloat16 and gs_out.dtype == torch.float32
    _check(lib().fp4_compute_global_scale(_dptr(x, "x"), x.shape[0], x.shape[1], _ld(x),
                                          _dptr(gs_out, "gs_out"), _stream(stream)),
           "fp4_compute_global_scale")


def fp4_compute_global_scale_alpha(x, gs_out, other_gs, alpha_out, stream=None):
    """S_global of x into gs_out and alpha = S_global * other_gs into alpha_out
    (float32 CUDA tensors of 1 element), one launch."""
    assert x.dtype == torch.bfloat16 and gs_out.dtype == torch.float32
    _check(lib().fp4_compute_global_scale_alpha(_dptr(x, "x"), x.shape[0], x.shape[1], _ld(x),
                                                _dptr(gs_out, "gs_out"), _dptr(other_gs, "other_gs"),
                                                _dptr(alpha_out, "alpha_out"), _stream(stream)),
           "fp4_compute_global_scale_alpha")


def fp4_compute_global_scales_pair(a, b, gs_a_out, gs_b_out, alpha_out=None, stream=None):
    """S_global of a and of b and (if alpha_out) alpha = gs_a * gs_b, one launch."""
    assert a.dtype == torch.bfloat16 and b.dtype == torch.bfloat16
    _check(lib().fp4_compute_global_scales_pair(_dptr(a, "a"), a.shape[0], a.shape[1], _ld(a),
                                                _dptr(b, "b"), b.shape[0], b.shape[1], _ld(b),
                                                _dptr(gs_a_out, "gs_a_out"), _dptr(gs_b_out, "gs_b_out"),
                                                _dptr(alpha_out, "alpha_out"), _stream(stream)),
           "fp4_compute_global_scales_pair")


def fp4_quantize(fmt, axis, x, packed_out, scales_out, global_scale=None, stream=None):
    assert x.dtype == torch.bfloat16
    _check(lib().fp4_quantize(int(fmt), int(axis), _dptr(x, "x"), x.shape[0], x.shape[1], _ld(x),
                              _dptr(packed_out, "packed_out"), _dptr(scales_out, "scales_out"),
                              _dptr(global_scale, "global_scale"), _stream(stream)),
           "fp4_quantize")


class GemmProblem(ctypes.Structure):
    """fp4_gemm_problem of include/fp4.h."""
    _fields_ = [("A", ctypes.c_void_p), ("sA", ctypes.c_void_p), ("B", ctypes.c_void_p),
                ("sB", ctypes.c_void_p), ("M", ctypes.c_int64), ("N", ctypes.c_int64),
                ("K", ctypes.c_int64), ("alpha", ctypes.c_void_p), ("D", ctypes.c_void_p),
                ("ldd", ctypes.c_int64)]


def _gemm_problems(items):
    arr = (GemmProblem * max(1, len(items)))()
    for i, (A, sA, B, sB, K, alpha, D) in enumerate(items):
        arr[i] = GemmProblem(_dptr(A, "A"), _dptr(sA, "sA"), _dptr(B, "B"), _dptr(sB, "sB"),
                             D.shape[0], D.shape[1], int(K), _dptr(alpha, "alpha"), _dptr(D, "D"),
                             D.stride(0))
    return arr


def fp4_gemm_grouped(fmt, items, stream=None):
    """Grouped GEMM; items are (A, sA, B, sB, K, alpha or None, D) tuples with
    D [M x N] bf16 (M, N taken from D)."""
    arr = _gemm_problems(items)
    _check(lib().fp4_gemm_grouped(int(fmt), len(items), ctypes.cast(arr, ctypes.c_void_p), _stream(stream)),
           "fp4_gemm_grouped")


def bind_gemm_grouped(fmt, items, stream=None):
    arr = _gemm_problems(items)
    call = BoundCall("fp4_gemm_grouped", int(fmt), len(items), ctypes.cast(arr, ctypes.c_void_p),
                     _stream(stream))
    call.keep = arr
    return call


def fp4_dequantize(fmt, packed, scales, global_scale, out, stream=None):
    """out[rows x k] (bf16) = q * S_block (* S_global), rounded once to BF16."""
    rows, k = out.shape[0], packed.shape[1] * 2
    _check(lib().fp4_dequantize(int(fmt), _dptr(packed, "packed"), _dptr(scales, "scales"),
                                _dptr(global_scale, "global_scale"), rows, k, _dptr(out, "out"),
                                out.stride(0), _stream(stream)), "fp4_dequantize")
    return out


class QuantizeDesc(ctypes.Structure):
    """fp4_quantize_desc of include/fp4.h."""
    _fields_ = [("in_bf16", ctypes.c_void_p), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("ld", ctypes.c_int64), ("packed_out", ctypes.c_void_p), ("scales_out", ctypes.c_void_p),
                ("global_scale", ctypes.c_void_p)]


def _quantize_descs(items):
    arr = (QuantizeDesc * max(1, len(items)))()
    for i, (x, packed_out, scales_out, gs) in enumerate(items):
        assert x.dtype == torch.bfloat16
        arr[i] = QuantizeDesc(_dptr(x, "x"), x.shape[0], x.shape[1], _ld(x),
                              _dptr(packed_out, "packed_out"), _dptr(scales_out, "scales_out"),
                              _dptr(gs, "global_scale"))
    return arr


def fp4_quantize_batch(fmt, items, stream=None):
    """Rowwise quantization of several tensors in one launch; items are
    (x, packed_out, scales_out, global_scale or None) tuples."""
    arr = _quantize_descs(items)
    _check(lib().fp4_quantize_batch(int(fmt), len(items), ctypes.cast(arr, ctypes.c_void_p),
                                    _stream(stream)), "fp4_quantize_batch")


def bind_quantize_batch(fmt, items, stream=None):
    arr = _quantize_descs(items)
    call = BoundCall("fp4_quantize_batch", int(fmt), len(items), ctypes.cast(arr, ctypes.c_void_p),
                     _stream(stream))
    call.keep = arr   # the descriptor array must outlive the bound call
    return call


def fp4_quantize_dynamic(x, packed_out, scales_out, gs_out, other_gs=None, alpha_out=None,
                         stream=None):
    """NVFP4: S_global of x, rowwise quantization with it and optionally
    alpha = S_global * other_gs, in one launch."""
    assert x.dtype == torch.bfloat16
    _check(lib().fp4_quantize_dynamic(NVFP4, _dptr(x, "x"), x.shape[0], x.shape[1], _ld(x),
                                      _dptr(packed_out, "packed_out"), _dptr(scales_out, "scales_out"),
                                      _dptr(gs_out, "gs_out"), _dptr(other_gs, "other_gs"),
                                      _dptr(alpha_out, "alpha_out"), _stream(stream)),
           "fp4_quantize_dynamic")


def bind_quantize_dynamic(x, packed_out, scales_out, gs_out, other_gs=None, alpha_out=None,
                          stream=None):
    return BoundCall("fp4_quantize_dynamic", NVFP4, _dptr(x, "x"), x.shape[0], x.shape[1], _ld(x),
                     _dptr(packed_out, "packed_out"), _dptr(scales_out, "scales_out"),
                     _dptr(gs_out, "gs_out"), _dptr(other_gs, "other_gs"),
                     _dptr(alpha_out, "alpha_out"), _stream(stream))


def fp4_alpha_from_global_scales(gsA, gsB, alpha_out, stream=None):
    _check(lib().fp4_alpha_from_global_scales(_dptr(gsA, "gsA"), _dptr(gsB, "gsB"),
                                              _dptr(alpha_out, "alpha_out"), _stream(stream)),
           "fp4_alpha_from_global_scales")


def fp4_gemm_workspace_bytes(fmt, M, N, K):
    return lib().fp4_gemm_workspace_bytes(int(fmt), int(M), int(N), int(K))


def fp4_gemm(fmt, A, sA, B, sB, M, N, K, alpha, D, workspace=None, kernel=GEMM_AUTO, stream=None):
    """D[M x N] (bf16, row stride D.stride(0)) = alpha * A_hat @ B_hat^T."""
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().fp4_gemm_with_kernel(int(fmt), _dptr(A, "A"), _dptr(sA, "sA"), _dptr(B, "B"),
                                      _dptr(sB, "sB"), int(M), int(N), int(K),
                                      _dptr(alpha, "alpha"), _dptr(D, "D"), D.stride(0),
                                      _dptr(workspace, "workspace"), ws_bytes, int(kernel),
                                      _stream(stream)),
           "fp4_gemm")


def fp4_gemm_decode_dynamic(x, W, sW, gsW, D, gs_out, alpha_out, workspace, stream=None):
    """NVFP4 decode GEMM quantizing the BF16 activation x [M x K] inside the
    kernel: gs_out = S_global(x), alpha_out = gs_out * gsW, D = alpha * x_hat W_hat^T."""
    assert x.dtype == torch.bfloat16
    M, K = x.shape
    N = W.shape[0]
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().fp4_gemm_decode_dynamic(_dptr(x, "x"), _ld(x), _dptr(W, "W"), _dptr(sW, "sW"),
                                         _dptr(gsW, "gsW"), M, N, K, _dptr(D, "D"), D.stride(0),
                                         _dptr(gs_out, "gs_out"), _dptr(alpha_out, "alpha_out"),
                                         _dptr(workspace, "workspace"), ws_bytes, _stream(stream)),
           "fp4_gemm_decode_dynamic")


def bind_gemm_decode_dynamic(x, W, sW, gsW, D, gs_out, alpha_out, workspace, stream=None):
    M, K = x.shape
    return BoundCall("fp4_gemm_decode_dynamic", _dptr(x, "x"), _ld(x), _dptr(W, "W"), _dptr(sW, "sW"),
                     _dptr(gsW, "gsW"), M, W.shape[0], K, _dptr(D, "D"), D.stride(0),
                     _dptr(gs_out, "gs_out"), _dptr(alpha_out, "alpha_out"), _dptr(workspace, "workspace"),
                     workspace.numel() * workspace.element_size(), _stream(stream))


def fp4_get_device_status(stream=None):
    return lib().fp4_get_device_status(_stream(stream))


def fp4_selftest_bounded_wait(stream=None):
    _check(lib().fp4_selftest_bounded_wait(_stream(stream)), "fp4_selftest_bounded_wait")


# ---------------------------------------------------------------------------
# Allocating conveniences (torch provides the memory; the library computes)
# ---------------------------------------------------------------------------
def quantize(x, fmt, axis=ROWWISE, global_scale=None, stream=None):
    """Quantize bf16 CUDA matrix x; returns (packed uint8 [R x K/2], scales uint8)."""
    rows, cols = x.shape
    out_rows, K = (rows, cols) if axis == ROWWISE else (cols, rows)
    packed = torch.empty((out_rows, K // 2), dtype=torch.uint8, device=x.device)
    scales = torch.empty((fp4_scale_bytes(fmt, out_rows, K),), dtype=torch.uint8, device=x.device)
    fp4_quantize(fmt, axis, x, packed, scales, global_scale, stream)
    return packed, scales


def global_scale(x, stream=None):
    gs = torch.empty((1,), dtype=torch.float32, device=x.device)
    fp4_compute_global_scale(x, gs, stream)
    return gs


def gemm(fmt, A, sA, B, sB, K, alpha=None, kernel=GEMM_AUTO, out=None, workspace=None, stream=None):
    """D = alpha * A_hat @ B_hat^T for packed operands; allocates D (and the
    decode workspace when it applies) unless given."""
    M, N = A.shape[0], B.shape[0]
    D = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    if workspace is None and kernel != GEMM_PREFILL:
        nb = fp4_gemm_workspace_bytes(fmt, M, N, K)
        if nb:
            workspace = torch.zeros((nb,), dtype=torch.uint8, device=A.device)
    fp4_gemm(fmt, A, sA, B, sB, M, N, K, alpha, D, workspace, kernel, stream)
    return D


# ---------------------------------------------------------------------------
# Pre-marshalled calls: the ctypes arguments are built once, each call then
# costs one foreign call (used where launch overhead matters, e.g. decode).
# ---------------------------------------------------------------------------
class BoundCall:
    def __init__(self, name, *cargs):
        self._f = getattr(lib(), name)
        self._args = cargs
        self.name = name

    def __call__(self):
        st = self._f(*self._args)
        if st != FP4_OK:
            _check(st, self.name)

    def on_stream(self, stream):
        """The same call issued on another stream (the stream is the last
        argument of every bound entry point)."""
        c = BoundCall(self.name, *self._args[:-1], _stream(stream))
        if hasattr(self, "keep"):
            c.keep = self.keep
        return c


def bind_global_scale(x, gs_out, stream=None):
    return BoundCall("fp4_compute_global_scale", _dptr(x, "x"), x.shape[0], x.shape[1], _ld(x),
                     _dptr(gs_out, "gs_out"), _stream(stream))


def bind_global_scale_alpha(x, gs_out, other_gs, alpha_out, stream=None):
    return BoundCall("fp4_compute_global_scale_alpha", _dptr(x, "x"), x.shape[0], x.shape[1], _ld(x),
                     _dptr(gs_out, "gs_out"), _dptr(other_gs, "other_gs"), _dptr(alpha_out, "alpha_out"),
                     _stream(stream))


def bind_global_scales_pair(a, b, gs_a_out, gs_b_out, alpha_out=None, stream=None):
    return BoundCall("fp4_compute_global_scales_pair", _dptr(a, "a"), a.shape[0], a.shape[1], _ld(a),
                     _dptr(b, "b"), b.shape[0], b.shape[1], _ld(b), _dptr(gs_a_out, "gs_a_out"),
                     _dptr(gs_b_out, "gs_b_out"), _dptr(alpha_out, "alpha_out"), _stream(stream))


def bind_quantize(fmt, axis, x, packed_out, scales_out, global_scale=None, stream=None):
    return BoundCall("fp4_quantize", int(fmt), int(axis), _dptr(x, "x"), x.shape[0], x.shape[1],
                     _ld(x), _dptr(packed_out, "packed_out"), _dptr(scales_out, "scales_out"),
                     _dptr(global_scale, "global_scale"), _stream(stream))


def bind_alpha(gsA, gsB, alpha_out, stream=None):
    return BoundCall("fp4_alpha_from_global_scales", _dptr(gsA, "gsA"), _dptr(gsB, "gsB"),
                     _dptr(alpha_out, "alpha_out"), _stream(stream))


def bind_gemm(fmt, A, sA, B, sB, M, N, K, alpha, D, workspace=None, kernel=GEMM_AUTO, stream=None):
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return BoundCall("fp4_gemm_with_kernel", int(fmt), _dptr(A, "A"), _dptr(sA, "sA"),
                     _dptr(B, "B"), _dptr(sB, "sB"), int(M), int(N), int(K),
                     _dptr(alpha, "alpha"), _dptr(D, "D"), D.stride(0),
                     _dptr(workspace, "workspace"), ws_bytes, int(kernel), _stream(stream))
