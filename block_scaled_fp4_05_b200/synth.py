"""Seeded synthetic BF16 inputs shaped like 70B-class projection layers.

This module is shared by the tests, the benchmark and the smoke check; it
holds no quantization or GEMM arithmetic, only random-number generation.

Recipe (one call = one tensor):
  * values: Philox-4x32-10 counter-based generator (numpy's implementation,
    keyed by (seed, tensor id)), standard normal FP32 samples times ``sigma``;
  * outlier channels: ``max(1, round(frac * cols))`` distinct columns drawn
    without replacement from a second Philox stream; each whole column is
    multiplied by ``factor`` in FP32 (the pages describe <0.1% of hidden
    channels spiking to 20-100x the rest);
  * exact zeros: each element set to +0.0 with probability ``zero_frac``
    (third Philox stream);
  * FP32 -> BF16 with round-to-nearest-even (torch CPU conversion).
Returned as a ``uint16`` numpy array of BF16 bit patterns, shape [rows, cols].
"""
import numpy as np
import torch


def _gen(seed, tensor_id, stream):
    return np.random.Generator(np.random.Philox(key=[int(seed), int(tensor_id) * 4 + int(stream)]))


def outlier_columns(cols, frac, seed, tensor_id):
    n = max(1, int(round(frac * cols)))
    return np.sort(_gen(seed, tensor_id, 1).choice(cols, size=n, replace=False))


def normal_bf16(rows, cols, seed, tensor_id=0, sigma=1.0, outlier_factor=None,
                outlier_frac=0.001, zero_frac=0.0):
    x = _gen(seed, tensor_id, 0).standard_normal((rows, cols), dtype=np.float32)
    if sigma != 1.0:
        x *= np.float32(sigma)
    if outlier_factor is not None:
        idx = outlier_columns(cols, outlier_frac, seed, tensor_id)
        x[:, idx] *= np.float32(outlier_factor)
    if zero_frac > 0.0:
        mask = _gen(seed, tensor_id, 2).random((rows, cols), dtype=np.float32) < zero_frac
        x[mask] = 0.0
    return f32_to_bf16_bits(x)


def f32_to_bf16_bits(x):
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b):
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def bits_to_torch(b):
    """uint16 bit array -> torch.bfloat16 CPU tensor (no copy of values)."""
    return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16)


# --------------------------------------------------------------------------
# The workloads (sizes, distributions and seeds of the five configurations).
# --------------------------------------------------------------------------
def tiny_nv():
    """NVFP4 quantize+GEMM tiny case: A 128x512, B 256x512, N(0,1), seed 0,
    0.1% of A's K columns scaled x50."""
    A = normal_bf16(128, 512, seed=0, tensor_id=0, outlier_factor=50.0)
    B = normal_bf16(256, 512, seed=0, tensor_id=1)
    return A, B


def square(n=4096):
    """Square case M=N=K=4096, N(0,1), seed 1, 0.1% outlier channels x50 in A."""
    A = normal_bf16(n, n, seed=1, tensor_id=0, outlier_factor=50.0)
    B = normal_bf16(n, n, seed=1, tensor_id=1)
    return A, B


def decode_weight(N=28672, K=8192):
    """Decode weight W [N x K], N(0, 0.02), seed 2."""
    return normal_bf16(N, K, seed=2, tensor_id=0, sigma=0.02)


def decode_activation(M, K=8192):
    """Decode activations [M x K], N(0,1), 0.1% outlier channels x100, seed 2."""
    return normal_bf16(M, K, seed=2, tensor_id=100 + M, outlier_factor=100.0)


def prefill(M=8192, N=28672, K=8192):
    """Prefill: A [M x K] N(0,1) with 0.1% outlier channels x50, W [N x K]
    N(0, 0.02), seed 3 (up-projection 8192x28672x8192; down-projection
    8192x8192x28672)."""
    A = normal_bf16(M, K, seed=3, tensor_id=0 if K == 8192 else 2, outlier_factor=50.0)
    W = normal_bf16(N, K, seed=3, tensor_id=1 if K == 8192 else 3, sigma=0.02)
    return A, W


def quant_sweep(rows, cols):
    """Quantizer sweep tensor: N(0,1), 0.1% outlier channels x100, 1% exact
    zeros, seed 4 (16384x16384 and 8192x28672)."""
    return normal_bf16(rows, cols, seed=4, tensor_id=rows * 7 + cols,
                       outlier_factor=100.0, zero_frac=0.01)
