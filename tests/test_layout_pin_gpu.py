"""Pin of the oracle's scale-tile layout against NVIDIA's own block-scaled
FP4 GEMM.

The oracle stores block scales in 512-byte tiles of 128 rows x 4 block
columns (byte of row r, block c at (r % 32) * 16 + ((r / 32) % 4) * 4 + c % 4,
column tiles fastest).  The pages only say that scale vectors are streamed
with the 4-bit tiles ("NVFP4 Architecture: Microscaling & 4-Bit LLMs on
Blackwell", "2. Hardware-Managed Tensor Core Dot-Products"); they fix no
layout.  This library's GEMM reads the same bytes through its own mapping, so
a mistake made consistently in the oracle and the kernels would pass every
parity test.  Here the oracle's bytes go, unchanged, to cuBLASLt's
block-scaled GEMM (reached through torch._scaled_mm: NVFP4 as
float4_e2m1fn_x2 operands with float8_e4m3fn scales, MXFP4 as the same codes
widened exactly to float8_e4m3fn with float8_e8m0fnu scales, i.e. MXFP8; both
in the library's 128x4 "blocked" scale layout), and its result must match
the oracle's FP64 GEMM of the same bytes.  Nothing of this repository's CUDA
library is involved: the only parties are the oracle and NVIDIA's library.
"""
import os

import numpy as np
import pytest
import torch

from block_scaled_fp4_05_b200 import synth
from gpu_util import assert_gemm_close, gemm_tolerance

pytestmark = pytest.mark.gpu

NV, MX = 0, 1


def _e2m1_values():
    """Value of each 4-bit code, from the page's code table (golden file);
    negative codes mirror with the sign bit."""
    path = os.path.join(os.path.dirname(__file__), "golden", "e2m1_code_table.txt")
    mag = {}
    with open(path) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            bits, val = line.split()[:2]
            mag[int(bits, 2)] = float(val)
    return np.array([mag[c & 7] * (-1.0 if c & 8 else 1.0) for c in range(16)], dtype=np.float32)


def cublas_block_scaled(fmt, pA, sA, pB, sB):
    """D = A_hat B_hat^T (BF16) by cuBLASLt from packed codes and tiled scales.

    NVFP4: the codes go in as float4_e2m1fn_x2 with float8_e4m3fn scales on
    16-element blocks.  MXFP4: torch reaches cuBLASLt's FP4 operands only with
    E4M3 scales, so the codes are widened to float8_e4m3fn (every E2M1 value
    is exact in E4M3) and the product runs as MXFP8, whose scales are E8M0 on
    32-element blocks in the same tiled layout; the scale bytes go in as they
    are."""
    sdt = torch.float8_e4m3fn if fmt == NV else torch.float8_e8m0fnu
    sa = torch.from_numpy(np.ascontiguousarray(sA)).cuda().view(sdt)
    sb = torch.from_numpy(np.ascontiguousarray(sB)).cuda().view(sdt)
    if fmt == NV:
        a = torch.from_numpy(np.ascontiguousarray(pA)).cuda().view(torch.float4_e2m1fn_x2)
        b = torch.from_numpy(np.ascontiguousarray(pB)).cuda().view(torch.float4_e2m1fn_x2)
    else:
        vals = _e2m1_values()

        def widen(p):
            codes = np.stack([p & 15, p >> 4], axis=-1).reshape(p.shape[0], -1)
            return torch.from_numpy(vals[codes]).cuda().to(torch.float8_e4m3fn)
        a, b = widen(pA), widen(pB)
    D = torch._scaled_mm(a, b.t(), sa, sb, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    return D.float().cpu().numpy().astype(np.float64)


def random_operand(rng, fmt, rows, K):
    """Random E2M1 codes and a random tiled scale buffer (every byte,
    padding rows included, drawn at random), with scales kept in a range
    where no product overflows."""
    k = 16 if fmt == NV else 32
    packed = rng.integers(0, 256, size=(rows, K // 2), dtype=np.uint8)
    nbytes = ((rows + 127) // 128) * ((K // k + 3) // 4) * 512
    if fmt == NV:
        # unsigned E4M3: exponent field 1..13, any mantissa -> 2^-6 .. 2^6 * 1.875
        e = rng.integers(1, 14, size=nbytes)
        m = rng.integers(0, 8, size=nbytes)
        scales = (e * 8 + m).astype(np.uint8)
    else:
        scales = rng.integers(120, 135, size=nbytes).astype(np.uint8)   # 2^-7 .. 2^7
    return packed, scales


def swapped_layout(scales):
    """The same tiles with the two row strides of the within-tile layout
    exchanged: the byte at (r%32)*16 + ((r/32)%4)*4 + c moves to
    ((r/32)%4)*128 + (r%32)*4 + c, a plausible transposition."""
    t = scales.reshape(-1, 32, 4, 4)          # [tile, r % 32, (r / 32) % 4, c]
    return np.ascontiguousarray(t.transpose(0, 2, 1, 3)).reshape(-1)


@pytest.mark.parametrize("fmt", [NV, MX])
@pytest.mark.parametrize("MNK", [(128, 256, 512), (256, 384, 1024), (208, 272, 768)])
def test_random_codes_and_scales_match_cublas(orc, fmt, MNK):
    M, N, K = MNK
    rng = np.random.default_rng(1000 + 7 * fmt + M)
    pA, sA = random_operand(rng, fmt, M, K)
    pB, sB = random_operand(rng, fmt, N, K)
    D_orc, S = orc.gemm(fmt, pA, sA, pB, sB, alpha=1.0)
    D_lib = cublas_block_scaled(fmt, pA, sA, pB, sB)
    assert_gemm_close(D_lib, D_orc, S, "cuBLASLt vs oracle %s fmt %d" % (MNK, fmt))

    # the pin discriminates: the oracle reading the bytes through a
    # transposed within-tile arrangement disagrees with the library
    D_wrong, S_wrong = orc.gemm(fmt, pA, swapped_layout(sA), pB, sB, alpha=1.0)
    bad = np.abs(D_lib - D_wrong) > gemm_tolerance(D_wrong, S_wrong)
    assert bad.mean() > 0.5, "a transposed scale layout would not be detected"


@pytest.mark.parametrize("fmt", [NV, MX])
def test_quantized_tiny_config_matches_cublas(orc, fmt):
    # the 128x512 / 256x512 inputs (outlier channel x50 in A), quantized by
    # the oracle; block scales only (alpha = 1), since the per-tensor factor
    # is outside what the library call multiplies
    A, B = synth.tiny_nv()
    gsA = orc.global_scale(A) if fmt == NV else 1.0
    gsB = orc.global_scale(B) if fmt == NV else 1.0
    pA, sA = orc.quantize(fmt, 0, A, gs=gsA)
    pB, sB = orc.quantize(fmt, 0, B, gs=gsB)
    D_orc, S = orc.gemm(fmt, pA, sA, pB, sB, alpha=1.0)
    D_lib = cublas_block_scaled(fmt, pA, sA, pB, sB)
    assert_gemm_close(D_lib, D_orc, S, "tiny config fmt %d" % fmt)


@pytest.mark.parametrize("fmt", [NV, MX])
def test_quantized_ragged_outliers_match_cublas(orc, fmt):
    # rows that straddle scale tiles (M = 304: three row tiles, the last one
    # partial) and outlier channels, so that the scales differ per row and
    # per block (the library wants N a multiple of 16)
    M, N, K = 304, 528, 1024
    A = synth.normal_bf16(M, K, seed=41, outlier_factor=50.0)
    B = synth.normal_bf16(N, K, seed=41, tensor_id=1, sigma=0.02)
    gsA = orc.global_scale(A) if fmt == NV else 1.0
    gsB = orc.global_scale(B) if fmt == NV else 1.0
    pA, sA = orc.quantize(fmt, 0, A, gs=gsA)
    pB, sB = orc.quantize(fmt, 0, B, gs=gsB)
    D_orc, S = orc.gemm(fmt, pA, sA, pB, sB, alpha=1.0)
    D_lib = cublas_block_scaled(fmt, pA, sA, pB, sB)
    assert_gemm_close(D_lib, D_orc, S, "ragged fmt %d" % fmt)
