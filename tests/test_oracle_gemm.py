"""Pins of the oracle's block-scaled GEMM (no GPU): closed forms, one-hot
selection, exact alpha scaling, every single-block code pair, and an
independent FP64 matmul of operands decoded here from the page's code table.
"""
import itertools

import numpy as np
import pytest

from block_scaled_fp4_05_b200 import synth
from test_oracle_formats import load_code_table

E2M1 = {}
for _c, _v in load_code_table():
    E2M1[_c] = _v
    E2M1[_c | 8] = -_v
E2M1_LUT = np.array([E2M1[c] for c in range(16)])

E4M3_ONE, E8M0_ONE = 0x38, 127


def pack_codes(codes):
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)


def tile_scales(orc, rm):
    rows, nsc = rm.shape
    out = np.zeros(orc.scale_bytes(rows, nsc), dtype=np.uint8)
    for r in range(rows):
        for c in range(nsc):
            out[orc.scale_offset(r, c, nsc)] = rm[r, c]
    return out


def scale_value(fmt, b):
    b = np.asarray(b, dtype=np.int64)
    if fmt == 1:
        return 2.0 ** (b - 127)
    e = (b >> 3) & 15
    m = b & 7
    return np.where(e == 0, m / 8.0 * 2.0 ** -6, (1 + m / 8.0) * 2.0 ** (e - 7))


@pytest.mark.parametrize("fmt", [0, 1])
def test_constant_operands_closed_form(orc, fmt):
    k = orc.block_size(fmt)
    M, N, K = 8, 16, 4 * k * 4
    one = E4M3_ONE if fmt == 0 else E8M0_ONE
    A = pack_codes(np.full((M, K), 2))          # 1.0
    B = pack_codes(np.full((N, K), 1))          # 0.5
    sA = tile_scales(orc, np.full((M, K // k), one, dtype=np.uint8))
    sB = tile_scales(orc, np.full((N, K // k), one, dtype=np.uint8))
    D, S = orc.gemm(fmt, A, sA, B, sB)
    assert np.all(D == 0.5 * K) and np.all(S == 0.5 * K)
    D2, _ = orc.gemm(fmt, A, sA, B, sB, alpha=2.0)
    assert np.all(D2 == 2 * D)
    D3, S3 = orc.gemm(fmt, A, sA, B, sB, alpha=-0.25)
    assert np.all(D3 == -0.125 * K) and np.all(S3 == 0.125 * K)


@pytest.mark.parametrize("fmt", [0, 1])
def test_one_hot_row_selects_column_of_b(orc, fmt):
    k = orc.block_size(fmt)
    rng = np.random.default_rng(3)
    M, N, K = 4, 24, 8 * k
    one = E4M3_ONE if fmt == 0 else E8M0_ONE
    codesA = np.zeros((M, K), dtype=np.uint8)
    js = [0, 5, K // 2 + 1, K - 1]
    for m, j in enumerate(js):
        codesA[m, j] = 2
    codesB = rng.integers(0, 16, (N, K)).astype(np.uint8)
    if fmt == 0:
        rmB = rng.integers(0x08, 0x70, (N, K // k)).astype(np.uint8)
    else:
        rmB = rng.integers(100, 150, (N, K // k)).astype(np.uint8)
    D, _ = orc.gemm(fmt, pack_codes(codesA), tile_scales(orc, np.full((M, K // k), one, np.uint8)),
                    pack_codes(codesB), tile_scales(orc, rmB))
    for m, j in enumerate(js):
        want = E2M1_LUT[codesB[:, j]] * scale_value(fmt, rmB[:, j // k])
        assert np.array_equal(D[m], want)


@pytest.mark.parametrize("fmt", [0, 1])
def test_every_single_block_code_pair(orc, fmt):
    k = orc.block_size(fmt)
    rng = np.random.default_rng(4)
    codes = np.arange(16, dtype=np.uint8)
    for trial in range(6):
        pos = int(rng.integers(0, k))
        codesA = np.zeros((16, k), dtype=np.uint8)
        codesB = np.zeros((16, k), dtype=np.uint8)
        codesA[:, pos] = codes
        codesB[:, pos] = codes
        if fmt == 0:
            sa, sb = rng.integers(1, 0x7F, 2)
        else:
            sa, sb = rng.integers(90, 165, 2)
        D, _ = orc.gemm(fmt, pack_codes(codesA), tile_scales(orc, np.full((16, 1), sa, np.uint8)),
                        pack_codes(codesB), tile_scales(orc, np.full((16, 1), sb, np.uint8)),
                        alpha=1.5)
        want = 1.5 * np.outer(E2M1_LUT, E2M1_LUT) * scale_value(fmt, sa) * scale_value(fmt, sb)
        assert np.array_equal(D, want)


@pytest.mark.parametrize("fmt", [0, 1])
def test_matches_independent_fp64_matmul(orc, fmt):
    M, N, K = 37, 52, 512
    A = synth.normal_bf16(M, K, seed=5, outlier_factor=30.0)
    B = synth.normal_bf16(N, K, seed=5, tensor_id=1)
    gsA = orc.global_scale(A) if fmt == 0 else 1.0
    gsB = orc.global_scale(B) if fmt == 0 else 1.0
    pA, sA, rA = orc.quantize(fmt, 0, A, gs=gsA, with_rowmajor_scales=True)
    pB, sB, rB = orc.quantize(fmt, 0, B, gs=gsB, with_rowmajor_scales=True)
    k = orc.block_size(fmt)

    def decode(p, rm):
        nib = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
        nib[:, 0::2] = p & 15
        nib[:, 1::2] = p >> 4
        return E2M1_LUT[nib] * np.repeat(scale_value(fmt, rm), k, axis=1)

    a_hat, b_hat = decode(pA, rA), decode(pB, rB)
    alpha = float(np.float32(gsA) * np.float32(gsB))
    D, S = orc.gemm(fmt, pA, sA, pB, sB, alpha=alpha)
    want = alpha * (a_hat @ b_hat.T)
    assert np.allclose(D, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    assert np.allclose(S, abs(alpha) * (np.abs(a_hat) @ np.abs(b_hat).T), rtol=1e-12)
    # the sampled form agrees with the full form
    ms = np.array([0, 3, 36, 17]); ns = np.array([0, 51, 7, 25])
    Dp, Sp = orc.gemm_pairs(fmt, pA, sA, pB, sB, ms, ns, alpha=alpha)
    assert np.array_equal(Dp, D[ms, ns]) and np.array_equal(Sp, S[ms, ns])


def test_nv_error_below_mx_error(orc):
    # invariant of the method: finer blocks and E4M3 scales reconstruct the
    # product more closely than 32-element power-of-two blocks
    M = N = K = 256
    A = synth.normal_bf16(M, K, seed=6, outlier_factor=50.0)
    B = synth.normal_bf16(N, K, seed=6, tensor_id=1)
    Af = synth.bf16_bits_to_f32(A).astype(np.float64)
    Bf = synth.bf16_bits_to_f32(B).astype(np.float64)
    ref = Af @ Bf.T
    err = {}
    for fmt in (0, 1):
        gsA = orc.global_scale(A) if fmt == 0 else 1.0
        gsB = orc.global_scale(B) if fmt == 0 else 1.0
        pA, sA = orc.quantize(fmt, 0, A, gs=gsA)
        pB, sB = orc.quantize(fmt, 0, B, gs=gsB)
        D, _ = orc.gemm(fmt, pA, sA, pB, sB, alpha=float(np.float32(gsA) * np.float32(gsB)))
        err[fmt] = np.linalg.norm(D - ref) / np.linalg.norm(ref)
    assert err[0] < err[1] < 0.2
