"""Pins of the oracle's block quantizer (no GPU): brute-force enumeration of
(block amax, value) rounding cases against a slow form written here, scale
layout invariants, outlier isolation, footprint and the pages' accuracy
narrative.
"""
import os

import numpy as np
import pytest
import torch

from block_scaled_fp4_05_b200 import synth
from test_oracle_formats import E2M1_MAGS, bf16_to_f32, nearest_e2m1_codes

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def unpack_nibbles(packed):
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 15
    out[..., 1::2] = p >> 4
    return out


def mx_bruteforce_blocks():
    """Blocks of 32: element 0 is the block amax; the other 31 slots hold, in
    turn, every BF16 magnitude v <= amax whose ratio v / 2^e lies in
    [2^-4, 6] (the range where rounding decisions happen), with alternating
    signs.  amax runs over every normal BF16 exponent and mantissas on both
    sides of the 1.5 boundary of the ceil(log2(amax/6)) rule."""
    blocks = []
    for ef in range(1, 255):
        for mant in (0, 1, 63, 64, 65, 127):
            amax_bits = (ef << 7) | mant
            amax = float(bf16_to_f32(np.array([amax_bits], dtype=np.uint16))[0])
            if amax < 1e-8:
                continue
            lo_ef = max(1, ef - 6)
            cand = np.arange(lo_ef << 7, amax_bits + 1, dtype=np.uint16)
            cand = cand[cand != amax_bits]
            for i in range(0, len(cand), 31):
                chunk = cand[i:i + 31]
                row = np.zeros(32, dtype=np.uint16)
                row[0] = amax_bits
                row[1:1 + len(chunk)] = chunk
                row[1::2] |= 0x8000  # alternate signs (odd slots negative)
                blocks.append(row)
    return np.array(blocks, dtype=np.uint16)


def test_mx_quantizer_bruteforce_amax_value_pairs(orc):
    x = mx_bruteforce_blocks()
    assert x.shape[0] > 20000
    packed, scales, rm = orc.quantize(orc.MXFP4, orc.ROWWISE, x, with_rowmajor_scales=True)
    xf = bf16_to_f32(x)
    amax = np.abs(xf.astype(np.float64)).max(axis=1)
    # slow form: smallest e with 6 * 2^e >= amax, via FP64 log2 and a check
    e = np.ceil(np.log2(np.maximum(amax, np.float64(np.float32(1e-8))) / 6.0))
    e = np.where(6.0 * 2.0 ** (e - 1) >= amax, e - 1, e)
    assert np.array_equal(rm[:, 0].astype(np.int64), e.astype(np.int64) + 127)
    ratio = (xf.astype(np.float64) / 2.0 ** e[:, None]).astype(np.float32)  # exact
    want = nearest_e2m1_codes(ratio.ravel()).reshape(x.shape)
    got = unpack_nibbles(packed)
    bad = np.argwhere(got != want)
    assert bad.size == 0, bad[:5]


def e4m3_nearest(t):
    """Independent E4M3 rounding for the NVFP4 check: torch's FP8 conversion
    (round-to-nearest-even) with saturation at 448."""
    t = np.asarray(t, dtype=np.float32)
    b = torch.from_numpy(np.minimum(t, np.float32(448.0)).copy()).to(torch.float8_e4m3fn)
    return b.view(torch.uint8).numpy(), b.float().numpy()


@pytest.mark.parametrize("gs", [1.0, 50.0 * 4.0 / 2688.0, 2.0 ** -10, 0.37])
def test_nv_quantizer_bruteforce_sampled(orc, gs):
    gs = np.float32(gs)
    rng = np.random.default_rng(7)
    nblk = 20000
    # amax spread over the whole useful range of t = amax / (6 gs)
    t_target = 2.0 ** rng.uniform(-12, 9.5, nblk)
    amax = (t_target * 6.0 * gs).astype(np.float32)
    amax_bits = synth.f32_to_bf16_bits(amax)
    amax = bf16_to_f32(amax_bits)
    # the other 15 slots: uniform fractions of amax plus exact tie points
    frac = rng.uniform(-1, 1, (nblk, 15)).astype(np.float32)
    vals_bits = synth.f32_to_bf16_bits(frac * amax[:, None])
    vals = bf16_to_f32(vals_bits)
    vals = np.where(np.abs(vals) > amax[:, None], np.copysign(amax[:, None], vals), vals)
    x = np.concatenate([amax_bits[:, None], synth.f32_to_bf16_bits(vals)], axis=1)
    x = np.ascontiguousarray(x, dtype=np.uint16)
    packed, scales, rm = orc.quantize(orc.NVFP4, orc.ROWWISE, x, gs=float(gs),
                                      with_rowmajor_scales=True)
    xf = bf16_to_f32(x)
    a = np.abs(xf).max(axis=1).astype(np.float32)
    # the reading's FP32 sequence, in numpy FP32
    t = a / (np.float32(6.0) * gs)
    sb, sbv = e4m3_nearest(t)
    assert np.array_equal(rm[:, 0], sb)
    eff = (sbv.astype(np.float32) * gs).astype(np.float32)
    with np.errstate(divide="ignore", over="ignore"):
        inv = np.where(eff == 0, np.float32(0), np.float32(1.0) / eff).astype(np.float32)
    inv = np.minimum(inv, np.finfo(np.float32).max)
    v = (xf * inv[:, None]).astype(np.float32)
    want = nearest_e2m1_codes(v.ravel()).reshape(x.shape)
    got = unpack_nibbles(packed)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("gs", [1.0, 50.0 * 4.0 / 2688.0, 2.0 ** -10, 0.37, 1e-38, 3e38])
def test_p1e8_quantizer_bruteforce_sampled(orc, gs):
    # E8M0 block scale on 16-element blocks under S_global: S_block = 2^e with
    # e the smallest integer such that 2^e >= max(amax / (6 gs), 1e-8) (the
    # ratio formed in FP32), capped at 127; elements times RN(1 / (2^e gs)).
    # The slow form below finds e with an FP64 log2 and checks both sides.
    gs = np.float32(gs)
    rng = np.random.default_rng(8)
    nblk = 20000
    amax = (2.0 ** rng.uniform(-20, 20, nblk)).astype(np.float32)
    amax_bits = synth.f32_to_bf16_bits(amax)
    amax_bits[:64] = synth.f32_to_bf16_bits(np.float32(6.0) * 2.0 ** np.arange(-32, 32).astype(np.float32))
    amax = bf16_to_f32(amax_bits)
    frac = rng.uniform(-1, 1, (nblk, 15)).astype(np.float32)
    vals = bf16_to_f32(synth.f32_to_bf16_bits(frac * amax[:, None]))
    vals = np.where(np.abs(vals) > amax[:, None], np.copysign(amax[:, None], vals), vals)
    x = np.ascontiguousarray(np.concatenate([amax_bits[:, None], synth.f32_to_bf16_bits(vals)], axis=1),
                             dtype=np.uint16)
    packed, scales, rm = orc.quantize(orc.P1E8, orc.ROWWISE, x, gs=float(gs), with_rowmajor_scales=True)
    xf = bf16_to_f32(x)
    a32 = np.abs(xf).max(axis=1).astype(np.float32)
    with np.errstate(over="ignore", divide="ignore"):
        ratio = (a32 / (np.float32(6.0) * gs)).astype(np.float32)
    r = np.maximum(ratio.astype(np.float64), np.float64(np.float32(1e-8)))
    with np.errstate(over="ignore", divide="ignore", invalid="ignore"):
        e = np.where(np.isinf(r), 200.0, np.ceil(np.log2(r)))
    e = np.where((e > -200) & (2.0 ** (e - 1) >= r), e - 1, e)   # smallest e with 2^e >= r
    e = np.minimum(e, 127).astype(np.int64)
    assert np.all((2.0 ** e.astype(np.float64) >= np.minimum(r, 2.0 ** 127)))
    assert np.array_equal(rm[:, 0].astype(np.int64), e + 127)
    eff = (np.ldexp(np.float32(1.0), e).astype(np.float32) * gs).astype(np.float32)
    with np.errstate(divide="ignore", over="ignore"):
        inv = np.where(eff == 0, np.float32(0), np.float32(1.0) / eff).astype(np.float32)
    inv = np.minimum(inv, np.finfo(np.float32).max)
    v = (xf * inv[:, None]).astype(np.float32)
    want = nearest_e2m1_codes(v.ravel()).reshape(x.shape)
    assert np.array_equal(unpack_nibbles(packed), want)


def test_colwise_is_rowwise_of_transpose(orc):
    x = synth.normal_bf16(96, 200, seed=11, outlier_factor=20.0)
    for fmt in (orc.NVFP4, orc.MXFP4):
        gs = orc.global_scale(x)
        pc, sc = orc.quantize(fmt, orc.COLWISE, x, gs=gs)
        pr, sr = orc.quantize(fmt, orc.ROWWISE, np.ascontiguousarray(x.T), gs=gs)
        assert np.array_equal(pc, pr) and np.array_equal(sc, sr)


def test_scale_layout_bijection_and_padding(orc):
    for rows, nsc in [(1, 4), (129, 8), (200, 12), (256, 4)]:
        offs = np.array([[orc.scale_offset(r, c, nsc) for c in range(nsc)] for r in range(rows)])
        total = orc.scale_bytes(rows, nsc)
        assert total == ((rows + 127) // 128) * ((nsc + 3) // 4) * 512
        assert offs.min() >= 0 and offs.max() < total
        assert len(np.unique(offs)) == rows * nsc
    x = synth.normal_bf16(130, 128, seed=12)
    for fmt in (orc.NVFP4, orc.MXFP4):
        p, s, rm = orc.quantize(fmt, orc.ROWWISE, x, gs=orc.global_scale(x), with_rowmajor_scales=True)
        nsc = rm.shape[1]
        hit = np.zeros(s.size, dtype=bool)
        for r in range(130):
            for c in range(nsc):
                o = orc.scale_offset(r, c, nsc)
                assert s[o] == rm[r, c]
                hit[o] = True
        assert np.all(s[~hit] == 0)  # padding rows 130..255 are zero


def test_block_sizes_and_scale_counts(orc):
    facts = {}
    with open(os.path.join(GOLDEN, "format_facts.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            k, v = line.split()[:2]
            facts[k] = float(v)
    assert orc.block_size(orc.NVFP4) == facts["nvfp4_block_size"] == 16
    assert orc.block_size(orc.MXFP4) == facts["mxfp4_block_size"] == 32
    x = synth.normal_bf16(128, 512, seed=13)
    _, _, rm_nv = orc.quantize(orc.NVFP4, orc.ROWWISE, x, with_rowmajor_scales=True)
    _, _, rm_mx = orc.quantize(orc.MXFP4, orc.ROWWISE, x, with_rowmajor_scales=True)
    assert rm_nv.size == 128 * 512 // 16 and rm_mx.size == 128 * 512 // 32


def test_footprint_matches_pages(orc):
    facts = {}
    with open(os.path.join(GOLDEN, "format_facts.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            k, v = line.split()[:2]
            facts[k] = float(v)
    R, K = 1024, 4096
    x = synth.normal_bf16(R, K, seed=14)
    bits = {}
    for fmt in (orc.NVFP4, orc.MXFP4):
        p, s = orc.quantize(fmt, orc.ROWWISE, x, gs=orc.global_scale(x))
        bits[fmt] = 8.0 * (p.nbytes + s.nbytes) / (R * K)
    assert bits[orc.NVFP4] == facts["bits_per_param_k16"] == 4.5
    assert bits[orc.MXFP4] == facts["bits_per_param_mxfp4"] == 4.25
    # "3.5x smaller than FP16, 1.8x smaller than FP8" (rounded on the page)
    assert abs(16.0 / bits[orc.NVFP4] - facts["reduction_vs_fp16"]) < 0.1
    assert round(8.0 / bits[orc.NVFP4], 1) == facts["reduction_vs_fp8"]
    # MXFP4: 46.8% less than FP8 (1 - 4.25/8 = 46.875%)
    assert abs(100 * (1 - bits[orc.MXFP4] / 8.0) - facts["mxfp4_saving_vs_fp8_percent"]) < 0.1
    # the footprint table: params * 4.5 bits, BF16 2 bytes, FP8 1 byte
    with open(os.path.join(GOLDEN, "footprint_table.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, pb, bf16, fp8, nv = line.split()
            params = float(pb) * 1e9
            assert round(params * 2 / 1e9, 1) == float(bf16)
            assert round(params * 1 / 1e9, 1) == float(fp8)
            assert round(params * bits[orc.NVFP4] / 8 / 1e9, 1) == float(nv), name


def test_outlier_isolation_mx_and_nv_fixed_gs(orc):
    # an outlier at index 14 widens only micro-block 0's scale
    x = synth.normal_bf16(1, 256, seed=15)
    y = x.copy()
    yf = bf16_to_f32(y)
    yf[0, 14] *= 100.0
    y = synth.f32_to_bf16_bits(yf)
    for fmt, k in ((orc.MXFP4, 32), (orc.NVFP4, 16)):
        gs = orc.global_scale(x)
        px, sx, rx = orc.quantize(fmt, orc.ROWWISE, x, gs=gs, with_rowmajor_scales=True)
        py, sy, ry = orc.quantize(fmt, orc.ROWWISE, y, gs=gs, with_rowmajor_scales=True)
        assert ry[0, 0] > rx[0, 0]
        assert np.array_equal(ry[0, 1:], rx[0, 1:])
        assert np.array_equal(px[0, k // 2:], py[0, k // 2:])
    # NVFP4 with a recomputed S_global: the per-tensor scale moves, so the
    # other blocks' E4M3 bytes legitimately move too
    gy = orc.global_scale(y)
    _, _, ry2 = orc.quantize(orc.NVFP4, orc.ROWWISE, y, gs=gy, with_rowmajor_scales=True)
    _, _, rx2 = orc.quantize(orc.NVFP4, orc.ROWWISE, x, gs=orc.global_scale(x), with_rowmajor_scales=True)
    assert not np.array_equal(ry2[0, 1:], rx2[0, 1:])


def test_naive_per_tensor_collapse_vs_microscaling(orc):
    # a 4096-dim activation with one 64.8 outlier: per-tensor scaling sends
    # the normal values to zero; micro-block scaling keeps them
    rng = np.random.default_rng(16)
    x = (rng.standard_normal(4096) * 0.1).astype(np.float32)
    x[1234] = 64.8
    xb = synth.f32_to_bf16_bits(x)
    xf = bf16_to_f32(xb)
    naive = orc.naive_per_tensor(xf)
    normal = np.ones(4096, dtype=bool)
    normal[1234] = False
    assert np.mean(naive[normal] == 0.0) > 0.99
    assert naive[1234] == pytest.approx(xf[1234], rel=1e-6)
    for fmt in (orc.MXFP4, orc.NVFP4):
        xr = xb.reshape(1, -1)
        p, s = orc.quantize(fmt, orc.ROWWISE, xr, gs=orc.global_scale(xr))
        deq = orc.dequantize(fmt, p, s, gs=orc.global_scale(xr) if fmt == orc.NVFP4 else 0.0)[0]
        assert np.mean(deq[normal] == 0.0) < 0.15


def snr_db(x, y):
    x = np.asarray(x, dtype=np.float64)
    return 10 * np.log10(np.sum(x ** 2) / np.sum((x - y) ** 2))


def test_emulation_script_experiment_ordering(orc):
    # the emulation script's experiment: 1024 values randn*0.5 (torch seed 42),
    # outliers 24.5 at 42 and -31.2 at 512, block size 16 with power-of-two
    # scales; the page prints no numbers, so only the ordering is pinned
    torch.manual_seed(42)
    x = (torch.randn(1024) * 0.5).numpy()
    x[42] = 24.5
    x[512] = -31.2
    naive = orc.naive_per_tensor(x)
    for page_tie in (False, True):
        blk = orc.block_pow2_roundtrip(x, 16, page_tie=page_tie)
        assert snr_db(x, blk) > snr_db(x, naive) + 10.0
    # same with the library formats on the BF16-rounded vector
    xb = synth.f32_to_bf16_bits(x).reshape(1, -1)
    xf = bf16_to_f32(xb)[0]
    for fmt in (orc.MXFP4, orc.NVFP4):
        gs = orc.global_scale(xb)
        p, s = orc.quantize(fmt, orc.ROWWISE, xb, gs=gs)
        deq = orc.dequantize(fmt, p, s, gs=gs if fmt == orc.NVFP4 else 0.0)[0]
        assert snr_db(xf, deq) > snr_db(xf, orc.naive_per_tensor(xf)) + 10.0


def test_reconstruction_error_bound(orc):
    # |x - x_hat| <= half the local grid step (1 in units of the block scale
    # where the E2M1 gap is 2) unless saturated: x / S within [0, 6]
    x = synth.normal_bf16(64, 512, seed=17, outlier_factor=80.0)
    xf = bf16_to_f32(x).astype(np.float64)
    p, s, rm = orc.quantize(orc.MXFP4, orc.ROWWISE, x, with_rowmajor_scales=True)
    deq = orc.dequantize(orc.MXFP4, p, s)
    S = np.repeat(2.0 ** (rm.astype(np.float64) - 127), 32, axis=1)
    r = np.abs(xf) / S
    step = np.select([r <= 2, r <= 4], [0.5, 1.0], 2.0)
    assert np.all(r <= 6.0)
    assert np.all(np.abs(xf - deq) <= 0.5 * step * S)


@pytest.mark.parametrize("fmt", ["nv", "mx", "p1e8"])
def test_dequantize_is_code_times_scales(orc, fmt):
    # x_hat = E2M1(code) * S_block (* S_global), written out here from the
    # packed nibbles and the row-major scale bytes: E4M3 for NVFP4 (torch's
    # FP8 decode), 2^(byte - 127) for the E8M0 formats
    f = {"nv": orc.NVFP4, "mx": orc.MXFP4, "p1e8": orc.P1E8}[fmt]
    k = 32 if fmt == "mx" else 16
    x = synth.normal_bf16(40, 512, seed=18, outlier_factor=80.0, zero_frac=0.05)
    gs = orc.global_scale(x) if fmt != "mx" else 1.0
    p, s, rm = orc.quantize(f, orc.ROWWISE, x, gs=gs, with_rowmajor_scales=True)
    deq = orc.dequantize(f, p, s, gs=gs if fmt != "mx" else 0.0)
    codes = unpack_nibbles(p).astype(np.int64)
    mags = np.array(E2M1_MAGS, dtype=np.float64)[codes & 7]
    vals = np.where(codes & 8, -mags, mags)
    if fmt == "nv":
        sv = torch.from_numpy(rm.copy()).view(torch.float8_e4m3fn).double().numpy()
    else:
        sv = 2.0 ** (rm.astype(np.float64) - 127)
    want = vals * np.repeat(sv, k, axis=1) * (float(np.float32(gs)) if fmt != "mx" else 1.0)
    assert np.array_equal(deq.reshape(want.shape), want)
    assert np.array_equal(np.signbit(deq.reshape(want.shape)), np.signbit(want))


def first_index_nearest_mags(v):
    """The emulation script's argmin rule written here: nearest magnitude,
    the lower grid index on a tie (so ties go to the smaller magnitude)."""
    a = np.abs(np.asarray(v, dtype=np.float32).astype(np.float64))
    d = np.abs(a[:, None] - E2M1_MAGS[None, :])
    return np.where(a >= 6.0, 6.0, E2M1_MAGS[d.argmin(axis=1)])


@pytest.mark.parametrize("k", [16, 32])
@pytest.mark.parametrize("page_tie", [False, True])
def test_block_pow2_roundtrip_and_naive_against_slow_forms(orc, k, page_tie):
    # the emulation script's block quantize / dequantize with power-of-two
    # scales (zero-padded last block) and the naive per-tensor baseline,
    # each written here from its definition
    rng = np.random.default_rng(19)
    x = (rng.standard_normal(1000) * 0.5).astype(np.float32)
    x[42], x[512] = 24.5, -31.2
    x[100:116] = 0.0
    x[200] = 0.75 * 2.0 ** -3   # a tie point
    got = orc.block_pow2_roundtrip(x, k, page_tie=page_tie)
    want = np.empty(x.size)
    for b0 in range(0, x.size, k):
        blk = x[b0:b0 + k]
        amax = max(float(np.abs(blk).max()), float(np.float32(1e-8)))
        e = int(np.ceil(np.log2(amax / 6.0)))
        if 6.0 * 2.0 ** (e - 1) >= amax:
            e -= 1
        v = (blk * np.float32(2.0 ** -e)).astype(np.float32)
        mags = first_index_nearest_mags(v) if page_tie else E2M1_MAGS[nearest_e2m1_codes(v) & 7]
        want[b0:b0 + k] = np.where(np.signbit(v), -mags, mags) * 2.0 ** e
    assert np.array_equal(got, want)
    s = np.float32(max(np.float32(np.abs(x).max()), np.float32(1e-8)) / np.float32(6.0))
    v = (x / s).astype(np.float32)
    mags = E2M1_MAGS[nearest_e2m1_codes(v) & 7]
    assert np.array_equal(orc.naive_per_tensor(x), np.where(np.signbit(v), -mags, mags) * float(s))
