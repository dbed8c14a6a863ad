"""Pins of the oracle's number formats against what the pages and independent
implementations fix (no GPU).

Each check compares the oracle's C code with something other than itself:
the code table the pages print, a nearest-value search written here in numpy,
the emulation script's own formula evaluated with torch, or torch's FP8
conversion.
"""
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
E2M1_MAGS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def all_finite_bf16_bits(nonneg_only=False):
    b = np.arange(0, 1 << 16, dtype=np.uint32)
    exp = (b >> 7) & 0xFF
    keep = exp != 0xFF
    if nonneg_only:
        keep &= b < 0x8000
    return b[keep].astype(np.uint16)


def bf16_to_f32(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


def nearest_e2m1_codes(v):
    """Independent nearest-E2M1 search: exact FP64 distance to the eight
    magnitudes, ties to the code with even mantissa bit, saturating at 6."""
    v = np.asarray(v, dtype=np.float32)
    a = np.abs(v.astype(np.float64))
    d = np.abs(a[:, None] - E2M1_MAGS[None, :])
    dmin = d.min(axis=1, keepdims=True)
    cand = d == dmin
    even = cand & (np.arange(8)[None, :] % 2 == 0)
    code = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    code = np.where(a >= 6.0, 7, code)
    return (code | (np.signbit(v).astype(np.int64) << 3)).astype(np.uint8)


def load_code_table():
    rows = []
    with open(os.path.join(GOLDEN, "e2m1_code_table.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            bits, val = line.split()
            rows.append((int(bits, 2), float(val)))
    return rows


def test_e2m1_decode_matches_page_code_table(orc):
    table = load_code_table()
    assert len(table) == 8
    for code, val in table:
        assert orc.e2m1_decode(code) == val
        # negative half mirrors with the sign bit; zero is signed
        neg = orc.e2m1_decode(code | 8)
        assert neg == -val and np.signbit(neg)


def test_e2m1_value_set_and_saturation(orc):
    vals = sorted({abs(orc.e2m1_decode(c)) for c in range(16)})
    assert vals == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert max(vals) == 6.0
    for v in [6.0, 6.5, 7.0, 100.0, 1e30, float("inf")]:
        assert orc.e2m1_encode(v) == 7
        assert orc.e2m1_encode(-v) == 15


def test_e2m1_roundtrip_all_codes(orc):
    for c in range(16):
        assert orc.e2m1_encode(orc.e2m1_decode(c)) == c


def test_e2m1_ties_to_even_and_page_tie_rule(orc):
    # decision points between neighbours: RNE picks the even-mantissa code
    rne = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for v, want in rne.items():
        assert orc.e2m1_decode(orc.e2m1_encode(v)) == want
        assert orc.e2m1_decode(orc.e2m1_encode(-v)) == -want
    # the emulation script's argmin keeps the smaller magnitude on a tie
    page = {0.25: 0.0, 0.75: 0.5, 1.25: 1.0, 1.75: 1.5, 2.5: 2.0, 3.5: 3.0, 5.0: 4.0}
    for v, want in page.items():
        assert orc.e2m1_decode(orc.e2m1_encode_first_index_tie(v)) == want
    # the two rules disagree exactly at 0.75, 1.75 and 3.5
    diff = [v for v in rne if rne[v] != page[v]]
    assert diff == [0.75, 1.75, 3.5]


def test_e2m1_signed_zero_and_negative_underflow(orc):
    assert orc.e2m1_encode(-0.0) == 8
    assert orc.e2m1_encode(0.0) == 0
    assert orc.e2m1_encode(-0.1) == 8
    assert orc.e2m1_encode(-0.25) == 8
    assert orc.e2m1_encode(0.2) == 0


def test_e2m1_encode_bruteforce_all_bf16_scaled(orc):
    base = bf16_to_f32(all_finite_bf16_bits())
    with np.errstate(over="ignore"):
        vals = np.concatenate([(base.astype(np.float64) * 2.0 ** j).astype(np.float32)
                               for j in range(-8, 9)])
    got = orc.e2m1_encode_array(vals)
    want = nearest_e2m1_codes(vals)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (vals[bad[:5]], got[bad[:5]], want[bad[:5]])


def test_e8m0_decode_definition(orc):
    for E in range(256):
        assert orc.e8m0_decode(E) == 2.0 ** (E - 127)


def test_mx_exponent_matches_page_formula_for_every_bf16_amax(orc):
    # the emulation script, step 2, literally: clamp(amax, min=1e-8),
    # ceil(log2(amax / 6.0)) in FP32 torch arithmetic
    a = bf16_to_f32(all_finite_bf16_bits(nonneg_only=True))
    t = torch.from_numpy(a.copy())
    page = torch.ceil(torch.log2(torch.clamp(t, min=1e-8) / 6.0)).numpy().astype(np.int64)
    got = orc.mx_exponent_array(a).astype(np.int64)
    assert np.array_equal(got, page)
    # zero block: clamp 1e-8 -> ceil(log2(1e-8/6)) = -29 -> E8M0 byte 98
    assert orc.e8m0_encode_block(0.0) == 98
    # byte range for finite BF16 input
    assert got.min() + 127 == 98 and got.max() + 127 == 253
    # definition: 6 * 2^e >= amax > 6 * 2^(e-1) above the clamp
    big = a >= 1e-8
    e = got[big].astype(np.float64)
    assert np.all(6.0 * 2.0 ** e >= a[big]) and np.all(6.0 * 2.0 ** (e - 1) < a[big])


def test_e4m3_decode_matches_torch_fp8(orc):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).float().numpy()
    for c in range(256):
        got = orc.e4m3_decode(c)
        if np.isnan(ref[c]):
            assert np.isnan(got), c
        else:
            assert got == float(ref[c]), c
    assert orc.e4m3_decode(0x7E) == 448.0


def e4m3_midpoints():
    vals = np.array([orc_val for orc_val in torch.arange(0, 0x7F, dtype=torch.int32)
                     .to(torch.uint8).view(torch.float8_e4m3fn).float().numpy()], dtype=np.float64)
    mids = (vals[:-1] + vals[1:]) / 2.0
    m32 = mids.astype(np.float32)
    return np.concatenate([m32, np.nextafter(m32, np.float32(0)), np.nextafter(m32, np.float32(1e9))])


def test_e4m3_encode_matches_torch_fp8_rne(orc):
    a = bf16_to_f32(all_finite_bf16_bits(nonneg_only=True))
    rng = np.random.default_rng(123)
    t = np.concatenate([a[a < 464.0], e4m3_midpoints(),
                        rng.uniform(0, 464, 200000).astype(np.float32),
                        (2.0 ** rng.uniform(-14, 8.8, 200000)).astype(np.float32)])
    t = t[t < 464.0]
    want = torch.from_numpy(t.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = orc.e4m3_encode_unsigned_array(t)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (t[bad[:5]], got[bad[:5]], want[bad[:5]])


def test_e4m3_encode_saturates_at_448(orc):
    for t in [448.0, 449.0, 464.0, 480.0, 1e6, 3e38, float("inf")]:
        assert orc.e4m3_encode_unsigned(t) == 0x7E
    assert orc.e4m3_encode_unsigned(2.0 ** -10) == 0          # tie -> even (0)
    assert orc.e4m3_encode_unsigned(1.5 * 2.0 ** -9) == 2     # tie -> even code
    assert orc.e4m3_encode_unsigned(2.0 ** -9) == 1           # smallest subnormal


def test_global_scale_maps_tensor_amax_block_to_e4m3_max(orc):
    # reading of "a scalar representing the maximum dynamic ceiling of the
    # entire tensor": the block holding the tensor's amax gets the largest
    # E4M3 block scale (448) and no block exceeds it
    from block_scaled_fp4_05_b200 import synth
    for seed in range(4):
        x = synth.normal_bf16(64, 256, seed=seed, outlier_factor=37.0)
        gs = orc.global_scale(x)
        p, s, rm = orc.quantize(orc.NVFP4, orc.ROWWISE, x, gs=gs, with_rowmajor_scales=True)
        assert rm.max() == 0x7E
        xf = bf16_to_f32(x).reshape(64, 16, 16)
        r, b = np.unravel_index(np.abs(xf).max(axis=2).argmax(), (64, 16))
        assert rm[r, b] == 0x7E
    assert orc.global_scale(np.zeros((4, 64), dtype=np.uint16)) == 1.0
    assert orc.global_scale_from_amax(2688.0) == 1.0
