"""Reconstruction (fp4_dequantize) parity and the accuracy comparison the
pages make: native W4A4 block-scaled GEMM against a W4A16 path (weights
reconstructed to BF16, activations kept in BF16) and against naive
per-tensor FP4, all measured against the unquantized product.

Pages: "NVFP4 Architecture: Microscaling & 4-Bit LLMs on Blackwell",
"The Outlier Problem" (a per-tensor scale collapses the small values) and
"End-to-End Implementation" (block scaling keeps them); "Extreme
Quantization and Precision Engineering ..." (W4A16 vs native W4A4)."""
import numpy as np
import pytest
import torch

from block_scaled_fp4_05_b200 import fp4, synth
from gpu_util import bf16_dev_to_f64, to_dev_bf16, to_dev_f32, to_dev_u8

pytestmark = pytest.mark.gpu


def f64_to_bf16_bits(x):
    """Exact FP64 -> BF16 round-to-nearest-even (one rounding), as bits."""
    x = np.asarray(x, dtype=np.float64)
    neg = np.signbit(x)
    a = np.abs(x)
    _, e = np.frexp(a)
    q_exp = np.where(e - 1 >= -126, e - 8, -133)      # quantum: 8 significant bits, or subnormal
    v = np.ldexp(np.round(np.ldexp(a, -q_exp)), q_exp)
    with np.errstate(over="ignore"):              # beyond the BF16 range: infinity
        bits = (v.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    return np.where(neg, bits | 0x8000, bits).astype(np.uint16)


def test_f64_to_bf16_helper_against_torch():
    # float32 inputs: torch's float32 -> bfloat16 conversion is RNE
    rng = np.random.default_rng(60)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
                        [0.0, -0.0, 1.0, 1.00390625, 1.005859375, 3e38, 1e-40]]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(f64_to_bf16_bits(x.astype(np.float64)), want)


@pytest.mark.parametrize("fmt", [fp4.NVFP4, fp4.MXFP4, fp4.P1E8])
# (33, 2176): a row is one whole 2048-code warp task plus a 128-code tail
@pytest.mark.parametrize("shape", [(1, 512), (200, 1024), (129, 8192), (33, 2176)])
def test_dequantize_matches_oracle(orc, fmt, shape):
    rows, K = shape
    x = synth.normal_bf16(rows, K, seed=61, outlier_factor=100.0, zero_frac=0.02)
    gs = orc.global_scale(x) if fmt != fp4.MXFP4 else 0.0
    p, s = orc.quantize(fmt, fp4.ROWWISE, x, gs=gs if fmt != fp4.MXFP4 else 1.0)
    want = f64_to_bf16_bits(orc.dequantize(fmt, p, s, gs=gs).reshape(rows, K))
    out = torch.full((rows, K + 8), float("nan"), dtype=torch.bfloat16, device="cuda")
    fp4.fp4_dequantize(fmt, to_dev_u8(p), to_dev_u8(s), to_dev_f32(gs) if fmt != fp4.MXFP4 else None,
                       out[:, :K])
    torch.cuda.synchronize()
    got = out[:, :K].cpu().view(torch.int16).numpy().view(np.uint16)
    bad = np.argwhere(got != want)
    assert bad.size == 0, (bad[:4].tolist(), got[tuple(bad[0])], want[tuple(bad[0])])
    assert torch.isnan(out[:, K:].float()).all()


@pytest.mark.parametrize("fmt", [fp4.NVFP4, fp4.MXFP4, fp4.P1E8])
@pytest.mark.parametrize("gs", [0.37, 3.1e-38, 2.0e36])
def test_dequantize_random_codes_and_scales(orc, fmt, gs):
    # every code with scale bytes drawn over the whole encoding (negative and
    # subnormal E4M3, E8M0 0..255; not the E4M3 NaN codes) and S_global
    # values whose products underflow to BF16 subnormals or overflow: the
    # rounding of every product, not only of the quantizer's usual range
    rows, K = 130, 1024
    rng = np.random.default_rng(63 + fmt)
    p = rng.integers(0, 256, size=(rows, K // 2), dtype=np.uint8)
    nb = fp4.fp4_scale_bytes(fmt, rows, K)
    s = rng.integers(0, 256, size=nb, dtype=np.uint8)
    if fmt == fp4.NVFP4:
        s[(s & 0x7F) == 0x7F] = 0x3F
    g = gs if fmt != fp4.MXFP4 else 0.0
    want = f64_to_bf16_bits(orc.dequantize(fmt, p, s, gs=g).reshape(rows, K))
    out = torch.full((rows, K + 8), float("nan"), dtype=torch.bfloat16, device="cuda")
    fp4.fp4_dequantize(fmt, to_dev_u8(p), to_dev_u8(s), to_dev_f32(g) if fmt != fp4.MXFP4 else None,
                       out[:, :K])
    torch.cuda.synchronize()
    got = out[:, :K].cpu().view(torch.int16).numpy().view(np.uint16)
    bad = np.argwhere(got != want)
    assert bad.size == 0, (bad[:4].tolist(), got[tuple(bad[0])], want[tuple(bad[0])])
    assert torch.isnan(out[:, K:].float()).all()


def snr_db(ref, got):
    return 10.0 * np.log10(np.sum(ref ** 2) / np.sum((got - ref) ** 2))


@pytest.mark.parametrize("MNK", [(16, 1024, 8192), (256, 512, 2048)])
def test_w4a4_vs_w4a16_vs_naive_per_tensor(orc, MNK, record_property):
    M, N, K = MNK
    A = synth.normal_bf16(M, K, seed=62, outlier_factor=100.0)          # activations with outlier channels
    W = synth.normal_bf16(N, K, seed=62, tensor_id=1, sigma=0.02)         # weights
    Af = synth.bits_to_torch(A).double().numpy()
    Wf = synth.bits_to_torch(W).double().numpy()
    ref = Af @ Wf.T
    Ad, Wd = to_dev_bf16(A), to_dev_bf16(W)
    snr = {}
    for fmt, name in ((fp4.NVFP4, "w4a4_nvfp4"), (fp4.MXFP4, "w4a4_mxfp4")):
        gA = fp4.global_scale(Ad) if fmt == fp4.NVFP4 else None
        gW = fp4.global_scale(Wd) if fmt == fp4.NVFP4 else None
        pA, sA = fp4.quantize(Ad, fmt, fp4.ROWWISE, gA)
        pW, sW = fp4.quantize(Wd, fmt, fp4.ROWWISE, gW)
        alpha = None
        if fmt == fp4.NVFP4:
            alpha = torch.empty(1, dtype=torch.float32, device="cuda")
            fp4.fp4_alpha_from_global_scales(gA, gW, alpha)
        D = fp4.gemm(fmt, pA, sA, pW, sW, K, alpha=alpha)
        torch.cuda.synchronize()
        snr[name] = snr_db(ref, bf16_dev_to_f64(D))
        if fmt == fp4.NVFP4:
            # W4A16: the same NVFP4 weights reconstructed to BF16, activations in BF16
            Wh = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
            fp4.fp4_dequantize(fmt, pW, sW, gW, Wh)
            torch.cuda.synchronize()
            snr["w4a16_nvfp4_weights"] = snr_db(ref, Af @ Wh.cpu().double().numpy().T)
    Aq = orc.naive_per_tensor(Af.astype(np.float32)).reshape(M, K)
    Wq = orc.naive_per_tensor(Wf.astype(np.float32)).reshape(N, K)
    snr["naive_per_tensor_fp4"] = snr_db(ref, Aq @ Wq.T)
    for k, v in snr.items():
        record_property(k, round(float(v), 2))
    print("SNR (dB) vs the unquantized product, %s:" % (MNK,),
          ", ".join("%s %.2f" % (k, v) for k, v in snr.items()))
    # the pages' orderings: weight-only beats W4A4; block scaling with the
    # finer E4M3 scale (16-element blocks) beats power-of-two scales on 32;
    # a single per-tensor scale collapses the non-outlier values
    assert snr["w4a16_nvfp4_weights"] > snr["w4a4_nvfp4"] > snr["w4a4_mxfp4"] > snr["naive_per_tensor_fp4"]
    assert snr["naive_per_tensor_fp4"] < 10.0 < snr["w4a4_mxfp4"]


def test_square_4096_error_nv_below_mx(record_property):
    # The 4096^3 inputs (outlier channels in A), quantized on the GPU in both
    # formats and multiplied by the GPU GEMM: relative Frobenius error and SNR
    # of D against the FP64 product of the original BF16 inputs (computed on
    # the GPU in FP64).  NVFP4's 16-element blocks with E4M3 scales must give
    # the smaller error (an invariant of the formats, not a pinned value).
    A, B = synth.square(4096)
    Ad, Bd = to_dev_bf16(A), to_dev_bf16(B)
    ref = Ad.double() @ Bd.double().T
    err = {}
    for fmt, name in ((fp4.NVFP4, "nvfp4"), (fp4.MXFP4, "mxfp4")):
        gA = fp4.global_scale(Ad) if fmt == fp4.NVFP4 else None
        gB = fp4.global_scale(Bd) if fmt == fp4.NVFP4 else None
        pA, sA = fp4.quantize(Ad, fmt, fp4.ROWWISE, gA)
        pB, sB = fp4.quantize(Bd, fmt, fp4.ROWWISE, gB)
        alpha = gA * gB if fmt == fp4.NVFP4 else None
        D = fp4.gemm(fmt, pA, sA, pB, sB, 4096, alpha=alpha, kernel=fp4.GEMM_PREFILL)
        torch.cuda.synchronize()
        assert fp4.fp4_get_device_status() == 0
        diff = D.double() - ref
        rel = float(torch.linalg.norm(diff) / torch.linalg.norm(ref))
        err[name] = (rel, -20.0 * np.log10(rel))
        record_property("rel_fro_" + name, rel)
    print("4096^3 relative Frobenius error / SNR: NVFP4 %.4f / %.2f dB, MXFP4 %.4f / %.2f dB" % (
        err["nvfp4"][0], err["nvfp4"][1], err["mxfp4"][0], err["mxfp4"][1]))
    assert err["nvfp4"][0] < err["mxfp4"][0]
    assert err["nvfp4"][0] < 0.2 and err["mxfp4"][0] < 0.3

