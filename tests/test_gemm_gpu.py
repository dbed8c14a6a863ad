"""GPU parity of the block-scaled GEMM kernels against the oracle (FP64
product of the dequantized operands), within the stated tolerance.  Operands
are quantized by the oracle and uploaded, so that the GEMM is tested on its
own; the end-to-end tests quantize on the GPU as well."""
import numpy as np
import pytest
import torch

from block_scaled_fp4_05_b200 import fp4, synth
from gpu_util import assert_gemm_close, bf16_dev_to_f64, to_dev_bf16, to_dev_f32, to_dev_u8

pytestmark = pytest.mark.gpu
FMTS = [fp4.NVFP4, fp4.MXFP4, fp4.P1E8]   # P1E8: 16-element blocks, E8M0 scales under S_global


def oracle_operands(orc, fmt, A_bits, B_bits):
    gsA = orc.global_scale(A_bits) if fmt != fp4.MXFP4 else 1.0
    gsB = orc.global_scale(B_bits) if fmt != fp4.MXFP4 else 1.0
    pA, sA = orc.quantize(fmt, 0, A_bits, gs=gsA)
    pB, sB = orc.quantize(fmt, 0, B_bits, gs=gsB)
    alpha = float(np.float32(gsA) * np.float32(gsB))
    return pA, sA, pB, sB, alpha


def run_gpu_gemm(fmt, pA, sA, pB, sB, K, alpha, kernel, ldd_pad=0):
    M, N = pA.shape[0], pB.shape[0]
    D = torch.full((M, N + ldd_pad), float("nan"), dtype=torch.bfloat16, device="cuda")
    Dv = D[:, :N]
    fp4.gemm(fmt, to_dev_u8(pA), to_dev_u8(sA), to_dev_u8(pB), to_dev_u8(sB), K,
             alpha=to_dev_f32(alpha), kernel=kernel, out=Dv)
    torch.cuda.synchronize()
    assert fp4.fp4_get_device_status() == 0
    if ldd_pad:
        assert torch.isnan(D[:, N:].float()).all()
    return bf16_dev_to_f64(Dv)


def test_constant_operands_exact():
    # A_hat = 1, B_hat = 0.5 -> D = 0.5 K exactly, no oracle involved
    for fmt in FMTS:
        k = fp4.block_size(fmt)
        M, N, K = 200, 264, 1024
        one = 0x38 if fmt == fp4.NVFP4 else 127
        A = torch.full((M, K // 2), 0x22, dtype=torch.uint8, device="cuda")
        B = torch.full((N, K // 2), 0x11, dtype=torch.uint8, device="cuda")
        sA = torch.full((fp4.fp4_scale_bytes(fmt, M, K),), one, dtype=torch.uint8, device="cuda")
        sB = torch.full((fp4.fp4_scale_bytes(fmt, N, K),), one, dtype=torch.uint8, device="cuda")
        for kernel in (fp4.GEMM_PREFILL,):
            D = fp4.gemm(fmt, A, sA, B, sB, K, kernel=kernel)
            torch.cuda.synchronize()
            assert torch.all(D.float() == 0.5 * K), (fmt, D.float().unique()[:8])


@pytest.mark.parametrize("fmt", FMTS)
def test_tiny_config(orc, fmt):
    A, B = synth.tiny_nv()
    pA, sA, pB, sB, alpha = oracle_operands(orc, fmt, A, B)
    D_orc, S = orc.gemm(fmt, pA, sA, pB, sB, alpha=alpha)
    D = run_gpu_gemm(fmt, pA, sA, pB, sB, 512, alpha, fp4.GEMM_PREFILL)
    assert_gemm_close(D, D_orc, S, "tiny")


@pytest.mark.parametrize("fmt", FMTS)
# K = 64: a single MMA per tile (NVFP4, P1E8); (130, 72, 64) also a ragged half tile
@pytest.mark.parametrize("MNK", [(1, 8, 128), (3, 24, 256), (129, 136, 384), (200, 264, 640),
                                 (300, 520, 1024), (128, 256, 2048), (257, 512, 128), (130, 72, 64)])
def test_prefill_ragged_shapes(orc, fmt, MNK):
    M, N, K = MNK
    if K % (128 if fmt == fp4.MXFP4 else 64):
        pytest.skip("K not supported by the format")
    A = synth.normal_bf16(M, K, seed=31, outlier_factor=50.0)
    B = synth.normal_bf16(N, K, seed=31, tensor_id=1, sigma=0.02)
    pA, sA, pB, sB, alpha = oracle_operands(orc, fmt, A, B)
    D_orc, S = orc.gemm(fmt, pA, sA, pB, sB, alpha=alpha)
    D = run_gpu_gemm(fmt, pA, sA, pB, sB, K, alpha, fp4.GEMM_PREFILL, ldd_pad=8)
    assert_gemm_close(D, D_orc, S, "prefill %s" % (MNK,))


@pytest.mark.parametrize("fmt", FMTS)
# (16, 38400, 1024) and (9, 38400, 1088): more weight tiles than SMs, so the
# decode schedule runs stream-K tiles and then whole tiles; 1088 adds a K tail
@pytest.mark.parametrize("MNK", [(1, 256, 512), (4, 1000, 1024), (16, 1024, 8192), (7, 136, 384),
                                 (16, 38400, 1024), (9, 38400, 1088), (5, 200, 64), (12, 520, 192)])
def test_decode_kernel_shapes(orc, fmt, MNK):
    M, N, K = MNK
    if K % (128 if fmt == fp4.MXFP4 else 64):
        pytest.skip("K not supported by the format")
    A = synth.normal_bf16(M, K, seed=32, outlier_factor=100.0)
    W = synth.normal_bf16(N, K, seed=32, tensor_id=1, sigma=0.02)
    pA, sA, pW, sW, alpha = oracle_operands(orc, fmt, A, W)
    D_orc, S = orc.gemm(fmt, pA, sA, pW, sW, alpha=alpha)
    D = run_gpu_gemm(fmt, pA, sA, pW, sW, K, alpha, fp4.GEMM_DECODE, ldd_pad=8)
    assert_gemm_close(D, D_orc, S, "decode %s" % (MNK,))
    D2 = run_gpu_gemm(fmt, pA, sA, pW, sW, K, alpha, fp4.GEMM_PREFILL)
    assert_gemm_close(D2, D_orc, S, "prefill-on-decode-shape %s" % (MNK,))


def test_decode_workspace_reused_across_shapes_stays_zeroed(orc):
    # one workspace, zeroed once, serves a sequence of shapes: every call
    # leaves the arrival counters (first 64 KB) at zero again
    fmt = fp4.NVFP4
    shapes = [(16, 1024, 8192), (3, 28672 // 4, 2048), (16, 1024, 8192), (1, 136, 384)]
    nb = max(fp4.fp4_gemm_workspace_bytes(fmt, *s) for s in shapes)
    ws = torch.zeros((nb,), dtype=torch.uint8, device="cuda")
    for i, (M, N, K) in enumerate(shapes):
        A = synth.normal_bf16(M, K, seed=40 + i, outlier_factor=100.0)
        W = synth.normal_bf16(N, K, seed=40 + i, tensor_id=1, sigma=0.02)
        pA, sA, pW, sW, alpha = oracle_operands(orc, fmt, A, W)
        D = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        fp4.fp4_gemm(fmt, to_dev_u8(pA), to_dev_u8(sA), to_dev_u8(pW), to_dev_u8(sW), M, N, K,
                     to_dev_f32(alpha), D, ws, kernel=fp4.GEMM_DECODE)
        torch.cuda.synchronize()
        assert fp4.fp4_get_device_status() == 0
        assert int(ws[:65536].count_nonzero().item()) == 0
        if N * K <= 1024 * 8192:
            D_orc, S = orc.gemm(fmt, pA, sA, pW, sW, alpha=alpha)
            assert_gemm_close(bf16_dev_to_f64(D), D_orc, S, "decode reuse %s" % ((M, N, K),))


def test_decode_workspace_not_zeroed_is_reported():
    # counters holding garbage: the kernel records it (no wait depends on
    # them) and the status call reports FP4_ERR_WORKSPACE
    fmt, M, N, K = fp4.NVFP4, 4, 512, 1024
    A = torch.randint(0, 256, (M, K // 2), dtype=torch.uint8, device="cuda")
    W = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device="cuda")
    sA = torch.full((fp4.fp4_scale_bytes(fmt, M, K),), 0x38, dtype=torch.uint8, device="cuda")
    sW = torch.full((fp4.fp4_scale_bytes(fmt, N, K),), 0x38, dtype=torch.uint8, device="cuda")
    ws = torch.full((fp4.fp4_gemm_workspace_bytes(fmt, M, N, K),), 0x7B, dtype=torch.uint8, device="cuda")
    D = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    fp4.fp4_gemm(fmt, A, sA, W, sW, M, N, K, None, D, ws, kernel=fp4.GEMM_DECODE)
    assert fp4.fp4_get_device_status() == 7
    assert fp4.fp4_get_device_status() == 0   # cleared
    ws.zero_()
    fp4.fp4_gemm(fmt, A, sA, W, sW, M, N, K, None, D, ws, kernel=fp4.GEMM_DECODE)
    assert fp4.fp4_get_device_status() == 0


@pytest.mark.parametrize("M", [1, 16])
def test_dynamic_activation_then_decode_with_static_weights(orc, M):
    # the chain a decode step runs: the activation is quantized with its own
    # S_global (which also writes alpha) and the GEMM, launched right behind
    # it with the weights marked static, requests weight tiles before the
    # quantizer has finished; operands, scales and alpha of the activation
    # must still be the quantizer's output
    fmt, N, K = fp4.NVFP4, 38400, 2048   # 300 weight tiles: stream-K and whole tiles
    A = synth.normal_bf16(M, K, seed=44, outlier_factor=100.0)
    W = synth.normal_bf16(N, K, seed=44, tensor_id=1, sigma=0.02)
    gW = orc.global_scale(W)
    pW, sW = orc.quantize(fmt, 0, W, gs=gW)
    Wd, sWd = to_dev_u8(pW), to_dev_u8(sW)
    Ad = to_dev_bf16(A)
    pA = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
    sA = torch.empty((fp4.fp4_scale_bytes(fmt, M, K),), dtype=torch.uint8, device="cuda")
    gA = torch.empty(1, dtype=torch.float32, device="cuda")
    alpha = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = torch.zeros((fp4.fp4_gemm_workspace_bytes(fmt, M, N, K),), dtype=torch.uint8, device="cuda")
    D = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    for _ in range(3):   # repeated back to back: each pair reads the previous pair's buffers
        pA.fill_(0xFF)
        fp4.fp4_quantize_dynamic(Ad, pA, sA, gA, to_dev_f32(gW), alpha)
        fp4.fp4_gemm(fmt, pA, sA, Wd, sWd, M, N, K, alpha, D, ws,
                     kernel=fp4.GEMM_DECODE | fp4.GEMM_B_STATIC)
    torch.cuda.synchronize()
    assert fp4.fp4_get_device_status() == 0
    g = orc.global_scale(A)
    qA, sqA = orc.quantize(fmt, 0, A, gs=g)
    D_orc, S = orc.gemm(fmt, qA, sqA, pW, sW, alpha=float(np.float32(g) * np.float32(gW)))
    assert_gemm_close(bf16_dev_to_f64(D), D_orc, S, "dynamic + decode, static weights")


def test_k_zero_and_empty():
    A = torch.empty((4, 0), dtype=torch.uint8, device="cuda")
    B = torch.empty((8, 0), dtype=torch.uint8, device="cuda")
    s = torch.zeros((512,), dtype=torch.uint8, device="cuda")
    D = torch.full((4, 8), 7.0, dtype=torch.bfloat16, device="cuda")
    fp4.fp4_gemm(fp4.NVFP4, A, s, B, s, 4, 8, 0, None, D)
    torch.cuda.synchronize()
    assert torch.all(D.float() == 0)
    fp4.fp4_gemm(fp4.NVFP4, A, s, B, s, 0, 8, 64, None, D)   # M == 0: no-op


def test_invalid_arguments_launch_nothing():
    d = torch.zeros((1024,), dtype=torch.uint8, device="cuda")
    D = torch.zeros((16, 16), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fp4.Fp4Error) as e:
        fp4.fp4_gemm(fp4.NVFP4, d, d, d, d, 16, 16, 96, None, D)   # K % 64
    assert e.value.status == 2
    with pytest.raises(fp4.Fp4Error) as e:
        fp4.fp4_gemm(fp4.MXFP4, d, d, d, d, 16, 16, 64, None, D)   # K % 128
    assert e.value.status == 2
    with pytest.raises(fp4.Fp4Error) as e:
        fp4.fp4_gemm(fp4.NVFP4, d[1:], d, d, d, 16, 16, 64, None, D)   # misaligned
    assert e.value.status == 3
    with pytest.raises(fp4.Fp4Error) as e:
        fp4.fp4_gemm(fp4.NVFP4, d, d, d, d, 32, 16, 64, None, D, kernel=fp4.GEMM_DECODE)
    assert e.value.status in (1, 2)


@pytest.mark.parametrize("fmt", FMTS)
def test_end_to_end_gpu_quantize_then_gemm(orc, fmt):
    A = synth.normal_bf16(333, 1024, seed=33, outlier_factor=50.0)
    B = synth.normal_bf16(264, 1024, seed=33, tensor_id=1)
    Ad, Bd = to_dev_bf16(A), to_dev_bf16(B)
    if fmt != fp4.MXFP4:
        gA, gB = fp4.global_scale(Ad), fp4.global_scale(Bd)
        alpha = torch.empty(1, dtype=torch.float32, device="cuda")
        fp4.fp4_alpha_from_global_scales(gA, gB, alpha)
    else:
        gA = gB = alpha = None
    pA, sA = fp4.quantize(Ad, fmt, fp4.ROWWISE, gA)
    pB, sB = fp4.quantize(Bd, fmt, fp4.ROWWISE, gB)
    D = fp4.gemm(fmt, pA, sA, pB, sB, 1024, alpha=alpha)
    torch.cuda.synchronize()
    pAo, sAo, pBo, sBo, alpha_o = oracle_operands(orc, fmt, A, B)
    D_orc, S = orc.gemm(fmt, pAo, sAo, pBo, sBo, alpha=alpha_o)
    assert_gemm_close(bf16_dev_to_f64(D), D_orc, S, "e2e")


# --------------------------------------------------------------------------
# full-size configurations, oracle on sampled output elements
# --------------------------------------------------------------------------
def sampled_check(orc, fmt, A_bits, B_bits, kernel, n_pairs=4096):
    M, K = A_bits.shape
    N = B_bits.shape[0]
    Ad, Bd = to_dev_bf16(A_bits), to_dev_bf16(B_bits)
    gsA = orc.global_scale(A_bits) if fmt != fp4.MXFP4 else 1.0
    gsB = orc.global_scale(B_bits) if fmt != fp4.MXFP4 else 1.0
    pA, sA = fp4.quantize(Ad, fmt, fp4.ROWWISE, to_dev_f32(gsA) if fmt != fp4.MXFP4 else None)
    pB, sB = fp4.quantize(Bd, fmt, fp4.ROWWISE, to_dev_f32(gsB) if fmt != fp4.MXFP4 else None)
    alpha = float(np.float32(gsA) * np.float32(gsB))
    D = fp4.gemm(fmt, pA, sA, pB, sB, K, alpha=to_dev_f32(alpha), kernel=kernel)
    torch.cuda.synchronize()
    assert fp4.fp4_get_device_status() == 0
    rng = np.random.default_rng(34)
    ms = np.concatenate([rng.integers(0, M, n_pairs), [0, M - 1, M - 1, 0]])
    ns = np.concatenate([rng.integers(0, N, n_pairs), [0, N - 1, 0, N - 1]])
    # oracle operands from the oracle's own quantizer, on the sampled rows only
    um, inv_m = np.unique(ms, return_inverse=True)
    un, inv_n = np.unique(ns, return_inverse=True)
    qA, sqA = orc.quantize(fmt, 0, np.ascontiguousarray(A_bits[um]), gs=gsA)
    qB, sqB = orc.quantize(fmt, 0, np.ascontiguousarray(B_bits[un]), gs=gsB)
    D_orc, S = orc.gemm_pairs(fmt, qA, sqA, qB, sqB, inv_m, inv_n, alpha=alpha)
    D_gpu = bf16_dev_to_f64(D)[ms, ns]
    assert_gemm_close(D_gpu, D_orc, S, "sampled")


@pytest.mark.parametrize("fmt", FMTS)
def test_square_4096_sampled(orc, fmt):
    # 256 tiles over 74 CTA pairs: the 34 tiles of the last wave run as 68
    # half tiles (256 x 128)
    A, B = synth.square(4096)
    sampled_check(orc, fmt, A, B, fp4.GEMM_PREFILL)


@pytest.mark.parametrize("fmt", FMTS)
def test_prefill_tail_halves_ragged(orc, fmt):
    # 8 x 11 = 88 tiles with both edges ragged (M = 2000, N = 2600): the 14
    # tiles of the last wave are split into column halves, the last of them
    # only 40 columns wide; the samples cover every output row and column
    # range, the split tiles included
    M, N, K = 2000, 2600, 1024
    A = synth.normal_bf16(M, K, seed=71, outlier_factor=100.0)
    B = synth.normal_bf16(N, K, seed=71, tensor_id=1, sigma=0.02)
    sampled_check(orc, fmt, A, B, fp4.GEMM_PREFILL, n_pairs=8192)


@pytest.mark.parametrize("M", [1, 4, 16])
def test_decode_config_sampled(orc, M):
    W = synth.decode_weight()
    A = synth.decode_activation(M)
    sampled_check(orc, fp4.NVFP4, A, W, fp4.GEMM_DECODE, n_pairs=2048)


@pytest.mark.parametrize("shape", [(8192, 28672, 8192), (8192, 8192, 28672)])
def test_prefill_config_sampled(orc, shape):
    M, N, K = shape
    A, W = synth.prefill(M, N, K)
    sampled_check(orc, fp4.NVFP4, A, W, fp4.GEMM_PREFILL, n_pairs=1024)


@pytest.mark.parametrize("fmt", FMTS)
def test_grouped_gemm_matches_oracle_per_problem(orc, fmt):
    # experts of an MoE layer: one weight shape, token counts from 0 to a few
    # hundred, plus one problem of another shape and one with K = 0; 18
    # problems, so the call makes two launches (16 + 2)
    rng = np.random.default_rng(36)
    K, N = 1024, 512
    shapes = [(int(m), N, K) for m in rng.integers(0, 300, 15)] + [(0, N, K), (40, 264, 640), (5, 136, 0)]
    items, checks = [], []
    for i, (M, Ni, Ki) in enumerate(shapes):
        if Ki and Ki % (128 if fmt == fp4.MXFP4 else 64):
            Ki = 768
        Ms = max(M, 1)
        A = synth.normal_bf16(Ms, max(Ki, 128), seed=37 + i, outlier_factor=50.0)[:M, :Ki]
        W = synth.normal_bf16(Ni, max(Ki, 128), seed=37 + i, tensor_id=1, sigma=0.02)[:, :Ki]
        D = torch.full((M, Ni + 8), float("nan"), dtype=torch.bfloat16, device="cuda")
        if M > 0 and Ki > 0:
            pA, sA, pW, sW, alpha = oracle_operands(orc, fmt, np.ascontiguousarray(A), np.ascontiguousarray(W))
            items.append((to_dev_u8(pA), to_dev_u8(sA), to_dev_u8(pW), to_dev_u8(sW), Ki, to_dev_f32(alpha),
                          D[:, :Ni]))
            checks.append((D, Ni, orc.gemm(fmt, pA, sA, pW, sW, alpha=alpha)))
        else:
            z = torch.zeros((64,), dtype=torch.uint8, device="cuda")
            items.append((z, z, z, z, Ki, None, D[:, :Ni]))
            checks.append((D, Ni, None))
    fp4.fp4_gemm_grouped(fmt, items)
    torch.cuda.synchronize()
    assert fp4.fp4_get_device_status() == 0
    for (M, Ni, Ki), (D, n_cols, want) in zip(shapes, checks):
        assert torch.isnan(D[:, n_cols:].float()).all()
        if M == 0:
            continue
        if want is None:   # K == 0
            assert torch.all(D[:, :n_cols].float() == 0)
            continue
        D_orc, S = want
        assert_gemm_close(bf16_dev_to_f64(D[:, :n_cols]), D_orc, S, "grouped %s" % ((M, Ni, Ki),))
