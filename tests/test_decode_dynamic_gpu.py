"""GPU parity of the decode GEMM that quantizes its activation inside the
kernel (fp4_gemm_decode_dynamic): S_global and alpha exactly as the oracle
forms them, D bit for bit equal to the two-step path (fp4_quantize_dynamic,
then the decode kernel on the packed activation) and within the GEMM
tolerance of the oracle's FP64 product of its own quantization."""
import numpy as np
import pytest
import torch

from block_scaled_fp4_05_b200 import fp4, synth
from gpu_util import assert_gemm_close, bf16_dev_to_f64, to_dev_bf16

pytestmark = pytest.mark.gpu


def run_case(orc, M, N, K, seed, lda_pad=0, n_pairs=None):
    A = synth.normal_bf16(M, K, seed=seed, tensor_id=100 + M, outlier_factor=100.0)
    W = synth.decode_weight(N, K) if seed == 2 else synth.normal_bf16(N, K, seed=seed, tensor_id=1, sigma=0.02)
    if lda_pad:
        big = np.zeros((M, K + lda_pad), dtype=np.uint16)
        big[:, :K] = A
        Ad = to_dev_bf16(big)[:, :K]
    else:
        Ad = to_dev_bf16(A)
    Wd = to_dev_bf16(W)
    gW = fp4.global_scale(Wd)
    pW, sW = fp4.quantize(Wd, fp4.NVFP4, fp4.ROWWISE, gW)
    ws = torch.zeros((fp4.fp4_gemm_workspace_bytes(fp4.NVFP4, M, N, K),), dtype=torch.uint8, device="cuda")
    D = torch.full((M, N + 8), float("nan"), dtype=torch.bfloat16, device="cuda")
    gA = torch.empty(1, dtype=torch.float32, device="cuda")
    al = torch.empty(1, dtype=torch.float32, device="cuda")
    fp4.fp4_gemm_decode_dynamic(Ad, pW, sW, gW, D[:, :N], gA, al, ws)
    # the two-step path on the same inputs
    pA, sA = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda"), \
        torch.empty((fp4.fp4_scale_bytes(fp4.NVFP4, M, K),), dtype=torch.uint8, device="cuda")
    gA2 = torch.empty(1, dtype=torch.float32, device="cuda")
    al2 = torch.empty(1, dtype=torch.float32, device="cuda")
    fp4.fp4_quantize_dynamic(Ad, pA, sA, gA2, gW, al2)
    D2 = fp4.gemm(fp4.NVFP4, pA, sA, pW, sW, K, alpha=al2, kernel=fp4.GEMM_DECODE, workspace=ws)
    torch.cuda.synchronize()
    assert fp4.fp4_get_device_status() == 0
    assert torch.isnan(D[:, N:].float()).all()
    g = np.float32(orc.global_scale(A))
    gw = np.float32(gW.item())
    assert np.float32(gA.item()) == g
    assert np.float32(al.item()) == g * gw
    d, d2 = bf16_dev_to_f64(D[:, :N]), bf16_dev_to_f64(D2)
    assert np.array_equal(d, d2), "in-kernel quantization differs from the two-step path"
    qA, qsA = orc.quantize(orc.NVFP4, orc.ROWWISE, A, gs=float(g))
    if n_pairs is None:
        qW, qsW = orc.quantize(orc.NVFP4, orc.ROWWISE, W, gs=float(gw))
        D_orc, S = orc.gemm(orc.NVFP4, qA, qsA, qW, qsW, alpha=float(g * gw))
        assert_gemm_close(d, D_orc, S, "decode dynamic %s" % ((M, N, K),))
    else:
        rng = np.random.default_rng(seed)
        ns = np.unique(np.concatenate([rng.integers(0, N, n_pairs), [0, N - 1]]))
        qW, qsW = orc.quantize(orc.NVFP4, orc.ROWWISE, np.ascontiguousarray(W[ns]), gs=float(gw))
        ms_i = np.repeat(np.arange(M), len(ns))
        ns_i = np.tile(np.arange(len(ns)), M)
        D_orc, S = orc.gemm_pairs(orc.NVFP4, qA, qsA, qW, qsW, ms_i, ns_i, alpha=float(g * gw))
        assert_gemm_close(d[ms_i, ns[ns_i]], D_orc, S, "decode dynamic sampled %s" % ((M, N, K),))


@pytest.mark.parametrize("MNK", [(1, 2048, 4096), (4, 1536, 2048), (16, 2048, 4096), (3, 1152, 1088),
                                 (16, 38400, 1088), (7, 640, 64)])
def test_decode_dynamic_matches_two_step_and_oracle(orc, MNK):
    # (16, 38400, 1088): more weight tiles than SMs (stream-K then whole
    # tiles) and a one-MMA K tail; (7, 640, 64): a single partial stage
    run_case(orc, *MNK, seed=61)


def test_decode_dynamic_strided_activation(orc):
    run_case(orc, 5, 1024, 2048, seed=62, lda_pad=64)


@pytest.mark.parametrize("M", [1, 16])
def test_decode_dynamic_full_size_sampled(orc, M):
    # the decode configuration: W 28672 x 8192, activation M x 8192
    run_case(orc, M, 28672, 8192, seed=2, n_pairs=512)
