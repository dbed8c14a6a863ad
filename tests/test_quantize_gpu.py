"""GPU parity of the quantizer kernels against the oracle: packed nibbles and
scale bytes must be identical, output guard bands untouched, scale padding
zero.  Runs the kernels through the C ABI (ctypes binding)."""
import numpy as np
import pytest
import torch

from block_scaled_fp4_05_b200 import fp4, synth
from gpu_util import Guarded, to_dev_bf16, to_dev_f32

pytestmark = pytest.mark.gpu

FMTS = [fp4.NVFP4, fp4.MXFP4, fp4.P1E8]   # P1E8: 16-element blocks, E8M0 scale under S_global


def gpu_quantize(fmt, axis, x_bits, gs):
    rows, cols = x_bits.shape
    out_rows, K = (rows, cols) if axis == fp4.ROWWISE else (cols, rows)
    x = to_dev_bf16(x_bits)
    packed = Guarded(out_rows * K // 2)
    scales = Guarded(fp4.fp4_scale_bytes(fmt, out_rows, K), fill=0x5A)
    gsd = to_dev_f32(gs) if fmt != fp4.MXFP4 else None
    fp4.fp4_quantize(fmt, axis, x, packed.view, scales.view, gsd)
    torch.cuda.synchronize()
    assert fp4.fp4_get_device_status() == 0
    assert packed.guards_intact() and scales.guards_intact()
    return packed.view.cpu().numpy().reshape(out_rows, K // 2), scales.view.cpu().numpy()


def check(orc, fmt, axis, x_bits, gs=None):
    if gs is None:
        gs = orc.global_scale(x_bits) if fmt != fp4.MXFP4 else 1.0
    p_gpu, s_gpu = gpu_quantize(fmt, axis, x_bits, gs)
    p_orc, s_orc = orc.quantize(fmt, axis, x_bits, gs=gs)
    bad = np.argwhere(p_gpu != p_orc)
    assert bad.size == 0, ("packed mismatch", bad[:4].tolist(), p_gpu[tuple(bad[0])], p_orc[tuple(bad[0])])
    bad = np.nonzero(s_gpu != s_orc)[0]
    assert bad.size == 0, ("scale mismatch", bad[:4].tolist(), s_gpu[bad[:4]], s_orc[bad[:4]])


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("axis", [fp4.ROWWISE, fp4.COLWISE])
def test_tiny_config(orc, fmt, axis):
    A, B = synth.tiny_nv()
    check(orc, fmt, axis, A)
    check(orc, fmt, axis, B)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("shape", [(1, 512), (3, 256), (129, 384), (200, 1024), (517, 2048),
                                   (33, 320), (130, 64)])   # NVFP4 only: a 64-column last tile
def test_rowwise_ragged_rows(orc, fmt, shape):
    if shape[1] % (4 * fp4.block_size(fmt)):
        pytest.skip("length not a multiple of 4 blocks")
    x = synth.normal_bf16(*shape, seed=21, outlier_factor=60.0, zero_frac=0.05)
    check(orc, fmt, fp4.ROWWISE, x)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("shape", [(128, 8), (256, 24), (384, 136), (512, 1000)])
def test_colwise_ragged_cols(orc, fmt, shape):
    if shape[0] % (4 * fp4.block_size(fmt)):
        pytest.skip("length not a multiple of 4 blocks")
    x = synth.normal_bf16(*shape, seed=22, outlier_factor=60.0, zero_frac=0.05)
    check(orc, fmt, fp4.COLWISE, x)


@pytest.mark.parametrize("fmt", FMTS)
def test_all_zero_and_signed_zero(orc, fmt):
    x = np.zeros((130, 256), dtype=np.uint16)
    x[1::2, 5::3] = 0x8000  # -0.0
    check(orc, fmt, fp4.ROWWISE, x, gs=1.0)
    check(orc, fmt, fp4.COLWISE, np.zeros((256, 136), dtype=np.uint16), gs=1.0)


@pytest.mark.parametrize("fmt", FMTS)
def test_rounding_ties_and_extremes(orc, fmt):
    # blocks whose elements land exactly on the E2M1 decision points, plus
    # the largest and smallest BF16 magnitudes and subnormals
    rng = np.random.default_rng(23)
    k = fp4.block_size(fmt)
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 0.5, 1.0, 3.0, 4.0], dtype=np.float32)
    rows = []
    for e in range(-20, 21):
        S = np.float32(2.0 ** e)
        vals = np.resize(np.concatenate([ties, -ties]), k) * S
        vals[0] = 6.0 * S   # amax = 6 S gives exponent e (MX)
        rows.append(vals)
    x = np.array(rows * 4, dtype=np.float32)
    x = np.concatenate([x] * (128 // k), axis=1) if k == 16 else np.concatenate([x] * 4, axis=1)
    xb = synth.f32_to_bf16_bits(x)
    extremes = np.array([0x7F7F, 0xFF7F, 0x0001, 0x8001, 0x0080, 0x007F, 0x3F80, 0xBF80],
                        dtype=np.uint16)
    xb[0, :8] = extremes
    xb[1, :k] = rng.integers(1, 0x80, k).astype(np.uint16)  # subnormal block
    check(orc, fmt, fp4.ROWWISE, xb, gs=1.0 if fmt == fp4.MXFP4 else 0.0625)
    check(orc, fmt, fp4.ROWWISE, xb)


@pytest.mark.parametrize("fmt", [fp4.NVFP4, fp4.P1E8])
def test_custom_global_scales(orc, fmt):
    # includes S_global so small that the effective block scale underflows
    # to zero (all codes +-0) and so large that every ratio is tiny
    x = synth.normal_bf16(256, 512, seed=24, outlier_factor=100.0)
    for gs in [1.0, 2.0 ** -12, 0.0371, 1000.0, 1e-38, 3e38]:
        check(orc, fmt, fp4.ROWWISE, x, gs=gs)
        check(orc, fmt, fp4.COLWISE, x, gs=gs)


@pytest.mark.parametrize("shape", [(1, 8), (128, 512), (333, 4104), (4096, 4096)])
def test_global_scale_matches_oracle(orc, shape):
    x = synth.normal_bf16(*shape, seed=25, outlier_factor=50.0)
    gs = fp4.global_scale(to_dev_bf16(x))
    torch.cuda.synchronize()
    assert np.float32(gs.item()) == np.float32(orc.global_scale(x))
    z = fp4.global_scale(torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda"))
    assert z.item() == 1.0


def test_global_scale_with_leading_dimension(orc):
    x = synth.normal_bf16(100, 256, seed=26, outlier_factor=10.0)
    big = np.zeros((100, 512), dtype=np.uint16)
    big[:, :256] = x
    big[3, 300] = synth.f32_to_bf16_bits(np.array([1e6], dtype=np.float32))[0]  # outside the view
    d = to_dev_bf16(big)
    gs = fp4.global_scale(d[:, :256])
    torch.cuda.synchronize()
    assert np.float32(gs.item()) == np.float32(orc.global_scale(x))


def test_global_scale_alpha_one_launch(orc):
    # S_global and alpha = S_global * other from one launch, on a strided view
    x = synth.normal_bf16(100, 256, seed=29, outlier_factor=30.0)
    big = np.zeros((100, 264), dtype=np.uint16)
    big[:, :256] = x
    d = to_dev_bf16(big)
    gs = torch.empty(1, dtype=torch.float32, device="cuda")
    al = torch.empty(1, dtype=torch.float32, device="cuda")
    other = to_dev_f32(0.0371)
    fp4.fp4_compute_global_scale_alpha(d[:, :256], gs, other, al)
    torch.cuda.synchronize()
    g = orc.global_scale(x)
    assert np.float32(gs.item()) == np.float32(g)
    assert np.float32(al.item()) == np.float32(g) * np.float32(0.0371)


@pytest.mark.parametrize("shapes", [((100, 256, 264), (64, 512, 512)), ((4096, 4096, 4096), (4096, 4096, 4096)),
                                    ((0, 64, 64), (33, 72, 80)), ((2048, 8192, 8192), (1, 8, 8))])
def test_global_scales_pair_one_launch(orc, shapes):
    # both operands' S_global and alpha from one launch, identical to the
    # single-tensor calls and to the oracle; strided views, an empty tensor
    # (S_global = 1) and tensors of very different sizes
    (ra, ca, la), (rb, cb, lb) = shapes
    xa = synth.normal_bf16(ra, ca, seed=31, outlier_factor=30.0) if ra else np.zeros((0, ca), np.uint16)
    xb = synth.normal_bf16(rb, cb, seed=31, tensor_id=1, outlier_factor=7.0)
    da, db = [to_dev_bf16(np.pad(x, ((0, 0), (0, l - x.shape[1])))) for x, l in ((xa, la), (xb, lb))]
    out = torch.zeros(3, dtype=torch.float32, device="cuda")
    fp4.fp4_compute_global_scales_pair(da[:, :ca], db[:, :cb], out[0:1], out[1:2], out[2:3])
    torch.cuda.synchronize()
    ga = np.float32(orc.global_scale(xa)) if ra else np.float32(1.0)
    gb = np.float32(orc.global_scale(xb))
    got = out.cpu().numpy()
    assert got[0] == ga and got[1] == gb and got[2] == ga * gb
    one = torch.empty(1, dtype=torch.float32, device="cuda")
    fp4.fp4_compute_global_scale(db[:, :cb], one)
    torch.cuda.synchronize()
    assert one.item() == got[1]


def test_global_scale_slot_ring_wraps(orc):
    # more calls than reduction slots, alternating two tensors: every call
    # leaves its slot zeroed, so the second use of each slot is exact again
    xs = [synth.normal_bf16(64, 512, seed=30, tensor_id=t, outlier_factor=20.0) for t in range(2)]
    want = [np.float32(orc.global_scale(x)) for x in xs]
    ds = [to_dev_bf16(x) for x in xs]
    out = torch.empty(1100, dtype=torch.float32, device="cuda")
    for i in range(1100):
        fp4.fp4_compute_global_scale(ds[i % 2], out[i:i + 1])
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    assert np.all(got[0::2] == want[0]) and np.all(got[1::2] == want[1])


def test_alpha_from_global_scales():
    a, b = to_dev_f32(0.0123), to_dev_f32(3.7)
    out = torch.empty(1, dtype=torch.float32, device="cuda")
    fp4.fp4_alpha_from_global_scales(a, b, out)
    torch.cuda.synchronize()
    assert np.float32(out.item()) == np.float32(0.0123) * np.float32(3.7)


# --------------------------------------------------------------------------
# full-size sweep tensors (16384 x 16384 and 8192 x 28672): GPU output on
# the whole tensor, oracle on a sample of output rows
# --------------------------------------------------------------------------
def sampled_rows_check(orc, fmt, axis, x_bits, n_rows=48):
    rows, cols = x_bits.shape
    gs = orc.global_scale(x_bits) if fmt != fp4.MXFP4 else 1.0
    x = to_dev_bf16(x_bits)
    packed, scales = fp4.quantize(x, fmt, axis, to_dev_f32(gs) if fmt != fp4.MXFP4 else None)
    torch.cuda.synchronize()
    assert fp4.fp4_get_device_status() == 0
    out_rows, K = (rows, cols) if axis == fp4.ROWWISE else (cols, rows)
    rng = np.random.default_rng(27)
    pick = np.unique(np.concatenate([[0, out_rows - 1], rng.integers(0, out_rows, n_rows)]))
    if axis == fp4.ROWWISE:
        sub = np.ascontiguousarray(x_bits[pick, :])
        p_orc, _, rm = orc.quantize(fmt, fp4.ROWWISE, sub, gs=gs, with_rowmajor_scales=True)
    else:
        sub = np.ascontiguousarray(x_bits[:, pick])
        p_orc, _, rm = orc.quantize(fmt, fp4.COLWISE, sub, gs=gs, with_rowmajor_scales=True)
    p_gpu = packed[torch.from_numpy(pick).cuda()].cpu().numpy()
    assert np.array_equal(p_gpu, p_orc)
    s_all = scales.cpu().numpy()
    nsc = K // fp4.block_size(fmt)
    cols_idx = np.arange(nsc)
    for i, r in enumerate(pick):
        offs = [orc.scale_offset(int(r), int(c), nsc) for c in cols_idx]
        assert np.array_equal(s_all[offs], rm[i])
    return gs


@pytest.mark.parametrize("fmt", [fp4.NVFP4, fp4.MXFP4])
@pytest.mark.parametrize("axis", [fp4.ROWWISE, fp4.COLWISE])
@pytest.mark.parametrize("shape", [(16384, 16384), (8192, 28672)])
def test_full_size_sweep_sampled(orc, fmt, axis, shape):
    x = synth.quant_sweep(*shape)
    sampled_rows_check(orc, fmt, axis, x)


@pytest.mark.parametrize("axis", [fp4.ROWWISE, fp4.COLWISE])
def test_full_size_sweep_sampled_p1e8(orc, axis):
    x = synth.quant_sweep(16384, 16384)
    sampled_rows_check(orc, fp4.P1E8, axis, x)


@pytest.mark.parametrize("shape", [(1, 8192), (4, 8192), (16, 8192), (16, 512), (3, 64), (1, 64),
                                   (200, 1024), (33, 8192), (300, 1024), (2048, 8192), (1000, 4160),
                                   (8192, 8192)])
def test_dynamic_quantize_matches_oracle(orc, shape):
    # one call: S_global, quantization with it, alpha = S_global * other; small tensors
    # take the single-launch cluster kernel, (33, 8192) and larger the two-launch path
    # (S_global + alpha, then the quantizer over the tiles in reverse order)
    x = synth.normal_bf16(*shape, seed=28, outlier_factor=100.0)
    rows, cols = shape
    xd = to_dev_bf16(x)
    packed = Guarded(rows * cols // 2)
    scales = Guarded(fp4.fp4_scale_bytes(fp4.NVFP4, rows, cols), fill=0x5A)
    gs = torch.empty(1, dtype=torch.float32, device="cuda")
    other = to_dev_f32(0.0123)
    alpha = torch.empty(1, dtype=torch.float32, device="cuda")
    fp4.fp4_quantize_dynamic(xd, packed.view, scales.view, gs, other, alpha)
    torch.cuda.synchronize()
    assert fp4.fp4_get_device_status() == 0
    assert packed.guards_intact() and scales.guards_intact()
    g = orc.global_scale(x)
    assert np.float32(gs.item()) == np.float32(g)
    assert np.float32(alpha.item()) == np.float32(g) * np.float32(0.0123)
    p_orc, s_orc = orc.quantize(fp4.NVFP4, fp4.ROWWISE, x, gs=g)
    assert np.array_equal(packed.view.cpu().numpy().reshape(rows, cols // 2), p_orc)
    assert np.array_equal(scales.view.cpu().numpy(), s_orc)


def _dynamic_check(orc, x, ld=None):
    rows, cols = x.shape
    if ld is None:
        xd = to_dev_bf16(x)
    else:   # a strided view: the rows of a wider matrix
        wide = np.zeros((rows, ld), dtype=np.uint16)
        wide[:, :cols] = x
        xd = to_dev_bf16(wide)[:, :cols]
    p = torch.empty((rows, cols // 2), dtype=torch.uint8, device="cuda")
    s = torch.empty((fp4.fp4_scale_bytes(fp4.NVFP4, rows, cols),), dtype=torch.uint8, device="cuda")
    gs = torch.empty(1, dtype=torch.float32, device="cuda")
    fp4.fp4_quantize_dynamic(xd, p, s, gs)
    torch.cuda.synchronize()
    assert fp4.fp4_get_device_status() == 0
    g = orc.global_scale(x)
    assert np.float32(gs.item()) == np.float32(g)
    p_orc, s_orc = orc.quantize(fp4.NVFP4, fp4.ROWWISE, x, gs=g)
    assert np.array_equal(p.cpu().numpy(), p_orc)
    assert np.array_equal(s.cpu().numpy(), s_orc)


@pytest.mark.parametrize("where", ["first", "middle", "last"])
def test_dynamic_quantize_large_amax_anywhere(orc, where):
    # the tensor's amax in one element of the first, a middle or the last tile:
    # every thread block's maximum must reach the reduction slot before the
    # last one forms S_global
    rows, cols = 1111, 2048
    x = synth.normal_bf16(rows, cols, seed=29)
    r, c = {"first": (0, 3), "middle": (555, 1030), "last": (rows - 1, cols - 1)}[where]
    x[r, c] = 0x4A80   # 4194304.0, far above the rest
    _dynamic_check(orc, x)


def test_dynamic_quantize_large_strided_and_zero(orc):
    x = synth.normal_bf16(700, 3072, seed=30, outlier_factor=50.0, zero_frac=0.1)
    _dynamic_check(orc, x, ld=3200)
    z = np.zeros((512, 4096), dtype=np.uint16)
    _dynamic_check(orc, z)   # amax 0: S_global 1, every code and scale 0


def test_dynamic_quantize_slot_ring_wraps(orc):
    # more calls than the 1024 reduction slots, two tensors alternating: each
    # call's S_global must be its own tensor's (a slot left dirty by the
    # previous use would carry the other tensor's amax or arrivals)
    rows, cols = 160, 8192   # above the single-cluster capacity: the S_global kernel's slots
    xa = synth.normal_bf16(rows, cols, seed=31, outlier_factor=100.0)
    xb = synth.normal_bf16(rows, cols, seed=32, sigma=0.01)
    xs = [to_dev_bf16(xa), to_dev_bf16(xb)]
    n = 1100
    p = torch.empty((rows, cols // 2), dtype=torch.uint8, device="cuda")
    s = torch.empty((fp4.fp4_scale_bytes(fp4.NVFP4, rows, cols),), dtype=torch.uint8, device="cuda")
    gs = torch.empty(n, dtype=torch.float32, device="cuda")
    for i in range(n):
        fp4.fp4_quantize_dynamic(xs[i % 2], p, s, gs[i:i + 1])
    torch.cuda.synchronize()
    assert fp4.fp4_get_device_status() == 0
    ga, gb = np.float32(orc.global_scale(xa)), np.float32(orc.global_scale(xb))
    got = gs.cpu().numpy()
    assert np.array_equal(got[0::2], np.full(n // 2, ga)) and np.array_equal(got[1::2], np.full(n // 2, gb))
    p_orc, s_orc = orc.quantize(fp4.NVFP4, fp4.ROWWISE, xb, gs=float(gb))
    assert np.array_equal(p.cpu().numpy(), p_orc) and np.array_equal(s.cpu().numpy(), s_orc)


def test_dynamic_quantize_all_zero_and_rejects_mx():
    x = torch.zeros((4, 128), dtype=torch.bfloat16, device="cuda")
    p = torch.empty((4, 64), dtype=torch.uint8, device="cuda")
    s = torch.empty((fp4.fp4_scale_bytes(fp4.NVFP4, 4, 128),), dtype=torch.uint8, device="cuda")
    gs = torch.empty(1, dtype=torch.float32, device="cuda")
    fp4.fp4_quantize_dynamic(x, p, s, gs)
    torch.cuda.synchronize()
    assert gs.item() == 1.0 and int(p.sum().item()) == 0
    import ctypes
    st = fp4.lib().fp4_quantize_dynamic(fp4.MXFP4, ctypes.c_void_p(x.data_ptr()), 4, 128, 128,
                                        ctypes.c_void_p(p.data_ptr()), ctypes.c_void_p(s.data_ptr()),
                                        ctypes.c_void_p(gs.data_ptr()), None, None, None)
    assert st == 1


@pytest.mark.parametrize("fmt", FMTS)
def test_batch_matches_oracle_per_tensor(orc, fmt):
    # ten tensors in one call (more than one launch's eight), ragged row
    # counts, one empty; each must equal its own fp4_quantize result
    shapes = [(517, 2048), (1, 512), (128, 256), (0, 256), (200, 1024), (3, 128), (129, 384),
              (64, 4096), (1000, 128), (7, 640)]
    items, expect = [], []
    for i, (r, c) in enumerate(shapes):
        x = synth.normal_bf16(max(r, 1), c, seed=50 + i, outlier_factor=60.0, zero_frac=0.02)[:r]
        gs = orc.global_scale(x) if (fmt != fp4.MXFP4 and r > 0) else 1.0
        packed = Guarded(max(1, r * c // 2))
        scales = Guarded(max(1, fp4.fp4_scale_bytes(fmt, r, c)), fill=0x5A)
        xd = to_dev_bf16(x) if r > 0 else torch.empty((0, c), dtype=torch.bfloat16, device="cuda")
        items.append((xd, packed.view, scales.view, to_dev_f32(gs) if fmt != fp4.MXFP4 else None))
        expect.append((x, gs, packed, scales))
    fp4.fp4_quantize_batch(fmt, items)
    torch.cuda.synchronize()
    assert fp4.fp4_get_device_status() == 0
    for (r, c), (x, gs, packed, scales) in zip(shapes, expect):
        assert packed.guards_intact() and scales.guards_intact()
        if r == 0:
            continue
        p_orc, s_orc = orc.quantize(fmt, fp4.ROWWISE, x, gs=gs)
        assert np.array_equal(packed.view.cpu().numpy().reshape(r, c // 2), p_orc), (r, c)
        assert np.array_equal(scales.view.cpu().numpy(), s_orc), (r, c)
