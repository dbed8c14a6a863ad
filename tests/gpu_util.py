"""Helpers shared by the GPU parity tests: host<->device transfer of BF16 bit
arrays, guard-banded output buffers and the GEMM acceptance check."""
import numpy as np
import torch

GUARD = 4096
GUARD_BYTE = 0xA5


def to_dev_bf16(bits):
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.cuda()


def to_dev_u8(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def to_dev_f32(x):
    return torch.tensor([float(np.float32(x))], dtype=torch.float32, device="cuda")


class Guarded:
    """A uint8 device buffer of `n` bytes with GUARD bytes of 0xA5 on each
    side; `view` is 256-byte aligned."""

    def __init__(self, n, fill=GUARD_BYTE):
        self.n = n
        self.raw = torch.full((n + 2 * GUARD + 256,), GUARD_BYTE, dtype=torch.uint8, device="cuda")
        off = (-self.raw.data_ptr()) % 256
        self.lo = off + GUARD
        self.view = self.raw[self.lo:self.lo + n]
        if fill != GUARD_BYTE:
            self.view.fill_(fill)

    def guards_intact(self):
        r = self.raw.cpu().numpy()
        return bool(np.all(r[:self.lo] == GUARD_BYTE) and np.all(r[self.lo + self.n:] == GUARD_BYTE))


def bf16_dev_to_f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def gemm_tolerance(D_oracle, S):
    """|D - D_oracle| <= 1e-3 * S + 2^-8 * |D_oracle| + 1e-6: the accuracy
    bound of the FP32 block-scaled accumulation (1e-3 of the sum of absolute
    products) plus half an ulp of the BF16 output rounding."""
    return 1e-3 * S + 2.0 ** -8 * np.abs(D_oracle) + 1e-6


def assert_gemm_close(D_gpu, D_oracle, S, what=""):
    tol = gemm_tolerance(D_oracle, S)
    err = np.abs(D_gpu - D_oracle)
    bad = np.argwhere(err > tol)
    assert bad.size == 0, "%s: %d/%d outside tolerance, first %s: gpu %r oracle %r tol %r" % (
        what, len(bad), err.size, bad[:3].tolist(),
        D_gpu[tuple(bad[0])] if bad.size else None,
        D_oracle[tuple(bad[0])] if bad.size else None,
        tol[tuple(bad[0])] if bad.size else None)
