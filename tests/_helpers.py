"""Shared test helpers: tolerance checks, host<->device marshalling, canaries.

The tolerance is the one the layer's numerics are held to (fp32 accumulation
on the GPU against the oracle's fp64 sums, both rounded once to BF16):
elementwise |y - y_ref| <= 2^-7 |y_ref| + 1e-3 max|y_ref| and normwise
||y - y_ref|| / ||y_ref|| <= 4e-3.
"""
from __future__ import annotations

import numpy as np
import torch

ELEM_REL = 2.0 ** -7
ELEM_ABS_OF_MAX = 1e-3
NORM_REL = 4e-3
SENTINEL = 0x7FC1  # a NaN pattern no kernel writes


def bits_to_f64(bits) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def assert_close(y_bits, ref_bits, what="", elementwise=True):
    """GEMV/GEMM tolerance: elementwise and normwise, against the oracle's BF16
    output.  elementwise=False keeps only the normwise bound (used where the
    reference is a different, coarser definition, e.g. an unfused chain that
    rounds an intermediate the fused kernel keeps in fp32)."""
    y = bits_to_f64(y_bits).ravel()
    r = bits_to_f64(ref_bits).ravel()
    assert y.shape == r.shape
    assert np.all(np.isfinite(y)), f"{what}: non-finite outputs"
    if r.size == 0:
        return
    mx = np.abs(r).max()
    bound = ELEM_REL * np.abs(r) + ELEM_ABS_OF_MAX * mx
    err = np.abs(y - r)
    bad = np.nonzero(err > bound)[0] if elementwise else np.zeros(0, dtype=np.int64)
    assert bad.size == 0, (f"{what}: {bad.size} elements outside tolerance; first at {bad[0]}: "
                           f"got {y[bad[0]]!r} want {r[bad[0]]!r} (bound {bound[bad[0]]:.3g})")
    nr = np.linalg.norm(r)
    if nr > 0:
        rel = np.linalg.norm(y - r) / nr
        assert rel <= NORM_REL, f"{what}: normwise relative error {rel:.3g} > {NORM_REL}"


def dev(a: np.ndarray) -> torch.Tensor:
    """numpy array (uint32 / uint16 bit patterns) -> CUDA tensor with the same bytes."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint32:
        t = torch.from_numpy(a.view(np.int32))
    elif a.dtype == np.uint16:
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(a)
    return t.cuda()


def host_bits(t: torch.Tensor) -> np.ndarray:
    """CUDA bf16 tensor -> uint16 bit patterns on the host."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


class Guarded:
    """A BF16 output buffer with sentinel guard bands on both sides."""

    def __init__(self, n: int, pad: int = 64, offset_elems: int = 0):
        self.n, self.pad = n, pad
        self.buf = torch.full((n + 2 * pad + offset_elems,), 0, dtype=torch.int16, device="cuda")
        self.buf.fill_(np.int16(np.uint16(SENTINEL).view(np.int16)))
        self.start = pad + offset_elems
        self.view = self.buf[self.start:self.start + n].view(torch.bfloat16)

    def data_ptr(self) -> int:
        return self.view.data_ptr()

    def value_bits(self) -> np.ndarray:
        return host_bits(self.view)

    def check_guards(self):
        h = self.buf.cpu().numpy().view(np.uint16)
        assert np.all(h[:self.start] == SENTINEL), "write before the output buffer"
        assert np.all(h[self.start + self.n:] == SENTINEL), "write past the output buffer"
