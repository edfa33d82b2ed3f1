"""CPU oracle for the 8-bit group-affine quantized linear layer (MlxInt8Weight page).

TEST INFRASTRUCTURE ONLY: the plain, slow, single-threaded reference the CUDA
library is checked against.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  It shares no
code with ``weight_only_quantized_mlx_b200`` and never imports it.

All arithmetic lives in ``mlxq_oracle.cpp``; this module only marshals numpy
arrays.  BF16 values travel as ``uint16`` bit patterns.  Shapes:

* ``packed``  uint32 ``[N, K/4]`` (byte j of word w is column 4w+j)
* ``scales``, ``biases``  uint16 (BF16 bits) ``[N, K/gs]``
* activations uint16 (BF16 bits) ``[K]`` or ``[m, K]``
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build as _build

_SIGS = None


def _signatures():
    u32p = ctypes.POINTER(ctypes.c_uint32)
    u16p = ctypes.POINTER(ctypes.c_uint16)
    u8p = ctypes.POINTER(ctypes.c_uint8)
    f32p = ctypes.POINTER(ctypes.c_float)
    f64p = ctypes.POINTER(ctypes.c_double)
    i64 = ctypes.c_int64
    W = [u32p, u16p, u16p, i64, i64, i64]
    return {
        "oracle_bf16_from_f32": (ctypes.c_uint16, [ctypes.c_float]),
        "oracle_bf16_from_f64": (ctypes.c_uint16, [ctypes.c_double]),
        "oracle_f16_from_f32": (ctypes.c_uint16, [ctypes.c_float]),
        "oracle_f32_from_bf16": (ctypes.c_float, [ctypes.c_uint16]),
        "oracle_silu": (ctypes.c_double, [ctypes.c_double]),
        "oracle_unpack": (None, [u32p, i64, i64, u8p]),
        "oracle_dequant_f32": (None, W + [f32p]),
        "oracle_dequant": (None, W + [u16p]),
        "oracle_dequant_f16": (None, W + [u16p]),
        "oracle_gemv_f64": (None, W + [u16p, f64p]),
        "oracle_gemv": (None, W + [u16p, u16p]),
        "oracle_silu_gate_f64": (None, W + [u16p, u16p, f64p]),
        "oracle_silu_gate": (None, W + [u16p, u16p, u16p]),
        "oracle_silu_gate_resid_f64": (None, W + [u16p, u16p, u16p, f64p]),
        "oracle_silu_gate_resid": (None, W + [u16p, u16p, u16p, u16p]),
        "oracle_silu_mul": (None, [u16p, u16p, i64, u16p]),
        "oracle_gemm_f64": (None, W + [u16p, i64, f64p]),
        "oracle_gemm": (None, W + [u16p, i64, u16p]),
        "oracle_quantize": (None, [u16p, i64, i64, i64, u32p, u16p, u16p]),
    }


def _p(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _vec(a, n, what):
    a = np.ascontiguousarray(a, dtype=np.uint16)
    if a.size != n:
        raise ValueError(f"{what} must hold {n} BF16 values")
    return a


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen BF16 bit patterns to float64 (exact: bits << 16 is the fp32 pattern)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


class Oracle:
    """numpy front end over one build of the oracle library.

    The default instance uses ``oracle/libmlxq_oracle.so``; the oracle's own
    tests also open deliberately broken builds through this class to show that
    the pins catch each planted mistake.
    """

    def __init__(self, path: str):
        L = ctypes.CDLL(path)
        for name, (res, args) in _signatures().items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        self.L = L
        self.path = path

    # ---- helpers -------------------------------------------------------------
    @staticmethod
    def _weight(packed, scales, biases, gs):
        packed = np.ascontiguousarray(packed, dtype=np.uint32)
        scales = np.ascontiguousarray(scales, dtype=np.uint16)
        biases = np.ascontiguousarray(biases, dtype=np.uint16)
        if packed.ndim != 2:
            raise ValueError("packed must be [N, K/4]")
        N, K = packed.shape[0], packed.shape[1] * 4
        if gs <= 0 or K % gs:
            raise ValueError("group_size must divide in_features")
        G = K // gs
        if scales.shape != (N, G) or biases.shape != (N, G):
            raise ValueError("scales/biases must be [N, K/gs]")
        args = [_p(packed, ctypes.c_uint32), _p(scales, ctypes.c_uint16),
                _p(biases, ctypes.c_uint16), N, K, gs]
        return args, (packed, scales, biases), N, K

    # ---- scalars ---------------------------------------------------------------
    def bf16_from_f32(self, v: float) -> int:
        return int(self.L.oracle_bf16_from_f32(float(v)))

    def bf16_from_f64(self, v: float) -> int:
        return int(self.L.oracle_bf16_from_f64(float(v)))

    def f32_from_bf16(self, h: int) -> float:
        return float(self.L.oracle_f32_from_bf16(int(h)))

    def silu(self, t: float) -> float:
        return float(self.L.oracle_silu(float(t)))

    def f64_to_bf16_array(self, v: np.ndarray) -> np.ndarray:
        """Round an fp64 array to BF16 bits, one rounding per element."""
        f = self.L.oracle_bf16_from_f64
        flat = np.ascontiguousarray(v, dtype=np.float64).ravel()
        out = np.fromiter((f(float(t)) for t in flat), dtype=np.uint16, count=flat.size)
        return out.reshape(np.shape(v))

    # ---- arrays ----------------------------------------------------------------
    def unpack(self, packed: np.ndarray) -> np.ndarray:
        packed = np.ascontiguousarray(packed, dtype=np.uint32)
        N, K = packed.shape[0], packed.shape[1] * 4
        q = np.empty((N, K), np.uint8)
        self.L.oracle_unpack(_p(packed, ctypes.c_uint32), N, K, _p(q, ctypes.c_uint8))
        return q

    def dequant_f32(self, packed, scales, biases, gs) -> np.ndarray:
        args, keep, N, K = self._weight(packed, scales, biases, gs)
        w = np.empty((N, K), np.float32)
        self.L.oracle_dequant_f32(*args, _p(w, ctypes.c_float))
        return w

    def quantize(self, w_bits, gs):
        """BF16 W [N, K] (bit patterns) -> (packed uint32 [N, K/4], scales,
        biases uint16 [N, K/gs]) by per-group min/max affine codes."""
        w = np.ascontiguousarray(w_bits, dtype=np.uint16)
        N, K = w.shape
        if gs <= 0 or K % gs or K % 4 or gs % 4:
            raise ValueError("quantize needs gs | K and 4 | gs")
        packed = np.empty((N, K // 4), np.uint32)
        scales = np.empty((N, K // gs), np.uint16)
        biases = np.empty((N, K // gs), np.uint16)
        self.L.oracle_quantize(_p(w, ctypes.c_uint16), N, K, gs, _p(packed, ctypes.c_uint32),
                               _p(scales, ctypes.c_uint16), _p(biases, ctypes.c_uint16))
        return packed, scales, biases

    def dequant_f16(self, packed, scales, biases, gs) -> np.ndarray:
        """FP16 bit patterns of fma_f32(s, q, b) rounded to nearest even, [N, K]."""
        args, keep, N, K = self._weight(packed, scales, biases, gs)
        w = np.empty((N, K), np.uint16)
        self.L.oracle_dequant_f16(*args, _p(w, ctypes.c_uint16))
        return w

    def f16_from_f32(self, v: float) -> int:
        return int(self.L.oracle_f16_from_f32(float(v)))

    def dequant(self, packed, scales, biases, gs) -> np.ndarray:
        """BF16 bit patterns of the dequantised weight, [N, K] row-major."""
        args, keep, N, K = self._weight(packed, scales, biases, gs)
        w = np.empty((N, K), np.uint16)
        self.L.oracle_dequant(*args, _p(w, ctypes.c_uint16))
        return w

    def gemv_f64(self, packed, scales, biases, gs, x) -> np.ndarray:
        args, keep, N, K = self._weight(packed, scales, biases, gs)
        x = _vec(x, K, "x")
        y = np.empty(N, np.float64)
        self.L.oracle_gemv_f64(*args, _p(x, ctypes.c_uint16), _p(y, ctypes.c_double))
        return y

    def gemv(self, packed, scales, biases, gs, x) -> np.ndarray:
        args, keep, N, K = self._weight(packed, scales, biases, gs)
        x = _vec(x, K, "x")
        y = np.empty(N, np.uint16)
        self.L.oracle_gemv(*args, _p(x, ctypes.c_uint16), _p(y, ctypes.c_uint16))
        return y

    def silu_gate_f64(self, packed, scales, biases, gs, gate, up) -> np.ndarray:
        args, keep, N, K = self._weight(packed, scales, biases, gs)
        gate, up = _vec(gate, K, "gate"), _vec(up, K, "up")
        y = np.empty(N, np.float64)
        self.L.oracle_silu_gate_f64(*args, _p(gate, ctypes.c_uint16),
                                    _p(up, ctypes.c_uint16), _p(y, ctypes.c_double))
        return y

    def silu_gate(self, packed, scales, biases, gs, gate, up) -> np.ndarray:
        args, keep, N, K = self._weight(packed, scales, biases, gs)
        gate, up = _vec(gate, K, "gate"), _vec(up, K, "up")
        y = np.empty(N, np.uint16)
        self.L.oracle_silu_gate(*args, _p(gate, ctypes.c_uint16),
                                _p(up, ctypes.c_uint16), _p(y, ctypes.c_uint16))
        return y

    def silu_gate_resid_f64(self, packed, scales, biases, gs, gate, up, x_resid) -> np.ndarray:
        args, keep, N, K = self._weight(packed, scales, biases, gs)
        gate, up = _vec(gate, K, "gate"), _vec(up, K, "up")
        r = _vec(x_resid, N, "x_resid")
        y = np.empty(N, np.float64)
        self.L.oracle_silu_gate_resid_f64(*args, _p(gate, ctypes.c_uint16),
                                          _p(up, ctypes.c_uint16), _p(r, ctypes.c_uint16),
                                          _p(y, ctypes.c_double))
        return y

    def silu_gate_resid(self, packed, scales, biases, gs, gate, up, x_resid) -> np.ndarray:
        args, keep, N, K = self._weight(packed, scales, biases, gs)
        gate, up = _vec(gate, K, "gate"), _vec(up, K, "up")
        r = _vec(x_resid, N, "x_resid")
        y = np.empty(N, np.uint16)
        self.L.oracle_silu_gate_resid(*args, _p(gate, ctypes.c_uint16),
                                      _p(up, ctypes.c_uint16), _p(r, ctypes.c_uint16),
                                      _p(y, ctypes.c_uint16))
        return y

    def silu_mul(self, gate, up) -> np.ndarray:
        """bf16(silu(gate) * up): the materialised intermediate of the unfused chain."""
        gate = np.ascontiguousarray(gate, dtype=np.uint16)
        up = _vec(up, gate.size, "up")
        h = np.empty(gate.size, np.uint16)
        self.L.oracle_silu_mul(_p(gate, ctypes.c_uint16), _p(up, ctypes.c_uint16),
                               gate.size, _p(h, ctypes.c_uint16))
        return h

    def gemm_f64(self, packed, scales, biases, gs, X) -> np.ndarray:
        args, keep, N, K = self._weight(packed, scales, biases, gs)
        X = np.ascontiguousarray(X, dtype=np.uint16)
        if X.ndim != 2 or X.shape[1] != K:
            raise ValueError("X must be [m, K]")
        m = X.shape[0]
        Y = np.empty((m, N), np.float64)
        self.L.oracle_gemm_f64(*args, _p(X, ctypes.c_uint16), m, _p(Y, ctypes.c_double))
        return Y

    def gemm(self, packed, scales, biases, gs, X) -> np.ndarray:
        args, keep, N, K = self._weight(packed, scales, biases, gs)
        X = np.ascontiguousarray(X, dtype=np.uint16)
        if X.ndim != 2 or X.shape[1] != K:
            raise ValueError("X must be [m, K]")
        m = X.shape[0]
        Y = np.empty((m, N), np.uint16)
        self.L.oracle_gemm(*args, _p(X, ctypes.c_uint16), m, _p(Y, ctypes.c_uint16))
        return Y


_default = None


def default() -> Oracle:
    """The oracle built from oracle/mlxq_oracle.cpp (compiled on first use)."""
    global _default
    if _default is None:
        _default = Oracle(_build.build())
    return _default


def __getattr__(name):
    # Module-level access (oracle.gemv(...)) goes to the default build.
    if name.startswith("_"):
        raise AttributeError(name)
    return getattr(default(), name)
