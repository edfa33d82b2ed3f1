"""Python binding of libmlxq.so, the B200 (sm_100a) library for the 8-bit
group-affine quantized linear layer of the "MlxInt8Weight" API page.

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  The functions carry the C names of ``include/mlxq.h``; buffers may be
given as torch tensors (their ``data_ptr()`` is passed) or as raw integer
device addresses, streams as ``torch.cuda.Stream`` objects, raw integers or
``None`` (torch's current stream).  A nonzero status raises :class:`MlxqError`.

There is no CPU fallback: importing the binding without the built library
raises ``ImportError`` (build it with ``python -m
weight_only_quantized_mlx_b200.build``).
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmlxq.so")

MLXQ_OK = 0
MLXQ_ERR_INVALID_ARG = 1
MLXQ_ERR_PARSE = 2
MLXQ_ERR_MISSING_TENSOR = 3
MLXQ_ERR_DTYPE = 4
MLXQ_ERR_SHAPE = 5
MLXQ_ERR_GROUP_SIZE = 6
MLXQ_ERR_UNSUPPORTED = 7
MLXQ_ERR_CUDA = 8
MLXQ_ERR_DEVICE_TIMEOUT = 9

MLXQ_GEMM_AUTO = 0
MLXQ_GEMM_ROWS = 1
MLXQ_GEMM_SMALLM = 2
MLXQ_GEMM_TCGEN05 = 3
MLXQ_GEMM_SMALLM_FFMA = 4
MLXQ_GEMM_SMALLM_GROUPS = 5
MLXQ_GEMM_SMALLM_TC = 6

MLXQ_WEIGHT_STATIC = 1

MLXQ_DTYPE_BF16 = 0
MLXQ_DTYPE_F16 = 1
MLXQ_DTYPE_F32 = 2

EXPORTS = ("mlxq_load", "mlxq_dequant", "mlxq_gemv", "mlxq_gemv_silu_gate",
           "mlxq_gemv_silu_gate_resid", "mlxq_gemm", "mlxq_gemm_with", "mlxq_gemm_noalloc", "mlxq_release",
           "mlxq_last_error", "mlxq_device_status", "mlxq_dequant_as", "mlxq_quantize", "mlxq_selftest_wait_timeout",
           "mlxq_selftest_fail_alloc")


class mlxq_weight(ctypes.Structure):
    """C ``mlxq_weight``: three device pointers and the dimensions."""
    _fields_ = [("packed", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("biases", ctypes.c_void_p), ("out_features", ctypes.c_uint32),
                ("in_features", ctypes.c_uint32), ("group_size", ctypes.c_uint32),
                ("flags", ctypes.c_uint32)]


class MlxqError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"mlxq error {code}: {message}")
        self.code = code


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is not built; run python -m weight_only_quantized_mlx_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        W = ctypes.POINTER(mlxq_weight)
        vp, u64, u32, i32 = ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int
        sigs = {
            "mlxq_load": [ctypes.c_char_p, ctypes.c_size_t, ctypes.c_char_p, u32, W],
            "mlxq_dequant": [W, vp, u64],
            "mlxq_gemv": [W, vp, vp, u64],
            "mlxq_gemv_silu_gate": [W, vp, vp, vp, u64],
            "mlxq_gemv_silu_gate_resid": [W, vp, vp, vp, vp, u64],
            "mlxq_gemm": [W, vp, vp, u32, u64],
            "mlxq_gemm_with": [W, vp, vp, u32, i32, u64],
            "mlxq_gemm_noalloc": [W, vp, vp, u32, u64],
            "mlxq_release": [W],
            "mlxq_last_error": [],
            "mlxq_device_status": [],
            "mlxq_quantize": [vp, W, u64],
            "mlxq_dequant_as": [W, vp, i32, u64],
            "mlxq_selftest_wait_timeout": [u32, u64],
            "mlxq_selftest_fail_alloc": [u32],
        }
        for name, args in sigs.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_char_p if name == "mlxq_last_error" else ctypes.c_int
        _lib = L
    return _lib


def _ptr(b):
    if b is None:
        return None
    if isinstance(b, int):
        return b
    return b.data_ptr()


def _stream(s) -> int:
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else 0
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(rc: int) -> None:
    if rc != MLXQ_OK:
        raise MlxqError(rc, mlxq_last_error())


def mlxq_last_error() -> str:
    return lib().mlxq_last_error().decode(errors="replace")


def mlxq_load(blob: bytes, base: str, group_size: int) -> mlxq_weight:
    w = mlxq_weight()
    _check(lib().mlxq_load(blob, len(blob), base.encode(), group_size, ctypes.byref(w)))
    return w


def mlxq_release(w: mlxq_weight) -> None:
    _check(lib().mlxq_release(ctypes.byref(w)))


def mlxq_dequant(w: mlxq_weight, out, stream=None) -> None:
    _check(lib().mlxq_dequant(ctypes.byref(w), _ptr(out), _stream(stream)))


def mlxq_gemv(w: mlxq_weight, x, y, stream=None) -> None:
    _check(lib().mlxq_gemv(ctypes.byref(w), _ptr(x), _ptr(y), _stream(stream)))


def mlxq_gemv_silu_gate(w: mlxq_weight, gate, up, y, stream=None) -> None:
    _check(lib().mlxq_gemv_silu_gate(ctypes.byref(w), _ptr(gate), _ptr(up), _ptr(y), _stream(stream)))


def mlxq_gemv_silu_gate_resid(w: mlxq_weight, gate, up, x_resid, y, stream=None) -> None:
    _check(lib().mlxq_gemv_silu_gate_resid(ctypes.byref(w), _ptr(gate), _ptr(up), _ptr(x_resid),
                                           _ptr(y), _stream(stream)))


def mlxq_gemm(w: mlxq_weight, x, y, m: int, stream=None) -> None:
    _check(lib().mlxq_gemm(ctypes.byref(w), _ptr(x), _ptr(y), m, _stream(stream)))


def mlxq_gemm_with(w: mlxq_weight, x, y, m: int, kernel: int, stream=None) -> None:
    _check(lib().mlxq_gemm_with(ctypes.byref(w), _ptr(x), _ptr(y), m, kernel, _stream(stream)))


def mlxq_gemm_noalloc(w: mlxq_weight, x, y, m: int, stream=None) -> None:
    _check(lib().mlxq_gemm_noalloc(ctypes.byref(w), _ptr(x), _ptr(y), m, _stream(stream)))


MLXQ_STATIC_SCRATCH_BYTES = 40 << 20


def mlxq_device_status() -> None:
    _check(lib().mlxq_device_status())


def mlxq_dequant_as(w: mlxq_weight, out, dtype: int, stream=None) -> None:
    _check(lib().mlxq_dequant_as(ctypes.byref(w), _ptr(out), dtype, _stream(stream)))


def mlxq_quantize(w_bf16, dst: mlxq_weight, stream=None) -> None:
    _check(lib().mlxq_quantize(_ptr(w_bf16), ctypes.byref(dst), _stream(stream)))


def mlxq_selftest_wait_timeout(limit_us: int, stream=None) -> None:
    _check(lib().mlxq_selftest_wait_timeout(limit_us, _stream(stream)))


def mlxq_selftest_fail_alloc(nth: int) -> None:
    _check(lib().mlxq_selftest_fail_alloc(nth))


def weight_view(packed, scales, biases, group_size: int, flags: int = 0) -> mlxq_weight:
    """A non-owning handle over caller-owned device tensors (packed uint32/int32
    [N, K/4], scales/biases bf16 [N, K/gs]).  Never pass it to mlxq_release."""
    N = packed.shape[0]
    K = packed.shape[1] * 4
    return mlxq_weight(_ptr(packed), _ptr(scales), _ptr(biases), N, K, group_size, flags)


class MlxInt8Weight:
    """The page's struct as a Python object: ``load`` / ``dequantize_to`` /
    ``gemv`` / ``gemv_silu_gate`` / ``gemv_silu_gate_resid`` / ``gemm`` /
    ``release``, each one call into the C ABI."""

    def __init__(self, handle: mlxq_weight, owned: bool):
        self.handle = handle
        self.owned = owned

    @classmethod
    def load(cls, blob: bytes, base: str, group_size: int, static: bool = False) -> "MlxInt8Weight":
        """static=True sets MLXQ_WEIGHT_STATIC (see include/mlxq.h): the caller
        promises that no kernel writes the weight while calls read it."""
        w = cls(mlxq_load(blob, base, group_size), True)
        if static:
            w.handle.flags |= MLXQ_WEIGHT_STATIC
        return w

    @property
    def out_features(self) -> int:
        return self.handle.out_features

    @property
    def in_features(self) -> int:
        return self.handle.in_features

    @property
    def group_size(self) -> int:
        return self.handle.group_size

    def dequantize_to(self, out, stream=None):
        mlxq_dequant(self.handle, out, stream)

    def gemv(self, x, y, stream=None):
        mlxq_gemv(self.handle, x, y, stream)

    def gemv_silu_gate(self, gate, up, y, stream=None):
        mlxq_gemv_silu_gate(self.handle, gate, up, y, stream)

    def gemv_silu_gate_resid(self, gate, up, x_resid, y, stream=None):
        mlxq_gemv_silu_gate_resid(self.handle, gate, up, x_resid, y, stream)

    def gemm(self, x, y, m: int, stream=None):
        mlxq_gemm(self.handle, x, y, m, stream)

    def release(self):
        if not self.owned:
            raise MlxqError(MLXQ_ERR_INVALID_ARG, "this handle does not own its buffers")
        mlxq_release(self.handle)
