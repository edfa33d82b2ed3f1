"""Seeded synthetic inputs for the 8-bit group-affine quantized linear layer.

The one module that both the CUDA path's tests/benchmark and the oracle's
checks draw inputs from.  It holds none of the layer's arithmetic: no
unpacking, no dequantisation, no products.  It only draws random numbers and
stores them in the weight's storage format:

* ``packed``: uint32 ``[N, K/4]``.  The codes q are i.i.d. uniform on 0..255;
  they are drawn directly as uniform 32-bit words, which is the same thing as
  four independent uniform bytes per word.
* ``scales``: BF16 ``[N, K/gs]`` = bf16(U(0.5, 1.5) * 2^-8).
* ``biases``: BF16 ``[N, K/gs]`` = bf16(-128 * scale + N(0, 1) * 2^-10), i.e.
  centred on the middle code so that W has mean close to zero.
* activations (x, gate, up, x_resid, X): bf16(N(0, 1)).

The weights and activations of the API page's workloads are those of a
language model's projections; no dataset or checkpoint is involved.  Draw
order from ``numpy.random.Generator(PCG64(seed))`` is fixed: packed words,
then scales, then bias noise, then activations.  BF16 rounding of the drawn
floats uses torch's float32 -> bfloat16 conversion (round to nearest even).
BF16 values are returned as uint16 bit patterns.
"""
from __future__ import annotations

import numpy as np
import torch


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float array -> BF16 bit patterns (uint16), via torch's RNE conversion."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Inverse storage view: BF16 bit patterns -> float32 values (exact)."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def weight(g: np.random.Generator, N: int, K: int, gs: int):
    """One synthetic quantized weight: (packed u32 [N,K/4], scales, biases u16 [N,K/gs])."""
    if K % 4 or gs <= 0 or K % gs:
        raise ValueError("need K % 4 == 0 and group_size | K")
    G = K // gs
    packed = g.integers(0, 1 << 32, size=(N, K // 4), dtype=np.uint32)
    scales = to_bf16_bits(g.uniform(0.5, 1.5, size=(N, G)) * 2.0 ** -8)
    s = bf16_bits_to_f32(scales).astype(np.float64)
    biases = to_bf16_bits(-128.0 * s + g.standard_normal(size=(N, G)) * 2.0 ** -10)
    return packed, scales, biases


def activations(g: np.random.Generator, *shape: int) -> np.ndarray:
    """BF16 bits of N(0, 1) draws."""
    return to_bf16_bits(g.standard_normal(size=shape))


def decode_pair(seed: int, N: int, K: int, gs: int):
    """(packed, scales, biases, x) of one seeded gemv problem."""
    g = rng(seed)
    packed, scales, biases = weight(g, N, K, gs)
    return packed, scales, biases, activations(g, K)


def safetensors_blob(tensors: dict) -> bytes:
    """Serialise {name: (dtype_str, shape, bytes)} in the safetensors layout:
    u64 little-endian header length, JSON header, then the raw data."""
    import json
    header, chunks, off = {}, [], 0
    for name, (dtype, shape, data) in tensors.items():
        header[name] = {"dtype": dtype, "shape": list(shape), "data_offsets": [off, off + len(data)]}
        chunks.append(data)
        off += len(data)
    h = json.dumps(header, separators=(",", ":")).encode()
    h += b" " * (-len(h) % 8)
    return len(h).to_bytes(8, "little") + h + b"".join(chunks)


def weight_blob(base: str, packed: np.ndarray, scales: np.ndarray, biases: np.ndarray) -> bytes:
    """A safetensors blob holding ``{base}.weight`` (U32), ``.scales``, ``.biases`` (BF16)."""
    return safetensors_blob({
        f"{base}.weight": ("U32", packed.shape, np.ascontiguousarray(packed, np.uint32).tobytes()),
        f"{base}.scales": ("BF16", scales.shape, np.ascontiguousarray(scales, np.uint16).tobytes()),
        f"{base}.biases": ("BF16", biases.shape, np.ascontiguousarray(biases, np.uint16).tobytes()),
    })
