"""Pins for the CPU oracle (no GPU).

Each ``pin_*`` function checks the oracle against something other than
itself: hand-derived golden values, closed forms, exact-integer cases, an
independently written dense brute force, and identities the MlxInt8Weight
page's definitions imply.  ``test_planted_mistakes`` then compiles copies of
the oracle with one deliberate mistake each and checks that some pin fails,
so a plausible slip (byte order, group index, dropped bias, silu sign, a
transposed output, a dropped residual, ties rounding away, double rounding)
cannot pass unnoticed.
"""
from __future__ import annotations

import math
import os
import shutil
import subprocess
import tempfile

import numpy as np
import pytest
import torch

import oracle
from oracle import Oracle, bf16_bits_to_f64
from oracle import build as oracle_build

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = os.path.join(HERE, "golden")


# ---------------------------------------------------------------------------
# independent helpers (written here, not shared with the oracle)
# ---------------------------------------------------------------------------
def pack_le(q: np.ndarray) -> np.ndarray:
    """uint8 [N, K] codes -> uint32 [N, K/4] words, byte j of a word = column 4w+j."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    N, K = q.shape
    return q.reshape(N, K // 4, 4).copy().view("<u4").reshape(N, K // 4).astype(np.uint32)


def unpack_by_bits(packed: np.ndarray) -> np.ndarray:
    """Second, deliberately naive unpack: assemble each code bit by bit."""
    N, W = packed.shape
    q = np.zeros((N, W * 4), np.int64)
    for k in range(W * 4):
        word = packed[:, k // 4].astype(np.int64)
        for b in range(8):
            q[:, k] |= ((word >> (8 * (k % 4) + b)) & 1) << b
    return q


def bf16_torch(a) -> np.ndarray:
    """float -> BF16 bits via torch (library RNE)."""
    t = torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def f32_bits(v) -> np.ndarray:
    return np.asarray(v, dtype=np.float32).view(np.uint32)


def dense_weight(packed, scales, biases, gs) -> np.ndarray:
    """Independent dense W (float64 of the BF16 values).  s*q is exact in
    float32 (8-bit by 8-bit significands), so float32 s*q + b rounds once,
    like a fused multiply-add."""
    q = unpack_by_bits(packed).astype(np.float32)
    N, K = q.shape
    g = np.arange(K) // gs
    s = bf16_bits_to_f64(scales).astype(np.float32)[:, g]
    b = bf16_bits_to_f64(biases).astype(np.float32)[:, g]
    w32 = (s * q).astype(np.float32) + b
    return bf16_bits_to_f64(bf16_torch(w32))


def read_kv(path):
    out = {}
    for line in open(path):
        line = line.split("#", 1)[0].strip()
        if not line:
            continue
        k, v = line.split(":", 1)
        out[k.strip()] = v.split()
    return out


def rand_weight(g, N, K, gs):
    q = g.integers(0, 256, size=(N, K), dtype=np.uint8)
    G = K // gs
    scales = bf16_torch(g.uniform(0.5, 1.5, size=(N, G)) * 2.0 ** -8)
    biases = bf16_torch(-128 * bf16_bits_to_f64(scales) + g.standard_normal((N, G)) * 2.0 ** -10)
    return pack_le(q), scales, biases, q


# ---------------------------------------------------------------------------
# pins (each takes an Oracle and raises AssertionError on a mismatch)
# ---------------------------------------------------------------------------
def pin_bf16_f32_table(o: Oracle):
    for line in open(os.path.join(GOLDEN, "bf16_rne_f32.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        f_hex, b_hex = line.split()[:2]
        v = np.array([int(f_hex, 16)], np.uint32).view(np.float32)[0]
        got = o.bf16_from_f32(v)
        assert got == int(b_hex, 16), f"{f_hex}: got {got:04X}, want {b_hex}"


def pin_bf16_f64_table(o: Oracle):
    for line in open(os.path.join(GOLDEN, "bf16_rne_f64.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        parts = line.split()
        # value expression = everything before the 4-hex-digit column
        idx = next(i for i, p in enumerate(parts) if len(p) == 4 and all(c in "0123456789ABCDEF" for c in p))
        expr = " ".join(parts[:idx])
        v = float(eval(expr, {"__builtins__": {}}, {}))
        got = o.bf16_from_f64(v)
        assert got == int(parts[idx], 16), f"{expr}: got {got:04X}, want {parts[idx]}"


def pin_bf16_two_routes_agree(o: Oracle):
    # On values that are already fp32 the single-rounding fp64 route and the
    # bit-pattern fp32 route are two independent implementations of one rule.
    g = np.random.default_rng(7)
    vals = np.concatenate([
        g.standard_normal(3000).astype(np.float32),
        (g.standard_normal(1000) * 1e-39).astype(np.float32),   # subnormal range
        (g.standard_normal(1000) * 1e37).astype(np.float32),
        (np.float32(1.0) + np.arange(0, 2 ** 16, 37, dtype=np.float32) * np.float32(2.0 ** -23)),
    ])
    for v in vals:
        if not np.isfinite(v):
            continue
        assert o.bf16_from_f64(float(v)) == o.bf16_from_f32(v), v
    # and both agree with torch's conversion on ordinary values
    ref = bf16_torch(vals[:3000])
    got = np.array([o.bf16_from_f32(v) for v in vals[:3000]], np.uint16)
    assert np.array_equal(ref, got)


def pin_unpack_word(o: Oracle):
    q = o.unpack(np.array([[0x04030201, 0xFDFCFBFA]], np.uint32))
    assert q.tolist() == [[1, 2, 3, 4, 250, 251, 252, 253]]
    g = np.random.default_rng(1)
    codes = g.integers(0, 256, size=(5, 24), dtype=np.uint8)
    assert np.array_equal(o.unpack(pack_le(codes)), codes)
    assert np.array_equal(unpack_by_bits(pack_le(codes)), codes)


def pin_identity_scale(o: Oracle):
    # s = 1, b = 0: W is the code itself; integers 0..255 are exact in BF16.
    g = np.random.default_rng(2)
    q = g.integers(0, 256, size=(3, 32), dtype=np.uint8)
    ones = np.full((3, 32 // 8), 0x3F80, np.uint16)
    zeros = np.zeros((3, 32 // 8), np.uint16)
    w = o.dequant(pack_le(q), ones, zeros, 8)
    want = (f32_bits(q.astype(np.float32)) >> 16).astype(np.uint16)
    assert np.array_equal(w, want)
    assert np.array_equal(o.dequant_f32(pack_le(q), ones, zeros, 8), q.astype(np.float32))


def pin_centred_scale(o: Oracle):
    # s = 2^-e, b = -128 * 2^-e: W = (q - 128) * 2^-e exactly.
    g = np.random.default_rng(3)
    q = g.integers(0, 256, size=(2, 64), dtype=np.uint8)
    for e in (0, 3, 8, 20):
        s = bf16_torch(np.full((2, 4), 2.0 ** -e))
        b = bf16_torch(np.full((2, 4), -128 * 2.0 ** -e))
        w = bf16_bits_to_f64(o.dequant(pack_le(q), s, b, 16))
        assert np.array_equal(w, (q.astype(np.float64) - 128) * 2.0 ** -e), e


def pin_group_index(o: Oracle):
    # one distinct power of two per group: each column must use group k // gs
    g = np.random.default_rng(4)
    for K, gs in ((64, 4), (64, 8), (96, 32), (48, 12)):
        G = K // gs
        q = g.integers(0, 256, size=(3, K), dtype=np.uint8)
        ex = (np.arange(3)[:, None] + np.arange(G)[None, :]) % 9
        s = bf16_torch(2.0 ** -ex.astype(np.float64))
        b = np.zeros((3, G), np.uint16)
        w = bf16_bits_to_f64(o.dequant(pack_le(q), s, b, gs))
        want = q.astype(np.float64) * 2.0 ** -ex[:, np.arange(K) // gs]
        assert np.array_equal(w, want), (K, gs)


def pin_worked_example(o: Oracle):
    d = read_kv(os.path.join(GOLDEN, "worked_example.txt"))
    gs = int(d["group_size"][0])
    packed = np.array([int(h, 16) for h in d["packed"]], np.uint32).reshape(2, 2)
    scales = np.array([int(h, 16) for h in d["scales"]], np.uint16).reshape(2, 2)
    biases = np.array([int(h, 16) for h in d["biases"]], np.uint16).reshape(2, 2)
    x = np.array([int(h, 16) for h in d["x"]], np.uint16)
    w = np.array([int(h, 16) for h in d["w"]], np.uint16).reshape(2, 8)
    assert np.array_equal(o.dequant(packed, scales, biases, gs), w)
    assert o.gemv_f64(packed, scales, biases, gs, x).tolist() == [float(v) for v in d["y_exact"]]
    assert o.gemv(packed, scales, biases, gs, x).tolist() == [int(h, 16) for h in d["y"]]
    Y = o.gemm(packed, scales, biases, gs, np.stack([x, x]))
    assert Y.tolist() == [[int(h, 16) for h in d["y"]]] * 2


def pin_bruteforce(o: Oracle):
    g = np.random.default_rng(5)
    for N, K, gs, m in ((1, 4, 4, 1), (3, 8, 4, 2), (5, 16, 8, 3), (16, 16, 16, 4),
                        (7, 12, 2, 3), (2, 16, 1, 5)):
        packed, scales, biases, _ = rand_weight(g, N, K, gs)
        W = dense_weight(packed, scales, biases, gs)
        assert np.array_equal(bf16_bits_to_f64(o.dequant(packed, scales, biases, gs)), W)
        X = bf16_torch(g.standard_normal((m, K)))
        ref = bf16_bits_to_f64(X) @ W.T
        got = o.gemm_f64(packed, scales, biases, gs, X)
        assert got.shape == (m, N)
        assert np.allclose(got, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max()), (N, K, gs, m)
        gv = o.gemv_f64(packed, scales, biases, gs, X[0])
        assert np.allclose(gv, ref[0], rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def pin_integer_exact(o: Oracle):
    # s = 1, b = 0 and small integer x: every sum is an exact integer.
    g = np.random.default_rng(6)
    N, K = 9, 256
    q = g.integers(0, 256, size=(N, K), dtype=np.uint8)
    xi = g.integers(-4, 5, size=K)
    ones = np.full((N, K // 64), 0x3F80, np.uint16)
    zeros = np.zeros((N, K // 64), np.uint16)
    x = bf16_torch(xi.astype(np.float32))
    exact = q.astype(np.int64) @ xi
    y64 = o.gemv_f64(pack_le(q), ones, zeros, 64, x)
    assert np.array_equal(y64, exact.astype(np.float64))
    want = bf16_torch(exact.astype(np.float32))  # |exact| < 2^24: float32 holds it exactly
    assert np.array_equal(o.gemv(pack_le(q), ones, zeros, 64, x), want)


def pin_silu_closed_forms(o: Oracle):
    assert o.silu(0.0) == 0.0
    # t*sigma(t) with sigma(ln 3) = 3/4
    assert math.isclose(o.silu(math.log(3.0)), 0.75 * math.log(3.0), rel_tol=1e-15)
    # sigma(1) = e / (e + 1)
    assert math.isclose(o.silu(1.0), math.e / (math.e + 1.0), rel_tol=1e-15)
    # silu(t) - silu(-t) = t (since sigma(t) + sigma(-t) = 1)
    for t in (0.1, 0.5, 2.0, 7.25, 30.0):
        assert math.isclose(o.silu(t) - o.silu(-t), t, rel_tol=1e-14), t
    # tails: silu(t) -> t for large t, -> 0 from below for very negative t
    assert math.isclose(o.silu(50.0), 50.0, rel_tol=1e-15)
    assert -1e-18 < o.silu(-50.0) < 0.0


def pin_silu_gate_zero(o: Oracle):
    g = np.random.default_rng(8)
    N, K, gs = 6, 64, 32
    packed, scales, biases, _ = rand_weight(g, N, K, gs)
    zero = np.zeros(K, np.uint16)
    up = bf16_torch(g.standard_normal(K))
    r = bf16_torch(g.standard_normal(N))
    assert np.array_equal(o.silu_gate_f64(packed, scales, biases, gs, zero, up), np.zeros(N))
    assert np.array_equal(o.silu_gate(packed, scales, biases, gs, zero, up), np.zeros(N, np.uint16))
    assert np.array_equal(o.silu_gate_resid(packed, scales, biases, gs, zero, up, r), r)


def pin_silu_gate_structure(o: Oracle):
    g = np.random.default_rng(9)
    N, K, gs = 7, 64, 16
    packed, scales, biases, _ = rand_weight(g, N, K, gs)
    W = dense_weight(packed, scales, biases, gs)
    gate = bf16_torch(g.standard_normal(K) * 3)
    up = bf16_torch(g.standard_normal(K))
    r = bf16_torch(g.standard_normal(N) * 4)
    h = np.array([o.silu(v) for v in bf16_bits_to_f64(gate)]) * bf16_bits_to_f64(up)
    ref = W @ h
    y = o.silu_gate_f64(packed, scales, biases, gs, gate, up)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    # up = 1 reduces the gate to W silu(gate)
    one = bf16_torch(np.ones(K))
    h1 = np.array([o.silu(v) for v in bf16_bits_to_f64(gate)])
    y1 = o.silu_gate_f64(packed, scales, biases, gs, gate, one)
    assert np.allclose(y1, W @ h1, rtol=1e-12, atol=1e-12 * np.abs(W @ h1).max())
    # the residual is added once: resid - plain = x_resid (up to the last fp64 rounding)
    yr = o.silu_gate_resid_f64(packed, scales, biases, gs, gate, up, r)
    diff = yr - y
    tol = 4 * np.spacing(np.maximum(np.abs(yr), np.abs(y)))
    assert np.all(np.abs(diff - bf16_bits_to_f64(r)) <= tol)
    # the materialised intermediate is bf16(silu(gate)*up)
    assert np.array_equal(o.silu_mul(gate, up), bf16_torch(h))


def pin_gemm_rows_are_gemv(o: Oracle):
    g = np.random.default_rng(10)
    N, K, gs = 11, 96, 32
    packed, scales, biases, _ = rand_weight(g, N, K, gs)
    X = bf16_torch(g.standard_normal((4, K)))
    Y = o.gemm(packed, scales, biases, gs, X)
    for i in range(4):
        assert np.array_equal(Y[i], o.gemv(packed, scales, biases, gs, X[i]))


# ---- quantize (the inverse of the format; the pages give no algorithm, so
# these pins check invariants of the min/max affine reading) ----------------
def pin_quantize_grid_identity(o: Oracle):
    # Weights that already lie on a grid s = 2^-e, b = -128 s, with every group
    # holding both code 0 and code 255: the group range is exactly 255 s, so
    # quantize must give back s, b and every code exactly.
    g = np.random.default_rng(40)
    N, K, gs = 3, 96, 32
    q = g.integers(0, 256, size=(N, K), dtype=np.uint8)
    q[:, ::gs] = 0
    q[:, 1::gs] = 255
    for e in (2, 8, 14):
        s = bf16_torch(np.full((N, K // gs), 2.0 ** -e))
        b = bf16_torch(np.full((N, K // gs), -128 * 2.0 ** -e))
        w = o.dequant(pack_le(q), s, b, gs)
        p2, s2, b2 = o.quantize(w, gs)
        assert np.array_equal(s2, s) and np.array_equal(b2, b), e
        assert np.array_equal(p2, pack_le(q)), e


def pin_quantize_error_bound(o: Oracle):
    # Round trip of arbitrary BF16 weights: each code is the nearest grid
    # point, so |W' - W| <= s / 2, except at the top of a group whose BF16
    # scale was rounded down, where code 255 falls short of the group maximum
    # by hi - (b + 255 s); plus the BF16 rounding of W' (half an ulp, <= 2^-8 |W'|) and of
    # the stored bias.  The group minimum maps to code 0.
    g = np.random.default_rng(41)
    N, K, gs = 4, 256, 64
    w = bf16_torch(g.standard_normal((N, K)) * 0.05)
    p, s, b = o.quantize(w, gs)
    w2 = bf16_bits_to_f64(o.dequant(p, s, b, gs))
    wf = bf16_bits_to_f64(w)
    sf = np.repeat(bf16_bits_to_f64(s), gs, axis=1)
    bf = np.repeat(bf16_bits_to_f64(b), gs, axis=1)
    lo = np.repeat(wf.reshape(N, K // gs, gs).min(axis=2), gs, axis=1)
    hi = np.repeat(wf.reshape(N, K // gs, gs).max(axis=2), gs, axis=1)
    top = np.maximum(sf / 2, hi - (bf + 255 * sf))
    assert np.all(np.abs(w2 - wf) <= top + 2.0 ** -8 * np.abs(w2) + np.abs(bf - lo) + 1e-12)
    codes = o.unpack(p).reshape(N, K // gs, gs)
    assert np.all(codes[np.arange(N)[:, None], np.arange(K // gs)[None, :],
                        wf.reshape(N, K // gs, gs).argmin(axis=2)] == 0)


def pin_quantize_constant_group(o: Oracle):
    # A constant group has range 0: scale 0, bias = the value, codes 0, and
    # dequantisation returns the value exactly.
    w = bf16_torch(np.array([[0.375] * 16 + [-2.5] * 16]))
    p, s, b = o.quantize(w, 16)
    assert np.array_equal(s, np.zeros((1, 2), np.uint16))
    assert np.array_equal(bf16_bits_to_f64(b), np.array([[0.375, -2.5]]))
    assert np.array_equal(p, np.zeros((1, 8), np.uint32))
    assert np.array_equal(o.dequant(p, s, b, 16), w)


def pin_f16_f32_table(o: Oracle):
    for line in open(os.path.join(GOLDEN, "fp16_rne_f32.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        f_hex, h_hex = line.split()[:2]
        v = np.array([int(f_hex, 16)], np.uint32).view(np.float32)[0]
        got = o.f16_from_f32(v)
        assert got == int(h_hex, 16), f"{f_hex}: got {got:04X}, want {h_hex}"


def pin_f16_matches_ieee_conversion(o: Oracle):
    # The same rule, implemented independently by numpy's IEEE float32 ->
    # float16 conversion, on random values across the normal, subnormal,
    # overflow and tie ranges.
    g = np.random.default_rng(11)
    vals = np.concatenate([
        g.standard_normal(4000).astype(np.float32),
        (g.standard_normal(2000) * 2.0 ** -18).astype(np.float32),     # subnormal FP16 range
        (g.uniform(6.0e4, 7.0e4, 1000) * g.choice([-1, 1], 1000)).astype(np.float32),  # overflow edge
        ((g.integers(-2048, 2048, 2000) + 0.5) * 2.0 ** -10).astype(np.float32),      # exact ties
    ])
    with np.errstate(over="ignore"):
        want = vals.astype(np.float16).view(np.uint16)
    got = np.array([o.f16_from_f32(v) for v in vals], np.uint16)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"{bad.size} mismatches, first {vals[bad[0]]!r}: {got[bad[0]]:04X} vs {want[bad[0]]:04X}"


def pin_dequant_f16(o: Oracle):
    # s = 1, b = 0: codes 0..255 are exact in FP16.  s = 1, b = 2048: 2048 + q
    # needs 12 bits, so odd q rounds to even: 2049 -> 2048, 2051 -> 2052.
    q = np.arange(256, dtype=np.uint8).reshape(1, 256)
    ones = np.full((1, 4), 0x3F80, np.uint16)
    w = o.dequant_f16(pack_le(q), ones, np.zeros((1, 4), np.uint16), 64)
    assert np.array_equal(w.view(np.float16).astype(np.float64), q.astype(np.float64))
    b2048 = np.full((1, 4), 0x4500, np.uint16)  # 2048 in BF16
    w = o.dequant_f16(pack_le(q), ones, b2048, 64).view(np.float16).astype(np.float64)[0]
    assert w[1] == 2048 and w[3] == 2052 and w[2] == 2050 and w[255] == 2048 + 256


PINS = [pin_bf16_f32_table, pin_bf16_f64_table, pin_bf16_two_routes_agree, pin_unpack_word,
        pin_identity_scale, pin_centred_scale, pin_group_index, pin_worked_example,
        pin_bruteforce, pin_integer_exact, pin_silu_closed_forms, pin_silu_gate_zero,
        pin_silu_gate_structure, pin_gemm_rows_are_gemv, pin_quantize_grid_identity,
        pin_quantize_error_bound, pin_quantize_constant_group, pin_dequant_f16, pin_f16_f32_table,
        pin_f16_matches_ieee_conversion]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(oracle.default())


# ---------------------------------------------------------------------------
# planted mistakes: every one must be caught by at least one pin
# ---------------------------------------------------------------------------
MUTANTS = {
    "big_endian_bytes": ("(word >> (8 * (k % 4)))", "(word >> (8 * (3 - k % 4)))"),
    "group_index_mod": ("const int64_t g = k / gs;", "const int64_t g = k % G;"),
    "dropped_bias": ("return std::fma(s, q, b);", "return s * q;"),
    "silu_sign": ("t / (1.0 + std::exp(-t))", "t / (1.0 + std::exp(t))"),
    "transposed_gemm_out": ("Y[i * N + n] = acc;", "Y[n * m + i] = acc;"),
    "dropped_resid": ("y[n] = static_cast<double>(bf16_to_f32(x_resid[n])) + y[n];", "y[n] = y[n];"),
    "ties_away": ("u + 0x7FFFu + lsb", "u + 0x8000u + 0u * lsb"),
    "double_rounding": ("if (std::isnan(v)) return 0x7FC0u;",
                        "if (std::isnan(v)) return 0x7FC0u;\n    return f32_to_bf16(static_cast<float>(v));"),
    "x_index_shift": ("acc += row[k] * static_cast<double>(bf16_to_f32(x[k]));",
                      "acc += row[k] * static_cast<double>(bf16_to_f32(x[(k + 1) % K]));"),
    "quant_divisor_256": ("f32_to_bf16(range / 255.0f)", "f32_to_bf16(range / 256.0f)"),
    "quant_bias_from_max": ("const uint16_t bb = f32_to_bf16(lo);", "const uint16_t bb = f32_to_bf16(hi);"),
    "quant_round_down": ("c = std::nearbyint(d / sf);", "c = std::floor(d / sf);"),
    "f16_ties_away": ("(rem == half && (mant & 1u))", "(rem == half)"),
    "f16_no_subnormals": ("if (shift > 24) return sign;", "if (E < -14) return sign;"),
}


def _build_mutant(tmp: str, name: str) -> str:
    src = open(oracle_build.SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation anchor for {name} not unique/found"
    path = os.path.join(tmp, f"{name}.cpp")
    open(path, "w").write(src.replace(old, new))
    lib = os.path.join(tmp, f"lib{name}.so")
    subprocess.run(["g++", *oracle_build.CXXFLAGS, path, "-o", lib], check=True)
    return lib


@pytest.mark.skipif(shutil.which("g++") is None, reason="g++ not available")
@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistakes(name):
    with tempfile.TemporaryDirectory() as tmp:
        o = Oracle(_build_mutant(tmp, name))
        caught = []
        for pin in PINS:
            try:
                pin(o)
            except AssertionError:
                caught.append(pin.__name__)
        assert caught, f"planted mistake {name} passed every pin"
