"""Host-side checks of the C ABI (no GPU needed).

* libmlxq.so loads and exports every function include/mlxq.h declares;
* mlxq_load rejects each malformed input the MlxInt8Weight page's `load`
  entry lists (missing tensor, weight not 2-D U32, scales/biases not BF16 of
  shape [N, K/gs], group_size not dividing in_features) plus malformed
  safetensors, before touching the GPU;
* compute calls reject null/released handles, bad group sizes, null or
  misaligned buffers and overlapping outputs before launching anything;
* release of an empty handle is refused (no double free).
"""
from __future__ import annotations

import ctypes
import json
import os
import re

import pytest

import synth
import weight_only_quantized_mlx_b200 as mq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"MLXQ_API\s+[\w\s\*]+?\b(mlxq_\w+)\s*\(", text)
    return names


def test_library_exports_every_declared_function():
    L = mq.lib()
    names = header_functions()
    assert set(names) == set(mq.EXPORTS), (sorted(names), mq.EXPORTS)
    for n in names:
        assert hasattr(L, n), n


def test_binding_names_match_c_names():
    for n in mq.EXPORTS:
        assert callable(getattr(mq, n))


def _blob(N=4, K=16, gs=8, wdtype="U32", sdtype="BF16", bdtype="BF16", wshape=None, sshape=None,
          bshape=None, drop=None, base="layer"):
    g = synth.rng(0)
    packed, scales, biases = synth.weight(g, N, K, gs)
    t = {
        f"{base}.weight": (wdtype, wshape or packed.shape, packed.tobytes()),
        f"{base}.scales": (sdtype, sshape or scales.shape, scales.tobytes()),
        f"{base}.biases": (bdtype, bshape or biases.shape, biases.tobytes()),
    }
    if drop:
        del t[f"{base}.{drop}"]
    return synth.safetensors_blob(t)


def _load_rc(blob, base="layer", gs=8):
    w = mq.mlxq_weight()
    rc = mq.lib().mlxq_load(blob, len(blob), base.encode(), gs, ctypes.byref(w))
    return rc, w


@pytest.mark.parametrize("drop", ["weight", "scales", "biases"])
def test_load_missing_tensor(drop):
    rc, w = _load_rc(_blob(drop=drop))
    assert rc == mq.MLXQ_ERR_MISSING_TENSOR
    assert drop in mq.mlxq_last_error()
    assert not w.packed and not w.scales and not w.biases


def test_load_wrong_base_name():
    rc, _ = _load_rc(_blob(), base="other")
    assert rc == mq.MLXQ_ERR_MISSING_TENSOR


def test_load_weight_not_u32():
    # same byte count, declared I32
    rc, _ = _load_rc(_blob(wdtype="I32"))
    assert rc == mq.MLXQ_ERR_DTYPE


def test_load_weight_not_2d():
    rc, _ = _load_rc(_blob(wshape=(4 * 4,)))  # 1-D view of the same 16 words
    assert rc == mq.MLXQ_ERR_SHAPE
    rc, _ = _load_rc(_blob(wshape=(2, 2, 4)))
    assert rc == mq.MLXQ_ERR_SHAPE


@pytest.mark.parametrize("which", ["scales", "biases"])
def test_load_tables_not_bf16(which):
    kw = {"sdtype": "F16"} if which == "scales" else {"bdtype": "F16"}
    rc, _ = _load_rc(_blob(**kw))
    assert rc == mq.MLXQ_ERR_DTYPE


@pytest.mark.parametrize("which", ["scales", "biases"])
def test_load_tables_wrong_shape(which):
    kw = {"sshape": (2, 4)} if which == "scales" else {"bshape": (8, 1)}
    rc, _ = _load_rc(_blob(**kw))
    assert rc == mq.MLXQ_ERR_SHAPE
    # right element count for another group size is still the wrong shape
    rc, _ = _load_rc(_blob(), gs=4)
    assert rc == mq.MLXQ_ERR_SHAPE


@pytest.mark.parametrize("gs", [0, 3, 5, 32])
def test_load_group_size_must_divide(gs):
    rc, _ = _load_rc(_blob(), gs=gs)
    assert rc == mq.MLXQ_ERR_GROUP_SIZE


@pytest.mark.parametrize("mutate", ["short", "hlen", "json", "trailing", "offsets", "size",
                                    "notobj", "baddim"])
def test_load_malformed_safetensors(mutate):
    blob = bytearray(_blob())
    hlen = int.from_bytes(blob[:8], "little")
    header = json.loads(bytes(blob[8:8 + hlen]))
    data = bytes(blob[8 + hlen:])

    def rebuild(h, d=data):
        hb = json.dumps(h).encode()
        return len(hb).to_bytes(8, "little") + hb + d

    if mutate == "short":
        b = bytes(blob[:5])
    elif mutate == "hlen":
        b = (len(blob)).to_bytes(8, "little") + bytes(blob[8:])
    elif mutate == "json":
        b = bytes(blob[:8]) + b"[" + bytes(blob[9:])  # "[" opened, "}" closes: invalid
    elif mutate == "trailing":
        hb = json.dumps(header).encode() + b" x"
        b = len(hb).to_bytes(8, "little") + hb + data
    elif mutate == "offsets":
        header["layer.scales"]["data_offsets"][1] += 10 ** 6
        b = rebuild(header)
    elif mutate == "size":
        header["layer.weight"]["shape"] = [4, 3]
        b = rebuild(header)
    elif mutate == "notobj":
        b = rebuild([1, 2, 3])
    else:
        header["layer.weight"]["shape"] = [4, -4]
        b = rebuild(header)
    rc, _ = _load_rc(b)
    assert rc == mq.MLXQ_ERR_PARSE, mq.mlxq_last_error()


def test_load_valid_blob_reaches_the_device_step():
    rc, w = _load_rc(_blob())
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:
        has_gpu = False
    if has_gpu:
        assert rc == mq.MLXQ_OK
        assert (w.out_features, w.in_features, w.group_size) == (4, 16, 8)
        mq.mlxq_release(w)
    else:
        assert rc == mq.MLXQ_ERR_CUDA  # validation passed; cudaMalloc had no device
        assert not w.packed


def test_load_null_arguments():
    L = mq.lib()
    w = mq.mlxq_weight()
    assert L.mlxq_load(None, 0, b"x", 8, ctypes.byref(w)) == mq.MLXQ_ERR_INVALID_ARG
    assert L.mlxq_load(b"12345678", 8, None, 8, ctypes.byref(w)) == mq.MLXQ_ERR_INVALID_ARG
    assert L.mlxq_load(b"12345678", 8, b"x", 8, None) == mq.MLXQ_ERR_INVALID_ARG


def _fake_weight(N=8, K=64, gs=32):
    # addresses are never dereferenced: every call below fails validation first
    return mq.mlxq_weight(0x10000, 0x20000, 0x30000, N, K, gs)


def test_unknown_weight_flags_are_refused():
    L = mq.lib()
    w = _fake_weight()
    w.flags = 0x2  # not a defined MLXQ_WEIGHT_* bit
    X, Y = 0x100000, 0x200000
    assert L.mlxq_gemv(ctypes.byref(w), X, Y, 0) == mq.MLXQ_ERR_INVALID_ARG
    assert "flags" in mq.mlxq_last_error()
    assert L.mlxq_dequant(ctypes.byref(w), Y, 0) == mq.MLXQ_ERR_INVALID_ARG


def test_weight_struct_layout_has_flags_last():
    # the C struct: three pointers, three uint32 dimensions, uint32 flags
    assert [f[0] for f in mq.mlxq_weight._fields_] == ["packed", "scales", "biases", "out_features",
                                                      "in_features", "group_size", "flags"]
    assert ctypes.sizeof(mq.mlxq_weight) == 3 * 8 + 4 * 4
    assert mq.MLXQ_WEIGHT_STATIC == 1


def test_release_twice_is_refused():
    w = mq.mlxq_weight()
    assert mq.lib().mlxq_release(ctypes.byref(w)) == mq.MLXQ_ERR_INVALID_ARG
    assert "released" in mq.mlxq_last_error()
    assert mq.lib().mlxq_release(None) == mq.MLXQ_ERR_INVALID_ARG


def test_calls_reject_released_or_null_handles():
    L = mq.lib()
    w = mq.mlxq_weight()
    X, Y = 0x100000, 0x200000
    assert L.mlxq_gemv(ctypes.byref(w), X, Y, 0) == mq.MLXQ_ERR_INVALID_ARG
    assert L.mlxq_gemv(None, X, Y, 0) == mq.MLXQ_ERR_INVALID_ARG
    assert L.mlxq_dequant(ctypes.byref(w), Y, 0) == mq.MLXQ_ERR_INVALID_ARG
    assert L.mlxq_gemm(ctypes.byref(w), X, Y, 4, 0) == mq.MLXQ_ERR_INVALID_ARG
    assert L.mlxq_gemv_silu_gate(ctypes.byref(w), X, X + 4096, Y, 0) == mq.MLXQ_ERR_INVALID_ARG
    assert L.mlxq_gemv_silu_gate_resid(ctypes.byref(w), X, X + 4096, Y, Y, 0) == mq.MLXQ_ERR_INVALID_ARG


def test_calls_reject_bad_group_size_and_k():
    L = mq.lib()
    X, Y = 0x100000, 0x200000
    for w, code in ((_fake_weight(gs=0), mq.MLXQ_ERR_GROUP_SIZE), (_fake_weight(gs=24), mq.MLXQ_ERR_GROUP_SIZE),
                    (_fake_weight(K=66, gs=2), mq.MLXQ_ERR_SHAPE)):
        assert L.mlxq_gemv(ctypes.byref(w), X, Y, 0) == code
        assert L.mlxq_dequant(ctypes.byref(w), Y, 0) == code


def test_calls_reject_null_and_misaligned_buffers():
    L = mq.lib()
    w = _fake_weight()
    assert L.mlxq_gemv(ctypes.byref(w), None, 0x200000, 0) == mq.MLXQ_ERR_INVALID_ARG
    assert L.mlxq_gemv(ctypes.byref(w), 0x100000, None, 0) == mq.MLXQ_ERR_INVALID_ARG
    assert L.mlxq_gemv(ctypes.byref(w), 0x100001, 0x200000, 0) == mq.MLXQ_ERR_INVALID_ARG
    assert L.mlxq_dequant(ctypes.byref(w), 0x200001, 0) == mq.MLXQ_ERR_INVALID_ARG
    assert L.mlxq_gemm(ctypes.byref(w), 0x100000, None, 3, 0) == mq.MLXQ_ERR_INVALID_ARG
    assert L.mlxq_gemm_with(ctypes.byref(w), 0x100000, 0x200000, 3, 99, 0) == mq.MLXQ_ERR_INVALID_ARG


def test_calls_reject_overlapping_outputs():
    L = mq.lib()
    w = _fake_weight(N=8, K=64)
    x = 0x100000
    assert L.mlxq_gemv(ctypes.byref(w), x, x + 8, 0) == mq.MLXQ_ERR_INVALID_ARG        # y inside x
    assert L.mlxq_gemv(ctypes.byref(w), x, 0x10000 + 16, 0) == mq.MLXQ_ERR_INVALID_ARG  # y inside packed
    r = 0x300000
    assert L.mlxq_gemv_silu_gate_resid(ctypes.byref(w), x, x + 256, r, r + 2, 0) == mq.MLXQ_ERR_INVALID_ARG
    assert L.mlxq_gemm(ctypes.byref(w), x, x + 64, 2, 0) == mq.MLXQ_ERR_INVALID_ARG
    assert L.mlxq_dequant(ctypes.byref(w), 0x30000 - 4, 0) == mq.MLXQ_ERR_INVALID_ARG


def test_zero_rows_are_a_no_op():
    L = mq.lib()
    w = _fake_weight()
    assert L.mlxq_gemm(ctypes.byref(w), None, None, 0, 0) == mq.MLXQ_OK


def test_python_error_type():
    with pytest.raises(mq.MlxqError) as ei:
        mq.mlxq_release(mq.mlxq_weight())
    assert ei.value.code == mq.MLXQ_ERR_INVALID_ARG


def test_product_path_has_no_oracle_dependency():
    # the binding and the CUDA sources never load, import or link the oracle
    pkg = os.path.join(ROOT, "weight_only_quantized_mlx_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                for needle in ("import oracle", "from oracle", "libmlxq_oracle", "mlxq_oracle"):
                    assert needle not in text, f"{f} references the oracle ({needle})"


def test_load_injected_alloc_failure_leaves_handle_untouched():
    # the first device allocation of the next load fails (no CUDA call is made)
    mq.mlxq_selftest_fail_alloc(1)
    try:
        rc, w = _load_rc(_blob())
    finally:
        mq.mlxq_selftest_fail_alloc(0)
    assert rc == mq.MLXQ_ERR_CUDA
    assert "uploading" in mq.mlxq_last_error()
    assert not w.packed and not w.scales and not w.biases and w.out_features == 0


def test_selftest_wait_timeout_rejects_bad_limits():
    for bad in (0, 1000001):
        with pytest.raises(mq.MlxqError) as e:
            mq.mlxq_selftest_wait_timeout(bad, 0)
        assert e.value.code == mq.MLXQ_ERR_INVALID_ARG


def test_quantize_validation_before_any_launch():
    # host checks only: fake (non-null, aligned) device addresses, nothing launched
    N, K = 8, 64
    base = 1 << 40
    def handle(gs, packed=base, scales=base + (1 << 20), biases=base + (2 << 20)):
        return mq.mlxq_weight(packed, scales, biases, N, K, gs)
    w = base + (3 << 20)
    for gs, code in ((6, mq.MLXQ_ERR_GROUP_SIZE), (2, mq.MLXQ_ERR_UNSUPPORTED), (0, mq.MLXQ_ERR_GROUP_SIZE)):
        with pytest.raises(mq.MlxqError) as e:
            mq.mlxq_quantize(w, handle(gs), 0)
        assert e.value.code == code, gs
    with pytest.raises(mq.MlxqError) as e:
        mq.mlxq_quantize(0, handle(16), 0)
    assert e.value.code == mq.MLXQ_ERR_INVALID_ARG
    with pytest.raises(mq.MlxqError) as e:   # the codes would overwrite the source
        mq.mlxq_quantize(base + 16, handle(16), 0)
    assert e.value.code == mq.MLXQ_ERR_INVALID_ARG and "overlap" in mq.mlxq_last_error()
    mq.mlxq_quantize(w, mq.mlxq_weight(base, base + 4096, base + 8192, 0, K, 16), 0)  # N = 0: no work


def test_weight_dimensions_beyond_any_device_are_rejected():
    base = 1 << 40
    w = mq.mlxq_weight(base, base + 4096, base + 8192, 0xFFFFFFF0, 0xFFFFFFF0, 16)
    with pytest.raises(mq.MlxqError) as e:
        mq.mlxq_dequant(w, base + (1 << 20), 0)
    assert e.value.code == mq.MLXQ_ERR_SHAPE


def test_gemm_rows_beyond_any_device_are_rejected():
    base = 1 << 40
    w = mq.mlxq_weight(base, base + (1 << 30), base + (2 << 30), 4096, 1 << 24, 64)
    with pytest.raises(mq.MlxqError) as e:
        mq.mlxq_gemm(w, base + (3 << 30), base + (4 << 30), 0xFFFFFFFF, 0)
    assert e.value.code == mq.MLXQ_ERR_SHAPE


def test_public_header_is_plain_c99(tmp_path):
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    src = tmp_path / "use_header.c"
    src.write_text('#include "mlxq.h"\n'
                   "int main(void) { mlxq_weight w = {0}; (void)w;\n"
                   "  return MLXQ_OK + MLXQ_DTYPE_F32 + MLXQ_GEMM_TCGEN05 - 5; }\n")
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", inc, "-c", str(src),
                        "-o", str(tmp_path / "use_header.o")], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_dequant_as_validation_before_any_launch():
    base = 1 << 40
    w = mq.mlxq_weight(base, base + (1 << 20), base + (2 << 20), 16, 64, 16)
    out = base + (3 << 20)
    for bad_dtype in (-1, 3):
        with pytest.raises(mq.MlxqError) as e:
            mq.mlxq_dequant_as(w, out, bad_dtype, 0)
        assert e.value.code == mq.MLXQ_ERR_INVALID_ARG
    with pytest.raises(mq.MlxqError) as e:      # FP32 output must be 4-byte aligned
        mq.mlxq_dequant_as(w, out + 2, mq.MLXQ_DTYPE_F32, 0)
    assert e.value.code == mq.MLXQ_ERR_INVALID_ARG and "aligned" in mq.mlxq_last_error()
    with pytest.raises(mq.MlxqError) as e:
        mq.mlxq_dequant_as(w, 0, mq.MLXQ_DTYPE_F16, 0)
    assert e.value.code == mq.MLXQ_ERR_INVALID_ARG
    with pytest.raises(mq.MlxqError) as e:      # output would overwrite the packed codes
        mq.mlxq_dequant_as(w, base, mq.MLXQ_DTYPE_F32, 0)
    assert e.value.code == mq.MLXQ_ERR_INVALID_ARG
