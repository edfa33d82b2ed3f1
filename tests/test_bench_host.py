"""Host-side pieces of bench.py that the reported numbers rest on."""
from __future__ import annotations

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_algorithmic_bytes():
    # decode gemv N = K = 4096, gs = 64: codes + scales + biases + x + y
    assert bench.gemv_bytes(4096, 4096, 64) == 4096 * 4096 + 4 * 4096 * 4096 // 64 + 2 * 4096 + 2 * 4096 == 17_842_176
    # the decode MLP chain: gate and up (14336 x 4096), then the fused down
    # projection (4096 x 14336) reading gate, up and the residual
    D, F, gs = 4096, 14336, 64
    chain = 2 * bench.gemv_bytes(F, D, gs) + (D * F + 4 * D * F // gs + 4 * F + 4 * D)
    assert chain == 187_318_272


def test_profile_traffic_only_for_the_profiled_source():
    srcs = ["weight_only_quantized_mlx_b200/csrc/gemv_mma.cu", "weight_only_quantized_mlx_b200/csrc/device_common.cuh"]
    t = bench.profile_traffic("gemv_decode_4096x4096_gs64", srcs)
    assert t is not None and 17e6 < t < 19e6       # the committed capture matches the source
    assert bench.profile_traffic("gemv_decode_4096x4096_gs64", srcs[:1]) is None  # another source: no figure
    assert bench.profile_traffic("no_such_profile", srcs) is None
