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


def test_profile_traffic_only_for_the_profiled_source(tmp_path):
    # a summary in the committed format, recorded for one source file
    src = tmp_path / "k.cu"
    src.write_text("kernel v1\n")
    (tmp_path / "profiles").mkdir()
    digest = bench.source_hash(["k.cu"], str(tmp_path))
    (tmp_path / "profiles" / "k_tag.md").write_text(
        "# k\n\n- dram__bytes_read.sum: `17.9` Mbyte\n"
        f"- traffic_bytes_per_launch: `17864448`\n- source_sha256: `{digest}` (of k.cu)\n")
    assert bench.profile_traffic("k_tag", ["k.cu"], str(tmp_path)) == 17864448.0
    assert bench.profile_traffic("no_such_profile", ["k.cu"], str(tmp_path)) is None
    src.write_text("kernel v2\n")  # the source changed since the capture: no figure
    assert bench.profile_traffic("k_tag", ["k.cu"], str(tmp_path)) is None


def test_committed_profiles_name_their_sources():
    # every committed summary that feeds a bench figure records a source hash
    for name in os.listdir(os.path.join(ROOT, "profiles")):
        text = open(os.path.join(ROOT, "profiles", name)).read()
        if "traffic_bytes_per_launch" in text:
            assert "source_sha256" in text, name
