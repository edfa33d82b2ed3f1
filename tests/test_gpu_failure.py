"""Failure detection on the GPU without a GPU fault.

* A bounded wait made to run out (an mbarrier nothing completes, 20 ms
  limit) sets the device status word; mlxq_device_status reports
  MLXQ_ERR_DEVICE_TIMEOUT once and clears it, and the context stays usable:
  the next gemv is still exact against the oracle.
* An allocation failure injected into mlxq_load at each of its three
  allocations returns MLXQ_ERR_CUDA, leaves the handle untouched and frees
  whatever it had allocated; a load after it succeeds.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

import oracle
import synth
import weight_only_quantized_mlx_b200 as mq
from _helpers import assert_close, dev, host_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "the -m gpu tests need a CUDA device"
    mq.mlxq_device_status()
    yield
    mq.mlxq_device_status()


def test_bounded_wait_runs_out_and_context_survives():
    mq.mlxq_selftest_wait_timeout(20000)  # 20 ms
    with pytest.raises(mq.MlxqError) as e:
        mq.mlxq_device_status()
    assert e.value.code == mq.MLXQ_ERR_DEVICE_TIMEOUT
    mq.mlxq_device_status()  # read once, then clear
    g = synth.rng(90)
    p, s, b = synth.weight(g, 256, 512, 64)
    x = synth.activations(g, 512)
    t = (dev(p), dev(s), dev(b))
    w = mq.weight_view(*t, 64)
    y = torch.empty(256, dtype=torch.bfloat16, device="cuda")
    mq.mlxq_gemv(w, dev(x), y)
    torch.cuda.synchronize()
    assert_close(host_bits(y), oracle.gemv(p, s, b, 64, x), "gemv after a timed-out wait")
    mq.mlxq_device_status()


@pytest.mark.parametrize("nth", [1, 2, 3])
def test_load_alloc_failure_frees_and_recovers(nth):
    g = synth.rng(91)
    p, s, b = synth.weight(g, 4096, 8192, 64)  # 32 MB of codes
    blob = synth.weight_blob("w", p, s, b)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    mq.mlxq_selftest_fail_alloc(nth)
    w = mq.mlxq_weight()
    try:
        rc = mq.lib().mlxq_load(blob, len(blob), b"w", 64, ctypes.byref(w))
    finally:
        mq.mlxq_selftest_fail_alloc(0)
    assert rc == mq.MLXQ_ERR_CUDA
    assert not w.packed and not w.scales and not w.biases
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] > free0 - (16 << 20)  # the 32 MB buffer was not kept
    ok = mq.MlxInt8Weight.load(blob, "w", 64)
    ok.release()
