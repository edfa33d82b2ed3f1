"""mlxq_gemm_noalloc: the gemm entry point that allocates no device memory.

It serves callers that cannot call cudaMalloc or a pool allocator (a fixed
memory budget set up front, a runtime that owns all device memory, a hot
loop that must not reach the allocator).  Its K-split partials live in the
library's static scratch array instead of the stream-ordered pool.  Checked
here: results equal mlxq_gemm bit for bit and the oracle within the gemm
tolerance; two calls in a row (no synchronisation between them, so the
second starts from the counters the first left behind) both stay exact; and
a call right after a bounded wait ran out (which makes mlxq_device_status
zero the array's tile counters) is still exact.

This file is collected last, so a run that stops at the first failure has
run every other test before it.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
import weight_only_quantized_mlx_b200 as mq
from _helpers import Guarded, assert_close, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "the -m gpu tests need a CUDA device"
    yield
    mq.mlxq_device_status()


def weight(seed, N, K, gs):
    g = synth.rng(seed)
    host = synth.weight(g, N, K, gs)
    t = tuple(dev(a) for a in host)
    return host, t, mq.weight_view(*t, gs), g


def call(fn, w, X, m, N):
    Y = Guarded(m * N)
    fn(w, X, Y.data_ptr(), m)
    torch.cuda.synchronize()
    Y.check_guards()
    return Y.value_bits().reshape(m, N)


# (N, K, gs, m): K split over CTAs (first three), whole tiles, and the
# weight-streaming kernel (m <= 32, no scratch at all)
SHAPES = [
    (512, 4096, 64, 64),
    (1000, 2048, 32, 200),
    (256, 4096, 128, 17 + 32),
    (256, 960, 64, 100),
    (300, 2048, 64, 24),
]


@pytest.mark.parametrize("N,K,gs,m", SHAPES)
def test_noalloc_matches_gemm_and_oracle(N, K, gs, m):
    host, keep, w, g = weight(70 + m, N, K, gs)
    X_bits = synth.activations(g, m, K)
    X = dev(X_bits)
    y_na = call(mq.mlxq_gemm_noalloc, w, X, m, N)
    y_ref = call(mq.mlxq_gemm, w, X, m, N)
    assert np.array_equal(y_na, y_ref)
    assert_close(y_na, oracle.gemm(*host, gs, X_bits), f"noalloc {N}x{K}/{gs} m={m}")


def test_noalloc_tail_split_matches_gemm():
    # 149 tiles: the last wave's tile splits K; both calls take the same plan
    N, K, gs, m = 256 * 149, 1024, 64, 32 + 8
    host, keep, w, g = weight(79, N, K, gs)
    X_bits = synth.activations(g, m, K)
    X = dev(X_bits)
    y_na = call(mq.mlxq_gemm_noalloc, w, X, m, N)
    y_ref = call(mq.mlxq_gemm, w, X, m, N)
    assert np.array_equal(y_na, y_ref)
    rows = np.concatenate([np.arange(0, 40), np.arange(N - 256, N)])
    p, s, b = host
    assert_close(y_na[:, rows], oracle.gemm(p[rows], s[rows], b[rows], gs, X_bits), "noalloc tail split")


def test_noalloc_two_calls_in_a_row():
    # different shapes, back to back on one stream with no synchronisation
    ha, keep_a, wa, ga = weight(80, 512, 4096, 64)  # keep_*: the device arrays the views point at
    hb, keep_b, wb, gb = weight(81, 1000, 2048, 32)
    Xa_bits, Xb_bits = synth.activations(ga, 64, 4096), synth.activations(gb, 200, 2048)
    Xa, Xb = dev(Xa_bits), dev(Xb_bits)
    Ya, Yb = Guarded(64 * 512), Guarded(200 * 1000)
    mq.mlxq_gemm_noalloc(wa, Xa, Ya.data_ptr(), 64)
    mq.mlxq_gemm_noalloc(wb, Xb, Yb.data_ptr(), 200)
    mq.mlxq_gemm_noalloc(wa, Xa, Ya.data_ptr(), 64)  # the first shape again, after the second
    torch.cuda.synchronize()
    Ya.check_guards()
    Yb.check_guards()
    ya, yb = Ya.value_bits().reshape(64, 512), Yb.value_bits().reshape(200, 1000)
    assert np.array_equal(ya, call(mq.mlxq_gemm, wa, Xa, 64, 512))
    assert np.array_equal(yb, call(mq.mlxq_gemm, wb, Xb, 200, 1000))
    assert_close(ya, oracle.gemm(*ha, 64, Xa_bits), "noalloc, first call")
    assert_close(yb, oracle.gemm(*hb, 32, Xb_bits), "noalloc, second call")


def test_noalloc_after_a_timed_out_wait():
    # A wait that ran out could have stopped a split between raising and
    # clearing a tile counter; reading the status zeroes the counters, and the
    # next split call must be exact again.
    host, keep, w, g = weight(83, 512, 4096, 64)
    m = 64
    X_bits = synth.activations(g, m, 4096)
    X = dev(X_bits)
    mq.mlxq_selftest_wait_timeout(20000)  # 20 ms
    with pytest.raises(mq.MlxqError) as e:
        mq.mlxq_device_status()
    assert e.value.code == mq.MLXQ_ERR_DEVICE_TIMEOUT
    y_na = call(mq.mlxq_gemm_noalloc, w, X, m, 512)
    y_ref = call(mq.mlxq_gemm, w, X, m, 512)
    assert np.array_equal(y_na, y_ref)
    assert_close(y_na, oracle.gemm(*host, 64, X_bits), "noalloc after a timed-out wait")
    mq.mlxq_device_status()


def test_noalloc_scratch_covers_every_split_on_this_gpu():
    # the largest split the kernel makes: one CTA per SM, 256 x 256 fp32 each
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert 4096 + sms * 256 * 256 * 4 <= mq.MLXQ_STATIC_SCRATCH_BYTES
