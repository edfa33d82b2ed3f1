"""GPU parity of the any-group-size kernels ("MlxInt8Weight" page, load:
group_size only has to divide in_features).  Group sizes that are multiples
of 4 but not of 16, or whose tables are not 16-byte multiples per row
((K / gs) % 8 != 0), through gemv, gemv_silu_gate(_resid), small-m gemm and
dequantize_to, against the oracle: dequant bit-exact, the rest within the
shared tolerance.  K % 16 == 0 in every shape (16-byte rows of codes)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
import weight_only_quantized_mlx_b200 as mq
from _helpers import Guarded, assert_close, dev, host_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    mq.lib()
    yield
    torch.cuda.synchronize()
    mq.mlxq_device_status()


class DevWeight:
    def __init__(self, packed, scales, biases, gs):
        self.host = (packed, scales, biases)
        self.t = (dev(packed), dev(scales), dev(biases))
        self.w = mq.weight_view(*self.t, gs)
        self.N, self.K = packed.shape[0], packed.shape[1] * 4


def make(seed, N, K, gs):
    g = synth.rng(seed)
    return DevWeight(*synth.weight(g, N, K, gs), gs), g


# (N, K, gs): odd N (a lone last row), G = K / gs with G % 8 != 0 in all but
# one, K long enough for several rounds of the lanes' 512-code steps
SHAPES = [(67, 1040, 4), (130, 1040, 8), (45, 1200, 12), (33, 1040, 20), (129, 1200, 48), (64, 960, 96),
          (31, 1280, 256), (301, 4096, 8), (5, 16, 4)]
IDS = [f"{n}x{k}/gs{gs}" for n, k, gs in SHAPES]


@pytest.mark.parametrize("N,K,gs", SHAPES, ids=IDS)
def test_dequant_any_group_size(N, K, gs):
    W, _ = make(20, N, K, gs)
    ref = oracle.dequant(*W.host, gs).ravel()
    for off in (0, 8):  # 32-byte and 16-byte aligned output
        out = Guarded(N * K, offset_elems=off)
        mq.mlxq_dequant(W.w, out.data_ptr())
        torch.cuda.synchronize()
        out.check_guards()
        assert np.array_equal(out.value_bits(), ref), f"offset {off}"


@pytest.mark.parametrize("N,K,gs", SHAPES, ids=IDS)
def test_gemv_any_group_size(N, K, gs):
    W, g = make(21, N, K, gs)
    x = synth.activations(g, K)
    y = Guarded(N)
    mq.mlxq_gemv(W.w, dev(x), y.data_ptr())
    torch.cuda.synchronize()
    y.check_guards()
    assert_close(y.value_bits(), oracle.gemv(*W.host, gs, x), f"gemv {N}x{K}/{gs}")


@pytest.mark.parametrize("N,K,gs", SHAPES, ids=IDS)
def test_silu_gate_any_group_size(N, K, gs):
    W, g = make(22, N, K, gs)
    gate, up, r = synth.activations(g, K), synth.activations(g, K), synth.activations(g, N)
    y = Guarded(N)
    mq.mlxq_gemv_silu_gate(W.w, dev(gate), dev(up), y.data_ptr())
    torch.cuda.synchronize()
    y.check_guards()
    assert_close(y.value_bits(), oracle.silu_gate(*W.host, gs, gate, up), f"silu {N}x{K}/{gs}")
    y2 = Guarded(N)
    mq.mlxq_gemv_silu_gate_resid(W.w, dev(gate), dev(up), dev(r), y2.data_ptr())
    torch.cuda.synchronize()
    y2.check_guards()
    assert_close(y2.value_bits(), oracle.silu_gate_resid(*W.host, gs, gate, up, r), f"resid {N}x{K}/{gs}")


@pytest.mark.parametrize("N,K,gs", SHAPES, ids=IDS)
@pytest.mark.parametrize("m", [1, 2, 3, 8, 9, 17, 32, 40])
def test_gemm_any_group_size(N, K, gs, m):
    W, g = make(23, N, K, gs)
    X = synth.activations(g, m, K)
    ref = oracle.gemm(*W.host, gs, X)
    for kernel in (mq.MLXQ_GEMM_SMALLM_FFMA, mq.MLXQ_GEMM_AUTO):
        Y = Guarded(m * N)
        mq.mlxq_gemm_with(W.w, dev(X), Y.data_ptr(), m, kernel)
        torch.cuda.synchronize()
        Y.check_guards()
        assert_close(Y.value_bits().reshape(m, N), ref, f"gemm m={m} {N}x{K}/{gs} kernel {kernel}")


def test_gemm_any_group_size_long_k_passes():
    # K = 28672: the rows of one pass must fit in shared memory, so passes of
    # fewer rows; sampled weight rows against the oracle
    N, K, gs, m = 600, 28672, 8, 5
    W, g = make(24, N, K, gs)
    X = synth.activations(g, m, K)
    Y = torch.empty(m * N, dtype=torch.bfloat16, device="cuda")
    mq.mlxq_gemm_with(W.w, dev(X), Y, m, mq.MLXQ_GEMM_SMALLM_FFMA)
    got = host_bits(Y).reshape(m, N)
    rows = np.array([0, 1, 2, 299, 300, 597, 598, 599])
    p, s, b = W.host
    assert_close(got[:, rows], oracle.gemm(p[rows], s[rows], b[rows], gs, X), "long-K gemm")


def test_gemv_decode_shape_gs8():
    # the decode projection shape at group_size 8 (the bench's any-gs row)
    p, s, b = synth.weight(synth.rng(25), 4096, 4096, 8)
    x = synth.activations(synth.rng(26), 4096)
    W = DevWeight(p, s, b, 8)
    y = Guarded(4096)
    mq.mlxq_gemv(W.w, dev(x), y.data_ptr())
    torch.cuda.synchronize()
    y.check_guards()
    assert_close(y.value_bits(), oracle.gemv(p, s, b, 8, x), "gemv 4096x4096/8")
    out = torch.empty(4096 * 4096, dtype=torch.bfloat16, device="cuda")
    mq.mlxq_dequant(W.w, out)
    assert np.array_equal(host_bits(out), oracle.dequant(p, s, b, 8).ravel())
