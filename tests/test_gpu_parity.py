"""GPU parity: every kernel of the library, called through the C ABI, against
the CPU oracle on the same seeded inputs.

* dequantize_to: bit-exact (BF16 bit patterns equal).
* gemv / gemv_silu_gate / gemv_silu_gate_resid / gemm: within the tolerance
  in tests/_helpers.py, elementwise and normwise.
Sizes span several pipeline stages / tiles with ragged tails, both the
vectorised and the generic kernel paths, and the workload shapes of the API
page's use (decode projections, a fused MLP, small-m and prefill gemm); at the
largest shapes the oracle is evaluated on sampled weight rows.  Output buffers
carry sentinel guard bands that must survive every call.
"""
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
    mq.mlxq_device_status()  # no kernel gave up a bounded wait


class DevWeight:
    def __init__(self, packed, scales, biases, gs):
        self.host = (packed, scales, biases)
        self.t = (dev(packed), dev(scales), dev(biases))
        self.gs = gs
        self.w = mq.weight_view(*self.t, gs)
        self.N, self.K = packed.shape[0], packed.shape[1] * 4


def make(seed, N, K, gs):
    g = synth.rng(seed)
    p, s, b = synth.weight(g, N, K, gs)
    return DevWeight(p, s, b, gs), g


def rows_subset(W: DevWeight, rows):
    p, s, b = W.host
    return p[rows], s[rows], b[rows]


# ---------------------------------------------------------------- dequantize_to
DEQ_SHAPES = [
    (256, 512, 64),    # the tiny workload
    (256, 512, 32), (256, 512, 128), (37, 1040, 16), (3, 64, 64), (1, 16, 16),
    (5, 12, 4), (9, 60, 12), (4, 8, 2), (6, 20, 20), (2, 4, 1),   # generic path
]


@pytest.mark.parametrize("N,K,gs", DEQ_SHAPES)
def test_dequant_bit_exact(N, K, gs):
    W, _ = make(0, N, K, gs)
    out = Guarded(N * K)
    mq.mlxq_dequant(W.w, out.data_ptr())
    torch.cuda.synchronize()
    out.check_guards()
    ref = oracle.dequant(*W.host, gs)
    assert np.array_equal(out.value_bits(), ref.ravel())


def test_dequant_misaligned_output_takes_generic_path():
    W, _ = make(1, 33, 256, 32)
    out = Guarded(33 * 256, offset_elems=1)  # 2-byte but not 16-byte aligned
    mq.mlxq_dequant(W.w, out.data_ptr())
    torch.cuda.synchronize()
    out.check_guards()
    assert np.array_equal(out.value_bits(), oracle.dequant(*W.host, 32).ravel())


@pytest.mark.parametrize("offset_elems", [8, 16])  # 16-byte aligned only; 32-byte aligned
def test_dequant_vector_paths_by_output_alignment(offset_elems):
    W, _ = make(3, 300, 1024 + 64, 64)  # several block steps and a ragged last one
    out = Guarded(300 * 1088, offset_elems=offset_elems)
    mq.mlxq_dequant(W.w, out.data_ptr())
    torch.cuda.synchronize()
    out.check_guards()
    assert np.array_equal(out.value_bits(), oracle.dequant(*W.host, 64).ravel())


def test_dequant_decode_workload_100_pairs():
    out = torch.empty(4096 * 4096, dtype=torch.bfloat16, device="cuda")
    for seed in range(100):
        p, s, b, _ = synth.decode_pair(seed, 4096, 4096, 64)
        W = DevWeight(p, s, b, 64)
        mq.mlxq_dequant(W.w, out)
        got = host_bits(out)
        ref = oracle.dequant(p, s, b, 64).ravel()
        assert np.array_equal(got, ref), f"seed {seed}"


def test_dequant_loaded_weight_and_release():
    g = synth.rng(5)
    p, s, b = synth.weight(g, 64, 256, 64)
    W = mq.MlxInt8Weight.load(synth.weight_blob("model.layers.0.mlp.down_proj", p, s, b),
                              "model.layers.0.mlp.down_proj", 64)
    assert (W.out_features, W.in_features, W.group_size) == (64, 256, 64)
    out = torch.empty(64 * 256, dtype=torch.bfloat16, device="cuda")
    W.dequantize_to(out)
    assert np.array_equal(host_bits(out), oracle.dequant(p, s, b, 64).ravel())
    W.release()
    with pytest.raises(mq.MlxqError):
        W.release()


# ---------------------------------------------------------------- gemv
GEMV_SHAPES = [
    (256, 512, 64),                     # tiny workload
    (4096, 4096, 64), (4096, 4096, 128), (4096, 4096, 32),
    (1000, 2048, 64), (333, 1024, 16), (17, 8192, 64),
    (2048, 14336, 64), (517, 14336, 128), (300, 28672, 64),  # 2 and 4 chunks per thread
    (6000, 8192, 64),                   # 41 rows per CTA: one 3-D code copy per stage, ragged last CTA
    (14336, 4096, 64), (10000, 2048, 32),  # 5 to 7 tiles per CTA: the 28-warp form, two items per warp
    (12000, 1024, 16), (11111, 4096, 64),  # (6 tiles; 76 rows per CTA with a ragged last CTA)
    (20000, 1024, 64), (40000, 512, 32),   # above 128 rows per SM: the tile-group kernel at m = 1
    (129, 256, 32), (7, 64, 64), (1, 16, 16),
    (45, 36, 12), (10, 100, 4), (3, 40000, 64),              # generic path
    (700, 4096, 256), (90, 8192, 256),                        # fp32-pipe stream kernel
]


def run_gemv(W, x_bits):
    x = dev(x_bits)
    y = Guarded(W.N)
    mq.mlxq_gemv(W.w, x, y.data_ptr())
    torch.cuda.synchronize()
    y.check_guards()
    return y.value_bits()


@pytest.mark.parametrize("N,K,gs", GEMV_SHAPES)
def test_gemv(N, K, gs):
    W, g = make(2, N, K, gs)
    x = synth.activations(g, K)
    assert_close(run_gemv(W, x), oracle.gemv(*W.host, gs, x), f"gemv {N}x{K}/{gs}")


def test_gemv_decode_workload_100_pairs():
    for seed in range(100):
        p, s, b, x = synth.decode_pair(seed, 4096, 4096, 64)
        W = DevWeight(p, s, b, 64)
        assert_close(run_gemv(W, x), oracle.gemv(p, s, b, 64, x), f"seed {seed}")


def test_gemv_misaligned_x_takes_generic_path():
    W, g = make(3, 200, 1024, 64)
    x_bits = synth.activations(g, 1024)
    buf = torch.empty(1024 + 8, dtype=torch.bfloat16, device="cuda")
    xs = buf[1:1025]
    xs.copy_(dev(x_bits))
    y = Guarded(200)
    mq.mlxq_gemv(W.w, xs, y.data_ptr())
    torch.cuda.synchronize()
    y.check_guards()
    assert_close(y.value_bits(), oracle.gemv(*W.host, 64, x_bits))


def test_gemv_integer_weights_are_exact():
    # s = 1, b = 0, small-integer x: every fp32 sum is exact, so the GPU must
    # return exactly the oracle's (exact) result.
    g = np.random.default_rng(11)
    N, K = 300, 4096
    q = g.integers(0, 256, size=(N, K), dtype=np.uint8)
    packed = q.reshape(N, K // 4, 4).view("<u4").reshape(N, K // 4).astype(np.uint32)
    s = np.full((N, K // 64), 0x3F80, np.uint16)
    b = np.zeros((N, K // 64), np.uint16)
    x = synth.to_bf16_bits(g.integers(-3, 4, size=K).astype(np.float32))
    W = DevWeight(packed, s, b, 64)
    got = run_gemv(W, x)
    assert np.array_equal(got, oracle.gemv(packed, s, b, 64, x))


# ---------------------------------------------------------------- silu gate (+ resid)
SILU_SHAPES = [(4096, 14336, 64), (256, 512, 64), (1000, 4096, 128), (77, 2048, 32), (14336, 2048, 64),
               (300, 28672, 64), (45, 36, 12),
               (500, 4096, 256), (64, 14336, 256)]   # group size the tensor-pipe kernel does not take


@pytest.mark.parametrize("N,K,gs", SILU_SHAPES)
def test_gemv_silu_gate(N, K, gs):
    W, g = make(4, N, K, gs)
    gate, up = synth.activations(g, K), synth.activations(g, K)
    y = Guarded(N)
    mq.mlxq_gemv_silu_gate(W.w, dev(gate), dev(up), y.data_ptr())
    torch.cuda.synchronize()
    y.check_guards()
    assert_close(y.value_bits(), oracle.silu_gate(*W.host, gs, gate, up), f"silu {N}x{K}")


@pytest.mark.parametrize("N,K,gs", SILU_SHAPES)
def test_gemv_silu_gate_resid(N, K, gs):
    W, g = make(5, N, K, gs)
    gate, up, r = synth.activations(g, K), synth.activations(g, K), synth.activations(g, N)
    y = Guarded(N)
    mq.mlxq_gemv_silu_gate_resid(W.w, dev(gate), dev(up), dev(r), y.data_ptr())
    torch.cuda.synchronize()
    y.check_guards()
    assert_close(y.value_bits(), oracle.silu_gate_resid(*W.host, gs, gate, up, r), f"resid {N}x{K}")


def test_resid_in_place():
    W, g = make(6, 1024, 4096, 64)
    gate, up, r = synth.activations(g, 4096), synth.activations(g, 4096), synth.activations(g, 1024)
    yr = dev(r)
    mq.mlxq_gemv_silu_gate_resid(W.w, dev(gate), dev(up), yr, yr)  # y == x_resid
    assert_close(host_bits(yr), oracle.silu_gate_resid(*W.host, 64, gate, up, r))


def test_zero_gate_gives_zero_and_residual():
    W, g = make(7, 512, 4096, 64)
    zero = np.zeros(4096, np.uint16)
    up, r = synth.activations(g, 4096), synth.activations(g, 512)
    y = torch.empty(512, dtype=torch.bfloat16, device="cuda")
    mq.mlxq_gemv_silu_gate(W.w, dev(zero), dev(up), y)
    assert np.all(host_bits(y) & 0x7FFF == 0)  # +-0
    mq.mlxq_gemv_silu_gate_resid(W.w, dev(zero), dev(up), dev(r), y)
    assert np.array_equal(host_bits(y), r)


def test_fused_mlp_chain():
    """x -> gate, up projections (N=14336, K=4096) -> silu_gate_resid down
    projection (N=4096, K=14336).  The down projection is checked against the
    oracle fed with the GPU's BF16 gate/up (full tolerance), and against the
    unfused chain that materialises silu(gate)*up in BF16 (normwise only: the
    fused call never rounds that intermediate, and the BF16 rounding of h moves
    near-zero outputs by more than the elementwise bound allows)."""
    D, F, gs = 4096, 14336, 64
    Wg, g = make(30, F, D, gs)
    Wu, _ = make(31, F, D, gs)
    Wd, _ = make(32, D, F, gs)
    x = synth.activations(g, D)
    xr = synth.activations(g, D)
    gate = torch.empty(F, dtype=torch.bfloat16, device="cuda")
    up = torch.empty(F, dtype=torch.bfloat16, device="cuda")
    xd = dev(x)
    mq.mlxq_gemv(Wg.w, xd, gate)
    mq.mlxq_gemv(Wu.w, xd, up)
    y = torch.empty(D, dtype=torch.bfloat16, device="cuda")
    mq.mlxq_gemv_silu_gate_resid(Wd.w, gate, up, dev(xr), y)
    gb, ub = host_bits(gate), host_bits(up)
    assert_close(gb, oracle.gemv(*Wg.host, gs, x), "gate proj")
    assert_close(ub, oracle.gemv(*Wu.host, gs, x), "up proj")
    assert_close(host_bits(y), oracle.silu_gate_resid(*Wd.host, gs, gb, ub, xr), "down (fused)")
    h = oracle.silu_mul(gb, ub)
    ref_unfused = oracle.f64_to_bf16_array(oracle.gemv_f64(*Wd.host, gs, h) +
                                           oracle.bf16_bits_to_f64(xr))
    assert_close(host_bits(y), ref_unfused, "down (unfused reference)", elementwise=False)


def test_fused_mlp_chain_concatenated_gate_up():
    """Gate and up loaded as one [2F, D] weight: one gemv gives [gate | up],
    and silu_gate_resid reads the two halves in place.  The [2F, D] weight may
    take a different kernel (or row split) than the [F, D] ones, so each half
    is held to the oracle's gemv of its own weight, and the down projection to
    the oracle fed with those halves."""
    D, F, gs = 4096, 14336, 64
    Wg, g = make(30, F, D, gs)
    Wu, _ = make(31, F, D, gs)
    Wd, _ = make(32, D, F, gs)
    Wgu = DevWeight(*(np.concatenate([a, b]) for a, b in zip(Wg.host, Wu.host)), gs)
    x = synth.activations(g, D)
    xr = synth.activations(g, D)
    xd, xrd = dev(x), dev(xr)
    gu = torch.empty(2 * F, dtype=torch.bfloat16, device="cuda")
    mq.mlxq_gemv(Wgu.w, xd, gu)
    y2 = torch.empty(D, dtype=torch.bfloat16, device="cuda")
    mq.mlxq_gemv_silu_gate_resid(Wd.w, gu[:F], gu[F:], xrd, y2)
    gub = host_bits(gu)
    assert_close(gub[:F], oracle.gemv(*Wg.host, gs, x), "gate half of [gate | up]")
    assert_close(gub[F:], oracle.gemv(*Wu.host, gs, x), "up half of [gate | up]")
    assert_close(host_bits(y2), oracle.silu_gate_resid(*Wd.host, gs, gub[:F], gub[F:], xr),
                 "down after concatenated gate/up")


# ---------------------------------------------------------------- dequant to FP16 / FP32
@pytest.mark.parametrize("N,K,gs", [(256, 512, 64), (37, 1040, 16), (9, 60, 12), (4096, 4096, 64)])
@pytest.mark.parametrize("dtype", ["f16", "f32"])
def test_dequant_as_bit_exact(N, K, gs, dtype):
    W, _ = make(70, N, K, gs)
    code, tdt, want = {"f16": (mq.MLXQ_DTYPE_F16, torch.float16, oracle.dequant_f16),
                       "f32": (mq.MLXQ_DTYPE_F32, torch.float32, oracle.dequant_f32)}[dtype]
    ref = want(*W.host, gs)
    for off in (0, 1):  # vector stores, and an output aligned only to its element
        buf = torch.empty(N * K + off, dtype=tdt, device="cuda")
        mq.mlxq_dequant_as(W.w, buf.data_ptr() + off * buf.element_size(), code)
        torch.cuda.synchronize()
        got = buf[off:].cpu().numpy().reshape(N, K)
        assert np.array_equal(got.view(np.uint16 if dtype == "f16" else np.uint32),
                              ref.view(np.uint16 if dtype == "f16" else np.uint32)), (dtype, off)
    out = torch.empty(N * K, dtype=torch.bfloat16, device="cuda")
    mq.mlxq_dequant_as(W.w, out, mq.MLXQ_DTYPE_BF16)  # BF16: the page's dequantize_to
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(out), oracle.dequant(*W.host, gs).ravel())


# ---------------------------------------------------------------- quantize
QUANT_SHAPES = [(256, 512, 64), (300, 1040, 16), (77, 2048, 32), (1, 64, 64), (128, 4096, 128), (5, 24, 4),
                (64, 512, 8), (16, 1024, 256), (33, 768, 48)]


def run_quantize(w_bits, gs, offset_elems=0):
    N, K = w_bits.shape
    src = torch.zeros(N * K + offset_elems, dtype=torch.int16, device="cuda")
    src[offset_elems:] = torch.from_numpy(w_bits.view(np.int16).ravel()).cuda()
    packed = torch.empty((N, K // 4), dtype=torch.int32, device="cuda")
    scales = torch.empty((N, K // gs), dtype=torch.int16, device="cuda")
    biases = torch.empty((N, K // gs), dtype=torch.int16, device="cuda")
    dst = mq.weight_view(packed, scales, biases, gs)
    mq.mlxq_quantize(src.data_ptr() + 2 * offset_elems, dst)
    torch.cuda.synchronize()
    return (packed.cpu().numpy().view(np.uint32), scales.cpu().numpy().view(np.uint16),
            biases.cpu().numpy().view(np.uint16)), (packed, scales, biases, dst)


@pytest.mark.parametrize("N,K,gs", QUANT_SHAPES)
def test_quantize_bit_exact(N, K, gs):
    g = synth.rng(60)
    w = synth.to_bf16_bits((g.standard_normal((N, K)) * 0.04).astype(np.float32))
    want = oracle.quantize(w, gs)
    for off in (0, 1):  # 8-byte loads, and a source that only allows 2-byte loads
        got, _ = run_quantize(w, gs, off)
        for a, b, what in zip(got, want, ("codes", "scales", "biases")):
            assert np.array_equal(a, b), f"{what} {N}x{K}/{gs} offset {off}"


def test_quantize_then_gemv():
    # the quantised weight goes straight into the other calls
    g = synth.rng(61)
    N, K, gs = 512, 2048, 64
    w = synth.to_bf16_bits((g.standard_normal((N, K)) * 0.05).astype(np.float32))
    host, (_, _, _, dst) = run_quantize(w, gs)
    x = synth.activations(g, K)
    y = torch.empty(N, dtype=torch.bfloat16, device="cuda")
    mq.mlxq_gemv(dst, dev(x), y)
    torch.cuda.synchronize()
    assert_close(host_bits(y), oracle.gemv(*host, gs, x), "gemv of a quantised weight")


def test_gemv_reads_a_weight_written_just_before():
    # Without MLXQ_WEIGHT_STATIC every read of the weight follows the previous
    # work on the stream: a gemv queued right behind the quantize that writes
    # its weight (no synchronisation in between) sees the new codes, round
    # after round.
    g = synth.rng(62)
    N, K, gs = 4096, 4096, 64
    dst_t = (torch.zeros(N, K // 4, dtype=torch.int32, device="cuda"),
             torch.zeros(N, K // gs, dtype=torch.int16, device="cuda"),
             torch.zeros(N, K // gs, dtype=torch.int16, device="cuda"))
    dst = mq.weight_view(*dst_t, gs)
    x = synth.activations(g, K)
    xd = dev(x)
    ws = [synth.to_bf16_bits((g.standard_normal((N, K)) * s).astype(np.float32)) for s in (0.05, 0.02, 0.08)]
    wd = [dev(w) for w in ws]
    ys = [torch.empty(N, dtype=torch.bfloat16, device="cuda") for _ in ws]
    torch.cuda.synchronize()
    for wi, yi in zip(wd, ys):
        mq.mlxq_quantize(wi, dst)
        mq.mlxq_gemv(dst, xd, yi)
    torch.cuda.synchronize()
    for w, yi in zip(ws, ys):
        assert_close(host_bits(yi), oracle.gemv(*oracle.quantize(w, gs), gs, x), "gemv right after quantize")


@pytest.mark.parametrize("N,K,gs", [(4096, 4096, 64), (4096, 14336, 64), (1000, 4096, 128), (333, 1024, 32)])
def test_static_weight_flag(N, K, gs):
    # MLXQ_WEIGHT_STATIC lets the weight's copies start before the previous
    # work has finished; the results are identical to the default
    W, g = make(63, N, K, gs)
    x = synth.activations(g, K)
    gate, up, r = synth.activations(g, K), synth.activations(g, K), synth.activations(g, N)
    Ws = DevWeight(*W.host, gs)
    Ws.w.flags = mq.MLXQ_WEIGHT_STATIC
    y0, y1 = run_gemv(W, x), run_gemv(Ws, x)
    assert np.array_equal(y0, y1)
    assert_close(y1, oracle.gemv(*W.host, gs, x), f"static gemv {N}x{K}")
    outs = []
    for Wx in (W, Ws):
        y = Guarded(N)
        mq.mlxq_gemv_silu_gate_resid(Wx.w, dev(gate), dev(up), dev(r), y.data_ptr())
        torch.cuda.synchronize()
        y.check_guards()
        outs.append(y.value_bits())
    assert np.array_equal(outs[0], outs[1])
    assert_close(outs[1], oracle.silu_gate_resid(*W.host, gs, gate, up, r), f"static resid {N}x{K}")


def test_static_weight_decode_chain():
    # a chain of static-weight gemvs, each reading the previous one's output,
    # with no synchronisation: the activations are still read after they are
    # written
    g = synth.rng(64)
    N = K = 4096
    Ws = []
    for _ in range(6):
        W, _ = make(int(g.integers(1 << 30)), N, K, 64)
        W.w.flags = mq.MLXQ_WEIGHT_STATIC
        Ws.append(W)
    x = synth.activations(g, K)
    bufs = [dev(x)] + [torch.empty(N, dtype=torch.bfloat16, device="cuda") for _ in Ws]
    for i, W in enumerate(Ws):
        mq.mlxq_gemv(W.w, bufs[i], bufs[i + 1])
    torch.cuda.synchronize()
    for i, W in enumerate(Ws):
        xin = host_bits(bufs[i])
        assert_close(host_bits(bufs[i + 1]), oracle.gemv(*W.host, 64, xin), f"chain step {i}")


def test_quantize_constant_and_signed_zero_groups():
    # range 0 (scale 0, codes 0) and groups of signed zeros: the first
    # minimum in column order decides the bias's sign, as in the oracle
    N, K, gs = 4, 64, 16
    w = np.zeros((N, K), np.uint16)
    w[0, :16] = 0x3EC0            # 0.375
    w[1, 16:32:2] = 0x8000        # -0 then +0 alternating
    w[2, 33:48:2] = 0x8000        # +0 first, then -0
    w[3] = synth.to_bf16_bits(np.linspace(-1, 1, K).astype(np.float32))
    got, _ = run_quantize(w, gs)
    for a, b in zip(got, oracle.quantize(w, gs)):
        assert np.array_equal(a, b)


# ---------------------------------------------------------------- gemm
def run_gemm(W, X_bits, m, kernel=mq.MLXQ_GEMM_AUTO):
    X = dev(X_bits)
    Y = Guarded(m * W.N)
    mq.mlxq_gemm_with(W.w, X, Y.data_ptr(), m, kernel)
    torch.cuda.synchronize()
    Y.check_guards()
    return Y.value_bits().reshape(m, W.N)


SMALLM_SHAPES = [(512, 1024, 64), (300, 4096, 32), (256, 14336, 128), (128, 28672, 64), (77, 512, 16),
                 (5000, 1152, 16), (2100, 2304, 32),   # several tile groups per CTA; K not a multiple of 512
                 (10000, 2048, 128),   # > 64 rows per CTA at group size 128: a table box per pair of stages
                 (9000, 8192, 64)]     # 31-61 rows per CTA: one 3-D code copy per stage


@pytest.mark.parametrize("N,K,gs", SMALLM_SHAPES)
@pytest.mark.parametrize("m", [1, 2, 3, 5, 8, 9, 16, 17, 32])
def test_gemm_smallm_tensor_pipe(N, K, gs, m):
    W, g = make(8, N, K, gs)
    X = synth.activations(g, m, K)
    ref = oracle.gemm(*W.host, gs, X)
    assert_close(run_gemm(W, X, m, mq.MLXQ_GEMM_SMALLM), ref, f"smallm m={m} {N}x{K}")
    assert_close(run_gemm(W, X, m, mq.MLXQ_GEMM_AUTO), ref, f"auto m={m} {N}x{K}")


# the tile-group kernel wants K % 128 == 0 and gs in {16, 32, 64}; the rows
# per CTA span one partial group, one or several full groups, and a ragged
# last tile
GROUP_SHAPES = [(512, 1024, 64), (300, 4096, 32), (77, 512, 16), (5000, 1152, 16), (2100, 2304, 32),
                (14336 + 8, 512, 64), (4096, 384, 16)]


@pytest.mark.parametrize("N,K,gs", GROUP_SHAPES)
@pytest.mark.parametrize("m", [1, 2, 7, 8, 9, 16, 17, 31, 32])
def test_gemm_smallm_tile_groups(N, K, gs, m):
    W, g = make(11, N, K, gs)
    X = synth.activations(g, m, K)
    ref = oracle.gemm(*W.host, gs, X)
    assert_close(run_gemm(W, X, m, mq.MLXQ_GEMM_SMALLM_GROUPS), ref, f"smallm-groups m={m} {N}x{K}")


# the tcgen05 small-m kernel: K % 128 == 0, gs 16..128 with (K/gs) % 8 == 0;
# several tile groups per CTA, partial last groups, a ragged last tile
TCSM_SHAPES = [(512, 1024, 64), (300, 4096, 32), (77, 512, 16), (5000, 1152, 16), (2100, 2304, 32),
               (14336 + 8, 512, 64), (256, 14336, 128), (40000 + 3, 1024, 128)]


@pytest.mark.parametrize("N,K,gs", TCSM_SHAPES)
@pytest.mark.parametrize("m", [1, 9, 16, 17, 32, 33, 64])
def test_gemm_smallm_tcgen05(N, K, gs, m):
    W, g = make(13, N, K, gs)
    X = synth.activations(g, m, K)
    ref = oracle.gemm(*W.host, gs, X)
    assert_close(run_gemm(W, X, m, mq.MLXQ_GEMM_SMALLM_TC), ref, f"smallm-tc m={m} {N}x{K}")
    if m > 32:
        assert_close(run_gemm(W, X, m, mq.MLXQ_GEMM_AUTO), ref, f"auto m={m} {N}x{K}")


def test_gemm_smallm_tile_groups_refuses_what_it_cannot_take():
    W, g = make(12, 256, 14336, 128)  # gs = 128: not taken
    X = dev(synth.activations(g, 4, 14336))
    Y = torch.empty(4 * 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mq.MlxqError) as e:
        mq.mlxq_gemm_with(W.w, X, Y.data_ptr(), 4, mq.MLXQ_GEMM_SMALLM_GROUPS)
    assert e.value.code == mq.MLXQ_ERR_UNSUPPORTED


@pytest.mark.parametrize("N,K,gs", SMALLM_SHAPES + [(300, 4096, 256)])
@pytest.mark.parametrize("m", [1, 2, 4, 5, 16, 32])
def test_gemm_smallm_fp32_pipes(N, K, gs, m):
    W, g = make(9, N, K, gs)
    X = synth.activations(g, m, K)
    ref = oracle.gemm(*W.host, gs, X)
    assert_close(run_gemm(W, X, m, mq.MLXQ_GEMM_SMALLM_FFMA), ref, f"smallm-ffma m={m} {N}x{K}")
    if m > 8:
        assert_close(run_gemm(W, X, m, mq.MLXQ_GEMM_AUTO), ref, f"auto m={m} {N}x{K}")


@pytest.mark.parametrize("m", [1, 3, 9])
def test_gemm_rows_path_and_generic_shapes(m):
    W, g = make(9, 45, 36, 12)  # generic shape: only the row passes take it
    X = synth.activations(g, m, 36)
    ref = oracle.gemm(*W.host, 12, X)
    assert_close(run_gemm(W, X, m, mq.MLXQ_GEMM_ROWS), ref)
    assert_close(run_gemm(W, X, m, mq.MLXQ_GEMM_AUTO), ref)


def test_gemm_m1_equals_gemv_bitwise():
    W, g = make(10, 1000, 4096, 64)
    x = synth.activations(g, 4096)
    assert np.array_equal(run_gemm(W, x.reshape(1, -1), 1)[0], run_gemv(W, x))


@pytest.mark.parametrize("NK", [(28672, 8192), (8192, 28672)])
@pytest.mark.parametrize("gs", [32, 64, 128])
def test_gemm_smallm_workload_sampled_rows(NK, gs):
    """The small-m batched-decode shapes at full size; the oracle checks a
    sample of 256 weight rows (first, last and random) for every m."""
    N, K = NK
    W, g = make(20 + gs, N, K, gs)
    pick = np.unique(np.concatenate([np.arange(64), np.arange(N - 64, N),
                                     np.random.default_rng(gs).choice(N, 128, replace=False)]))
    sub = rows_subset(W, pick)
    for m in (1, 2, 4, 8, 16, 32):
        X = synth.activations(g, m, K)
        got = run_gemm(W, X, m)
        ref = oracle.gemm(*sub, gs, X)
        assert_close(got[:, pick], ref, f"{N}x{K}/{gs} m={m}")


def test_empty_shapes():
    """N = 0: nothing is written; K = 0: y = 0 (plus the residual); m = 0: no-op."""
    e32, e16 = np.zeros((0, 16), np.uint32), np.zeros((0, 2), np.uint16)
    W0 = mq.MlxInt8Weight.load(synth.weight_blob("e", e32, e16, e16), "e", 32)
    y = Guarded(8)
    x = dev(synth.activations(synth.rng(1), 64))
    mq.mlxq_gemv(W0.handle, x, y.data_ptr())
    mq.mlxq_dequant(W0.handle, y.data_ptr())
    mq.mlxq_gemm(W0.handle, x, y.data_ptr(), 0)
    mq.mlxq_gemm(W0.handle, x, y.data_ptr(), 3)
    torch.cuda.synchronize()
    y.check_guards()
    assert np.all(y.value_bits() == 0x7FC1)
    W0.release()

    k32, k16 = np.zeros((16, 0), np.uint32), np.zeros((16, 0), np.uint16)
    Wk = mq.MlxInt8Weight.load(synth.weight_blob("k", k32, k16, k16), "k", 4)
    assert (Wk.out_features, Wk.in_features) == (16, 0)
    yk = torch.full((16,), 3.0, dtype=torch.bfloat16, device="cuda")
    mq.mlxq_gemv(Wk.handle, None, yk)
    assert np.all(host_bits(yk) & 0x7FFF == 0)
    r = dev(synth.activations(synth.rng(2), 16))
    mq.mlxq_gemv_silu_gate_resid(Wk.handle, None, None, r, yk)
    assert np.array_equal(host_bits(yk), host_bits(r))
    Wk.release()


# ---------------------------------------------------------------- tensor-core gemm
TC_SHAPES = [
    (128, 64, 64, 32),      # one tile, one k-block
    (256, 512, 64, 64),
    (300, 1040, 16, 100),   # ragged N, ragged K (16.25 k-blocks), ragged m
    (257, 4096, 128, 257),  # two m tiles, last one ragged
    (512, 2048, 32, 512),
    (1000, 960, 64, 333),
]


@pytest.mark.parametrize("N,K,gs,m", TC_SHAPES)
def test_gemm_tcgen05(N, K, gs, m):
    W, g = make(40, N, K, gs)
    X = synth.activations(g, m, K)
    ref = oracle.gemm(*W.host, gs, X)
    assert_close(run_gemm(W, X, m, mq.MLXQ_GEMM_TCGEN05), ref, f"tc {N}x{K}/{gs} m={m}")
    if m >= 64:
        assert_close(run_gemm(W, X, m, mq.MLXQ_GEMM_AUTO), ref, f"auto {N}x{K}/{gs} m={m}")


# Shapes with fewer tiles than SMs: the tile's K is split over several CTAs
# whose fp32 partials are summed by the last one to finish.
TC_SPLIT_SHAPES = [
    (256, 4096, 128, 64),   # 1 tile, 8 splits; 128-wide groups, so splits start inside a scale box
    (300, 3088, 16, 40),    # ragged K (48.25 k-blocks), 2 tiles x 6 splits
    (1000, 2048, 32, 200),  # 4 tiles x 4 splits, ragged N
    (130, 8192, 64, 17),    # one 32-column tile, 16 splits
    (256, 1088, 64, 48),    # 17 groups per row: scales by direct loads, 2 splits
]


@pytest.mark.parametrize("N,K,gs,m", TC_SPLIT_SHAPES)
def test_gemm_tcgen05_split_k(N, K, gs, m):
    W, g = make(41, N, K, gs)
    X = synth.activations(g, m, K)
    ref = oracle.gemm(*W.host, gs, X)
    y1 = run_gemm(W, X, m, mq.MLXQ_GEMM_TCGEN05)
    assert_close(y1, ref, f"tc split {N}x{K}/{gs} m={m}")
    # the partials are added in split order whichever CTA finishes last
    y2 = run_gemm(W, X, m, mq.MLXQ_GEMM_TCGEN05)
    assert np.array_equal(y1, y2)


# More tiles than SMs with a partial last wave: whole tiles fill the full
# waves and the last wave's tiles split K over the SMs it would leave idle.
# (N, K, gs, m) -> tiles: 149 (1 split tile), 160 (12 split tiles, BN 256),
# 151 with a ragged last weight tile and ragged m.
TC_TAIL_SHAPES = [
    (256 * 149, 1024, 64, 32),
    (256 * 40, 1024, 32, 1024),
    (256 * 150 + 77, 2048, 128, 40),
]


@pytest.mark.parametrize("N,K,gs,m", TC_TAIL_SHAPES)
def test_gemm_tcgen05_tail_split(N, K, gs, m):
    W, g = make(42, N, K, gs)
    X = synth.activations(g, m, K)
    y1 = run_gemm(W, X, m, mq.MLXQ_GEMM_TCGEN05)
    y2 = run_gemm(W, X, m, mq.MLXQ_GEMM_TCGEN05)
    assert np.array_equal(y1, y2)  # split tiles are summed in split order
    pick_w = np.unique(np.concatenate([tile_edges(N, 256), np.arange(N - 300, N),
                                       np.random.default_rng(N).choice(N, 64, replace=False)]))
    pick_x = np.unique(np.concatenate([tile_edges(m, 256), np.random.default_rng(m).choice(m, min(m, 24), replace=False)]))
    ref = oracle.gemm(*rows_subset(W, pick_w), gs, X[pick_x])
    assert_close(y1[np.ix_(pick_x, pick_w)], ref, f"tc tail {N}x{K}/{gs} m={m}")


def test_gemm_tcgen05_integer_weights_exact():
    # s = 1, b = 0 and small-integer X: every BF16 product and fp32 partial sum is
    # an exact integer below 2^24, so the tensor-core result must equal the
    # oracle's exact result bit for bit.
    g = np.random.default_rng(12)
    N, K, m = 256, 1024, 96
    q = g.integers(0, 256, size=(N, K), dtype=np.uint8)
    packed = q.reshape(N, K // 4, 4).view("<u4").reshape(N, K // 4).astype(np.uint32)
    s = np.full((N, K // 64), 0x3F80, np.uint16)
    b = np.zeros((N, K // 64), np.uint16)
    X = synth.to_bf16_bits(g.integers(-2, 3, size=(m, K)).astype(np.float32))
    W = DevWeight(packed, s, b, 64)
    assert np.array_equal(run_gemm(W, X, m, mq.MLXQ_GEMM_TCGEN05), oracle.gemm(packed, s, b, 64, X))


def tile_edges(n, tile):
    """First and last index of every `tile`-sized block of range(n) (the last
    block may be ragged)."""
    starts = np.arange(0, n, tile)
    return np.unique(np.concatenate([starts, np.minimum(starts + tile, n) - 1]))


@pytest.mark.parametrize("NK", [(4096, 14336), (14336, 4096)])
def test_gemm_prefill_workload_sampled(NK):
    """The prefill shapes at full size (m up to 8192, and a ragged m) through
    the tensor-core kernel.  The oracle checks, element by element, at least
    64 rows of X - the first and last row of every 256-row activation tile,
    the ragged last tile included, plus seeded random rows - against the
    first and last row of every 256-row weight tile plus seeded random
    weight rows."""
    N, K = NK
    W, g = make(50 + N // 1024, N, K, 64)
    pick_w = np.unique(np.concatenate([tile_edges(N, 256), np.random.default_rng(N).choice(N, 64, replace=False)]))
    sub = rows_subset(W, pick_w)
    for m in (512, 2048, 4096, 8192, 1000):
        X = synth.activations(g, m, K)
        got = run_gemm(W, X, m)  # auto: the tensor-core kernel at these m
        edges = tile_edges(m, 256)
        rest = np.setdiff1d(np.arange(m), edges)
        extra = np.random.default_rng(m).choice(rest, max(16, 64 - edges.size), replace=False)
        pick_x = np.unique(np.concatenate([edges, extra]))
        assert pick_x.size >= 64
        ref = oracle.gemm(*sub, 64, X[pick_x])
        assert_close(got[np.ix_(pick_x, pick_w)], ref, f"prefill {N}x{K} m={m}")
