// The m = 1 kernels of the "MlxInt8Weight" page: mlx_int8_gemv (y = W x),
// mlx_int8_gemv_silu_gate (y = W (silu(gate)*up)) and gemv_silu_gate_resid
// (the same plus x_resid), as one HBM-streaming kernel with a compile-time
// prologue/epilogue mode.
//
// Design (sm_100a):
//  * One CTA per SM owns a contiguous range of weight rows.  Because the
//    packed weight is row-major, those rows are one contiguous byte range;
//    a producer lane streams them into a ring of shared-memory stages with
//    1-D bulk copies (cp.async.bulk, L2 evict-first), B rows per stage, the
//    matching scale and bias rows alongside.  Completion is an mbarrier
//    transaction count; consumers free a stage with an mbarrier arrive.
//  * Consumer thread t owns the same 16-code chunks of every row (chunk
//    c = t + j*T), so its slice of h = x (or silu(gate)*up, fp32, computed
//    once in registers, not stored to global memory) is loaded once.
//  * Per chunk: unpack 16 codes (byte -> fp32 through the 2^23 exponent
//    trick), w = fma(s, q, b) in fp32, round to BF16 (so W equals the BF16
//    weight the page's dequantize_to produces), fp32 FMA with h, using the
//    paired fp32 instructions (FFMA2/FADD2) of sm_100.
//  * Rows are reduced in groups of 8: a transposing butterfly across the
//    warp (4 shuffles per row per thread instead of 5 per row per value),
//    then the warps' partial sums through shared memory, in a fixed order.
//  * Every pipeline wait is bounded (device_common.cuh).
#include "device_common.cuh"
#include "kernels.h"

namespace mlxq {
namespace {

struct GemvParams {
    const uint8_t* packed;  // [N, K] bytes (uint32 words viewed as bytes)
    const uint16_t* scales;
    const uint16_t* biases;
    const uint16_t* x;
    const uint16_t* gate;
    const uint16_t* up;
    const uint16_t* resid;
    uint16_t* y;
    int64_t N;
    int K, G, C, cpg;  // C = K/16 chunks per row; cpg = group_size/16
    int T;             // consumer threads (multiple of 32)
    int S;             // pipeline stages
    int i0;            // first X row of this pass (small-m gemm)
    uint32_t stage_bytes;
    unsigned int* status;
};

// The 16 BF16 weights of one 16-byte chunk, as fp32 pairs:
// w[i] = bf16(fma(s, q[2i], b)), bf16(fma(s, q[2i+1], b)).
__device__ __forceinline__ void dequant16(uint4 wq, float s, float b, float2 (&w)[8]) {
    const float2 s2 = make_float2(s, s);
    const float2 b2 = make_float2(b, b);
    const float2 m2 = make_float2(-kMagic, -kMagic);
    const uint32_t words[4] = {wq.x, wq.y, wq.z, wq.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t u = words[i];
        const float2 q01 = __fadd2_rn(make_float2(code_magic<0>(u), code_magic<1>(u)), m2);
        const float2 q23 = __fadd2_rn(make_float2(code_magic<2>(u), code_magic<3>(u)), m2);
        w[2 * i] = round_bf16x2(__ffma2_rn(q01, s2, b2));
        w[2 * i + 1] = round_bf16x2(__ffma2_rn(q23, s2, b2));
    }
}

// sum_i w_i * h_i over one chunk (two interleaved fp32 partial sums).
__device__ __forceinline__ float dot16(const float2 (&w)[8], const float2* h) {
    float2 acc = __fmul2_rn(w[0], h[0]);
#pragma unroll
    for (int i = 1; i < 8; ++i) acc = __ffma2_rn(w[i], h[i], acc);
    return acc.x + acc.y;
}

// Reduce 8 per-row partials across a warp.  Returns, in every lane, the warp
// total of row (lane >> 2) & 7.
__device__ __forceinline__ float warp_reduce_rows8(const float (&p)[8], int lane) {
    const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
    float q4[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float send = b4 ? p[i] : p[i + 4];
        const float keep = b4 ? p[i + 4] : p[i];
        q4[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, 16);
    }
    float q2[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float send = b3 ? q4[i] : q4[i + 2];
        const float keep = b3 ? q4[i + 2] : q4[i];
        q2[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, 8);
    }
    const float send = b2 ? q2[0] : q2[1];
    const float keep = b2 ? q2[1] : q2[0];
    float v = keep + __shfl_xor_sync(0xFFFFFFFFu, send, 4);
    v += __shfl_xor_sync(0xFFFFFFFFu, v, 1);
    v += __shfl_xor_sync(0xFFFFFFFFu, v, 2);
    return v;
}

__device__ __forceinline__ float silu_f32(float t) { return t / (1.0f + expf(-t)); }

// MT activation rows per pass: MT = 1 for the gemv family, MT <= 4 for the
// CUDA-core small-m gemm (X rows i0 .. i0+MT-1; Y row-major [m, N]).
template <int MODE, int CPT, int B, int MT>
__global__ void __launch_bounds__(544, 1) k_gemv_stream(const GemvParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int T = p.T;
    const int S = p.S;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int nwc = T >> 5;

    uint8_t* stage_base = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(S) * p.stage_bytes);
    uint64_t* empty = full + S;
    float* red = reinterpret_cast<float*>(empty + S);  // [2][MT][8][nwc]

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), nwc);
        }
        mbar_fence_init();
    }
    __syncthreads();

    const int64_t rb = static_cast<int64_t>(blockIdx.x) * p.N / gridDim.x;
    const int64_t re = static_cast<int64_t>(blockIdx.x + 1) * p.N / gridDim.x;
    const uint32_t pk_bytes = static_cast<uint32_t>(B) * p.K;
    const uint32_t sb_bytes = static_cast<uint32_t>(B) * p.G * 2;

    if (warp == nwc) {
        // ---------------- producer ----------------
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            int t = 0;
            bool ok = true;
            for (int64_t g0 = rb; g0 < re; g0 += 8) {
                const int rows_g = static_cast<int>(re - g0 < 8 ? re - g0 : 8);
                for (int j = 0; j * B < rows_g; ++j, ++t) {
                    const int s = t % S;
                    if (t >= S && ok) ok = mbar_wait(smem_u32(&empty[s]), ((t / S) - 1) & 1, p.status);
                    const int nr = rows_g - j * B < B ? rows_g - j * B : B;
                    const int64_t r0 = g0 + j * B;
                    const uint32_t dst = smem_u32(stage_base + static_cast<size_t>(s) * p.stage_bytes);
                    const uint32_t bar = smem_u32(&full[s]);
                    const uint32_t wbytes = static_cast<uint32_t>(nr) * p.K;
                    const uint32_t sbytes = static_cast<uint32_t>(nr) * p.G * 2;
                    mbar_arrive_expect_tx(bar, wbytes + 2 * sbytes);
                    bulk_g2s(dst, p.packed + r0 * p.K, wbytes, bar, pol);
                    bulk_g2s(dst + pk_bytes, p.scales + r0 * p.G, sbytes, bar, pol);
                    bulk_g2s(dst + pk_bytes + sb_bytes, p.biases + r0 * p.G, sbytes, bar, pol);
                }
            }
            // Do not leave while copies may still be landing (only matters if
            // a wait above gave up).
            const int first = t > S ? t - S : 0;
            for (int u = first; u < t; ++u) {
                if (!mbar_wait(smem_u32(&full[u % S]), (u / S) & 1, p.status)) break;
            }
        }
        return;
    }

    // ---------------- consumers ----------------
    // this thread's chunks, their groups, and its slice of h (per X row)
    float2 h[MT][CPT][8];
    int cg[CPT];
    bool cval[CPT];
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
        const int c = tid + j * T;
        cval[j] = c < p.C;
        cg[j] = cval[j] ? c / p.cpg : 0;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            if (!cval[j]) {
#pragma unroll
                for (int i = 0; i < 8; ++i) h[mt][j][i] = make_float2(0.f, 0.f);
            } else if (MODE == GEMV_PLAIN) {
                const uint16_t* xr = p.x + static_cast<int64_t>(p.i0 + mt) * p.K + c * 16;
                const uint4 a = ldg_nc_v4(xr);
                const uint4 bq = ldg_nc_v4(xr + 8);
                const uint32_t u[8] = {a.x, a.y, a.z, a.w, bq.x, bq.y, bq.z, bq.w};
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    h[mt][j][i] = make_float2(bf16_bits_to_f32(u[i] & 0xFFFFu), bf16_bits_to_f32(u[i] >> 16));
            } else {
                const uint4 ga = ldg_nc_v4(p.gate + c * 16);
                const uint4 gb = ldg_nc_v4(p.gate + c * 16 + 8);
                const uint4 ua = ldg_nc_v4(p.up + c * 16);
                const uint4 ub = ldg_nc_v4(p.up + c * 16 + 8);
                const uint32_t g[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
                const uint32_t u[8] = {ua.x, ua.y, ua.z, ua.w, ub.x, ub.y, ub.z, ub.w};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float g0 = bf16_bits_to_f32(g[i] & 0xFFFFu), g1 = bf16_bits_to_f32(g[i] >> 16);
                    const float u0 = bf16_bits_to_f32(u[i] & 0xFFFFu), u1 = bf16_bits_to_f32(u[i] >> 16);
                    h[mt][j][i] = make_float2(silu_f32(g0) * u0, silu_f32(g1) * u1);
                }
            }
        }
    }

    bool ok = true;
    int t = 0;
    int buf = 0;
    for (int64_t g0 = rb; g0 < re; g0 += 8, buf ^= 1) {
        const int rows_g = static_cast<int>(re - g0 < 8 ? re - g0 : 8);
        float part[MT][8];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int i = 0; i < 8; ++i) part[mt][i] = 0.f;
#pragma unroll
        for (int j = 0; j < 8 / B; ++j) {
            if (j * B < rows_g) {
                const int s = t % S;
                if (ok) ok = mbar_wait(smem_u32(&full[s]), (t / S) & 1, p.status);
                const uint32_t base = smem_u32(stage_base + static_cast<size_t>(s) * p.stage_bytes);
                const int nr = rows_g - j * B < B ? rows_g - j * B : B;
#pragma unroll
                for (int b = 0; b < B; ++b) {
                    if (b < nr) {
#pragma unroll
                        for (int jc = 0; jc < CPT; ++jc) {
                            if (cval[jc]) {
                                const int c = tid + jc * T;
                                const uint4 wq = lds128(base + static_cast<uint32_t>(b) * p.K + c * 16);
                                const uint32_t sidx = static_cast<uint32_t>(b * p.G + cg[jc]) * 2;
                                const float sc = bf16_bits_to_f32(lds16(base + pk_bytes + sidx));
                                const float bi = bf16_bits_to_f32(lds16(base + pk_bytes + sb_bytes + sidx));
                                float2 w[8];
                                dequant16(wq, sc, bi, w);
#pragma unroll
                                for (int mt = 0; mt < MT; ++mt) part[mt][j * B + b] += dot16(w, h[mt][jc]);
                            }
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
                ++t;
            }
        }
        float* rbuf = red + buf * MT * 8 * nwc;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const float v = warp_reduce_rows8(part[mt], lane);
            if ((lane & 3) == 0) rbuf[(mt * 8 + ((lane >> 2) & 7)) * nwc + warp] = v;
        }
        named_bar_sync(1, T);
        // warp w finishes outputs w, w + nwc, ...: one partial per lane, then
        // a fixed shuffle tree (deterministic order)
        for (int o = warp; o < 8 * MT; o += nwc) {
            const int mt = o >> 3, r = o & 7;
            float acc = lane < nwc ? rbuf[(mt * 8 + r) * nwc + lane] : 0.f;
#pragma unroll
            for (int sh = 16; sh > 0; sh >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, sh);
            if (lane == 0 && r < rows_g) {
                const int64_t row = g0 + r;
                if (MODE == GEMV_SILU_RESID) acc += bf16_bits_to_f32(p.resid[row]);
                const __nv_bfloat16 ob = __float2bfloat16_rn(acc);
                p.y[static_cast<int64_t>(p.i0 + mt) * p.N + row] = *reinterpret_cast<const uint16_t*>(&ob);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Generic path: any K % 4 == 0, any group size, any 2-byte aligned vectors.
// One warp per row, one packed word per lane per step.
template <int MODE>
__global__ void __launch_bounds__(256) k_gemv_generic(const GemvParams p, int64_t gs) {
    const int warps = blockDim.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t wpr = p.K / 4;
    for (int64_t row = static_cast<int64_t>(blockIdx.x) * warps + (threadIdx.x >> 5); row < p.N;
         row += static_cast<int64_t>(gridDim.x) * warps) {
        const uint32_t* prow = reinterpret_cast<const uint32_t*>(p.packed) + row * wpr;
        float acc = 0.f;
        for (int64_t kw = lane; kw < wpr; kw += 32) {
            const uint32_t w = prow[kw];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int64_t k = kw * 4 + j;
                const int64_t gi = row * p.G + k / gs;
                const float wf = __bfloat162float(__float2bfloat16_rn(
                    __fmaf_rn(bf16_bits_to_f32(p.scales[gi]), static_cast<float>((w >> (8 * j)) & 0xFFu),
                              bf16_bits_to_f32(p.biases[gi]))));
                float hk;
                if (MODE == GEMV_PLAIN) {
                    hk = bf16_bits_to_f32(p.x[k]);
                } else {
                    hk = silu_f32(bf16_bits_to_f32(p.gate[k])) * bf16_bits_to_f32(p.up[k]);
                }
                acc = __fmaf_rn(wf, hk, acc);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
        if (lane == 0) {
            if (MODE == GEMV_SILU_RESID) acc += bf16_bits_to_f32(p.resid[row]);
            const __nv_bfloat16 o = __float2bfloat16_rn(acc);
            p.y[row] = *reinterpret_cast<const uint16_t*>(&o);
        }
    }
}

inline bool a16(const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; }

template <int MODE, int CPT, int B, int MT>
cudaError_t launch_stream_t(const GemvParams& p, int grid, size_t smem, cudaStream_t stream) {
    auto kern = k_gemv_stream<MODE, CPT, B, MT>;
    static std::atomic<int> configured[64];
    cudaError_t e = ensure_dynamic_smem(kern, smem, configured);
    if (e != cudaSuccess) return e;
    kern<<<grid, p.T + 32, smem, stream>>>(p);
    return cudaGetLastError();
}

// The (CPT, B) pairs that the host plan below can produce: CPT = 1 goes with
// B in {2, 4, 8} (K <= 8192), CPT = 2 and CPT = 4 with B = 1.
template <int MODE, int MT>
cudaError_t launch_stream_cb(const GemvParams& p, int CPT, int B, int grid, size_t smem,
                             cudaStream_t stream) {
    if (CPT == 1) {
        if (B == 8) return launch_stream_t<MODE, 1, 8, MT>(p, grid, smem, stream);
        if (B == 4) return launch_stream_t<MODE, 1, 4, MT>(p, grid, smem, stream);
        return launch_stream_t<MODE, 1, 2, MT>(p, grid, smem, stream);
    }
    if constexpr (MT <= 2) {
        if (CPT == 2) return launch_stream_t<MODE, 2, 1, MT>(p, grid, smem, stream);
    }
    if constexpr (MT == 1) {
        return launch_stream_t<MODE, 4, 1, MT>(p, grid, smem, stream);
    }
    return cudaErrorInvalidValue;
}

struct StreamPlan {
    bool vec;
    int CPT, B, T, S, grid;
    uint32_t stage_bytes;
    size_t smem;
};

StreamPlan plan_stream(const WeightView& w, bool acts_aligned, int max_mt) {
    const DeviceInfo& dev = device_info();
    StreamPlan pl{};
    pl.vec = w.K > 0 && w.K % 16 == 0 && w.gs % 16 == 0 && w.G % 8 == 0 && w.K <= 32768 &&
             a16(w.packed) && a16(w.scales) && a16(w.biases) && acts_aligned;
    if (!pl.vec) return pl;
    const int C = static_cast<int>(w.K / 16);
    pl.CPT = C <= 512 ? 1 : (C <= 1024 ? 2 : 4);
    pl.T = ((C + pl.CPT - 1) / pl.CPT + 31) / 32 * 32;
    pl.B = 1;
    if (pl.CPT == 1) {
        pl.B = 2;
        while (pl.B < 8 && static_cast<int64_t>(pl.B) * 2 * w.K <= 16384) pl.B *= 2;
    }
    const uint32_t stage = static_cast<uint32_t>(pl.B * w.K + 4 * pl.B * w.G);
    pl.stage_bytes = (stage + 127u) / 128u * 128u;
    const size_t tail = 2 * 8 * sizeof(uint64_t) + 2 * max_mt * 8 * (pl.T / 32) * sizeof(float);
    const size_t budget = static_cast<size_t>(dev.max_smem_optin) - tail - 256;
    int S = static_cast<int>(budget / pl.stage_bytes);
    if (S > 8) S = 8;
    if (S < 2) {
        pl.vec = false;
        return pl;
    }
    pl.S = S;
    pl.grid = static_cast<int>(w.N < dev.sm_count ? w.N : dev.sm_count);
    pl.smem = static_cast<size_t>(S) * pl.stage_bytes + 2 * S * sizeof(uint64_t) + tail;
    return pl;
}

GemvParams base_params(const WeightView& w, const StreamPlan& pl) {
    GemvParams p{};
    p.packed = reinterpret_cast<const uint8_t*>(w.packed);
    p.scales = w.scales;
    p.biases = w.biases;
    p.N = w.N;
    p.K = static_cast<int>(w.K);
    p.G = static_cast<int>(w.G);
    p.C = static_cast<int>(w.K / 16);
    p.cpg = static_cast<int>(w.gs / 16 > 0 ? w.gs / 16 : 1);
    p.T = pl.T;
    p.S = pl.S;
    p.stage_bytes = pl.stage_bytes;
    p.status = device_status_ptr();
    return p;
}

}  // namespace

cudaError_t launch_gemv(const WeightView& w, int mode, const void* x, const void* gate,
                        const void* up, const void* resid, void* y, cudaStream_t stream) {
    if (w.N == 0) return cudaSuccess;
    if (gemv_la_supported(w, mode, x, gate, up)) return launch_gemv_la(w, mode, x, gate, up, resid, y, stream);
    // Above 128 rows per SM (beyond k_gemv_la), the tile-group kernel at m = 1
    // (plain gemv only) measured faster than the per-row-pair stream kernel:
    // 28672x8192 3829 vs 3704 GB/s, 57344x4096 4042 vs 3379.
    if (mode == GEMV_PLAIN && (w.N + device_info().sm_count - 1) / device_info().sm_count > 128 &&
        smallm_supported(w, 1, x))
        return launch_smallm(w, x, y, 1, stream);
    if (stream_mma_supported(w, mode, 1, x, gate, up))
        return launch_stream_mma(w, mode, 1, x, gate, up, resid, y, stream);
    const bool acts_aligned = (mode == GEMV_PLAIN) ? a16(x) : (a16(gate) && a16(up));
    const StreamPlan pl = plan_stream(w, acts_aligned, 1);
    GemvParams p = base_params(w, pl);
    p.x = static_cast<const uint16_t*>(x);
    p.gate = static_cast<const uint16_t*>(gate);
    p.up = static_cast<const uint16_t*>(up);
    p.resid = static_cast<const uint16_t*>(resid);
    p.y = static_cast<uint16_t*>(y);
    p.i0 = 0;
    if (!pl.vec && anygs_gemv_supported(w, mode)) return launch_anygs_gemv(w, mode, x, gate, up, resid, y, stream);
    if (!pl.vec) {
        const int sms = device_info().sm_count;
        const int64_t blocks64 = (w.N + 7) / 8;
        const int blocks = static_cast<int>(blocks64 < sms * 16 ? blocks64 : sms * 16);
        switch (mode) {
            case GEMV_PLAIN: k_gemv_generic<GEMV_PLAIN><<<blocks, 256, 0, stream>>>(p, w.gs); break;
            case GEMV_SILU: k_gemv_generic<GEMV_SILU><<<blocks, 256, 0, stream>>>(p, w.gs); break;
            default: k_gemv_generic<GEMV_SILU_RESID><<<blocks, 256, 0, stream>>>(p, w.gs); break;
        }
        return cudaGetLastError();
    }
    switch (mode) {
        case GEMV_PLAIN: return launch_stream_cb<GEMV_PLAIN, 1>(p, pl.CPT, pl.B, pl.grid, pl.smem, stream);
        case GEMV_SILU: return launch_stream_cb<GEMV_SILU, 1>(p, pl.CPT, pl.B, pl.grid, pl.smem, stream);
        default: return launch_stream_cb<GEMV_SILU_RESID, 1>(p, pl.CPT, pl.B, pl.grid, pl.smem, stream);
    }
}

// ---- CUDA-core small-m gemm: passes of MT <= 4 X rows over the weight stream ----
static int max_mt_for(int CPT) { return CPT == 1 ? 4 : (CPT == 2 ? 2 : 1); }

bool gemm_smallm_supported(const WeightView& w, int64_t m) {
    if (m < 1 || m > kSmallMMax) return false;
    const StreamPlan pl = plan_stream(w, true, 4);
    return pl.vec;
}

cudaError_t launch_gemm_smallm(const WeightView& w, const void* X, void* Y, int64_t m,
                               cudaStream_t stream) {
    if (w.N == 0 || m == 0) return cudaSuccess;
    const StreamPlan pl0 = plan_stream(w, a16(X) && (w.K * 2) % 16 == 0, 4);
    if (!pl0.vec) return cudaErrorInvalidValue;
    const int max_mt = max_mt_for(pl0.CPT);
    const StreamPlan pl = plan_stream(w, true, max_mt);
    GemvParams p = base_params(w, pl);
    p.x = static_cast<const uint16_t*>(X);
    p.y = static_cast<uint16_t*>(Y);
    for (int64_t i0 = 0; i0 < m; i0 += max_mt) {
        const int mt = static_cast<int>(m - i0 < max_mt ? m - i0 : max_mt);
        p.i0 = static_cast<int>(i0);
        cudaError_t e;
        switch (mt) {
            case 1: e = launch_stream_cb<GEMV_PLAIN, 1>(p, pl.CPT, pl.B, pl.grid, pl.smem, stream); break;
            case 2: e = launch_stream_cb<GEMV_PLAIN, 2>(p, pl.CPT, pl.B, pl.grid, pl.smem, stream); break;
            case 3: e = launch_stream_cb<GEMV_PLAIN, 3>(p, pl.CPT, pl.B, pl.grid, pl.smem, stream); break;
            default: e = launch_stream_cb<GEMV_PLAIN, 4>(p, pl.CPT, pl.B, pl.grid, pl.smem, stream); break;
        }
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace mlxq
