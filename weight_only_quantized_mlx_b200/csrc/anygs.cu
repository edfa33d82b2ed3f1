// Vectorised kernels for any group size the format allows with 4-code words
// ("MlxInt8Weight" page, load: group_size only has to divide in_features):
// group_size % 4 == 0, in_features % 16 == 0.  The tensor-pipe and TMA
// kernels want group_size in {16, 32, 64, 128} (or a multiple of 16) and
// 16-byte aligned table rows; these take the rest (4, 8, 12, 20, 48, 96, ...,
// and tables of any length), still with 16-byte loads of the codes.
//
// A 4-code word never straddles a group (group_size % 4 == 0), so a word
// has one (scale, bias) pair.  A lane walks 16-code chunks k0, k0 + 512, ...
// of its rows and keeps the chunk's first group and its offset in the group
// up to date by addition, so no division runs in the loop.
//
//   k_anygs_gemv    y = W h (+ resid) with h = x rows (MT of them per pass)
//                   or silu(gate) * up; each warp takes two weight rows at a
//                   time (paired in fp32x2 operations), lanes split K, the
//                   activations sit in shared memory, and the weight element
//                   is the BF16 value dequantize_to writes
//   k_dequant_anygs dequantize_to: one 16-code chunk per thread per step, 32
//                   (or 2 x 16) bytes stored
#include <atomic>

#include "device_common.cuh"
#include "kernels.h"

namespace mlxq {
namespace {

constexpr int kAgWarps = 8;
constexpr int kAgThreads = kAgWarps * 32;
// chunks per lane whose loads are issued together: 4 with one activation row
// per pass, 2 with more (registers)
template <int MT>
constexpr int ag_unroll() { return MT == 1 ? 4 : 2; }

struct AgParams {
    const uint8_t* packed;   // [N, K] codes, 16-byte aligned rows
    const uint16_t* scales;  // [N, G]
    const uint16_t* biases;  // [N, G]
    const uint16_t* x;       // plain: X [m, K]
    const uint16_t* gate;    // silu modes: [K]
    const uint16_t* up;
    const uint16_t* resid;   // GEMV_SILU_RESID: [N]
    uint16_t* y;             // [m, N]
    int64_t N;
    int K, G, gs;
    int step_g, step_r;      // 512 codes = step_g groups + step_r codes
    int i0, mt;              // X rows i0 .. i0 + mt - 1 in this pass
};

__device__ __forceinline__ float silu_ag(float t) { return t / (1.0f + expf(-t)); }

// groups passed from the chunk's first group to word j: (r + 4 j) / gs for
// r < gs, with at most three steps (gs >= 4)
__device__ __forceinline__ int word_group_step(int r, int j, int gs) {
    const int t = r + 4 * j;
    return (t >= gs) + (t >= 2 * gs) + (t >= 3 * gs);
}

// The BF16-rounded weights of byte J of word u (row r0) and of word v (row
// r1), as an fp32 pair: paired subtract and fma, one two-value pack.
template <int J>
__device__ __forceinline__ float2 weight_pair(uint32_t u, uint32_t v, float2 s2, float2 b2) {
    const float2 q = __fadd2_rn(make_float2(code_magic<J>(u), code_magic<J>(v)), make_float2(-kMagic, -kMagic));
    const float2 f = __ffma2_rn(q, s2, b2);
    const uint32_t w = pack_bf16x2(f.x, f.y);
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// MT: activation rows per pass (plain mode); 1 for the silu modes.
template <int MODE, int MT>
__global__ void __launch_bounds__(kAgThreads) k_anygs_gemv(const AgParams p) {
    constexpr int kAgUnroll = ag_unroll<MT>();
    extern __shared__ __align__(16) uint8_t smem_ag[];
    const int lane = threadIdx.x & 31;
    const int K = p.K;
    // activations: plain -> BF16 [MT][K]; silu -> fp32 h [K]
    pdl_launch_dependents();
    pdl_wait();
    // (16-byte loads when the vectors are 16-byte aligned, K % 16 == 0 keeping
    // every row aligned; several loads in flight per thread either way)
    if (MODE == GEMV_PLAIN) {
        if ((reinterpret_cast<uintptr_t>(p.x) & 15u) == 0) {
            uint4* xs = reinterpret_cast<uint4*>(smem_ag);
            const int k8 = K / 8;
#pragma unroll 4
            for (int e = threadIdx.x; e < MT * k8; e += kAgThreads) {
                const int i = e / k8, c = e - i * k8;
                xs[e] = (i < p.mt) ? ldg_nc_v4(p.x + static_cast<int64_t>(p.i0 + i) * K + 8 * c)
                                   : make_uint4(0u, 0u, 0u, 0u);
            }
        } else {
            uint16_t* xs = reinterpret_cast<uint16_t*>(smem_ag);
#pragma unroll 8
            for (int e = threadIdx.x; e < MT * K; e += kAgThreads) {
                const int i = e / K, k = e - i * K;
                xs[e] = (i < p.mt) ? p.x[static_cast<int64_t>(p.i0 + i) * K + k] : uint16_t(0);
            }
        }
    } else {
        float* hs = reinterpret_cast<float*>(smem_ag);
        if (((reinterpret_cast<uintptr_t>(p.gate) | reinterpret_cast<uintptr_t>(p.up)) & 15u) == 0) {
#pragma unroll 2
            for (int c = threadIdx.x; c < K / 8; c += kAgThreads) {
                const uint4 gv = ldg_nc_v4(p.gate + 8 * c), uv = ldg_nc_v4(p.up + 8 * c);
                const uint32_t gg[4] = {gv.x, gv.y, gv.z, gv.w}, uu[4] = {uv.x, uv.y, uv.z, uv.w};
                float h[8];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    h[2 * i] = silu_ag(bf16_bits_to_f32(gg[i] & 0xFFFFu)) * bf16_bits_to_f32(uu[i] & 0xFFFFu);
                    h[2 * i + 1] = silu_ag(bf16_bits_to_f32(gg[i] >> 16)) * bf16_bits_to_f32(uu[i] >> 16);
                }
                reinterpret_cast<float4*>(hs)[2 * c] = make_float4(h[0], h[1], h[2], h[3]);
                reinterpret_cast<float4*>(hs)[2 * c + 1] = make_float4(h[4], h[5], h[6], h[7]);
            }
        } else {
#pragma unroll 8
            for (int k = threadIdx.x; k < K; k += kAgThreads)
                hs[k] = silu_ag(bf16_bits_to_f32(p.gate[k])) * bf16_bits_to_f32(p.up[k]);
        }
    }
    __syncthreads();

    const int64_t pairs = (p.N + 1) / 2;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * kAgWarps;
    const int chunks = K / 16;
    for (int64_t pr = static_cast<int64_t>(blockIdx.x) * kAgWarps + (threadIdx.x >> 5); pr < pairs; pr += warps) {
        const int64_t r0 = 2 * pr;
        const bool has1 = r0 + 1 < p.N;
        const int64_t r1 = has1 ? r0 + 1 : r0;
        const uint8_t* w0 = p.packed + r0 * K;
        const uint8_t* w1 = p.packed + r1 * K;
        const uint16_t* s0 = p.scales + r0 * p.G;
        const uint16_t* s1 = p.scales + r1 * p.G;
        const uint16_t* b0 = p.biases + r0 * p.G;
        const uint16_t* b1 = p.biases + r1 * p.G;
        float2 acc[MT];  // (row r0, row r1)
#pragma unroll
        for (int i = 0; i < MT; ++i) acc[i] = make_float2(0.f, 0.f);
        // the lane's first chunk starts at code 16 * lane
        int g = (16 * lane) / p.gs;
        int r = 16 * lane - g * p.gs;
        for (int c0 = lane; c0 < chunks; c0 += 32 * kAgUnroll) {
            uint4 q0[kAgUnroll], q1[kAgUnroll];
            float sc0[kAgUnroll][4], bi0[kAgUnroll][4], sc1[kAgUnroll][4], bi1[kAgUnroll][4];
            int gu = g, ru = r;
#pragma unroll
            for (int u = 0; u < kAgUnroll; ++u) {
                const int c = c0 + 32 * u;
                if (c < chunks) {
                    q0[u] = ldg_nc_v4(w0 + 16 * c);
                    q1[u] = ldg_nc_v4(w1 + 16 * c);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int gj = gu + word_group_step(ru, j, p.gs);
                        sc0[u][j] = bf16_bits_to_f32(__ldg(s0 + gj));
                        bi0[u][j] = bf16_bits_to_f32(__ldg(b0 + gj));
                        sc1[u][j] = bf16_bits_to_f32(__ldg(s1 + gj));
                        bi1[u][j] = bf16_bits_to_f32(__ldg(b1 + gj));
                    }
                }
                // next chunk of this lane: 512 codes on
                gu += p.step_g;
                ru += p.step_r;
                if (ru >= p.gs) {
                    ru -= p.gs;
                    ++gu;
                }
            }
            g = gu;
            r = ru;
#pragma unroll
            for (int u = 0; u < kAgUnroll; ++u) {
                const int c = c0 + 32 * u;
                if (c < chunks) {
                    const uint32_t a0[4] = {q0[u].x, q0[u].y, q0[u].z, q0[u].w};
                    const uint32_t a1[4] = {q1[u].x, q1[u].y, q1[u].z, q1[u].w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        // the two rows side by side in paired fp32 operations
                        const float2 s2 = make_float2(sc0[u][j], sc1[u][j]);
                        const float2 b2 = make_float2(bi0[u][j], bi1[u][j]);
                        float2 v[4];
                        v[0] = weight_pair<0>(a0[j], a1[j], s2, b2);
                        v[1] = weight_pair<1>(a0[j], a1[j], s2, b2);
                        v[2] = weight_pair<2>(a0[j], a1[j], s2, b2);
                        v[3] = weight_pair<3>(a0[j], a1[j], s2, b2);
                        const int k = 16 * c + 4 * j;
                        if (MODE == GEMV_PLAIN) {
                            const uint16_t* xs = reinterpret_cast<const uint16_t*>(smem_ag);
#pragma unroll
                            for (int i = 0; i < MT; ++i) {
                                const uint2 xv = *reinterpret_cast<const uint2*>(xs + i * K + k);
                                const float x0 = __uint_as_float(xv.x << 16), x1 = __uint_as_float(xv.x & 0xFFFF0000u);
                                const float x2 = __uint_as_float(xv.y << 16), x3 = __uint_as_float(xv.y & 0xFFFF0000u);
                                acc[i] = __ffma2_rn(v[0], make_float2(x0, x0), acc[i]);
                                acc[i] = __ffma2_rn(v[1], make_float2(x1, x1), acc[i]);
                                acc[i] = __ffma2_rn(v[2], make_float2(x2, x2), acc[i]);
                                acc[i] = __ffma2_rn(v[3], make_float2(x3, x3), acc[i]);
                            }
                        } else {
                            const float4 h = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(smem_ag) + k);
                            acc[0] = __ffma2_rn(v[0], make_float2(h.x, h.x), acc[0]);
                            acc[0] = __ffma2_rn(v[1], make_float2(h.y, h.y), acc[0]);
                            acc[0] = __ffma2_rn(v[2], make_float2(h.z, h.z), acc[0]);
                            acc[0] = __ffma2_rn(v[3], make_float2(h.w, h.w), acc[0]);
                        }
                    }
                }
            }
        }
        // the lanes' partial sums, in a fixed butterfly order
        float acc0[MT], acc1[MT];
#pragma unroll
        for (int i = 0; i < MT; ++i) {
            acc0[i] = acc[i].x;
            acc1[i] = acc[i].y;
        }
#pragma unroll
        for (int i = 0; i < MT; ++i) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                acc0[i] += __shfl_xor_sync(0xFFFFFFFFu, acc0[i], o);
                acc1[i] += __shfl_xor_sync(0xFFFFFFFFu, acc1[i], o);
            }
        }
        if (lane == 0) {
#pragma unroll
            for (int i = 0; i < MT; ++i) {
                if (i < p.mt) {
                    float y0 = acc0[i], y1 = acc1[i];
                    if (MODE == GEMV_SILU_RESID) {
                        y0 += bf16_bits_to_f32(p.resid[r0]);
                        if (has1) y1 += bf16_bits_to_f32(p.resid[r1]);
                    }
                    uint16_t* yrow = p.y + static_cast<int64_t>(p.i0 + i) * p.N;
                    yrow[r0] = __bfloat16_as_ushort(__float2bfloat16_rn(y0));
                    if (has1) yrow[r1] = __bfloat16_as_ushort(__float2bfloat16_rn(y1));
                }
            }
        }
    }
}

// dequantize_to: one 16-code chunk per thread per step over a balanced
// contiguous range per block; V8 as in the group-size-16 kernel.
template <bool V8>
__global__ void __launch_bounds__(256) k_dequant_anygs(const uint8_t* __restrict__ packed,
                                                       const uint16_t* __restrict__ scales,
                                                       const uint16_t* __restrict__ biases,
                                                       uint4* __restrict__ out, uint64_t nchunks,
                                                       uint32_t chunks_per_row, uint32_t gs, uint32_t G) {
    pdl_launch_dependents();
    pdl_wait();
    const uint64_t lo = nchunks * blockIdx.x / gridDim.x;
    const uint64_t hi = nchunks * (blockIdx.x + 1) / gridDim.x;
    for (uint64_t c = lo + threadIdx.x; c < hi; c += 256) {
        const uint32_t n = static_cast<uint32_t>(c / chunks_per_row);
        const uint32_t k0 = 16u * static_cast<uint32_t>(c - static_cast<uint64_t>(n) * chunks_per_row);
        const uint32_t g0 = k0 / gs;
        const int r = static_cast<int>(k0 - g0 * gs);
        const uint4 wq = ldg_nc_v4(packed + 16 * c);
        const uint32_t words[4] = {wq.x, wq.y, wq.z, wq.w};
        uint32_t o[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint64_t gi = static_cast<uint64_t>(n) * G + g0 + word_group_step(r, j, static_cast<int>(gs));
            const float s = bf16_bits_to_f32(__ldg(scales + gi));
            const float b = bf16_bits_to_f32(__ldg(biases + gi));
            const uint32_t w = words[j];
            o[2 * j] = pack_bf16x2(__fmaf_rn(s, code_magic<0>(w) - kMagic, b), __fmaf_rn(s, code_magic<1>(w) - kMagic, b));
            o[2 * j + 1] = pack_bf16x2(__fmaf_rn(s, code_magic<2>(w) - kMagic, b), __fmaf_rn(s, code_magic<3>(w) - kMagic, b));
        }
        uint4* dst = out + 2 * c;
        if constexpr (V8) {
            stg_cs_v8(dst, o);
        } else {
            __stcs(dst, make_uint4(o[0], o[1], o[2], o[3]));
            __stcs(dst + 1, make_uint4(o[4], o[5], o[6], o[7]));
        }
    }
}

inline bool al(const void* q, uintptr_t a) { return (reinterpret_cast<uintptr_t>(q) & (a - 1)) == 0; }

// Shared memory of the activations: plain MT x K BF16, silu K fp32.
size_t ag_smem(int mode, int mt, int64_t K) {
    return mode == GEMV_PLAIN ? static_cast<size_t>(mt) * K * 2 : static_cast<size_t>(K) * 4;
}

constexpr size_t kAgSmemMax = 112 * 1024;  // two blocks per SM

bool ag_shape_ok(const WeightView& w) {
    return w.K >= 16 && w.K % 16 == 0 && w.gs >= 4 && w.gs % 4 == 0 && w.K <= (1 << 20) && al(w.packed, 16) &&
           w.N <= (int64_t{1} << 40);
}

template <int MODE, int MT>
cudaError_t launch_ag_t(const AgParams& p, size_t smem, cudaStream_t stream) {
    auto kern = k_anygs_gemv<MODE, MT>;
    static std::atomic<int> configured[64];
    cudaError_t e = ensure_dynamic_smem(kern, smem, configured);
    if (e != cudaSuccess) return e;
    const int sms = device_info().sm_count;
    const int64_t pairs = (p.N + 1) / 2;
    const int64_t want = (pairs + kAgWarps - 1) / kAgWarps;
    const int64_t cap = static_cast<int64_t>(sms) * (smem > kAgSmemMax / 2 ? 2 : 4);
    const int grid = static_cast<int>(want < cap ? want : cap);
    return launch_pdl(kern, dim3(grid), dim3(kAgThreads), smem, stream, p);
}

AgParams ag_params(const WeightView& w) {
    AgParams p{};
    p.packed = reinterpret_cast<const uint8_t*>(w.packed);
    p.scales = w.scales;
    p.biases = w.biases;
    p.N = w.N;
    p.K = static_cast<int>(w.K);
    p.G = static_cast<int>(w.G);
    p.gs = static_cast<int>(w.gs);
    p.step_g = 512 / p.gs;
    p.step_r = 512 % p.gs;
    return p;
}

}  // namespace

bool anygs_gemv_supported(const WeightView& w, int mode) {
    return ag_shape_ok(w) && ag_smem(mode, 1, w.K) <= kAgSmemMax;
}

cudaError_t launch_anygs_gemv(const WeightView& w, int mode, const void* x, const void* gate, const void* up,
                              const void* resid, void* y, cudaStream_t stream) {
    if (!anygs_gemv_supported(w, mode)) return cudaErrorInvalidValue;
    AgParams p = ag_params(w);
    p.x = static_cast<const uint16_t*>(x);
    p.gate = static_cast<const uint16_t*>(gate);
    p.up = static_cast<const uint16_t*>(up);
    p.resid = static_cast<const uint16_t*>(resid);
    p.y = static_cast<uint16_t*>(y);
    p.i0 = 0;
    p.mt = 1;
    const size_t smem = ag_smem(mode, 1, w.K);
    switch (mode) {
        case GEMV_PLAIN: return launch_ag_t<GEMV_PLAIN, 1>(p, smem, stream);
        case GEMV_SILU: return launch_ag_t<GEMV_SILU, 1>(p, smem, stream);
        default: return launch_ag_t<GEMV_SILU_RESID, 1>(p, smem, stream);
    }
}

bool anygs_gemm_supported(const WeightView& w, int64_t m) {
    return m >= 1 && m <= (int64_t{1} << 31) && ag_shape_ok(w) && ag_smem(GEMV_PLAIN, 1, w.K) <= kAgSmemMax;
}

// Passes of up to 8 X rows (fewer when K is long: the rows must fit in
// shared memory); every pass streams the weight once.
cudaError_t launch_anygs_gemm(const WeightView& w, const void* X, void* Y, int64_t m, cudaStream_t stream) {
    if (!anygs_gemm_supported(w, m)) return cudaErrorInvalidValue;
    AgParams p = ag_params(w);
    p.x = static_cast<const uint16_t*>(X);
    p.y = static_cast<uint16_t*>(Y);
    int mt_max = 8;
    while (mt_max > 1 && ag_smem(GEMV_PLAIN, mt_max, w.K) > kAgSmemMax) mt_max /= 2;
    for (int64_t i0 = 0; i0 < m; i0 += mt_max) {
        const int64_t left = m - i0;
        p.i0 = static_cast<int>(i0);
        p.mt = static_cast<int>(left < mt_max ? left : mt_max);
        const int mt = p.mt > 4 ? 8 : (p.mt > 2 ? 4 : p.mt);  // instantiated widths: 1, 2, 4, 8
        const size_t smem = ag_smem(GEMV_PLAIN, mt, w.K);
        cudaError_t e;
        switch (mt) {
            case 1: e = launch_ag_t<GEMV_PLAIN, 1>(p, smem, stream); break;
            case 2: e = launch_ag_t<GEMV_PLAIN, 2>(p, smem, stream); break;
            case 4: e = launch_ag_t<GEMV_PLAIN, 4>(p, smem, stream); break;
            default: e = launch_ag_t<GEMV_PLAIN, 8>(p, smem, stream); break;
        }
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

bool anygs_dequant_supported(const WeightView& w, const void* out) {
    return ag_shape_ok(w) && al(out, 16) && w.K / 16 < (int64_t{1} << 32) && w.G < (int64_t{1} << 32);
}

cudaError_t launch_anygs_dequant(const WeightView& w, void* out, cudaStream_t stream) {
    if (!anygs_dequant_supported(w, out)) return cudaErrorInvalidValue;
    const uint64_t nchunks = static_cast<uint64_t>(w.N) * static_cast<uint64_t>(w.K / 16);
    if (nchunks == 0) return cudaSuccess;
    const int sms = device_info().sm_count;
    const uint64_t want = (nchunks + 255) / 256;
    const uint64_t cap = static_cast<uint64_t>(sms) * 8;
    const int blocks = static_cast<int>(want < cap ? want : cap);
    const bool v8 = al(out, 32);
    auto kern = v8 ? k_dequant_anygs<true> : k_dequant_anygs<false>;
    return launch_pdl(kern, dim3(blocks), dim3(256), 0, stream, reinterpret_cast<const uint8_t*>(w.packed),
                      w.scales, w.biases, reinterpret_cast<uint4*>(out), nchunks,
                      static_cast<uint32_t>(w.K / 16), static_cast<uint32_t>(w.gs), static_cast<uint32_t>(w.G));
}

}  // namespace mlxq
