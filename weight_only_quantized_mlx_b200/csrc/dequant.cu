// mlx_int8_dequant ("MlxInt8Weight" page, dequantize_to): write the full
// weight as BF16, out[n, k] = bf16_rne(fma_f32(scale[n,g], q[n,k], bias[n,g])).
//
// HBM-bound streaming kernel: each thread turns one 16-byte word group (16
// codes) into two 16-byte BF16 stores.  s*q is exact in fp32, so the only
// roundings are the fp32 add inside the fma and the final RNE to BF16; the
// result is bit-identical to any correct fp32 implementation of the formula.
#include <cuda_fp16.h>

#include <atomic>
#include <cstring>

#include "device_common.cuh"
#include "kernels.h"

namespace mlxq {
namespace {

// Fast path: K % 16 == 0, group_size % 16 == 0, 16-byte aligned buffers.
// A chunk is 16 codes (one 16-byte load, 32 bytes stored) and never
// straddles a group.  Each block owns a balanced contiguous range of chunks
// and walks it kDqU * 256 chunks per step; a thread issues all kDqU loads
// (and their table loads) before its first store, so each SM keeps enough
// bytes in flight to cover HBM latency.
// The grid is one resident wave and is launched as a programmatic dependent:
// the output is written only after the previous kernel on the stream has
// finished; a weight marked static is also read before that point.
// V8: the output is 32-byte aligned and each chunk is one 32-byte store
// (whole sectors); otherwise two 16-byte stores.
constexpr int kDqU = 4;
template <bool V8>
__global__ void __launch_bounds__(256) k_dequant_vec16(const uint4* __restrict__ packed,
                                                       const uint16_t* __restrict__ scales,
                                                       const uint16_t* __restrict__ biases,
                                                       uint4* __restrict__ out, uint32_t nchunks,
                                                       uint32_t chunks_per_row, uint32_t chunks_per_group,
                                                       uint32_t G, int pre_wait) {
    pdl_launch_dependents();
    bool waited = pre_wait == 0;
    if (waited) pdl_wait();
    // this block's share: a balanced contiguous range of chunks
    const uint64_t lo = static_cast<uint64_t>(nchunks) * blockIdx.x / gridDim.x;
    const uint64_t hi = static_cast<uint64_t>(nchunks) * (blockIdx.x + 1) / gridDim.x;
    for (uint64_t base = lo; base < hi; base += kDqU * 256u) {
        uint4 wq[kDqU];
        float s[kDqU], b[kDqU];
#pragma unroll
        for (int u = 0; u < kDqU; ++u) {
            const uint64_t c = base + u * 256u + threadIdx.x;
            if (c < hi) {
                const uint32_t n = static_cast<uint32_t>(c) / chunks_per_row;
                const uint32_t j = static_cast<uint32_t>(c) - n * chunks_per_row;
                const uint64_t gi = static_cast<uint64_t>(n) * G + j / chunks_per_group;
                wq[u] = ldg_nc_v4(packed + c);
                s[u] = bf16_bits_to_f32(__ldg(scales + gi));
                b[u] = bf16_bits_to_f32(__ldg(biases + gi));
            }
        }
        if (!waited) {
            pdl_wait();
            waited = true;
        }
#pragma unroll
        for (int u = 0; u < kDqU; ++u) {
            const uint64_t c = base + u * 256u + threadIdx.x;
            if (c < hi) {
                const uint32_t words[4] = {wq[u].x, wq[u].y, wq[u].z, wq[u].w};
                uint32_t o[8];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t w = words[i];
                    const float q0 = code_magic<0>(w) - kMagic;
                    const float q1 = code_magic<1>(w) - kMagic;
                    const float q2 = code_magic<2>(w) - kMagic;
                    const float q3 = code_magic<3>(w) - kMagic;
                    o[2 * i] = pack_bf16x2(__fmaf_rn(s[u], q0, b[u]), __fmaf_rn(s[u], q1, b[u]));
                    o[2 * i + 1] = pack_bf16x2(__fmaf_rn(s[u], q2, b[u]), __fmaf_rn(s[u], q3, b[u]));
                }
                uint4* dst = out + 2ull * c;
                if constexpr (V8) {
                    stg_cs_v8(dst, o);
                } else {
                    __stcs(dst, make_uint4(o[0], o[1], o[2], o[3]));
                    __stcs(dst + 1, make_uint4(o[4], o[5], o[6], o[7]));
                }
            }
        }
    }
    if (!waited) pdl_wait();
}

// Any shape the format allows (K % 4 == 0, any group_size dividing K, any
// 2-byte aligned output): one thread per packed word, scalar stores.
__global__ void __launch_bounds__(256) k_dequant_generic(const uint32_t* __restrict__ packed,
                                                         const uint16_t* __restrict__ scales,
                                                         const uint16_t* __restrict__ biases,
                                                         uint16_t* __restrict__ out, int64_t nwords,
                                                         int64_t K, int64_t gs, int64_t G) {
    const int64_t wpr = K / 4;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t wi = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; wi < nwords;
         wi += stride) {
        const int64_t n = wi / wpr;
        const int64_t k0 = (wi - n * wpr) * 4;
        const uint32_t w = packed[wi];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t k = k0 + j;
            const int64_t gi = n * G + k / gs;
            const float s = bf16_bits_to_f32(scales[gi]);
            const float b = bf16_bits_to_f32(biases[gi]);
            const float q = static_cast<float>((w >> (8 * j)) & 0xFFu);
            const __nv_bfloat16 v = __float2bfloat16_rn(__fmaf_rn(s, q, b));
            out[n * K + k] = *reinterpret_cast<const uint16_t*>(&v);
        }
    }
}

// dequantize_to in a wider format (no page entry; the dequant-to-f16/f32
// variants of the quantized-storage page): FP32 keeps the fma result itself,
// FP16 rounds it to nearest even.  One thread per packed word (4 outputs),
// one vector store when the output is aligned for it.
template <typename T>
__global__ void __launch_bounds__(256) k_dequant_wide(const uint32_t* __restrict__ packed,
                                                      const uint16_t* __restrict__ scales,
                                                      const uint16_t* __restrict__ biases, T* __restrict__ out,
                                                      int64_t nwords, int64_t K, int64_t gs, int64_t G, bool vec) {
    const int64_t wpr = K / 4;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t wi = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; wi < nwords; wi += stride) {
        const int64_t n = wi / wpr;
        const int64_t k0 = (wi - n * wpr) * 4;
        const uint32_t w = __ldg(packed + wi);
        float v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t gi = n * G + (k0 + j) / gs;
            v[j] = __fmaf_rn(bf16_bits_to_f32(__ldg(scales + gi)), static_cast<float>((w >> (8 * j)) & 0xFFu),
                             bf16_bits_to_f32(__ldg(biases + gi)));
        }
        T* dst = out + n * K + k0;
        if constexpr (sizeof(T) == 4) {
            if (vec) {
                __stcs(reinterpret_cast<float4*>(dst), make_float4(v[0], v[1], v[2], v[3]));
            } else {
#pragma unroll
                for (int j = 0; j < 4; ++j) dst[j] = v[j];
            }
        } else {
            const __half h[4] = {__float2half_rn(v[0]), __float2half_rn(v[1]), __float2half_rn(v[2]),
                                 __float2half_rn(v[3])};
            if (vec) {
                uint2 u;
                std::memcpy(&u, h, 8);
                *reinterpret_cast<uint2*>(dst) = u;
            } else {
#pragma unroll
                for (int j = 0; j < 4; ++j) dst[j] = h[j];
            }
        }
    }
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

cudaError_t launch_dequant(const WeightView& w, void* out, cudaStream_t stream) {
    const int64_t total = w.N * w.K;
    if (total == 0) return cudaSuccess;
    const int sms = device_info().sm_count;
    const bool vec = (w.K % 16 == 0) && (w.gs % 16 == 0) && aligned16(w.packed) &&
                     aligned16(out) && total / 16 < (int64_t{1} << 32) && w.G < (int64_t{1} << 32);
    if (vec) {
        const int64_t nchunks = total / 16;
        const int64_t tiles = (nchunks + kDqU * 256 - 1) / (kDqU * 256);
        const bool v8 = (reinterpret_cast<uintptr_t>(out) & 31u) == 0;
        auto kern = v8 ? k_dequant_vec16<true> : k_dequant_vec16<false>;
        static std::atomic<int> per_sm[2];  // resident blocks per SM, asked once per variant
        if (per_sm[v8].load() == 0) {
            int b = 0;
            cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kern, 256, 0);
            if (e != cudaSuccess) return e;
            per_sm[v8].store(b > 0 ? b : 1);
        }
        const int64_t wave = static_cast<int64_t>(sms) * per_sm[v8].load();  // one resident wave
        const int blocks = static_cast<int>(tiles < wave ? tiles : wave);
        const int pre_wait = (w.flags & MLXQ_WEIGHT_STATIC) ? 1 : 0;
        cudaError_t e = launch_pdl(kern, dim3(blocks), dim3(256), 0, stream,
                                   reinterpret_cast<const uint4*>(w.packed), w.scales, w.biases,
                                   reinterpret_cast<uint4*>(out), static_cast<uint32_t>(nchunks),
                                   static_cast<uint32_t>(w.K / 16), static_cast<uint32_t>(w.gs / 16),
                                   static_cast<uint32_t>(w.G), pre_wait);
        if (e != cudaSuccess) return e;
    } else if (anygs_dequant_supported(w, out)) {
        return launch_anygs_dequant(w, out, stream);
    } else {
        const int64_t nwords = total / 4;
        int64_t blocks = (nwords + 255) / 256;
        const int64_t cap = static_cast<int64_t>(sms) * 32;
        if (blocks > cap) blocks = cap;
        k_dequant_generic<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
            w.packed, w.scales, w.biases, static_cast<uint16_t*>(out), nwords, w.K, w.gs, w.G);
    }
    return cudaGetLastError();
}

cudaError_t launch_dequant_as(const WeightView& w, void* out, int dtype, cudaStream_t stream) {
    if (dtype == 0) return launch_dequant(w, out, stream);  // BF16: the page's dequantize_to
    const int64_t nwords = w.N * w.K / 4;
    if (nwords == 0) return cudaSuccess;
    int64_t blocks = (nwords + 255) / 256;
    const int64_t cap = static_cast<int64_t>(device_info().sm_count) * 32;
    if (blocks > cap) blocks = cap;
    const uintptr_t a = reinterpret_cast<uintptr_t>(out);
    if (dtype == 2) {
        k_dequant_wide<float><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
            w.packed, w.scales, w.biases, static_cast<float*>(out), nwords, w.K, w.gs, w.G, (a & 15u) == 0);
    } else {
        k_dequant_wide<__half><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
            w.packed, w.scales, w.biases, static_cast<__half*>(out), nwords, w.K, w.gs, w.G, (a & 7u) == 0);
    }
    return cudaGetLastError();
}

}  // namespace mlxq
