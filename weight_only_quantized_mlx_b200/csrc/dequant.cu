// mlx_int8_dequant ("MlxInt8Weight" page, dequantize_to): write the full
// weight as BF16, out[n, k] = bf16_rne(fma_f32(scale[n,g], q[n,k], bias[n,g])).
//
// HBM-bound streaming kernel: each thread turns one 16-byte word group (16
// codes) into two 16-byte BF16 stores.  s*q is exact in fp32, so the only
// roundings are the fp32 add inside the fma and the final RNE to BF16; the
// result is bit-identical to any correct fp32 implementation of the formula.
#include <cuda_fp16.h>

#include <cstring>

#include "device_common.cuh"
#include "kernels.h"

namespace mlxq {
namespace {

// Fast path: K % 16 == 0, group_size % 16 == 0, 16-byte aligned buffers.
// One thread per 16-code chunk; a chunk never straddles a group.
__global__ void __launch_bounds__(256) k_dequant_vec16(const uint4* __restrict__ packed,
                                                       const uint16_t* __restrict__ scales,
                                                       const uint16_t* __restrict__ biases,
                                                       uint4* __restrict__ out, int64_t nchunks,
                                                       int64_t chunks_per_row,
                                                       int64_t chunks_per_group, int64_t G) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; c < nchunks;
         c += stride) {
        const int64_t n = c / chunks_per_row;
        const int64_t j = c - n * chunks_per_row;
        const int64_t gi = n * G + j / chunks_per_group;
        const uint4 wq = ldg_nc_v4(packed + c);
        const float s = bf16_bits_to_f32(__ldg(scales + gi));
        const float b = bf16_bits_to_f32(__ldg(biases + gi));
        const uint32_t words[4] = {wq.x, wq.y, wq.z, wq.w};
        uint32_t o[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t w = words[i];
            const float q0 = code_magic<0>(w) - kMagic;
            const float q1 = code_magic<1>(w) - kMagic;
            const float q2 = code_magic<2>(w) - kMagic;
            const float q3 = code_magic<3>(w) - kMagic;
            o[2 * i] = pack_bf16x2(__fmaf_rn(s, q0, b), __fmaf_rn(s, q1, b));
            o[2 * i + 1] = pack_bf16x2(__fmaf_rn(s, q2, b), __fmaf_rn(s, q3, b));
        }
        uint4* dst = out + 2 * c;
        __stcs(dst, make_uint4(o[0], o[1], o[2], o[3]));
        __stcs(dst + 1, make_uint4(o[4], o[5], o[6], o[7]));
    }
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
                     aligned16(out);
    if (vec) {
        const int64_t nchunks = total / 16;
        int64_t blocks = (nchunks + 255) / 256;
        const int64_t cap = static_cast<int64_t>(sms) * 32;
        if (blocks > cap) blocks = cap;
        k_dequant_vec16<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
            reinterpret_cast<const uint4*>(w.packed), w.scales, w.biases,
            reinterpret_cast<uint4*>(out), nchunks, w.K / 16, w.gs / 16, w.G);
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
