// BF16 -> 8-bit group-affine codes: the inverse of the "MlxInt8Weight"
// format (packed bytes in uint32 words, BF16 scale and bias per group).  The
// pages give no quantizer algorithm; this is the plain min/max affine one:
// per row and group of gs columns, all in fp32 with every operation rounded
// to nearest even,
//   lo, hi = min, max;  s = bf16((hi - lo) / 255);  b = bf16(lo);
//   q = clamp(rint((w - b) / s), 0, 255)   (q = 0 when s == 0).
// HBM-bound: 2 bytes read and 1 + 4/gs bytes written per weight.  The
// quotient is computed approximately and made exact only near a tie, so the
// codes equal those of the correctly rounded division.
//
// k_quantize_lanes (gs = 8..256, a power of two, 16-byte aligned source):
// gs/8 consecutive lanes share a group, each loading 8 BF16 (16 bytes,
// coalesced across the warp) and writing 8 codes (8 bytes).  The group's
// minimum and maximum are combined over adjacent blocks of lanes (xor
// offsets 1, 2, 4, ...) with strict compares that keep the earlier block's
// value on a tie - the same result as a scan in column order, down to the
// sign of a zero minimum.
// k_quantize (any other group size or alignment): one thread per group, a
// scan for the range, then the codes.
#include "device_common.cuh"
#include "kernels.h"

namespace mlxq {
namespace {

__global__ void __launch_bounds__(256) k_quantize(const uint16_t* __restrict__ w, int64_t N, int64_t K, int gs,
                                                  int64_t G, uint32_t* __restrict__ packed,
                                                  uint16_t* __restrict__ scales, uint16_t* __restrict__ biases) {
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= N * G) return;
    const int64_t n = idx / G, g = idx - n * G;
    const uint16_t* src = w + n * K + g * gs;
    const bool v8 = (reinterpret_cast<uintptr_t>(src) & 7u) == 0;  // four BF16 per load
    float lo = bf16_bits_to_f32(__ldg(src)), hi = lo;
    if (v8) {
        for (int j = 0; j < gs; j += 4) {
            const uint2 u = __ldg(reinterpret_cast<const uint2*>(src + j));
            const float f[4] = {bf16_bits_to_f32(u.x & 0xFFFFu), bf16_bits_to_f32(u.x >> 16),
                                bf16_bits_to_f32(u.y & 0xFFFFu), bf16_bits_to_f32(u.y >> 16)};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (f[i] < lo) lo = f[i];
                if (f[i] > hi) hi = f[i];
            }
        }
    } else {
        for (int j = 1; j < gs; ++j) {
            const float v = bf16_bits_to_f32(__ldg(src + j));
            if (v < lo) lo = v;
            if (v > hi) hi = v;
        }
    }
    const __nv_bfloat16 sb = __float2bfloat16_rn(__fdiv_rn(__fsub_rn(hi, lo), 255.0f));
    const __nv_bfloat16 bb = __float2bfloat16_rn(lo);
    const float sf = __bfloat162float(sb), bf = __bfloat162float(bb);
    uint32_t* dst = packed + n * (K / 4) + g * (gs / 4);
    for (int j = 0; j < gs; j += 4) {
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float c = 0.0f;
            if (sf != 0.0f) {
                c = rintf(__fdiv_rn(__fsub_rn(bf16_bits_to_f32(__ldg(src + j + i)), bf), sf));
                if (c < 0.0f) c = 0.0f;
                if (c > 255.0f) c = 255.0f;
            }
            word |= static_cast<uint32_t>(c) << (8 * i);
        }
        dst[j / 4] = word;
    }
    scales[idx] = *reinterpret_cast<const uint16_t*>(&sb);
    biases[idx] = *reinterpret_cast<const uint16_t*>(&bb);
}

// Combine this lane's running minimum/maximum with the block of lanes at
// xor distance `o`; the lower block holds the earlier columns.
__device__ __forceinline__ void combine_range(float& lo, float& hi, int o, int lane) {
    const float olo = __shfl_xor_sync(0xFFFFFFFFu, lo, o);
    const float ohi = __shfl_xor_sync(0xFFFFFFFFu, hi, o);
    if (lane & o) {  // this lane is in the later block: keep its value only when strictly beyond
        lo = lo < olo ? lo : olo;
        hi = hi > ohi ? hi : ohi;
    } else {
        lo = olo < lo ? olo : lo;
        hi = ohi > hi ? ohi : hi;
    }
}

template <int L>  // lanes per group = gs / 8
__global__ void __launch_bounds__(256) k_quantize_lanes(const uint16_t* __restrict__ w, int64_t tasks,
                                                        uint32_t* __restrict__ packed, uint16_t* __restrict__ scales,
                                                        uint16_t* __restrict__ biases) {
    const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;  // 8-column chunk
    const int lane = threadIdx.x & 31;
    const bool live = t < tasks;  // whole groups are live or not, so shuffles stay within live groups
    const uint4 u = live ? __ldg(reinterpret_cast<const uint4*>(w) + t) : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t h[4] = {u.x, u.y, u.z, u.w};
    float f[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = bf16_bits_to_f32(h[i] & 0xFFFFu);
        f[2 * i + 1] = bf16_bits_to_f32(h[i] >> 16);
    }
    float lo = f[0], hi = f[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) {
        if (f[i] < lo) lo = f[i];
        if (f[i] > hi) hi = f[i];
    }
#pragma unroll
    for (int o = 1; o < L; o <<= 1) combine_range(lo, hi, o, lane);
    const __nv_bfloat16 sb = __float2bfloat16_rn(__fdiv_rn(__fsub_rn(hi, lo), 255.0f));
    const __nv_bfloat16 bb = __float2bfloat16_rn(lo);
    const float sf = __bfloat162float(sb), bf = __bfloat162float(bb);
    uint32_t word[2] = {0u, 0u};
    // An approximate quotient rounds to the same integer as the correctly
    // rounded one unless it lies within a few ulps of a half-integer; there,
    // and for operands outside the range where the approximation holds, the
    // correctly rounded division decides.
    const float as = fabsf(sf);
    const bool fast_ok = as > 0x1p-100f && as < 0x1p100f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float c = 0.0f;
        if (sf != 0.0f) {
            const float d = __fsub_rn(f[i], bf);
            float qv;
            if (fast_ok && fabsf(d) < 0x1p100f) {
                qv = __fdividef(d, sf);
                if (fabsf(qv - floorf(qv) - 0.5f) < 0x1p-10f) qv = __fdiv_rn(d, sf);
            } else {
                qv = __fdiv_rn(d, sf);
            }
            c = rintf(qv);
            if (c < 0.0f) c = 0.0f;
            if (c > 255.0f) c = 255.0f;
        }
        word[i >> 2] |= static_cast<uint32_t>(c) << (8 * (i & 3));
    }
    if (!live) return;
    reinterpret_cast<uint2*>(packed)[t] = make_uint2(word[0], word[1]);
    if ((lane & (L - 1)) == 0) {
        const int64_t grp = t / L;
        scales[grp] = *reinterpret_cast<const uint16_t*>(&sb);
        biases[grp] = *reinterpret_cast<const uint16_t*>(&bb);
    }
}

template <int L>
cudaError_t launch_lanes(const void* w, const WeightView& dst, cudaStream_t stream) {
    const int64_t tasks = dst.N * dst.K / 8;
    const int64_t blocks = (tasks + 255) / 256;
    if (blocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
    k_quantize_lanes<L><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        static_cast<const uint16_t*>(w), tasks, const_cast<uint32_t*>(dst.packed), const_cast<uint16_t*>(dst.scales),
        const_cast<uint16_t*>(dst.biases));
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize(const void* w, const WeightView& dst, cudaStream_t stream) {
    const int64_t groups = dst.N * dst.G;
    if (groups == 0) return cudaSuccess;
    const bool lanes_ok = (reinterpret_cast<uintptr_t>(w) & 15u) == 0 && (reinterpret_cast<uintptr_t>(dst.packed) & 7u) == 0;
    if (lanes_ok) {
        switch (dst.gs) {
            case 8: return launch_lanes<1>(w, dst, stream);
            case 16: return launch_lanes<2>(w, dst, stream);
            case 32: return launch_lanes<4>(w, dst, stream);
            case 64: return launch_lanes<8>(w, dst, stream);
            case 128: return launch_lanes<16>(w, dst, stream);
            case 256: return launch_lanes<32>(w, dst, stream);
            default: break;
        }
    }
    const int64_t blocks = (groups + 255) / 256;
    if (blocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
    k_quantize<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        static_cast<const uint16_t*>(w), dst.N, dst.K, static_cast<int>(dst.gs), dst.G,
        const_cast<uint32_t*>(dst.packed), const_cast<uint16_t*>(dst.scales), const_cast<uint16_t*>(dst.biases));
    return cudaGetLastError();
}

}  // namespace mlxq
