// Tensor-core gemm for large m ("MlxInt8Weight" page, gemm: Y = X W^T).
//
// The page's kernel computes one output element per thread; here the
// contraction runs on the sm_100 tensor cores instead:
//
//   CTA tile: 128 weight rows (MMA M) x BN activation rows (MMA N), full K.
//   warp 0      TMA producer: per 64-wide k-block, the packed bytes of the
//               128 weight rows (2-D tensor copy, no swizzle) and the BN x 64
//               BF16 activation tile (2-D tensor copy, 128-byte swizzle).
//   warp 1      allocates TMEM (BN fp32 columns x 128 lanes) and, from one
//               lane, issues tcgen05.mma kind::f16 (BF16 x BF16 -> fp32),
//               4 per k-block, committing each stage back to the producer.
//   warps 2-9   dequantise the packed tile to BF16 straight into the MMA's
//               A operand layout (K-major, 128-byte swizzle) - exactly the
//               BF16 weight dequantize_to writes - then, after the last
//               k-block, read the accumulators (tcgen05.ld) and store Y.
//
// The accumulator is D[w_row][x_row] (TMEM lane = weight row), so each warp's
// stores of one output row of Y are 32 consecutive BF16 values.  All pipeline
// waits are bounded; no cluster multicast is used.
#include "device_common.cuh"
#include "kernels.h"
#include "tensor_map.h"

namespace mlxq {
namespace {

constexpr int kBM = 128;                // weight rows per tile (MMA M)
constexpr int kBK = 64;                 // k per stage: one 128-byte row of BF16
constexpr int kDequantWarps = 8;
constexpr int kThreads = (2 + kDequantWarps) * 32;
constexpr uint32_t kStageA = kBM * 128;  // BF16 A tile
constexpr uint32_t kStageP = kBM * kBK;  // packed codes

struct TcParams {
    const uint16_t* scales;
    const uint16_t* biases;
    uint16_t* Y;
    int N, K, G, gs, m;
    int BN, S, num_kb;
    uint32_t stage_bytes, idesc, tmem_cols;
    unsigned int* status;
};

// ---- tcgen05 / TMEM primitives ------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
        "%12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

// Shared-memory matrix descriptor for a K-major operand stored as rows of
// 128 bytes with the 128-byte swizzle, 8-row core groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);  // start address (16-byte units)
    d |= static_cast<uint64_t>(1u) << 16;                 // leading byte offset (unused here)
    d |= static_cast<uint64_t>(1024u >> 4) << 32;         // stride byte offset: 8 rows x 128 B
    d |= static_cast<uint64_t>(1u) << 46;                 // descriptor version of sm_100
    d |= static_cast<uint64_t>(2u) << 61;                 // layout: 128-byte swizzle
    return d;
}

__global__ void __launch_bounds__(kThreads, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tm_packed, const __grid_constant__ CUtensorMap tm_x,
              const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);  // 1024-byte aligned (swizzle atoms)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = p.S;
    const int n0 = blockIdx.x * kBM;
    const int m0 = blockIdx.y * p.BN;
    const uint32_t stage_x = static_cast<uint32_t>(p.BN) * 128u;

    uint64_t* pfull = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(S) * p.stage_bytes);
    uint64_t* full = pfull + S;
    uint64_t* empty = full + S;
    uint64_t* accum = empty + S;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
    const uint32_t sbase = smem_u32(smem);
    auto A_of = [&](int s) { return sbase + static_cast<uint32_t>(s) * p.stage_bytes; };
    auto X_of = [&](int s) { return A_of(s) + kStageA; };
    auto P_of = [&](int s) { return X_of(s) + stage_x; };

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_u32(&pfull[s]), 1);
            mbar_init(smem_u32(&full[s]), 1 + kDequantWarps);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        mbar_init(smem_u32(accum), 1);
        mbar_fence_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), p.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_d = *tmem_slot;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            prefetch_tmap(&tm_packed);
            prefetch_tmap(&tm_x);
            const uint64_t pol_w = policy_evict_first();
            const uint64_t pol_x = policy_evict_last();
            bool ok = true;
            for (int kb = 0; kb < p.num_kb; ++kb) {
                const int s = kb % S;
                if (kb >= S && ok) ok = mbar_wait(smem_u32(&empty[s]), ((kb / S) - 1) & 1, p.status);
                mbar_arrive_expect_tx(smem_u32(&pfull[s]), kStageP);
                tma_load_2d(P_of(s), &tm_packed, kb * kBK, n0, smem_u32(&pfull[s]), pol_w);
                mbar_arrive_expect_tx(smem_u32(&full[s]), stage_x);
                tma_load_2d(X_of(s), &tm_x, kb * kBK, m0, smem_u32(&full[s]), pol_x);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            bool ok = true;
            for (int kb = 0; kb < p.num_kb; ++kb) {
                const int s = kb % S;
                if (ok) ok = mbar_wait(smem_u32(&full[s]), (kb / S) & 1, p.status);
                tc_fence_after();
                const uint64_t ad = sw128_kmajor_desc(A_of(s));
                const uint64_t bd = sw128_kmajor_desc(X_of(s));
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk) {
                    // advance 16 BF16 (32 bytes) along K inside the swizzled row
                    umma_bf16(tmem_d, ad + 2u * kk, bd + 2u * kk, p.idesc, (kb | kk) != 0);
                }
                umma_commit(smem_u32(&empty[s]));
            }
            umma_commit(smem_u32(accum));
        }
        __syncwarp();
    } else {
        // ---------------- dequant, then epilogue ----------------
        const int dt = (warp - 2) * 32 + lane;  // 0 .. 255
        const int chunk = dt & 3;               // 16-code chunk of the 64-code k-block
        const int rbase = dt >> 2;              // rows rbase and rbase + 64
        bool ok = true;
        // scale/bias of the next k-block, loaded one block ahead
        float sc[2], bi[2];
        auto load_sb = [&](int kb, float (&s_)[2], float (&b_)[2]) {
            int g = (kb * kBK + chunk * 16) / p.gs;
            if (g > p.G - 1) g = p.G - 1;
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int n = n0 + rbase + 64 * i;
                if (n < p.N) {
                    s_[i] = bf16_bits_to_f32(__ldg(p.scales + static_cast<int64_t>(n) * p.G + g));
                    b_[i] = bf16_bits_to_f32(__ldg(p.biases + static_cast<int64_t>(n) * p.G + g));
                } else {
                    s_[i] = 0.f;
                    b_[i] = 0.f;
                }
            }
        };
        load_sb(0, sc, bi);
        for (int kb = 0; kb < p.num_kb; ++kb) {
            const int s = kb % S;
            float scn[2] = {0.f, 0.f}, bin[2] = {0.f, 0.f};
            if (kb + 1 < p.num_kb) load_sb(kb + 1, scn, bin);
            if (ok) ok = mbar_wait(smem_u32(&pfull[s]), (kb / S) & 1, p.status);
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int row = rbase + 64 * i;
                const uint4 wq = lds128(P_of(s) + row * kBK + chunk * 16);
                const uint32_t words[4] = {wq.x, wq.y, wq.z, wq.w};
                uint32_t o[8];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t u = words[j];
                    const float q0 = code_magic<0>(u) - kMagic, q1 = code_magic<1>(u) - kMagic;
                    const float q2 = code_magic<2>(u) - kMagic, q3 = code_magic<3>(u) - kMagic;
                    o[2 * j] = pack_bf16x2(__fmaf_rn(sc[i], q0, bi[i]), __fmaf_rn(sc[i], q1, bi[i]));
                    o[2 * j + 1] = pack_bf16x2(__fmaf_rn(sc[i], q2, bi[i]), __fmaf_rn(sc[i], q3, bi[i]));
                }
                // logical 16-byte chunks 2*chunk and 2*chunk+1 of this 128-byte row,
                // placed by the 128-byte swizzle (chunk index ^ row % 8)
                const uint32_t rowa = A_of(s) + static_cast<uint32_t>(row) * 128u;
                const uint32_t sw = static_cast<uint32_t>(row & 7);
                sts128(rowa + (((2u * chunk) ^ sw) << 4), o[0], o[1], o[2], o[3]);
                sts128(rowa + (((2u * chunk + 1u) ^ sw) << 4), o[4], o[5], o[6], o[7]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&full[s]));
            sc[0] = scn[0];
            sc[1] = scn[1];
            bi[0] = bin[0];
            bi[1] = bin[1];
        }
        // epilogue: TMEM lane = weight row, column = activation row
        if (ok) ok = mbar_wait(smem_u32(accum), 0, p.status);
        tc_fence_after();
        const int q = warp & 3;                // TMEM lane quadrant this warp may access
        const int half = (warp - 2) >> 2;      // which half of the BN columns
        const int row = q * 32 + lane;
        const int n = n0 + row;
        const int cols = p.BN >> 1;
        for (int c0 = half * cols; c0 < (half + 1) * cols; c0 += 16) {
            uint32_t r[16];
            tmem_ld16(tmem_d + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(c0), r);
            tmem_ld_wait();
            if (n < p.N) {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int i = m0 + c0 + j;
                    if (i < p.m) {
                        const __nv_bfloat16 v = __float2bfloat16_rn(__uint_as_float(r[j]));
                        p.Y[static_cast<int64_t>(i) * p.N + n] = *reinterpret_cast<const uint16_t*>(&v);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_d, p.tmem_cols);
    }
}

// ---- host side -----------------------------------------------------------------------
int pick_bn(int64_t m) {
    int64_t bn = (m + 31) / 32 * 32;
    return static_cast<int>(bn > 256 ? 256 : bn);
}

}  // namespace

bool gemm_tc_supported(const WeightView& w, int64_t m, const void* X, const void* Y) {
    (void)Y;
    if (m < 1 || w.N < 1 || w.K < 16) return false;
    if (w.K % 16 != 0 || w.gs % 16 != 0) return false;
    if ((reinterpret_cast<uintptr_t>(X) & 15u) != 0 || (reinterpret_cast<uintptr_t>(w.packed) & 15u) != 0)
        return false;
    if (w.N > (1ll << 31) - 1 || w.K > (1ll << 31) - 1 || m > (1ll << 31) - 1) return false;
    int major = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device_info().device);
    if (major != 10) return false;
    return tensor_maps_available();
}

cudaError_t launch_gemm_tc(const WeightView& w, const void* X, void* Y, int64_t m, cudaStream_t stream) {
    const DeviceInfo& dev = device_info();
    TcParams p{};
    p.scales = w.scales;
    p.biases = w.biases;
    p.Y = static_cast<uint16_t*>(Y);
    p.N = static_cast<int>(w.N);
    p.K = static_cast<int>(w.K);
    p.G = static_cast<int>(w.G);
    p.gs = static_cast<int>(w.gs);
    p.m = static_cast<int>(m);
    p.BN = pick_bn(m);
    p.num_kb = static_cast<int>((w.K + kBK - 1) / kBK);
    p.stage_bytes = kStageA + static_cast<uint32_t>(p.BN) * 128u + kStageP;
    const size_t tail = 1024 /*alignment slack*/ + 64 * sizeof(uint64_t);
    int S = static_cast<int>((static_cast<size_t>(dev.max_smem_optin) - tail) / p.stage_bytes);
    if (S > 6) S = 6;
    if (S < 2) return cudaErrorInvalidValue;
    p.S = S;
    p.idesc = (1u << 4)                                   // D: fp32
              | (1u << 7)                                 // A: BF16
              | (1u << 10)                                // B: BF16
              | (static_cast<uint32_t>(p.BN >> 3) << 17)  // N
              | (static_cast<uint32_t>(kBM >> 4) << 24);  // M
    uint32_t cols = 32;
    while (cols < static_cast<uint32_t>(p.BN)) cols <<= 1;
    p.tmem_cols = cols;
    p.status = device_status_ptr();

    TensorMaps3 wm;
    if (!weight_tensor_maps(w, kBM, kBK, CU_TENSOR_MAP_SWIZZLE_NONE, 0, &wm)) return cudaErrorInvalidValue;
    const CUtensorMap& tm_packed = wm.packed;
    CUtensorMap tm_x;
    if (!encode_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, const_cast<void*>(X), static_cast<uint64_t>(w.K),
                   static_cast<uint64_t>(m), static_cast<uint64_t>(w.K) * 2, kBK, static_cast<uint32_t>(p.BN),
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;

    const size_t smem = static_cast<size_t>(S) * p.stage_bytes + tail;
    static std::atomic<int> configured[64];
    cudaError_t e = ensure_dynamic_smem(k_gemm_tc, smem, configured);
    if (e != cudaSuccess) return e;
    const dim3 grid(static_cast<unsigned>((w.N + kBM - 1) / kBM), static_cast<unsigned>((m + p.BN - 1) / p.BN));
    if (grid.y > 65535) return cudaErrorInvalidValue;
    k_gemm_tc<<<grid, kThreads, smem, stream>>>(tm_packed, tm_x, p);
    return cudaGetLastError();
}

}  // namespace mlxq
