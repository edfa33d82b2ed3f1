// m = 1 stream kernel of the "MlxInt8Weight" page: gemv (y = W x),
// gemv_silu_gate (y = W (silu(gate) * up)) and gemv_silu_gate_resid (the same
// plus x_resid).
//
// k_gemv_la: one CTA per SM owns R consecutive weight rows (R ~ N / #SMs),
// in 16-row MMA tiles ("pairs" of 8-row octets).  A producer lane streams K in
// stages of 512 * CPL codes with 2-D tensor copies: 4 * CPL boxes of [R rows
// x 128 bytes] (128-byte swizzle) plus the stage's [R x groups] scale and
// bias boxes.  A stage's work items are (tile, 64 * CPL-code slice) pairs; the
// 16 consumer warps take fixed items, so every warp keeps its own
// accumulators.  Per 16-code chunk and pair of rows (g, g + 8) a lane
// dequantises with paired fp32 operations, one code of row g beside one of
// row g + 8 (so the scale and bias pairs need no duplication), rounds to BF16
// (the exact weight dequantize_to writes), and feeds the A fragment of
// mma.sync m16n8k16 (BF16 in, fp32 accumulate), alternating two accumulators
// so consecutive MMAs do not wait on each other.  Every lane loads the
// activation as its own B column, so all 8 columns of D hold the same sums
// (the silu variants: even columns the BF16 high part of h, odd columns the
// low part).  The items' partial sums meet in shared memory in a fixed order.
//
// All waits are bounded.  After a wait gives up, the producer stops issuing
// copies and, before the CTA exits, waits (bounded) for the copies it has in
// flight, so no copy lands in shared memory the CTA no longer owns.
#include <cstring>

#include "device_common.cuh"
#include "kernels.h"
#include "tensor_map.h"

namespace mlxq {
namespace {

constexpr int kLaMaxPairs = 8;   // 16-row tiles per CTA (R <= 128)
constexpr int kLaMaxStages = 8;
constexpr int kLaSlices = 8;     // 64 * CPL-code slices of a stage, one per item

struct LaParams {
    const uint16_t* x;
    const uint16_t* gate;
    const uint16_t* up;
    const uint16_t* resid;
    uint16_t* y;
    int N, K, G;
    int R, npair;            // rows per CTA; 16-row tiles covering them
    int num_kb, S;           // stages; ring depth
    int gpk;                 // scale groups per stage
    int Kpad;                // num_kb * stage width (activation staging, zero past K)
    int pf_stages;           // stages prefetched to L2 before the dependency wait
    int pre_wait;            // stages copied into shared memory before it (static weights; <= S)
    uint32_t box_rows;       // rows of one 128-code column in shared memory (R, or npair * 16)
    uint32_t box_bytes;      // box_rows * 128 bytes
    int codes3;              // > 0: 3-D copies of this many 128-code columns each
    uint32_t tab_off;        // tables within a stage: after the columns and the rows a tile reads past R
    uint32_t sb_bytes;       // one table (scales or biases) of a stage, 128-byte padded
    uint32_t stage_bytes;    // 1024-byte multiple
    uint32_t xs_off, red_off, bar_off;  // from the 1024-aligned shared-memory base
    unsigned int* status;
};

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One word (4 codes) of row g (u) and of row g + 8 (v) -> the A fragment
// registers of one MMA: a0 = row g codes 0,1; a1 = row g+8 codes 0,1;
// a2 = row g codes 2,3; a3 = row g+8 codes 2,3.  s2 / b2 = (row g, row g+8).
__device__ __forceinline__ void dequant_rows(uint32_t u, uint32_t v, float2 s2, float2 b2, uint32_t& a0,
                                             uint32_t& a1, uint32_t& a2, uint32_t& a3) {
    const float2 m2 = make_float2(-kMagic, -kMagic);
    const float2 w0 = __ffma2_rn(__fadd2_rn(make_float2(code_magic<0>(u), code_magic<0>(v)), m2), s2, b2);
    const float2 w1 = __ffma2_rn(__fadd2_rn(make_float2(code_magic<1>(u), code_magic<1>(v)), m2), s2, b2);
    const float2 w2 = __ffma2_rn(__fadd2_rn(make_float2(code_magic<2>(u), code_magic<2>(v)), m2), s2, b2);
    const float2 w3 = __ffma2_rn(__fadd2_rn(make_float2(code_magic<3>(u), code_magic<3>(v)), m2), s2, b2);
    a0 = pack_bf16x2(w0.x, w1.x);
    a1 = pack_bf16x2(w0.y, w1.y);
    a2 = pack_bf16x2(w2.x, w3.x);
    a3 = pack_bf16x2(w2.y, w3.y);
}

__device__ __forceinline__ float silu_fast(float t) { return __fdividef(t, 1.0f + __expf(-t)); }

// W consumer warps (+ one producer warp).  A stage's work items are
// (16-row tile, 64 * CPL-code slice) pairs, npair * 8 of them; warp w takes
// items w, w + W, ... (at most JMAX), the same ones in every stage, so each
// item has its own accumulators.  CPL: 16-code chunks per lane per item (1 or
// 2; stages of 512 * CPL codes); GS: group size.
template <int MODE, int CPL, int GS, int W, int JMAX>
__global__ void __launch_bounds__((W + 1) * 32, 1)
    k_gemv_la(const __grid_constant__ CUtensorMap tm_packed, const __grid_constant__ CUtensorMap tm_scales,
              const __grid_constant__ CUtensorMap tm_biases, const __grid_constant__ CUtensorMap tm_codes3,
              const LaParams p) {
    constexpr int kKB = 64 * CPL * kLaSlices;  // codes per stage
    constexpr int kNB = kKB / 128;      // 128-code boxes per stage
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tq = lane & 3;
    const int S = p.S;
    const int r0 = blockIdx.x * p.R;
    const int rows = min(p.R, p.N - r0);  // >= 1
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.bar_off);
    uint64_t* empty = full + kLaMaxStages;
    const uint32_t xs = sbase + p.xs_off;
    float* red = reinterpret_cast<float*>(smem + p.red_off);
    auto stage_of = [&](int s) { return sbase + static_cast<uint32_t>(s) * p.stage_bytes; };

    pdl_launch_dependents();  // the next launch in the stream may be scheduled now
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), W);
        }
        mbar_fence_init();
    }
    __syncthreads();

    if (warp == W) {
        // ---------------- producer ----------------
        if (lane == 0) {
            prefetch_tmap(p.codes3 ? &tm_codes3 : &tm_packed);
            prefetch_tmap(&tm_scales);
            prefetch_tmap(&tm_biases);
            // Warm L2 with the first stages while the previous launch finishes
            // (when their copies must wait for it).
            for (int kb = 0; kb < p.pf_stages; ++kb) {
                for (int b = 0; b < kNB && kb * kKB + 128 * b < p.K; ++b)
                    tma_prefetch_l2_2d(&tm_packed, kb * kKB + 128 * b, r0);
                tma_prefetch_l2_2d(&tm_scales, kb * p.gpk, r0);
                tma_prefetch_l2_2d(&tm_biases, kb * p.gpk, r0);
            }
            const uint64_t pol = policy_evict_first();
            bool ok = true;
            int issued = 0;
            // Stages [0, pre_wait) of a weight no running kernel writes are
            // copied before the dependency wait; everything else after it.
            if (p.pre_wait == 0) pdl_wait();
            for (int kb = 0; kb < p.num_kb; ++kb) {
                if (kb == p.pre_wait && kb > 0) pdl_wait();
                const int s = kb % S;
                if (kb >= S) ok = mbar_wait(smem_u32(&empty[s]), ((kb / S) - 1) & 1, p.status);
                if (!ok) break;  // stop issuing: consumers may still be reading this slot
                const int col0 = kb * kKB;
                int nbox = (p.K - col0 + 127) / 128;
                if (nbox > kNB) nbox = kNB;
                const uint32_t bar = smem_u32(&full[s]);
                const uint32_t st = stage_of(s);
                if (p.codes3) {
                    // copies of [codes3 columns][R rows][128 bytes], zero past K
                    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(kNB) * 128u * p.R +
                                                   2u * static_cast<uint32_t>(p.R) * p.gpk * 2u);
                    for (int j = 0; j < kNB; j += p.codes3)
                        tma_load_3d(st + static_cast<uint32_t>(j) * p.box_bytes, &tm_codes3, 0, r0, kb * kNB + j, bar, pol);
                } else {
                    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nbox) * 128u * p.R +
                                                   2u * static_cast<uint32_t>(p.R) * p.gpk * 2u);
                    for (int b = 0; b < nbox; ++b)
                        tma_load_2d(st + static_cast<uint32_t>(b) * p.box_bytes, &tm_packed, col0 + 128 * b, r0, bar, pol);
                }
                tma_load_2d(st + p.tab_off, &tm_scales, kb * p.gpk, r0, bar, pol);
                tma_load_2d(st + p.tab_off + p.sb_bytes, &tm_biases, kb * p.gpk, r0, bar, pol);
                issued = kb + 1;
            }
            if (p.pre_wait >= p.num_kb) pdl_wait();
            // Leave only once every issued copy has landed (bounded; normally
            // the consumers have already waited for all of them).
            for (int kb = issued > S ? issued - S : 0; kb < issued; ++kb)
                if (!mbar_wait(smem_u32(&full[kb % S]), (kb / S) & 1, p.status)) break;
        }
        return;
    }

    // ---------------- consumers ----------------
    const int ctid = threadIdx.x;  // 0 .. 32 W - 1
    pdl_wait();  // activations, residual and the output belong to earlier work
    // Stage the activation operand, zero from K to Kpad: x (plain), or the
    // BF16 high and low parts of h = silu(gate) * up (rows 0 and 1).
    for (int k = ctid * 8; k < p.Kpad; k += W * 32 * 8) {
        if (MODE == GEMV_PLAIN) {
            const uint4 v = k < p.K ? ldg_nc_v4(p.x + k) : make_uint4(0u, 0u, 0u, 0u);
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(xs + 2u * k), "r"(v.x), "r"(v.y),
                         "r"(v.z), "r"(v.w)
                         : "memory");
        } else {
            uint32_t hi[4] = {0u, 0u, 0u, 0u}, lo[4] = {0u, 0u, 0u, 0u};
            if (k < p.K) {
                const uint4 gv = ldg_nc_v4(p.gate + k);
                const uint4 uv = ldg_nc_v4(p.up + k);
                const uint32_t gg[4] = {gv.x, gv.y, gv.z, gv.w}, uu[4] = {uv.x, uv.y, uv.z, uv.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float h0 = silu_fast(bf16_bits_to_f32(gg[i] & 0xFFFFu)) * bf16_bits_to_f32(uu[i] & 0xFFFFu);
                    const float h1 = silu_fast(bf16_bits_to_f32(gg[i] >> 16)) * bf16_bits_to_f32(uu[i] >> 16);
                    hi[i] = pack_bf16x2(h0, h1);
                    lo[i] = pack_bf16x2(h0 - bf16_bits_to_f32(hi[i] & 0xFFFFu), h1 - bf16_bits_to_f32(hi[i] >> 16));
                }
            }
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(xs + 2u * k), "r"(hi[0]), "r"(hi[1]),
                         "r"(hi[2]), "r"(hi[3])
                         : "memory");
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(xs + 2u * (p.Kpad + k)), "r"(lo[0]),
                         "r"(lo[1]), "r"(lo[2]), "r"(lo[3])
                         : "memory");
        }
    }
    named_bar_sync(1, W * 32);

    // This warp's items (the same in every stage): tile pj, slice sl -> box
    // b and this lane's 16-code chunks c = 2 tq + h (h = the slice's parity,
    // or ci when CPL == 2), so the 8 lanes of a shared-memory phase read 8
    // distinct 16-byte bank groups.
    const int items = p.npair * kLaSlices;
    // activation row this lane feeds as its B column (silu: high / low part)
    const uint32_t xrow = (MODE == GEMV_PLAIN) ? xs : xs + static_cast<uint32_t>(g & 1) * 2u * p.Kpad;
    const uint32_t sb8 = static_cast<uint32_t>(8 * p.gpk) * 2u;  // table offset of row g + 8
    float acc[JMAX][2][4];
#pragma unroll
    for (int j = 0; j < JMAX; ++j)
#pragma unroll
        for (int h = 0; h < 2; ++h) acc[j][h][0] = acc[j][h][1] = acc[j][h][2] = acc[j][h][3] = 0.f;

    bool ok = true;
    for (int kb = 0; kb < p.num_kb; ++kb) {
        const int s = kb % S;
        if (ok) ok = mbar_wait(smem_u32(&full[s]), (kb / S) & 1, p.status);
        const uint32_t st = stage_of(s);
        const uint32_t sca = st + p.tab_off;
        const uint32_t bia = sca + p.sb_bytes;
#pragma unroll
        for (int j = 0; j < JMAX; ++j) {
            const int it = warp + W * j;
            if (it < items) {  // warp-uniform
                const int pj = it / kLaSlices, sl = it % kLaSlices;
                const uint32_t row = static_cast<uint32_t>(16 * pj + g);
                // An item is CPL / 2 boxes (one half box when CPL == 1); per box
                // the lane takes chunks 2 tq and 2 tq + 1 (CPL >= 2) or the
                // slice's one (CPL == 1), which share a scale group when the
                // group spans 32 codes or more.
#pragma unroll
                for (int hb = 0; hb < (CPL + 1) / 2; ++hb) {
                    constexpr int kC = CPL == 1 ? 1 : 2;  // chunks of this box
                    constexpr bool kOneGroup = kC == 1 || GS >= 32;
                    const int b = CPL == 1 ? (sl >> 1) : sl * (CPL / 2) + hb;
                    const uint32_t boxa = st + static_cast<uint32_t>(b) * p.box_bytes + row * 128u;
                    // operands, shared memory -> registers
                    uint4 xa[kC], xb[kC], wu[kC], wv[kC];
                    float2 s2[kOneGroup ? 1 : kC], b2[kOneGroup ? 1 : kC];
#pragma unroll
                    for (int ci = 0; ci < kC; ++ci) {
                        const int c = 2 * tq + (CPL == 1 ? (sl & 1) : ci);
                        const uint32_t xa_addr = xrow + 2u * static_cast<uint32_t>(kb * kKB + 128 * b + 16 * c);
                        xa[ci] = lds128(xa_addr);
                        xb[ci] = lds128(xa_addr + 16u);
                        // the 128-byte swizzle keys on the line's index within the
                        // 1024-byte aligned stage: column b's rows follow column b - 1's
                        const uint32_t swz = static_cast<uint32_t>(c ^ ((b * static_cast<int>(p.box_rows) + g) & 7)) << 4;
                        wu[ci] = lds128(boxa + swz);
                        wv[ci] = lds128(boxa + 8u * 128u + swz);
                        if (!kOneGroup || ci == 0) {
                            const uint32_t so = (row * p.gpk + static_cast<uint32_t>((128 * b + 16 * c) / GS)) * 2u;
                            s2[ci] = make_float2(bf16_bits_to_f32(lds16(sca + so)), bf16_bits_to_f32(lds16(sca + so + sb8)));
                            b2[ci] = make_float2(bf16_bits_to_f32(lds16(bia + so)), bf16_bits_to_f32(lds16(bia + so + sb8)));
                        }
                    }
#pragma unroll
                    for (int ci = 0; ci < kC; ++ci) {
                        const uint32_t uu[4] = {wu[ci].x, wu[ci].y, wu[ci].z, wu[ci].w};
                        const uint32_t vv[4] = {wv[ci].x, wv[ci].y, wv[ci].z, wv[ci].w};
                        const uint32_t xw[8] = {xa[ci].x, xa[ci].y, xa[ci].z, xa[ci].w, xb[ci].x, xb[ci].y, xb[ci].z, xb[ci].w};
                        const int gi = kOneGroup ? 0 : ci;
#pragma unroll
                        for (int w4 = 0; w4 < 4; ++w4) {
                            uint32_t a0, a1, a2, a3;
                            dequant_rows(uu[w4], vv[w4], s2[gi], b2[gi], a0, a1, a2, a3);
                            // two accumulators, so consecutive MMAs do not wait on each other
                            mma_bf16_16816(acc[j][w4 & 1], a0, a1, a2, a3, xw[2 * w4], xw[2 * w4 + 1]);
                        }
                    }
                }
            }
        }
        // release the slot only after computing: an arrive right after the
        // loads would make the warp wait for them before any arithmetic
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
    }

    // ---- cross-warp sum in a fixed order: red[slice][row] ----
    const int R16 = p.npair * 16;
    if (tq == 0) {
#pragma unroll
        for (int j = 0; j < JMAX; ++j) {
            const int it = warp + W * j;
            if (it < items) {
                const int pj = it / kLaSlices, sl = it % kLaSlices;
                // D columns 0 (and 1: the low part of h) of rows g and g + 8
                const float c0 = acc[j][0][0] + acc[j][1][0], c1 = acc[j][0][1] + acc[j][1][1];
                const float c2 = acc[j][0][2] + acc[j][1][2], c3 = acc[j][0][3] + acc[j][1][3];
                red[sl * R16 + 16 * pj + g] = MODE == GEMV_PLAIN ? c0 : c0 + c1;
                red[sl * R16 + 16 * pj + g + 8] = MODE == GEMV_PLAIN ? c2 : c2 + c3;
            }
        }
    }
    named_bar_sync(1, W * 32);
    for (int r = ctid; r < rows; r += W * 32) {
        float v = 0.f;
#pragma unroll
        for (int sl = 0; sl < kLaSlices; ++sl) v += red[sl * R16 + r];
        const int n = r0 + r;
        if (MODE == GEMV_SILU_RESID) v += bf16_bits_to_f32(p.resid[n]);
        const __nv_bfloat16 o = __float2bfloat16_rn(v);
        p.y[n] = *reinterpret_cast<const uint16_t*>(&o);
    }
}

struct LaMaps {
    TensorMaps3 w;        // 2-D maps: codes [R x 128 bytes], scales and biases [R x gpk]
    CUtensorMap codes3;   // 3-D map of the codes: one box is a stage's columns
};

constexpr int kLaW = 16;        // consumer warps
// Code copies: one 2-D copy per 128-code column when the ring holds all of K
// (every stage is issued at once, and many small copies in flight land
// sooner: decode 4096 x 4096, 6.30 us against 6.45-6.78 with 3-D copies);
// one 3-D copy per stage when the ring is shorter than K and a CTA has at
// most 64 rows (8192 x 28672: 4414 -> 4767 GB/s; 4096 x 14336 down
// projection 19.0 -> 18.6 us); per-column copies again above 64 rows.

template <int MODE, int CPL, int GS, int JMAX>
cudaError_t launch_la_t(const LaMaps& tm, const LaParams& p, int grid, size_t smem, cudaStream_t stream) {
    auto kern = k_gemv_la<MODE, CPL, GS, kLaW, JMAX>;
    static std::atomic<int> configured[64];
    cudaError_t e = ensure_dynamic_smem(kern, smem, configured);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kern, dim3(grid), dim3((kLaW + 1) * 32), smem, stream, tm.w.packed, tm.w.scales, tm.w.biases,
                   tm.codes3, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// Configurations the plan produces: CPL 2 (1024-code stages) up to four
// tiles, CPL 1 (512) above, with 1, 2 or 4 items per warp; group size 128
// always takes CPL 2 (16-byte table rows).
template <int MODE, int CPL, int GS>
cudaError_t launch_la_j(const LaMaps& tm, const LaParams& p, int jmax, int grid, size_t smem,
                        cudaStream_t stream) {
    if (jmax == 1) return launch_la_t<MODE, CPL, GS, 1>(tm, p, grid, smem, stream);
    if constexpr (CPL <= 2) {
        if (jmax == 2) return launch_la_t<MODE, CPL, GS, 2>(tm, p, grid, smem, stream);
        if constexpr (CPL == 1 || GS == 128) return launch_la_t<MODE, CPL, GS, 4>(tm, p, grid, smem, stream);
    }
    return cudaErrorInvalidValue;
}

template <int MODE, int GS>
cudaError_t launch_la_cpl(const LaMaps& tm, const LaParams& p, int cpl, int jmax, int grid, size_t smem,
                          cudaStream_t stream) {
    if (cpl == 2) return launch_la_j<MODE, 2, GS>(tm, p, jmax, grid, smem, stream);
    if constexpr (GS != 128) return launch_la_j<MODE, 1, GS>(tm, p, jmax, grid, smem, stream);
    return cudaErrorInvalidValue;
}

template <int MODE>
cudaError_t launch_la_mode(const LaMaps& tm, const LaParams& p, int gs, int cpl, int jmax, int grid,
                           size_t smem, cudaStream_t stream) {
    switch (gs) {
        case 16: return launch_la_cpl<MODE, 16>(tm, p, cpl, jmax, grid, smem, stream);
        case 32: return launch_la_cpl<MODE, 32>(tm, p, cpl, jmax, grid, smem, stream);
        case 64: return launch_la_cpl<MODE, 64>(tm, p, cpl, jmax, grid, smem, stream);
        case 128: return launch_la_cpl<MODE, 128>(tm, p, cpl, jmax, grid, smem, stream);
        default: return cudaErrorInvalidValue;
    }
}

bool a16(const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; }

// Stage geometry of a weight; false if the kernel cannot take it.
struct LaPlan {
    int cpl, R, npair, grid, num_kb, S, gpk, Kpad, pf_stages, jmax;
    uint32_t box_rows, box_bytes, tab_off, sb_bytes, stage_bytes, xs_off, red_off, bar_off;
    int codes3;
    size_t smem;
};

// Stage geometry for R rows per CTA and CPL chunks per lane per item within
// `budget` bytes of shared memory; false if not even `min_stages` stages fit.
bool plan_geometry(const WeightView& w, int mode, int R, int cpl, size_t budget, int min_stages, LaPlan& pl) {
    pl.R = R;
    pl.npair = (R + 15) / 16;
    pl.cpl = cpl;
    const int kb = 64 * cpl * kLaSlices;
    pl.grid = static_cast<int>((w.N + R - 1) / R);
    pl.gpk = kb / static_cast<int>(w.gs);
    if (pl.gpk < 8) return false;  // a stage's table rows must be 16-byte multiples
    pl.num_kb = static_cast<int>((w.K + kb - 1) / kb);
    pl.Kpad = pl.num_kb * kb;
    pl.sb_bytes = (static_cast<uint32_t>(pl.npair) * 16u * pl.gpk * 2u + 127u) / 128u * 128u;
    const uint32_t xs_bytes = static_cast<uint32_t>((mode == GEMV_PLAIN ? 2 : 4) * pl.Kpad);
    const uint32_t red_bytes = static_cast<uint32_t>(kLaSlices * pl.npair * 16 * 4);
    const size_t fixed = 1024 + xs_bytes + red_bytes + 2 * kLaMaxStages * sizeof(uint64_t);
    const int items = pl.npair * kLaSlices;
    const int j = (items + kLaW - 1) / kLaW;
    pl.jmax = j <= 1 ? 1 : (j <= 2 ? 2 : 4);
    // The stage layout for codes3 columns per 3-D copy (0: 2-D copies).
    // 3-D columns hold exactly R rows (K % 128 == 0); 2-D columns are padded
    // to whole tiles.  A tile reads rows up to npair * 16 - 1 of every column,
    // so the tables start past that.
    auto layout = [&](int codes3) -> bool {
        pl.codes3 = codes3;
        pl.box_rows = codes3 ? static_cast<uint32_t>(R) : static_cast<uint32_t>(pl.npair) * 16u;
        pl.box_bytes = pl.box_rows * 128u;
        pl.tab_off = (static_cast<uint32_t>(kb / 128) * pl.box_bytes +
                      (static_cast<uint32_t>(pl.npair) * 16u - pl.box_rows) * 128u + 127u) / 128u * 128u;
        pl.stage_bytes = (pl.tab_off + 2u * pl.sb_bytes + 1023u) / 1024u * 1024u;
        if (budget < fixed + static_cast<size_t>(min_stages) * pl.stage_bytes) return false;
        int S = static_cast<int>((budget - fixed) / pl.stage_bytes);
        if (S > kLaMaxStages) S = kLaMaxStages;
        if (S > pl.num_kb) S = pl.num_kb;
        pl.S = S;
        pl.xs_off = static_cast<uint32_t>(S) * pl.stage_bytes;
        pl.red_off = pl.xs_off + xs_bytes;
        pl.bar_off = (pl.red_off + red_bytes + 7u) / 8u * 8u;
        pl.smem = 1024 + pl.bar_off + 2 * kLaMaxStages * sizeof(uint64_t);
        return true;
    };
    if (!layout(0)) return false;
    if (pl.S < pl.num_kb && w.K % 128 == 0 && R <= 64 && !layout(kb / 128)) return false;
    const int S = pl.S;
    // L2 prefetch of the first stages before the dependency wait, only when
    // the ring is shorter than K: otherwise every stage's copy is issued at
    // once right after the wait, and issuing the prefetches first would only
    // delay those copies
    pl.pf_stages = S < pl.num_kb ? S : 0;
    return true;
}

bool plan_la(const WeightView& w, int mode, LaPlan& pl) {
    const DeviceInfo& dev = device_info();
    if (w.N < 1 || w.K < 16 || w.K % 16 != 0 || w.K > 32768 || w.N > (1 << 30)) return false;
    if (w.gs != 16 && w.gs != 32 && w.gs != 64 && w.gs != 128) return false;
    if (w.G % 8 != 0) return false;  // table rows must be 16-byte multiples for the tensor copies
    const int64_t sms = dev.sm_count;
    if ((w.N + sms - 1) / sms > kLaMaxPairs * 16) return false;  // at most 128 rows per SM, one CTA per SM
    const int R = static_cast<int>((w.N + sms - 1) / sms);
    const int npair = (R + 15) / 16;
    // Codes per stage: fewer, larger stages mean fewer stage synchronisations
    // and one scale/bias load for two chunks, as long as the ring stays deep
    // enough: 1024 codes for up to four tiles, 512 above (group size 128
    // needs >= 1024).  (2048-code stages for one or two tiles measured no
    // better at the decode shape.)
    const size_t budget = static_cast<size_t>(dev.max_smem_optin);
    const int cpl = (w.gs == 128 || npair <= 4) ? 2 : 1;
    return plan_geometry(w, mode, R, cpl, budget, 1, pl);
}

}  // namespace

bool gemv_la_supported(const WeightView& w, int mode, const void* x, const void* gate, const void* up) {
    LaPlan pl;
    if (!plan_la(w, mode, pl)) return false;
    if (!a16(w.packed) || !a16(w.scales) || !a16(w.biases)) return false;
    if (mode == GEMV_PLAIN ? !a16(x) : (!a16(gate) || !a16(up))) return false;
    return tensor_maps_available();
}

cudaError_t launch_gemv_la(const WeightView& w, int mode, const void* x, const void* gate, const void* up,
                           const void* resid, void* y, cudaStream_t stream) {
    LaPlan pl;
    if (!plan_la(w, mode, pl)) return cudaErrorInvalidValue;
    LaParams p{};
    p.x = static_cast<const uint16_t*>(x);
    p.gate = static_cast<const uint16_t*>(gate);
    p.up = static_cast<const uint16_t*>(up);
    p.resid = static_cast<const uint16_t*>(resid);
    p.y = static_cast<uint16_t*>(y);
    p.N = static_cast<int>(w.N);
    p.K = static_cast<int>(w.K);
    p.G = static_cast<int>(w.G);
    p.R = pl.R;
    p.npair = pl.npair;
    p.num_kb = pl.num_kb;
    p.S = pl.S;
    p.gpk = pl.gpk;
    p.Kpad = pl.Kpad;
    // a static weight: the ring's first stages are copied before the dependency wait
    p.pre_wait = (w.flags & MLXQ_WEIGHT_STATIC) ? pl.S : 0;
    p.pf_stages = (w.flags & MLXQ_WEIGHT_STATIC) ? 0 : pl.pf_stages;
    p.box_rows = pl.box_rows;
    p.box_bytes = pl.box_bytes;
    p.codes3 = pl.codes3;
    p.tab_off = pl.tab_off;
    p.sb_bytes = pl.sb_bytes;
    p.stage_bytes = pl.stage_bytes;
    p.xs_off = pl.xs_off;
    p.red_off = pl.red_off;
    p.bar_off = pl.bar_off;
    p.status = device_status_ptr();
    LaMaps maps;
    if (!weight_tensor_maps(w, pl.R, 128, CU_TENSOR_MAP_SWIZZLE_128B, pl.gpk, &maps.w)) return cudaErrorInvalidValue;
    std::memset(&maps.codes3, 0, sizeof(maps.codes3));
    if (pl.codes3 && !encode_3d_chunks(&maps.codes3, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w.packed, static_cast<uint64_t>(w.K),
                                       static_cast<uint64_t>(w.N), static_cast<uint64_t>(w.K), 128,
                                       static_cast<uint32_t>(pl.R), static_cast<uint32_t>(pl.codes3)))
        return cudaErrorInvalidValue;
    const int gs = static_cast<int>(w.gs);
    switch (mode) {
        case GEMV_PLAIN: return launch_la_mode<GEMV_PLAIN>(maps, p, gs, pl.cpl, pl.jmax, pl.grid, pl.smem, stream);
        case GEMV_SILU: return launch_la_mode<GEMV_SILU>(maps, p, gs, pl.cpl, pl.jmax, pl.grid, pl.smem, stream);
        default: return launch_la_mode<GEMV_SILU_RESID>(maps, p, gs, pl.cpl, pl.jmax, pl.grid, pl.smem, stream);
    }
}

}  // namespace mlxq
