// Stream kernels for the "MlxInt8Weight" page's gemv, gemv_silu_gate,
// gemv_silu_gate_resid (m = 1) and small-m gemm (m <= 32), with the
// multiply-adds on the tensor pipe.
//
// Why: the work is HBM-bound, one weight byte per code, and at ~6.5 TB/s a
// B200 SM must turn ~23 codes per clock into products.  Done on the fp32
// pipes (unpack, fma, BF16 round, fma with h) that is ~8 issued instructions
// per code, which the SM cannot sustain.  Here each code costs only the
// dequantisation (byte -> fp32 via the 2^23 exponent trick, fp32 fma with
// scale and bias, RNE to BF16 - the exact BF16 weight of dequantize_to); the
// products and fp32 sums run in mma.sync m16n8k16 (BF16 in, fp32
// accumulate), with the dequantised weights going straight from registers
// into the A fragment.
//
// Layout (per MMA): A = dequantised weights, 16 rows x 16 codes (lane (g, t)
// holds rows g and g + 8 of a row pair); B = activations, 16 codes x 8
// activation rows; D = 16 weight rows x 8 activation rows.  The k order
// inside each MMA is a fixed permutation that A and B share (sums are
// order-free up to fp32 rounding).
//
// Data movement: one CTA owns R consecutive weight rows (R ~ N / #SMs, so HBM
// work is balanced to one row); a producer lane streams K in stages of
// 128 * NB codes with 2-D tensor copies: NB boxes of [R rows x 128 bytes]
// with the 128-byte swizzle (conflict-free fragment loads), plus the
// matching [R x groups] scale and bias boxes.  Consumer warp w takes box
// w % NB of every stage for its subset of row pairs.  Activations:
//   m == 1 (k_stream_mma): x - or, for the silu variants, h = silu(gate)*up
//          split into a BF16 high and a BF16 low part, so h keeps ~16 bits
//          and is never written to global memory - is staged once per CTA;
//   m > 1 (k_stream_mma_xs): each stage's activation slice arrives by TMA
//          with its weight boxes ([8 NT rows x 64 columns] boxes, 128-byte
//          swizzle, zero past m and K).
// The warps' partial results are summed in shared memory in a fixed order.
#include "device_common.cuh"
#include "kernels.h"
#include "tensor_map.h"

namespace mlxq {
namespace {

constexpr int kWarps = 16;                    // consumer warps
constexpr int kThreads = (kWarps + 1) * 32;   // + producer warp
constexpr int kMaxRows = 128;                 // rows per CTA (16 octets)

struct MmaParams {
    const uint16_t* X;      // [m, K] activations (m > 1) or x (m == 1, plain)
    const uint16_t* gate;
    const uint16_t* up;
    const uint16_t* resid;
    uint16_t* Y;            // [m, N]
    int N, K, G, gs, m;
    int R, R16;             // rows per CTA, rounded up to 16
    int num_kb, S;
    int gpk;                // scale groups per table box row: max(8, groups per stage)
    int gstage;             // scale groups per stage = 128 * NB / gs
    int tpair;              // 1: gstage < 8, one table box serves a pair of stages
    uint32_t box_rows;      // rows of one 128-code column in shared memory (R16, or R with 3-D copies)
    uint32_t box_bytes;     // box_rows * 128
    int codes3;             // 1: tm_packed is a 3-D map and one copy brings a stage's NB columns
    uint32_t tab_off;       // tables within a stage (past every row a tile reads)
    uint32_t sb_bytes;      // R16 * gpk * 2, rounded up to 128
    uint32_t stage_bytes;
    uint32_t x_off;         // m > 1: offset of the stage's activation boxes (1024-aligned)
    uint32_t xbox_bytes;    // m > 1: one [8 NT rows x 64 columns] BF16 box, 128-byte swizzle
    int x3;                 // m > 1 and K % 64 == 0: the stage's boxes come as one 3-D copy
    uint32_t x_tx;          // m > 1: activation bytes per stage (0 for m == 1)
    uint32_t xs_bytes;      // activation staging (m == 1)
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

// Dequantise one word (4 codes) to two BF16 pairs: codes (0,1) and (2,3).
__device__ __forceinline__ void dequant_word(uint32_t u, float2 s2, float2 b2, uint32_t& lo, uint32_t& hi) {
    const float2 m2 = make_float2(-kMagic, -kMagic);
    const float2 q01 = __fadd2_rn(make_float2(code_magic<0>(u), code_magic<1>(u)), m2);
    const float2 q23 = __fadd2_rn(make_float2(code_magic<2>(u), code_magic<3>(u)), m2);
    const float2 w01 = __ffma2_rn(q01, s2, b2);
    const float2 w23 = __ffma2_rn(q23, s2, b2);
    lo = pack_bf16x2(w01.x, w01.y);
    hi = pack_bf16x2(w23.x, w23.y);
}

__device__ __forceinline__ float silu_f32(float t) { return t / (1.0f + expf(-t)); }

// MMA orientation: A = dequantised weights (16 rows x 16 codes: lane (g, t)
// holds rows g and g+8), B = activations (16 codes x 8 activation rows),
// D = 16 weight rows x 8 activation rows.  Weight rows are handled in
// "pairs" of octets (16 rows).
//
// NB: 128-code boxes per stage; consumer warp w takes box w % NB and row
// pairs p = w / NB + j * (kWarps / NB).  PW: most pairs one warp holds.
// NT: activation column tiles of 8 (m <= 8 * NT).
//
// XS: m > 1, the activations arrive by TMA with each stage (tm_x); without
// it (m == 1) they are staged once per CTA from global memory.
template <int MODE, int NB, int PW, int NT, bool XS>
__device__ __forceinline__ void stream_mma(const CUtensorMap& tm_packed, const CUtensorMap& tm_scales,
                                           const CUtensorMap& tm_biases, const CUtensorMap* tm_x,
                                           const MmaParams& p) {
    constexpr int kKB = 128 * NB;
    constexpr int kSub = kWarps / NB;  // row-pair subsets
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tq = lane & 3;
    const int S = p.S;
    const int r0 = blockIdx.x * p.R;
    const int rows = min(p.R, p.N - r0);  // valid rows of this CTA (>= 1)
    const int npair = (rows + 15) >> 4;

    const uint32_t sbase = smem_u32(smem);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(S) * p.stage_bytes + p.xs_bytes);
    uint64_t* empty = full + S;
    const uint32_t xs = sbase + static_cast<uint32_t>(S) * p.stage_bytes;  // activation staging
    auto stage_of = [&](int s) { return sbase + static_cast<uint32_t>(s) * p.stage_bytes; };

    pdl_launch_dependents();  // the next kernel in the stream may be scheduled
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), kWarps);
        }
        mbar_fence_init();
    }
    __syncthreads();

    if (warp == kWarps) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            prefetch_tmap(&tm_packed);
            prefetch_tmap(&tm_scales);
            prefetch_tmap(&tm_biases);
            // Warm L2 with the first stages while earlier kernels finish
            // (L2 is coherent, so this is safe before the dependency wait;
            // every load into shared memory comes after it).
            for (int kb = 0; kb < S && kb < p.num_kb; ++kb) {
                const int col0 = kb * kKB;
                if (!p.codes3)
                    for (int b = 0; b < NB && col0 + 128 * b < p.K; ++b) tma_prefetch_l2_2d(&tm_packed, col0 + 128 * b, r0);
                tma_prefetch_l2_2d(&tm_scales, (p.tpair ? (kb & ~1) : kb) * p.gstage, r0);
                tma_prefetch_l2_2d(&tm_biases, (p.tpair ? (kb & ~1) : kb) * p.gstage, r0);
            }
            if constexpr (XS) prefetch_tmap(tm_x);
            pdl_wait();
            const uint64_t pol = policy_evict_first();
            [[maybe_unused]] const uint64_t pol_x = XS ? policy_evict_last() : 0ull;  // every CTA reads the same activations
            bool ok = true;
            int issued = 0;
            for (int kb = 0; kb < p.num_kb; ++kb) {
                const int s = kb % S;
                if (kb >= S) ok = mbar_wait(smem_u32(&empty[s]), ((kb / S) - 1) & 1, p.status);
                if (!ok) break;  // consumers may still be reading this slot: issue nothing more
                const int col0 = kb * kKB;
                int nbox = (p.K - col0 + 127) / 128;
                if (nbox > NB) nbox = NB;
                const uint32_t bar = smem_u32(&full[s]);
                const uint32_t st = stage_of(s);
                if (p.codes3) {  // one copy: [NB columns][R rows][128 bytes], zero past K
                    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(NB) * 128u * p.R +
                                                   2u * static_cast<uint32_t>(p.R) * p.gpk * 2u + p.x_tx);
                    tma_load_3d(st, &tm_packed, 0, r0, kb * NB, bar, pol);
                } else {
                    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nbox) * 128u * p.R +
                                                   2u * static_cast<uint32_t>(p.R) * p.gpk * 2u + p.x_tx);
                    for (int b = 0; b < nbox; ++b)
                        tma_load_2d(st + static_cast<uint32_t>(b) * p.box_bytes, &tm_packed, col0 + 128 * b, r0, bar, pol);
                }
                // the table box starts at the stage's first group, or at its
                // pair's (fewer than 8 groups per stage: 16-byte boxes)
                const int g0 = (p.tpair ? (kb & ~1) : kb) * p.gstage;
                tma_load_2d(st + p.tab_off, &tm_scales, g0, r0, bar, pol);
                tma_load_2d(st + p.tab_off + p.sb_bytes, &tm_biases, g0, r0, bar, pol);
                if constexpr (XS) {  // the stage's activation columns, all 8 NT rows (zero past m and K)
                    if (p.x3) {  // one 3-D copy: [kKB / 64 planes][8 NT rows][64 columns]
                        tma_load_3d(st + p.x_off, tm_x, 0, 0, col0 / 64, bar, pol_x);
                    } else {
                        for (int j = 0; j < kKB / 64; ++j)
                            tma_load_2d(st + p.x_off + static_cast<uint32_t>(j) * p.xbox_bytes, tm_x, col0 + 64 * j, 0,
                                        bar, pol_x);
                    }
                }
                issued = kb + 1;
            }
            // every issued copy has landed before the CTA may exit
            for (int kb = issued > S ? issued - S : 0; kb < issued; ++kb)
                if (!mbar_wait(smem_u32(&full[kb % S]), (kb / S) & 1, p.status)) break;
        }
        return;
    }

    // ---------------- consumers ----------------
    const int ctid = threadIdx.x;  // 0 .. 32*kWarps-1
    pdl_wait();  // activations, residual and the output belong to earlier work
    if (p.m == 1) {
        // stage the activation operand: x (plain) or the BF16 high/low split
        // of h = silu(gate)*up (silu variants: activation columns 0 and 1)
        if (MODE == GEMV_PLAIN) {
            for (int k = ctid * 8; k < p.K; k += kWarps * 32 * 8) {
                const uint4 v = ldg_nc_v4(p.X + k);
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(xs + 2u * k), "r"(v.x), "r"(v.y),
                             "r"(v.z), "r"(v.w)
                             : "memory");
            }
        } else {
            for (int k = ctid * 8; k < p.K; k += kWarps * 32 * 8) {
                const uint4 gv = ldg_nc_v4(p.gate + k);
                const uint4 uv = ldg_nc_v4(p.up + k);
                const uint32_t gg[4] = {gv.x, gv.y, gv.z, gv.w}, uu[4] = {uv.x, uv.y, uv.z, uv.w};
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float h0 = silu_f32(bf16_bits_to_f32(gg[i] & 0xFFFFu)) * bf16_bits_to_f32(uu[i] & 0xFFFFu);
                    const float h1 = silu_f32(bf16_bits_to_f32(gg[i] >> 16)) * bf16_bits_to_f32(uu[i] >> 16);
                    hi[i] = pack_bf16x2(h0, h1);
                    lo[i] = pack_bf16x2(h0 - bf16_bits_to_f32(hi[i] & 0xFFFFu), h1 - bf16_bits_to_f32(hi[i] >> 16));
                }
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(xs + 2u * k), "r"(hi[0]), "r"(hi[1]),
                             "r"(hi[2]), "r"(hi[3])
                             : "memory");
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(xs + 2u * (p.K + k)), "r"(lo[0]),
                             "r"(lo[1]), "r"(lo[2]), "r"(lo[3])
                             : "memory");
            }
        }
        named_bar_sync(1, kWarps * 32);
    }

    const int box = warp % NB;
    const int sub = warp / NB;
    // Every warp runs the same trip counts (CTA-uniform), so the mma.sync loop
    // has no divergent branches: a pair index past the CTA's rows re-reads the
    // CTA's last pair, a box past K re-reads box 0 with zero activations, and
    // those results are never stored.
    const int pw_u = (npair + kSub - 1) / kSub;  // pairs per warp (uniform)
    float acc[PW][NT][4];
#pragma unroll
    for (int j = 0; j < PW; ++j)
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[j][t][0] = acc[j][t][1] = acc[j][t][2] = acc[j][t][3] = 0.f;

    // loop-invariant pieces: group index of each chunk, swizzled offsets of
    // rows g and g + 8 of every pair (both have row % 8 == g)
    int grp[2];
    uint32_t swz[2];
#pragma unroll
    for (int ci = 0; ci < 2; ++ci) {
        const int c = tq + 4 * ci;
        grp[ci] = (box * 128 + 16 * c) / p.gs;
        // the 128-byte swizzle keys on the line's index within the 1024-byte
        // aligned stage: column `box`'s rows follow the previous columns'
        swz[ci] = static_cast<uint32_t>(c ^ ((box * static_cast<int>(p.box_rows) + g) & 7)) << 4;
    }
    uint32_t rowoff[PW];
    uint32_t sbo[PW];
#pragma unroll
    for (int j = 0; j < PW; ++j) {
        int pidx = sub + j * kSub;
        if (pidx > npair - 1) pidx = npair - 1;
        const int row = 16 * pidx + g;
        rowoff[j] = static_cast<uint32_t>(row) * 128u;
        sbo[j] = static_cast<uint32_t>(row * p.gpk + grp[0]) * 2u;
    }
    const uint32_t sgrp1 = static_cast<uint32_t>(grp[1] - grp[0]) * 2u;
    const uint32_t sbo8 = static_cast<uint32_t>(8 * p.gpk) * 2u;
    // activation column this lane feeds (B column g of each 8-column tile)
    const bool plain1 = (p.m == 1 && MODE == GEMV_PLAIN);
    // staged rows: x (plain, row 0) or h high/low (silu, rows 0 and 1); any
    // other lane reads row 0 and discards it, so every load stays inside
    const uint32_t xrow_off = (p.m == 1 && MODE != GEMV_PLAIN && g < 2) ? 2u * static_cast<uint32_t>(g * p.K) : 0u;
    bool colv[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        const int col = 8 * t + g;
        colv[t] = plain1 ? col == 0 : (p.m == 1 ? col < 2 : col < p.m);
    }
    bool ok = true;
    for (int kb = 0; kb < p.num_kb; ++kb) {
        const int s = kb % S;
        if (ok) ok = mbar_wait(smem_u32(&full[s]), (kb / S) & 1, p.status);
        const int col0 = kb * kKB + box * 128;
        const bool box_in = col0 < p.K;
        const uint32_t st = stage_of(s);
        const uint32_t boxa = st + static_cast<uint32_t>(box_in ? box : 0) * p.box_bytes;
        // tables: this stage's groups start (kb & 1) * gstage into a paired box
        const uint32_t sca = st + p.tab_off + (p.tpair ? static_cast<uint32_t>((kb & 1) * p.gstage) * 2u : 0u);
        const uint32_t bia = sca + p.sb_bytes;
#pragma unroll
        for (int ci = 0; ci < 2; ++ci) {
            const int kc = col0 + 16 * (tq + 4 * ci);
            const bool kin = box_in && kc < p.K;
            const int kcs = kin ? kc : 0;  // a valid address when out of range
            // B fragments: activation column (8 t + g) at this lane's 16 codes
            uint32_t b[NT][8];
            if constexpr (!XS) {
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    uint4 v0, v1;
                    if (p.m == 1) {
                        const uint32_t base = xs + xrow_off + 2u * static_cast<uint32_t>(kcs);
                        v0 = lds128(base);
                        v1 = lds128(base + 16);
                    } else {
                        const int colr = colv[t] ? 8 * t + g : 0;
                        const uint16_t* xr = p.X + static_cast<int64_t>(colr) * p.K + kcs;
                        v0 = ldg_nc_v4(xr);
                        v1 = ldg_nc_v4(xr + 8);
                    }
                    const bool live = kin && colv[t];
                    b[t][0] = live ? v0.x : 0u; b[t][1] = live ? v0.y : 0u;
                    b[t][2] = live ? v0.z : 0u; b[t][3] = live ? v0.w : 0u;
                    b[t][4] = live ? v1.x : 0u; b[t][5] = live ? v1.y : 0u;
                    b[t][6] = live ? v1.z : 0u; b[t][7] = live ? v1.w : 0u;
                }
            } else {
                // staged by TMA with the stage (zero past m and K): 64-column
                // box 2 box + ci, row 8 t + g, 16-byte chunks 2 tq and 2 tq + 1
                // placed by the 128-byte swizzle (chunk ^ row % 8; row % 8 == g)
                const uint32_t xb = st + p.x_off + static_cast<uint32_t>(2 * box + ci) * p.xbox_bytes;
                const uint32_t c0 = static_cast<uint32_t>((2 * tq) ^ g) << 4;
                const uint32_t c1 = static_cast<uint32_t>((2 * tq + 1) ^ g) << 4;
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    const uint32_t ra = xb + static_cast<uint32_t>(8 * t + g) * 128u;
                    const uint4 v0 = lds128(ra + c0), v1 = lds128(ra + c1);
                    b[t][0] = v0.x; b[t][1] = v0.y; b[t][2] = v0.z; b[t][3] = v0.w;
                    b[t][4] = v1.x; b[t][5] = v1.y; b[t][6] = v1.z; b[t][7] = v1.w;
                }
            }
            const uint32_t sgo = ci ? sgrp1 : 0u;
            // row pairs in groups of two: load both, then interleave the MMAs
#pragma unroll
            for (int j0 = 0; j0 < PW; j0 += 2) {
                if (j0 < pw_u) {  // CTA-uniform
                    uint4 wlo[2], whi[2];
                    float2 slo[2], blo[2], shi[2], bhi[2];
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        const int j = (j0 + jj < PW) ? j0 + jj : j0;
                        wlo[jj] = lds128(boxa + rowoff[j] + swz[ci]);
                        whi[jj] = lds128(boxa + rowoff[j] + 8u * 128u + swz[ci]);
                        const uint32_t sidx = sbo[j] + sgo;
                        const float s0 = bf16_bits_to_f32(lds16(sca + sidx));
                        const float b0 = bf16_bits_to_f32(lds16(bia + sidx));
                        const float s1 = bf16_bits_to_f32(lds16(sca + sidx + sbo8));
                        const float b1 = bf16_bits_to_f32(lds16(bia + sidx + sbo8));
                        slo[jj] = make_float2(s0, s0);
                        blo[jj] = make_float2(b0, b0);
                        shi[jj] = make_float2(s1, s1);
                        bhi[jj] = make_float2(b1, b1);
                    }
#pragma unroll
                    for (int w4 = 0; w4 < 4; ++w4) {
#pragma unroll
                        for (int jj = 0; jj < 2; ++jj) {
                            const int j = j0 + jj;
                            if (j < PW && (jj == 0 || j0 + 1 < pw_u)) {  // CTA-uniform
                                const uint32_t ul = w4 == 0 ? wlo[jj].x : w4 == 1 ? wlo[jj].y : w4 == 2 ? wlo[jj].z : wlo[jj].w;
                                const uint32_t uh = w4 == 0 ? whi[jj].x : w4 == 1 ? whi[jj].y : w4 == 2 ? whi[jj].z : whi[jj].w;
                                uint32_t a0, a2, a1, a3;
                                dequant_word(ul, slo[jj], blo[jj], a0, a2);  // row g: codes (0,1), (2,3)
                                dequant_word(uh, shi[jj], bhi[jj], a1, a3);  // row g + 8
#pragma unroll
                                for (int t = 0; t < NT; ++t)
                                    mma_bf16_16816(acc[j][t], a0, a1, a2, a3, b[t][2 * w4], b[t][2 * w4 + 1]);
                            }
                        }
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
    }
    const int my_pairs = npair > sub ? (npair - sub + kSub - 1) / kSub : 0;

    // ---- cross-warp sum (fixed order) in the freed stage area ----
    named_bar_sync(1, kWarps * 32);  // every warp is done with the stage buffers
    const int ncol = (p.m == 1) ? 1 : p.m;   // output columns (activation rows)
    const int R16 = p.R16;
    float* red = reinterpret_cast<float*>(smem);  // [kWarps][ncol][R16]
#pragma unroll
    for (int j = 0; j < PW; ++j) {
        if (j < my_pairs) {
            const int row = 16 * (sub + j * kSub) + g;
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                // c0/c2: column 8t + 2tq, c1/c3: column 8t + 2tq + 1; rows g, g+8
                if (p.m == 1) {
                    if (t == 0 && tq == 0) {
                        float v0 = acc[j][0][0], v1 = acc[j][0][2];
                        if (MODE != GEMV_PLAIN) {  // columns 0 (high) and 1 (low) of h
                            v0 += acc[j][0][1];
                            v1 += acc[j][0][3];
                        }
                        red[(warp * ncol) * R16 + row] = v0;
                        red[(warp * ncol) * R16 + row + 8] = v1;
                    }
                } else {
                    const int c = 8 * t + 2 * tq;
                    if (c < ncol) {
                        red[(warp * ncol + c) * R16 + row] = acc[j][t][0];
                        red[(warp * ncol + c) * R16 + row + 8] = acc[j][t][2];
                    }
                    if (c + 1 < ncol) {
                        red[(warp * ncol + c + 1) * R16 + row] = acc[j][t][1];
                        red[(warp * ncol + c + 1) * R16 + row + 8] = acc[j][t][3];
                    }
                }
            }
        }
    }
    named_bar_sync(1, kWarps * 32);
    const int nout = ncol * rows;
    for (int idx = ctid; idx < nout; idx += kWarps * 32) {
        const int i = idx / rows, r = idx - i * rows;
        const int w0 = ((r >> 4) % kSub) * NB;  // the NB warps that own this row pair
        float v = 0.f;
        for (int bb = 0; bb < NB; ++bb) v += red[((w0 + bb) * ncol + i) * R16 + r];
        const int n = r0 + r;
        if (MODE == GEMV_SILU_RESID) v += bf16_bits_to_f32(p.resid[n]);
        const __nv_bfloat16 o = __float2bfloat16_rn(v);
        p.Y[static_cast<int64_t>(i) * p.N + n] = *reinterpret_cast<const uint16_t*>(&o);
    }
}

template <int MODE, int NB, int PW, int NT>
__global__ void __launch_bounds__(kThreads, 1)
    k_stream_mma(const __grid_constant__ CUtensorMap tm_packed, const __grid_constant__ CUtensorMap tm_scales,
                 const __grid_constant__ CUtensorMap tm_biases, const MmaParams p) {
    stream_mma<MODE, NB, PW, NT, false>(tm_packed, tm_scales, tm_biases, nullptr, p);
}

template <int NB, int PW, int NT>
__global__ void __launch_bounds__(kThreads, 1)
    k_stream_mma_xs(const __grid_constant__ CUtensorMap tm_packed, const __grid_constant__ CUtensorMap tm_scales,
                    const __grid_constant__ CUtensorMap tm_biases, const __grid_constant__ CUtensorMap tm_x,
                    const MmaParams p) {
    stream_mma<GEMV_PLAIN, NB, PW, NT, true>(tm_packed, tm_scales, tm_biases, &tm_x, p);
}

template <int MODE, int NB, int PW, int NT>
cudaError_t launch_t(const TensorMaps3& tm, const CUtensorMap& tmx, const MmaParams& p, int grid, size_t smem,
                     cudaStream_t stream) {
    cudaError_t e;
    if (p.x_tx) {  // m > 1
        auto kern = k_stream_mma_xs<NB, PW, NT>;
        static std::atomic<int> configured[64];
        e = ensure_dynamic_smem(kern, smem, configured);
        if (e != cudaSuccess) return e;
        e = launch_pdl(kern, dim3(grid), dim3(kThreads), smem, stream, tm.packed, tm.scales, tm.biases, tmx, p);
    } else {
        auto kern = k_stream_mma<MODE, NB, PW, NT>;
        static std::atomic<int> configured[64];
        e = ensure_dynamic_smem(kern, smem, configured);
        if (e != cudaSuccess) return e;
        e = launch_pdl(kern, dim3(grid), dim3(kThreads), smem, stream, tm.packed, tm.scales, tm.biases, p);
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int MODE, int NT>
cudaError_t launch_pw(const TensorMaps3& tm, const CUtensorMap& tmx, const MmaParams& p, int nb, int npair, int grid,
                      size_t smem, cudaStream_t stream) {
    // rows per CTA are capped by NT on the host, so at most 4 / NT pairs per warp
    const int sub = kWarps / nb;
    const int pw = (npair + sub - 1) / sub;
    if (nb == 8) {
        if (pw <= 1) return launch_t<MODE, 8, 1, NT>(tm, tmx, p, grid, smem, stream);
        if constexpr (NT <= 2) {
            if (pw <= 2) return launch_t<MODE, 8, 2, NT>(tm, tmx, p, grid, smem, stream);
        }
        if constexpr (NT == 1) return launch_t<MODE, 8, 4, NT>(tm, tmx, p, grid, smem, stream);
        return cudaErrorInvalidValue;
    }
    if (pw <= 1) return launch_t<MODE, 4, 1, NT>(tm, tmx, p, grid, smem, stream);
    if constexpr (NT <= 2) return launch_t<MODE, 4, 2, NT>(tm, tmx, p, grid, smem, stream);
    return cudaErrorInvalidValue;
}

bool a16(const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; }

}  // namespace

bool stream_mma_supported(const WeightView& w, int mode, int64_t m, const void* x, const void* gate,
                          const void* up) {
    if (m < 1 || m > kStreamMmaMaxM || w.N < 1 || w.K < 16 || w.K % 16 != 0) return false;
    // scale boxes of 128*NB/gs groups (NB = 8 always possible): need (1024/gs) % 8 == 0
    if (w.gs % 16 != 0 || 1024 % w.gs != 0 || (1024 / w.gs) % 8 != 0 || w.G % 8 != 0) return false;
    if (!a16(w.packed) || !a16(w.scales) || !a16(w.biases)) return false;
    if (mode == GEMV_PLAIN ? !a16(x) : (!a16(gate) || !a16(up))) return false;
    if (mode != GEMV_PLAIN && m != 1) return false;
    if (w.K > 32768 || w.N > (1 << 30)) return false;
    return tensor_maps_available();
}

cudaError_t launch_stream_mma(const WeightView& w, int mode, int64_t m, const void* x, const void* gate,
                              const void* up, const void* resid, void* y, cudaStream_t stream) {
    const DeviceInfo& dev = device_info();
    MmaParams p{};
    p.X = static_cast<const uint16_t*>(x);
    p.gate = static_cast<const uint16_t*>(gate);
    p.up = static_cast<const uint16_t*>(up);
    p.resid = static_cast<const uint16_t*>(resid);
    p.Y = static_cast<uint16_t*>(y);
    p.N = static_cast<int>(w.N);
    p.K = static_cast<int>(w.K);
    p.G = static_cast<int>(w.G);
    p.gs = static_cast<int>(w.gs);
    p.m = static_cast<int>(m);
    // rows per CTA: balance the weight bytes over the SMs to one row, at most
    // max_rows per CTA (more CTAs than SMs when N is large); wider activation
    // tiles (m > 8) hold more registers per row pair, so fewer rows
    const int nt = m <= 8 ? 1 : (m <= 16 ? 2 : 4);
    const int64_t max_rows = nt == 1 ? kMaxRows : (nt == 2 ? 64 : 32);
    const int64_t per_sm = (w.N + dev.sm_count - 1) / dev.sm_count;
    const int64_t waves = (per_sm + max_rows - 1) / max_rows;
    int64_t R = (w.N + dev.sm_count * waves - 1) / (dev.sm_count * waves);
    if (R < 1) R = 1;
    p.R = static_cast<int>(R);
    p.R16 = (p.R + 15) / 16 * 16;
    // boxes per stage: 8 while that keeps >= 3 stages in shared memory, else 4
    // (when the group size allows 4: a stage's scale box must span >= 8 groups)
    // (a stage with fewer than 8 scale groups shares one 8-group table box
    // with the next stage)
    const int nb = (p.R16 <= 64 || w.K <= 1024) ? 8 : 4;
    const int kKB = 128 * nb;
    if (kKB % w.gs != 0) return cudaErrorInvalidValue;
    p.gstage = static_cast<int>(kKB / w.gs);
    p.tpair = p.gstage < 8 ? 1 : 0;
    if (p.tpair && (8 % p.gstage != 0 || 2 * p.gstage != 8)) return cudaErrorInvalidValue;
    if (!p.tpair && p.gstage % 8 != 0) return cudaErrorInvalidValue;
    p.gpk = p.tpair ? 8 : p.gstage;
    p.num_kb = static_cast<int>((w.K + kKB - 1) / kKB);
    p.sb_bytes = (static_cast<uint32_t>(p.R16) * p.gpk * 2u + 127u) / 128u * 128u;
    p.xs_bytes = (m == 1) ? static_cast<uint32_t>((mode == GEMV_PLAIN ? 2 : 4) * w.K + 127) / 128u * 128u : 0u;
    const uint32_t red_bytes = kWarps * static_cast<uint32_t>(m) * static_cast<uint32_t>(p.R16) * 4u;
    const size_t fixed = 1024 + p.xs_bytes + 2 * 16 * sizeof(uint64_t);
    const size_t full_budget = static_cast<size_t>(dev.max_smem_optin);
    const size_t half_budget = full_budget / 2 - 1024;
    size_t smem = 0;
    // The stage layout with 2-D copies of one column each (codes3 = 0,
    // columns padded to whole tiles) or one 3-D copy of all NB columns
    // (columns of exactly R rows; a tile reads rows up to R16 - 1 of every
    // column, so the tables start past that).  One CTA per SM when the grid
    // is one wave, else sized for two per SM if that still leaves two stages.
    auto layout = [&](int codes3) -> bool {
        p.codes3 = codes3;
        p.box_rows = codes3 ? static_cast<uint32_t>(p.R) : static_cast<uint32_t>(p.R16);
        p.box_bytes = p.box_rows * 128u;
        p.tab_off = (static_cast<uint32_t>(nb) * p.box_bytes + (static_cast<uint32_t>(p.R16) - p.box_rows) * 128u + 127u) /
                    128u * 128u;
        p.stage_bytes = p.tab_off + 2u * p.sb_bytes;
        p.stage_bytes = (p.stage_bytes + 1023u) / 1024u * 1024u;  // keep every stage 1024-byte aligned
        p.x_off = 0;
        p.xbox_bytes = 0;
        p.x_tx = 0;
        if (m > 1) {  // the stage's activation slice: kKB / 64 boxes of [8 nt rows x 64 columns]
            p.x_off = p.stage_bytes;
            p.xbox_bytes = static_cast<uint32_t>(8 * nt) * 128u;
            p.x_tx = static_cast<uint32_t>(kKB / 64) * p.xbox_bytes;
            p.stage_bytes += p.x_tx;
        }
        int S = static_cast<int>((full_budget - fixed) / p.stage_bytes);
        if (waves > 1 && half_budget > fixed && (half_budget - fixed) / p.stage_bytes >= 2)
            S = static_cast<int>((half_budget - fixed) / p.stage_bytes);
        if (S > p.num_kb) S = p.num_kb;
        if (S > 8) S = 8;
        if (S < 1) return false;
        smem = static_cast<size_t>(S) * p.stage_bytes + fixed;
        if (static_cast<size_t>(S) * p.stage_bytes < red_bytes) smem = red_bytes + fixed;  // room for the final sum
        if (smem > static_cast<size_t>(dev.max_smem_optin)) return false;
        p.S = S;
        return true;
    };
    if (!layout(0)) return cudaErrorInvalidValue;
    // one copy per stage pays when the ring is shorter than K and the rows are
    // few (the m = 1 kernel measured the same)
    if (p.S < p.num_kb && w.K % 128 == 0 && p.R <= 64 && !layout(1)) return cudaErrorInvalidValue;
    p.status = device_status_ptr();

    TensorMaps3 maps;
    if (!weight_tensor_maps(w, p.R, 128, CU_TENSOR_MAP_SWIZZLE_128B, p.gpk, &maps)) return cudaErrorInvalidValue;
    CUtensorMap tmx = maps.packed;  // m == 1: not read
    if (p.codes3 && !encode_3d_chunks(&maps.packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w.packed, static_cast<uint64_t>(w.K),
                                      static_cast<uint64_t>(w.N), static_cast<uint64_t>(w.K), 128,
                                      static_cast<uint32_t>(p.R), static_cast<uint32_t>(nb)))
        return cudaErrorInvalidValue;
    // m > 1: the activation boxes; as 3-D planes of 64 columns (one copy per
    // stage, the same shared-memory layout) when K % 64 == 0
    p.x3 = (m > 1 && w.K % 64 == 0) ? 1 : 0;
    if (p.x3 && !encode_3d_chunks(&tmx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, static_cast<uint64_t>(w.K),
                                  static_cast<uint64_t>(m), static_cast<uint64_t>(w.K) * 2, 64,
                                  static_cast<uint32_t>(8 * nt), static_cast<uint32_t>(kKB / 64)))
        return cudaErrorInvalidValue;
    if (m > 1 && !p.x3 && !encode_2d(&tmx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, static_cast<uint64_t>(w.K),
                                     static_cast<uint64_t>(m), static_cast<uint64_t>(w.K) * 2, 64,
                                     static_cast<uint32_t>(8 * nt), CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const int grid = static_cast<int>((w.N + p.R - 1) / p.R);
    const int npair = p.R16 / 16;
    if (nt == 2) return launch_pw<GEMV_PLAIN, 2>(maps, tmx, p, nb, npair, grid, smem, stream);
    if (nt == 4) return launch_pw<GEMV_PLAIN, 4>(maps, tmx, p, nb, npair, grid, smem, stream);
    switch (mode) {
        case GEMV_PLAIN: return launch_pw<GEMV_PLAIN, 1>(maps, tmx, p, nb, npair, grid, smem, stream);
        case GEMV_SILU: return launch_pw<GEMV_SILU, 1>(maps, tmx, p, nb, npair, grid, smem, stream);
        default: return launch_pw<GEMV_SILU_RESID, 1>(maps, tmx, p, nb, npair, grid, smem, stream);
    }
}

}  // namespace mlxq
