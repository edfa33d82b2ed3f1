// Tensor-core gemm for m > 32 ("MlxInt8Weight" page, gemm: Y = X W^T).
//
// The page's kernel computes one output element per thread; here the
// contraction runs on the sm_100 tensor cores (tcgen05) instead.
//
//   tile: 256 weight rows (two MMA M=128 halves) x BN activation rows (MMA N),
//         over the k-blocks of one K split (64 codes per k-block)
//   warp 0      TMA: the BN x 64 BF16 activation tile of each k-block
//               (128-byte swizzle, the MMA's B operand)
//   warp 1      allocates TMEM (2 x BN fp32 columns x 128 lanes) and, from one
//               lane, issues tcgen05.mma kind::f16 (BF16 x BF16 -> fp32),
//               8 per k-block, committing each stage back to the producers
//   warp 2      TMA: packed codes of the 256 rows, and 8-group boxes of their
//               scales and biases
//   warps 3-10  dequantise the codes to BF16 straight into the MMA's A
//               operand layout (K-major, 128-byte swizzle) - exactly the BF16
//               weight dequantize_to writes
//   warps 11-18 after a unit's last k-block, read the accumulators
//               (tcgen05.ld) and store Y (or the unit's fp32 partial)
//
// When the tiles alone would leave SMs idle (fewer tiles than SMs, or the
// tiles of a partial last wave), those tiles' K is split over several CTAs:
// each stores its fp32 partial tile, and the last to finish (a per-tile
// counter) adds them in split order, so the result does not depend on which
// CTA finishes when.  The tiles of the full waves stay whole.  The accumulator is D[w_row][x_row]
// (TMEM lane = weight row), so a warp's stores of one output row of Y are 32
// consecutive BF16 values.  All pipeline waits are bounded; no cluster
// multicast is used.  After a wait gives up, the producers and the MMA thread
// issue nothing more, and before TMEM is freed and the CTA exits they wait
// (bounded) for the copies and MMAs they already issued.
#include <mutex>

#include "device_common.cuh"
#include "kernels.h"
#include "tensor_map.h"

namespace mlxq {

// Scratch of mlxq_gemm_noalloc, compiled into the library (zero when the
// module loads): per-tile counters, then the fp32 partials.  Every split
// gemm leaves the counters it used at zero, so calls need no reset.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];
namespace {

constexpr int kBM = 256;                // weight rows per tile: two MMA M=128 halves
constexpr int kHM = 128;                // rows per MMA half
constexpr int kBK = 64;                 // k per stage: one 128-byte row of BF16
constexpr int kDequantWarps = 8;
constexpr int kEpilogueWarps = 8;       // two per TMEM lane quadrant (one per accumulator half)
constexpr int kFirstDequant = 3;        // warps: 0 X producer, 1 MMA, 2 weight producer
constexpr int kFirstEpilogue = kFirstDequant + kDequantWarps;
constexpr int kThreads = (kFirstEpilogue + kEpilogueWarps) * 32;
constexpr uint32_t kStageA = kBM * 128;  // BF16 A tile (two 128-row halves)
constexpr uint32_t kStageP = kBM * kBK;  // packed codes of one k-block
constexpr int kSbGroups = 8;             // scale groups per scale/bias box (16 bytes per row)
constexpr uint32_t kStageSB = kBM * kSbGroups * 2;  // one box of scales (or biases)
constexpr int kXBoxRows = 32;            // activation rows per TMA box
constexpr int kSP = 3;                   // packed-code slots
constexpr int kSSB = 2;                  // scale/bias slots

struct TcParams {
    uint16_t* Y;
    int N, K, G, gs, m;
    int BN, S, SX, num_kb;  // S: A-tile stages, SX: activation-tile stages
    int sg;          // k-blocks covered by one scale/bias box (8 * gs / 64)
    int sb_tma;      // 1: scales/biases by TMA boxes; 0 (rows not 16-byte multiples): direct loads
    int ks;          // K splits of each split tile (1: no tile is split)
    int full_units;  // units 0 .. full_units - 1: whole tiles 0 .. full_units - 1
    int tail0, ntail;  // then tiles tail0 .. tail0 + ntail - 1, each in ks K splits
    float* ws;       // ks > 1: fp32 partials [ntail * ks][BN][kBM] of the split tiles
    unsigned int* counters;  // ks > 1: per split tile arrival counts, zero between launches
    const uint16_t* scales;
    const uint16_t* biases;
    uint32_t idesc, tmem_cols;
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

// Sum the ks fp32 partials of one tile in split order and store BF16 Y.
// Thread et of the 256 epilogue threads takes float4 chunks (4 rows of one
// column) et, et + 256, ...; the loads of four splits and kRedU chunks are in
// flight together.
constexpr int kRedU = 4;
__device__ __forceinline__ void reduce_partials(const TcParams& p, int tile, int n0, int m0, int cols, int et) {
    const float* base = p.ws + static_cast<int64_t>(tile - p.tail0) * p.ks * p.BN * kBM;
    const int64_t part = static_cast<int64_t>(p.BN) * kBM;  // floats per partial
    const int nchunk = cols * (kBM / 4);
    const bool vec_store = (p.N % 4 == 0) && ((reinterpret_cast<uintptr_t>(p.Y) & 7u) == 0);
    for (int f0 = et; f0 < nchunk; f0 += kEpilogueWarps * 32 * kRedU) {
        float4 acc[kRedU];
#pragma unroll
        for (int u = 0; u < kRedU; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int sp0 = 0; sp0 < p.ks; sp0 += 4) {
            float4 v[4][kRedU];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int u = 0; u < kRedU; ++u) {
                    const int f = f0 + u * kEpilogueWarps * 32;
                    v[i][u] = (sp0 + i < p.ks && f < nchunk)
                                  ? __ldcg(reinterpret_cast<const float4*>(base + (sp0 + i) * part) + f)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int u = 0; u < kRedU; ++u) {
                    acc[u].x += v[i][u].x; acc[u].y += v[i][u].y;
                    acc[u].z += v[i][u].z; acc[u].w += v[i][u].w;
                }
        }
#pragma unroll
        for (int u = 0; u < kRedU; ++u) {
            const int f = f0 + u * kEpilogueWarps * 32;
            if (f >= nchunk) continue;
            const int c = f / (kBM / 4);
            const int n = n0 + (f % (kBM / 4)) * 4;
            uint16_t* y = p.Y + static_cast<int64_t>(m0 + c) * p.N + n;
            const uint32_t lo = pack_bf16x2(acc[u].x, acc[u].y), hi = pack_bf16x2(acc[u].z, acc[u].w);
            if (vec_store && n + 3 < p.N) {
                *reinterpret_cast<uint2*>(y) = make_uint2(lo, hi);
            } else {
                const uint16_t h[4] = {static_cast<uint16_t>(lo), static_cast<uint16_t>(lo >> 16),
                                       static_cast<uint16_t>(hi), static_cast<uint16_t>(hi >> 16)};
                for (int i = 0; i < 4 && n + i < p.N; ++i) y[i] = h[i];
            }
        }
    }
}

// Persistent: CTA b processes units b, b + gridDim.x, ... (a unit is one K
// split of one tile, weight-row tile fastest).  A tile is 256 weight rows x
// BN activation rows: two M=128 MMAs per 16-wide k step share the activation
// (B) tile.  All operand bytes arrive by
// TMA: the activation tile into the (A, X) stage ring, the packed codes into
// their own ring, and the scales/biases as 8-group boxes into a third ring;
// the dequant warps read only shared memory.  The two fp32 accumulators fill
// TMEM (2 x BN <= 512 columns).
__global__ void __launch_bounds__(kThreads, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_packed,
              const __grid_constant__ CUtensorMap tm_scales, const __grid_constant__ CUtensorMap tm_biases,
              const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);  // 1024-byte aligned (swizzle atoms)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = p.S;
    const uint32_t stage_x = static_cast<uint32_t>(p.BN) * 128u;
    const int tiles_n = (p.N + kBM - 1) / kBM;
    const int tiles_m = (p.m + p.BN - 1) / p.BN;
    const int num_tiles = tiles_n * tiles_m;
    const int num_units = p.full_units + p.ntail * p.ks;
    const int my_units = blockIdx.x < num_units ? (num_units - 1 - blockIdx.x) / gridDim.x + 1 : 0;

    // shared memory: S A tiles | SX activation tiles | kSP packed slots |
    // kSSB (scales, biases) slots | barriers.  The activation ring is the
    // deeper one: its tiles come from L2/HBM, the A tiles from the dequant warps.
    const int SX = p.SX;
    const uint32_t sbase = smem_u32(smem);
    const uint32_t x_base = sbase + static_cast<uint32_t>(S) * kStageA;
    const uint32_t p_base = x_base + static_cast<uint32_t>(SX) * stage_x;
    const uint32_t sb_base = p_base + kSP * kStageP;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + (sb_base + kSSB * 2 * kStageSB - sbase));
    uint64_t* empty = full + S;      // A tile s: written (dequant) / read (MMA)
    uint64_t* xfull = empty + S;     // activation tile: landed (TMA) / read (MMA)
    uint64_t* xempty = xfull + SX;
    uint64_t* pfull = xempty + SX;
    uint64_t* pempty = pfull + kSP;
    uint64_t* sbfull = pempty + kSP;
    uint64_t* sbempty = sbfull + kSSB;
    uint64_t* acc_full = sbempty + kSSB;
    uint64_t* acc_empty = acc_full + 1;
    uint64_t* drain = acc_empty + 1;  // the MMA thread's last commit (teardown)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    uint32_t* last_flag = tmem_slot + 1;  // epilogue: this CTA completed the tile
    auto A_of = [&](int s) { return sbase + static_cast<uint32_t>(s) * kStageA; };
    auto X_of = [&](int s) { return x_base + static_cast<uint32_t>(s) * stage_x; };
    auto P_of = [&](int s) { return p_base + static_cast<uint32_t>(s) * kStageP; };
    auto SC_of = [&](int s) { return sb_base + static_cast<uint32_t>(s) * 2u * kStageSB; };
    auto BI_of = [&](int s) { return SC_of(s) + kStageSB; };
    // Work unit t of this CTA: a tile (weight-row tile fastest) and the
    // k-blocks [kb0, kb1) of its K split.  The first full_units units are
    // whole tiles; the rest are the ks splits of the tiles from tail0 on (the
    // tiles of a partial last wave, or every tile when there are fewer tiles
    // than SMs).
    (void)num_tiles;
    auto unit_of = [&](int t, int& tile, int& split, int& n0, int& m0, int& kb0, int& kb1) {
        const int u = blockIdx.x + t * gridDim.x;
        if (u < p.full_units) {
            tile = u;
            split = -1;  // a whole tile
            kb0 = 0;
            kb1 = p.num_kb;
        } else {
            const int v = u - p.full_units;
            tile = p.tail0 + v % p.ntail;
            split = v / p.ntail;
            kb0 = static_cast<int>(static_cast<int64_t>(split) * p.num_kb / p.ks);
            kb1 = static_cast<int>(static_cast<int64_t>(split + 1) * p.num_kb / p.ks);
        }
        n0 = (tile % tiles_n) * kBM;
        m0 = (tile / tiles_n) * p.BN;
    };

    pdl_launch_dependents();
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_u32(&full[s]), kDequantWarps);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int s = 0; s < SX; ++s) {
            mbar_init(smem_u32(&xfull[s]), 1);
            mbar_init(smem_u32(&xempty[s]), 1);
        }
        for (int s = 0; s < kSP; ++s) {
            mbar_init(smem_u32(&pfull[s]), 1);
            mbar_init(smem_u32(&pempty[s]), kDequantWarps);
        }
        for (int s = 0; s < kSSB; ++s) {
            mbar_init(smem_u32(&sbfull[s]), 1);
            mbar_init(smem_u32(&sbempty[s]), kDequantWarps);
        }
        mbar_init(smem_u32(acc_full), 1);
        mbar_init(smem_u32(acc_empty), kEpilogueWarps);
        mbar_init(smem_u32(drain), 1);
        mbar_fence_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 2 * p.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_wait();  // activations, weights and Y belong to earlier work

    if (warp == 0) {
        // ---------------- activation producer ----------------
        if (lane == 0) {
            prefetch_tmap(&tm_x);
            const uint64_t pol = policy_evict_last();  // each activation tile serves every weight tile
            bool ok = true;
            int it = 0;
            for (int t = 0; t < my_units && ok; ++t) {
                int tile, split, n0, m0, kb0, kb1;
                unit_of(t, tile, split, n0, m0, kb0, kb1);
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % SX;
                    if (it >= SX) ok = mbar_wait(smem_u32(&xempty[s]), ((it / SX) - 1) & 1, p.status);
                    if (!ok) break;  // the slot may still be in use: issue nothing more
                    mbar_arrive_expect_tx(smem_u32(&xfull[s]), stage_x);
                    for (int r = 0; r < p.BN; r += kXBoxRows)
                        tma_load_2d(X_of(s) + static_cast<uint32_t>(r) * 128u, &tm_x, kb * kBK, m0 + r,
                                    smem_u32(&xfull[s]), pol);
                }
            }
            // every issued copy has landed before the CTA may exit
            for (int u = it > SX ? it - SX : 0; u < it; ++u)
                if (!mbar_wait(smem_u32(&xfull[u % SX]), (u / SX) & 1, p.status)) break;
        }
    } else if (warp == 2) {
        // ---------------- weight producer: packed codes, scales, biases ----------------
        if (lane == 0) {
            prefetch_tmap(&tm_packed);
            prefetch_tmap(&tm_scales);
            prefetch_tmap(&tm_biases);
            const uint64_t pol = policy_evict_last();  // each weight tile serves every activation tile
            bool ok = true;
            int it = 0, sbi = 0;
            for (int t = 0; t < my_units && ok; ++t) {
                int tile, split, n0, m0, kb0, kb1;
                unit_of(t, tile, split, n0, m0, kb0, kb1);
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    if (p.sb_tma && (kb == kb0 || kb % p.sg == 0)) {  // the scale/bias box holding kb
                        const int ss = sbi % kSSB;
                        if (sbi >= kSSB) ok = mbar_wait(smem_u32(&sbempty[ss]), ((sbi / kSSB) - 1) & 1, p.status);
                        if (!ok) break;  // the slot may still be in use: issue nothing more
                        mbar_arrive_expect_tx(smem_u32(&sbfull[ss]), 2u * kStageSB);
                        const int g0 = (kb / p.sg) * kSbGroups;
                        tma_load_2d(SC_of(ss), &tm_scales, g0, n0, smem_u32(&sbfull[ss]), pol);
                        tma_load_2d(BI_of(ss), &tm_biases, g0, n0, smem_u32(&sbfull[ss]), pol);
                        ++sbi;
                    }
                    const int sp = it % kSP;
                    if (it >= kSP) ok = mbar_wait(smem_u32(&pempty[sp]), ((it / kSP) - 1) & 1, p.status);
                    if (!ok) break;
                    mbar_arrive_expect_tx(smem_u32(&pfull[sp]), kStageP);
                    tma_load_2d(P_of(sp), &tm_packed, kb * kBK, n0, smem_u32(&pfull[sp]), pol);
                }
            }
            // every issued copy has landed before the CTA may exit (on a
            // break above, `it` counts the code loads actually issued)
            for (int u = it > kSP ? it - kSP : 0; u < it; ++u)
                if (!mbar_wait(smem_u32(&pfull[u % kSP]), (u / kSP) & 1, p.status)) break;
            for (int u = sbi > kSSB ? sbi - kSSB : 0; u < sbi; ++u)
                if (!mbar_wait(smem_u32(&sbfull[u % kSSB]), (u / kSSB) & 1, p.status)) break;
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            bool ok = true;
            int it = 0;
            for (int t = 0; t < my_units && ok; ++t) {
                int tile, split, n0, m0, kb0, kb1;
                unit_of(t, tile, split, n0, m0, kb0, kb1);
                // the epilogue must have drained the accumulators (previous unit)
                if (t >= 1) ok = mbar_wait(smem_u32(acc_empty), (t - 1) & 1, p.status);
                if (!ok) break;  // issue no MMA into accumulators still being read
                tc_fence_after();
                const uint32_t d0 = tmem_base, d1 = tmem_base + p.tmem_cols;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % S, sx = it % SX;
                    ok = mbar_wait(smem_u32(&full[s]), (it / S) & 1, p.status);
                    if (ok) ok = mbar_wait(smem_u32(&xfull[sx]), (it / SX) & 1, p.status);
                    if (!ok) break;  // operands not there: issue nothing more
                    tc_fence_after();
                    const uint64_t a0 = sw128_kmajor_desc(A_of(s));
                    const uint64_t a1 = sw128_kmajor_desc(A_of(s) + kHM * 128u);
                    const uint64_t bd = sw128_kmajor_desc(X_of(sx));
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        // advance 16 BF16 (32 bytes) along K inside the swizzled rows
                        const uint32_t acc = (kb != kb0 || kk != 0) ? 1u : 0u;
                        umma_bf16(d0, a0 + 2u * kk, bd + 2u * kk, p.idesc, acc);
                        umma_bf16(d1, a1 + 2u * kk, bd + 2u * kk, p.idesc, acc);
                    }
                    umma_commit(smem_u32(&empty[s]));
                    umma_commit(smem_u32(&xempty[sx]));
                }
                if (ok) umma_commit(smem_u32(acc_full));
            }
            // every MMA this thread issued has finished before TMEM is freed
            umma_commit(smem_u32(drain));
            mbar_wait(smem_u32(drain), 0, p.status);
        }
        __syncwarp();
    } else if (warp < kFirstEpilogue) {
        // ---------------- dequant: packed codes -> BF16 A operand ----------------
        const int dt = (warp - kFirstDequant) * 32 + lane;  // 0 .. 255
        const int chunk = dt & 3;                           // 16-code chunk of the 64-code k-block
        const int rbase = dt >> 2;                          // rows rbase + 64 i, i = 0..3
        bool ok = true;
        const float2 m2 = make_float2(-kMagic, -kMagic);
        int it = 0, sbi = 0;
        for (int t = 0; t < my_units; ++t) {
            int tile, split, n0, m0, kb0, kb1;
            unit_of(t, tile, split, n0, m0, kb0, kb1);
            for (int kb = kb0; kb < kb1; ++kb, ++it) {
                const int ss = sbi % kSSB;
                if (p.sb_tma && (kb == kb0 || kb % p.sg == 0) && ok)
                    ok = mbar_wait(smem_u32(&sbfull[ss]), (sbi / kSSB) & 1, p.status);
                const int sp = it % kSP;
                if (ok) ok = mbar_wait(smem_u32(&pfull[sp]), (it / kSP) & 1, p.status);
                // this thread's codes and the scale/bias of their group, for its 4 rows
                const int gl = ((kb % p.sg) * kBK + chunk * 16) / p.gs;  // group within the box
                uint4 wq[4];
                float2 s2[4], b2[4];
                const int k0 = kb * kBK + chunk * 16;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int drow = rbase + 64 * i;
                    wq[i] = lds128(P_of(sp) + static_cast<uint32_t>(drow * kBK + chunk * 16));
                    float sv = 0.f, bv = 0.f;
                    if (p.sb_tma) {
                        const uint32_t so = static_cast<uint32_t>(drow * kSbGroups + gl) * 2u;
                        sv = bf16_bits_to_f32(lds16(SC_of(ss) + so));
                        bv = bf16_bits_to_f32(lds16(BI_of(ss) + so));
                    } else if (n0 + drow < p.N && k0 < p.K) {
                        const int64_t gi = static_cast<int64_t>(n0 + drow) * p.G + k0 / p.gs;
                        sv = bf16_bits_to_f32(__ldg(p.scales + gi));
                        bv = bf16_bits_to_f32(__ldg(p.biases + gi));
                    }
                    s2[i] = make_float2(sv, sv);
                    b2[i] = make_float2(bv, bv);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&pempty[sp]));  // packed slot read
                if (p.sb_tma && (kb % p.sg == p.sg - 1 || kb == kb1 - 1)) {
                    if (lane == 0) mbar_arrive(smem_u32(&sbempty[ss]));  // last use of this box
                    ++sbi;
                }
                const int s = it % S;
                // the MMA that last read this stage's A tile must be done
                if (it >= S && ok) ok = mbar_wait(smem_u32(&empty[s]), ((it / S) - 1) & 1, p.status);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int drow = rbase + 64 * i;  // 0..255: half drow >> 7
                    const uint32_t words[4] = {wq[i].x, wq[i].y, wq[i].z, wq[i].w};
                    uint32_t o[8];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t u = words[j];
                        const float2 q01 = __fadd2_rn(make_float2(code_magic<0>(u), code_magic<1>(u)), m2);
                        const float2 q23 = __fadd2_rn(make_float2(code_magic<2>(u), code_magic<3>(u)), m2);
                        const float2 w01 = __ffma2_rn(q01, s2[i], b2[i]);
                        const float2 w23 = __ffma2_rn(q23, s2[i], b2[i]);
                        o[2 * j] = pack_bf16x2(w01.x, w01.y);
                        o[2 * j + 1] = pack_bf16x2(w23.x, w23.y);
                    }
                    // logical 16-byte chunks 2*chunk and 2*chunk+1 of this 128-byte row,
                    // placed by the 128-byte swizzle (chunk index ^ row % 8)
                    const uint32_t rowa = A_of(s) + static_cast<uint32_t>(drow) * 128u;
                    const uint32_t sw = static_cast<uint32_t>(drow & 7);
                    sts128(rowa + (((2u * chunk) ^ sw) << 4), o[0], o[1], o[2], o[3]);
                    sts128(rowa + (((2u * chunk + 1u) ^ sw) << 4), o[4], o[5], o[6], o[7]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&full[s]));
            }
        }
    } else {
        // ---------------- epilogue: TMEM -> BF16 Y ----------------
        // TMEM lane = weight row within a half, column = activation row
        const int ew = warp - kFirstEpilogue;  // 0..7
        const int q = warp & 3;                // lane quadrant this warp may access
        const int half = ew >> 2;              // accumulator half
        const int row = half * kHM + q * 32 + lane;
        bool ok = true;
        for (int t = 0; t < my_units; ++t) {
            int tile, split, n0, m0, kb0, kb1;
            unit_of(t, tile, split, n0, m0, kb0, kb1);
            if (ok) ok = mbar_wait(smem_u32(acc_full), t & 1, p.status);
            tc_fence_after();
            const uint32_t d = tmem_base + static_cast<uint32_t>(half) * p.tmem_cols +
                               (static_cast<uint32_t>(q * 32) << 16);
            const int n = n0 + row;
            const int cols = p.m - m0 < p.BN ? p.m - m0 : p.BN;
            if (split < 0 || p.ks == 1) {
                for (int c0 = 0; c0 < cols; c0 += 16) {
                    uint32_t r[16];
                    tmem_ld16(d + static_cast<uint32_t>(c0), r);
                    tmem_ld_wait();
                    if (n < p.N) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            if (c0 + j < cols) {
                                const __nv_bfloat16 v = __float2bfloat16_rn(__uint_as_float(r[j]));
                                p.Y[static_cast<int64_t>(m0 + c0 + j) * p.N + n] = *reinterpret_cast<const uint16_t*>(&v);
                            }
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(acc_empty));
                continue;
            }
            // K split: store this split's fp32 partial ([column][row], so a
            // warp's stores are 128 contiguous bytes), free the accumulators,
            // and let the tile's last unit to finish add the ks partials in
            // split order (the same order whichever unit is last).
            float* part = p.ws + (static_cast<int64_t>(tile - p.tail0) * p.ks + split) * p.BN * kBM;
            for (int c0 = 0; c0 < cols; c0 += 16) {
                uint32_t r[16];
                tmem_ld16(d + static_cast<uint32_t>(c0), r);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    if (c0 + j < cols) __stcg(part + static_cast<int64_t>(c0 + j) * kBM + row, __uint_as_float(r[j]));
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(acc_empty));
            __threadfence();  // this thread's partial is visible before the tile's count moves
            named_bar_sync(1, kEpilogueWarps * 32);
            if (ew == 0 && lane == 0) {
                const unsigned int prev = atomicAdd(p.counters + (tile - p.tail0), 1u);
                const bool last = prev == static_cast<unsigned int>(p.ks - 1);
                if (last) p.counters[tile - p.tail0] = 0u;  // zero again for the next launch
                *reinterpret_cast<volatile uint32_t*>(last_flag) = last ? 1u : 0u;
            }
            named_bar_sync(1, kEpilogueWarps * 32);
            const bool last = *reinterpret_cast<volatile uint32_t*>(last_flag) != 0u;
            if (last) {
                __threadfence();
                reduce_partials(p, tile, n0, m0, cols, ew * 32 + lane);
            }
            named_bar_sync(1, kEpilogueWarps * 32);  // the flag is read before the next unit rewrites it
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 2 * p.tmem_cols);
    }
}

// ---- host side -----------------------------------------------------------------------
int pick_bn(int64_t m) {
    int64_t bn = (m + 31) / 32 * 32;
    return static_cast<int>(bn > 256 ? 256 : bn);
}

// The library's own stream-ordered pool for split-K partials, one per device:
// it keeps its memory between calls (the device's default pool hands memory
// back at every synchronisation, and mapping it again costs more than the
// kernel).
cudaError_t workspace_pool(int device, cudaMemPool_t* out) {
    static std::mutex mu;
    static cudaMemPool_t pools[64];
    static bool made[64];
    if (device < 0 || device >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!made[device]) {
        cudaMemPoolProps props{};
        props.allocType = cudaMemAllocationTypePinned;
        props.handleTypes = cudaMemHandleTypeNone;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = device;
        cudaError_t e = cudaMemPoolCreate(&pools[device], &props);
        if (e != cudaSuccess) return e;
        uint64_t keep = ~0ull;
        e = cudaMemPoolSetAttribute(pools[device], cudaMemPoolAttrReleaseThreshold, &keep);
        if (e != cudaSuccess) return e;
        made[device] = true;
    }
    *out = pools[device];
    return cudaSuccess;
}

constexpr int kMinKbPerSplit = 8;  // 512 codes: a split shorter than this is mostly pipeline fill

constexpr size_t kCounterBytes = 4096;  // room for 1024 tile counters

cudaError_t static_scratch_base(int device, unsigned char** out) {
    static std::mutex mu;
    static unsigned char* base[64];
    if (device < 0 || device >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (base[device] == nullptr) {
        void* a = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&a, g_static_scratch);
        if (e != cudaSuccess) return e;
        base[device] = static_cast<unsigned char*>(a);
    }
    *out = base[device];
    return cudaSuccess;
}

}  // namespace

// Synchronous: called from mlxq_device_status after a device-wide sync.
cudaError_t reset_static_scratch_counters() {
    const DeviceInfo& dev = device_info();
    unsigned char* base = nullptr;
    cudaError_t e = static_scratch_base(dev.device, &base);
    if (e != cudaSuccess) return e;
    return cudaMemset(base, 0, kCounterBytes);
}

namespace {

// Which tiles split K, and into how many parts.
//  - Fewer tiles than SMs: every tile splits, into as many parts as keep all
//    splits in one wave (units <= SMs), each >= kMinKbPerSplit k-blocks.
//  - Otherwise whole tiles fill the full waves, and the R tiles of a partial
//    last wave split over the SMs that wave would leave idle (R * ks <= SMs,
//    each split >= kMinKbPerTail k-blocks): the last wave then takes 1/ks of
//    a tile's time instead of a whole tile's.
constexpr int kMinKbPerTail = 4;
struct SplitPlan {
    int full_units, tail0, ntail, ks;
};
SplitPlan plan_splits(int64_t tiles, int num_kb, int sm_count) {
    SplitPlan sp{static_cast<int>(tiles), 0, 0, 1};
    if (tiles < sm_count) {
        int64_t ks = sm_count / tiles;
        const int64_t by_k = num_kb / kMinKbPerSplit;
        if (ks > by_k) ks = by_k;
        if (ks < 1) ks = 1;
        sp = SplitPlan{0, 0, static_cast<int>(tiles), static_cast<int>(ks)};
        return sp;
    }
    const int64_t r = tiles % sm_count;
    if (r == 0) return sp;
    int64_t ks = sm_count / r;
    const int64_t by_k = num_kb / kMinKbPerTail;
    if (ks > by_k) ks = by_k;
    if (ks < 2) return sp;
    sp.full_units = static_cast<int>(tiles - r);
    sp.tail0 = static_cast<int>(tiles - r);
    sp.ntail = static_cast<int>(r);
    sp.ks = static_cast<int>(ks);
    return sp;
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

size_t gemm_tc_scratch_bytes(const WeightView& w, int64_t m) {
    const DeviceInfo& dev = device_info();
    const int bn = pick_bn(m);
    const int num_kb = static_cast<int>((w.K + kBK - 1) / kBK);
    const int64_t tiles = ((w.N + kBM - 1) / kBM) * ((m + bn - 1) / bn);
    const SplitPlan sp = plan_splits(tiles, num_kb, dev.sm_count);
    if (sp.ks == 1) return 0;
    return kCounterBytes + static_cast<size_t>(sp.ntail) * sp.ks * bn * kBM * sizeof(float);
}

cudaError_t launch_gemm_tc(const WeightView& w, const void* X, void* Y, int64_t m, cudaStream_t stream,
                           TcScratch scratch) {
    const DeviceInfo& dev = device_info();
    TcParams p{};
    p.Y = static_cast<uint16_t*>(Y);
    p.N = static_cast<int>(w.N);
    p.K = static_cast<int>(w.K);
    p.G = static_cast<int>(w.G);
    p.gs = static_cast<int>(w.gs);
    p.m = static_cast<int>(m);
    p.BN = pick_bn(m);
    p.num_kb = static_cast<int>((w.K + kBK - 1) / kBK);
    p.sg = static_cast<int>(kSbGroups * w.gs / kBK);
    p.sb_tma = (w.G % 8 == 0) ? 1 : 0;
    const int64_t tiles = ((w.N + kBM - 1) / kBM) * ((m + p.BN - 1) / p.BN);
    if (tiles > (1ll << 30)) return cudaErrorInvalidValue;
    const SplitPlan sp = plan_splits(tiles, p.num_kb, dev.sm_count);
    p.ks = sp.ks;
    p.full_units = sp.full_units;
    p.tail0 = sp.tail0;
    p.ntail = sp.ntail;
    p.scales = w.scales;
    p.biases = w.biases;
    // two A tiles (filled on the SM by the dequant warps), then as many
    // activation tiles (fetched from L2/HBM, ~2 us away) as shared memory holds
    const size_t stage_x = static_cast<size_t>(p.BN) * 128u;
    const size_t fixed = 1024 /*alignment slack*/ + kSP * kStageP + kSSB * 2 * kStageSB + 64 * sizeof(uint64_t);
    const size_t budget = static_cast<size_t>(dev.max_smem_optin);
    p.S = 2;
    if (fixed + 2 * kStageA + 2 * stage_x > budget) return cudaErrorInvalidValue;
    int SX = static_cast<int>((budget - fixed - 2 * kStageA) / stage_x);
    if (SX > 8) SX = 8;
    p.SX = SX;
    p.idesc = (1u << 4)                                   // D: fp32
              | (1u << 7)                                 // A: BF16
              | (1u << 10)                                // B: BF16
              | (static_cast<uint32_t>(p.BN >> 3) << 17)  // N
              | (static_cast<uint32_t>(kHM >> 4) << 24);  // M
    uint32_t cols = 32;
    while (cols < static_cast<uint32_t>(p.BN)) cols <<= 1;
    p.tmem_cols = cols;  // per accumulator half; two halves allocated
    p.status = device_status_ptr();

    TensorMaps3 wm;
    if (!weight_tensor_maps(w, kBM, kBK, CU_TENSOR_MAP_SWIZZLE_NONE, p.sb_tma ? kSbGroups : 0, &wm))
        return cudaErrorInvalidValue;
    CUtensorMap tm_x;
    if (!encode_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, const_cast<void*>(X), static_cast<uint64_t>(w.K),
                   static_cast<uint64_t>(m), static_cast<uint64_t>(w.K) * 2, kBK, kXBoxRows,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;

    const size_t smem = 2 * kStageA + static_cast<size_t>(SX) * stage_x + fixed;
    static std::atomic<int> configured[64];
    cudaError_t e = ensure_dynamic_smem(k_gemm_tc, smem, configured);
    if (e != cudaSuccess) return e;
    const int64_t units = static_cast<int64_t>(p.full_units) + static_cast<int64_t>(p.ntail) * p.ks;
    const int grid = static_cast<int>(units < dev.sm_count ? units : dev.sm_count);
    if (p.ks == 1) {
        e = launch_pdl(k_gemm_tc, dim3(grid), dim3(kThreads), smem, stream, tm_x, wm.packed, wm.scales, wm.biases, p);
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    }
    const size_t part_bytes = static_cast<size_t>(p.ntail) * p.ks * p.BN * kBM * sizeof(float);
    if (static_cast<size_t>(p.ntail) * sizeof(unsigned int) > kCounterBytes) return cudaErrorInvalidValue;
    if (scratch == TC_SCRATCH_STATIC) {
        // the library's static buffer: counters already zero, nothing allocated
        if (kCounterBytes + part_bytes > kStaticScratchBytes) return cudaErrorMemoryAllocation;
        unsigned char* base = nullptr;
        e = static_scratch_base(dev.device, &base);
        if (e != cudaSuccess) return e;
        p.counters = reinterpret_cast<unsigned int*>(base);
        p.ws = reinterpret_cast<float*>(base + kCounterBytes);
        e = launch_pdl(k_gemm_tc, dim3(grid), dim3(kThreads), smem, stream, tm_x, wm.packed, wm.scales, wm.biases, p);
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    }
    // K split: the fp32 partials and the per-tile counters come from the
    // library's stream-ordered pool, allocated and freed in order on the stream
    const size_t bytes = part_bytes + static_cast<size_t>(p.ntail) * sizeof(unsigned int);
    cudaMemPool_t pool;
    e = workspace_pool(dev.device, &pool);
    if (e != cudaSuccess) return e;
    void* ws = nullptr;
    e = cudaMallocFromPoolAsync(&ws, bytes, pool, stream);
    if (e != cudaSuccess) return e;
    p.ws = static_cast<float*>(ws);
    p.counters = reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(ws) + part_bytes);
    e = cudaMemsetAsync(p.counters, 0, static_cast<size_t>(p.ntail) * sizeof(unsigned int), stream);
    if (e == cudaSuccess)
        e = launch_pdl(k_gemm_tc, dim3(grid), dim3(kThreads), smem, stream, tm_x, wm.packed, wm.scales, wm.biases, p);
    if (e == cudaSuccess) e = cudaGetLastError();
    const cudaError_t ef = cudaFreeAsync(ws, stream);
    return e != cudaSuccess ? e : ef;
}

}  // namespace mlxq
