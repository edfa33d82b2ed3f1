// Small-m gemm on the tcgen05 tensor cores ("MlxInt8Weight" page, gemm:
// Y = X W^T for 8 < m <= 64), weight-streaming: every weight byte is read
// from HBM once and dequantised once.
//
// Swap-AB: the dequantised weight is the MMA's A operand (M = 128 weight
// rows) and the activations are B (N = m rounded up to 16, 32 or 64), so the
// m activation rows cost the tensor core, not the dequantising warps: the
// consumers' work per code is the same at m = 64 as at m = 16.
//
// One CTA per SM owns a balanced range of 16-row tiles and walks it in
// groups of up to 8 tiles (128 rows).  Each group streams K in 128-code
// stages:
//   warp 0      TMA: per stage one box of the group's codes ([rows x 128
//               bytes], 128-byte swizzle) into the code ring; per 16 scale
//               groups one [rows x 16] box each of scales and biases
//   warp 2      TMA: per stage one 3-D box of the activation columns ([2
//               k-blocks][BN rows][64 columns], 128-byte swizzle, zero past m
//               and K) into its own ring, so a code slot is free again as soon
//               as the codes are dequantised, not when the MMAs are done
//   warp 1      allocates TMEM (one fp32 accumulator of BN columns) and, from
//               one lane, issues tcgen05.mma kind::f16 (BF16 x BF16 -> fp32):
//               8 per stage, A from the stage's A tile, B from its activation
//               box
//   warps 3-18  dequantise the stage's codes into the A tile (K-major,
//               128-byte swizzle: the BF16 weight dequantize_to writes), and
//               at the end of a group read the accumulator (tcgen05.ld) and
//               store the group's outputs
// A tile rows past the group's rows are never written; the MMA rows they
// feed are never read.  All waits are bounded; after one gives up, the
// producer and the MMA thread issue nothing more and wait (bounded) for what
// they already issued before TMEM is freed and the CTA exits.
#include <atomic>

#include "device_common.cuh"
#include "kernels.h"
#include "tensor_map.h"

namespace mlxq {
namespace {

constexpr int kStW = 16;             // dequantising warps
constexpr int kStThreads = (kStW + 3) * 32;
constexpr int kStKB = 128;           // codes per stage (two 64-code k-blocks)
constexpr int kStMaxS = 8;           // code ring depth
constexpr int kStMaxX = 4;           // activation ring depth
constexpr int kStTabGroups = 16;     // scale groups per table box
constexpr uint32_t kStA = 128u * 128u;  // one k-block's A tile: 128 rows x 128 bytes
constexpr int kStMaxGP = 8;          // tiles per group
constexpr int kStNA = 2;             // A tiles in flight (two k-blocks each)

struct StParams {
    uint16_t* Y;  // [m, N]
    int N, K, m, gs;
    int P;              // 16-row tiles
    int gp;             // tiles per group (<= 8)
    int num_kb;         // stages per group pass
    int S, SX;          // code ring depth, activation ring depth
    int tab_every;      // stages per table box (16 * gs / 128)
    uint32_t code_bytes;   // codes box of a stage: gp * 16 rows x 128 bytes (1024-byte multiple)
    uint32_t x_bytes;      // activation box of a stage: 2 x BN x 128 bytes (1024-byte multiple)
    uint32_t tab_bytes;    // one table box: gp * 16 rows x 32 bytes
    uint32_t x_off, a_off, t_off, bar_off;  // from the 1024-aligned shared-memory base
    uint32_t idesc;
    unsigned int* status;
};

struct StMaps {
    CUtensorMap codes[kStMaxGP], sc[kStMaxGP], bi[kStMaxGP], x;
};

// ---- tcgen05 / TMEM primitives ----
__device__ __forceinline__ void st_tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void st_tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void st_tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void st_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void st_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void st_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void st_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
__device__ __forceinline__ void st_ld4(uint32_t taddr, uint32_t (&r)[4]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
}
__device__ __forceinline__ void st_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void st_sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}
// K-major operand in rows of 128 bytes with the 128-byte swizzle, 8-row
// core groups 1024 bytes apart (the UMMA shared-memory descriptor).
__device__ __forceinline__ uint64_t st_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(1u) << 16;
    d |= static_cast<uint64_t>(1024u >> 4) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    d |= static_cast<uint64_t>(2u) << 61;
    return d;
}

// BN: MMA N = activation rows per pass, padded (16, 32 or 64); GS: group size.
template <int BN, int GS>
__global__ void __launch_bounds__(kStThreads, 1) k_smallm_tc(const __grid_constant__ StMaps maps, const StParams p) {
    constexpr int kTabEvery = kStTabGroups * GS / kStKB;  // stages per table box
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = p.S, SX = p.SX;
    const int t0 = static_cast<int>(static_cast<int64_t>(p.P) * blockIdx.x / gridDim.x);
    const int t1 = static_cast<int>(static_cast<int64_t>(p.P) * (blockIdx.x + 1) / gridDim.x);
    const int ngroups = (t1 - t0 + p.gp - 1) / p.gp;
    uint64_t* cfull = reinterpret_cast<uint64_t*>(smem + p.bar_off);  // codes landed (TMA)
    uint64_t* cempty = cfull + kStMaxS;  // codes read (16 warps)
    uint64_t* xfull = cempty + kStMaxS;  // activation box landed (TMA)
    uint64_t* xempty = xfull + kStMaxX;  // activation box read by the MMAs (commit)
    uint64_t* tfull = xempty + kStMaxX;  // table box landed
    uint64_t* tempty = tfull + 2;        // table box read
    uint64_t* afull = tempty + 2;        // A tile written (16 warps)
    uint64_t* aempty = afull + kStNA;    // A tile read by the MMAs (commit)
    uint64_t* dfull = aempty + kStNA;    // the group's accumulator complete (commit)
    uint64_t* dempty = dfull + 1;        // the accumulator read out (16 warps)
    uint64_t* drain = dempty + 1;        // the MMA thread's last commit
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    auto codes_of = [&](int s) { return sbase + static_cast<uint32_t>(s) * p.code_bytes; };
    auto x_of = [&](int s) { return sbase + p.x_off + static_cast<uint32_t>(s) * p.x_bytes; };
    auto a_of = [&](int a) { return sbase + p.a_off + static_cast<uint32_t>(a) * 2u * kStA; };
    auto tab_of = [&](int t) { return sbase + p.t_off + static_cast<uint32_t>(t) * 2u * p.tab_bytes; };
    constexpr uint32_t kTmemCols = BN < 32 ? 32u : static_cast<uint32_t>(BN);

    pdl_launch_dependents();
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_u32(&cfull[s]), 1);
            mbar_init(smem_u32(&cempty[s]), kStW);
        }
        for (int s = 0; s < SX; ++s) {
            mbar_init(smem_u32(&xfull[s]), 1);
            mbar_init(smem_u32(&xempty[s]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&tfull[i]), 1);
            mbar_init(smem_u32(&tempty[i]), kStW);
        }
        for (int i = 0; i < kStNA; ++i) {
            mbar_init(smem_u32(&afull[i]), kStW);
            mbar_init(smem_u32(&aempty[i]), 1);
        }
        mbar_init(smem_u32(dfull), 1);
        mbar_init(smem_u32(dempty), kStW);
        mbar_init(smem_u32(drain), 1);
        mbar_fence_init();
    }
    if (warp == 1) {
        st_tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        st_tmem_relinquish();
    }
    st_fence_before();
    __syncthreads();
    st_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_wait();  // activations, weights and Y belong to earlier work

    if (warp == 0) {
        // ---------------- codes and tables producer ----------------
        if (lane == 0) {
            prefetch_tmap(&maps.codes[p.gp - 1]);
            prefetch_tmap(&maps.sc[p.gp - 1]);
            prefetch_tmap(&maps.bi[p.gp - 1]);
            const uint64_t pol = policy_evict_first();
            bool ok = true;
            int it = 0, ti = 0;
            for (int grp = 0; grp < ngroups && ok; ++grp) {
                const int ta = t0 + grp * p.gp;
                const int nt = min(p.gp, t1 - ta);
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    if (kb % kTabEvery == 0) {
                        const int ts = ti % 2;
                        if (ti >= 2) ok = mbar_wait(smem_u32(&tempty[ts]), ((ti / 2) - 1) & 1, p.status);
                        if (!ok) break;  // the box may still be in use: issue nothing more
                        const uint32_t tb = smem_u32(&tfull[ts]);
                        mbar_arrive_expect_tx(tb, 2u * static_cast<uint32_t>(nt) * 16u * 2u * kStTabGroups);
                        tma_load_2d(tab_of(ts), &maps.sc[nt - 1], (kb / kTabEvery) * kStTabGroups, ta * 16, tb, pol);
                        tma_load_2d(tab_of(ts) + p.tab_bytes, &maps.bi[nt - 1], (kb / kTabEvery) * kStTabGroups,
                                    ta * 16, tb, pol);
                        ++ti;
                    }
                    const int s = it % S;
                    if (it >= S) ok = mbar_wait(smem_u32(&cempty[s]), ((it / S) - 1) & 1, p.status);
                    if (!ok) break;
                    const uint32_t fb = smem_u32(&cfull[s]);
                    mbar_arrive_expect_tx(fb, static_cast<uint32_t>(nt) * 16u * 128u);
                    tma_load_2d(codes_of(s), &maps.codes[nt - 1], kb * kStKB, ta * 16, fb, pol);
                    ++it;
                }
            }
            // every issued copy has landed before the CTA may exit
            for (int u = it > S ? it - S : 0; u < it; ++u)
                if (!mbar_wait(smem_u32(&cfull[u % S]), (u / S) & 1, p.status)) break;
            for (int u = ti > 2 ? ti - 2 : 0; u < ti; ++u)
                if (!mbar_wait(smem_u32(&tfull[u % 2]), (u / 2) & 1, p.status)) break;
        }
    } else if (warp == 2) {
        // ---------------- activation producer ----------------
        if (lane == 0) {
            prefetch_tmap(&maps.x);
            const uint64_t pol_x = policy_evict_last();  // every CTA reads the same activations
            bool ok = true;
            int it = 0;
            for (int grp = 0; grp < ngroups && ok; ++grp) {
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    const int s = it % SX;
                    if (it >= SX) ok = mbar_wait(smem_u32(&xempty[s]), ((it / SX) - 1) & 1, p.status);
                    if (!ok) break;
                    const uint32_t fb = smem_u32(&xfull[s]);
                    mbar_arrive_expect_tx(fb, p.x_bytes);
                    tma_load_3d(x_of(s), &maps.x, 0, 0, kb * 2, fb, pol_x);
                    ++it;
                }
            }
            for (int u = it > SX ? it - SX : 0; u < it; ++u)
                if (!mbar_wait(smem_u32(&xfull[u % SX]), (u / SX) & 1, p.status)) break;
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            bool ok = true;
            int it = 0;
            for (int grp = 0; grp < ngroups && ok; ++grp) {
                // the previous group's accumulator has been read out
                if (grp >= 1) ok = mbar_wait(smem_u32(dempty), (grp - 1) & 1, p.status);
                if (!ok) break;
                st_fence_after();
                for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
                    const int sx = it % SX, a = it % kStNA;
                    ok = mbar_wait(smem_u32(&afull[a]), (it / kStNA) & 1, p.status);
                    if (ok) ok = mbar_wait(smem_u32(&xfull[sx]), (it / SX) & 1, p.status);
                    if (!ok) break;  // operands not there: issue nothing more
                    st_fence_after();
#pragma unroll
                    for (int kbi = 0; kbi < 2; ++kbi) {
                        const uint64_t ad = st_desc(a_of(a) + static_cast<uint32_t>(kbi) * kStA);
                        const uint64_t bd = st_desc(x_of(sx) + static_cast<uint32_t>(kbi * BN) * 128u);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)  // 16 BF16 (32 bytes) along K per MMA
                            st_mma(tmem_base, ad + 2u * kk, bd + 2u * kk, p.idesc, (kb | kbi | kk) != 0 ? 1u : 0u);
                    }
                    st_commit(smem_u32(&aempty[a]));
                    st_commit(smem_u32(&xempty[sx]));
                }
                if (ok) st_commit(smem_u32(dfull));
            }
            // every MMA this thread issued has finished before TMEM is freed
            st_commit(smem_u32(drain));
            mbar_wait(smem_u32(drain), 0, p.status);
        }
        __syncwarp();
    } else {
        // ---------------- dequantising warps; then each group's outputs ----------------
        const int dw = warp - 3;        // 0 .. 15
        const int dt = dw * 32 + lane;  // 0 .. 511
        const float2 m2 = make_float2(-kMagic, -kMagic);
        bool ok = true;
        int it = 0, ti = 0;
        for (int grp = 0; grp < ngroups; ++grp) {
            const int ta = t0 + grp * p.gp;
            const int nt = min(p.gp, t1 - ta);
            const int units = nt * 16 * 8;  // (row, 16-code chunk) pairs of a stage
            // This thread's units (at most two), the same in every stage of the
            // group.  16 consecutive units cover rows 2b and 2b + 1; each 8-lane
            // phase takes four chunks of one row and the other four of the other
            // row, so its code loads and its A stores each hit 8 distinct 16-byte
            // bank groups.
            uint32_t ld_off[2], st0[2], st1[2], trow[2];
            int cch[2];
            bool has[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int u = dt + i * kStW * 32;
                has[i] = u < units;
                const int q = u & 15, tq = (q >> 2) & 1;
                const int r = 2 * (u >> 4) + (tq ^ (q >> 3));
                const int c = (q & 3) + 4 * tq;
                const uint32_t sw = static_cast<uint32_t>(r & 7);
                ld_off[i] = static_cast<uint32_t>(r) * 128u + ((static_cast<uint32_t>(c) ^ sw) << 4);
                // chunk c lands in k-block c / 4 of the A tile, 16-byte units
                // 2 (c % 4) and 2 (c % 4) + 1 of row r, placed by the swizzle
                const uint32_t arow = static_cast<uint32_t>(c >> 2) * kStA + static_cast<uint32_t>(r) * 128u;
                st0[i] = arow + (((2u * static_cast<uint32_t>(c & 3)) ^ sw) << 4);
                st1[i] = arow + (((2u * static_cast<uint32_t>(c & 3) + 1u) ^ sw) << 4);
                trow[i] = static_cast<uint32_t>(r * kStTabGroups) * 2u;
                cch[i] = c;
            }
            for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
                const int ts = ti % 2;
                if (kb % kTabEvery == 0 && ok) ok = mbar_wait(smem_u32(&tfull[ts]), (ti / 2) & 1, p.status);
                const int s = it % S, a = it % kStNA;
                if (ok) ok = mbar_wait(smem_u32(&cfull[s]), (it / S) & 1, p.status);
                // the MMAs that last read this A tile are done
                if (it >= kStNA && ok) ok = mbar_wait(smem_u32(&aempty[a]), ((it / kStNA) - 1) & 1, p.status);
                const uint32_t cs = codes_of(s), as = a_of(a);
                const uint32_t sca = tab_of(ts), bia = sca + p.tab_bytes;
                const int gbase = (kb % kTabEvery) * kStKB;  // codes of the table box before this stage
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    if (!has[i]) continue;
                    const uint4 wq = lds128(cs + ld_off[i]);
                    const uint32_t so = trow[i] + static_cast<uint32_t>((gbase + 16 * cch[i]) / GS) * 2u;
                    const float sv = bf16_bits_to_f32(lds16(sca + so)), bv = bf16_bits_to_f32(lds16(bia + so));
                    const float2 s2 = make_float2(sv, sv), b2 = make_float2(bv, bv);
                    const uint32_t words[4] = {wq.x, wq.y, wq.z, wq.w};
                    uint32_t o[8];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t v = words[j];
                        const float2 q01 = __fadd2_rn(make_float2(code_magic<0>(v), code_magic<1>(v)), m2);
                        const float2 q23 = __fadd2_rn(make_float2(code_magic<2>(v), code_magic<3>(v)), m2);
                        const float2 w01 = __ffma2_rn(q01, s2, b2);
                        const float2 w23 = __ffma2_rn(q23, s2, b2);
                        o[2 * j] = pack_bf16x2(w01.x, w01.y);
                        o[2 * j + 1] = pack_bf16x2(w23.x, w23.y);
                    }
                    st_sts128(as + st0[i], o[0], o[1], o[2], o[3]);
                    st_sts128(as + st1[i], o[4], o[5], o[6], o[7]);
                }
                fence_proxy_async_smem();  // the tensor core reads the A tile through the async proxy
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(smem_u32(&afull[a]));
                    mbar_arrive(smem_u32(&cempty[s]));  // this warp is done with the stage's codes
                }
                if (kb % kTabEvery == kTabEvery - 1 || kb == p.num_kb - 1) {
                    if (lane == 0) mbar_arrive(smem_u32(&tempty[ts]));
                    ++ti;
                }
            }
            // ---- the group's outputs: TMEM lane = weight row, column = activation row ----
            if (ok) ok = mbar_wait(smem_u32(dfull), grp & 1, p.status);
            st_fence_after();
            const int q = warp & 3;          // the TMEM lane quadrant this warp may read
            const int wq = dw >> 2;          // this warp's quarter of the BN columns
            const int row = 32 * q + lane;   // weight row within the group
            const int n = ta * 16 + row;
            const bool live = row < nt * 16 && n < p.N;
#pragma unroll
            for (int c4 = 0; c4 < BN / 16; ++c4) {
                const int c0 = wq * (BN / 4) + 4 * c4;
                uint32_t r4[4];
                st_ld4(tmem_base + static_cast<uint32_t>(c0) + (static_cast<uint32_t>(32 * q) << 16), r4);
                st_ld_wait();
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int i = c0 + j;
                    if (live && i < p.m) {
                        const __nv_bfloat16 v = __float2bfloat16_rn(__uint_as_float(r4[j]));
                        p.Y[static_cast<int64_t>(i) * p.N + n] = *reinterpret_cast<const uint16_t*>(&v);
                    }
                }
            }
            st_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(dempty));
        }
    }
    st_fence_before();
    __syncthreads();
    if (warp == 1) {
        st_fence_after();
        st_tmem_dealloc(tmem_base, kTmemCols);
    }
}

bool st_a16(const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; }

struct StPlan {
    int bn, grid;
    StParams p;
    size_t smem;
};

constexpr size_t kStBarBytes = 512;

bool plan_st(const WeightView& w, int64_t m, StPlan& pl) {
    const DeviceInfo& dev = device_info();
    if (m < 1 || m > 64 || w.N < 1 || w.K < kStKB || w.K % kStKB != 0 || w.N > (1 << 30) || w.K > (1 << 30))
        return false;
    if (w.gs != 16 && w.gs != 32 && w.gs != 64 && w.gs != 128) return false;
    if (w.G % 8 != 0) return false;  // table rows must be 16-byte multiples for the tensor copies
    StParams& p = pl.p;
    p = StParams{};
    pl.bn = m <= 16 ? 16 : (m <= 32 ? 32 : 64);
    p.N = static_cast<int>(w.N);
    p.K = static_cast<int>(w.K);
    p.m = static_cast<int>(m);
    p.gs = static_cast<int>(w.gs);
    p.P = static_cast<int>((w.N + 15) / 16);
    pl.grid = p.P < dev.sm_count ? p.P : dev.sm_count;
    const int tmax = (p.P + pl.grid - 1) / pl.grid;  // most tiles a CTA owns
    const int ng = (tmax + kStMaxGP - 1) / kStMaxGP;
    p.gp = (tmax + ng - 1) / ng;
    p.num_kb = p.K / kStKB;
    p.tab_every = kStTabGroups * p.gs / kStKB;
    p.code_bytes = static_cast<uint32_t>(p.gp) * 16u * 128u;
    p.x_bytes = 2u * static_cast<uint32_t>(pl.bn) * 128u;
    p.tab_bytes = static_cast<uint32_t>(p.gp) * 16u * 2u * kStTabGroups;
    const size_t a_bytes = static_cast<size_t>(kStNA) * 2 * kStA;
    const size_t fixed = 1024 + a_bytes + 4 * static_cast<size_t>(p.tab_bytes) + kStBarBytes;
    const size_t budget = static_cast<size_t>(dev.max_smem_optin);
    p.SX = kStMaxX;
    if (budget < fixed + static_cast<size_t>(p.SX) * p.x_bytes + 2 * static_cast<size_t>(p.code_bytes)) return false;
    int S = static_cast<int>((budget - fixed - static_cast<size_t>(p.SX) * p.x_bytes) / p.code_bytes);
    if (S > kStMaxS) S = kStMaxS;
    p.S = S;
    p.x_off = static_cast<uint32_t>(S) * p.code_bytes;
    p.a_off = p.x_off + static_cast<uint32_t>(p.SX) * p.x_bytes;
    p.t_off = p.a_off + static_cast<uint32_t>(a_bytes);
    p.bar_off = p.t_off + 4u * p.tab_bytes;
    pl.smem = 1024 + p.bar_off + kStBarBytes;
    p.idesc = (1u << 4)                                   // D: fp32
              | (1u << 7)                                 // A: BF16
              | (1u << 10)                                // B: BF16
              | (static_cast<uint32_t>(pl.bn >> 3) << 17)  // N
              | (static_cast<uint32_t>(128 >> 4) << 24);   // M
    return true;
}

template <int BN, int GS>
cudaError_t launch_st_t(const StMaps& maps, const StParams& p, int grid, size_t smem, cudaStream_t stream) {
    auto kern = k_smallm_tc<BN, GS>;
    static std::atomic<int> configured[64];
    cudaError_t e = ensure_dynamic_smem(kern, smem, configured);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kern, dim3(grid), dim3(kStThreads), smem, stream, maps, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int BN>
cudaError_t launch_st_gs(const StMaps& maps, const StParams& p, int grid, size_t smem, cudaStream_t stream) {
    switch (p.gs) {
        case 16: return launch_st_t<BN, 16>(maps, p, grid, smem, stream);
        case 32: return launch_st_t<BN, 32>(maps, p, grid, smem, stream);
        case 64: return launch_st_t<BN, 64>(maps, p, grid, smem, stream);
        default: return launch_st_t<BN, 128>(maps, p, grid, smem, stream);
    }
}

}  // namespace

bool smallm_tc_supported(const WeightView& w, int64_t m, const void* X) {
    StPlan pl;
    if (!plan_st(w, m, pl)) return false;
    if (!st_a16(w.packed) || !st_a16(w.scales) || !st_a16(w.biases) || !st_a16(X)) return false;
    int major = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device_info().device);
    if (major != 10) return false;
    return tensor_maps_available();
}

// Measured faster than the alternatives for 32 < m <= 64 with at least 6
// tiles of 16 rows per SM (its A tile always has 128 rows, so shorter row
// ranges per SM waste it); below m = 32 the mma.sync stream kernels win.
bool smallm_tc_preferred(const WeightView& w, int64_t m, const void* X) {
    if (m <= 32 || !smallm_tc_supported(w, m, X)) return false;
    return (w.N + 15) / 16 >= 6 * static_cast<int64_t>(device_info().sm_count);
}

cudaError_t launch_smallm_tc(const WeightView& w, const void* X, void* Y, int64_t m, cudaStream_t stream) {
    StPlan pl;
    if (!plan_st(w, m, pl)) return cudaErrorInvalidValue;
    StParams p = pl.p;
    p.Y = static_cast<uint16_t*>(Y);
    p.status = device_status_ptr();
    StMaps maps;
    for (int t = 0; t < p.gp; ++t) {
        TensorMaps3 tm;
        if (!weight_tensor_maps(w, (t + 1) * 16, 128, CU_TENSOR_MAP_SWIZZLE_128B, kStTabGroups, &tm))
            return cudaErrorInvalidValue;
        maps.codes[t] = tm.packed;
        maps.sc[t] = tm.scales;
        maps.bi[t] = tm.biases;
    }
    if (!encode_3d_chunks(&maps.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, static_cast<uint64_t>(w.K),
                          static_cast<uint64_t>(m), static_cast<uint64_t>(w.K) * 2, 64,
                          static_cast<uint32_t>(pl.bn), 2))
        return cudaErrorInvalidValue;
    switch (pl.bn) {
        case 16: return launch_st_gs<16>(maps, p, pl.grid, pl.smem, stream);
        case 32: return launch_st_gs<32>(maps, p, pl.grid, pl.smem, stream);
        default: return launch_st_gs<64>(maps, p, pl.grid, pl.smem, stream);
    }
}

}  // namespace mlxq
