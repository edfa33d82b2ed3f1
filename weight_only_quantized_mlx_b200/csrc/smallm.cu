// Small-m gemm of the "MlxInt8Weight" page (Y = X W^T for 1 <= m <= 32):
// every weight byte is read from HBM once and dequantised once, and each
// dequantised fragment feeds all m activation rows.
//
// One CTA per SM owns a balanced range of 16-row weight tiles ("pairs" of
// 8-row octets) and walks it in groups of GP tiles; each group streams K in
// 512-code stages.  Per stage a producer lane issues a handful of large
// tensor copies (a copy costs tens of nanoseconds however small its box, so
// many small boxes starve the stream): one 3-D box of the group's rows over
// the stage's four 128-code columns (128-byte swizzle), the group's [rows x
// groups] scale and bias boxes, and one 3-D box of the stage's activation
// slice ([8 columns of 64] x [8 NT rows], zero past m and K).  A CTA's last
// group may hold fewer than GP tiles; there is a map for every group height,
// so every group takes the same three copies and a CTA never loads rows it
// does not own.
//
// A stage's work items are (tile, 64-code slice) pairs; the 16 consumer warps
// take fixed items, and all items of a warp share its slice, so the warp loads
// the activation fragments once per stage for all its tiles.  Per 16-code
// chunk and pair of rows (g, g + 8) a lane dequantises with paired fp32
// operations (one code of row g beside one of row g + 8), rounds to BF16 (the
// exact weight dequantize_to writes) and feeds the A fragment of mma.sync
// m16n8k16 for each of the NT 8-row activation tiles (BF16 in, fp32
// accumulate).  At the end of a group the slices' partial sums meet in shared
// memory in a fixed order and the group's outputs are written.
//
// All waits are bounded.  After a wait gives up, the producer stops issuing
// copies and, before the CTA exits, waits (bounded) for the copies it has in
// flight.
#include "device_common.cuh"
#include "kernels.h"
#include "tensor_map.h"

namespace mlxq {
namespace {

constexpr int kSmW = 16;           // consumer warps
constexpr int kSmSlices = 8;       // 64-code slices of a 512-code stage
constexpr int kSmKB = 512;         // codes per stage
constexpr int kSmNB = kSmKB / 128; // 128-code columns per stage
constexpr int kSmMaxStages = 8;
constexpr uint32_t kTileBox = 16u * 128u;  // one tile's box of one column

struct SmParams {
    uint16_t* Y;  // [m, N]
    int N, K, G, m;
    int P;        // 16-row tiles of the weight
    int num_kb, S, gpk;
    uint32_t col_bytes;   // one 128-code column of a group: GP tiles
    uint32_t tab_bytes;   // one table (scales or biases) of a group, 128-byte padded
    uint32_t x_off;       // activation boxes within a stage
    uint32_t xbox_bytes;  // one [8 NT rows x 64 columns] box
    uint32_t stage_bytes, red_off, bar_off;
    unsigned int* status;
};

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One word (4 codes) of row g (u) and of row g + 8 (v) -> A fragment
// registers: a0 = row g codes 0,1; a1 = row g+8 codes 0,1; a2 = row g codes
// 2,3; a3 = row g+8 codes 2,3.  s2 / b2 = (row g, row g+8).
__device__ __forceinline__ void dequant_pair(uint32_t u, uint32_t v, float2 s2, float2 b2, uint32_t& a0,
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

// NT: 8-row activation tiles (m <= 8 NT); GP: weight tiles per group (the
// warps' items per stage are GP * 8, JMAX = GP / 2 per warp); GS: group size.
// Tensor maps of one launch: for a group of t + 1 tiles, pg[t] (3-D codes box
// of the group's rows over a stage's columns) and sg[t] / bg[t] (the group's
// scale / bias rows); x the stage's activation slice (3-D box).
constexpr int kSmMaxGP = 4;
struct SmMaps {
    CUtensorMap pg[kSmMaxGP], sg[kSmMaxGP], bg[kSmMaxGP], x;
};

template <int NT, int GP, int GS>
__global__ void __launch_bounds__((kSmW + 1) * 32, 1)
    k_smallm(const __grid_constant__ SmMaps maps, const SmParams p) {
    constexpr int JMAX = GP * kSmSlices / kSmW;
    static_assert(JMAX >= 1 && GP * kSmSlices == JMAX * kSmW, "items must divide evenly over the warps");
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tq = lane & 3;
    const int S = p.S;
    // this CTA's tiles: a balanced share of all P
    const int t0 = static_cast<int>(static_cast<int64_t>(p.P) * blockIdx.x / gridDim.x);
    const int t1 = static_cast<int>(static_cast<int64_t>(p.P) * (blockIdx.x + 1) / gridDim.x);
    const int ngroups = (t1 - t0 + GP - 1) / GP;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.bar_off);
    uint64_t* empty = full + kSmMaxStages;
    float* red = reinterpret_cast<float*>(smem + p.red_off);
    auto stage_of = [&](int s) { return sbase + static_cast<uint32_t>(s) * p.stage_bytes; };

    pdl_launch_dependents();
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), kSmW);
        }
        mbar_fence_init();
    }
    __syncthreads();

    if (warp == kSmW) {
        // ---------------- producer ----------------
        if (lane == 0) {
            prefetch_tmap(&maps.pg[GP - 1]);
            prefetch_tmap(&maps.sg[GP - 1]);
            prefetch_tmap(&maps.bg[GP - 1]);
            prefetch_tmap(&maps.x);
            pdl_wait();
            const uint64_t pol = policy_evict_first();
            const uint64_t pol_x = policy_evict_last();  // every CTA reads the same activations
            const uint32_t tab_tile = 16u * static_cast<uint32_t>(p.gpk) * 2u;
            bool ok = true;
            int it = 0;
            for (int grp = 0; grp < ngroups && ok; ++grp) {
                const int ta = t0 + grp * GP;
                const int nt = min(GP, t1 - ta);
                for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
                    const int s = it % S;
                    if (it >= S) ok = mbar_wait(smem_u32(&empty[s]), ((it / S) - 1) & 1, p.status);
                    if (!ok) break;  // consumers may still be reading this slot: issue nothing more
                    const int col0 = kb * kSmKB;
                    int nbox = (p.K - col0 + 127) / 128;
                    if (nbox > kSmNB) nbox = kSmNB;
                    const uint32_t bar = smem_u32(&full[s]);
                    const uint32_t st = stage_of(s);
                    const uint32_t sca = st + kSmNB * p.col_bytes;
                    const uint32_t x_tx = static_cast<uint32_t>(kSmKB / 64) * p.xbox_bytes;
                    // the group's rows over the stage's columns, and its tables
                    // (past K the boxes read zeros)
                    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nt) * (kSmNB * kTileBox + 2u * tab_tile) + x_tx);
                    tma_load_3d(st, &maps.pg[nt - 1], 0, ta * 16, kb * kSmNB, bar, pol);
                    tma_load_2d(sca, &maps.sg[nt - 1], kb * p.gpk, ta * 16, bar, pol);
                    tma_load_2d(sca + p.tab_bytes, &maps.bg[nt - 1], kb * p.gpk, ta * 16, bar, pol);
                    tma_load_3d(st + p.x_off, &maps.x, 0, 0, kb * (kSmKB / 64), bar, pol_x);
                }
            }
            // every issued copy has landed before the CTA may exit
            for (int u = it > S ? it - S : 0; u < it; ++u)
                if (!mbar_wait(smem_u32(&full[u % S]), (u / S) & 1, p.status)) break;
        }
        return;
    }

    // ---------------- consumers ----------------
    const int ctid = threadIdx.x;
    pdl_wait();  // the output belongs to earlier work
    const int sl = warp % kSmSlices;  // this warp's slice, the same for all its items
    const int b = sl >> 1;            // 128-code column
    const int c = 2 * tq + (sl & 1);  // this lane's 16-code chunk of the column
    const uint32_t swz = static_cast<uint32_t>(c ^ g) << 4;
    // activation fragments: box 2 b + c / 4 of the stage, 16-byte units
    // 2 (c % 4) and 2 (c % 4) + 1 of row 8 t + g, placed by the swizzle
    const uint32_t xbox = static_cast<uint32_t>(2 * b + (c >> 2)) * p.xbox_bytes;
    const uint32_t xu0 = static_cast<uint32_t>((2 * (c & 3)) ^ g) << 4;
    const uint32_t xu1 = static_cast<uint32_t>((2 * (c & 3) + 1) ^ g) << 4;
    const uint32_t tab_tile = 16u * static_cast<uint32_t>(p.gpk) * 2u;
    const uint32_t grp_off = static_cast<uint32_t>((128 * b + 16 * c) / GS) * 2u;
    const int GR = GP * 16;  // rows of a group
    bool ok = true;
    int it = 0;
    for (int grp = 0; grp < ngroups; ++grp) {
        const int ta = t0 + grp * GP;
        const int nt = min(GP, t1 - ta);
        float acc[JMAX][NT][4];
#pragma unroll
        for (int j = 0; j < JMAX; ++j)
#pragma unroll
            for (int t = 0; t < NT; ++t) acc[j][t][0] = acc[j][t][1] = acc[j][t][2] = acc[j][t][3] = 0.f;
        for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
            const int s = it % S;
            if (ok) ok = mbar_wait(smem_u32(&full[s]), (it / S) & 1, p.status);
            const uint32_t st = stage_of(s);
            uint32_t bx[NT][8];
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const uint32_t ra = st + p.x_off + xbox + static_cast<uint32_t>(8 * t + g) * 128u;
                const uint4 v0 = lds128(ra + xu0), v1 = lds128(ra + xu1);
                bx[t][0] = v0.x; bx[t][1] = v0.y; bx[t][2] = v0.z; bx[t][3] = v0.w;
                bx[t][4] = v1.x; bx[t][5] = v1.y; bx[t][6] = v1.z; bx[t][7] = v1.w;
            }
#pragma unroll
            for (int j = 0; j < JMAX; ++j) {
                const int q = (warp + kSmW * j) / kSmSlices;  // tile within the group
                if (q < nt) {  // warp-uniform
                    // the group's box: [column][nt * 16 rows][128 bytes]
                    const uint32_t boxa = st + static_cast<uint32_t>(b * nt + q) * kTileBox +
                                          static_cast<uint32_t>(g) * 128u + swz;
                    const uint4 wu = lds128(boxa), wv = lds128(boxa + 8u * 128u);
                    const uint32_t sca = st + kSmNB * p.col_bytes + static_cast<uint32_t>(q) * tab_tile;
                    const uint32_t so = static_cast<uint32_t>(g * p.gpk) * 2u + grp_off;
                    const uint32_t so8 = so + static_cast<uint32_t>(8 * p.gpk) * 2u;
                    const float2 s2 = make_float2(bf16_bits_to_f32(lds16(sca + so)), bf16_bits_to_f32(lds16(sca + so8)));
                    const float2 b2 = make_float2(bf16_bits_to_f32(lds16(sca + p.tab_bytes + so)),
                                                  bf16_bits_to_f32(lds16(sca + p.tab_bytes + so8)));
                    const uint32_t uu[4] = {wu.x, wu.y, wu.z, wu.w}, vv[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                    for (int w4 = 0; w4 < 4; ++w4) {
                        uint32_t a0, a1, a2, a3;
                        dequant_pair(uu[w4], vv[w4], s2, b2, a0, a1, a2, a3);
#pragma unroll
                        for (int t = 0; t < NT; ++t)
                            mma_16816(acc[j][t], a0, a1, a2, a3, bx[t][2 * w4], bx[t][2 * w4 + 1]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
        }
        // ---- the group's outputs: slices summed in a fixed order ----
        // red[slice][activation row][group row]
#pragma unroll
        for (int j = 0; j < JMAX; ++j) {
            const int q = (warp + kSmW * j) / kSmSlices;
            if (q < nt) {
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    const int i = 8 * t + 2 * tq;  // D columns i, i + 1; rows g, g + 8
                    float* rb = red + (sl * 8 * NT + i) * GR + 16 * q + g;
                    if (i < p.m) {
                        rb[0] = acc[j][t][0];
                        rb[8] = acc[j][t][2];
                    }
                    if (i + 1 < p.m) {
                        rb[GR] = acc[j][t][1];
                        rb[GR + 8] = acc[j][t][3];
                    }
                }
            }
        }
        named_bar_sync(1, kSmW * 32);
        const int rows = min(nt * 16, p.N - ta * 16);
        for (int o = ctid; o < p.m * rows; o += kSmW * 32) {
            const int i = o / rows, r = o - i * rows;
            float v = 0.f;
#pragma unroll
            for (int q = 0; q < kSmSlices; ++q) v += red[(q * 8 * NT + i) * GR + r];
            const __nv_bfloat16 ob = __float2bfloat16_rn(v);
            p.Y[static_cast<int64_t>(i) * p.N + ta * 16 + r] = *reinterpret_cast<const uint16_t*>(&ob);
        }
        named_bar_sync(1, kSmW * 32);  // red is read before the next group writes it
    }
}

template <int NT, int GP, int GS>
cudaError_t launch_sm_t(const SmMaps& m, const SmParams& p, int grid, size_t smem, cudaStream_t stream) {
    auto kern = k_smallm<NT, GP, GS>;
    static std::atomic<int> configured[64];
    cudaError_t e = ensure_dynamic_smem(kern, smem, configured);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kern, dim3(grid), dim3((kSmW + 1) * 32), smem, stream, m, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int NT, int GP>
cudaError_t launch_sm_gs(const SmMaps& m, const SmParams& p, int gs, int grid, size_t smem, cudaStream_t stream) {
    switch (gs) {
        case 16: return launch_sm_t<NT, GP, 16>(m, p, grid, smem, stream);
        case 32: return launch_sm_t<NT, GP, 32>(m, p, grid, smem, stream);
        default: return launch_sm_t<NT, GP, 64>(m, p, grid, smem, stream);
    }
}

bool a16(const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; }

struct SmPlan {
    int nt, gp, grid, S;
    SmParams p;
    size_t smem;
};

bool plan_sm(const WeightView& w, int64_t m, SmPlan& pl) {
    const DeviceInfo& dev = device_info();
    // K % 128 == 0: the 3-D views of the codes (128-byte columns) and of the
    // activations (64-column blocks)
    if (m < 1 || m > 32 || w.N < 1 || w.K < 128 || w.K % 128 != 0 || w.N > (1 << 30) || w.K > (1 << 30)) return false;
    // 512-code stages: a stage's table rows (512 / gs groups) must be 16-byte
    // multiples, and a 16-code chunk must not straddle a group
    if (w.gs != 16 && w.gs != 32 && w.gs != 64) return false;
    if (w.G % 8 != 0) return false;
    pl.nt = m <= 8 ? 1 : (m <= 16 ? 2 : 4);
    pl.gp = pl.nt == 4 ? 2 : 4;
    SmParams& p = pl.p;
    p = SmParams{};
    p.N = static_cast<int>(w.N);
    p.K = static_cast<int>(w.K);
    p.G = static_cast<int>(w.G);
    p.m = static_cast<int>(m);
    p.P = static_cast<int>((w.N + 15) / 16);
    p.gpk = kSmKB / static_cast<int>(w.gs);
    p.num_kb = static_cast<int>((w.K + kSmKB - 1) / kSmKB);
    p.col_bytes = static_cast<uint32_t>(pl.gp) * kTileBox;  // largest group
    p.tab_bytes = (static_cast<uint32_t>(pl.gp) * 16u * p.gpk * 2u + 127u) / 128u * 128u;
    p.xbox_bytes = static_cast<uint32_t>(8 * pl.nt) * 128u;
    p.x_off = kSmNB * p.col_bytes + 2u * p.tab_bytes;
    p.x_off = (p.x_off + 1023u) / 1024u * 1024u;  // swizzled boxes start on 1024-byte boundaries
    p.stage_bytes = p.x_off + static_cast<uint32_t>(kSmKB / 64) * p.xbox_bytes;
    p.stage_bytes = (p.stage_bytes + 1023u) / 1024u * 1024u;
    const uint32_t red_bytes = static_cast<uint32_t>(kSmSlices * 8 * pl.nt * pl.gp * 16 * 4);
    const size_t fixed = 1024 + red_bytes + 2 * kSmMaxStages * sizeof(uint64_t);
    const size_t budget = static_cast<size_t>(dev.max_smem_optin);
    if (budget < fixed + 2 * static_cast<size_t>(p.stage_bytes)) return false;
    int S = static_cast<int>((budget - fixed) / p.stage_bytes);
    if (S > kSmMaxStages) S = kSmMaxStages;
    pl.S = S;
    p.S = S;
    p.red_off = static_cast<uint32_t>(S) * p.stage_bytes;
    p.bar_off = p.red_off + red_bytes;
    pl.smem = 1024 + p.bar_off + 2 * kSmMaxStages * sizeof(uint64_t);
    pl.grid = p.P < dev.sm_count ? p.P : dev.sm_count;
    return true;
}

}  // namespace

bool smallm_supported(const WeightView& w, int64_t m, const void* X) {
    SmPlan pl;
    if (!plan_sm(w, m, pl)) return false;
    if (!a16(w.packed) || !a16(w.scales) || !a16(w.biases) || !a16(X)) return false;
    return tensor_maps_available();
}

bool smallm_preferred(const WeightView& w, int64_t m, const void* X) {
    if (m <= 8 || !smallm_supported(w, m, X)) return false;
    return (w.N + 15) / 16 >= 6 * static_cast<int64_t>(device_info().sm_count);
}

cudaError_t launch_smallm(const WeightView& w, const void* X, void* Y, int64_t m, cudaStream_t stream) {
    SmPlan pl;
    if (!plan_sm(w, m, pl)) return cudaErrorInvalidValue;
    SmParams p = pl.p;
    p.Y = static_cast<uint16_t*>(Y);
    p.status = device_status_ptr();
    SmMaps mp;
    for (int t = 0; t < pl.gp; ++t) {
        TensorMaps3 tabs;
        if (!weight_tensor_maps(w, (t + 1) * 16, 128, CU_TENSOR_MAP_SWIZZLE_128B, p.gpk, &tabs) ||
            !encode_3d_chunks(&mp.pg[t], CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w.packed, static_cast<uint64_t>(w.K),
                              static_cast<uint64_t>(w.N), static_cast<uint64_t>(w.K), 128,
                              static_cast<uint32_t>((t + 1) * 16), kSmNB))
            return cudaErrorInvalidValue;
        mp.sg[t] = tabs.scales;
        mp.bg[t] = tabs.biases;
    }
    if (!encode_3d_chunks(&mp.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, static_cast<uint64_t>(w.K),
                          static_cast<uint64_t>(m), static_cast<uint64_t>(w.K) * 2, 64,
                          static_cast<uint32_t>(8 * pl.nt), kSmKB / 64))
        return cudaErrorInvalidValue;
    const int gs = static_cast<int>(w.gs);
    if (pl.nt == 1) return launch_sm_gs<1, 4>(mp, p, gs, pl.grid, pl.smem, stream);
    if (pl.nt == 2) return launch_sm_gs<2, 4>(mp, p, gs, pl.grid, pl.smem, stream);
    return launch_sm_gs<4, 2>(mp, p, gs, pl.grid, pl.smem, stream);
}

}  // namespace mlxq
