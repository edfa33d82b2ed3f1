// Plain, slow, single-threaded CPU oracle for the 8-bit group-affine
// quantized linear layer ("MlxInt8Weight" API page).
//
// TEST INFRASTRUCTURE ONLY. This file is the independent checker of the CUDA
// library. Only the test suite, the smoke check and the CPU-baseline leg of the
// benchmark may load it. It shares no code, header, table or helper with the
// CUDA path under weight_only_quantized_mlx_b200/csrc, and it includes nothing
// from there.
//
// Build: g++ -O2 -ffp-contract=off -shared -fPIC (see oracle/build.py).
// -ffp-contract=off keeps every multiply and add a separately rounded
// operation unless std::fma is written explicitly.
//
// What each function follows (MlxInt8Weight page):
//   * struct fields "packed", "scales", "biases": packed is
//     [out_features, in_features/4] bytes held in uint32 words; scales and
//     biases are [out_features, in_features/group_size] BF16, one per group.
//   * "load": group_size must divide in_features.
//   * "dequantize_to": the full dequantised weight, BF16.  The
//     quantized-storage page also names dequantisation to f16 and f32: the
//     fp32 affine value itself, and that value rounded to FP16 (nearest even).
//   * "gemv": y = W x.
//   * "gemv_silu_gate": y = W (silu(gate) * up).
//   * "gemv_silu_gate_resid": y[n] = x_resid[n] + sum_k W[n,k]*(silu(gate[k])*up[k]).
//   * "gemm": Y = X W^T, X [m, in_features], Y [m, out_features].
//   * quantize (no page entry: the inverse of the format, which the head
//     builder of the model pages applies to BF16 projections; the pages give
//     no algorithm).  Parity unpinned against the pages: the min/max affine
//     reading below is pinned by invariants only (grid identity, error bound,
//     constant groups).
//
// Readings taken where the page is silent:
//   * q[n,k] is byte (k mod 4) of word packed[n, k/4], little-endian
//     (byte j = bits 8j..8j+7), unsigned 0..255.
//   * W[n,k] = bf16_rne( fma_f32(s[n,g], q[n,k], b[n,g]) ), g = floor(k/gs):
//     groups are gs consecutive columns of one row.
//   * Products accumulate in fp64 in the order k = 0..K-1 over the BF16 W.
//   * silu(t) = t / (1 + exp(-t)), in fp64; silu(gate)*up is NOT rounded.
//   * Each output is rounded once, fp64 -> BF16, round to nearest even.
//
// Parity status: every function pinned (see tests/test_oracle.py), except
// that oracle_quantize's algorithm itself has no page to be checked against.
//
// quantize reading (per row, per group of gs columns, all fp32, each
// operation rounded to nearest even, no fused operations):
//   lo = min, hi = max of the group;  s = bf16((hi - lo) / 255);
//   b = bf16(lo);  q = clamp(rint((w - b) / s), 0, 255), or q = 0 if s == 0.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

// ---- BF16 (1 sign, 8 exponent, 7 stored significand bits) -----------------

// fp32 -> bf16, round to nearest, ties to even, written on the bit pattern.
// NaN stays NaN (quiet bit forced); infinities and overflow behave as IEEE.
uint16_t f32_to_bf16(float v) {
    uint32_t u;
    std::memcpy(&u, &v, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu) != 0u) {
        return static_cast<uint16_t>((u >> 16) | 0x0040u);  // quiet NaN
    }
    const uint32_t lsb = (u >> 16) & 1u;       // last kept bit
    const uint32_t rounded = u + 0x7FFFu + lsb;  // half-way goes to even
    return static_cast<uint16_t>(rounded >> 16);
}

// fp64 -> bf16 with ONE rounding (nearest, ties to even). Written from the
// format's definition: a bf16 number is an integer multiple of its quantum
// 2^(e-8) where 2^(e-1) <= |v| < 2^e, the quantum never going below the
// subnormal step 2^-133; magnitudes that round to 2^128 or above overflow.
uint16_t f64_to_bf16(double v) {
    if (std::isnan(v)) return 0x7FC0u;
    if (v == 0.0) return std::signbit(v) ? 0x8000u : 0x0000u;
    if (std::isinf(v)) return v > 0 ? 0x7F80u : 0xFF80u;
    int e = 0;
    std::frexp(v, &e);                       // |v| = m * 2^e, 0.5 <= m < 1
    const int qexp = (e < -125 ? -125 : e) - 8;  // quantum 2^qexp
    double r = std::nearbyint(std::ldexp(v, -qexp));  // ties to even (default mode)
    r = std::ldexp(r, qexp);
    if (std::fabs(r) >= std::ldexp(1.0, 128)) return v > 0 ? 0x7F80u : 0xFF80u;
    const float f = static_cast<float>(r);  // exact: r has <= 8 significant bits
    uint32_t u;
    std::memcpy(&u, &f, 4);
    return static_cast<uint16_t>(u >> 16);
}

// ---- FP16 (IEEE binary16: 1 sign, 5 exponent, 10 stored significand bits) --

// fp32 -> fp16, round to nearest, ties to even, written on the fp32 bit
// pattern.  A finite fp32 value is sig * 2^(E - 23) with a 24-bit integer
// significand sig (implicit bit included for normal numbers).  Its fp16
// quantum is 2^(max(E, -14) - 10): 10 fraction bits for normal numbers, the
// fixed subnormal step 2^-24 below 2^-14.  The dropped low bits of sig decide
// the rounding (above half: up; exactly half: to the even neighbour).  A carry
// out of the significand moves into the exponent field by itself, so the
// largest subnormal rounds up to the smallest normal and 65520 and above
// overflow to infinity.  NaN stays NaN (quiet bit set, top payload bits kept).
uint16_t f32_to_f16(float v) {
    uint32_t u;
    std::memcpy(&u, &v, 4);
    const uint16_t sign = static_cast<uint16_t>((u >> 16) & 0x8000u);
    const uint32_t a = u & 0x7FFFFFFFu;
    if (a > 0x7F800000u) return static_cast<uint16_t>(sign | 0x7E00u | ((a >> 13) & 0x3FFu));
    if (a == 0x7F800000u) return static_cast<uint16_t>(sign | 0x7C00u);
    const int biased = static_cast<int>(a >> 23);
    const uint32_t sig = biased == 0 ? (a & 0x7FFFFFu) : ((a & 0x7FFFFFu) | 0x800000u);
    const int E = biased == 0 ? -126 : biased - 127;
    if (E > 15) return static_cast<uint16_t>(sign | 0x7C00u);  // |v| >= 2^16
    const int qe = (E < -14 ? -14 : E) - 10;                   // fp16 quantum 2^qe
    const int shift = qe - (E - 23);                           // dropped bits, >= 13
    if (shift > 24) return sign;  // |v| < 2^-25: below half the smallest subnormal
    uint32_t mant = sig >> shift;
    const uint32_t rem = sig & ((1u << shift) - 1u);
    const uint32_t half = 1u << (shift - 1);
    if (rem > half || (rem == half && (mant & 1u))) mant += 1u;
    const uint32_t bits = (static_cast<uint32_t>((E < -14 ? -14 : E) + 14) << 10) + mant;
    return static_cast<uint16_t>(sign | (bits >= 0x7C00u ? 0x7C00u : bits));
}

float bf16_to_f32(uint16_t h) {
    const uint32_t u = static_cast<uint32_t>(h) << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return f;
}

// ---- the weight encoding ----------------------------------------------------

// Code q[n,k]: byte (k mod 4) of word packed[n, k/4], little-endian.
inline uint32_t code_at(const uint32_t* packed, int64_t K, int64_t n, int64_t k) {
    const uint32_t word = packed[n * (K / 4) + k / 4];
    return (word >> (8 * (k % 4))) & 0xFFu;
}

// fp32 value of the affine map before rounding: fma(s, q, b).
inline float affine_f32(const uint32_t* packed, const uint16_t* scales,
                        const uint16_t* biases, int64_t K, int64_t gs,
                        int64_t n, int64_t k) {
    const int64_t G = K / gs;
    const int64_t g = k / gs;
    const float s = bf16_to_f32(scales[n * G + g]);
    const float b = bf16_to_f32(biases[n * G + g]);
    const float q = static_cast<float>(code_at(packed, K, n, k));
    return std::fma(s, q, b);
}

// Row n of the BF16 weight, widened to double (exact).
void weight_row_f64(const uint32_t* packed, const uint16_t* scales,
                    const uint16_t* biases, int64_t K, int64_t gs, int64_t n,
                    double* row) {
    for (int64_t k = 0; k < K; ++k) {
        const uint16_t w = f32_to_bf16(affine_f32(packed, scales, biases, K, gs, n, k));
        row[k] = static_cast<double>(bf16_to_f32(w));
    }
}

double silu_f64(double t) { return t / (1.0 + std::exp(-t)); }

}  // namespace

extern "C" {

// ---- scalar conversions (exposed so the tests can pin them) ---------------
uint16_t oracle_bf16_from_f32(float v) { return f32_to_bf16(v); }
uint16_t oracle_bf16_from_f64(double v) { return f64_to_bf16(v); }
uint16_t oracle_f16_from_f32(float v) { return f32_to_f16(v); }
float oracle_f32_from_bf16(uint16_t h) { return bf16_to_f32(h); }
double oracle_silu(double t) { return silu_f64(t); }

// ---- unpack: q[n,k] for the whole [N, K] weight ---------------------------
void oracle_unpack(const uint32_t* packed, int64_t N, int64_t K, uint8_t* q) {
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            q[n * K + k] = static_cast<uint8_t>(code_at(packed, K, n, k));
}

// ---- dequantize_to ----------------------------------------------------------
// fp32 affine values before the BF16 rounding.
void oracle_dequant_f32(const uint32_t* packed, const uint16_t* scales,
                        const uint16_t* biases, int64_t N, int64_t K, int64_t gs,
                        float* w) {
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            w[n * K + k] = affine_f32(packed, scales, biases, K, gs, n, k);
}

// fp32 affine values rounded to FP16 (nearest even), as bit patterns.
void oracle_dequant_f16(const uint32_t* packed, const uint16_t* scales,
                        const uint16_t* biases, int64_t N, int64_t K, int64_t gs,
                        uint16_t* w) {
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            w[n * K + k] = f32_to_f16(affine_f32(packed, scales, biases, K, gs, n, k));
}

// The BF16 weight, row-major [N, K], as bit patterns.
void oracle_dequant(const uint32_t* packed, const uint16_t* scales,
                    const uint16_t* biases, int64_t N, int64_t K, int64_t gs,
                    uint16_t* w) {
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            w[n * K + k] = f32_to_bf16(affine_f32(packed, scales, biases, K, gs, n, k));
}

// ---- gemv: y = W x ------------------------------------------------------------
void oracle_gemv_f64(const uint32_t* packed, const uint16_t* scales,
                     const uint16_t* biases, int64_t N, int64_t K, int64_t gs,
                     const uint16_t* x, double* y) {
    std::vector<double> row(static_cast<size_t>(K));
    for (int64_t n = 0; n < N; ++n) {
        weight_row_f64(packed, scales, biases, K, gs, n, row.data());
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k) acc += row[k] * static_cast<double>(bf16_to_f32(x[k]));
        y[n] = acc;
    }
}

void oracle_gemv(const uint32_t* packed, const uint16_t* scales,
                 const uint16_t* biases, int64_t N, int64_t K, int64_t gs,
                 const uint16_t* x, uint16_t* y) {
    std::vector<double> acc(static_cast<size_t>(N));
    oracle_gemv_f64(packed, scales, biases, N, K, gs, x, acc.data());
    for (int64_t n = 0; n < N; ++n) y[n] = f64_to_bf16(acc[n]);
}

// ---- silu gate: h[k] = silu(gate[k]) * up[k] (fp64, never rounded) ---------
void oracle_silu_gate_f64(const uint32_t* packed, const uint16_t* scales,
                          const uint16_t* biases, int64_t N, int64_t K, int64_t gs,
                          const uint16_t* gate, const uint16_t* up, double* y) {
    std::vector<double> h(static_cast<size_t>(K));
    for (int64_t k = 0; k < K; ++k)
        h[k] = silu_f64(bf16_to_f32(gate[k])) * static_cast<double>(bf16_to_f32(up[k]));
    std::vector<double> row(static_cast<size_t>(K));
    for (int64_t n = 0; n < N; ++n) {
        weight_row_f64(packed, scales, biases, K, gs, n, row.data());
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k) acc += row[k] * h[k];
        y[n] = acc;
    }
}

void oracle_silu_gate(const uint32_t* packed, const uint16_t* scales,
                      const uint16_t* biases, int64_t N, int64_t K, int64_t gs,
                      const uint16_t* gate, const uint16_t* up, uint16_t* y) {
    std::vector<double> acc(static_cast<size_t>(N));
    oracle_silu_gate_f64(packed, scales, biases, N, K, gs, gate, up, acc.data());
    for (int64_t n = 0; n < N; ++n) y[n] = f64_to_bf16(acc[n]);
}

// ---- silu gate + residual: y[n] = x_resid[n] + sum_k W[n,k] h[k] -------------
void oracle_silu_gate_resid_f64(const uint32_t* packed, const uint16_t* scales,
                                const uint16_t* biases, int64_t N, int64_t K,
                                int64_t gs, const uint16_t* gate, const uint16_t* up,
                                const uint16_t* x_resid, double* y) {
    oracle_silu_gate_f64(packed, scales, biases, N, K, gs, gate, up, y);
    for (int64_t n = 0; n < N; ++n) y[n] = static_cast<double>(bf16_to_f32(x_resid[n])) + y[n];
}

void oracle_silu_gate_resid(const uint32_t* packed, const uint16_t* scales,
                            const uint16_t* biases, int64_t N, int64_t K, int64_t gs,
                            const uint16_t* gate, const uint16_t* up,
                            const uint16_t* x_resid, uint16_t* y) {
    std::vector<double> acc(static_cast<size_t>(N));
    oracle_silu_gate_resid_f64(packed, scales, biases, N, K, gs, gate, up, x_resid, acc.data());
    for (int64_t n = 0; n < N; ++n) y[n] = f64_to_bf16(acc[n]);
}

// BF16-materialised silu(gate)*up, for the unfused-chain comparison.
void oracle_silu_mul(const uint16_t* gate, const uint16_t* up, int64_t K, uint16_t* h) {
    for (int64_t k = 0; k < K; ++k)
        h[k] = f64_to_bf16(silu_f64(bf16_to_f32(gate[k])) * static_cast<double>(bf16_to_f32(up[k])));
}

// ---- gemm: Y[i,n] = sum_k X[i,k] W[n,k], X [m, K], Y [m, N] ----------------
void oracle_gemm_f64(const uint32_t* packed, const uint16_t* scales,
                     const uint16_t* biases, int64_t N, int64_t K, int64_t gs,
                     const uint16_t* X, int64_t m, double* Y) {
    std::vector<double> xd(static_cast<size_t>(m * K));
    for (int64_t t = 0; t < m * K; ++t) xd[t] = static_cast<double>(bf16_to_f32(X[t]));
    std::vector<double> row(static_cast<size_t>(K));
    for (int64_t n = 0; n < N; ++n) {
        weight_row_f64(packed, scales, biases, K, gs, n, row.data());
        for (int64_t i = 0; i < m; ++i) {
            const double* xi = xd.data() + i * K;
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += xi[k] * row[k];
            Y[i * N + n] = acc;
        }
    }
}

void oracle_gemm(const uint32_t* packed, const uint16_t* scales,
                 const uint16_t* biases, int64_t N, int64_t K, int64_t gs,
                 const uint16_t* X, int64_t m, uint16_t* Y) {
    std::vector<double> acc(static_cast<size_t>(m * N));
    oracle_gemm_f64(packed, scales, biases, N, K, gs, X, m, acc.data());
    for (int64_t t = 0; t < m * N; ++t) Y[t] = f64_to_bf16(acc[t]);
}

// quantize: BF16 W [N, K] -> packed codes, BF16 scales and biases [N, K/gs].
void oracle_quantize(const uint16_t* w, int64_t N, int64_t K, int64_t gs, uint32_t* packed,
                     uint16_t* scales, uint16_t* biases) {
    const int64_t G = K / gs;
    std::vector<uint8_t> q(static_cast<size_t>(K));
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t g = 0; g < G; ++g) {
            const uint16_t* src = w + n * K + g * gs;
            float lo = bf16_to_f32(src[0]), hi = lo;
            for (int64_t j = 1; j < gs; ++j) {
                const float v = bf16_to_f32(src[j]);
                if (v < lo) lo = v;
                if (v > hi) hi = v;
            }
            const float range = hi - lo;
            const uint16_t sb = f32_to_bf16(range / 255.0f);
            const uint16_t bb = f32_to_bf16(lo);
            const float sf = bf16_to_f32(sb), bf = bf16_to_f32(bb);
            for (int64_t j = 0; j < gs; ++j) {
                float c = 0.0f;
                if (sf != 0.0f) {
                    const float d = bf16_to_f32(src[j]) - bf;
                    c = std::nearbyint(d / sf);  // default rounding: to nearest, ties to even
                    if (c < 0.0f) c = 0.0f;
                    if (c > 255.0f) c = 255.0f;
                }
                q[static_cast<size_t>(g * gs + j)] = static_cast<uint8_t>(c);
            }
            scales[n * G + g] = sb;
            biases[n * G + g] = bb;
        }
        for (int64_t k4 = 0; k4 < K / 4; ++k4) {
            uint32_t word = 0;
            for (int j = 0; j < 4; ++j) word |= static_cast<uint32_t>(q[static_cast<size_t>(4 * k4 + j)]) << (8 * j);
            packed[n * (K / 4) + k4] = word;
        }
    }
}

}  // extern "C"
