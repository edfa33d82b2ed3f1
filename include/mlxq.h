/*
 * mlxq.h - C ABI of the B200 (sm_100a) library for the 8-bit group-affine
 * quantized linear layer described on the "MlxInt8Weight" API page.
 *
 * The weight format (page: struct MlxInt8Weight, fields packed/scales/biases):
 *   packed  uint32 [out_features, in_features/4], row-major.  Each word holds
 *           four unsigned 8-bit codes; byte j (bits 8j..8j+7) of word w of a
 *           row is the code of column 4w+j (little-endian).
 *   scales  BF16 [out_features, in_features/group_size], row-major.
 *   biases  BF16 [out_features, in_features/group_size], row-major.
 *   Weight element: W[n,k] = bf16( fma_f32(scale[n,g], q[n,k], bias[n,g]) ),
 *   g = k / group_size (groups are group_size consecutive columns of a row).
 *
 * Conventions for every call:
 *   - Device pointers are plain CUDA device addresses.  BF16 buffers hold
 *     IEEE bfloat16 values (2 bytes each), contiguous, row-major.
 *   - `stream` is a cudaStream_t value cast to uint64_t (0 = legacy default
 *     stream).  Kernel calls are asynchronous on that stream; inputs must stay
 *     valid and outputs untouched by others until the stream passes the call.
 *   - Every call returns MLXQ_OK (0) or one of the MLXQ_ERR_* codes below and
 *     launches nothing when it fails validation.  mlxq_last_error() gives a
 *     human-readable message for the last failure on the calling thread.
 *   - Accumulation is fp32 on the GPU; each output element is rounded once to
 *     BF16 (round to nearest even).
 *   - Outputs may not overlap inputs, except y == x_resid exactly (each
 *     output element reads its own residual before its single write).  Other
 *     overlaps that the library can see are rejected with MLXQ_ERR_INVALID_ARG.
 *   - Device memory: mlxq_load allocates the weight's three buffers.  When
 *     mlxq_gemm splits K over CTAs it takes fp32 partials from a stream-ordered
 *     pool the library owns (allocated and freed in order on `stream`); the
 *     pool keeps its memory between calls.  No other call allocates device
 *     memory; mlxq_gemm_noalloc is mlxq_gemm without any allocation.
 */
#ifndef MLXQ_H
#define MLXQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MLXQ_API __attribute__((visibility("default")))
#else
#define MLXQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum {
    MLXQ_OK = 0,
    MLXQ_ERR_INVALID_ARG = 1,    /* null/released handle, null or misaligned pointer, overlap */
    MLXQ_ERR_PARSE = 2,          /* malformed safetensors blob */
    MLXQ_ERR_MISSING_TENSOR = 3, /* {base}.weight / .scales / .biases absent */
    MLXQ_ERR_DTYPE = 4,          /* weight not U32, or scales/biases not BF16 */
    MLXQ_ERR_SHAPE = 5,          /* weight not 2-D, or scales/biases not [N, K/gs] */
    MLXQ_ERR_GROUP_SIZE = 6,     /* group_size == 0 or group_size does not divide in_features */
    MLXQ_ERR_UNSUPPORTED = 7,    /* valid request outside what the kernels handle */
    MLXQ_ERR_CUDA = 8,           /* CUDA allocation, copy or launch error */
    MLXQ_ERR_DEVICE_TIMEOUT = 9  /* a kernel gave up a bounded wait (see mlxq_device_status) */
};

/*
 * One quantized linear weight resident on the GPU (page: struct
 * MlxInt8Weight).  N = out_features, K = in_features, gs = group_size.
 * A handle filled by mlxq_load owns its three buffers and must be freed once
 * with mlxq_release.  A caller may instead fill the struct with device
 * buffers it owns (same layouts); such a handle must not be passed to
 * mlxq_release.  `flags` is 0 or a combination of MLXQ_WEIGHT_* below;
 * mlxq_load sets it to 0 and a caller may change it afterwards.
 */
typedef struct mlxq_weight {
    void* packed;          /* uint32 [N, K/4] */
    void* scales;          /* bf16  [N, K/gs] */
    void* biases;          /* bf16  [N, K/gs] */
    uint32_t out_features; /* N */
    uint32_t in_features;  /* K (a multiple of 4) */
    uint32_t group_size;   /* gs, divides K */
    uint32_t flags;        /* MLXQ_WEIGHT_* */
} mlxq_weight;

/*
 * MLXQ_WEIGHT_STATIC: the caller guarantees that while a call that reads this
 * weight is queued or running, no kernel on any stream writes its packed,
 * scales or biases buffers (true of weights loaded once and then only read,
 * as in decoding).  The m = 1 kernels and dequantize_to may then read the
 * weight before the previous work on the stream has finished; activations,
 * residuals and outputs are still touched only after it.  Off (0) by default:
 * every read of the weight then comes after the previous work on the stream.
 */
#define MLXQ_WEIGHT_STATIC 1u

/*
 * mlxq_load (page: MlxInt8Weight::load).  Parses an in-memory safetensors
 * blob (host memory, `blob_len` bytes: u64 little-endian header length, JSON
 * header, data), finds "{base}.weight" (U32, 2-D [N, K/4]), "{base}.scales"
 * and "{base}.biases" (BF16, [N, K/gs]), allocates three device buffers with
 * cudaMalloc on the current device and copies the tensors in (synchronous).
 * On success *out owns the buffers.  Fails, allocating nothing, with
 * MLXQ_ERR_PARSE, _MISSING_TENSOR, _DTYPE, _SHAPE or _GROUP_SIZE exactly as
 * the page lists; MLXQ_ERR_CUDA if allocation or the copy fails (partial
 * allocations are freed).  *out is zeroed on failure.
 */
MLXQ_API int mlxq_load(const void* blob, size_t blob_len, const char* base, uint32_t group_size,
              mlxq_weight* out);

/*
 * mlxq_dequant (page: MlxInt8Weight::dequantize_to, kernel mlx_int8_dequant).
 * Writes the full dequantised weight as BF16 to `out`, row-major [N, K]:
 * out must hold at least N*K*2 bytes (device).  Bytes past N*K*2 are not
 * touched.  Bit-exact: each element is bf16_rne(fma_f32(s, q, b)).
 */
MLXQ_API int mlxq_dequant(const mlxq_weight* w, void* out, uint64_t stream);

/*
 * mlxq_gemv (page: MlxInt8Weight::gemv, kernel mlx_int8_gemv).
 * y = W x.  x: BF16 [K] (device); y: BF16, at least N elements (device).
 */
MLXQ_API int mlxq_gemv(const mlxq_weight* w, const void* x, void* y, uint64_t stream);

/*
 * mlxq_gemv_silu_gate (page: MlxInt8Weight::gemv_silu_gate, kernel
 * mlx_int8_gemv_silu_gate).  y = W (silu(gate) * up), silu(t) = t/(1+e^-t),
 * in one launch; the product silu(gate)*up exists only on chip (registers and
 * shared memory), it is not stored to global memory.  gate, up: BF16 [K];
 * y: BF16 [N].
 */
MLXQ_API int mlxq_gemv_silu_gate(const mlxq_weight* w, const void* gate, const void* up, void* y,
                        uint64_t stream);

/*
 * mlxq_gemv_silu_gate_resid (page: MlxInt8Weight::gemv_silu_gate_resid).
 * y[n] = x_resid[n] + sum_k W[n,k] * (silu(gate[k]) * up[k]), one launch.
 * gate, up: BF16 [K]; x_resid, y: BF16 [N].  y may equal x_resid exactly.
 */
MLXQ_API int mlxq_gemv_silu_gate_resid(const mlxq_weight* w, const void* gate, const void* up,
                              const void* x_resid, void* y, uint64_t stream);

/*
 * mlxq_gemm (page: MlxInt8Weight::gemm, kernel mlx_int8_gemm).
 * Y = X W^T.  X: BF16 [m, K] row-major; Y: BF16 [m, N] row-major.  m == 0 is
 * a no-op.  The kernel is chosen from m: weight-streaming kernels for small m
 * (every weight byte read once, dequantised in registers) or the tcgen05
 * tensor-core kernel for larger m (weight tiles dequantised to BF16 in shared
 * memory, fp32 accumulators in TMEM).  When m leaves SMs idle, the
 * tensor-core kernel splits K over CTAs; their fp32 partials live in a
 * stream-ordered memory pool owned by the library, allocated and freed in
 * order on `stream`.  Callers that must not allocate use mlxq_gemm_noalloc.
 */
MLXQ_API int mlxq_gemm(const mlxq_weight* w, const void* x, void* y, uint32_t m, uint64_t stream);

/* Size of the scratch buffer compiled into the library for mlxq_gemm_noalloc:
 * enough for every K split on a GPU with up to 148 SMs (at most one CTA per SM
 * per split tile, 256 x 256 fp32 partials each) plus the tile counters. */
#define MLXQ_STATIC_SCRATCH_BYTES (40u << 20)

/*
 * mlxq_gemm_noalloc (page: MlxInt8Weight::gemm, kernel mlx_int8_gemm).
 * mlxq_gemm that allocates no device memory, for callers that cannot call
 * cudaMalloc or a pool allocator: code running where allocation is not
 * allowed or not wanted (a fixed memory budget set up front, a runtime that
 * owns all device memory itself, or a hot loop that must not reach the
 * allocator).  Same arguments, layout, kernel choice and results (bit for
 * bit) as mlxq_gemm.  Where mlxq_gemm takes the K-split partials from its
 * memory pool, this call uses the library's static scratch buffer: a
 * file-scope device array of MLXQ_STATIC_SCRATCH_BYTES that every GPU which
 * loads the library holds until the process exits.
 *   - A call whose split would need more than that returns
 *     MLXQ_ERR_UNSUPPORTED and launches nothing.
 *   - The first call on a device that splits K looks up the array's device
 *     address (cudaGetSymbolAddress) with that device current; make that
 *     first call before any stream capture on the device.
 *   - The buffer is one per device and shared by every call, and it keeps
 *     the last call's contents (each split leaves its tile counters at zero
 *     for the next).  Calls that overlap on the GPU race on it: issue calls
 *     that split K on one stream, or order them with events.
 */
MLXQ_API int mlxq_gemm_noalloc(const mlxq_weight* w, const void* x, void* y, uint32_t m, uint64_t stream);

/* Kernel selection for mlxq_gemm_with (tests and benchmarks pin a path). */
enum {
    MLXQ_GEMM_AUTO = 0,        /* what mlxq_gemm picks */
    MLXQ_GEMM_ROWS = 1,        /* m independent passes of the gemv kernel */
    MLXQ_GEMM_SMALLM = 2,      /* weight-streaming kernel, products on the tensor pipe
                                  (mma.sync fragments), m <= 32: each CTA streams its
                                  rows in pairs of 8-row octets */
    MLXQ_GEMM_TCGEN05 = 3,     /* tcgen05 tensor-core kernel (TMEM accumulators) */
    MLXQ_GEMM_SMALLM_FFMA = 4, /* weight-streaming kernel on the fp32 pipes: m <= 32
                                  when group_size % 16 == 0; any m, in passes of up to
                                  8 rows, for other group sizes with group_size % 4 == 0
                                  and in_features % 16 == 0 */
    MLXQ_GEMM_SMALLM_GROUPS = 5, /* weight-streaming kernel on the tensor pipe, m <= 32:
                                  each SM walks a balanced range of 16-row tiles in
                                  groups; in_features % 128 == 0, group_size 16/32/64 */
    MLXQ_GEMM_SMALLM_TC = 6    /* weight-streaming kernel on tcgen05, m <= 64: the
                                  dequantised weight is the M = 128 operand, the
                                  activations the N operand; in_features % 128 == 0,
                                  group_size 16/32/64/128, (in/group_size) % 8 == 0 */
};

/* mlxq_gemm with an explicit kernel; MLXQ_ERR_UNSUPPORTED if that kernel
 * cannot take this shape. */
MLXQ_API int mlxq_gemm_with(const mlxq_weight* w, const void* x, void* y, uint32_t m, int kernel,
                   uint64_t stream);

/* Output formats of mlxq_dequant_as. */
enum { MLXQ_DTYPE_BF16 = 0, MLXQ_DTYPE_F16 = 1, MLXQ_DTYPE_F32 = 2 };

/*
 * mlxq_dequant_as (dequantize_to in another format; the dequantize-to-f16
 * and -f32 variants of the quantized-storage page).  Writes the full
 * weight, row-major [N, K], to out (N * K elements of the format, aligned to
 * its size):
 *   MLXQ_DTYPE_BF16  exactly mlxq_dequant;
 *   MLXQ_DTYPE_F32   fma_f32(s, q, b) itself (no further rounding);
 *   MLXQ_DTYPE_F16   fma_f32(s, q, b) rounded to FP16, nearest even.
 * MLXQ_ERR_INVALID_ARG for an unknown dtype or a null/misaligned/overlapping
 * out.
 */
MLXQ_API int mlxq_dequant_as(const mlxq_weight* w, void* out, int dtype, uint64_t stream);

/*
 * mlxq_quantize (no page entry: the inverse of the format; the pages give no
 * quantizer algorithm, so the plain per-group min/max affine one is used).
 * w_bf16: BF16 [out_features, in_features] row-major, device.  dst: a handle
 * whose packed/scales/biases point at caller-owned device buffers of the
 * format's sizes and whose dimensions and group_size (a multiple of 4, dividing
 * in_features) describe w.  Per row and group, in fp32, each operation
 * rounded to nearest even:
 *   s = bf16((max - min) / 255), b = bf16(min),
 *   q = clamp(rint((w - b) / s), 0, 255)  (all q = 0 when s == 0),
 * codes little-endian in the words.  The result is a weight every other call
 * takes.  Source and destination must not overlap (MLXQ_ERR_INVALID_ARG).
 */
MLXQ_API int mlxq_quantize(const void* w_bf16, const mlxq_weight* dst, uint64_t stream);

/*
 * Self-tests of the failure paths (no page entry; used by the tests).
 *
 * mlxq_selftest_wait_timeout: launches one warp on `stream` that waits,
 * through the same bounded mbarrier wait every kernel uses, on a barrier that
 * nothing completes.  After limit_us microseconds (1 .. 1,000,000) the wait
 * gives up, sets the device status word and the kernel returns: nothing
 * faults, traps or hangs, and the context stays usable.  The next
 * mlxq_device_status then returns MLXQ_ERR_DEVICE_TIMEOUT (and clears it).
 *
 * mlxq_selftest_fail_alloc: makes the nth device allocation made by mlxq_load
 * from now on fail as if cudaMalloc had run out of memory (nth = 1: the next
 * one; 0 cancels).  mlxq_load then returns MLXQ_ERR_CUDA, frees what it had
 * allocated and leaves the handle untouched.
 */
MLXQ_API int mlxq_selftest_wait_timeout(uint32_t limit_us, uint64_t stream);
MLXQ_API int mlxq_selftest_fail_alloc(uint32_t nth);

/*
 * mlxq_release (page: MlxInt8Weight::release).  Frees the three buffers of a
 * handle filled by mlxq_load and zeroes the handle.  The buffers are freed
 * exactly once: a second call on the same handle returns MLXQ_ERR_INVALID_ARG.
 */
MLXQ_API int mlxq_release(mlxq_weight* w);

/* Message for the last nonzero status returned on this thread ("" if none). */
MLXQ_API const char* mlxq_last_error(void);

/*
 * Waits for the current device to go idle, then reads and clears the
 * library's device status word.  Returns MLXQ_OK, or MLXQ_ERR_DEVICE_TIMEOUT
 * if some kernel since the last check gave up a bounded wait (its outputs are
 * then not valid), or MLXQ_ERR_CUDA.  Kernels never hang or trap on a stalled
 * pipeline: they record the timeout here and return.  On a timeout it also
 * zeroes the tile counters of mlxq_gemm_noalloc's static scratch, which an
 * interrupted K split may have left raised.
 */
MLXQ_API int mlxq_device_status(void);

#ifdef __cplusplus
}
#endif

#endif /* MLXQ_H */
