// Host-side launch interface between the C ABI (abi.cu) and the kernels.
// Every launcher validates nothing: abi.cu has already checked pointers,
// shapes and alignment.  Each returns the launch status (cudaGetLastError).
#pragma once

#include "mlxq.h"

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <utility>

namespace mlxq {

struct WeightView {
    const uint32_t* packed;  // [N, K/4]
    const uint16_t* scales;  // [N, G] bf16 bits
    const uint16_t* biases;  // [N, G] bf16 bits
    int64_t N, K, gs, G;
    uint32_t flags;          // MLXQ_WEIGHT_*
};

enum GemvMode { GEMV_PLAIN = 0, GEMV_SILU = 1, GEMV_SILU_RESID = 2 };

// Device properties of the current device (cached per device).
struct DeviceInfo {
    int device;
    int sm_count;
    int max_smem_optin;
    int smem_per_sm;  // shared memory of one SM (bytes), for co-resident CTAs
};
const DeviceInfo& device_info();

// Address of the library's device status word on the current device.
unsigned int* device_status_ptr();

// Raise a kernel's dynamic shared-memory limit to `bytes` once per device
// (cudaFuncSetAttribute is a host round trip; launches then skip it).
// `configured` is the calling launch site's own per-device record (one static
// array per kernel instance: kernels of one signature share a function type).
template <typename Kernel>
cudaError_t ensure_dynamic_smem(Kernel kern, size_t bytes, std::atomic<int> (&configured)[64]) {
    const int dev = device_info().device;
    const int want = static_cast<int>(bytes);
    if (configured[dev].load(std::memory_order_relaxed) >= want) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, want);
    if (e == cudaSuccess) {
        int cur = configured[dev].load(std::memory_order_relaxed);
        while (cur < want && !configured[dev].compare_exchange_weak(cur, want)) {
        }
    }
    return e;
}

// Launch with programmatic stream serialization (PDL): the kernel may start
// while the previous one in the stream finishes; kernels launched this way
// call griddepcontrol.wait before touching any input or output in memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// mlx_int8_dequant: out [N, K] bf16.
cudaError_t launch_dequant(const WeightView& w, void* out, cudaStream_t stream);
// dtype: 0 BF16 (launch_dequant), 1 FP16, 2 FP32.
cudaError_t launch_dequant_as(const WeightView& w, void* out, int dtype, cudaStream_t stream);

// mlx_int8_gemv family (m = 1): y = W h (+ resid), h = x or silu(gate)*up.
cudaError_t launch_gemv(const WeightView& w, int mode, const void* x, const void* gate,
                        const void* up, const void* resid, void* y, cudaStream_t stream);

// m = 1 stream kernel (gemv and its silu variants) with fixed per-warp work
// items; N up to 128 rows per SM.
bool gemv_la_supported(const WeightView& w, int mode, const void* x, const void* gate, const void* up);
cudaError_t launch_gemv_la(const WeightView& w, int mode, const void* x, const void* gate, const void* up,
                           const void* resid, void* y, cudaStream_t stream);

// Tensor-pipe stream kernel (mma.sync fragments) for m <= kStreamMmaMaxM:
// gemv and its silu variants (m == 1) and small-m gemm (plain mode).
constexpr int kStreamMmaMaxM = 32;
bool stream_mma_supported(const WeightView& w, int mode, int64_t m, const void* x, const void* gate,
                          const void* up);
cudaError_t launch_stream_mma(const WeightView& w, int mode, int64_t m, const void* x, const void* gate,
                              const void* up, const void* resid, void* y, cudaStream_t stream);

// Small-m gemm, 1 <= m <= 32, weight tiles walked in groups by one CTA per
// SM (tensor-pipe fragments, activations copied with each stage).
bool smallm_supported(const WeightView& w, int64_t m, const void* X);
// Small m on tcgen05 (swap-AB: weights as the M = 128 operand), 1 <= m <= 64.
bool smallm_tc_supported(const WeightView& w, int64_t m, const void* X);
bool smallm_tc_preferred(const WeightView& w, int64_t m, const void* X);
cudaError_t launch_smallm_tc(const WeightView& w, const void* X, void* Y, int64_t m, cudaStream_t stream);
// supported, and measured faster than the per-row-pair streaming kernel:
// 8 < m and at least 6 tiles of 16 rows per SM
bool smallm_preferred(const WeightView& w, int64_t m, const void* X);
cudaError_t launch_smallm(const WeightView& w, const void* X, void* Y, int64_t m, cudaStream_t stream);

// Any group size with 4-code words (gs % 4 == 0, K % 16 == 0, 16-byte
// aligned codes; tables and activations need only 2-byte alignment).
bool anygs_gemv_supported(const WeightView& w, int mode);
cudaError_t launch_anygs_gemv(const WeightView& w, int mode, const void* x, const void* gate, const void* up,
                              const void* resid, void* y, cudaStream_t stream);
bool anygs_gemm_supported(const WeightView& w, int64_t m);
cudaError_t launch_anygs_gemm(const WeightView& w, const void* X, void* Y, int64_t m, cudaStream_t stream);
bool anygs_dequant_supported(const WeightView& w, const void* out);  // out 16-byte aligned
cudaError_t launch_anygs_dequant(const WeightView& w, void* out, cudaStream_t stream);

// CUDA-core small-m gemm: Y [m, N] = X [m, K] W^T, 2 <= m <= kSmallMMax.
constexpr int kSmallMMax = 32;
bool gemm_smallm_supported(const WeightView& w, int64_t m);
cudaError_t launch_gemm_smallm(const WeightView& w, const void* X, void* Y, int64_t m,
                               cudaStream_t stream);

// tcgen05 tensor-core gemm.
bool gemm_tc_supported(const WeightView& w, int64_t m, const void* X, const void* Y);
// BF16 W [N, K] (row-major) -> codes, scales and biases of `dst`.
cudaError_t launch_quantize(const void* w, const WeightView& dst, cudaStream_t stream);

// Self-test: one bounded wait that runs out after limit_ns (status word set).
cudaError_t launch_wait_timeout_selftest(unsigned long long limit_ns, cudaStream_t stream);

// Where the K-split partials of the tcgen05 gemm live: the library's
// stream-ordered pool, or the static buffer of mlxq_gemm_noalloc.
enum TcScratch { TC_SCRATCH_POOL = 0, TC_SCRATCH_STATIC = 1 };
constexpr size_t kStaticScratchBytes = MLXQ_STATIC_SCRATCH_BYTES;
// Zero the tile counters of the static scratch (after a timed-out wait).
cudaError_t reset_static_scratch_counters();
// Scratch bytes a tcgen05 gemm of this shape needs (0: no K split).
size_t gemm_tc_scratch_bytes(const WeightView& w, int64_t m);
cudaError_t launch_gemm_tc(const WeightView& w, const void* X, void* Y, int64_t m, cudaStream_t stream,
                           TcScratch scratch = TC_SCRATCH_POOL);

}  // namespace mlxq
