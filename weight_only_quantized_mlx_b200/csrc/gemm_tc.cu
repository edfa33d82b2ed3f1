// tcgen05 tensor-core gemm for large m ("MlxInt8Weight" page, gemm).
#include "device_common.cuh"
#include "kernels.h"

namespace mlxq {

bool gemm_tc_supported(const WeightView&, int64_t, const void*, const void*) { return false; }

cudaError_t launch_gemm_tc(const WeightView&, const void*, void*, int64_t, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace mlxq
