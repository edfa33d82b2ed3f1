#include "tensor_map.h"

#include <cudaTypedefs.h>

#include <cstring>
#include <map>
#include <mutex>
#include <tuple>

namespace mlxq {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode;
}

using Key = std::tuple<const void*, const void*, const void*, int64_t, int64_t, int64_t, int, int, int, int, int>;
std::mutex g_mu;
std::map<Key, TensorMaps3> g_cache;
constexpr size_t kMaxEntries = 4096;

}  // namespace

bool tensor_maps_available() { return encoder() != nullptr; }

bool encode_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
               uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
    auto enc = encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_3d_chunks(CUtensorMap* map, CUtensorMapDataType dt, uint32_t elem_bytes, const void* base, uint64_t inner,
                      uint64_t outer, uint64_t row_bytes, uint32_t chunk, uint32_t box_outer, uint32_t box_chunks) {
    auto enc = encoder();
    if (!enc || chunk == 0 || inner % chunk != 0) return false;
    const cuuint64_t dims[3] = {chunk, outer, inner / chunk};
    const cuuint64_t strides[2] = {row_bytes, static_cast<cuuint64_t>(chunk) * elem_bytes};
    const cuuint32_t box[3] = {chunk, box_outer, box_chunks};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool weight_tensor_maps(const WeightView& w, int box_rows, int box_k_bytes, CUtensorMapSwizzle packed_sw,
                        int box_groups, TensorMaps3* out) {
    int dev = 0;
    cudaGetDevice(&dev);
    const Key key{w.packed, w.scales, w.biases, w.N, w.K, w.gs, box_rows, box_k_bytes,
                  static_cast<int>(packed_sw), box_groups, dev};
    {
        std::lock_guard<std::mutex> lk(g_mu);
        auto it = g_cache.find(key);
        if (it != g_cache.end()) {
            *out = it->second;
            return true;
        }
    }
    TensorMaps3 t;
    std::memset(&t, 0, sizeof(t));
    if (!encode_2d(&t.packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.packed, static_cast<uint64_t>(w.K),
                   static_cast<uint64_t>(w.N), static_cast<uint64_t>(w.K), static_cast<uint32_t>(box_k_bytes),
                   static_cast<uint32_t>(box_rows), packed_sw))
        return false;
    if (box_groups > 0) {
        const uint64_t G = static_cast<uint64_t>(w.G);
        if (!encode_2d(&t.scales, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w.scales, G, static_cast<uint64_t>(w.N), G * 2,
                       static_cast<uint32_t>(box_groups), static_cast<uint32_t>(box_rows), CU_TENSOR_MAP_SWIZZLE_NONE))
            return false;
        if (!encode_2d(&t.biases, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w.biases, G, static_cast<uint64_t>(w.N), G * 2,
                       static_cast<uint32_t>(box_groups), static_cast<uint32_t>(box_rows), CU_TENSOR_MAP_SWIZZLE_NONE))
            return false;
    }
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_cache.size() >= kMaxEntries) g_cache.clear();
    g_cache[key] = t;
    *out = t;
    return true;
}

}  // namespace mlxq
