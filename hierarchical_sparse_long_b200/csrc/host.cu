// Host-side helpers shared by the launchers: TMA tensor maps over rows of
// bf16 values (cached per thread, since encoding one is a driver call on
// every launch otherwise) and the per-device dynamic shared-memory attribute
// of a kernel (set once per kernel and device).
#include <cudaTypedefs.h>
#include <mutex>
#include <utility>
#include <vector>

#include "common.cuh"

namespace hga {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

struct MapEntry {
    const void *base;
    unsigned long long rows;
    unsigned box_rows;
    CUtensorMap map;
};
constexpr int kMapCache = 16;
thread_local MapEntry t_maps[kMapCache];
thread_local int t_map_next = 0;

struct GroupMapEntry {
    const void *base;
    int D;
    unsigned long long rows, groups, stride;
    CUtensorMap map;
};
thread_local GroupMapEntry t_gmaps[kMapCache];
thread_local int t_gmap_next = 0;

std::mutex g_attr_mu;
std::vector<std::pair<std::pair<const void *, int>, int>> g_attr;  // (kernel, device) -> bytes set

}  // namespace

bool tma_encoder_available() {
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode != nullptr;
}

bool tma_rows_map(CUtensorMap *map, const void *base, unsigned long long rows, unsigned box_rows) {
    for (const MapEntry &e : t_maps)
        if (e.base == base && e.rows == rows && e.box_rows == box_rows && base != nullptr) {
            *map = e.map;
            return true;
        }
    if (!tma_encoder_available()) return false;
    const cuuint64_t dims[2] = {128, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {128 * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    if (g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    MapEntry &slot = t_maps[t_map_next];
    t_map_next = (t_map_next + 1) % kMapCache;
    slot.base = base;
    slot.rows = rows;
    slot.box_rows = box_rows;
    slot.map = *map;
    return true;
}

bool tma_group_rows_map(CUtensorMap *map, const void *base, int D, unsigned long long rows,
                        unsigned long long groups, unsigned long long group_stride_rows) {
    for (const GroupMapEntry &e : t_gmaps)
        if (e.base == base && e.D == D && e.rows == rows && e.groups == groups && e.stride == group_stride_rows &&
            base != nullptr) {
            *map = e.map;
            return true;
        }
    if (!tma_encoder_available() || rows == 0 || groups == 0 || (D != 64 && D != 128)) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)groups};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)(group_stride_rows * D * 2)};
    const cuuint32_t box[3] = {64, 64, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    GroupMapEntry &slot = t_gmaps[t_gmap_next];
    t_gmap_next = (t_gmap_next + 1) % kMapCache;
    slot.base = base;
    slot.D = D;
    slot.rows = rows;
    slot.groups = groups;
    slot.stride = group_stride_rows;
    slot.map = *map;
    return true;
}

cudaError_t set_max_dynamic_smem(const void *kernel, int bytes) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_attr_mu);
    for (auto &kv : g_attr)
        if (kv.first.first == kernel && kv.first.second == dev) {
            if (kv.second >= bytes) return cudaSuccess;
            e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
            if (e == cudaSuccess) kv.second = bytes;
            return e;
        }
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) g_attr.push_back({{kernel, dev}, bytes});
    return e;
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) {
        cudaGetLastError();
        return 148;
    }
    return n;
}

}  // namespace hga
