// nle_api.cpp -- status strings, version, device-property cache and the
// tensor-map encoder (cuTensorMapEncodeTiled reached through the runtime's
// driver entry point, so libnle.so does not link libcuda directly).
#include <mutex>
#include <set>
#include <utility>

#include "nle.h"
#include "nle_host.h"

namespace nle {

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mutex;
DeviceInfo g_info[kMaxDevices];
bool g_have[kMaxDevices] = {};

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
bool g_encode_tried = false;

EncodeTiledFn encode_fn()
{
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_encode_tried) {
        g_encode_tried = true;
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    return g_encode;
}
} // namespace

bool current_device_info(DeviceInfo *info, int *device)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return false;
    *device = dev;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (g_have[dev]) {
            *info = g_info[dev];
            return true;
        }
    }
    DeviceInfo d;
    if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return false;
    std::lock_guard<std::mutex> lock(g_mutex);
    g_info[dev] = d;
    g_have[dev] = true;
    *info = d;
    return true;
}

bool allow_max_dynamic_smem(const void *fn, int device, int smem_optin)
{
    static std::mutex mu;
    static std::set<std::pair<const void *, int>> done;
    std::lock_guard<std::mutex> lock(mu);
    if (done.count({fn, device}))
        return true;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_optin) != cudaSuccess)
        return false;
    done.insert({fn, device});
    return true;
}

bool encode_tmap_bf16_2d(CUtensorMap *map, const void *base, uint64_t cols, uint64_t rows,
                         uint64_t row_stride_elems, uint32_t box_cols, uint32_t box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {row_stride_elems * 2};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [rows][heads][64] bf16 (row stride `row_stride_elems`) viewed as a 3-D
// tensor ordered (d, row, head), so that a box of (64, box_rows, box_heads)
// lands in shared memory head-major: box_rows rows of 128 B per head.
bool encode_tmap_bf16_heads(CUtensorMap *map, const void *base, uint64_t rows, uint64_t heads,
                            uint64_t row_stride_elems, uint32_t box_rows, uint32_t box_heads)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    const cuuint64_t dims[3] = {64, rows, heads};
    const cuuint64_t strides[2] = {row_stride_elems * 2, 128};
    const cuuint32_t box[3] = {64, box_rows, box_heads};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

} // namespace nle

extern "C" int nle_version(void) { return NLE_ABI_VERSION; }

extern "C" const char *nle_status_string(int status)
{
    switch (status) {
    case NLE_OK:
        return "NLE_OK";
    case NLE_ERR_INVALID_ARG:
        return "NLE_ERR_INVALID_ARG: invalid argument";
    case NLE_ERR_UNSUPPORTED:
        return "NLE_ERR_UNSUPPORTED: unsupported size or device";
    case NLE_ERR_MISALIGNED:
        return "NLE_ERR_MISALIGNED: pointer or stride not 16-byte aligned";
    case NLE_ERR_CUDA:
        return "NLE_ERR_CUDA: CUDA launch or query failed";
    case NLE_ERR_TIMEOUT:
        return "NLE_ERR_TIMEOUT: bounded in-kernel wait expired";
    default:
        return "unknown nle status";
    }
}
