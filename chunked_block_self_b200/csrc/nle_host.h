// nle_host.h -- host-side helpers shared by the launchers.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace nle {

struct DeviceInfo {
    int sm_count = 0;
    int smem_optin = 0;   // max dynamic shared memory per block (opt-in)
    int cc_major = 0;
    int cc_minor = 0;
};

// Properties of the current device (queried once per device, thread-safe).
// Returns false if the CUDA runtime call fails.
bool current_device_info(DeviceInfo *info, int *device);

// 2-D bf16 tensor map over a [rows][row_stride] matrix where only the first
// `cols` elements of each row are addressed; box = {box_cols, box_rows},
// 128-byte swizzle, zero fill outside the bounds.
bool encode_tmap_bf16_2d(CUtensorMap *map, const void *base, uint64_t cols, uint64_t rows,
                         uint64_t row_stride_elems, uint32_t box_cols, uint32_t box_rows);
// [rows][heads][64] bf16 as a 3-D tensor (d, row, head): boxes of
// (64, box_rows, box_heads) land head-major in shared memory; 128-byte
// swizzle, zero fill outside the tensor.
bool encode_tmap_bf16_heads(CUtensorMap *map, const void *base, uint64_t rows, uint64_t heads,
                            uint64_t row_stride_elems, uint32_t box_rows, uint32_t box_heads);

// Lets `fn` launch with any dynamic shared memory size up to the device's
// opt-in maximum (cudaFuncAttributeMaxDynamicSharedMemorySize set once per
// kernel and device, under a lock; the attribute only ever grows, so
// concurrent callers cannot undo each other).  Returns false if the CUDA
// call fails.
bool allow_max_dynamic_smem(const void *fn, int device, int smem_optin);

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

} // namespace nle
