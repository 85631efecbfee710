// common.cuh -- host-side helpers shared by the C-ABI entry points:
// argument checks, the per-device error word, TMA descriptor encoding.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <atomic>
#include <cstddef>
#include <cstdint>
#include <initializer_list>

#include "svdq.h"   // include/ is on the include path (see build.py)

namespace svdq {

// Row ranges handed to kernels by value (host segments are copied in).
constexpr int kMaxSegments = 64;

struct SegTable {
    int n;
    int64_t begin[kMaxSegments];
    int64_t prefix[kMaxSegments + 1];   // prefix[s] = rows in segments before s
};

// Validate host segments against [0, M) and fill a SegTable.  NULL/0 selects all rows.
inline int make_seg_table(const svdq_seg* segs, int n_seg, int64_t M, SegTable* t) {
    if (n_seg < 0 || n_seg > kMaxSegments) return SVDQ_ERR_INVALID_ARG;
    if (n_seg > 0 && segs == nullptr) return SVDQ_ERR_INVALID_ARG;
    if (segs == nullptr) {
        t->n = 1;
        t->begin[0] = 0;
        t->prefix[0] = 0;
        t->prefix[1] = M;
        return SVDQ_OK;
    }
    t->n = n_seg;
    t->prefix[0] = 0;
    for (int s = 0; s < n_seg; ++s) {
        if (segs[s].begin < 0 || segs[s].end < segs[s].begin || segs[s].end > M) return SVDQ_ERR_INVALID_ARG;
        t->begin[s] = segs[s].begin;
        t->prefix[s + 1] = t->prefix[s] + (segs[s].end - segs[s].begin);
    }
    return SVDQ_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Current device's error word (a __device__ variable of this library).
uint32_t* device_error_word();

// Current device is sm_100 (B200 class)?  Cached per device.
bool device_is_sm100();

// Number of SMs of the current device (cached).
int device_sm_count();

// Encode a 2-D tiled tensor map (dims/strides in elements of `dtype`).
bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, uint32_t elem_bytes,
                    const void* base, uint64_t inner, uint64_t outer, uint64_t row_stride_bytes,
                    uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle);

// Unswizzled 3-D map of bytes: dims {d0, d1, d2} (d0 innermost, contiguous),
// byte strides s1 (dimension 1) and s2 (dimension 2), box {b0, b1, b2}.
bool encode_tmap_3d_u8(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
                       uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2);

// Current device ordinal, or -1.
int current_device_index();

// Debug library only (SVDQ_DEBUG_CHECKS=1), identity otherwise: the extent a
// kernel checks its stores of output `site` against -- `extent`, or the
// smaller value a test armed with svdq_debug_limit_extent (consumed here).
int64_t debug_extent(uint32_t site, int64_t extent);

// Debug library only, true otherwise: every non-null pointer is device (or
// managed) memory of the current device.  Entry points return
// SVDQ_ERR_INVALID_ARG when it fails.
bool debug_ptrs_ok(std::initializer_list<const void*> ptrs);

// Raise a kernel's dynamic shared memory limit to `bytes`, once per device
// (`done` is a per-kernel bit set over device ordinals 0..63).
template <typename Kernel>
inline bool set_dynamic_smem_once(Kernel kern, uint32_t bytes, std::atomic<uint64_t>& done) {
    const int dev = current_device_index();
    if (dev < 0) return false;
    const uint64_t bit = uint64_t(1) << (dev & 63);
    if (done.load(std::memory_order_acquire) & bit) return true;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)) !=
        cudaSuccess)
        return false;
    done.fetch_or(bit, std::memory_order_release);
    return true;
}

// Largest grid of `kern` (blockDim `threads`, `smem` dynamic bytes) whose CTAs
// can all be resident at once on the current device: what a cooperative launch
// may use.  0 if the occupancy query fails.
template <typename Kernel>
inline int64_t coresident_grid(Kernel kern, int threads, size_t smem) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem) != cudaSuccess) return 0;
    return static_cast<int64_t>(per_sm) * device_sm_count();
}

inline int launch_status(cudaError_t e) {
    if (e == cudaSuccess) return SVDQ_OK;
    return SVDQ_ERR_CUDA;
}

}  // namespace svdq
