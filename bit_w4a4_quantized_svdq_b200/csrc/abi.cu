// abi.cu -- library-wide C-ABI entries (status strings, sizes, the device
// error word) and the host helpers the kernel entry points share.
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "sm100.cuh"

namespace svdq {

// One error word per device (each device's copy of this module holds its own).
__device__ uint32_t g_device_error;

namespace {
constexpr int kMaxDevices = 64;
uint32_t* g_err_ptr[kMaxDevices] = {};
int g_is_sm100[kMaxDevices] = {};      // 0 unknown, 1 yes, 2 no (guarded by g_mutex)
std::atomic<int> g_sm_count[kMaxDevices] = {};
std::mutex g_mutex;

int current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
    return dev;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
}  // namespace

int current_device_index() { return current_device(); }

// Armed extent limits + 1 per store site (0: none armed).
std::atomic<int64_t> g_extent_limit[kSiteCount] = {};

int64_t debug_extent(uint32_t site, int64_t extent) {
#if SVDQ_DEBUG_CHECKS
    if (site < kSiteCount) {
        const int64_t lim = g_extent_limit[site].exchange(0, std::memory_order_acq_rel) - 1;
        if (lim >= 0 && lim < extent) return lim;
    }
#else
    (void)site;
#endif
    return extent;
}

bool debug_ptrs_ok(std::initializer_list<const void*> ptrs) {
#if SVDQ_DEBUG_CHECKS
    const int dev = current_device();
    if (dev < 0) return false;
    for (const void* p : ptrs) {
        if (p == nullptr) continue;
        cudaPointerAttributes at{};
        if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
            (void)cudaGetLastError();
            return false;
        }
        const bool on_device = at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged;
        if (!on_device || at.device != dev) return false;
    }
#else
    (void)ptrs;
#endif
    return true;
}

uint32_t* device_error_word() {
    const int dev = current_device();
    if (dev < 0) return nullptr;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_err_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
        g_err_ptr[dev] = static_cast<uint32_t*>(p);
    }
    return g_err_ptr[dev];
}

bool device_is_sm100() {
    const int dev = current_device();
    if (dev < 0) return false;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_is_sm100[dev] == 0) {
        int major = 0, minor = 0, sms = 0;
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        g_is_sm100[dev] = (major == 10 && minor == 0) ? 1 : 2;
        g_sm_count[dev].store(sms, std::memory_order_release);
    }
    return g_is_sm100[dev] == 1;
}

int device_sm_count() {
    const int dev = current_device();
    if (dev < 0) return 0;
    if (g_sm_count[dev].load(std::memory_order_acquire) == 0) device_is_sm100();
    return g_sm_count[dev].load(std::memory_order_acquire);
}

static bool load_encoder() {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_encode == nullptr) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr)
            return false;
        g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    return true;
}

bool encode_tmap_3d_u8(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
                       uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2) {
    if (!load_encoder()) return false;
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {s1, s2};
    const cuuint32_t box[3] = {b0, b1, b2};
    const cuuint32_t estr[3] = {1, 1, 1};
    std::memset(map, 0, sizeof(*map));
    const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box,
                                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, uint32_t elem_bytes,
                    const void* base, uint64_t inner, uint64_t outer, uint64_t row_stride_bytes,
                    uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
    if (!load_encoder()) return false;
    (void)elem_bytes;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_stride_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    std::memset(map, 0, sizeof(*map));
    const CUresult r = g_encode(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace svdq

extern "C" {

const char* svdq_status_string(int status) {
    switch (status) {
        case SVDQ_OK: return "ok";
        case SVDQ_ERR_INVALID_ARG: return "invalid argument";
        case SVDQ_ERR_UNSUPPORTED: return "unsupported shape";
        case SVDQ_ERR_MISALIGNED: return "misaligned pointer or stride";
        case SVDQ_ERR_CUDA: return "CUDA error";
        case SVDQ_ERR_TIMEOUT: return "device wait timed out";
        case SVDQ_ERR_NO_DEVICE: return "no sm_100 device";
        case SVDQ_ERR_SCRATCH_TOO_SMALL: return "problem exceeds the library's static scratch array";
        case SVDQ_ERR_BOUNDS: return "a device store fell outside its output (debug library)";
        default: return "unknown status";
    }
}

int svdq_version(void) { return 100; }

size_t svdq_sf_bytes(int64_t rows, int64_t K) {
    if (rows < 0 || K <= 0 || K % 64 != 0) return 0;
    const int64_t padded = (rows + 127) / 128 * 128;
    return static_cast<size_t>(padded) * static_cast<size_t>(K / 16);
}

int svdq_device_error(void* stream, uint32_t* code) {
    if (code == nullptr) return SVDQ_ERR_INVALID_ARG;
    *code = 0;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SVDQ_ERR_CUDA;
    uint32_t* word = svdq::device_error_word();
    if (word == nullptr) return SVDQ_ERR_CUDA;
    uint32_t v = 0;
    if (cudaMemcpy(&v, word, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return SVDQ_ERR_CUDA;
    if (v != 0) {
        const uint32_t zero = 0;
        if (cudaMemcpy(word, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return SVDQ_ERR_CUDA;
    }
    *code = v;
    if (v == 0) return SVDQ_OK;
    return v >= svdq::kErrBounds ? SVDQ_ERR_BOUNDS : SVDQ_ERR_TIMEOUT;
}

int svdq_debug_build(void) { return SVDQ_DEBUG_CHECKS ? 1 : 0; }

int svdq_debug_limit_extent(int site, int64_t extent) {
#if SVDQ_DEBUG_CHECKS
    if (site < 1 || site >= static_cast<int>(svdq::kSiteCount) || extent < 0) return SVDQ_ERR_INVALID_ARG;
    svdq::g_extent_limit[site].store(extent + 1, std::memory_order_release);
    return SVDQ_OK;
#else
    (void)site;
    (void)extent;
    return SVDQ_ERR_UNSUPPORTED;
#endif
}

}  // extern "C"
