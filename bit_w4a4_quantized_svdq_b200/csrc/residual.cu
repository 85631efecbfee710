// residual.cu -- offline weight conversion: the residual the 4-bit weight
// encodes once the low-rank branch has taken the top singular directions
// ("MiniMax-H3 . SVDQuant W4A4 (int4, rank 32, GPTQ)", opening section:
// outliers absorbed into a 16-bit low-rank branch, the residual quantised).
//
//   R[n, k] = W[n, k] * lambda[k] - lambda[k] * sum_j down[j, k] * up[n, j]
//
// in fp64 with the j sum in index order, then fp64 -> fp32 -> bf16, each step
// round-to-nearest.  Products of bf16 values are exact in fp64, so the sum is
// the same whether or not the compiler fuses multiply and add; the two
// rounding steps that matter use explicit _rn intrinsics.
#include "common.cuh"
#include "sm100.cuh"

namespace svdq {
namespace {

constexpr int kMaxRank = 32;
constexpr int kTileK = 256;     // one thread per k, one block row of up values in shared memory

__global__ void __launch_bounds__(kTileK)
residual_kernel(const uint16_t* __restrict__ W, int64_t N, int64_t K, int64_t ldw,
                const float* __restrict__ lambda, const uint16_t* __restrict__ down,
                const uint16_t* __restrict__ up, int r, uint16_t* __restrict__ R, int rows_per_block,
                int64_t ext, uint32_t* err) {
    __shared__ double up_s[kMaxRank];
    const int64_t k = static_cast<int64_t>(blockIdx.x) * kTileK + threadIdx.x;
    const int64_t n0 = static_cast<int64_t>(blockIdx.y) * rows_per_block;
    const int64_t n1 = min(n0 + rows_per_block, N);
    double dk[kMaxRank];
    double lam = 1.0;
    if (k < K) {
        if (lambda) lam = static_cast<double>(lambda[k]);
#pragma unroll
        for (int j = 0; j < kMaxRank; ++j)
            dk[j] = j < r ? static_cast<double>(__uint_as_float(static_cast<uint32_t>(down[j * K + k]) << 16)) : 0.0;
    }
    for (int64_t n = n0; n < n1; ++n) {
        __syncthreads();
        if (threadIdx.x < r)
            up_s[threadIdx.x] = static_cast<double>(__uint_as_float(static_cast<uint32_t>(up[n * r + threadIdx.x]) << 16));
        __syncthreads();
        if (k < K) {
            double acc = 0.0;
#pragma unroll
            for (int j = 0; j < kMaxRank; ++j)
                if (j < r) acc = __dadd_rn(acc, __dmul_rn(dk[j], up_s[j]));
            const double w = static_cast<double>(__uint_as_float(static_cast<uint32_t>(W[n * ldw + k]) << 16));
            const double v = __dsub_rn(__dmul_rn(w, lam), __dmul_rn(lam, acc));
            const float f = __double2float_rn(v);
            if (store_ok(n * K + k, 1, ext, err, kSiteResidual))
                R[n * K + k] = __bfloat16_as_ushort(__float2bfloat16_rn(f));
        }
    }
}

}  // namespace
}  // namespace svdq

extern "C" int svdq_residual(const void* W, int64_t N, int64_t K, int64_t ldw, const float* lambda,
                             const void* down, const void* up, int r, void* R, void* stream) {
    using namespace svdq;
    if (W == nullptr || R == nullptr || N < 1 || K < 1 || ldw < K) return SVDQ_ERR_INVALID_ARG;
    if (r < 0 || r > kMaxRank) return SVDQ_ERR_UNSUPPORTED;
    if (r > 0 && (down == nullptr || up == nullptr)) return SVDQ_ERR_INVALID_ARG;
    if (!device_is_sm100()) return SVDQ_ERR_NO_DEVICE;
    if (!debug_ptrs_ok({W, lambda, down, up, R})) return SVDQ_ERR_INVALID_ARG;
    uint32_t* err = device_error_word();
    if (err == nullptr) return SVDQ_ERR_CUDA;
    const int rows_per_block = 16;
    const int64_t gy = (N + rows_per_block - 1) / rows_per_block;
    if (gy > 65535) return SVDQ_ERR_UNSUPPORTED;
    dim3 grid(static_cast<unsigned>((K + kTileK - 1) / kTileK), static_cast<unsigned>(gy));
    residual_kernel<<<grid, kTileK, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint16_t*>(W), N, K, ldw, lambda, static_cast<const uint16_t*>(down),
        static_cast<const uint16_t*>(up), r, static_cast<uint16_t*>(R), rows_per_block,
        debug_extent(kSiteResidual, N * K), err);
    return launch_status(cudaGetLastError());
}
