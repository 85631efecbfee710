// grid.cu -- lambda candidates over a migration-strength grid.
//
// "MiniMax-H3 NVFP4 -- what the smoothing scale should be calibrated on",
// section "Calibration": the smoothing scale is chosen from a grid of
// candidates built from absmax statistics (39 candidates in the pages' runs).
// Each candidate is lambda_j(alpha) = ax_j^alpha / aw_j^(1 - alpha), the
// square-root rule of the calibration kernel being alpha = 0.5:
//
//   lambda_j = RN32(2^(alpha log2 ax_j - (1 - alpha) log2 aw_j))   (fp64 inside)
//   1 where ax_j or aw_j is 0;  inv_lambda_j = RN32(1 / lambda_j)
//   s_g      = RN32(max_j RN32(ax_j * inv_lambda_j) / 2688), 1 if that max is 0
//
// i.e. each candidate's lambda, 1/lambda and static activation tensor scale, in
// the form svdq_quantize_act and svdq_residual take them.  One CTA per
// candidate; the products and the difference in the exponent are written with
// explicit round-to-nearest operations so no contraction changes them.
#include "common.cuh"
#include "sm100.cuh"

namespace svdq {
namespace {

constexpr int kGridThreads = 256;

__global__ void __launch_bounds__(kGridThreads)
lambda_grid_kernel(const float* __restrict__ ax, const float* __restrict__ aw, const float* __restrict__ alpha,
                   int64_t K, float* __restrict__ lam, float* __restrict__ inv, float* __restrict__ s_g,
                   int64_t ext, int64_t ext_sg, uint32_t* err) {
    __shared__ float s_top[kGridThreads / 32];
    const int c = blockIdx.x;
    const double a = static_cast<double>(__ldg(alpha + c));
    const double b = 1.0 - a;                         // exact: alpha is an fp32 value
    float top = 0.0f;
    for (int64_t j = threadIdx.x; j < K; j += kGridThreads) {
        const float x = __ldg(ax + j);
        const float w = __ldg(aw + j);
        float l = 1.0f;
        if (x > 0.0f && w > 0.0f) {
            const double t = __dsub_rn(__dmul_rn(a, log2(static_cast<double>(x))),
                                       __dmul_rn(b, log2(static_cast<double>(w))));
            l = __double2float_rn(exp2(t));
        }
        const float il = __frcp_rn(l);
        if (store_ok(static_cast<int64_t>(c) * K + j, 1, ext, err, kSiteGrid)) {
            lam[static_cast<int64_t>(c) * K + j] = l;
            inv[static_cast<int64_t>(c) * K + j] = il;
        }
        top = fmaxf(top, __fmul_rn(x, il));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) top = fmaxf(top, __shfl_xor_sync(0xffffffffu, top, o));
    if ((threadIdx.x & 31) == 0) s_top[threadIdx.x >> 5] = top;
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = 0.0f;
        for (int i = 0; i < kGridThreads / 32; ++i) m = fmaxf(m, s_top[i]);
        if (store_ok(c, 1, ext_sg, err, kSiteGrid)) s_g[c] = m > 0.0f ? __fdiv_rn(m, 2688.0f) : 1.0f;
    }
}

}  // namespace
}  // namespace svdq

extern "C" int svdq_lambda_grid(const float* amax_x, const float* amax_w, int64_t K, const float* alpha, int n_alpha,
                                float* lambda, float* inv_lambda, float* s_g, void* stream) {
    using namespace svdq;
    if (amax_x == nullptr || amax_w == nullptr || alpha == nullptr || lambda == nullptr || inv_lambda == nullptr ||
        s_g == nullptr)
        return SVDQ_ERR_INVALID_ARG;
    if (K < 1 || n_alpha < 1 || n_alpha > 65535) return SVDQ_ERR_INVALID_ARG;
    const uintptr_t any = reinterpret_cast<uintptr_t>(amax_x) | reinterpret_cast<uintptr_t>(amax_w) |
                          reinterpret_cast<uintptr_t>(alpha) | reinterpret_cast<uintptr_t>(lambda) |
                          reinterpret_cast<uintptr_t>(inv_lambda) | reinterpret_cast<uintptr_t>(s_g);
    if (any & 3u) return SVDQ_ERR_MISALIGNED;
    if (!device_is_sm100()) return SVDQ_ERR_NO_DEVICE;
    if (!debug_ptrs_ok({amax_x, amax_w, alpha, lambda, inv_lambda, s_g})) return SVDQ_ERR_INVALID_ARG;
    uint32_t* err = device_error_word();
    if (err == nullptr) return SVDQ_ERR_CUDA;
    lambda_grid_kernel<<<static_cast<unsigned>(n_alpha), kGridThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        amax_x, amax_w, alpha, K, lambda, inv_lambda, s_g, debug_extent(kSiteGrid, K * n_alpha), n_alpha, err);
    return launch_status(cudaGetLastError());
}
