// proxy.cu -- the bits-lost proxy: how many bits the input channels of a linear
// lose to the shared NVFP4 group scale, per modality and per lambda candidate.
//
// "MiniMax-H3 NVFP4 -- what the smoothing scale should be calibrated on",
// section "Why": 16 consecutive input channels share one FP8 scale set by the
// group's absmax, so a channel whose own absmax is below the group's loses
// log2(group_absmax / channel_absmax) bits, and lambda reshapes that profile
// because the kernel sees X / lambda.  The figure needs only statistics: the
// per-modality channel absmax that the calibration pass produces (one fp32
// vector per modality, svdq_calib_lambda over that modality's rows) and one
// 1/lambda vector per candidate, so a whole lambda grid is scored in one launch
// of a few microseconds, without a GEMM.
//
// One CTA per (modality, candidate).  Each thread takes whole 16-channel
// groups: in fp32 the smoothed statistic RN(ax * (1/lambda)) (what the
// activation quantiser's group scale sees; the maximum over rows commutes with
// the monotone rounded product) and the group maximum, then in fp64 the sum of
// log2(group / channel) over the channels whose statistic is nonzero (a zero
// channel has nothing to lose).  A fixed-order reduction makes the result
// deterministic; the mean is that sum over the number of channels counted.
#include "common.cuh"
#include "sm100.cuh"

namespace svdq {
namespace {

constexpr int kProxyThreads = 256;
constexpr int kGroup = 16;

__global__ void __launch_bounds__(kProxyThreads)
bits_lost_kernel(const float* __restrict__ ax, int64_t ld_ax, const float* __restrict__ inv_lam, int64_t ld_lam,
                 int64_t K, int n_mod, double* __restrict__ bits, int64_t ext, uint32_t* err) {
    __shared__ double s_sum[kProxyThreads / 32];
    __shared__ unsigned long long s_cnt[kProxyThreads / 32];
    const int mod = blockIdx.x;
    const int cand = blockIdx.y;
    const float* a = ax + static_cast<int64_t>(mod) * ld_ax;
    const float* il = inv_lam != nullptr ? inv_lam + static_cast<int64_t>(cand) * ld_lam : nullptr;
    double sum = 0.0;
    unsigned long long cnt = 0;
    for (int64_t g = threadIdx.x; g < K / kGroup; g += kProxyThreads) {
        float c[kGroup];
        float gmax = 0.0f;
#pragma unroll
        for (int j = 0; j < kGroup; ++j) {
            const float v = __ldg(a + g * kGroup + j);
            c[j] = il != nullptr ? __fmul_rn(v, __ldg(il + g * kGroup + j)) : v;
            gmax = fmaxf(gmax, c[j]);
        }
#pragma unroll
        for (int j = 0; j < kGroup; ++j) {
            if (c[j] > 0.0f) {
                sum += log2(static_cast<double>(gmax) / static_cast<double>(c[j]));
                ++cnt;
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        sum += __shfl_xor_sync(0xffffffffu, sum, o);
        cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    }
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) {
        s_sum[warp] = sum;
        s_cnt[warp] = cnt;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double total = 0.0;
        unsigned long long n = 0;
        for (int w = 0; w < kProxyThreads / 32; ++w) {
            total += s_sum[w];
            n += s_cnt[w];
        }
        const int64_t off = static_cast<int64_t>(cand) * n_mod + mod;
        if (store_ok(off, 1, ext, err, kSiteBits)) bits[off] = n > 0 ? total / static_cast<double>(n) : 0.0;
    }
}

}  // namespace
}  // namespace svdq

extern "C" int svdq_bits_lost(const float* amax_x, int64_t ld_amax, int n_mod, const float* inv_lambda,
                              int64_t ld_lam, int n_cand, int64_t K, double* bits, void* stream) {
    using namespace svdq;
    if (amax_x == nullptr || bits == nullptr) return SVDQ_ERR_INVALID_ARG;
    if (n_mod < 1 || n_mod > 65535 || n_cand < 1 || n_cand > 65535) return SVDQ_ERR_INVALID_ARG;
    if (K < kGroup || K % kGroup != 0 || ld_amax < K) return SVDQ_ERR_INVALID_ARG;
    if (inv_lambda == nullptr ? n_cand != 1 : ld_lam < K) return SVDQ_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(amax_x) & 3u) || (reinterpret_cast<uintptr_t>(inv_lambda) & 3u) ||
        (reinterpret_cast<uintptr_t>(bits) & 7u))
        return SVDQ_ERR_MISALIGNED;
    if (!device_is_sm100()) return SVDQ_ERR_NO_DEVICE;
    if (!debug_ptrs_ok({amax_x, inv_lambda, bits})) return SVDQ_ERR_INVALID_ARG;
    uint32_t* err = device_error_word();
    if (err == nullptr) return SVDQ_ERR_CUDA;
    bits_lost_kernel<<<dim3(static_cast<unsigned>(n_mod), static_cast<unsigned>(n_cand)), kProxyThreads, 0,
                       static_cast<cudaStream_t>(stream)>>>(amax_x, ld_amax, inv_lambda, ld_lam, K, n_mod, bits,
                                                       debug_extent(kSiteBits, int64_t(n_mod) * n_cand), err);
    return launch_status(cudaGetLastError());
}
