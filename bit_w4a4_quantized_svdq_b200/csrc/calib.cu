// calib.cu -- per-channel absmax over selected rows, the smoothing scale
// lambda and the static activation tensor scale.
//
// "MiniMax-H3 NVFP4 -- what the smoothing scale should be calibrated on",
// section "Calibration" (activation absmax accumulated under a modality mask)
// and section "Why" (the kernel sees X / lambda); "DeltaQuant on MiniMax-H3",
// section "The activation scale bound held" (static tensor scale from a bound).
//
// Bandwidth-bound: each element is read once with 16-byte loads.  |bf16| is
// the bit pattern with the sign cleared, and for non-negative values integer
// order equals value order, so two channels at a time reduce with one
// packed 16-bit unsigned max (__vmaxu2).  Per-block results merge with an
// integer atomicMax on the fp32 bit pattern (exact, order independent).
#include "common.cuh"
#include "sm100.cuh"

namespace svdq {
namespace {

constexpr int kColsPerThread = 8;             // one 16-byte load
constexpr int kThreadsX = 32;                 // 256 channels per block
constexpr int kThreadsY = 8;
constexpr int kRowsPerThread = 16;            // independent loads in flight per thread (one round)
constexpr int kRounds = 4;                    // rounds per block: 512 rows, so few atomics per column
constexpr int kRowsPerBlock = kThreadsY * kRowsPerThread * kRounds;

struct AbsmaxJob {
    const uint16_t* base;
    int64_t ld;
    SegTable segs;
    int64_t total_rows;
    uint32_t* out_bits;
};

// blockIdx.z selects the job (0: activations over the selected rows, 1: the weight).
__global__ void __launch_bounds__(kThreadsX * kThreadsY)
col_absmax_kernel(AbsmaxJob job0, AbsmaxJob job1, int64_t K) {
    __shared__ uint32_t red[kThreadsY][kThreadsX][kColsPerThread / 2];
    const AbsmaxJob& job = blockIdx.z == 0 ? job0 : job1;
    const int64_t v0 = static_cast<int64_t>(blockIdx.y) * kRowsPerBlock;
    if (v0 >= job.total_rows) return;                       // uniform per block
    const int64_t v1 = min(v0 + kRowsPerBlock, job.total_rows);
    const int64_t col0 = (static_cast<int64_t>(blockIdx.x) * kThreadsX + threadIdx.x) * kColsPerThread;
    const bool col_ok = col0 < K;
    uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;
    if (col_ok) {
      int s = 0;
      for (int round = 0; round < kRounds; ++round) {
        uint4 q[kRowsPerThread];
#pragma unroll
        for (int i = 0; i < kRowsPerThread; ++i) {
            const int64_t v = v0 + threadIdx.y + static_cast<int64_t>(round * kRowsPerThread + i) * kThreadsY;
            if (v < v1) {
                while (s + 1 < job.segs.n && v >= job.segs.prefix[s + 1]) ++s;   // v increases with i
                const int64_t row = job.segs.begin[s] + (v - job.segs.prefix[s]);
                q[i] = __ldg(reinterpret_cast<const uint4*>(job.base + row * job.ld + col0));
            } else {
                q[i] = make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int i = 0; i < kRowsPerThread; ++i) {
            m0 = __vmaxu2(m0, q[i].x & 0x7FFF7FFFu);
            m1 = __vmaxu2(m1, q[i].y & 0x7FFF7FFFu);
            m2 = __vmaxu2(m2, q[i].z & 0x7FFF7FFFu);
            m3 = __vmaxu2(m3, q[i].w & 0x7FFF7FFFu);
        }
      }
    }
    red[threadIdx.y][threadIdx.x][0] = m0;
    red[threadIdx.y][threadIdx.x][1] = m1;
    red[threadIdx.y][threadIdx.x][2] = m2;
    red[threadIdx.y][threadIdx.x][3] = m3;
    __syncthreads();
    if (threadIdx.y == 0 && col_ok) {
        for (int y = 1; y < kThreadsY; ++y) {
            m0 = __vmaxu2(m0, red[y][threadIdx.x][0]);
            m1 = __vmaxu2(m1, red[y][threadIdx.x][1]);
            m2 = __vmaxu2(m2, red[y][threadIdx.x][2]);
            m3 = __vmaxu2(m3, red[y][threadIdx.x][3]);
        }
        const uint32_t w[4] = {m0, m1, m2, m3};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            // bf16 -> fp32 bit pattern is a 16-bit left shift.
            const uint32_t lo = (w[i] & 0xFFFFu) << 16;
            const uint32_t hi = w[i] & 0xFFFF0000u;
            if (lo) atomicMax(job.out_bits + col0 + 2 * i, lo);
            if (hi) atomicMax(job.out_bits + col0 + 2 * i + 1, hi);
        }
    }
}

__global__ void __launch_bounds__(1024)
lambda_kernel(const float* __restrict__ ax, const float* __restrict__ aw, int64_t K,
              float* __restrict__ lambda, float* __restrict__ inv_lambda, float* __restrict__ s_g) {
    __shared__ float red[32];
    float top = 0.0f;
    for (int64_t j = threadIdx.x; j < K; j += blockDim.x) {
        const float a = ax[j];
        float lam = 1.0f;
        if (aw != nullptr) {
            const float b = aw[j];
            if (a > 0.0f && b > 0.0f) lam = __fsqrt_rn(__fdiv_rn(a, b));
        }
        const float il = __frcp_rn(lam);
        lambda[j] = lam;
        if (inv_lambda) inv_lambda[j] = il;
        top = fmaxf(top, __fmul_rn(a, il));
    }
    for (int o = 16; o > 0; o >>= 1) top = fmaxf(top, __shfl_xor_sync(0xffffffffu, top, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = top;
    __syncthreads();
    if (threadIdx.x < 32) {
        top = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0f;
        for (int o = 16; o > 0; o >>= 1) top = fmaxf(top, __shfl_xor_sync(0xffffffffu, top, o));
        if (threadIdx.x == 0) s_g[0] = top > 0.0f ? __fdiv_rn(top, 2688.0f) : 1.0f;
    }
}

// Column absmax of X over `segs` (and of W over all of its rows, if given) in one launch.
int launch_col_absmax(const void* X, int64_t K, int64_t ldx, const SegTable& segs, float* out_x,
                      const void* W, int64_t N, int64_t ldw, float* out_w, cudaStream_t st) {
    AbsmaxJob jx{static_cast<const uint16_t*>(X), ldx, segs, segs.prefix[segs.n], reinterpret_cast<uint32_t*>(out_x)};
    AbsmaxJob jw = jx;
    if (W != nullptr) {
        SegTable all;
        make_seg_table(nullptr, 0, N, &all);
        jw = AbsmaxJob{static_cast<const uint16_t*>(W), ldw, all, N, reinterpret_cast<uint32_t*>(out_w)};
    }
    if (cudaMemsetAsync(out_x, 0, sizeof(float) * K, st) != cudaSuccess) return SVDQ_ERR_CUDA;
    if (W != nullptr && cudaMemsetAsync(out_w, 0, sizeof(float) * K, st) != cudaSuccess) return SVDQ_ERR_CUDA;
    const int64_t rows = max(jx.total_rows, W != nullptr ? jw.total_rows : int64_t(0));
    if (rows == 0) return SVDQ_OK;
    const int64_t gx = (K + kThreadsX * kColsPerThread - 1) / (kThreadsX * kColsPerThread);
    const int64_t gy = (rows + kRowsPerBlock - 1) / kRowsPerBlock;
    // 65535 blocks of 512 rows in y: about 33 million rows per call.
    if (gy > 65535) return SVDQ_ERR_UNSUPPORTED;
    dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy), W != nullptr ? 2u : 1u);
    col_absmax_kernel<<<grid, dim3(kThreadsX, kThreadsY), 0, st>>>(jx, jw, K);
    return launch_status(cudaGetLastError());
}

}  // namespace
}  // namespace svdq

extern "C" int svdq_calib_lambda(const void* X, int64_t M, int64_t K, int64_t ldx,
                                 const svdq_seg* segs, int n_seg,
                                 const void* W, int64_t N, int64_t ldw,
                                 float* amax_x, float* amax_w, float* lambda, float* inv_lambda,
                                 float* s_g, void* stream) {
    using namespace svdq;
    if (X == nullptr || amax_x == nullptr || lambda == nullptr || s_g == nullptr) return SVDQ_ERR_INVALID_ARG;
    if (M < 1 || K < 8 || K % 8 != 0 || ldx < K) return SVDQ_ERR_INVALID_ARG;
    if (W != nullptr && (amax_w == nullptr || N < 1 || ldw < K)) return SVDQ_ERR_INVALID_ARG;
    if (!aligned16(X) || (ldx * 2) % 16 != 0) return SVDQ_ERR_MISALIGNED;
    if (W != nullptr && (!aligned16(W) || (ldw * 2) % 16 != 0)) return SVDQ_ERR_MISALIGNED;
    SegTable table;
    int st = make_seg_table(segs, n_seg, M, &table);
    if (st != SVDQ_OK) return st;
    if (!device_is_sm100()) return SVDQ_ERR_NO_DEVICE;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    st = launch_col_absmax(X, K, ldx, table, amax_x, W, N, ldw, amax_w, cs);
    if (st != SVDQ_OK) return st;
    lambda_kernel<<<1, 1024, 0, cs>>>(amax_x, W != nullptr ? amax_w : nullptr, K, lambda, inv_lambda, s_g);
    return launch_status(cudaGetLastError());
}
