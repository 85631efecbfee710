// calib.cu -- per-channel absmax over selected rows, the smoothing scale
// lambda and the static activation tensor scale.
//
// "MiniMax-H3 NVFP4 -- what the smoothing scale should be calibrated on",
// section "Calibration" (activation absmax accumulated under a modality mask)
// and section "Why" (the kernel sees X / lambda); "DeltaQuant on MiniMax-H3",
// section "The activation scale bound held" (static tensor scale from a bound).
//
// Bandwidth-bound: every selected element of X and every element of W is read
// once, with 16-byte loads.  |bf16| is the bit pattern with the sign cleared,
// and for non-negative values integer order equals value order, so two
// channels reduce per packed 16-bit unsigned max (__vmaxu2).
//
// Work split: the columns are cut into 256-channel strips (a warp reads one
// 512-byte row segment per load) and the rows of each matrix into equal
// chunks, sized on the host so that the CTAs (strip x chunk, both matrices)
// fill every SM about once at four CTAs per SM.  Each CTA merges its strip's
// maxima into the outputs with integer atomicMax on the fp32 bit patterns
// (exact and order independent).
//
// Completion without scratch memory: the first lambda word of each strip
// counts, for the duration of the call, the CTAs of that strip that are done;
// the last one forms lambda and 1/lambda for the strip's 256 channels.  The
// strip maxima of RN(ax / lambda) / 2688 meet in the bits of the s_g output
// (atomicMax; division by 2688 is monotonic, so the max of the quotients is
// the quotient of the max), and lambda[1] counts finished strips; the last
// strip writes the final s_g (1 when every maximum is 0) and lambda[1].  So the
// call is two launches: a zeroing kernel and the reduction.
#include "common.cuh"
#include "sm100.cuh"

namespace svdq {
namespace {

constexpr int kThreads = 256;                 // 8 warps
constexpr int kWarps = kThreads / 32;
constexpr int kColsPerLane = 8;               // one 16-byte load
constexpr int kStripCols = 32 * kColsPerLane; // 256 channels per CTA
constexpr int kUnroll = 8;                    // independent 16-byte loads in flight per thread
constexpr int kCtasPerSm = 4;

struct MatJob {
    const uint16_t* base;
    int64_t ld;          // elements
    int64_t rows;        // selected rows
    int64_t chunk;       // rows per CTA
    int64_t n_chunks;
    uint32_t* out_bits;  // fp32 absmax as bit patterns
};

struct CalibArgs {
    MatJob job[2];       // 0: activations over the selected rows, 1: the weight (all rows)
    SegTable segs;       // row selection of job 0
    int64_t K;
    int64_t strips;
    int64_t ctas_job0;   // strips * job[0].n_chunks
    uint32_t ctas_per_strip;  // job[0].n_chunks + job[1].n_chunks
    const float* ax;     // == job[0].out_bits (as float)
    const float* aw;     // nullptr when there is no weight
    float* lambda;
    float* inv_lambda;
    float* s_g;          // holds max(strip maxima) until the last strip writes the scale
};

__global__ void __launch_bounds__(256)
calib_zero_kernel(float* ax, float* aw, int64_t K, float* lambda, float* s_g) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < K; j += stride) {
        ax[j] = 0.0f;
        if (aw) aw[j] = 0.0f;
        if (j % kStripCols == 0 || j == 1) lambda[j] = 0.0f;   // strip counters, strips-done counter
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) *reinterpret_cast<uint32_t*>(s_g) = 0u;
}

__device__ __forceinline__ float lambda_of(float x, const float* aw, int64_t j) {
    if (aw == nullptr) return 1.0f;
    const float w = __ldcg(aw + j);
    return (x > 0.0f && w > 0.0f) ? __fsqrt_rn(__fdiv_rn(x, w)) : 1.0f;
}

// The last CTA of a strip: lambda_j = sqrt(ax_j / aw_j) (1 where either absmax
// is 0) and 1/lambda_j for the strip's channels, then the strip's share of
// s_g = max_j(ax_j / lambda_j) / (6 * 448).
__device__ void strip_lambda(const CalibArgs& a, int64_t strip) {
    __shared__ float red[kWarps];
    __shared__ uint32_t strips_done;
    const int64_t j = strip * kStripCols + threadIdx.x;
    float v = 0.0f;
    if (j < a.K) {
        const float x = __ldcg(a.ax + j);
        const float lam = lambda_of(x, a.aw, j);
        const float il = __frcp_rn(lam);
        if (j != 1) a.lambda[j] = lam;          // lambda[1] is the strips-done counter until the end
        if (a.inv_lambda) a.inv_lambda[j] = il;
        v = __fmul_rn(x, il);
    }
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kWarps; ++w) v = fmaxf(v, red[w]);
        const float q = __fdiv_rn(v, 2688.0f);
        if (q > 0.0f) atomicMax(reinterpret_cast<uint32_t*>(a.s_g), __float_as_uint(q));
        __threadfence();
        strips_done = atomicAdd(reinterpret_cast<uint32_t*>(a.lambda + 1), 1u);
        if (strips_done == static_cast<uint32_t>(a.strips) - 1) {
            __threadfence();
            const float m = __uint_as_float(atomicAdd(reinterpret_cast<uint32_t*>(a.s_g), 0u));
            const float x1 = __ldcg(a.ax + 1);
            a.lambda[1] = lambda_of(x1, a.aw, 1);
            *a.s_g = m > 0.0f ? m : 1.0f;
        }
    }
}

__global__ void __launch_bounds__(kThreads, kCtasPerSm)
calib_absmax_kernel(const __grid_constant__ CalibArgs a) {
    __shared__ uint32_t red[kWarps][32][kColsPerLane / 2];
    __shared__ uint32_t is_last;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t b = blockIdx.x;
    const bool is_w = b >= a.ctas_job0;
    const int64_t local = is_w ? b - a.ctas_job0 : b;
    const MatJob& job = a.job[is_w ? 1 : 0];
    uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;
    {
        const int64_t strip = local % a.strips;
        const int64_t chunk = local / a.strips;
        const int64_t col0 = strip * kStripCols + lane * kColsPerLane;
        const int64_t v_end = min(job.rows, (chunk + 1) * job.chunk);
        int64_t v = chunk * job.chunk + warp;
        // Virtual (selected) row -> physical row: keep the current segment's
        // end and offset in registers; only a crossing re-reads the table.
        int s = 0;
        int64_t seg_end = job.rows, off = 0;
        if (!is_w) {
            while (s + 1 < a.segs.n && v >= a.segs.prefix[s + 1]) ++s;
            seg_end = a.segs.prefix[s + 1];
            off = a.segs.begin[s] - a.segs.prefix[s];
        }
        if (col0 < a.K) {
            const uint16_t* colp = job.base + col0;
            for (; v < v_end; v += kWarps * kUnroll) {
                uint4 q[kUnroll];
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    const int64_t vv = v + u * kWarps;
                    q[u] = make_uint4(0, 0, 0, 0);
                    if (vv < v_end) {
                        if (vv >= seg_end) {       // rare: the chunk crosses a segment boundary
                            while (s + 1 < a.segs.n && vv >= a.segs.prefix[s + 1]) ++s;
                            seg_end = a.segs.prefix[s + 1];
                            off = a.segs.begin[s] - a.segs.prefix[s];
                        }
                        q[u] = ldg_stream_v4(colp + (vv + off) * job.ld);
                    }
                }
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    m0 = __vmaxu2(m0, q[u].x & 0x7FFF7FFFu);
                    m1 = __vmaxu2(m1, q[u].y & 0x7FFF7FFFu);
                    m2 = __vmaxu2(m2, q[u].z & 0x7FFF7FFFu);
                    m3 = __vmaxu2(m3, q[u].w & 0x7FFF7FFFu);
                }
            }
        }
    }
    red[warp][lane][0] = m0;
    red[warp][lane][1] = m1;
    red[warp][lane][2] = m2;
    red[warp][lane][3] = m3;
    __syncthreads();
    {
        // thread t owns channel t of the strip
        const int t = threadIdx.x;
        const int src_lane = t / kColsPerLane, word = (t % kColsPerLane) / 2, hi = t & 1;
        uint32_t m = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) m = max(m, (red[w][src_lane][word] >> (16 * hi)) & 0xFFFFu);
        const int64_t col = (local % a.strips) * kStripCols + t;
        if (m != 0 && col < a.K) atomicMax(job.out_bits + col, m << 16);   // bf16 -> fp32 bits
    }
    // Completion count of the strip: its last CTA sees every other CTA's atomics.
    const int64_t strip = local % a.strips;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t prev = atomicAdd(reinterpret_cast<uint32_t*>(a.lambda + strip * kStripCols), 1u);
        is_last = (prev == a.ctas_per_strip - 1) ? 1u : 0u;
    }
    __syncthreads();
    if (is_last) {
        __threadfence();
        strip_lambda(a, strip);
    }
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
    if ((reinterpret_cast<uintptr_t>(s_g) | reinterpret_cast<uintptr_t>(amax_x)) & 3u) return SVDQ_ERR_MISALIGNED;
    if (W != nullptr && (reinterpret_cast<uintptr_t>(amax_w) & 3u)) return SVDQ_ERR_MISALIGNED;
    CalibArgs a{};
    int st = make_seg_table(segs, n_seg, M, &a.segs);
    if (st != SVDQ_OK) return st;
    if (!device_is_sm100()) return SVDQ_ERR_NO_DEVICE;
    const int64_t sms = device_sm_count() > 0 ? device_sm_count() : 148;

    a.K = K;
    a.strips = (K + kStripCols - 1) / kStripCols;
    const int64_t rx = a.segs.prefix[a.segs.n];
    const int64_t rw = W != nullptr ? N : 0;
    // Rows per CTA: the smallest multiple of 8 whose CTA count fits kCtasPerSm per SM.
    const int64_t slots = sms * kCtasPerSm;
    const int64_t total_rows = a.strips * (rx + rw);
    int64_t chunk = (total_rows + slots - 1) / slots;
    chunk = (chunk + 7) / 8 * 8;
    if (chunk < 8) chunk = 8;
    auto n_chunks = [&](int64_t rows) { return rows > 0 ? (rows + chunk - 1) / chunk : int64_t(0); };
    while (a.strips * (n_chunks(rx) + n_chunks(rw)) > slots && chunk < (rx > rw ? rx : rw)) chunk += 8;
    a.job[0] = MatJob{static_cast<const uint16_t*>(X), ldx, rx, chunk, n_chunks(rx), reinterpret_cast<uint32_t*>(amax_x)};
    a.job[1] = MatJob{static_cast<const uint16_t*>(W), ldw, rw, chunk, n_chunks(rw), reinterpret_cast<uint32_t*>(amax_w)};
    if (a.job[0].n_chunks + a.job[1].n_chunks == 0) a.job[0].n_chunks = 1;   // no rows: one idle CTA per strip
    a.ctas_job0 = a.strips * a.job[0].n_chunks;
    a.ctas_per_strip = static_cast<uint32_t>(a.job[0].n_chunks + a.job[1].n_chunks);
    const int64_t total = a.strips * a.ctas_per_strip;
    if (total > 0x7FFFFFFF) return SVDQ_ERR_UNSUPPORTED;
    a.ax = amax_x;
    a.aw = W != nullptr ? amax_w : nullptr;
    a.lambda = lambda;
    a.inv_lambda = inv_lambda;
    a.s_g = s_g;

    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const int64_t zb = (K + 255) / 256;
    calib_zero_kernel<<<static_cast<unsigned>(zb < sms ? zb : sms), 256, 0, cs>>>(
        amax_x, W != nullptr ? amax_w : nullptr, K, lambda, s_g);
    st = launch_status(cudaGetLastError());
    if (st != SVDQ_OK) return st;
    calib_absmax_kernel<<<static_cast<unsigned>(total), kThreads, 0, cs>>>(a);
    return launch_status(cudaGetLastError());
}
