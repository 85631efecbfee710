// calib.cu -- per-channel absmax over selected rows, the smoothing scale
// lambda and the static activation tensor scale.
//
// "MiniMax-H3 NVFP4 -- what the smoothing scale should be calibrated on",
// section "Calibration" (activation absmax accumulated under a modality mask)
// and section "Why" (the kernel sees X / lambda); "DeltaQuant on MiniMax-H3",
// section "The activation scale bound held" (static tensor scale from a bound).
//
// Bandwidth-bound: every selected element of X and every element of W is read
// once.  |bf16| is the bit pattern with the sign cleared, and for non-negative
// values integer order equals value order, so two channels reduce per packed
// 16-bit unsigned max (__vmaxu2).
//
// Streaming: the channels are cut into bands of 2048 and the rows of each
// matrix (the selected rows of X, counted across its row segments, then the
// rows of W) into chunks; one 1024-thread CTA takes one (band, chunk) item: 256
// thread columns of 8 channels by 4 row slices, each thread reading its 16 bytes
// of every fourth row of the chunk with streaming loads, eight rows in flight
// (128 KB per SM).  A row's band is 4 KB of contiguous memory and the CTAs of a
// wave together cover whole rows: the wider a row's piece, the closer plain
// loads come to the copy bandwidth (4 KB pieces 5.6 TB/s, 1 KB pieces 4.8 TB/s
// on the 16384 x 20480 input).  The running maxima stay in registers (four
// packed words per thread), meet across the row slices in shared memory, and
// are merged into the outputs once per item (integer atomicMax on the fp32 bit
// patterns: exact and order independent).  One atomic per channel per item is
// what sizes the items: one CTA per SM, so the chunks per band are the SMs over
// the bands.
//
// Completion without scratch memory: the first lambda word of each band
// counts, for the duration of the call, the items merged into that band; the
// CTA whose merge is the band's last forms lambda and 1/lambda for its 2048
// channels.  The band maxima of RN(ax / lambda) / 2688 meet in the bits of the
// s_g output (atomicMax; division by 2688 is monotonic, so the max of the
// quotients is the quotient of the max), and lambda[1] counts finished bands;
// the last band writes the final s_g (1 when every maximum is 0) and lambda[1].
// So the call is two launches: a zeroing kernel and the reduction.  The
// reduction is a programmatic dependent of the zeroing kernel: its loads of X
// and W run while the zeroing finishes, and it waits for it
// (griddepcontrol.wait) before its first write to the outputs.
#include <algorithm>

#include "common.cuh"
#include "sm100.cuh"

namespace svdq {
namespace {

constexpr int kThreads = 1024;
constexpr int kColThreads = 256;              // thread columns of a band
constexpr int kRowSlices = kThreads / kColThreads;   // rows r, r + 4, ... per slice
constexpr int kBandCols = kColThreads * 8;    // channels per band (16 bytes of bf16 per thread)
constexpr int kRowsInFlight = 8;              // rows loaded per thread before they are reduced

struct CalibArgs {
    const uint16_t* x;
    int64_t ldx;
    const uint16_t* w;                        // nullptr when the weight is not read here
    int64_t ldw;
    SegTable segs;                            // selected rows of X
    int64_t K;
    int64_t bands;
    int64_t chunk_rows;                       // rows per chunk (both matrices)
    int64_t chunks[2];                        // chunks of X's selected rows, of W's rows
    int64_t rows[2];                          // selected rows of X, rows of W
    uint32_t* out_bits[2];                    // absmax of X, of W (fp32 bit patterns)
    const float* ax;
    const float* aw;                          // nullptr: lambda = 1
    float* lambda;
    float* inv_lambda;
    float* s_g;                               // holds max(band maxima) until the last band writes the scale
    uint32_t* err;
    int64_t ext_amax, ext_lambda;             // store-check extents (debug library): K each
};

__global__ void __launch_bounds__(256)
calib_zero_kernel(float* ax, float* aw, int64_t K, float* lambda, float* s_g, int64_t ext, uint32_t* err) {
    pdl_launch_dependents();                  // the reduction may start streaming at once
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < K; j += stride) {
        if (!store_ok(j, 1, ext, err, kSiteCalibZero)) continue;
        ax[j] = 0.0f;
        if (aw) aw[j] = 0.0f;
        if (j % kBandCols == 0 || j == 1) lambda[j] = 0.0f;   // band counters, bands-done counter
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) *reinterpret_cast<uint32_t*>(s_g) = 0u;
}

__device__ __forceinline__ float lambda_of(float x, const float* aw, int64_t j) {
    if (aw == nullptr) return 1.0f;
    const float w = __ldcg(aw + j);
    return (x > 0.0f && w > 0.0f) ? __fsqrt_rn(__fdiv_rn(x, w)) : 1.0f;
}

__device__ __forceinline__ float block_max(float v, float* red) {
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    if (threadIdx.x == 0)
        for (int w = 1; w < kThreads / 32; ++w) v = fmaxf(v, red[w]);
    return v;                                 // valid in thread 0
}

// By the CTA that made a band's last merge: lambda_j = sqrt(ax_j / aw_j) (1
// where either absmax is 0) and 1/lambda_j for the band's channels, then the
// band's share of s_g = max_j(ax_j / lambda_j) / (6 * 448).
__device__ void band_lambda(const CalibArgs& a, int64_t band) {
    __shared__ float red[kThreads / 32];
    const int64_t j1 = min(a.K, (band + 1) * kBandCols);
    float v = 0.0f;
    for (int64_t j = band * kBandCols + threadIdx.x; j < j1; j += kThreads) {
        const float x = __ldcg(a.ax + j);
        const float lam = lambda_of(x, a.aw, j);
        const float il = __frcp_rn(lam);
        if (store_ok(j, 1, a.ext_lambda, a.err, kSiteCalibLambda)) {
            if (j != 1) a.lambda[j] = lam;          // lambda[1] is the bands-done counter until the end
            if (a.inv_lambda) a.inv_lambda[j] = il;
        }
        v = fmaxf(v, __fmul_rn(x, il));
    }
    v = block_max(v, red);
    if (threadIdx.x == 0) {
        const float q = __fdiv_rn(v, 2688.0f);
        if (q > 0.0f) atomicMax(reinterpret_cast<uint32_t*>(a.s_g), __float_as_uint(q));
        __threadfence();
        const uint32_t done = atomicAdd(reinterpret_cast<uint32_t*>(a.lambda + 1), 1u);
        if (done == static_cast<uint32_t>(a.bands) - 1) {
            __threadfence();
            const float m = __uint_as_float(atomicAdd(reinterpret_cast<uint32_t*>(a.s_g), 0u));
            const float x1 = __ldcg(a.ax + 1);
            a.lambda[1] = lambda_of(x1, a.aw, 1);
            *a.s_g = m > 0.0f ? m : 1.0f;
        }
    }
}

__device__ __forceinline__ void max_row(uint32_t (&m)[4], const uint4& q) {
    m[0] = __vmaxu2(m[0], q.x & 0x7FFF7FFFu);
    m[1] = __vmaxu2(m[1], q.y & 0x7FFF7FFFu);
    m[2] = __vmaxu2(m[2], q.z & 0x7FFF7FFFu);
    m[3] = __vmaxu2(m[3], q.w & 0x7FFF7FFFu);
}

// Keeps the compiler from interleaving the maxima with the loads (which would
// leave one load in flight at a time): the loaded values pass through here first.
__device__ __forceinline__ void in_flight(uint4 (&q)[kRowsInFlight]) {
    static_assert(kRowsInFlight == 8, "one operand list per load");
    asm volatile(""
                 : "+r"(q[0].x), "+r"(q[0].y), "+r"(q[0].z), "+r"(q[0].w), "+r"(q[1].x), "+r"(q[1].y), "+r"(q[1].z),
                   "+r"(q[1].w), "+r"(q[2].x), "+r"(q[2].y), "+r"(q[2].z), "+r"(q[2].w), "+r"(q[3].x), "+r"(q[3].y),
                   "+r"(q[3].z), "+r"(q[3].w), "+r"(q[4].x), "+r"(q[4].y), "+r"(q[4].z), "+r"(q[4].w), "+r"(q[5].x),
                   "+r"(q[5].y), "+r"(q[5].z), "+r"(q[5].w), "+r"(q[6].x), "+r"(q[6].y), "+r"(q[6].z), "+r"(q[6].w),
                   "+r"(q[7].x), "+r"(q[7].y), "+r"(q[7].z), "+r"(q[7].w));
}

// Maxima of this thread's 8 channels (column `col`) over rows r0, r0 + step,
// ... below r1 of a matrix with row stride ld, kRowsInFlight rows loaded before
// they are reduced.
__device__ __forceinline__ void max_rows(uint32_t (&m)[4], const uint16_t* base, int64_t ld, int64_t r0, int64_t r1,
                                         int step, int64_t col) {
    const int64_t stride = ld * step;
    const uint16_t* p = base + r0 * ld + col;
    int64_t r = r0;
    for (; r + (kRowsInFlight - 1) * step < r1; r += kRowsInFlight * step, p += kRowsInFlight * stride) {
        uint4 q[kRowsInFlight];
#pragma unroll
        for (int i = 0; i < kRowsInFlight; ++i) q[i] = __ldcs(reinterpret_cast<const uint4*>(p + i * stride));
        in_flight(q);                          // all eight loads issue before the first max waits for one
#pragma unroll
        for (int i = 0; i < kRowsInFlight; ++i) max_row(m, q[i]);
    }
    for (; r < r1; r += step, p += stride) max_row(m, __ldcs(reinterpret_cast<const uint4*>(p)));
}

__global__ void __launch_bounds__(kThreads, 1)
calib_rows_kernel(const __grid_constant__ CalibArgs a) {
    __shared__ uint32_t is_last;
    __shared__ uint4 slice_max[kRowSlices - 1][kColThreads];
    const int64_t band = blockIdx.x % a.bands;
    const int64_t chunk = blockIdx.x / a.bands;
    const int job = chunk < a.chunks[0] ? 0 : 1;
    const int64_t c = job ? chunk - a.chunks[0] : chunk;
    const int64_t p0 = c * a.chunk_rows;
    const int64_t p1 = min(p0 + a.chunk_rows, a.rows[job]);
    const int tc = threadIdx.x % kColThreads, tr = threadIdx.x / kColThreads;
    const int64_t col = band * kBandCols + tc * 8;
    const bool active = col < a.K;             // K % 8 == 0: a thread's 8 channels are all in or all out
    uint32_t m[4] = {0u, 0u, 0u, 0u};
    if (active && p0 < p1) {
        if (job == 0) {
            // the chunk's selected rows, segment by segment; this slice takes every
            // kRowSlices-th of them, counted from the chunk's first
            int s = 0;
            while (s + 1 < a.segs.n && p0 >= a.segs.prefix[s + 1]) ++s;
            for (int64_t p = p0; p < p1; ++s) {
                const int64_t e = min(p1, a.segs.prefix[s + 1]);
                const int64_t first = p + ((tr - (p - p0)) % kRowSlices + kRowSlices) % kRowSlices;
                const int64_t row = a.segs.begin[s] + (first - a.segs.prefix[s]);
                if (first < e) max_rows(m, a.x, a.ldx, row, row + (e - first), kRowSlices, col);
                p = e;
            }
        } else {
            max_rows(m, a.w, a.ldw, p0 + tr, p1, kRowSlices, col);
        }
    }
    // the row slices meet in shared memory: slice 0 keeps the band's maxima
    if (tr > 0) slice_max[tr - 1][tc] = make_uint4(m[0], m[1], m[2], m[3]);
    __syncthreads();
    if (tr == 0) {
#pragma unroll
        for (int i = 0; i < kRowSlices - 1; ++i) max_row(m, slice_max[i][tc]);
    }
    pdl_wait();                                // the zeroing kernel's writes are complete and visible
    if (active && tr == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t v = (m[i] >> (16 * h)) & 0xFFFFu;
                const int64_t j = col + 2 * i + h;
                if (v != 0 && store_ok(j, 1, a.ext_amax, a.err, kSiteCalibAmax))
                    atomicMax(a.out_bits[job] + j, v << 16);          // bf16 -> fp32 bits
            }
        }
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        is_last = 0u;
        const int64_t ctr = band * kBandCols;
        if (store_ok(ctr, 1, a.ext_lambda, a.err, kSiteCalibLambda)) {
            const uint32_t prev = atomicAdd(reinterpret_cast<uint32_t*>(a.lambda + ctr), 1u);
            const int64_t items = a.chunks[0] + a.chunks[1];
            is_last = (static_cast<int64_t>(prev) == items - 1) ? 1u : 0u;
        }
    }
    __syncthreads();
    if (is_last) {
        __threadfence();
        band_lambda(a, band);
    }
}

// Shared by both entry points.  W != NULL: the weight's absmax is reduced into
// amax_w here.  W == NULL and aw_in != NULL: aw_in is the stored absmax of the
// weight (an input).  Both NULL: lambda = 1.
int calib_launch(const void* X, int64_t M, int64_t K, int64_t ldx, const svdq_seg* segs, int n_seg,
                 const void* W, int64_t N, int64_t ldw, const float* aw_in,
                 float* amax_x, float* amax_w, float* lambda, float* inv_lambda, float* s_g, void* stream) {
    if (X == nullptr || amax_x == nullptr || lambda == nullptr || s_g == nullptr) return SVDQ_ERR_INVALID_ARG;
    if (M < 1 || K < 8 || K % 8 != 0 || ldx < K) return SVDQ_ERR_INVALID_ARG;
    if (W != nullptr && (amax_w == nullptr || N < 1 || ldw < K)) return SVDQ_ERR_INVALID_ARG;
    if (!aligned16(X) || (ldx * 2) % 16 != 0) return SVDQ_ERR_MISALIGNED;
    if (W != nullptr && (!aligned16(W) || (ldw * 2) % 16 != 0)) return SVDQ_ERR_MISALIGNED;
    if ((reinterpret_cast<uintptr_t>(s_g) | reinterpret_cast<uintptr_t>(amax_x)) & 3u) return SVDQ_ERR_MISALIGNED;
    if (W != nullptr && (reinterpret_cast<uintptr_t>(amax_w) & 3u)) return SVDQ_ERR_MISALIGNED;
    if (aw_in != nullptr && (reinterpret_cast<uintptr_t>(aw_in) & 3u)) return SVDQ_ERR_MISALIGNED;
    if (M > 0x7FFFFFFF || N > 0x7FFFFFFF || K > (int64_t(1) << 30)) return SVDQ_ERR_UNSUPPORTED;
    CalibArgs a{};
    int st = make_seg_table(segs, n_seg, M, &a.segs);
    if (st != SVDQ_OK) return st;
    if (!device_is_sm100()) return SVDQ_ERR_NO_DEVICE;
    if (!debug_ptrs_ok({X, W, aw_in, amax_x, amax_w, lambda, inv_lambda, s_g})) return SVDQ_ERR_INVALID_ARG;
    uint32_t* err = device_error_word();
    if (err == nullptr) return SVDQ_ERR_CUDA;
    const int64_t sms = device_sm_count() > 0 ? device_sm_count() : 148;

    a.x = static_cast<const uint16_t*>(X);
    a.ldx = ldx;
    a.w = static_cast<const uint16_t*>(W);
    a.ldw = ldw;
    a.K = K;
    a.bands = (K + kBandCols - 1) / kBandCols;
    a.rows[0] = a.segs.prefix[a.segs.n];
    a.rows[1] = W != nullptr ? N : 0;
    // Items (band x chunk): one wave of one CTA per SM (the chunks per band are
    // the SMs over the bands, rounded down); chunks no shorter than the rows in
    // flight.  With no rows at all, one empty chunk per band still forms lambda = 1.
    const int64_t total_rows = a.rows[0] + a.rows[1];
    const int64_t chunks_wanted = std::max<int64_t>(1, sms / a.bands);
    // the two matrices' chunks round up separately: lengthen the chunks until
    // their sum fits the wave
    for (int64_t t = chunks_wanted; t >= 1; --t) {
        a.chunk_rows = std::max<int64_t>(kRowsInFlight, (total_rows + t - 1) / t);
        a.chunks[0] = (a.rows[0] + a.chunk_rows - 1) / a.chunk_rows;
        a.chunks[1] = (a.rows[1] + a.chunk_rows - 1) / a.chunk_rows;
        if (a.chunks[0] + a.chunks[1] <= chunks_wanted) break;
    }
    if (a.chunks[0] + a.chunks[1] == 0) a.chunks[0] = 1;
    const int64_t grid = a.bands * (a.chunks[0] + a.chunks[1]);
    if (grid > 0x7FFFFFFF) return SVDQ_ERR_UNSUPPORTED;
    a.out_bits[0] = reinterpret_cast<uint32_t*>(amax_x);
    a.out_bits[1] = reinterpret_cast<uint32_t*>(amax_w);
    a.ax = amax_x;
    a.aw = W != nullptr ? amax_w : aw_in;
    a.lambda = lambda;
    a.inv_lambda = inv_lambda;
    a.s_g = s_g;
    a.err = err;
    a.ext_amax = debug_extent(kSiteCalibAmax, K);
    a.ext_lambda = debug_extent(kSiteCalibLambda, K);

    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const int64_t zb = (K + 255) / 256;
    // the stored weight absmax is an input: only the outputs are zeroed
    calib_zero_kernel<<<static_cast<unsigned>(zb < sms ? zb : sms), 256, 0, cs>>>(
        amax_x, W != nullptr ? amax_w : nullptr, K, lambda, s_g, debug_extent(kSiteCalibZero, K), err);
    st = launch_status(cudaGetLastError());
    if (st != SVDQ_OK) return st;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = cs;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return launch_status(cudaLaunchKernelEx(&cfg, calib_rows_kernel, a));
}

}  // namespace
}  // namespace svdq

extern "C" int svdq_calib_lambda(const void* X, int64_t M, int64_t K, int64_t ldx,
                                 const svdq_seg* segs, int n_seg,
                                 const void* W, int64_t N, int64_t ldw,
                                 float* amax_x, float* amax_w, float* lambda, float* inv_lambda,
                                 float* s_g, void* stream) {
    return svdq::calib_launch(X, M, K, ldx, segs, n_seg, W, N, ldw, nullptr, amax_x, amax_w, lambda, inv_lambda,
                              s_g, stream);
}

extern "C" int svdq_calib_lambda_stored_w(const void* X, int64_t M, int64_t K, int64_t ldx,
                                          const svdq_seg* segs, int n_seg, const float* amax_w,
                                          float* amax_x, float* lambda, float* inv_lambda, float* s_g,
                                          void* stream) {
    if (amax_w == nullptr) return SVDQ_ERR_INVALID_ARG;
    return svdq::calib_launch(X, M, K, ldx, segs, n_seg, nullptr, 0, 0, amax_w, amax_x, nullptr, lambda,
                              inv_lambda, s_g, stream);
}
