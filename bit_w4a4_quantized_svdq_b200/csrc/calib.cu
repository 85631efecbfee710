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
// Streaming: the work is cut into units of 32 rows x 256 channels (a strip of
// channels; rows counted from the start of each selected row segment), ordered
// matrix, strip, segment, row box.  One persistent CTA per SM takes a
// contiguous range of units; its producer warp brings each unit into an
// 8-slot shared-memory ring with a TMA tensor load (a constant 128 KB in
// flight per SM), its 8 consumer warps keep a running max per channel of the
// current strip and merge it into the outputs (integer atomicMax on the fp32
// bit patterns: exact, order independent) whenever the strip changes.
//
// Completion without scratch memory: the first lambda word of each strip
// counts, for the duration of the call, the merges into that strip; the CTA
// whose merge is the strip's last (the number of merges follows from the unit
// ranges) forms lambda and 1/lambda for the strip's 256 channels.  The strip
// maxima of RN(ax / lambda) / 2688 meet in the bits of the s_g output
// (atomicMax; division by 2688 is monotonic, so the max of the quotients is
// the quotient of the max), and lambda[1] counts finished strips; the last
// strip writes the final s_g (1 when every maximum is 0) and lambda[1].  So the
// call is two launches: a zeroing kernel and the reduction.  The reduction is a
// programmatic dependent of the zeroing kernel: its loads of X and W start while
// the zeroing runs, and its consumers wait for it (griddepcontrol.wait) before
// their first write to the outputs.
#include "common.cuh"
#include "sm100.cuh"

namespace svdq {
namespace {

constexpr int kStripCols = 256;               // channels per unit (512 bytes per row)
constexpr int kBoxRows = 32;                  // rows per unit
constexpr int kSlots = 8;                     // ring slots of 16 KB
constexpr int kConsumerWarps = 8;             // 4 rows of each unit per warp
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;     // + producer warp
constexpr uint32_t kUnitBytes = kBoxRows * kStripCols * 2;   // 16 KB
constexpr uint32_t kSmemBytes = kSlots * kUnitBytes + 256;

struct CalibArgs {
    SegTable segs;                            // row selection of X
    int64_t box_prefix[kMaxSegments + 1];     // row boxes before segment s (X)
    int64_t boxes[2];                         // row boxes per strip: X (all segments), W
    int64_t units[2];                         // strips * boxes
    int64_t n_units;                          // units[0] + units[1]
    int64_t N;                                // rows of W
    int64_t K;
    int64_t strips;
    uint32_t* out_bits[2];                    // absmax of X, of W (fp32 bit patterns)
    const float* ax;
    const float* aw;                          // nullptr when there is no weight
    float* lambda;
    float* inv_lambda;
    float* s_g;                               // holds max(strip maxima) until the last strip writes the scale
    uint32_t* err;
    int64_t ext_amax, ext_lambda;             // store-check extents (debug library): K each
    // Time-out test (armed from the host, one call): CTA 0's producer leaves its
    // ring unit `skip_unit` unloaded, so a consumer's wait for it runs out after
    // `wait_limit` cycles; -1 = off.  Every other CTA and call runs normally.
    int64_t skip_unit;
    long long wait_limit;
};

__global__ void __launch_bounds__(256)
calib_zero_kernel(float* ax, float* aw, int64_t K, float* lambda, float* s_g, int64_t ext, uint32_t* err) {
    pdl_launch_dependents();                  // the reduction may start streaming at once
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < K; j += stride) {
        if (!store_ok(j, 1, ext, err, kSiteCalibZero)) continue;
        ax[j] = 0.0f;
        if (aw) aw[j] = 0.0f;
        if (j % kStripCols == 0 || j == 1) lambda[j] = 0.0f;   // strip counters, strips-done counter
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) *reinterpret_cast<uint32_t*>(s_g) = 0u;
}

__device__ __forceinline__ void consumers_sync() {
    asm volatile("bar.sync 1, %0;" :: "n"(kConsumers) : "memory");
}

__device__ __forceinline__ float lambda_of(float x, const float* aw, int64_t j) {
    if (aw == nullptr) return 1.0f;
    const float w = __ldcg(aw + j);
    return (x > 0.0f && w > 0.0f) ? __fsqrt_rn(__fdiv_rn(x, w)) : 1.0f;
}

// By the consumer threads of the CTA that made a strip's last merge:
// lambda_j = sqrt(ax_j / aw_j) (1 where either absmax is 0) and 1/lambda_j for
// the strip's channels, then the strip's share of s_g = max_j(ax_j / lambda_j) / (6 * 448).
__device__ void strip_lambda(const CalibArgs& a, int64_t strip) {
    __shared__ float red[kConsumerWarps];
    const int64_t j = strip * kStripCols + threadIdx.x;
    float v = 0.0f;
    if (j < a.K) {
        const float x = __ldcg(a.ax + j);
        const float lam = lambda_of(x, a.aw, j);
        const float il = __frcp_rn(lam);
        if (store_ok(j, 1, a.ext_lambda, a.err, kSiteCalibLambda)) {
            if (j != 1) a.lambda[j] = lam;      // lambda[1] is the strips-done counter until the end
            if (a.inv_lambda) a.inv_lambda[j] = il;
        }
        v = __fmul_rn(x, il);
    }
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    consumers_sync();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kConsumerWarps; ++w) v = fmaxf(v, red[w]);
        const float q = __fdiv_rn(v, 2688.0f);
        if (q > 0.0f) atomicMax(reinterpret_cast<uint32_t*>(a.s_g), __float_as_uint(q));
        __threadfence();
        const uint32_t done = atomicAdd(reinterpret_cast<uint32_t*>(a.lambda + 1), 1u);
        if (done == static_cast<uint32_t>(a.strips) - 1) {
            __threadfence();
            const float m = __uint_as_float(atomicAdd(reinterpret_cast<uint32_t*>(a.s_g), 0u));
            const float x1 = __ldcg(a.ax + 1);
            a.lambda[1] = lambda_of(x1, a.aw, 1);
            *a.s_g = m > 0.0f ? m : 1.0f;
        }
    }
    consumers_sync();
}

// CTA that owns unit u when n units are split into g contiguous ranges
// [i n / g, (i + 1) n / g).
__device__ __forceinline__ int64_t unit_owner(int64_t u, int64_t g, int64_t n) {
    return ((u + 1) * g - 1) / n;
}

// Merges a strip receives: one per CTA whose range meets the strip's units of a matrix.
__device__ int64_t strip_merges(const CalibArgs& a, int64_t strip, int64_t g) {
    int64_t m = 0;
    int64_t base = 0;
    for (int j = 0; j < 2; ++j) {
        if (a.boxes[j] > 0) {
            const int64_t first = base + strip * a.boxes[j];
            const int64_t last = first + a.boxes[j] - 1;
            m += unit_owner(last, g, a.n_units) - unit_owner(first, g, a.n_units) + 1;
        }
        base += a.units[j];
    }
    return m;
}

__global__ void __launch_bounds__(kThreads, 1)
calib_stream_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                    const __grid_constant__ CalibArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kSlots * kUnitBytes);
    uint64_t* empty = full + kSlots;
    uint32_t* meta = reinterpret_cast<uint32_t*>(empty + kSlots);          // per slot: strip, matrix, rows
    volatile uint32_t* abort_flag = meta + kSlots;
    __shared__ uint32_t red[kConsumerWarps][32][4];
    __shared__ uint32_t is_last;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t G = gridDim.x;
    const int64_t g = blockIdx.x;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kSlots; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    pdl_launch_dependents();                  // the quantiser's set-up may overlap this kernel

    if (a.n_units == 0) {
        // No rows selected and no weight: one CTA per strip forms lambda = 1.
        pdl_wait();
        if (warp < kConsumerWarps) strip_lambda(a, g);
        return;
    }
    const int64_t u_begin = g * a.n_units / G;
    const int64_t u_end = (g + 1) * a.n_units / G;
    const int64_t skip = g == 0 ? a.skip_unit : -1;
    const long long limit = skip >= 0 ? a.wait_limit : kWaitLimitCycles;

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tmap_x);
            if (a.units[1] > 0) prefetch_tmap(&tmap_w);
            int i = 0;
            for (int64_t u = u_begin; u < u_end; ++u, ++i) {
                const int s = i % kSlots;
                const uint32_t ph = (i / kSlots) & 1;
                if (!mbar_wait_limit(&empty[s], ph ^ 1, abort_flag, a.err, kErrWaitEmpty, limit)) break;
                if (i == skip) continue;              // time-out test: this unit never arrives
                const int job = u < a.units[0] ? 0 : 1;
                const int64_t local = job ? u - a.units[0] : u;
                const int64_t strip = local / a.boxes[job];
                const int64_t b = local % a.boxes[job];
                int64_t row0, valid;
                if (job == 0) {
                    int seg = 0;
                    while (seg + 1 < a.segs.n && b >= a.box_prefix[seg + 1]) ++seg;
                    const int64_t in_seg = (b - a.box_prefix[seg]) * kBoxRows;
                    row0 = a.segs.begin[seg] + in_seg;
                    valid = min(static_cast<int64_t>(kBoxRows), a.segs.prefix[seg + 1] - a.segs.prefix[seg] - in_seg);
                } else {
                    row0 = b * kBoxRows;
                    valid = min(static_cast<int64_t>(kBoxRows), a.N - row0);
                }
                meta[s] = (static_cast<uint32_t>(strip) << 8) | (static_cast<uint32_t>(job) << 7) |
                          static_cast<uint32_t>(valid);
                mbar_arrive_expect_tx(&full[s], kUnitBytes);
                tma_load_2d(smem + s * kUnitBytes, job ? &tmap_w : &tmap_x, &full[s],
                            static_cast<int32_t>(strip * kStripCols), static_cast<int32_t>(row0));
            }
            for (int j = (i > kSlots ? i - kSlots : 0); j < i; ++j) {   // bounded drain
                if (j == skip) continue;
                const long long t0 = clock64();
                while (!mbar_try_wait(&full[j % kSlots], (j / kSlots) & 1) && clock64() - t0 < kWaitLimitCycles) {}
            }
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    pdl_wait();                               // the zeroing kernel's writes are complete and visible
    uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;
    int64_t cur = -1;                          // (strip << 1) | matrix of the running maxima
    auto merge = [&](int64_t key) {
        const int job = static_cast<int>(key & 1);
        const int64_t strip = key >> 1;
        red[warp][lane][0] = m0;
        red[warp][lane][1] = m1;
        red[warp][lane][2] = m2;
        red[warp][lane][3] = m3;
        m0 = m1 = m2 = m3 = 0;
        consumers_sync();
        {
            // thread t owns channel t of the strip
            const int t = threadIdx.x;
            const int src_lane = t / 8, word = (t % 8) / 2, hi = t & 1;
            uint32_t m = 0;
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) m = max(m, (red[w][src_lane][word] >> (16 * hi)) & 0xFFFFu);
            const int64_t col = strip * kStripCols + t;
            if (m != 0 && col < a.K && store_ok(col, 1, a.ext_amax, a.err, kSiteCalibAmax))
                atomicMax(a.out_bits[job] + col, m << 16);   // bf16 -> fp32 bits
        }
        __threadfence();
        consumers_sync();
        if (threadIdx.x == 0) {
            is_last = 0u;
            if (store_ok(strip * kStripCols, 1, a.ext_lambda, a.err, kSiteCalibLambda)) {
                const uint32_t prev = atomicAdd(reinterpret_cast<uint32_t*>(a.lambda + strip * kStripCols), 1u);
                is_last = (static_cast<int64_t>(prev) == strip_merges(a, strip, G) - 1) ? 1u : 0u;
            }
        }
        consumers_sync();
        if (is_last) {
            __threadfence();
            strip_lambda(a, strip);
        }
    };
    int i = 0;
    for (int64_t u = u_begin; u < u_end; ++u, ++i) {
        const int s = i % kSlots;
        const uint32_t ph = (i / kSlots) & 1;
        if (!mbar_wait_limit(&full[s], ph, abort_flag, a.err, kErrWaitFull, limit)) break;
        const uint32_t md = meta[s];
        const int64_t key = (static_cast<int64_t>(md >> 8) << 1) | ((md >> 7) & 1);
        const int valid = static_cast<int>(md & 0x7Fu);
        if (key != cur) {                      // the same decision in every consumer warp
            if (cur >= 0) merge(cur);
            cur = key;
        }
        const uint8_t* tile = smem + s * kUnitBytes;
#pragma unroll
        for (int rr = 0; rr < kBoxRows / kConsumerWarps; ++rr) {
            const int r = warp * (kBoxRows / kConsumerWarps) + rr;
            if (r < valid) {
                const uint4 q = *reinterpret_cast<const uint4*>(tile + r * (kStripCols * 2) + lane * 16);
                m0 = __vmaxu2(m0, q.x & 0x7FFF7FFFu);
                m1 = __vmaxu2(m1, q.y & 0x7FFF7FFFu);
                m2 = __vmaxu2(m2, q.z & 0x7FFF7FFFu);
                m3 = __vmaxu2(m3, q.w & 0x7FFF7FFFu);
            }
        }
        consumed(m0, m1, m2, m3);                     // the unit's loads are in these maxima
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (cur >= 0) merge(cur);
}

// One-shot time-out test arming (see svdq_debug_arm_calib_timeout).
std::atomic<long long> g_arm_skip{-1};
std::atomic<long long> g_arm_limit{0};

}  // namespace
}  // namespace svdq

extern "C" int svdq_debug_arm_calib_timeout(int64_t unit, int64_t wait_limit_cycles) {
    if (unit < 0 || wait_limit_cycles < 100000) return SVDQ_ERR_INVALID_ARG;
    svdq::g_arm_limit.store(wait_limit_cycles);
    svdq::g_arm_skip.store(unit);
    return SVDQ_OK;
}

namespace svdq {
namespace {

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

    a.K = K;
    a.N = W != nullptr ? N : 0;
    a.strips = (K + kStripCols - 1) / kStripCols;
    a.box_prefix[0] = 0;
    for (int s = 0; s < a.segs.n; ++s) {
        const int64_t rows = a.segs.prefix[s + 1] - a.segs.prefix[s];
        a.box_prefix[s + 1] = a.box_prefix[s] + (rows + kBoxRows - 1) / kBoxRows;
    }
    a.boxes[0] = a.box_prefix[a.segs.n];
    a.boxes[1] = (a.N + kBoxRows - 1) / kBoxRows;
    a.units[0] = a.strips * a.boxes[0];
    a.units[1] = a.strips * a.boxes[1];
    a.n_units = a.units[0] + a.units[1];
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
    a.skip_unit = g_arm_skip.exchange(-1);       // armed by the time-out test for this one call
    a.wait_limit = a.skip_unit >= 0 ? g_arm_limit.load() : kWaitLimitCycles;
    if (a.strips >= (int64_t(1) << 24)) return SVDQ_ERR_UNSUPPORTED;
    const int64_t grid = a.n_units == 0 ? a.strips : (a.n_units < sms ? a.n_units : sms);

    CUtensorMap tx, tw;
    if (!encode_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, K, M, ldx * 2, kStripCols, kBoxRows,
                        CU_TENSOR_MAP_SWIZZLE_NONE))
        return SVDQ_ERR_CUDA;
    tw = tx;
    if (W != nullptr && !encode_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W, K, N, ldw * 2, kStripCols,
                                        kBoxRows, CU_TENSOR_MAP_SWIZZLE_NONE))
        return SVDQ_ERR_CUDA;

    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const int64_t zb = (K + 255) / 256;
    // the stored weight absmax is an input: only the outputs are zeroed
    calib_zero_kernel<<<static_cast<unsigned>(zb < sms ? zb : sms), 256, 0, cs>>>(
        amax_x, W != nullptr ? amax_w : nullptr, K, lambda, s_g, debug_extent(kSiteCalibZero, K), err);
    st = launch_status(cudaGetLastError());
    if (st != SVDQ_OK) return st;
    const uint32_t smem = kSmemBytes + 1024;
    static std::atomic<uint64_t> smem_set{0};
    if (!set_dynamic_smem_once(calib_stream_kernel, smem, smem_set)) return SVDQ_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = cs;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return launch_status(cudaLaunchKernelEx(&cfg, calib_stream_kernel, tx, tw, a));
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
