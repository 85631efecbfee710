// score.cu -- per-segment relative L2 error of a quantised layer output
// against the bf16 layer ("MiniMax-H3 NVFP4 -- what the smoothing scale should
// be calibrated on", section "The metric that picks the winner also hides the
// cost": candidates scored by rel-L2 vs bf16 on proportional rows and on 4096
// rows per modality).
//
// Bandwidth-bound two-pass reduction with a fixed order, so results are
// bitwise reproducible: pass 1 writes one fp64 partial sum per (segment,
// 16384-element chunk) to the caller's workspace; pass 2 sums each segment's
// partials in index order and forms num, den and rel.  Pass 1 has two forms
// that reduce a chunk with the same thread mapping and tree, so they agree bit
// for bit: rows stored back to back stream through persistent CTAs (a producer
// warp bulk-copies whole chunks into a shared-memory ring, eight consumer warps
// reduce them, a grid barrier, then the final sums); strided rows take one block
// per chunk with 8 independent 16-byte loads per thread and input in flight.
#include <mutex>

#include <cooperative_groups.h>

#include "common.cuh"
#include "sm100.cuh"

namespace svdq {
namespace {

constexpr int kThreads = 256;
constexpr int kVecPerThread = 8;                    // 16-byte vectors of each input per thread
constexpr int64_t kElemsPerChunk = int64_t(kThreads) * kVecPerThread * 8;   // 16384 elements per block

// Segment s covers the flat element range [0, rows_s * N) of its rows; block
// `chunk` sums elements [c * kElemsPerChunk, (c + 1) * kElemsPerChunk) of one segment.
struct ChunkPlan {
    int n;                                           // segments
    int64_t begin[kMaxSegments];                     // first row of segment s
    int64_t elems[kMaxSegments];                     // rows_s * N
    int64_t chunk_prefix[kMaxSegments + 1];          // first chunk index of segment s
};

inline void make_plan(const svdq_seg* segs, int n_seg, int64_t N, ChunkPlan* p) {
    p->n = n_seg;
    p->chunk_prefix[0] = 0;
    for (int s = 0; s < n_seg; ++s) {
        p->begin[s] = segs[s].begin;
        p->elems[s] = (segs[s].end - segs[s].begin) * N;
        const int64_t chunks = p->elems[s] > 0 ? (p->elems[s] + kElemsPerChunk - 1) / kElemsPerChunk : 1;
        p->chunk_prefix[s + 1] = p->chunk_prefix[s] + chunks;
    }
}

__device__ __forceinline__ double block_sum(double v, double* sh) {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) sh[w] = v;
    __syncthreads();
    v = (threadIdx.x < (kThreads >> 5)) ? sh[threadIdx.x] : 0.0;
    if (w == 0)
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;   // valid in thread 0
}

// Eight element pairs: differences and squares in fp32 (the difference of two
// bf16 values and its square carry at most a 2^-24 relative rounding each), the
// 8-term partial sums are added to the fp64 accumulators.
__device__ __forceinline__ void accum8(const uint4& qa, const uint4& qb, double& num, double& den) {
    const uint32_t wa[4] = {qa.x, qa.y, qa.z, qa.w};
    const uint32_t wb[4] = {qb.x, qb.y, qb.z, qb.w};
    float n8 = 0.0f, d8 = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float r_lo = bf16_lo(wb[i]), r_hi = bf16_hi(wb[i]);
        const float e_lo = __fsub_rn(bf16_lo(wa[i]), r_lo);
        const float e_hi = __fsub_rn(bf16_hi(wa[i]), r_hi);
        n8 = __fmaf_rn(e_lo, e_lo, n8);
        n8 = __fmaf_rn(e_hi, e_hi, n8);
        d8 = __fmaf_rn(r_lo, r_lo, d8);
        d8 = __fmaf_rn(r_hi, r_hi, d8);
    }
    num += static_cast<double>(n8);
    den += static_cast<double>(d8);
}

__global__ void __launch_bounds__(kThreads)
score_partial_kernel(const uint16_t* __restrict__ yq, const uint16_t* __restrict__ yr, int64_t N, int64_t ld,
                     ChunkPlan plan, double* __restrict__ partial, int64_t ext_part, uint32_t* err) {
    __shared__ double sh[kThreads / 32];
    const int64_t chunk = blockIdx.x;
    int s = 0;
    while (s + 1 < plan.n && chunk >= plan.chunk_prefix[s + 1]) ++s;
    const int64_t e0 = (chunk - plan.chunk_prefix[s]) * kElemsPerChunk;
    const int64_t e1 = min(e0 + kElemsPerChunk, plan.elems[s]);
    const uint16_t* qa = yq + plan.begin[s] * ld;
    const uint16_t* qb = yr + plan.begin[s] * ld;
    double num = 0.0, den = 0.0;
    if (N % 8 == 0) {
        // 16-byte vectors; a vector never straddles a row because N % 8 == 0.
        uint4 va[kVecPerThread], vb[kVecPerThread];
#pragma unroll
        for (int i = 0; i < kVecPerThread; ++i) {
            const int64_t e = e0 + (static_cast<int64_t>(i) * kThreads + threadIdx.x) * 8;
            if (e < e1) {
                const int64_t off = (ld == N) ? e : (e / N) * ld + (e % N);   // contiguous rows: no division
                va[i] = __ldg(reinterpret_cast<const uint4*>(qa + off));
                vb[i] = __ldg(reinterpret_cast<const uint4*>(qb + off));
            } else {
                va[i] = make_uint4(0, 0, 0, 0);
                vb[i] = make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int i = 0; i < kVecPerThread; ++i) accum8(va[i], vb[i], num, den);
    } else {
        for (int64_t e = e0 + threadIdx.x; e < e1; e += kThreads) {
            const int64_t off = (ld == N) ? e : (e / N) * ld + (e % N);
            const float r = __uint_as_float(static_cast<uint32_t>(qb[off]) << 16);
            const float d = __fsub_rn(__uint_as_float(static_cast<uint32_t>(qa[off]) << 16), r);
            num += static_cast<double>(__fmul_rn(d, d));
            den += static_cast<double>(__fmul_rn(r, r));
        }
    }
    num = block_sum(num, sh);
    den = block_sum(den, sh);
    if (threadIdx.x == 0 && store_ok(2 * chunk, 2, ext_part, err, kSiteScorePart)) {
        partial[2 * chunk] = num;
        partial[2 * chunk + 1] = den;
    }
}

__global__ void __launch_bounds__(kThreads)
score_finalize_kernel(ChunkPlan plan, const double* __restrict__ partial, double* __restrict__ num_out,
                      double* __restrict__ den_out, double* __restrict__ rel_out, int64_t ext_out, uint32_t* err) {
    __shared__ double sh[kThreads / 32];
    const int s = blockIdx.x;
    double num = 0.0, den = 0.0;
    for (int64_t c = plan.chunk_prefix[s] + threadIdx.x; c < plan.chunk_prefix[s + 1]; c += kThreads) {
        num += partial[2 * c];
        den += partial[2 * c + 1];
    }
    num = block_sum(num, sh);
    den = block_sum(den, sh);
    if (threadIdx.x == 0 && store_ok(s, 1, ext_out, err, kSiteScoreOut)) {
        num_out[s] = num;
        den_out[s] = den;
        double rel;
        if (den > 0.0) rel = sqrt(num / den);
        else rel = (num == 0.0) ? 0.0 : __longlong_as_double(0x7FF0000000000000LL);
        rel_out[s] = rel;
    }
}

// ---------------------------------------------------------------------------
// Streaming version for rows stored back to back (ld == N, N % 8 == 0): every
// chunk is one contiguous run of 2 x 32 KB, so a producer warp copies whole
// chunks with bulk copies into a 3-slot shared-memory ring (192 KB in flight
// per SM) while 8 consumer warps reduce earlier chunks.  One persistent CTA
// per SM takes chunks c = blockIdx.x, blockIdx.x + gridDim.x, ... so the CTAs
// together stream through memory in order.  Each chunk is reduced by the same
// thread mapping and the same reduction tree as score_partial_kernel: the
// partial sums are bitwise the same.
// ---------------------------------------------------------------------------
constexpr int kStreamSlots = 3;
constexpr int kStreamConsumerWarps = kThreads / 32;            // 8
constexpr int kStreamThreads = kThreads + 32;                  // + producer warp
constexpr uint32_t kChunkBytes = kElemsPerChunk * 2;           // 32 KB per input
constexpr uint32_t kStreamSmem = kStreamSlots * 2 * kChunkBytes + 256;

__device__ __forceinline__ double consumer_sum(double v, double* sh) {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    asm volatile("bar.sync 1, %0;" :: "n"(kThreads) : "memory");
    if (l == 0) sh[w] = v;
    asm volatile("bar.sync 1, %0;" :: "n"(kThreads) : "memory");
    v = (threadIdx.x < (kThreads >> 5)) ? sh[threadIdx.x] : 0.0;
    if (w == 0)
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;   // valid in thread 0
}

__device__ __forceinline__ void consumers_sync_all() {
    asm volatile("bar.sync 1, %0;" :: "n"(kThreads) : "memory");
}

__global__ void __launch_bounds__(kStreamThreads, 1)
score_stream_kernel(const uint16_t* __restrict__ yq, const uint16_t* __restrict__ yr, int64_t N,
                    const __grid_constant__ ChunkPlan plan, int64_t n_chunks, double* __restrict__ partial,
                    double* __restrict__ num_out, double* __restrict__ den_out, double* __restrict__ rel_out,
                    uint32_t* err, int64_t ext_part, int64_t ext_out, int64_t skip_chunk, long long wait_limit) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStreamSlots * 2 * kChunkBytes);
    uint64_t* empty = full + kStreamSlots;
    uint32_t* n_elems = reinterpret_cast<uint32_t*>(empty + kStreamSlots);    // per slot
    volatile uint32_t* abort_flag = n_elems + kStreamSlots;
    __shared__ double sh[kThreads / 32];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // Time-out test (armed from the host, one call): CTA 0's producer leaves its
    // chunk number `skip_chunk` uncopied and the CTA's waits give up after
    // `wait_limit` cycles; -1 = off.
    const int64_t skip = blockIdx.x == 0 ? skip_chunk : -1;
    const long long limit = skip >= 0 ? wait_limit : kWaitLimitCycles;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStreamSlots; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kStreamConsumerWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kStreamConsumerWarps) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int i = 0;
            int seg = 0;
            for (int64_t c = blockIdx.x; c < n_chunks; c += gridDim.x, ++i) {
                const int s = i % kStreamSlots;
                const uint32_t ph = (i / kStreamSlots) & 1;
                if (!mbar_wait_limit(&empty[s], ph ^ 1, abort_flag, err, kErrWaitEmpty, limit)) break;
                if (i == skip) continue;              // time-out test: this chunk never arrives
                while (seg + 1 < plan.n && c >= plan.chunk_prefix[seg + 1]) ++seg;   // c increases
                const int64_t e0 = (c - plan.chunk_prefix[seg]) * kElemsPerChunk;
                const int64_t e1 = min(e0 + kElemsPerChunk, plan.elems[seg]);
                const uint32_t n = e1 > e0 ? static_cast<uint32_t>(e1 - e0) : 0u;
                n_elems[s] = n;
                mbar_arrive_expect_tx(&full[s], 4u * n);
                if (n) {
                    const int64_t off = plan.begin[seg] * N + e0;
                    uint8_t* dst = smem + s * 2 * kChunkBytes;
                    bulk_load(dst, yq + off, 2u * n, &full[s]);
                    bulk_load(dst + kChunkBytes, yr + off, 2u * n, &full[s]);
                }
            }
            for (int j = (i > kStreamSlots ? i - kStreamSlots : 0); j < i; ++j) {   // bounded drain
                if (j == skip) continue;
                const long long t0 = clock64();
                while (!mbar_try_wait(&full[j % kStreamSlots], (j / kStreamSlots) & 1) &&
                       clock64() - t0 < kWaitLimitCycles) {}
            }
        }
    } else {
        // ------------------------------------------------------------ consumers
        int i = 0;
        for (int64_t c = blockIdx.x; c < n_chunks; c += gridDim.x, ++i) {
            const int s = i % kStreamSlots;
            const uint32_t ph = (i / kStreamSlots) & 1;
            if (!mbar_wait_limit(&full[s], ph, abort_flag, err, kErrWaitFull, limit)) break;
            const uint32_t n = n_elems[s];
            const uint8_t* qa = smem + s * 2 * kChunkBytes;
            const uint8_t* qb = qa + kChunkBytes;
            uint4 va[kVecPerThread], vb[kVecPerThread];
#pragma unroll
            for (int v = 0; v < kVecPerThread; ++v) {
                const uint32_t e = (static_cast<uint32_t>(v) * kThreads + threadIdx.x) * 8;
                if (e < n) {
                    va[v] = *reinterpret_cast<const uint4*>(qa + 2 * e);
                    vb[v] = *reinterpret_cast<const uint4*>(qb + 2 * e);
                } else {
                    va[v] = make_uint4(0, 0, 0, 0);
                    vb[v] = make_uint4(0, 0, 0, 0);
                }
            }
            double num = 0.0, den = 0.0;
#pragma unroll
            for (int v = 0; v < kVecPerThread; ++v) accum8(va[v], vb[v], num, den);
            num = consumer_sum(num, sh);
            den = consumer_sum(den, sh);
            // The slot is released once the loaded values have been used (the
            // shuffles of the sums read them): a release with shared-memory loads
            // still in flight could let the next copy land under them.
            if (lane == 0) mbar_arrive(&empty[s]);
            if (threadIdx.x == 0 && store_ok(2 * c, 2, ext_part, err, kSiteScorePart)) {
                partial[2 * c] = num;
                partial[2 * c + 1] = den;
            }
        }
    }

    // Every chunk's partial is written: CTA s sums segment s's partials in index
    // order, with the same tree as score_finalize_kernel (the launch is
    // cooperative, so all CTAs are resident and the grid barrier is safe).
    cooperative_groups::this_grid().sync();
    if (warp < kStreamConsumerWarps) {
        for (int s = blockIdx.x; s < plan.n; s += gridDim.x) {
            double num = 0.0, den = 0.0;
            for (int64_t c = plan.chunk_prefix[s] + threadIdx.x; c < plan.chunk_prefix[s + 1]; c += kThreads) {
                num += __ldcg(partial + 2 * c);
                den += __ldcg(partial + 2 * c + 1);
            }
            num = consumer_sum(num, sh);
            den = consumer_sum(den, sh);
            if (threadIdx.x == 0 && store_ok(s, 1, ext_out, err, kSiteScoreOut)) {
                num_out[s] = num;
                den_out[s] = den;
                double rel;
                if (den > 0.0) rel = sqrt(num / den);
                else rel = (num == 0.0) ? 0.0 : __longlong_as_double(0x7FF0000000000000LL);
                rel_out[s] = rel;
            }
            consumers_sync_all();
        }
    }
}

}  // namespace

// One-shot time-out test arming (see svdq_debug_arm_score_timeout).
std::atomic<long long> g_arm_skip{-1};
std::atomic<long long> g_arm_limit{0};

// Shared by the entry point below; `partial` must hold 2 doubles per chunk.
int score_lambda_launch(const void* Yq, const void* Yref, int64_t M, int64_t N, int64_t ld,
                        const svdq_seg* segs, int n_seg, double* num, double* den, double* rel,
                        double* partial, size_t partial_bytes, cudaStream_t cs) {
    ChunkPlan plan;
    make_plan(segs, n_seg, N, &plan);
    const int64_t chunks = plan.chunk_prefix[n_seg];
    if (partial_bytes < static_cast<size_t>(chunks) * 2 * sizeof(double)) return SVDQ_ERR_INVALID_ARG;
    if (chunks > 0x7FFFFFFF) return SVDQ_ERR_UNSUPPORTED;
    if (!debug_ptrs_ok({Yq, Yref, num, den, rel, partial})) return SVDQ_ERR_INVALID_ARG;
    uint32_t* err = device_error_word();
    if (err == nullptr) return SVDQ_ERR_CUDA;
    const int64_t ext_part = debug_extent(kSiteScorePart, static_cast<int64_t>(partial_bytes / sizeof(double)));
    const int64_t ext_out = debug_extent(kSiteScoreOut, n_seg);
    if (ld == N && N % 8 == 0) {
        static std::atomic<uint64_t> smem_set{0};
        if (!set_dynamic_smem_once(score_stream_kernel, kStreamSmem, smem_set)) return SVDQ_ERR_CUDA;
        // cooperative: never more CTAs than can be resident together
        const int64_t resident = coresident_grid(score_stream_kernel, kStreamThreads, kStreamSmem);
        if (resident < 1) return SVDQ_ERR_CUDA;
        const int64_t sms = device_sm_count() > 0 ? device_sm_count() : 148;
        int64_t grid = chunks < sms ? chunks : sms;
        if (grid > resident) grid = resident;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
        cfg.blockDim = dim3(kStreamThreads, 1, 1);
        cfg.dynamicSmemBytes = kStreamSmem;
        cfg.stream = cs;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        const int64_t skip = g_arm_skip.exchange(-1);     // armed by the time-out test for this one call
        const long long limit = skip >= 0 ? g_arm_limit.load() : kWaitLimitCycles;
        return launch_status(cudaLaunchKernelEx(&cfg, score_stream_kernel, static_cast<const uint16_t*>(Yq),
                                                static_cast<const uint16_t*>(Yref), N, plan, chunks, partial, num,
                                                den, rel, err, ext_part, ext_out, skip, limit));
    } else {
        score_partial_kernel<<<static_cast<unsigned>(chunks), kThreads, 0, cs>>>(
            static_cast<const uint16_t*>(Yq), static_cast<const uint16_t*>(Yref), N, ld, plan, partial, ext_part, err);
    }
    if (cudaGetLastError() != cudaSuccess) return SVDQ_ERR_CUDA;
    score_finalize_kernel<<<n_seg, kThreads, 0, cs>>>(plan, partial, num, den, rel, ext_out, err);
    return launch_status(cudaGetLastError());
}

int score_lambda_check(const void* Yq, const void* Yref, int64_t M, int64_t N, int64_t ld,
                       const svdq_seg* segs, int n_seg, const double* num, const double* den,
                       const double* rel) {
    if (Yq == nullptr || Yref == nullptr || num == nullptr || den == nullptr || rel == nullptr)
        return SVDQ_ERR_INVALID_ARG;
    if (segs == nullptr || n_seg < 1 || n_seg > kMaxSegments) return SVDQ_ERR_INVALID_ARG;
    if (M < 1 || N < 1 || ld < N) return SVDQ_ERR_INVALID_ARG;
    for (int s = 0; s < n_seg; ++s)
        if (segs[s].begin < 0 || segs[s].end < segs[s].begin || segs[s].end > M) return SVDQ_ERR_INVALID_ARG;
    if (!aligned16(Yq) || !aligned16(Yref) || (ld * 2) % 16 != 0) return SVDQ_ERR_MISALIGNED;
    return SVDQ_OK;
}

size_t score_partial_bytes(const svdq_seg* segs, int n_seg, int64_t N) {
    if (segs == nullptr || n_seg < 1 || n_seg > kMaxSegments || N < 1) return 0;
    int64_t chunks = 0;
    for (int s = 0; s < n_seg; ++s) {
        const int64_t elems = (segs[s].end - segs[s].begin) * N;
        chunks += elems > 0 ? (elems + kElemsPerChunk - 1) / kElemsPerChunk : 1;
    }
    return static_cast<size_t>(chunks) * 2 * sizeof(double);
}

}  // namespace svdq

extern "C" int svdq_debug_arm_score_timeout(int64_t chunk, int64_t wait_limit_cycles) {
    if (chunk < 0 || wait_limit_cycles < 100000) return SVDQ_ERR_INVALID_ARG;
    svdq::g_arm_limit.store(wait_limit_cycles);
    svdq::g_arm_skip.store(chunk);
    return SVDQ_OK;
}

extern "C" size_t svdq_score_workspace_bytes(const svdq_seg* segs, int n_seg, int64_t N) {
    const size_t b = svdq::score_partial_bytes(segs, n_seg, N);
    return b == 0 ? 0 : (b + 255) / 256 * 256;
}

extern "C" int svdq_score_lambda(const void* Yq, const void* Yref, int64_t M, int64_t N, int64_t ld,
                                 const svdq_seg* segs, int n_seg,
                                 double* num, double* den, double* rel,
                                 void* workspace, size_t workspace_bytes, void* stream) {
    using namespace svdq;
    int st = score_lambda_check(Yq, Yref, M, N, ld, segs, n_seg, num, den, rel);
    if (st != SVDQ_OK) return st;
    if (workspace == nullptr) return SVDQ_ERR_INVALID_ARG;
    if (!aligned16(workspace)) return SVDQ_ERR_MISALIGNED;
    if (!device_is_sm100()) return SVDQ_ERR_NO_DEVICE;
    return score_lambda_launch(Yq, Yref, M, N, ld, segs, n_seg, num, den, rel,
                               static_cast<double*>(workspace), workspace_bytes,
                               static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------
// Scoring without a caller workspace.
//
// Some callers cannot allocate device memory while they score: code running
// inside a framework's memory pool that forbids side allocations, a
// pre-recorded launch sequence whose buffers were fixed in advance, or a
// plugin host that hands out only input and output tensors.  For them the
// per-block partial sums live in a fixed array inside this library instead of
// a workspace argument.  The array is a __device__ variable, so every GPU that
// loads the library holds it (kStaticScoreBytes) until the process exits.
// ---------------------------------------------------------------------------
namespace svdq {
namespace {

constexpr size_t kStaticScoreBytes = size_t(1) << 20;   // 65536 partial-sum pairs

static __device__ __align__(256) double g_score_scratch[kStaticScoreBytes / sizeof(double)];

constexpr int kMaxDevicesStatic = 64;
double* g_score_scratch_ptr[kMaxDevicesStatic] = {};
std::mutex g_score_scratch_mutex;

// Host code may not hand the array's name to a kernel: on the host it is only a
// stand-in for the device variable.  Its device address is looked up once per
// device, with that device current.
double* static_scratch_for_current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevicesStatic) return nullptr;
    std::lock_guard<std::mutex> lock(g_score_scratch_mutex);
    if (g_score_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_score_scratch) != cudaSuccess || p == nullptr) return nullptr;
        g_score_scratch_ptr[dev] = static_cast<double*>(p);
    }
    return g_score_scratch_ptr[dev];
}

}  // namespace
}  // namespace svdq

extern "C" size_t svdq_score_static_max_bytes(void) { return svdq::kStaticScoreBytes; }

extern "C" int svdq_score_lambda_static(const void* Yq, const void* Yref, int64_t M, int64_t N, int64_t ld,
                                        const svdq_seg* segs, int n_seg,
                                        double* num, double* den, double* rel, void* stream) {
    using namespace svdq;
    int st = score_lambda_check(Yq, Yref, M, N, ld, segs, n_seg, num, den, rel);
    if (st != SVDQ_OK) return st;
    const size_t need = score_partial_bytes(segs, n_seg, N);
    if (need > kStaticScoreBytes) return SVDQ_ERR_SCRATCH_TOO_SMALL;
    if (!device_is_sm100()) return SVDQ_ERR_NO_DEVICE;
    double* scratch = static_scratch_for_current_device();
    if (scratch == nullptr) return SVDQ_ERR_CUDA;
    // Every partial-sum slot a call reads is written by the same call first, so
    // the previous call's contents need no clearing.
    return score_lambda_launch(Yq, Yref, M, N, ld, segs, n_seg, num, den, rel, scratch, kStaticScoreBytes,
                               static_cast<cudaStream_t>(stream));
}
