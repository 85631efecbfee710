// sm100.cuh -- thin wrappers over the sm_100a PTX this library uses:
// mbarriers, TMA (cp.async.bulk[.tensor]), and the tcgen05 tensor-core path
// (tensor-memory allocation, MMA issue, commit, shared->tensor-memory copy of
// block scales, tensor-memory loads).  Every wait is bounded.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

namespace svdq {

// ---------------------------------------------------------------------------
// Device error word (one per device; read by svdq_device_error on the host)
// ---------------------------------------------------------------------------
enum DevErr : uint32_t {
    kErrNone = 0,
    kErrWaitFull = 1,      // consumer waited too long for a TMA stage
    kErrWaitEmpty = 2,     // producer waited too long for a free stage
    kErrWaitAccum = 3,     // MMA issuer waited too long for the accumulator
    kErrWaitMma = 4,       // epilogue waited too long for the MMA result
    kErrWaitLowRank = 5,   // low-rank operand stage wait ran out
    kErrWaitRef = 6,       // scoring epilogue waited too long for a reference strip or its slot
};

// About 2-4 s of SM cycles at the clocks this part runs: far above any
// legitimate wait, short enough to return control on a lost arrival.
constexpr long long kWaitLimitCycles = 4000000000LL;

// ---------------------------------------------------------------------------
// Store checks of the debug library (compiled with SVDQ_DEBUG_CHECKS=1)
// ---------------------------------------------------------------------------
// Every plain global store of an output goes through store_ok(), and every TMA
// store's box origin through box_ok().  The extent is the output's documented
// size, computed on the host apart from the kernel's index arithmetic.  In the
// debug library a store outside it is skipped and kErrBounds + site goes into
// the error word (the first error wins), so the kernel runs on and the host
// reads SVDQ_ERR_BOUNDS.  In the release library both return true and compile
// away.
#ifndef SVDQ_DEBUG_CHECKS
#define SVDQ_DEBUG_CHECKS 0
#endif
constexpr uint32_t kErrBounds = 0x100u;
enum StoreSite : uint32_t {
    kSiteCalibZero = 1,       // calibration: zeroing of absmax, counters, scale
    kSiteCalibAmax = 2,       // calibration: per-channel absmax merge
    kSiteCalibLambda = 3,     // calibration: lambda, 1/lambda, strip counters, scale
    kSiteQuantCodes = 4,      // NVFP4 quantiser: packed codes
    kSiteQuantSf = 5,         // NVFP4 quantiser: swizzled scale bytes
    kSiteQuantD = 6,          // NVFP4 quantiser: low-rank down-projection D
    kSiteLinearBox = 7,       // linear: TMA store box origin of Y
    kSiteLinearF32 = 8,       // linear: fp32 output
    kSiteLinearScore = 9,     // fused scoring: per-CTA partials and the result
    kSiteScorePart = 10,      // scoring: per-CTA partial sums
    kSiteScoreOut = 11,       // scoring: num, den, rel
    kSiteResidual = 12,       // residual weight
    kSiteGrid = 13,           // lambda grid: lambda, 1/lambda, scale
    kSiteBits = 14,           // bits lost
    kSiteMxCodes = 15,        // MXFP8 quantiser: codes
    kSiteMxSf = 16,           // MXFP8 quantiser: scale bytes
    kSiteCount = 17
};

// A store of `width` elements at element offset `off` into an output of
// `extent` elements.
__device__ __forceinline__ bool store_ok(int64_t off, int64_t width, int64_t extent, uint32_t* err,
                                         uint32_t site) {
#if SVDQ_DEBUG_CHECKS
    if (off >= 0 && off + width <= extent) return true;
    atomicCAS(err, 0u, kErrBounds + site);
    return false;
#else
    (void)off; (void)width; (void)extent; (void)err; (void)site;
    return true;
#endif
}

// A TMA store box starting at (x, y) of a tensor of dims {dx, dy}: the origin
// must lie inside (the copy clips the far edges; a negative origin is not allowed).
__device__ __forceinline__ bool box_ok(int64_t x, int64_t y, int64_t dx, int64_t dy, uint32_t* err,
                                       uint32_t site) {
#if SVDQ_DEBUG_CHECKS
    if (x >= 0 && y >= 0 && x < dx && y < dy) return true;
    atomicCAS(err, 0u, kErrBounds + site);
    return false;
#else
    (void)x; (void)y; (void)dx; (void)dy; (void)err; (void)site;
    return true;
#endif
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t lane_id() {
    uint32_t l;
    asm volatile("mov.u32 %0, %%laneid;" : "=r"(l));
    return l;
}

// Streaming 16-byte global load: read-only path, no L1 allocation (the data
// is used once).
__device__ __forceinline__ uint4 ldg_stream_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 :: "r"(smem_u32(bar)), "r"(bytes) : "memory");
}

// A consumer's values computed from a shared-memory stage, tied in place
// before it releases the stage: the compiler may not sink their computation
// past this point, and since a warp issues in order and these instructions wait
// for the loads they read, the release below cannot be issued while a load of
// the stage is still in flight (the next copy into the stage could otherwise
// land under it).
__device__ __forceinline__ void consumed(uint32_t a, uint32_t b) { asm volatile("" :: "r"(a), "r"(b) : "memory"); }
__device__ __forceinline__ void consumed(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("" :: "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity to complete.  On timeout
// (`limit` cycles) it records `code` in the device error word, raises the
// CTA-wide abort flag (so the other roles stop waiting too) and returns false.
// It also returns false at once when another role already raised the abort flag.
__device__ __forceinline__ bool mbar_wait_limit(uint64_t* bar, uint32_t parity, volatile uint32_t* abort_flag,
                                                uint32_t* err_word, uint32_t code, long long limit) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long start = clock64();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - start > limit) {
            *abort_flag = 1u;
            atomicCAS(err_word, 0u, code);
            return false;
        }
    }
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile uint32_t* abort_flag,
                                          uint32_t* err_word, uint32_t code) {
    return mbar_wait_limit(bar, parity, abort_flag, err_word, code, kWaitLimitCycles);
}

// ---------------------------------------------------------------------------
// TMA and bulk copies (global -> shared, completion on an mbarrier)
// ---------------------------------------------------------------------------
// Named barrier `kId` over `kCount` threads that also returns the OR of `pred`
// over them: every participant takes the same decision from it.
template <int kId, int kCount>
__device__ __forceinline__ bool bar_sync_or(bool pred) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(out) : "r"(pred ? 1u : 0u), "n"(kId), "n"(kCount) : "memory");
    return out != 0u;
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" :: "l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];"
        :: "r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1),
           "r"(smem_u32(bar))
        : "memory");
}

// L2 policy for data read or written once: its lines are the first evicted, so
// a stream does not push out operands that other CTAs still re-read.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// L2 policy for data many CTAs re-read over the kernel's life: its lines are
// kept in preference to normal ones.
__device__ __forceinline__ uint64_t l2_evict_last_policy() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ void tma_load_2d_hint(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                                 int32_t c0, int32_t c1, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;"
        :: "r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1),
           "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// 3-D tensor load (box in the order of the map's dimensions) into shared memory.
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1, int32_t c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];"
        :: "r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2),
           "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_load_3d_hint(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                                 int32_t c0, int32_t c1, int32_t c2, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4}], [%5], %6;"
        :: "r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2),
           "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// Contiguous copy; both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        :: "r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// shared -> global tiled bulk store (TMA), tracked by the issuing thread's bulk group.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* smem_src, int32_t c0, int32_t c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
                 :: "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(smem_src)), "r"(c0), "r"(c1) : "memory");
}

__device__ __forceinline__ void tma_store_2d_hint(const CUtensorMap* map, const void* smem_src, int32_t c0, int32_t c1,
                                                  uint64_t policy) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group.L2::cache_hint [%0, {%2, %3}], [%1], %4;"
                 :: "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(smem_src)), "r"(c0), "r"(c1), "l"(policy)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit_group() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until every committed bulk store of this thread has finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read_all() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// Wait until every committed bulk store of this thread has completed.
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Make generic-proxy shared-memory writes visible to the async proxy (TMA / tensor core).
__device__ __forceinline__ void fence_async_shared() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory, MMA, commit, copies, loads
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_result, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32(smem_result)), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrive on `bar` once every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(smem_u32(bar)) : "memory");
}

// D(tmem) (+)= A(smem) * B(smem)^T, bf16 inputs, fp32 accumulation.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

// D(tmem) (+)= (A * SFA)(smem) * (B * SFB)(smem)^T, E2M1 inputs, one E4M3 scale
// per 16 elements (scales in tensor memory), fp32 accumulation.
__device__ __forceinline__ void mma_nvf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate),
           "r"(sfa_tmem), "r"(sfb_tmem) : "memory");
}

// Block-scaled FP8 MMA: kind::mxf8f6f4, one E8M0 scale per 32 elements
// (scale_vec::1X), K = 32 per instruction.  Each 32-bit tensor-memory scale word
// holds four scale bytes; the instruction descriptor's scale ids pick the byte.
__device__ __forceinline__ void mma_mxf8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale.scale_vec::1X [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate),
           "r"(sfa_tmem), "r"(sfb_tmem) : "memory");
}

// Copy a 32-row x 128-bit shared-memory block into tensor memory, replicated
// into all four 32-lane quarters (the layout block scales are read from).
__device__ __forceinline__ void tc_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" :: "r"(taddr), "l"(sdesc) : "memory");
}

// Each thread of the warp reads 32 consecutive 32-bit columns of its own lane.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// Each thread of the warp writes 16 consecutive 32-bit columns of its own lane.
__device__ __forceinline__ void tmem_st_32x32b_x1(uint32_t taddr, uint32_t r) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" :: "r"(taddr), "r"(r) : "memory");
}

__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
        :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
           "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

// Each thread of the warp writes 32 consecutive 32-bit columns of its own lane.
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
        :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
           "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
           "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
           "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// tcgen05.ld writes its destination registers asynchronously: they hold the
// loaded values only after tcgen05.wait::ld.  To the compiler the registers are
// ready as soon as the load's asm statement ends, so it may move their uses
// above a plain wait.  These waits also pass the registers through the asm
// statement ("+r"), so every use depends on the wait.  After one wait, further
// arrays loaded before it are tied with tmem_ld_tie (an empty asm, ordered
// after the wait as both are volatile).
__device__ __forceinline__ void tmem_ld_tie(uint32_t (&r)[32]) {
    asm volatile(""
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                   "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                   "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
}

__device__ __forceinline__ void tmem_ld_tie(uint32_t (&r)[16]) {
    asm volatile(""
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15])
                 :
                 : "memory");
}

template <int N>
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[N]) {
    tmem_ld_wait();
    tmem_ld_tie(r);
}

// ---------------------------------------------------------------------------
// Thread-block clusters
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Programmatic dependent launch.  The first kernel lets the next one in the
// stream (launched with programmatic stream serialization) start early; that
// kernel must wait for the first one's completion and memory before it touches
// anything the first one writes.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void pdl_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Full cluster barrier (every thread of every CTA of the cluster).
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Descriptors
// ---------------------------------------------------------------------------
// Shared-memory matrix descriptor, K-major operand in the 128-byte swizzle
// canonical layout: rows of 128 bytes, 8-row groups 1024 bytes apart.  The
// tile base must be 1024-byte aligned; stepping along K inside the 128-byte
// row adds the byte offset to the start address.
__device__ __forceinline__ uint64_t desc_kmajor_sw128(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);      // start address, bits [0,14)
    d |= static_cast<uint64_t>(1024u >> 4) << 32;                 // stride byte offset, bits [32,46)
    d |= static_cast<uint64_t>(1u) << 46;                         // descriptor version (sm_100)
    d |= static_cast<uint64_t>(2u) << 61;                         // layout: 128-byte swizzle
    return d;
}

// Descriptor of a plain (unswizzled) block of 32 rows x 16 bytes, rows
// contiguous, 8-row core matrices 128 bytes apart: the source of tc_cp_32x128b_x4.
__device__ __forceinline__ uint64_t desc_sf_block(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(128u >> 4) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    return d;
}

// Instruction descriptor, kind::f16 with bf16 A/B, fp32 D, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(uint32_t m, uint32_t n) {
    return (1u << 4)            // D format: f32
         | (1u << 7)            // A format: bf16
         | (1u << 10)           // B format: bf16
         | ((n >> 3) << 17)     // N / 8
         | ((m >> 4) << 24);    // M / 16
}

// Instruction descriptor, kind::mxf4nvf4 with E2M1 A/B, E4M3 block scales
// (one per 16 elements), both K-major, scale ids 0, K = 64 per instruction.
__host__ __device__ constexpr uint32_t idesc_nvf4(uint32_t m, uint32_t n) {
    return (1u << 7)            // A format: E2M1
         | (1u << 10)           // B format: E2M1
         | ((n >> 3) << 17)     // N / 8
         | (0u << 23)           // scale format: E4M3
         | ((m >> 4) << 24);    // M / 16
}

// Instruction descriptor, kind::mxf8f6f4 with E4M3 A/B and E8M0 block scales (one
// per 32 elements), both K-major, K = 32 per instruction; `sf_id` selects the
// byte of the A and B scale words this instruction uses.
__host__ __device__ constexpr uint32_t idesc_mxf8(uint32_t m, uint32_t n, uint32_t sf_id) {
    return (sf_id << 4)         // B scale factor id
         | (0u << 7)            // A format: E4M3
         | (0u << 10)           // B format: E4M3
         | ((n >> 3) << 17)     // N / 8
         | (1u << 23)           // scale format: E8M0
         | ((m >> 4) << 24)     // M / 16
         | (sf_id << 29);       // A scale factor id
}

// ---------------------------------------------------------------------------
// Conversions through the hardware round-to-nearest-even instructions
// ---------------------------------------------------------------------------
// Two fp32 -> two E2M1 codes in one byte; `lo` goes to the low nibble.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .b8 b;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b, %2, %1;\n\t"
        "cvt.u32.u8 %0, b;\n\t}"
        : "=r"(out) : "f"(lo), "f"(hi));
    return out;
}

// Eight fp32 -> eight E2M1 codes packed little-endian (element 0 in bits 0..3).
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float (&q)[8]) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(q[0]), "f"(q[1]), "f"(q[2]), "f"(q[3]), "f"(q[4]), "f"(q[5]), "f"(q[6]), "f"(q[7]));
    return out;
}

// Non-negative fp32 -> E4M3 byte (round to nearest even, saturate at 448).
__device__ __forceinline__ uint32_t cvt_e4m3(float t) {
    uint16_t out;
    asm volatile("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(out) : "f"(t), "f"(0.0f));
    return out & 0xFFu;
}

// E4M3 byte -> fp32 (exact: every E4M3 value is an fp16 value).
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
    uint32_t h2;
    const uint16_t in = static_cast<uint16_t>(b & 0xFFu);
    asm volatile("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    const uint16_t h = static_cast<uint16_t>(h2 & 0xFFFFu);
    float f;
    asm volatile("cvt.f32.f16 %0, %1;" : "=f"(f) : "h"(h));
    return f;
}


// ---------------------------------------------------------------------------
// Packed fp32 pairs (sm_100 f32x2 arithmetic: two IEEE round-to-nearest
// operations per instruction, identical results to two scalar ones)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ void unpack_f32x2(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// Two bf16 (low half = element 0) -> their exact fp32 values as a pair.
__device__ __forceinline__ uint64_t bf16x2_to_f32x2(uint32_t w) {
    return pack_f32x2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// max_j |x_j| over 16 values held as 8 pairs (balanced tree).
__device__ __forceinline__ float absmax16(const uint64_t (&x)[8]) {
    float m[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float lo, hi;
        unpack_f32x2(x[j], lo, hi);
        m[j] = fmaxf(fabsf(lo), fabsf(hi));
    }
    const float a = fmaxf(m[0], m[1]), b = fmaxf(m[2], m[3]), c = fmaxf(m[4], m[5]), e = fmaxf(m[6], m[7]);
    return fmaxf(fmaxf(a, b), fmaxf(c, e));
}

// Two non-negative fp32 -> two E4M3 bytes (RNE, saturating at 448): `lo` in
// bits 0..7, `hi` in bits 8..15.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
    uint16_t out;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(hi), "f"(lo));
    return out;
}

// Four fp32 pairs -> eight E2M1 codes, pair j in byte j, element 2j in its low nibble.
__device__ __forceinline__ uint32_t cvt_e2m1x8_pairs(uint64_t p0, uint64_t p1, uint64_t p2, uint64_t p3) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        ".reg .f32 l0, h0, l1, h1, l2, h2, l3, h3;\n\t"
        "mov.b64 {l0, h0}, %1;\n\t"
        "mov.b64 {l1, h1}, %2;\n\t"
        "mov.b64 {l2, h2}, %3;\n\t"
        "mov.b64 {l3, h3}, %4;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, h0, l0;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, h1, l1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, h2, l2;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, h3, l3;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out) : "l"(p0), "l"(p1), "l"(p2), "l"(p3));
    return out;
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

}  // namespace svdq
