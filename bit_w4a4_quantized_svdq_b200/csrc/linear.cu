// linear.cu -- the fused W4A4 linear: block-scaled NVFP4 GEMM on the tcgen05
// tensor cores with the low-rank up-projection, the tensor scales and the bias
// in the same accumulator / epilogue.
//
// "MiniMax-H3 . SVDQuant W4A4 (int4, rank 32, GPTQ)", opening section: 4-bit
// activations times the 4-bit residual weight plus the 16-bit rank-32 branch,
// executed as one fused kernel (the "Measured" table contrasts it with an
// unfused dequantise-then-GEMM path).  "MiniMax-H3 NVFP4 -- what the smoothing
// scale should be calibrated on", section "Why": one E4M3 scale per 16
// consecutive channels.
//
//   Y[m, n] = alpha * (sum_k A[m,k] B[n,k] + sum_j D'[m,j] up[n,j]) + bias[n]
//   alpha   = s_g_act * s_g_w,   D' = D / alpha (split into bf16 hi + lo)
//
// One persistent CTA per SM walks 128 x 256 output tiles (in bands of the
// operand walked fastest, so that band stays in L2).  Warps:
//   0     operand producer: per 256-channel stage, A codes 128 x 128 B and B
//         codes 256 x 128 B (128-byte swizzle) into a four-stage ring; each
//         tile's first ring position is its low-rank stage, handed to the
//         epilogue warps to fill
//   1     tcgen05 issuer and tensor-memory owner: per tile 4 kind::f16 MMAs for
//         the low-rank term (K = 64: 32 ranks of D'_hi then 32 of D'_lo
//         against up twice), which start the accumulator; then per stage one
//         barrier wait and 4 kind::mxf4nvf4 block16 MMAs (K = 64 each)
//   2..5  block-scale writers: each stage's scale atoms, shared memory ->
//         registers -> tensor memory (tcgen05.st, one warp per lane quarter),
//         into a per-stage buffer, then an arrival on the stage's barrier; this
//         keeps the tensor pipe free for MMAs
//   6..13 epilogue (two warps per tensor-memory lane quarter): the next tile's
//         low-rank stage (D' hi/lo and up in the swizzled operand layout), then
//         tensor memory -> registers, alpha and bias, bf16 rows staged in shared
//         memory and written by TMA bulk stores (fp32 rows: plain stores); the
//         accumulator is released as soon as it has been read, so the stores
//         overlap the next tile's main loop
//   14    scale producer: the scale atoms of two stages at a time (A 4 KB, W
//         8 KB, two 3-D tensor loads) into a 2-slot ring, from its own thread so
//         the operand copies never queue behind them
// Instantiations (linear_kernel<out fp32, score, MXFP8>):
//   <0|1, 0, 0>  svdq_linear: the NVFP4 linear, bf16 or fp32 output
//   <0, 1, 0>    svdq_linear_score: the same over a three-stage ring, with the tile
//                scored against a bf16 reference in the epilogue (reference strips by
//                TMA into a 48 KB epilogue area, per-row exact fp32 pair sums,
//                per-segment fp64 sums, a grid barrier and a final sum in CTA order);
//                writing Y is optional
//   <0, 0, 1>    svdq_linear_mxfp8: E4M3 operands with E8M0 scales per 32 on
//                kind::mxf8f6f4 MMAs; 128 channels per stage, one scale atom per 128
//                rows per stage serving its four K = 32 MMAs through the scale ids;
//                no tensor scales, no low-rank branch
//
// What paces the main loop (measured on B200 with a stripped main-loop kernel):
// the tensor pipe keeps only a short queue, so every instruction the issuing
// thread runs between MMAs shows up as idle tensor cycles (hence one barrier
// wait per stage, stage and phase kept as counters, descriptors precomputed);
// and the TMA unit spends a roughly fixed time per copy, so the scale atoms
// travel in as few copies as possible (two per two stages instead of three per
// stage).
#include <cooperative_groups.h>

#include "common.cuh"
#include "sm100.cuh"

namespace svdq {
namespace {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBKBytes = 128;                 // packed FP4 bytes per row per stage (256 channels)
constexpr int kBK = 256;                      // channels per stage
constexpr int kThreads = 480;                 // 15 warps
constexpr int kSfWarp0 = 2;                   // warps 2..5 write block scales into tensor memory
constexpr int kSfWarps = 4;
constexpr int kEpiWarp0 = 6;                  // warps 6..13: epilogue
constexpr int kEpiWarps = 8;
constexpr int kSfLoadWarp = 14;               // warp 14: scale-atom copies
static_assert(kSfWarp0 == 2 && kSfWarp0 + kSfWarps == kEpiWarp0 && kEpiWarp0 + kEpiWarps == kSfLoadWarp &&
                  kSfLoadWarp + 1 == kThreads / 32,
              "warp roles: 0 operand producer, 1 MMA issuer, 2..5 scale writers, 6..13 epilogue, 14 scale "
              "producer; each group of four consecutive warps covers the four tensor-memory lane quarters "
              "(warp % 4)");

constexpr uint32_t kATile = kBM * kBKBytes;          // 16 KB
constexpr uint32_t kBTile = kBN * kBKBytes;          // 32 KB
constexpr uint32_t kStageBytes = kATile + kBTile;
// Scale atoms (512 B per 128 rows x 64 channels) of two consecutive stages:
// A: 8 atoms of the tile's row block; W: 8 atoms of each of its two row blocks.
constexpr uint32_t kSfaPair = 4096;
constexpr uint32_t kSfSlot = kSfaPair + 8192;        // 12 KB
// Scoring: reference strips of 128 rows x 64 bf16 columns, three in the epilogue area.
constexpr uint32_t kStripBytes = kBM * 128;
constexpr uint32_t kScoreBytes = 2 * kBM * 16 + kMaxSegments * 16 + kMaxSegments * 8;
constexpr uint32_t kYStageBytes = 1024;              // per epilogue warp: 32 rows x 16 bf16 columns

// Shared-memory layout.  The low-rank operands of a tile travel through the
// operand ring as one more stage (written by the epilogue warps), so the ring
// takes all the room the rest leaves: four 48 KB stages, or three where the
// scoring epilogue needs 48 KB for its reference strips.
template <bool kScore>
struct LinLayout {
    static constexpr int kStages = kScore ? 3 : 4;
    static constexpr uint32_t kOffStages = 0;
    static constexpr uint32_t kOffSf = kStages * kStageBytes;              // 2 slots, multiple of 1024
    static constexpr uint32_t kOffEpi = kOffSf + 2 * kSfSlot;              // output staging / reference strips
    static constexpr uint32_t kEpiBytes = kScore ? 3 * kStripBytes : kEpiWarps * kYStageBytes;
    static constexpr uint32_t kOffBar = kOffEpi + kEpiBytes;
    static constexpr uint32_t kOffBias = kOffBar + 256;                    // 2 x 256 bf16 bias staging
    static constexpr uint32_t kOffScore = kOffBias + 2 * kBN * 2;          // scoring: row and segment sums
    static constexpr uint32_t kBytes = kOffScore + (kScore ? kScoreBytes : 0);
    static_assert(kBytes + 1024 <= 232448, "fits the 227 KB opt-in shared memory of one CTA");
};

// Tensor-memory columns: accumulator [0, 256), then one block-scale buffer per
// pipeline stage (48 columns each: A scales 4 per MMA, B scales 8 per MMA).
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemSf0 = 256;
constexpr uint32_t kTmemSfStride = 48;
constexpr uint32_t kTmemSfbOff = 16;
static_assert(kTmemSf0 + 4 * kTmemSfStride <= kTmemCols, "accumulator and four scale buffers fit tensor memory");

struct LinearArgs {
    const uint8_t* a_sf;
    const uint8_t* w_sf;
    const float* D;
    const uint16_t* up;
    const uint16_t* bias;
    void* Y;
    int64_t ldy;
    int64_t M, N, K;
    const float* s_g_act;
    const float* s_g_w;
    int r;
    int m_tiles, n_tiles;
    int n_fastest;            // tile order: 1 = N fastest (the weight stays in L2), 0 = M fastest
    int band;                 // blocks of the fastest-walked operand per band (see tile_coords)
    uint32_t* err;
    // Scoring fused into the epilogue (bf16 output only; the reference comes by tensor map).
    int write_y;              // 0: the output itself is not written
    double* seg_part;         // [gridDim.x][n_seg][2] per-CTA (num, den) of every segment
    double* num;
    double* den;
    double* rel;
    SegTable segs;
    // Store-check extents (debug library): Y's columns and rows for TMA box
    // origins, fp32 Y elements ((M - 1) ldy + N), workspace doubles, segments.
    int64_t ext_box_x, ext_box_y, ext_y32, ext_part, ext_seg;
};

// Scoring of eight output elements against the reference: the fp32 8-term
// partial sums of the standalone scoring kernel (differences and squares in fp32,
// in column order).
__device__ __forceinline__ void score8(const uint32_t (&q)[4], const uint4& rv, float& n8, float& d8) {
    const uint32_t wr[4] = {rv.x, rv.y, rv.z, rv.w};
    n8 = 0.0f;
    d8 = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float r_lo = bf16_lo(wr[i]), r_hi = bf16_hi(wr[i]);
        const float e_lo = __fsub_rn(bf16_lo(q[i]), r_lo);
        const float e_hi = __fsub_rn(bf16_hi(q[i]), r_hi);
        n8 = __fmaf_rn(e_lo, e_lo, n8);
        n8 = __fmaf_rn(e_hi, e_hi, n8);
        d8 = __fmaf_rn(r_lo, r_lo, d8);
        d8 = __fmaf_rn(r_hi, r_hi, d8);
    }
}

// hi + lo += x for an unevaluated fp32 pair: TwoSum (Knuth, TAOCP vol. 2,
// 4.2.2; Moller 1965) makes s + e == hi + x exactly, the rounding errors gather
// in lo.  A row's partials summed this way stay within a few units of 2^-48 of
// their exact sum, so the one fp64 conversion per row replaces an fp64 addition
// per partial (fp64 instructions slow the tensor-core main loop that shares the SM).
__device__ __forceinline__ void pair_add(float& hi, float& lo, float x) {
    const float s = __fadd_rn(hi, x);
    const float bp = __fsub_rn(s, hi);
    const float ap = __fsub_rn(s, bp);
    const float e = __fadd_rn(__fsub_rn(hi, ap), __fsub_rn(x, bp));
    hi = s;
    lo = __fadd_rn(lo, e);
}

// Output tile -> (M block, N block).  The order decides what the CTAs working
// at the same time share: the smaller operand's blocks are walked fastest, so
// each block of the other operand is read once while the smaller one is re-read
// from L2.  When the smaller operand itself is larger than what the L2 keeps for
// the SMs that read it (the 52 MB weight of the 16384 x 20480 -> 5120 layer was
// read from DRAM again on every pass of the persistent grid), it is walked in
// bands of `band` blocks: every block of the other operand passes under one band
// before the next band starts, so the band stays resident and the larger operand
// is read once per band.
struct TileOrder {
    int m_tiles, n_tiles, n_fastest, band;
};

__device__ __forceinline__ void tile_coords(const TileOrder& a, int tile, int& m_blk, int& n_blk) {
    const int fast_tiles = a.n_fastest ? a.n_tiles : a.m_tiles;
    const int slow_tiles = a.n_fastest ? a.m_tiles : a.n_tiles;
    const int per_band = a.band * slow_tiles;                // tiles of one full band
    const int b = tile / per_band;
    const int r = tile - b * per_band;
    const int f0 = b * a.band;
    const int width = min(a.band, fast_tiles - f0);          // the last band may be narrower
    const int fast = f0 + r % width, slow = r / width;
    if (a.n_fastest) {
        n_blk = fast;
        m_blk = slow;
    } else {
        m_blk = fast;
        n_blk = slow;
    }
}

__device__ __forceinline__ void tile_coords(const LinearArgs& a, int tile, int& m_blk, int& n_blk) {
    tile_coords(TileOrder{a.m_tiles, a.n_tiles, a.n_fastest, a.band}, tile, m_blk, n_blk);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t out;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(out) : "f"(hi), "f"(lo));
    return out;
}

// The tile's low-rank operands, written by the epilogue warps into the ring
// slot that follows the tile's last K stage: A = D' of the tile's 128 rows as
// bf16 hi (ranks 0..31) | lo (32..63), B = up of its 256 columns twice, both in
// the 128-byte-swizzled K-major layout the MMAs read, D' = D / alpha.  The
// global reads (the tile's D rows and up rows) are issued before the wait for
// the slot (go_bar: the producer found the slot free), so only shared-memory
// stores follow it.  Every epilogue thread calls this; whether to go on is
// decided together (no warp is ever left waiting at the named barrier); four
// warps arrive on the slot's barrier, the count the scale writers give an
// ordinary stage, and one on done_bar.
__device__ __forceinline__ bool lr_stage(const LinearArgs& a, uint8_t* slot, uint64_t* go_bar, uint32_t parity,
                                         uint64_t* full_bar, uint64_t* done_bar, int m_blk, int n_blk,
                                         float inv_alpha, int etid, volatile uint32_t* abort_flag) {
    const int r = a.r;
    const int arow = etid >> 1, h = etid & 1;               // A row of this thread and its 16 ranks
    float dv[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) dv[j] = 0.0f;
    const int64_t gm = static_cast<int64_t>(m_blk) * kBM + arow;
    if (gm < a.M && 16 * h < r) {
        const float4* src = reinterpret_cast<const float4*>(a.D + gm * r + 16 * h);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 v = __ldg(src + q);
            dv[4 * q] = v.x; dv[4 * q + 1] = v.y; dv[4 * q + 2] = v.z; dv[4 * q + 3] = v.w;
        }
    }
    uint4 u[4];                                              // B row etid: up[n, 0..31] (zero past r)
    const int64_t gn = static_cast<int64_t>(n_blk) * kBN + etid;
    const uint4* usrc = reinterpret_cast<const uint4*>(a.up + gn * r);
#pragma unroll
    for (int c = 0; c < 4; ++c) u[c] = (c * 8 < r && gn < a.N) ? __ldg(usrc + c) : make_uint4(0, 0, 0, 0);
    // D' = D / alpha as bf16 hi + lo pairs, formed before the wait
    uint32_t hi[8], lo[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float x0 = __fmul_rn(dv[2 * j], inv_alpha);
        const float x1 = __fmul_rn(dv[2 * j + 1], inv_alpha);
        hi[j] = pack_bf16x2(x0, x1);
        lo[j] = pack_bf16x2(__fsub_rn(x0, bf16_lo(hi[j])), __fsub_rn(x1, bf16_hi(hi[j])));
    }
    const bool ok = mbar_wait(go_bar, parity, abort_flag, a.err, kErrWaitLowRank);
    if (ok) {
        uint8_t* rowp = slot + arow * 128;
        const int sw = arow & 7;
        *reinterpret_cast<uint4*>(rowp + (((2 * h) ^ sw) << 4)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(rowp + (((2 * h + 1) ^ sw) << 4)) = make_uint4(hi[4], hi[5], hi[6], hi[7]);
        *reinterpret_cast<uint4*>(rowp + (((4 + 2 * h) ^ sw) << 4)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        *reinterpret_cast<uint4*>(rowp + (((5 + 2 * h) ^ sw) << 4)) = make_uint4(lo[4], lo[5], lo[6], lo[7]);
        uint8_t* browp = slot + kATile + etid * 128;
        const int swb = etid & 7;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            *reinterpret_cast<uint4*>(browp + ((c ^ swb) << 4)) = u[c];
            *reinterpret_cast<uint4*>(browp + (((c + 4) ^ swb) << 4)) = u[c];
        }
    }
    fence_async_shared();                                    // the tensor core reads these stores
    const bool fail = bar_sync_or<1, kEpiWarps * 32>(!ok);
    if (!fail && (etid & 31) == 0 && etid < 4 * 32) mbar_arrive(full_bar);
    if (!fail && etid == 0) mbar_arrive(done_bar);
    return !fail;
}

// The scale atoms of two stages per copy pair into a 2-slot ring (`ring`,
// kSfSlot bytes a slot), in the operand producer's tile order, as far ahead as
// the writers free the slots.  Issued from their own thread (warp 14): TMA issue
// from one thread is serial, so the operand copies never queue behind these.
template <bool kMx>
__device__ __forceinline__ void scale_producer(const CUtensorMap* tmap_sfa, const CUtensorMap* tmap_sfb,
                                            TileOrder order, uint32_t* err, uint8_t* ring, uint64_t* sf_data,
                                            uint64_t* sf_free, volatile uint32_t* abort_flag, int num_tiles,
                                            int k_stages) {
    constexpr uint32_t kSfaPairT = kMx ? 1024 : kSfaPair;          // A scale bytes of two stages
    constexpr uint32_t kSfSlotT = kMx ? 3072 : kSfSlot;            // A + W scale bytes of two stages
    constexpr int kSfHalvesPerStage = kMx ? 2 : 8;                  // 256-byte scale pieces per row block
    prefetch_tmap(tmap_sfa);
    prefetch_tmap(tmap_sfb);
    pdl_wait();                                   // the activation scales are written
    const uint64_t pol_keep = l2_evict_last_policy(), pol_once = l2_evict_first_policy();
    const uint64_t pol_a = order.n_fastest ? pol_once : pol_keep;
    const uint64_t pol_b = order.n_fastest ? pol_keep : pol_once;
    int issued = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        int m_blk, n_blk;
        tile_coords(order, tile, m_blk, n_blk);
        for (int kb = 0; kb < k_stages; kb += 2) {
            const int slot = issued & 1;
            if (issued >= 2 &&
                !mbar_wait(&sf_free[slot], ((issued >> 1) & 1) ^ 1, abort_flag, err, kErrWaitEmpty)) {
                ok = false;
                break;
            }
            uint8_t* dst = ring + slot * kSfSlot;
            mbar_arrive_expect_tx(&sf_data[slot], kSfSlotT);
            // scale atoms of stages kb and kb + 1 (a last odd stage reads zeros past K)
            tma_load_3d_hint(dst, tmap_sfa, &sf_data[slot], 0, kb * kSfHalvesPerStage, m_blk, pol_a);
            tma_load_3d_hint(dst + kSfaPairT, tmap_sfb, &sf_data[slot], 0, kb * kSfHalvesPerStage, 2 * n_blk,
                             pol_b);
            ++issued;
        }
    }
    // Bounded drain of the copies still in flight.
    for (int q = (issued > 2 ? issued - 2 : 0); q < issued; ++q) {
        const long long t0 = clock64();
        while (!mbar_try_wait(&sf_data[q & 1], (q >> 1) & 1) && clock64() - t0 < kWaitLimitCycles) {}
    }
}

template <bool kOutF32, bool kScore, bool kMx>
__global__ void __launch_bounds__(kThreads, 1)
linear_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
              const __grid_constant__ CUtensorMap tmap_y, const __grid_constant__ CUtensorMap tmap_r,
              const __grid_constant__ CUtensorMap tmap_sfa,
              const __grid_constant__ CUtensorMap tmap_sfb, LinearArgs args) {
    using L = LinLayout<kScore>;
    constexpr int kStagesT = L::kStages;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
    uint64_t* empty = full + kStagesT;
    uint64_t* acc_full = empty + kStagesT;
    uint64_t* acc_empty = acc_full + 1;
    uint64_t* sf_data = acc_empty + 1;                      // 2 slots: scale atoms landed
    uint64_t* sf_free = sf_data + 2;                        // 2 slots: the writers have read them
    uint64_t* strip_full = sf_free + 2;                     // scoring: reference strips 0..3 landed
    uint64_t* ring_free0 = strip_full + 4;                  // scoring: column half 0 done with slot 0
    uint64_t* lr_go = ring_free0 + 1;                       // producer: this tile's low-rank slot is free
    uint64_t* lr_done = lr_go + 1;                          // epilogue: this tile's low-rank stage is written
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(lr_done + 1);
    volatile uint32_t* abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5;
    const uint32_t lane = threadIdx.x & 31;
    const int num_tiles = args.m_tiles * args.n_tiles;
    // Format constants.  NVFP4: 256 channels per 128-byte stage row, four scale
    // atoms per 128 rows per stage (one per MMA of K = 64).  MXFP8: 128 channels
    // per stage row, one scale atom per 128 rows per stage whose four bytes serve
    // the stage's four MMAs of K = 32 (scale ids 0..3).
    constexpr int kStageK = kMx ? 128 : kBK;
    constexpr uint32_t kSfaPairT = kMx ? 1024 : kSfaPair;          // A scale bytes of two stages
    constexpr uint32_t kTmemSfStrideT = kMx ? 16 : kTmemSfStride;
    constexpr uint32_t kTmemSfbOffT = kMx ? 4 : kTmemSfbOff;
    // a last partial stage reads zero codes and zero scales past K (TMA fill): it adds nothing
    const int k_stages = static_cast<int>((args.K + kStageK - 1) / kStageK);
    const bool has_lr = args.r > 0;
    // Ring positions per tile: the low-rank stage, then the K stages.
    const int span = k_stages + (has_lr ? 1 : 0);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStagesT; ++s) {
            // operand bytes + the stage's scales in tensor memory (low-rank stage:
            // the producer's arrival + four epilogue warps' operand stores)
            mbar_init(&full[s], 1 + kSfWarps);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sf_data[i], 1);
            mbar_init(&sf_free[i], kSfWarps);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, kEpiWarps);
        for (int i = 0; i < 4; ++i) mbar_init(&strip_full[i], 1);
        mbar_init(ring_free0, kEpiWarps / 2);
        mbar_init(lr_go, 1);
        mbar_init(lr_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&tmap_a);
            prefetch_tmap(&tmap_b);
            pdl_wait();                               // the activation codes are written
            // L2 policies: the operand walked fastest over the tiles (the smaller
            // one) is re-read by every block row (or column) of the other, so it
            // is kept; the other streams through once.
            const uint64_t pol_keep = l2_evict_last_policy(), pol_once = l2_evict_first_policy();
            const uint64_t pol_a = args.n_fastest ? pol_once : pol_keep;
            const uint64_t pol_b = args.n_fastest ? pol_keep : pol_once;
            int s = 0, it = 0, lr_tiles = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                int m_blk, n_blk;
                tile_coords(args, tile, m_blk, n_blk);
                if (has_lr) {
                    // The low-rank stage opens the tile: the epilogue warps fill this
                    // slot.  The producer walks the ring in order, so its wait for
                    // the slot's previous MMAs is the safe one (a parity wait tells
                    // only one phase from the next); it hands the free slot to the
                    // epilogue through lr_go, once the epilogue has written the
                    // previous tile's stage (lr_done), so neither barrier ever runs
                    // two phases ahead of its waiter.  Its arrival on full stands
                    // for the copies.
                    if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, args.err, kErrWaitEmpty)) { ok = false; break; }
                    if (lr_tiles > 0 &&
                        !mbar_wait(lr_done, (lr_tiles - 1) & 1, abort_flag, args.err, kErrWaitLowRank)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive(&full[s]);
                    mbar_arrive(lr_go);
                    ++lr_tiles;
                    ++it;
                    if (++s == kStagesT) { s = 0; ph ^= 1u; }
                }
                for (int kb = 0; kb < k_stages; ++kb, ++it) {
                    if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, args.err, kErrWaitEmpty)) { ok = false; break; }
                    uint8_t* st = smem + L::kOffStages + s * kStageBytes;
                    mbar_arrive_expect_tx(&full[s], kStageBytes);
                    tma_load_2d_hint(st, &tmap_a, &full[s], kb * kBKBytes, m_blk * kBM, pol_a);
                    tma_load_2d_hint(st + kATile, &tmap_b, &full[s], kb * kBKBytes, n_blk * kBN, pol_b);
                    if (++s == kStagesT) { s = 0; ph ^= 1u; }
                }
            }
            // Bounded drain of the copies still in flight.
            for (int i = (it > kStagesT ? it - kStagesT : 0); i < it; ++i) {
                const long long t0 = clock64();
                while (!mbar_try_wait(&full[i % kStagesT], (i / kStagesT) & 1) && clock64() - t0 < kWaitLimitCycles) {}
            }
        }
    } else if (warp == kSfLoadWarp) {
        // ------------------------------------------------------------ scale-atom producer
        if (lane == 0)
            scale_producer<kMx>(&tmap_sfa, &tmap_sfb, TileOrder{args.m_tiles, args.n_tiles, args.n_fastest, args.band},
                                args.err, smem + L::kOffSf, sf_data, sf_free, abort_flag, num_tiles, k_stages);
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // Kept to the minimum between MMAs: one wait per stage (the barrier counts
        // the operand bytes and the four scale writers), counters instead of
        // divisions, descriptors advanced by constant offsets.
        if (lane == 0) {
            const uint32_t idesc_f4 = idesc_nvf4(kBM, kBN);
            const uint32_t idesc_lr = idesc_bf16(kBM, kBN);
            const uint64_t da0 = desc_kmajor_sw128(smem_u32(smem + L::kOffStages));
            const uint64_t db0 = desc_kmajor_sw128(smem_u32(smem + L::kOffStages + kATile));
            constexpr uint64_t kStageDesc = kStageBytes >> 4;     // descriptor address field counts 16 bytes
            int s = 0, local = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++local) {
                if (!mbar_wait(acc_empty, (local & 1) ^ 1, abort_flag, args.err, kErrWaitAccum)) break;
                tc_fence_after();
                if (has_lr) {
                    // The low-rank term opens the tile and initialises the
                    // accumulator: 4 kind::f16 MMAs (K = 64: 32 ranks of D'_hi, then
                    // 32 of D'_lo, against up twice) from the ring slot the epilogue
                    // warps filled while the previous tile was finishing.
                    if (!mbar_try_wait(&full[s], ph) &&
                        !mbar_wait(&full[s], ph, abort_flag, args.err, kErrWaitLowRank))
                        break;
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(smem + L::kOffStages + s * kStageBytes);
                    const uint32_t b0 = a0 + kATile;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(tmem, desc_kmajor_sw128(a0 + kk * 32), desc_kmajor_sw128(b0 + kk * 32), idesc_lr,
                                 kk == 0 ? 0u : 1u);
                    tc_commit(&empty[s]);
                    if (++s == kStagesT) { s = 0; ph ^= 1u; }
                }
                const uint32_t acc0 = has_lr ? 1u : 0u;            // the first K stage starts the sum without it
                for (int kb = 0; kb < k_stages; ++kb) {
                    if (!mbar_try_wait(&full[s], ph) &&
                        !mbar_wait(&full[s], ph, abort_flag, args.err, kErrWaitFull)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t da = da0 + kStageDesc * s, db = db0 + kStageDesc * s;
                    const uint32_t sf = tmem + kTmemSf0 + s * kTmemSfStrideT;
                    const uint32_t acc = kb == 0 ? acc0 : 1u;
                    if constexpr (kMx) {
                        mma_mxf8(tmem, da, db, idesc_mxf8(kBM, kBN, 0), sf, sf + kTmemSfbOffT, acc);
                        mma_mxf8(tmem, da + 2, db + 2, idesc_mxf8(kBM, kBN, 1), sf, sf + kTmemSfbOffT, 1u);
                        mma_mxf8(tmem, da + 4, db + 4, idesc_mxf8(kBM, kBN, 2), sf, sf + kTmemSfbOffT, 1u);
                        mma_mxf8(tmem, da + 6, db + 6, idesc_mxf8(kBM, kBN, 3), sf, sf + kTmemSfbOffT, 1u);
                    } else {
                        mma_nvf4(tmem, da, db, idesc_f4, sf, sf + kTmemSfbOff, acc);
                        mma_nvf4(tmem, da + 2, db + 2, idesc_f4, sf + 4, sf + kTmemSfbOff + 8, 1u);
                        mma_nvf4(tmem, da + 4, db + 4, idesc_f4, sf + 8, sf + kTmemSfbOff + 16, 1u);
                        mma_nvf4(tmem, da + 6, db + 6, idesc_f4, sf + 12, sf + kTmemSfbOff + 24, 1u);
                    }
                    tc_commit(&empty[s]);
                    if (++s == kStagesT) { s = 0; ph ^= 1u; }
                }
                if (!ok) break;
                tc_commit(acc_full);
            }
        }
    } else if (warp < kEpiWarp0) {
        // ------------------------------------------------------------ block-scale writers
        // Each warp copies the stage's scale atoms from the shared-memory ring
        // into its own tensor-memory lane quarter with tcgen05.st, then arrives
        // on the stage's barrier.  The block-scaled MMA of lane quarter q reads
        // the W scales of all 256 columns (so every quarter holds all of them)
        // and, of the four A-scale columns of an MMA (rows 32 j + lane in column
        // j), only column q: each writer stores just that one (the same output
        // bit for bit as storing all four).  Unlike a shared->tensor copy issued by
        // the MMA thread, these stores run alongside the MMAs instead of in front
        // of them.  Ring slot: released after the stores of its last stage.
        // Tensor-memory buffer s: written only after the MMAs of its previous
        // use have completed (the stage's empty barrier).  Low-rank stages are
        // the epilogue's: the writers only step over them.
        const uint32_t tq = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        int s = 0, it = 0, pair = -1;
        uint32_t ph = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
            if (has_lr) {                                   // the tile's low-rank stage is the epilogue's
                ++it;
                if (++s == kStagesT) { s = 0; ph ^= 1u; }
            }
            for (int kb = 0; kb < k_stages; ++kb, ++it) {
                if ((kb & 1) == 0) ++pair;
                const int slot = pair & 1;
                if (!mbar_try_wait(&sf_data[slot], (pair >> 1) & 1) &&
                    !mbar_wait(&sf_data[slot], (pair >> 1) & 1, abort_flag, args.err, kErrWaitFull)) {
                    ok = false;
                    break;
                }
                // Slot layout: A atoms [8][512] of the two stages, then W row block
                // 2n and 2n + 1, [8][512] each.  Column layout of one tensor-memory
                // buffer: A scales of MMA kk at 4 kk + (row / 32); W scales of MMA
                // kk at 16 + 8 kk + (row / 32), rows 128..255 at + 4.  Lane i reads
                // row i of each 512-byte atom: its 4 words are the 4 columns.
                uint32_t ra[4], rb[kMx ? 8 : 32];
                if constexpr (kMx) {
                    // MXFP8: the stage's one A atom and one W atom per 128-row block
                    // (slot layout: A [2 stages][512], then W [2 row blocks][2 stages][512]).
                    const uint8_t* sfa = smem + L::kOffSf + slot * kSfSlot + (kb & 1) * 512;
                    const uint8_t* sfb = smem + L::kOffSf + slot * kSfSlot + kSfaPairT + (kb & 1) * 512;
                    const uint4 a = *reinterpret_cast<const uint4*>(sfa + lane * 16);
                    const uint4 x = *reinterpret_cast<const uint4*>(sfb + lane * 16);
                    const uint4 y = *reinterpret_cast<const uint4*>(sfb + 1024 + lane * 16);
                    ra[0] = a.x; ra[1] = a.y; ra[2] = a.z; ra[3] = a.w;
                    rb[0] = x.x; rb[1] = x.y; rb[2] = x.z; rb[3] = x.w;
                    rb[4] = y.x; rb[5] = y.y; rb[6] = y.z; rb[7] = y.w;
                } else {
                    const uint8_t* sfa = smem + L::kOffSf + slot * kSfSlot + (kb & 1) * 2048;
                    const uint8_t* sfb = smem + L::kOffSf + slot * kSfSlot + kSfaPair + (kb & 1) * 2048;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        // A: only this lane quarter's rows (word `warp & 3` of the lane's 16 bytes)
                        ra[q] = *reinterpret_cast<const uint32_t*>(sfa + q * 512 + lane * 16 + (warp & 3) * 4);
                        const uint4 x = *reinterpret_cast<const uint4*>(sfb + q * 512 + lane * 16);
                        const uint4 y = *reinterpret_cast<const uint4*>(sfb + 4096 + q * 512 + lane * 16);
                        rb[8 * q] = x.x; rb[8 * q + 1] = x.y; rb[8 * q + 2] = x.z; rb[8 * q + 3] = x.w;
                        rb[8 * q + 4] = y.x; rb[8 * q + 5] = y.y; rb[8 * q + 6] = y.z; rb[8 * q + 7] = y.w;
                    }
                }
                if (it >= kStagesT && !mbar_try_wait(&empty[s], ph ^ 1) &&
                    !mbar_wait(&empty[s], ph ^ 1, abort_flag, args.err, kErrWaitEmpty)) {
                    ok = false;
                    break;
                }
                const uint32_t base = tq + kTmemSf0 + s * kTmemSfStrideT;
                if constexpr (kMx) {
                    // columns: A 0..3, W rows 0..127 at 4..7 and rows 128..255 at 8..11
                    const uint32_t r[16] = {ra[0], ra[1], ra[2], ra[3], rb[0], rb[1], rb[2], rb[3],
                                            rb[4], rb[5], rb[6], rb[7], 0u, 0u, 0u, 0u};
                    tmem_st_32x32b_x16(base, r);
                } else {
                    // A scales of MMA kk sit in columns 4 kk .. 4 kk + 3 (rows 32 j + lane in
                    // column 4 kk + j); lane quarter q reads only column 4 kk + q, so each
                    // writer stores that one.  W scales: all 32 columns in every quarter.
#pragma unroll
                    for (int q = 0; q < 4; ++q) tmem_st_32x32b_x1(base + 4 * q + (warp & 3), ra[q]);
                    tmem_st_32x32b_x32(base + kTmemSfbOff, rb);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&full[s]);
                // The ring slot is released only now: the shared-memory loads above
                // are complete once the tensor-memory stores that read their
                // registers have been issued, and a slot released with loads still
                // in flight could be refilled by the next copy under them.
                if (lane == 0 && ((kb & 1) == 1 || kb == k_stages - 1)) mbar_arrive(&sf_free[slot]);
                if (++s == kStagesT) { s = 0; ph ^= 1u; }
            }
        }
    } else if constexpr (kScore) {
        // ------------------------------------------------------------ epilogue with scoring
        // The plain epilogue's output path plus the tile's scoring against the
        // reference output.  The reference comes in by TMA as strips of 128 rows x
        // 64 columns (16 KB, 128-byte swizzle) into a three-slot ring in the
        // epilogue area, which the previous tile's strips (and the output stores
        // that read them) have left by the barrier that ends each tile.  Strips 0 and 2 (the first 64 columns of each
        // column half) and strip 1 go out at "accumulator full"; strip 3 takes
        // strip 0's slot once the four warps of column half 0 are done with it.
        // Each lane scores its own row against its converted output values, so no
        // value moves between lanes; the bf16 output, when written, is staged over
        // the reference chunks it replaces (each lane rewrites exactly the bytes it
        // read) and leaves by a TMA store.  The tile loop is left only at its top,
        // through a barrier that ORs the abort flag over the epilogue warps, so a
        // wait that runs out never strands the other warps at a barrier.
        const int ew = warp - kEpiWarp0;                    // 0..7
        const int quarter = warp & 3;                       // lane quarter this warp may access
        const int half = ew >> 2;                           // column half of the tile
        const int etid = ew * 32 + lane;                    // 0..255
        const uint32_t tbase = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + half * (kBN / 2);
        uint16_t* bias_s = reinterpret_cast<uint16_t*>(smem + L::kOffBias);
        uint8_t* ring = smem + L::kOffEpi;
        double2* rowsum = reinterpret_cast<double2*>(smem + L::kOffScore);   // [column half][tile row] (num, den)
        double2* segsum = rowsum + 2 * kBM;                              // [segment] this CTA's (num, den)
        int2* segrows = reinterpret_cast<int2*>(segsum + kMaxSegments);  // [segment] rows [begin, end)
        const int n_seg = args.segs.n;
        pdl_wait();                                   // inputs of the earlier kernels are written
        const float alpha = __fmul_rn(__ldg(args.s_g_act), __ldg(args.s_g_w));
        const float inv_alpha = __frcp_rn(alpha);
        for (int i = etid; i < kMaxSegments; i += kEpiWarps * 32) {
            segsum[i] = make_double2(0.0, 0.0);
            if (i < n_seg) {
                const int64_t b = args.segs.begin[i];
                const int64_t e = b + (args.segs.prefix[i + 1] - args.segs.prefix[i]);
                segrows[i] = make_int2(static_cast<int>(b), static_cast<int>(e));
            }
        }
        if (etid == 0) prefetch_tmap(&tmap_r);
        const int32_t M32 = static_cast<int32_t>(args.M);
        // the first tile's low-rank stage (ring position 0); a failure raises the
        // abort flag, which the loop top reads
        if (has_lr && static_cast<int>(blockIdx.x) < num_tiles) {
            int m_0, n_0;
            tile_coords(args, blockIdx.x, m_0, n_0);
            lr_stage(args, smem + L::kOffStages, lr_go, 0u, &full[0], lr_done, m_0, n_0, inv_alpha, etid, abort_flag);
        }
        int local = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
            int m_blk, n_blk;
            tile_coords(args, tile, m_blk, n_blk);
            const int32_t col0 = n_blk * kBN;
            const int32_t m0 = m_blk * kBM;
            uint16_t* bt = bias_s + (local & 1) * kBN;
            bt[etid] = (args.bias && col0 + etid < args.N) ? args.bias[col0 + etid] : static_cast<uint16_t>(0);
            // bias staged, the previous tile's row sums consumed; leave together on abort
            if (bar_sync_or<1, kEpiWarps * 32>(*abort_flag != 0u)) break;
            if (has_lr && tile + static_cast<int>(gridDim.x) < num_tiles) {
                // the next tile's low-rank stage (its first ring position), written
                // while this tile's last K stages run
                const int64_t p = static_cast<int64_t>(local + 1) * span;
                const int slot = static_cast<int>(p % kStagesT);
                int m_nx, n_nx;
                tile_coords(args, tile + static_cast<int>(gridDim.x), m_nx, n_nx);
                if (!lr_stage(args, smem + L::kOffStages + slot * kStageBytes, lr_go,
                              static_cast<uint32_t>((local + 1) & 1), &full[slot], lr_done, m_nx, n_nx, inv_alpha,
                              etid, abort_flag))
                    continue;                                // the abort flag is up: the loop top leaves
            }
            bool ok = __all_sync(0xffffffffu, mbar_wait(acc_full, local & 1, abort_flag, args.err, kErrWaitMma));
            tc_fence_after();
            if (ok && etid == 0) {
#pragma unroll
                for (int i = 0; i < 3; ++i) {               // slots 0, 1, 2 <- strips 0, 2, 1
                    const int strip = i == 0 ? 0 : 3 - i;
                    mbar_arrive_expect_tx(&strip_full[strip], kStripBytes);
                    tma_load_2d(ring + i * kStripBytes, &tmap_r, &strip_full[strip], col0 + strip * 64, m0);
                }
            }
            const uint16_t* bw = bt + half * (kBN / 2);
            // This warp's 128 accumulator columns as bf16 pairs (pk[h][j]: columns
            // 64 h + 2 j, 64 h + 2 j + 1), the accumulator released after the last read.
            // The first two 32-column pieces are read together, the last two one at
            // a time (the first half's values are held meanwhile).
            uint32_t pk[2][32];
            if (ok) {
                auto convert = [&](const uint32_t (&v)[32], int c) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const uint32_t bb = *reinterpret_cast<const uint32_t*>(bw + c * 32 + 2 * j);
                        pk[c >> 1][(c & 1) * 16 + j] = pack_bf16x2(fmaf(alpha, __uint_as_float(v[2 * j]), bf16_lo(bb)),
                                                                   fmaf(alpha, __uint_as_float(v[2 * j + 1]), bf16_hi(bb)));
                    }
                };
                {
                    uint32_t v[2][32];
                    tmem_ld_32x32b_x32(tbase, v[0]);
                    tmem_ld_32x32b_x32(tbase + 32, v[1]);
                    tmem_ld_wait(v[0]);
                    tmem_ld_tie(v[1]);
                    convert(v[0], 0);
                    convert(v[1], 1);
                }
#pragma unroll
                for (int c = 2; c < 4; ++c) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(tbase + c * 32, v);
                    tmem_ld_wait(v);
                    if (c == 3) {                   // the accumulator has been read: next tile's MMAs may start
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(acc_empty);
                    }
                    convert(v, c);
                }
            }
            // The row's 8-column groups in column order: fp32 within a group, exact
            // fp32 pairs across, fp64 from the row on.
            float nh = 0.0f, nl = 0.0f, dh = 0.0f, dl = 0.0f;
            const int32_t grow0 = m0 + quarter * 32;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                // half 0: strips 0 (slot 0), 1 (slot 2); half 1: strips 2 (slot 1), 3 (slot 0 again).
                // Each strip has its own barrier, completed once per tile.
                const int strip = 2 * half + h;
                const int slot = h == 0 ? half : 2 - 2 * half;
                if (ok)
                    ok = __all_sync(0xffffffffu, mbar_wait(&strip_full[strip], local & 1, abort_flag, args.err, kErrWaitRef));
                uint8_t* part = ring + slot * kStripBytes + quarter * 4096;
                if (ok) {
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        uint4* p = reinterpret_cast<uint4*>(part + lane * 128 + ((c ^ (lane & 7)) << 4));
                        const uint4 rv = *p;
                        const uint32_t q[4] = {pk[h][4 * c], pk[h][4 * c + 1], pk[h][4 * c + 2], pk[h][4 * c + 3]};
                        float n8, d8;
                        score8(q, rv, n8, d8);
                        pair_add(nh, nl, n8);
                        pair_add(dh, dl, d8);
                        if (args.write_y) *p = make_uint4(q[0], q[1], q[2], q[3]);
                    }
                    if (args.write_y) {
                        fence_async_shared();
                        __syncwarp();
                        const int32_t bx = col0 + half * (kBN / 2) + h * 64;
                        if (lane == 0 && grow0 < M32 && bx < args.N &&
                            box_ok(bx, grow0, args.ext_box_x, args.ext_box_y, args.err, kSiteLinearBox)) {
                            // boxes wholly past row M or column N are skipped
                            tma_store_2d(&tmap_y, part, bx, grow0);
                            bulk_commit_group();
                        }
                    }
                }
                if (h == 0 && half == 0) {
                    // slot 0 is free for strip 3 once column half 0's four warps (and their stores) are done with it
                    if (args.write_y && lane == 0) bulk_wait_read_all();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(ring_free0);
                    if (ew == 0) {
                        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(ring_free0, local & 1, abort_flag, args.err, kErrWaitRef));
                        if (ok && lane == 0) {
                            mbar_arrive_expect_tx(&strip_full[3], kStripBytes);
                            tma_load_2d(ring, &tmap_r, &strip_full[3], col0 + 3 * 64, m0);
                        }
                    }
                }
            }
            if (args.write_y && lane == 0) bulk_wait_read_all();   // the ring is no longer read
            __syncwarp();
            rowsum[half * kBM + quarter * 32 + lane] =
                grow0 + static_cast<int32_t>(lane) < M32
                    ? make_double2(static_cast<double>(nh) + static_cast<double>(nl),
                                   static_cast<double>(dh) + static_cast<double>(dl))
                    : make_double2(0.0, 0.0);
            asm volatile("bar.sync 1, %0;" :: "n"(kEpiWarps * 32) : "memory");
            // The tile's rows of each segment (both halves of a row together, lanes
            // striding over the rows, then a fixed shuffle tree); segment s belongs
            // to epilogue warp s mod 8.
            const int32_t m1 = min(m0 + kBM, M32);
            for (int sg = ew; sg < n_seg; sg += kEpiWarps) {
                const int2 se = segrows[sg];
                const int lo = max(se.x, m0), hi = min(se.y, m1);
                if (lo >= hi) continue;
                double n = 0.0, d = 0.0;
                for (int rr = lo - m0 + static_cast<int>(lane); rr < hi - m0; rr += 32) {
                    const double2 a = rowsum[rr], b = rowsum[kBM + rr];
                    n += a.x + b.x;
                    d += a.y + b.y;
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    n += __shfl_xor_sync(0xffffffffu, n, o);
                    d += __shfl_xor_sync(0xffffffffu, d, o);
                }
                if (lane == 0) {
                    segsum[sg].x += n;
                    segsum[sg].y += d;
                }
            }
        }
        if (args.write_y) {
            if (lane == 0) bulk_wait_all();          // bulk stores complete before the CTA exits
            __syncwarp();
        }
        for (int sg = ew; sg < n_seg; sg += kEpiWarps) {
            const int64_t off = (static_cast<int64_t>(blockIdx.x) * n_seg + sg) * 2;
            if (lane == 0 && store_ok(off, 2, args.ext_part, args.err, kSiteLinearScore)) {
                args.seg_part[off] = segsum[sg].x;
                args.seg_part[off + 1] = segsum[sg].y;
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // Two warps per tensor-memory lane quarter, each owning 128 of the 256
        // columns.  Per tile: the bias is staged in shared memory; the tile's
        // low-rank stage is written into the ring (lr_stage); then, at
        // "accumulator full", the warp reads all its 128 columns (two 32-column
        // loads per wait), releases the accumulator and only then applies alpha
        // and bias and stores, so the next tile's MMAs start as early as possible.
        // bf16 rows leave in eight TMA stores of 16 columns x 32 rows through the
        // warp's 1 KB staging buffer (bulk stores keep scattered per-row writes off
        // the load/store path the tensor core reads its operands through); fp32
        // rows with plain stores.  The loop is left only at its top, all warps
        // together, so a wait that runs out never strands a warp at a barrier.
        const int ew = warp - kEpiWarp0;                    // 0..7
        const int quarter = warp & 3;                       // lane quarter this warp may access
        const int half = ew >> 2;                           // column half of the tile
        const int etid = ew * 32 + lane;                    // 0..255
        const uint32_t tbase = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + half * (kBN / 2);
        uint16_t* bias_s = reinterpret_cast<uint16_t*>(smem + L::kOffBias);
        uint8_t* stg = smem + L::kOffEpi + ew * kYStageBytes;
        const uint64_t pol_y = l2_evict_first_policy();
        pdl_wait();                                   // inputs of the earlier kernels are written
        const float alpha = kMx ? 1.0f : __fmul_rn(__ldg(args.s_g_act), __ldg(args.s_g_w));
        const float inv_alpha = __frcp_rn(alpha);
        // the first tile's low-rank stage (ring position 0); a failure raises the
        // abort flag, which the loop top reads
        if (has_lr && static_cast<int>(blockIdx.x) < num_tiles) {
            int m_0, n_0;
            tile_coords(args, blockIdx.x, m_0, n_0);
            lr_stage(args, smem + L::kOffStages, lr_go, 0u, &full[0], lr_done, m_0, n_0, inv_alpha, etid, abort_flag);
        }
        int local = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
            int m_blk, n_blk;
            tile_coords(args, tile, m_blk, n_blk);
            const int64_t col0 = static_cast<int64_t>(n_blk) * kBN;
            uint16_t* bt = bias_s + (local & 1) * kBN;
            bt[etid] = (args.bias && col0 + etid < args.N) ? args.bias[col0 + etid] : static_cast<uint16_t>(0);
            // bias staged; leave together on abort
            if (bar_sync_or<1, kEpiWarps * 32>(*abort_flag != 0u)) break;
            if (has_lr && tile + static_cast<int>(gridDim.x) < num_tiles) {
                // the next tile's low-rank stage (its first ring position), written
                // while this tile's last K stages run
                const int64_t p = static_cast<int64_t>(local + 1) * span;
                const int slot = static_cast<int>(p % kStagesT);
                int m_nx, n_nx;
                tile_coords(args, tile + static_cast<int>(gridDim.x), m_nx, n_nx);
                if (!lr_stage(args, smem + L::kOffStages + slot * kStageBytes, lr_go,
                              static_cast<uint32_t>((local + 1) & 1), &full[slot], lr_done, m_nx, n_nx, inv_alpha,
                              etid, abort_flag))
                    continue;                                // the abort flag is up: the loop top leaves
            }
            if (!mbar_wait(acc_full, local & 1, abort_flag, args.err, kErrWaitMma)) continue;
            tc_fence_after();
            const int64_t row = static_cast<int64_t>(m_blk) * kBM + quarter * 32 + lane;
            const int64_t ccol = col0 + half * (kBN / 2);   // first output column of this warp
            const uint16_t* bw = bt + half * (kBN / 2);
            if constexpr (!kOutF32) {
                // pk[16 c + j]: columns 32 c + 2 j and 32 c + 2 j + 1 of this warp, as bf16
                uint32_t pk[64];
                auto convert = [&](const uint32_t (&v)[32], int c) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const uint32_t bb = *reinterpret_cast<const uint32_t*>(bw + c * 32 + 2 * j);
                        pk[c * 16 + j] = pack_bf16x2(fmaf(alpha, __uint_as_float(v[2 * j]), bf16_lo(bb)),
                                                     fmaf(alpha, __uint_as_float(v[2 * j + 1]), bf16_hi(bb)));
                    }
                };
                {
                    uint32_t v[2][32];
                    tmem_ld_32x32b_x32(tbase, v[0]);
                    tmem_ld_32x32b_x32(tbase + 32, v[1]);
                    tmem_ld_wait(v[0]);
                    tmem_ld_tie(v[1]);
                    convert(v[0], 0);
                    convert(v[1], 1);
                }
                {
                    // one piece at a time: the converted columns and one load fit the registers
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(tbase + 64, v);
                    tmem_ld_wait(v);
                    convert(v, 2);
                    tmem_ld_32x32b_x32(tbase + 96, v);
                    tmem_ld_wait(v);
                    tc_fence_before();              // the accumulator has been read: next tile's MMAs may start
                    __syncwarp();
                    if (lane == 0) mbar_arrive(acc_empty);
                    convert(v, 3);
                }
                const int32_t grow0 = static_cast<int32_t>(m_blk * kBM + quarter * 32);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (lane == 0) bulk_wait_read_all();    // the previous box has left the buffer
                    __syncwarp();
                    uint4* dst = reinterpret_cast<uint4*>(stg + lane * 32);
                    dst[0] = make_uint4(pk[8 * j], pk[8 * j + 1], pk[8 * j + 2], pk[8 * j + 3]);
                    dst[1] = make_uint4(pk[8 * j + 4], pk[8 * j + 5], pk[8 * j + 6], pk[8 * j + 7]);
                    fence_async_shared();
                    __syncwarp();
                    if (lane == 0 && grow0 < args.M && ccol + 16 * j < args.N &&   // boxes wholly past M or N are skipped
                        box_ok(ccol + 16 * j, grow0, args.ext_box_x, args.ext_box_y, args.err, kSiteLinearBox)) {
                        // the output is not read again here: first out of L2, so it does
                        // not push out the operands other tiles still read
                        tma_store_2d_hint(&tmap_y, stg, static_cast<int32_t>(ccol) + 16 * j, grow0, pol_y);
                        bulk_commit_group();
                    }
                }
            } else {
                const bool row_ok = row < args.M;
#pragma unroll 1
                for (int c = 0; c < kBN / 2 / 32; ++c) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(tbase + c * 32, v);
                    tmem_ld_wait(v);
                    if (row_ok && ccol + c * 32 < args.N) {           // N % 128 == 0: chunks are whole
                        const int64_t off = row * args.ldy + ccol + c * 32;
                        float* dst = static_cast<float*>(args.Y) + off;
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            if (!store_ok(off + 4 * q, 4, args.ext_y32, args.err, kSiteLinearF32)) continue;
                            float y[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int j = 4 * q + e;
                                const float bj = __uint_as_float(static_cast<uint32_t>(bw[c * 32 + j]) << 16);
                                y[e] = fmaf(alpha, __uint_as_float(v[j]), bj);
                            }
                            reinterpret_cast<float4*>(dst)[q] = make_float4(y[0], y[1], y[2], y[3]);
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acc_empty);
            }
        }
        if constexpr (!kOutF32) {
            if (lane == 0) bulk_wait_all();          // bulk stores complete before the CTA exits
            __syncwarp();
        }
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    if constexpr (kScore) {
        {
            // Every CTA's segment sums are written (the launch is cooperative, so all
            // CTAs are resident and the grid barrier is safe); CTA 0 adds them in
            // CTA order.
            cooperative_groups::this_grid().sync();
            if (blockIdx.x == 0 && warp == kEpiWarp0) {
                const int n = args.segs.n;
                for (int sg = 0; sg < n; ++sg) {
                    double num = 0.0, den = 0.0;
                    for (int c = lane; c < static_cast<int>(gridDim.x); c += 32) {
                        num += __ldcg(args.seg_part + (static_cast<int64_t>(c) * n + sg) * 2);
                        den += __ldcg(args.seg_part + (static_cast<int64_t>(c) * n + sg) * 2 + 1);
                    }
                    for (int o = 16; o > 0; o >>= 1) {
                        num += __shfl_xor_sync(0xffffffffu, num, o);
                        den += __shfl_xor_sync(0xffffffffu, den, o);
                    }
                    if (lane == 0 && store_ok(sg, 1, args.ext_seg, args.err, kSiteLinearScore)) {
                        args.num[sg] = num;
                        args.den[sg] = den;
                        double rel;
                        if (den > 0.0) rel = sqrt(num / den);
                        else rel = (num == 0.0) ? 0.0 : __longlong_as_double(0x7FF0000000000000LL);
                        args.rel[sg] = rel;
                    }
                }
            }
        }
    }
}

// Persistent grid: one CTA per SM (at most one fits), never more CTAs than tiles;
// with scoring (a cooperative launch) never more than can be resident at once.
inline int linear_grid(int m_tiles, int n_tiles, int64_t resident = 0) {
    const int64_t tiles = static_cast<int64_t>(m_tiles) * n_tiles;
    const int sms = device_sm_count() > 0 ? device_sm_count() : 148;
    int64_t g = tiles < sms ? tiles : sms;
    if (resident > 0 && g > resident) g = resident;
    return static_cast<int>(g);
}

// `ws_bytes`: the scoring workspace (per-CTA segment sums), checked against the grid.
template <bool kOutF32, bool kScore, bool kMx = false>
int launch_linear(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& ty, const CUtensorMap& tr,
                  const CUtensorMap& tsa, const CUtensorMap& tsb, const LinearArgs& a, cudaStream_t st,
                  size_t ws_bytes = 0) {
    static_assert(!(kOutF32 && kScore), "scoring is fused into the bf16 epilogue only");
    const uint32_t smem = LinLayout<kScore>::kBytes + 1024;
    auto kern = linear_kernel<kOutF32, kScore, kMx>;
    static std::atomic<uint64_t> smem_set{0};
    if (!set_dynamic_smem_once(kern, smem, smem_set)) return SVDQ_ERR_CUDA;
    int64_t resident = 0;
    if (kScore) {
        resident = coresident_grid(kern, kThreads, smem);
        if (resident < 1) return SVDQ_ERR_CUDA;
    }
    const int grid = linear_grid(a.m_tiles, a.n_tiles, resident);
    if (kScore && ws_bytes < static_cast<size_t>(grid) * a.segs.n * 2 * sizeof(double)) return SVDQ_ERR_INVALID_ARG;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    if (kScore) {
        attr[0].id = cudaLaunchAttributeCooperative;      // scoring ends with a grid barrier
        attr[0].val.cooperative = 1;
    } else {
        // a programmatic dependent of the quantiser: set-up overlaps its tail
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
    }
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return launch_status(cudaLaunchKernelEx(&cfg, kern, ta, tb, ty, tr, tsa, tsb, a));
}

// Validation, tensor maps and kernel arguments shared by the entry points.
int linear_prepare(const uint8_t* a_codes, const uint8_t* a_sf, const float* s_g_act, const float* D, int r,
                   const uint8_t* w_codes, const uint8_t* w_sf, const float* s_g_w, const void* up,
                   const void* bias, void* Y, int64_t ldy, int out_dtype, int64_t M, int64_t N, int64_t K,
                   CUtensorMap* ta, CUtensorMap* tb, CUtensorMap* ty, CUtensorMap* tsa, CUtensorMap* tsb,
                   LinearArgs* a, bool mx = false, bool score = false) {
    // mx: MXFP8 operands (one byte per element, E8M0 scales per 32, no tensor
    // scales, no low-rank branch); otherwise NVFP4 (two elements per byte).
    if (a_codes == nullptr || a_sf == nullptr || w_codes == nullptr || w_sf == nullptr ||
        (!mx && (s_g_act == nullptr || s_g_w == nullptr)))
        return SVDQ_ERR_INVALID_ARG;
    if (M < 1 || N < 1 || K < 1 || (Y != nullptr && ldy < N)) return SVDQ_ERR_INVALID_ARG;
    if (out_dtype != 0 && out_dtype != 1) return SVDQ_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(s_g_act) & 3u) || (reinterpret_cast<uintptr_t>(s_g_w) & 3u))
        return SVDQ_ERR_MISALIGNED;
    if (mx ? r != 0 : (r != 0 && r != 16 && r != 32)) return SVDQ_ERR_UNSUPPORTED;
    if ((r > 0) != (D != nullptr) || (r > 0) != (up != nullptr)) return SVDQ_ERR_INVALID_ARG;
    if (K % (mx ? 128 : 64) != 0 || N % 128 != 0) return SVDQ_ERR_UNSUPPORTED;
    if (M > (int64_t(1) << 31) - 128 || N > (int64_t(1) << 31) - 256 || K > (int64_t(1) << 30))
        return SVDQ_ERR_UNSUPPORTED;
    const int64_t m_tiles = (M + 127) / 128, n_tiles = (N + 255) / 256;
    if (m_tiles * n_tiles > 0x7FFFFFFF) return SVDQ_ERR_UNSUPPORTED;
    if (!aligned16(a_codes) || !aligned16(a_sf) || !aligned16(w_codes) || !aligned16(w_sf) || !aligned16(Y))
        return SVDQ_ERR_MISALIGNED;
    if (Y != nullptr && (ldy * (out_dtype ? 4 : 2)) % 16 != 0) return SVDQ_ERR_MISALIGNED;
    if (r > 0 && (!aligned16(D) || !aligned16(up))) return SVDQ_ERR_MISALIGNED;
    if (bias && !aligned16(bias)) return SVDQ_ERR_MISALIGNED;
    if (!device_is_sm100()) return SVDQ_ERR_NO_DEVICE;
    if (!debug_ptrs_ok({a_codes, a_sf, s_g_act, D, w_codes, w_sf, s_g_w, up, bias, Y})) return SVDQ_ERR_INVALID_ARG;
    uint32_t* err = device_error_word();
    if (err == nullptr) return SVDQ_ERR_CUDA;

    const int64_t row_bytes = mx ? K : K / 2;
    if (!encode_tmap_2d(ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a_codes, row_bytes, M, row_bytes, 128, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tmap_2d(tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w_codes, row_bytes, N, row_bytes, 128, 256,
                        CU_TENSOR_MAP_SWIZZLE_128B))
        return SVDQ_ERR_CUDA;
    // bf16 output boxes: 16 columns x 32 rows unswizzled (the plain epilogue's
    // 1 KB staging), or 64 x 32 with the 128-byte swizzle of the scoring
    // epilogue's reference strips
    *ty = *ta;
    if (out_dtype == 0 && Y != nullptr &&
        !encode_tmap_2d(ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Y, N, M, ldy * 2, score ? 64 : 16, 32,
                        score ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE))
        return SVDQ_ERR_CUDA;
    // Scale atoms viewed as [row block][atoms x 2 halves][256 bytes]: one box
    // holds the atoms of two stages (A: one row block, W: two).  NVFP4: K / 64
    // atoms per row block, 4 per stage; MXFP8: K / 128 atoms, 1 per stage.
    const uint64_t halves = mx ? static_cast<uint64_t>(K / 128) * 2 : static_cast<uint64_t>(K / 64) * 2;
    const uint32_t box_halves = mx ? 4 : 16;
    if (!encode_tmap_3d_u8(tsa, a_sf, 256, halves, static_cast<uint64_t>(m_tiles), 256, halves * 256, 256,
                           box_halves, 1) ||
        !encode_tmap_3d_u8(tsb, w_sf, 256, halves, static_cast<uint64_t>(N / 128), 256, halves * 256, 256,
                           box_halves, 2))
        return SVDQ_ERR_CUDA;
    *a = LinearArgs{};
    a->a_sf = a_sf;
    a->w_sf = w_sf;
    a->D = D;
    a->up = static_cast<const uint16_t*>(up);
    a->bias = static_cast<const uint16_t*>(bias);
    a->Y = Y;
    a->ldy = ldy;
    a->M = M;
    a->N = N;
    a->K = K;
    a->s_g_act = s_g_act;
    a->s_g_w = s_g_w;
    a->r = r;
    a->m_tiles = static_cast<int>(m_tiles);
    a->n_tiles = static_cast<int>(n_tiles);
    a->n_fastest = N <= M ? 1 : 0;                       // the weight is the smaller operand
    {
        // Bands of the fastest-walked operand no larger than kBandBytes (the
        // whole operand when it is smaller): each die's L2 half (~63 MB) must
        // hold the band and the other operand's blocks in flight.
        constexpr int64_t kBandBytes = int64_t(40) << 20;
        const int64_t fast_tiles = a->n_fastest ? n_tiles : m_tiles;
        const int64_t block_bytes = (a->n_fastest ? int64_t(kBN) : int64_t(kBM)) * row_bytes;
        const int64_t bands = (fast_tiles * block_bytes + kBandBytes - 1) / kBandBytes;
        a->band = static_cast<int>((fast_tiles + bands - 1) / bands);
    }
    a->err = err;
    a->write_y = Y != nullptr ? 1 : 0;
    a->ext_box_x = debug_extent(kSiteLinearBox, N);
    a->ext_box_y = M;
    a->ext_y32 = debug_extent(kSiteLinearF32, (M - 1) * ldy + N);
    return SVDQ_OK;
}

}  // namespace
}  // namespace svdq

extern "C" int svdq_linear(const uint8_t* a_codes, const uint8_t* a_sf, const float* s_g_act,
                           const float* D, int r,
                           const uint8_t* w_codes, const uint8_t* w_sf, const float* s_g_w,
                           const void* up, const void* bias,
                           void* Y, int64_t ldy, int out_dtype,
                           int64_t M, int64_t N, int64_t K, void* stream) {
    using namespace svdq;
    if (Y == nullptr) return SVDQ_ERR_INVALID_ARG;
    CUtensorMap ta, tb, ty, tsa, tsb;
    LinearArgs a;
    const int st0 = linear_prepare(a_codes, a_sf, s_g_act, D, r, w_codes, w_sf, s_g_w, up, bias, Y, ldy, out_dtype,
                                   M, N, K, &ta, &tb, &ty, &tsa, &tsb, &a);
    if (st0 != SVDQ_OK) return st0;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return out_dtype ? launch_linear<true, false>(ta, tb, ty, ta, tsa, tsb, a, st)
                     : launch_linear<false, false>(ta, tb, ty, ta, tsa, tsb, a, st);
}

extern "C" int svdq_linear_mxfp8(const uint8_t* a_codes, const uint8_t* a_sf, const uint8_t* w_codes,
                                 const uint8_t* w_sf, const void* bias, void* Y, int64_t ldy, int64_t M, int64_t N,
                                 int64_t K, void* stream) {
    using namespace svdq;
    if (Y == nullptr) return SVDQ_ERR_INVALID_ARG;
    CUtensorMap ta, tb, ty, tsa, tsb;
    LinearArgs a;
    const int st0 = linear_prepare(a_codes, a_sf, nullptr, nullptr, 0, w_codes, w_sf, nullptr, nullptr, bias, Y, ldy,
                                   0, M, N, K, &ta, &tb, &ty, &tsa, &tsb, &a, true);
    if (st0 != SVDQ_OK) return st0;
    return launch_linear<false, false, true>(ta, tb, ty, ta, tsa, tsb, a, static_cast<cudaStream_t>(stream));
}

extern "C" size_t svdq_linear_score_workspace_bytes(int n_seg) {
    if (n_seg < 1 || n_seg > svdq::kMaxSegments) return 0;
    return static_cast<size_t>(1024) * static_cast<size_t>(n_seg) * 2 * sizeof(double);
}

extern "C" int svdq_linear_score(const uint8_t* a_codes, const uint8_t* a_sf, const float* s_g_act,
                                 const float* D, int r,
                                 const uint8_t* w_codes, const uint8_t* w_sf, const float* s_g_w,
                                 const void* up, const void* bias,
                                 void* Y, int64_t ldy,
                                 const void* Yref, int64_t ldr,
                                 const svdq_seg* segs, int n_seg,
                                 double* num, double* den, double* rel,
                                 void* workspace, size_t workspace_bytes,
                                 int64_t M, int64_t N, int64_t K, void* stream) {
    using namespace svdq;
    if (Yref == nullptr || num == nullptr || den == nullptr || rel == nullptr || workspace == nullptr)
        return SVDQ_ERR_INVALID_ARG;
    if (segs == nullptr || n_seg < 1 || n_seg > kMaxSegments || ldr < N) return SVDQ_ERR_INVALID_ARG;
    if (!aligned16(Yref) || (ldr * 2) % 16 != 0 || (reinterpret_cast<uintptr_t>(workspace) & 7u) ||
        (reinterpret_cast<uintptr_t>(num) & 7u) || (reinterpret_cast<uintptr_t>(den) & 7u) ||
        (reinterpret_cast<uintptr_t>(rel) & 7u))
        return SVDQ_ERR_MISALIGNED;
    CUtensorMap ta, tb, ty, tsa, tsb;
    LinearArgs a;
    const int st0 = linear_prepare(a_codes, a_sf, s_g_act, D, r, w_codes, w_sf, s_g_w, up, bias, Y, ldy, 0, M, N,
                                   K, &ta, &tb, &ty, &tsa, &tsb, &a, false, true);
    if (st0 != SVDQ_OK) return st0;
    if (workspace_bytes < static_cast<size_t>(n_seg) * 2 * sizeof(double)) return SVDQ_ERR_INVALID_ARG;
    const int sst = make_seg_table(segs, n_seg, M, &a.segs);
    if (sst != SVDQ_OK) return sst;
    // The reference in strips of 64 columns x 128 rows, 128-byte swizzle (rows past M read as zeros).
    CUtensorMap tr;
    if (!encode_tmap_2d(&tr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Yref, N, M, ldr * 2, 64, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B))
        return SVDQ_ERR_CUDA;
    if (!debug_ptrs_ok({Yref, num, den, rel, workspace})) return SVDQ_ERR_INVALID_ARG;
    a.seg_part = static_cast<double*>(workspace);
    a.num = num;
    a.den = den;
    a.rel = rel;
    a.ext_part = debug_extent(kSiteLinearScore, static_cast<int64_t>(workspace_bytes / sizeof(double)));
    a.ext_seg = n_seg;
    return launch_linear<false, true>(ta, tb, ty, tr, tsa, tsb, a, static_cast<cudaStream_t>(stream),
                                      workspace_bytes);
}
