// quantize.cu -- per-token NVFP4 quantisation of smoothed activations, fused
// with the low-rank down-projection D = X down^T = (X / lambda) L1.
//
// "MiniMax-H3 NVFP4 -- what the smoothing scale should be calibrated on",
// section "Why": 16 consecutive input channels share one FP8 (E4M3) scale set
// by the group absmax, and the kernel sees X / lambda.  "MiniMax-H3 . SVDQuant
// W4A4 (int4, rank 32, GPTQ)", opening section: activations are quantised per
// token at run time and a 16-bit rank-32 branch carries the outliers.
// "DeltaQuant on MiniMax-H3", section "The activation scale bound held": the
// tensor scale is static and saturated groups are counted at run time.
//
// Work split: the rows are cut into G groups of R consecutive rows (R <= 112,
// the last group shorter) and K into S slices of consecutive 64-channel chunks
// (S <= 4, the CTAs of one thread-block cluster): one CTA per (group, slice).
// R and S are chosen so that G * S comes close to the SM count (at most one
// CTA fits per SM), with no more clusters than fit at once: 128 CTAs of 128
// rows at 4096 rows (S = 4: 32 clusters of 4 fit, 37 do not), 147 of 112 rows
// at 16384 rows (S = 1), 140 of 88 rows at 12288 rows.  Whole 128-row tiles
// would leave 20 to 52 SMs without work at the larger sizes.  The partial D
// tiles of a cluster are summed in cluster-rank order through distributed
// shared memory, so D is deterministic.  Without a split along K (S = 1) the
// CTA needs no D partial in shared memory: its room goes to a deeper ring of
// 12 stages of 112-row slots, and D goes from tensor memory to global memory.
//
// Layout of one CTA (30 warps) over its group's rows and its slice of K:
//   warp 28      TMA producer: R x 64 bf16 tiles of X (128-byte swizzle), the
//                matching r x 64 tile of the down weight and 64 values of
//                1/lambda into an 8-stage ring, or the 12-stage one without a
//                split (a multiple of the 4 quantiser teams)
//   warp 29      tcgen05 issuer: D_partial(tmem, fp32) += X_tile * down_tile^T
//                (M = 128: rows of a stage slot past R are never stored)
//   warps 0..27  quantisers, in four teams of 7 that take the stages in
//                turn (the time per stage is set by how many stages are being
//                quantised at once, not by the rows of a stage: four teams of
//                112 rows beat three of 128); a lane owns one 16-channel group in each of two rows
//                (two independent dependency chains), reads them from the
//                swizzled tile, multiplies by 1/lambda and later by 1/S with
//                packed f32x2 multiplies, forms the E4M3 scales of both rows
//                with one conversion and the E2M1 codes with the hardware RNE
//                conversions, and stores 8-byte code words and 4-byte scale
//                words; 1/S comes from a per-CTA table over the 127 finite
//                non-negative E4M3 bytes (S = RN(dec(byte) * s_g), 1/S = RN(1/S)),
//                built once at CTA start;
//                warps 0..3 (one per tensor-memory lane quarter) finally read
//                D_partial from tensor memory (and, without a split, store it).
// The kernel is a programmatic dependent of the one before it in the stream:
// barrier set-up, tensor-memory allocation and the tensor-map prefetch run
// before griddepcontrol.wait, and it lets its own dependent (the linear) start
// launching at once.  Memory traffic per element: 2 bytes in, 0.5625 out.
#include "common.cuh"
#include "sm100.cuh"

namespace svdq {
namespace {

constexpr int kBM = 128;               // rows of a stage slot (the MMA's M); a group holds at most this many
constexpr int kBK = 64;                // channels per stage (128 bytes of bf16)
// Quantiser teams take the stages in turn; each warp of a team takes 16 rows
// of a stage (4 groups of 16 channels).  Groups of up to 112 rows: four teams
// of 7 warps over an 8-stage ring; of up to 128 rows: three teams of 8 over 9
// stages (the host picks by the rows; a template parameter, so the ring and
// team arithmetic stays constant).  The time per stage is set by how many
// stages are being quantised at once, so the four-team shape is the faster one,
// and the deep ring (12 stages, no split) faster still: more stages in flight.
constexpr int kStages = 9;            // ring slots laid out (the 4-team shape uses 8)
constexpr int kQuantWarps = 28;
constexpr int kGroupRows = 7 * 16;    // rows a group holds with four teams
constexpr int kProducerWarp = kQuantWarps;
constexpr int kMmaWarp = kQuantWarps + 1;
constexpr int kThreads = (kQuantWarps + 2) * 32;
// Stage i sits in slot i % stages and is quantised by team i % teams.  A
// parity wait only tells the current phase from the one before it, so a slot
// must always be consumed by the same team (stages is a multiple of teams):
// otherwise a team a whole ring lap ahead could take the slot's unfinished
// phase for its own (completed) one.
static_assert(kStages % 3 == 0 && 8 <= kStages && 4 * 7 <= kQuantWarps && 3 * 8 <= kQuantWarps,
              "both team shapes fit the warps and the ring");
constexpr int kMaxSplit = 4;          // CTAs of a cluster along K
constexpr int kDeepStages = 12;       // the deep ring: groups of <= 112 rows, no split along K

// Shared-memory layout: kNumStages slots of kSlotRows x 64 bf16 of X (the MMA
// reads 128 rows from a slot; rows past the group's are never stored, and a
// 112-row slot's last ones lie in the next slot or, for the last slot, in the
// down tiles: in bounds either way), the matching down tiles, the D partial
// when a cluster sums D along K (kPart), 1/lambda per stage, the 1/S table and
// the barriers.
template <int R, int kSlotRows, int kNumStages, bool kPart>
struct QSmem {
    static constexpr uint32_t kXTile = kSlotRows * kBK * 2;                        // 16 or 14 KB (1 KB multiples)
    static constexpr int kStagesL = kNumStages;
    static constexpr uint32_t kDownTileBytes = R * kBK * 2;
    static constexpr uint32_t kXOff = 0;
    static constexpr uint32_t kDownOff = kNumStages * kXTile;
    static constexpr uint32_t kPartStride = R + 4;                                 // floats per row (padded)
    static constexpr uint32_t kPartOff = kDownOff + kNumStages * kDownTileBytes;  // D partial [128][R + 4] fp32
    static constexpr uint32_t kIlamOff = kPartOff + (kPart && R > 0 ? kBM * kPartStride * 4 : 0);   // 1/lambda, 64 fp32 per stage
    static constexpr uint32_t kTabOff = kIlamOff + kNumStages * kBK * 4;           // 1/S per E4M3 byte, 128 fp32
    static constexpr uint32_t kBarOff = kTabOff + 128 * 4;                         // full, empty [kNumStages], dfull, ...
    static constexpr uint32_t kBytes = kBarOff + 256;
    static_assert(kXTile % 1024 == 0, "slots keep the 128-byte swizzle's 1 KB alignment");
    static_assert(2 * kNumStages * 8 + 24 <= 256, "the barriers fit their area");
    static_assert(kBytes + 1024 <= 232448, "fits the 227 KB opt-in shared memory of one CTA");
};

// The three shapes: kTeamWarps = 8 (three teams, 9 stages of 128-row slots);
// kTeamWarps = 7 (four teams, 8 of the 9 laid-out stages); kDeep (four teams of 7
// over 12 stages of 112-row slots, no D partial in shared memory: D goes from
// tensor memory straight to global memory, so only without a split along K).
template <int R, int kTeamWarps, bool kDeep>
using QLayout = QSmem<R, kDeep ? kGroupRows : kBM, kDeep ? kDeepStages : kStages, !kDeep>;

struct QuantArgs {
    const float* inv_lambda;
    const float* s_g;
    int64_t M, K;
    uint8_t* codes;
    uint8_t* sf;
    float* D;
    uint32_t* sat_count;
    uint32_t* err;
    int64_t ext_codes, ext_sf, ext_d;   // store-check extents (debug library): M K / 2 bytes, the scale bytes, M R floats
    int n_chunks;      // K / 64
    int split;         // CTAs along K (cluster size when R > 0)
    int rows;          // rows per group (the TMA box height), <= 128
};

__device__ __forceinline__ float4 ld_dsmem_f32x4(uint32_t local_addr, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(remote) : "memory");
    return v;
}

// E4M3 scale byte and saturation (t > 448) of t = RN(a / d), a >= 0, d > 0.  With y = RN(1 / d): |a y - a / d| <= 2^-24 a / d < 1 ulp,
// rounding a y to q adds at most 1/2 ulp and t is within 1/2 ulp of a / d, so
// |q - t| < 2 ulp (a power-of-two boundary between them only widens the
// bit-pattern steps used below).  E4M3 rounding and the test t > 448 are
// monotonic in t: when the floats 3 steps below and above q give the same byte
// and the same test, t gives them too.  Otherwise -- near a rounding boundary
// of the byte, at 448, or for a = 0 -- the exact quotient decides.
__device__ __forceinline__ uint32_t scale_byte_checked(float a, float d, float rd, uint32_t& sat) {
    const float q = __fmul_rn(a, rd);
    const uint32_t qb = __float_as_uint(q);
    const float lo = __uint_as_float(qb - 3u), hi = __uint_as_float(qb + 3u);
    const uint32_t b2 = cvt_e4m3x2(lo, hi);
    const bool sat_lo = lo > 448.0f, sat_hi = hi > 448.0f;
    if (a != 0.0f && qb >= 3u && (b2 & 0xFFu) == (b2 >> 8) && sat_lo == sat_hi) {
        sat += sat_lo ? 1u : 0u;
        return b2 & 0xFFu;
    }
    const float t = __fdiv_rn(a, d);
    sat += t > 448.0f ? 1u : 0u;
    return cvt_e4m3x2(t, 0.0f) & 0xFFu;
}

template <int R, int kTeamWarps, bool kDeep>
__global__ void __launch_bounds__(kThreads)
quantize_act_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_down,
                    QuantArgs args) {
    using L = QLayout<R, kTeamWarps, kDeep>;
    static_assert(kTeamWarps == 7 || kTeamWarps == 8, "the two team shapes");
    static_assert(!kDeep || kTeamWarps == 7, "the deep ring is laid out for 112-row groups");
    constexpr int kTeams = kQuantWarps / kTeamWarps;                 // 4 or 3
    constexpr int kStagesT = kDeep ? kDeepStages : (kTeamWarps == 7 ? 8 : 9);   // a multiple of the teams
    static_assert(kStagesT % kTeams == 0 && kStagesT <= L::kStagesL, "every slot is consumed by one team");
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
    uint64_t* empty = full + L::kStagesL;
    uint64_t* dfull = empty + L::kStagesL;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(dfull + 1);
    volatile uint32_t* abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5;
    const uint32_t lane = threadIdx.x & 31;
    const int64_t row_base = static_cast<int64_t>(blockIdx.x) * args.rows;   // first row of this group
    // Box rows that are real rows or zero fill inside the scale array's 128-row
    // padding (their scale bytes are written); rows of the box at or past M are
    // zero-filled by TMA.
    const int64_t m_pad = (args.M + 127) / 128 * 128;
    const int box_rows = static_cast<int>(min(static_cast<int64_t>(args.rows), m_pad - row_base));
    const int ky = blockIdx.y;
    const int c_begin = static_cast<int>(static_cast<int64_t>(ky) * args.n_chunks / args.split);
    const int c_end = static_cast<int>(static_cast<int64_t>(ky + 1) * args.n_chunks / args.split);
    const int n_local = c_end - c_begin;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStagesT; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kTeamWarps + (R > 0 ? 1 : 0));
        }
        mbar_init(dfull, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (R > 0 && warp == kMmaWarp) {
        tmem_alloc(tmem_slot, 32);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_d = (R > 0) ? *tmem_slot : 0u;
    pdl_launch_dependents();                  // the next kernel's set-up may overlap this one

    if (warp == kProducerWarp) {
        if (lane == 0) {
            prefetch_tmap(&tmap_x);
            if (R > 0) prefetch_tmap(&tmap_down);
            pdl_wait();                           // X, 1/lambda and the tensor scale are written
            const uint32_t x_bytes = static_cast<uint32_t>(args.rows) * kBK * 2;
            int issued = 0;
            for (int i = 0; i < n_local; ++i) {
                const int s = i % kStagesT;
                const uint32_t ph = (i / kStagesT) & 1;
                if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, args.err, kErrWaitEmpty)) break;
                const int col = (c_begin + i) * kBK;
                mbar_arrive_expect_tx(&full[s], x_bytes + L::kDownTileBytes + (args.inv_lambda ? kBK * 4 : 0));
                if (args.inv_lambda)
                    bulk_load(smem + L::kIlamOff + s * kBK * 4, args.inv_lambda + col, kBK * 4, &full[s]);
                tma_load_2d(smem + L::kXOff + s * L::kXTile, &tmap_x, &full[s], col,
                            static_cast<int32_t>(row_base));
                if (R > 0)
                    tma_load_2d(smem + L::kDownOff + s * L::kDownTileBytes, &tmap_down, &full[s], col, 0);
                ++issued;
            }
            // Wait (bounded) for the copies still in flight before the CTA may exit.
            for (int i = (issued > kStagesT ? issued - kStagesT : 0); i < issued; ++i) {
                const long long t0 = clock64();
                while (!mbar_try_wait(&full[i % kStagesT], (i / kStagesT) & 1) &&
                       clock64() - t0 < kWaitLimitCycles) {}
            }
        }
    } else if (warp == kMmaWarp) {
        if (R > 0 && lane == 0) {
            const uint32_t idesc = idesc_bf16(kBM, R);
            for (int i = 0; i < n_local; ++i) {
                const int s = i % kStagesT;
                const uint32_t ph = (i / kStagesT) & 1;
                if (!mbar_wait(&full[s], ph, abort_flag, args.err, kErrWaitFull)) break;
                tc_fence_after();
                const uint32_t a0 = smem_u32(smem + L::kXOff + s * L::kXTile);
                const uint32_t b0 = smem_u32(smem + L::kDownOff + s * L::kDownTileBytes);
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk)
                    mma_bf16(tmem_d, desc_kmajor_sw128(a0 + kk * 32), desc_kmajor_sw128(b0 + kk * 32), idesc,
                             (i > 0 || kk > 0) ? 1u : 0u);
                tc_commit(&empty[s]);
            }
            tc_commit(dfull);
        }
    } else {
        // ------------------------------------------------------------ quantisers
        pdl_wait();                               // the tensor scale is written
        if (threadIdx.x < 128) {
            // 1/S for every scale byte the RNE-satfinite conversion can produce (0x00..0x7E).
            const float s_g0 = __ldg(args.s_g);
            const float S = __fmul_rn(e4m3_to_f32(threadIdx.x), s_g0);
            reinterpret_cast<float*>(smem + L::kTabOff)[threadIdx.x] =
                (threadIdx.x == 0x7F || S == 0.0f) ? 0.0f : __frcp_rn(S);
        }
        asm volatile("bar.sync 1, %0;" :: "n"(kQuantWarps * 32) : "memory");
        const float s_g = __ldg(args.s_g);
        const float d = __fmul_rn(6.0f, s_g);
        const float rd = __frcp_rn(d);
        const int64_t M = args.M;
        const int64_t half_k = args.K >> 1;
        const int64_t atoms_k = args.K >> 6;
        const bool has_il = args.inv_lambda != nullptr;
        const float* rs_tab = reinterpret_cast<const float*>(smem + L::kTabOff);
        uint32_t sat = 0;
        // Team (stage parity), rows and group of this lane: rows r0 and r0 + 8
        // of the tile, channels 16 b .. 16 b + 15 of the stage; the group's two
        // 16-byte halves are chunks 2b and 2b+1 of the row's 128-byte line
        // (both rows have the same swizzle phase, r0 % 8 == (r0 + 8) % 8).
        const int team = warp / kTeamWarps;      // >= teams: a spare warp, no stages
        const int rw = lane >> 2;
        const int b = lane & 3;
        const int r0 = (warp % kTeamWarps) * 16 + rw;
        const int r1 = r0 + 8;
        const int64_t grow0 = row_base + r0;
        const int64_t grow1 = grow0 + 8;
        // rows past the box hold stale shared memory: nothing of them is stored or counted
        const bool box0 = r0 < box_rows, box1 = r1 < box_rows;
        const bool code0 = box0 && grow0 < M, code1 = box1 && grow1 < M;
        const int ph0 = ((2 * b) ^ (r0 & 7)) << 4;
        const int ph1 = ((2 * b + 1) ^ (r0 & 7)) << 4;
        const uint64_t one2 = pack_f32x2(1.0f, 1.0f);
        // A warp whose 16 rows all lie past this group's box has nothing to
        // quantise: it only keeps the ring's protocol (wait for each of its
        // team's stages, release it), so the work per stage follows the rows.
        const bool idle = (warp % kTeamWarps) * 16 >= box_rows;
        for (int i = team < kTeams ? team : n_local; i < n_local; i += kTeams) {
            const int s = i % kStagesT;
            const uint32_t ph = (i / kStagesT) & 1;
            if (!mbar_wait(&full[s], ph, abort_flag, args.err, kErrWaitFull)) break;
            if (idle) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
                continue;
            }
            const int chunk = c_begin + i;
            const uint8_t* tile = smem + L::kXOff + s * L::kXTile;
            const uint4 u0 = *reinterpret_cast<const uint4*>(tile + r0 * 128 + ph0);
            const uint4 u1 = *reinterpret_cast<const uint4*>(tile + r0 * 128 + ph1);
            const uint4 v0 = *reinterpret_cast<const uint4*>(tile + (r0 + 8) * 128 + ph0);
            const uint4 v1 = *reinterpret_cast<const uint4*>(tile + (r0 + 8) * 128 + ph1);
            uint64_t il[8];
            if (has_il) {
                const ulonglong2* ilp = reinterpret_cast<const ulonglong2*>(smem + L::kIlamOff + s * kBK * 4 + b * 64);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const ulonglong2 t = ilp[q];
                    il[2 * q] = t.x;
                    il[2 * q + 1] = t.y;
                }
            } else {
#pragma unroll
                for (int q = 0; q < 8; ++q) il[q] = one2;
            }
            const uint32_t wa[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
            const uint32_t wb[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            // xs = RN(x * (1/lambda)), element pairs (2j, 2j+1) of each row
            uint64_t xa[8], xb[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                xa[j] = mul_f32x2(bf16x2_to_f32x2(wa[j]), il[j]);
                xb[j] = mul_f32x2(bf16x2_to_f32x2(wb[j]), il[j]);
            }
            const float aa = absmax16(xa), ab = absmax16(xb);
            // Scale bytes and saturation of both rows from t = RN(a / d), through
            // the product with 1/d where that is provably the same (see scale_from_amax).
            uint32_t sat_a = 0, sat_b = 0;
            const uint32_t sf2 = scale_byte_checked(aa, d, rd, sat_a) |
                                 (scale_byte_checked(ab, d, rd, sat_b) << 8);   // byte 0: row r0, byte 1: row r0 + 8
            const float rsa = rs_tab[sf2 & 0xFFu], rsb = rs_tab[sf2 >> 8];
            const uint64_t ra = pack_f32x2(rsa, rsa), rb = pack_f32x2(rsb, rsb);
            uint64_t qa[8], qb[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                qa[j] = mul_f32x2(xa[j], ra);
                qb[j] = mul_f32x2(xb[j], rb);
            }
            const uint2 ca = make_uint2(cvt_e2m1x8_pairs(qa[0], qa[1], qa[2], qa[3]),
                                        cvt_e2m1x8_pairs(qa[4], qa[5], qa[6], qa[7]));
            const uint2 cb = make_uint2(cvt_e2m1x8_pairs(qb[0], qb[1], qb[2], qb[3]),
                                        cvt_e2m1x8_pairs(qb[4], qb[5], qb[6], qb[7]));
            sat += (box0 ? sat_a : 0u) + (box1 ? sat_b : 0u);
            // scale words of both rows: bytes of lanes 4 rw .. 4 rw + 3 (groups b = 0..3)
            const uint32_t n1 = __shfl_down_sync(0xffffffffu, sf2, 1);
            const uint32_t n2 = __shfl_down_sync(0xffffffffu, sf2, 2);
            const uint32_t n3 = __shfl_down_sync(0xffffffffu, sf2, 3);
            const uint32_t x01 = __byte_perm(sf2, n1, 0x5140);   // a0 b0 a1 b1
            const uint32_t x23 = __byte_perm(n2, n3, 0x5140);    // c0 d0 c1 d1
            consumed(ca.x, ca.y, cb.x, cb.y);            // every loaded value of the stage is in these
            consumed(x01, x23);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);        // shared memory of this stage no longer read
            const int64_t coff = chunk * (kBK / 2) + b * 8;
            if (code0 && store_ok(coff + grow0 * half_k, 8, args.ext_codes, args.err, kSiteQuantCodes))
                *reinterpret_cast<uint2*>(args.codes + coff + grow0 * half_k) = ca;
            if (code1 && store_ok(coff + grow1 * half_k, 8, args.ext_codes, args.err, kSiteQuantCodes))
                *reinterpret_cast<uint2*>(args.codes + coff + grow1 * half_k) = cb;
            if (b == 0) {
                // a row's word in its 128-row block's 512-byte atom of this chunk
                const int64_t o0 = ((grow0 >> 7) * atoms_k + chunk) * 512 + (grow0 & 31) * 16 + ((grow0 >> 5) & 3) * 4;
                const int64_t o1 = ((grow1 >> 7) * atoms_k + chunk) * 512 + (grow1 & 31) * 16 + ((grow1 >> 5) & 3) * 4;
                if (box0 && store_ok(o0, 4, args.ext_sf, args.err, kSiteQuantSf))
                    *reinterpret_cast<uint32_t*>(args.sf + o0) = __byte_perm(x01, x23, 0x5410);
                if (box1 && store_ok(o1, 4, args.ext_sf, args.err, kSiteQuantSf))
                    *reinterpret_cast<uint32_t*>(args.sf + o1) = __byte_perm(x01, x23, 0x7632);
            }
        }
        // Padding rows of the scale array past the last group's box (the box ends
        // before the 128-row boundary): zero scale words for this CTA's chunks.
        if (row_base + args.rows < m_pad && row_base + args.rows >= M) {
            const int64_t pad0 = row_base + args.rows;
            const int64_t n_pad = (m_pad - pad0) * n_local;
            for (int64_t t = threadIdx.x; t < n_pad; t += kQuantWarps * 32) {
                const int64_t row = pad0 + t / n_local;
                const int64_t chunk = c_begin + t % n_local;
                const int64_t off = ((row >> 7) * atoms_k + chunk) * 512 + (row & 31) * 16 + ((row >> 5) & 3) * 4;
                if (store_ok(off, 4, args.ext_sf, args.err, kSiteQuantSf))
                    *reinterpret_cast<uint32_t*>(args.sf + off) = 0u;
            }
        }
        // saturation count: one atomic per warp
        for (int o = 16; o > 0; o >>= 1) sat += __shfl_xor_sync(0xffffffffu, sat, o);
        if (lane == 0 && sat && args.sat_count) atomicAdd(args.sat_count, sat);

        if (kDeep && R > 0 && warp < 4) {
            // No split along K: this CTA's D rows go from tensor memory straight to
            // global memory (one warp per lane quarter, a thread per row).
            const int row = warp * 32 + lane;
            const int64_t grow = row_base + row;
            const bool row_ok = row < args.rows && grow < args.M;
            if (mbar_wait(dfull, 0, abort_flag, args.err, kErrWaitMma)) {
                tc_fence_after();
                const uint32_t taddr = tmem_d + (static_cast<uint32_t>(warp * 32) << 16);
                uint32_t v[R > 16 ? 32 : 16];
                if constexpr (R == 32) tmem_ld_32x32b_x32(taddr, v);
                else tmem_ld_32x32b_x16(taddr, v);
                tmem_ld_wait(v);
                if (row_ok) {
                    float4* dst = reinterpret_cast<float4*>(args.D + grow * R);
#pragma unroll
                    for (int q = 0; q < R / 4; ++q)
                        if (store_ok(grow * R + 4 * q, 4, args.ext_d, args.err, kSiteQuantD))
                            dst[q] = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                                 __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
                }
            }
            tc_fence_before();
        } else if (R > 0 && warp < 4) {   // one warp per tensor-memory lane quarter
            float* part = reinterpret_cast<float*>(smem + L::kPartOff) + (warp * 32 + lane) * L::kPartStride;
            if (mbar_wait(dfull, 0, abort_flag, args.err, kErrWaitMma)) {
                tc_fence_after();
                const uint32_t taddr = tmem_d + (static_cast<uint32_t>(warp * 32) << 16);
                if constexpr (R == 32) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(taddr, v);
                    tmem_ld_wait(v);
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<float4*>(part + j) = make_float4(
                            __uint_as_float(v[j]), __uint_as_float(v[j + 1]), __uint_as_float(v[j + 2]),
                            __uint_as_float(v[j + 3]));
                } else {
                    uint32_t v[16];
                    tmem_ld_32x32b_x16(taddr, v);
                    tmem_ld_wait(v);
#pragma unroll
                    for (int j = 0; j < 16; j += 4)
                        *reinterpret_cast<float4*>(part + j) = make_float4(
                            __uint_as_float(v[j]), __uint_as_float(v[j + 1]), __uint_as_float(v[j + 2]),
                            __uint_as_float(v[j + 3]));
                }
            } else {
#pragma unroll
                for (int j = 0; j < R; ++j) part[j] = 0.0f;
            }
            tc_fence_before();
        }
    }

    __syncwarp();   // reconverge each warp before the warp-aligned cluster barrier
    if constexpr (R > 0) {
        // Sum the split-K partials in cluster-rank order (deterministic).  Every
        // CTA of the cluster takes a share of the ranks (in groups of 4): it
        // issues all its 16-byte loads from the peers' shared memory first and
        // then adds them, so the loads' latencies overlap.
        cluster_sync_all();
        if (!kDeep && warp < 4) {
            constexpr int kNq = R / 4;                           // float4 groups per row
            constexpr int kMaxQ = (kNq + 1) / 2 + 1;             // groups one CTA takes (split >= 2), or all
            const int split = args.split;
            const int cr = static_cast<int>(cluster_ctarank());
            const int q0 = cr * kNq / split, q1 = (cr + 1) * kNq / split;
            const int row = warp * 32 + lane;
            const int64_t grow = row_base + row;
            const bool row_ok = row < args.rows && grow < args.M;
            const uint32_t base = smem_u32(smem + L::kPartOff) + row * L::kPartStride * 4;
            if (split == 1) {
                if (row_ok) {
                    const float4* src = reinterpret_cast<const float4*>(smem + L::kPartOff) + row * (L::kPartStride / 4);
                    float4* dst = reinterpret_cast<float4*>(args.D + grow * R);
#pragma unroll
                    for (int q = 0; q < kNq; ++q)
                        if (store_ok(grow * R + 4 * q, 4, args.ext_d, args.err, kSiteQuantD)) dst[q] = src[q];
                }
            } else {
                // two groups at a time: at most 8 remote 16-byte loads in flight per thread
                for (int t0 = 0; t0 < kMaxQ; t0 += 2) {
                    float4 got[2][kMaxSplit];
#pragma unroll
                    for (int t = 0; t < 2; ++t)
#pragma unroll
                        for (int c = 0; c < kMaxSplit; ++c)
                            if (q0 + t0 + t < q1 && c < split)
                                got[t][c] = ld_dsmem_f32x4(base + (q0 + t0 + t) * 16, c);
                    if (row_ok) {
                        float4* dst = reinterpret_cast<float4*>(args.D + grow * R);
#pragma unroll
                        for (int t = 0; t < 2; ++t) {
                            if (q0 + t0 + t < q1) {
                                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                                for (int c = 0; c < kMaxSplit; ++c) {
                                    if (c < split) {
                                        acc.x += got[t][c].x; acc.y += got[t][c].y;
                                        acc.z += got[t][c].z; acc.w += got[t][c].w;
                                    }
                                }
                                if (store_ok(grow * R + 4 * (q0 + t0 + t), 4, args.ext_d, args.err, kSiteQuantD))
                                    dst[q0 + t0 + t] = acc;
                            }
                        }
                    }
                }
            }
        }
        cluster_sync_all();
        if (warp == kMmaWarp) {
            tc_fence_after();
            tmem_dealloc(tmem_d, 32);
        }
    }
}

// Work split of an M x K problem over `sms` SMs (one CTA fits per SM): K slices
// per row group (a cluster, at most 4, only when whole 128-row tiles leave SMs
// for it) and rows per group (at most 128, at least 16 where M allows) so that
// groups x slices comes as close to the SM count as the rows allow.
struct QuantPlan {
    int split;
    int rows;
    int64_t groups;
};

inline QuantPlan plan_quantize(int64_t M, int n_chunks, int64_t sms, int64_t max_clusters) {
    QuantPlan p{};
    const int64_t m_tiles = (M + kBM - 1) / kBM;
    const int64_t per_tile = sms / m_tiles;
    p.split = static_cast<int>(per_tile < 1 ? 1 : (per_tile > kMaxSplit ? kMaxSplit : per_tile));
    if (p.split > n_chunks) p.split = n_chunks;
    int64_t groups_max = sms / p.split > 0 ? sms / p.split : 1;
    // clusters are placed whole inside a GPC: never more than fit at once
    if (p.split > 1 && max_clusters > 0 && groups_max > max_clusters) groups_max = max_clusters;
    int64_t rows = (M + groups_max - 1) / groups_max;
    rows = (rows + 7) / 8 * 8;                    // whole 8-row swizzle groups
    if (rows > kBM) rows = kBM;                   // more rows than one wave holds: whole 128-row groups
    if (rows > M) rows = M;
    p.rows = static_cast<int>(rows);
    p.groups = (M + rows - 1) / rows;
    return p;
}

template <int R>
int launch_quantize(const void* X, int64_t M, int64_t K, int64_t ldx, const QuantArgs& base, const void* down,
                    cudaStream_t st) {
    QuantArgs a = base;
    a.n_chunks = static_cast<int>(K / kBK);
    const int64_t sms = device_sm_count() > 0 ? device_sm_count() : 148;
    // The three-team and the four-team shape share threads and shared memory
    // (the ring is laid out for 9 stages), so the cluster occupancy below holds
    // for either; the deep shape runs without clusters.
    const uint32_t smem = QLayout<R, 8, false>::kBytes + 1024;
    const uint32_t smem_deep = QLayout<R, 7, true>::kBytes + 1024;
    auto kern4 = quantize_act_kernel<R, 7, false>;
    auto kern3 = quantize_act_kernel<R, 8, false>;
    auto kern_deep = quantize_act_kernel<R, 7, true>;
    static std::atomic<uint64_t> smem_set4{0}, smem_set3{0}, smem_set_deep{0};
    if (!set_dynamic_smem_once(kern4, smem, smem_set4) || !set_dynamic_smem_once(kern3, smem, smem_set3) ||
        !set_dynamic_smem_once(kern_deep, smem_deep, smem_set_deep))
        return SVDQ_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    // clusters of 4 along K that fit on the device at once (0: unknown)
    int max_clusters = 0;
    if (R > 0) {
        cfg.gridDim = dim3(1, kMaxSplit, 1);
        attr[0].val.clusterDim.y = kMaxSplit;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&max_clusters, kern3, &cfg) != cudaSuccess) max_clusters = 0;
    }
    const QuantPlan plan = plan_quantize(M, a.n_chunks, sms, max_clusters);
    if (plan.groups > 0x7FFFFFFF) return SVDQ_ERR_UNSUPPORTED;
    a.split = plan.split;
    a.rows = plan.rows;

    CUtensorMap tx, td;
    if (!encode_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, K, M, ldx * 2, kBK,
                        static_cast<uint32_t>(plan.rows), CU_TENSOR_MAP_SWIZZLE_128B))
        return SVDQ_ERR_CUDA;
    if (R > 0) {
        if (!encode_tmap_2d(&td, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, down, K, R, K * 2, kBK, R,
                            CU_TENSOR_MAP_SWIZZLE_128B))
            return SVDQ_ERR_CUDA;
    } else {
        td = tx;
    }

    cfg.gridDim = dim3(static_cast<unsigned>(plan.groups), static_cast<unsigned>(plan.split), 1);
    attr[0].val.clusterDim.y = (R > 0) ? plan.split : 1;
    cfg.numAttrs = 2;
    // groups of up to 112 rows whose D needs no sum across a cluster: the deep ring
    if (plan.rows <= kGroupRows && (R == 0 || plan.split == 1)) {
        cfg.dynamicSmemBytes = smem_deep;
        return launch_status(cudaLaunchKernelEx(&cfg, kern_deep, tx, td, a));
    }
    return launch_status(plan.rows <= kGroupRows ? cudaLaunchKernelEx(&cfg, kern4, tx, td, a)
                                                 : cudaLaunchKernelEx(&cfg, kern3, tx, td, a));
}

}  // namespace
}  // namespace svdq

extern "C" int svdq_quantize_act(const void* X, int64_t M, int64_t K, int64_t ldx,
                                 const float* inv_lambda, const float* s_g,
                                 const void* down, int r,
                                 uint8_t* codes, uint8_t* sf, float* D, uint32_t* sat_count,
                                 void* stream) {
    using namespace svdq;
    if (X == nullptr || codes == nullptr || sf == nullptr || s_g == nullptr) return SVDQ_ERR_INVALID_ARG;
    if (M < 1 || K < 64 || ldx < K) return SVDQ_ERR_INVALID_ARG;
    if (K % 64 != 0) return SVDQ_ERR_UNSUPPORTED;
    if (reinterpret_cast<uintptr_t>(s_g) & 3u) return SVDQ_ERR_MISALIGNED;
    if (r != 0 && r != 16 && r != 32) return SVDQ_ERR_UNSUPPORTED;
    if ((r > 0) != (down != nullptr) || (r > 0) != (D != nullptr)) return SVDQ_ERR_INVALID_ARG;
    if (M > (int64_t(1) << 31) - 128 || K > (int64_t(1) << 30)) return SVDQ_ERR_UNSUPPORTED;
    if (!aligned16(X) || (ldx * 2) % 16 != 0 || !aligned16(codes) || !aligned16(sf)) return SVDQ_ERR_MISALIGNED;
    if (inv_lambda && !aligned16(inv_lambda)) return SVDQ_ERR_MISALIGNED;
    if (r > 0 && (!aligned16(down) || !aligned16(D))) return SVDQ_ERR_MISALIGNED;
    if (sat_count && (reinterpret_cast<uintptr_t>(sat_count) & 3u)) return SVDQ_ERR_MISALIGNED;
    if (!device_is_sm100()) return SVDQ_ERR_NO_DEVICE;
    if (!debug_ptrs_ok({X, inv_lambda, s_g, down, codes, sf, D, sat_count})) return SVDQ_ERR_INVALID_ARG;
    uint32_t* err = device_error_word();
    if (err == nullptr) return SVDQ_ERR_CUDA;
    QuantArgs a{};
    a.inv_lambda = inv_lambda;
    a.s_g = s_g;
    a.M = M;
    a.K = K;
    a.codes = codes;
    a.sf = sf;
    a.D = D;
    a.sat_count = sat_count;
    a.err = err;
    a.ext_codes = debug_extent(kSiteQuantCodes, M * (K / 2));
    a.ext_sf = debug_extent(kSiteQuantSf, static_cast<int64_t>(svdq_sf_bytes(M, K)));
    a.ext_d = debug_extent(kSiteQuantD, M * r);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // Rows of the last 128-row block beyond M hold zero scale bytes: the kernel
    // writes every row of every tile (zero-filled by TMA), so no memset is needed.
    switch (r) {
        case 0: return launch_quantize<0>(X, M, K, ldx, a, down, st);
        case 16: return launch_quantize<16>(X, M, K, ldx, a, down, st);
        default: return launch_quantize<32>(X, M, K, ldx, a, down, st);
    }
}
