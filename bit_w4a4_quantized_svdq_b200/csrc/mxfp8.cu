// mxfp8.cu -- MXFP8 quantisation for the W8A8 variant of the linear.
//
// "MiniMax-H3 -- MXFP8 (weight-quantized, vLLM-Omni native layout)", section
// "Quant format": OCP microscaling FP8, E4M3 elements with one E8M0 scale per 32
// consecutive elements, symmetric round-to-nearest; weights quantised once,
// activations dynamically per token and 32 channels.  Per block:
//
//   e     = floor(log2 amax) - 8, clamped to [-127, 127]; -127 for an all-zero block
//   scale = e + 127 (E8M0 byte)
//   code  = E4M3(v * 2^-e), nearest, ties to even, saturating at 448, sign kept
//
// floor(log2 amax) is the unbiased exponent of amax (a bf16 value, exact in
// fp32); amax below the normal range gives e < -127 and so -127.  2^-e is built
// from its exponent bits (e <= 119 for any bf16 input, so it is a normal fp32),
// which makes v * 2^-e exact up to fp32 underflow, where E4M3 rounds to zero anyway.
//
// Bandwidth-bound: 2 bytes in, 1 byte of code and 1/32 byte of scale out per
// element.  A warp takes 256 consecutive elements of a row: each lane loads 8
// (16 bytes, so every load instruction is one contiguous 512-byte piece), four
// lanes share a block's amax through two shuffles, each lane writes its 8 codes
// (a contiguous 256-byte store per warp), and lanes 0 and 16 each write the 4
// scale bytes of one 128-channel atom row as one word.  Rows from M up to the
// 128-row padding of the scale layout get zero scales.
#include "common.cuh"
#include "sm100.cuh"

namespace svdq {
namespace {

constexpr int kMxThreads = 256;
constexpr int kMxSegs = 4;                     // 256-element segments per warp and iteration (loads in flight)

// Byte offset of scale [row, block] in the tensor-core scale-factor layout:
// 128-row x 4-block atoms of 512 bytes, row r at (r % 32) * 16 + (r / 32 % 4) * 4,
// atoms along K first.
__device__ __forceinline__ int64_t mx_sf_offset(int64_t row, int64_t blk, int64_t blocks_per_row) {
    const int64_t atom = (row >> 7) * (blocks_per_row >> 2) + (blk >> 2);
    return atom * 512 + (row & 31) * 16 + ((row >> 5) & 3) * 4 + (blk & 3);
}

__global__ void __launch_bounds__(kMxThreads)
mx_quantize_kernel(const uint16_t* __restrict__ X, int64_t M, int64_t K, int64_t ldx, uint32_t n_units,
                   uint8_t* __restrict__ codes, uint8_t* __restrict__ sf, int64_t ext_codes, int64_t ext_sf,
                   uint32_t* err) {
    const int lane = threadIdx.x & 31;
    const uint32_t segs_per_row = static_cast<uint32_t>((K + 255) / 256);
    const uint32_t warps = gridDim.x * (kMxThreads / 32);
    const int64_t blocks_per_row = K / 32;
    for (uint32_t u0 = (blockIdx.x * (kMxThreads / 32) + (threadIdx.x >> 5)) * kMxSegs; u0 < n_units;
         u0 += warps * kMxSegs) {
        // (row, segment) of the warp's units: one division, then carried along the row
        int64_t rows[kMxSegs], cols[kMxSegs];
        {
            uint32_t row = u0 / segs_per_row, seg = u0 - row * segs_per_row;
#pragma unroll
            for (int i = 0; i < kMxSegs; ++i) {
                rows[i] = row;
                cols[i] = static_cast<int64_t>(seg) * 256 + lane * 8;
                if (++seg == segs_per_row) {
                    seg = 0;
                    ++row;
                }
            }
        }
        uint4 v[kMxSegs];
#pragma unroll
        for (int i = 0; i < kMxSegs; ++i) {
            v[i] = (u0 + i < n_units && rows[i] < M && cols[i] < K)
                       ? __ldg(reinterpret_cast<const uint4*>(X + rows[i] * ldx + cols[i]))
                       : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int i = 0; i < kMxSegs; ++i) {
            if (u0 + i >= n_units) break;            // warp-uniform
            const int64_t row = rows[i];
            const int64_t col = cols[i];
            const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
            // |bf16| as bits with the sign cleared: integer order is value order
            uint32_t m2 = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) m2 = __vmaxu2(m2, w[j] & 0x7FFF7FFFu);
            uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
            m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
            m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
            const int bexp = static_cast<int>(m >> 7);                  // biased exponent of amax (bf16 = fp32's)
            const int e = bexp == 0 ? -127 : max(bexp - 127 - 8, -127);
            const float inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);   // 2^-e
            const uint64_t inv2 = pack_f32x2(inv, inv);
            uint32_t q[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                float p0, p1, p2, p3;
                unpack_f32x2(mul_f32x2(bf16x2_to_f32x2(w[2 * j]), inv2), p0, p1);
                unpack_f32x2(mul_f32x2(bf16x2_to_f32x2(w[2 * j + 1]), inv2), p2, p3);
                q[j] = cvt_e4m3x2(p0, p1) | (cvt_e4m3x2(p2, p3) << 16);
            }
            if (row < M && col < K && store_ok(row * K + col, 8, ext_codes, err, kSiteMxCodes))
                *reinterpret_cast<uint2*>(codes + row * K + col) = make_uint2(q[0], q[1]);
            // scale bytes of blocks 4g .. 4g + 3 of this segment: lanes 16 g, 16 g + 4, + 8, + 12
            const uint32_t sb = static_cast<uint32_t>(e + 127);
            const uint32_t s1 = __shfl_down_sync(0xffffffffu, sb, 4);
            const uint32_t s2 = __shfl_down_sync(0xffffffffu, sb, 8);
            const uint32_t s3 = __shfl_down_sync(0xffffffffu, sb, 12);
            if ((lane & 15) == 0 && col < K) {
                const int64_t off = mx_sf_offset(row, col / 32, blocks_per_row);
                if (store_ok(off, 4, ext_sf, err, kSiteMxSf))
                    *reinterpret_cast<uint32_t*>(sf + off) = sb | (s1 << 8) | (s2 << 16) | (s3 << 24);
            }
        }
    }
}

}  // namespace
}  // namespace svdq

extern "C" size_t svdq_mxfp8_sf_bytes(int64_t rows, int64_t K) {
    if (rows < 1 || K < 128 || K % 128 != 0) return 0;
    return static_cast<size_t>((rows + 127) / 128 * 128) * static_cast<size_t>(K / 32);
}

extern "C" int svdq_quantize_mxfp8(const void* X, int64_t M, int64_t K, int64_t ldx, uint8_t* codes, uint8_t* sf,
                                   void* stream) {
    using namespace svdq;
    if (X == nullptr || codes == nullptr || sf == nullptr) return SVDQ_ERR_INVALID_ARG;
    if (M < 1 || K < 128 || ldx < K) return SVDQ_ERR_INVALID_ARG;
    if (K % 128 != 0) return SVDQ_ERR_UNSUPPORTED;
    if (M > (int64_t(1) << 40) || K > (int64_t(1) << 30)) return SVDQ_ERR_UNSUPPORTED;
    if (!aligned16(X) || (ldx * 2) % 16 != 0 || !aligned16(codes) || (reinterpret_cast<uintptr_t>(sf) & 3u))
        return SVDQ_ERR_MISALIGNED;
    if (!device_is_sm100()) return SVDQ_ERR_NO_DEVICE;
    if (!debug_ptrs_ok({X, codes, sf})) return SVDQ_ERR_INVALID_ARG;
    uint32_t* err = device_error_word();
    if (err == nullptr) return SVDQ_ERR_CUDA;
    const int64_t rows_pad = (M + 127) / 128 * 128;
    const int64_t units = rows_pad * ((K + 255) / 256);            // 256-element row segments
    if (units > 0x7FFFFFFFLL) return SVDQ_ERR_UNSUPPORTED;
    const int64_t warps_needed = (units + kMxSegs - 1) / kMxSegs;
    const int sms = device_sm_count() > 0 ? device_sm_count() : 148;
    const int64_t blocks = std::min<int64_t>((warps_needed + 7) / 8, static_cast<int64_t>(sms) * 8);
    mx_quantize_kernel<<<static_cast<unsigned>(blocks), kMxThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint16_t*>(X), M, K, ldx, static_cast<uint32_t>(units), codes, sf,
        debug_extent(kSiteMxCodes, M * K), debug_extent(kSiteMxSf, static_cast<int64_t>(svdq_mxfp8_sf_bytes(M, K))),
        err);
    return launch_status(cudaGetLastError());
}
