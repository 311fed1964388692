// fp8.cu -- FP8 expert weights: quantise (bf16 -> E4M3 codes + E8M0 scales),
// dequantise, and the re-tiling into the layout the FP8 variant of the
// tensor-core FFN streams.
//
// Pages: the "MiMo-V2.5-Pro-FP4-DFlash" model card's section 2 "FP4
// Quantization" sets the MXFP4 experts against an FP8 baseline, and its
// introduction notes that even 8-bit weights carry heavy memory-bandwidth
// costs at the trillion-parameter scale. The pages give no FP8 layout; the
// reading here keeps the MX scheme of the FP4 experts with E4M3 elements: one
// E8M0 scale per 32 elements along K, scale exponent floor(log2 amax) - 8 (8
// is the exponent of E4M3's largest power of two, as 2 is E2M1's), elements
// rounded to nearest E4M3 with ties to even, saturating at 448, sign bit kept.
#include "common.cuh"

namespace mxmoe {
namespace {

// floor(log2 |v|) of a non-zero bf16 magnitude given by its 15 low bits.
__device__ __forceinline__ int bf16_mag_floor_log2(uint32_t mag)
{
    const uint32_t ex = mag >> 7;
    if (ex)
        return (int)ex - 127;
    return (31 - __clz((int)mag)) - 133;  // subnormal: mantissa * 2^-133
}

// One warp per (row, 256-element chunk); lane = (block b = lane/4, part =
// lane%4) owns 8 consecutive elements of block b.
__global__ void __launch_bounds__(256) quantize_fp8_kernel(const uint16_t *__restrict__ w, int64_t rows, int64_t K,
                                                           uint8_t *__restrict__ codes, uint8_t *__restrict__ scales)
{
    const int lane = threadIdx.x & 31;
    const int64_t nchunk = (K + 255) / 256;
    const int64_t total = rows * nchunk;
    const int64_t warp0 = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x / 32);
    for (int64_t item = warp0; item < total; item += nwarps) {
        const int64_t r = item / nchunk;
        const int64_t k = (item % nchunk) * 256 + (lane >> 2) * 32 + (lane & 3) * 8;
        const bool valid = k < K;  // K % 32 == 0: a block is all valid or all invalid
        uint4 v = make_uint4(0, 0, 0, 0);
        if (valid)
            v = __ldg(reinterpret_cast<const uint4 *>(w + r * K + k));
        const uint32_t e16[8] = {v.x & 0xFFFF, v.x >> 16, v.y & 0xFFFF, v.y >> 16,
                                 v.z & 0xFFFF, v.z >> 16, v.w & 0xFFFF, v.w >> 16};
        uint32_t amax = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            amax = max(amax, e16[i] & 0x7FFF);
        amax = max(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
        amax = max(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
        int e = amax ? bf16_mag_floor_log2(amax) - 8 : -127;
        e = max(-127, min(e, 127));
        // 2^-e as a float: e <= 126 gives a normal 2^(-e) (at most 2^127);
        // e = 127 the subnormal 2^-127. |x| * 2^-e is exact in float: it is at
        // most 2^9 for every block, and no bf16 value falls below float's
        // subnormal range when scaled up.
        const float inv = (e <= 126) ? __uint_as_float((uint32_t)(127 - e) << 23) : __uint_as_float(0x00400000u);
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
            const float q0 = __uint_as_float((e16[i] & 0x7FFF) << 16) * inv;
            const float q1 = __uint_as_float((e16[i + 1] & 0x7FFF) << 16) * inv;
            uint16_t pair;  // element i in the low byte: round to nearest even, saturating at 448
            asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pair) : "f"(q1), "f"(q0));
            const uint32_t two = (uint32_t)pair | ((e16[i] >> 15) << 7) | ((e16[i + 1] >> 15) << 15);
            if (i < 4)
                lo |= two << (8 * i);
            else
                hi |= two << (8 * (i - 4));
        }
        if (valid) {
            *reinterpret_cast<uint2 *>(codes + r * K + k) = make_uint2(lo, hi);
            if ((lane & 3) == 0)
                scales[r * (K / 32) + k / 32] = (uint8_t)(e + 127);
        }
    }
}

// Value of an E4M3 code from its fields: sign bit 7, exponent e = bits 6..3
// (bias 7), mantissa m = bits 2..0; e == 0 gives (m/8) * 2^-6; 0x7F / 0xFF are
// NaN (never produced by the quantiser).
__device__ __forceinline__ float e4m3_decode(uint32_t c)
{
    const uint32_t e = (c >> 3) & 15u, m = c & 7u;
    float mag;
    if (e == 15u && m == 7u)
        mag = __uint_as_float(0x7FC00000u);
    else if (e)
        mag = __uint_as_float(((e + 120u) << 23) | (m << 20));
    else
        mag = (float)m * 0.001953125f;  // m * 2^-9
    return (c & 0x80u) ? -mag : mag;
}

__global__ void __launch_bounds__(256) dequantize_fp8_kernel(const uint8_t *__restrict__ codes,
                                                             const uint8_t *__restrict__ scales, int64_t rows,
                                                             int64_t K, float *__restrict__ out)
{
    const int64_t n = rows * K;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / K, k = i % K;
        out[i] = e4m3_decode(codes[i]) * e8m0_to_float(scales[r * (K / 32) + k / 32]);
    }
}

// Prepacked FP8 blob:
//   [gate/up code boxes][down code boxes][gate/up scale images][down scale images]
// A code box is one 256-row tile by 128 values of K: 256 rows of 128 bytes
// (32 KB, contiguous), boxes ordered by (expert, tile, K chunk). Gate/up tile
// t holds gate rows 128t .. 128t+127 (tile rows 0..127) and then the matching
// up rows (tile rows 128..255); down rows keep their order and are padded to a
// multiple of 256 with zero codes and zero scale bytes. The scale images of a
// box are two 512-byte images, one per row half g: byte (r % 32) * 16 +
// (r / 32) * 4 + kb holds the scale of tile row 128g + r, k32 block kb of the
// box -- the order in which tcgen05.cp places them in tensor memory.
__device__ __forceinline__ int64_t fp8_tile_src_row(bool gate_up, int64_t lr_all, int I)
{
    if (!gate_up)
        return lr_all;
    const int64_t t = lr_all >> 8;
    const int lr = (int)(lr_all & 255);
    return lr < 128 ? 128 * t + lr : (int64_t)I + 128 * t + (lr - 128);
}

// One thread per 16 bytes of the code boxes. rows: real rows per expert;
// rows_pad: padded (multiple of 256); K a multiple of 128.
__global__ void __launch_bounds__(256) prepack_fp8_rows_kernel(const uint8_t *__restrict__ codes, int E,
                                                               int64_t rows, int64_t rows_pad, int K, bool gate_up,
                                                               int I, uint8_t *__restrict__ dst)
{
    const int nchunk = K / 128;
    const int64_t tiles = rows_pad / 256;
    const int64_t total = (int64_t)E * rows_pad * nchunk * 8;  // 16-byte units
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < total; u += (int64_t)gridDim.x * blockDim.x) {
        const int part = (int)(u & 7);         // 16-byte part of a 128-byte box row
        const int lr = (int)((u >> 3) & 255);  // box row
        const int64_t box = u >> 11;           // (e * tiles + t) * nchunk + c
        const int c = (int)(box % nchunk);
        const int64_t tile_id = box / nchunk;
        const int64_t e = tile_id / tiles, t = tile_id % tiles;
        const int64_t row = fp8_tile_src_row(gate_up, t * 256 + lr, I);
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (row < rows)
            v = __ldg(reinterpret_cast<const uint4 *>(codes + (e * rows + row) * K + (int64_t)c * 128 + part * 16));
        reinterpret_cast<uint4 *>(dst)[u] = v;
    }
}

// One thread per byte of the scale images.
__global__ void __launch_bounds__(256) prepack_fp8_sf_kernel(const uint8_t *__restrict__ sc, int E, int64_t rows,
                                                             int64_t rows_pad, int K, bool gate_up, int I,
                                                             uint8_t *__restrict__ dst)
{
    const int nchunk = K / 128;
    const int64_t tiles = rows_pad / 256;
    const int64_t total = (int64_t)E * tiles * nchunk * 1024;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int b = (int)(i & 511);
        const int g = (int)((i >> 9) & 1);
        const int64_t box = i >> 10;
        const int c = (int)(box % nchunk);
        const int64_t tile_id = box / nchunk;
        const int64_t e = tile_id / tiles, t = tile_id % tiles;
        const int m = (b >> 4) + 32 * ((b & 15) >> 2), kb = b & 3;
        const int64_t row = fp8_tile_src_row(gate_up, t * 256 + 128 * g + m, I);
        dst[i] = row < rows ? sc[(e * rows + row) * (K / 32) + 4 * c + kb] : (uint8_t)0;
    }
}

int fp8_grid_for(int64_t work, int per_block)
{
    const int64_t g = (work + per_block - 1) / per_block;
    const int64_t cap = 148LL * 32;
    return (int)(g < 1 ? 1 : (g > cap ? cap : g));
}

int64_t fp8_pad256(int64_t v) { return (v + 255) & ~int64_t(255); }

}  // namespace
}  // namespace mxmoe

using namespace mxmoe;

extern "C" MXMOE_API int mxmoe_quantize_fp8(const void *w, int64_t rows, int64_t K, uint8_t *codes, uint8_t *scales,
                                            void *stream)
{
    if (rows <= 0 || K <= 0 || K % 32)
        return fail(MXMOE_ERR_INVALID_SHAPE,
                    "mxmoe_quantize_fp8: rows=%lld K=%lld (K must be a positive multiple of 32)", (long long)rows,
                    (long long)K);
    if (!w || !codes || !scales)
        return fail(MXMOE_ERR_NULL, "mxmoe_quantize_fp8: NULL pointer");
    if (!aligned16(w) || (reinterpret_cast<uintptr_t>(codes) & 7))
        return fail(MXMOE_ERR_ALIGNMENT, "mxmoe_quantize_fp8: w needs 16-byte and codes 8-byte alignment");
    if (int rc = check_device())
        return rc;
    const int64_t warps = rows * ((K + 255) / 256);
    quantize_fp8_kernel<<<fp8_grid_for(warps, 8), 256, 0, (cudaStream_t)stream>>>(static_cast<const uint16_t *>(w),
                                                                                 rows, K, codes, scales);
    return check_launch("quantize_fp8_kernel");
}

extern "C" MXMOE_API int mxmoe_dequantize_fp8(const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t K,
                                              float *out, void *stream)
{
    if (rows <= 0 || K <= 0 || K % 32)
        return fail(MXMOE_ERR_INVALID_SHAPE, "mxmoe_dequantize_fp8: rows=%lld K=%lld", (long long)rows,
                    (long long)K);
    if (!codes || !scales || !out)
        return fail(MXMOE_ERR_NULL, "mxmoe_dequantize_fp8: NULL pointer");
    if (int rc = check_device())
        return rc;
    dequantize_fp8_kernel<<<fp8_grid_for(rows * K, 256), 256, 0, (cudaStream_t)stream>>>(codes, scales, rows, K, out);
    return check_launch("dequantize_fp8_kernel");
}

extern "C" MXMOE_API int64_t mxmoe_prepacked_size_fp8(int E, int H, int I)
{
    if (E <= 0 || H <= 0 || I <= 0 || H % 128 || I % 128)
        return -1;
    const int64_t Hp = fp8_pad256(H);
    return (int64_t)E * (2 * (int64_t)I * H + Hp * I) * 33 / 32;
}

extern "C" MXMOE_API int mxmoe_prepack_experts_fp8(const uint8_t *codes13, const uint8_t *sc13, const uint8_t *codes2,
                                                   const uint8_t *sc2, int E, int H, int I, void *prepacked,
                                                   void *stream)
{
    if (mxmoe_prepacked_size_fp8(E, H, I) < 0)
        return fail(MXMOE_ERR_INVALID_SHAPE,
                    "mxmoe_prepack_experts_fp8: E=%d H=%d I=%d (need H %% 128 == 0, I %% 128 == 0)", E, H, I);
    if (!codes13 || !sc13 || !codes2 || !sc2 || !prepacked)
        return fail(MXMOE_ERR_NULL, "mxmoe_prepack_experts_fp8: NULL pointer");
    if ((reinterpret_cast<uintptr_t>(prepacked) & 31) || !aligned16(codes13) || !aligned16(codes2))
        return fail(MXMOE_ERR_ALIGNMENT,
                    "mxmoe_prepack_experts_fp8: prepacked needs 32-byte, codes13/codes2 16-byte alignment");
    if (int rc = check_device())
        return rc;
    const int64_t Hp = fp8_pad256(H);
    uint8_t *w13 = static_cast<uint8_t *>(prepacked);
    uint8_t *w2 = w13 + (int64_t)E * 2 * I * H;
    uint8_t *sf13 = w2 + (int64_t)E * Hp * I;
    uint8_t *sf2 = sf13 + (int64_t)E * 2 * I * (H / 32);
    cudaStream_t st = (cudaStream_t)stream;
    prepack_fp8_rows_kernel<<<fp8_grid_for((int64_t)E * 2 * I * (H / 16), 256), 256, 0, st>>>(codes13, E, 2 * I,
                                                                                              2 * I, H, true, I, w13);
    if (int rc = check_launch("prepack_fp8_rows_kernel(gate/up)"))
        return rc;
    prepack_fp8_rows_kernel<<<fp8_grid_for((int64_t)E * Hp * (I / 16), 256), 256, 0, st>>>(codes2, E, H, Hp, I, false,
                                                                                           I, w2);
    if (int rc = check_launch("prepack_fp8_rows_kernel(down)"))
        return rc;
    prepack_fp8_sf_kernel<<<fp8_grid_for((int64_t)E * 2 * I * (H / 32), 256), 256, 0, st>>>(sc13, E, 2 * I, 2 * I, H,
                                                                                            true, I, sf13);
    if (int rc = check_launch("prepack_fp8_sf_kernel(gate/up)"))
        return rc;
    prepack_fp8_sf_kernel<<<fp8_grid_for((int64_t)E * Hp * (I / 32), 256), 256, 0, st>>>(sc2, E, H, Hp, I, false, I,
                                                                                         sf2);
    return check_launch("prepack_fp8_sf_kernel(down)");
}
