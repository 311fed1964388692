// quant.cu -- MXFP4 weight format: quantise (bf16 -> E2M1 nibbles + E8M0
// scales), dequantise, and the re-tiling of expert weights into the layout
// the FFN kernels stream.
//
// Format: "MiMo-V2.5-Pro-FP4-DFlash" model card, section 2 "FP4
// Quantization" (MXFP4, block size 32, experts only). The pages give no scale
// or rounding rule; the OCP MX convention is used: block scale exponent
// floor(log2 amax) - 2, elements rounded to nearest E2M1 with ties to even,
// saturating at 6, sign bit kept.
#include "common.cuh"

namespace mxmoe {
namespace {

// floor(log2 |v|) of a non-zero bf16 magnitude given by its 15 low bits.
__device__ __forceinline__ int bf16_floor_log2(uint32_t mag)
{
    uint32_t ex = mag >> 7;
    if (ex)
        return (int)ex - 127;
    return (31 - __clz((int)mag)) - 133;  // subnormal: mantissa * 2^-133
}

// One warp per (row, 256-element chunk); lane = (block b = lane/4, part =
// lane%4) owns 8 consecutive elements of block b.
__global__ void __launch_bounds__(256) quantize_kernel(const uint16_t *__restrict__ w, int64_t rows, int64_t K,
                                                       uint8_t *__restrict__ packed, uint8_t *__restrict__ scales)
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
        uint32_t e16[8] = {v.x & 0xFFFF, v.x >> 16, v.y & 0xFFFF, v.y >> 16,
                           v.z & 0xFFFF, v.z >> 16, v.w & 0xFFFF, v.w >> 16};
        uint32_t amax = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            amax = max(amax, e16[i] & 0x7FFF);
        amax = max(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
        amax = max(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
        int e = amax ? bf16_floor_log2(amax) - 2 : -127;
        e = max(-127, min(e, 127));
        // 2^-e as a float (e in [-127, 127]); 2^127 is normal, 2^-127 is the
        // subnormal 0x00400000.
        const float inv = (e <= 126) ? __uint_as_float((uint32_t)(127 - e) << 23) : __uint_as_float(0x00400000u);
        uint32_t out = 0;
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
            const float q0 = __uint_as_float((e16[i] & 0x7FFF) << 16) * inv;
            const float q1 = __uint_as_float((e16[i + 1] & 0x7FFF) << 16) * inv;
            uint32_t byte;
            asm("{\n\t.reg .b8 t;\n\t"
                "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
                "cvt.u32.u8 %0, t;\n\t}"
                : "=r"(byte)
                : "f"(q1), "f"(q0));
            byte |= ((e16[i] >> 15) << 3) | ((e16[i + 1] >> 15) << 7);
            out |= (byte & 0xFF) << (4 * i);
        }
        if (valid) {
            *reinterpret_cast<uint32_t *>(packed + r * (K / 2) + k / 2) = out;
            if ((lane & 3) == 0)
                scales[r * (K / 32) + k / 32] = (uint8_t)(e + 127);
        }
    }
}

// Value of an E2M1 code from its fields: exponent e = bits 2..1, mantissa m =
// bit 0, sign bit 3; e == 0 gives m * 0.5, otherwise 2^(e-1) * (1 + m/2).
__device__ __forceinline__ float e2m1_decode(uint32_t c)
{
    const uint32_t e = (c >> 1) & 3u, m = c & 1u;
    const float mag = e ? __uint_as_float(((e + 126u) << 23) | (m << 22)) : 0.5f * (float)m;
    return (c & 8u) ? -mag : mag;
}

__global__ void __launch_bounds__(256) dequantize_kernel(const uint8_t *__restrict__ packed,
                                                         const uint8_t *__restrict__ scales, int64_t rows,
                                                         int64_t K, float *__restrict__ out)
{
    const int64_t nbytes = rows * (K / 2);
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nbytes;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / (K / 2), kk = (i % (K / 2)) * 2;
        const float s = e8m0_to_float(scales[r * (K / 32) + kk / 32]);
        const uint32_t byte = packed[i];
        const float lo = e2m1_decode(byte & 0xF), hi = e2m1_decode(byte >> 4);
        *reinterpret_cast<float2 *>(out + r * K + kk) = make_float2(lo * s, hi * s);
    }
}

// Prepacked blob for the tensor-core FFN:
//   [gate/up code boxes][down code boxes][gate/up scale images][down scale images]
// A code box is one 256-row wide tile by 256 values of K: 256 rows of 128
// bytes (32 KB, contiguous), boxes ordered by (expert, tile, K chunk). Gate/up
// tile t holds gate rows 128t .. 128t+127 (tile rows 0..127) and then the
// matching up rows (tile rows 128..255); down rows keep their order. The
// scale images of a box are four 512-byte images ordered (K half h, row half
// g): byte (r % 32) * 16 + (r / 32) * 4 + kb holds the scale of tile row
// 128g + r, k32 block 4h + kb of the box. K is padded to a multiple of 256 and
// the down rows to a multiple of 256 with zero codes and zero scale bytes; at
// H, I multiples of 256 the blob is a byte permutation of the canonical format.
__device__ __forceinline__ int64_t tile_src_row(bool gate_up, int64_t lr_all, int I)
{
    if (!gate_up)
        return lr_all;
    const int64_t t = lr_all >> 8;
    const int lr = (int)(lr_all & 255);
    return lr < 128 ? 128 * t + lr : (int64_t)I + 128 * t + (lr - 128);
}

// One thread per 16 bytes of the code boxes. rows: real rows per expert;
// rows_pad: padded (multiple of 256); K real, K padded to a multiple of 256.
__global__ void __launch_bounds__(256) prepack_rows_kernel(const uint8_t *__restrict__ packed, int E, int64_t rows,
                                                           int64_t rows_pad, int K, bool gate_up, int I,
                                                           uint8_t *__restrict__ dst)
{
    const int nchunk = (K + 255) / 256;
    const int64_t tiles = rows_pad / 256;
    const int64_t total = (int64_t)E * rows_pad * nchunk * 8;  // 16-byte units
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < total; u += (int64_t)gridDim.x * blockDim.x) {
        const int part = (int)(u & 7);          // 16-byte part of a 128-byte box row
        const int lr = (int)((u >> 3) & 255);   // box row
        const int64_t box = u >> 11;            // (e * tiles + t) * nchunk + c
        const int c = (int)(box % nchunk);
        const int64_t tile_id = box / nchunk;
        const int64_t e = tile_id / tiles, t = tile_id % tiles;
        const int64_t row = tile_src_row(gate_up, t * 256 + lr, I);
        const int64_t byte = (int64_t)c * 128 + part * 16;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (row < rows && byte < K / 2)
            v = __ldg(reinterpret_cast<const uint4 *>(packed + (e * rows + row) * (K / 2) + byte));
        reinterpret_cast<uint4 *>(dst)[u] = v;
    }
}

// One thread per byte of the scale images.
__global__ void __launch_bounds__(256) prepack_sf_kernel(const uint8_t *__restrict__ sc, int E, int64_t rows,
                                                         int64_t rows_pad, int K, bool gate_up, int I,
                                                         uint8_t *__restrict__ dst)
{
    const int nchunk = (K + 255) / 256;
    const int64_t tiles = rows_pad / 256;
    const int64_t total = (int64_t)E * tiles * nchunk * 2048;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int b = (int)(i & 511);
        const int g = (int)((i >> 9) & 1), h = (int)((i >> 10) & 1);
        const int64_t box = i >> 11;
        const int c = (int)(box % nchunk);
        const int64_t tile_id = box / nchunk;
        const int64_t e = tile_id / tiles, t = tile_id % tiles;
        const int m = (b >> 4) + 32 * ((b & 15) >> 2), kb = b & 3;
        const int64_t row = tile_src_row(gate_up, t * 256 + 128 * g + m, I);
        const int blk = 8 * c + 4 * h + kb;
        dst[i] = (row < rows && blk < K / 32) ? sc[(e * rows + row) * (K / 32) + blk] : (uint8_t)0;
    }
}

int grid_for(int64_t work, int per_block)
{
    int64_t g = (work + per_block - 1) / per_block;
    int64_t cap = 148LL * 32;
    return (int)(g < 1 ? 1 : (g > cap ? cap : g));
}

}  // namespace
}  // namespace mxmoe

using namespace mxmoe;

extern "C" MXMOE_API int mxmoe_quantize(const void *w, int64_t rows, int64_t K, uint8_t *packed, uint8_t *scales,
                                        void *stream)
{
    if (rows <= 0 || K <= 0 || K % 32)
        return fail(MXMOE_ERR_INVALID_SHAPE, "mxmoe_quantize: rows=%lld K=%lld (K must be a positive multiple of 32)",
                    (long long)rows, (long long)K);
    if (!w || !packed || !scales)
        return fail(MXMOE_ERR_NULL, "mxmoe_quantize: NULL pointer");
    if (!aligned16(w))
        return fail(MXMOE_ERR_ALIGNMENT, "mxmoe_quantize: w must be 16-byte aligned");
    if (int rc = check_device())
        return rc;
    const int64_t warps = rows * ((K + 255) / 256);
    quantize_kernel<<<grid_for(warps, 8), 256, 0, (cudaStream_t)stream>>>(static_cast<const uint16_t *>(w), rows,
                                                                          K, packed, scales);
    return check_launch("quantize_kernel");
}

extern "C" MXMOE_API int mxmoe_dequantize(const uint8_t *packed, const uint8_t *scales, int64_t rows, int64_t K,
                                          float *out, void *stream)
{
    if (rows <= 0 || K <= 0 || K % 32)
        return fail(MXMOE_ERR_INVALID_SHAPE, "mxmoe_dequantize: rows=%lld K=%lld", (long long)rows, (long long)K);
    if (!packed || !scales || !out)
        return fail(MXMOE_ERR_NULL, "mxmoe_dequantize: NULL pointer");
    if ((reinterpret_cast<uintptr_t>(out) & 7) != 0)
        return fail(MXMOE_ERR_ALIGNMENT, "mxmoe_dequantize: out must be 8-byte aligned");
    if (int rc = check_device())
        return rc;
    dequantize_kernel<<<grid_for(rows * (K / 2), 256), 256, 0, (cudaStream_t)stream>>>(packed, scales, rows, K,
                                                                                      out);
    return check_launch("dequantize_kernel");
}

static int64_t pad256(int64_t v) { return (v + 255) & ~int64_t(255); }

extern "C" MXMOE_API int64_t mxmoe_prepacked_size(int E, int H, int I)
{
    if (E <= 0 || H <= 0 || I <= 0 || H % 128 || I % 128)
        return -1;
    const int64_t Hp = pad256(H), Ip = pad256(I);
    return (int64_t)E * (2 * (int64_t)I * Hp + Hp * Ip) * 17 / 32;
}

extern "C" MXMOE_API int mxmoe_prepack_experts(const uint8_t *packed13, const uint8_t *sc13, const uint8_t *packed2,
                                               const uint8_t *sc2, int E, int H, int I, void *prepacked,
                                               void *stream)
{
    if (mxmoe_prepacked_size(E, H, I) < 0)
        return fail(MXMOE_ERR_INVALID_SHAPE,
                    "mxmoe_prepack_experts: E=%d H=%d I=%d (need H %% 128 == 0, I %% 128 == 0)", E, H, I);
    if (!packed13 || !sc13 || !packed2 || !sc2 || !prepacked)
        return fail(MXMOE_ERR_NULL, "mxmoe_prepack_experts: NULL pointer");
    if ((reinterpret_cast<uintptr_t>(prepacked) & 31) || !aligned16(packed13) || !aligned16(packed2))
        return fail(MXMOE_ERR_ALIGNMENT,
                    "mxmoe_prepack_experts: prepacked needs 32-byte, packed13/packed2 16-byte alignment");
    if (int rc = check_device())
        return rc;
    const int64_t Hp = pad256(H), Ip = pad256(I);
    uint8_t *w13 = static_cast<uint8_t *>(prepacked);
    uint8_t *w2 = w13 + (int64_t)E * 2 * I * (Hp / 2);
    uint8_t *sf13 = w2 + (int64_t)E * Hp * (Ip / 2);
    uint8_t *sf2 = sf13 + (int64_t)E * 2 * I * (Hp / 32);
    cudaStream_t st = (cudaStream_t)stream;
    prepack_rows_kernel<<<grid_for((int64_t)E * 2 * I * (Hp / 32), 256), 256, 0, st>>>(packed13, E, 2 * I, 2 * I, H,
                                                                                        true, I, w13);
    if (int rc = check_launch("prepack_rows_kernel(gate/up)"))
        return rc;
    prepack_rows_kernel<<<grid_for((int64_t)E * Hp * (Ip / 32), 256), 256, 0, st>>>(packed2, E, H, Hp, I, false, I,
                                                                                    w2);
    if (int rc = check_launch("prepack_rows_kernel(down)"))
        return rc;
    prepack_sf_kernel<<<grid_for((int64_t)E * 2 * I * (Hp / 32), 256), 256, 0, st>>>(sc13, E, 2 * I, 2 * I, H, true,
                                                                                      I, sf13);
    if (int rc = check_launch("prepack_sf_kernel(gate/up)"))
        return rc;
    prepack_sf_kernel<<<grid_for((int64_t)E * Hp * (Ip / 32), 256), 256, 0, st>>>(sc2, E, H, Hp, I, false, I, sf2);
    return check_launch("prepack_sf_kernel(down)");
}
