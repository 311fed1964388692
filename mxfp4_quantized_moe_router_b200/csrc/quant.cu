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

// Canonical expert row of slab s (0..3), row r16 (0..15) of tile `tile`.
// Gate/up part: tile = 32 intermediate columns; slabs 0,1 are gate rows,
// slabs 2,3 the matching up rows (offset I). Down part: 64 consecutive rows.
__device__ __forceinline__ int64_t tile_row(bool gate_up, int tile, int s, int r16, int I)
{
    if (gate_up)
        return (int64_t)(s >= 2 ? I : 0) + tile * 32 + (s & 1) * 16 + r16;
    return (int64_t)tile * 64 + s * 16 + r16;
}

// One block per (expert, tile, chunk) of one matrix (gate/up or down).
__global__ void __launch_bounds__(256) prepack_kernel(const uint8_t *__restrict__ packed,
                                                      const uint8_t *__restrict__ sc, int E, int rows_per_expert,
                                                      int K, int tiles_per_expert, bool gate_up, int I,
                                                      uint8_t *__restrict__ dst)
{
    const int nchunk = (K + kChunkK - 1) / kChunkK;
    const int64_t blk = blockIdx.x;
    const int c = (int)(blk % nchunk);
    const int tile = (int)((blk / nchunk) % tiles_per_expert);
    const int e = (int)(blk / ((int64_t)nchunk * tiles_per_expert));
    const int k0 = c * kChunkK;
    const int kw = min(kChunkK, K - k0);
    const int64_t ebase = (int64_t)e * rows_per_expert;
    uint8_t *out = dst + ((int64_t)e * tiles_per_expert + tile) * wtile_bytes(K) + (int64_t)c * wchunk_bytes(kChunkK);
    // nibble part: word index = ((w*2 + half)*32 + lane)*4 + jj
    const int nwords = (int)(wchunk_nibble_bytes(kw) / 4);
    for (int i = threadIdx.x; i < nwords; i += blockDim.x) {
        const int jj = i & 3, lane = (i >> 2) & 31, half = (i >> 7) & 1, w = i >> 8;
        const int g = lane >> 2, t = lane & 3;
        const int s = 2 * half + (jj >> 1), step = jj & 1;
        uint32_t word = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int r16 = (b & 1) ? g + 8 : g;
            const int kk = k0 + 32 * w + 16 * step + 2 * t + ((b & 2) ? 8 : 0);
            const int64_t row = ebase + tile_row(gate_up, tile, s, r16, I);
            word |= (uint32_t)packed[row * (K / 2) + kk / 2] << (8 * b);
        }
        reinterpret_cast<uint32_t *>(out)[i] = word;
    }
    // scale part: byte index = ((w*8 + g)*4 + s)*2 + r2
    uint8_t *osc = out + wchunk_nibble_bytes(kw);
    const int nsc = 2 * kw;
    for (int i = threadIdx.x; i < nsc; i += blockDim.x) {
        const int r2 = i & 1, s = (i >> 1) & 3, g = (i >> 3) & 7, w = i >> 6;
        const int r16 = r2 ? g + 8 : g;
        const int64_t row = ebase + tile_row(gate_up, tile, s, r16, I);
        osc[i] = sc[row * (K / 32) + (k0 + 32 * w) / 32];
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

extern "C" MXMOE_API int64_t mxmoe_prepacked_size(int E, int H, int I)
{
    if (E <= 0 || H <= 0 || I <= 0 || H % 64 || I % 32)
        return -1;
    return (int64_t)E * ((int64_t)(I / 32) * wtile_bytes(H) + (int64_t)(H / 64) * wtile_bytes(I));
}

extern "C" MXMOE_API int mxmoe_prepack_experts(const uint8_t *packed13, const uint8_t *sc13, const uint8_t *packed2,
                                               const uint8_t *sc2, int E, int H, int I, void *prepacked,
                                               void *stream)
{
    if (mxmoe_prepacked_size(E, H, I) < 0)
        return fail(MXMOE_ERR_INVALID_SHAPE, "mxmoe_prepack_experts: E=%d H=%d I=%d (need H %% 64 == 0, I %% 32 == 0)",
                    E, H, I);
    if (!packed13 || !sc13 || !packed2 || !sc2 || !prepacked)
        return fail(MXMOE_ERR_NULL, "mxmoe_prepack_experts: NULL pointer");
    if (!aligned16(prepacked))
        return fail(MXMOE_ERR_ALIGNMENT, "mxmoe_prepack_experts: prepacked must be 16-byte aligned");
    if (int rc = check_device())
        return rc;
    uint8_t *dst = static_cast<uint8_t *>(prepacked);
    cudaStream_t st = (cudaStream_t)stream;
    const int64_t blocks13 = (int64_t)E * (I / 32) * ((H + kChunkK - 1) / kChunkK);
    prepack_kernel<<<(unsigned)blocks13, 256, 0, st>>>(packed13, sc13, E, 2 * I, H, I / 32, true, I, dst);
    if (int rc = check_launch("prepack_kernel(gate/up)"))
        return rc;
    uint8_t *dst2 = dst + (int64_t)E * (I / 32) * wtile_bytes(H);
    const int64_t blocks2 = (int64_t)E * (H / 64) * ((I + kChunkK - 1) / kChunkK);
    prepack_kernel<<<(unsigned)blocks2, 256, 0, st>>>(packed2, sc2, E, H, I, H / 64, false, I, dst2);
    return check_launch("prepack_kernel(down)");
}
