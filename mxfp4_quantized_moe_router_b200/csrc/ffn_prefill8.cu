// ffn_prefill8.cu -- both stages of the expert FFN for large token counts on
// block-scaled tcgen05 tensor cores, the MXFP4 weights fed as stored.
//
// Pages: "MiMo-V2.5-Pro-FP4-DFlash" model card, section 2 "FP4 Quantization"
// (MXFP4 experts, block size 32); nxbn.cn MiMo-V2.5-Pro-FP4-DFlash article,
// architecture section (384 experts, 8 per token, hidden 6144). The expert is
// read as a SwiGLU FFN with no biases: h = silu(W_gate x) * (W_up x),
// y = W_down h.
//
// When an expert sees hundreds of tokens the FFN is bound by the tensor cores.
// tcgen05.mma.kind::mxf8f6f4.block_scale takes the E2M1 weight codes as they
// are stored (the TMA unpacks them to one byte per value, 16U4_ALIGN16B) with
// their UE8M0 scales applied in hardware, so no instruction touches a weight.
// The activations enter as E4M3 terms with one UE8M0 scale per 32 values
// each: x as two terms (exact for every bf16 element within 2^-13 of its
// 32-block's maximum, smaller ones within 2^-21 of it), h as three (about 12
// significant bits). A term's MMAs accumulate into the same accumulator as the
// others' (terms stacked along K); at the fp8 rate two terms cost one bf16
// MMA, three cost one and a half.
//  * A work item is (expert, pass of up to 224 tokens, one 256-row box of the
//    prepacked blob) = two 128-row tiles: gate rows and up rows of the same
//    128 h columns (gate/up), or two 128-row halves of 256 output columns
//    (down). A stage is 128 values of K.
//  * Two rings: weight stages (one TMA box of 256 rows x 128 values, unpacked
//    to 32 KB, plus the blob's two 512-byte scale images of that K half),
//    activation-term stages (one 28 KB tile of 224 rows x 128 E4M3 values of
//    one term, already in the 128-byte-swizzled layout, plus its two scale
//    images), each with its own producer warp.
//  * One MMA thread copies each stage's scale images into tensor memory
//    (tcgen05.cp, one column slot per ring slot) and issues the MMAs of both
//    tiles: M = 128, N = the pass's tokens rounded up to 16, K = 32.
//  * Accumulators: tile 0 at tensor-memory column 0, tile 1 at 256 (224
//    columns each); the scale slots sit in the columns between and after.
//  * Eight epilogue warps, two per accumulator lane quarter taking alternate
//    32-token chunks: gate/up computes h = silu(g) u for each token (lane = h
//    column, so a warp holds one 32-block of h per token: its maximum is one
//    redux.sync), encodes h into its three E4M3 terms in the layout the down
//    stage reads; down writes y in fp32.
//  * Items go round-robin over a persistent grid of one CTA per SM.
// All waits are bounded; on a timeout the kernel records MXMOE_ERR_TIMEOUT in
// the workspace status word and returns.
#include <algorithm>

#include <cudaTypedefs.h>

#include "common.cuh"
#include "tcgen05.cuh"

namespace mxmoe {
namespace {

constexpr uint64_t kQWaitNs = 2000000000ull;  // bounded waits: 2 s
constexpr int kQThreads = 384;                // 12 warps: see the role list at the kernel
constexpr int kQTok = 224;                    // tokens per pass (N <= 224)
constexpr int kQK = 128;                      // K per stage
constexpr int kQAStages = 3;                  // weight ring
constexpr int kQBStages = 4;                  // activation-term ring
constexpr int kQABytes = 256 * kQK;           // a weight stage in shared memory: 256 rows x 128 values, one byte each
constexpr int kQATx = 256 * kQK / 2;          // its TMA transaction bytes (the packed codes)
constexpr int kQBBytes = kQTok * kQK;         // an activation-term stage: 224 rows x 128 E4M3 values
constexpr int kQSfBytes = 1024;               // two 512-byte scale images

// Tensor memory: accumulators of tiles 0 and 1 at columns 0 and 256; weight
// scale slots (8 columns: tile j at +4j) at 224 + 8s; activation scale slots
// (8 columns: rows 0..127 at +0, 128..255 at +4) at 480 + 8s.
constexpr uint32_t kQAccCols = 256;
constexpr uint32_t kQSfaCol0 = 224;
constexpr uint32_t kQSfbCol0 = 480;
static_assert(kQSfaCol0 + 8 * kQAStages <= kQAccCols && kQSfbCol0 + 8 * kQBStages <= 512, "tensor memory columns");

// shared memory: weight ring | its scale images | term ring | their scale images | barriers | misc
constexpr size_t kQOffAsf = (size_t)kQAStages * kQABytes;
constexpr size_t kQOffB = kQOffAsf + (size_t)kQAStages * kQSfBytes;
constexpr size_t kQOffBsf = kQOffB + (size_t)kQBStages * kQBBytes;
constexpr size_t kQOffBar = kQOffBsf + (size_t)kQBStages * kQSfBytes;
// full_a, empty_a, full_b, empty_b, accfull, accempty, mma_done
constexpr int kQBars = 2 * kQAStages + 2 * kQBStages + 3;
constexpr size_t kQOffMisc = (kQOffBar + kQBars * 8 + 15) & ~size_t(15);
constexpr size_t kQSmem = 1024 + kQOffMisc + 64;
static_assert(kQSmem <= 232448, "shared memory");
static_assert(kQBBytes % 1024 == 0 && kQABytes % 1024 == 0, "swizzled tiles start on 1024-byte boundaries");

struct Q8Params {
    int pairs;                  // 256-row blob boxes per expert: I/128 (gate/up) or Hp/256 (down)
    int nkb;                    // 128-value K stages: H/128 (gate/up) or I/128 (down)
    int nchunk;                 // 256-value chunks per blob row (K padded to 256)
    int H, I, E;
    const int32_t *offsets;     // [E+1]
    const int32_t *pass_start;  // [E+1]: 224-token passes before each expert
    const uint8_t *act;         // activation terms: [pass][stage][term][224 x 128]
    const uint8_t *act_sf;      // their scale images: [pass][stage][term][1024]
    const uint8_t *wsf;         // scale images of the stage's blob part: [box][chunk][2048]
    uint8_t *h_terms;           // gate/up out: h's terms, [pass][I/128][3][224 x 128]
    uint8_t *h_sf;              // and their scale images
    float *y;                   // down out: [rows, H]
    int *status;
};

// Token passes of up to `tok` rows before each expert: pass_start[e] = sum
// over e' < e of ceil(n_e' / tok), e = 0 .. E (E <= 1024), counting only
// experts with at least min_rows rows (the others run on the E2M1-term
// kernel). One block of 1024 threads; also clears the status word (when given).
__global__ void __launch_bounds__(1024) prefill_passes_kernel(const int32_t *__restrict__ offsets, int E,
                                                              int min_rows, int tok, int32_t *__restrict__ pass_start,
                                                              int *status)
{
    grid_dep_wait();  // the preceding kernel's results (chained launch)
    grid_dep_launch();
    __shared__ int32_t s_warp[32];
    const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
    const int n_e = e < E ? __ldg(offsets + e + 1) - __ldg(offsets + e) : 0;
    const int c = n_e >= min_rows ? (n_e + tok - 1) / tok : 0;
    int incl = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
        if (lane >= off)
            incl += o;
    }
    if (lane == 31)
        s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = s_warp[lane], wi = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xFFFFFFFFu, wi, off);
            if (lane >= off)
                wi += o;
        }
        s_warp[lane] = wi - w;  // passes before this warp's experts
    }
    __syncthreads();
    const int excl = s_warp[warp] + incl - c;
    if (e <= E)
        pass_start[e] = excl;  // e == E: the total
    if (e == 0 && status)
        *status = 0;
}

// slot_row[src_row[r]] = r: the grouped row of each (token, slot) pair.
__global__ void __launch_bounds__(256) slot_rows_kernel(const int32_t *__restrict__ src_row, int rows,
                                                        int32_t *__restrict__ slot_row)
{
    grid_dep_wait();  // the preceding kernel's results (chained launch)
    grid_dep_launch();
    for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < rows; r += gridDim.x * blockDim.x)
        slot_row[__ldg(src_row + r)] = r;
}

// Byte of the scale of activation row m (of the pass), 32-block kb of a
// stage, in the term's two 512-byte images (rows 0..127, 128..255): lane
// m % 32, column (m % 128) / 32 of image m / 128, byte kb -- the order in which
// tcgen05.cp places a 32-lane x 16-byte image in tensor memory.
__device__ __forceinline__ int q8_sf_byte(int m, int kb)
{
    return (m >> 7) * 512 + (m & 31) * 16 + ((m & 127) >> 5) * 4 + kb;
}

// Byte offset of row m, byte b (0..127) of a 128-byte-swizzled tile (16-byte
// chunk c of row m at chunk c ^ (m % 8)).
__device__ __forceinline__ int q8_swz(int m, int b) { return m * 128 + ((((b >> 4) ^ (m & 7))) << 4) + (b & 15); }

__device__ __forceinline__ float q8_pow2(int s)  // 2^s for s in [-126, 127]
{
    return __uint_as_float((uint32_t)(s + 127) << 23);
}

// E4M3 code of v (round to nearest even, saturating), and the code's value.
__device__ __forceinline__ uint32_t q8_e4m3(float v)
{
    uint16_t pair;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pair) : "f"(0.f), "f"(v));
    return pair & 0xFFu;
}

__device__ __forceinline__ float q8_e4m3_value(uint32_t code)
{
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)code));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

// E4M3 codes of two values in one conversion: lo's code in bits 0..7, hi's in 8..15.
__device__ __forceinline__ uint32_t q8_e4m3x2(float lo, float hi)
{
    uint16_t pair;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pair) : "f"(hi), "f"(lo));
    return pair;
}

// The values of two E4M3 codes (bits 0..7 and 8..15): every E4M3 value is an
// f16 value, so a conversion to f16x2 and two widenings give them exactly.
__device__ __forceinline__ float2 q8_e4m3x2_values(uint32_t codes)
{
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)codes));
    return __half22float2(*reinterpret_cast<const __half2 *>(&h2));
}

// Byte transpose in groups of 4 lanes: lane 4j + r holds bytes k = 0..3 (its
// values for 4 items k); afterwards it holds item r's bytes of lanes 4j .. 4j+3
// (sel1 = r & 1 ? 0x3715 : 0x6240, sel2 = r & 2 ? 0x3276 : 0x5410).
__device__ __forceinline__ uint32_t q8_t4(uint32_t w, uint32_t sel1, uint32_t sel2)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(w), "r"(__shfl_xor_sync(0xFFFFFFFFu, w, 1)), "r"(sel1));
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(w) : "r"(d), "r"(__shfl_xor_sync(0xFFFFFFFFu, d, 2)), "r"(sel2));
    return w;
}

// Instruction descriptor of kind::mxf8f6f4.block_scale: A = E2M1 (the
// weights, one per byte), B = E4M3 (the activation terms), UE8M0 scales, both
// K-major, M = 128, N = n, scale byte sf_id (the 32-block of a 4-block column)
// for both operands.
__device__ __forceinline__ uint32_t q8_idesc(int n, uint32_t sf_id)
{
    return (sf_id << 4) | (5u << 7) | (0u << 10) | ((uint32_t)(n >> 3) << 17) | (1u << 23) | (8u << 24) |
           (sf_id << 29);
}

__device__ __forceinline__ void q8_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate, uint32_t sfa_tmem, uint32_t sfb_tmem)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// Work items: (pass of up to 224 tokens, 256-row blob box), passes in expert
// order: item i is box i % pairs of pass i / pairs. CTA b takes items b,
// b + G, b + 2G, ... (G CTAs). Every role decodes the same items.
struct QItem {
    int e, box, r0, nt;
    int64_t pass;
};

__device__ __forceinline__ QItem q8_item(int64_t idx, const int32_t *__restrict__ pass_start,
                                         const int32_t *__restrict__ off, int E, int pairs)
{
    QItem it;
    it.pass = idx / pairs;
    it.box = (int)(idx % pairs);
    int lo = 0, hi = E;  // expert of the pass: largest e with pass_start[e] <= pass
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(pass_start + mid) <= it.pass)
            lo = mid;
        else
            hi = mid;
    }
    it.e = lo;
    it.r0 = __ldg(off + lo) + (int)(it.pass - __ldg(pass_start + lo)) * kQTok;
    it.nt = min(kQTok, __ldg(off + lo + 1) - it.r0);
    return it;
}

// Lane 0 waits on an mbarrier; the warp follows its verdict. On a timeout or
// an abort raised elsewhere the status word gets MXMOE_ERR_TIMEOUT.
__device__ __forceinline__ bool q8_warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag, int *status)
{
    int okv = 1;
    if ((threadIdx.x & 31) == 0 && (*abort_flag || !mbar_wait_bounded(bar, parity, kQWaitNs))) {
        set_status(status, MXMOE_ERR_TIMEOUT);
        *abort_flag = 1;
        okv = 0;
    }
    return __shfl_sync(0xFFFFFFFFu, okv, 0) != 0;
}

// x rows in grouped order as two E4M3 terms per value, tiled as the stage
// reads them: the tile of (pass, stage, term) holds the pass's 224 rows x 128
// values, 128-byte swizzled, with two 512-byte scale images. For a 32-block
// whose largest magnitude has exponent E (at least -116, so that every scale
// stays a normal UE8M0 value): term 0 = x / 2^(E-7) rounded to E4M3, term 1 =
// the exact remainder / 2^(E-11) rounded to E4M3. Rows of experts with fewer
// than min_rows rows are skipped (the E2M1-term kernel takes them).
// A warp takes (token t, a range of the 128-value stages; `groups` ranges
// per token so that small token counts still fill the GPU): lane j < k finds
// where slot j goes, every lane keeps each slot's tile row offset for its own
// 4 bytes, then per stage the warp reads x[t] once (lane l: values 4l .. 4l+3,
// a 32-block being eight lanes; the loads of NL stages issued together),
// encodes, and writes every slot's two terms; lane j writes slot j's four
// block scales of both terms as one word each.
constexpr int kQMaxK = 32;

template <int KMAX>
__global__ void __launch_bounds__(256) x8_terms_kernel(const uint16_t *__restrict__ x,
                                                       const int32_t *__restrict__ slot_row,
                                                       const int32_t *__restrict__ offsets,
                                                       const int32_t *__restrict__ pass_start, int E, int min_rows,
                                                       int k, int T, int H, int groups, uint8_t *__restrict__ terms,
                                                       uint8_t *__restrict__ sf)
{
    grid_dep_wait();  // the preceding kernel's results (chained launch)
    grid_dep_launch();
    const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5;
    const int nkb = H / kQK;
    const int per = (nkb + groups - 1) / groups;
    if (__ldg(pass_start + E) == 0)  // no expert for this kernel
        return;
    const int64_t units = (int64_t)T * groups;
    for (int64_t u = (int64_t)blockIdx.x * 8 + wl; u < units; u += (int64_t)gridDim.x * 8) {
        const int t = (int)(u / groups), g = (int)(u % groups);
        const int kb0 = g * per, kb1 = min(nkb, kb0 + per);
        int64_t my_pass = -1;  // lane j < k: slot j's pass (or -1: the E2M1-term kernel's expert) and row
        int my_row = 0;
        if (lane < k) {
            const int r = __ldg(slot_row + (int64_t)t * k + lane);
            int lo = 0, hi = E;  // expert of row r: largest e with offsets[e] <= r
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (__ldg(offsets + mid) <= r)
                    lo = mid;
                else
                    hi = mid;
            }
            const int local = r - __ldg(offsets + lo);
            if (__ldg(offsets + lo + 1) - __ldg(offsets + lo) >= min_rows)
                my_pass = __ldg(pass_start + lo) + local / kQTok;
            my_row = local % kQTok;
        }
        if (!__any_sync(0xFFFFFFFFu, my_pass >= 0) || kb0 >= kb1)
            continue;
        int64_t tb[KMAX];  // slot j: byte offset of this lane's 4 bytes in the slot's row of stage 0, term 0
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            const long long pj = __shfl_sync(0xFFFFFFFFu, (long long)my_pass, j);
            const int rj = __shfl_sync(0xFFFFFFFFu, my_row, j);
            tb[j] = (j < k && pj >= 0) ? pj * nkb * 2 * (int64_t)kQBBytes + q8_swz(rj, 4 * lane) : -1;
        }
        const int64_t sbase = my_pass >= 0 ? my_pass * nkb * 2 * (int64_t)kQSfBytes + q8_sf_byte(my_row, 0) : -1;
        const uint2 *src = reinterpret_cast<const uint2 *>(x + (int64_t)t * H);
        constexpr int NL = KMAX > 8 ? 2 : 4;  // stages whose x loads are in flight together
        for (int kq = kb0; kq < kb1; kq += NL) {
            uint2 raws[NL];
#pragma unroll
            for (int i = 0; i < NL; ++i)
                raws[i] = kq + i < kb1 ? __ldg(src + (kq + i) * 32 + lane) : make_uint2(0u, 0u);
#pragma unroll
            for (int i = 0; i < NL; ++i) {
                const int kb = kq + i;
                if (kb >= kb1)
                    break;
                const uint2 raw = raws[i];
                float v[4] = {__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xFFFF0000u),
                              __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xFFFF0000u)};
                uint32_t m = 0;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    m = max(m, __float_as_uint(v[j]) & 0x7FFFFFFFu);
                m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
                m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
                m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 4));
                const int Eb = max((int)(m >> 23) - 127, -116);
                const float inv0 = q8_pow2(7 - Eb), inv1 = q8_pow2(11 - Eb), sc0 = q8_pow2(Eb - 7);
                uint32_t w0 = 0, w1 = 0;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t c0 = q8_e4m3(v[j] * inv0);
                    const float rem = v[j] - q8_e4m3_value(c0) * sc0;  // exact
                    const uint32_t c1 = q8_e4m3(rem * inv1);
                    w0 |= c0 << (8 * j);
                    w1 |= c1 << (8 * j);
                }
                // the stage's four block scale bytes of term 0 (E - 7 + 127); term 1's are 4 less (E - 11 + 127)
                const uint32_t s0 = (uint32_t)(__shfl_sync(0xFFFFFFFFu, Eb, 0) + 120) |
                                    ((uint32_t)(__shfl_sync(0xFFFFFFFFu, Eb, 8) + 120) << 8) |
                                    ((uint32_t)(__shfl_sync(0xFFFFFFFFu, Eb, 16) + 120) << 16) |
                                    ((uint32_t)(__shfl_sync(0xFFFFFFFFu, Eb, 24) + 120) << 24);
                const int64_t koff = (int64_t)kb * 2 * kQBBytes;
#pragma unroll
                for (int j = 0; j < KMAX; ++j)
                    if (tb[j] >= 0) {
                        *reinterpret_cast<uint32_t *>(terms + tb[j] + koff) = w0;
                        *reinterpret_cast<uint32_t *>(terms + tb[j] + koff + kQBBytes) = w1;
                    }
                if (sbase >= 0) {
                    uint8_t *s = sf + sbase + (int64_t)kb * 2 * kQSfBytes;
                    *reinterpret_cast<uint32_t *>(s) = s0;
                    *reinterpret_cast<uint32_t *>(s + kQSfBytes) = s0 - 0x04040404u;
                }
            }
        }
    }
}

// Warp roles (12 warps).
constexpr int kQWarpB = 0;      // activation-term producer
constexpr int kQWarpMma = 1;    // MMA thread (and the scale-image copies)
constexpr int kQWarpA = 2;      // weight producer
constexpr int kQEpiWarp0 = 4;   // epilogue warps 4..11 (lane quarter w % 4, token chunks of parity (w - 4) / 4)
constexpr int kQEpiWarps = 8;
static_assert(kQThreads == 32 * (kQEpiWarp0 + kQEpiWarps), "warp roles");

__device__ __forceinline__ float q8_silu(float g) { return __fdividef(g, 1.f + __expf(-g)); }

template <bool GATE_UP>
__global__ void __launch_bounds__(kQThreads, 1)
    ffn_f8_kernel(const __grid_constant__ CUtensorMap tmW, const Q8Params p)
{
    constexpr int NTERMS = GATE_UP ? 2 : 3;  // x as two terms, h as three
    if (__ldg(p.pass_start + p.E) == 0) {  // no expert for this kernel
        grid_dep_wait();
        grid_dep_launch();
        return;
    }
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem, *sAsf = smem + kQOffAsf, *sB = smem + kQOffB, *sBsf = smem + kQOffBsf;
    uint64_t *full_a = reinterpret_cast<uint64_t *>(smem + kQOffBar);
    uint64_t *empty_a = full_a + kQAStages;
    uint64_t *full_b = empty_a + kQAStages;
    uint64_t *empty_b = full_b + kQBStages;
    uint64_t *accfull = empty_b + kQBStages;
    uint64_t *accempty = accfull + 1;
    uint64_t *mma_done = accempty + 1;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + kQOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int E = p.E, pairs = p.pairs;
    if (tid == 32) {
        for (int s = 0; s < kQAStages; ++s) {
            mbar_init(&full_a[s], 1);
            mbar_init(&empty_a[s], 1);
        }
        for (int s = 0; s < kQBStages; ++s) {
            mbar_init(&full_b[s], 1);
            mbar_init(&empty_b[s], 1);
        }
        mbar_init(accfull, 1);
        mbar_init(accempty, kQEpiWarps);
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kQWarpMma)
        tc::alloc(tslot, 512);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *tslot;
    const int64_t total = (int64_t)__ldg(p.pass_start + E) * pairs;
    const int64_t G = gridDim.x;
    const int n_items = (int)(total > blockIdx.x ? (total - blockIdx.x + G - 1) / G : 0);
#define ITEM(i) q8_item(blockIdx.x + (int64_t)(i) * G, p.pass_start, p.offsets, E, pairs)
    const int nkb = p.nkb;
    // Chained launch: the weight producer fills its ring before waiting for
    // the preceding kernel (weights, offsets and the pass table are older than
    // it); every other role waits here.
    if (!((warp == kQWarpB || warp == kQWarpA) && lane == 0))
        grid_dep_wait();

    if (warp == kQWarpB || warp == kQWarpA) {
        // ---------------------------------------------------------- producers
        // Warp 0: activation-term stages (one bulk copy of a 28 KB tile and
        // one of its two scale images each), kept in L2 for the pass's other
        // boxes. Warp 2: weight stages (the box's 256 rows x 128 values of one
        // K half, unpacked by the TMA, and the blob's scale images of that half).
        if (lane == 0) {
            const bool is_b = warp == kQWarpB;
            const int S = is_b ? kQBStages : kQAStages;
            uint64_t *full = is_b ? full_b : full_a;
            uint64_t *empty = is_b ? empty_b : empty_a;
            const uint64_t pol = is_b ? policy_evict_last() : policy_evict_normal();
            int s = 0;
            uint32_t ph = 0;
            int64_t issued = 0;
            bool ok = true;
            auto load_a = [&](int sl, int64_t box, int kb) {
                const int64_t chunk = box * p.nchunk + (kb >> 1);  // 256-value chunk of the box
                mbar_arrive_expect_tx(&full[sl], (uint32_t)(kQATx + kQSfBytes));
                tc::tma_load_2d(sA + (size_t)sl * kQABytes, &tmW, 128 * (kb & 1), (int)(chunk * 256), &full[sl], pol);
                bulk_g2s_hint(sAsf + (size_t)sl * kQSfBytes, p.wsf + chunk * 2048 + (kb & 1) * kQSfBytes, kQSfBytes,
                              &full[sl], pol);
            };
            int64_t pre = 0;  // weight loads issued before the wait (slots 0 .. pre-1, first use)
            if (!is_b)
                for (int i = 0; i < n_items && pre < S; ++i) {
                    const QItem it = ITEM(i);
                    for (int kb = 0; kb < nkb && pre < S; ++kb, ++pre)
                        load_a((int)pre, (int64_t)it.e * pairs + it.box, kb);
                }
            grid_dep_wait();
            for (int i = 0; i < n_items && ok; ++i) {
                const QItem it = ITEM(i);
                const int64_t box = (int64_t)it.e * pairs + it.box;
                for (int kb = 0; kb < nkb && ok; ++kb) {
                    for (int t = 0; t < (is_b ? NTERMS : 1); ++t) {
                        if (issued >= pre) {
                            if (*abort_flag || !mbar_wait_bounded(&empty[s], ph ^ 1u, kQWaitNs)) {
                                ok = false;
                                break;
                            }
                            if (is_b) {
                                // the pass's rows only (the MMA reads N = nt rounded up to 16 of them)
                                const int64_t tile = (it.pass * nkb + kb) * NTERMS + t;
                                const uint32_t bytes = (uint32_t)((it.nt + 15) & ~15) * kQK;
                                mbar_arrive_expect_tx(&full[s], bytes + (uint32_t)kQSfBytes);
                                bulk_g2s_hint(sB + (size_t)s * kQBBytes, p.act + tile * kQBBytes, bytes, &full[s],
                                              pol);
                                bulk_g2s_hint(sBsf + (size_t)s * kQSfBytes, p.act_sf + tile * kQSfBytes, kQSfBytes,
                                              &full[s], pol);
                            } else {
                                load_a(s, box, kb);
                            }
                        }
                        ++issued;
                        if (++s == S) {
                            s = 0;
                            ph ^= 1u;
                        }
                    }
                }
            }
            if (!ok) {
                set_status(p.status, MXMOE_ERR_TIMEOUT);
                *abort_flag = 1;
            }
            issued = issued > pre ? issued : pre;  // the loads issued before the wait included
            for (int64_t f = issued > S ? issued - S : 0; f < issued; ++f)  // no copy in flight at exit
                if (!mbar_wait_bounded(&full[f % S], (uint32_t)((f / S) & 1), kQWaitNs)) {
                    set_status(p.status, MXMOE_ERR_TIMEOUT);
                    break;
                }
        }
    } else if (warp == kQWarpMma) {
        // ---------------------------------------------------------------- MMA
        // For every stage: the weight scale images into slot sa's columns, then
        // per term its scale images into slot sb's columns and, for each of the
        // stage's four 32-blocks, one MMA per tile: D_j += A_j * B_t^T. The
        // whole warp runs the loop (lane 0 waits, the verdict is shared); one
        // elected lane issues. Descriptors are stepped from per-ring bases.
        const bool leader = tc::elect_one();
        const uint64_t a_desc0 = tc::smem_desc(smem_u32(sA), 16, 1024, 2);
        const uint64_t b_desc0 = tc::smem_desc(smem_u32(sB), 16, 1024, 2);
        const uint32_t sfa_s0 = smem_u32(sAsf), sfb_s0 = smem_u32(sBsf);
        int sa = 0, sb = 0;
        uint32_t pha = 0, phb = 0;
        bool ok = true, any = false;
        for (int i = 0; i < n_items && ok; ++i) {
            const QItem it = ITEM(i);
            ok = q8_warp_wait(accempty, ((uint32_t)i & 1u) ^ 1u, abort_flag, p.status);
            if (!ok)
                break;
            tc::fence_after();
            const int n = (it.nt + 15) & ~15;
            uint32_t idesc[4];
#pragma unroll
            for (int k32 = 0; k32 < 4; ++k32)
                idesc[k32] = q8_idesc(n, (uint32_t)k32);
            for (int kb = 0; kb < nkb && ok; ++kb) {
                ok = q8_warp_wait(&full_a[sa], pha, abort_flag, p.status);
                if (!ok)
                    break;
                tc::fence_after();
                const uint32_t sfa_t = tmem + kQSfaCol0 + 8 * sa;
                const uint64_t a_desc = a_desc0 + (uint64_t)((sa * kQABytes) >> 4);
                if (leader) {
                    const uint32_t sfa_s = sfa_s0 + sa * kQSfBytes;
                    tc::cp_32x128b_warpx4(sfa_t, tc::smem_desc(sfa_s, 16, 128, 0));
                    tc::cp_32x128b_warpx4(sfa_t + 4, tc::smem_desc(sfa_s + 512, 16, 128, 0));
                }
                for (int t = 0; t < NTERMS; ++t) {
                    ok = q8_warp_wait(&full_b[sb], phb, abort_flag, p.status);
                    if (!ok)
                        break;
                    tc::fence_after();
                    if (leader) {
                        const uint32_t sfb_t = tmem + kQSfbCol0 + 8 * sb;
                        const uint32_t sfb_s = sfb_s0 + sb * kQSfBytes;
                        tc::cp_32x128b_warpx4(sfb_t, tc::smem_desc(sfb_s, 16, 128, 0));
                        tc::cp_32x128b_warpx4(sfb_t + 4, tc::smem_desc(sfb_s + 512, 16, 128, 0));
                        const uint64_t b_desc = b_desc0 + (uint64_t)((sb * kQBBytes) >> 4);
                        const uint32_t first = (kb > 0 || t > 0) ? 1u : 0u;
#pragma unroll
                        for (int k32 = 0; k32 < 4; ++k32)
#pragma unroll
                            for (int j = 0; j < 2; ++j)  // + 32 bytes of K per 32-block, + 16 KB per tile
                                q8_mma(tmem + (uint32_t)j * kQAccCols, a_desc + (uint64_t)(2 * k32 + 1024 * j),
                                       b_desc + (uint64_t)(2 * k32), idesc[k32], k32 > 0 ? 1u : first,
                                       (sfa_t + 4 * j) | ((uint32_t)k32 << 30), sfb_t | ((uint32_t)k32 << 30));
                        tc::commit(&empty_b[sb]);
                    }
                    __syncwarp();
                    any = true;
                    if (++sb == kQBStages) {
                        sb = 0;
                        phb ^= 1u;
                    }
                }
                if (ok && leader)
                    tc::commit(&empty_a[sa]);
                __syncwarp();
                if (++sa == kQAStages) {
                    sa = 0;
                    pha ^= 1u;
                }
            }
            if (ok && leader)
                tc::commit(accfull);
            __syncwarp();
        }
        if (!ok && lane == 0) {
            set_status(p.status, MXMOE_ERR_TIMEOUT);
            *abort_flag = 1;
        }
        if (any && leader) {  // every MMA and copy of ours completes before tensor memory is released
            tc::commit(mma_done);
            if (!mbar_wait_bounded(mma_done, 0, kQWaitNs))
                set_status(p.status, MXMOE_ERR_TIMEOUT);
        }
        __syncwarp();
    } else if (warp >= kQEpiWarp0) {
        // ----------------------------------------------------------- epilogue
        // Warp quarter q reads accumulator lanes 32q .. 32q+31 of both tiles,
        // 32 columns (tokens) at a time: chunks 2c + half for half = (warp - 4) / 4.
        const int q = warp & 3, half = (warp - kQEpiWarp0) >> 2;
        const uint32_t acc0 = tmem + ((uint32_t)(32 * q) << 16), acc1 = acc0 + kQAccCols;
        bool aborted = false;
        for (int i = 0; i < n_items; ++i) {
            const QItem it = ITEM(i);
            const int nt = it.nt;
            if (!aborted)
                aborted = !q8_warp_wait(accfull, (uint32_t)(i & 1), abort_flag, p.status);
            tc::fence_after();
            if (GATE_UP) {
                // lane: h column 128 box + 32q + lane (gate row of tile 0, up row of tile 1), value 32q + lane of
                // down stage `box`; the warp holds its 32-block q for every token
                const int nkb_d = p.I / kQK;
                uint8_t *hb = p.h_terms + ((it.pass * nkb_d + it.box) * 3) * (int64_t)kQBBytes;
                uint8_t *hs = p.h_sf + ((it.pass * nkb_d + it.box) * 3) * (int64_t)kQSfBytes;
                // Codes are made with lane = h column 32q + lane, four tokens per step; a byte transpose in
                // groups of 4 lanes leaves lane 4j + r with token r's codes of columns 32q + 4j .. 4j+3, one
                // word per term. off[s]: that word in the rows of the step's token r, by swizzle phase 4s + r
                // (chunks start at multiples of 32 tokens, so the phase is fixed by the step).
                const int r = lane & 3, c4 = 32 * q + 4 * (lane >> 2);
                const uint32_t sel1 = (r & 1) ? 0x3715u : 0x6240u, sel2 = (r & 2) ? 0x3276u : 0x5410u;
                int off[2];
#pragma unroll
                for (int s2 = 0; s2 < 2; ++s2)
                    off[s2] = r * 128 + (((c4 >> 4) ^ (4 * s2 + r)) << 4) + (c4 & 15);
                for (int n0 = 32 * half; n0 < nt && !aborted; n0 += 64) {
                    uint8_t *hrow = hb + (int64_t)n0 * 128;  // row n0 of the tiles
                    float g[32], u[32];
                    tc::ld_32x32b_x32(acc0 + (uint32_t)n0, g);
                    tc::ld_32x32b_x32(acc1 + (uint32_t)n0, u);
                    int Eown = 0;  // the block exponent of token n0 + lane, for the scale bytes written below
#pragma unroll
                    for (int t = 0; t < 32; t += 4) {
                        if (n0 + t >= nt)
                            break;
                        uint32_t w[3] = {0u, 0u, 0u};  // byte k of term i's word: the code of token t + k
#pragma unroll
                        for (int pr = 0; pr < 2; ++pr) {  // tokens t + 2pr, t + 2pr + 1, converted together
                            const int ta = t + 2 * pr;
                            const float ha = q8_silu(g[ta]) * u[ta], hb2 = q8_silu(g[ta + 1]) * u[ta + 1];
                            const uint32_t ma = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(ha) & 0x7FFFFFFFu);
                            const uint32_t mb = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(hb2) & 0x7FFFFFFFu);
                            const int Ea = max((int)(ma >> 23) - 127, -112), Eb = max((int)(mb >> 23) - 127, -112);
                            // on the scale of term 0 (h / 2^(E-7), below 256 in magnitude); each remainder is
                            // exact and times 16 is the next term's scale (2^(E-11), then 2^(E-15))
                            const float aa = ha * q8_pow2(7 - Ea), ab = hb2 * q8_pow2(7 - Eb);
                            const uint32_t c0 = q8_e4m3x2(aa, ab);
                            const float2 v0 = q8_e4m3x2_values(c0);
                            const float ba = (aa - v0.x) * 16.f, bb = (ab - v0.y) * 16.f;
                            const uint32_t c1 = q8_e4m3x2(ba, bb);
                            const float2 v1 = q8_e4m3x2_values(c1);
                            const uint32_t c2 = q8_e4m3x2((ba - v1.x) * 16.f, (bb - v1.y) * 16.f);
                            w[0] |= c0 << (16 * pr);
                            w[1] |= c1 << (16 * pr);
                            w[2] |= c2 << (16 * pr);
                            Eown = lane == ta ? Ea : (lane == ta + 1 ? Eb : Eown);
                        }
#pragma unroll
                        for (int i = 0; i < 3; ++i)
                            w[i] = q8_t4(w[i], sel1, sel2);
                        if (n0 + t + r < nt) {
                            uint32_t *pw = reinterpret_cast<uint32_t *>(hrow + t * 128 + off[(t >> 2) & 1]);
                            pw[0] = w[0];
                            pw[kQBBytes / 4] = w[1];
                            pw[2 * kQBBytes / 4] = w[2];
                        }
                    }
                    // scale bytes of the three terms: lane j those of token n0 + j, 32-block q of the stage
                    if (n0 + lane < nt) {
                        const int f = q8_sf_byte(n0 + lane, q);
                        hs[f] = (uint8_t)(Eown - 7 + 127);
                        hs[kQSfBytes + f] = (uint8_t)(Eown - 11 + 127);
                        hs[2 * kQSfBytes + f] = (uint8_t)(Eown - 15 + 127);
                    }
                }
            } else {
                // lane: y columns 256 box + 32q + lane (tile 0) and 256 box + 128 + 32q + lane (tile 1)
                const int c0 = 256 * it.box + 32 * q + lane, c1 = c0 + 128;
                float *dst = p.y + (int64_t)it.r0 * p.H;
                for (int n0 = 32 * half; n0 < nt && !aborted; n0 += 64) {
                    float v0[32], v1[32];
                    tc::ld_32x32b_x32(acc0 + (uint32_t)n0, v0);
                    tc::ld_32x32b_x32(acc1 + (uint32_t)n0, v1);
#pragma unroll
                    for (int t = 0; t < 32; ++t)
                        if (n0 + t < nt) {
                            if (c0 < p.H)
                                dst[(int64_t)(n0 + t) * p.H + c0] = v0[t];
                            if (c1 < p.H)
                                dst[(int64_t)(n0 + t) * p.H + c1] = v1[t];
                        }
                }
            }
            tc::fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(accempty);
        }
    }
    tc::fence_before();
    __syncthreads();
    if (warp == kQWarpMma) {
        tc::fence_after();
        tc::dealloc(tmem, 512);
    }
#undef ITEM
}

template <bool GATE_UP>
int launch_f8_stage(const CUtensorMap &tmW, const Q8Params &p, cudaStream_t st)
{
    static thread_local int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        if (cudaFuncSetAttribute(ffn_f8_kernel<GATE_UP>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kQSmem) !=
            cudaSuccess)
            return fail(MXMOE_ERR_CUDA, "ffn_f8_kernel: cannot reserve %zu bytes of shared memory", kQSmem);
        configured_dev = dev;
    }
    return launch_kernel(GATE_UP ? "ffn_f8_kernel<gate_up>" : "ffn_f8_kernel<down>", ffn_f8_kernel<GATE_UP>,
                         num_sms(), kQThreads, kQSmem, st, tmW, p);
}

}  // namespace

// A 2-D tensor map: `outer` rows of row_bytes bytes, `inner` elements of
// `type` each, boxes of box_inner x box_outer.
int encode2d_any(CUtensorMap *m, CUtensorMapDataType type, const void *base, uint64_t inner, uint64_t outer,
             uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle, const char *what)
{
    auto enc = tensor_map_encoder();
    if (!enc)
        return fail(MXMOE_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer}, es[2] = {1, 1};
    CUresult r = enc(m, type, 2, const_cast<void *>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(MXMOE_ERR_CUDA, "cuTensorMapEncodeTiled (%s) failed: %d", what, (int)r);
    return MXMOE_OK;
}

// Token passes of up to `tok` rows before each expert with at least min_rows
// rows (pass_start, E + 1 ints; E <= 1024); clears the status word when given.
int run_pass_prefix(const int32_t *offsets, int E, int min_rows, int tok, int32_t *pass_start, int *status,
                    cudaStream_t st)
{
    return launch_kernel("prefill_passes_kernel", prefill_passes_kernel, 1, 1024, 0, st, offsets, E, min_rows, tok,
                         pass_start, status);
}

// slot_row[src_row[r]] = r for the rows grouped pairs.
int run_slot_rows(const int32_t *src_row, int rows, int32_t *slot_row, cudaStream_t st)
{
    const int blocks = (int)std::min<int64_t>(((int64_t)rows + 255) / 256, (int64_t)num_sms() * 4);
    return launch_kernel("slot_rows_kernel", slot_rows_kernel, blocks < 1 ? 1 : blocks, 256, 0, st, src_row, rows,
                         slot_row);
}

// Upper bound on the 224-token passes of `rows` grouped rows over E experts
// when only experts with at least min_rows rows count.
int64_t f8_max_passes(int64_t rows, int E, int min_rows)
{
    const int64_t experts = min_rows > 0 ? std::min<int64_t>(E, rows / min_rows) : E;
    return (rows + kQTok - 1) / kQTok + experts;
}

// Bytes of one stage's activation terms (NTERMS 2 for x, 3 for h) over all
// passes, and of their scale images.
int64_t f8_terms_bytes(int64_t passes, int K, int nterms) { return passes * (K / kQK) * nterms * (int64_t)kQBBytes; }
int64_t f8_sf_bytes(int64_t passes, int K, int nterms) { return passes * (K / kQK) * nterms * (int64_t)kQSfBytes; }

// Before the gate/up stage: the 224-token passes before each expert with at
// least min_rows rows (pass_start), then those experts' x rows as two E4M3
// terms per value tiled per (pass, stage, term) into x_terms / x_sf, through
// slot_row (the grouped row of each (token, slot)); clears the status word
// when given. E <= 1024, k <= 32.
int run_f8_prep(const void *x, const int32_t *offsets, const int32_t *src_row, int k, int rows, int E, int H,
                int min_rows, int32_t *pass_start, int32_t *slot_row, uint8_t *x_terms, uint8_t *x_sf, int *status,
                cudaStream_t st)
{
    if (int rc = run_pass_prefix(offsets, E, min_rows, kQTok, pass_start, status, st))
        return rc;
    if (int rc = run_slot_rows(src_row, rows, slot_row, st))
        return rc;
    const int T = rows / k;
    // stage ranges per token: about 48 warps per SM in all
    const int nkb = H / kQK;
    const int groups = (int)std::max<int64_t>(1, std::min<int64_t>(nkb, ((int64_t)num_sms() * 48 + T - 1) / T));
    const int64_t units = (int64_t)T * groups;
    const int blocks = (int)std::min<int64_t>((units + 7) / 8, (int64_t)num_sms() * 8);
    if (k <= 8)
        return launch_kernel("x8_terms_kernel", x8_terms_kernel<8>, blocks < 1 ? 1 : blocks, 256, 0, st,
                             static_cast<const uint16_t *>(x), slot_row, offsets, pass_start, E, min_rows, k, T, H,
                             groups, x_terms, x_sf);
    return launch_kernel("x8_terms_kernel", x8_terms_kernel<kQMaxK>, blocks < 1 ? 1 : blocks, 256, 0, st,
                         static_cast<const uint16_t *>(x), slot_row, offsets, pass_start, E, min_rows, k, T, H, groups,
                         x_terms, x_sf);
}

// One FFN stage on the block-scaled fp8-kind tensor cores.
//  gate/up: terms = x's (run_f8_prep); w, sf = the gate/up code boxes and
//           scale images of the blob; writes h's three terms (h_terms, h_sf).
//  down:    terms = h's; w, sf = the down part of the blob; writes y (fp32
//           [rows][H]).
int run_f8_stage(bool gate_up, const uint8_t *terms, const uint8_t *terms_sf, const int32_t *offsets,
                 const int32_t *pass_start, const uint8_t *w, const uint8_t *sf, int E, int H, int I, uint8_t *h_terms,
                 uint8_t *h_sf, float *y, int *status, cudaStream_t st)
{
    const int K = gate_up ? H : I;
    const int nchunk = (K + 255) / 256;
    const int pairs = gate_up ? I / 128 : (H + 255) / 256;
    const int64_t blob_rows = (int64_t)E * pairs * nchunk * 256;
    CUtensorMap tmW;  // the packed codes (a 128-byte row = 256 values), unpacked to a byte each, 128 values x 256 rows
    if (int rc = encode2d_any(&tmW, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, w, 256, (uint64_t)blob_rows, 128, 128, 256,
                              CU_TENSOR_MAP_SWIZZLE_128B, "fp8-kind stage weights"))
        return rc;
    Q8Params p{};
    p.pairs = pairs;
    p.nkb = K / kQK;
    p.nchunk = nchunk;
    p.H = H;
    p.I = I;
    p.E = E;
    p.offsets = offsets;
    p.pass_start = pass_start;
    p.act = terms;
    p.act_sf = terms_sf;
    p.wsf = sf;
    p.h_terms = h_terms;
    p.h_sf = h_sf;
    p.y = y;
    p.status = status;
    return gate_up ? launch_f8_stage<true>(tmW, p, st) : launch_f8_stage<false>(tmW, p, st);
}

}  // namespace mxmoe
