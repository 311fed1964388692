// ffn_prefill.cu -- the gate/up stage of the expert FFN for large token counts,
// on bf16 tcgen05 tensor cores with the MXFP4 weights dequantised in shared
// memory.
//
// Pages: "MiMo-V2.5-Pro-FP4-DFlash" model card, section 2 "FP4 Quantization"
// (MXFP4 experts, block size 32); nxbn.cn MiMo-V2.5-Pro-FP4-DFlash article,
// architecture section (384 experts, 8 per token, hidden 6144). The expert is
// read as a SwiGLU FFN with no biases; h = silu(W_gate x) * (W_up x).
//
// When an expert sees hundreds of tokens the stage is bound by the tensor
// cores, not by the weight stream, and the E2M1 activation terms of the decode
// kernel would spend most of every MMA on terms. Here each weight tile is
// dequantised once per pass of up to 256 tokens, exactly (an E2M1 value times
// its power-of-two scale is a bf16 value), and multiplied with the bf16 x rows
// as they are (tcgen05.mma.kind::f16, fp32 accumulation):
//  * a producer warp brings, per 64-value K step, the packed codes of 64 gate
//    and 64 up rows (two TMA boxes of the prepacked blob), the scale images of
//    their 256-K chunk, and 256 grouped x rows (one TMA box);
//  * four dequantising warps write the 128 x 64 bf16 weight tile into shared
//    memory in the 128-byte-swizzled K-major layout the MMA reads, one row per
//    thread; tile row 32q + w is gate row 16q + w (w < 16) or the matching up
//    row (w >= 16), so gate and up of one column meet in one warp;
//  * an MMA warp issues four M = 128, N <= 256, K = 16 MMAs per step into one
//    of two accumulators (128 lanes x 256 columns each);
//  * four epilogue warps apply SwiGLU and write h in fp32 (grouped rows),
//    which the down stage then encodes into its E2M1 digit terms.
// All waits are bounded; on a timeout the kernel records MXMOE_ERR_TIMEOUT in
// the workspace status word and returns.
#include <algorithm>
#include <mutex>

#include <cudaTypedefs.h>

#include "common.cuh"
#include "tcgen05.cuh"

namespace mxmoe {
namespace {

constexpr uint64_t kPWaitNs = 2000000000ull;  // bounded waits: 2 s
constexpr int kPThreads = 320;    // producer, MMA, 4 dequantising warps, 4 epilogue warps
constexpr int kPStages = 4;
constexpr int kPK = 64;           // K per step
constexpr int kPTok = 256;        // tokens per pass (MMA N at most)
constexpr int kPXBytes = kPTok * 128;  // x step: 256 rows x 64 bf16
constexpr int kPABytes = 128 * 128;    // bf16 weight step: 128 rows x 64 bf16
constexpr int kPWBytes = 128 * 32;     // packed codes of a step: 128 rows x 64 codes
constexpr int kPSfBytes = 2048;        // scale images of one 256-K chunk of a 256-row blob box
constexpr int kPMaxE = 1024;

struct PrefillParams {
    int tiles;                // 128-row (64 gate + 64 up) weight tiles per expert: I / 64
    int H, I, E, rows;
    int nchunk;               // 256-K chunks per blob row (H padded to 256)
    const int32_t *offsets;   // [E+1]
    const uint8_t *sf13;      // gate/up scale images of the prepacked blob
    float *h;                 // out: [rows, I] fp32
    int *status;
};

// shared memory: x steps | bf16 weight steps | packed code steps | scale images | barriers | misc | offsets
constexpr size_t kPOffA = (size_t)kPStages * kPXBytes;
constexpr size_t kPOffW = kPOffA + (size_t)kPStages * kPABytes;
constexpr size_t kPOffSf = kPOffW + (size_t)kPStages * kPWBytes;
constexpr size_t kPOffBar = kPOffSf + (size_t)kPStages * kPSfBytes;
constexpr int kPBars = 3 * kPStages + 5;  // full, aready, empty per stage; accfull[2], accempty[2], mma_done
constexpr size_t kPOffMisc = (kPOffBar + kPBars * 8 + 15) & ~size_t(15);
constexpr size_t kPOffOffsets = kPOffMisc + 64;
constexpr size_t kPOffItems = kPOffOffsets + (kPMaxE + 1) * 4;  // items before each expert [kPMaxE + 1]
constexpr size_t kPSmem = 1024 + kPOffItems + (kPMaxE + 1) * 4;
static_assert(kPSmem <= 232448, "shared memory");

// x rows gathered into grouped order (row r = token src_row[r] / k), so that
// a pass of an expert is a contiguous row range for TMA; 16 bytes per thread.
// Block 0 also clears the status word.
__global__ void __launch_bounds__(256) x_gather_kernel(const uint16_t *__restrict__ x,
                                                       const int32_t *__restrict__ src_row, int k, int rows, int H,
                                                       uint16_t *__restrict__ x_perm, int *status)
{
    if (blockIdx.x == 0 && threadIdx.x == 0 && status)
        *status = 0;
    const int per_row = H / 8;  // 16-byte units
    const int64_t total = (int64_t)rows * per_row;
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < total; u += (int64_t)gridDim.x * blockDim.x) {
        const int r = (int)(u / per_row), c = (int)(u % per_row);
        const int tok = src_row[r] / k;
        reinterpret_cast<uint4 *>(x_perm)[u] = __ldg(reinterpret_cast<const uint4 *>(x + (int64_t)tok * H) + c);
    }
}

// Work items: (expert, pass of up to 256 tokens, 128-row weight tile), in that
// order. CTA b takes items b, b + G, b + 2G, ... (G CTAs), so that at any time
// the grid works on a few consecutive expert passes and their x rows stay in
// L2 while every weight tile is read once. Every role decodes the same items.
struct PItem {
    int e, pass, tile, r0, nt;
};

__device__ __forceinline__ PItem decode_item(int64_t idx, const int32_t *items, const int32_t *off, int E, int tiles)
{
    int lo = 0, hi = E;  // largest e with items[e] <= idx
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (items[mid] <= idx)
            lo = mid;
        else
            hi = mid;
    }
    PItem it;
    it.e = lo;
    const int local = (int)(idx - items[lo]);
    it.pass = local / tiles;
    it.tile = local % tiles;
    it.r0 = off[lo] + it.pass * kPTok;
    it.nt = min(kPTok, off[lo + 1] - it.r0);
    return it;
}

__device__ __forceinline__ uint32_t idesc_bf16(int n)  // kind::f16, bf16 x bf16 -> f32, K-major, M = 128
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | (8u << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0)
        : "memory");
}

__global__ void __launch_bounds__(kPThreads, 1)
    ffn_bf16_gate_up_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                            const PrefillParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sX = smem, *sA = smem + kPOffA, *sW = smem + kPOffW, *sSf = smem + kPOffSf;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kPOffBar);
    uint64_t *aready = full + kPStages;
    uint64_t *empty = aready + kPStages;
    uint64_t *accfull = empty + kPStages;  // [2]
    uint64_t *accempty = accfull + 2;      // [2]
    uint64_t *mma_done = accempty + 2;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + kPOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);
    int32_t *s_off = reinterpret_cast<int32_t *>(smem + kPOffOffsets);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int E = p.E, tiles = p.tiles;
    for (int e = tid; e <= E; e += kPThreads)
        s_off[e] = p.offsets[e];
    __syncthreads();
    int32_t *s_items = reinterpret_cast<int32_t *>(smem + kPOffItems);
    if (warp == 0) {  // items before each expert: sum of ceil(n_e / 256) * tiles
        int carry = 0;
        for (int b = 0; b <= E; b += 32) {
            const int e = b + lane;
            const int c = e < E ? tiles * ((s_off[e + 1] - s_off[e] + kPTok - 1) / kPTok) : 0;
            int incl = c;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
                if (lane >= off)
                    incl += o;
            }
            if (e <= E)
                s_items[e] = carry + incl - c;
            carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
    }
    if (tid == 32) {
        for (int s = 0; s < kPStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&aready[s], 4);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accfull[b], 1);
            mbar_init(&accempty[b], 4);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1)
        tc::alloc(tslot, 512);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *tslot;
    const int64_t total = s_items[E];
    const int64_t G = gridDim.x;
    const int n_items = (int)(total > blockIdx.x ? (total - blockIdx.x + G - 1) / G : 0);
#define ITEM(i) decode_item(blockIdx.x + (int64_t)(i) * G, s_items, s_off, E, tiles)
    const int nks = p.H / kPK;            // K steps
    const int wtiles = p.I / 128;         // 256-row blob tiles per expert (gate/up)

    if (warp == 0) {
        // ----------------------------------------------------------- producer
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_first();
            const uint64_t pol_x = policy_evict_last();
            int s = 0;
            uint32_t ph = 0;
            int64_t issued = 0;
            bool ok = true;
            for (int i = 0; i < n_items && ok; ++i) {
                const PItem it = ITEM(i);
                const int r0 = it.r0;
                const int64_t tile_box = (int64_t)it.e * wtiles + (it.tile >> 1);  // blob 256-row tile
                const int half = it.tile & 1;
                for (int ks = 0; ks < nks; ++ks) {
                    if (*abort_flag || !mbar_wait_bounded(&empty[s], ph ^ 1u, kPWaitNs)) {
                        ok = false;
                        break;
                    }
                    const int c = ks >> 2;  // 256-K chunk
                    const int64_t row0 = (tile_box * p.nchunk + c) * 256;
                    mbar_arrive_expect_tx(&full[s], (uint32_t)(kPWBytes + kPSfBytes + kPXBytes));
                    uint8_t *w = sW + (size_t)s * kPWBytes;
                    tc::tma_load_2d(w, &tmW, 32 * (ks & 3), (int)(row0 + 64 * half), &full[s], pol_w);
                    tc::tma_load_2d(w + kPWBytes / 2, &tmW, 32 * (ks & 3), (int)(row0 + 128 + 64 * half), &full[s],
                                    pol_w);
                    bulk_g2s_hint(sSf + (size_t)s * kPSfBytes, p.sf13 + (tile_box * p.nchunk + c) * kPSfBytes,
                                  kPSfBytes, &full[s], pol_w);
                    tc::tma_load_2d(sX + (size_t)s * kPXBytes, &tmX, kPK * ks, r0, &full[s], pol_x);
                    ++issued;
                    if (++s == kPStages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (!ok) {
                set_status(p.status, MXMOE_ERR_TIMEOUT);
                *abort_flag = 1;
            }
            for (int64_t f = issued > kPStages ? issued - kPStages : 0; f < issued; ++f)
                if (!mbar_wait_bounded(&full[f % kPStages], (uint32_t)((f / kPStages) & 1), kPWaitNs)) {
                    set_status(p.status, MXMOE_ERR_TIMEOUT);
                    break;
                }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            bool ok = true, any = false;
            for (int i = 0; i < n_items && ok; ++i) {
                const PItem it = ITEM(i);
                const int buf = i & 1;
                const uint32_t use = (uint32_t)(i >> 1);
                if (*abort_flag || !mbar_wait_bounded(&accempty[buf], (use & 1u) ^ 1u, kPWaitNs)) {
                    ok = false;
                    break;
                }
                tc::fence_after();
                const uint32_t idesc = idesc_bf16((it.nt + 15) & ~15);  // N: the pass's tokens, rounded up to 16
                const uint32_t d_tmem = tmem + (uint32_t)buf * 256;
                for (int ks = 0; ks < nks; ++ks) {
                    if (*abort_flag || !mbar_wait_bounded(&full[s], ph, kPWaitNs) ||
                        !mbar_wait_bounded(&aready[s], ph, kPWaitNs)) {
                        ok = false;
                        break;
                    }
                    tc::fence_after();
                    const uint32_t a_base = smem_u32(sA + (size_t)s * kPABytes);
                    const uint32_t b_base = smem_u32(sX + (size_t)s * kPXBytes);
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4)  // 16 values of K per MMA
                        mma_bf16(d_tmem, tc::smem_desc(a_base + 32 * k4, 16, 1024, 2),
                                 tc::smem_desc(b_base + 32 * k4, 16, 1024, 2), idesc, (ks > 0 || k4 > 0) ? 1u : 0u);
                    tc::commit(&empty[s]);
                    any = true;
                    if (++s == kPStages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (ok)
                    tc::commit(&accfull[buf]);
            }
            if (!ok) {
                set_status(p.status, MXMOE_ERR_TIMEOUT);
                *abort_flag = 1;
            }
            if (any) {
                tc::commit(mma_done);
                if (!mbar_wait_bounded(mma_done, 0, kPWaitNs))
                    set_status(p.status, MXMOE_ERR_TIMEOUT);
            }
        }
    } else if (warp <= 5) {
        // ------------------------------------------------------ dequantising
        // Thread m writes tile row m: gate row 16q + w of the tile's 64 gate
        // rows (w < 16) or the matching up row, from the packed step in shared
        // memory and its two E8M0 scales, as 64 bf16 values (exact) in the
        // 128-byte swizzle: 16-byte chunk c of row m lands at chunk c ^ (m % 8).
        const int m = tid - 64;
        const int q = m >> 5, w = m & 31;
        const int src = (w < 16 ? 0 : kPWBytes / 2) + (16 * q + (w & 15)) * 32;
        int s = 0;
        uint32_t ph = 0;
        bool aborted = false;
        for (int i = 0; i < n_items; ++i) {
            const PItem it = ITEM(i);
            // row of the 256-row blob box: gate rows 0..127, up rows 128..255
            const int R = (w < 16 ? 0 : 128) + 64 * (it.tile & 1) + 16 * q + (w & 15);
            const int img = (R >> 7), rr = R & 127;
            const int img_byte = (rr & 31) * 16 + (rr >> 5) * 4;
            for (int ks = 0; ks < nks; ++ks) {
                if (!aborted) {  // lane 0 waits; the warp follows its verdict
                    int okv = 1;
                    if (lane == 0 && (*abort_flag || !mbar_wait_bounded(&full[s], ph, kPWaitNs))) {
                        set_status(p.status, MXMOE_ERR_TIMEOUT);
                        *abort_flag = 1;
                        okv = 0;
                    }
                    aborted = !__shfl_sync(0xFFFFFFFFu, okv, 0);
                }
                if (!aborted) {
                    const uint8_t *wrow = sW + (size_t)s * kPWBytes + src;
                    const uint4 c0 = *reinterpret_cast<const uint4 *>(wrow);
                    const uint4 c1 = *reinterpret_cast<const uint4 *>(wrow + 16);
                    // k32 blocks 2(ks%4) and 2(ks%4)+1 of the chunk: K half (ks%4)/2, bytes 2(ks%2), +1
                    const int q4 = ks & 3;
                    const uint8_t *sfp = sSf + (size_t)s * kPSfBytes + ((q4 >> 1) * 2 + img) * 512 + img_byte +
                                         2 * (q4 & 1);
                    const float sc0 = e8m0_to_float(sfp[0]), sc1 = e8m0_to_float(sfp[1]);
                    uint8_t *arow = sA + (size_t)s * kPABytes + m * 128;
                    const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {  // 8 values per 16-byte chunk
                        const float sc = ch < 4 ? sc0 : sc1;
                        uint32_t hh[4];
                        e2m1x4_to_f16x2x4(words[ch], hh[0], hh[1], hh[2], hh[3]);
                        uint32_t out[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const __half2 hv = *reinterpret_cast<const __half2 *>(&hh[j]);
                            const __nv_bfloat162 b =
                                __floats2bfloat162_rn(__low2float(hv) * sc, __high2float(hv) * sc);
                            out[j] = *reinterpret_cast<const uint32_t *>(&b);
                        }
                        *reinterpret_cast<uint4 *>(arow + ((ch ^ (m & 7)) << 4)) =
                            make_uint4(out[0], out[1], out[2], out[3]);
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                }
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&aready[s]);
                if (++s == kPStages) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
    } else {
        // ----------------------------------------------------------- epilogue
        // Warp quarter q holds accumulator lanes 32q .. 32q+31: lanes w < 16
        // the gate rows of h columns 64 * tile + 16q + w, lanes w + 16 the
        // matching up rows; columns are the pass's tokens.
        const int q = warp & 3;
        bool aborted = false;
        for (int i = 0; i < n_items; ++i) {
            const PItem it = ITEM(i);
            const int buf = i & 1;
            const uint32_t use = (uint32_t)(i >> 1);
            if (!aborted) {
                int okv = 1;
                if (lane == 0 && (*abort_flag || !mbar_wait_bounded(&accfull[buf], use & 1u, kPWaitNs))) {
                    set_status(p.status, MXMOE_ERR_TIMEOUT);
                    *abort_flag = 1;
                    okv = 0;
                }
                aborted = !__shfl_sync(0xFFFFFFFFu, okv, 0);
            }
            tc::fence_after();
            const int nt = it.nt;
            const int64_t r0 = it.r0;
            const int col = 64 * it.tile + 16 * q + (lane & 15);
            for (int n0 = 0; n0 < nt && !aborted; n0 += 32) {
                float v[32];
                tc::ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * 256 + n0), v);
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float g = v[j];
                    const float u = __shfl_down_sync(0xFFFFFFFFu, g, 16);
                    if (lane < 16 && n0 + j < nt)
                        p.h[(r0 + n0 + j) * p.I + col] = g / (1.f + expf(-g)) * u;
                }
            }
            tc::fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&accempty[buf]);
        }
    }
    tc::fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after();
        tc::dealloc(tmem, 512);
    }
#undef ITEM
}

int encode2d(CUtensorMap *m, CUtensorMapDataType type, const void *base, uint64_t inner, uint64_t outer,
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

}  // namespace

// Gate/up stage on bf16 tensor cores: x rows gathered into grouped order, then
// h = silu(W_gate x) * (W_up x) for every grouped row into h (fp32 [T*k, I]).
// w13 / sf13: the gate/up code boxes and scale images of the prepacked blob.
// Requires I % 64 == 0 (I % 128 == 0 holds for every accepted shape).
int run_bf16_gate_up(const void *x, const int32_t *offsets, const int32_t *src_row, const uint8_t *w13,
                     const uint8_t *sf13, int T, int k, int E, int H, int I, uint16_t *x_perm, float *h, int *status,
                     cudaStream_t st)
{
    const int rows = T * k;
    {
        const int64_t units = (int64_t)rows * (H / 8);
        const int blocks = (int)std::min<int64_t>((units + 255) / 256, (int64_t)num_sms() * 8);
        x_gather_kernel<<<blocks < 1 ? 1 : blocks, 256, 0, st>>>(static_cast<const uint16_t *>(x), src_row, k, rows,
                                                                  H, x_perm, status);
        if (int rc = check_launch("x_gather_kernel"))
            return rc;
    }
    const int nchunk = (H + 255) / 256;
    const int64_t blob_rows = (int64_t)E * (I / 128) * nchunk * 256;
    CUtensorMap tmW, tmX;
    if (int rc = encode2d(&tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, w13, 128, (uint64_t)blob_rows, 128, 32, 64,
                          CU_TENSOR_MAP_SWIZZLE_NONE, "prefill weights"))
        return rc;
    if (int rc = encode2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x_perm, (uint64_t)H, (uint64_t)rows,
                          (uint64_t)H * 2, kPK, kPTok, CU_TENSOR_MAP_SWIZZLE_128B, "prefill x"))
        return rc;
    static thread_local int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        if (cudaFuncSetAttribute(ffn_bf16_gate_up_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kPSmem) != cudaSuccess)
            return fail(MXMOE_ERR_CUDA, "ffn_bf16_gate_up_kernel: cannot reserve %zu bytes of shared memory", kPSmem);
        configured_dev = dev;
    }
    PrefillParams p{};
    p.tiles = I / 64;
    p.H = H;
    p.I = I;
    p.E = E;
    p.rows = rows;
    p.nchunk = nchunk;
    p.offsets = offsets;
    p.sf13 = sf13;
    p.h = h;
    p.status = status;
    ffn_bf16_gate_up_kernel<<<num_sms(), kPThreads, kPSmem, st>>>(tmW, tmX, p);
    return check_launch("ffn_bf16_gate_up_kernel");
}

}  // namespace mxmoe
