// ffn_prefill.cu -- both stages of the expert FFN for large token counts, on
// bf16 tcgen05 tensor cores with the MXFP4 weights dequantised in shared
// memory.
//
// Pages: "MiMo-V2.5-Pro-FP4-DFlash" model card, section 2 "FP4 Quantization"
// (MXFP4 experts, block size 32); nxbn.cn MiMo-V2.5-Pro-FP4-DFlash article,
// architecture section (384 experts, 8 per token, hidden 6144). The expert is
// read as a SwiGLU FFN with no biases: h = silu(W_gate x) * (W_up x),
// y = W_down h.
//
// When an expert sees hundreds of tokens the FFN is bound by the tensor cores,
// and the E2M1 activation terms of the decode kernel would spend most of every
// MMA on terms. Here each weight tile is dequantised once per pass of up to 256
// tokens, exactly (an E2M1 value times its power-of-two scale is a bf16 value),
// and multiplied with bf16 activations (tcgen05.mma.kind::f16, fp32
// accumulation): x as it is (exact), h as two bf16 terms hi + lo (within 2^-15
// of h), which the down stage stacks along K so that one accumulator column
// sums both.
//  * A work item is (expert, pass of up to 256 tokens, one 256-row box of the
//    prepacked blob) = two 128-row MMA tiles. A K step is 64 values.
//  * Three rings in shared memory, each with its own producer or writer, so
//    that no role waits on another's latency: activation steps (bulk copies,
//    2 x 32 KB; one step per K step for gate/up, two for down: hi then lo),
//    packed weights with their scale images (TMA + bulk copy, 3 x 17 KB of two
//    K steps each, issued by a second producer warp ahead), and dequantised
//    bf16 weight tiles (3 x 32 KB, written by sixteen warps, two threads per
//    row, in the 128-byte-swizzled K-major layout the MMA reads).
//  * Two MMA warps each own one tile and one accumulator (128 lanes x 256
//    columns, together all of tensor memory), so that the tiles' MMAs are
//    issued independently and each accumulator has its own epilogue warps.
//  * Eight epilogue warps, four per accumulator, drain both at once: gate/up
//    applies SwiGLU (tile row 32q + w is gate row 16q + w of the tile's 64,
//    w < 16, or the matching up row) and writes h as bf16 hi/lo terms; down
//    writes y in fp32.
//  * Items go round-robin over a persistent grid of one CTA per SM, so the
//    few expert passes in flight keep their activations in L2 while every
//    weight box is read once per pass.
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
constexpr int kPThreads = 896;  // 28 warps: see the role list at the kernel
constexpr int kPK = 64;         // K per step
constexpr int kPTok = 256;      // tokens per pass
constexpr int kPBStages = 2;    // activation ring
constexpr int kPWStages = 3;    // packed weight ring (a slot holds two K steps)
constexpr int kPAStages = 3;    // dequantised weight ring (a third slot measured faster than a third activation slot)
constexpr int kPBBytes = kPTok * 128;  // activation step: 256 rows x 64 bf16
constexpr int kPABytes = 128 * 128;    // one bf16 weight tile step: 128 rows x 64 bf16
constexpr int kPWBytes = 256 * 64;     // packed codes of two K steps: 256 rows x 128 codes
constexpr int kPSfBytes = 1024;        // their two scale images (one K half of a chunk, both row halves)
struct PrefillParams {
    int pairs;                // 256-row blob boxes per expert: I/128 (gate/up) or Hp/256 (down)
    int K;                    // H (gate/up) or I (down)
    int nchunk;               // 256-K chunks per blob row (K padded to 256)
    int H, I, E, rows;
    const int32_t *offsets;   // [E+1]
    const int32_t *pass_start;  // [E+1]: 256-token passes before each expert
    const uint8_t *act;       // tiled activations: x, or h's hi and lo (one 32 KB block per pass, K step, term)
    const uint8_t *sf;        // scale images of the stage's blob part
    uint8_t *h_tiled;         // gate/up out: h hi, lo tiled for the down stage
    float *y;                 // down out: [rows, H]
    int *status;
};

// shared memory: activation ring | dequantised ring (2 tiles a step) | packed ring | scale images | barriers |
// misc
constexpr size_t kPOffA = (size_t)kPBStages * kPBBytes;
constexpr size_t kPOffW = kPOffA + (size_t)kPAStages * 2 * kPABytes;
constexpr size_t kPOffSf = kPOffW + (size_t)kPWStages * kPWBytes;
constexpr size_t kPOffBar = kPOffSf + (size_t)kPWStages * kPSfBytes;
// full_b, empty_b, full_w, empty_w, aready, aempty, accfull[2], accempty[2], mma_done[2]
constexpr int kPBars = 2 * kPBStages + 2 * kPWStages + 2 * kPAStages + 6;
constexpr size_t kPOffMisc = (kPOffBar + kPBars * 8 + 15) & ~size_t(15);
constexpr size_t kPSmem = 1024 + kPOffMisc + 64;
static_assert(kPSmem <= 232448, "shared memory");

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

// x rows in grouped order, tiled as the bf16 stage reads them: the block of
// (pass, K step) holds the pass's 256 rows x 64 values in the 128-byte
// swizzle (16-byte chunk c of row m at chunk c ^ (m % 8)), 32 KB, so that one
// bulk copy brings a whole activation step. Grouped row r of expert e is row
// r - offsets[e] - 256 p of pass p of e; rows past an expert's last token are
// left as they are (the FFN ignores their columns), and rows of experts with
// fewer than min_rows rows are skipped. One warp per token: lane j < k finds
// where the token's slot j goes, then the warp reads x[t] once and writes it
// to every such place.
constexpr int kTileMaxK = 32;

__global__ void __launch_bounds__(256) x_tile_kernel(const uint16_t *__restrict__ x,
                                                     const int32_t *__restrict__ slot_row,
                                                     const int32_t *__restrict__ offsets,
                                                     const int32_t *__restrict__ pass_start, int E, int min_rows,
                                                     int k, int T, int H, uint8_t *__restrict__ x_tiled)
{
    grid_dep_wait();  // the preceding kernel's results (chained launch)
    grid_dep_launch();
    __shared__ int64_t s_dst[8][kTileMaxK];  // per warp: byte offset of slot j's row in x_tiled, or -1
    const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5;
    const int nks = H / kPK;
    if (__ldg(pass_start + E) == 0)  // no expert for the bf16 kernel
        return;
    for (int t = blockIdx.x * 8 + wl; t < T; t += gridDim.x * 8) {
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
            int64_t d = -1;
            if (__ldg(offsets + lo + 1) - __ldg(offsets + lo) >= min_rows) {
                const int64_t pass = __ldg(pass_start + lo) + local / kPTok;
                const int m = local % kPTok;
                d = (pass * nks * kPTok + m) * 128 + m % 8;  // m % 8 rides along for the swizzle
            }
            s_dst[wl][lane] = d;
        }
        __syncwarp();
        const uint4 *src = reinterpret_cast<const uint4 *>(x + (int64_t)t * H);
        for (int c8 = lane; c8 < H / 8; c8 += 32) {  // 16-byte chunk c8: K step c8 / 8, chunk c8 % 8
            const uint4 v = __ldg(src + c8);
            const int c = c8 & 7;
            const int64_t step = (int64_t)(c8 >> 3) * kPBBytes;
            for (int j = 0; j < k; ++j) {
                const int64_t d = s_dst[wl][j];
                if (d >= 0) {
                    const int64_t row = d & ~int64_t(7);
                    *reinterpret_cast<uint4 *>(x_tiled + row + step + ((c ^ (int)(d & 7)) << 4)) = v;
                }
            }
        }
        __syncwarp();
    }
}

// Work items: (pass of up to 256 tokens, 256-row blob box), passes in expert
// order: item i is box i % pairs of pass i / pairs. CTA b takes items b,
// b + G, b + 2G, ... (G CTAs), so that at any time the grid works on a few
// consecutive passes and their activation steps stay in L2 while every weight
// box is read once per pass. Every role decodes the same items.
struct PItem {
    int e, box, r0, nt;
    int64_t pass;  // global pass index: the block row of the tiled activations
};

__device__ __forceinline__ PItem decode_item(int64_t idx, const int32_t *__restrict__ pass_start,
                                             const int32_t *__restrict__ off, int E, int pairs)
{
    PItem it;
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
    it.r0 = __ldg(off + lo) + (int)(it.pass - __ldg(pass_start + lo)) * kPTok;
    it.nt = min(kPTok, __ldg(off + lo + 1) - it.r0);
    return it;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Byte tables for dequantising E2M1 codes with prmt: entry i (i = 0..7) is the
// bf16 value of the E2M1 magnitude i (0, 0.5, 1, 1.5, 2, 3, 4, 6) times the
// block scale f, rounded to nearest (exact for every scale that keeps the
// products normal). lo0/lo1 hold the entries' low bytes (entries 0-3, 4-7),
// hi0/hi1 their high bytes; the sign bit of every entry is 0.
struct Bf16Tab {
    uint32_t lo0, lo1, hi0, hi1;
};

__device__ __forceinline__ uint32_t bf16x2_bits(float a, float b)  // a in the low half
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&v);
}

// Table for the E8M0 scale byte s (f = 2^(s-127)). For 2 <= s <= 252 every
// product is a normal bf16 number, whose bits are the unscaled entry's bits
// plus (s-127) << 7 (the exponent field): four integer multiply-adds, each
// adding to both 16-bit halves of a packed pair (no half carries or borrows
// in that range). Other scales take the rounding path through fp32.
__device__ __forceinline__ Bf16Tab e2m1_table(uint32_t s)
{
    uint32_t p0, p1, p2, p3;
    if (s - 2u <= 250u) {
        const uint32_t d = (uint32_t)(((int)s - 127) * 128);
        p0 = (0x3F00u + d) << 16;  // entries 0 (stays 0) and 0.5
        p1 = 0x3FC03F80u + d * 0x10001u;
        p2 = 0x40404000u + d * 0x10001u;
        p3 = 0x40C04080u + d * 0x10001u;
    } else {
        const float f = e8m0_to_float(s);
        p0 = bf16x2_bits(0.f, 0.5f * f);
        p1 = bf16x2_bits(f, 1.5f * f);
        p2 = bf16x2_bits(2.f * f, 3.f * f);
        p3 = bf16x2_bits(4.f * f, 6.f * f);
    }
    return {prmt(p0, p1, 0x6420u), prmt(p2, p3, 0x6420u), prmt(p0, p1, 0x7531u), prmt(p2, p3, 0x7531u)};
}

// Eight E2M1 codes (element j in bits 4j .. 4j+3; bit 3 of a code is its
// sign) -> eight bf16 values, element 2i in the low half of word i. The code
// nibbles select table bytes directly; the signs come from prmt's
// sign-replicate mode (selector bit 3 set), reading the code bytes as they
// are (odd elements) and shifted left by 4 (even elements).
__device__ __forceinline__ uint4 e2m1x8_to_bf16x8(uint32_t w, const Bf16Tab &t)
{
    const uint32_t w4 = w << 4;
    const uint32_t c0 = w & 0x77777777u, c1 = c0 >> 16;  // prmt reads the low 16 selector bits
    const uint32_t l0 = prmt(t.lo0, t.lo1, c0), l1 = prmt(t.lo0, t.lo1, c1);
    const uint32_t h0 = prmt(t.hi0, t.hi1, c0) | (prmt(w4, w, 0xD9C8u) & 0x80808080u);
    const uint32_t h1 = prmt(t.hi0, t.hi1, c1) | (prmt(w4, w, 0xFBEAu) & 0x80808080u);
    return make_uint4(prmt(l0, h0, 0x5140u), prmt(l0, h0, 0x7362u), prmt(l1, h1, 0x5140u), prmt(l1, h1, 0x7362u));
}

// Lane 0 waits on an mbarrier; the warp follows its verdict. On a timeout or
// an abort raised elsewhere the status word gets MXMOE_ERR_TIMEOUT.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag, int *status)
{
    int okv = 1;
    if ((threadIdx.x & 31) == 0 && (*abort_flag || !mbar_wait_bounded(bar, parity, kPWaitNs))) {
        set_status(status, MXMOE_ERR_TIMEOUT);
        *abort_flag = 1;
        okv = 0;
    }
    return __shfl_sync(0xFFFFFFFFu, okv, 0) != 0;
}

// Warp roles (28 warps).
constexpr int kPWarpB = 0;      // activation producer
constexpr int kPWarpMma = 1;    // MMA warps 1, 2 (tile / accumulator 0, 1)
constexpr int kPWarpW = 3;      // packed weight producer
constexpr int kPDeqWarp0 = 4;   // dequantising warps 4 .. 19
constexpr int kPEpiWarp0 = 20;  // epilogue warps 20 .. 27 (accumulator (w - 20) / 4, lane quarter w % 4)
constexpr int kPDeqWarps = kPEpiWarp0 - kPDeqWarp0;
static_assert(kPThreads == 32 * (kPEpiWarp0 + 8), "warp roles");

__device__ __forceinline__ float silu_fast(float g)  // g * sigmoid(g), ex2 / rcp approximations
{
    return __fdividef(g, 1.f + __expf(-g));
}

// Ring position: slot and phase parity of the n-th use of an S-slot ring.
template <int S>
struct Ring {
    int slot = 0;
    uint32_t phase = 0;
    __device__ __forceinline__ void next()
    {
        if (++slot == S) {
            slot = 0;
            phase ^= 1u;
        }
    }
};

template <bool GATE_UP>
__global__ void __launch_bounds__(kPThreads, 1)
    ffn_bf16_kernel(const __grid_constant__ CUtensorMap tmW, const PrefillParams p)
{
    constexpr int NB = GATE_UP ? 1 : 2;  // activation steps per K step: x, or h's hi then lo
    if (__ldg(p.pass_start + p.E) == 0) {  // no expert for this kernel (the E2M1-term kernel took them all)
        grid_dep_wait();                    // a chained CTA ends after the preceding kernel
        grid_dep_launch();
        return;
    }
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sB = smem, *sA = smem + kPOffA, *sW = smem + kPOffW, *sSf = smem + kPOffSf;
    uint64_t *full_b = reinterpret_cast<uint64_t *>(smem + kPOffBar);
    uint64_t *empty_b = full_b + kPBStages;
    uint64_t *full_w = empty_b + kPBStages;
    uint64_t *empty_w = full_w + kPWStages;
    uint64_t *aready = empty_w + kPWStages;
    uint64_t *aempty = aready + kPAStages;
    uint64_t *accfull = aempty + kPAStages;  // [2]: one accumulator per MMA warp
    uint64_t *accempty = accfull + 2;        // [2]
    uint64_t *mma_done = accempty + 2;       // [2]
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + kPOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int E = p.E, pairs = p.pairs;
    if (tid == 32) {
        for (int s = 0; s < kPBStages; ++s) {
            mbar_init(&full_b[s], 1);
            mbar_init(&empty_b[s], 2);
        }
        for (int s = 0; s < kPWStages; ++s) {
            mbar_init(&full_w[s], 1);
            mbar_init(&empty_w[s], kPDeqWarps);
        }
        for (int s = 0; s < kPAStages; ++s) {
            mbar_init(&aready[s], kPDeqWarps);
            mbar_init(&aempty[s], 2);
        }
        for (int j = 0; j < 2; ++j) {
            mbar_init(&accfull[j], 1);
            mbar_init(&accempty[j], 4);
            mbar_init(&mma_done[j], 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kPWarpMma)
        tc::alloc(tslot, 512);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *tslot;
    const int64_t total = (int64_t)__ldg(p.pass_start + E) * pairs;
    const int64_t G = gridDim.x;
    const int n_items = (int)(total > blockIdx.x ? (total - blockIdx.x + G - 1) / G : 0);
#define ITEM(i) decode_item(blockIdx.x + (int64_t)(i) * G, p.pass_start, p.offsets, E, pairs)
    const int nks = p.K / kPK;  // K steps (even: K is a multiple of 128)
    // Chained launch: the weight producer fills its ring before waiting for
    // the preceding kernel (weights, offsets and the pass table are older than
    // it); every other role waits here. The next kernel is let start only as
    // this one's CTAs exit (an earlier trigger measured slower).
    if (!((warp == kPWarpB || warp == kPWarpW) && lane == 0))
        grid_dep_wait();

    if (warp == kPWarpB || warp == kPWarpW) {
        // ---------------------------------------------------------- producers
        // Warp 0: the activation steps (x rows of the pass; for down h's hi
        // rows then lo rows), one bulk copy of a tiled 32 KB block each, kept
        // in L2 for the other boxes of the pass.
        // Warp 3: packed weights of two K steps (64 bytes of each of the box's
        // 256 rows) with their scale images.
        if (lane == 0) {
            const bool is_b = warp == kPWarpB;
            const int S = is_b ? kPBStages : kPWStages;
            uint64_t *full = is_b ? full_b : full_w;
            uint64_t *empty = is_b ? empty_b : empty_w;
            const uint64_t pol = is_b ? policy_evict_last() : policy_evict_normal();
            int s = 0;
            uint32_t ph = 0;
            int64_t issued = 0;
            bool ok = true;
            // packed weights and scale images of K steps ks, ks + 1 of a box into slot sl
            auto load_w = [&](int sl, int64_t box, int ks) {
                const int64_t chunk = box * p.nchunk + (ks >> 2);  // 256-K chunk of the box
                mbar_arrive_expect_tx(&full[sl], (uint32_t)(kPWBytes + kPSfBytes));
                tc::tma_load_2d(sW + (size_t)sl * kPWBytes, &tmW, 64 * ((ks & 3) >> 1), (int)(chunk * 256), &full[sl],
                                pol);
                bulk_g2s_hint(sSf + (size_t)sl * kPSfBytes, p.sf + chunk * 2048 + ((ks & 3) >> 1) * kPSfBytes,
                              kPSfBytes, &full[sl], pol);
            };
            int64_t pre = 0;  // weight loads issued before the wait (slots 0 .. pre-1, first use)
            if (!is_b)
                for (int i = 0; i < n_items && pre < S; ++i) {
                    const PItem it = ITEM(i);
                    for (int ks = 0; ks < nks && pre < S; ks += 2, ++pre)
                        load_w((int)pre, (int64_t)it.e * pairs + it.box, ks);
                }
            grid_dep_wait();
            for (int i = 0; i < n_items && ok; ++i) {
                const PItem it = ITEM(i);
                const int64_t box = (int64_t)it.e * pairs + it.box;
                for (int ks = 0; ks < nks && ok; ks += is_b ? 1 : 2) {
                    for (int b = 0; b < (is_b ? NB : 1); ++b) {
                        if (issued >= pre) {
                            if (*abort_flag || !mbar_wait_bounded(&empty[s], ph ^ 1u, kPWaitNs)) {
                                ok = false;
                                break;
                            }
                            if (is_b) {
                                mbar_arrive_expect_tx(&full[s], (uint32_t)kPBBytes);
                                bulk_g2s_hint(sB + (size_t)s * kPBBytes,
                                              p.act + ((it.pass * nks + ks) * NB + b) * (int64_t)kPBBytes, kPBBytes,
                                              &full[s], pol);
                            } else {
                                load_w(s, box, ks);
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
                if (!mbar_wait_bounded(&full[f % S], (uint32_t)((f / S) & 1), kPWaitNs)) {
                    set_status(p.status, MXMOE_ERR_TIMEOUT);
                    break;
                }
        }
    } else if (warp == kPWarpMma || warp == kPWarpMma + 1) {
        // ---------------------------------------------------------------- MMA
        // Warp 1 + j multiplies weight tile j of every K step into accumulator
        // j (tensor memory columns 256j ..): D[row][n] += A_j[row][k] * B[n][k],
        // B the step's activation rows (down: hi, then lo, into the same D).
        if (lane == 0) {
            const int j = warp - kPWarpMma;
            const uint32_t d_tmem = tmem + (uint32_t)j * 256;
            Ring<kPBStages> rb;
            Ring<kPAStages> ra;
            bool ok = true, any = false;
            for (int i = 0; i < n_items && ok; ++i) {
                const PItem it = ITEM(i);
                if (*abort_flag || !mbar_wait_bounded(&accempty[j], (uint32_t)(i & 1) ^ 1u, kPWaitNs)) {
                    ok = false;
                    break;
                }
                tc::fence_after();
                const uint32_t idesc = tc::idesc_bf16((it.nt + 15) & ~15);  // N: the pass's tokens, rounded up to 16
                for (int ks = 0; ks < nks && ok; ++ks) {
                    if (*abort_flag || !mbar_wait_bounded(&aready[ra.slot], ra.phase, kPWaitNs)) {
                        ok = false;
                        break;
                    }
                    const uint32_t a_base = smem_u32(sA + (size_t)(2 * ra.slot + j) * kPABytes);
                    for (int b = 0; b < NB; ++b) {
                        if (*abort_flag || !mbar_wait_bounded(&full_b[rb.slot], rb.phase, kPWaitNs)) {
                            ok = false;
                            break;
                        }
                        tc::fence_after();
                        const uint32_t b_base = smem_u32(sB + (size_t)rb.slot * kPBBytes);
#pragma unroll
                        for (int k4 = 0; k4 < 4; ++k4)  // 16 values of K per MMA
                            tc::mma_bf16(d_tmem, tc::smem_desc(a_base + 32 * k4, 16, 1024, 2),
                                     tc::smem_desc(b_base + 32 * k4, 16, 1024, 2), idesc,
                                     (ks > 0 || b > 0 || k4 > 0) ? 1u : 0u);
                        tc::commit(&empty_b[rb.slot]);
                        any = true;
                        rb.next();
                    }
                    if (ok)
                        tc::commit(&aempty[ra.slot]);
                    ra.next();
                }
                if (ok)
                    tc::commit(&accfull[j]);
            }
            if (!ok) {
                set_status(p.status, MXMOE_ERR_TIMEOUT);
                *abort_flag = 1;
            }
            if (any) {
                tc::commit(&mma_done[j]);
                if (!mbar_wait_bounded(&mma_done[j], 0, kPWaitNs))
                    set_status(p.status, MXMOE_ERR_TIMEOUT);
            }
        }
    } else if (warp >= kPDeqWarp0 && warp < kPEpiWarp0) {
        // ------------------------------------------------------ dequantising
        // Thread (k, j, m) writes half k of row m of weight tile j: 32 bf16
        // values (exact: an E2M1 value times a power of two) from the packed
        // step and the E8M0 scale of its 32-value block, by table lookups (no
        // conversion instructions per value), in the 128-byte swizzle (16-byte
        // chunk c of row m at chunk c ^ (m % 8); half k is chunks 4k .. 4k+3).
        //  gate/up: tile j holds gate rows 64j .. 64j+63 of the box (its rows
        //           0..127) and the matching up rows (box rows 128..255); row
        //           32q + w is gate row 16q + w of the 64 for w < 16, else the
        //           up row of the same h column;
        //  down:    tile j is box rows 128j .. 128j+127.
        const int d = tid - 32 * kPDeqWarp0;
        const int k = d >> 8, j = (d >> 7) & 1, m = d & 127;
        const int q = m >> 5, w = m & 31;
        const int R = GATE_UP ? (w < 16 ? 0 : 128) + 64 * j + 16 * q + (w & 15) : 128 * j + m;  // box row
        const int img = R >> 7, rr = R & 127;
        const int sf_byte = img * 512 + (rr & 31) * 16 + (rr >> 5) * 4;
        Ring<kPWStages> rw;
        Ring<kPAStages> ra;
        bool aborted = false;
        for (int i = 0; i < n_items; ++i) {
            for (int ks = 0; ks < nks; ++ks) {
                if (!aborted && !(ks & 1))  // a packed slot holds steps ks, ks + 1
                    aborted = !warp_wait(&full_w[rw.slot], rw.phase, abort_flag, p.status);
                uint4 c = make_uint4(0, 0, 0, 0);
                uint32_t e = 0;
                if (!aborted) {
                    c = *reinterpret_cast<const uint4 *>(sW + (size_t)rw.slot * kPWBytes + R * 64 + 32 * (ks & 1) +
                                                         16 * k);
                    // k32 block 2(ks%4) + k of the chunk: byte 2(ks%2) + k of the row's scale word in the
                    // image of this K half
                    e = sSf[(size_t)rw.slot * kPSfBytes + sf_byte + 2 * (ks & 1) + k];
                }
                if (ks & 1) {
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&empty_w[rw.slot]);
                    rw.next();
                }
                if (!aborted)
                    aborted = !warp_wait(&aempty[ra.slot], ra.phase ^ 1u, abort_flag, p.status);
                if (!aborted) {
                    const Bf16Tab t = e2m1_table(e);
                    uint8_t *arow = sA + (size_t)(2 * ra.slot + j) * kPABytes + m * 128;
                    const uint32_t words[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {  // 8 values per 16-byte chunk
                        const int ch = 4 * k + q4;
                        *reinterpret_cast<uint4 *>(arow + ((ch ^ (m & 7)) << 4)) = e2m1x8_to_bf16x8(words[q4], t);
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                }
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&aready[ra.slot]);
                ra.next();
            }
        }
    } else if (warp >= kPEpiWarp0) {
        // ----------------------------------------------------------- epilogue
        // Warps 12..15 drain accumulator 0, warps 16..19 accumulator 1; warp
        // quarter q reads lanes 32q .. 32q+31, 32 columns (tokens) at a time.
        const int j = (warp - kPEpiWarp0) >> 2, q = warp & 3;
        const uint32_t acc = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(256 * j);
        bool aborted = false;
        for (int i = 0; i < n_items; ++i) {
            const PItem it = ITEM(i);
            const int nt = it.nt;
            const int64_t r0 = it.r0;
            if (!aborted)
                aborted = !warp_wait(&accfull[j], (uint32_t)(i & 1), abort_flag, p.status);
            tc::fence_after();
            if (GATE_UP) {
                // lane w < 16 holds the gate rows of h column 128 box + 64j + 16q + w, lane w + 16 the up rows.
                // Each round the two swap half their tokens, so that lane w finishes token t and lane w + 16
                // token t + 16 of the 32: h = silu(g) u as bf16 hi (h rounded to 8 significant bits) and lo
                // (the exact remainder h - hi cut to 8 bits): hi + lo within 2^-15 of h, no conversions.
                // h column 128 box + 64j + 16q + w is value 16q + w of down K step 2 box + j: chunk 2q + w / 8 of
                // its row in the tiled hi block of (pass, K step), the lo block 32 KB after it.
                const bool upper = lane >= 16;
                const int w = lane & 15, c = 2 * q + (w >> 3);
                uint8_t *hb = p.h_tiled + ((it.pass * (p.I / kPK) + 2 * it.box + j) * 2) * (int64_t)kPBBytes + (w & 7) * 2;
                for (int n0 = 0; n0 < nt && !aborted; n0 += 32) {
                    float v[32];
                    tc::ld_32x32b_x32(acc + (uint32_t)n0, v);
#pragma unroll
                    for (int t = 0; t < 16; ++t) {
                        const float send = upper ? v[t] : v[t + 16];
                        const float recv = __shfl_xor_sync(0xFFFFFFFFu, send, 16);
                        const float g = upper ? recv : v[t];
                        const float u = upper ? v[t + 16] : recv;
                        const float h = silu_fast(g) * u;
                        const uint32_t hi = (__float_as_uint(h) + 0x8000u) & 0xFFFF0000u;
                        const uint32_t lo = __float_as_uint(h - __uint_as_float(hi));
                        const int m = n0 + t + (upper ? 16 : 0);  // row of the pass
                        if (m < nt) {
                            uint8_t *o = hb + m * 128 + ((c ^ (m & 7)) << 4);
                            *reinterpret_cast<uint16_t *>(o) = (uint16_t)(hi >> 16);
                            *reinterpret_cast<uint16_t *>(o + kPBBytes) = (uint16_t)(lo >> 16);
                        }
                    }
                }
            } else {
                // lane: y column 256 box + 128j + 32q + lane; accumulator column n: token n of the pass
                const int col = 256 * it.box + 128 * j + 32 * q + lane;
                float *dst = p.y + r0 * p.H + col;
                const bool col_ok = col < p.H;
                for (int n0 = 0; n0 < nt && !aborted; n0 += 32) {
                    float v[32];
                    tc::ld_32x32b_x32(acc + (uint32_t)n0, v);
#pragma unroll
                    for (int t = 0; t < 32; ++t)
                        if (col_ok && n0 + t < nt)
                            dst[(int64_t)(n0 + t) * p.H] = v[t];
                }
            }
            tc::fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&accempty[j]);
        }
    }
    tc::fence_before();
    __syncthreads();
    if (warp == kPWarpMma) {
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

template <bool GATE_UP>
int launch_bf16_stage(const CUtensorMap &tmW, const PrefillParams &p, cudaStream_t st)
{
    static thread_local int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        if (cudaFuncSetAttribute(ffn_bf16_kernel<GATE_UP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kPSmem) != cudaSuccess)
            return fail(MXMOE_ERR_CUDA, "ffn_bf16_kernel: cannot reserve %zu bytes of shared memory", kPSmem);
        configured_dev = dev;
    }
    return launch_kernel(GATE_UP ? "ffn_bf16_kernel<gate_up>" : "ffn_bf16_kernel<down>", ffn_bf16_kernel<GATE_UP>,
                         num_sms(), kPThreads, kPSmem, st, tmW, p);
}

}  // namespace

// A 2-D tensor map (rows of row_bytes bytes, `inner` elements of `type` each),
// for the other prefill kernel file.
int encode2d_any(CUtensorMap *m, CUtensorMapDataType type, const void *base, uint64_t inner, uint64_t outer,
                 uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle,
                 const char *what)
{
    return encode2d(m, type, base, inner, outer, row_bytes, box_inner, box_outer, swizzle, what);
}

// Upper bound on the 256-token passes of `rows` grouped rows over E experts
// when only experts with at least min_rows rows count: sum of ceil(n_e / 256)
// <= rows / 256 + (number of such experts). Sizes the tiled activations.
int64_t bf16_max_passes(int64_t rows, int E, int min_rows)
{
    const int64_t experts = min_rows > 0 ? std::min<int64_t>(E, rows / min_rows) : E;
    return (rows + kPTok - 1) / kPTok + experts;
}

// Before the gate/up stage: the passes before each expert with at least
// min_rows rows (pass_start, E + 1 ints), then those experts' x rows tiled per
// (pass, K step) into x_tiled (bf16_max_passes(rows, E, min_rows) * 256 * H *
// 2 bytes), through slot_row (rows ints: the grouped row of each (token,
// slot)); clears the status word when status is given. E <= 1024 and
// k <= 32 (every accepted shape).
// Passes of up to `tok` rows before each expert with at least min_rows rows
// (pass_start, E + 1 ints; E <= 1024); clears the status word when given.
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

int run_bf16_prep(const void *x, const int32_t *offsets, const int32_t *src_row, int k, int rows, int E, int H,
                  int min_rows, int32_t *pass_start, int32_t *slot_row, uint8_t *x_tiled, int *status,
                  cudaStream_t st)
{
    if (int rc = run_pass_prefix(offsets, E, min_rows, kPTok, pass_start, status, st))
        return rc;
    if (int rc = run_slot_rows(src_row, rows, slot_row, st))
        return rc;
    const int T = rows / k;
    const int blocks = (int)std::min<int64_t>(((int64_t)T + 7) / 8, (int64_t)num_sms() * 8);
    return launch_kernel("x_tile_kernel", x_tile_kernel, blocks < 1 ? 1 : blocks, 256, 0, st,
                         static_cast<const uint16_t *>(x), slot_row, offsets, pass_start, E, min_rows, k, T, H, x_tiled);
}

// One FFN stage on bf16 tensor cores over the grouped rows.
//  gate/up: act_tiled = x tiled by run_bf16_prep; w, sf = the gate/up code
//           boxes and scale images of the prepacked blob; writes h_tiled
//           (bf16_max_passes(rows, E) * 256 * I * 4 bytes: h = hi + lo).
//  down:    act_tiled = h_tiled; w, sf = the down part of the blob; writes y
//           (fp32 [rows][H]).
// pass_start comes from run_bf16_prep. Needs H % 128 == 0 and I % 128 == 0
// (every accepted shape).
int run_bf16_stage(bool gate_up, const uint8_t *act_tiled, const int32_t *offsets, const int32_t *pass_start,
                   const uint8_t *w, const uint8_t *sf, int rows, int E, int H, int I, uint8_t *h_tiled, float *y,
                   int *status, cudaStream_t st)
{
    const int K = gate_up ? H : I;
    const int nchunk = (K + 255) / 256;
    const int pairs = gate_up ? I / 128 : (H + 255) / 256;
    const int64_t blob_rows = (int64_t)E * pairs * nchunk * 256;
    CUtensorMap tmW;
    if (int rc = encode2d(&tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, w, 128, (uint64_t)blob_rows, 128, 64, 256,
                          CU_TENSOR_MAP_SWIZZLE_NONE, "bf16 stage weights"))
        return rc;
    PrefillParams p{};
    p.pairs = pairs;
    p.K = K;
    p.nchunk = nchunk;
    p.H = H;
    p.I = I;
    p.E = E;
    p.rows = rows;
    p.offsets = offsets;
    p.pass_start = pass_start;
    p.act = act_tiled;
    p.sf = sf;
    p.h_tiled = h_tiled;
    p.y = y;
    p.status = status;
    return gate_up ? launch_bf16_stage<true>(tmW, p, st) : launch_bf16_stage<false>(tmW, p, st);
}

}  // namespace mxmoe
