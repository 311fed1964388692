// ffn.cu -- grouped SwiGLU expert FFN over MXFP4 weights on tcgen05 block-scaled
// tensor cores, the weighted combine, and their entry points.
//
// Pages: "MiMo-V2.5-Pro-FP4-DFlash" model card, section 2 "FP4 Quantization"
// (the MoE experts, which hold the vast majority of parameters, are MXFP4 with
// block size 32) and introduction (lower bit width per parameter translates
// directly into faster decoding: the layer is bound by streaming expert
// weights); nxbn.cn MiMo-V2.5-Pro-FP4-DFlash article, architecture section
// (384 experts, 8 per token, hidden 6144). The expert is read as a SwiGLU FFN
// (h = silu(W_gate x) * (W_up x), y = W_down h) with no biases.
//
// Design (one B200, sm_100a):
//  * The weights stay MXFP4 all the way into the tensor core:
//    tcgen05.mma.kind::mxf4.block_scale multiplies packed E2M1 weight codes by
//    packed E2M1 activation codes, applies both operands' UE8M0 scales per 32
//    elements of K in hardware and accumulates in fp32 in tensor memory. No
//    instruction touches a weight element.
//  * The weights are the N operand, 256 rows per MMA, so that each MMA
//    covers 8 KB of weight codes (256 rows x 64 values of K): the fewest MMAs
//    per weight byte, and the weight stream, not the tensor pipe (about a
//    third busy), sets the pace.
//  * Activations become kT = 8 E2M1 terms per value: the balanced base-8
//    digits (each in -4..4, all exact E2M1 values) of the value on the grid
//    2^(E-22), E the exponent of its 32-value block's largest magnitude; term
//    t carries scale 2^(E-1-3t). That is exact for every bf16 x within 2^-15
//    of its block maximum and keeps h to within 2^-23 of its block maximum.
//    The terms of a token are consecutive MMA rows (row = token * kT + term;
//    M = 128 rows = 16 tokens); the epilogue adds them.
//  * Weight boxes (256 rows x 256 K, 32 KB, contiguous in the prepacked blob)
//    and their scale images (2 KB) stream through a 5-deep ring; activation
//    terms (one 4-D TMA box per chunk) and their scale images (written by the
//    producing kernel directly in tensor-memory image order, one per token
//    pass and 128 columns) through a 3-deep ring. tcgen05.cp moves the scale
//    images into tensor memory.
//  * Warp roles per CTA: a producer warp, an MMA warp and four epilogue warps.
//    The epilogue sums a token's terms with a 3-round butterfly that leaves
//    each lane 8 finished columns of every 64, then releases the accumulator.
//  * Stage 1 (gate/up): a 256-row tile is 128 gate rows and the matching 128
//    up rows; SwiGLU and the term encoding of h (with its scale images) are
//    fused into the epilogue. Stage 2 (down): a tile is 256 output rows.
//  * Work items (expert, tile, token pass of up to NT tokens) go round-robin
//    over a persistent grid of one CTA per SM (CTA b takes items b, b + G,
//    ...), so that the passes of one weight tile run side by side and share
//    its boxes in L2.
//  * FP8 expert weights (E4M3 codes, one E8M0 scale per 32; the pages' FP8
//    baseline, model card section 2) run through the same kernel with
//    tcgen05.mma.kind::mxf8f6f4.block_scale: the E4M3 weights are the N
//    operand as they are stored (256 rows x 128 values of K per 32 KB box),
//    the activations the same E2M1 digit terms, unpacked to one byte per
//    value by the TMA (16U4_ALIGN16B), with the same UE8M0 scale images.
#include <float.h>
#include <limits.h>

#include <algorithm>
#include <mutex>

#include <cudaTypedefs.h>

#include "common.cuh"
#include "router_dev.cuh"
#include "tcgen05.cuh"

namespace mxmoe {
int64_t f8_max_passes(int64_t rows, int E, int min_rows);
int64_t f8_terms_bytes(int64_t passes, int K, int nterms);
int64_t f8_sf_bytes(int64_t passes, int K, int nterms);
int run_f8_prep(const void *x, const int32_t *offsets, const int32_t *src_row, int k, int rows, int E, int H,
                int min_rows, int32_t *pass_start, int32_t *slot_row, uint8_t *x_terms, uint8_t *x_sf, int *status,
                cudaStream_t st);
int run_f8_stage(bool gate_up, const uint8_t *terms, const uint8_t *terms_sf, const int32_t *offsets,
                 const int32_t *pass_start, const uint8_t *w, const uint8_t *sf, int E, int H, int I, uint8_t *h_terms,
                 uint8_t *h_sf, float *y, int *status, cudaStream_t st);
namespace {

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bounded waits: 2 s
constexpr int kT = 8;            // E2M1 terms per activation value
constexpr int kKC = 256;         // K per chunk (one weight box)
constexpr int kWBox = 32768;     // bytes of a weight box: 256 rows x 128 bytes
constexpr int kWSf = 2048;       // its scale images: (K half, row half) x 512 bytes
constexpr int kAStage = 16384;   // shared bytes the MMA reads for A: 128 rows x 128 bytes
constexpr int kSFImg = 512;      // scale image: 32 lanes x 16 bytes
constexpr int kThreads = 224;    // producer, MMA, 4 epilogue warps, scale-copy warp
constexpr int kMaxE = 1024;

struct FfnParams {
    int tiles;                  // 256-row tiles per expert: I/128 (gate/up) or H/256 (down)
    int K;                      // reduction length (H or I)
    int rows;                   // activation rows (T*k)
    const uint8_t *wsf;         // weight scale images [E*tiles][K/256][2048]
    const uint8_t *asf;         // activation scale images [pass][K/128][512]
    const int32_t *offsets;     // [E+1]
    const int32_t *pass_start;  // [E+1]: first token pass of each expert
    int E;
    uint8_t *h_terms;           // gate/up output: terms of h (term_offset layout)
    uint8_t *h_sf;              // gate/up output: their scale images
    int I;
    float *y_out;               // down output: [rows, H]
    int H;
    int hot_rows;               // experts with at least this many rows are left to the large-token kernel
    int *status;
    int wait_first;             // chained after a kernel that wrote the offsets: every thread waits first
};

__host__ __device__ __forceinline__ int64_t pad256(int64_t v) { return (v + 255) & ~int64_t(255); }

// Byte offset of the E2M1 code byte holding columns k, k+1 (k even) of term t
// of activation row r, in a term tensor laid out [K/256][rows][kT][128]: the
// terms of one 256-column chunk of a token pass are consecutive 128-byte rows.
__host__ __device__ __forceinline__ int64_t term_offset(int64_t rows, int t, int64_t r, int k)
{
    return (((int64_t)(k >> 8) * rows + r) * kT + t) * 128 + ((k & 255) >> 1);
}

// Byte offset, within the scale images of one token pass and 128-column half
// (512 bytes), of the scale of term t of pass row n for 32-block kb of the
// half: MMA row m = n * kT + t sits in tensor-memory lane m % 32, column m / 32.
__host__ __device__ __forceinline__ int image_byte(int n, int t, int kb)
{
    const int m = n * kT + t;
    return (m & 31) * 16 + (m >> 5) * 4 + kb;
}

// Upper bound on token passes: every pass holds at least one row, and there
// are at most ceil(rows / 8) + (non-empty experts) of them.
inline int64_t max_passes(int64_t rows)
{
    return std::min<int64_t>(rows, (rows + 7) / 8 + std::min<int64_t>(kMaxE, rows));
}

template <int NT>
struct Cfg {
    static constexpr int kM = NT * kT;  // MMA rows in use
    static constexpr int kATx = kM * 128;
    static constexpr int kStagesW = 5, kStagesA = 3;
    // shared memory: W stages | A stages | W scale images | A scale images | barriers | tslot, cursor
    static constexpr size_t kOffA = (size_t)kStagesW * kWBox;
    static constexpr size_t kOffSfw = kOffA + (size_t)kStagesA * kAStage;
    static constexpr size_t kOffSfa = kOffSfw + (size_t)kStagesW * kWSf;
    static constexpr size_t kOffBar = kOffSfa + (size_t)kStagesA * 2 * kSFImg;
    static constexpr int kBars = 2 * kStagesW + 2 * kStagesA + 3 + kStagesA + 1;
    // two barrier sets: the persistent layer kernel gives each FFN stage its own
    static constexpr size_t kOffMisc = (kOffBar + 2 * kBars * 8 + 15) & ~size_t(15);
    static constexpr size_t kOffItems = kOffMisc + 64;  // items before each expert [kMaxE + 1]
    static constexpr size_t kSmem = 1024 + kOffItems + (kMaxE + 1) * 4;
    // Tensor memory: the accumulator (128 lanes x 256 columns), then per weight
    // stage two 8-column scale groups (K halves; 256 rows = 8 columns) and per
    // activation stage two 4-column groups.
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kSfwCol0 = 256;
    static constexpr uint32_t kSfaCol0 = kSfwCol0 + 16 * kStagesW;
    static_assert(NT == 8 || NT == 16, "token pass");
    static_assert(kSfaCol0 + 8 * kStagesA <= kTmemCols, "tensor memory columns");
    static_assert(kSmem <= 232448, "shared memory");
};

// Instruction descriptor of kind::mxf4.block_scale: A and B E2M1, UE8M0
// scales, both K-major, M = 128, N = n, scale byte pair sf_id (0 or 2) of
// each operand's scale column.
__device__ __forceinline__ uint32_t idesc_mxf4(int n, uint32_t sf_id)
{
    return (sf_id << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | (1u << 23) | (8u << 24) |
           (sf_id << 29);
}

__device__ __forceinline__ void mma_mxf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate, uint32_t sfa_tmem, uint32_t sfb_tmem)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// Instruction descriptor of kind::mxf8f6f4.block_scale with A = E2M1 (the
// activation terms, one per byte), B = E4M3 (FP8 weights), UE8M0 scales, both
// K-major, M = 128, N = n, scale byte sf_id (0..3: the k32 block of a 4-block
// scale column) for both operands.
__device__ __forceinline__ uint32_t idesc_e2m1_x_e4m3(int n, uint32_t sf_id)
{
    return (sf_id << 4) | (5u << 7) | (0u << 10) | ((uint32_t)(n >> 3) << 17) | (1u << 23) | (8u << 24) |
           (sf_id << 29);
}

// D (+)= A * B^T over 32 values of K, one UE8M0 scale per 32 values for each
// operand (the scale bytes picked by the descriptor's sf_id).
__device__ __forceinline__ void mma_mxf8f6f4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate, uint32_t sfa_tmem, uint32_t sfb_tmem)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// Work items of one FFN stage: (expert, 256-row tile, token pass), expert-major,
// then tile, then pass. CTA b takes items b, b + G, b + 2G, ... (G CTAs), so
// the passes of one weight tile run on neighbouring CTAs at about the same
// time and all but the first read its boxes from L2. Every role decodes the
// same items.
struct Item {
    int e, tile, pass, r0, nt;
};

template <int NT>
__device__ __forceinline__ Item decode_item(int64_t idx, const int32_t *items, const int32_t *offsets, int E,
                                            int tiles)
{
    int lo = 0, hi = E;  // largest e with items[e] <= idx
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (items[mid] <= idx)
            lo = mid;
        else
            hi = mid;
    }
    const int base = offsets[lo], n_e = offsets[lo + 1] - base;
    const int npass = (n_e + NT - 1) / NT;
    const int local = (int)(idx - items[lo]);
    Item it;
    it.e = lo;
    it.tile = local / npass;
    it.pass = local % npass;
    it.r0 = base + it.pass * NT;
    it.nt = min(NT, n_e - it.pass * NT);
    return it;
}

__device__ __forceinline__ float pow2f(int s)  // 2^s for s in [-126, 127]
{
    return __uint_as_float((uint32_t)(s + 127) << 23);
}

// Exponent E of a 32-value activation block whose largest magnitude is m:
// floor(log2 m), raised to -104 for tiny or zero blocks so that every term's
// scale 2^(E - 1 - 3t) stays a normal UE8M0 value.
__device__ __forceinline__ int act_block_exp(float m)
{
    const uint32_t b = __float_as_uint(m);
    return max((int)(b >> 23) - 127, -104);
}

__device__ __forceinline__ uint32_t byte_perm(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// The kT balanced base-8 digits of 8 activation values v[0..7] of a block of
// exponent E, as E2M1 codes: v ~= sum_t d_t * 2^(E - 1 - 3t), d_t in {-4..4}
// (all exact E2M1 values), t = 0 most significant; word[t] holds value j's
// code of d_t in nibble j. The digits are exact for any v that is a multiple
// of 2^(E - 22) -- every bf16 value within 2^-15 of its block maximum -- and
// otherwise represent v rounded to that grid (within 2^-23 of the block
// maximum).
// iv = v * 2^(22 - E) rounded, |iv| <= 2^23. Adding 4 at each of the 7 low
// base-8 positions (u = iv + 4 * (8^0 + ... + 8^6)) turns the low digits, in
// [-4, 3], into plain base-8 digits d + 4 (no carries), and what is left
// above them (an arithmetic shift by 21) is the top digit, in [-4, 4]. Each
// value's seven low digits + 4 are spread to nibbles 0..6 of a word and its
// top digit + 4 (0..8) put in nibble 7; an 8 x 8 nibble transpose (two
// byte-permute stages, one of nibble masks) gathers digit t of the 8 values
// into one word, in the nibble order 0 2 4 6 1 3 5 7; a byte-permute lookup
// turns four digits into their codes at a time, bytes of even and odd values
// then interleaved to nibbles. A selector nibble of 8 (a top digit of 4)
// reads 0 (the sign of table byte 0) and takes code 6 from a second lookup.
__device__ __forceinline__ void act_words(const float (&v)[8], int E, uint32_t (&word)[kT])
{
    static_assert(kT == 8, "one word per digit of 8 values");
    const float s = pow2f(22 - E);
    uint32_t x[8];
#pragma unroll
    for (int p = 0; p < 8; ++p) {
        const int u = (int)rintf(v[p < 4 ? 2 * p : 2 * p - 7] * s) + 0x124924;
        uint32_t f = (uint32_t)u;
        f = (f & 0xFFFu) | ((f << 4) & 0x01FF0000u);        // digits 4..6 to bits 16..24
        f = (f & 0x003F003Fu) | ((f << 2) & 0x3F003F00u);   // digits 2, 3 and 6 to the odd bytes
        f = (f & 0x07070707u) | ((f << 1) & 0x70707070u);   // odd digits to the high nibbles
        x[p] = f | (((uint32_t)(u + 0x800000) << 7) & 0xF0000000u);
    }
#pragma unroll
    for (int p = 0; p < 4; ++p) {  // 4 x 4 blocks of nibbles
        const uint32_t a = x[p], b = x[p + 4];
        x[p] = byte_perm(a, b, 0x5410u);
        x[p + 4] = byte_perm(a, b, 0x7632u);
    }
#pragma unroll
    for (int p = 0; p < 8; p += (p & 1) ? 3 : 1) {  // 2 x 2 blocks: pairs (0,2) (1,3) (4,6) (5,7)
        const uint32_t a = x[p], b = x[p + 2];
        x[p] = byte_perm(a, b, 0x6240u);
        x[p + 2] = byte_perm(a, b, 0x7351u);
    }
#pragma unroll
    for (int p = 0; p < 8; p += 2) {  // single nibbles
        const uint32_t a = x[p], b = x[p + 1];
        x[p] = (a & 0x0F0F0F0Fu) | ((b << 4) & 0xF0F0F0F0u);
        x[p + 1] = ((a >> 4) & 0x0F0F0F0Fu) | (b & 0xF0F0F0F0u);
    }
    // codes of digit + 4 = 0..7 (d = -4..3): 0xE 0xD 0xC 0xA 0x0 0x2 0x4 0x5 (bit 3 the sign)
    constexpr uint32_t kLo = 0x0A0C0D0Eu, kHi = 0x05040200u;
#pragma unroll
    for (int m = 0; m < 7; ++m)  // x[m]: the digits of weight 8^m, term kT - 1 - m
        word[kT - 1 - m] = byte_perm(kLo, kHi, x[m]) | (byte_perm(kLo, kHi, x[m] >> 16) << 4);
    const uint32_t y = x[7];
    const uint32_t lo = byte_perm(kLo, kHi, y) | (byte_perm(0x80u, 0u, y) & 0x06060606u);
    const uint32_t hi = byte_perm(kLo, kHi, y >> 16) | (byte_perm(0x80u, 0u, y >> 16) & 0x06060606u);
    word[0] = lo | (hi << 4);
}

// Shared-memory view of one FFN stage: rings, scale images, barrier set
// `set` (0 or 1) and the per-expert item table.
template <int NT>
struct StageSmem {
    uint8_t *sW, *sA, *sSfw, *sSfa;
    uint64_t *fullW, *emptyW, *fullA, *emptyA, *accfull, *accempty, *mma_done, *sfready, *cp_done;
    uint32_t *tslot;
    volatile int *abort_flag;
    int32_t *s_items;
    __device__ __forceinline__ StageSmem(uint8_t *smem, int set)
    {
        using C = Cfg<NT>;
        sW = smem;
        sA = smem + C::kOffA;
        sSfw = smem + C::kOffSfw;
        sSfa = smem + C::kOffSfa;
        fullW = reinterpret_cast<uint64_t *>(smem + C::kOffBar) + set * C::kBars;
        emptyW = fullW + C::kStagesW;
        fullA = emptyW + C::kStagesW;
        emptyA = fullA + C::kStagesA;
        accfull = emptyA + C::kStagesA;
        accempty = accfull + 1;
        mma_done = accempty + 1;
        sfready = mma_done + 1;  // [kStagesA]: a chunk's scale images are in tensor memory
        cp_done = sfready + C::kStagesA;
        tslot = reinterpret_cast<uint32_t *>(smem + C::kOffMisc);
        abort_flag = reinterpret_cast<volatile int *>(tslot + 1);
        s_items = reinterpret_cast<int32_t *>(smem + C::kOffItems);
    }
};

// Items of every expert and their prefix (s_items), the stage's barriers,
// a cleared abort flag. Called by every thread of the block; ends with a
// block-wide barrier.
template <int NT>
__device__ __forceinline__ void stage_prepare(const FfnParams &p, const StageSmem<NT> &S)
{
    using C = Cfg<NT>;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int E = p.E, tiles = p.tiles;
    int32_t *s_items = S.s_items;
    for (int e = tid; e < E; e += blockDim.x) {  // items of expert e: tiles * ceil(n_e / NT), none if it is hot
        const int n_e = p.offsets[e + 1] - p.offsets[e];
        s_items[e] = n_e >= p.hot_rows ? 0 : tiles * ((n_e + NT - 1) / NT);
    }
    __syncthreads();
    if (warp == 0) {  // exclusive prefix, in place; s_items[E] = all items
        int carry = 0;
        for (int b = 0; b <= E; b += 32) {
            const int e = b + lane;
            const int c = e < E ? s_items[e] : 0;
            int incl = c;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
                if (lane >= off)
                    incl += o;
            }
            __syncwarp();
            if (e <= E)
                s_items[e] = carry + incl - c;
            carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
    }
    if (tid == 32) {
        for (int s = 0; s < C::kStagesW; ++s) {
            mbar_init(&S.fullW[s], 1);
            mbar_init(&S.emptyW[s], 1);
        }
        for (int s = 0; s < C::kStagesA; ++s) {
            mbar_init(&S.fullA[s], 1);
            mbar_init(&S.emptyA[s], 1);
        }
        mbar_init(S.accfull, 1);
        mbar_init(S.accempty, 4);
        mbar_init(S.mma_done, 1);
        for (int s = 0; s < C::kStagesA; ++s)
            mbar_init(&S.sfready[s], 1);
        mbar_init(S.cp_done, 1);
        *S.abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
}

// The chained launch's producer wait: the preceding kernel's results.
struct WaitChained {
    __device__ __forceinline__ bool operator()() const
    {
        grid_dep_wait();
        return true;
    }
};

// The roles of one FFN stage, warps 0..6 of the block (warp 0 producer, 1 MMA,
// 2..5 epilogue, 6 scale copies; any further warps return at once). The
// producer fills its weight ring first, then calls producer_wait() (false:
// give up) before it loads any activation; every other role must have waited
// for its inputs before it is called. No block-wide barrier inside; the
// caller ends the stage with tc::fence_before() and __syncthreads().
// GATE_UP = true: stage 1 (x terms in; h terms and their scale images out).
// GATE_UP = false: stage 2 (h terms in; float rows out).
// FP8 = true: E4M3 weights (128 values of K per box, kind::mxf8f6f4, the
// activation terms unpacked to a byte each by the TMA); else MXFP4 weights
// (256 values of K per box, kind::mxf4).
template <int NT, bool GATE_UP, bool FP8, class ProducerWait>
__device__ __forceinline__ void stage_roles(const CUtensorMap &tmW, const CUtensorMap &tmA, const FfnParams &p,
                                            const StageSmem<NT> &S, uint32_t tmem, ProducerWait producer_wait)
{
    using C = Cfg<NT>;
    uint8_t *sW = S.sW, *sA = S.sA, *sSfw = S.sSfw, *sSfa = S.sSfa;
    uint64_t *fullW = S.fullW, *emptyW = S.emptyW, *fullA = S.fullA, *emptyA = S.emptyA;
    uint64_t *accfull = S.accfull, *accempty = S.accempty, *mma_done = S.mma_done, *sfready = S.sfready;
    uint64_t *cp_done = S.cp_done;
    volatile int *abort_flag = S.abort_flag;
    const int32_t *s_items = S.s_items;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int E = p.E, tiles = p.tiles;
    const int64_t G = gridDim.x, total = s_items[E];
    const int n_items = (int)(total > blockIdx.x ? (total - blockIdx.x + G - 1) / G : 0);
#define ITEM(i) decode_item<NT>(blockIdx.x + (int64_t)(i) * G, s_items, p.offsets, E, tiles)
    // MXFP4: 256-value chunks (the last may hold one 128-column half);
    // FP8: 128-value chunks, each one half
    const int nchunk = FP8 ? p.K / 128 : (p.K + kKC - 1) / kKC;
    const int khalves = p.K / 128;
    constexpr int kWSfBox = FP8 ? 1024 : kWSf;  // a box's weight scale images

    if (warp == 0) {
        // ----------------------------------------------------------- producer
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_first();
            const uint64_t pol_a = policy_evict_last();
            int sw = 0, sa = 0;
            uint32_t phw = 0, pha = 0;
            int64_t issued_w = 0, issued_a = 0;
            bool ok = true;
            auto load_w = [&](int sl, int64_t box) {  // weight box and its scale images into slot sl
                mbar_arrive_expect_tx(&fullW[sl], (uint32_t)(kWBox + kWSfBox));
                tc::tma_load_2d(sW + (size_t)sl * kWBox, &tmW, 0, (int)(box * 256), &fullW[sl], pol_w);
                bulk_g2s_hint(sSfw + sl * kWSf, p.wsf + box * kWSfBox, kWSfBox, &fullW[sl], pol_w);
            };
            int64_t pre_w = 0;  // weight boxes issued before the wait (slots 0 .. pre_w-1, first use)
            for (int i = 0; i < n_items && pre_w < C::kStagesW; ++i) {
                const Item it = ITEM(i);
                const int64_t box0 = ((int64_t)it.e * tiles + it.tile) * nchunk;
                for (int c = 0; c < nchunk && pre_w < C::kStagesW; ++c, ++pre_w)
                    load_w((int)pre_w, box0 + c);
            }
            if (!producer_wait())
                ok = false;
            for (int i = 0; i < n_items && ok; ++i) {
                const Item it = ITEM(i);
                const int64_t box0 = ((int64_t)it.e * tiles + it.tile) * nchunk;
                const int64_t pass_id = (int64_t)p.pass_start[it.e] + it.pass;
                const int r0 = it.r0;
                for (int c = 0; c < nchunk; ++c) {
                    if (issued_w >= pre_w) {
                        if (*abort_flag || !mbar_wait_bounded(&emptyW[sw], phw ^ 1u, kWaitLimitNs)) {
                            ok = false;
                            break;
                        }
                        load_w(sw, box0 + c);
                    }
                    ++issued_w;
                    if (*abort_flag || !mbar_wait_bounded(&emptyA[sa], pha ^ 1u, kWaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    if (FP8) {
                        // K half c of the packed terms, unpacked to a byte per value (the transaction
                        // counts the packed bytes: 64 per row), and its one scale image
                        mbar_arrive_expect_tx(&fullA[sa], (uint32_t)(C::kM * 64 + kSFImg));
                        tc::tma_load_4d(sA + (size_t)sa * kAStage, &tmA, 128 * (c & 1), 0, r0, c >> 1, &fullA[sa],
                                        pol_a);
                        bulk_g2s_hint(sSfa + sa * 2 * kSFImg, p.asf + (pass_id * khalves + c) * kSFImg, kSFImg,
                                      &fullA[sa], pol_a);
                    } else {
                        const int nh = min(2, khalves - 2 * c);  // K halves in this chunk
                        mbar_arrive_expect_tx(&fullA[sa], (uint32_t)(C::kATx + nh * kSFImg));
                        tc::tma_load_4d(sA + (size_t)sa * kAStage, &tmA, 0, 0, r0, c, &fullA[sa], pol_a);
                        bulk_g2s_hint(sSfa + sa * 2 * kSFImg, p.asf + (pass_id * khalves + 2 * c) * kSFImg,
                                      (uint32_t)(nh * kSFImg), &fullA[sa], pol_a);
                    }
                    ++issued_a;
                    if (++sw == C::kStagesW) {
                        sw = 0;
                        phw ^= 1u;
                    }
                    if (++sa == C::kStagesA) {
                        sa = 0;
                        pha ^= 1u;
                    }
                }
            }
            if (!ok) {
                set_status(p.status, MXMOE_ERR_TIMEOUT);
                *abort_flag = 1;
            }
            // Drain: no copy of ours may still be landing when the CTA ends (the
            // weight loads issued before the wait included).
            issued_w = issued_w > pre_w ? issued_w : pre_w;
            for (int64_t f = issued_w > C::kStagesW ? issued_w - C::kStagesW : 0; f < issued_w; ++f)
                if (!mbar_wait_bounded(&fullW[f % C::kStagesW], (uint32_t)((f / C::kStagesW) & 1), kWaitLimitNs)) {
                    set_status(p.status, MXMOE_ERR_TIMEOUT);
                    break;
                }
            for (int64_t f = issued_a > C::kStagesA ? issued_a - C::kStagesA : 0; f < issued_a; ++f)
                if (!mbar_wait_bounded(&fullA[f % C::kStagesA], (uint32_t)((f / C::kStagesA) & 1), kWaitLimitNs)) {
                    set_status(p.status, MXMOE_ERR_TIMEOUT);
                    break;
                }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA
        if (lane == 0) {
            int sw = 0, sa = 0;
            uint32_t phw = 0, pha = 0;
            bool ok = true, any = false;
            for (int i = 0; i < n_items && ok; ++i) {
                if (*abort_flag || !mbar_wait_bounded(accempty, ((uint32_t)i & 1u) ^ 1u, kWaitLimitNs)) {
                    ok = false;
                    break;
                }
                tc::fence_after();
                for (int c = 0; c < nchunk; ++c) {
                    if (*abort_flag || !mbar_wait_bounded(&fullW[sw], phw, kWaitLimitNs) ||
                        !mbar_wait_bounded(&fullA[sa], pha, kWaitLimitNs) ||
                        !mbar_wait_bounded(&sfready[sa], pha, kWaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    tc::fence_after();
                    const uint32_t sfw_t = tmem + C::kSfwCol0 + 16 * sw;  // + 8 per K half, + 4 per row half
                    const uint32_t sfa_t = tmem + C::kSfaCol0 + 8 * sa;   // + 4 per K half
                    const uint32_t a_base = smem_u32(sA + (size_t)sa * kAStage);
                    const uint32_t w_base = smem_u32(sW + (size_t)sw * kWBox);
                    if (FP8) {
#pragma unroll
                        for (int k = 0; k < 4; ++k) {  // 32 values of K (32 bytes of both operands) per MMA
                            const uint32_t id = (uint32_t)k;
                            mma_mxf8f6f4(tmem, tc::smem_desc(a_base + k * 32, 16, 1024, 2),
                                         tc::smem_desc(w_base + k * 32, 16, 1024, 2), idesc_e2m1_x_e4m3(256, id),
                                         (c > 0 || k > 0) ? 1u : 0u, sfa_t | (id << 30), sfw_t | (id << 30));
                        }
                    } else {
                        const int nk = 2 * min(2, khalves - 2 * c);  // a half chunk takes two MMAs
                        for (int k = 0; k < nk; ++k) {  // 64 values of K per MMA
                            const uint32_t h = (uint32_t)(k >> 1), id = 2u * (uint32_t)(k & 1);
                            mma_mxf4(tmem, tc::smem_desc(a_base + k * 32, 16, 1024, 2),
                                     tc::smem_desc(w_base + k * 32, 16, 1024, 2), idesc_mxf4(256, id),
                                     (c > 0 || k > 0) ? 1u : 0u, (sfa_t + 4 * h) | (id << 30),
                                     (sfw_t + 8 * h) | (id << 30));
                        }
                    }
                    tc::commit(&emptyW[sw]);  // frees both stages once these MMAs are done
                    tc::commit(&emptyA[sa]);
                    any = true;
                    if (++sw == C::kStagesW) {
                        sw = 0;
                        phw ^= 1u;
                    }
                    if (++sa == C::kStagesA) {
                        sa = 0;
                        pha ^= 1u;
                    }
                }
                if (ok)
                    tc::commit(accfull);
            }
            if (!ok) {
                set_status(p.status, MXMOE_ERR_TIMEOUT);
                *abort_flag = 1;
            }
            // Every MMA of ours completes before tensor memory is released.
            if (any) {
                tc::commit(mma_done);
                if (!mbar_wait_bounded(mma_done, 0, kWaitLimitNs))
                    set_status(p.status, MXMOE_ERR_TIMEOUT);
            }
        }
    } else if (warp == 6) {
        // ---------------------------------------------------- scale images
        // Moves each chunk's scale images from shared into tensor memory and
        // signals sfready, so the MMA warp issues nothing but MMAs. A slot's
        // columns are rewritten only after its full barrier fired again, i.e.
        // after the MMAs that read them completed.
        if (lane == 0) {
            int sw = 0, sa = 0;
            uint32_t phw = 0, pha = 0;
            bool ok = true, any = false;
            const int64_t total = (int64_t)n_items * nchunk;
            for (int64_t j = 0; j < total; ++j) {
                const int c = (int)(j % nchunk);
                if (*abort_flag || !mbar_wait_bounded(&fullW[sw], phw, kWaitLimitNs) ||
                    !mbar_wait_bounded(&fullA[sa], pha, kWaitLimitNs)) {
                    ok = false;
                    break;
                }
                tc::fence_after();
                const uint32_t sfw_t = tmem + C::kSfwCol0 + 16 * sw;
                const uint32_t sfa_t = tmem + C::kSfaCol0 + 8 * sa;
                const uint32_t sfw_s = smem_u32(sSfw + sw * kWSf);
                const uint32_t sfa_s = smem_u32(sSfa + sa * 2 * kSFImg);
#pragma unroll
                for (int img = 0; img < (FP8 ? 2 : 4); ++img)
                    tc::cp_32x128b_warpx4(sfw_t + 4 * img, tc::smem_desc(sfw_s + img * kSFImg, 16, 128, 0));
                for (int h = 0; h < (FP8 ? 1 : min(2, khalves - 2 * c)); ++h)
                    tc::cp_32x128b_warpx4(sfa_t + 4 * h, tc::smem_desc(sfa_s + h * kSFImg, 16, 128, 0));
                tc::commit(&sfready[sa]);
                any = true;
                if (++sw == C::kStagesW) {
                    sw = 0;
                    phw ^= 1u;
                }
                if (++sa == C::kStagesA) {
                    sa = 0;
                    pha ^= 1u;
                }
            }
            if (!ok) {
                set_status(p.status, MXMOE_ERR_TIMEOUT);
                *abort_flag = 1;
            }
            // Every copy of ours completes before tensor memory is released.
            if (any) {
                tc::commit(cp_done);
                if (!mbar_wait_bounded(cp_done, 0, kWaitLimitNs))
                    set_status(p.status, MXMOE_ERR_TIMEOUT);
            }
        }
    } else if (warp <= 5) {
        // ----------------------------------------------------------- epilogue
        // Warp quarter q reads accumulator lanes 32q .. 32q+31: tokens 4q .. 4q+3
        // of the pass, term tl = lane % 8 in each. A warp that gives up on a wait
        // stops reading tensor memory and writing outputs.
        const int q = warp & 3;
        const int tl = lane & 7;
        const int n = 4 * q + (lane >> 3);  // token within the pass
        const bool has_rows = 4 * q < NT;   // this quarter holds MMA rows in use
        bool aborted = false;
        for (int i = 0; i < n_items; ++i) {
            const Item it = ITEM(i);
            if (!aborted) {  // lane 0 waits; the warp follows its verdict
                int ok = 1;
                if (lane == 0 && (*abort_flag || !mbar_wait_bounded(accfull, (uint32_t)i & 1u, kWaitLimitNs))) {
                    set_status(p.status, MXMOE_ERR_TIMEOUT);
                    *abort_flag = 1;
                    ok = 0;
                }
                aborted = !__shfl_sync(0xFFFFFFFFu, ok, 0);
            }
            tc::fence_after();
            // v[b][j]: column 64b + 8tl + j of the token's term sum
            float v[4][8];
#pragma unroll
            for (int b = 0; b < 4; ++b)
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    v[b][j] = 0.f;
            if (!aborted && has_rows) {
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    float x[64];
                    tc::ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(64 * b), x);
                    tc::ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(64 * b + 32), x + 32);
                    // reduce-scatter over the 8 term lanes of each token
#pragma unroll
                    for (int round = 0; round < 3; ++round) {
                        const int half = 32 >> round, mask = 4 >> round;
                        const bool up = (tl & mask) != 0;
#pragma unroll
                        for (int j = 0; j < half; ++j) {
                            const float send = up ? x[j] : x[j + half];
                            const float keep = up ? x[j + half] : x[j];
                            x[j] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, mask);
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        v[b][j] = x[j];
                }
            }
            tc::fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(accempty);
            const int ntile = it.nt;
            const bool valid = !aborted && has_rows && n < ntile;
            if (GATE_UP) {
                // h columns 64b + 8tl + j of the tile (b = 0, 1): gate = v[b], up = v[b + 2]
                float hv[2][8];
#pragma unroll
                for (int b = 0; b < 2; ++b)
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float g = v[b][j];
                        hv[b][j] = valid ? g / (1.f + expf(-g)) * v[b + 2][j] : 0.f;
                    }
                const int r = it.r0 + n;
                const int64_t img = ((int64_t)p.pass_start[it.e] + it.pass) * (p.I / 128) + it.tile;
#pragma unroll
                for (int b = 0; b < 2; ++b) {
                    // the 32-block of these 8 columns spans the lanes tl ^ {0..3}
                    float m = 0.f;
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        m = fmaxf(m, fabsf(hv[b][j]));
                    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
                    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
                    const int E_blk = act_block_exp(m);
                    uint32_t word[kT];
                    act_words(hv[b], E_blk, word);
                    if (valid) {
                        const int col = 128 * it.tile + 64 * b + 8 * tl;
#pragma unroll
                        for (int t = 0; t < kT; ++t) {
                            *reinterpret_cast<uint32_t *>(p.h_terms + term_offset(p.rows, t, r, col)) = word[t];
                            if ((tl & 3) == 0)
                                p.h_sf[img * kSFImg + image_byte(n, t, 2 * b + (tl >> 2))] =
                                    (uint8_t)(E_blk - 1 - 3 * t + 127);
                        }
                    }
                }
            } else if (valid) {
                float *yrow = p.y_out + (int64_t)(it.r0 + n) * p.H + 256 * it.tile + 8 * tl;
                const int ncols = min(256, p.H - 256 * it.tile);  // 128 in a padded last tile
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    if (64 * b >= ncols)
                        break;
                    float4 *dst = reinterpret_cast<float4 *>(yrow + 64 * b);
                    dst[0] = make_float4(v[b][0], v[b][1], v[b][2], v[b][3]);
                    dst[1] = make_float4(v[b][4], v[b][5], v[b][6], v[b][7]);
                }
            }
        }
    }
#undef ITEM
}

// One FFN stage over all experts as its own (chained) launch.
template <int NT, bool GATE_UP, bool FP8 = false>
__global__ void __launch_bounds__(kThreads, 1)
    ffn_mxf4_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmA,
                    const FfnParams p)
{
    using C = Cfg<NT>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const StageSmem<NT> S(smem, 0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (p.wait_first)  // the offsets and the pass table are the preceding kernel's results
        grid_dep_wait();
    stage_prepare<NT>(p, S);
    if (warp == 1)
        tc::alloc(S.tslot, C::kTmemCols);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *S.tslot;
    // Chained launch: the producer fills the weight ring before waiting for
    // the preceding kernel (weights and offsets are older than it; the
    // activation terms, their scale images and the pass table are its
    // results); every other thread waits here. The next kernel is let start
    // only as this one's CTAs exit: triggered earlier, its CTAs sat resident
    // and waiting beside these, which measured slower.
    if (!(warp == 0 && lane == 0))
        grid_dep_wait();
    stage_roles<NT, GATE_UP, FP8>(tmW, tmA, p, S, tmem, WaitChained{});
    tc::fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after();
        tc::dealloc(tmem, C::kTmemCols);
    }
}

// Token passes of each expert: pass_start[e] = sum over e' < e of
// ceil(n_e' / nt), from the block's copy of the offsets, for one block's warp
// 0 (E <= kMaxE).
__device__ void pass_prefix(const int32_t *offsets, int E, int nt, int32_t *out)
{
    const int lane = threadIdx.x & 31;
    int carry = 0;
    for (int b = 0; b <= E; b += 32) {
        const int e = b + lane;
        const int c = e < E ? (offsets[e + 1] - offsets[e] + nt - 1) / nt : 0;
        int incl = c;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
            if (lane >= off)
                incl += o;
        }
        if (e <= E)
            out[e] = carry + incl - c;
        carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
}

// One unit (grouped row r, 256-value chunk c; u = r * chunks + c) of the
// activation terms: row r holds token src_row[r] / k; one warp, lane l holding
// values 8l .. 8l+7 of the chunk (one 16-byte load), a 32-value block being
// four lanes; each of the kT terms of the chunk leaves as one 128-byte row of
// 32-bit stores, in the term_offset layout, with their scale images (one per
// token pass and 128 columns). Rows of experts with at least hot_rows rows are
// skipped (the large-token kernel takes those experts). s_off / s_pass: the offsets
// and the token-pass prefix in shared memory. The three steps (locate, load,
// encode) are separate so that a warp can keep several units' loads in
// flight. COHERENT: src_row was written earlier in the same launch (read
// through L2, not the read-only path).
struct ActUnit {
    int r, c, n, tok;
    int64_t img_row;
    bool skip;
};

template <bool COHERENT>
__device__ __forceinline__ ActUnit act_unit_locate(int64_t u, const int32_t *__restrict__ src_row,
                                                   const int32_t *s_off, const int32_t *s_pass, int E, int k, int H,
                                                   int nt, int hot_rows)
{
    const int nch = (H + kKC - 1) / kKC;
    ActUnit a;
    a.r = (int)(u / nch);
    a.c = (int)(u % nch);
    int lo = 0, hi = E;  // expert of row r: largest e with s_off[e] <= r
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_off[mid] <= a.r)
            lo = mid;
        else
            hi = mid;
    }
    a.skip = s_off[lo + 1] - s_off[lo] >= hot_rows;  // the large-token kernel takes this expert
    const int local = a.r - s_off[lo];
    a.img_row = ((int64_t)s_pass[lo] + local / nt) * (H / 128);
    a.n = local % nt;
    a.tok = a.skip ? 0 : (COHERENT ? __ldcg(src_row + a.r) : __ldg(src_row + a.r)) / k;
    return a;
}

__device__ __forceinline__ uint4 act_unit_load(const ActUnit &a, const uint16_t *__restrict__ act, int H)
{
    const int col = a.c * kKC + 8 * (threadIdx.x & 31);
    if (a.skip || col >= H)  // H % 128 == 0: in a half chunk lanes 0..15 are live
        return make_uint4(0, 0, 0, 0);
    return __ldg(reinterpret_cast<const uint4 *>(act + (int64_t)a.tok * H + col));
}

__device__ __forceinline__ void act_unit_encode(const ActUnit &a, uint4 raw, int rows, int H,
                                                uint8_t *__restrict__ terms, uint8_t *__restrict__ sf)
{
    const int lane = threadIdx.x & 31;
    const int kb = lane >> 2, q = lane & 3;  // the lane's 32-block within the chunk; its place in the block
    const int col = a.c * kKC + 8 * lane;
    const bool live = col < H;
    float v[8];
    const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        v[2 * j] = __uint_as_float(w4[j] << 16);
        v[2 * j + 1] = __uint_as_float(w4[j] & 0xFFFF0000u);
    }
    float m = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j)
        m = fmaxf(m, fabsf(v[j]));
    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
    const int E_blk = act_block_exp(m);
    uint32_t word[kT];  // value j of the lane: nibble j (element 2i in the low nibble of byte i)
    act_words(v, E_blk, word);
    if (live) {
        uint32_t *tp = reinterpret_cast<uint32_t *>(terms + term_offset(rows, 0, a.r, col));
#pragma unroll
        for (int t = 0; t < kT; ++t)  // term t sits 128 bytes after term t-1
            tp[32 * t] = word[t];
        // scales of the block: lane q of it writes terms q and q + 4
        uint8_t *sp = sf + (a.img_row + 2 * a.c + (kb >> 2)) * kSFImg;
        sp[image_byte(a.n, q, kb & 3)] = (uint8_t)(E_blk - 1 - 3 * q + 127);
        sp[image_byte(a.n, q + 4, kb & 3)] = (uint8_t)(E_blk - 1 - 3 * (q + 4) + 127);
    }
}

// Activation rows -> kT E2M1 terms per value in grouped row order (act_terms_unit
// over every (row, 256-value chunk)). Block 0 also writes pass_start for the FFN
// stages and clears the status word (when given).
__global__ void __launch_bounds__(256) act_terms_kernel(const uint16_t *__restrict__ act, const int32_t *__restrict__ src_row,
                                                      const int32_t *__restrict__ offsets, int E, int k, int rows,
                                                      int H, int nt, int hot_rows, uint8_t *__restrict__ terms,
                                                      uint8_t *__restrict__ sf, int32_t *__restrict__ pass_start_out,
                                                      int *status)
{
    grid_dep_wait();  // the preceding kernel's results (chained launch)
    grid_dep_launch();
    __shared__ int32_t s_off[kMaxE + 1], s_pass[kMaxE + 1];
    const int warp = threadIdx.x >> 5;
    for (int e = threadIdx.x; e <= E; e += blockDim.x)
        s_off[e] = offsets[e];
    __syncthreads();
    if (warp == 0)
        pass_prefix(s_off, E, nt, s_pass);
    __syncthreads();
    if (blockIdx.x == 0) {
        for (int e = threadIdx.x; e <= E; e += blockDim.x)
            pass_start_out[e] = s_pass[e];
        if (threadIdx.x == 0 && status)
            *status = 0;
    }
    // Units (row, chunk) go round-robin over the warps (warp g: units g,
    // g + W, ...), so that skipped rows of hot experts, which are contiguous,
    // do not leave some warps idle while others carry double work.
    const int nch = (H + kKC - 1) / kKC;
    const int64_t total = (int64_t)rows * nch;
    const int64_t nwarps = (int64_t)gridDim.x * 8, gw = (int64_t)blockIdx.x * 8 + warp;
    for (int64_t u = gw; u < total; u += nwarps) {
        const ActUnit a = act_unit_locate<false>(u, src_row, s_off, s_pass, E, k, H, nt, hot_rows);
        if (!a.skip)
            act_unit_encode(a, act_unit_load(a, act, H), rows, H, terms, sf);
    }
}

// y[t, c] = sum_j w[t, j] * y_perm[dst_of[t*k + j], c], j in order.
__global__ void __launch_bounds__(256) combine_kernel(const float *__restrict__ y_perm,
                                                      const int32_t *__restrict__ dst_of,
                                                      const float *__restrict__ w, int T, int k, int H,
                                                      float *__restrict__ y)
{
    grid_dep_wait();  // the preceding kernel's results (chained launch)
    grid_dep_launch();
    const int t = blockIdx.y;
    const int c4 = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= T || c4 * 4 >= H)
        return;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
        const float wj = w[(int64_t)t * k + j];
        const float4 v = __ldg(reinterpret_cast<const float4 *>(y_perm + (int64_t)dst_of[(int64_t)t * k + j] * H) + c4);
        acc.x = fmaf(wj, v.x, acc.x);
        acc.y = fmaf(wj, v.y, acc.y);
        acc.z = fmaf(wj, v.z, acc.z);
        acc.w = fmaf(wj, v.w, acc.w);
    }
    reinterpret_cast<float4 *>(y + (int64_t)t * H)[c4] = acc;
}

// ---------------------------------------------------------------------------
// The whole layer as one persistent kernel (decode-sized token counts): the
// execution model of the pages' serving engine -- a resident engine kernel
// that removes the gaps at operator boundaries and keeps prefetching while
// the tensor cores compute ("Xiaomi MiMo-V2.5-Pro-UltraSpeed 發佈說明",
// agentlenshq.com, section "TileRT 執行模型").
// ---------------------------------------------------------------------------
// One CTA per SM, all co-resident (cooperative launch), 8 warps. The layer's
// steps run as phases separated by grid-wide barriers, so no launch boundary
// sits between them:
//   1. router GEMM tiles (all warps; the same tiles and split sums as the
//      chained router_gemm_kernel);                                  barrier 1
//   2. routing, a warp per token;                                    barrier 2
//   3. grouping by expert (CTA 0; offsets, src_row, dst_of, passes); barrier 3
//   4. gate/up: warps 1..7 encode the activation terms while the producer warp
//      already streams its first weight boxes; then the FFN roles; barrier 4
//      is the terms' completion, which only the producer's activation loads
//      and the other roles wait for;
//   5. down: the FFN roles again (second barrier set);              barrier 5
//   6. the weighted combine (all warps).                            barrier 6
// Every barrier wait is bounded (2 s); a CTA that gives up records
// MXMOE_ERR_TIMEOUT in the status word, which every waiter polls, so the
// others stop at their next barrier. Memory written by one phase and read by
// the next crosses CTAs through L2 (a release fence and atomic arrival, an
// acquire load, then ld.global.cg or the TMA), and generic-proxy writes read by
// the TMA are ordered with proxy fences on both sides.
constexpr int kFusedThreads = 256;
constexpr int kFusedMaxE = 384;      // routing keeps 12 logits per lane
constexpr int kFusedMaxPairs = 4096;  // grouping in one CTA's shared memory
constexpr int kFusedLocalRoute = 64;  // up to this many tokens CTA 0 routes them (no grid-wide barrier)

struct FusedParams {
    const uint16_t *x, *wg;
    const float *bias;
    int T, H, I, E, k, nsplit;
    float *partials;  // router partial sums [nsplit, T, E]
    int32_t *ids;
    float *w;
    int32_t *offsets, *src_row, *dst_of;  // the grouping (offsets also in gu / dn)
    int32_t *pass_start;                  // token passes before each expert (also in gu / dn)
    uint8_t *x_terms, *x_sf;              // the activation terms of x and their scale images
    float *y_perm, *y;
    unsigned *barrier;  // grid barrier arrivals, zero at launch
    int *status;
    FfnParams gu, dn;
};

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned *p)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Arrival of the CTA at the next grid barrier, by one thread, after a
// block-wide barrier that followed every thread's writes of the phase (and
// each thread's proxy fence, so that the TMA of other CTAs sees them).
__device__ __forceinline__ void grid_arrive(unsigned *ctr)
{
    __threadfence();
    atomicAdd(ctr, 1u);
}

// Waits until `target` arrivals; false on a timeout (recorded) or when another
// CTA has recorded a failure.
__device__ __forceinline__ bool grid_wait(const unsigned *ctr, unsigned target, int *status)
{
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_u32(ctr) < target) {
        if (*reinterpret_cast<volatile int *>(status) != 0)
            return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            set_status(status, MXMOE_ERR_TIMEOUT);
            return false;
        }
        __nanosleep(64);
    }
    asm volatile("fence.proxy.async.global;" ::: "memory");
    return true;
}

__device__ __forceinline__ void proxy_fence_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// Block-wide: arrive at barrier n and wait for it (every thread gets the verdict).
__device__ __forceinline__ bool grid_sync(const FusedParams &fp, unsigned n, int *s_flag)
{
    proxy_fence_global();
    __syncthreads();
    if (threadIdx.x == 0) {
        grid_arrive(fp.barrier);
        *s_flag = grid_wait(fp.barrier, n * gridDim.x, fp.status);
    }
    __syncthreads();
    return *s_flag != 0;
}

// The producer's wait before its first activation load: barrier n.
struct WaitGrid {
    const unsigned *ctr;
    unsigned target;
    int *status;
    __device__ __forceinline__ bool operator()() const { return grid_wait(ctr, target, status); }
};

// Grouping of the T*k pairs by expert in one CTA (phase 3): counts, prefix,
// token passes of NT rows, then the pairs placed in index order by warp 0, 32
// at a time: lanes holding the same expert (match_any) take consecutive
// places in lane order after that expert's earlier pairs (stable).
template <int NT>
__device__ void fused_group(const FusedParams &fp, int32_t *s_ids, int32_t *s_cnt, int32_t *s_off)
{
    const int n = fp.T * fp.k, E = fp.E;
    const int tid = threadIdx.x, lane = tid & 31;
    for (int q = tid; q < n; q += blockDim.x)
        s_ids[q] = __ldcg(fp.ids + q);
    for (int e = tid; e < E; e += blockDim.x)
        s_cnt[e] = 0;
    __syncthreads();
    for (int q = tid; q < n; q += blockDim.x)
        atomicAdd(&s_cnt[s_ids[q]], 1);
    __syncthreads();
    if (tid < 32) {  // exclusive prefixes of the counts (offsets) and of ceil(count / NT) (passes)
        int carry = 0, carry_p = 0;
        for (int b = 0; b <= E; b += 32) {
            const int e = b + lane;
            const int c = e < E ? s_cnt[e] : 0, cp = (c + NT - 1) / NT;
            int incl = c, incl_p = cp;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
                const int op = __shfl_up_sync(0xFFFFFFFFu, incl_p, off);
                if (lane >= off) {
                    incl += o;
                    incl_p += op;
                }
            }
            if (e <= E) {
                s_off[e] = carry + incl - c;
                fp.offsets[e] = carry + incl - c;
                fp.pass_start[e] = carry_p + incl_p - cp;
            }
            carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
            carry_p += __shfl_sync(0xFFFFFFFFu, incl_p, 31);
        }
    }
    __syncthreads();
    if (tid < 32) {  // s_cnt becomes each expert's next free place
        for (int e = lane; e < E; e += 32)
            s_cnt[e] = s_off[e];
        __syncwarp();
        for (int base = 0; base < n; base += 32) {
            const int q = base + lane;
            const int e = q < n ? s_ids[q] : -1;
            const uint32_t same = __match_any_sync(0xFFFFFFFFu, e);
            const int rank = __popc(same & ((1u << lane) - 1u));
            const int pos = e >= 0 ? s_cnt[e] + rank : 0;
            __syncwarp();
            if (e >= 0 && rank == 0)
                s_cnt[e] += __popc(same);
            __syncwarp();
            if (q < n) {
                fp.src_row[pos] = q;
                fp.dst_of[q] = pos;
            }
        }
    }
}

template <int NT>
__global__ void __launch_bounds__(kFusedThreads, 1)
    fused_layer_kernel(const __grid_constant__ CUtensorMap tmW13, const __grid_constant__ CUtensorMap tmX,
                       const __grid_constant__ CUtensorMap tmW2, const __grid_constant__ CUtensorMap tmH,
                       const FusedParams fp)
{
    using C = Cfg<NT>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const StageSmem<NT> S1(smem, 0), S2(smem, 1);
    // two flags in the spare words after the stages' tensor-memory slot and abort flag
    int &s_flag = *reinterpret_cast<int *>(smem + C::kOffMisc + 8);
    int &s_flag2 = *reinterpret_cast<int *>(smem + C::kOffMisc + 12);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int T = fp.T, E = fp.E, k = fp.k, H = fp.H;
    const int G = gridDim.x;
    if (warp == 1)
        tc::alloc(S1.tslot, C::kTmemCols);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *S1.tslot;
    int32_t *s_scratch = reinterpret_cast<int32_t *>(S1.sA);  // the activation ring is free until stage 1 loads

    // 1. router GEMM tiles
    {
        RouterRed &red = *reinterpret_cast<RouterRed *>(S1.sA);
        const int ex = (E + kRgExperts - 1) / kRgExperts, ty = (T + kRgTokens - 1) / kRgTokens;
        const int ntiles = ex * ty * fp.nsplit;
        for (int vt = blockIdx.x; vt < ntiles; vt += G)
            router_tile(fp.x, fp.wg, fp.bias, T, H, E, fp.partials, vt % ex, (vt / ex) % ty, vt / (ex * ty), fp.nsplit,
                        red);
    }
    unsigned nbar = 1;
    bool alive = grid_sync(fp, nbar, &s_flag);
    // 2. routing, a warp per token (the partial sums were written in this launch by other CTAs and were never
    // read before on this SM, so the read-only path holds no stale copy of them). Up to kFusedLocalRoute
    // tokens CTA 0 routes them all itself and goes on to the grouping without a grid-wide barrier.
    const bool local_route = T <= kFusedLocalRoute;
    if (alive && (!local_route || blockIdx.x == 0))
        for (int tok = (local_route ? 0 : blockIdx.x * 8) + warp; tok < T; tok += local_route ? 8 : G * 8)
            route_token<kFusedMaxE / 32, 4>(fp.partials, fp.nsplit, fp.nsplit > 1 ? fp.bias : nullptr, T, E, k,
                                            fp.ids, fp.w, tok);
    if (!local_route)
        alive = alive && grid_sync(fp, ++nbar, &s_flag);
    else
        __syncthreads();  // CTA 0's ids and weights, for its own grouping
    // 3. grouping (CTA 0)
    if (alive && blockIdx.x == 0)
        fused_group<NT>(fp, s_scratch, s_scratch + kFusedMaxPairs, s_scratch + kFusedMaxPairs + kFusedMaxE);
    alive = alive && grid_sync(fp, ++nbar, &s_flag);

    // 4. gate/up: warps 1..7 encode the activation terms while the producer (warp 0) streams its first weight
    // boxes and then waits for barrier 4 before loading activations
    if (alive) {
        int32_t *s_off = s_scratch, *s_pass = s_scratch + kFusedMaxE + 1;
        for (int e = tid; e <= E; e += blockDim.x) {
            s_off[e] = __ldcg(fp.offsets + e);
            s_pass[e] = __ldcg(fp.pass_start + e);
        }
        stage_prepare<NT>(fp.gu, S1);  // ends with a block-wide barrier
        const WaitGrid w4{fp.barrier, (++nbar) * G, fp.status};
        if (warp == 0) {
            stage_roles<NT, true, false>(tmW13, tmX, fp.gu, S1, tmem, w4);
        } else {
            const int nch = (H + kKC - 1) / kKC;
            const int64_t total = (int64_t)T * k * nch;
            const int64_t nworkers = (int64_t)G * 7, gw = (int64_t)blockIdx.x * 7 + (warp - 1);
            // four units per warp at a time: their row lookups, then their x loads, in flight together
            for (int64_t u0 = gw; u0 < total; u0 += 4 * nworkers) {
                ActUnit a[4];
                uint4 raw[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int64_t u = u0 + j * nworkers;
                    a[j] = act_unit_locate<true>(u < total ? u : u0, fp.src_row, s_off, s_pass, E, k, H, NT, INT_MAX);
                    a[j].skip = u >= total;
                }
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    raw[j] = act_unit_load(a[j], fp.x, H);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (!a[j].skip)
                        act_unit_encode(a[j], raw[j], T * k, H, fp.x_terms, fp.x_sf);
            }
            proxy_fence_global();
            named_bar_sync(1, 7 * 32);  // warps 1..7: this CTA's terms are written
            if (tid == 32) {
                grid_arrive(fp.barrier);
                s_flag2 = w4();
            }
            named_bar_sync(1, 7 * 32);
            if (s_flag2)
                stage_roles<NT, true, false>(tmW13, tmX, fp.gu, S1, tmem, w4);
            else if (tid == 32)
                *S1.abort_flag = 1;
        }
        tc::fence_before();
        __syncthreads();
        if (tid == 0)  // one verdict for the whole CTA
            s_flag = s_flag2 != 0 && *reinterpret_cast<volatile int *>(fp.status) == 0;
        __syncthreads();
        alive = s_flag != 0;
    }
    // 5. down
    if (alive) {
        proxy_fence_global();  // this thread's h writes, for the other CTAs' TMA
        __syncthreads();
        if (tid == 0)
            grid_arrive(fp.barrier);
        stage_prepare<NT>(fp.dn, S2);
        const WaitGrid w5{fp.barrier, (++nbar) * G, fp.status};
        if (warp == 0) {
            stage_roles<NT, false, false>(tmW2, tmH, fp.dn, S2, tmem, w5);
        } else {
            if (tid == 32)
                s_flag2 = w5();
            named_bar_sync(1, 7 * 32);
            if (s_flag2)
                stage_roles<NT, false, false>(tmW2, tmH, fp.dn, S2, tmem, w5);
            else if (tid == 32)
                *S2.abort_flag = 1;
        }
        tc::fence_before();
        __syncthreads();
        alive = s_flag2 != 0;
    }
    // 6. combine: y[t, c] = sum over j, in order, of w[t, j] * y_perm[dst_of[t*k + j], c]
    alive = alive && grid_sync(fp, ++nbar, &s_flag);
    if (alive) {
        const int H4 = H / 4;
        for (int64_t u = (int64_t)blockIdx.x * blockDim.x + tid; u < (int64_t)T * H4; u += (int64_t)G * blockDim.x) {
            const int t = (int)(u / H4), c4 = (int)(u % H4);
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int j = 0; j < k; ++j) {
                const float wj = __ldcg(fp.w + (int64_t)t * k + j);
                const int r = __ldcg(fp.dst_of + (int64_t)t * k + j);
                const float4 v = __ldcg(reinterpret_cast<const float4 *>(fp.y_perm + (int64_t)r * H) + c4);
                acc.x = fmaf(wj, v.x, acc.x);
                acc.y = fmaf(wj, v.y, acc.y);
                acc.z = fmaf(wj, v.z, acc.z);
                acc.w = fmaf(wj, v.w, acc.w);
            }
            reinterpret_cast<float4 *>(fp.y + (int64_t)t * H)[c4] = acc;
        }
    }
    tc::fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after();
        tc::dealloc(tmem, C::kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
struct FfnWs {
    int *status;
    int32_t *pass_start;  // [kMaxE + 1]: token passes before each expert
    uint8_t *x_terms;     // term_offset layout, K = H
    uint8_t *x_sf;        // scale images [pass][H/128][512]
    uint8_t *h_terms;     // term_offset layout, K = I
    uint8_t *h_sf;        // scale images [pass][I/128][512]
    int32_t *f8_pass_start;  // large-token kernel: its token passes before each expert [kMaxE + 1]
    int32_t *slot_row;    // large-token kernel: grouped row of each (token, slot) [rows]
    uint8_t *x_tiled;     // large-token kernel: x's two E4M3 terms per (pass, stage, term) as the shared-memory image
    uint8_t *x8_sf;       // their scale images
    uint8_t *h_tiled;     // large-token kernel: h's three E4M3 terms likewise
    uint8_t *h8_sf;       // their scale images
};

// The front of a decode-sized layer step as one cooperative launch: router
// GEMM tiles, routing, grouping and the activation terms -- the persistent
// layer kernel's first phases (the same device code, so the results are
// bit-identical to the chained kernels'), with only two grid-wide barriers up
// to kFusedLocalRoute tokens (CTA 0 routes and groups them alone) and no
// launch boundary between the steps. The FFN stages follow as chained launches.
constexpr size_t kFrontSmem = sizeof(RouterRed) > (size_t)(kFusedMaxPairs + 2 * kFusedMaxE + 1) * 4
                                  ? sizeof(RouterRed)
                                  : (size_t)(kFusedMaxPairs + 2 * kFusedMaxE + 1) * 4;

template <int NT>
__global__ void __launch_bounds__(kFusedThreads, 1) front_kernel(const FusedParams fp)
{
    extern __shared__ __align__(16) uint8_t front_smem[];
    __shared__ int s_flag;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int T = fp.T, E = fp.E, k = fp.k, H = fp.H;
    const int G = gridDim.x;
    int32_t *s_scratch = reinterpret_cast<int32_t *>(front_smem);
    // 1. router GEMM tiles
    {
        RouterRed &red = *reinterpret_cast<RouterRed *>(front_smem);
        const int ex = (E + kRgExperts - 1) / kRgExperts, ty = (T + kRgTokens - 1) / kRgTokens;
        const int ntiles = ex * ty * fp.nsplit;
        for (int vt = blockIdx.x; vt < ntiles; vt += G)
            router_tile(fp.x, fp.wg, fp.bias, T, H, E, fp.partials, vt % ex, (vt / ex) % ty, vt / (ex * ty), fp.nsplit,
                        red);
    }
    unsigned nbar = 1;
    bool alive = grid_sync(fp, nbar, &s_flag);
    // 2. routing, a warp per token (partial sums written in this launch by other CTAs, never read before on this
    // SM); up to kFusedLocalRoute tokens CTA 0 routes them all and groups them without another grid barrier
    const bool local_route = T <= kFusedLocalRoute;
    if (alive && (!local_route || blockIdx.x == 0))
        for (int tok = (local_route ? 0 : blockIdx.x * 8) + warp; tok < T; tok += local_route ? 8 : G * 8)
            route_token<kFusedMaxE / 32, 4>(fp.partials, fp.nsplit, fp.nsplit > 1 ? fp.bias : nullptr, T, E, k,
                                            fp.ids, fp.w, tok);
    if (!local_route)
        alive = alive && grid_sync(fp, ++nbar, &s_flag);
    else
        __syncthreads();
    // 3. grouping (CTA 0): offsets, src_row, dst_of and the token passes
    if (alive && blockIdx.x == 0)
        fused_group<NT>(fp, s_scratch, s_scratch + kFusedMaxPairs, s_scratch + kFusedMaxPairs + kFusedMaxE);
    alive = alive && grid_sync(fp, ++nbar, &s_flag);
    // 4. the activation terms of every grouped row (all warps, round-robin over (row, 256-value chunk))
    if (alive) {
        int32_t *s_off = s_scratch, *s_pass = s_scratch + kFusedMaxE + 1;
        for (int e = tid; e <= E; e += blockDim.x) {
            s_off[e] = __ldcg(fp.offsets + e);
            s_pass[e] = __ldcg(fp.pass_start + e);
        }
        __syncthreads();
        const int nch = (H + kKC - 1) / kKC;
        const int64_t total = (int64_t)T * k * nch;
        const int64_t nworkers = (int64_t)G * (kFusedThreads / 32), gw = (int64_t)blockIdx.x * (kFusedThreads / 32) + warp;
        for (int64_t u = gw; u < total; u += nworkers) {
            const ActUnit a = act_unit_locate<true>(u, fp.src_row, s_off, s_pass, E, k, H, NT, INT_MAX);
            act_unit_encode(a, act_unit_load(a, fp.x, H), T * k, H, fp.x_terms, fp.x_sf);
        }
    }
}

// Token counts at which both FFN stages run on the large-token kernel
// (ffn_prefill8.cu: block-scaled fp8-kind tensor cores, the E2M1 weights as
// stored, x as two E4M3 terms and h as three) for every expert, instead of
// the E2M1-term MMAs: from 16384 grouped rows (2048 tokens at top-8), where
// experts see hundreds of tokens and the stages are bound by the tensor cores.
constexpr int64_t kLargeRows = 16384;
bool use_large_path(int T, int k) { return (int64_t)T * k >= kLargeRows; }

// Below that, experts with at least kHotRows rows (a skewed router) still go
// to the large-token kernel, the rest to the E2M1-term kernel: the E2M1-term
// kernel multiplies 8 terms per activation value and re-streams the expert's
// weights for every 16-token pass, so from about a hundred tokens per expert
// the large-token kernel is cheaper (cuts of 64, 128, 256 and 512 rows
// measured within noise of each other). Only token counts that can produce
// such an expert (T >= kHotRows) launch its kernels.
constexpr int kHotRows = 128;
bool use_hybrid(int T, int k) { return !use_large_path(T, k) && T >= kHotRows; }
int large_min_rows(int T, int k) { return use_large_path(T, k) ? 0 : kHotRows; }

// fp8: the FP8-weight FFN, which runs every expert on the E2M1-term kernel.
int64_t ffn_ws_layout(int T, int k, int E, int H, int I, FfnWs *ws, void *base, bool fp8 = false)
{
    int64_t off = 0;
    auto take = [&](int64_t bytes) {
        int64_t o = off;
        off = align256(off + bytes);
        return o;
    };
    const int64_t rows = (int64_t)T * k;
    const int64_t passes = max_passes(rows);
    const int64_t o_status = take(16);
    const int64_t o_ps = take((kMaxE + 1) * 4);
    const bool terms = fp8 || !use_large_path(T, k);        // the E2M1-term kernel runs
    const bool large = !fp8 && (!terms || use_hybrid(T, k));  // the large-token kernel runs
    const int64_t o_xt = take(terms ? rows * kT * pad256(H) / 2 : 0);
    const int64_t o_xs = take(terms ? passes * (H / 128) * kSFImg : 0);
    const int64_t o_ht = take(terms ? rows * kT * pad256(I) / 2 : 0);
    const int64_t o_hs = take(terms ? passes * (I / 128) * kSFImg : 0);
    const int64_t o_bps = take(large ? (kMaxE + 1) * 4 : 0);
    const int64_t o_sr = take(large ? rows * 4 : 0);
    const int64_t bp = large ? f8_max_passes(rows, E, large_min_rows(T, k)) : 0;  // 224-token passes, at most
    const int64_t o_xp = take(f8_terms_bytes(bp, H, 2));
    const int64_t o_x8s = take(f8_sf_bytes(bp, H, 2));
    const int64_t o_h2 = take(f8_terms_bytes(bp, I, 3));
    const int64_t o_h8s = take(f8_sf_bytes(bp, I, 3));
    if (ws && base) {
        uint8_t *b = static_cast<uint8_t *>(base);
        ws->status = reinterpret_cast<int *>(b + o_status);
        ws->pass_start = reinterpret_cast<int32_t *>(b + o_ps);
        ws->x_terms = b + o_xt;
        ws->x_sf = b + o_xs;
        ws->h_terms = b + o_ht;
        ws->h_sf = b + o_hs;
        ws->f8_pass_start = large ? reinterpret_cast<int32_t *>(b + o_bps) : nullptr;
        ws->slot_row = large ? reinterpret_cast<int32_t *>(b + o_sr) : nullptr;
        ws->x_tiled = large ? b + o_xp : nullptr;
        ws->x8_sf = large ? b + o_x8s : nullptr;
        ws->h_tiled = large ? b + o_h2 : nullptr;
        ws->h8_sf = large ? b + o_h8s : nullptr;
    }
    return off;
}


int encode(CUtensorMap *m, int rank, const void *base, const cuuint64_t *dims, const cuuint64_t *strides,
           const cuuint32_t *box, CUtensorMapL2promotion promo, const char *what,
           CUtensorMapDataType type = CU_TENSOR_MAP_DATA_TYPE_UINT8)
{
    auto enc = tensor_map_encoder();
    if (!enc)
        return fail(MXMOE_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const cuuint32_t es[5] = {1, 1, 1, 1, 1};
    CUresult r = enc(m, type, (cuuint32_t)rank, const_cast<void *>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(MXMOE_ERR_CUDA, "cuTensorMapEncodeTiled (%s) failed: %d", what, (int)r);
    return MXMOE_OK;
}

// The code boxes of one weight matrix (all experts) as rows of 128 bytes; a
// request brings one box (256 rows), with the 128-byte swizzle.
int encode_weights(CUtensorMap *m, const void *base, int64_t n_boxes)
{
    const cuuint64_t dims[2] = {128, (cuuint64_t)(n_boxes * 256)};
    const cuuint64_t strides[1] = {128};
    const cuuint32_t box[2] = {128, 256};
    return encode(m, 2, base, dims, strides, box, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, "weights");
}

// Activation terms (term_offset layout), dims {128, kT, rows, K/256}; a
// request brings all terms of nt rows of one chunk. Rows past the end read as
// zero.
int encode_terms(CUtensorMap *m, const void *base, int64_t rows, int K, int nt)
{
    const cuuint64_t dims[4] = {128, (cuuint64_t)kT, (cuuint64_t)rows, (cuuint64_t)((K + kKC - 1) / kKC)};
    const cuuint64_t strides[3] = {128, (cuuint64_t)(kT * 128), (cuuint64_t)(rows * kT * 128)};
    const cuuint32_t box[4] = {128, (cuuint32_t)kT, (cuuint32_t)nt, 1};
    return encode(m, 4, base, dims, strides, box, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, "activation terms");
}

// The same terms for the FP8 kernel: the 4-bit codes unpacked by the TMA into
// one byte per value (16U4_ALIGN16B; dims and box counted in values), a
// request bringing one 128-value K half of all terms of nt rows.
int encode_terms_unpacked(CUtensorMap *m, const void *base, int64_t rows, int K, int nt)
{
    const cuuint64_t dims[4] = {256, (cuuint64_t)kT, (cuuint64_t)rows, (cuuint64_t)((K + kKC - 1) / kKC)};
    const cuuint64_t strides[3] = {128, (cuuint64_t)(kT * 128), (cuuint64_t)(rows * kT * 128)};
    const cuuint32_t box[4] = {128, (cuuint32_t)kT, (cuuint32_t)nt, 1};
    return encode(m, 4, base, dims, strides, box, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, "unpacked activation terms",
                  CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B);
}

template <int NT, bool GATE_UP, bool FP8 = false>
int launch_ffn(const void *codes, const uint8_t *act_terms, const FfnParams &p, cudaStream_t st)
{
    using C = Cfg<NT>;
    auto kernel = ffn_mxf4_kernel<NT, GATE_UP, FP8>;
    static thread_local int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem) != cudaSuccess)
            return fail(MXMOE_ERR_CUDA, "ffn_mxf4_kernel: cannot reserve %zu bytes of shared memory", C::kSmem);
        configured_dev = dev;
    }
    CUtensorMap tmW, tmA;
    const int64_t chunks = FP8 ? p.K / 128 : (p.K + kKC - 1) / kKC;
    if (int rc = encode_weights(&tmW, codes, (int64_t)p.E * p.tiles * chunks))
        return rc;
    if (int rc = FP8 ? encode_terms_unpacked(&tmA, act_terms, p.rows, p.K, NT)
                     : encode_terms(&tmA, act_terms, p.rows, p.K, NT))
        return rc;
    const char *name = FP8 ? (GATE_UP ? "ffn_mxf4_kernel<gate_up, fp8 weights>" : "ffn_mxf4_kernel<down, fp8 weights>")
                           : (GATE_UP ? "ffn_mxf4_kernel<gate_up>" : "ffn_mxf4_kernel<down>");
    return launch_kernel(name, kernel, num_sms(), kThreads, C::kSmem, st, tmW, tmA, p);
}

// Token rows per pass: 8 up to 8 tokens (an expert then never sees more than
// 8 rows), else 16.
int token_tile(int T) { return T <= 8 ? 8 : 16; }

// The shapes every FFN entry point (and the layer) accepts.
bool shapes_ok(int T, int k, int E, int H, int I)
{
    return !(T < 0 || k < 1 || k > 32 || E <= 0 || E > kMaxE || H <= 0 || I <= 0 || H % 128 || I % 128 ||
             H > 32768 || I > 32768 || (int64_t)T * k > (1 << 22) || (int64_t)E * I * H / 128 >= (1LL << 31));
}

int validate_ffn(int T, int k, int E, int H, int I)
{
    if (!shapes_ok(T, k, E, H, I))
        return fail(MXMOE_ERR_INVALID_SHAPE,
                    "expert FFN: T=%d k=%d E=%d H=%d I=%d (need H, I multiples of 128 up to 32768, 1 <= k <= 32, "
                    "E <= 1024, T*k <= 2^22, E*I*H < 2^38)",
                    T, k, E, H, I);
    return MXMOE_OK;
}

// The four parts of the prepacked blob.
struct Blob {
    const uint8_t *w13, *w2, *sf13, *sf2;
};

Blob blob_parts(const void *prepacked, int E, int H, int I)
{
    const uint8_t *b = static_cast<const uint8_t *>(prepacked);
    Blob o;
    o.w13 = b;
    const int64_t Hp = pad256(H), Ip = pad256(I);
    o.w2 = o.w13 + (int64_t)E * 2 * I * (Hp / 2);
    o.sf13 = o.w2 + (int64_t)E * Hp * (Ip / 2);
    o.sf2 = o.sf13 + (int64_t)E * 2 * I * (Hp / 32);
    return o;
}

}  // namespace

// clear_status: whether this call starts a new status record (the layer
// clears it itself before the router, which may record a timeout in it).
int run_ffn_gate_up(const void *x, const int32_t *offsets, const int32_t *src_row, const void *prepacked, int T,
                    int k, int E, int H, int I, void *workspace, bool clear_status, cudaStream_t st)
{
    FfnWs ws;
    ffn_ws_layout(T, k, E, H, I, &ws, workspace);
    int *clear = clear_status ? ws.status : nullptr;
    const int rows = T * k;
    const int nt = token_tile(T);
    const Blob bl = blob_parts(prepacked, E, H, I);
    if (!use_large_path(T, k)) {  // E2M1-term kernel: every expert, or (hybrid) those below kHotRows rows
        const int hot_rows = use_hybrid(T, k) ? kHotRows : INT_MAX;
        const int64_t warps = (int64_t)rows * ((H + kKC - 1) / kKC);
        const int blocks = (int)std::min<int64_t>((warps + 7) / 8, (int64_t)num_sms() * 8);
        if (int rc = launch_kernel("act_terms_kernel", act_terms_kernel, blocks < 1 ? 1 : blocks, 256, 0, st,
                                   static_cast<const uint16_t *>(x), src_row, offsets, E, k, rows, H, nt, hot_rows,
                                   ws.x_terms, ws.x_sf, ws.pass_start, clear))
            return rc;
        clear = nullptr;  // cleared once, before anything could record a timeout
        FfnParams p{};
        p.tiles = I / 128;
        p.K = H;
        p.rows = rows;
        p.wsf = bl.sf13;
        p.asf = ws.x_sf;
        p.offsets = offsets;
        p.pass_start = ws.pass_start;
        p.E = E;
        p.h_terms = ws.h_terms;
        p.h_sf = ws.h_sf;
        p.I = I;
        p.y_out = nullptr;
        p.H = H;
        p.hot_rows = hot_rows;
        p.status = ws.status;
        if (int rc = nt == 8 ? launch_ffn<8, true>(bl.w13, ws.x_terms, p, st)
                             : launch_ffn<16, true>(bl.w13, ws.x_terms, p, st))
            return rc;
        if (!use_hybrid(T, k))
            return MXMOE_OK;
    }
    // large-token kernel: every expert, or (hybrid) those with at least kHotRows rows; x as two E4M3 terms,
    // h leaves as three
    if (int rc = run_f8_prep(x, offsets, src_row, k, rows, E, H, large_min_rows(T, k), ws.f8_pass_start, ws.slot_row,
                             ws.x_tiled, ws.x8_sf, clear, st))
        return rc;
    return run_f8_stage(true, ws.x_tiled, ws.x8_sf, offsets, ws.f8_pass_start, bl.w13, bl.sf13, E, H, I, ws.h_tiled,
                        ws.h8_sf, nullptr, ws.status, st);
}

int run_ffn_down(const int32_t *offsets, const void *prepacked, int T, int k, int E, int H, int I, float *y_perm,
                 void *workspace, cudaStream_t st)
{
    FfnWs ws;
    ffn_ws_layout(T, k, E, H, I, &ws, workspace);
    const int rows = T * k;
    const int nt = token_tile(T);
    const Blob bl = blob_parts(prepacked, E, H, I);
    if (!use_large_path(T, k)) {
        FfnParams p{};
        p.tiles = (int)(pad256(H) / 256);
        p.K = I;
        p.rows = rows;
        p.wsf = bl.sf2;
        p.asf = ws.h_sf;
        p.offsets = offsets;
        p.pass_start = ws.pass_start;
        p.E = E;
        p.h_terms = nullptr;
        p.h_sf = nullptr;
        p.I = I;
        p.y_out = y_perm;
        p.H = H;
        p.hot_rows = use_hybrid(T, k) ? kHotRows : INT_MAX;
        p.status = ws.status;
        if (int rc = nt == 8 ? launch_ffn<8, false>(bl.w2, ws.h_terms, p, st)
                             : launch_ffn<16, false>(bl.w2, ws.h_terms, p, st))
            return rc;
        if (!use_hybrid(T, k))
            return MXMOE_OK;
    }
    return run_f8_stage(false, ws.h_tiled, ws.h8_sf, offsets, ws.f8_pass_start, bl.w2, bl.sf2, E, H, I, nullptr,
                        nullptr, y_perm, ws.status, st);
}

// The FP8-weight FFN: both stages on the E2M1-term kernel with kind::mxf8f6f4
// for every expert and token count.
struct Fp8Blob {
    const uint8_t *w13, *w2, *sf13, *sf2;
};

Fp8Blob fp8_blob_parts(const void *prepacked, int E, int H, int I)
{
    const uint8_t *b = static_cast<const uint8_t *>(prepacked);
    const int64_t Hp = pad256(H);
    Fp8Blob o;
    o.w13 = b;
    o.w2 = o.w13 + (int64_t)E * 2 * I * H;
    o.sf13 = o.w2 + (int64_t)E * Hp * I;
    o.sf2 = o.sf13 + (int64_t)E * 2 * I * (H / 32);
    return o;
}

int run_expert_ffn_fp8(const void *x, const int32_t *offsets, const int32_t *src_row, const void *prepacked, int T,
                       int k, int E, int H, int I, float *y_perm, void *workspace, bool clear_status, cudaStream_t st)
{
    FfnWs ws;
    ffn_ws_layout(T, k, E, H, I, &ws, workspace, true);
    const int rows = T * k;
    const int nt = token_tile(T);
    const Fp8Blob bl = fp8_blob_parts(prepacked, E, H, I);
    const int64_t warps = (int64_t)rows * ((H + kKC - 1) / kKC);
    const int blocks = (int)std::min<int64_t>((warps + 7) / 8, (int64_t)num_sms() * 8);
    if (int rc = launch_kernel("act_terms_kernel", act_terms_kernel, blocks < 1 ? 1 : blocks, 256, 0, st,
                               static_cast<const uint16_t *>(x), src_row, offsets, E, k, rows, H, nt, INT_MAX,
                               ws.x_terms, ws.x_sf, ws.pass_start, clear_status ? ws.status : nullptr))
        return rc;
    FfnParams p{};
    p.tiles = I / 128;
    p.K = H;
    p.rows = rows;
    p.wsf = bl.sf13;
    p.asf = ws.x_sf;
    p.offsets = offsets;
    p.pass_start = ws.pass_start;
    p.E = E;
    p.h_terms = ws.h_terms;
    p.h_sf = ws.h_sf;
    p.I = I;
    p.H = H;
    p.hot_rows = INT_MAX;
    p.status = ws.status;
    if (int rc = nt == 8 ? launch_ffn<8, true, true>(bl.w13, ws.x_terms, p, st)
                         : launch_ffn<16, true, true>(bl.w13, ws.x_terms, p, st))
        return rc;
    p.tiles = (int)(pad256(H) / 256);
    p.K = I;
    p.wsf = bl.sf2;
    p.asf = ws.h_sf;
    p.h_terms = nullptr;
    p.h_sf = nullptr;
    p.y_out = y_perm;
    return nt == 8 ? launch_ffn<8, false, true>(bl.w2, ws.h_terms, p, st)
                   : launch_ffn<16, false, true>(bl.w2, ws.h_terms, p, st);
}

int64_t ffn_workspace_bytes_fp8(int T, int k, int E, int H, int I)
{
    return ffn_ws_layout(T, k, E, H, I, nullptr, nullptr, true);
}

// Whether the persistent layer kernel takes these sizes: every expert on the
// E2M1-term kernel, the grouping in one CTA, routing with 12 logits a lane.
bool fused_layer_ok(int T, int k, int E, int H, int I)
{
    return T >= 1 && T <= 256 && (int64_t)T * k <= kFusedMaxPairs && E <= kFusedMaxE && E >= k && k <= 32 &&
           shapes_ok(T, k, E, H, I);
}

template <int NT>
int launch_fused(const FusedParams &fp, const uint8_t *w13, const uint8_t *w2, const uint8_t *h_terms,
                 cudaStream_t st)
{
    using C = Cfg<NT>;
    auto kernel = fused_layer_kernel<NT>;
    static thread_local int configured_dev = -1;
    static thread_local int grid = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem) != cudaSuccess)
            return fail(MXMOE_ERR_CUDA, "fused_layer_kernel: cannot reserve %zu bytes of shared memory", C::kSmem);
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kFusedThreads, C::kSmem) != cudaSuccess ||
            per_sm < 1)
            return fail(MXMOE_ERR_CUDA, "fused_layer_kernel: no CTA fits on an SM");
        grid = num_sms();  // one CTA per SM, all resident at once
        configured_dev = dev;
    }
    CUtensorMap tmW13, tmX, tmW2, tmH;
    const int rows = fp.T * fp.k;
    if (int rc = encode_weights(&tmW13, w13, (int64_t)fp.E * fp.gu.tiles * ((fp.H + kKC - 1) / kKC)))
        return rc;
    if (int rc = encode_terms(&tmX, fp.x_terms, rows, fp.H, NT))
        return rc;
    if (int rc = encode_weights(&tmW2, w2, (int64_t)fp.E * fp.dn.tiles * ((fp.I + kKC - 1) / kKC)))
        return rc;
    if (int rc = encode_terms(&tmH, h_terms, rows, fp.I, NT))
        return rc;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kFusedThreads);
    cfg.dynamicSmemBytes = C::kSmem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;  // the grid-wide barriers need every CTA resident
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, tmW13, tmX, tmW2, tmH, fp);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(MXMOE_ERR_CUDA, "fused_layer_kernel: %s", cudaGetErrorString(e));
    }
    return check_launch("fused_layer_kernel");
}

// The whole layer in one persistent launch (fused_layer_ok sizes). ffn_ws: the
// FFN workspace of (T, k, E, H, I); its first 16 bytes (status word, barrier
// counter) are cleared here, before the launch. partials: [nsplit, T, E].
int run_fused_layer(const void *x, const void *wg, const float *bias, const void *prepacked, int T, int H, int I,
                    int E, int k, int nsplit, float *partials, int32_t *ids, float *w, int32_t *offsets,
                    int32_t *src_row, int32_t *dst_of, float *y_perm, float *y, void *ffn_ws, cudaStream_t st)
{
    FfnWs ws;
    ffn_ws_layout(T, k, E, H, I, &ws, ffn_ws);
    if (cudaMemsetAsync(ws.status, 0, 16, st) != cudaSuccess)
        return fail(MXMOE_ERR_CUDA, "persistent layer: cannot clear the status word");
    const Blob bl = blob_parts(prepacked, E, H, I);
    const int nt = token_tile(T);
    FusedParams fp{};
    fp.x = static_cast<const uint16_t *>(x);
    fp.wg = static_cast<const uint16_t *>(wg);
    fp.bias = bias;
    fp.T = T;
    fp.H = H;
    fp.I = I;
    fp.E = E;
    fp.k = k;
    fp.nsplit = nsplit;
    fp.partials = partials;
    fp.ids = ids;
    fp.w = w;
    fp.offsets = offsets;
    fp.src_row = src_row;
    fp.dst_of = dst_of;
    fp.pass_start = ws.pass_start;
    fp.x_terms = ws.x_terms;
    fp.x_sf = ws.x_sf;
    fp.y_perm = y_perm;
    fp.y = y;
    fp.barrier = reinterpret_cast<unsigned *>(reinterpret_cast<uint8_t *>(ws.status) + 8);
    fp.status = ws.status;
    FfnParams &gu = fp.gu;
    gu.tiles = I / 128;
    gu.K = H;
    gu.rows = T * k;
    gu.wsf = bl.sf13;
    gu.asf = ws.x_sf;
    gu.offsets = offsets;
    gu.pass_start = ws.pass_start;
    gu.E = E;
    gu.h_terms = ws.h_terms;
    gu.h_sf = ws.h_sf;
    gu.I = I;
    gu.H = H;
    gu.hot_rows = INT_MAX;
    gu.status = ws.status;
    FfnParams &dn = fp.dn;
    dn = gu;
    dn.tiles = (int)(pad256(H) / 256);
    dn.K = I;
    dn.wsf = bl.sf2;
    dn.asf = ws.h_sf;
    dn.h_terms = nullptr;
    dn.h_sf = nullptr;
    dn.y_out = y_perm;
    return nt == 8 ? launch_fused<8>(fp, bl.w13, bl.w2, ws.h_terms, st)
                   : launch_fused<16>(fp, bl.w13, bl.w2, ws.h_terms, st);
}

int run_expert_ffn(const void *x, const int32_t *offsets, const int32_t *src_row, const void *prepacked, int T,
                   int k, int E, int H, int I, float *y_perm, void *workspace, bool clear_status, cudaStream_t st)
{
    if (int rc = run_ffn_gate_up(x, offsets, src_row, prepacked, T, k, E, H, I, workspace, clear_status, st))
        return rc;
    return run_ffn_down(offsets, prepacked, T, k, E, H, I, y_perm, workspace, st);
}

int run_combine(const float *y_perm, const int32_t *dst_of, const float *w, int T, int k, int H, float *y,
                cudaStream_t st)
{
    dim3 grid((H / 4 + 255) / 256, T);
    return launch_kernel("combine_kernel", combine_kernel, grid, 256, 0, st, y_perm, dst_of, w, T, k, H, y);
}

// Shapes the front kernel takes: the E2M1-term path without hot experts
// (T < kHotRows), at most kFusedMaxPairs pairs and kFusedMaxE experts, and
// the mma.sync router (T < 512).
bool front_ok(int T, int k, int E, int H, int I)
{
    return T >= 1 && T < kHotRows && !use_large_path(T, k) && (int64_t)T * k <= kFusedMaxPairs && k <= E &&
           E <= kFusedMaxE && shapes_ok(T, k, E, H, I);
}

template <int NT>
int launch_front(const FusedParams &fp, cudaStream_t st)
{
    auto kernel = front_kernel<NT>;
    static thread_local int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kFrontSmem) != cudaSuccess)
            return fail(MXMOE_ERR_CUDA, "front_kernel: cannot reserve %zu bytes of shared memory", kFrontSmem);
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kFusedThreads, kFrontSmem) != cudaSuccess ||
            per_sm < 1)
            return fail(MXMOE_ERR_CUDA, "front_kernel: no CTA fits on an SM");
        configured_dev = dev;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(num_sms());  // one CTA per SM, all resident at once
    cfg.blockDim = dim3(kFusedThreads);
    cfg.dynamicSmemBytes = kFrontSmem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;  // the grid-wide barriers need every CTA resident
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    chain_next();  // a plain launch, first of the layer's chain
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, fp);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(MXMOE_ERR_CUDA, "front_kernel: %s", cudaGetErrorString(e));
    }
    return check_launch("front_kernel");
}

// The layer for front_ok shapes: the front kernel (router, routing, grouping,
// activation terms), then the gate/up and down stages on the E2M1-term kernel
// and the combine, chained. The gate/up stage reads the grouping that its
// predecessor wrote, so all its threads wait for it first (FfnParams::wait_first).
int run_layer_front(const void *x, const void *wg, const float *bias, const void *prepacked, int T, int H, int I,
                    int E, int k, int nsplit, float *partials, int32_t *ids, float *w, int32_t *offsets,
                    int32_t *src_row, int32_t *dst_of, float *y_perm, float *y, void *ffn_ws, cudaStream_t st)
{
    FfnWs ws;
    ffn_ws_layout(T, k, E, H, I, &ws, ffn_ws);
    if (cudaMemsetAsync(ws.status, 0, 16, st) != cudaSuccess)  // the status word and the grid barrier's count
        return fail(MXMOE_ERR_CUDA, "layer: cannot clear the status word");
    const Blob bl = blob_parts(prepacked, E, H, I);
    const int nt = token_tile(T);
    FusedParams fp{};
    fp.x = static_cast<const uint16_t *>(x);
    fp.wg = static_cast<const uint16_t *>(wg);
    fp.bias = bias;
    fp.T = T;
    fp.H = H;
    fp.I = I;
    fp.E = E;
    fp.k = k;
    fp.nsplit = nsplit;
    fp.partials = partials;
    fp.ids = ids;
    fp.w = w;
    fp.offsets = offsets;
    fp.src_row = src_row;
    fp.dst_of = dst_of;
    fp.pass_start = ws.pass_start;
    fp.x_terms = ws.x_terms;
    fp.x_sf = ws.x_sf;
    fp.barrier = reinterpret_cast<unsigned *>(reinterpret_cast<uint8_t *>(ws.status) + 8);
    fp.status = ws.status;
    ChainScope chain;
    if (int rc = nt == 8 ? launch_front<8>(fp, st) : launch_front<16>(fp, st))
        return rc;
    FfnParams p{};
    p.tiles = I / 128;
    p.K = H;
    p.rows = T * k;
    p.wsf = bl.sf13;
    p.asf = ws.x_sf;
    p.offsets = offsets;
    p.pass_start = ws.pass_start;
    p.E = E;
    p.h_terms = ws.h_terms;
    p.h_sf = ws.h_sf;
    p.I = I;
    p.y_out = nullptr;
    p.H = H;
    p.hot_rows = INT_MAX;
    p.status = ws.status;
    p.wait_first = 1;
    if (int rc = nt == 8 ? launch_ffn<8, true>(bl.w13, ws.x_terms, p, st) : launch_ffn<16, true>(bl.w13, ws.x_terms, p, st))
        return rc;
    if (int rc = run_ffn_down(offsets, prepacked, T, k, E, H, I, y_perm, ffn_ws, st))
        return rc;
    return run_combine(y_perm, dst_of, w, T, k, H, y, st);
}

int64_t ffn_workspace_bytes(int T, int k, int E, int H, int I)
{
    return ffn_ws_layout(T, k, E, H, I, nullptr, nullptr);
}

int validate_ffn_shapes(int T, int k, int E, int H, int I) { return validate_ffn(T, k, E, H, I); }
bool ffn_shapes_ok(int T, int k, int E, int H, int I) { return shapes_ok(T, k, E, H, I); }

}  // namespace mxmoe

using namespace mxmoe;

extern "C" MXMOE_API int64_t mxmoe_ffn_workspace_size(int T, int k, int E, int H, int I)
{
    if (!ffn_shapes_ok(T, k, E, H, I))
        return -1;
    return ffn_workspace_bytes(T, k, E, H, I);
}

static int check_ffn_args(const char *fn, int T, int k, int E, int H, int I, void *workspace, int64_t workspace_bytes,
                          bool fp8 = false)
{
    if (int rc = validate_ffn_shapes(T, k, E, H, I))
        return rc;
    const int64_t need = fp8 ? ffn_workspace_bytes_fp8(T, k, E, H, I) : ffn_workspace_bytes(T, k, E, H, I);
    if (!workspace || workspace_bytes < need)
        return fail(MXMOE_ERR_WORKSPACE, "%s: workspace of %lld bytes, need %lld", fn, (long long)workspace_bytes,
                    (long long)need);
    if (reinterpret_cast<uintptr_t>(workspace) & 255)
        return fail(MXMOE_ERR_ALIGNMENT, "%s: workspace needs 256-byte alignment", fn);
    return MXMOE_OK;
}

static bool aligned32(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

extern "C" MXMOE_API int mxmoe_expert_ffn(const void *x, const int32_t *offsets, const int32_t *src_row,
                                          const void *prepacked, int T, int k, int E, int H, int I, float *y_perm,
                                          void *workspace, int64_t workspace_bytes, void *stream)
{
    if (int rc = check_ffn_args("mxmoe_expert_ffn", T, k, E, H, I, workspace, workspace_bytes))
        return rc;
    if (T == 0)
        return MXMOE_OK;
    if (!x || !offsets || !src_row || !prepacked || !y_perm)
        return fail(MXMOE_ERR_NULL, "mxmoe_expert_ffn: NULL pointer");
    if (!aligned16(x) || !aligned32(prepacked) || !aligned16(y_perm))
        return fail(MXMOE_ERR_ALIGNMENT, "mxmoe_expert_ffn: x and y_perm need 16-byte, prepacked 32-byte alignment");
    if (int rc = check_device())
        return rc;
    ChainScope chain;
    return run_expert_ffn(x, offsets, src_row, prepacked, T, k, E, H, I, y_perm, workspace, true,
                          (cudaStream_t)stream);
}

extern "C" MXMOE_API int mxmoe_ffn_gate_up(const void *x, const int32_t *offsets, const int32_t *src_row,
                                           const void *prepacked, int T, int k, int E, int H, int I, void *workspace,
                                           int64_t workspace_bytes, void *stream)
{
    if (int rc = check_ffn_args("mxmoe_ffn_gate_up", T, k, E, H, I, workspace, workspace_bytes))
        return rc;
    if (T == 0)
        return MXMOE_OK;
    if (!x || !offsets || !src_row || !prepacked)
        return fail(MXMOE_ERR_NULL, "mxmoe_ffn_gate_up: NULL pointer");
    if (!aligned16(x) || !aligned32(prepacked))
        return fail(MXMOE_ERR_ALIGNMENT, "mxmoe_ffn_gate_up: x needs 16-byte, prepacked 32-byte alignment");
    if (int rc = check_device())
        return rc;
    ChainScope chain;
    return run_ffn_gate_up(x, offsets, src_row, prepacked, T, k, E, H, I, workspace, true, (cudaStream_t)stream);
}

extern "C" MXMOE_API int mxmoe_ffn_down(const int32_t *offsets, const void *prepacked, int T, int k, int E, int H,
                                        int I, float *y_perm, void *workspace, int64_t workspace_bytes, void *stream)
{
    if (int rc = check_ffn_args("mxmoe_ffn_down", T, k, E, H, I, workspace, workspace_bytes))
        return rc;
    if (T == 0)
        return MXMOE_OK;
    if (!offsets || !prepacked || !y_perm)
        return fail(MXMOE_ERR_NULL, "mxmoe_ffn_down: NULL pointer");
    if (!aligned32(prepacked) || !aligned16(y_perm))
        return fail(MXMOE_ERR_ALIGNMENT, "mxmoe_ffn_down: prepacked needs 32-byte, y_perm 16-byte alignment");
    if (int rc = check_device())
        return rc;
    ChainScope chain;
    return run_ffn_down(offsets, prepacked, T, k, E, H, I, y_perm, workspace, (cudaStream_t)stream);
}

extern "C" MXMOE_API int mxmoe_combine(const float *y_perm, const int32_t *dst_of, const float *w, int T, int k,
                                       int H, float *y, void *stream)
{
    if (T < 0 || T > 65535 || k < 1 || H <= 0 || H % 4)
        return fail(MXMOE_ERR_INVALID_SHAPE,
                    "mxmoe_combine: T=%d k=%d H=%d (H must be a multiple of 4, T at most 65535)", T, k, H);
    if (T == 0)
        return MXMOE_OK;
    if (!y_perm || !dst_of || !w || !y)
        return fail(MXMOE_ERR_NULL, "mxmoe_combine: NULL pointer");
    if (!aligned16(y_perm) || !aligned16(y))
        return fail(MXMOE_ERR_ALIGNMENT, "mxmoe_combine: y_perm and y must be 16-byte aligned");
    if (int rc = check_device())
        return rc;
    return run_combine(y_perm, dst_of, w, T, k, H, y, (cudaStream_t)stream);
}

extern "C" MXMOE_API int64_t mxmoe_ffn_workspace_size_fp8(int T, int k, int E, int H, int I)
{
    if (!ffn_shapes_ok(T, k, E, H, I))
        return -1;
    return ffn_workspace_bytes_fp8(T, k, E, H, I);
}

extern "C" MXMOE_API int mxmoe_expert_ffn_fp8(const void *x, const int32_t *offsets, const int32_t *src_row,
                                              const void *prepacked, int T, int k, int E, int H, int I, float *y_perm,
                                              void *workspace, int64_t workspace_bytes, void *stream)
{
    if (int rc = check_ffn_args("mxmoe_expert_ffn_fp8", T, k, E, H, I, workspace, workspace_bytes, true))
        return rc;
    if (T == 0)
        return MXMOE_OK;
    if (!x || !offsets || !src_row || !prepacked || !y_perm)
        return fail(MXMOE_ERR_NULL, "mxmoe_expert_ffn_fp8: NULL pointer");
    if (!aligned16(x) || !aligned32(prepacked) || !aligned16(y_perm))
        return fail(MXMOE_ERR_ALIGNMENT,
                    "mxmoe_expert_ffn_fp8: x and y_perm need 16-byte, prepacked 32-byte alignment");
    if (int rc = check_device())
        return rc;
    ChainScope chain;
    return run_expert_ffn_fp8(x, offsets, src_row, prepacked, T, k, E, H, I, y_perm, workspace, true,
                              (cudaStream_t)stream);
}
