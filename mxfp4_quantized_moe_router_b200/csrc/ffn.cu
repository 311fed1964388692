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
//    tcgen05.mma.kind::mxf8f6f4.block_scale multiplies E2M1 weight codes by
//    E4M3 activation codes and applies both operands' UE8M0 scales per 32
//    elements of K in hardware, accumulating in fp32 in tensor memory. No
//    instruction touches a weight element.
//  * Weight tiles (128 rows x 128 K, one contiguous 8 KB box of the
//    prepacked blob) arrive by TMA with the fp4 unpack (16U4_ALIGN16B), their
//    scale images (512 B) by a bulk copy, and the scale images move into
//    tensor memory by tcgen05.cp.
//  * Activations are exact sums of E4M3 terms with one power-of-two scale per
//    32 values: x (bf16) = 2 terms, exact for every element within 2^-14 of
//    its block maximum; h (fp32) = 3 terms, about 12 significant bits. The
//    terms are stacked along N (term t of token n is B row t*NT + n), so one
//    MMA per 32 values of K covers all of them and the epilogue adds the term
//    columns.
//  * Activations are stored in grouped (expert-sorted) row order, so a token
//    pass of an expert is a contiguous row range: one 3-D TMA box per K step
//    brings all of its terms.
//  * Warp roles per CTA: a producer warp (TMA and bulk copies into an S-stage
//    ring), an MMA warp (tcgen05.cp of the scale images, the MMAs, commits),
//    four epilogue warps reading the fp32 accumulators from tensor memory
//    (two accumulator buffers, so item i's epilogue overlaps item i+1's MMAs;
//    within an item the k32 blocks rotate over independent accumulators so
//    the short MMAs of decode-sized N do not serialise on one accumulator).
//  * Stage 1 (gate/up): a 128-row tile is 64 gate rows and the 64 matching up
//    rows, interleaved by 16 so gate and up of one column meet in one warp;
//    SwiGLU and the 3-term encoding of h are fused into the epilogue.
//    Stage 2 (down): a tile is 128 output rows.
//  * Work items (expert, tile, token pass) are split contiguously over a
//    persistent grid of one CTA per SM.
#include <float.h>

#include <algorithm>
#include <mutex>

#include <cudaTypedefs.h>

#include "common.cuh"
#include "tcgen05.cuh"

namespace mxmoe {
namespace {

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bounded waits: 2 s
constexpr int kKC = 128;            // K per chunk (one 128 x 128 fp4 box of the prepacked blob)
constexpr int kChunkSmem = 16384;   // shared-memory bytes of an unpacked chunk box
constexpr int kChunkTx = 8192;      // TMA transaction bytes of a chunk box (its packed size)
constexpr int kSFImg = 512;         // scale image: 32 lanes x 16 bytes
constexpr int kThreads = 192;       // producer, MMA, 4 epilogue warps

struct FfnParams {
    int tiles_per_expert;     // 2I/128 (gate/up) or H/128 (down)
    int K;                    // reduction length (H or I)
    int rows_act;             // rows of the activation term tensors (T*k)
    const uint8_t *sfa;       // weight scale images [E*tiles][K/128][512]
    const int32_t *offsets;   // [E+1]
    int E;
    uint8_t *h_terms;         // gate/up output: terms of h (term_offset layout)
    uint8_t *h_rec;           // gate/up output: their scale records (rec_offset layout)
    int I;
    float *y_out;             // down output: [rows, H]
    int H;
    int *status;
};

// Byte offset of term t of activation row r, column k, in a term tensor laid
// out [K/128][nterms][rows][128]: the terms of one 128-column chunk of a token
// pass are nterms runs of consecutive 128-byte rows.
__host__ __device__ __forceinline__ int64_t term_offset(int nterms, int64_t rows, int t, int64_t r, int k)
{
    return (((int64_t)(k >> 7) * nterms + t) * rows + r) * 128 + (k & 127);
}

// Byte offset of the UE8M0 scale of term t, row r, for the 32-block holding
// column k, in a scale-record array of 16-byte records. With 8-token passes
// (per_term) a record holds one term of one chunk (byte = k32 block), planes
// chunk * nterms + t: the records of a pass and chunk then form that chunk's
// B scale image, image row t * 8 + n. With 32-token passes a record holds all
// terms of one chunk (byte 4t + k32 block), planes = chunks: image row n then
// serves the stacked rows t * 32 + n through its t-th 32-bit column.
__host__ __device__ __forceinline__ int64_t rec_offset(bool per_term, int nterms, int64_t rows, int t, int64_t r,
                                                       int k)
{
    const int c = k >> 7, kb = (k >> 5) & 3;
    if (per_term)
        return (((int64_t)c * nterms + t) * rows + r) * 16 + kb;
    return ((int64_t)c * rows + r) * 16 + 4 * t + kb;
}

__host__ __device__ __forceinline__ int64_t rec_planes(bool per_term, int nterms, int K)
{
    return per_term ? (int64_t)(K / kKC) * nterms : K / kKC;
}

template <int NT, int NTERMS>
struct Cfg {
    static constexpr bool kPerTerm = NT <= 8;
    static constexpr int kCPS = NT <= 8 ? 4 : 2;  // chunks per stage (one weight TMA request)
    // Weight ring (codes + scale images, from HBM) and activation ring (terms +
    // scale records, L2-resident), advanced together once per stage.
    static constexpr int kStagesA = NT <= 8 ? 3 : (NTERMS == 2 ? 5 : 4);
    static constexpr int kStagesB = NT <= 8 ? 2 : 3;
    static constexpr int kAStage = kCPS * kChunkSmem;
    static constexpr int kATx = kCPS * kChunkTx;
    static constexpr int kSfaStage = kCPS * kSFImg;
    static constexpr int kBChunk = NTERMS * NT * 128;  // one chunk's terms, rows t*NT + n
    static constexpr int kBStage = kCPS * kBChunk;
    static constexpr int kSfbZ = kPerTerm ? NTERMS * kCPS : kCPS;  // record planes per stage
    static constexpr int kSfbTx = 16 * NT * kSfbZ;
    static constexpr int kSfbImg = kSfbTx / kCPS;  // one chunk's B scale image
    // a 32-lane tcgen05.cp of the last image reads up to 512 bytes
    static constexpr int kSfbStage = kSfbTx + (kSfbImg < kSFImg ? kSFImg - kSfbImg : 0);
    static constexpr int kN = NTERMS * NT;  // MMA N: the stacked terms
    static constexpr int kXchg = 8 * NT;    // [pair][parity][quarter][NT] block maxima
    // shared memory: A stages | B stages | A scale images | B scale images | xchg | barriers | tslot, cursor
    static constexpr size_t kOffB = (size_t)kStagesA * kAStage;
    static constexpr size_t kOffSfa = kOffB + (size_t)kStagesB * kBStage;
    static constexpr size_t kOffSfb = kOffSfa + (size_t)kStagesA * kSfaStage;
    static constexpr size_t kOffXchg = kOffSfb + (size_t)kStagesB * kSfbStage;
    static constexpr size_t kOffBar = (kOffXchg + kXchg * 4 + 127) & ~size_t(127);
    static constexpr int kBars = 2 * kStagesA + 2 * kStagesB + 5;
    static constexpr size_t kOffMisc = (kOffBar + kBars * 8 + 15) & ~size_t(15);
    static constexpr size_t kSmem = 1024 + kOffMisc + 64;
    // Tensor memory: two accumulator buffers (item i and i+1), each holding
    // kChains independent accumulators of kN columns (32-column aligned): the
    // k32 blocks of an item rotate over the chains so that consecutive small-N
    // MMAs do not wait on each other. Then the scale columns: per stage and
    // chunk one group of 4 for A and one for B. An MMA's scale address must be
    // a group base (a multiple of 4 columns).
    static constexpr int kChains = NT <= 8 ? 4 : 2;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kAccStride = (kN + 31) & ~31;
    static constexpr uint32_t kBufCols = kChains * kAccStride;
    static constexpr uint32_t kSfaCol0 = 2 * kBufCols;
    static constexpr uint32_t kSfaCols = 4 * kCPS;
    static constexpr uint32_t kSfbCol0 = kSfaCol0 + kStagesA * kSfaCols;
    static constexpr uint32_t kSfbCols = 4 * kCPS;
    static_assert(NT <= 32 && NTERMS <= 3 && kN <= 256 && kN % 8 == 0, "MMA shape");
    static_assert(!kPerTerm || kN <= 32, "a per-term B scale image has at most 32 rows");
    static_assert(kSfbStage % 128 == 0 && kSfbImg % 16 == 0, "scale image alignment");
    static_assert(kSfbCol0 + kStagesB * kSfbCols <= kTmemCols, "tensor memory columns");
    static_assert(kAStage % 1024 == 0 && kBChunk % 1024 == 0 && kOffB % 1024 == 0, "128-byte swizzle atoms");
    static_assert(kSmem <= 232448, "shared memory");
};

// Work items of one FFN stage: (expert, weight tile, token pass), expert-major,
// then tile, then pass, so that the passes of one weight tile are adjacent
// (the repeated weight boxes then come from L2). A CTA takes a contiguous
// range of items and every role walks it with its own cursor.
template <int NT>
struct ItemCursor {
    const int32_t *offsets;
    int E, tiles;
    int e, tile, pass, npass, base, n_e;

    __device__ __forceinline__ void load_expert()
    {
        base = offsets[e];
        n_e = offsets[e + 1] - base;
        npass = (n_e + NT - 1) / NT;
    }
    __device__ __forceinline__ void start(const int32_t *off, int E_, int tiles_, int e0, int local)
    {
        offsets = off;
        E = E_;
        tiles = tiles_;
        e = e0;
        if (e >= E)
            return;
        load_expert();
        tile = npass ? local / npass : 0;
        pass = npass ? local % npass : 0;
    }
    __device__ __forceinline__ void next()
    {
        if (++pass < npass)
            return;
        pass = 0;
        if (++tile < tiles)
            return;
        tile = 0;
        do {
            ++e;
            if (e >= E)
                return;
            load_expert();
        } while (npass == 0);
    }
    __device__ __forceinline__ int r0() const { return base + pass * NT; }
    __device__ __forceinline__ int nt() const { return min(NT, n_e - pass * NT); }
};

// Activation value v (already divided by its block's 2^s, |v| < 256) as
// NTERMS E4M3 codes c_t with v ~= sum_t c_t * 16^-t (exact for 8-bit v).
template <int NTERMS>
__device__ __forceinline__ void split_terms(float v, uint32_t (&code)[NTERMS])
{
    float r = v;
#pragma unroll
    for (int t = 0; t < NTERMS; ++t) {
        code[t] = tc::f32_to_e4m3(r);
        r = (r - tc::e4m3_to_f32(code[t])) * 16.f;
    }
}

// Scale exponent s of a 32-value activation block with maximum m: m / 2^s
// lands in [128, 256); clamped so that every term's scale byte s - 4t + 127
// stays in [0, 254].
__device__ __forceinline__ int act_block_exp(float m)
{
    const int s = m > 0.f ? tc::floor_log2(m) - 7 : 0;
    return max(-119, min(s, 127));
}

// One FFN stage over all experts.
// GATE_UP = true: stage 1 (x terms in; h terms and records out).
// GATE_UP = false: stage 2 (h terms in; float rows out).
template <int NT, int NTERMS, bool GATE_UP>
__global__ void __launch_bounds__(kThreads, 1)
    ffn_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmSfb, const FfnParams p)
{
    using C = Cfg<NT, NTERMS>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem, *sB = smem + C::kOffB, *sSfa = smem + C::kOffSfa, *sSfb = smem + C::kOffSfb;
    float *xchg = reinterpret_cast<float *>(smem + C::kOffXchg);
    uint64_t *fullA = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
    uint64_t *emptyA = fullA + C::kStagesA;
    uint64_t *fullB = emptyA + C::kStagesA;
    uint64_t *emptyB = fullB + C::kStagesB;
    uint64_t *accfull = emptyB + C::kStagesB;  // [2]
    uint64_t *accempty = accfull + 2;          // [2]
    uint64_t *mma_done = accempty + 2;         // [1]
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + C::kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);
    int *cur = reinterpret_cast<int *>(tslot + 2);  // [0] first expert, [1] first item within it, [2] item count

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int E = p.E, tiles = p.tiles_per_expert;

    if (warp == 0) {
        // Items of expert e: tiles * ceil(n_e / NT). Pass 1 counts them all;
        // pass 2 finds the expert holding this CTA's first item.
        int64_t total = 0;
        for (int b = 0; b < E; b += 32) {
            const int e = b + lane;
            const int n_e = e < E ? p.offsets[e + 1] - p.offsets[e] : 0;
            int64_t c = (int64_t)tiles * ((n_e + NT - 1) / NT);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                c += __shfl_xor_sync(0xFFFFFFFFu, c, off);
            total += c;
        }
        const int64_t i_begin = total * blockIdx.x / gridDim.x;
        const int64_t i_end = total * (blockIdx.x + 1) / gridDim.x;
        if (lane == 0) {
            cur[0] = E;
            cur[1] = 0;
            cur[2] = (int)(i_end - i_begin);
        }
        __syncwarp();
        int64_t carry = 0;
        for (int b = 0; b < E && i_end > i_begin; b += 32) {
            const int e = b + lane;
            const int n_e = e < E ? p.offsets[e + 1] - p.offsets[e] : 0;
            const int64_t c = (int64_t)tiles * ((n_e + NT - 1) / NT);
            int64_t incl = c;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int64_t o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
                if (lane >= off)
                    incl += o;
            }
            const int64_t excl = carry + incl - c;
            if (c > 0 && excl <= i_begin && i_begin < excl + c) {
                cur[0] = e;
                cur[1] = (int)(i_begin - excl);
            }
            carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
    }
    if (tid == 32) {
        for (int s = 0; s < C::kStagesA; ++s) {
            mbar_init(&fullA[s], 1);
            mbar_init(&emptyA[s], 1);
        }
        for (int s = 0; s < C::kStagesB; ++s) {
            mbar_init(&fullB[s], 1);
            mbar_init(&emptyB[s], 1);
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
        tc::alloc(tslot, C::kTmemCols);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *tslot;
    const int n_items = cur[2];
    ItemCursor<NT> it;
    it.start(p.offsets, E, tiles, cur[0], cur[1]);
    const int nchunk = p.K / kKC;
    const int nstage = (nchunk + C::kCPS - 1) / C::kCPS;

    if (warp == 0) {
        // ----------------------------------------------------------- producer
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_first();
            const uint64_t pol_a = policy_evict_last();
            int sa = 0, sb = 0;
            uint32_t pha = 0, phb = 0;
            int64_t issued_a = 0, issued_b = 0;
            bool ok = true;
            for (int i = 0; i < n_items && ok; ++i, it.next()) {
                const int64_t box0 = ((int64_t)it.e * tiles + it.tile) * nchunk;
                const int r0 = it.r0();
                for (int st = 0; st < nstage; ++st) {
                    const int c0 = st * C::kCPS, nc = min(C::kCPS, nchunk - c0);
                    if (*abort_flag || !mbar_wait_bounded(&emptyA[sa], pha ^ 1u, kWaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&fullA[sa], (uint32_t)(C::kATx + nc * kSFImg));
                    tc::tma_load_3d(sA + (size_t)sa * C::kAStage, &tmA, 0, 0, (int)(box0 + c0), &fullA[sa], pol_w);
                    bulk_g2s_hint(sSfa + sa * C::kSfaStage, p.sfa + (box0 + c0) * kSFImg, (uint32_t)(nc * kSFImg),
                                  &fullA[sa], pol_w);
                    ++issued_a;
                    if (*abort_flag || !mbar_wait_bounded(&emptyB[sb], phb ^ 1u, kWaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&fullB[sb], (uint32_t)(C::kBStage + C::kSfbTx));
                    tc::tma_load_4d(sB + (size_t)sb * C::kBStage, &tmB, 0, r0, 0, c0, &fullB[sb], pol_a);
                    tc::tma_load_3d(sSfb + sb * C::kSfbStage, &tmSfb, 0, r0, C::kPerTerm ? c0 * NTERMS : c0,
                                    &fullB[sb], pol_a);
                    ++issued_b;
                    if (++sa == C::kStagesA) {
                        sa = 0;
                        pha ^= 1u;
                    }
                    if (++sb == C::kStagesB) {
                        sb = 0;
                        phb ^= 1u;
                    }
                }
            }
            if (!ok) {
                set_status(p.status, MXMOE_ERR_TIMEOUT);
                *abort_flag = 1;
            }
            // Drain: no copy of ours may still be landing when the CTA ends.
            for (int64_t f = issued_a > C::kStagesA ? issued_a - C::kStagesA : 0; f < issued_a; ++f)
                if (!mbar_wait_bounded(&fullA[f % C::kStagesA], (uint32_t)((f / C::kStagesA) & 1), kWaitLimitNs)) {
                    set_status(p.status, MXMOE_ERR_TIMEOUT);
                    break;
                }
            for (int64_t f = issued_b > C::kStagesB ? issued_b - C::kStagesB : 0; f < issued_b; ++f)
                if (!mbar_wait_bounded(&fullB[f % C::kStagesB], (uint32_t)((f / C::kStagesB) & 1), kWaitLimitNs)) {
                    set_status(p.status, MXMOE_ERR_TIMEOUT);
                    break;
                }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA
        if (lane == 0) {
            int sa = 0, sb = 0;
            uint32_t pha = 0, phb = 0;
            bool ok = true, any = false;
            for (int i = 0; i < n_items && ok; ++i) {
                const int buf = i & 1;
                const uint32_t use = (uint32_t)(i >> 1);
                if (*abort_flag || !mbar_wait_bounded(&accempty[buf], (use & 1u) ^ 1u, kWaitLimitNs)) {
                    ok = false;
                    break;
                }
                tc::fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)buf * C::kBufCols;
                for (int st = 0; st < nstage; ++st) {
                    const int nc = min(C::kCPS, nchunk - st * C::kCPS);
                    if (*abort_flag || !mbar_wait_bounded(&fullA[sa], pha, kWaitLimitNs) ||
                        !mbar_wait_bounded(&fullB[sb], phb, kWaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    tc::fence_after();
                    const uint32_t sfa_t = tmem + C::kSfaCol0 + C::kSfaCols * sa;
                    const uint32_t sfb_t = tmem + C::kSfbCol0 + C::kSfbCols * sb;
                    const uint32_t a_base = smem_u32(sA + (size_t)sa * C::kAStage);
                    const uint32_t b_base = smem_u32(sB + (size_t)sb * C::kBStage);
                    const uint32_t sfa_s = smem_u32(sSfa + sa * C::kSfaStage);
                    const uint32_t sfb_s = smem_u32(sSfb + sb * C::kSfbStage);
                    for (int j = 0; j < nc; ++j)
                        tc::cp_32x128b_warpx4(sfa_t + 4 * j, tc::smem_desc(sfa_s + j * kSFImg, 16, 128, 0));
                    for (int j = 0; j < nc; ++j)
                        tc::cp_32x128b_warpx4(sfb_t + 4 * j, tc::smem_desc(sfb_s + j * C::kSfbImg, 16, 128, 0));
                    for (int j = 0; j < nc; ++j) {
                        const uint32_t sfa_j = sfa_t + 4 * j;
                        const uint32_t sfb_j = sfb_t + 4 * j;
#pragma unroll
                        for (int kb = 0; kb < 4; ++kb) {
                            const uint64_t adesc =
                                tc::smem_desc(a_base + j * kChunkSmem + kb * 32, 16, 1024, 2);
                            const uint64_t bdesc = tc::smem_desc(b_base + j * C::kBChunk + kb * 32, 16, 1024, 2);
                            const uint32_t idesc = tc::idesc_e2m1_e4m3(C::kN, (uint32_t)kb);
                            const int step = 4 * j + kb;
                            const int chain = step % C::kChains;
                            tc::mma_mxf8f6f4(d_tmem + (uint32_t)chain * C::kAccStride, adesc, bdesc, idesc,
                                             (st > 0 || step >= C::kChains) ? 1u : 0u, sfa_j | ((uint32_t)kb << 30),
                                             sfb_j | ((uint32_t)kb << 30));
                        }
                    }
                    tc::commit(&emptyA[sa]);  // frees both stages once these MMAs are done
                    tc::commit(&emptyB[sb]);
                    any = true;
                    if (++sa == C::kStagesA) {
                        sa = 0;
                        pha ^= 1u;
                    }
                    if (++sb == C::kStagesB) {
                        sb = 0;
                        phb ^= 1u;
                    }
                }
                if (ok)
                    tc::commit(&accfull[buf]);
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
    } else {
        // ----------------------------------------------------------- epilogue
        // A warp that gives up on a wait stops reading tensor memory and writing
        // outputs but keeps taking part in the pair barriers.
        const int q = warp & 3;  // tensor-memory lane quarter: rows 32q .. 32q+31
        const int pair = q >> 1;
        bool aborted = false;
        for (int i = 0; i < n_items; ++i, it.next()) {
            const int buf = i & 1;
            const uint32_t use = (uint32_t)(i >> 1);
            const int r0 = it.r0(), ntile = it.nt();
            if (!aborted && (*abort_flag || !mbar_wait_bounded(&accfull[buf], use & 1u, kWaitLimitNs))) {
                if (lane == 0) {
                    set_status(p.status, MXMOE_ERR_TIMEOUT);
                    *abort_flag = 1;
                }
                aborted = true;
            }
            tc::fence_after();
            float acc[NT];
#pragma unroll
            for (int j0 = 0; j0 < NT; j0 += 8) {
                float v8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                if (!aborted && j0 < ntile) {
                    // chains, then term columns t*NT + n, added in that order
#pragma unroll
                    for (int a = 0; a < C::kChains; ++a)
#pragma unroll
                        for (int t = 0; t < NTERMS; ++t) {
                            float w8[8];
                            tc::ld_32x32b_x8(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)buf * C::kBufCols +
                                                 (uint32_t)(a * C::kAccStride + t * NT + j0),
                                             w8);
#pragma unroll
                            for (int k = 0; k < 8; ++k)
                                v8[k] = (a | t) ? v8[k] + w8[k] : w8[k];
                        }
                }
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    acc[j0 + k] = v8[k];
            }
            tc::fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&accempty[buf]);
            if (GATE_UP) {
                // lanes 0..15 hold gate column col, lanes 16..31 the up column col
                const int col = 64 * it.tile + 16 * q + (lane & 15);
                float *xb = xchg + (pair * 2 + (i & 1)) * 2 * NT;
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    const float g = acc[n];
                    const float u = __shfl_down_sync(0xFFFFFFFFu, g, 16);
                    const float h = (n < ntile) ? g / (1.f + expf(-g)) * u : 0.f;
                    float m = (lane < 16) ? fabsf(h) : 0.f;
#pragma unroll
                    for (int off = 8; off > 0; off >>= 1)
                        m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
                    acc[n] = h;
                    if (lane == 0)
                        xb[(q & 1) * NT + n] = m;  // this quarter's half-block maximum
                }
                named_bar_sync(2 + pair, 64);
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    if (aborted || n >= ntile)
                        continue;
                    const float bm = fmaxf(xb[n], xb[NT + n]);
                    const int s = act_block_exp(bm);
                    const float inv = __uint_as_float((uint32_t)(127 - s) << 23);  // 2^-s
                    const int r = r0 + n;
                    if (lane < 16) {
                        uint32_t code[3];
                        split_terms<3>(acc[n] * inv, code);
#pragma unroll
                        for (int t = 0; t < 3; ++t)
                            p.h_terms[term_offset(3, p.rows_act, t, r, col)] = (uint8_t)code[t];
                    }
                    if (lane == 0 && !(q & 1)) {
#pragma unroll
                        for (int t = 0; t < 3; ++t)
                            p.h_rec[rec_offset(C::kPerTerm, 3, p.rows_act, t, r, col)] = (uint8_t)(s - 4 * t + 127);
                    }
                }
            } else if (!aborted) {
                float *yrow = p.y_out + (int64_t)r0 * p.H + 128 * it.tile + 32 * q + lane;
#pragma unroll
                for (int n = 0; n < NT; ++n)
                    if (n < ntile)
                        yrow[(int64_t)n * p.H] = acc[n];
            }
        }
    }
    tc::fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after();
        tc::dealloc(tmem, C::kTmemCols);
    }
}

// x rows (bf16) -> 2 E4M3 terms per value in grouped row order (row r holds
// token src_row[r] / k), in the term_offset layout, and their UE8M0 scales per
// 32-value block in the rec_offset layout. One warp per 32-value block.
// Block 0 also clears the status word.
__global__ void __launch_bounds__(256) x_terms_kernel(const uint16_t *__restrict__ x, const int32_t *__restrict__ src_row,
                                                      int k, int rows, int H, uint8_t *__restrict__ terms,
                                                      uint8_t *__restrict__ rec, bool per_term, int *status)
{
    if (blockIdx.x == 0 && threadIdx.x == 0 && status)
        *status = 0;
    const int lane = threadIdx.x & 31;
    const int nkb = H / 32;
    const int64_t total = (int64_t)rows * nkb;
    for (int64_t w = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); w < total; w += (int64_t)gridDim.x * 8) {
        const int r = (int)(w / nkb), kb = (int)(w % nkb);
        const int tok = src_row[r] / k;
        const int col = kb * 32 + lane;
        const float v = __uint_as_float((uint32_t)x[(int64_t)tok * H + col] << 16);
        float m = fabsf(v);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
        const int s = act_block_exp(m);
        const float inv = __uint_as_float((uint32_t)(127 - s) << 23);
        uint32_t code[2];
        split_terms<2>(v * inv, code);
        terms[term_offset(2, rows, 0, r, col)] = (uint8_t)code[0];
        terms[term_offset(2, rows, 1, r, col)] = (uint8_t)code[1];
        if (lane == 0) {
            rec[rec_offset(per_term, 2, rows, 0, r, col)] = (uint8_t)(s + 127);
            rec[rec_offset(per_term, 2, rows, 1, r, col)] = (uint8_t)(s - 4 + 127);
        }
    }
}

// y[t, c] = sum_j w[t, j] * y_perm[dst_of[t*k + j], c], j in order.
__global__ void __launch_bounds__(256) combine_kernel(const float *__restrict__ y_perm,
                                                      const int32_t *__restrict__ dst_of,
                                                      const float *__restrict__ w, int T, int k, int H,
                                                      float *__restrict__ y)
{
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
// Host side
// ---------------------------------------------------------------------------
struct FfnWs {
    int *status;
    uint8_t *x_terms;  // [H/128][2][rows][128]
    uint8_t *x_rec;    // records (rec_offset layout)
    uint8_t *h_terms;  // [I/128][3][rows][128]
    uint8_t *h_rec;    // records (rec_offset layout)
};

int64_t ffn_ws_layout(int T, int k, int H, int I, FfnWs *ws, void *base)
{
    int64_t off = 0;
    auto take = [&](int64_t bytes) {
        int64_t o = off;
        off = align256(off + bytes);
        return o;
    };
    const int64_t rows = (int64_t)T * k;
    // record planes for either record layout
    const int64_t xr_planes = std::max(rec_planes(true, 2, H), rec_planes(false, 2, H));
    const int64_t hr_planes = std::max(rec_planes(true, 3, I), rec_planes(false, 3, I));
    const int64_t o_status = take(16);
    const int64_t o_xt = take(2 * rows * H);
    const int64_t o_xr = take(xr_planes * rows * 16);
    const int64_t o_ht = take(3 * rows * I);
    const int64_t o_hr = take(hr_planes * rows * 16);
    if (ws && base) {
        uint8_t *b = static_cast<uint8_t *>(base);
        ws->status = reinterpret_cast<int *>(b + o_status);
        ws->x_terms = b + o_xt;
        ws->x_rec = b + o_xr;
        ws->h_terms = b + o_ht;
        ws->h_rec = b + o_hr;
    }
    return off;
}

int num_sms()
{
    static thread_local int cached_dev = -1, cached = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev != cached_dev) {
        cudaDeviceGetAttribute(&cached, cudaDevAttrMultiProcessorCount, dev);
        cached_dev = dev;
    }
    return cached > 0 ? cached : 148;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void *ptr = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

int encode(CUtensorMap *m, CUtensorMapDataType type, int rank, const void *base, const cuuint64_t *dims,
           const cuuint64_t *strides, const cuuint32_t *box, CUtensorMapSwizzle swizzle, CUtensorMapL2promotion promo,
           const char *what)
{
    auto enc = tensor_map_encoder();
    if (!enc)
        return fail(MXMOE_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const cuuint32_t es[5] = {1, 1, 1, 1, 1};
    CUresult r = enc(m, type, (cuuint32_t)rank, const_cast<void *>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(MXMOE_ERR_CUDA, "cuTensorMapEncodeTiled (%s) failed: %d", what, (int)r);
    return MXMOE_OK;
}

// The code boxes of one weight matrix (all experts): n_boxes boxes of 128
// rows x 128 fp4 codes (64 bytes a row, 8 KB a box), read `cps` consecutive
// boxes per request, each unpacked into one 16-byte slot per 16 codes with the
// 128-byte swizzle. Boxes past the end read as zero.
int encode_weights(CUtensorMap *m, const void *base, int64_t n_boxes, int cps)
{
    const cuuint64_t dims[3] = {128, 128, (cuuint64_t)n_boxes};
    const cuuint64_t strides[2] = {64, kChunkTx};
    const cuuint32_t box[3] = {128, 128, (cuuint32_t)cps};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, "weights");
}

// Activation terms in the term_offset layout, dims {128, rows, nterms,
// chunks}; a request brings nt rows x all terms x cps chunks. Rows and chunks
// past the end read as zero.
int encode_terms(CUtensorMap *m, const void *base, int64_t rows, int K, int nterms, int nt, int cps)
{
    const cuuint64_t dims[4] = {128, (cuuint64_t)rows, (cuuint64_t)nterms, (cuuint64_t)(K / kKC)};
    const cuuint64_t strides[3] = {128, (cuuint64_t)(rows * 128), (cuuint64_t)(rows * 128 * nterms)};
    const cuuint32_t box[4] = {128, (cuuint32_t)nt, (cuuint32_t)nterms, (cuuint32_t)cps};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_128B, "activation terms");
}

// Scale records (rec_offset layout), dims {16, rows, planes}; a request brings
// nt rows x z planes.
int encode_records(CUtensorMap *m, const void *base, int64_t rows, int64_t planes, int nt, int z)
{
    const cuuint64_t dims[3] = {16, (cuuint64_t)rows, (cuuint64_t)planes};
    const cuuint64_t strides[2] = {16, (cuuint64_t)(rows * 16)};
    const cuuint32_t box[3] = {16, (cuuint32_t)nt, (cuuint32_t)z};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, "activation scale records");
}

template <int NT, int NTERMS, bool GATE_UP>
int launch_ffn(const void *codes, const uint8_t *act_terms, const uint8_t *act_rec, FfnParams p, cudaStream_t st)
{
    using C = Cfg<NT, NTERMS>;
    static thread_local int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        if (cudaFuncSetAttribute(ffn_tc_kernel<NT, NTERMS, GATE_UP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)C::kSmem) != cudaSuccess)
            return fail(MXMOE_ERR_CUDA, "ffn_tc_kernel: cannot reserve %zu bytes of shared memory", C::kSmem);
        configured_dev = dev;
    }
    const int64_t n_boxes = (int64_t)p.E * p.tiles_per_expert * (p.K / kKC);
    CUtensorMap tmA, tmB, tmSfb;
    if (int rc = encode_weights(&tmA, codes, n_boxes, C::kCPS))
        return rc;
    if (int rc = encode_terms(&tmB, act_terms, p.rows_act, p.K, NTERMS, NT, C::kCPS))
        return rc;
    if (int rc = encode_records(&tmSfb, act_rec, p.rows_act, rec_planes(C::kPerTerm, NTERMS, p.K), NT, C::kSfbZ))
        return rc;
    ffn_tc_kernel<NT, NTERMS, GATE_UP><<<num_sms(), kThreads, C::kSmem, st>>>(tmA, tmB, tmSfb, p);
    return check_launch(GATE_UP ? "ffn_tc_kernel<gate_up>" : "ffn_tc_kernel<down>");
}

// Token rows per pass: 8 while the mean rows per expert is at most 8 (decode
// and verify blocks), else 32.
int token_tile(int T, int k, int E) { return (int64_t)T * k <= 8LL * E ? 8 : 32; }

int validate_ffn(int T, int k, int E, int H, int I)
{
    if (T < 0 || k < 1 || k > 32 || E <= 0 || E > 1024 || H <= 0 || I <= 0 || H % 128 || I % 128 || H > 32768 ||
        I > 32768 || (int64_t)T * k > (1 << 22))
        return fail(MXMOE_ERR_INVALID_SHAPE,
                    "expert FFN: T=%d k=%d E=%d H=%d I=%d (need H, I multiples of 128 up to 32768, 1 <= k <= 32, "
                    "E <= 1024, T*k <= 2^22)",
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
    o.w2 = o.w13 + (int64_t)E * 2 * I * (H / 2);
    o.sf13 = o.w2 + (int64_t)E * H * (I / 2);
    o.sf2 = o.sf13 + (int64_t)E * 2 * I * (H / 32);
    return o;
}

}  // namespace

int run_ffn_gate_up(const void *x, const int32_t *offsets, const int32_t *src_row, const void *prepacked, int T,
                    int k, int E, int H, int I, void *workspace, cudaStream_t st)
{
    FfnWs ws;
    ffn_ws_layout(T, k, H, I, &ws, workspace);
    const int rows = T * k;
    const int nt = token_tile(T, k, E);
    {
        const int64_t warps = (int64_t)rows * (H / 32);
        const int blocks = (int)std::min<int64_t>((warps + 7) / 8, (int64_t)num_sms() * 16);
        x_terms_kernel<<<blocks < 1 ? 1 : blocks, 256, 0, st>>>(static_cast<const uint16_t *>(x), src_row, k, rows,
                                                                 H, ws.x_terms, ws.x_rec, nt <= 8, ws.status);
        if (int rc = check_launch("x_terms_kernel"))
            return rc;
    }
    const Blob bl = blob_parts(prepacked, E, H, I);
    FfnParams p{};
    p.tiles_per_expert = 2 * I / 128;
    p.K = H;
    p.rows_act = rows;
    p.sfa = bl.sf13;
    p.offsets = offsets;
    p.E = E;
    p.h_terms = ws.h_terms;
    p.h_rec = ws.h_rec;
    p.I = I;
    p.y_out = nullptr;
    p.H = H;
    p.status = ws.status;
    if (nt == 8)
        return launch_ffn<8, 2, true>(bl.w13, ws.x_terms, ws.x_rec, p, st);
    return launch_ffn<32, 2, true>(bl.w13, ws.x_terms, ws.x_rec, p, st);
}

int run_ffn_down(const int32_t *offsets, const void *prepacked, int T, int k, int E, int H, int I, float *y_perm,
                 void *workspace, cudaStream_t st)
{
    FfnWs ws;
    ffn_ws_layout(T, k, H, I, &ws, workspace);
    const int rows = T * k;
    const int nt = token_tile(T, k, E);
    const Blob bl = blob_parts(prepacked, E, H, I);
    FfnParams p{};
    p.tiles_per_expert = H / 128;
    p.K = I;
    p.rows_act = rows;
    p.sfa = bl.sf2;
    p.offsets = offsets;
    p.E = E;
    p.h_terms = nullptr;
    p.h_rec = nullptr;
    p.I = I;
    p.y_out = y_perm;
    p.H = H;
    p.status = ws.status;
    if (nt == 8)
        return launch_ffn<8, 3, false>(bl.w2, ws.h_terms, ws.h_rec, p, st);
    return launch_ffn<32, 3, false>(bl.w2, ws.h_terms, ws.h_rec, p, st);
}

int run_expert_ffn(const void *x, const int32_t *offsets, const int32_t *src_row, const void *prepacked, int T,
                   int k, int E, int H, int I, float *y_perm, void *workspace, cudaStream_t st)
{
    if (int rc = run_ffn_gate_up(x, offsets, src_row, prepacked, T, k, E, H, I, workspace, st))
        return rc;
    return run_ffn_down(offsets, prepacked, T, k, E, H, I, y_perm, workspace, st);
}

int run_combine(const float *y_perm, const int32_t *dst_of, const float *w, int T, int k, int H, float *y,
                cudaStream_t st)
{
    dim3 grid((H / 4 + 255) / 256, T);
    combine_kernel<<<grid, 256, 0, st>>>(y_perm, dst_of, w, T, k, H, y);
    return check_launch("combine_kernel");
}

int64_t ffn_workspace_bytes(int T, int k, int H, int I) { return ffn_ws_layout(T, k, H, I, nullptr, nullptr); }

int validate_ffn_shapes(int T, int k, int E, int H, int I) { return validate_ffn(T, k, E, H, I); }

}  // namespace mxmoe

using namespace mxmoe;

extern "C" MXMOE_API int64_t mxmoe_ffn_workspace_size(int T, int k, int E, int H, int I)
{
    if (T < 0 || k < 1 || k > 32 || E <= 0 || E > 1024 || H <= 0 || I <= 0 || H % 128 || I % 128 || H > 32768 ||
        I > 32768 || (int64_t)T * k > (1 << 22))
        return -1;
    return ffn_workspace_bytes(T, k, H, I);
}

static int check_ffn_args(const char *fn, int T, int k, int E, int H, int I, void *workspace, int64_t workspace_bytes)
{
    if (int rc = validate_ffn_shapes(T, k, E, H, I))
        return rc;
    if (!workspace || workspace_bytes < ffn_workspace_bytes(T, k, H, I))
        return fail(MXMOE_ERR_WORKSPACE, "%s: workspace of %lld bytes, need %lld", fn, (long long)workspace_bytes,
                    (long long)ffn_workspace_bytes(T, k, H, I));
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
    return run_expert_ffn(x, offsets, src_row, prepacked, T, k, E, H, I, y_perm, workspace, (cudaStream_t)stream);
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
    return run_ffn_gate_up(x, offsets, src_row, prepacked, T, k, E, H, I, workspace, (cudaStream_t)stream);
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
    return run_ffn_down(offsets, prepacked, T, k, E, H, I, y_perm, workspace, (cudaStream_t)stream);
}

extern "C" MXMOE_API int mxmoe_combine(const float *y_perm, const int32_t *dst_of, const float *w, int T, int k,
                                       int H, float *y, void *stream)
{
    if (T < 0 || k < 1 || H <= 0 || H % 4)
        return fail(MXMOE_ERR_INVALID_SHAPE, "mxmoe_combine: T=%d k=%d H=%d (H must be a multiple of 4)", T, k, H);
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
