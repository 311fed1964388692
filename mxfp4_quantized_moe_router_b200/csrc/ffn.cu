// ffn.cu -- grouped SwiGLU expert FFN over MXFP4 weights (W4A16), the
// weighted combine, and the whole-layer chain.
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
//  * Weights are streamed once per (tile, token pass) from the prepacked blob
//    by 1-D bulk async copies (cp.async.bulk + mbarrier transaction counts)
//    into a multi-stage shared-memory ring filled by one producer warp.
//  * Eight consumer warps split each 256-wide K chunk into k32 blocks (one
//    MXFP4 scale block each). A warp decodes its E2M1 nibbles in registers
//    (cvt.rn.f16x2.e2m1x2, exact) straight into m16n8k16 tensor-core
//    fragments and multiplies them with f16 activations (ldmatrix), fp32
//    accumulation. Per k32 block the partial product is scaled by the weight
//    row's E8M0 scale times the activation block's power-of-two factor.
//  * Activations travel in "act16" rows: f16 values pre-multiplied by a
//    per-32-block power of two that puts the block maximum in [2^14, 2^15),
//    plus the inverse factors (exact for bf16 x; h keeps 11 bits).
//  * Stage 1 (gate/up): a tile is 32 intermediate columns (32 gate rows + the
//    32 matching up rows), so SwiGLU is fused into the epilogue, which writes
//    h directly as one act16 block (the k32 block the down GEMM consumes).
//  * Stage 2 (down): a tile is 64 output rows.
//  * Work items (expert, tile, token pass) are split contiguously over a
//    persistent grid sized to the SM count, so each CTA streams consecutive
//    tiles without gaps and passes over the same tile hit L2.
#include <float.h>

#include <algorithm>

#include "common.cuh"

namespace mxmoe {
namespace {

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bounded waits: 2 s
// Shared-memory row stride of one token's activation chunk: 1088 bytes of h16
// chunk (or 1024 of x16) plus 16 so that ldmatrix rows hit distinct banks.
constexpr int kActStride = act_chunk_bytes(kChunkK) + 16;

struct StageParams {
    const uint8_t *wblob;     // first tile of this matrix in the prepacked blob
    int tiles_per_expert;     // I/32 (gate/up) or H/64 (down)
    int K;                    // reduction length
    const uint8_t *act;       // x16 rows (gate/up) or h16 rows (down)
    int64_t act_row_bytes;
    const float *act_inv;     // gate/up: per-token inverse factor of x16
    const int32_t *offsets;   // [E+1]
    const int32_t *src_row;   // gate/up: token = src_row[r] / k; down: row r itself
    int k;
    int E;
    uint8_t *h_out;           // gate/up: h16 rows [T*k]
    int64_t h_row_bytes;
    int I;
    float *y_out;             // down: [T*k, H]
    int H;
    int *status;
};

template <int NT>
struct StageCfg {
    static constexpr int kNTiles = NT / 8;
    static constexpr int kStages = 3;
    static constexpr int kWBytes = (int)wchunk_bytes(kChunkK);  // 17408
    static constexpr int kStageBytes = kWBytes + NT * kActStride;
    static constexpr int kRedFloats = 4 * 4 * 16 * NT;  // half the consumer warps' partials
    static constexpr int kItemCap = 1025;                // item prefix for E <= 1024
    static constexpr size_t kSmem = (size_t)kStages * kStageBytes + (size_t)kRedFloats * 4 +
                                    (size_t)kItemCap * 4 + 2 * kStages * 8 + 64 + 128;
    static constexpr int kMinBlocks = NT <= 8 ? 2 : 1;
};

struct Item {
    int e, tile, r0, nt;
};

template <int NT>
__device__ __forceinline__ Item decode_item(int64_t idx, const int *item_start, const int32_t *offsets, int E,
                                            int tiles_per_expert)
{
    int lo = 0, hi = E;  // largest e with item_start[e] <= idx
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (item_start[mid] <= idx)
            lo = mid;
        else
            hi = mid;
    }
    const int e = lo;
    const int n_e = offsets[e + 1] - offsets[e];
    const int passes = (n_e + NT - 1) / NT;
    const int local = (int)(idx - item_start[e]);
    Item it;
    it.e = e;
    it.tile = local / passes;
    const int pass = local % passes;
    it.r0 = offsets[e] + pass * NT;
    it.nt = min(NT, n_e - pass * NT);
    return it;
}

// One k32 block of one chunk for one consumer warp: 4 slabs x 16 rows x 32 K of
// weights against NT activation columns. The E2M1 codes of each slab become
// f16 A fragments in registers (exact); two m16n8k16 MMAs give the block's
// partial sums, which are scaled by the weight row's E8M0 scale (and, for the
// h16 input, by the activation block's inverse factor) into the accumulators.
template <int NT, bool ACT_BLOCK_SCALES>
__device__ __forceinline__ void consume_block(const uint8_t *sb, int kw, int b, int lane,
                                              float (&acc)[4][NT / 8][4])
{
    constexpr int NTL = NT / 8;
    const int g = lane >> 2, t = lane & 3;
    const uint4 a01 = *reinterpret_cast<const uint4 *>(sb + b * 1024 + lane * 16);
    const uint4 a23 = *reinterpret_cast<const uint4 *>(sb + b * 1024 + 512 + lane * 16);
    const uint2 scw = *reinterpret_cast<const uint2 *>(sb + wchunk_nibble_bytes(kw) + b * 64 + g * 8);
    const uint8_t *act = sb + StageCfg<NT>::kWBytes;
    uint32_t bf[NTL][4];
    float sb0[NTL], sb1[NTL];
#pragma unroll
    for (int j = 0; j < NTL; ++j) {
        const uint32_t addr = smem_u32(act + (8 * j + (lane & 7)) * kActStride + (b * 32 + (lane >> 3) * 8) * 2);
        ldmatrix_x4(bf[j][0], bf[j][1], bf[j][2], bf[j][3], addr);
        if (ACT_BLOCK_SCALES) {
            sb0[j] = *reinterpret_cast<const float *>(act + (8 * j + 2 * t) * kActStride + kw * 2 + b * 4);
            sb1[j] = *reinterpret_cast<const float *>(act + (8 * j + 2 * t + 1) * kActStride + kw * 2 + b * 4);
        }
    }
    float sc[8];  // slab s: rows g -> sc[2s], g+8 -> sc[2s+1]
    e8m0x4_to_float(scw.x, sc[0], sc[1], sc[2], sc[3]);
    e8m0x4_to_float(scw.y, sc[4], sc[5], sc[6], sc[7]);
    const uint32_t words[8] = {a01.x, a01.y, a01.z, a01.w, a23.x, a23.y, a23.z, a23.w};
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        uint32_t A0[4], A1[4];
        e2m1x4_to_f16x2x4(words[2 * s], A0[0], A0[1], A0[2], A0[3]);
        e2m1x4_to_f16x2x4(words[2 * s + 1], A1[0], A1[1], A1[2], A1[3]);
#pragma unroll
        for (int j = 0; j < NTL; ++j) {
            float tmp[4] = {0.f, 0.f, 0.f, 0.f};
            mma_f16_16816(tmp, A0, bf[j][0], bf[j][1], tmp);
            mma_f16_16816(tmp, A1, bf[j][2], bf[j][3], tmp);
            if (ACT_BLOCK_SCALES) {
                acc[s][j][0] = fmaf(tmp[0], sc[2 * s] * sb0[j], acc[s][j][0]);
                acc[s][j][1] = fmaf(tmp[1], sc[2 * s] * sb1[j], acc[s][j][1]);
                acc[s][j][2] = fmaf(tmp[2], sc[2 * s + 1] * sb0[j], acc[s][j][2]);
                acc[s][j][3] = fmaf(tmp[3], sc[2 * s + 1] * sb1[j], acc[s][j][3]);
            } else {
                acc[s][j][0] = fmaf(tmp[0], sc[2 * s], acc[s][j][0]);
                acc[s][j][1] = fmaf(tmp[1], sc[2 * s], acc[s][j][1]);
                acc[s][j][2] = fmaf(tmp[2], sc[2 * s + 1], acc[s][j][2]);
                acc[s][j][3] = fmaf(tmp[3], sc[2 * s + 1], acc[s][j][3]);
            }
        }
    }
}

// GATE_UP = true: stage 1 (x16 input, SwiGLU epilogue writing h16);
// GATE_UP = false: stage 2 (h16 input, float output rows).
template <int NT, bool GATE_UP>
__global__ void __launch_bounds__(288, StageCfg<NT>::kMinBlocks) ffn_stage_kernel(const StageParams p)
{
    using C = StageCfg<NT>;
    constexpr bool kBlockScales = !GATE_UP;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    uint8_t *stages = smem;
    float *red = reinterpret_cast<float *>(smem + (size_t)C::kStages * C::kStageBytes);
    int *item_start = reinterpret_cast<int *>(red + C::kRedFloats);
    uint64_t *full = reinterpret_cast<uint64_t *>(item_start + C::kItemCap + 1);
    full = reinterpret_cast<uint64_t *>((reinterpret_cast<uintptr_t>(full) + 7) & ~uintptr_t(7));
    uint64_t *empty = full + C::kStages;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + C::kStages);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int E = p.E;

    // item prefix: items of expert e = tiles_per_expert * ceil(n_e / NT)
    if (warp == 0) {
        int carry = 0;
        for (int base = 0; base < E; base += 32) {
            const int e = base + lane;
            const int n_e = e < E ? p.offsets[e + 1] - p.offsets[e] : 0;
            const int c = p.tiles_per_expert * ((n_e + NT - 1) / NT);
            int incl = c;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
                if (lane >= off)
                    incl += o;
            }
            if (e < E)
                item_start[e] = carry + incl - c;
            carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
        if (lane == 0)
            item_start[E] = carry;
    }
    if (tid == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    const int64_t n_items = item_start[E];
    const int64_t i_begin = n_items * blockIdx.x / gridDim.x;
    const int64_t i_end = n_items * (blockIdx.x + 1) / gridDim.x;
    const int nchunk = (p.K + kChunkK - 1) / kChunkK;
    const int64_t tile_bytes = wtile_bytes(p.K);

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------- producer
        const uint64_t pol_w = policy_evict_first();
        const uint64_t pol_a = policy_evict_last();
        int stage = 0;
        uint32_t phase = 0;
        int64_t issued = 0;
        bool ok = true;
        for (int64_t idx = i_begin; idx < i_end && ok; ++idx) {
            const Item it = decode_item<NT>(idx, item_start, p.offsets, E, p.tiles_per_expert);
            const uint8_t *wsrc = p.wblob + ((int64_t)it.e * p.tiles_per_expert + it.tile) * tile_bytes;
            const uint8_t *arow = p.act;
            if (lane < it.nt) {
                const int r = it.r0 + lane;
                arow += (GATE_UP ? (int64_t)(p.src_row[r] / p.k) : (int64_t)r) * p.act_row_bytes;
            }
            for (int c = 0; c < nchunk; ++c) {
                const int kw = min(kChunkK, p.K - c * kChunkK);
                if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, kWaitLimitNs) || *abort_flag) {
                    if (lane == 0) {
                        set_status(p.status, MXMOE_ERR_TIMEOUT);
                        *abort_flag = 1;
                    }
                    ok = false;
                    break;
                }
                uint8_t *sbuf = stages + (size_t)stage * C::kStageBytes;
                const uint32_t abytes = (uint32_t)(kBlockScales ? act_chunk_bytes(kw) : kw * 2);
                const int64_t aoff = (int64_t)c * (kBlockScales ? act_chunk_bytes(kChunkK) : kChunkK * 2);
                if (lane == 0) {
                    mbar_arrive_expect_tx(&full[stage], (uint32_t)wchunk_bytes(kw) + (uint32_t)it.nt * abytes);
                    bulk_g2s_hint(sbuf, wsrc + (int64_t)c * C::kWBytes, (uint32_t)wchunk_bytes(kw), &full[stage],
                                  pol_w);
                }
                __syncwarp();
                if (lane < it.nt)
                    bulk_g2s_hint(sbuf + C::kWBytes + lane * kActStride, arow + aoff, abytes, &full[stage], pol_a);
                ++issued;
                if (++stage == C::kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        // Drain: make sure no copy of ours is still landing in shared memory.
        if (lane == 0) {
            const int64_t first = issued > C::kStages ? issued - C::kStages : 0;
            for (int64_t f = first; f < issued; ++f) {
                const int s = (int)(f % C::kStages);
                const uint32_t par = (uint32_t)((f / C::kStages) & 1);
                if (!mbar_wait_bounded(&full[s], par, kWaitLimitNs)) {
                    set_status(p.status, MXMOE_ERR_TIMEOUT);
                    break;
                }
            }
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    // A consumer that gives up on a wait never leaves early: it stops reading
    // shared memory and writing outputs but keeps taking part in the named
    // barriers, so no other warp can be left waiting.
    const int g = lane >> 2, t = lane & 3;
    int stage = 0;
    uint32_t phase = 0;
    bool aborted = false;
    for (int64_t idx = i_begin; idx < i_end; ++idx) {
        const Item it = decode_item<NT>(idx, item_start, p.offsets, E, p.tiles_per_expert);
        aborted = aborted || *abort_flag;
        float acc[4][C::kNTiles][4];
#pragma unroll
        for (int s = 0; s < 4; ++s)
#pragma unroll
            for (int j = 0; j < C::kNTiles; ++j)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    acc[s][j][i] = 0.f;
        for (int c = 0; c < nchunk; ++c) {
            const int kw = min(kChunkK, p.K - c * kChunkK);
            if (!aborted && (!mbar_wait_bounded(&full[stage], phase, kWaitLimitNs) || *abort_flag)) {
                if (lane == 0) {
                    set_status(p.status, MXMOE_ERR_TIMEOUT);
                    *abort_flag = 1;
                }
                aborted = true;
            }
            const uint8_t *sbuf = stages + (size_t)stage * C::kStageBytes;
            if (!aborted) {
                // warp w takes k32 blocks 2w and 2w+1 of the chunk
                if (2 * warp * 32 < kw)
                    consume_block<NT, kBlockScales>(sbuf, kw, 2 * warp, lane, acc);
                if ((2 * warp + 1) * 32 < kw)
                    consume_block<NT, kBlockScales>(sbuf, kw, 2 * warp + 1, lane, acc);
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&empty[stage]);
            if (++stage == C::kStages) {
                stage = 0;
                phase ^= 1u;
            }
        }
        // ------------------------------------------------------------ epilogue
        // Two-level reduction over the 8 warps in a fixed order: warps 4..7
        // store, warps 0..3 add their own partials, then the output threads add
        // the four sums. red[((w*4 + s)*16 + row16)*NT + n], w < 4.
        auto store_acc = [&](int w, bool add) {
#pragma unroll
            for (int s = 0; s < 4; ++s)
#pragma unroll
                for (int j = 0; j < C::kNTiles; ++j) {
                    const int n0 = 8 * j + 2 * t;
                    float *rw = red + ((w * 4 + s) * 16) * NT;
                    const float v[4] = {acc[s][j][0], acc[s][j][1], acc[s][j][2], acc[s][j][3]};
                    float *d[4] = {&rw[g * NT + n0], &rw[g * NT + n0 + 1], &rw[(g + 8) * NT + n0],
                                   &rw[(g + 8) * NT + n0 + 1]};
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        *d[i] = add ? *d[i] + v[i] : v[i];
                }
        };
        if (warp >= 4)
            store_acc(warp - 4, false);
        named_bar_sync(1, kConsumerWarps * 32);
        if (warp < 4)
            store_acc(warp, true);
        named_bar_sync(1, kConsumerWarps * 32);
        aborted = aborted || *abort_flag;
        if (aborted) {
            // nothing to write
        } else if (GATE_UP) {
            // 32 h columns x nt tokens; warp -> token, lane -> column
            const int col = lane, sg = col >> 4, r16 = col & 15;
            const int hcol0 = it.tile * 32;
            const int hc = hcol0 / kChunkK;
            const int kwc = min(kChunkK, p.I - hc * kChunkK);
            for (int n = warp; n < it.nt; n += kConsumerWarps) {
                float gs = 0.f, us = 0.f;
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    gs += red[((w * 4 + sg) * 16 + r16) * NT + n];
                    us += red[((w * 4 + 2 + sg) * 16 + r16) * NT + n];
                }
                const float xinv = p.act_inv[p.src_row[it.r0 + n] / p.k];
                gs *= xinv;
                us *= xinv;
                const float h = gs / (1.f + expf(-gs)) * us;
                float m = fabsf(h);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1)
                    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
                float mul, inv;
                act_block_factor(m, mul, inv);
                uint8_t *row = p.h_out + (int64_t)(it.r0 + n) * p.h_row_bytes + (int64_t)hc * act_chunk_bytes(kChunkK);
                reinterpret_cast<unsigned short *>(row)[(hcol0 - hc * kChunkK) + col] =
                    __half_as_ushort(__float2half_rn(h * mul));
                if (lane == 0)
                    reinterpret_cast<float *>(row + kwc * 2)[(hcol0 - hc * kChunkK) / 32] = inv;
            }
        } else {
            for (int n = warp; n < it.nt; n += kConsumerWarps) {
                float *yrow = p.y_out + (int64_t)(it.r0 + n) * p.H + it.tile * 64;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int rr = lane + 32 * half, s = rr >> 4, r16 = rr & 15;
                    float v = 0.f;
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        v += red[((w * 4 + s) * 16 + r16) * NT + n];
                    yrow[rr] = v;
                }
            }
        }
        named_bar_sync(1, kConsumerWarps * 32);
    }
}

// bf16 rows -> x16 rows: one block per row; pass 1 finds max |x| of the row,
// pass 2 writes x * 2^(14 - floor(log2 max)) as f16 and stores the inverse
// factor. Block 0 also clears the status word.
__global__ void __launch_bounds__(256) act_convert_kernel(const uint16_t *__restrict__ x, int64_t rows, int K,
                                                          uint16_t *__restrict__ out, float *__restrict__ inv_out,
                                                          int *status)
{
    __shared__ float wmax[8];
    if (blockIdx.x == 0 && threadIdx.x == 0 && status)
        *status = 0;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n16 = K / 8;  // 16-byte groups of 8 values
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        const uint4 *src = reinterpret_cast<const uint4 *>(x + r * K);
        float m = 0.f;
        for (int i = threadIdx.x; i < n16; i += blockDim.x) {
            const uint4 v = __ldg(src + i);
            const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q)
                m = fmaxf(m, fmaxf(fabsf(__uint_as_float(wv[q] << 16)), fabsf(__uint_as_float(wv[q] & 0xFFFF0000u))));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
        if (lane == 0)
            wmax[warp] = m;
        __syncthreads();
        m = wmax[0];
#pragma unroll
        for (int w = 1; w < 8; ++w)
            m = fmaxf(m, wmax[w]);
        float mul, inv;
        act_block_factor(m, mul, inv);
        uint4 *dst = reinterpret_cast<uint4 *>(out + r * K);
        for (int i = threadIdx.x; i < n16; i += blockDim.x) {
            const uint4 v = __ldg(src + i);
            const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
            uint32_t hv[4];
#pragma unroll
            for (int q = 0; q < 4; ++q)
                hv[q] = (uint32_t)__half_as_ushort(__float2half_rn(__uint_as_float(wv[q] << 16) * mul)) |
                        ((uint32_t)__half_as_ushort(__float2half_rn(__uint_as_float(wv[q] & 0xFFFF0000u) * mul))
                         << 16);
            dst[i] = make_uint4(hv[0], hv[1], hv[2], hv[3]);
        }
        if (threadIdx.x == 0)
            inv_out[r] = inv;
        __syncthreads();  // wmax is reused by the next row
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
    uint16_t *x16;
    float *xinv;
    uint8_t *h16;
};

int64_t ffn_ws_layout(int T, int k, int H, int I, FfnWs *ws, void *base)
{
    int64_t off = 0;
    auto take = [&](int64_t bytes) {
        int64_t o = off;
        off = align256(off + bytes);
        return o;
    };
    const int64_t o_status = take(16);
    const int64_t o_x16 = take((int64_t)T * H * 2);
    const int64_t o_xinv = take((int64_t)T * 4);
    const int64_t o_h16 = take((int64_t)T * k * act_row_bytes(I));
    if (ws && base) {
        uint8_t *b = static_cast<uint8_t *>(base);
        ws->status = reinterpret_cast<int *>(b + o_status);
        ws->x16 = reinterpret_cast<uint16_t *>(b + o_x16);
        ws->xinv = reinterpret_cast<float *>(b + o_xinv);
        ws->h16 = b + o_h16;
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

template <int NT, bool GATE_UP>
int launch_stage(const StageParams &p, cudaStream_t st)
{
    using C = StageCfg<NT>;
    static thread_local int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        if (cudaFuncSetAttribute(ffn_stage_kernel<NT, GATE_UP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)C::kSmem) != cudaSuccess)
            return fail(MXMOE_ERR_CUDA, "ffn_stage_kernel: cannot reserve %zu bytes of shared memory", C::kSmem);
        configured_dev = dev;
    }
    int per_sm = 1;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, ffn_stage_kernel<NT, GATE_UP>, 288, C::kSmem);
    if (per_sm < 1)
        per_sm = 1;
    ffn_stage_kernel<NT, GATE_UP><<<num_sms() * per_sm, 288, C::kSmem, st>>>(p);
    return check_launch(GATE_UP ? "ffn_stage_kernel<gate_up>" : "ffn_stage_kernel<down>");
}

template <bool GATE_UP>
int launch_stage_nt(int T, const StageParams &p, cudaStream_t st)
{
    if (T <= 8)
        return launch_stage<8, GATE_UP>(p, st);
    return launch_stage<32, GATE_UP>(p, st);
}

int validate_ffn(int T, int k, int E, int H, int I)
{
    if (T < 0 || k < 1 || k > 32 || E <= 0 || E > 1024 || H <= 0 || I <= 0 || H % 64 || I % 32 ||
        (int64_t)T * k > (1 << 24))
        return fail(MXMOE_ERR_INVALID_SHAPE,
                    "expert FFN: T=%d k=%d E=%d H=%d I=%d (need H %% 64 == 0, I %% 32 == 0, 1 <= k <= 32, E <= 1024)",
                    T, k, E, H, I);
    return MXMOE_OK;
}

}  // namespace

int run_ffn_gate_up(const void *x, const int32_t *offsets, const int32_t *src_row, const void *prepacked, int T,
                    int k, int E, int H, int I, void *workspace, cudaStream_t st)
{
    FfnWs ws;
    ffn_ws_layout(T, k, H, I, &ws, workspace);
    {
        int blocks = (int)std::min<int64_t>((int64_t)T, (int64_t)num_sms() * 8);
        act_convert_kernel<<<blocks < 1 ? 1 : blocks, 256, 0, st>>>(static_cast<const uint16_t *>(x), T, H, ws.x16,
                                                                    ws.xinv, ws.status);
        if (int rc = check_launch("act_convert_kernel"))
            return rc;
    }
    StageParams p1{};
    p1.wblob = static_cast<const uint8_t *>(prepacked);
    p1.tiles_per_expert = I / 32;
    p1.K = H;
    p1.act = reinterpret_cast<const uint8_t *>(ws.x16);
    p1.act_row_bytes = (int64_t)H * 2;
    p1.act_inv = ws.xinv;
    p1.offsets = offsets;
    p1.src_row = src_row;
    p1.k = k;
    p1.E = E;
    p1.h_out = ws.h16;
    p1.h_row_bytes = act_row_bytes(I);
    p1.I = I;
    p1.y_out = nullptr;
    p1.H = H;
    p1.status = ws.status;
    return launch_stage_nt<true>(T, p1, st);
}

int run_ffn_down(const int32_t *offsets, const void *prepacked, int T, int k, int E, int H, int I, float *y_perm,
                 void *workspace, cudaStream_t st)
{
    FfnWs ws;
    ffn_ws_layout(T, k, H, I, &ws, workspace);
    StageParams p2{};
    p2.wblob = static_cast<const uint8_t *>(prepacked) + (int64_t)E * (I / 32) * wtile_bytes(H);
    p2.tiles_per_expert = H / 64;
    p2.K = I;
    p2.act = ws.h16;
    p2.act_row_bytes = act_row_bytes(I);
    p2.act_inv = nullptr;
    p2.offsets = offsets;
    p2.src_row = nullptr;
    p2.k = k;
    p2.E = E;
    p2.h_out = nullptr;
    p2.h_row_bytes = 0;
    p2.I = I;
    p2.y_out = y_perm;
    p2.H = H;
    p2.status = ws.status;
    return launch_stage_nt<false>(T, p2, st);
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
    if (T < 0 || k < 1 || k > 32 || E <= 0 || E > 1024 || H <= 0 || I <= 0 || H % 64 || I % 32)
        return -1;
    return ffn_workspace_bytes(T, k, H, I);
}

extern "C" MXMOE_API int mxmoe_expert_ffn(const void *x, const int32_t *offsets, const int32_t *src_row,
                                          const void *prepacked, int T, int k, int E, int H, int I, float *y_perm,
                                          void *workspace, int64_t workspace_bytes, void *stream)
{
    if (int rc = validate_ffn_shapes(T, k, E, H, I))
        return rc;
    if (!workspace || workspace_bytes < ffn_workspace_bytes(T, k, H, I))
        return fail(MXMOE_ERR_WORKSPACE, "mxmoe_expert_ffn: workspace of %lld bytes, need %lld",
                    (long long)workspace_bytes, (long long)ffn_workspace_bytes(T, k, H, I));
    if (T == 0)
        return MXMOE_OK;
    if (!x || !offsets || !src_row || !prepacked || !y_perm)
        return fail(MXMOE_ERR_NULL, "mxmoe_expert_ffn: NULL pointer");
    if (!aligned16(x) || !aligned16(prepacked) || !aligned16(y_perm) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255))
        return fail(MXMOE_ERR_ALIGNMENT,
                    "mxmoe_expert_ffn: x, prepacked, y_perm need 16-byte and workspace 256-byte alignment");
    if (int rc = check_device())
        return rc;
    return run_expert_ffn(x, offsets, src_row, prepacked, T, k, E, H, I, y_perm, workspace, (cudaStream_t)stream);
}

static int check_ffn_args(const char *fn, int T, int k, int E, int H, int I, void *workspace,
                          int64_t workspace_bytes)
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
    if (!aligned16(x) || !aligned16(prepacked))
        return fail(MXMOE_ERR_ALIGNMENT, "mxmoe_ffn_gate_up: x and prepacked need 16-byte alignment");
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
    if (!aligned16(prepacked) || !aligned16(y_perm))
        return fail(MXMOE_ERR_ALIGNMENT, "mxmoe_ffn_down: prepacked and y_perm need 16-byte alignment");
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
