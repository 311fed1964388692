// router_dev.cuh -- device code of the router GEMM tile and of the routing
// of one token, shared by the chained kernels (router.cu) and the persistent
// layer kernel (fused.cu).
//
// Pages: nxbn.cn MiMo-V2.5-Pro-FP4-DFlash article, architecture section: 384
// experts, 8 activated per token, hidden size 6144. The router function is
// read as the usual MoE gate: softmax over all expert logits, the top k kept
// (a tie going to the lower expert index), their weights renormalised to sum 1.
#pragma once

#include "common.cuh"

namespace mxmoe {

// ---------------------------------------------------------------------------
// Router GEMM (small T; from 512 tokens the tcgen05 kernel of router_tc.cu
// runs instead): logits[t, e] = sum_k x[t, k] Wg[e, k] + bias[e].
// CTA tile: 16 experts x 32 tokens x (K / splits); 8 warps split the tile's
// K range (warp w takes its k32 blocks w, w+8, ...), partial sums reduced in
// shared memory in a fixed order. With more than one split each tile writes
// its partial sums to out[z][t][e] (no bias) and routing adds the splits in
// order.
// Tensor cores with bf16 operands and fp32 accumulation: every bf16 product is
// exact in fp32. A and B fragments are loaded straight from global memory
// with the K order permuted identically on both operands (lane t holds 8
// consecutive k), which leaves the dot products unchanged.
// ---------------------------------------------------------------------------
constexpr int kRgExperts = 16, kRgTokens = 32, kRgWarps = 8, kRgUnroll = 4;

// Shared memory of one router tile: the 8 warps' partial sums.
struct RouterRed {
    float red[kRgWarps][kRgExperts][kRgTokens + 1];
};

// One CTA tile of the router GEMM (256 threads, all of them call it): experts
// 16 bx .. 16 bx + 15, tokens 32 by .. 32 by + 31, K split bz of nz (the k32
// blocks [nkb bz / nz, nkb (bz + 1) / nz)). Ends with a block-wide barrier, so
// that a CTA can run several tiles in a row.
__device__ __forceinline__ void router_tile(const uint16_t *__restrict__ x, const uint16_t *__restrict__ wg,
                                            const float *__restrict__ bias, int T, int H, int E,
                                            float *__restrict__ logits, int bx, int by, int bz, int nz, RouterRed &sm)
{
    float(&red)[kRgWarps][kRgExperts][kRgTokens + 1] = sm.red;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int e0 = bx * kRgExperts, t0 = by * kRgTokens;
    const int nkb_all = H / 32;
    const int kb_lo = (int)((int64_t)nkb_all * bz / nz);
    const int kb_hi = (int)((int64_t)nkb_all * (bz + 1) / nz);
    logits += (int64_t)bz * T * E;
    float acc[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int i = 0; i < 4; ++i)
            acc[j][i] = 0.f;
    const bool ra = e0 + g < E, rb = e0 + g + 8 < E;
    const uint16_t *wa = wg + (int64_t)(e0 + g) * H + 8 * t;
    const uint16_t *wb = wg + (int64_t)(e0 + g + 8) * H + 8 * t;
    for (int kb0 = kb_lo + warp; kb0 < kb_hi; kb0 += kRgWarps * kRgUnroll) {
        uint4 A[kRgUnroll][2];
        uint4 B[kRgUnroll][4];
#pragma unroll
        for (int u = 0; u < kRgUnroll; ++u) {
            const int kb = kb0 + u * kRgWarps;
            const bool kv = kb < kb_hi;
            A[u][0] = (kv && ra) ? __ldg(reinterpret_cast<const uint4 *>(wa + kb * 32)) : make_uint4(0, 0, 0, 0);
            A[u][1] = (kv && rb) ? __ldg(reinterpret_cast<const uint4 *>(wb + kb * 32)) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int tok = t0 + 8 * j + g;
                B[u][j] = (kv && tok < T)
                              ? __ldg(reinterpret_cast<const uint4 *>(x + (int64_t)tok * H + kb * 32 + 8 * t))
                              : make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int u = 0; u < kRgUnroll; ++u) {
            const uint32_t a0[4] = {A[u][0].x, A[u][1].x, A[u][0].y, A[u][1].y};
            const uint32_t a1[4] = {A[u][0].z, A[u][1].z, A[u][0].w, A[u][1].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                mma_bf16_16816(acc[j], a0, B[u][j].x, B[u][j].y, acc[j]);
                mma_bf16_16816(acc[j], a1, B[u][j].z, B[u][j].w, acc[j]);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        red[warp][g][8 * j + 2 * t] = acc[j][0];
        red[warp][g][8 * j + 2 * t + 1] = acc[j][1];
        red[warp][g + 8][8 * j + 2 * t] = acc[j][2];
        red[warp][g + 8][8 * j + 2 * t + 1] = acc[j][3];
    }
    __syncthreads();
    for (int o = threadIdx.x; o < kRgExperts * kRgTokens; o += blockDim.x) {
        const int er = o % kRgExperts, tc = o / kRgExperts;
        const int e = e0 + er, tok = t0 + tc;
        if (e < E && tok < T) {
            float s = 0.f;
#pragma unroll
            for (int w = 0; w < kRgWarps; ++w)
                s += red[w][er][tc];
            if (bias && nz == 1)
                s += bias[e];
            logits[(int64_t)tok * E + e] = s;
        }
    }
    __syncthreads();
}


// Routing key of (logit v, expert e): unsigned order is the selection order
// (larger logit first, then the lower expert). The logit's bits are mapped to
// an order-preserving unsigned value (negative: all bits flipped; otherwise
// the sign bit set), with -0 taken as +0 so that the two tie; the low half is
// the complement of e.
__device__ __forceinline__ uint64_t route_key(float v, int e)
{
    uint32_t u = __float_as_uint(v);
    if (u == 0x80000000u)
        u = 0;
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((uint64_t)u << 32) | (uint32_t)~e;
}

__device__ __forceinline__ float route_key_value(uint64_t key)
{
    const uint32_t u = (uint32_t)(key >> 32);
    return __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
}

// One warp routes token tok (E <= 32 * V): lane l holds the logits of experts
// l, l + 32, ..., summed over the splits in split order (G splits' loads in
// flight at a time; G = 1 takes a single split) plus the bias, as routing
// keys. k rounds of a warp-wide maximum of the keys not yet taken pick the
// experts, with no block-wide barrier, so that 8 tokens share a 256-thread
// block.
template <int V, int G>
__device__ __forceinline__ void route_token(const float *__restrict__ logits, int nsplit, const float *__restrict__ bias,
                                            int T, int E, int k, int32_t *__restrict__ ids, float *__restrict__ w,
                                            int tok)
{
    const int lane = threadIdx.x & 31;
    const float *l = logits + (int64_t)tok * E;
    float v[V];
#pragma unroll
    for (int i = 0; i < V; ++i) {
        const int e = lane + 32 * i;
        v[i] = e < E ? __ldg(l + e) : 0.f;
    }
    if (G > 1) {
        int z = 1;
        for (; z + G - 1 < nsplit; z += G) {
            float pz[G][V];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float *lz = l + (int64_t)(z + g) * T * E;
#pragma unroll
                for (int i = 0; i < V; ++i) {
                    const int e = lane + 32 * i;
                    pz[g][i] = e < E ? __ldg(lz + e) : 0.f;
                }
            }
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int i = 0; i < V; ++i)
                    v[i] += pz[g][i];
        }
        for (; z < nsplit; ++z) {
            const float *lz = l + (int64_t)z * T * E;
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const int e = lane + 32 * i;
                v[i] += e < E ? __ldg(lz + e) : 0.f;
            }
        }
    }
    uint64_t key[V];
#pragma unroll
    for (int i = 0; i < V; ++i) {
        const int e = lane + 32 * i;
        key[i] = e < E ? route_key(bias ? v[i] + __ldg(bias + e) : v[i], e) : 0ull;  // 0: never picked
    }
    uint64_t sel = 0;  // lane j < k: the key of the j-th pick
    uint32_t taken = 0;  // bit i: key[i] already picked
    for (int j = 0; j < k; ++j) {
        uint64_t best = 0;
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const uint64_t c = ((taken >> i) & 1u) ? 0ull : key[i];
            best = c > best ? c : best;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const uint64_t o = __shfl_xor_sync(0xFFFFFFFFu, best, off);
            best = o > best ? o : best;
        }
        const uint32_t e = ~(uint32_t)best;
        if (best != 0 && (e & 31u) == (uint32_t)lane)  // the owner drops the pick from its candidates
            taken |= 1u << (e >> 5);
        if (lane == j)
            sel = best;
    }
    // weights: exp(l_j - l_max) / sum over the selected, summed in slot order
    const float sel_v = route_key_value(sel);
    const float top = __shfl_sync(0xFFFFFFFFu, sel_v, 0);
    const float ex = lane < k ? expf(sel_v - top) : 0.f;
    float ssum = 0.f;
    for (int j = 0; j < k; ++j)
        ssum += __shfl_sync(0xFFFFFFFFu, ex, j);
    if (lane < k) {
        ids[(int64_t)tok * k + lane] = (int32_t)~(uint32_t)sel;
        w[(int64_t)tok * k + lane] = ex / ssum;
    }
}


}  // namespace mxmoe
