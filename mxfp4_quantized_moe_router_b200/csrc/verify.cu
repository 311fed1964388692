// verify.cu -- block verification of a speculative draft: which of a block's
// drafted tokens the backbone accepts, and the token it emits after them.
//
// Page: "MiMo-V2.5-Pro-FP4-DFlash" (alphaneural mirror), section 3
// "Block-Diffusion Speculative Decoding (DFlash)": the drafter fills a whole
// block of masked positions (at most 8) in one forward pass, the backbone
// verifies the block in one step, and rejection-sampling verification keeps
// the output lossless. Read as the standard speculative-sampling test, taken
// position by position in block order: p_i = softmax(z_i / tau) of the
// backbone's logits at block position i, q_i = softmax(w_i / tau) of the
// drafter's; draft token d_i is accepted when u_i q_i(d_i) < p_i(d_i); at the
// first rejection j the emitted token is drawn from max(0, p_j - q_j), after
// K acceptances from p_K, both by inverse CDF in token order with u_K (the
// smallest v whose running sum exceeds u_K times the total). tau = 0 is
// greedy verification: d_i is accepted while it is the argmax of z_i (ties to
// the lower index), and the emitted token is the argmax at the first
// mismatch. A draft token outside [0, V) is never accepted.
//
// Design (one B200): the work is a pass over every logit row of the block
// (K + 1 backbone rows, and K drafter rows when sampling), so it is bound by
// HBM. Four chained kernels:
//  1. verify_rows_kernel: one CTA per (row, 8192-logit chunk) -- max, the sum
//     of exp((z - max) / tau) and the argmax of the chunk, written as a
//     partial; coalesced loads, one pass, no atomics.
//  2. verify_decide_kernel: one CTA per block, a warp per row, merging the
//     rows' partials in chunk order (max, rescaled sums, argmax), then
//     thread 0 takes the position-by-position decisions; greedy verification
//     ends here.
//  3. verify_draw_sums_kernel: one CTA per (block, chunk) of the drawn row,
//     summing the draw's weights (residual, or p_K unnormalised).
//  4. verify_draw_pick_kernel: one CTA per block: block-wide scans find the
//     chunk where the running sum of the chunk sums passes u_K times the
//     total, then the token inside that chunk.
// Every reduction runs in a fixed order, so results are bit-reproducible.
#include <float.h>
#include <math.h>

#include <algorithm>

#include "common.cuh"

namespace mxmoe {
namespace {

constexpr int kVThreads = 256;
constexpr int kVPer = 32;                       // logits per thread per chunk
constexpr int kVChunk = kVThreads * kVPer;      // 8192 logits (32 KB) per chunk
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kVMaxChunks = 2048;               // vocabulary up to 2^24 (the draw's chunk sums in shared memory)

struct RowPart {
    float m;    // chunk maximum
    float s;    // sum over the chunk of 2^((z - m) k), k = log2(e) / tau (0 when greedy)
    float amax; // argmax value
    int arg;    // argmax index (lowest on ties), INT_MAX when the chunk holds nothing above -inf
};

struct DrawInfo {
    int n;       // accepted drafts; the draw uses position n's rows
    float mp, sp; // backbone row n: merged maximum and sum
    float mq, sq; // drafter row n (n < K): merged maximum and sum
};

__device__ __forceinline__ bool arg_better(float v, int i, float bv, int bi)
{
    return v > bv || (v == bv && i < bi);
}

// Block-wide (value, index) argmax and sum; every thread gets the results.
__device__ __forceinline__ void block_argmax(float &v, int &i, float *sv, int *si)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xFFFFFFFFu, v, off);
        const int oi = __shfl_xor_sync(0xFFFFFFFFu, i, off);
        if (arg_better(ov, oi, v, i)) {
            v = ov;
            i = oi;
        }
    }
    if (lane == 0) {
        sv[warp] = v;
        si[warp] = i;
    }
    __syncthreads();
    v = sv[0];
    i = si[0];
    for (int w = 1; w < kVThreads / 32; ++w)
        if (arg_better(sv[w], si[w], v, i)) {
            v = sv[w];
            i = si[w];
        }
    __syncthreads();
}

__device__ __forceinline__ float block_sum(float x, float *sx)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        x += __shfl_xor_sync(0xFFFFFFFFu, x, off);
    if (lane == 0)
        sx[warp] = x;
    __syncthreads();
    float t = 0.f;
    for (int w = 0; w < kVThreads / 32; ++w)
        t += sx[w];
    __syncthreads();
    return t;
}

// Row r of a block's rows: backbone rows 0..K, then (sampling) drafter rows.
__device__ __forceinline__ const float *row_ptr(const float *target, const float *draft, int K, int64_t V, int rows,
                                                int r)
{
    const int b = r / rows, j = r % rows;
    return j <= K ? target + ((int64_t)b * (K + 1) + j) * V : draft + ((int64_t)b * K + (j - K - 1)) * V;
}

__global__ void __launch_bounds__(kVThreads) verify_rows_kernel(const float *__restrict__ target,
                                                                const float *__restrict__ draft, int K, int64_t V,
                                                                int rows, float k, int nchunk,
                                                                RowPart *__restrict__ part)
{
    grid_dep_wait();  // the preceding kernel's results (chained launch)
    grid_dep_launch();
    __shared__ float sv[kVThreads / 32];
    __shared__ int si[kVThreads / 32];
    const int c = blockIdx.x, r = blockIdx.y;
    const float *row = row_ptr(target, draft, K, V, rows, r);
    const int64_t v0 = (int64_t)c * kVChunk + threadIdx.x;
    float x[kVPer];
#pragma unroll
    for (int i = 0; i < kVPer; ++i) {
        const int64_t v = v0 + (int64_t)i * kVThreads;
        x[i] = v < V ? __ldcs(row + v) : -INFINITY;  // streamed once
    }
    float bv = -INFINITY;
    int bi = INT_MAX;
#pragma unroll
    for (int i = 0; i < kVPer; ++i)  // indices rise with i: strict > keeps the lowest
        if (x[i] > bv) {
            bv = x[i];
            bi = (int)(v0 + (int64_t)i * kVThreads);
        }
    block_argmax(bv, bi, sv, si);
    float s = 0.f;
    if (k > 0.f && bv > -INFINITY) {
#pragma unroll
        for (int i = 0; i < kVPer; ++i)
            s += exp2f((x[i] - bv) * k);
        s = block_sum(s, sv);
    }
    if (threadIdx.x == 0)
        part[(int64_t)r * nchunk + c] = RowPart{bv, s, bv, bi};
}

// Merge of row r's chunk partials by one warp, in chunk order per lane and a
// fixed shuffle tree: maximum, sum rescaled to it, argmax.
__device__ __forceinline__ void merge_row(const RowPart *__restrict__ part, int64_t r, int nchunk, float k, float &m,
                                          float &s, int &arg)
{
    const int lane = threadIdx.x & 31;
    float lm = -INFINITY, ls = 0.f, av = -INFINITY;
    int ai = INT_MAX;
    for (int c = lane; c < nchunk; c += 32) {
        const RowPart p = part[r * nchunk + c];
        if (p.m > lm) {
            ls = (lm > -INFINITY ? ls * exp2f((lm - p.m) * k) : 0.f) + p.s;
            lm = p.m;
        } else if (p.m > -INFINITY) {
            ls += p.s * exp2f((p.m - lm) * k);
        }
        if (arg_better(p.amax, p.arg, av, ai)) {
            av = p.amax;
            ai = p.arg;
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float om = __shfl_xor_sync(0xFFFFFFFFu, lm, off);
        const float os = __shfl_xor_sync(0xFFFFFFFFu, ls, off);
        const float nm = fmaxf(lm, om);
        ls = (lm > -INFINITY ? ls * exp2f((lm - nm) * k) : 0.f) + (om > -INFINITY ? os * exp2f((om - nm) * k) : 0.f);
        lm = nm;
        const float ov = __shfl_xor_sync(0xFFFFFFFFu, av, off);
        const int oi = __shfl_xor_sync(0xFFFFFFFFu, ai, off);
        if (arg_better(ov, oi, av, ai)) {
            av = ov;
            ai = oi;
        }
    }
    m = lm;
    s = ls;
    arg = ai;
}

// One CTA per block, one warp per row (up to 32 warps): the warps merge the
// block's rows in parallel, the drafts' logits are read in the same round,
// and thread 0 takes the position-by-position decisions from shared memory.
__global__ void __launch_bounds__(1024) verify_decide_kernel(const float *__restrict__ target,
                                                            const float *__restrict__ draft,
                                                            const int32_t *__restrict__ dtok,
                                                            const float *__restrict__ u, int K, int64_t V, int rows,
                                                            float k, int nchunk, const RowPart *__restrict__ part,
                                                            DrawInfo *__restrict__ info, int32_t *__restrict__ accepted,
                                                            int32_t *__restrict__ tokens)
{
    grid_dep_wait();  // the preceding kernel's results (chained launch)
    grid_dep_launch();
    __shared__ float s_m[2 * 32 + 1], s_s[2 * 32 + 1];
    __shared__ int s_arg[2 * 32 + 1];
    __shared__ float s_zd[32], s_wd[32], s_u[33];
    __shared__ int s_d[32];
    __shared__ int s_n, s_out;
    const int b = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t *db = dtok + (int64_t)b * K;
    if (threadIdx.x < K)
        s_d[threadIdx.x] = db[threadIdx.x];
    if (threadIdx.x >= 64 && threadIdx.x <= 64 + K)
        s_u[threadIdx.x - 64] = u[(int64_t)b * (K + 1) + threadIdx.x - 64];
    for (int r = warp; r < rows; r += (int)(blockDim.x >> 5)) {
        float m, s;
        int arg;
        merge_row(part, (int64_t)b * rows + r, nchunk, k, m, s, arg);
        if (lane == 0) {
            s_m[r] = m;
            s_s[r] = s;
            s_arg[r] = arg;
        }
    }
    if (k > 0.f && threadIdx.x < 64) {  // the drafts' logits: backbone (threads 0..31) and drafter (32..63)
        const int i = threadIdx.x & 31;
        if (i < K) {
            const int32_t d = db[i];
            const bool ok = d >= 0 && (int64_t)d < V;
            if (threadIdx.x < 32)
                s_zd[i] = ok ? __ldg(target + ((int64_t)b * (K + 1) + i) * V + d) : 0.f;
            else
                s_wd[i] = ok ? __ldg(draft + ((int64_t)b * K + i) * V + d) : 0.f;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int n = 0, out = -1;
        if (k == 0.f) {  // greedy: the leading drafts that are their row's argmax
            while (n < K && s_d[n] >= 0 && (int64_t)s_d[n] < V && s_arg[n] == s_d[n])
                ++n;
            out = s_arg[n];
        } else {
            for (; n < K; ++n) {
                const int32_t d = s_d[n];
                if (d < 0 || (int64_t)d >= V)
                    break;
                const float pd = exp2f((s_zd[n] - s_m[n]) * k) / s_s[n];
                const float qd = exp2f((s_wd[n] - s_m[K + 1 + n]) * k) / s_s[K + 1 + n];
                if (!(s_u[n] * qd < pd))
                    break;
            }
            DrawInfo di;
            di.n = n;
            di.mp = s_m[n];
            di.sp = s_s[n];
            di.mq = n < K ? s_m[K + 1 + n] : 0.f;
            di.sq = n < K ? s_s[K + 1 + n] : 1.f;
            info[b] = di;
        }
        accepted[b] = n;
        s_n = n;
        s_out = out;
    }
    __syncthreads();
    if (threadIdx.x <= K) {  // the accepted drafts, then the emitted token (greedy; sampling draws it later), then -1
        const int i = threadIdx.x, n = s_n;
        tokens[(int64_t)b * (K + 1) + i] = i < n ? s_d[i] : (i == n ? s_out : -1);
    }
}

// Weight of token v in the draw of block b: the residual max(0, p - q), or
// (no drafter row) p_K unnormalised. rp, rq: 1 / (the rows' sums).
__device__ __forceinline__ float draw_weight(const float *zrow, const float *wrow, const DrawInfo &di, float k,
                                             float rp, float rq, int64_t v)
{
    const float p = exp2f((__ldg(zrow + v) - di.mp) * k);
    if (!wrow)
        return p;
    const float q = exp2f((__ldg(wrow + v) - di.mq) * k);
    return fmaxf(p * rp - q * rq, 0.f);
}

__global__ void __launch_bounds__(kVThreads) verify_draw_sums_kernel(const float *__restrict__ target,
                                                                     const float *__restrict__ draft, int K,
                                                                     int64_t V, float k, int nchunk,
                                                                     const DrawInfo *__restrict__ info,
                                                                     float *__restrict__ csum)
{
    grid_dep_wait();  // the preceding kernel's results (chained launch)
    grid_dep_launch();
    __shared__ float sx[kVThreads / 32];
    const int c = blockIdx.x, b = blockIdx.y;
    const DrawInfo di = info[b];
    const float *zrow = target + ((int64_t)b * (K + 1) + di.n) * V;
    const float *wrow = di.n < K ? draft + ((int64_t)b * K + di.n) * V : nullptr;
    const float rp = 1.f / di.sp, rq = 1.f / di.sq;
    const int64_t v0 = (int64_t)c * kVChunk + threadIdx.x;
    float zx[kVPer], wx[kVPer];  // every load in flight before the arithmetic
#pragma unroll
    for (int i = 0; i < kVPer; ++i) {
        const int64_t v = v0 + (int64_t)i * kVThreads;
        zx[i] = v < V ? __ldg(zrow + v) : -INFINITY;
        wx[i] = (v < V && wrow) ? __ldg(wrow + v) : -INFINITY;
    }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < kVPer; ++i) {
        const float p = exp2f((zx[i] - di.mp) * k);
        s += wrow ? fmaxf(p * rp - exp2f((wx[i] - di.mq) * k) * rq, 0.f) : p;
    }
    s = block_sum(s, sx);
    if (threadIdx.x == 0)
        csum[(int64_t)b * nchunk + c] = s;
}

// Exclusive running sums of x over the block's threads, in thread order
// (warp shuffles, then the warps' totals); also the block total.
__device__ __forceinline__ float block_exclusive_scan(float x, float *s_warp, float &total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float incl = x;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
        if (lane >= off)
            incl += o;
    }
    if (lane == 31)
        s_warp[warp] = incl;
    __syncthreads();
    float before = 0.f;
    total = 0.f;
    for (int w = 0; w < kVThreads / 32; ++w) {
        if (w < warp)
            before += s_warp[w];
        total += s_warp[w];
    }
    __syncthreads();
    return before + incl - x;
}

__global__ void __launch_bounds__(kVThreads) verify_draw_pick_kernel(const float *__restrict__ target,
                                                                     const float *__restrict__ draft,
                                                                     const float *__restrict__ u, int K, int64_t V,
                                                                     float k, int nchunk,
                                                                     const DrawInfo *__restrict__ info,
                                                                     const float *__restrict__ csum,
                                                                     int32_t *__restrict__ tokens)
{
    grid_dep_wait();  // the preceding kernel's results (chained launch)
    grid_dep_launch();
    __shared__ float s_warp[kVThreads / 32];
    __shared__ float s_incl[kVMaxChunks];  // running sums of the chunk sums, in chunk order
    __shared__ float s_w[kVChunk + kVChunk / 32];  // the chosen chunk's weights, one pad word per 32
    __shared__ int s_pick, s_last, s_cpick, s_clast;
    const int b = blockIdx.x, t = threadIdx.x;
    const float uk = __ldg(u + (int64_t)b * (K + 1) + K);  // issued before the dependent loads
    const DrawInfo di = info[b];
    const float rp = 1.f / di.sp, rq = 1.f / di.sq;
    const float *zrow = target + ((int64_t)b * (K + 1) + di.n) * V;
    const float *wrow = di.n < K ? draft + ((int64_t)b * K + di.n) * V : nullptr;
    const float *cs = csum + (int64_t)b * nchunk;
    if (t == 0) {
        s_pick = INT_MAX;
        s_last = -1;
        s_cpick = INT_MAX;
        s_clast = -1;
    }
    // 1. running sums of the chunk sums (block scans in rounds of 256
    // chunks), then the first chunk where they pass u_K times the total
    float carry = 0.f;
    for (int c0 = 0; c0 < nchunk; c0 += kVThreads) {
        const float x = c0 + t < nchunk ? cs[c0 + t] : 0.f;
        float rtot;
        const float ex = block_exclusive_scan(x, s_warp, rtot);
        if (c0 + t < nchunk) {
            s_incl[c0 + t] = carry + ex + x;
            if (x > 0.f)
                atomicMax(&s_clast, c0 + t);
        }
        carry += rtot;
    }
    __syncthreads();
    const float total = s_incl[nchunk - 1];
    const float thr = uk * total;
    for (int c0 = t; c0 < nchunk; c0 += kVThreads)
        if (s_incl[c0] > thr)
            atomicMin(&s_cpick, c0);
    __syncthreads();
    const bool scan = s_cpick != INT_MAX;  // rounding may leave the running sum at or below the threshold
    const int c = scan ? s_cpick : (s_clast >= 0 ? s_clast : 0);
    const float before_chunk = (scan && c > 0) ? s_incl[c - 1] : 0.f;
    // 2. within chunk c: the weights, loaded coalesced (thread t: logits
    // t + 256 i), into shared memory padded by one word per 32 so that
    // thread t then reads its own run [32 t, 32 t + 32) without bank
    // conflicts, and scans it in order
    {
        const int64_t cbase = (int64_t)c * kVChunk;
        float zx[kVPer], wx[kVPer];
#pragma unroll
        for (int i = 0; i < kVPer; ++i) {
            const int64_t v = cbase + t + (int64_t)i * kVThreads;
            zx[i] = v < V ? __ldg(zrow + v) : -INFINITY;
            wx[i] = (v < V && wrow) ? __ldg(wrow + v) : -INFINITY;
        }
#pragma unroll
        for (int i = 0; i < kVPer; ++i) {
            const int e = t + i * kVThreads;
            const float p = exp2f((zx[i] - di.mp) * k);
            s_w[e + (e >> 5)] = wrow ? fmaxf(p * rp - exp2f((wx[i] - di.mq) * k) * rq, 0.f) : p;
        }
    }
    __syncthreads();
    const int64_t base = (int64_t)c * kVChunk + (int64_t)t * kVPer;
    float w[kVPer];
    float tsum = 0.f;
#pragma unroll
    for (int i = 0; i < kVPer; ++i) {
        const int e = t * kVPer + i;
        w[i] = s_w[e + (e >> 5)];
        tsum += w[i];
    }
    float ctot;
    float run = before_chunk + block_exclusive_scan(tsum, s_warp, ctot);
    int last = -1;
#pragma unroll
    for (int i = 0; i < kVPer; ++i) {
        run += w[i];
        if (w[i] > 0.f) {
            last = (int)(base + i);
            if (scan && run > thr) {
                atomicMin(&s_pick, last);
                break;
            }
        }
    }
    if (last >= 0)
        atomicMax(&s_last, last);
    __syncthreads();
    if (t == 0)  // no token passed (rounding): the chunk's last token with a weight
        tokens[(int64_t)b * (K + 1) + di.n] = s_pick != INT_MAX ? s_pick : (s_last >= 0 ? s_last : 0);
}

}  // namespace

// Workspace layout: partials [B][rows][nchunk], then DrawInfo [B], then chunk sums [B][nchunk].
int64_t verify_ws_layout(int B, int K, int64_t V, bool sampling, RowPart **part, DrawInfo **info, float **csum,
                         void *base)
{
    const int rows = sampling ? 2 * K + 1 : K + 1;
    const int64_t nchunk = (V + kVChunk - 1) / kVChunk;
    int64_t off = 0;
    auto take = [&](int64_t bytes) {
        const int64_t o = off;
        off = align256(off + bytes);
        return o;
    };
    const int64_t o_part = take((int64_t)B * rows * nchunk * (int64_t)sizeof(RowPart));
    const int64_t o_info = take((int64_t)B * (int64_t)sizeof(DrawInfo));
    const int64_t o_csum = take((int64_t)B * nchunk * (int64_t)sizeof(float));
    if (base) {
        uint8_t *p = static_cast<uint8_t *>(base);
        *part = reinterpret_cast<RowPart *>(p + o_part);
        *info = reinterpret_cast<DrawInfo *>(p + o_info);
        *csum = reinterpret_cast<float *>(p + o_csum);
    }
    return off;
}

}  // namespace mxmoe

using namespace mxmoe;

// Blocks per call: the row pass puts B (2K + 1) rows on the grid's y extent.
static bool verify_blocks_ok(int B, int K) { return (int64_t)B * (2 * K + 1) <= 65535; }

extern "C" MXMOE_API int64_t mxmoe_verify_workspace_size(int B, int K, int64_t V)
{
    if (B < 0 || K < 1 || K > 32 || V < 1 || V > (int64_t)kVMaxChunks * kVChunk || !verify_blocks_ok(B, K))
        return -1;
    return verify_ws_layout(B, K, V, true, nullptr, nullptr, nullptr, nullptr);
}

extern "C" MXMOE_API int mxmoe_verify_block(const float *target_logits, const float *draft_logits,
                                            const int32_t *draft_tokens, const float *uniforms, int B, int K,
                                            int64_t V, float temperature, int32_t *accepted, int32_t *tokens,
                                            void *workspace, int64_t workspace_bytes, void *stream)
{
    if (B < 0 || K < 1 || K > 32 || V < 1 || V > (int64_t)kVMaxChunks * kVChunk || !verify_blocks_ok(B, K))
        return fail(MXMOE_ERR_INVALID_SHAPE,
                    "mxmoe_verify_block: B=%d K=%d V=%lld (need 1 <= K <= 32, V <= 2^24, B (2K+1) <= 65535)", B, K,
                    (long long)V);
    if (!(temperature >= 0.f) || isinf(temperature))
        return fail(MXMOE_ERR_INVALID_SHAPE, "mxmoe_verify_block: temperature must be finite and >= 0");
    const bool sampling = temperature > 0.f;
    // The kernels scale logits by log2(e) / temperature; a positive temperature
    // so small that this factor overflows float would turn (z - max) * k into
    // 0 * inf = NaN at the row maximum.
    if (sampling && isinf(kLog2e / temperature))
        return fail(MXMOE_ERR_INVALID_SHAPE,
                    "mxmoe_verify_block: temperature %g is too small (log2(e) / temperature overflows float); "
                    "use 0 for greedy verification",
                    (double)temperature);
    if (workspace_bytes < mxmoe_verify_workspace_size(B, K, V))
        return fail(MXMOE_ERR_WORKSPACE, "mxmoe_verify_block: workspace of %lld bytes, need %lld",
                    (long long)workspace_bytes, (long long)mxmoe_verify_workspace_size(B, K, V));
    if (B == 0)
        return MXMOE_OK;
    if (!target_logits || !draft_tokens || !uniforms || !accepted || !tokens || !workspace ||
        (sampling && !draft_logits))
        return fail(MXMOE_ERR_NULL, "mxmoe_verify_block: NULL pointer");
    if (reinterpret_cast<uintptr_t>(workspace) & 255)
        return fail(MXMOE_ERR_ALIGNMENT, "mxmoe_verify_block: workspace needs 256-byte alignment");
    if (int rc = check_device())
        return rc;
    RowPart *part;
    DrawInfo *info;
    float *csum;
    verify_ws_layout(B, K, V, sampling, &part, &info, &csum, workspace);
    const int rows = sampling ? 2 * K + 1 : K + 1;
    const int nchunk = (int)((V + kVChunk - 1) / kVChunk);
    const float k = sampling ? kLog2e / temperature : 0.f;
    cudaStream_t st = (cudaStream_t)stream;
    ChainScope chain;
    if (int rc = launch_kernel("verify_rows_kernel", verify_rows_kernel, dim3(nchunk, B * rows), kVThreads, 0, st,
                               target_logits, draft_logits, K, V, rows, k, nchunk, part))
        return rc;
    const int decide_threads = std::min(1024, std::max(128, 32 * rows));  // a warp per row
    if (int rc = launch_kernel("verify_decide_kernel", verify_decide_kernel, B, decide_threads, 0, st, target_logits,
                               draft_logits, draft_tokens, uniforms, K, V, rows, k, nchunk, part, info, accepted,
                               tokens))
        return rc;
    if (!sampling)
        return MXMOE_OK;
    if (int rc = launch_kernel("verify_draw_sums_kernel", verify_draw_sums_kernel, dim3(nchunk, B), kVThreads, 0, st,
                               target_logits, draft_logits, K, V, k, nchunk, info, csum))
        return rc;
    return launch_kernel("verify_draw_pick_kernel", verify_draw_pick_kernel, B, kVThreads, 0, st, target_logits,
                         draft_logits, uniforms, K, V, k, nchunk, info, csum, tokens);
}
