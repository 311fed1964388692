// router.cu -- router GEMM (float32 logits), top-k routing, and the stable
// grouping of (token, slot) pairs by expert.
//
// Pages: nxbn.cn MiMo-V2.5-Pro-FP4-DFlash article, architecture section: 384
// experts, 8 activated per token, hidden size 6144. The router function is not
// on the pages; it is read as the usual MoE gate: softmax over all expert
// logits, the top k kept (a tie going to the lower expert index) and their
// weights renormalised to sum 1.
#include <float.h>

#include <algorithm>

#include "common.cuh"
#include "router_dev.cuh"

namespace mxmoe {
bool use_router_tc(int T, int H);
int router_tc_splits(int T, int H, int E);
int run_router_gemm_tc(const void *x, const void *wg, const float *bias, int T, int H, int E, float *out, int nsplit,
                       int *status, cudaStream_t st);
namespace {

// Router GEMM for small T: one tile per CTA (grid: expert tiles x token tiles x K splits).
__global__ void __launch_bounds__(256) router_gemm_kernel(const uint16_t *__restrict__ x,
                                                          const uint16_t *__restrict__ wg,
                                                          const float *__restrict__ bias, int T, int H, int E,
                                                          float *__restrict__ logits)
{
    grid_dep_wait();  // the preceding kernel's results (chained launch)
    grid_dep_launch();
    __shared__ RouterRed red;
    router_tile(x, wg, bias, T, H, E, logits, blockIdx.x, blockIdx.y, blockIdx.z, gridDim.z, red);
}

// ---------------------------------------------------------------------------
// Top-k routing for more than 1024 experts: one 128-thread block per token
// (up to 4096 experts). Thread i holds logits i,
// i+128, ...; k rounds of a block arg-max (larger value first, then lower
// index): thread, warp (shuffles), then the four warp winners in shared
// memory, combined in the same order by every thread.
// ---------------------------------------------------------------------------
constexpr int kRouteThreads = 128;

__device__ __forceinline__ bool route_better(float ov, int oi, float bv, int bi)
{
    return oi != 0x7FFFFFFF && (bi == 0x7FFFFFFF || ov > bv || (ov == bv && oi < bi));
}

// With nsplit > 1 the logits are the sum, in split order, of nsplit partial
// [T, E] arrays plus bias (the split router GEMM's output). E <= 128 * V.
template <int V>
__global__ void __launch_bounds__(kRouteThreads) route_kernel(const float *__restrict__ logits, int nsplit,
                                                              const float *__restrict__ bias, int T, int E, int k,
                                                              int32_t *__restrict__ ids, float *__restrict__ w)
{
    grid_dep_wait();  // the preceding kernel's results (chained launch)
    grid_dep_launch();
    __shared__ float s_bv[kRouteThreads / 32];
    __shared__ int s_bi[kRouteThreads / 32];
    __shared__ float s_sel_v[32];
    __shared__ int s_sel_i[32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tok = blockIdx.x;
    if (tok >= T)
        return;
    const float *l = logits + (int64_t)tok * E;
    float v[V];
#pragma unroll
    for (int i = 0; i < V; ++i) {
        const int e = tid + kRouteThreads * i;
        v[i] = e < E ? l[e] : -FLT_MAX;
    }
    // add the other splits in split order, four splits' loads at a time
    int z = 1;
    for (; z + 3 < nsplit; z += 4) {
        float pz[4][V];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const float *lz = l + (int64_t)(z + g) * T * E;
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const int e = tid + kRouteThreads * i;
                pz[g][i] = e < E ? lz[e] : 0.f;
            }
        }
#pragma unroll
        for (int g = 0; g < 4; ++g)
#pragma unroll
            for (int i = 0; i < V; ++i)
                v[i] += pz[g][i];
    }
    for (; z < nsplit; ++z) {
        const float *lz = l + (int64_t)z * T * E;
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int e = tid + kRouteThreads * i;
            v[i] += e < E ? lz[e] : 0.f;
        }
    }
    if (bias) {
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int e = tid + kRouteThreads * i;
            if (e < E)
                v[i] += bias[e];
        }
    }
    uint32_t taken = 0;
    for (int j = 0; j < k; ++j) {
        float bv = -FLT_MAX;
        int bi = 0x7FFFFFFF;
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int e = tid + kRouteThreads * i;
            if (e < E && !((taken >> i) & 1u) && route_better(v[i], e, bv, bi)) {
                bv = v[i];
                bi = e;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, off);
            const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, off);
            if (route_better(ov, oi, bv, bi)) {
                bv = ov;
                bi = oi;
            }
        }
        if (lane == 0) {
            s_bv[warp] = bv;
            s_bi[warp] = bi;
        }
        __syncthreads();
        bv = s_bv[0];
        bi = s_bi[0];
#pragma unroll
        for (int q = 1; q < kRouteThreads / 32; ++q)
            if (route_better(s_bv[q], s_bi[q], bv, bi)) {
                bv = s_bv[q];
                bi = s_bi[q];
            }
        if (bi != 0x7FFFFFFF && bi % kRouteThreads == tid)
            taken |= 1u << (bi / kRouteThreads);
        if (tid == 0) {
            s_sel_v[j] = bv;
            s_sel_i[j] = bi;
        }
        __syncthreads();
    }
    // weights: exp(l_j - l_max) / sum over the selected, summed in slot order
    if (warp == 0) {
        const float ex = (lane < k) ? expf(s_sel_v[lane < k ? lane : 0] - s_sel_v[0]) : 0.f;
        float s = 0.f;
        for (int j = 0; j < k; ++j)
            s += __shfl_sync(0xFFFFFFFFu, ex, j);
        if (lane < k) {
            ids[(int64_t)tok * k + lane] = s_sel_i[lane];
            w[(int64_t)tok * k + lane] = ex / s;
        }
    }
}

// ---------------------------------------------------------------------------
// Stable grouping by expert: one CTA of 1024 threads. Counts -> exclusive scan
// -> offsets; then pairs are placed chunk by chunk (1024 pairs in index order),
// each pair's rank = earlier chunks' count for its expert + count among lower
// warps of the chunk + count among lower lanes of its warp.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) permute_kernel(const int32_t *__restrict__ ids, int n, int E,
                                                       int32_t *__restrict__ offsets, int32_t *__restrict__ src_row,
                                                       int32_t *__restrict__ dst_of)
{
    grid_dep_wait();  // the preceding kernel's results (chained launch)
    grid_dep_launch();
    extern __shared__ int32_t sm[];
    int32_t *cursor = sm;            // [E]
    int32_t *wcnt = sm + E;          // [32][E]
    int32_t *total = sm + 33 * E;    // [E]: pairs of the current chunk per expert
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int e = tid; e < E; e += blockDim.x)
        cursor[e] = 0;
    __syncthreads();
    for (int p = tid; p < n; p += blockDim.x)
        atomicAdd(&cursor[min(max(ids[p], 0), E - 1)], 1);
    __syncthreads();
    if (warp == 0) {  // exclusive scan of counts by one warp
        int carry = 0;
        for (int base = 0; base < E; base += 32) {
            const int e = base + lane;
            const int c = e < E ? cursor[e] : 0;
            int incl = c;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
                if (lane >= off)
                    incl += o;
            }
            if (e < E) {
                cursor[e] = carry + incl - c;
                offsets[e] = carry + incl - c;
            }
            carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
        if (lane == 0)
            offsets[E] = carry;
    }
    __syncthreads();
    for (int base = 0; base < n; base += blockDim.x) {
        for (int i = tid; i < 32 * E; i += blockDim.x)
            wcnt[i] = 0;
        __syncthreads();
        const int p = base + tid;
        const bool valid = p < n;
        const int e = valid ? min(max(ids[p], 0), E - 1) : -1;
        const uint32_t vmask = __ballot_sync(0xFFFFFFFFu, valid);
        const uint32_t same = __match_any_sync(0xFFFFFFFFu, e) & vmask;
        const int in_warp = __popc(same & ((1u << lane) - 1u));
        if (valid && in_warp == 0)
            wcnt[warp * E + e] = __popc(same);
        __syncthreads();
        for (int ee = tid; ee < E; ee += blockDim.x) {  // exclusive scan over warps, per expert
            int run = 0;
            for (int w = 0; w < 32; ++w) {
                const int c = wcnt[w * E + ee];
                wcnt[w * E + ee] = run;
                run += c;
            }
            total[ee] = run;
        }
        __syncthreads();
        if (valid) {
            const int pos = cursor[e] + wcnt[warp * E + e] + in_warp;
            src_row[pos] = p;
            dst_of[p] = pos;
        }
        __syncthreads();
        for (int ee = tid; ee < E; ee += blockDim.x)
            cursor[ee] += total[ee];
        __syncthreads();
    }
}

// One warp per token, 8 tokens a block (E <= 32 * V), no block-wide barrier.
template <int V, int G>
__global__ void __launch_bounds__(256) route_warp_kernel(const float *__restrict__ logits, int nsplit,
                                                         const float *__restrict__ bias, int T, int E, int k,
                                                         int32_t *__restrict__ ids, float *__restrict__ w)
{
    grid_dep_wait();  // the preceding kernel's results (chained launch)
    grid_dep_launch();
    const int tok = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (tok < T)
        route_token<V, G>(logits, nsplit, bias, T, E, k, ids, w, tok);
}

// ---------------------------------------------------------------------------
// Multi-block stable grouping (many pairs; E <= 1024): the same result as
// permute_kernel from three launches over blocks of 1024 pairs.
//  1. permute_count_kernel: pairs of block b per expert -> counts[e][b].
//  2. permute_scan_kernel: block e turns counts[e][.] into its exclusive
//     prefix over blocks and writes the expert's total.
//  3. permute_scatter_kernel: each block scans the totals into the expert
//     offsets (block 0 writes them) and places its pairs: position =
//     offset[e] + pairs of e in earlier blocks + earlier pairs of e in this
//     block (warp match, then warps in order), so the order within an expert
//     stays ascending.
// ---------------------------------------------------------------------------
constexpr int kPmBlock = 1024;
constexpr int kPmMaxE = 1024;  // experts the grouping kernels take (shared memory: 34 ints per expert)

__global__ void __launch_bounds__(kPmBlock) permute_count_kernel(const int32_t *__restrict__ ids, int n, int E,
                                                                 int32_t *__restrict__ counts)
{
    grid_dep_wait();  // the preceding kernel's results (chained launch)
    grid_dep_launch();
    extern __shared__ int32_t cnt[];  // [E]
    const int tid = threadIdx.x, nb = gridDim.x;
    for (int e = tid; e < E; e += kPmBlock)
        cnt[e] = 0;
    __syncthreads();
    const int p = blockIdx.x * kPmBlock + tid;
    if (p < n)
        atomicAdd(&cnt[min(max(ids[p], 0), E - 1)], 1);
    __syncthreads();
    for (int e = tid; e < E; e += kPmBlock)
        counts[(int64_t)e * nb + blockIdx.x] = cnt[e];
}

// Exclusive scan of v over the block's 1024 threads; returns the prefix and
// puts the block total in *total (shared scratch s_warp[32]).
__device__ __forceinline__ int block_excl_scan_1024(int v, int32_t *s_warp, int *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
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
        const int w = s_warp[lane];
        int wi = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xFFFFFFFFu, wi, off);
            if (lane >= off)
                wi += o;
        }
        s_warp[lane] = wi - w;
        if (lane == 31)
            s_warp[32] = wi;
    }
    __syncthreads();
    const int r = s_warp[warp] + incl - v;
    *total = s_warp[32];
    __syncthreads();  // s_warp free again
    return r;
}

__global__ void __launch_bounds__(kPmBlock) permute_scan_kernel(int32_t *__restrict__ counts, int nb,
                                                                int32_t *__restrict__ totals)
{
    grid_dep_wait();  // the preceding kernel's results (chained launch)
    grid_dep_launch();
    __shared__ int32_t s_warp[33];
    int32_t *c = counts + (int64_t)blockIdx.x * nb;
    int carry = 0;
    for (int base = 0; base < nb; base += kPmBlock) {
        const int i = base + threadIdx.x;
        const int v = i < nb ? c[i] : 0;
        int tot;
        const int ex = block_excl_scan_1024(v, s_warp, &tot);
        if (i < nb)
            c[i] = carry + ex;
        carry += tot;
    }
    if (threadIdx.x == 0)
        totals[blockIdx.x] = carry;
}

__global__ void __launch_bounds__(kPmBlock) permute_scatter_kernel(const int32_t *__restrict__ ids, int n, int E,
                                                                   const int32_t *__restrict__ counts,
                                                                   const int32_t *__restrict__ totals,
                                                                   int32_t *__restrict__ offsets,
                                                                   int32_t *__restrict__ src_row,
                                                                   int32_t *__restrict__ dst_of)
{
    grid_dep_wait();  // the preceding kernel's results (chained launch)
    grid_dep_launch();
    extern __shared__ int32_t sm[];
    int32_t *base_e = sm;      // [E]: first position of this block's pairs of expert e
    int32_t *wcnt = sm + E;    // [32][E]: per warp, then exclusive over warps
    __shared__ int32_t s_warp[33];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nb = gridDim.x;
    {  // expert offsets: exclusive scan of the totals (E <= 1024: one expert per thread)
        const int t = tid < E ? totals[tid] : 0;
        int all;
        const int off = block_excl_scan_1024(t, s_warp, &all);
        if (tid < E) {
            base_e[tid] = off + counts[(int64_t)tid * nb + blockIdx.x];
            if (blockIdx.x == 0)
                offsets[tid] = off;
        }
        if (blockIdx.x == 0 && tid == 0)
            offsets[E] = all;
    }
    for (int i = tid; i < 32 * E; i += kPmBlock)
        wcnt[i] = 0;
    __syncthreads();
    const int p = blockIdx.x * kPmBlock + tid;
    const bool valid = p < n;
    const int e = valid ? min(max(ids[p], 0), E - 1) : -1;
    const uint32_t vmask = __ballot_sync(0xFFFFFFFFu, valid);
    const uint32_t same = __match_any_sync(0xFFFFFFFFu, e) & vmask;
    const int in_warp = __popc(same & ((1u << lane) - 1u));
    if (valid && in_warp == 0)
        wcnt[warp * E + e] = __popc(same);
    __syncthreads();
    for (int ee = tid; ee < E; ee += kPmBlock) {  // exclusive over warps, per expert
        int run = 0;
        for (int w = 0; w < 32; ++w) {
            const int c = wcnt[w * E + ee];
            wcnt[w * E + ee] = run;
            run += c;
        }
    }
    __syncthreads();
    if (valid) {
        const int pos = base_e[e] + wcnt[warp * E + e] + in_warp;
        src_row[pos] = p;
        dst_of[p] = pos;
    }
}

}  // namespace
}  // namespace mxmoe

using namespace mxmoe;

extern "C" MXMOE_API int mxmoe_router_gemm(const void *x, const void *wg, const float *bias, int T, int H, int E,
                                           float *logits, void *stream)
{
    if (T < 0 || E <= 0 || H <= 0 || H % 32)
        return fail(MXMOE_ERR_INVALID_SHAPE, "mxmoe_router_gemm: T=%d H=%d E=%d (H must be a positive multiple of 32)",
                    T, H, E);
    if (T == 0)
        return MXMOE_OK;
    if (!x || !wg || !logits)
        return fail(MXMOE_ERR_NULL, "mxmoe_router_gemm: NULL pointer");
    if (!aligned16(x) || !aligned16(wg))
        return fail(MXMOE_ERR_ALIGNMENT, "mxmoe_router_gemm: x and wg must be 16-byte aligned");
    if (int rc = check_device())
        return rc;
    if (use_router_tc(T, H))
        return run_router_gemm_tc(x, wg, bias, T, H, E, logits, 1, nullptr, (cudaStream_t)stream);
    dim3 grid((E + kRgExperts - 1) / kRgExperts, (T + kRgTokens - 1) / kRgTokens, 1);
    return launch_kernel("router_gemm_kernel", router_gemm_kernel, grid, 256, 0, (cudaStream_t)stream,
                         static_cast<const uint16_t *>(x), static_cast<const uint16_t *>(wg), bias, T, H, E, logits);
}

namespace mxmoe {

template <int V>
int launch_route_warp(const float *logits, int nsplit, const float *bias, int T, int E, int k, int32_t *ids, float *w,
                      int blocks, cudaStream_t st)
{
    constexpr int G = V <= 16 ? 4 : 2;  // split loads in flight (registers)
    if (nsplit == 1)
        return launch_kernel("route_warp_kernel", route_warp_kernel<V, 1>, blocks, 256, 0, st, logits, nsplit, bias, T,
                             E, k, ids, w);
    return launch_kernel("route_warp_kernel", route_warp_kernel<V, G>, blocks, 256, 0, st, logits, nsplit, bias, T, E,
                         k, ids, w);
}

// Top-k routing of T tokens: a warp per token up to 1024 experts, else the
// block-per-token kernel.
int launch_route(const float *logits, int nsplit, const float *bias, int T, int E, int k, int32_t *ids, float *w,
                 cudaStream_t st)
{
    if (E <= 1024) {  // a warp per token
        const int blocks = (T + 7) / 8;
        if (E <= 128)
            return launch_route_warp<4>(logits, nsplit, bias, T, E, k, ids, w, blocks, st);
        if (E <= 256)
            return launch_route_warp<8>(logits, nsplit, bias, T, E, k, ids, w, blocks, st);
        if (E <= 384)
            return launch_route_warp<12>(logits, nsplit, bias, T, E, k, ids, w, blocks, st);
        if (E <= 512)
            return launch_route_warp<16>(logits, nsplit, bias, T, E, k, ids, w, blocks, st);
        return launch_route_warp<32>(logits, nsplit, bias, T, E, k, ids, w, blocks, st);
    }
    return launch_kernel("route_kernel", route_kernel<32>, T, kRouteThreads, 0, st, logits, nsplit, bias, T, E, k, ids,
                         w);
}

// K splits for the layer's router GEMM: as many as keep all tiles in one
// wave of one tile per SM (the persistent layer kernel runs a tile per CTA;
// the chained kernel's CTAs all fit at once either way), at most 8, each
// split at least 8 k32 blocks (one per warp).
int router_splits(int T, int H, int E)
{
    if (use_router_tc(T, H))
        return router_tc_splits(T, H, E);
    const int64_t base = (int64_t)((E + kRgExperts - 1) / kRgExperts) * ((T + kRgTokens - 1) / kRgTokens);
    int z = (int)(num_sms() / std::max<int64_t>(base, 1));
    z = std::max(1, std::min(z, 8));
    z = std::min(z, std::max(1, (H / 32) / 8));
    return z;
}

// Router GEMM into nsplit partial arrays (nsplit = router_splits(T, H, E))
// plus routing that sums them (the layer path). partials: float [nsplit, T, E].
// status: where a timeout of the tcgen05 router is recorded.
int run_router_and_route(const void *x, const void *wg, const float *bias, int T, int H, int E, int k,
                         float *partials, int nsplit, int32_t *ids, float *w, int *status, cudaStream_t st)
{
    if (use_router_tc(T, H)) {
        if (int rc = run_router_gemm_tc(x, wg, bias, T, H, E, partials, nsplit, status, st))
            return rc;
        return launch_route(partials, nsplit, nsplit > 1 ? bias : nullptr, T, E, k, ids, w, st);
    }
    dim3 grid((E + kRgExperts - 1) / kRgExperts, (T + kRgTokens - 1) / kRgTokens, nsplit);
    if (int rc = launch_kernel("router_gemm_kernel", router_gemm_kernel, grid, 256, 0, st,
                               static_cast<const uint16_t *>(x), static_cast<const uint16_t *>(wg), bias, T, H, E,
                               partials))
        return rc;
    return launch_route(partials, nsplit, nsplit > 1 ? bias : nullptr, T, E, k, ids, w, st);
}

}  // namespace mxmoe

extern "C" MXMOE_API int mxmoe_route(const float *logits, int T, int E, int k, int32_t *ids, float *w, void *stream)
{
    if (T < 0 || E <= 0 || E > 4096 || k < 1 || k > E || k > 32)
        return fail(MXMOE_ERR_INVALID_SHAPE, "mxmoe_route: T=%d E=%d k=%d (need 1 <= k <= min(E, 32), E <= 4096)", T,
                    E, k);
    if (T == 0)
        return MXMOE_OK;
    if (!logits || !ids || !w)
        return fail(MXMOE_ERR_NULL, "mxmoe_route: NULL pointer");
    if (int rc = check_device())
        return rc;
    return launch_route(logits, 1, nullptr, T, E, k, ids, w, (cudaStream_t)stream);
}

namespace mxmoe {

// Scratch ints of the multi-block grouping: counts [E][blocks] + totals [E].
int64_t permute_scratch_ints(int n, int E) { return (int64_t)E * ((n + kPmBlock - 1) / kPmBlock) + E; }
bool use_multiblock_permute(int n, int E) { return n > 4 * kPmBlock && E <= kPmMaxE; }

// The layer path's grouping: the multi-block kernels when use_multiblock_permute
// (scratch: permute_scratch_ints(n, E) ints), else permute_kernel.
int run_permute(const int32_t *ids, int T, int k, int E, int32_t *offsets, int32_t *src_row, int32_t *dst_of,
                int32_t *scratch, cudaStream_t st)
{
    const int n = T * k;
    if (!use_multiblock_permute(n, E) || !scratch)
        return mxmoe_permute(ids, T, k, E, offsets, src_row, dst_of, st);
    const int nb = (n + kPmBlock - 1) / kPmBlock;
    int32_t *counts = scratch, *totals = scratch + (int64_t)E * nb;
    const size_t smem_scatter = (size_t)33 * E * sizeof(int32_t);
    static thread_local int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        if (cudaFuncSetAttribute(permute_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(33 * kPmBlock * sizeof(int32_t))) != cudaSuccess)
            return fail(MXMOE_ERR_CUDA, "permute_scatter_kernel: cannot reserve shared memory");
        configured_dev = dev;
    }
    if (int rc = launch_kernel("permute_count_kernel", permute_count_kernel, nb, kPmBlock, E * sizeof(int32_t), st,
                               ids, n, E, counts))
        return rc;
    if (int rc = launch_kernel("permute_scan_kernel", permute_scan_kernel, E, kPmBlock, 0, st, counts, nb, totals))
        return rc;
    return launch_kernel("permute_scatter_kernel", permute_scatter_kernel, nb, kPmBlock, smem_scatter, st, ids, n, E,
                         counts, totals, offsets, src_row, dst_of);
}

}  // namespace mxmoe

extern "C" MXMOE_API int mxmoe_permute(const int32_t *ids, int T, int k, int E, int32_t *offsets, int32_t *src_row,
                                       int32_t *dst_of, void *stream)
{
    if (T < 0 || k < 1 || E <= 0 || E > kPmMaxE || (int64_t)T * k > (1 << 24))
        return fail(MXMOE_ERR_INVALID_SHAPE, "mxmoe_permute: T=%d k=%d E=%d (need E <= %d, T*k <= 2^24)", T, k, E,
                    kPmMaxE);
    if (!offsets || (T > 0 && (!ids || !src_row || !dst_of)))
        return fail(MXMOE_ERR_NULL, "mxmoe_permute: NULL pointer");
    if (int rc = check_device())
        return rc;
    const size_t smem = (size_t)(E + 32 * E + E) * sizeof(int32_t);  // <= 136 KB for E <= 1024
    static thread_local int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        if (cudaFuncSetAttribute(permute_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(34 * kPmMaxE * sizeof(int32_t))) != cudaSuccess)
            return fail(MXMOE_ERR_CUDA, "mxmoe_permute: cannot reserve shared memory");
        configured_dev = dev;
    }
    return launch_kernel("permute_kernel", permute_kernel, 1, 1024, smem, (cudaStream_t)stream, ids, T * k, E, offsets,
                         src_row, dst_of);
}

extern "C" MXMOE_API int64_t mxmoe_permute_scratch_size(int T, int k, int E)
{
    if (T < 0 || k < 1 || E <= 0 || E > kPmMaxE || (int64_t)T * k > (1 << 24))
        return -1;
    return permute_scratch_ints(T * k, E) * (int64_t)sizeof(int32_t);
}

extern "C" MXMOE_API int mxmoe_permute_ws(const int32_t *ids, int T, int k, int E, int32_t *offsets,
                                          int32_t *src_row, int32_t *dst_of, void *scratch, int64_t scratch_bytes,
                                          void *stream)
{
    if (T < 0 || k < 1 || E <= 0 || E > kPmMaxE || (int64_t)T * k > (1 << 24))
        return fail(MXMOE_ERR_INVALID_SHAPE, "mxmoe_permute_ws: T=%d k=%d E=%d", T, k, E);
    if (!scratch || scratch_bytes < mxmoe_permute_scratch_size(T, k, E))
        return fail(MXMOE_ERR_WORKSPACE, "mxmoe_permute_ws: scratch of %lld bytes, need %lld",
                    (long long)scratch_bytes, (long long)mxmoe_permute_scratch_size(T, k, E));
    if (!offsets || (T > 0 && (!ids || !src_row || !dst_of)))
        return fail(MXMOE_ERR_NULL, "mxmoe_permute_ws: NULL pointer");
    if (int rc = check_device())
        return rc;
    ChainScope chain;
    return run_permute(ids, T, k, E, offsets, src_row, dst_of, static_cast<int32_t *>(scratch),
                       (cudaStream_t)stream);
}
