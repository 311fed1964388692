// ep.cu -- expert parallelism: the layer's experts split over G ranks, each
// rank holding one contiguous range of E/G experts. The kernels here are the
// compute on either side of the two all-to-all exchanges:
//   dispatch (sender): tokens' rows in the grouped order of mxmoe_permute,
//     which is also destination-rank order, with each row's expert id local
//     to its owner and the row count per destination rank;
//   expert FFN (receiver): the received rows grouped by local expert, run
//     through the rank's expert shard, and returned in receive order.
// The exchanges themselves (NCCL all-to-all over NVLink, through
// torch.distributed) and the final weighted combine (mxmoe_combine, on the
// sender) sit around them.
//
// Pages: the model is served with expert parallelism (the SGLang launch in
// the "MiMo-V2.5-Pro-FP4-DFlash" model card's deployment section and in the
// nxbn.cn article's SGLang deployment section pass --ep-size 16); 384
// experts, 8 per token (nxbn.cn article, architecture section).
#include "common.cuh"

namespace mxmoe {
int run_permute(const int32_t *ids, int T, int k, int E, int32_t *offsets, int32_t *src_row, int32_t *dst_of,
                int32_t *scratch, cudaStream_t st);
int64_t permute_scratch_ints(int n, int E);
int run_expert_ffn(const void *x, const int32_t *offsets, const int32_t *src_row, const void *prepacked, int T,
                   int k, int E, int H, int I, float *y_perm, void *workspace, bool clear_status, cudaStream_t st);
int64_t ffn_workspace_bytes(int T, int k, int E, int H, int I);
bool ffn_shapes_ok(int T, int k, int E, int H, int I);

namespace {

// Sender side: one warp per grouped row r. send_x[r] = x[src_row[r] / k]
// (H bf16 values, 16-byte copies), send_local[r] = expert of r minus the first
// expert of its owner rank; block 0 also writes send_counts[g], the rows of
// experts [g E/G, (g+1) E/G).
__global__ void __launch_bounds__(256) ep_dispatch_kernel(const uint16_t *__restrict__ x,
                                                          const int32_t *__restrict__ offsets,
                                                          const int32_t *__restrict__ src_row, int n, int k, int E,
                                                          int G, int H, uint16_t *__restrict__ send_x,
                                                          int32_t *__restrict__ send_local,
                                                          int32_t *__restrict__ send_counts)
{
    grid_dep_wait();  // the preceding kernel's results (chained launch)
    grid_dep_launch();
    const int per = E / G;
    if (blockIdx.x == 0)
        for (int g = threadIdx.x; g < G; g += blockDim.x)
            send_counts[g] = __ldg(offsets + (g + 1) * per) - __ldg(offsets + g * per);
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < n; r += warps) {
        if (lane == 0) {
            int lo = 0, hi = E;  // expert of row r: largest e with offsets[e] <= r
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (__ldg(offsets + mid) <= r)
                    lo = mid;
                else
                    hi = mid;
            }
            send_local[r] = lo - (lo / per) * per;
        }
        const uint4 *src = reinterpret_cast<const uint4 *>(x + (int64_t)(__ldg(src_row + r) / k) * H);
        uint4 *dst = reinterpret_cast<uint4 *>(send_x + r * H);
        for (int c = lane; c < H / 8; c += 32)
            dst[c] = __ldg(src + c);
    }
}

// dst[i] = src[idx[i]] for rows of H floats: one warp per row, 16-byte copies.
__global__ void __launch_bounds__(256) gather_rows_kernel(const float *__restrict__ src,
                                                          const int32_t *__restrict__ idx, int n, int H,
                                                          float *__restrict__ dst)
{
    grid_dep_wait();  // the preceding kernel's results (chained launch)
    grid_dep_launch();
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t i = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); i < n; i += warps) {
        const float4 *s = reinterpret_cast<const float4 *>(src + (int64_t)__ldg(idx + i) * H);
        float4 *d = reinterpret_cast<float4 *>(dst + i * H);
        for (int c = lane; c < H / 4; c += 32)
            d[c] = __ldg(s + c);
    }
}

// Receiver workspace: [FFN workspace (status word first) | offsets | src_row |
// dst_of | grouping scratch | y_perm].
struct EpWs {
    void *ffn;
    int32_t *offsets, *src_row, *dst_of, *scratch;
    float *y_perm;
};

int64_t ep_ws_layout(int n, int E_local, int H, int I, EpWs *ws, void *base)
{
    int64_t off = 0;
    auto take = [&](int64_t bytes) {
        const int64_t o = off;
        off = align256(off + bytes);
        return o;
    };
    const int64_t o_ffn = take(ffn_workspace_bytes(n, 1, E_local, H, I));
    const int64_t o_off = take((int64_t)(E_local + 1) * 4);
    const int64_t o_src = take((int64_t)n * 4);
    const int64_t o_dst = take((int64_t)n * 4);
    const int64_t o_scr = take(permute_scratch_ints(n, E_local) * 4);
    const int64_t o_yp = take((int64_t)n * H * 4);
    if (ws && base) {
        uint8_t *b = static_cast<uint8_t *>(base);
        ws->ffn = b + o_ffn;
        ws->offsets = reinterpret_cast<int32_t *>(b + o_off);
        ws->src_row = reinterpret_cast<int32_t *>(b + o_src);
        ws->dst_of = reinterpret_cast<int32_t *>(b + o_dst);
        ws->scratch = reinterpret_cast<int32_t *>(b + o_scr);
        ws->y_perm = reinterpret_cast<float *>(b + o_yp);
    }
    return off;
}

int rows_grid(int64_t n)
{
    const int64_t blocks = (n + 7) / 8;
    const int64_t cap = (int64_t)num_sms() * 8;
    return (int)(blocks < 1 ? 1 : (blocks > cap ? cap : blocks));
}

}  // namespace
}  // namespace mxmoe

using namespace mxmoe;

extern "C" MXMOE_API int mxmoe_ep_dispatch(const void *x, const int32_t *offsets, const int32_t *src_row, int T,
                                           int k, int E, int G, int H, void *send_x, int32_t *send_local,
                                           int32_t *send_counts, void *stream)
{
    if (T < 0 || k < 1 || k > 32 || E < 1 || E > 1024 || G < 1 || E % G || H <= 0 || H % 8 ||
        (int64_t)T * k > (1 << 24))
        return fail(MXMOE_ERR_INVALID_SHAPE,
                    "mxmoe_ep_dispatch: T=%d k=%d E=%d G=%d H=%d (need E <= 1024 a multiple of G, H %% 8 == 0, "
                    "T*k <= 2^24)",
                    T, k, E, G, H);
    if (!offsets || !send_counts || (T > 0 && (!x || !src_row || !send_x || !send_local)))
        return fail(MXMOE_ERR_NULL, "mxmoe_ep_dispatch: NULL pointer");
    if ((T > 0 && (!aligned16(x) || !aligned16(send_x))))
        return fail(MXMOE_ERR_ALIGNMENT, "mxmoe_ep_dispatch: x and send_x need 16-byte alignment");
    if (int rc = check_device())
        return rc;
    const int n = T * k;
    if (n == 0) {  // nothing to send (and mxmoe_permute wrote no offsets)
        if (cudaMemsetAsync(send_counts, 0, sizeof(int32_t) * G, (cudaStream_t)stream) != cudaSuccess)
            return fail(MXMOE_ERR_CUDA, "mxmoe_ep_dispatch: cannot clear send_counts");
        return MXMOE_OK;
    }
    return launch_kernel("ep_dispatch_kernel", ep_dispatch_kernel, rows_grid(n), 256, 0, (cudaStream_t)stream,
                         static_cast<const uint16_t *>(x), offsets, src_row, n, k, E, G, H,
                         static_cast<uint16_t *>(send_x), send_local, send_counts);
}

extern "C" MXMOE_API int64_t mxmoe_ep_workspace_size(int n_recv, int E_local, int H, int I)
{
    if (n_recv < 0 || !ffn_shapes_ok(n_recv, 1, E_local, H, I))
        return -1;
    return ep_ws_layout(n_recv, E_local, H, I, nullptr, nullptr);
}

extern "C" MXMOE_API int mxmoe_ep_expert_ffn(const void *x_recv, const int32_t *recv_local, int n_recv, int E_local,
                                             int H, int I, const void *prepacked_local, float *y_recv,
                                             void *workspace, int64_t workspace_bytes, void *stream)
{
    if (n_recv < 0 || !ffn_shapes_ok(n_recv, 1, E_local, H, I))
        return fail(MXMOE_ERR_INVALID_SHAPE,
                    "mxmoe_ep_expert_ffn: n_recv=%d E_local=%d H=%d I=%d (the expert FFN's shapes with k = 1)",
                    n_recv, E_local, H, I);
    const int64_t need = ep_ws_layout(n_recv, E_local, H, I, nullptr, nullptr);
    if (!workspace || workspace_bytes < need)
        return fail(MXMOE_ERR_WORKSPACE, "mxmoe_ep_expert_ffn: workspace of %lld bytes, need %lld",
                    (long long)workspace_bytes, (long long)need);
    if (reinterpret_cast<uintptr_t>(workspace) & 255)
        return fail(MXMOE_ERR_ALIGNMENT, "mxmoe_ep_expert_ffn: workspace needs 256-byte alignment");
    if (n_recv == 0)
        return MXMOE_OK;
    if (!x_recv || !recv_local || !prepacked_local || !y_recv)
        return fail(MXMOE_ERR_NULL, "mxmoe_ep_expert_ffn: NULL pointer");
    if (!aligned16(x_recv) || !aligned16(y_recv) || (reinterpret_cast<uintptr_t>(prepacked_local) & 31))
        return fail(MXMOE_ERR_ALIGNMENT,
                    "mxmoe_ep_expert_ffn: x_recv and y_recv need 16-byte, prepacked_local 32-byte alignment");
    if (int rc = check_device())
        return rc;
    EpWs ws;
    ep_ws_layout(n_recv, E_local, H, I, &ws, workspace);
    cudaStream_t st = (cudaStream_t)stream;
    ChainScope chain;
    // group the received rows by local expert (k = 1: row i is pair i)
    if (int rc = run_permute(recv_local, n_recv, 1, E_local, ws.offsets, ws.src_row, ws.dst_of, ws.scratch, st))
        return rc;
    if (int rc = run_expert_ffn(x_recv, ws.offsets, ws.src_row, prepacked_local, n_recv, 1, E_local, H, I, ws.y_perm,
                                ws.ffn, true, st))
        return rc;
    return launch_kernel("gather_rows_kernel", gather_rows_kernel, rows_grid(n_recv), 256, 0, st, ws.y_perm,
                         ws.dst_of, n_recv, H, y_recv);
}
