// api.cu -- error reporting, device checks, workspace sizing, the
// whole-layer entry point and the status read-back of libmxmoe.
#include <stdarg.h>
#include <stdio.h>

#include <mutex>

#include "common.cuh"

namespace mxmoe {

static thread_local char g_err[512] = "";

// SM count of the current device (the persistent grids' size), cached per thread.
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

// cuTensorMapEncodeTiled from the driver, looked up once.
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


int fail(int code, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return code;
}

namespace {
thread_local int t_chain_depth = 0;
thread_local bool t_chain_started = false;
}  // namespace

ChainScope::ChainScope()
{
    if (t_chain_depth++ == 0)
        t_chain_started = false;
}

ChainScope::~ChainScope() { --t_chain_depth; }

bool chain_next()
{
    const bool chained = t_chain_depth > 0 && t_chain_started;
    t_chain_started = true;
    return chained;
}

int check_launch(const char *what)
{
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return fail(MXMOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return MXMOE_OK;
}

int check_device()
{
    static thread_local int cached_dev = -2, cached_ok = 0;
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return fail(MXMOE_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev != cached_dev) {
        int major = 0;
        e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        if (e != cudaSuccess)
            return fail(MXMOE_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
        cached_ok = (major == 10);
        cached_dev = dev;
    }
    if (!cached_ok)
        return fail(MXMOE_ERR_DEVICE, "device %d is not compute capability 10.x (sm_100a build)", dev);
    return MXMOE_OK;
}

// defined in ffn.cu
int run_expert_ffn(const void *x, const int32_t *offsets, const int32_t *src_row, const void *prepacked, int T,
                   int k, int E, int H, int I, float *y_perm, void *workspace, bool clear_status, cudaStream_t st);
int run_combine(const float *y_perm, const int32_t *dst_of, const float *w, int T, int k, int H, float *y,
                cudaStream_t st);
int64_t ffn_workspace_bytes(int T, int k, int E, int H, int I);
int run_expert_ffn_fp8(const void *x, const int32_t *offsets, const int32_t *src_row, const void *prepacked, int T,
                       int k, int E, int H, int I, float *y_perm, void *workspace, bool clear_status, cudaStream_t st);
int64_t ffn_workspace_bytes_fp8(int T, int k, int E, int H, int I);
bool fused_layer_ok(int T, int k, int E, int H, int I);
int run_fused_layer(const void *x, const void *wg, const float *bias, const void *prepacked, int T, int H, int I,
                    int E, int k, int nsplit, float *partials, int32_t *ids, float *w, int32_t *offsets,
                    int32_t *src_row, int32_t *dst_of, float *y_perm, float *y, void *ffn_ws, cudaStream_t st);
int validate_ffn_shapes(int T, int k, int E, int H, int I);
bool ffn_shapes_ok(int T, int k, int E, int H, int I);
int router_splits(int T, int H, int E);
int64_t permute_scratch_ints(int n, int E);
int run_permute(const int32_t *ids, int T, int k, int E, int32_t *offsets, int32_t *src_row, int32_t *dst_of,
                int32_t *scratch, cudaStream_t st);
bool front_ok(int T, int k, int E, int H, int I);
int run_layer_front(const void *x, const void *wg, const float *bias, const void *prepacked, int T, int H, int I,
                    int E, int k, int nsplit, float *partials, int32_t *ids, float *w, int32_t *offsets,
                    int32_t *src_row, int32_t *dst_of, float *y_perm, float *y, void *ffn_ws, cudaStream_t st);
int run_router_and_route(const void *x, const void *wg, const float *bias, int T, int H, int E, int k,
                         float *partials, int nsplit, int32_t *ids, float *w, int *status, cudaStream_t st);

namespace {

// Layer workspace: the FFN workspace first (so the status word sits at offset
// 0), then logits, routing and grouping arrays and the per-pair outputs.
struct LayerWs {
    void *ffn;
    float *logits;
    int32_t *ids;
    float *w;
    int32_t *offsets, *src_row, *dst_of;
    int32_t *permute_scratch;
    float *y_perm;
};

int64_t layer_ws_layout(int T, int H, int I, int E, int k, LayerWs *ws, void *base, bool fp8 = false)
{
    int64_t off = 0;
    auto take = [&](int64_t bytes) {
        int64_t o = off;
        off = align256(off + bytes);
        return o;
    };
    const int64_t n = (int64_t)T * k;
    const int64_t o_ffn = take(fp8 ? ffn_workspace_bytes_fp8(T, k, E, H, I) : ffn_workspace_bytes(T, k, E, H, I));
    const int64_t o_logits = take((int64_t)router_splits(T, H, E) * T * E * 4);
    const int64_t o_ids = take(n * 4);
    const int64_t o_w = take(n * 4);
    const int64_t o_off = take((int64_t)(E + 1) * 4);
    const int64_t o_src = take(n * 4);
    const int64_t o_dst = take(n * 4);
    const int64_t o_pm = take(permute_scratch_ints((int)n, E) * 4);
    const int64_t o_yp = take(n * H * 4);
    if (ws && base) {
        uint8_t *b = static_cast<uint8_t *>(base);
        ws->ffn = b + o_ffn;
        ws->logits = reinterpret_cast<float *>(b + o_logits);
        ws->ids = reinterpret_cast<int32_t *>(b + o_ids);
        ws->w = reinterpret_cast<float *>(b + o_w);
        ws->offsets = reinterpret_cast<int32_t *>(b + o_off);
        ws->src_row = reinterpret_cast<int32_t *>(b + o_src);
        ws->dst_of = reinterpret_cast<int32_t *>(b + o_dst);
        ws->permute_scratch = reinterpret_cast<int32_t *>(b + o_pm);
        ws->y_perm = reinterpret_cast<float *>(b + o_yp);
    }
    return off;
}

}  // namespace
}  // namespace mxmoe

using namespace mxmoe;

extern "C" MXMOE_API const char *mxmoe_version(void) { return "mxmoe 0.1.0 (sm_100a)"; }

extern "C" MXMOE_API const char *mxmoe_last_error(void) { return g_err; }

// Token limit of the layer and of the combine: one grid row per token.
constexpr int kMaxLayerTokens = 65535;

extern "C" MXMOE_API int64_t mxmoe_workspace_size(int T, int H, int I, int E, int k)
{
    // exactly the shapes mxmoe_layer_forward accepts
    if (T > kMaxLayerTokens || k > E || !ffn_shapes_ok(T, k, E, H, I))
        return -1;
    return layer_ws_layout(T, H, I, E, k, nullptr, nullptr);
}

namespace {
// Token counts up to which mxmoe_layer_forward runs the whole layer as one
// persistent kernel. None: measured on one verify block (8 tokens), the
// persistent kernel's grid-wide barriers cost about as much as the chained
// launches' gaps, which programmatic dependent launch already hides (0.2494
// vs 0.2459 ms per layer step), so the chained launches stay the default.
constexpr int kPersistentMaxTokens = 0;

enum class LayerPath { kAuto, kChained, kPersistent };

// The whole layer; fp8 selects the FP8-weight expert FFN (prepacked by
// mxmoe_prepack_experts_fp8) instead of the MXFP4 one; path picks the chained
// launches or the persistent kernel (kAuto: by size).
int layer_forward(const char *fn, bool fp8, LayerPath path, const void *x, const void *wg, const float *bias, const void *prepacked,
                  int T, int H, int I, int E, int k, float *y, int32_t *ids_out, float *w_out, void *workspace,
                  int64_t workspace_bytes, void *stream)
{
    if (k > E)
        return fail(MXMOE_ERR_INVALID_SHAPE, "%s: k=%d > E=%d", fn, k, E);
    if (T > kMaxLayerTokens)
        return fail(MXMOE_ERR_INVALID_SHAPE, "%s: T=%d > %d (the combine's grid)", fn, T, kMaxLayerTokens);
    if (int rc = validate_ffn_shapes(T, k, E, H, I))
        return rc;
    const int64_t need = layer_ws_layout(T, H, I, E, k, nullptr, nullptr, fp8);
    if (!workspace || workspace_bytes < need)
        return fail(MXMOE_ERR_WORKSPACE, "%s: workspace of %lld bytes, need %lld", fn, (long long)workspace_bytes,
                    (long long)need);
    if (T == 0)
        return MXMOE_OK;
    if (!x || !wg || !prepacked || !y)
        return fail(MXMOE_ERR_NULL, "%s: NULL pointer", fn);
    if (!aligned16(x) || !aligned16(wg) || !aligned16(prepacked) || !aligned16(y) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255))
        return fail(MXMOE_ERR_ALIGNMENT, "%s: x, wg, prepacked, y need 16-byte and workspace 256-byte alignment", fn);
    if (path == LayerPath::kPersistent && (fp8 || !fused_layer_ok(T, k, E, H, I)))
        return fail(MXMOE_ERR_INVALID_SHAPE,
                    "%s: T=%d k=%d E=%d (the persistent layer takes 1 <= T <= 256, T*k <= 4096, k <= E <= 384)", fn,
                    T, k, E);
    if (int rc = check_device())
        return rc;
    LayerWs ws;
    layer_ws_layout(T, H, I, E, k, &ws, workspace, fp8);
    int32_t *ids = ids_out ? ids_out : ws.ids;
    float *w = w_out ? w_out : ws.w;
    cudaStream_t st = (cudaStream_t)stream;
    const bool persistent = path == LayerPath::kPersistent ||
                            (path == LayerPath::kAuto && !fp8 && T <= kPersistentMaxTokens && fused_layer_ok(T, k, E, H, I));
    if (persistent)
        return run_fused_layer(x, wg, bias, prepacked, T, H, I, E, k, router_splits(T, H, E), ws.logits, ids, w,
                               ws.offsets, ws.src_row, ws.dst_of, ws.y_perm, y, ws.ffn, st);
    // decode-sized steps: router, routing, grouping and the activation terms in one cooperative launch, then the
    // FFN stages and the combine chained (mxmoe_layer_forward_chained keeps one launch per step)
    if (path == LayerPath::kAuto && !fp8 && front_ok(T, k, E, H, I))
        return run_layer_front(x, wg, bias, prepacked, T, H, I, E, k, router_splits(T, H, E), ws.logits, ids, w,
                               ws.offsets, ws.src_row, ws.dst_of, ws.y_perm, y, ws.ffn, st);
    // one status record for the whole layer (the FFN workspace's first word): cleared here, so that a timeout
    // of the router kernel survives to mxmoe_read_status
    int *status = static_cast<int *>(ws.ffn);
    if (cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess)
        return fail(MXMOE_ERR_CUDA, "%s: cannot clear the status word", fn);
    ChainScope chain;  // the router GEMM starts after the clear; every later kernel is chained
    if (int rc = run_router_and_route(x, wg, bias, T, H, E, k, ws.logits, router_splits(T, H, E), ids, w, status,
                                      st))
        return rc;
    if (int rc = run_permute(ids, T, k, E, ws.offsets, ws.src_row, ws.dst_of, ws.permute_scratch, st))
        return rc;
    if (int rc = fp8 ? run_expert_ffn_fp8(x, ws.offsets, ws.src_row, prepacked, T, k, E, H, I, ws.y_perm, ws.ffn,
                                          false, st)
                     : run_expert_ffn(x, ws.offsets, ws.src_row, prepacked, T, k, E, H, I, ws.y_perm, ws.ffn, false,
                                      st))
        return rc;
    return run_combine(ws.y_perm, ws.dst_of, w, T, k, H, y, st);
}
}  // namespace

extern "C" MXMOE_API int mxmoe_layer_forward(const void *x, const void *wg, const float *bias, const void *prepacked,
                                             int T, int H, int I, int E, int k, float *y, int32_t *ids_out,
                                             float *w_out, void *workspace, int64_t workspace_bytes, void *stream)
{
    return layer_forward("mxmoe_layer_forward", false, LayerPath::kAuto, x, wg, bias, prepacked, T, H, I, E, k, y,
                         ids_out, w_out, workspace, workspace_bytes, stream);
}

extern "C" MXMOE_API int mxmoe_layer_forward_chained(const void *x, const void *wg, const float *bias,
                                                     const void *prepacked, int T, int H, int I, int E, int k, float *y,
                                                     int32_t *ids_out, float *w_out, void *workspace,
                                                     int64_t workspace_bytes, void *stream)
{
    return layer_forward("mxmoe_layer_forward_chained", false, LayerPath::kChained, x, wg, bias, prepacked, T, H, I,
                         E, k, y, ids_out, w_out, workspace, workspace_bytes, stream);
}

extern "C" MXMOE_API int mxmoe_layer_forward_persistent(const void *x, const void *wg, const float *bias,
                                                        const void *prepacked, int T, int H, int I, int E, int k,
                                                        float *y, int32_t *ids_out, float *w_out, void *workspace,
                                                        int64_t workspace_bytes, void *stream)
{
    return layer_forward("mxmoe_layer_forward_persistent", false, LayerPath::kPersistent, x, wg, bias, prepacked, T,
                         H, I, E, k, y, ids_out, w_out, workspace, workspace_bytes, stream);
}

extern "C" MXMOE_API int64_t mxmoe_workspace_size_fp8(int T, int H, int I, int E, int k)
{
    if (T > kMaxLayerTokens || k > E || !ffn_shapes_ok(T, k, E, H, I))
        return -1;
    return layer_ws_layout(T, H, I, E, k, nullptr, nullptr, true);
}

extern "C" MXMOE_API int mxmoe_layer_forward_fp8(const void *x, const void *wg, const float *bias,
                                                 const void *prepacked, int T, int H, int I, int E, int k, float *y,
                                                 int32_t *ids_out, float *w_out, void *workspace,
                                                 int64_t workspace_bytes, void *stream)
{
    return layer_forward("mxmoe_layer_forward_fp8", true, LayerPath::kChained, x, wg, bias, prepacked, T, H, I, E, k,
                         y, ids_out, w_out, workspace, workspace_bytes, stream);
}

namespace mxmoe {
namespace {
// One thread waits on an mbarrier that nothing arrives on (phase 0 of a fresh
// barrier with one expected arrival never completes) until the bounded wait
// gives up.
__global__ void wait_timeout_kernel(int *status, uint64_t limit_ns)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0)
        *status = mbar_wait_bounded(&bar, 0, limit_ns) ? MXMOE_OK : MXMOE_ERR_TIMEOUT;
}
}  // namespace
}  // namespace mxmoe

extern "C" MXMOE_API int mxmoe_selftest_wait_timeout(int *status, int limit_us, void *stream)
{
    if (!status)
        return fail(MXMOE_ERR_NULL, "mxmoe_selftest_wait_timeout: NULL status");
    if (limit_us < 1 || limit_us > 1000000)
        return fail(MXMOE_ERR_INVALID_SHAPE, "mxmoe_selftest_wait_timeout: limit_us=%d (1 .. 1000000)", limit_us);
    if (int rc = check_device())
        return rc;
    wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(status, (uint64_t)limit_us * 1000ull);
    return check_launch("wait_timeout_kernel");
}

extern "C" MXMOE_API int mxmoe_read_status(const void *workspace, int *status, void *stream)
{
    if (!workspace || !status)
        return fail(MXMOE_ERR_NULL, "mxmoe_read_status: NULL pointer");
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess)
        return fail(MXMOE_ERR_CUDA, "mxmoe_read_status: %s", cudaGetErrorString(e));
    int v = 0;
    e = cudaMemcpy(&v, workspace, sizeof v, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess)
        return fail(MXMOE_ERR_CUDA, "mxmoe_read_status: %s", cudaGetErrorString(e));
    *status = v;
    return MXMOE_OK;
}
