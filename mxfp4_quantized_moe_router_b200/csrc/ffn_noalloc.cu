// ffn_noalloc.cu -- a variant of mxmoe_expert_ffn for callers that cannot
// allocate device memory: its scratch is a fixed static device array inside
// the library instead of a caller-provided workspace.
//
// Who needs it: code whose device memory is entirely owned by some other
// allocator (for example an engine that reserves all free memory for its own
// pool at start-up and forbids further cudaMalloc), and latency-critical
// loops where cudaMalloc/cudaFree, which may synchronise the device, are not
// allowed. Such a caller can pass its inputs and outputs and nothing else.
#include <mutex>

#include <cuda.h>

#include "common.cuh"

namespace mxmoe {
int run_expert_ffn(const void *x, const int32_t *offsets, const int32_t *src_row, const void *prepacked, int T,
                   int k, int E, int H, int I, float *y_perm, void *workspace, bool clear_status, cudaStream_t st);
int64_t ffn_workspace_bytes(int T, int k, int E, int H, int I);
int validate_ffn_shapes(int T, int k, int E, int H, int I);
}  // namespace mxmoe

namespace {

constexpr int64_t kStaticScratchBytes = 8LL << 20;  // 8 MiB per device
constexpr int kMaxDevices = 64;

// The shared scratch. Every GPU on which the library's device code is loaded
// holds these 8 MiB until the process exits. In host code this name is only a
// host-side stand-in: its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_ffn_scratch[kStaticScratchBytes];

std::mutex g_setup_mutex;
// Looked-up addresses, one per device ordinal, each tagged with the CUDA
// context it was looked up in. The array's address belongs to the module
// loaded in that context: after cudaDeviceReset, or in another context on the
// same device, the library's device code is loaded again and the array may sit
// elsewhere, so a lookup made in an earlier context is never reused.
struct ScratchEntry {
    CUcontext ctx;
    void *ptr;
};
ScratchEntry g_scratch[kMaxDevices] = {};

PFN_cuCtxGetCurrent_v4000 ctx_getter()
{
    static std::once_flag once;
    static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    });
    return fn;
}

// The scratch array's device address in the current device's current context.
// The lookup (cudaGetSymbolAddress, which also makes the device's primary
// context current if none is) runs on the first call in each context, under a
// lock; later calls in the same context reuse it.
int scratch_for_current_device(void **out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return mxmoe::fail(MXMOE_ERR_CUDA, "mxmoe_expert_ffn_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices)
        return mxmoe::fail(MXMOE_ERR_DEVICE, "mxmoe_expert_ffn_noalloc: device ordinal %d out of range", dev);
    auto get_ctx = ctx_getter();
    if (!get_ctx)
        return mxmoe::fail(MXMOE_ERR_CUDA, "mxmoe_expert_ffn_noalloc: cuCtxGetCurrent is not available");
    CUcontext ctx = nullptr;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (get_ctx(&ctx) == CUDA_SUCCESS && ctx && ctx == g_scratch[dev].ctx && g_scratch[dev].ptr) {
        *out = g_scratch[dev].ptr;
        return MXMOE_OK;
    }
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_ffn_scratch);
    if (e != cudaSuccess || !p)
        return mxmoe::fail(MXMOE_ERR_CUDA, "mxmoe_expert_ffn_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    ctx = nullptr;
    if (get_ctx(&ctx) != CUDA_SUCCESS || !ctx)
        return mxmoe::fail(MXMOE_ERR_CUDA, "mxmoe_expert_ffn_noalloc: no current CUDA context");
    g_scratch[dev] = {ctx, p};
    *out = p;
    return MXMOE_OK;
}

}  // namespace

extern "C" MXMOE_API int mxmoe_expert_ffn_noalloc(const void *x, const int32_t *offsets, const int32_t *src_row,
                                                  const void *prepacked, int T, int k, int E, int H, int I,
                                                  float *y_perm, int *status, void *stream)
{
    using namespace mxmoe;
    if (int rc = validate_ffn_shapes(T, k, E, H, I))
        return rc;
    const int64_t need = ffn_workspace_bytes(T, k, E, H, I);
    if (need > kStaticScratchBytes)
        return fail(MXMOE_ERR_WORKSPACE,
                    "mxmoe_expert_ffn_noalloc: these sizes need %lld bytes of scratch, more than the fixed %lld "
                    "(use mxmoe_expert_ffn with a workspace)",
                    (long long)need, (long long)kStaticScratchBytes);
    if (T == 0)
        return MXMOE_OK;
    if (!x || !offsets || !src_row || !prepacked || !y_perm)
        return fail(MXMOE_ERR_NULL, "mxmoe_expert_ffn_noalloc: NULL pointer");
    if (!aligned16(x) || (reinterpret_cast<uintptr_t>(prepacked) & 31) || !aligned16(y_perm))
        return fail(MXMOE_ERR_ALIGNMENT,
                    "mxmoe_expert_ffn_noalloc: x and y_perm need 16-byte, prepacked 32-byte alignment");
    if (int rc = check_device())
        return rc;
    void *scratch = nullptr;
    if (int rc = scratch_for_current_device(&scratch))
        return rc;
    cudaStream_t st = (cudaStream_t)stream;
    // The first kernel of the chain clears the status word at the start of the
    // scratch; every other scratch byte that can reach the outputs is written
    // earlier in the same call, so nothing else needs clearing between calls.
    ChainScope chain;
    if (int rc = run_expert_ffn(x, offsets, src_row, prepacked, T, k, E, H, I, y_perm, scratch, true, st))
        return rc;
    if (status) {
        cudaError_t e = cudaMemcpyAsync(status, scratch, sizeof(int), cudaMemcpyDeviceToDevice, st);
        if (e != cudaSuccess)
            return fail(MXMOE_ERR_CUDA, "mxmoe_expert_ffn_noalloc: status copy: %s", cudaGetErrorString(e));
    }
    return MXMOE_OK;
}
