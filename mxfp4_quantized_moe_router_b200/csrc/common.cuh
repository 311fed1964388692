// common.cuh -- shared device/host helpers of libmxmoe (sm_100a only).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include "../../include/mxmoe.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libmxmoe is built for sm_100a only"
#endif

namespace mxmoe {

// ---------------------------------------------------------------------------
// SM count of the current device and the driver's cuTensorMapEncodeTiled
// (defined in api.cu)
int num_sms();
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// Host-side error reporting (defined in api.cu)
// ---------------------------------------------------------------------------
int fail(int code, const char *fmt, ...);
int check_launch(const char *what);
int check_device();  // MXMOE_ERR_DEVICE unless the current device is CC 10.x

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------------------------
// Launch chains (programmatic dependent launch). Inside a ChainScope -- one
// per C entry point that launches kernels -- every kernel started through
// launch_kernel after the first may begin while its predecessor on the stream
// is still running. Every such kernel runs grid_dep_wait() in each thread that
// touches its predecessor's results (and in each CTA before it exits), and
// grid_dep_launch() only after that wait. So when a chained kernel begins,
// every kernel before its predecessor has completed: what it reads before its
// own wait (routing offsets, pass tables, weights) was written by those. The
// first kernel of a scope is launched plainly, after all earlier work on the
// stream, so a chain never overlaps the caller's own kernels.
// ---------------------------------------------------------------------------
struct ChainScope {
    ChainScope();
    ~ChainScope();
    ChainScope(const ChainScope &) = delete;
    ChainScope &operator=(const ChainScope &) = delete;
};
bool chain_next();  // whether the next launch may overlap its predecessor; marks the chain as started

// Launches kernel<<<grid, block, smem, st>>>(args...) (chained when inside a
// ChainScope after its first launch); MXMOE_OK or MXMOE_ERR_CUDA naming what.
template <typename... P, typename... A>
int launch_kernel(const char *what, void (*kernel)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                  A &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    if (chain_next()) {
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<A &&>(args)...);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(MXMOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    }
    return check_launch(what);
}

inline int64_t align256(int64_t v) { return (v + 255) & ~int64_t(255); }

// ---------------------------------------------------------------------------
// Device status word (first 16 bytes of a workspace)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void set_status(int *status, int code)
{
    if (status)
        atomicCAS(status, 0, code);
}

#if defined(__CUDACC__)

// Programmatic dependent launch: grid_dep_wait() returns once the kernel this
// one was chained after has completed and its writes are visible (at once
// when it was launched plainly); grid_dep_launch() lets the next chained
// kernel start its own prologue.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ uint64_t globaltimer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------------------
// mbarrier (shared::cta) and 1-D bulk async copies
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// try_wait that may suspend the thread for up to `hint_ns` nanoseconds while
// the phase is incomplete, instead of returning at once: a waiting thread then
// takes no issue slots from the warps doing work.
__device__ __forceinline__ bool mbar_try_wait_suspend(uint64_t *bar, uint32_t parity, uint32_t hint_ns)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Bounded wait: gives up after about `limit_ns` nanoseconds and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, uint64_t limit_ns)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait_suspend(bar, parity, 20000u))
            return true;
        if (globaltimer_ns() - t0 > limit_ns)
            return false;
    }
}

// Global -> shared bulk copy with an L2 cache policy, completion signalled on
// `bar` (complete_tx). dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s_hint(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                              uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], "
        "%4;" ::"r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t policy_evict_normal()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t policy_evict_last()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// Named barrier over `nthreads` threads (multiple of 32) of the block.
__device__ __forceinline__ void named_bar_sync(int id, int nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------------------
// Tensor-core and conversion primitives
// ---------------------------------------------------------------------------
// d = a(16x16 bf16, row) * b(16x8 bf16, col) + c, fp32 accumulate (mma.sync).
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                                               const float (&c)[4])
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]),
          "f"(c[3]));
}

// E8M0 scale byte -> float 2^(S-127) (S = 0 is the subnormal 2^-127).
__device__ __forceinline__ float e8m0_to_float(uint32_t s)
{
    return __uint_as_float(s ? (s << 23) : 0x00400000u);
}

#endif  // __CUDACC__

}  // namespace mxmoe
