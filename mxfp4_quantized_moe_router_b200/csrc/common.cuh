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

// ---------------------------------------------------------------------------
// Layout constants shared by the prepack and FFN kernels
// ---------------------------------------------------------------------------
constexpr int kBlock = 32;       // MXFP4 block: elements per E8M0 scale
constexpr int kChunkK = 512;     // K elements per streamed chunk (16 k32 blocks)
constexpr int kTileRows = 64;    // weight rows per tile (4 slabs of 16)
constexpr int kConsumerWarps = 8;

// Bytes of one weight chunk covering kw (multiple of 32, <= kChunkK) K
// elements: nibbles 64 rows * kw/2 = 32*kw, then scales 64 rows * kw/32 = 2*kw.
// Inside a chunk, k32 block b owns nibble bytes [1024 b, 1024 b + 1024) and
// scale bytes [32 kw + 64 b, 32 kw + 64 b + 64).
__host__ __device__ constexpr int64_t wchunk_bytes(int kw) { return 34LL * kw; }
__host__ __device__ constexpr int64_t wchunk_nibble_bytes(int kw) { return 32LL * kw; }
// Bytes of a whole weight tile covering K (multiple of 32): 34*K.
__host__ __device__ constexpr int64_t wtile_bytes(int64_t K) { return 34LL * K; }

// Activation row formats.
//  * "x16" (gate/up input): a row of K values is K f16 values, each the bf16
//    input times one power-of-two factor per row; the inverse factors are
//    kept in a separate float array.
//  * "h16" (down input): a row of K values (K multiple of 32) is stored chunk
//    by chunk (chunks of up to kChunkK values); a chunk of kw values is kw
//    f16 values, each pre-multiplied by its 32-value block's power-of-two
//    factor, then kw/32 float inverse factors, padded to a multiple of 16
//    bytes.
__host__ __device__ constexpr int act_scale_bytes(int kw) { return ((kw / 32) * 4 + 15) & ~15; }
__host__ __device__ constexpr int act_chunk_bytes(int kw) { return kw * 2 + act_scale_bytes(kw); }
__host__ __device__ inline int64_t act_row_bytes(int64_t K)
{
    int64_t full = K / kChunkK, rem = K % kChunkK;
    return full * act_chunk_bytes(kChunkK) + (rem ? act_chunk_bytes((int)rem) : 0);
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

// Global -> shared bulk copy, completion signalled on `bar` (complete_tx).
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

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

// Named barrier over `nthreads` threads (multiple of 32).
__device__ __forceinline__ void named_bar_sync(int id, int nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------------------
// Tensor-core and conversion primitives
// ---------------------------------------------------------------------------
// Two E2M1 codes (one byte, element 2j in the low nibble) -> f16x2 (exact;
// the low half holds the low nibble's value).
__device__ __forceinline__ void e2m1x4_to_f16x2x4(uint32_t four_bytes, uint32_t &h0, uint32_t &h1, uint32_t &h2,
                                                  uint32_t &h3)
{
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3)
        : "r"(four_bytes));
}

// d = a(16x16 f16, row) * b(16x8 f16, col) + c, fp32 accumulate.
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                                              const float (&c)[4])
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]),
          "f"(c[3]));
}

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

__device__ __forceinline__ void ldmatrix_x4(uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3,
                                            uint32_t saddr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(saddr));
}

// E8M0 scale byte -> float 2^(S-127) (S = 0 is the subnormal 2^-127).
__device__ __forceinline__ float e8m0_to_float(uint32_t s)
{
    return __uint_as_float(s ? (s << 23) : 0x00400000u);
}

// The four E8M0 bytes of a word as floats 2^(S-127), byte 0 first. Two
// instructions per scale; a zero byte (2^-127) reads as 0.0, a difference of
// at most 6 * 2^-127 per weight.
__device__ __forceinline__ void e8m0x4_to_float(uint32_t w, float &f0, float &f1, float &f2, float &f3)
{
    f0 = __uint_as_float((w << 23) & 0x7F800000u);
    f1 = __uint_as_float((w << 15) & 0x7F800000u);
    f2 = __uint_as_float((w << 7) & 0x7F800000u);
    f3 = __uint_as_float((w >> 1) & 0x7F800000u);
}

// Power-of-two factor that maps a block maximum m (> 0, finite) into
// [2^14, 2^15), and its inverse; exponent clamped so both stay normal floats.
__device__ __forceinline__ void act_block_factor(float m, float &mul, float &inv)
{
    int fl;
    if (m > 0.f) {
        uint32_t b = __float_as_uint(m);
        int be = (int)(b >> 23);
        fl = be ? be - 127 : (31 - __clz((int)(b & 0x7FFFFF))) - 149;
    } else {
        fl = 0;
    }
    fl = max(-100, min(fl, 127));
    mul = __uint_as_float((uint32_t)(127 + 14 - fl) << 23);  // 2^(14 - fl), fl <= 127 -> >= 2^-113
    inv = __uint_as_float((uint32_t)(127 - 14 + fl) << 23);  // 2^(fl - 14), fl >= -100 -> >= 2^-114
}

#endif  // __CUDACC__

}  // namespace mxmoe
