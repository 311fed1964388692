// router_tc.cu -- the router GEMM on tcgen05 tensor cores, for many tokens.
//
// Pages: nxbn.cn MiMo-V2.5-Pro-FP4-DFlash article, architecture section (384
// experts, hidden size 6144): logits[t, e] = sum_k x[t, k] Wg[e, k] + bias[e]
// in fp32 from bf16 operands. Every bf16 product is exact in fp32; only the
// order of the fp32 additions differs from the small-T kernel.
//
// A work item is (128 experts, 256 tokens, one of nsplit K ranges): Wg rows
// are the MMA's M (A operand), tokens its N (B operand), so that the
// accumulator lane is an expert and the epilogue's stores of one token row are
// 32 consecutive experts. One CTA per item: a producer thread streams A and B
// steps of 64 values of K by TMA (128-byte swizzle) through a 4-stage ring,
// one thread issues the MMAs (kind::f16, 4 per step) into a 256-column
// accumulator, and the four warps then store fp32 logits (with the bias only
// when nsplit == 1: otherwise the routing kernel adds the split partial sums
// in order and then the bias). All waits are bounded; a timeout sets
// MXMOE_ERR_TIMEOUT in *status when status is given.
#include <algorithm>

#include <cudaTypedefs.h>

#include "common.cuh"
#include "tcgen05.cuh"

namespace mxmoe {
namespace {

constexpr uint64_t kRtWaitNs = 2000000000ull;
constexpr int kRtStages = 4;
constexpr int kRtK = 64;                // K per step
constexpr int kRtExp = 128, kRtTok = 256;
constexpr int kRtABytes = kRtExp * 128;  // 128 experts x 64 bf16
constexpr int kRtBBytes = kRtTok * 128;  // 256 tokens x 64 bf16
constexpr size_t kRtOffBar = (size_t)kRtStages * (kRtABytes + kRtBBytes);
constexpr size_t kRtSmem = 1024 + kRtOffBar + (2 * kRtStages + 1) * 8 + 16;

struct RtParams {
    int T, E, ksteps;  // K steps per split
    int etiles, ttiles;
    const float *bias;  // used when out has one split
    int nsplit;
    float *out;  // [nsplit][T][E]
    int *status;
};

__global__ void __launch_bounds__(128, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const RtParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem, *sB = smem + (size_t)kRtStages * kRtABytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kRtOffBar);
    uint64_t *empty = full + kRtStages;
    uint64_t *accfull = empty + kRtStages;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(accfull + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);

    grid_dep_wait();  // the preceding kernel's results (chained launch); the next one starts as CTAs exit
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // item: expert tile fastest, so that the CTAs of one token tile run together and share x in L2
    const int et = blockIdx.x % p.etiles;
    const int tt = (blockIdx.x / p.etiles) % p.ttiles;
    const int z = blockIdx.x / (p.etiles * p.ttiles);
    const int e0 = et * kRtExp, t0 = tt * kRtTok, k0 = z * p.ksteps;
    if (tid == 0) {
        for (int s = 0; s < kRtStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accfull, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1)
        tc::alloc(tslot, 256);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *tslot;
    const int nk = p.ksteps;

    if (warp == 0 && lane == 0) {
        // producer
        const uint64_t pol_a = policy_evict_last(), pol_b = policy_evict_normal();
        int s = 0;
        uint32_t ph = 0;
        int issued = 0;
        for (int ks = 0; ks < nk; ++ks) {
            if (*abort_flag || !mbar_wait_bounded(&empty[s], ph ^ 1u, kRtWaitNs)) {
                set_status(p.status, MXMOE_ERR_TIMEOUT);
                *abort_flag = 1;
                break;
            }
            mbar_arrive_expect_tx(&full[s], (uint32_t)(kRtABytes + kRtBBytes));
            tc::tma_load_2d(sA + (size_t)s * kRtABytes, &tmA, kRtK * (k0 + ks), e0, &full[s], pol_a);
            tc::tma_load_2d(sB + (size_t)s * kRtBBytes, &tmB, kRtK * (k0 + ks), t0, &full[s], pol_b);
            ++issued;
            if (++s == kRtStages) {
                s = 0;
                ph ^= 1u;
            }
        }
        for (int f = issued > kRtStages ? issued - kRtStages : 0; f < issued; ++f)  // no copy in flight at exit
            if (!mbar_wait_bounded(&full[f % kRtStages], (uint32_t)((f / kRtStages) & 1), kRtWaitNs)) {
                set_status(p.status, MXMOE_ERR_TIMEOUT);
                break;
            }
    } else if (warp == 1 && lane == 0) {
        // MMA: D[e][t] += Wg[e][k] x[t][k]
        const uint32_t idesc = tc::idesc_bf16(kRtTok);
        int s = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int ks = 0; ks < nk; ++ks) {
            if (*abort_flag || !mbar_wait_bounded(&full[s], ph, kRtWaitNs)) {
                set_status(p.status, MXMOE_ERR_TIMEOUT);
                *abort_flag = 1;
                ok = false;
                break;
            }
            tc::fence_after();
            const uint32_t a_base = smem_u32(sA + (size_t)s * kRtABytes);
            const uint32_t b_base = smem_u32(sB + (size_t)s * kRtBBytes);
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4)
                tc::mma_bf16(tmem, tc::smem_desc(a_base + 32 * k4, 16, 1024, 2),
                             tc::smem_desc(b_base + 32 * k4, 16, 1024, 2), idesc, (ks > 0 || k4 > 0) ? 1u : 0u);
            tc::commit(&empty[s]);
            if (++s == kRtStages) {
                s = 0;
                ph ^= 1u;
            }
        }
        tc::commit(accfull);  // also when aborted: every issued MMA completes before the epilogue
        if (!ok)
            set_status(p.status, MXMOE_ERR_TIMEOUT);
    }
    __syncwarp();
    // epilogue: warp q holds experts e0 + 32q + lane; accumulator column n is token t0 + n
    {
        int okv = 1;
        if (lane == 0 && !mbar_wait_bounded(accfull, 0, kRtWaitNs)) {
            set_status(p.status, MXMOE_ERR_TIMEOUT);
            okv = 0;
        }
        const bool ok = __shfl_sync(0xFFFFFFFFu, okv, 0) != 0 && nk > 0;
        tc::fence_after();
        const int e = e0 + 32 * warp + lane;
        const bool e_ok = e < p.E;
        const float b = (p.nsplit == 1 && p.bias && e_ok) ? p.bias[e] : 0.f;
        float *dst = p.out + (size_t)z * p.T * p.E + (size_t)t0 * p.E + e;
        const int nt = min(kRtTok, p.T - t0);
        for (int n0 = 0; n0 < nt && ok; n0 += 32) {
            float v[32];
            tc::ld_32x32b_x32(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)n0, v);
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (e_ok && n0 + j < nt)
                    dst[(size_t)(n0 + j) * p.E] = v[j] + b;
        }
    }
    tc::fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after();
        tc::dealloc(tmem, 256);
    }
}

int encode_bf16_rows(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows, uint32_t box_rows,
                     const char *what)
{
    auto enc = tensor_map_encoder();
    if (!enc)
        return fail(MXMOE_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kRtK, box_rows}, es[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(MXMOE_ERR_CUDA, "cuTensorMapEncodeTiled (%s) failed: %d", what, (int)r);
    return MXMOE_OK;
}

}  // namespace

// Token counts from which the router GEMM runs on tcgen05 (H a multiple of 64).
constexpr int kRouterTcMinT = 512;
bool use_router_tc(int T, int H) { return T >= kRouterTcMinT && H % kRtK == 0; }

// K splits for the tcgen05 router: enough items to cover the GPU, each split
// at least 8 K steps.
int router_tc_splits(int T, int H, int E)
{
    const int64_t base = (int64_t)((E + kRtExp - 1) / kRtExp) * ((T + kRtTok - 1) / kRtTok);
    const int nks = H / kRtK;
    int z = (int)std::max<int64_t>(1, (int64_t)num_sms() / std::max<int64_t>(base, 1));
    z = std::min(std::min(z, 8), std::max(1, nks / 8));
    while (z > 1 && nks % z)  // equal splits
        --z;
    return z;
}

// logits (nsplit == 1: with the bias) or per-split partial sums into out
// [nsplit][T][E]. x [T][H], wg [E][H] bf16, 16-byte aligned.
int run_router_gemm_tc(const void *x, const void *wg, const float *bias, int T, int H, int E, float *out, int nsplit,
                       int *status, cudaStream_t st)
{
    CUtensorMap tmA, tmB;
    if (int rc = encode_bf16_rows(&tmA, wg, (uint64_t)H, (uint64_t)E, kRtExp, "router weights"))
        return rc;
    if (int rc = encode_bf16_rows(&tmB, x, (uint64_t)H, (uint64_t)T, kRtTok, "router x"))
        return rc;
    static thread_local int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        if (cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRtSmem) !=
            cudaSuccess)
            return fail(MXMOE_ERR_CUDA, "router_tc_kernel: cannot reserve %zu bytes of shared memory", kRtSmem);
        configured_dev = dev;
    }
    RtParams p{};
    p.T = T;
    p.E = E;
    p.ksteps = H / kRtK / nsplit;
    p.etiles = (E + kRtExp - 1) / kRtExp;
    p.ttiles = (T + kRtTok - 1) / kRtTok;
    p.bias = bias;
    p.nsplit = nsplit;
    p.out = out;
    p.status = status;
    const int grid = p.etiles * p.ttiles * nsplit;
    return launch_kernel("router_tc_kernel", router_tc_kernel, grid, 128, kRtSmem, st, tmA, tmB, p);
}

}  // namespace mxmoe
