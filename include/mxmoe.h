/*
 * mxmoe.h -- C ABI of libmxmoe.so: the MXFP4 MoE expert layer of a
 * decode/verify step on one NVIDIA B200 (sm_100a).
 *
 * The layer (pages: "MiMo-V2.5-Pro-FP4-DFlash" model card, section 2 "FP4
 * Quantization" -- MoE experts stored as MXFP4 with block size 32, the rest at
 * higher precision; nxbn.cn MiMo-V2.5-Pro-FP4-DFlash article, architecture
 * section -- 384 experts, 8 activated per token, hidden size 6144):
 *
 *   logits = x Wg^T (+ bias)               mxmoe_router_gemm
 *   ids, w = top-k of softmax(logits)      mxmoe_route
 *   group (token, slot) pairs by expert    mxmoe_permute
 *   h = silu(W_gate x) * (W_up x)          mxmoe_ffn_gate_up (stage 1)
 *   y_e = W_down h                         mxmoe_ffn_down (stage 2)
 *   (both stages)                          mxmoe_expert_ffn
 *   y = sum_j w_j y_{e_j}                  mxmoe_combine
 *   all of the above in one call           mxmoe_layer_forward
 * plus the weight-format entry points mxmoe_quantize / mxmoe_dequantize and
 * the kernel-layout re-tiling mxmoe_prepack_experts.
 *
 * Conventions for every entry point:
 *  - Pointers named as device memory must be device (or managed) memory that
 *    the caller owns and keeps alive until the stream work finishes. No entry
 *    point allocates device memory; scratch comes from a caller-provided
 *    workspace sized by the matching *_workspace_size query.
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream). Nothing synchronises the host except
 *    mxmoe_read_status.
 *  - Every call returns an mxmoe_status. Argument problems are detected on the
 *    host before anything is enqueued. On failure mxmoe_last_error() returns a
 *    message for the calling thread.
 *  - bf16 tensors are passed as raw 16-bit words (const void*), row-major.
 *  - Entry points are thread-safe: they keep no host state besides the
 *    per-thread error message.
 */
#ifndef MXMOE_H
#define MXMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MXMOE_API __attribute__((visibility("default")))

enum mxmoe_status {
    MXMOE_OK = 0,
    MXMOE_ERR_INVALID_SHAPE = 1, /* a size is out of range or not a required multiple */
    MXMOE_ERR_ALIGNMENT = 2,     /* a pointer is not 16-byte aligned (bulk copies need it) */
    MXMOE_ERR_NULL = 3,          /* a required pointer is NULL */
    MXMOE_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed */
    MXMOE_ERR_TIMEOUT = 5,       /* device side: a bounded wait gave up (read via mxmoe_read_status) */
    MXMOE_ERR_DEVICE = 6,        /* the current device is not compute capability 10.0 */
    MXMOE_ERR_WORKSPACE = 7      /* workspace NULL or smaller than the size query returns */
};

/* Library version string, e.g. "mxmoe 0.1.0". Never fails. */
MXMOE_API const char *mxmoe_version(void);

/* Message describing the last failing call made by this thread ("" if none).
 * The pointer stays valid until this thread's next failing call. */
MXMOE_API const char *mxmoe_last_error(void);

/* ------------------------------------------------------------------------ */
/* Weight format                                                             */
/* ------------------------------------------------------------------------ */

/* MXFP4 quantiser (model card, section 2: MXFP4, block size 32; the pages fix
 * no scale or rounding rule, so the OCP MX convention is used).
 *   w       device, bf16 [rows, K] row-major.
 *   packed  device, uint8 [rows, K/2]: element 2j of a row in the low nibble
 *           of byte j, element 2j+1 in the high nibble. E2M1 codes: bit 3
 *           sign, bits 2..1 exponent (bias 1), bit 0 mantissa.
 *   scales  device, uint8 [rows, K/32], one E8M0 byte per 32-element block.
 * Per block: e = floor(log2 max|x|) - 2 clamped to [-127, 127] (e = -127 for
 * an all-zero block), scale byte e + 127, each element |x|/2^e rounded to
 * nearest E2M1 with ties to the even mantissa and saturation at 6, sign bit
 * copied. Non-finite inputs are outside the contract.
 * Errors: K % 32 != 0 or rows/K <= 0 -> INVALID_SHAPE; NULL -> NULL;
 * w not 16-byte aligned or K % 8 != 0 -> ALIGNMENT (only the alignment of w
 * matters; packed and scales are written bytewise). */
MXMOE_API int mxmoe_quantize(const void *w, int64_t rows, int64_t K, uint8_t *packed, uint8_t *scales,
                             void *stream);

/* Inverse of the format above: out[r, k] = E2M1(code) * 2^(S - 127) as float.
 *   packed device uint8 [rows, K/2], scales device uint8 [rows, K/32],
 *   out device float [rows, K]. Errors as for mxmoe_quantize. */
MXMOE_API int mxmoe_dequantize(const uint8_t *packed, const uint8_t *scales, int64_t rows, int64_t K, float *out,
                               void *stream);

/* Bytes of the prepacked expert blob for E experts of hidden size H and
 * intermediate size I: E * (2*I*Hp + Hp*Ip) * 17/32 with Hp, Ip = H, I rounded
 * up to multiples of 256, i.e. the bytes of the packed codes plus scales
 * (E * 3 * H * I * 17/32) when H and I are multiples of 256, and those bytes
 * padded with zero codes and zero scale bytes otherwise. Returns -1 unless H and I are positive
 * multiples of 128.
 */
MXMOE_API int64_t mxmoe_prepacked_size(int E, int H, int I);

/* Re-tile canonical MXFP4 expert weights into the layout the tensor-core FFN
 * streams (a pure byte permutation; nothing is re-rounded).
 *   packed13 device uint8 [E, 2I, H/2], sc13 device uint8 [E, 2I, H/32]:
 *            rows 0..I-1 of each expert are the gate projection, rows
 *            I..2I-1 the up projection (each row a K = H vector).
 *   packed2  device uint8 [E, H, I/2], sc2 device uint8 [E, H, I/32]: down
 *            projection (each row a K = I vector).
 *   prepacked device, mxmoe_prepacked_size(E, H, I) bytes, 32-byte aligned.
 * Layout of the blob: [gate/up code boxes][down code boxes][gate/up scale
 * images][down scale images]. A code box is a 256-row tile by 256 values of
 * K: 256 rows of 128 bytes (32 KB), contiguous, boxes ordered by (expert,
 * tile, K chunk). Gate/up tile t holds gate rows 128t .. 128t+127 and then the
 * matching up rows I + 128t .. I + 128t+127; down rows keep their order. The
 * scale images of a box are four 512-byte images ordered (K half h, row half
 * g): byte (r % 32) * 16 + (r / 32) * 4 + kb is the scale of tile row
 * 128g + r, 32-block 4h + kb of the box. K, and the down rows, are padded to
 * multiples of 256 with zero codes and zero scale bytes (no padding when H and
 * I are multiples of 256: the blob is then a byte permutation of the inputs).
 * Errors: shapes as in mxmoe_prepacked_size -> INVALID_SHAPE; NULL -> NULL;
 * prepacked not 32-byte or packed13/packed2 not 16-byte aligned -> ALIGNMENT.
 */
MXMOE_API int mxmoe_prepack_experts(const uint8_t *packed13, const uint8_t *sc13, const uint8_t *packed2,
                                    const uint8_t *sc2, int E, int H, int I, void *prepacked, void *stream);

/* ------------------------------------------------------------------------ */
/* Router                                                                    */
/* ------------------------------------------------------------------------ */

/* Router logits in float32: logits[t, e] = sum_k x[t, k] * Wg[e, k] + bias[e]
 * (products of bf16 values are exact in float32; the sum is float32).
 *   x device bf16 [T, H]; wg device bf16 [E, H]; bias device float [E] or
 *   NULL for no bias; logits device float [T, E].
 * Errors: T < 0, E <= 0, H <= 0 or H % 32 != 0 -> INVALID_SHAPE; x, wg not
 * 16-byte aligned -> ALIGNMENT. T == 0 is a no-op. */
MXMOE_API int mxmoe_router_gemm(const void *x, const void *wg, const float *bias, int T, int H, int E,
                                float *logits, void *stream);

/* Top-k routing (384 experts, 8 per token in the layer on the pages).
 * For each token: the k largest logits, a tie going to the lower expert
 * index, in descending order; weights w_j = exp(l_j - l_max) / sum over the
 * selected k, which equals a softmax over all E renormalised over the k.
 *   logits device float [T, E]; ids device int32 [T, k]; w device float [T, k].
 * Errors: k < 1, k > E, k > 32, E > 4096 or T < 0 -> INVALID_SHAPE. */
MXMOE_API int mxmoe_route(const float *logits, int T, int E, int k, int32_t *ids, float *w, void *stream);

/* Group the T*k (token, slot) pairs by expert (stable), so that each
 * expert's rows are contiguous for the grouped FFN. The pages route every
 * token to 8 of 384 experts (nxbn.cn MiMo-V2.5-Pro-FP4-DFlash article,
 * architecture section) and give no grouping rule; this is the plain
 * counting-sort reading: experts ascending, pairs in (t, j) order within an
 * expert.
 *   ids device int32 [T, k], every id in [0, E).
 *   offsets device int32 [E+1]: pairs routed to experts < e.
 *   src_row device int32 [T*k]: pair index t*k + j at each grouped position;
 *           experts ascending, within an expert (t, j) ascending.
 *   dst_of  device int32 [T*k]: grouped position of pair t*k + j.
 * Errors: T*k > 2^24 or E > 1024 -> INVALID_SHAPE. Ids outside [0, E) are
 * outside the contract (they are clamped into range, not reported). */
MXMOE_API int mxmoe_permute(const int32_t *ids, int T, int k, int E, int32_t *offsets, int32_t *src_row,
                            int32_t *dst_of, void *stream);

/* mxmoe_permute for many pairs, with caller scratch: the same outputs (bit for
 * bit) from a multi-block grouping when T*k > 4096 (otherwise it
 * runs mxmoe_permute's kernel and leaves the scratch alone).
 *   scratch device, >= mxmoe_permute_scratch_size(T, k, E) bytes, 16-byte
 *   aligned, contents not kept between calls.
 * Errors: those of mxmoe_permute; scratch NULL or too small ->
 * WORKSPACE. */
MXMOE_API int mxmoe_permute_ws(const int32_t *ids, int T, int k, int E, int32_t *offsets, int32_t *src_row,
                               int32_t *dst_of, void *scratch, int64_t scratch_bytes, void *stream);

/* Scratch bytes for mxmoe_permute_ws (-1 on bad sizes). */
MXMOE_API int64_t mxmoe_permute_scratch_size(int T, int k, int E);

/* ------------------------------------------------------------------------ */
/* Experts                                                                   */
/* ------------------------------------------------------------------------ */

/* Workspace bytes needed by mxmoe_expert_ffn for these sizes (-1 on bad
 * sizes). */
MXMOE_API int64_t mxmoe_ffn_workspace_size(int T, int k, int E, int H, int I);

/* Grouped SwiGLU expert FFN over MXFP4 weights (W4A16), fp32 accumulation.
 * For every grouped position r (pair p = src_row[r] = t*k + j, routed to the
 * expert e with offsets[e] <= r < offsets[e+1]):
 *   g = W_gate[e] x_t, u = W_up[e] x_t, h = silu(g) * u, y_perm[r] = W_down[e] h.
 *   x device bf16 [T, H]; offsets, src_row as produced by mxmoe_permute;
 *   prepacked device blob from mxmoe_prepack_experts; y_perm device float
 *   [T*k, H]; workspace device, >= mxmoe_ffn_workspace_size bytes, 256-byte
 *   aligned. Its first 16 bytes hold the device status word of the call.
 * The products run on tcgen05 block-scaled tensor cores (E2M1 weights x E2M1
 * activation terms, UE8M0 scales per 32, fp32 accumulation): x and h each
 * enter as eight E2M1 terms per value (balanced base-8 digits on the grid
 * 2^(E-22), E the exponent of the value's 32-block maximum), every term with
 * its own scale per 32 values. That represents every bf16 x within 2^-15 of
 * its block maximum exactly and any other value (smaller x, fp32 h) to within
 * 2^-23 of the block maximum. From 16384 grouped rows (and, from 128 tokens,
 * for experts with at least 128 rows) both stages run on the large-token
 * kernel instead (tcgen05 kind::mxf8f6f4 block-scaled MMAs): the E2M1 weight
 * codes and their scales as stored, x as two E4M3 terms per value (exact for
 * every bf16 x within 2^-13 of its 32-block maximum, smaller ones within
 * 2^-21 of it), h as three E4M3 terms on scales 2^(E-7), 2^(E-11), 2^(E-15)
 * of its 32-block maximum 2^E (within about 2^-16 of the block maximum).
 * Errors: H or I not a multiple of 128 or above 32768, k > 32, E > 1024,
 * T*k > 2^22, E*I*H >= 2^38 -> INVALID_SHAPE; workspace
 * too small -> WORKSPACE; x, y_perm not 16-byte or prepacked not 32-byte
 * aligned -> ALIGNMENT. Device-side wait timeouts -> mxmoe_read_status. */
MXMOE_API int mxmoe_expert_ffn(const void *x, const int32_t *offsets, const int32_t *src_row, const void *prepacked,
                               int T, int k, int E, int H, int I, float *y_perm, void *workspace,
                               int64_t workspace_bytes, void *stream);

/* Stage 1 of mxmoe_expert_ffn on its own: for every grouped position r,
 * h[r] = silu(W_gate[e] x_t) * (W_up[e] x_t), written into the workspace for
 * mxmoe_ffn_down: as 8 E2M1 digit terms per value with their scale images,
 * or, for experts that the large-token kernel takes (every expert from 16384
 * grouped rows; from 128 tokens, experts with at least 128 rows), as three
 * E4M3 terms per value with their scale images, tiled per 224-token pass in
 * the layout that kernel reads.
 * Arguments, layout and errors as for mxmoe_expert_ffn (workspace from
 * mxmoe_ffn_workspace_size, 256-byte aligned). */
MXMOE_API int mxmoe_ffn_gate_up(const void *x, const int32_t *offsets, const int32_t *src_row, const void *prepacked,
                                int T, int k, int E, int H, int I, void *workspace, int64_t workspace_bytes,
                                void *stream);

/* Stage 2 of mxmoe_expert_ffn on its own: y_perm[r] = W_down[e] h[r] for every
 * grouped position r, reading the h that mxmoe_ffn_gate_up left in the same
 * workspace (call it first, on the same stream). y_perm device float
 * [T*k, H], 16-byte aligned. Errors as for mxmoe_expert_ffn. */
MXMOE_API int mxmoe_ffn_down(const int32_t *offsets, const void *prepacked, int T, int k, int E, int H, int I,
                             float *y_perm, void *workspace, int64_t workspace_bytes, void *stream);

/* Workspace-free variant of mxmoe_expert_ffn for callers that cannot
 * allocate device memory: for example a process whose device memory is all
 * reserved by another allocator's pool, or a latency-critical loop in which
 * cudaMalloc (which may synchronise the device) is not allowed. There is no
 * counterpart on the pages; it exists only for such callers.
 * Arguments, layout and results are those of mxmoe_expert_ffn, minus the
 * workspace. Scratch is a fixed 8 MiB static device array inside the library
 * (held on every GPU where the library's device code is loaded, until the
 * process exits); sizes whose mxmoe_ffn_workspace_size exceeds 8 MiB are
 * rejected with MXMOE_ERR_WORKSPACE before anything is enqueued (the
 * 6144/2048/top-8 layer fits up to 15 tokens).
 *   status  device int or NULL: when given, receives the call's device status
 *           word (MXMOE_OK or MXMOE_ERR_TIMEOUT) in stream order.
 * The first call in each CUDA context of a device looks up the array's
 * device address (once per context, under a lock); make that first call
 * before any stream capture. A device reset (cudaDeviceReset) or a new
 * context reloads the library's device code, which invalidates an earlier
 * lookup: the next call then looks the address up again. The call
 * allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 * All calls share the one array and it keeps the last call's contents (the
 * call itself clears what must start at zero), so calls whose work overlaps
 * on the GPU (different streams, or several host threads) race: serialise
 * them, for example on one stream. */
MXMOE_API int mxmoe_expert_ffn_noalloc(const void *x, const int32_t *offsets, const int32_t *src_row,
                                       const void *prepacked, int T, int k, int E, int H, int I, float *y_perm,
                                       int *status, void *stream);

/* Weighted combine: y[t, c] = sum over j = 0..k-1 (in order) of
 * w[t, j] * y_perm[dst_of[t*k + j], c], float32: each token's output is its
 * selected experts' outputs weighted by its routing weights (the 8 activated
 * experts of the nxbn.cn article's architecture section; the pages give no
 * summation order, so slots are added in order).
 *   y_perm device float [T*k, H]; dst_of device int32 [T*k]; w device float
 *   [T, k]; y device float [T, H].
 * Errors: H % 4 != 0 or T > 65535 -> INVALID_SHAPE; y_perm, y not 16-byte aligned ->
 * ALIGNMENT. */
MXMOE_API int mxmoe_combine(const float *y_perm, const int32_t *dst_of, const float *w, int T, int k, int H,
                            float *y, void *stream);

/* ------------------------------------------------------------------------ */
/* Whole layer                                                               */
/* ------------------------------------------------------------------------ */

/* Workspace bytes needed by mxmoe_layer_forward; -1 for exactly the shapes
 * that mxmoe_layer_forward rejects with INVALID_SHAPE. */
MXMOE_API int64_t mxmoe_workspace_size(int T, int H, int I, int E, int k);

/* The whole MoE expert layer for T tokens: router GEMM, route, permute,
 * expert FFN, combine, in stream order, with no host synchronisation.
 *   x device bf16 [T, H]; wg device bf16 [E, H]; bias device float [E] or
 *   NULL; prepacked device blob (mxmoe_prepack_experts); y device float
 *   [T, H]; ids_out device int32 [T, k] or NULL; w_out device float [T, k]
 *   or NULL; workspace device, >= mxmoe_workspace_size bytes, 256-byte
 *   aligned (its first 16 bytes hold the device status word).
 * Errors: the union of the steps' errors (so T <= 65535, the combine's limit). */
MXMOE_API int mxmoe_layer_forward(const void *x, const void *wg, const float *bias, const void *prepacked, int T,
                                  int H, int I, int E, int k, float *y, int32_t *ids_out, float *w_out,
                                  void *workspace, int64_t workspace_bytes, void *stream);

/* ------------------------------------------------------------------------ */
/* FP8 expert weights                                                        */
/* ------------------------------------------------------------------------ */
/* The model card's section 2 ("FP4 Quantization") sets the MXFP4 experts
 * against an FP8 baseline, and its introduction says that even 8-bit weights
 * carry heavy memory-bandwidth costs at this scale, so lowering the bit width
 * speeds up decoding. These entry points run the same layer with FP8 expert
 * weights, to measure that. The pages give no FP8 layout; the reading is the
 * MX scheme of the FP4 experts with E4M3 elements ("MXFP8"): one E8M0 scale
 * per 32 elements along K, scale exponent e = floor(log2 amax) - 8 clamped to
 * [-127, 127] (-127 for an all-zero block; 8 is the exponent of E4M3's
 * largest power of two), each element |x| / 2^e rounded to nearest E4M3 with
 * ties to the even mantissa, saturating at 448, sign bit copied. E4M3 codes:
 * bit 7 sign, bits 6..3 exponent (bias 7), bits 2..0 mantissa; exponent 0 is
 * subnormal; 0x7F / 0xFF (NaN) are never produced. */

/* bf16 [rows, K] -> E4M3 codes uint8 [rows, K] (one byte per element) and
 * scales uint8 [rows, K/32], all device memory.
 * Errors: K % 32 != 0 or rows/K <= 0 -> INVALID_SHAPE; NULL -> NULL; w not
 * 16-byte or codes not 8-byte aligned -> ALIGNMENT. */
MXMOE_API int mxmoe_quantize_fp8(const void *w, int64_t rows, int64_t K, uint8_t *codes, uint8_t *scales,
                                 void *stream);

/* out[r, k] = E4M3(codes[r, k]) * 2^(scales[r, k/32] - 127) as float (device
 * memory). Errors as for mxmoe_quantize_fp8. */
MXMOE_API int mxmoe_dequantize_fp8(const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t K, float *out,
                                   void *stream);

/* Bytes of the prepacked FP8 blob: E * (2*I*H + Hp*I) * 33/32, Hp = H rounded
 * up to a multiple of 256. -1 unless H and I are positive multiples of 128. */
MXMOE_API int64_t mxmoe_prepacked_size_fp8(int E, int H, int I);

/* Re-tile FP8 expert weights for the FP8 FFN (a byte permutation plus
 * zero padding of the down rows to a multiple of 256).
 *   codes13 device uint8 [E, 2I, H], sc13 [E, 2I, H/32] (gate rows 0..I-1,
 *   up rows I..2I-1); codes2 [E, H, I], sc2 [E, H, I/32] (down);
 *   prepacked device, mxmoe_prepacked_size_fp8 bytes, 32-byte aligned.
 * Layout: [gate/up code boxes][down code boxes][gate/up scale images][down
 * scale images]. A code box is a 256-row tile by 128 values of K (256 rows of
 * 128 bytes, 32 KB, contiguous), boxes ordered by (expert, tile, K chunk);
 * gate/up tile t holds gate rows 128t .. 128t+127, then the matching up rows.
 * A box's scale images are two 512-byte images, one per row half g: byte
 * (r % 32) * 16 + (r / 32) * 4 + kb is the scale of tile row 128g + r, k32
 * block kb of the box.
 * Errors: shapes -> INVALID_SHAPE; NULL -> NULL; prepacked not 32-byte or
 * codes13/codes2 not 16-byte aligned -> ALIGNMENT. */
MXMOE_API int mxmoe_prepack_experts_fp8(const uint8_t *codes13, const uint8_t *sc13, const uint8_t *codes2,
                                        const uint8_t *sc2, int E, int H, int I, void *prepacked, void *stream);

/* Workspace bytes for mxmoe_expert_ffn_fp8 (-1 on bad sizes). */
MXMOE_API int64_t mxmoe_ffn_workspace_size_fp8(int T, int k, int E, int H, int I);

/* mxmoe_expert_ffn with FP8 expert weights (blob from
 * mxmoe_prepack_experts_fp8): the same grouped SwiGLU FFN, arguments, layout
 * and errors, workspace from mxmoe_ffn_workspace_size_fp8. Both stages run on
 * tcgen05.mma.kind::mxf8f6f4.block_scale at every token count: E4M3 weights
 * as stored times the E2M1 digit terms of x and h (the same terms, and the
 * same error bound, as the MXFP4 kernel), UE8M0 scales per 32 applied in
 * hardware, fp32 accumulation. */
MXMOE_API int mxmoe_expert_ffn_fp8(const void *x, const int32_t *offsets, const int32_t *src_row,
                                   const void *prepacked, int T, int k, int E, int H, int I, float *y_perm,
                                   void *workspace, int64_t workspace_bytes, void *stream);

/* Workspace bytes for mxmoe_layer_forward_fp8 (-1 for exactly the shapes it
 * rejects with INVALID_SHAPE). */
MXMOE_API int64_t mxmoe_workspace_size_fp8(int T, int H, int I, int E, int k);

/* mxmoe_layer_forward with FP8 expert weights: router GEMM, route, permute,
 * mxmoe_expert_ffn_fp8's FFN, combine. Arguments and errors as for
 * mxmoe_layer_forward, prepacked from mxmoe_prepack_experts_fp8, workspace
 * from mxmoe_workspace_size_fp8. */
MXMOE_API int mxmoe_layer_forward_fp8(const void *x, const void *wg, const float *bias, const void *prepacked, int T,
                                      int H, int I, int E, int k, float *y, int32_t *ids_out, float *w_out,
                                      void *workspace, int64_t workspace_bytes, void *stream);

/* ------------------------------------------------------------------------ */
/* Expert parallelism                                                        */
/* ------------------------------------------------------------------------ */
/* The pages serve the model with expert parallelism (--ep-size 16 in the
 * SGLang launch of the "MiMo-V2.5-Pro-FP4-DFlash" model card's deployment
 * section and of the nxbn.cn article's SGLang deployment section). With G
 * ranks, rank g holds experts [g E/G, (g+1) E/G) (E a multiple of G) as its
 * own prepacked blob, and each rank routes its own tokens. One layer step on
 * rank g:
 *   1. mxmoe_router_gemm + mxmoe_route on its tokens (all E experts);
 *   2. mxmoe_permute: pairs grouped by expert -- also by owner rank;
 *   3. mxmoe_ep_dispatch: the rows to send, their local expert ids and the
 *      row count per destination rank;
 *   4. all-to-all of the counts, then of the rows and ids (the caller's
 *      collective library, e.g. NCCL through torch.distributed);
 *   5. mxmoe_ep_expert_ffn on the received rows with the rank's experts;
 *   6. all-to-all back (the reverse splits): the output rows land in the
 *      grouped order of step 2;
 *   7. mxmoe_combine with step 2's dst_of and step 1's weights.
 * The result equals mxmoe_layer_forward of the whole layer on the rank's
 * tokens up to float summation order. */

/* Sender side of the dispatch, after mxmoe_permute.
 *   x device bf16 [T, H]; offsets, src_row from mxmoe_permute over E experts.
 *   send_x device bf16 [T*k, H]: send_x[r] = x[src_row[r] / k] (grouped
 *   order, so rank g's rows are offsets[g E/G] .. offsets[(g+1) E/G]).
 *   send_local device int32 [T*k]: the expert of row r minus the first
 *   expert of its owner rank.
 *   send_counts device int32 [G]: rows destined to each rank.
 * Errors: E > 1024 or not a multiple of G, k > 32, H % 8 != 0, T*k > 2^24 ->
 * INVALID_SHAPE; NULL -> NULL; x, send_x not 16-byte aligned -> ALIGNMENT. */
MXMOE_API int mxmoe_ep_dispatch(const void *x, const int32_t *offsets, const int32_t *src_row, int T, int k, int E,
                                int G, int H, void *send_x, int32_t *send_local, int32_t *send_counts, void *stream);

/* Workspace bytes for mxmoe_ep_expert_ffn (-1 on bad sizes). */
MXMOE_API int64_t mxmoe_ep_workspace_size(int n_recv, int E_local, int H, int I);

/* Receiver side: the rank's experts applied to the rows it received.
 *   x_recv device bf16 [n_recv, H]; recv_local device int32 [n_recv], each
 *   in [0, E_local); prepacked_local: mxmoe_prepack_experts of the rank's
 *   E_local experts; y_recv device float [n_recv, H]: y_recv[i] = the FFN of
 *   expert recv_local[i] on x_recv[i] (receive order); workspace device,
 *   >= mxmoe_ep_workspace_size bytes, 256-byte aligned (its first 16 bytes
 *   hold the device status word, read with mxmoe_read_status).
 * The rows are grouped by local expert (mxmoe_permute with k = 1), run
 * through mxmoe_expert_ffn and gathered back into receive order.
 * Errors: the expert FFN's shapes with T = n_recv, k = 1 -> INVALID_SHAPE;
 * workspace -> WORKSPACE / ALIGNMENT; NULL -> NULL. */
MXMOE_API int mxmoe_ep_expert_ffn(const void *x_recv, const int32_t *recv_local, int n_recv, int E_local, int H,
                                  int I, const void *prepacked_local, float *y_recv, void *workspace,
                                  int64_t workspace_bytes, void *stream);

/* The layer of mxmoe_layer_forward as one persistent kernel: one CTA per SM,
 * all resident (a cooperative launch), running the router GEMM, routing,
 * grouping, the activation terms, both FFN stages (tcgen05 block-scaled MMA,
 * the same items as mxmoe_expert_ffn's E2M1-term kernel) and the combine as
 * phases separated by grid-wide barriers, so that no launch boundary sits
 * between the layer's steps and the weight stream of the gate/up stage starts
 * while the activation terms are still being encoded. This is the execution
 * model of the pages' serving engine, applied to this layer: a persistent
 * engine kernel that stays resident, removes the gaps at operator boundaries
 * and keeps prefetching while the tensor cores compute ("Xiaomi
 * MiMo-V2.5-Pro-UltraSpeed 發佈說明", agentlenshq.com, section "TileRT 執行模型").
 * This entry point takes the path for any supported size,
 * mxmoe_layer_forward_chained never; mxmoe_layer_forward keeps the chained
 * launches (measured as fast or faster: on one verify block the grid-wide
 * barriers cost about what the chained launches' gaps do).
 * Arguments, layout, results and workspace as for mxmoe_layer_forward (ids and
 * weights identical; y equal up to float summation order, which is the same
 * as the chained path's). Every grid-wide wait is bounded (2 s): a CTA that
 * gives up records MXMOE_ERR_TIMEOUT in the status word (mxmoe_read_status)
 * and the others stop at their next barrier.
 * Errors: those of mxmoe_layer_forward; and T > 256, T*k > 4096 or E > 384 ->
 * INVALID_SHAPE. */
MXMOE_API int mxmoe_layer_forward_persistent(const void *x, const void *wg, const float *bias, const void *prepacked,
                                             int T, int H, int I, int E, int k, float *y, int32_t *ids_out,
                                             float *w_out, void *workspace, int64_t workspace_bytes, void *stream);

/* mxmoe_layer_forward as the chain of separate launches at every size (never
 * the persistent kernel). Arguments, results and errors as for
 * mxmoe_layer_forward. */
MXMOE_API int mxmoe_layer_forward_chained(const void *x, const void *wg, const float *bias, const void *prepacked,
                                          int T, int H, int I, int E, int k, float *y, int32_t *ids_out, float *w_out,
                                          void *workspace, int64_t workspace_bytes, void *stream);

/* Test of the device-side timeout path (failure detection): one thread waits
 * on a shared-memory mbarrier that nothing ever arrives on, through the same
 * bounded wait that every wait of the FFN and router kernels uses, with a
 * limit of limit_us microseconds, then writes MXMOE_ERR_TIMEOUT to *status
 * (MXMOE_OK if the wait had completed) and the kernel returns normally, so the
 * context stays usable. No counterpart on the pages.
 *   status device int; limit_us 1 .. 1000000.
 * Errors: status NULL -> NULL; limit_us out of range -> INVALID_SHAPE. */
MXMOE_API int mxmoe_selftest_wait_timeout(int *status, int limit_us, void *stream);

/* Synchronise `stream`, then read the device status word that the last
 * mxmoe_expert_ffn / mxmoe_layer_forward call on this workspace left:
 * MXMOE_OK, or MXMOE_ERR_TIMEOUT if a bounded device-side wait gave up.
 *   workspace device (as passed to the call); *status host int. */
MXMOE_API int mxmoe_read_status(const void *workspace, int *status, void *stream);

/* ------------------------------------------------------------------------
 * Block verification of a speculative draft
 *
 * "MiMo-V2.5-Pro-FP4-DFlash" (alphaneural mirror), section 3
 * "Block-Diffusion Speculative Decoding (DFlash)": the drafter proposes a
 * block of tokens (at most 8) in one pass and the backbone verifies the whole
 * block in one step; rejection-sampling verification keeps the output
 * lossless. Reading (the pages give no formula): the standard
 * speculative-sampling test in block order. With p_i = softmax(z_i / tau) of
 * the backbone's logits at block position i and q_i = softmax(w_i / tau) of
 * the drafter's, draft token d_i is accepted when u_i q_i(d_i) < p_i(d_i);
 * at the first rejection j the emitted token is drawn from max(0, p_j - q_j),
 * after K acceptances from p_K, both by inverse CDF in token order with u_K
 * (the smallest v whose running sum exceeds u_K times the total). tau = 0 is
 * greedy verification: d_i is accepted while it is the argmax of z_i (ties
 * to the lower index) and the emitted token is the argmax at the first
 * mismatch. A draft token outside [0, V) is never accepted. Arithmetic is
 * fp32; a decision whose two sides are within float rounding of each other
 * (a uniform on a threshold) may differ from an exact evaluation.
 * ------------------------------------------------------------------------ */

/* Workspace bytes for mxmoe_verify_block with these sizes; -1 if invalid. */
MXMOE_API int64_t mxmoe_verify_workspace_size(int B, int K, int64_t V);

/* Verify B blocks of K drafted tokens.
 *   target_logits device float [B, K+1, V]: the backbone's logits at the K
 *       block positions and the position after the block.
 *   draft_logits device float [B, K, V]: the drafter's logits (may be NULL
 *       when temperature == 0).
 *   draft_tokens device int32 [B, K]; uniforms device float [B, K+1] in
 *       [0, 1): u_0 .. u_{K-1} for the acceptance tests, u_K for the draw.
 *   temperature >= 0, finite (0: greedy).
 *   accepted device int32 [B]: accepted drafts n (0 .. K).
 *   tokens device int32 [B, K+1]: the n accepted drafts, then the emitted
 *       token, then -1.
 *   workspace device, >= mxmoe_verify_workspace_size(B, K, V) bytes,
 *       256-byte aligned; contents not kept between calls.
 * Errors: K < 1, K > 32, V < 1, V > 2^24, B < 0, B (2K + 1) > 65535 -> INVALID_SHAPE;
 * a negative or non-finite temperature, or a positive one so small that
 * log2(e) / temperature overflows float (below about 4e-39) -> INVALID_SHAPE; NULL pointers ->
 * NULL; workspace too small -> WORKSPACE, misaligned -> ALIGNMENT. */
MXMOE_API int mxmoe_verify_block(const float *target_logits, const float *draft_logits,
                                 const int32_t *draft_tokens, const float *uniforms, int B, int K, int64_t V,
                                 float temperature, int32_t *accepted, int32_t *tokens, void *workspace,
                                 int64_t workspace_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MXMOE_H */
