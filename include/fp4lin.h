/*
 * fp4lin.h -- C ABI of the B200 (sm_100a) NVFP4 / MXFP4 W4A4 linear layer and
 * NVFP4 KV cache.
 *
 * The formats (web pages cited by title and section):
 *   - E2M1 elements, 1 sign / 2 exponent / 1 mantissa bit, about -6..6:
 *     "FP4 auf Blackwell: Was NVFP4 fuer lokale KI wirklich aendert",
 *     section "Was NVFP4 von frueheren 4-Bit-Formaten unterscheidet";
 *     "FP8, NVFP4 czy AWQ?", section "Czym roznia sie FP8, NVFP4, MXFP4 i AWQ?".
 *   - NVFP4: 16-value blocks, one E4M3 (FP8) scale per block plus one FP32
 *     scale per tensor (same two sections).
 *   - MXFP4 (OCP Microscaling): 32-value blocks, power-of-two E8M0 scale
 *     (same two sections).
 *   - Blockwise Hadamard rotation of the activations, computed online, with
 *     the rotation folded into the weights: the MR-GPTQ abstract
 *     (hyper.ai/de/papers/2509.23202), "Abstract".
 *   - KV cache written in NVFP4, dequantised to FP8 before attention: the
 *     NVFP4 KV-cache story (hyper.ai/de/stories/e1307393ec176dd2b0276468adeec3f9,
 *     one untitled paragraph).
 *
 * Conventions for every entry point:
 *   - All data pointers are DEVICE pointers on the current CUDA device; the
 *     caller allocates and owns every buffer.  The library allocates no
 *     memory and keeps no state beyond cached kernel attributes and one
 *     device status word per device (see fp4lin_device_status).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call only enqueues work on it and returns without
 *     synchronising; results are ready when the stream is.
 *   - Arguments are checked on the host before anything is launched; on any
 *     error nothing is launched and a status below is returned.
 *   - bf16 means IEEE bfloat16 stored as 16-bit words; codes pack two E2M1
 *     values per byte, element 2i in the low nibble and 2i+1 in the high
 *     nibble, K (the row) contiguous.
 *   - "Tensor-core scale layout": scale bytes of a [rows, sf_cols] matrix
 *     grouped into atoms of 128 rows x 4 scale columns (512 bytes); atom
 *     (rt, ct) starts at byte (rt * ceil(sf_cols/4) + ct) * 512, and inside
 *     an atom the scale of row r, column c sits at byte
 *     (r % 32) * 16 + ((r % 128) / 32) * 4 + c % 4.  The buffer holds
 *     fp4lin_scale_bytes(rows, sf_cols) bytes; padding bytes are written 0.
 *     This is the layout the sm_100 block-scaled tensor-core MMA reads.
 */
#ifndef FP4LIN_H
#define FP4LIN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every entry point. */
enum fp4lin_status {
    FP4LIN_OK = 0,
    FP4LIN_ERR_INVALID_ARGUMENT = 1, /* null pointer, size <= 0, bad option value */
    FP4LIN_ERR_UNSUPPORTED_SHAPE = 2, /* a size the kernels do not support (see each call) */
    FP4LIN_ERR_MISALIGNED = 3,       /* a pointer or leading dimension breaks the 16-byte rule */
    FP4LIN_ERR_CUDA = 4,             /* a CUDA runtime call or kernel launch failed */
    FP4LIN_ERR_TIMEOUT = 5,          /* a device-side wait gave up (reported by fp4lin_device_status) */
    FP4LIN_ERR_DEVICE = 6,           /* the current device is not compute capability 10.0 (B200) */
    FP4LIN_ERR_WORKSPACE = 7,        /* workspace null or smaller than required */
    FP4LIN_ERR_OUT_OF_RANGE = 8,     /* a KV position outside [0, Lcap) (reported by fp4lin_device_status) */
    FP4LIN_ERR_NUMERIC = 9           /* a factorisation met a pivot that is not positive and finite
                                        (reported by fp4lin_device_status) */
};

/* Library version, MAJOR*10000 + MINOR*100 + PATCH. */
int fp4lin_version(void);

/* Bytes of a tensor-core-layout scale buffer for `rows` rows and `sf_cols`
 * scale columns: ceil(rows/128)*128 * ceil(sf_cols/4)*4. */
int64_t fp4lin_scale_bytes(int64_t rows, int64_t sf_cols);

/* Bytes of workspace nvfp4_quantize needs when compute_global_scale = 1
 * (a constant 4096: one float per partial-maximum block). */
size_t nvfp4_quantize_workspace_bytes(int64_t rows, int64_t cols);

/* Bytes of workspace that lets nvfp4_gemm / mxfp4_gemm split K over more
 * CTAs for this shape (0 when the shape needs no split).  A smaller
 * workspace is accepted: the GEMM then runs without the split. */
size_t fp4lin_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);

/*
 * NVFP4 quantisation of a bf16 matrix, optionally rotated.
 * Defined by: "FP4 auf Blackwell: Was NVFP4 fuer lokale KI wirklich aendert", section
 * "Was NVFP4 von frueheren 4-Bit-Formaten unterscheidet" (E2M1 elements, E4M3 block scale per 16
 * values, one FP32 scale per tensor); "FP8, NVFP4 czy AWQ?", section "Czym roznia sie FP8, NVFP4, MXFP4 i AWQ?",
 * NVFP4 bullet (16-element blocks, FP8 E4M3 scale); the rotation: the MR-GPTQ abstract (hyper.ai/de/papers/2509.23202), "Abstract"
 * (blockwise Hadamard transforms, activations rotated online).
 *
 *   x       [rows, cols] bf16, row stride ld_x elements.
 *   hadamard 0 (none) or 16: rotate every 16-value block along the row by
 *           the Sylvester Hadamard matrix scaled by 1/4 before quantising.
 *   compute_global_scale
 *           1: g is OUTPUT -- g = max|x'| / (6*448) over the (rotated)
 *              tensor, or 1 when that is not > 0; needs `workspace`.
 *           0: g is INPUT (device float, must be > 0 and finite).
 *   g       device pointer to one float (the FP32 tensor scale).
 *   codes   [rows, cols/2] bytes, E2M1 pairs.
 *   scales  tensor-core scale layout of the [rows, cols/16] E4M3 block
 *           scales, fp4lin_scale_bytes(rows, cols/16) bytes.
 * Per 16-value block: t = (amax/6)/g, sf = E4M3 round-to-nearest-even with
 * saturation at 448, d = dec(sf)*g, r = d > 0 ? 1/d : 0, codes =
 * E2M1 round-to-nearest-even of x'*r with saturation at 6 (sign kept).
 * Shapes: rows >= 1, cols a multiple of 64, ld_x >= cols and a multiple of
 * 8; x, codes, scales 16-byte aligned.
 */
int nvfp4_quantize(const void *x, int64_t rows, int64_t cols, int64_t ld_x,
                   int hadamard, int compute_global_scale, float *g,
                   uint8_t *codes, uint8_t *scales,
                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * y[M, N] = A[M, K] * W[N, K]^T for NVFP4 operands, FP32 accumulation on the
 * tensor cores.  Defined by: "FP4 auf Blackwell: Was NVFP4 fuer lokale KI wirklich aendert", section
 * "Was NVFP4 von frueheren 4-Bit-Formaten unterscheidet"
 * (Blackwell's 5th-generation tensor cores apply the two-level scaling in
 * hardware); "FP8, NVFP4 czy AWQ?", section "Dlaczego W8A8 i W4A16 to nie to
 * samo?" (W4A4: weights and activations both 4-bit, the product on low-precision
 * tensor cores).  Result: y = bf16_round(g_a * g_w * acc).
 * The library picks the kernel (CTA pairs over 256 x 256 tiles for M >= 256
 * without a K split, else one CTA per tile; FP4LIN_GEMM_KERNEL=single or =pair
 * forces one); every choice gives the same bytes.
 *   a_codes [M, K/2], a_scales tensor-core layout of [M, K/16];
 *   w_codes [N, K/2], w_scales tensor-core layout of [N, K/16];
 *   g_a, g_w device floats; y bf16 with row stride ldy elements.
 * Shapes: M, N >= 1; K a multiple of 64; ldy >= N and a multiple of 8;
 * all pointers 16-byte aligned.  workspace may be NULL (see
 * fp4lin_gemm_workspace_bytes).
 */
int nvfp4_gemm(const uint8_t *a_codes, const uint8_t *a_scales, const float *g_a,
               const uint8_t *w_codes, const uint8_t *w_scales, const float *g_w,
               void *y, int64_t M, int64_t N, int64_t K, int64_t ldy,
               void *workspace, size_t workspace_bytes, void *stream);

/*
 * MXFP4 quantisation.  Defined by: "FP4 auf Blackwell: Was NVFP4 fuer lokale KI wirklich aendert", section
 * "Was NVFP4 von frueheren 4-Bit-Formaten unterscheidet"
 * (MXFP4: 32-value blocks scaled by powers of two); "FP8, NVFP4 czy AWQ?", section "Czym roznia sie FP8, NVFP4, MXFP4 i AWQ?",
 * MXFP4 bullet (the OCP Microscaling standard's E8M0 block scale); the 32-wide
 * rotation: the MR-GPTQ abstract (hyper.ai/de/papers/2509.23202), "Abstract".
 * 32-value blocks, E8M0 scale byte = clamp(X + 127, 0,
 * 254) with X = floor(log2 amax) - 2, codes = E2M1 of x' * 2^-X.
 *   hadamard 0 or 32 (rotate each 32-value block by H_32 / sqrt(32)).
 *   codes [rows, cols/2]; scales tensor-core layout of [rows, cols/32].
 * Shapes as nvfp4_quantize.
 */
int mxfp4_quantize(const void *x, int64_t rows, int64_t cols, int64_t ld_x,
                   int hadamard, uint8_t *codes, uint8_t *scales, void *stream);

/* y = A * W^T for MXFP4 operands (E8M0 scales, no tensor scale); otherwise
 * as nvfp4_gemm.
 * Defined by: "FP4 auf Blackwell: Was NVFP4 fuer lokale KI wirklich aendert", section
 * "Was NVFP4 von frueheren 4-Bit-Formaten unterscheidet"
 * (MXFP4 blocks of 32 with power-of-two scales, multiplied on the block-scaled
 * tensor cores); "FP8, NVFP4 czy AWQ?", section "Czym roznia sie FP8, NVFP4, MXFP4 i AWQ?", MXFP4 bullet. */
int mxfp4_gemm(const uint8_t *a_codes, const uint8_t *a_scales,
               const uint8_t *w_codes, const uint8_t *w_scales,
               void *y, int64_t M, int64_t N, int64_t K, int64_t ldy,
               void *workspace, size_t workspace_bytes, void *stream);

/*
 * Append T new K (or V) rows per (batch, head) to an NVFP4 cache.
 * Defined by: the NVFP4 KV-cache story (hyper.ai/de/stories/e1307393ec176dd2b0276468adeec3f9,
 * one untitled paragraph), its statement that new K/V vectors are written to the
 * cache in NVFP4 and the KV tensors are dequantised to FP8 before attention.
 *   kv_new       bf16 [B, H, T, D] contiguous.
 *   pos          device int32 [B]: row t of batch b goes to position pos[b] + t.
 *   g            device float, the static FP32 tensor scale (> 0).
 *   cache_codes  [B, H, Lcap, D/2] bytes.
 *   cache_scales [B, H, Lcap, D/16] E4M3 bytes, row-major (not the
 *                tensor-core layout: attention reads the FP8 copy).
 * Each row is quantised along D exactly like nvfp4_quantize with static g.
 * A position outside [0, Lcap) is skipped and recorded as
 * FP4LIN_ERR_OUT_OF_RANGE in the device status word.
 * Shapes: D a multiple of 16; pointers 16-byte aligned except pos (4).
 */
int kv_nvfp4_store(const void *kv_new, const int32_t *pos, const float *g,
                   uint8_t *cache_codes, uint8_t *cache_scales,
                   int B, int H, int T, int64_t Lcap, int D, void *stream);

/*
 * Dequantise the first L positions of every (batch, head) of an NVFP4 cache
 * to FP8 E4M3 for attention.
 * Defined by: the NVFP4 KV-cache story (hyper.ai/de/stories/e1307393ec176dd2b0276468adeec3f9,
 * one untitled paragraph), its statement that new K/V vectors are written to the
 * cache in NVFP4 and the KV tensors are dequantised to FP8 before attention.
 *   out_fp8[b,h,l,d] = E4M3_rne(e2m1(code) * dec(sf) / 8), out_scale = 8 * g,
 * so that value = fp8 * out_scale.  The product is exact, so the E4M3
 * rounding is the only rounding.
 *   out_fp8 [B, H, L, D] bytes; out_scale device float.
 * Shapes: 1 <= L <= Lcap; D a multiple of 16; pointers 16-byte aligned
 * except g and out_scale (4).
 */
int kv_nvfp4_load_fp8(const uint8_t *cache_codes, const uint8_t *cache_scales,
                      const float *g, int64_t L, uint8_t *out_fp8, float *out_scale,
                      int B, int H, int64_t Lcap, int D, void *stream);

/*
 * Synchronise `stream`, then read and clear this device's status word.
 * Returns FP4LIN_OK, or the first device-side error recorded since the last
 * call (FP4LIN_ERR_TIMEOUT, FP4LIN_ERR_OUT_OF_RANGE), or FP4LIN_ERR_CUDA if
 * the synchronisation itself failed.
 */
int fp4lin_device_status(void *stream);

/*
 * Diagnostic: run the library's own element conversions on n floats.
 *   e2m1[i] = E2M1 code (low nibble) of in[i], round-to-nearest-even,
 *             saturating at 6, sign kept;
 *   e4m3[i] = E4M3 byte of in[i], round-to-nearest-even, saturating at 448.
 * These are the device functions every quantiser uses.  n >= 1.
 */
int fp4lin_convert_selftest(const float *in, uint8_t *e2m1, uint8_t *e4m3, int64_t n,
                            void *stream);

/*
 * Diagnostic of the device-side wait limit.  One CTA runs two waits on
 * shared-memory barriers through the same bounded-wait routine the GEMM
 * pipelines use: wait 1 with a limit of limit_ns nanoseconds, wait 0 with the
 * library's 1 s limit but giving up as soon as another wait of the CTA has
 * expired (the GEMM's abort rule).
 *   arrive = 1: each barrier is arrived on first; both waits succeed and the
 *               device status stays FP4LIN_OK.
 *   arrive = 0: nothing arrives.  Wait 1 expires after limit_ns and records
 *               FP4LIN_ERR_TIMEOUT in the device status; wait 0 then gives
 *               up.  The kernel returns normally: the context stays usable.
 * result: device, 4 x uint64, 8-byte aligned, written by the kernel:
 *   result[0], result[1] = 1 if wait 0 / wait 1 saw its barrier complete;
 *   result[2], result[3] = nanoseconds wait 0 / wait 1 took (global timer).
 * limit_ns in [1000, 100000000] (1 us .. 100 ms), else
 * FP4LIN_ERR_INVALID_ARGUMENT, as for arrive not 0 or 1 or result NULL.
 */
int fp4lin_wait_selftest(uint64_t limit_ns, int arrive, uint64_t *result, void *stream);

/*
 * nvfp4_quantize with the tensor scale computed (compute_global_scale = 1),
 * for callers that cannot allocate device memory: plug-ins whose host
 * framework owns the whole device memory pool and forbids raw cudaMalloc, or
 * latency-critical loops where a cudaMalloc/cudaFree would synchronise the
 * device.  The paper has no counterpart: this is an interface convenience.
 *
 * Instead of a caller workspace, the per-CTA maxima of the tensor-scale pass
 * live in a fixed array inside the library: 1024 floats (4 KB) that every
 * device which loads the library holds until the process exits.  The pass uses
 * at most 1024 CTAs, so every shape nvfp4_quantize accepts fits; a grid that
 * would need more partials is rejected with FP4LIN_ERR_UNSUPPORTED_SHAPE.
 * The call allocates nothing (no cudaMalloc, cudaFree or allocating library
 * routine).  The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) and caches it; make that first call before any
 * stream capture.  The cached address belongs to the device's primary context
 * as it was at that first call: after cudaDeviceReset on a device, do not call
 * this entry point on that device again in the same process (the address
 * would be stale); nvfp4_quantize with a caller workspace is unaffected.  All calls on a device share the array and it keeps the last
 * call's contents (nothing in it has to start at zero: each call overwrites
 * every partial it reads), so calls that overlap on the GPU -- on different
 * streams without ordering -- race and must be avoided.
 * Arguments, results and errors otherwise as nvfp4_quantize; g is OUTPUT.
 */
int nvfp4_quantize_noalloc(const void *x, int64_t rows, int64_t cols, int64_t ld_x,
                           int hadamard, float *g, uint8_t *codes, uint8_t *scales,
                           void *stream);

/*
 * Decode attention read straight from the NVFP4 KV cache (the story on NVFP4 KV
 * caches: new K/V rows are stored in NVFP4 and dequantised to FP8 before
 * attention).  The K and V values are exactly the FP8 values kv_nvfp4_load_fp8
 * would write, times 8 g_k / 8 g_v, but they are formed on chip: the FP8 copy
 * is neither written nor read.  Query head j of batch b uses kv head j / G:
 *   s_l = (q . k_l) / sqrt(D) for l < L, p = softmax(s), out = sum_l p_l v_l,
 * in binary32 (a split over L merged with rescaled sums).
 *   q: bf16 [B, H*G, D]; caches as kv_nvfp4_store; g_k, g_v device floats;
 *   out: float32 [B, H*G, D].
 * Shapes: D = 128, 1 <= G <= 8, 1 <= L <= Lcap, B*H <= 65535.  codes, q, out,
 * workspace 16-byte aligned, scales 8-byte aligned.  workspace of at least
 * kv_attention_workspace_bytes(B, H, G, L, D) bytes (else FP4LIN_ERR_WORKSPACE).
 */
size_t kv_attention_workspace_bytes(int B, int H, int G, int64_t L, int D);
int kv_nvfp4_attention(const void *q, const uint8_t *k_codes, const uint8_t *k_scales,
                       const float *g_k, const uint8_t *v_codes, const uint8_t *v_scales,
                       const float *g_v, int64_t L, float *out, int B, int H, int G,
                       int64_t Lcap, int D, void *workspace, size_t workspace_bytes, void *stream);

/*
 * nvfp4_gemm whose output is also NVFP4-quantised for the next layer, inside the
 * GEMM's epilogue (or its split-K reduction), so a chain of layers need not
 * write and re-read bf16.  The output is first rounded to bf16 exactly as
 * nvfp4_gemm rounds it; then each 16-value block of each output row is rotated
 * by H_16/4 when hadamard = 16 and encoded as nvfp4_quantize does with the
 * STATIC tensor scale *g_y: the codes and scales equal those of
 * nvfp4_quantize(y, hadamard, *g_y) applied to the bf16 y, bit for bit.
 *   y: bf16 [M, N] with row stride ldy, or NULL (then only the codes are written);
 *   y_codes [M, N/2]; y_scales tensor-core layout of [M, N/16] (padding zeroed).
 * Shapes as nvfp4_gemm and N a multiple of 64 (FP4LIN_ERR_UNSUPPORTED_SHAPE).
 * g_y device float (4-byte aligned); y_codes, y_scales 16-byte aligned.
 * Errors as nvfp4_gemm; hadamard not 0 or 16, or a null g_y, y_codes or
 * y_scales, give FP4LIN_ERR_INVALID_ARGUMENT.
 */
int nvfp4_gemm_quant(const uint8_t *a_codes, const uint8_t *a_scales, const float *g_a,
                     const uint8_t *w_codes, const uint8_t *w_scales, const float *g_w,
                     void *y, int64_t ldy, int hadamard, const float *g_y,
                     uint8_t *y_codes, uint8_t *y_scales, int64_t M, int64_t N, int64_t K,
                     void *workspace, size_t workspace_bytes, void *stream);

/*
 * NVFP4 quantisation with the block scale that minimises the block's squared
 * error (page "FP4 auf Blackwell: Was NVFP4 fuer lokale KI wirklich aendert",
 * section "Was NVFP4 von frueheren 4-Bit-Formaten unterscheidet": the scaling
 * algorithm picks the factor with the least mean squared error over the 16
 * values of a block).  Meant for weights, offline.  The tensor scale g is
 * nvfp4_quantize's (amax / 2688, computed or given); for every 16-value block
 * all 127 non-negative finite E4M3 codes c are tried: d = RN32(dec(c) * g),
 * r = RN32(1/d) (0 when d = 0), q_i = E2M1(RN32(x_i * r)), error = binary32
 * sum in order i = 0..15 of RN32(RN32(x_i - RN32(e2m1(q_i) * d))^2); the least
 * error wins, ties to the smaller code.  Tensors whose amax is below ~1e-32
 * (where 1/d overflows for small codes) are outside the specified range.
 * Arguments, layouts, workspace and errors exactly as nvfp4_quantize.
 */
int nvfp4_quantize_mse(const void *x, int64_t rows, int64_t cols, int64_t ld_x,
                       int hadamard, int compute_global_scale, float *g,
                       uint8_t *codes, uint8_t *scales,
                       void *workspace, size_t workspace_bytes, void *stream);

/*
 * MXFP4 quantisation with the E8M0 scale rounded to the nearest power of two
 * (same page and section: E8M0 rounds the scale factor to the nearest power
 * of two): the ideal scale amax/6 goes to the nearer of the two powers of two
 * around it, by value, ties upward.  With e = floor(log2 amax) that is
 * X = e - 2 when amax >= 1.125 * 2^e, else X = e - 3 (values then saturate at
 * 6); byte = clamp(X + 127, 0, 254), codes = E2M1 of x' * 2^-X.
 * Arguments, layouts and errors exactly as mxfp4_quantize.
 */
int mxfp4_quantize_nearest(const void *x, int64_t rows, int64_t cols, int64_t ld_x,
                           int hadamard, uint8_t *codes, uint8_t *scales, void *stream);

/*
 * Decode linear layer with the activation quantiser fused into the GEMM: the
 * bf16 activations go straight in, and the GEMM's own warps encode each
 * 16-row operand tile into shared memory as it is needed (the activations'
 * online rotation and quantisation, MR-GPTQ abstract, "Abstract"; the native
 * block-scaled FP4 product, "FP4 auf Blackwell", section "Was NVFP4 von
 * frueheren 4-Bit-Formaten unterscheidet").  No codes or scales of the
 * activations are written to memory and no quantiser is launched (one amax
 * pass when the tensor scale is computed).  The result equals, bit for bit,
 * nvfp4_quantize(x, hadamard, compute_global_scale, g_a) followed by
 * nvfp4_gemm(codes, scales, g_a, w_codes, w_scales, g_w, y); with
 * compute_global_scale = 1, *g_a is written with the same amax / 2688.
 *   x: bf16 [M, K], row stride ld_x (multiple of 8 elements, 16-byte aligned);
 *   w_codes / w_scales / g_w: the weights as nvfp4_gemm takes them (N x K);
 *   y: bf16 [M, N], row stride ldy (multiple of 8).
 * 1 <= M <= 16 (larger M: FP4LIN_ERR_UNSUPPORTED_SHAPE; use nvfp4_quantize +
 * nvfp4_gemm), K a multiple of 64.  workspace: at least
 * nvfp4_linear_decode_workspace_bytes(M, N, K) bytes (16-byte aligned): the
 * amax partials, then the split-K partial sums; with less (or NULL, only
 * allowed when compute_global_scale = 0) the GEMM runs without a K split.
 * Errors as nvfp4_quantize and nvfp4_gemm.
 */
size_t nvfp4_linear_decode_workspace_bytes(int64_t M, int64_t N, int64_t K);
int nvfp4_linear_decode(const void *x, int64_t M, int64_t K, int64_t ld_x, int hadamard,
                        int compute_global_scale, float *g_a,
                        const uint8_t *w_codes, const uint8_t *w_scales, const float *g_w,
                        void *y, int64_t N, int64_t ldy,
                        void *workspace, size_t workspace_bytes, void *stream);

/*
 * MR-GPTQ weight quantisation (offline): GPTQ's error-correcting column sweep
 * on the blockwise-Hadamard-rotated weights (MR-GPTQ abstract, "Abstract":
 * GPTQ adapted to FP4 with blockwise Hadamard transforms; "FP8, NVFP4 czy
 * AWQ?", section "Czym roznia sie FP8, NVFP4, MXFP4 i AWQ?": GPTQ quantises
 * weights layer by layer with error correction).  For every row of
 * W' = W blockdiag(H_b / sqrt b) (b = hadamard; 0 = no rotation), binary32:
 * for j = 0 .. K-1: at the first column of each 16- (NVFP4) or 32-value
 * (MXFP4) block, the block's scale is fixed from the row's current values by
 * the format's rule (nvfp4_quantize's, relative to the tensor scale *g; or
 * mxfp4_quantize's); q = the dequantised code of w_j; e = (w_j - q) / U[j][j];
 * then w_k = fma(-e, U[j][k], w_k) for every k > j, in increasing j.
 *   w: bf16 [N, K], row stride ld_w (multiple of 8), the weights as
 *      nvfp4_quantize / mxfp4_quantize take them (unrotated);
 *   u: float [K, K], row stride ld_u >= K (a multiple of 4; u 16-byte
 *      aligned): the upper Cholesky factor U of the damped inverse Hessian of
 *      the (rotated) layer inputs, H^-1 = U^T U; only entries with row <=
 *      column are read; U[j][j] > 0;
 *   codes [N, K/2], scales: tensor-core layout of [N, K/16] or [N, K/32] --
 *      ready for nvfp4_gemm / mxfp4_gemm with activations rotated the same way;
 *   g (NVFP4): the tensor scale; compute_global_scale = 1 writes the rotated
 *      W's amax / 2688 there (as nvfp4_quantize), 0 reads it;
 *   workspace: gptq_workspace_bytes(N, K) bytes, 16-byte aligned (W' in
 *      binary32, the errors of two 256-column superblocks, the tensor-scale
 *      partials).
 * The work forks from `stream` onto two streams the call creates (the column
 * sweep at the highest priority, the bulk corrections at the lowest) and joins
 * back into it before the call returns; both are released with the call.
 * K a multiple of 64.  Errors as nvfp4_quantize; a workspace below the size
 * gives FP4LIN_ERR_WORKSPACE.  Time grows as N K^2 (binary32 multiply-adds).
 */
size_t gptq_workspace_bytes(int64_t N, int64_t K);
/*
 * GPTQ's input from calibration activations: the factor u that the MR-GPTQ
 * entry points above take.  Defined by: the MR-GPTQ abstract
 * (hyper.ai/de/papers/2509.23202), "Abstract" -- MR-GPTQ is a variant of the
 * classic GPTQ algorithm with blockwise Hadamard transforms, so its Hessian
 * is that of the rotated layer inputs.  In binary64:
 *   x' = x blockdiag(H_b / sqrt b)   (b = hadamard: 16, 32, or 0 = none)
 *   H  = x'^T x' + damp * mean(diag(x'^T x')) * I
 *   u  = the upper triangular factor with positive diagonal, H^-1 = u^T u,
 *        rounded to float (entries below the diagonal written 0).
 * u is found without forming H^-1: with P the reversal of the K indices,
 * P H P = L L^T (blocked Cholesky, 64 x 64 blocks) and u = P L^-1 P.
 *   x: double [T, K], row stride ld_x >= K (8-byte aligned), the calibration
 *      activations (T tokens), unrotated;
 *   damp >= 0 (GPTQ's usual choice is 0.01);
 *   u: float [K, K], row stride ld_u >= K, 4-byte aligned;
 *   workspace: gptq_hessian_workspace_bytes(T, K) bytes, 16-byte aligned:
 *      8 * (T K + 2 K^2 + 128 K) bytes (the rotated activations, the
 *      Hessian's factor and its inverse, and 64-row blocks of products).
 * T >= 1; K a multiple of 64.  If H is not positive definite (a pivot not
 * positive and finite, e.g. all-zero or non-finite x with damp = 0),
 * FP4LIN_ERR_NUMERIC is recorded in the device status word (see
 * fp4lin_device_status) and u is not meaningful.  Other errors as
 * nvfp4_quantize; a workspace below the size gives FP4LIN_ERR_WORKSPACE.
 * Time grows as T K^2 + K^3 (binary64 multiply-adds).
 */
size_t gptq_hessian_workspace_bytes(int64_t T, int64_t K);
int gptq_hessian_factor(const double *x, int64_t T, int64_t K, int64_t ld_x, int hadamard,
                        double damp, float *u, int64_t ld_u,
                        void *workspace, size_t workspace_bytes, void *stream);
int nvfp4_gptq_quantize(const void *w, int64_t N, int64_t K, int64_t ld_w, int hadamard,
                        const float *u, int64_t ld_u, int compute_global_scale, float *g,
                        uint8_t *codes, uint8_t *scales,
                        void *workspace, size_t workspace_bytes, void *stream);
int mxfp4_gptq_quantize(const void *w, int64_t N, int64_t K, int64_t ld_w, int hadamard,
                        const float *u, int64_t ld_u, uint8_t *codes, uint8_t *scales,
                        void *workspace, size_t workspace_bytes, void *stream);
/*
 * nvfp4_gptq_quantize with each 16-value block's scale chosen, from the row's
 * current values at the block's first column, as nvfp4_quantize_mse chooses it
 * (least squared error over all 127 E4M3 codes, ties to the smaller code): the
 * format-specific scale of the MR-GPTQ abstract read as NVFP4's best scale.
 * Arguments and errors as nvfp4_gptq_quantize; slower (127 candidates per block).
 */
int nvfp4_gptq_quantize_mse(const void *w, int64_t N, int64_t K, int64_t ld_w, int hadamard,
                            const float *u, int64_t ld_u, int compute_global_scale, float *g,
                            uint8_t *codes, uint8_t *scales,
                            void *workspace, size_t workspace_bytes, void *stream);

/*
 * Decode weights in tile order.  The decode-sized GEMM (M <= 16) streams the
 * weights 128 rows x 256 values at a time.  In the row-major layout each such
 * stage is 128 strided runs of 128 bytes; prepared once in tile order, each
 * stage is one contiguous 16 KB block that a bulk copy lands in shared memory
 * as the exact 128-byte-swizzled operand image (16-byte chunk c of row r at
 * position c ^ (r % 8)).  Tile (mt, kt) -- rows 128 mt .. +127, code bytes
 * 128 kt .. +127 -- starts at byte (mt * ceil(K/256) + kt) * 16384; rows past N
 * and bytes past K/2 are zero.  The scales stay in the tensor-core layout.
 *   fp4lin_tiled_weight_bytes(N, K): the tiled buffer's size.
 *   fp4lin_tile_weights: codes [N, K/2] (as nvfp4_quantize writes them) -> tiled.
 *   nvfp4_gemm_tiled, nvfp4_linear_decode_tiled: nvfp4_gemm / nvfp4_linear_decode
 *   with the weights' codes in tile order (w_tiled); same results, bit for bit;
 *   M <= 16 (else FP4LIN_ERR_UNSUPPORTED_SHAPE).  K a multiple of 64; pointers
 *   16-byte aligned.  Errors as the untiled calls.
 */
size_t fp4lin_tiled_weight_bytes(int64_t N, int64_t K);
int fp4lin_tile_weights(const uint8_t *codes, int64_t N, int64_t K, uint8_t *tiled, void *stream);
int nvfp4_gemm_tiled(const uint8_t *a_codes, const uint8_t *a_scales, const float *g_a,
                     const uint8_t *w_tiled, const uint8_t *w_scales, const float *g_w,
                     void *y, int64_t M, int64_t N, int64_t K, int64_t ldy,
                     void *workspace, size_t workspace_bytes, void *stream);
int nvfp4_linear_decode_tiled(const void *x, int64_t M, int64_t K, int64_t ld_x, int hadamard,
                              int compute_global_scale, float *g_a,
                              const uint8_t *w_tiled, const uint8_t *w_scales, const float *g_w,
                              void *y, int64_t N, int64_t ldy,
                              void *workspace, size_t workspace_bytes, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* FP4LIN_H */
