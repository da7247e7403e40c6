/*
 * oracle.c -- the oracle: a plain, slow CPU reference for the NVFP4 / MXFP4
 * W4A4 linear layer and the NVFP4 KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may load it: only
 * tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference
 * legs do.  It shares no code, table or constant with the CUDA library.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -fopenmp -shared -fPIC.
 * Floating point is IEEE binary32 / binary64 with round-to-nearest-even and
 * no contraction, so every float expression below is evaluated exactly as
 * written, in the order written.
 *
 * Sources (web pages, cited by title and section):
 *   [FP4-BW]  "FP4 auf Blackwell: Was NVFP4 fuer lokale KI wirklich aendert"
 *             (aisyndicate.ch), section "Was NVFP4 von frueheren
 *             4-Bit-Formaten unterscheidet".
 *   [PL]      "FP8, NVFP4 czy AWQ? Kwantyzacja modeli na GPU Blackwell w
 *             praktyce" (pimento.cloud), section "Czym roznia sie FP8, NVFP4,
 *             MXFP4 i AWQ?".
 *   [MRGPTQ]  the MR-GPTQ abstract (hyper.ai/de/papers/2509.23202), "Abstract".
 *   [KV]      the NVFP4 KV-cache story (hyper.ai/de/stories/...).
 *
 * Readings where the pages are silent, garbled or in conflict:
 *   R1 E2M1 has exponent bias 1 (the pages give "about -6 to 6", which with
 *      1 sign / 2 exponent / 1 mantissa bit forces bias 1); encoding rounds to
 *      nearest, ties to the even code, saturates at 6, keeps the sign of zero.
 *   R2 E4M3 (the FP8 block scale) follows the OFP8 definition: bias 7, max 448,
 *      no infinities, S.1111.111 = NaN; encoding rounds to nearest even and
 *      saturates to 448 ("satfinite").
 *   R3 NVFP4: FP32 tensor scale g = amax_t / (6*448) (1 when that is not > 0);
 *      block scale sf = E4M3((amax_b / 6) / g); elements v = x * (1 / (dec(sf)*g)).
 *   R4 MXFP4 (OCP MX): scale exponent X = floor(log2 amax_b) - 2, stored as
 *      clamp(X + 127, 0, 254); elements v = x * 2^-X.
 *   R5 Blockwise Hadamard: Sylvester H_b, applied as an in-place fast
 *      Walsh-Hadamard transform with butterfly strides 1, 2, 4, ... and the
 *      pair (u, w) -> (u + w, u - w), then one multiply by RN32(1/sqrt(b)).
 *   R6 Codes: element 2i in the low nibble, 2i+1 in the high nibble.
 *   R7 Tensor-core scale layout: 128-row x 4-column atoms of 512 bytes, atoms
 *      ordered row-tile-major; in an atom, byte (r%32)*16 + ((r%128)/32)*4 + c%4.
 *   R8 KV: static per-tensor g; dequantised FP8 = E4M3(e2m1 * dec(sf) / 8),
 *      attention-side scale 8*g.
 *   R9 NVFP4 "MSE-optimal" block scale ([FP4-BW]: the scale minimises the mean
 *      squared error over the block's 16 values): every non-negative finite
 *      E4M3 code c = 0..126 is tried with d = RN32(dec(c)*g), r = RN32(1/d)
 *      (0 when d = 0), q_i = E2M1(RN32(x_i*r)); its error is the binary32 sum,
 *      in order i = 0..15, of RN32(RN32(x_i - RN32(e2m1(q_i)*d))^2); the
 *      smallest error wins, ties to the smaller code.  g is R3's.
 *   R10 MXFP4 "nearest power of two" ([FP4-BW]: the scale is rounded to the
 *      nearest power of two): the ideal scale amax/6 is rounded to the nearer
 *      of the two powers of two around it, by value, ties upward.  With
 *      e = floor(log2 amax) that is X = e-2 when amax >= 1.125*2^e, else e-3.
 *   R11 Decode attention over the NVFP4 KV cache ([KV] says only that the FP8
 *      copy feeds attention): G query heads per kv head (query head j uses kv
 *      head j / G), scores q . k / sqrt(D) over positions 0..L-1, softmax, the
 *      p-weighted sum of the values; q bf16, output fp32; no mask beyond L.
 *   R12 MR-GPTQ ([MRGPTQ]: GPTQ adapted to FP4 through blockwise Hadamard
 *      transforms; [PL]: GPTQ quantises weights layer by layer with error
 *      correction).  GPTQ's published column sweep, on the rotated weights
 *      W' = W R (R = blockdiag(H_b / sqrt b), b = the format's block, or no
 *      rotation) and the Hessian of the rotated inputs: U is the upper
 *      Cholesky factor of the damped inverse Hessian (H^-1 = U^T U), an input.
 *      Column j of every row: at the first column of each block (16 or 32) the
 *      block's scale is fixed from the row's current values of that block by
 *      the format's own rule (R3 with the static tensor scale g of the
 *      rotated W, or R4); q = the dequantised code; e = (w_j - q) / U[j][j];
 *      then w_k <- fma(-e, U[j][k], w_k) for every k > j, in binary32, so each
 *      value receives its corrections one at a time in increasing j.  Variant
 *      (NVFP4): the block scale chosen by R9 (least squared error over all 127
 *      E4M3 codes) from the block's current values, the abstract's
 *      format-specific optimisation read as the format's best scale.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define EXPORT __attribute__((visibility("default")))

/* ------------------------------------------------------------------ formats */

/* E2M1 magnitudes of codes 0..7 ([FP4-BW]: 1 sign, 2 exponent, 1 mantissa
 * bit; [PL]: range about +-6).  Code bit 3 is the sign. */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

EXPORT double oracle_e2m1_decode(uint8_t code)
{
    double m = E2M1_MAG[code & 7];
    return (code & 8) ? -m : m;
}

/* Nearest E2M1 magnitude, ties to the even code (the one whose mantissa bit,
 * the code's bit 0, is clear); anything beyond 6 becomes 6 (saturation).
 * The sign bit copies the input's sign, so small negatives give -0 (code 8). */
EXPORT uint8_t oracle_e2m1_encode(float v)
{
    double a = fabs((double)v);
    if (a > 6.0)
        a = 6.0; /* saturate first: far out, the distances to 4 and 6 round to the same double */
    int best = 0;
    double bd = a;
    for (int c = 1; c < 8; ++c) {
        double d = fabs(a - E2M1_MAG[c]);
        if (d < bd || (d == bd && (c & 1) == 0)) {
            best = c;
            bd = d;
        }
    }
    return (uint8_t)(best | (signbit(v) ? 8 : 0));
}

/* E4M3 (OFP8): s eeee mmm, bias 7; e = 0 is subnormal m*2^-9; S.1111.111 is NaN. */
EXPORT double oracle_e4m3_decode(uint8_t b)
{
    int e = (b >> 3) & 15, m = b & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp((double)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */
    return (b & 0x80) ? -v : v;
}

/* Nearest finite E4M3 value by search over the 127 non-negative finite codes,
 * ties to the even code; values above 448 become 448 (satfinite). */
EXPORT uint8_t oracle_e4m3_encode(float v)
{
    double a = fabs((double)v);
    if (a > 448.0)
        a = 448.0; /* satfinite */
    int best = 0;
    double bd = a;
    for (int c = 1; c <= 126; ++c) {
        double d = fabs(a - oracle_e4m3_decode((uint8_t)c));
        if (d < bd || (d == bd && (c & 1) == 0)) {
            best = c;
            bd = d;
        }
    }
    return (uint8_t)(best | (signbit(v) ? 0x80 : 0));
}

/* E8M0 ([FP4-BW], [PL]): a power of two 2^(e-127); 255 is NaN. */
EXPORT double oracle_e8m0_decode(uint8_t b)
{
    if (b == 255)
        return NAN;
    return ldexp(1.0, (int)b - 127);
}

static float bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round a double to the nearest bf16 (8 significant bits, ties to even) in one
 * step -- no detour through float, which would round twice. */
EXPORT uint16_t oracle_bf16_rn(double v)
{
    float f;
    uint32_t u;
    if (isnan(v))
        return 0x7FC0;
    double a = fabs(v);
    if (a == 0.0 || isinf(v)) {
        f = (float)v;
    } else {
        int e;
        frexp(a, &e);                 /* a in [2^(e-1), 2^e) */
        int ulp_exp = e - 8;          /* 8 significant bits */
        if (ulp_exp < -133)
            ulp_exp = -133;           /* bf16 subnormal spacing */
        double q = nearbyint(ldexp(a, -ulp_exp));
        double r = ldexp(q, ulp_exp);
        f = (float)r;                 /* exact, or +inf past the bf16 range */
        if (v < 0)
            f = -f;
    }
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------ rotation */

/* Sylvester Hadamard matrix: H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]]. */
EXPORT void oracle_hadamard_matrix(int b, int8_t *H)
{
    H[0] = 1;
    for (int n = 1; n < b; n <<= 1)
        for (int i = 0; i < n; ++i)
            for (int j = 0; j < n; ++j) {
                int8_t h = H[i * b + j];
                H[i * b + (j + n)] = h;
                H[(i + n) * b + j] = h;
                H[(i + n) * b + (j + n)] = (int8_t)-h;
            }
}

/* Normalisation 1/sqrt(b) rounded once to binary32. */
EXPORT float oracle_hadamard_norm(int b)
{
    return (float)(1.0 / sqrt((double)b));
}

/* In-place blockwise rotation x <- H_b x / sqrt(b) of one block of b values
 * ([MRGPTQ]: blockwise Hadamard transforms; reading R5 fixes the order). */
EXPORT void oracle_fwht(float *x, int b)
{
    for (int h = 1; h < b; h <<= 1)
        for (int i = 0; i < b; ++i)
            if ((i & h) == 0) {
                float u = x[i], w = x[i + h];
                x[i] = u + w;
                x[i + h] = u - w;
            }
    float c = oracle_hadamard_norm(b);
    for (int i = 0; i < b; ++i)
        x[i] = x[i] * c;
}

/* Load block `blk` (width b) of row `r`, rotated when `hadamard` is b. */
static void load_block(const uint16_t *x, int64_t ld, int64_t r, int64_t blk, int b,
                       int hadamard, float *out)
{
    const uint16_t *p = x + r * ld + blk * b;
    for (int i = 0; i < b; ++i)
        out[i] = bf16_to_f32(p[i]);
    if (hadamard == b)
        oracle_fwht(out, b);
}

/* ------------------------------------------------------------------ NVFP4 */

/* FP32 tensor scale, the second scaling level ([FP4-BW]; [PL]): reading R3,
 * g = amax_t / (6 * 448) over the (rotated) tensor, 1 when that is not > 0. */
EXPORT float oracle_nvfp4_tensor_scale(const uint16_t *x, int64_t rows, int64_t cols,
                                       int64_t ld, int hadamard)
{
    float amax = 0.0f, blk[16];
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < cols / 16; ++k) {
            load_block(x, ld, r, k, 16, hadamard, blk);
            for (int i = 0; i < 16; ++i)
                if (fabsf(blk[i]) > amax)
                    amax = fabsf(blk[i]);
        }
    float g = amax / 2688.0f;
    if (!(g > 0.0f))
        g = 1.0f;
    return g;
}

/* One 16-value block: E4M3 block scale relative to g, then E2M1 codes
 * ([FP4-BW]: one FP8 scale per 16 values plus one FP32 scale per tensor;
 * [PL]: E2M1, 16-value blocks; reading R3 for the exact steps). */
static uint8_t nvfp4_block(const float *x, float g, uint8_t *codes)
{
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i)
        if (fabsf(x[i]) > amax)
            amax = fabsf(x[i]);
    float t = (amax / 6.0f) / g;
    uint8_t sf = oracle_e4m3_encode(t);
    float d = (float)oracle_e4m3_decode(sf) * g;
    float rcp = (d > 0.0f) ? 1.0f / d : 0.0f;
    for (int i = 0; i < 16; ++i)
        codes[i] = oracle_e2m1_encode(x[i] * rcp);
    return sf;
}

/* One 16-value block with the MSE-optimal E4M3 block scale ([FP4-BW]: the
 * scaling algorithm picks the factor with the least mean squared error over
 * the block's 16 values; reading R9 for the candidate set, the arithmetic and
 * the tie rule).  Every candidate is tried: a brute-force search. */
static uint8_t nvfp4_block_mse(const float *x, float g, uint8_t *codes)
{
    int best = -1;
    float best_err = 0.0f;
    uint8_t q[16];
    for (int c = 0; c <= 126; ++c) {
        float d = (float)oracle_e4m3_decode((uint8_t)c) * g;
        float rcp = (d > 0.0f) ? 1.0f / d : 0.0f;
        float err = 0.0f;
        for (int i = 0; i < 16; ++i) {
            q[i] = oracle_e2m1_encode(x[i] * rcp);
            float t = (float)oracle_e2m1_decode(q[i]) * d;
            float diff = x[i] - t;
            err = err + diff * diff;
        }
        if (best < 0 || err < best_err) {
            best = c;
            best_err = err;
            memcpy(codes, q, 16);
        }
    }
    return (uint8_t)best;
}

/* NVFP4 quantisation with the MSE-optimal block scales (R9); same layouts and
 * tensor scale as oracle_nvfp4_quantize. */
EXPORT void oracle_nvfp4_quantize_mse(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                                      int hadamard, float g, uint8_t *codes, uint8_t *sf)
{
    int64_t nb = cols / 16;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < nb; ++k) {
            float blk[16];
            uint8_t c[16];
            load_block(x, ld, r, k, 16, hadamard, blk);
            sf[r * nb + k] = nvfp4_block_mse(blk, g, c);
            for (int j = 0; j < 8; ++j)
                codes[r * (cols / 2) + k * 8 + j] = (uint8_t)(c[2 * j] | (c[2 * j + 1] << 4));
        }
}

/* NVFP4 quantisation of a bf16 [rows, cols] matrix (row stride ld elements).
 * codes: [rows, cols/2] packed (R6).  sf: [rows, cols/16] row-major E4M3. */
EXPORT void oracle_nvfp4_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                                  int hadamard, float g, uint8_t *codes, uint8_t *sf)
{
    int64_t nb = cols / 16;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < nb; ++k) {
            float blk[16];
            uint8_t c[16];
            load_block(x, ld, r, k, 16, hadamard, blk);
            sf[r * nb + k] = nvfp4_block(blk, g, c);
            for (int j = 0; j < 8; ++j)
                codes[r * (cols / 2) + k * 8 + j] = (uint8_t)(c[2 * j] | (c[2 * j + 1] << 4));
        }
}

/* ------------------------------------------------------------------ MXFP4 */

/* One 32-value block with a power-of-two E8M0 scale ([FP4-BW]: MXFP4 from the
 * OCP Microscaling spec, E8M0 scaling, 32 values per block; [PL]: OCP,
 * 32-value blocks, power-of-two E8M0 scale; reading R4 for the exponent rule,
 * or R10 when `nearest`). */
static uint8_t mxfp4_block(const float *x, uint8_t *codes, int nearest)
{
    float amax = 0.0f;
    for (int i = 0; i < 32; ++i)
        if (fabsf(x[i]) > amax)
            amax = fabsf(x[i]);
    int byte;
    if (amax == 0.0f) {
        byte = 0;
    } else {
        int e;
        frexp((double)amax, &e);    /* amax = f * 2^e, f in [0.5, 1): floor(log2 amax) = e - 1 */
        int X = (e - 1) - 2;        /* 2 = exponent of E2M1's largest power of two, 4 */
        if (nearest && (double)amax < 1.125 * ldexp(1.0, e - 1))
            X -= 1;                 /* amax/6 < 1.5 * 2^(X-1): the lower power of two is nearer */
        byte = X + 127;
        if (byte < 0)
            byte = 0;
        if (byte > 254)
            byte = 254;
    }
    float s = ldexpf(1.0f, 127 - byte); /* 2^-X, exact */
    for (int i = 0; i < 32; ++i)
        codes[i] = oracle_e2m1_encode(x[i] * s);
    return (uint8_t)byte;
}

/* MXFP4 quantisation.  codes: [rows, cols/2]; sf: [rows, cols/32] row-major E8M0.
 * nearest = 0: the OCP exponent rule (R4); 1: the nearest power of two (R10). */
static void mxfp4_quantize_rule(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                                int hadamard, uint8_t *codes, uint8_t *sf, int nearest)
{
    int64_t nb = cols / 32;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < nb; ++k) {
            float blk[32];
            uint8_t c[32];
            load_block(x, ld, r, k, 32, hadamard, blk);
            sf[r * nb + k] = mxfp4_block(blk, c, nearest);
            for (int j = 0; j < 16; ++j)
                codes[r * (cols / 2) + k * 16 + j] = (uint8_t)(c[2 * j] | (c[2 * j + 1] << 4));
        }
}

EXPORT void oracle_mxfp4_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                                  int hadamard, uint8_t *codes, uint8_t *sf)
{
    mxfp4_quantize_rule(x, rows, cols, ld, hadamard, codes, sf, 0);
}

EXPORT void oracle_mxfp4_quantize_nearest(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                                          int hadamard, uint8_t *codes, uint8_t *sf)
{
    mxfp4_quantize_rule(x, rows, cols, ld, hadamard, codes, sf, 1);
}

/* ------------------------------------------------------------------ MR-GPTQ (R12) */

/* GPTQ ([PL]: weights quantised with error correction) in the MR-GPTQ form
 * ([MRGPTQ]: blockwise Hadamard rotations), reading R12.  GPTQ sweeps the
 * columns in order and corrects the later columns of every row by the same
 * rule; no step mixes two rows, so the sweep is done here one row at a time.
 * group: 16 (NVFP4, E4M3 scales relative to g) or 32 (MXFP4, E8M0 scales).
 * codes [N, K/2] (R6); sf [N, K/group] row-major; err [N, K] (optional): the
 * scaled errors e, the quantities GPTQ feeds back. */
static void gptq_sweep(const uint16_t *w, int64_t N, int64_t K, int64_t ld, int group, int hadamard,
                       const float *u, float g, int mse, uint8_t *codes, uint8_t *sf, float *err)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t n = 0; n < N; ++n) {
        float *row = malloc((size_t)K * sizeof(float));
        for (int64_t b = 0; b < K / group; ++b)
            load_block(w, ld, n, b, group, hadamard, row + b * group);
        float d = 0.0f, rcp = 0.0f, down = 1.0f, up = 1.0f;
        for (int64_t j = 0; j < K; ++j) {
            if (j % group == 0) { /* the block's scale, from its current values */
                float amax = 0.0f;
                for (int i = 0; i < group; ++i)
                    if (fabsf(row[j + i]) > amax)
                        amax = fabsf(row[j + i]);
                if (group == 16) { /* R3, or R9 with mse */
                    uint8_t scratch[16];
                    float t = (amax / 6.0f) / g;
                    uint8_t s = mse ? nvfp4_block_mse(row + j, g, scratch) : oracle_e4m3_encode(t);
                    d = (float)oracle_e4m3_decode(s) * g;
                    rcp = (d > 0.0f) ? 1.0f / d : 0.0f;
                    sf[n * (K / 16) + j / 16] = s;
                } else { /* R4 */
                    int byte = 0;
                    if (amax > 0.0f) {
                        int e;
                        frexp((double)amax, &e);
                        byte = (e - 1) - 2 + 127;
                        if (byte < 0)
                            byte = 0;
                        if (byte > 254)
                            byte = 254;
                    }
                    down = ldexpf(1.0f, 127 - byte);
                    up = ldexpf(1.0f, byte - 127);
                    sf[n * (K / 32) + j / 32] = (uint8_t)byte;
                }
            }
            uint8_t c = oracle_e2m1_encode(group == 16 ? row[j] * rcp : row[j] * down);
            float q = (float)oracle_e2m1_decode(c) * (group == 16 ? d : up);
            uint8_t *cb = codes + n * (K / 2) + j / 2;
            *cb = (j & 1) ? (uint8_t)(*cb | (c << 4)) : c;
            float e = (row[j] - q) / u[j * K + j];
            if (err)
                err[n * K + j] = e;
            for (int64_t k = j + 1; k < K; ++k)
                row[k] = fmaf(-e, u[j * K + k], row[k]);
        }
        free(row);
    }
}

EXPORT void oracle_gptq(const uint16_t *w, int64_t N, int64_t K, int64_t ld, int group, int hadamard,
                        const float *u, float g, uint8_t *codes, uint8_t *sf, float *err)
{
    gptq_sweep(w, N, K, ld, group, hadamard, u, g, 0, codes, sf, err);
}

/* MR-GPTQ with R9's MSE-optimal NVFP4 block scales (group 16). */
EXPORT void oracle_gptq_mse(const uint16_t *w, int64_t N, int64_t K, int64_t ld, int hadamard, const float *u,
                            float g, uint8_t *codes, uint8_t *sf, float *err)
{
    gptq_sweep(w, N, K, ld, 16, hadamard, u, g, 1, codes, sf, err);
}

/* ------------------------------------------------------------------ scale layout (R7) */

EXPORT int64_t oracle_tc_scale_bytes(int64_t rows, int64_t sf_cols)
{
    return ((rows + 127) / 128) * 128 * (((sf_cols + 3) / 4) * 4);
}

/* Row-major [rows, sf_cols] scale bytes -> the tensor-core atom layout; padding is 0. */
EXPORT void oracle_tc_scale_layout(const uint8_t *lin, int64_t rows, int64_t sf_cols, uint8_t *out)
{
    int64_t katoms = (sf_cols + 3) / 4;
    memset(out, 0, (size_t)oracle_tc_scale_bytes(rows, sf_cols));
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < sf_cols; ++c) {
            int64_t atom = (r / 128) * katoms + c / 4;
            int64_t off = atom * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4);
            out[off] = lin[r * sf_cols + c];
        }
}

/* ------------------------------------------------------------------ GEMM reference */

/* Dequantise rows of a packed FP4 matrix: out[r][k] = e2m1(code) * dec(sf) * g,
 * exactly, in binary64.  block = 16 with E4M3 scales (sf_kind 0) or 32 with
 * E8M0 scales (sf_kind 1); sf is row-major [rows, cols/block]. */
EXPORT void oracle_dequant(const uint8_t *codes, const uint8_t *sf, int64_t rows, int64_t cols,
                           int block, int sf_kind, double g, double *out)
{
    int64_t nb = cols / block;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < cols; ++k) {
            uint8_t byte = codes[r * (cols / 2) + k / 2];
            uint8_t c = (k & 1) ? (byte >> 4) : (byte & 15);
            uint8_t s = sf[r * nb + k / block];
            double sc = sf_kind ? oracle_e8m0_decode(s) : oracle_e4m3_decode(s);
            out[r * cols + k] = oracle_e2m1_decode(c) * sc * g;
        }
}

/* y = A W^T and s = sum |a_k w_k| in binary64 for A [M,K], W [N,K] (the plain
 * definition of the linear layer over the dequantised operands). */
EXPORT void oracle_gemm_abt(const double *A, const double *W, int64_t M, int64_t N, int64_t K,
                            double *y, double *s)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0, mag = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double p = A[m * K + k] * W[n * K + k];
                acc += p;
                mag += fabs(p);
            }
            y[m * N + n] = acc;
            s[m * N + n] = mag;
        }
}

EXPORT int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------ KV cache ([KV]) */

/* Append T new rows per (b, h) at positions pos[b] .. pos[b]+T-1: each row of D
 * values is NVFP4-quantised along D in 16-blocks with the static FP32 scale g.
 * kv_new: bf16 [B,H,T,D]; cache codes [B,H,Lcap,D/2]; cache sf [B,H,Lcap,D/16]. */
EXPORT void oracle_kv_store(const uint16_t *kv_new, const int32_t *pos, float g,
                            uint8_t *cache_codes, uint8_t *cache_sf, int B, int H, int T,
                            int64_t Lcap, int D)
{
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            for (int t = 0; t < T; ++t) {
                int64_t src_row = ((int64_t)b * H + h) * T + t;
                int64_t dst_row = ((int64_t)b * H + h) * Lcap + pos[b] + t;
                oracle_nvfp4_quantize(kv_new + src_row * D, 1, D, D, 0, g,
                                      cache_codes + dst_row * (D / 2), cache_sf + dst_row * (D / 16));
            }
}

/* Dequantise the first L positions of every (b, h) to FP8 E4M3 (reading R8):
 * fp8 = E4M3(e2m1(c) * dec(sf) / 8).  The product is exact in binary32, so the
 * E4M3 rounding is the only rounding.  out: [B,H,L,D]. */
EXPORT void oracle_kv_load_fp8(const uint8_t *cache_codes, const uint8_t *cache_sf, int64_t L,
                               int B, int H, int64_t Lcap, int D, uint8_t *out)
{
    for (int64_t bh = 0; bh < (int64_t)B * H; ++bh)
        for (int64_t l = 0; l < L; ++l) {
            int64_t row = bh * Lcap + l;
            for (int d = 0; d < D; ++d) {
                uint8_t byte = cache_codes[row * (D / 2) + d / 2];
                uint8_t c = (d & 1) ? (byte >> 4) : (byte & 15);
                double v = oracle_e2m1_decode(c) * oracle_e4m3_decode(cache_sf[row * (D / 16) + d / 16]) * 0.125;
                out[(bh * L + l) * D + d] = oracle_e4m3_encode((float)v);
            }
        }
}

/* The FP8 value (R8) of one cached element, times 8g: the value attention reads. */
static double kv_fp8_value(const uint8_t *codes_row, const uint8_t *sf_row, int d, double g8)
{
    uint8_t byte = codes_row[d / 2];
    uint8_t c = (d & 1) ? (byte >> 4) : (byte & 15);
    double v = oracle_e2m1_decode(c) * oracle_e4m3_decode(sf_row[d / 16]) * 0.125;
    return oracle_e4m3_decode(oracle_e4m3_encode((float)v)) * g8;
}

/* Decode attention over the cache as attention reads it after the FP8 load ([KV]:
 * new K/V rows stored in NVFP4 and dequantised to FP8 before attention; reading
 * R11 for the attention itself): query head j of batch b uses kv head h = j / G;
 * k_l, v_l are the FP8 values of position l times 8g; s_l = (q . k_l) / sqrt(D);
 * p = softmax(s) over l < L; o = sum_l p_l v_l.  binary64 throughout.
 * q: bf16 [B, H*G, D]; caches as oracle_kv_store; out: [B, H*G, D]. */
EXPORT void oracle_kv_attention(const uint16_t *q, const uint8_t *kc, const uint8_t *ks, float gk,
                                const uint8_t *vc, const uint8_t *vs, float gv, int64_t L, int B, int H,
                                int G, int64_t Lcap, int D, double *out)
{
    const double gk8 = 8.0 * (double)gk, gv8 = 8.0 * (double)gv, inv_sqrt_d = 1.0 / sqrt((double)D);
#pragma omp parallel for schedule(dynamic)
    for (int64_t bh = 0; bh < (int64_t)B * H; ++bh) {
        double *kv = (double *)malloc((size_t)L * D * sizeof(double));
        double *vv = (double *)malloc((size_t)L * D * sizeof(double));
        double *s = (double *)malloc((size_t)L * sizeof(double));
        for (int64_t l = 0; l < L; ++l) {
            int64_t row = bh * Lcap + l;
            for (int d = 0; d < D; ++d) {
                kv[l * D + d] = kv_fp8_value(kc + row * (D / 2), ks + row * (D / 16), d, gk8);
                vv[l * D + d] = kv_fp8_value(vc + row * (D / 2), vs + row * (D / 16), d, gv8);
            }
        }
        const int64_t b = bh / H, h = bh % H;
        for (int j = 0; j < G; ++j) {
            const uint16_t *qr = q + ((b * H + h) * G + j) * (int64_t)D;
            double m = -INFINITY;
            for (int64_t l = 0; l < L; ++l) {
                double acc = 0.0;
                for (int d = 0; d < D; ++d)
                    acc += (double)bf16_to_f32(qr[d]) * kv[l * D + d];
                s[l] = acc * inv_sqrt_d;
                if (s[l] > m)
                    m = s[l];
            }
            double sum = 0.0;
            for (int64_t l = 0; l < L; ++l) {
                s[l] = exp(s[l] - m);
                sum += s[l];
            }
            double *o = out + ((b * H + h) * G + j) * (int64_t)D;
            for (int d = 0; d < D; ++d) {
                double acc = 0.0;
                for (int64_t l = 0; l < L; ++l)
                    acc += s[l] * vv[l * D + d];
                o[d] = acc / sum;
            }
        }
        free(kv);
        free(vv);
        free(s);
    }
}
