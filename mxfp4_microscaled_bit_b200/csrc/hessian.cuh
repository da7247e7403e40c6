// hessian.cuh -- GPTQ's input, prepared on the GPU in binary64: the upper triangular factor U
// with H^-1 = U^T U of the damped Hessian H = x'^T x' + damp * mean(diag) * I of the
// calibration activations x [T, K], rotated blockwise (x' = x H_b / sqrt(b) per b-value block
// along K, b = 16 or 32, or no rotation).
//
// MR-GPTQ is "a variant of the classic GPTQ algorithm" with blockwise Hadamard transforms
// (the MR-GPTQ abstract, hyper.ai/de/papers/2509.23202, "Abstract"); GPTQ's column sweep
// reads the inverse Hessian through exactly this factor.
//
// The factor without an explicit inverse.  Let P reverse the order of K indices.  The
// Cholesky factorisation P H P = Lr Lr^T (Lr lower, positive diagonal) gives
// H = (P Lr P)(P Lr P)^T, so H^-1 = (P Lr^-1 P)^T (P Lr^-1 P), and U = P Lr^-1 P is upper
// triangular with a positive diagonal: the unique such factor.  The rotation pass writes
// x' with its columns reversed, so the Gram product of that copy is P H P directly; one
// blocked Cholesky and one blocked triangular inverse follow, and the output pass undoes P.
//
// Kernels (all binary64, 64 x 64 blocks):
//   hess_rotate_kernel     x -> x'P (rotated, columns reversed)
//   dgemm_kernel           C = beta C + alpha A B^T with general strides (lower-triangle
//                          option, batched): the Gram product, the Cholesky trailing
//                          updates and the inverse's block products
//   hess_damp_kernel       diag += damp * mean(diag) (fixed summation order)
//   chol_diag_kernel       Cholesky of one diagonal block and the inverse of its factor
//   chol_panel_kernel      the panel below it times that inverse, transposed
//   hess_out_kernel        U(i, j) = float(Lr^-1(K-1-i, K-1-j)), zero below the diagonal
// A non-positive (or non-finite) pivot records FP4LIN_ERR_NUMERIC in the device status word.
#pragma once

#include "common.cuh"

namespace fp4lin {

constexpr int HB = 64;  // block size of the factorisation and of the GEMM tiles

// x' = rotated x, written column-reversed: xr[t][K-1-i] = x'[t][i].  One thread per b-value
// block (B = 1: no rotation).  Butterflies (u, w) -> (u + w, u - w) at strides 1, 2, ..., then
// one multiply by 1/sqrt(b).
template <int B>
__global__ void __launch_bounds__(256) hess_rotate_kernel(const double *x, int64_t T, int64_t K, int64_t ld_x,
                                                          double *xr)
{
    const int64_t nb = K / B, total = T * nb;
    const double s = B == 1 ? 1.0 : 1.0 / sqrt((double)B);
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / nb, blk = i - t * nb;
        double v[B];
#pragma unroll
        for (int j = 0; j < B; ++j)
            v[j] = x[t * ld_x + blk * B + j];
#pragma unroll
        for (int h = 1; h < B; h <<= 1)
#pragma unroll
            for (int j = 0; j < B; ++j)
                if ((j & h) == 0) {
                    const double u = v[j], w = v[j + h];
                    v[j] = u + w;
                    v[j + h] = u - w;
                }
        double *dst = xr + t * K + (K - 1 - blk * B);
#pragma unroll
        for (int j = 0; j < B; ++j)
            dst[-j] = B == 1 ? v[j] : v[j] * s;
    }
}

// C(m, n) = beta * C(m, n) + alpha * sum_k A(m, k) B(n, k) for m < M, n < N, with
// A(m, k) = a[m * sam + k * sak], B(n, k) = b[n * sbn + k * sbk], C(m, n) = c[m * ldc + n];
// batch z offsets a, b and c by z * bza, z * bzb, z * bzc.  LOWER: only m >= n is computed and
// written (tiles wholly above the diagonal are skipped).  AK / BK: the operand is contiguous
// along k (sak or sbk == 1), else along m / n (sam or sbn == 1); this picks the loads' order
// only.  beta == 0 writes without reading C.  64 x 64 tiles, 16 values of k per stage, 256
// threads with a 4 x 4 block of C each.
struct DgemmArgs {
    const double *a, *b;
    double *c;
    int64_t M, N, Kd;
    int64_t sam, sak, sbn, sbk, ldc;
    int64_t bza, bzb, bzc;
    double alpha, beta;
};

template <bool AK, bool BK, bool LOWER>
__global__ void __launch_bounds__(256) dgemm_kernel(DgemmArgs p)
{
    constexpr int TK = 16;
    __shared__ double As[TK][HB + 1], Bs[TK][HB + 1];
    const int64_t m0 = (int64_t)blockIdx.y * HB, n0 = (int64_t)blockIdx.x * HB;
    if (LOWER && m0 + HB - 1 < n0)
        return;
    const int64_t z = blockIdx.z;
    const double *a = p.a + z * p.bza, *b = p.b + z * p.bzb;
    double *c = p.c + z * p.bzc;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    double acc[4][4] = {};
    for (int64_t k0 = 0; k0 < p.Kd; k0 += TK) {
        // stage 64 x 16 of each operand: 4 values per thread
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            int mm, kk;
            if (AK) {  // consecutive threads walk k
                mm = (tid >> 4) + 16 * r;
                kk = tid & 15;
            } else {   // consecutive threads walk m
                mm = tid & 63;
                kk = (tid >> 6) + 4 * r;
            }
            const int64_t gm = m0 + mm, gk = k0 + kk;
            As[kk][mm] = (gm < p.M && gk < p.Kd) ? a[gm * p.sam + gk * p.sak] : 0.0;
            int nn, kb;
            if (BK) {
                nn = (tid >> 4) + 16 * r;
                kb = tid & 15;
            } else {
                nn = tid & 63;
                kb = (tid >> 6) + 4 * r;
            }
            const int64_t gn = n0 + nn, gkb = k0 + kb;
            Bs[kb][nn] = (gn < p.N && gkb < p.Kd) ? b[gn * p.sbn + gkb * p.sbk] : 0.0;
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < TK; ++k) {
            double av[4], bv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                av[i] = As[k][ty * 4 + i];
                bv[i] = Bs[k][tx * 4 + i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    acc[i][j] = fma(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t m = m0 + ty * 4 + i;
        if (m >= p.M)
            continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t n = n0 + tx * 4 + j;
            if (n >= p.N || (LOWER && m < n))
                continue;
            double *dst = c + m * p.ldc + n;
            *dst = p.beta == 0.0 ? p.alpha * acc[i][j] : fma(p.alpha, acc[i][j], p.beta * *dst);
        }
    }
}

// diag(a) += damp * mean(diag(a)); one CTA, the sum in a fixed order.
__global__ void __launch_bounds__(256) hess_damp_kernel(double *a, int64_t K, double damp)
{
    __shared__ double part[256];
    double s = 0.0;
    for (int64_t i = threadIdx.x; i < K; i += 256)
        s += a[i * K + i];
    part[threadIdx.x] = s;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if (threadIdx.x < w)
            part[threadIdx.x] += part[threadIdx.x + w];
        __syncthreads();
    }
    const double add = damp * (part[0] / (double)K);
    for (int64_t i = threadIdx.x; i < K; i += 256)
        a[i * K + i] += add;
}

// Cholesky of diagonal block kb of a (lower triangle read), in place, and the inverse of the
// factor into dinv[kb] (64 x 64, row-major, zeros above the diagonal).  One CTA of 256 threads.
__global__ void __launch_bounds__(256) chol_diag_kernel(double *a, int64_t K, int kb, double *dinv)
{
    __shared__ double L[HB][HB + 1];
    __shared__ int bad;
    const int tid = threadIdx.x;
    double *blk = a + (int64_t)kb * HB * K + (int64_t)kb * HB;
    for (int e = tid; e < HB * HB; e += 256) {
        const int r = e >> 6, c = e & 63;
        L[r][c] = c <= r ? blk[(int64_t)r * K + c] : 0.0;
    }
    if (tid == 0)
        bad = 0;
    __syncthreads();
    for (int j = 0; j < HB; ++j) {
        if (tid == 0) {
            const double d = L[j][j];
            if (!(d > 0.0) || !isfinite(d)) {
                bad = 1;
                L[j][j] = 1.0;
            } else {
                L[j][j] = sqrt(d);
            }
        }
        __syncthreads();
        const double piv = L[j][j];
        for (int i = j + 1 + tid; i < HB; i += 256)
            L[i][j] /= piv;
        __syncthreads();
        // trailing update of the block: L[i][k] -= L[i][j] L[k][j], j < k <= i
        for (int e = tid; e < HB * HB; e += 256) {
            const int i = e >> 6, k = e & 63;
            if (k > j && k <= i)
                L[i][k] -= L[i][j] * L[k][j];
        }
        __syncthreads();
    }
    if (tid == 0 && bad)
        report_error(FP4LIN_ERR_NUMERIC);
    // dinv[kb] = L^-1 by forward substitution, one column per thread; each thread reads back
    // only the entries of its own column it has written
    double *dv = dinv + (int64_t)kb * HB * HB;
    if (tid < HB) {
        const int c = tid;
        for (int i = 0; i < HB; ++i) {
            if (i < c) {
                dv[i * HB + c] = 0.0;
                continue;
            }
            double s = i == c ? 1.0 : 0.0;
            for (int k = c; k < i; ++k)
                s -= L[i][k] * dv[k * HB + c];
            dv[i * HB + c] = s / L[i][i];
        }
    }
    for (int e = tid; e < HB * HB; e += 256) {
        const int r = e >> 6, c = e & 63;
        if (c <= r)
            blk[(int64_t)r * K + c] = L[r][c];
    }
}

// Panel below diagonal block kb: a[i, kb] <- a[i, kb] * dinv[kb]^T for block rows i > kb
// (blockIdx.x = i - kb - 1).  Each CTA owns its 64 x 64 block, so it works in place.
__global__ void __launch_bounds__(256) chol_panel_kernel(double *a, int64_t K, int kb, const double *dinv)
{
    __shared__ double P[HB][HB + 1];
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int64_t i = kb + 1 + blockIdx.x;
    double *blk = a + i * HB * K + (int64_t)kb * HB;
    const double *dv = dinv + (int64_t)kb * HB * HB;  // 32 KB, read through the L1 by every thread
    for (int e = tid; e < HB * HB; e += 256) {
        const int r = e >> 6, c = e & 63;
        P[r][c] = blk[(int64_t)r * K + c];
    }
    __syncthreads();
    double acc[4][4] = {};
    for (int k = 0; k < HB; ++k) {
        double pv[4], dw[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            pv[q] = P[ty * 4 + q][k];
            dw[q] = __ldg(dv + (tx * 4 + q) * HB + k);
        }
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c)
                acc[r][c] = fma(pv[r], dw[c], acc[r][c]);
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c)
            blk[(int64_t)(ty * 4 + r) * K + tx * 4 + c] = acc[r][c];
}

// X's diagonal blocks from the stored block inverses; everything above them zero.
__global__ void __launch_bounds__(256) hess_inv_init_kernel(double *xinv, int64_t K, const double *dinv)
{
    const int64_t total = K * K;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = e / K, c = e - r * K;
        const int64_t br = r / HB, bc = c / HB;
        double v = 0.0;
        if (br == bc)
            v = dinv[br * HB * HB + (r - br * HB) * HB + (c - bc * HB)];
        if (br >= bc)  // blocks below the diagonal are overwritten later; zero them anyway
            xinv[e] = br == bc ? v : 0.0;
        else
            xinv[e] = 0.0;
    }
}

// u(i, j) = float(xinv(K-1-i, K-1-j)) for i <= j, 0 below the diagonal.
__global__ void __launch_bounds__(256) hess_out_kernel(const double *xinv, int64_t K, float *u, int64_t ld_u)
{
    const int64_t total = K * K;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = e / K, j = e - i * K;
        u[i * ld_u + j] = i <= j ? (float)xinv[(K - 1 - i) * K + (K - 1 - j)] : 0.0f;
    }
}

}  // namespace fp4lin
