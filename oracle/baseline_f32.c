/*
 * baseline_f32.c -- the CPU baseline the benchmark times: the grouped GEMMs
 * of a MoE expert layer on bf16 inputs with fp32 accumulation, OpenMP over
 * experts x row blocks.
 *
 * TEST INFRASTRUCTURE ONLY, like the rest of oracle/: it is a reported
 * baseline, never a parity reference (the fp64 oracle in mxfp8_oracle.c is
 * that).  It computes the grouped GEMM's definition (iitak.ru, "NVIDIA ...
 * JAX", Transformer Engine paragraph: every expert on its own token rows)
 *   Y_e = X_e W_e^T,  dX_e = dY_e W_e,  dW_e = dY_e^T X_e
 * with bf16 operands widened to fp32 and fp32 sums.  Loops are blocked over
 * 8 rows so each weight row is read once per block, and written so the
 * compiler vectorises the inner loops (8 partial sums per dot product); it is
 * built with -O3 and FMA contraction, so its rounding differs from a plain
 * left-to-right fp32 sum.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define RB 8   /* rows per block */

static inline float bf(uint16_t b) { uint32_t u = (uint32_t)b << 16; float f; memcpy(&f, &u, 4); return f; }

static int32_t group_of(const int32_t* offs, int32_t E, int64_t r)
{
    int32_t lo = 0, hi = E - 1;
    while (lo < hi) {
        int32_t mid = (lo + hi + 1) / 2;
        if (offs[mid] <= r) lo = mid; else hi = mid - 1;
    }
    return lo;
}

static int bad_offsets(const int32_t* offs, int32_t E, int64_t M)
{
    int32_t e;
    if (offs[0] != 0 || offs[E] != M) return 1;
    for (e = 0; e < E; ++e) if (offs[e + 1] < offs[e]) return 1;
    return 0;
}

/* Y = X_e W_e^T for rows [row_lo, row_hi) (a bounded sample). */
int orc_baseline_fwd_f32(const uint16_t* X, const uint16_t* W, const int32_t* offs, int32_t E,
                         int64_t M, int64_t N, int64_t K, int64_t row_lo, int64_t row_hi, float* Y)
{
    int64_t nblk = (row_hi - row_lo + RB - 1) / RB;
    int fail = 0;
    if (bad_offsets(offs, E, M) || K % 8 != 0) return 1;
#pragma omp parallel
    {
        float* xf = (float*)malloc(sizeof(float) * RB * K);
        int64_t b;
        if (!xf) fail = 1;
#pragma omp for schedule(dynamic, 1)
        for (b = 0; b < nblk; ++b) {
            int64_t i0 = row_lo + b * RB, n, k;
            int r, nr = 0, l;
            int32_t e[RB];
            if (!xf) continue;
            /* a block may cross an expert boundary: every row keeps its own expert */
            for (r = 0; r < RB && i0 + r < row_hi; ++r) {
                e[r] = group_of(offs, E, i0 + r);
                for (k = 0; k < K; ++k) xf[r * K + k] = bf(X[(i0 + r) * K + k]);
                nr = r + 1;
            }
            for (n = 0; n < N; ++n) {
                for (r = 0; r < nr; ++r) {
                    const uint16_t* w = W + ((int64_t)e[r] * N + n) * K;
                    const float* x = xf + r * K;
                    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0}, s = 0.0f;
                    for (k = 0; k < K; k += 8)
                        for (l = 0; l < 8; ++l) acc[l] += x[k + l] * bf(w[k + l]);
                    for (l = 0; l < 8; ++l) s += acc[l];
                    Y[(i0 + r) * N + n] = s;
                }
            }
        }
        free(xf);
    }
    return fail;
}

/* dX = dY_e W_e for rows [row_lo, row_hi). */
int orc_baseline_dgrad_f32(const uint16_t* dY, const uint16_t* W, const int32_t* offs, int32_t E,
                           int64_t M, int64_t N, int64_t K, int64_t row_lo, int64_t row_hi, float* dX)
{
    int64_t nblk = (row_hi - row_lo + RB - 1) / RB, b;
    if (bad_offsets(offs, E, M)) return 1;
#pragma omp parallel for schedule(dynamic, 1)
    for (b = 0; b < nblk; ++b) {
        int64_t i0 = row_lo + b * RB, n, k;
        int r, nr = (int)(row_hi - i0 < RB ? row_hi - i0 : RB);
        int32_t e[RB];
        for (r = 0; r < nr; ++r) {
            e[r] = group_of(offs, E, i0 + r);
            for (k = 0; k < K; ++k) dX[(i0 + r) * K + k] = 0.0f;
        }
        for (n = 0; n < N; ++n)
            for (r = 0; r < nr; ++r) {
                const float d = bf(dY[(i0 + r) * N + n]);
                const uint16_t* w = W + ((int64_t)e[r] * N + n) * K;
                float* out = dX + (i0 + r) * K;
                for (k = 0; k < K; ++k) out[k] += d * bf(w[k]);
            }
    }
    return 0;
}

/* dW_e = dY_e^T X_e for output rows n in [n_lo, n_hi) of every expert. */
int orc_baseline_wgrad_f32(const uint16_t* dY, const uint16_t* X, const int32_t* offs, int32_t E,
                           int64_t M, int64_t N, int64_t K, int64_t n_lo, int64_t n_hi, float* dW)
{
    int64_t nb = (n_hi - n_lo + RB - 1) / RB, en;
    if (bad_offsets(offs, E, M)) return 1;
#pragma omp parallel for schedule(dynamic, 1)
    for (en = 0; en < (int64_t)E * nb; ++en) {
        int32_t e = (int32_t)(en / nb);
        int64_t n0 = n_lo + (en % nb) * RB, i, k;
        int r, nr = (int)(n_hi - n0 < RB ? n_hi - n0 : RB);
        for (r = 0; r < nr; ++r)
            for (k = 0; k < K; ++k) dW[((int64_t)e * N + n0 + r) * K + k] = 0.0f;
        for (i = offs[e]; i < offs[e + 1]; ++i) {
            const uint16_t* x = X + i * K;
            for (r = 0; r < nr; ++r) {
                const float d = bf(dY[i * N + n0 + r]);
                float* out = dW + ((int64_t)e * N + n0 + r) * K;
                for (k = 0; k < K; ++k) out[k] += d * bf(x[k]);
            }
        }
    }
    return 0;
}
