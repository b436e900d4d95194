/*
 * mxfp8_oracle.c -- plain, slow CPU oracle for MXFP8 quantisation and the
 * dropless grouped GEMM of a Mixture-of-Experts expert layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only the tests, the package's smoke check and the CPU
 * baseline leg of the benchmark use it.  It shares no source with the CUDA
 * library (no headers, helpers or tables) and includes nothing from it.
 *
 * What it follows:
 *   - MXFP8 is a microscaling format in which a block of 32 consecutive
 *     elements shares one exponent (opensourcebeat.com, "Enabling up to 41%
 *     faster pre-training: MXFP8 and DeepEP ...", FAQ "What is MXFP8?").
 *     The block rules are those of the OCP Microscaling (MX) v1.0
 *     specification: E8M0 scale X = 2^(floor(log2(amax)) - emax),
 *     emax = 8 for E4M3, clamped to the E8M0 range; element = E4M3(v / X)
 *     with round-to-nearest-even and saturation to +-448.
 *   - The grouped GEMM computes every expert on its real token count, with
 *     no padding to a capacity (iitak.ru, "NVIDIA ... JAX", paragraph on the
 *     Transformer Engine grouped GEMM): Y_e = X_e W_e^T, dX_e = dY_e W_e,
 *     dW_e = dY_e^T X_e, each per expert e over rows offs[e]..offs[e+1]-1.
 *
 * Readings where the pages are silent:
 *   - an all-zero block has scale exponent -127 (byte 0x00) and zero codes;
 *   - the sign of zero survives quantisation (-0 and negative underflow
 *     encode as 0x80), as IEEE round-to-nearest-even gives;
 *   - a block whose amax is Inf or NaN is outside the contract; it gets the
 *     NaN scale byte 0xFF and NaN codes 0x7F;
 *   - colwise blocks restart at every group offset; a group's last block may
 *     be short and its amax is over the real rows only.
 *
 * Data layouts (a format definition, restated here independently of the
 * CUDA library):
 *   rowwise: codes keep the [R, C] input layout.  Scales form a logical
 *     matrix S[pr, j] (pr = padded row, j = 32-block index along C) in which
 *     each group's rows start at a multiple of 128 (pr = 128*RB_g + t for
 *     row offs[g] + t, RB_g = sum over h<g of ceil(m_h/128)).
 *   colwise: codes are transposed, qT[c, P_g + t] for element (offs[g]+t, c),
 *     P_g = sum over h<g of round_up(m_h, 32); the pad columns up to
 *     round_up(m_g, 32) hold 0x00.  Scales form S^T[c, 4*RB_g + t/32].
 *   Both scale matrices are stored in 512-byte atoms of 128 rows x 4 block
 *     columns; atom (rb, cb) sits at byte (rb*pitch + cb)*512 and element
 *     (row, col) inside it at (row%32)*16 + ((row%128)/32)*4 + col%4.  Pad
 *     bytes inside a written atom are 0x00.  pitch = ceil(C/128) for rowwise,
 *     ceil(R/128) + G - 1 for colwise.  The colwise code row stride is
 *     ldT = round_up(round_up(R, 32) + 32*(G-1), 128), at least 128.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* Scalars                                                              */
/* ------------------------------------------------------------------ */

/* bf16 is the top half of an IEEE binary32; widening to double is exact. */
double orc_bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* E4M3 "fn": sign, 4 exponent bits with bias 7, 3 mantissa bits.  No
 * infinities; S.1111.111 is NaN.  Normal: (1 + m/8) * 2^(e-7), e = 1..15
 * (e = 15 only with m <= 6, max 448).  Subnormal: m * 2^-9. */
double orc_e4m3_decode(uint8_t b)
{
    int s = b >> 7, e = (b >> 3) & 0xF, m = b & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* Round v to the nearest E4M3 value, ties to the even mantissa, saturating
 * finite overflow to +-448; the sign survives on zero. */
uint8_t orc_e4m3_encode(double v)
{
    uint8_t sign;
    double a, quantum, n, fl, rem, k, r, f;
    int ex, e_biased, m;

    if (isnan(v)) return 0x7F;
    sign = signbit(v) ? 0x80 : 0x00;
    a = fabs(v);
    /* Values above 448 would round to 448 (below the 464 midpoint) or past
     * the largest finite value; saturation maps both to 448. */
    if (a > 448.0) return (uint8_t)(sign | 0x7E);
    if (a < ldexp(1.0, -6)) {
        quantum = ldexp(1.0, -9);                  /* subnormal spacing */
    } else {
        frexp(a, &ex);                             /* a = f*2^ex, f in [0.5,1) */
        quantum = ldexp(1.0, (ex - 1) - 3);        /* 2^(floor(log2 a) - 3) */
    }
    n = a / quantum;                               /* exact: power-of-two divide */
    fl = floor(n);
    rem = n - fl;                                  /* exact */
    if (rem > 0.5) k = fl + 1.0;
    else if (rem < 0.5) k = fl;
    else k = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
    r = k * quantum;                               /* exact, r <= 448 */
    if (r == 0.0) return sign;
    if (r < ldexp(1.0, -6)) {
        m = (int)(r / ldexp(1.0, -9));
        return (uint8_t)(sign | m);
    }
    f = frexp(r, &ex);
    e_biased = (ex - 1) + 7;
    m = (int)((f * 2.0 - 1.0) * 8.0);
    return (uint8_t)(sign | (e_biased << 3) | m);
}

/* Shared block exponent s = floor(log2(amax)) - 8, clamped to [-127, 127];
 * floor(log2) is read off the binary exponent, not a log function.  amax = 0
 * gives -127.  Returns 128 for a non-finite amax (NaN scale). */
int orc_scale_exponent(double amax)
{
    int ex, s;
    if (isnan(amax) || isinf(amax)) return 128;
    if (amax == 0.0) return -127;
    frexp(amax, &ex);
    s = (ex - 1) - 8;
    if (s < -127) s = -127;
    if (s > 127) s = 127;
    return s;
}

uint8_t orc_scale_byte(int s) { return (uint8_t)(s + 127); }   /* 128 -> 0xFF */

/* Array forms of the scalar rules, for exhaustive checks. */
void orc_e4m3_encode_array(const double* v, int64_t n, uint8_t* out)
{
    int64_t i;
    for (i = 0; i < n; ++i) out[i] = orc_e4m3_encode(v[i]);
}

void orc_e4m3_decode_array(const uint8_t* b, int64_t n, double* out)
{
    int64_t i;
    for (i = 0; i < n; ++i) out[i] = orc_e4m3_decode(b[i]);
}

void orc_scale_exponent_array(const double* amax, int64_t n, int32_t* out)
{
    int64_t i;
    for (i = 0; i < n; ++i) out[i] = orc_scale_exponent(amax[i]);
}

double orc_scale_value(uint8_t byte)
{
    if (byte == 0xFF) return NAN;
    return ldexp(1.0, (int)byte - 127);
}

/* Quantise one block of n <= 32 bf16 values read at x[i*stride]. */
void orc_quantize_block(const uint16_t* x, int n, int64_t stride, uint8_t* codes,
                        int64_t code_stride, uint8_t* scale_byte)
{
    double amax = 0.0;
    int i, s;
    for (i = 0; i < n; ++i) {
        double a = fabs(orc_bf16_to_double(x[i * stride]));
        if (isnan(a)) { amax = NAN; break; }
        if (a > amax) amax = a;
    }
    s = orc_scale_exponent(amax);
    *scale_byte = orc_scale_byte(s);
    for (i = 0; i < n; ++i) {
        if (s == 128) codes[i * code_stride] = 0x7F;
        else codes[i * code_stride] = orc_e4m3_encode(ldexp(orc_bf16_to_double(x[i * stride]), -s));
    }
}

/* ------------------------------------------------------------------ */
/* Layout helpers                                                       */
/* ------------------------------------------------------------------ */

static int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
static int64_t rup(int64_t a, int64_t b) { return cdiv(a, b) * b; }

/* Byte offset of logical scale element (row, col) in the atom layout. */
int64_t orc_sf_offset(int64_t row, int64_t col, int64_t pitch)
{
    int64_t atom = (row / 128) * pitch + col / 4;
    return atom * 512 + (row % 32) * 16 + ((row % 128) / 32) * 4 + (col % 4);
}

int64_t orc_rowwise_pitch(int64_t C) { return cdiv(C, 128); }

int64_t orc_colwise_pitch(int64_t R, int32_t G)
{
    return R == 0 ? 0 : cdiv(R, 128) + G - 1;
}

int64_t orc_colwise_ld(int64_t R, int32_t G)
{
    int64_t ld = rup(rup(R, 32) + 32 * (int64_t)(G - 1), 128);
    return ld < 128 ? 128 : ld;
}

/* Default offsets: one group holding all rows. */
static void group_bounds(const int32_t* offs, int32_t G, int64_t R, int32_t g,
                         int64_t* lo, int64_t* hi)
{
    if (offs) { *lo = offs[g]; *hi = offs[g + 1]; }
    else { *lo = 0; *hi = R; }
}

/* Prefixes RB_g (128-row blocks before group g) and P_g (32-padded rows). */
static void group_prefixes(const int32_t* offs, int32_t G, int64_t R, int64_t* RB, int64_t* P)
{
    int32_t g;
    RB[0] = 0; P[0] = 0;
    for (g = 0; g < G; ++g) {
        int64_t lo, hi;
        group_bounds(offs, G, R, g, &lo, &hi);
        RB[g + 1] = RB[g] + cdiv(hi - lo, 128);
        P[g + 1] = P[g] + rup(hi - lo, 32);
    }
}

/* Returns 0 if offs[0] = 0, offs non-decreasing and offs[G] = R. */
int orc_check_offsets(const int32_t* offs, int32_t G, int64_t R)
{
    int32_t g;
    if (!offs) return 0;
    if (offs[0] != 0 || offs[G] != R) return 1;
    for (g = 0; g < G; ++g) if (offs[g + 1] < offs[g]) return 1;
    return 0;
}

/* ------------------------------------------------------------------ */
/* Whole-tensor quantisers in the library layout                        */
/* ------------------------------------------------------------------ */

/* x: bf16 [R, C] row-major, C % 32 == 0.  q: [R, C].  sf: scale atoms,
 * at least RB_G * pitch * 512 bytes; only that prefix is written. */
int orc_quantize_rowwise(const uint16_t* x, int64_t R, int64_t C, const int32_t* offs,
                         int32_t G, uint8_t* q, uint8_t* sf)
{
    int64_t pitch = orc_rowwise_pitch(C), nb = C / 32;
    int64_t *RB, *P;
    int32_t g;
    if (C % 32 != 0 || G < 1 || orc_check_offsets(offs, G, R)) return 1;
    RB = (int64_t*)malloc(sizeof(int64_t) * (G + 1));
    P = (int64_t*)malloc(sizeof(int64_t) * (G + 1));
    group_prefixes(offs, G, R, RB, P);
    memset(sf, 0, (size_t)(RB[G] * pitch * 512));
    for (g = 0; g < G; ++g) {
        int64_t lo, hi, r;
        group_bounds(offs, G, R, g, &lo, &hi);
        /* rows are independent: threads only split the loop */
#pragma omp parallel for schedule(static)
        for (r = lo; r < hi; ++r) {
            int64_t pr = 128 * RB[g] + (r - lo), j;
            for (j = 0; j < nb; ++j) {
                uint8_t sb;
                orc_quantize_block(x + r * C + 32 * j, 32, 1, q + r * C + 32 * j, 1, &sb);
                sf[orc_sf_offset(pr, j, pitch)] = sb;
            }
        }
    }
    free(RB); free(P);
    return 0;
}

/* x: bf16 [R, C].  qT: [C, ldT] with ldT = orc_colwise_ld(R, G); columns
 * P_G..ldT-1 are not written.  sfT: pitch = orc_colwise_pitch(R, G); atoms
 * (rb, cb) with cb < RB_G are written, for rb < ceil(C/128). */
int orc_quantize_colwise(const uint16_t* x, int64_t R, int64_t C, const int32_t* offs,
                         int32_t G, uint8_t* qT, uint8_t* sfT)
{
    int64_t ldT = orc_colwise_ld(R, G), pitch = orc_colwise_pitch(R, G);
    int64_t *RB, *P, c, rb, cb;
    int32_t g;
    if (C % 32 != 0 || G < 1 || orc_check_offsets(offs, G, R)) return 1;
    RB = (int64_t*)malloc(sizeof(int64_t) * (G + 1));
    P = (int64_t*)malloc(sizeof(int64_t) * (G + 1));
    group_prefixes(offs, G, R, RB, P);
    for (rb = 0; rb < cdiv(C, 128); ++rb)
        for (cb = 0; cb < RB[G]; ++cb)
            memset(sfT + (rb * pitch + cb) * 512, 0, 512);
    for (g = 0; g < G; ++g) {
        int64_t lo, hi, m;
        group_bounds(offs, G, R, g, &lo, &hi);
        m = hi - lo;
        /* columns are independent: threads only split the loop */
#pragma omp parallel for schedule(static)
        for (c = 0; c < C; ++c) {
            int64_t t0;
            for (t0 = 0; t0 < m; t0 += 32) {
                int n = (int)(m - t0 < 32 ? m - t0 : 32);
                uint8_t sb;
                orc_quantize_block(x + (lo + t0) * C + c, n, C, qT + c * ldT + P[g] + t0, 1, &sb);
                sfT[orc_sf_offset(c, 4 * RB[g] + t0 / 32, pitch)] = sb;
            }
            for (t0 = m; t0 < rup(m, 32); ++t0) qT[c * ldT + P[g] + t0] = 0;
        }
    }
    free(RB); free(P);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Dequantisation from the library layout                               */
/* ------------------------------------------------------------------ */

/* out: fp64 [R, C] = code * 2^s for every element. */
int orc_dequantize_rowwise(const uint8_t* q, const uint8_t* sf, int64_t R, int64_t C,
                           const int32_t* offs, int32_t G, double* out)
{
    int64_t pitch = orc_rowwise_pitch(C);
    int64_t *RB, *P;
    int32_t g;
    if (C % 32 != 0 || G < 1 || orc_check_offsets(offs, G, R)) return 1;
    RB = (int64_t*)malloc(sizeof(int64_t) * (G + 1));
    P = (int64_t*)malloc(sizeof(int64_t) * (G + 1));
    group_prefixes(offs, G, R, RB, P);
    for (g = 0; g < G; ++g) {
        int64_t lo, hi, r;
        group_bounds(offs, G, R, g, &lo, &hi);
#pragma omp parallel for schedule(static)
        for (r = lo; r < hi; ++r) {
            int64_t pr = 128 * RB[g] + (r - lo), c;
            for (c = 0; c < C; ++c)
                out[r * C + c] = orc_e4m3_decode(q[r * C + c]) *
                                 orc_scale_value(sf[orc_sf_offset(pr, c / 32, pitch)]);
        }
    }
    free(RB); free(P);
    return 0;
}

/* out: fp64 [R, C] (un-transposed) from the colwise layout. */
int orc_dequantize_colwise(const uint8_t* qT, const uint8_t* sfT, int64_t R, int64_t C,
                           const int32_t* offs, int32_t G, double* out)
{
    int64_t ldT = orc_colwise_ld(R, G), pitch = orc_colwise_pitch(R, G);
    int64_t *RB, *P;
    int32_t g;
    if (C % 32 != 0 || G < 1 || orc_check_offsets(offs, G, R)) return 1;
    RB = (int64_t*)malloc(sizeof(int64_t) * (G + 1));
    P = (int64_t*)malloc(sizeof(int64_t) * (G + 1));
    group_prefixes(offs, G, R, RB, P);
    for (g = 0; g < G; ++g) {
        int64_t lo, hi, t;
        group_bounds(offs, G, R, g, &lo, &hi);
#pragma omp parallel for schedule(static)
        for (t = 0; t < hi - lo; ++t) {
            int64_t c;
            for (c = 0; c < C; ++c)
                out[(lo + t) * C + c] = orc_e4m3_decode(qT[c * ldT + P[g] + t]) *
                                        orc_scale_value(sfT[orc_sf_offset(c, 4 * RB[g] + t / 32, pitch)]);
        }
    }
    free(RB); free(P);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Grouped GEMMs: the plain definition in fp64 on dense operands        */
/* ------------------------------------------------------------------ */

/* Y[i, n] = sum_k X[i, k] * W[e, n, k] for rows i of expert e. */
int orc_gemm_fwd(const double* X, const double* W, const int32_t* offs, int32_t E,
                 int64_t M, int64_t N, int64_t K, double* Y)
{
    int32_t e;
    if (orc_check_offsets(offs, E, M)) return 1;
    for (e = 0; e < E; ++e) {
        int64_t i, n, k;
        for (i = offs[e]; i < offs[e + 1]; ++i)
            for (n = 0; n < N; ++n) {
                double acc = 0.0;
                for (k = 0; k < K; ++k) acc += X[i * K + k] * W[((int64_t)e * N + n) * K + k];
                Y[i * N + n] = acc;
            }
    }
    return 0;
}

/* dX[i, k] = sum_n dY[i, n] * W[e, n, k] for rows i of expert e. */
int orc_gemm_dgrad(const double* dY, const double* W, const int32_t* offs, int32_t E,
                   int64_t M, int64_t N, int64_t K, double* dX)
{
    int32_t e;
    if (orc_check_offsets(offs, E, M)) return 1;
    for (e = 0; e < E; ++e) {
        int64_t i, n, k;
        for (i = offs[e]; i < offs[e + 1]; ++i)
            for (k = 0; k < K; ++k) {
                double acc = 0.0;
                for (n = 0; n < N; ++n) acc += dY[i * N + n] * W[((int64_t)e * N + n) * K + k];
                dX[i * K + k] = acc;
            }
    }
    return 0;
}

/* dW[e, n, k] = sum over rows i of expert e of dY[i, n] * X[i, k]; zero
 * for an expert with no rows. */
int orc_gemm_wgrad(const double* dY, const double* X, const int32_t* offs, int32_t E,
                   int64_t M, int64_t N, int64_t K, double* dW)
{
    int32_t e;
    if (orc_check_offsets(offs, E, M)) return 1;
    for (e = 0; e < E; ++e) {
        int64_t i, n, k;
        for (n = 0; n < N; ++n)
            for (k = 0; k < K; ++k) {
                double acc = 0.0;
                for (i = offs[e]; i < offs[e + 1]; ++i) acc += dY[i * N + n] * X[i * K + k];
                dW[((int64_t)e * N + n) * K + k] = acc;
            }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Sampled outputs straight from quantised operands (full-size checks)  */
/* ------------------------------------------------------------------ */

/* The group g with offs[g] <= r < offs[g+1]: the last g with offs[g] <= r
 * (empty groups before it share its offset and are skipped). */
static int32_t group_of_row(const int32_t* offs, int32_t G, int64_t r)
{
    int32_t lo = 0, hi = G - 1;
    while (lo < hi) {
        int32_t mid = (lo + hi + 1) / 2;
        if (offs[mid] <= r) lo = mid; else hi = mid - 1;
    }
    return lo;
}

typedef struct {
    const uint8_t* q; const uint8_t* sf; int64_t R, C; const int32_t* offs; int32_t G;
    int64_t pitch, ldT; int64_t *RB, *P; int colwise;
} orc_operand;

static void operand_init(orc_operand* o, const uint8_t* q, const uint8_t* sf, int64_t R,
                         int64_t C, const int32_t* offs, int32_t G, int colwise)
{
    o->q = q; o->sf = sf; o->R = R; o->C = C; o->offs = offs; o->G = G; o->colwise = colwise;
    o->pitch = colwise ? orc_colwise_pitch(R, G) : orc_rowwise_pitch(C);
    o->ldT = orc_colwise_ld(R, G);
    o->RB = (int64_t*)malloc(sizeof(int64_t) * (G + 1));
    o->P = (int64_t*)malloc(sizeof(int64_t) * (G + 1));
    group_prefixes(offs, G, R, o->RB, o->P);
}

static void operand_free(orc_operand* o) { free(o->RB); free(o->P); }

/* Dequantised logical element (r, c) of an operand of logical shape [R, C]. */
static double operand_at(const orc_operand* o, int64_t r, int64_t c)
{
    int32_t g = o->offs ? group_of_row(o->offs, o->G, r) : 0;
    int64_t lo = o->offs ? o->offs[g] : 0, t = r - lo;
    if (!o->colwise)
        return orc_e4m3_decode(o->q[r * o->C + c]) *
               orc_scale_value(o->sf[orc_sf_offset(128 * o->RB[g] + t, c / 32, o->pitch)]);
    return orc_e4m3_decode(o->q[c * o->ldT + o->P[g] + t]) *
           orc_scale_value(o->sf[orc_sf_offset(c, 4 * o->RB[g] + t / 32, o->pitch)]);
}

/* fwd sample: Y[rows[s], cols[s]]; X rowwise [M, K] grouped by offs, W
 * rowwise [E*N, K] quantised as one group. */
int orc_sample_fwd(const uint8_t* xq, const uint8_t* xs, const uint8_t* wq, const uint8_t* ws,
                   const int32_t* offs, int32_t E, int64_t M, int64_t N, int64_t K,
                   int64_t ns, const int64_t* rows, const int64_t* cols, double* out)
{
    orc_operand X, W;
    int64_t s;
    if (orc_check_offsets(offs, E, M)) return 1;
    operand_init(&X, xq, xs, M, K, offs, E, 0);
    operand_init(&W, wq, ws, (int64_t)E * N, K, NULL, 1, 0);
    for (s = 0; s < ns; ++s) {
        int64_t i = rows[s], n = cols[s], k;
        int32_t e = group_of_row(offs, E, i);
        double acc = 0.0;
        for (k = 0; k < K; ++k) acc += operand_at(&X, i, k) * operand_at(&W, (int64_t)e * N + n, k);
        out[s] = acc;
    }
    operand_free(&X); operand_free(&W);
    return 0;
}

/* dgrad sample: dX[rows[s], cols[s]]; dY rowwise [M, N] grouped by offs,
 * W colwise (logical [E*N, K], one group). */
int orc_sample_dgrad(const uint8_t* dyq, const uint8_t* dys, const uint8_t* wqT,
                     const uint8_t* wsT, const int32_t* offs, int32_t E, int64_t M, int64_t N,
                     int64_t K, int64_t ns, const int64_t* rows, const int64_t* cols, double* out)
{
    orc_operand D, W;
    int64_t s;
    if (orc_check_offsets(offs, E, M)) return 1;
    operand_init(&D, dyq, dys, M, N, offs, E, 0);
    operand_init(&W, wqT, wsT, (int64_t)E * N, K, NULL, 1, 1);
    for (s = 0; s < ns; ++s) {
        int64_t i = rows[s], k = cols[s], n;
        int32_t e = group_of_row(offs, E, i);
        double acc = 0.0;
        for (n = 0; n < N; ++n) acc += operand_at(&D, i, n) * operand_at(&W, (int64_t)e * N + n, k);
        out[s] = acc;
    }
    operand_free(&D); operand_free(&W);
    return 0;
}

/* wgrad sample: dW[experts[s], rows[s], cols[s]]; dY and X colwise, both
 * grouped by offs. */
int orc_sample_wgrad(const uint8_t* dyqT, const uint8_t* dysT, const uint8_t* xqT,
                     const uint8_t* xsT, const int32_t* offs, int32_t E, int64_t M, int64_t N,
                     int64_t K, int64_t ns, const int32_t* experts, const int64_t* rows,
                     const int64_t* cols, double* out)
{
    orc_operand D, X;
    int64_t s;
    if (orc_check_offsets(offs, E, M)) return 1;
    operand_init(&D, dyqT, dysT, M, N, offs, E, 1);
    operand_init(&X, xqT, xsT, M, K, offs, E, 1);
    for (s = 0; s < ns; ++s) {
        int32_t e = experts[s];
        int64_t n = rows[s], k = cols[s], i;
        double acc = 0.0;
        for (i = offs[e]; i < offs[e + 1]; ++i) acc += operand_at(&D, i, n) * operand_at(&X, i, k);
        out[s] = acc;
    }
    operand_free(&D); operand_free(&X);
    return 0;
}

/* ------------------------------------------------------------------ */
/* CPU baseline: bf16 inputs, fp32 accumulation, rows split over threads */
/* ------------------------------------------------------------------ */

int orc_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* The timed fp32 baselines (orc_baseline_fwd/dgrad/wgrad_f32) live in
 * baseline_f32.c, built with optimisation flags of their own. */

/* Whole-tensor quantiser timing helper for the CPU baseline: rowwise over
 * rows [row_lo, row_hi) of a single-group tensor (codes and logical scales). */
int orc_baseline_quantize_rows(const uint16_t* x, int64_t C, int64_t row_lo, int64_t row_hi,
                               uint8_t* q, uint8_t* s_logical)
{
    int64_t r;
#pragma omp parallel for schedule(static)
    for (r = row_lo; r < row_hi; ++r) {
        int64_t j;
        for (j = 0; j < C / 32; ++j)
            orc_quantize_block(x + r * C + 32 * j, 32, 1, q + r * C + 32 * j, 1, s_logical + r * (C / 32) + j);
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* MoE token dispatch plan and combine (permute / unpermute)            */
/* ------------------------------------------------------------------ */
/* The grouped GEMM consumes each expert's tokens as one contiguous run of
 * rows, every token with its real count (iitak.ru, "NVIDIA ... JAX",
 * paragraph on the Transformer Engine grouped GEMM; the all-to-all that
 * sends tokens to experts and the one that brings results back are on
 * opensourcebeat.com, section "Двухсторонняя атака: MXFP8 и DeepEP").
 * Routing gives token t its k experts idx[t*k + j], j = 0..k-1.  The plan
 * lists the (token, slot) pairs grouped by expert, in ascending (token,
 * slot) order inside an expert:
 *   offs[e]      exclusive prefix of the per-expert pair counts, offs[E] = T*k;
 *   perm[r]      token of permuted row r;
 *   inv[t*k+j]   permuted row of pair (t, j).
 * Returns -1 if an expert id is out of range. */
int orc_moe_plan(const int32_t* idx, int64_t T, int32_t k, int32_t E, int32_t* offs, int32_t* perm,
                 int32_t* inv)
{
    int64_t* fill = (int64_t*)calloc((size_t)E + 1, sizeof(int64_t));
    int64_t i, t;
    int32_t e, j;
    for (i = 0; i < T * k; ++i) {
        if (idx[i] < 0 || idx[i] >= E) { free(fill); return -1; }
        fill[idx[i]] += 1;
    }
    offs[0] = 0;
    for (e = 0; e < E; ++e) offs[e + 1] = offs[e] + (int32_t)fill[e];
    for (e = 0; e < E; ++e) fill[e] = 0;
    for (t = 0; t < T; ++t) {
        for (j = 0; j < k; ++j) {
            int32_t ee = idx[t * k + j];
            int64_t r = offs[ee] + fill[ee]++;
            perm[r] = (int32_t)t;
            inv[t * k + j] = (int32_t)r;
        }
    }
    free(fill);
    return 0;
}

/* Nearest-even bf16 bits of a double (8 significant bits, exponent range of
 * fp32: normals from 2^-126, subnormals in steps of 2^-133, overflow to Inf
 * at and above 2^128 - 2^119, the midpoint past the largest finite value). */
uint16_t orc_bf16_from_double(double v)
{
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    double a = fabs(v), q, m, fl, rem;
    int e;
    if (isnan(v)) return (uint16_t)(sign | 0x7FC0u);
    if (a >= ldexp(1.0, 128) - ldexp(1.0, 119)) return (uint16_t)(sign | 0x7F80u);
    if (a == 0.0) return sign;
    frexp(a, &e);                       /* a = f * 2^e, f in [0.5, 1) */
    e = e - 1;                          /* a in [2^e, 2^(e+1)) */
    if (e < -126) e = -126;             /* subnormal range: fixed quantum */
    q = ldexp(1.0, e - 7);              /* spacing of bf16 values there */
    m = a / q;                          /* exact: q is a power of two */
    fl = floor(m);
    rem = m - fl;
    if (rem > 0.5 || (rem == 0.5 && fmod(fl, 2.0) != 0.0)) fl += 1.0;
    a = fl * q;                         /* the rounded magnitude, exact */
    {
        /* encode: normal if a >= 2^-126, else subnormal */
        uint32_t bits;
        float f = (float)a;             /* exact: a has at most 8 significant bits */
        memcpy(&bits, &f, 4);
        return (uint16_t)(sign | (uint16_t)(bits >> 16));
    }
}

/* Combine: y[t, c] = sum over j of w[t*k+j] * yp[inv[t*k+j], c], summed in
 * fp64 and rounded once to bf16.  yp: bf16 [rows, C]; y: bf16 [T, C]. */
int orc_moe_combine(const uint16_t* yp, int64_t rows, int64_t C, const int32_t* inv, const float* w,
                    int64_t T, int32_t k, uint16_t* y)
{
    int64_t t;
    for (t = 0; t < T * k; ++t)
        if (inv[t] < 0 || inv[t] >= rows) return -1;
    for (t = 0; t < T; ++t) {
        int64_t c;
        for (c = 0; c < C; ++c) {
            double acc = 0.0;
            int32_t j;
            for (j = 0; j < k; ++j)
                acc += (double)w[t * k + j] * orc_bf16_to_double(yp[(int64_t)inv[t * k + j] * C + c]);
            y[t * C + c] = orc_bf16_from_double(acc);
        }
    }
    return 0;
}

void orc_bf16_from_double_array(const double* v, int64_t n, uint16_t* out)
{
    int64_t i;
    for (i = 0; i < n; ++i) out[i] = orc_bf16_from_double(v[i]);
}

/* ------------------------------------------------------------------ */
/* SwiGLU between the two grouped linears of an expert                  */
/* ------------------------------------------------------------------ */
/* The MXFP8 speed-up comes from the expert pipeline as a whole
 * (opensourcebeat.com, section "Двухсторонняя атака: MXFP8 и DeepEP"); the
 * DeepSeek-V3 and Llama 4 experts the workloads model apply SwiGLU between
 * their gate/up and down projections.  The pages give no formula, so the
 * plainest reading: the gate/up output Y [M, 2I] holds the gate in columns
 * 0 .. I-1 and the up projection in columns I .. 2I-1, and
 *   h[i, j] = silu(g) * u = g * u / (1 + exp(-g)),  g = Y[i, j], u = Y[i, I + j],
 * evaluated in fp64 and rounded once to bf16 (nearest even). */
double orc_silu(double g) { return g / (1.0 + exp(-g)); }

int orc_swiglu(const double* Y, int64_t M, int64_t I, uint16_t* h)
{
    int64_t i;
    if (M < 0 || I <= 0) return 1;
#pragma omp parallel for schedule(static)
    for (i = 0; i < M; ++i) {
        int64_t j;
        for (j = 0; j < I; ++j) {
            double g = Y[i * 2 * I + j], u = Y[i * 2 * I + I + j];
            h[i * I + j] = orc_bf16_from_double(orc_silu(g) * u);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Expert-parallel dispatch: the plan, and MXFP8 rows sent once per rank */
/* ------------------------------------------------------------------ */
/* Each MoE layer sends every token to the GPUs holding its experts and
 * brings the results back (opensourcebeat.com, section "Двухсторонняя
 * атака: MXFP8 и DeepEP"); a token needed by several experts of one
 * destination crosses the network once and is copied there (iitak.ru,
 * "NVIDIA ... JAX", paragraph on NCCL EP).  Readings where the pages are
 * silent: P ranks own E/P consecutive experts each (rank p owns experts
 * p*E/P .. (p+1)*E/P - 1); a token travels as one record per destination
 * rank, carrying the token's row as rowwise MXFP8 (its codes, then its
 * 32-block scale bytes); each (token, slot) pair routed to that rank travels
 * as a pair entry (local expert id, record index).  Send order: destination
 * rank, then token, then slot, all ascending. */

/* idx: int32 [T, k] global expert ids.  Outputs, in send order:
 *   counts[p]         records sent to rank p;  counts[P + p]  pairs sent to p
 *   rec_token[i]      token of record i (records of rank p after those of
 *                     ranks < p)
 *   pair_expert[s]    local expert id (e mod E/P) of pair s
 *   pair_rec[s]       record of pair s, counted from the first record sent
 *                     to the same rank
 *   ret_pos[t*k + j]  pair index s of slot (t, j) -- the row at which its
 *                     expert output comes back -- or -1 when the id is
 *                     outside [0, E) (such a slot is not sent).
 * Returns the number of slots with an id outside [0, E), or -1 when P < 1
 * or E is not a positive multiple of P. */
int64_t orc_ep_plan(const int32_t* idx, int64_t T, int32_t k, int32_t E, int32_t P, int32_t* counts,
                    int32_t* rec_token, int32_t* pair_expert, int32_t* pair_rec, int32_t* ret_pos)
{
    int64_t t, rec = 0, pair = 0, bad = 0;
    int32_t p, j, epr;
    if (P < 1 || E < 1 || E % P != 0 || k < 1) return -1;
    epr = E / P;
    for (t = 0; t < T * k; ++t) {
        ret_pos[t] = -1;
        if (idx[t] < 0 || idx[t] >= E) bad += 1;
    }
    for (p = 0; p < P; ++p) {
        int64_t rec0 = rec, pair0 = pair;
        for (t = 0; t < T; ++t) {
            int64_t mine = -1;   /* this token's record for rank p, once made */
            for (j = 0; j < k; ++j) {
                int32_t e = idx[t * k + j];
                if (e < 0 || e >= E || e / epr != p) continue;
                if (mine < 0) {
                    mine = rec - rec0;
                    rec_token[rec++] = (int32_t)t;
                }
                pair_expert[pair] = e % epr;
                pair_rec[pair] = (int32_t)mine;
                ret_pos[t * k + j] = (int32_t)pair;
                pair += 1;
            }
        }
        counts[p] = (int32_t)(rec - rec0);
        counts[P + p] = (int32_t)(pair - pair0);
    }
    return bad;
}

/* Bytes of one record holding a row of C elements: C codes, C/32 scale
 * bytes, zero padding to a multiple of 16. */
int64_t orc_ep_record_bytes(int64_t C) { return rup(C + C / 32, 16); }

/* x: bf16 [T, C], C % 32 == 0.  Record i holds the MXFP8 rowwise encoding
 * of row rec_token[i]: byte 32b + n is the code of element 32b + n, byte
 * C + b the scale byte of block b, the rest zero.  A token index outside
 * [0, T) gives an all-zero record. */
int orc_ep_pack(const uint16_t* x, int64_t T, int64_t C, const int32_t* rec_token, int64_t R, uint8_t* rec)
{
    int64_t stride = orc_ep_record_bytes(C), i;
    if (C % 32 != 0 || C <= 0) return 1;
#pragma omp parallel for schedule(static)
    for (i = 0; i < R; ++i) {
        uint8_t* r = rec + i * stride;
        int64_t t = rec_token[i], b;
        memset(r, 0, (size_t)stride);
        if (t < 0 || t >= T) continue;
        for (b = 0; b < C / 32; ++b) orc_quantize_block(x + t * C + 32 * b, 32, 1, r + 32 * b, 1, r + C + b);
    }
    return 0;
}

/* Receiving side: R records and M pairs arrived from P source ranks, each
 * source's records and pairs after those of lower ranks.  src_base[q] is
 * the first pair and src_base[P + 1 + q] the first record from source q
 * (src_base[P], src_base[2P + 1] the totals).  Grouped row r (rows grouped
 * by local expert with offs, G groups) is pair perm[r]; its record is
 * src_base[P + 1 + q] + pair_rec[perm[r]] for the source q whose pairs hold
 * perm[r].  Writes the rowwise MXFP8 layout of the grouped rows: codes
 * q [M, C] and scale atoms (pitch ceil(C/128), the first RB_G * pitch * 512
 * bytes).  Returns 1 on bad sizes, offsets or an index out of range. */
int orc_ep_unpack(const uint8_t* rec, int64_t R, int64_t C, const int32_t* pair_rec, const int32_t* src_base,
                  int32_t P, const int32_t* perm, int64_t M, const int32_t* offs, int32_t G, uint8_t* q,
                  uint8_t* sf)
{
    int64_t stride = orc_ep_record_bytes(C), pitch = orc_rowwise_pitch(C), nb = C / 32;
    int64_t *RB, *Pp;
    int32_t g;
    int bad = 0;
    if (C % 32 != 0 || C <= 0 || G < 1 || P < 1 || orc_check_offsets(offs, G, M)) return 1;
    if (src_base[P] != M || src_base[2 * P + 1] != R) return 1;
    RB = (int64_t*)malloc(sizeof(int64_t) * (G + 1));
    Pp = (int64_t*)malloc(sizeof(int64_t) * (G + 1));
    group_prefixes(offs, G, M, RB, Pp);
    memset(sf, 0, (size_t)(RB[G] * pitch * 512));
    for (g = 0; g < G; ++g) {
        int64_t lo, hi, r;
        group_bounds(offs, G, M, g, &lo, &hi);
        for (r = lo; r < hi; ++r) {
            int64_t s = perm[r], i, j, src = 0;
            if (s < 0 || s >= M) { bad = 1; continue; }
            while (src + 1 < P && src_base[src + 1] <= s) src += 1;
            i = (int64_t)src_base[P + 1 + src] + pair_rec[s];
            if (i < 0 || i >= R) { bad = 1; continue; }
            memcpy(q + r * C, rec + i * stride, (size_t)C);
            for (j = 0; j < nb; ++j) sf[orc_sf_offset(128 * RB[g] + (r - lo), j, pitch)] = rec[i * stride + C + j];
        }
    }
    free(RB); free(Pp);
    return bad;
}

/* ------------------------------------------------------------------ */
/* NVFP4: 4-bit E2M1 elements, 16-element blocks with E4M3 scales and   */
/* one fp32 scale per tensor                                             */
/* ------------------------------------------------------------------ */
/* The pages name NVFP4 only as the format NVIDIA's MoE training adds next
 * (iitak.ru, "NVIDIA в 10 раз ускорила обучение моделей-«смесей экспертов»
 * на JAX", closing paragraph).  Its rules here are NVIDIA's public NVFP4
 * definition, read plainly:
 *   - E2M1 element: sign, 2 exponent bits (bias 1), 1 mantissa bit; values
 *     0, 0.5, 1, 1.5, 2, 3, 4, 6; round to nearest even, saturate at 6.
 *   - tensor scale S = (448 * 6) / amax(tensor) in fp32 (1 when amax = 0);
 *   - a block of 16 shares the E4M3 scale sf = E4M3(amax_b * S / 6), and an
 *     element is E2M1((x * S) / sf); the fp32 operations are rounded to
 *     nearest in exactly this order (the decision that picks each code is
 *     taken in fp32, as the GPU takes it); sf = 0 gives zero codes.
 *   - value = code * sf / S. */
double orc_e2m1_decode(uint8_t nib)
{
    int s = (nib >> 3) & 1, e = (nib >> 1) & 3, m = nib & 1;
    double v = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -v : v;
}

uint8_t orc_e2m1_encode(double v)
{
    uint8_t sign = signbit(v) ? 8 : 0;
    double a = fabs(v), q, n, fl, rem, k, r;
    int ex;
    if (a >= 6.0) return (uint8_t)(sign | 7);          /* saturate (and 6 itself) */
    if (a < 1.0) q = 0.5;                              /* subnormal spacing, and [0.5, 1) */
    else { frexp(a, &ex); q = ldexp(1.0, (ex - 1) - 1); }   /* 2^(floor(log2 a) - 1) */
    n = a / q;
    fl = floor(n);
    rem = n - fl;
    if (rem > 0.5) k = fl + 1.0;
    else if (rem < 0.5) k = fl;
    else k = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
    r = k * q;
    if (r >= 6.0) return (uint8_t)(sign | 7);
    if (r == 0.0) return sign;
    if (r < 1.0) return (uint8_t)(sign | 1);           /* 0.5 */
    frexp(r, &ex);
    {
        int e = ex;                                    /* r in [2^(ex-1), 2^ex): biased exponent ex */
        int m = (r / ldexp(1.0, ex - 1) > 1.0) ? 1 : 0;
        return (uint8_t)(sign | (e << 1) | m);
    }
}

float orc_nvfp4_tensor_scale(float amax)
{
    return amax == 0.0f ? 1.0f : 2688.0f / amax;
}

/* One block of n <= 16 bf16 elements (stride apart): the E4M3 scale byte and
 * one E2M1 nibble per element (low 4 bits of codes[i * code_stride]). */
void orc_nvfp4_quantize_block(const uint16_t* x, int n, int64_t stride, float S, uint8_t* codes,
                              int64_t code_stride, uint8_t* scale_byte)
{
    float amax = 0.0f, t, u, r;
    int i;
    uint8_t sf;
    for (i = 0; i < n; ++i) {
        float a = fabsf((float)orc_bf16_to_double(x[i * stride]));
        if (a > amax) amax = a;
    }
    t = amax * S;
    u = t / 6.0f;
    sf = orc_e4m3_encode((double)u);
    r = (float)orc_e4m3_decode(sf);
    *scale_byte = sf;
    for (i = 0; i < n; ++i) {
        if (r == 0.0f) {
            codes[i * code_stride] = 0;
        } else {
            float w = ((float)orc_bf16_to_double(x[i * stride]) * S) / r;
            codes[i * code_stride] = orc_e2m1_encode((double)w);
        }
    }
}

static int64_t nv_pitch_row(int64_t C) { return cdiv(C, 64); }

int64_t orc_nvfp4_colwise_pitch(int64_t R, int32_t G) { return R == 0 ? 0 : cdiv(R, 64) + G - 1; }

int64_t orc_nvfp4_colwise_ld(int64_t R, int32_t G)
{
    int64_t ld = rup(rup(R, 32) + 32 * (int64_t)(G - 1), 256);
    return ld < 256 ? 256 : ld;                         /* elements; bytes = ld / 2 */
}

/* Rowwise NVFP4 of x [R, C] (C % 64 == 0) with groups offs: packed codes
 * q [R, C/2] (element c in the low nibble of byte c/2 when c is even),
 * scales in 512-byte atoms of 128 rows x 4 blocks, rows of group g padded to
 * a multiple of 128 as for MXFP8, pitch ceil(C/64). */
int orc_nvfp4_quantize_rowwise(const uint16_t* x, int64_t R, int64_t C, const int32_t* offs, int32_t G,
                               float S, uint8_t* q, uint8_t* sf)
{
    int64_t* RB = (int64_t*)calloc((size_t)G + 1, sizeof(int64_t));
    int64_t* P = (int64_t*)calloc((size_t)G + 1, sizeof(int64_t));
    int64_t pitch = nv_pitch_row(C);
    int32_t g;
    if (orc_check_offsets(offs, G, R) != 0 || C % 64 != 0) { free(RB); free(P); return -1; }
    group_prefixes(offs, G, R, RB, P);
    for (g = 0; g < G; ++g) {
        int64_t lo, hi, r;
        group_bounds(offs, G, R, g, &lo, &hi);
        for (r = lo; r < hi; ++r) {
            int64_t pr = 128 * RB[g] + (r - lo), j;
            for (j = 0; j < C / 16; ++j) {
                uint8_t nib[16], sb;
                int i;
                orc_nvfp4_quantize_block(x + r * C + 16 * j, 16, 1, S, nib, 1, &sb);
                for (i = 0; i < 16; i += 2)
                    q[r * (C / 2) + 8 * j + i / 2] = (uint8_t)(nib[i] | (nib[i + 1] << 4));
                sf[orc_sf_offset(pr, j, pitch)] = sb;
            }
        }
    }
    free(RB); free(P);
    return 0;
}

/* Colwise NVFP4: blocks of 16 rows restarting at every group offset (a
 * group's last block may be short), codes transposed and packed along rows:
 * qT [C, ld/2] bytes, element (offs[g] + t, c) at nibble P_g + t of row c
 * (P_g = sum over h < g of round_up(m_h, 32); pad nibbles 0).  Scales
 * S^T[c, 4*RB64_g + t/16], RB64_g = sum over h < g of ceil(m_h/64), pitch
 * orc_nvfp4_colwise_pitch(R, G). */
int orc_nvfp4_quantize_colwise(const uint16_t* x, int64_t R, int64_t C, const int32_t* offs, int32_t G,
                               float S, uint8_t* qT, uint8_t* sfT)
{
    int64_t ld = orc_nvfp4_colwise_ld(R, G), pitch = orc_nvfp4_colwise_pitch(R, G);
    int64_t p0 = 0, rb64 = 0;
    int32_t g;
    if (orc_check_offsets(offs, G, R) != 0 || C % 64 != 0) return -1;
    for (g = 0; g < G; ++g) {
        int64_t lo, hi, m, c;
        group_bounds(offs, G, R, g, &lo, &hi);
        m = hi - lo;
        for (c = 0; c < C; ++c) {
            int64_t b;
            for (b = 0; b < cdiv(m, 16); ++b) {
                int64_t n = m - 16 * b < 16 ? m - 16 * b : 16, i;
                uint8_t nib[16], sb;
                orc_nvfp4_quantize_block(x + (lo + 16 * b) * C + c, (int)n, C, S, nib, 1, &sb);
                for (i = 0; i < n; ++i) {
                    int64_t col = p0 + 16 * b + i;
                    uint8_t* dst = qT + c * (ld / 2) + col / 2;
                    *dst = (uint8_t)((col & 1) ? ((*dst & 0x0F) | (nib[i] << 4)) : ((*dst & 0xF0) | nib[i]));
                }
                sfT[orc_sf_offset(c, 4 * rb64 + b, pitch)] = sb;
            }
        }
        p0 += rup(m, 32);
        rb64 += cdiv(m, 64);
    }
    return 0;
}

/* Dequantisation back to fp64 (value = code * sf / S), same layouts. */
int orc_nvfp4_dequantize_rowwise(const uint8_t* q, const uint8_t* sf, int64_t R, int64_t C, const int32_t* offs,
                                 int32_t G, float S, double* out)
{
    int64_t* RB = (int64_t*)calloc((size_t)G + 1, sizeof(int64_t));
    int64_t* P = (int64_t*)calloc((size_t)G + 1, sizeof(int64_t));
    int64_t pitch = nv_pitch_row(C);
    int32_t g;
    if (orc_check_offsets(offs, G, R) != 0) { free(RB); free(P); return -1; }
    group_prefixes(offs, G, R, RB, P);
    for (g = 0; g < G; ++g) {
        int64_t r, lo, hi;
        group_bounds(offs, G, R, g, &lo, &hi);
        for (r = lo; r < hi; ++r) {
            int64_t pr = 128 * RB[g] + (r - lo), c;
            for (c = 0; c < C; ++c) {
                uint8_t byte = q[r * (C / 2) + c / 2];
                uint8_t nib = (c & 1) ? (byte >> 4) : (byte & 0xF);
                double s = orc_e4m3_decode(sf[orc_sf_offset(pr, c / 16, pitch)]);
                out[r * C + c] = orc_e2m1_decode(nib) * s / (double)S;
            }
        }
    }
    free(RB); free(P);
    return 0;
}

int orc_nvfp4_dequantize_colwise(const uint8_t* qT, const uint8_t* sfT, int64_t R, int64_t C,
                                 const int32_t* offs, int32_t G, float S, double* out)
{
    int64_t ld = orc_nvfp4_colwise_ld(R, G), pitch = orc_nvfp4_colwise_pitch(R, G);
    int64_t p0 = 0, rb64 = 0;
    int32_t g;
    if (orc_check_offsets(offs, G, R) != 0) return -1;
    for (g = 0; g < G; ++g) {
        int64_t lo, hi, m, t, c;
        group_bounds(offs, G, R, g, &lo, &hi);
        m = hi - lo;
        for (t = 0; t < m; ++t)
            for (c = 0; c < C; ++c) {
                int64_t col = p0 + t;
                uint8_t byte = qT[c * (ld / 2) + col / 2];
                uint8_t nib = (col & 1) ? (byte >> 4) : (byte & 0xF);
                double s = orc_e4m3_decode(sfT[orc_sf_offset(c, 4 * rb64 + t / 16, pitch)]);
                out[(lo + t) * C + c] = orc_e2m1_decode(nib) * s / (double)S;
            }
        p0 += rup(m, 32);
        rb64 += cdiv(m, 64);
    }
    return 0;
}

void orc_e2m1_encode_array(const double* v, int64_t n, uint8_t* out)
{
    int64_t i;
    for (i = 0; i < n; ++i) out[i] = orc_e2m1_encode(v[i]);
}
