/*
 * gptq_oracle.c -- plain, slow, float64 CPU reference for GPTQ layer-wise
 * weight quantization (asymmetric group-wise INT-b, fp16 scale, b-bit zero).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes or
 * calls this file; only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark may load it.  It shares no code, header, table or
 * helper with the CUDA path.
 *
 * Sources (the pages this follows; see each function):
 *   [P1] "模型量化技术(下)：权重量化与激活量化、KL散度校准、GPTQ/AWQ量化方法",
 *        section "GPTQ：基于二阶信息的后训练量化" (Hessian from layer inputs,
 *        quantize column by column, compensate the remaining columns).
 *   [P3] "INT4/INT8 量化推理：从 GPTQ 到 AWQ 的取舍", section 一 (group of 128
 *        consecutive weights sharing an fp16 scale and a 4-bit zero point,
 *        66.5 bytes per 128 weights) and section 三 (objective: match the
 *        layer output; H from the calibration inputs; per-column error pushed
 *        onto the not-yet-quantized columns through H^-1).
 *   [P4] "大模型量化的“校准”艺术", section 2.1 (min-max: map [min,max]
 *        linearly onto the integer range) and section 2.2 (the column loop).
 *   [P5] "GPTQ / AWQ / SqueezeLLM", section 一 (H = 2 X^T X / n, damping,
 *        processing in blocks, approximate decomposition of H^-1,
 *        importance ordering).
 *
 * Readings where the pages are silent or garbled (each is listed in the
 * design notes of the repository):
 *   - U is the upper Cholesky factor of (H + lambda I)^-1, U^T U = H_l^-1;
 *     row j of U is the row of the inverse of the not-yet-quantized
 *     sub-Hessian scaled by 1/sqrt of its diagonal, so the sweep below is the
 *     exact sequential optimal-brain-surgeon update the pages describe.
 *   - lambda = damp_rel * mean(diag H); quantization of a group happens at its
 *     first column from the row's values after every earlier update.
 *   - Group range always includes 0: mn = min(0, min w), mx = max(0, max w);
 *     an all-zero group uses [-1, 1].
 *   - Quantization decisions (min/max, scale, zero point, code) are taken in
 *     IEEE fp32 from the fp32-rounded current weight, matching the fp32 working
 *     copy of the pages' code; all error-feedback arithmetic here is fp64.
 *   - s is rounded to fp16 (round-to-nearest-even) before use, clamped to the
 *     positive finite fp16 range [2^-24, 65504]; z = clamp(rne(-mn/s), 0, maxq).
 *   - code = clamp(rne(w/s) + z, 0, maxq), rne = round half to even.
 *
 * Build: gcc -O2 -ffp-contract=off -fopenmp -shared -fPIC (no fast-math: the
 * fp32 decisions must be IEEE single-precision operations).
 */
#include <stdint.h>
#include <stddef.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* IEEE binary16 <-> binary32/64, written from the format definition.        */
/* ------------------------------------------------------------------------ */

double orc_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int man = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)man, -24);              /* subnormal: man * 2^-24 */
    else if (e == 31)
        v = man ? NAN : INFINITY;
    else
        v = ldexp((double)(man | 0x400), e - 25); /* 1.man * 2^(e-15) */
    return sign ? -v : v;
}

/* Round a finite binary32 value to binary16, round-half-to-even. */
uint16_t orc_float_to_half_rne(float f)
{
    double a = fabs((double)f);
    uint16_t sign = signbit(f) ? 0x8000 : 0;
    if (isnan(f)) return 0x7e00;
    if (a >= 65520.0) return sign | 0x7c00;       /* halfway to 2^16 or more */
    if (a < ldexp(1.0, -14)) {                    /* subnormal range */
        double q = nearbyint(a / ldexp(1.0, -24)); /* exact scaling, RNE */
        return sign | (uint16_t)q;                /* q == 1024 encodes 2^-14 */
    }
    int ex;
    frexp(a, &ex);                                /* a = f * 2^ex, f in [0.5,1) */
    int e = ex - 1;                               /* 2^e <= a < 2^(e+1) */
    double quantum = ldexp(1.0, e - 10);
    double q = nearbyint(a / quantum);            /* 1024 .. 2048 */
    if (q >= 2048.0) { q = 1024.0; e += 1; }
    if (e > 15) return sign | 0x7c00;
    return sign | (uint16_t)(((e + 15) << 10) | ((int)q - 1024));
}

/* ------------------------------------------------------------------------ */
/* Group parameters and codes: [P3] sec. 一, [P4] sec. 2.1.                   */
/* ------------------------------------------------------------------------ */

typedef struct {
    uint16_t s16;   /* fp16 bit pattern of the scale */
    float s;        /* the same scale as fp32 (exact) */
    float s_pre;    /* fp32 scale before fp16 rounding */
    int z;          /* zero point, 0..maxq */
    float zq;       /* -mn / s in fp32, the value the zero point rounds */
} orc_gparams;

static orc_gparams orc_group_params(const double* w, int len, int maxq)
{
    float mn = 0.0f, mx = 0.0f;                   /* range includes 0 */
    for (int k = 0; k < len; ++k) {
        float x = (float)w[k];
        if (x < mn) mn = x;
        if (x > mx) mx = x;
    }
    if (mn == mx) { mn = -1.0f; mx = 1.0f; }      /* all-zero group */
    orc_gparams g;
    g.s_pre = (mx - mn) / (float)maxq;
    uint16_t h = orc_float_to_half_rne(g.s_pre);
    if ((h & 0x7fff) == 0) h = 0x0001;            /* smallest positive fp16 */
    if ((h & 0x7fff) >= 0x7c00) h = 0x7bff;       /* largest finite fp16 */
    g.s16 = h;
    g.s = (float)orc_half_to_double(h);
    g.zq = -mn / g.s;
    float zf = rintf(g.zq);
    if (zf < 0.0f) zf = 0.0f;
    if (zf > (float)maxq) zf = (float)maxq;
    g.z = (int)zf;
    return g;
}

/* code = clamp(rne(x/s) + z, 0, maxq), decided in fp32. */
static int orc_code(float x, float s, int z, int maxq)
{
    float c = rintf(x / s) + (float)z;
    if (!(c > 0.0f)) c = 0.0f;                    /* also maps NaN to 0 */
    if (c > (float)maxq) c = (float)maxq;
    return (int)c;
}

/* Distance of x/s (fp32) from the nearest rounding boundary k+0.5. */
static float orc_tie_distance(float x, float s)
{
    float t = x / s;
    float f = t - floorf(t);
    return fabsf(f - 0.5f);
}

/* ------------------------------------------------------------------------ */
/* Hessian: [P1] H = X^T X; [P3] H = 2 X X^T (X as d x n); [P5] H = 2 X^T X/n.*/
/* S = sum over tokens of x_t^T x_t, fp16 inputs promoted exactly.           */
/* ------------------------------------------------------------------------ */

void orc_hessian_accumulate(const uint16_t* X, int64_t n, int64_t d, double* S)
{
    double* xr = (double*)malloc(sizeof(double) * (size_t)d);
    for (int64_t t = 0; t < n; ++t) {
        for (int64_t i = 0; i < d; ++i) xr[i] = orc_half_to_double(X[t * d + i]);
        #pragma omp parallel for schedule(static)
        for (int64_t i = 0; i < d; ++i) {
            double xi = xr[i];
            if (xi == 0.0) continue;
            double* row = S + i * d;
            for (int64_t j = 0; j < d; ++j) row[j] += xi * xr[j];
        }
    }
    free(xr);
}

/* ------------------------------------------------------------------------ */
/* Finalize: H = 2 S / n ([P5]), act-order permutation, relative damping.   */
/* perm: stable descending argsort of diag(H) (ties: lower index first).     */
/* Returns 0, or 3 when mean(diag H) <= 0 (no damping can be formed).        */
/* ------------------------------------------------------------------------ */

static const double* orc_sort_keys;
static int orc_cmp_desc_stable(const void* a, const void* b)
{
    int32_t ia = *(const int32_t*)a, ib = *(const int32_t*)b;
    double ka = orc_sort_keys[ia], kb = orc_sort_keys[ib];
    if (ka > kb) return -1;
    if (ka < kb) return 1;
    return (ia < ib) ? -1 : (ia > ib);
}

/* The act-order permutation alone (stable descending argsort of diag). */
void orc_act_order_perm(const double* diag, int64_t d, int32_t* perm)
{
    for (int64_t i = 0; i < d; ++i) perm[i] = (int32_t)i;
    orc_sort_keys = diag;
    qsort(perm, (size_t)d, sizeof(int32_t), orc_cmp_desc_stable);
}

int orc_finalize(const double* S, int64_t n, int64_t d, double damp_rel,
                 int act_order, double* H, double* Hd, int32_t* perm, double* lam_out)
{
    double scale = 2.0 / (double)n;
    double* diag = (double*)malloc(sizeof(double) * (size_t)d);
    for (int64_t i = 0; i < d; ++i) diag[i] = scale * S[i * d + i];
    for (int64_t i = 0; i < d; ++i) perm[i] = (int32_t)i;
    if (act_order) {
        orc_sort_keys = diag;
        qsort(perm, (size_t)d, sizeof(int32_t), orc_cmp_desc_stable);
    }
    for (int64_t i = 0; i < d; ++i)
        for (int64_t j = 0; j < d; ++j)
            H[i * d + j] = scale * S[(int64_t)perm[i] * d + perm[j]];
    double mean = 0.0;
    for (int64_t i = 0; i < d; ++i) mean += H[i * d + i];
    mean /= (double)d;
    free(diag);
    double lam = damp_rel * mean;
    if (lam_out) *lam_out = lam;
    memcpy(Hd, H, sizeof(double) * (size_t)(d * d));
    for (int64_t i = 0; i < d; ++i) Hd[i * d + i] += lam;
    return (mean > 0.0) ? 0 : 3;
}

/* ------------------------------------------------------------------------ */
/* Dense linear algebra (own code, no LAPACK).                               */
/* ------------------------------------------------------------------------ */

/* Lower Cholesky A = L L^T, column by column; returns 0 or the 1-based index
 * of the first non-positive pivot (LAPACK convention). */
int orc_cholesky_lower(const double* A, int64_t d, double* L)
{
    memset(L, 0, sizeof(double) * (size_t)(d * d));
    for (int64_t j = 0; j < d; ++j) {
        const double* lj = L + j * d;
        double s = A[j * d + j];
        for (int64_t k = 0; k < j; ++k) s -= lj[k] * lj[k];
        if (!(s > 0.0)) return (int)(j + 1);
        double piv = sqrt(s);
        L[j * d + j] = piv;
        #pragma omp parallel for schedule(static)
        for (int64_t i = j + 1; i < d; ++i) {
            const double* li = L + i * d;
            double t = A[i * d + j];
            for (int64_t k = 0; k < j; ++k) t -= li[k] * lj[k];
            L[i * d + j] = t / piv;
        }
    }
    return 0;
}

/* Inverse of a lower-triangular L, returned TRANSPOSED: LinvT[j][i] =
 * (L^-1)[i][j], i.e. row j of LinvT is column j of L^-1 (forward substitution
 * of L x = e_j). Columns are independent. */
void orc_trtri_lower_T(const double* L, int64_t d, double* LinvT)
{
    memset(LinvT, 0, sizeof(double) * (size_t)(d * d));
    #pragma omp parallel for schedule(dynamic, 8)
    for (int64_t j = 0; j < d; ++j) {
        double* x = LinvT + j * d;
        for (int64_t i = j; i < d; ++i) {
            const double* li = L + i * d;
            double t = (i == j) ? 1.0 : 0.0;
            for (int64_t k = j; k < i; ++k) t -= li[k] * x[k];
            x[i] = t / li[i];
        }
    }
}

/* U = upper Cholesky factor of Hd^-1 by the plain route: L = chol(Hd),
 * Hd^-1 = L^-T L^-1, L2 = chol(Hd^-1), U = L2^T.  Returns the info of the
 * first factorization (0 when Hd is positive definite). */
int orc_hinv_upper_chol(const double* Hd, int64_t d, double* U)
{
    size_t dd = (size_t)(d * d);
    double* L = (double*)malloc(sizeof(double) * dd);
    double* LinvT = (double*)malloc(sizeof(double) * dd);
    int info = orc_cholesky_lower(Hd, d, L);
    if (info) { free(L); free(LinvT); return info; }
    orc_trtri_lower_T(L, d, LinvT);
    /* Hinv[i][j] = sum_k Linv[k][i] Linv[k][j] = dot(LinvT row i, row j). */
    double* Hinv = L;  /* reuse */
    #pragma omp parallel for schedule(dynamic, 8)
    for (int64_t i = 0; i < d; ++i) {
        const double* a = LinvT + i * d;
        for (int64_t j = i; j < d; ++j) {
            const double* b = LinvT + j * d;
            double t = 0.0;
            for (int64_t k = j; k < d; ++k) t += a[k] * b[k];  /* nonzero k >= max(i,j) */
            Hinv[i * d + j] = t;
            Hinv[j * d + i] = t;
        }
    }
    double* L2 = LinvT;  /* reuse */
    int info2 = orc_cholesky_lower(Hinv, d, L2);
    for (int64_t i = 0; i < d; ++i)
        for (int64_t j = 0; j < d; ++j)
            U[i * d + j] = (j >= i) ? L2[j * d + i] : 0.0;
    free(L); free(LinvT);
    return info2 ? -info2 : 0;
}

/* ------------------------------------------------------------------------ */
/* The column sweep: [P1] GPTQ pseudocode, [P3] sec. 三 loop, [P4] sec. 2.2 */
/* steps 1-5, [P5] sec. 一 (with U in place of the pages' H_inv rows).       */
/*                                                                           */
/* W: m x d float64 in sweep order (already permuted when act-order is on). */
/* U: d x d upper.  Outputs per row r and column j (sweep order):            */
/*   codes[r*d+j], scales16[r*G+gi], zeros[r*G+gi], row_loss[r] = sum E_j^2 */
/*   s_pre[r*G+gi] (fp32 scale before fp16 rounding).                        */
/* Teacher forcing (all nullable): when forced_codes[r*d+j] >= 0 the code is */
/* taken from it; when forced_s16 is given the group parameters are taken    */
/* from forced_s16/forced_z.  own_codes/tie_dist record the oracle's own     */
/* decision and the distance of w/s from the nearest rounding boundary;      */
/* own_s16/own_z/z_tie (m x G) record the oracle's own group parameters on   */
/* the (forced) trajectory and the distance of -mn/s from the nearest        */
/* rounding boundary k + 0.5 (nullable; bookkeeping only).                  */
/* ------------------------------------------------------------------------ */

void orc_quantize_rows(const double* W, const double* U, int64_t m, int64_t d,
                       int bits, int64_t group_size,
                       uint8_t* codes, uint16_t* scales16, uint8_t* zeros,
                       double* row_loss, float* s_pre,
                       const int16_t* forced_codes, const uint16_t* forced_s16,
                       const uint8_t* forced_z, uint8_t* own_codes, float* tie_dist,
                       uint16_t* own_s16, uint8_t* own_z, float* z_tie,
                       double* Wq_out)
{
    int maxq = (1 << bits) - 1;
    int64_t g = (group_size <= 0) ? d : group_size;
    int64_t G = (d + g - 1) / g;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < m; ++r) {
        double* w = (double*)malloc(sizeof(double) * (size_t)d);
        memcpy(w, W + r * d, sizeof(double) * (size_t)d);
        orc_gparams gp = {0, 1.0f, 1.0f, 0, 0.0f};
        double loss = 0.0;
        for (int64_t j = 0; j < d; ++j) {
            if (j % g == 0) {
                int64_t len = (j + g <= d) ? g : d - j;
                int64_t gi = j / g;
                orc_gparams own = orc_group_params(w + j, (int)len, maxq);
                if (s_pre) s_pre[r * G + gi] = own.s_pre;
                if (own_s16) own_s16[r * G + gi] = own.s16;
                if (own_z) own_z[r * G + gi] = (uint8_t)own.z;
                if (z_tie) z_tie[r * G + gi] = fabsf((own.zq - floorf(own.zq)) - 0.5f);
                gp = own;
                if (forced_s16) {
                    gp.s16 = forced_s16[r * G + gi];
                    gp.s = (float)orc_half_to_double(gp.s16);
                    gp.z = forced_z[r * G + gi];
                }
                scales16[r * G + gi] = gp.s16;
                zeros[r * G + gi] = (uint8_t)gp.z;
            }
            float x = (float)w[j];
            int c = orc_code(x, gp.s, gp.z, maxq);
            if (own_codes) own_codes[r * d + j] = (uint8_t)c;
            if (tie_dist) tie_dist[r * d + j] = orc_tie_distance(x, gp.s);
            if (forced_codes && forced_codes[r * d + j] >= 0) c = forced_codes[r * d + j];
            codes[r * d + j] = (uint8_t)c;
            double q = (double)gp.s * (double)(c - gp.z);
            double e = w[j] - q;
            const double* uj = U + j * d;
            double E = e / uj[j];
            loss += E * E;
            w[j] = q;
            for (int64_t k = j + 1; k < d; ++k) w[k] -= E * uj[k];
        }
        if (Wq_out) memcpy(Wq_out + r * d, w, sizeof(double) * (size_t)d);
        row_loss[r] = loss;
        free(w);
    }
}

/* Round-to-nearest baseline ([P2] "算法本质", [P4] sec. 2.1): the same group
 * quantizer on the original W, with no error feedback. */
void orc_rtn(const double* W, int64_t m, int64_t d, int bits, int64_t group_size,
             uint8_t* codes, uint16_t* scales16, uint8_t* zeros, float* s_pre)
{
    int maxq = (1 << bits) - 1;
    int64_t g = (group_size <= 0) ? d : group_size;
    int64_t G = (d + g - 1) / g;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < m; ++r) {
        const double* w = W + r * d;
        for (int64_t gi = 0; gi < G; ++gi) {
            int64_t j0 = gi * g;
            int64_t len = (j0 + g <= d) ? g : d - j0;
            orc_gparams gp = orc_group_params(w + j0, (int)len, maxq);
            scales16[r * G + gi] = gp.s16;
            zeros[r * G + gi] = (uint8_t)gp.z;
            if (s_pre) s_pre[r * G + gi] = gp.s_pre;
            for (int64_t j = j0; j < j0 + len; ++j)
                codes[r * d + j] = (uint8_t)orc_code((float)w[j], gp.s, gp.z, maxq);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Packing ([P3] sec. 一 storage arithmetic): 8 four-bit codes per uint32,   */
/* lowest column in the lowest nibble; zero points two per byte, even group */
/* in the low nibble, an odd group count padded with a zero nibble.          */
/* ------------------------------------------------------------------------ */

void orc_pack_int4(const uint8_t* codes, const uint8_t* zeros, int64_t m, int64_t d,
                   int64_t G, uint32_t* qweight, uint8_t* qzeros)
{
    int64_t W8 = d / 8, Gb = (G + 1) / 2;
    for (int64_t r = 0; r < m; ++r) {
        for (int64_t w = 0; w < W8; ++w) {
            uint32_t v = 0;
            for (int k = 0; k < 8; ++k)
                v |= (uint32_t)(codes[r * d + 8 * w + k] & 0xf) << (4 * k);
            qweight[r * W8 + w] = v;
        }
        for (int64_t b = 0; b < Gb; ++b) {
            uint8_t lo = zeros[r * G + 2 * b] & 0xf;
            uint8_t hi = (2 * b + 1 < G) ? (zeros[r * G + 2 * b + 1] & 0xf) : 0;
            qzeros[r * Gb + b] = (uint8_t)(lo | (hi << 4));
        }
    }
}

void orc_unpack_int4(const uint32_t* qweight, const uint8_t* qzeros, int64_t m, int64_t d,
                     int64_t G, uint8_t* codes, uint8_t* zeros)
{
    int64_t W8 = d / 8, Gb = (G + 1) / 2;
    for (int64_t r = 0; r < m; ++r) {
        for (int64_t w = 0; w < W8; ++w)
            for (int k = 0; k < 8; ++k)
                codes[r * d + 8 * w + k] = (uint8_t)((qweight[r * W8 + w] >> (4 * k)) & 0xf);
        for (int64_t gi = 0; gi < G; ++gi) {
            uint8_t b = qzeros[r * Gb + gi / 2];
            zeros[r * G + gi] = (gi & 1) ? (uint8_t)(b >> 4) : (uint8_t)(b & 0xf);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* b-bit packing (b in 2..8) for the other widths the INT4/INT8 page names   */
/* beside the 4-bit storage of its sec. 一: each row's codes form one        */
/* little-endian bit stream, code k in bits [b k, b k + b), stored as uint32 */
/* words; the row's zero points form a second stream stored as bytes, its    */
/* last byte padded with zero bits.  For b = 4 this is the INT4 layout.      */
/* ------------------------------------------------------------------------ */

void orc_pack_bits(const uint8_t* codes, const uint8_t* zeros, int64_t m, int64_t d, int64_t G,
                   int bits, uint32_t* qweight, uint8_t* qzeros)
{
    int64_t nw = d * bits / 32, nb = (G * bits + 7) / 8;
    uint32_t mask = (1u << bits) - 1u;
    for (int64_t r = 0; r < m; ++r) {
        for (int64_t w = 0; w < nw; ++w) qweight[r * nw + w] = 0;
        for (int64_t k = 0; k < d; ++k) {
            uint64_t bit = (uint64_t)k * (uint64_t)bits;
            uint32_t c = codes[r * d + k] & mask;
            for (int t = 0; t < bits; ++t) {            /* one bit at a time */
                uint64_t pos = bit + (uint64_t)t;
                if ((c >> t) & 1u) qweight[r * nw + (int64_t)(pos / 32)] |= 1u << (pos % 32);
            }
        }
        for (int64_t b = 0; b < nb; ++b) qzeros[r * nb + b] = 0;
        for (int64_t gi = 0; gi < G; ++gi) {
            uint64_t bit = (uint64_t)gi * (uint64_t)bits;
            uint32_t z = zeros[r * G + gi] & mask;
            for (int t = 0; t < bits; ++t) {
                uint64_t pos = bit + (uint64_t)t;
                if ((z >> t) & 1u) qzeros[r * nb + (int64_t)(pos / 8)] |= (uint8_t)(1u << (pos % 8));
            }
        }
    }
}

void orc_unpack_bits(const uint32_t* qweight, const uint8_t* qzeros, int64_t m, int64_t d,
                     int64_t G, int bits, uint8_t* codes, uint8_t* zeros)
{
    int64_t nw = d * bits / 32, nb = (G * bits + 7) / 8;
    for (int64_t r = 0; r < m; ++r) {
        for (int64_t k = 0; k < d; ++k) {
            uint32_t c = 0;
            for (int t = 0; t < bits; ++t) {
                uint64_t pos = (uint64_t)k * (uint64_t)bits + (uint64_t)t;
                c |= ((qweight[r * nw + (int64_t)(pos / 32)] >> (pos % 32)) & 1u) << t;
            }
            codes[r * d + k] = (uint8_t)c;
        }
        for (int64_t gi = 0; gi < G; ++gi) {
            uint32_t z = 0;
            for (int t = 0; t < bits; ++t) {
                uint64_t pos = (uint64_t)gi * (uint64_t)bits + (uint64_t)t;
                z |= ((uint32_t)(qzeros[r * nb + (int64_t)(pos / 8)] >> (pos % 8)) & 1u) << t;
            }
            zeros[r * G + gi] = (uint8_t)z;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Layer loss ([P3] sec. 三 objective, [P5] sec. 一 "F-norm squared"):       */
/* tr(D H D^T) with D = W - Q, for a symmetric H (fp64).                     */
/* ------------------------------------------------------------------------ */

double orc_trace_quadratic(const double* D, const double* H, int64_t m, int64_t d)
{
    double total = 0.0;
    #pragma omp parallel for reduction(+:total) schedule(static)
    for (int64_t r = 0; r < m; ++r) {
        const double* dr = D + r * d;
        double acc = 0.0;
        for (int64_t i = 0; i < d; ++i) {
            if (dr[i] == 0.0) continue;
            const double* hi = H + i * d;
            double t = 0.0;
            for (int64_t j = 0; j < d; ++j) t += hi[j] * dr[j];
            acc += dr[i] * t;
        }
        total += acc;
    }
    return total;
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
