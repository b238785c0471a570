/*
 * stq_oracle.cpp -- plain, single-threaded CPU oracle for the quantized
 * Delta-rule recurrent-state decode step.
 *
 * TEST INFRASTRUCTURE ONLY (see stq_oracle.h).  Built with
 * -O2 -ffp-contract=off and no fast-math, so every float expression below is
 * evaluated exactly as written: one IEEE rounding per +, -, *, /, and fmaf
 * only where it is spelled out.
 *
 * Three evaluations of the step live here:
 *   orc_step_f64        the plain definition in double precision, natural key
 *                       order;
 *   orc_step_f32_plain  the plain fp32 evaluation: every column sum one fma
 *                       chain over the key channels in natural order; the
 *                       anchor the GPU is compared with under the rounding-
 *                       band rule (codes may differ only where the fp32
 *                       rounding of any evaluation order can move the
 *                       pre-rounding value across a boundary);
 *   orc_step_f32        the canonical fp32 evaluation, the decode kernel's own
 *                       summation order, which the GPU must reproduce bit for
 *                       bit (a second, stricter check).  The pages fix no fp32
 *                       evaluation order; this one is the kernel's:
 *                   - the state is handled in column-normalised units
 *                     T = S / c (so the value-column scale c_j leaves the
 *                     inner loops);
 *                   - a column sum sum_s w_s T_sj deals the stored rows
 *                     of every 16-row block into four slices of 4
 *                     consecutive rows (slice (s mod 16) / 4); the rows of
 *                     one slice in one half of the page (s / 64) form a
 *                     chain p = fmaf(w_s, T_sj, p) from p = 0 in ascending
 *                     s; per slice the two half partials are added, and the
 *                     four slice sums by a pairwise tree in slice order,
 *                     (R0 + R1) + (R2 + R3);
 *                   - requantization rounds the exact product T' * inv once
 *                     (to an integer, ties to even);
 *                   - inv = qmax / m rounded toward zero, which keeps every
 *                     scaled value inside [-qmax, qmax].
 *                 orc_step_f64 pins both fp32 evaluations to the mathematics.
 *
 * parity pins: every function here is pinned by tests/test_oracle_*.py
 * (closed forms, brute force at d_k = d_v = 4, invariants, library
 * routines).  No function is "parity unpinned".
 */
#include "stq_oracle.h"

#include <cmath>
#include <cstring>
#include <vector>
#include <algorithm>

/* the canonical column-sum partition (see the header comment) */
static const int ORC_BLOCK_ROWS = 16;   /* rows of a block */
static const int ORC_SLICE_ROWS = 4;    /* consecutive rows of a block in one slice */
static const int ORC_HALF_ROWS = 64;    /* rows whose slice rows form one chain */

/* ------------------------------------------------------------------------ */
/* format helpers                                                           */
/* ------------------------------------------------------------------------ */

static int group_of_row(const orc_format *f, int s)
{
    int acc = 0;
    for (int g = 0; g < f->n_groups; ++g) {
        acc += f->group_rows[g];
        if (s < acc) return g;
    }
    return -1;
}

extern "C" int orc_format_check(const orc_format *f)
{
    if (!f) return -1;
    if (f->d_k < 1 || f->d_v < 1 || f->d_k > 4096 || f->d_v > 4096) return -2;
    if (f->n_groups < 1 || f->n_groups > ORC_MAX_GROUPS) return -3;
    int total = 0;
    for (int g = 0; g < f->n_groups; ++g) {
        if (f->group_rows[g] < 1) return -4;
        total += f->group_rows[g];
        int kind = f->group_kind[g];
        if (kind == ORC_KIND_INT) {
            if (f->group_bits[g] < 2 || f->group_bits[g] > 8) return -5;
        } else if (kind != ORC_KIND_FP16 && kind != ORC_KIND_FP32) {
            return -6;
        }
    }
    if (total != f->d_k) return -7;
    return 0;
}

extern "C" int orc_row_kind(const orc_format *f, int s)
{
    return f->group_kind[group_of_row(f, s)];
}

extern "C" int orc_row_qmax(const orc_format *f, int s)
{
    int g = group_of_row(f, s);
    if (f->group_kind[g] != ORC_KIND_INT) return 0;
    return (1 << (f->group_bits[g] - 1)) - 1;
}

/* Planes of a b-bit code: the binary decomposition of b, widest plane first,
 * the widest plane holding the lowest bits.  FP16 rows are one 16-bit plane. */
static int planes_of(int kind, int bits, int width[3], int low[3])
{
    if (kind == ORC_KIND_FP16) { width[0] = 16; low[0] = 0; return 1; }
    if (bits == 8) { width[0] = 8; low[0] = 0; return 1; }
    int n = 0, lo = 0;
    for (int w = 4; w >= 1; w >>= 1) {
        if (bits & w) { width[n] = w; low[n] = lo; lo += w; ++n; }
    }
    return n;
}

static int packable(const orc_format *f)
{
    if (orc_format_check(f) != 0) return 0;
    if (f->d_k != 128 || f->d_v != 128) return 0;
    for (int g = 0; g < f->n_groups; ++g) {
        if (f->group_rows[g] % 16 != 0) return 0;
        if (f->group_kind[g] == ORC_KIND_FP32) return 0;
    }
    return 1;
}

static int n_int_rows(const orc_format *f)
{
    int n = 0;
    for (int g = 0; g < f->n_groups; ++g)
        if (f->group_kind[g] == ORC_KIND_INT) n += f->group_rows[g];
    return n;
}

extern "C" long orc_page_bytes(const orc_format *f)
{
    if (!packable(f)) return -1;
    long bytes = 0;
    for (int blk = 0; blk < 8; ++blk) {
        int g = group_of_row(f, 16 * blk);
        int width[3], low[3];
        int np = planes_of(f->group_kind[g], f->group_bits[g], width, low);
        for (int p = 0; p < np; ++p) bytes += 256L * width[p];
    }
    bytes += 4L * n_int_rows(f);
    if (f->col_scales) bytes += 4L * 128;
    return bytes;
}

/* ------------------------------------------------------------------------ */
/* scalar building blocks                                                   */
/* ------------------------------------------------------------------------ */

static float bits_to_f32(uint32_t u) { float x; std::memcpy(&x, &u, 4); return x; }
static uint32_t f32_to_bits(float x) { uint32_t u; std::memcpy(&u, &x, 4); return u; }

/* IEEE 754 binary16, round to nearest, ties to even, with subnormals;
 * written from the format's definition: value = (-1)^s 2^(e-15) (1 + m/1024)
 * for 1 <= e <= 30, (-1)^s 2^-14 (m/1024) for e = 0. */
extern "C" uint16_t orc_f32_to_f16_rn(float x)
{
    uint32_t u = f32_to_bits(x);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    float ax = std::fabs(x);
    if (std::isnan(x)) return (uint16_t)(sign | 0x7E00u);
    if (std::isinf(x)) return (uint16_t)(sign | 0x7C00u);
    /* largest finite half is 65504; the midpoint to the next (virtual) value
     * 65536 is 65520, which ties to the even significand, i.e. overflows */
    if (ax >= 65520.0f) return (uint16_t)(sign | 0x7C00u);
    if (ax < 0x1p-14f) {
        /* subnormal range: multiples of 2^-24 */
        double t = (double)ax * 0x1p24;          /* exact */
        double n = std::nearbyint(t);            /* ties to even */
        return (uint16_t)(sign | (uint16_t)n);   /* n == 1024 is the smallest normal */
    }
    int e = std::ilogb(ax);                      /* -14 .. 15 */
    double t = std::ldexp((double)ax, 10 - e);   /* in [1024, 2048), exact */
    double n = std::nearbyint(t);
    if (n >= 2048.0) { n = 1024.0; e += 1; }
    if (e > 15) return (uint16_t)(sign | 0x7C00u);
    return (uint16_t)(sign | (uint16_t)((e + 15) << 10) | (uint16_t)((int)n - 1024));
}

extern "C" float orc_f16_to_f32(uint16_t h)
{
    int s = (h >> 15) & 1, e = (h >> 10) & 0x1F, m = h & 0x3FF;
    double v;
    if (e == 0) v = std::ldexp((double)m, -24);
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = std::ldexp((double)(1024 + m), e - 25);
    return (float)(s ? -v : v);
}

/* a / b rounded toward zero (a, b > 0 finite): the largest float q with
 * q * b <= a.  Products of two floats are exact in double. */
extern "C" float orc_div_rz(float a, float b)
{
    float q = (float)((double)a / (double)b);
    while ((double)q * (double)b > (double)a) q = std::nextafter(q, 0.0f);
    for (;;) {
        float up = std::nextafter(q, INFINITY);
        if ((double)up * (double)b <= (double)a) q = up; else break;
    }
    return q;
}

extern "C" void orc_f32_to_f16_rn_n(const float *x, uint16_t *out, long n)
{
    for (long i = 0; i < n; ++i) out[i] = orc_f32_to_f16_rn(x[i]);
}

extern "C" void orc_f16_to_f32_n(const uint16_t *x, float *out, long n)
{
    for (long i = 0; i < n; ++i) out[i] = orc_f16_to_f32(x[i]);
}

extern "C" void orc_div_rz_n(const float *a, const float *b, float *out, long n)
{
    for (long i = 0; i < n; ++i) out[i] = orc_div_rz(a[i], b[i]);
}

/* pcg4d, the four-word hash of Jarzynski and Olano, "Hash Functions for GPU
 * Rendering" (Journal of Computer Graphics Techniques 9(3), 2020): a linear
 * congruential step on each word (multiplier 1664525, increment 1013904223),
 * then each word plus the product of two others, a 16-bit xorshift of every
 * word, and the products once more.  Every step is invertible, so the map is
 * a bijection of the 128-bit input. */
extern "C" void orc_pcg4d(const uint32_t in[4], uint32_t out[4])
{
    uint32_t x = in[0], y = in[1], z = in[2], w = in[3];
    x = x * 1664525u + 1013904223u;
    y = y * 1664525u + 1013904223u;
    z = z * 1664525u + 1013904223u;
    w = w * 1664525u + 1013904223u;
    x += y * w;
    y += z * x;
    z += x * y;
    w += y * z;
    x ^= x >> 16;
    y ^= y >> 16;
    z ^= z >> 16;
    w ^= w >> 16;
    x += y * w;
    y += z * x;
    z += x * y;
    w += y * z;
    out[0] = x; out[1] = y; out[2] = z; out[3] = w;
}

/* Stochastic-rounding offset for element (s, j) of page (b, h) at a step.
 * One hash serves a 2-row x 4-column tile: input (tile index, step,
 * request ^ low seed word, head ^ high seed word).  Word 2*(s & 1) +
 * ((j >> 1) & 1) of the output holds columns j & ~1 (high 16 bits) and j | 1
 * (low 16 bits).  u = h16 / 65536 in [0, 1), exactly; the rounded code is
 * floor(x + u), x the exact scaled value. */
extern "C" float orc_sr_offset(uint64_t seed, uint32_t step, uint32_t b, uint32_t h,
                               int s, int j, int d_v)
{
    uint32_t quads = (uint32_t)((d_v + 3) / 4);
    uint32_t in[4] = { (uint32_t)(s >> 1) * quads + (uint32_t)(j >> 2), step,
                       b ^ (uint32_t)seed, h ^ (uint32_t)(seed >> 32) };
    uint32_t out[4];
    orc_pcg4d(in, out);
    uint32_t word = out[((s & 1) << 1) | ((j >> 1) & 1)];
    uint32_t h16 = (j & 1) ? (word & 0xFFFFu) : (word >> 16);
    return (float)h16 * 0x1p-16f;
}

/* ------------------------------------------------------------------------ */
/* requantization of one stored row (shared by quantize and step)          */
/* ------------------------------------------------------------------------ */

static double dist_to_half(double x)
{
    return std::fabs(x - (std::floor(x) + 0.5));
}

static double dist_to_int(double x)
{
    return std::fabs(x - std::nearbyint(x));
}

static double f16_margin(float x)
{
    double ax = std::fabs((double)x);
    double spacing;
    if (ax < 0x1p-14) spacing = 0x1p-24;
    else spacing = std::ldexp(1.0, std::ilogb(ax) - 10);
    return dist_to_half(ax / spacing);
}

static void requant_row(const orc_format *f, int s, const float *Tp, orc_page *p,
                        uint64_t seed, uint32_t step, uint32_t b, uint32_t h,
                        int use_sr, double *margin)
{
    const int d_v = f->d_v;
    const int kind = orc_row_kind(f, s);
    int32_t *code = p->code + (size_t)s * d_v;
    if (kind == ORC_KIND_FP32) {
        for (int j = 0; j < d_v; ++j) {
            code[j] = (int32_t)f32_to_bits(Tp[j]);
            if (margin) margin[j] = INFINITY;
        }
        p->r[s] = 0.0f;
        return;
    }
    if (kind == ORC_KIND_FP16) {
        for (int j = 0; j < d_v; ++j) {
            code[j] = (int32_t)orc_f32_to_f16_rn(Tp[j]);
            if (margin) margin[j] = f16_margin(Tp[j]);
        }
        p->r[s] = 0.0f;
        return;
    }
    const int qmax = orc_row_qmax(f, s);
    float m = 0.0f;
    for (int j = 0; j < d_v; ++j) {
        float a = std::fabs(Tp[j]);
        if (a > m) m = a;
    }
    float r, inv;
    if (m > 0.0f) {
        r = m / (float)qmax;
        inv = orc_div_rz((float)qmax, m);
    } else {
        r = 0.0f;
        inv = 0.0f;
    }
    p->r[s] = r;
    for (int j = 0; j < d_v; ++j) {
        double x = (double)Tp[j] * (double)inv;    /* exact */
        double zr;
        if (!use_sr) {
            zr = std::nearbyint(x);
            if (margin) margin[j] = dist_to_half(x);
        } else {
            /* floor(x + u) of the exact sum: x >= fl + 1 - u compares two
             * exact doubles (fl an integer, u on the 2^-16 grid) */
            double u = (double)orc_sr_offset(seed, step, b, h, s, j, d_v);
            double fl = std::floor(x);
            zr = (x >= fl + 1.0 - u) ? fl + 1.0 : fl;
            if (margin) margin[j] = dist_to_int(x + u);
        }
        if (!(zr == zr)) zr = 0.0;                 /* non-finite input */
        if (zr > qmax) zr = qmax;
        if (zr < -qmax) zr = -qmax;
        code[j] = (int32_t)zr;
    }
}

/* value held by element (s, j): the integer code, or the float it encodes */
static float element_value(const orc_format *f, const orc_page *p, int s, int j)
{
    int32_t c = p->code[(size_t)s * f->d_v + j];
    int kind = orc_row_kind(f, s);
    if (kind == ORC_KIND_INT) return (float)c;
    if (kind == ORC_KIND_FP16) return orc_f16_to_f32((uint16_t)c);
    return bits_to_f32((uint32_t)c);
}

/* ------------------------------------------------------------------------ */
/* calibration: precision map                                               */
/* ------------------------------------------------------------------------ */

extern "C" int orc_rank_rows(const orc_format *f, int B, int H, const float *S,
                             const float *row_weight, int32_t *perm_out)
{
    if (orc_format_check(f) != 0 || B < 1 || H < 1 || !S || !perm_out) return -1;
    const int d_k = f->d_k, d_v = f->d_v;
    std::vector<double> score(d_k);
    std::vector<int> order(d_k);
    for (int h = 0; h < H; ++h) {
        /* score = row-mean-square summed over the batch, times the optional
         * retention weight; the constant 1 / (B d_v) is left out (it does
         * not change the ranking).  In double: per request the row's sum of
         * squares (columns in order), added over the requests in order. */
        for (int kap = 0; kap < d_k; ++kap) {
            double acc = 0.0;
            for (int b = 0; b < B; ++b) {
                const float *row = S + (((size_t)b * H + h) * d_k + kap) * d_v;
                double rs = 0.0;
                for (int j = 0; j < d_v; ++j) rs += (double)row[j] * (double)row[j];
                acc += rs;
            }
            if (row_weight) acc *= (double)row_weight[(size_t)h * d_k + kap];
            score[kap] = acc;
        }
        for (int kap = 0; kap < d_k; ++kap) order[kap] = kap;
        /* descending score; equal scores keep ascending key channel */
        std::stable_sort(order.begin(), order.end(),
                         [&](int a, int b2) { return score[a] > score[b2]; });
        /* the best-ranked rows go to the first (widest) group; inside a group
         * rows are stored in ascending key channel */
        int32_t *perm = perm_out + (size_t)h * d_k;
        int start = 0;
        for (int g = 0; g < f->n_groups; ++g) {
            int n = f->group_rows[g];
            std::vector<int> members(order.begin() + start, order.begin() + start + n);
            std::sort(members.begin(), members.end());
            for (int i = 0; i < n; ++i) perm[start + i] = members[i];
            start += n;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* quantize / dequantize                                                    */
/* ------------------------------------------------------------------------ */

extern "C" int orc_quantize_page(const orc_format *f, const float *S_nat,
                                 const int32_t *perm, orc_page *out)
{
    if (orc_format_check(f) != 0 || !S_nat || !perm || !out) return -1;
    const int d_k = f->d_k, d_v = f->d_v;
    std::vector<float> ic(d_v);
    for (int j = 0; j < d_v; ++j) {
        float c = 1.0f;
        if (f->col_scales) {
            float m = 0.0f;
            for (int kap = 0; kap < d_k; ++kap) {
                float a = std::fabs(S_nat[(size_t)kap * d_v + j]);
                if (a > m) m = a;
            }
            c = (m > 0.0f) ? m : 1.0f;
        }
        out->c[j] = c;
        ic[j] = f->col_scales ? 1.0f / c : 1.0f;
    }
    std::vector<float> T(d_v);
    for (int s = 0; s < d_k; ++s) {
        const float *row = S_nat + (size_t)perm[s] * d_v;
        for (int j = 0; j < d_v; ++j) T[j] = row[j] * ic[j];
        /* the initial quantization always rounds to nearest */
        requant_row(f, s, T.data(), out, 0, 0, 0, 0, 0, nullptr);
    }
    return 0;
}

extern "C" int orc_dequantize_page(const orc_format *f, const orc_page *p,
                                   const int32_t *perm, float *S_nat)
{
    if (orc_format_check(f) != 0 || !p || !perm || !S_nat) return -1;
    const int d_k = f->d_k, d_v = f->d_v;
    for (int s = 0; s < d_k; ++s) {
        int kind = orc_row_kind(f, s);
        float rs = (kind == ORC_KIND_INT) ? p->r[s] : 1.0f;
        for (int j = 0; j < d_v; ++j) {
            float x = element_value(f, p, s, j);
            float c = f->col_scales ? p->c[j] : 1.0f;
            S_nat[(size_t)perm[s] * d_v + j] = (x * rs) * c;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* joint fit of the row and column scales (STEPQuant's scale fitting)       */
/* ------------------------------------------------------------------------ */

/* Codes of INT row s for float scales r and c: the nearest code to
 * S / (r c) (the product r c exact in double, one correctly rounded double
 * division, ties to even), clamped to [-qmax, qmax]; 0 where r c is 0. */
static void fit_codes_row(const orc_format *f, int s, const float *S_row, float r, const float *c, int32_t *z)
{
    const int qmax = orc_row_qmax(f, s);
    for (int j = 0; j < f->d_v; ++j) {
        const double d = (double)r * (double)c[j];
        double n = (d > 0.0) ? std::nearbyint((double)S_row[j] / d) : 0.0;
        if (n > qmax) n = qmax;
        if (n < -qmax) n = -qmax;
        z[j] = (int32_t)n;
    }
}

/* sum over INT rows of w_kappa sum_j (S - z r c)^2, in double */
static double fit_objective(const orc_format *f, const float *S_nat, const int32_t *perm, const float *w_nat,
                            const std::vector<int32_t> &z, const std::vector<float> &r, const std::vector<float> &c)
{
    double e = 0.0;
    for (int s = 0; s < f->d_k; ++s) {
        if (orc_row_kind(f, s) != ORC_KIND_INT) continue;
        const int kap = perm[s];
        double row = 0.0;
        for (int j = 0; j < f->d_v; ++j) {
            const double d = (double)S_nat[(size_t)kap * f->d_v + j]
                             - (double)z[(size_t)s * f->d_v + j] * (double)r[s] * (double)c[j];
            row += d * d;
        }
        e += (w_nat ? (double)w_nat[kap] : 1.0) * row;
    }
    return e;
}

extern "C" int orc_quantize_page_fit(const orc_format *f, const float *S_nat, const int32_t *perm,
                                     const float *impact_nat, int iters, orc_page *out, double *err_out)
{
    if (orc_format_check(f) != 0 || !S_nat || !perm || !out || iters < 0) return -1;
    const int d_k = f->d_k, d_v = f->d_v;
    /* start from the absmax scales */
    int rc = orc_quantize_page(f, S_nat, perm, out);
    if (rc != 0) return rc;
    std::vector<float> r(out->r, out->r + d_k), c(out->c, out->c + d_v);
    std::vector<int32_t> z((size_t)d_k * d_v, 0);
    std::vector<int> row_of(d_k);
    for (int s = 0; s < d_k; ++s) row_of[perm[s]] = s;
    for (int it = 0; it < iters; ++it) {
        /* the nearest codes for the current scales */
        for (int s = 0; s < d_k; ++s)
            if (orc_row_kind(f, s) == ORC_KIND_INT)
                fit_codes_row(f, s, S_nat + (size_t)perm[s] * d_v, r[s], c.data(), z.data() + (size_t)s * d_v);
        if (err_out) err_out[it] = fit_objective(f, S_nat, perm, impact_nat, z, r, c);
        /* row scales: least squares of each row with its codes and c fixed,
         * r_s = sum_j S z c / sum_j (z c)^2 (the row's impact weight cancels) */
        for (int s = 0; s < d_k; ++s) {
            if (orc_row_kind(f, s) != ORC_KIND_INT) continue;
            const float *Sr = S_nat + (size_t)perm[s] * d_v;
            double num = 0.0, den = 0.0;
            for (int j = 0; j < d_v; ++j) {
                const double zc = (double)z[(size_t)s * d_v + j] * (double)c[j];
                num += (double)Sr[j] * zc;
                den += zc * zc;
            }
            if (den > 0.0) r[s] = (float)(num / den);
        }
        /* column scales: impact-weighted least squares of each column with
         * the codes and r fixed, c_j = sum_kappa w S z r / sum_kappa w (z r)^2,
         * over the INT rows in natural key order */
        if (f->col_scales) {
            for (int j = 0; j < d_v; ++j) {
                double num = 0.0, den = 0.0;
                for (int kap = 0; kap < d_k; ++kap) {
                    const int s = row_of[kap];
                    if (orc_row_kind(f, s) != ORC_KIND_INT) continue;
                    const double w = impact_nat ? (double)impact_nat[kap] : 1.0;
                    const double zr = (double)z[(size_t)s * d_v + j] * (double)r[s];
                    num += w * ((double)S_nat[(size_t)kap * d_v + j] * zr);
                    den += w * (zr * zr);
                }
                if (den > 0.0) c[j] = (float)(num / den);
            }
        }
    }
    /* final codes for the fitted scales; float rows as the quantizer stores them */
    for (int s = 0; s < d_k; ++s) {
        const float *Sr = S_nat + (size_t)perm[s] * d_v;
        if (orc_row_kind(f, s) == ORC_KIND_INT) {
            if (iters > 0) fit_codes_row(f, s, Sr, r[s], c.data(), out->code + (size_t)s * d_v);
            else for (int j = 0; j < d_v; ++j) z[(size_t)s * d_v + j] = out->code[(size_t)s * d_v + j];
            out->r[s] = r[s];
        } else if (iters > 0) {
            std::vector<float> T(d_v);
            for (int j = 0; j < d_v; ++j) T[j] = Sr[j] * (f->col_scales ? 1.0f / c[j] : 1.0f);
            requant_row(f, s, T.data(), out, 0, 0, 0, 0, 0, nullptr);
        }
    }
    for (int j = 0; j < d_v; ++j) out->c[j] = c[j];
    if (err_out) {
        std::vector<int32_t> zf(out->code, out->code + (size_t)d_k * d_v);
        err_out[iters] = fit_objective(f, S_nat, perm, impact_nat, zf, r, c);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* decode step: canonical fp32 evaluation                                   */
/* ------------------------------------------------------------------------ */

static float tree_sum(const float *P, int n)
{
    if (n == 1) return P[0];
    int m = (n + 1) / 2;
    return tree_sum(P, m) + tree_sum(P + m, n - m);
}

/* out_j = sum over stored rows s of w[perm[s]] * X[s][j] in the canonical
 * order: chain (slice, half) over the rows s with (s mod 16) / 4 == slice and
 * s / 64 == half, ascending; per slice a tree over its non-empty half
 * chains, then a tree over the non-empty slices in slice order. */
static void column_sum(const orc_format *f, const int32_t *perm, const float *w_nat,
                       const float *X, float *out)
{
    const int d_k = f->d_k, d_v = f->d_v;
    const int n_slice = ORC_BLOCK_ROWS / ORC_SLICE_ROWS;
    const int n_half = (d_k + ORC_HALF_ROWS - 1) / ORC_HALF_ROWS;
    std::vector<float> P(n_half), R(n_slice);
    for (int j = 0; j < d_v; ++j) {
        int nr = 0;
        for (int w = 0; w < n_slice; ++w) {
            int np = 0;
            for (int h = 0; h < n_half; ++h) {
                float acc = 0.0f;
                bool any = false;
                for (int s = h * ORC_HALF_ROWS; s < std::min(d_k, (h + 1) * ORC_HALF_ROWS); ++s) {
                    if ((s % ORC_BLOCK_ROWS) / ORC_SLICE_ROWS != w) continue;
                    acc = std::fmaf(w_nat[perm[s]], X[(size_t)s * d_v + j], acc);
                    any = true;
                }
                if (any) P[np++] = acc;
            }
            if (np > 0) R[nr++] = tree_sum(P.data(), np);
        }
        out[j] = tree_sum(R.data(), nr);
    }
}

/* The plain evaluation: out_j = sum over key channels kappa = 0 .. d_k - 1 in
 * natural order of w[kappa] * X[s(kappa)][j] (s(kappa): the stored row that
 * holds channel kappa), one fma chain from +0.  Nothing in it follows a
 * thread mapping; it is the sum of the definition written left to right. */
static void column_sum_plain(const orc_format *f, const int32_t *perm, const float *w_nat,
                             const float *X, float *out)
{
    const int d_k = f->d_k, d_v = f->d_v;
    std::vector<int> row_of(d_k);
    for (int s = 0; s < d_k; ++s) row_of[perm[s]] = s;
    for (int j = 0; j < d_v; ++j) {
        float acc = 0.0f;
        for (int kap = 0; kap < d_k; ++kap)
            acc = std::fmaf(w_nat[kap], X[(size_t)row_of[kap] * d_v + j], acc);
        out[j] = acc;
    }
}

static void column_sum_in(int plain, const orc_format *f, const int32_t *perm, const float *w_nat,
                          const float *X, float *out)
{
    if (plain) column_sum_plain(f, perm, w_nat, X, out);
    else column_sum(f, perm, w_nat, X, out);
}

static int step_f32(int plain, const orc_format *f, orc_page *page, const int32_t *perm,
                    const float *q, const float *k, const float *v,
                    const float *alpha, float beta, float *o_out,
                    uint64_t seed, uint32_t step, uint32_t b, uint32_t h,
                    float *Tp_out, double *margin_out)
{
    if (orc_format_check(f) != 0 || !page || !perm || !q || !k || !v || !alpha || !o_out)
        return -1;
    const int d_k = f->d_k, d_v = f->d_v;
    std::vector<float> ic(d_v), a(d_k), T((size_t)d_k * d_v), Tp((size_t)d_k * d_v);
    std::vector<float> u(d_v), e(d_v), ot(d_v);

    for (int j = 0; j < d_v; ++j) ic[j] = f->col_scales ? 1.0f / page->c[j] : 1.0f;

    /* dequantize into column-normalised units and decay: T = z * (alpha r) */
    for (int s = 0; s < d_k; ++s) {
        float al = f->gate_vector ? alpha[perm[s]] : alpha[0];
        a[s] = (orc_row_kind(f, s) == ORC_KIND_INT) ? al * page->r[s] : al;
        for (int j = 0; j < d_v; ++j)
            T[(size_t)s * d_v + j] = element_value(f, page, s, j) * a[s];
    }
    /* prediction (A S)^T k, then the error e = v - prediction (both / c) */
    column_sum_in(plain, f, perm, k, T.data(), u.data());
    for (int j = 0; j < d_v; ++j) e[j] = v[j] * ic[j] - u[j];
    /* rank-1 delta update T' = T + (beta k) e^T */
    for (int s = 0; s < d_k; ++s) {
        float bk = beta * k[perm[s]];
        for (int j = 0; j < d_v; ++j) {
            size_t i = (size_t)s * d_v + j;
            Tp[i] = std::fmaf(bk, e[j], T[i]);
        }
    }
    /* readout o = S'^T q */
    column_sum_in(plain, f, perm, q, Tp.data(), ot.data());
    for (int j = 0; j < d_v; ++j) o_out[j] = f->col_scales ? page->c[j] * ot[j] : ot[j];
    if (Tp_out) std::memcpy(Tp_out, Tp.data(), sizeof(float) * Tp.size());
    /* requantize in place; c is unchanged */
    for (int s = 0; s < d_k; ++s)
        requant_row(f, s, Tp.data() + (size_t)s * d_v, page, seed, step, b, h,
                    f->stochastic, margin_out ? margin_out + (size_t)s * d_v : nullptr);
    return 0;
}

extern "C" int orc_step_f32(const orc_format *f, orc_page *page, const int32_t *perm,
                            const float *q, const float *k, const float *v,
                            const float *alpha, float beta, float *o_out,
                            uint64_t seed, uint32_t step, uint32_t b, uint32_t h,
                            float *Tp_out, double *margin_out)
{
    return step_f32(0, f, page, perm, q, k, v, alpha, beta, o_out, seed, step, b, h, Tp_out, margin_out);
}

extern "C" int orc_step_f32_plain(const orc_format *f, orc_page *page, const int32_t *perm,
                                  const float *q, const float *k, const float *v,
                                  const float *alpha, float beta, float *o_out,
                                  uint64_t seed, uint32_t step, uint32_t b, uint32_t h,
                                  float *Tp_out, double *margin_out)
{
    return step_f32(1, f, page, perm, q, k, v, alpha, beta, o_out, seed, step, b, h, Tp_out, margin_out);
}

/* ------------------------------------------------------------------------ */
/* decode step: plain definition in fp64                                    */
/* ------------------------------------------------------------------------ */

/* ------------------------------------------------------------------------ */
/* per-window decode                                                        */
/* ------------------------------------------------------------------------ */

/* x . y over n channels (natural order) in the canonical order: lane l holds
 * the fma chain over channels 4l .. 4l+3 from +0; the n / 4 lane partials
 * (a power of two) are combined by an xor butterfly, offsets n/8 .. 1 */
static float lane_dot(const float *x, const float *y, int n)
{
    const int lanes = n / 4;
    std::vector<float> p(lanes), nx(lanes);
    for (int l = 0; l < lanes; ++l) {
        float acc = 0.0f;
        for (int i = 0; i < 4; ++i) acc = std::fmaf(x[4 * l + i], y[4 * l + i], acc);
        p[l] = acc;
    }
    for (int off = lanes / 2; off >= 1; off /= 2) {
        for (int l = 0; l < lanes; ++l) nx[l] = p[l] + p[l ^ off];
        p.swap(nx);
    }
    return p[0];
}

/* x . y over n channels as one fma chain in channel order, from +0 */
static float plain_dot(const float *x, const float *y, int n)
{
    float acc = 0.0f;
    for (int i = 0; i < n; ++i) acc = std::fmaf(x[i], y[i], acc);
    return acc;
}

static int window_step_f32(int plain, const orc_format *f, orc_page *page, const int32_t *perm,
                           float *P, float *K, float *D, int t, int commit,
                           const float *q, const float *k, const float *v,
                           const float *alpha, float beta, float *o_out,
                           uint64_t seed, uint32_t step, uint32_t b, uint32_t h,
                           double *margin_out)
{
    if (orc_format_check(f) != 0 || !page || !perm || !P || !K || !D || t < 0 || !q || !k || !v ||
        !alpha || !o_out)
        return -1;
    const int d_k = f->d_k, d_v = f->d_v;
    if (d_k % 4 != 0) return -1;
    std::vector<float> ic(d_v), Z((size_t)d_k * d_v), af(d_k), wk(d_k), wq(d_k), u(d_v), ot(d_v);
    for (int j = 0; j < d_v; ++j) ic[j] = f->col_scales ? 1.0f / page->c[j] : 1.0f;

    /* decay: the window's cumulative product and the earlier entries' keys */
    for (int kap = 0; kap < d_k; ++kap) {
        const float al = f->gate_vector ? alpha[kap] : alpha[0];
        const float p0 = (t == 0) ? 1.0f : P[kap];   /* a window starts from no decay */
        P[kap] = p0 * al;
        for (int tau = 0; tau < t; ++tau) K[(size_t)tau * d_k + kap] = K[(size_t)tau * d_k + kap] * al;
    }
    /* the fixed page as exact values Z (INT rows: z, FP16 rows: h) and one
     * factor per stored row, the window's decay times the row scale:
     * a'_s = P'_kappa r_s (FP16 rows: P'_kappa) */
    for (int s = 0; s < d_k; ++s) {
        const int kap = perm[s];
        const float rs = (orc_row_kind(f, s) == ORC_KIND_INT) ? page->r[s] : 1.0f;
        af[s] = P[kap] * rs;
        for (int j = 0; j < d_v; ++j) Z[(size_t)s * d_v + j] = element_value(f, page, s, j);
    }
    /* row weights by key channel: k a', q a' */
    for (int s = 0; s < d_k; ++s) {
        const int kap = perm[s];
        wk[kap] = k[kap] * af[s];
        wq[kap] = q[kap] * af[s];
    }
    /* prediction from the page and the earlier entries */
    column_sum_in(plain, f, perm, wk.data(), Z.data(), u.data());
    for (int tau = 0; tau < t; ++tau) {
        const float a = plain ? plain_dot(K + (size_t)tau * d_k, k, d_k) : lane_dot(K + (size_t)tau * d_k, k, d_k);
        for (int j = 0; j < d_v; ++j) u[j] = std::fmaf(a, D[(size_t)tau * d_v + j], u[j]);
    }
    /* this step's entry */
    for (int j = 0; j < d_v; ++j) {
        const float e = v[j] * ic[j] - u[j];
        D[(size_t)t * d_v + j] = beta * e;
    }
    for (int kap = 0; kap < d_k; ++kap) K[(size_t)t * d_k + kap] = k[kap];
    /* readout from the page and every entry */
    column_sum_in(plain, f, perm, wq.data(), Z.data(), ot.data());
    for (int tau = 0; tau <= t; ++tau) {
        const float bq = plain ? plain_dot(K + (size_t)tau * d_k, q, d_k) : lane_dot(K + (size_t)tau * d_k, q, d_k);
        for (int j = 0; j < d_v; ++j) ot[j] = std::fmaf(bq, D[(size_t)tau * d_v + j], ot[j]);
    }
    for (int j = 0; j < d_v; ++j) o_out[j] = f->col_scales ? page->c[j] * ot[j] : ot[j];

    if (commit) {
        /* T = Z a' + sum_tau K[tau] D[tau]^T, requantized once */
        std::vector<float> row(d_v);
        for (int s = 0; s < d_k; ++s) {
            const int kap = perm[s];
            for (int j = 0; j < d_v; ++j) {
                float x = Z[(size_t)s * d_v + j] * af[s];
                for (int tau = 0; tau <= t; ++tau)
                    x = std::fmaf(K[(size_t)tau * d_k + kap], D[(size_t)tau * d_v + j], x);
                row[j] = x;
            }
            requant_row(f, s, row.data(), page, seed, step, b, h, f->stochastic,
                        margin_out ? margin_out + (size_t)s * d_v : nullptr);
        }
        for (int kap = 0; kap < d_k; ++kap) P[kap] = 1.0f;
    }
    return 0;
}

extern "C" int orc_window_step_f32(const orc_format *f, orc_page *page, const int32_t *perm,
                                   float *P, float *K, float *D, int t, int commit,
                                   const float *q, const float *k, const float *v,
                                   const float *alpha, float beta, float *o_out,
                                   uint64_t seed, uint32_t step, uint32_t b, uint32_t h,
                                   double *margin_out)
{
    return window_step_f32(0, f, page, perm, P, K, D, t, commit, q, k, v, alpha, beta, o_out, seed, step, b, h,
                           margin_out);
}

extern "C" int orc_window_step_f32_plain(const orc_format *f, orc_page *page, const int32_t *perm,
                                         float *P, float *K, float *D, int t, int commit,
                                         const float *q, const float *k, const float *v,
                                         const float *alpha, float beta, float *o_out,
                                         uint64_t seed, uint32_t step, uint32_t b, uint32_t h,
                                         double *margin_out)
{
    return window_step_f32(1, f, page, perm, P, K, D, t, commit, q, k, v, alpha, beta, o_out, seed, step, b, h,
                           margin_out);
}


/* ------------------------------------------------------------------------ */
/* prefill: a prompt of L tokens through one page, one requantization       */
/* ------------------------------------------------------------------------ */

static int prefill_f32(int plain, const orc_format *f, orc_page *page, const int32_t *perm, int L,
                       const float *q, const float *k, const float *v,
                       const float *alpha, const float *beta, float *o_out,
                       uint64_t seed, uint32_t step, uint32_t b, uint32_t h,
                       float *Tp_out, double *margin_out)
{
    if (orc_format_check(f) != 0 || !page || !perm || L < 1 || !q || !k || !v || !alpha || !beta || !o_out)
        return -1;
    const int d_k = f->d_k, d_v = f->d_v;
    const int na = f->gate_vector ? d_k : 1;
    std::vector<float> ic(d_v), T((size_t)d_k * d_v), u(d_v), e(d_v), ot(d_v);
    for (int j = 0; j < d_v; ++j) ic[j] = f->col_scales ? 1.0f / page->c[j] : 1.0f;

    for (int l = 0; l < L; ++l) {
        const float *ql = q + (size_t)l * d_k, *kl = k + (size_t)l * d_k, *vl = v + (size_t)l * d_v;
        const float *al = alpha + (size_t)l * na;
        /* decay: the first token dequantizes the page with the gate folded
         * into the row scale, T = z (alpha r), as the decode step does; later
         * tokens decay the fp32 state in place, T = alpha T */
        for (int s = 0; s < d_k; ++s) {
            const float a_s = f->gate_vector ? al[perm[s]] : al[0];
            if (l == 0) {
                const float a = (orc_row_kind(f, s) == ORC_KIND_INT) ? a_s * page->r[s] : a_s;
                for (int j = 0; j < d_v; ++j) T[(size_t)s * d_v + j] = element_value(f, page, s, j) * a;
            } else {
                for (int j = 0; j < d_v; ++j) T[(size_t)s * d_v + j] = a_s * T[(size_t)s * d_v + j];
            }
        }
        /* the decode step's prediction, rank-1 update and readout */
        column_sum_in(plain, f, perm, kl, T.data(), u.data());
        for (int j = 0; j < d_v; ++j) e[j] = vl[j] * ic[j] - u[j];
        for (int s = 0; s < d_k; ++s) {
            const float bk = beta[l] * kl[perm[s]];
            for (int j = 0; j < d_v; ++j) {
                const size_t i = (size_t)s * d_v + j;
                T[i] = std::fmaf(bk, e[j], T[i]);
            }
        }
        column_sum_in(plain, f, perm, ql, T.data(), ot.data());
        for (int j = 0; j < d_v; ++j) o_out[(size_t)l * d_v + j] = f->col_scales ? page->c[j] * ot[j] : ot[j];
    }
    if (Tp_out) std::memcpy(Tp_out, T.data(), sizeof(float) * T.size());
    for (int s = 0; s < d_k; ++s)
        requant_row(f, s, T.data() + (size_t)s * d_v, page, seed, step, b, h, f->stochastic,
                    margin_out ? margin_out + (size_t)s * d_v : nullptr);
    return 0;
}

extern "C" int orc_prefill_f32(const orc_format *f, orc_page *page, const int32_t *perm, int L,
                               const float *q, const float *k, const float *v,
                               const float *alpha, const float *beta, float *o_out,
                               uint64_t seed, uint32_t step, uint32_t b, uint32_t h,
                               float *Tp_out, double *margin_out)
{
    return prefill_f32(0, f, page, perm, L, q, k, v, alpha, beta, o_out, seed, step, b, h, Tp_out, margin_out);
}

extern "C" int orc_prefill_f32_plain(const orc_format *f, orc_page *page, const int32_t *perm, int L,
                                     const float *q, const float *k, const float *v,
                                     const float *alpha, const float *beta, float *o_out,
                                     uint64_t seed, uint32_t step, uint32_t b, uint32_t h,
                                     float *Tp_out, double *margin_out)
{
    return prefill_f32(1, f, page, perm, L, q, k, v, alpha, beta, o_out, seed, step, b, h, Tp_out, margin_out);
}


/* ------------------------------------------------------------------------ */
/* prefill, chunkwise form (the chunk algebra in fp64)                      */
/* ------------------------------------------------------------------------ */

extern "C" int orc_prefill_chunked_f64(const orc_format *f, const orc_page *page, const int32_t *perm, int L, int C,
                                       const float *q, const float *k, const float *v,
                                       const float *alpha, const float *beta, double *o_out, double *Sp_out)
{
    if (orc_format_check(f) != 0 || !page || !perm || L < 1 || C < 1 || !q || !k || !v || !alpha || !beta || !o_out)
        return -1;
    const int d_k = f->d_k, d_v = f->d_v;
    const int na = f->gate_vector ? d_k : 1;
    /* the page's state in natural key order, in double */
    std::vector<double> S((size_t)d_k * d_v);
    for (int s = 0; s < d_k; ++s) {
        const double rs = (orc_row_kind(f, s) == ORC_KIND_INT) ? (double)page->r[s] : 1.0;
        for (int j = 0; j < d_v; ++j)
            S[(size_t)perm[s] * d_v + j] = (double)element_value(f, page, s, j) * rs
                                           * (f->col_scales ? (double)page->c[j] : 1.0);
    }
    for (int t0 = 0; t0 < L; t0 += C) {
        const int n = std::min(C, L - t0);
        /* cumulative decay of the chunk's tokens per key channel: gam[i][c] =
         * prod of the gates of tokens t0 .. t0 + i */
        auto gate = [&](int i, int c) {
            return (double)alpha[(size_t)(t0 + i) * na + (f->gate_vector ? c : 0)];
        };
        std::vector<double> gam((size_t)n * d_k);
        for (int i = 0; i < n; ++i)
            for (int c = 0; c < d_k; ++c)
                gam[(size_t)i * d_k + c] = (i == 0 ? 1.0 : gam[(size_t)(i - 1) * d_k + c]) * gate(i, c);
        /* the decay from token j to token i (j <= i), gam_i / gam_j, taken as
         * the product of the gates of tokens j + 1 .. i (1 for j = i): defined
         * where a gate is zero or the cumulative decay vanishes */
        std::vector<double> rho((size_t)n * n * d_k);
        auto R = [&](int i, int j, int c) -> double & { return rho[((size_t)i * n + j) * d_k + c]; };
        for (int i = 0; i < n; ++i)
            for (int c = 0; c < d_k; ++c) {
                R(i, i, c) = 1.0;
                for (int j = i - 1; j >= 0; --j) R(i, j, c) = R(i, j + 1, c) * gate(j + 1, c);
            }
        /* A[i][j] (j < i) = beta_i sum_c k_ic k_jc rho_ijc;
         * E = (I + A)^-1 R, R_i = beta_i (v_i - (gam_i k_i)^T S0), by forward
         * substitution: E_i = R_i - sum_{j<i} A_ij E_j */
        std::vector<double> E((size_t)n * d_v);
        for (int i = 0; i < n; ++i) {
            const float *ki = k + (size_t)(t0 + i) * d_k;
            const double bi = (double)beta[t0 + i];
            for (int j = 0; j < d_v; ++j) {
                double pred = 0.0;
                for (int c = 0; c < d_k; ++c) pred += gam[(size_t)i * d_k + c] * (double)ki[c] * S[(size_t)c * d_v + j];
                E[(size_t)i * d_v + j] = bi * ((double)v[(size_t)(t0 + i) * d_v + j] - pred);
            }
            for (int jt = 0; jt < i; ++jt) {
                const float *kj = k + (size_t)(t0 + jt) * d_k;
                double a = 0.0;
                for (int c = 0; c < d_k; ++c)
                    a += (double)ki[c] * (double)kj[c] * R(i, jt, c);
                a *= bi;
                for (int j = 0; j < d_v; ++j) E[(size_t)i * d_v + j] -= a * E[(size_t)jt * d_v + j];
            }
        }
        /* o_i = (gam_i q_i)^T S0 + sum_{j<=i} (sum_c q_ic k_jc rho_ijc) E_j */
        for (int i = 0; i < n; ++i) {
            const float *qi = q + (size_t)(t0 + i) * d_k;
            double *oi = o_out + (size_t)(t0 + i) * d_v;
            for (int j = 0; j < d_v; ++j) {
                double acc = 0.0;
                for (int c = 0; c < d_k; ++c) acc += gam[(size_t)i * d_k + c] * (double)qi[c] * S[(size_t)c * d_v + j];
                oi[j] = acc;
            }
            for (int jt = 0; jt <= i; ++jt) {
                const float *kj = k + (size_t)(t0 + jt) * d_k;
                double pw = 0.0;
                for (int c = 0; c < d_k; ++c)
                    pw += (double)qi[c] * (double)kj[c] * R(i, jt, c);
                for (int j = 0; j < d_v; ++j) oi[j] += pw * E[(size_t)jt * d_v + j];
            }
        }
        /* S <- diag(gam_n) S0 + sum_j (rho_nj k_j) E_j^T */
        for (int c = 0; c < d_k; ++c) {
            const double gn = gam[(size_t)(n - 1) * d_k + c];
            for (int j = 0; j < d_v; ++j) {
                double acc = gn * S[(size_t)c * d_v + j];
                for (int jt = 0; jt < n; ++jt)
                    acc += R(n - 1, jt, c) * (double)k[(size_t)(t0 + jt) * d_k + c]
                           * E[(size_t)jt * d_v + j];
                S[(size_t)c * d_v + j] = acc;
            }
        }
    }
    if (Sp_out) std::memcpy(Sp_out, S.data(), sizeof(double) * S.size());
    return 0;
}

/* ------------------------------------------------------------------------ */
/* lifetime weights from gate samples                                       */
/* ------------------------------------------------------------------------ */

extern "C" int orc_lifetime_weights(const orc_format *f, int B, int H, int n_samples, const float *alpha,
                                    float *row_weight)
{
    if (orc_format_check(f) != 0 || B < 1 || H < 1 || n_samples < 1 || !alpha || !row_weight) return -1;
    const int d_k = f->d_k;
    const int na = f->gate_vector ? d_k : 1;
    for (int h = 0; h < H; ++h) {
        for (int kap = 0; kap < d_k; ++kap) {
            /* the mean gate over the samples and requests, in double: one
             * sum from 0, samples in order, the requests of each in order */
            double sum = 0.0;
            for (int t = 0; t < n_samples; ++t)
                for (int b = 0; b < B; ++b)
                    sum += (double)alpha[(((size_t)t * B + b) * H + h) * na + (f->gate_vector ? kap : 0)];
            const double mean = sum / ((double)n_samples * (double)B);
            /* expected persistence under geometric decay: 1 / (1 - mean),
             * capped at 2^24 (a gate of one keeps its content for ever) */
            const double gap = 1.0 - mean;
            const double w = (gap <= 0x1p-24) ? 0x1p24 : 1.0 / gap;
            row_weight[(size_t)h * d_k + kap] = (float)w;
        }
    }
    return 0;
}

extern "C" int orc_step_f64(const orc_format *f, const orc_page *page, const int32_t *perm,
                            const float *q, const float *k, const float *v,
                            const float *alpha, float beta, double *o_out, double *Sp_out)
{
    if (orc_format_check(f) != 0 || !page || !perm || !q || !k || !v || !alpha || !o_out)
        return -1;
    const int d_k = f->d_k, d_v = f->d_v;
    std::vector<double> AS((size_t)d_k * d_v), Sp((size_t)d_k * d_v), pred(d_v);
    /* S in natural key order, in double, then A S */
    for (int s = 0; s < d_k; ++s) {
        int kap = perm[s];
        int kind = orc_row_kind(f, s);
        double rs = (kind == ORC_KIND_INT) ? (double)page->r[s] : 1.0;
        double al = f->gate_vector ? (double)alpha[kap] : (double)alpha[0];
        for (int j = 0; j < d_v; ++j) {
            double c = f->col_scales ? (double)page->c[j] : 1.0;
            double Sij = (double)element_value(f, page, s, j) * rs * c;
            AS[(size_t)kap * d_v + j] = al * Sij;
        }
    }
    for (int j = 0; j < d_v; ++j) {
        double acc = 0.0;
        for (int kap = 0; kap < d_k; ++kap) acc += (double)k[kap] * AS[(size_t)kap * d_v + j];
        pred[j] = acc;
    }
    for (int kap = 0; kap < d_k; ++kap)
        for (int j = 0; j < d_v; ++j)
            Sp[(size_t)kap * d_v + j] = AS[(size_t)kap * d_v + j]
                                        + (double)beta * (double)k[kap] * ((double)v[j] - pred[j]);
    for (int j = 0; j < d_v; ++j) {
        double acc = 0.0;
        for (int kap = 0; kap < d_k; ++kap) acc += (double)q[kap] * Sp[(size_t)kap * d_v + j];
        o_out[j] = acc;
    }
    if (Sp_out) std::memcpy(Sp_out, Sp.data(), sizeof(double) * Sp.size());
    return 0;
}

/* ------------------------------------------------------------------------ */
/* packed byte layout                                                       */
/* ------------------------------------------------------------------------ */
/*
 * A page is: the code region, then r (fp32, one per INT row, stored order),
 * then c (fp32 x 128) when the format has column scales.
 *
 * The code region is eight blocks of 16 stored rows in order.  A block is the
 * planes of its rows' codes, widest plane first (an INT code of b bits is
 * split into planes of widths given by the binary decomposition of b, the
 * widest plane holding the low bits; an FP16 row is one 16-bit plane).  INT
 * codes are stored biased: u = z + 2^(b-1).
 *
 * A plane of width w covers 16 rows x 128 columns in 256 w bytes.  Column
 * quad l (columns 4l .. 4l+3) owns 2w little-endian 32-bit words of it.  For
 * w <= 8, word n holds rows n*(8/w) + sigma, sigma = 0 .. 8/w - 1: column
 * 4l + beta sits in byte beta, bits [w sigma, w sigma + w).  For w = 16, word n
 * holds row n/2, columns 4l + 2(n%2) (low half) and 4l + 2(n%2) + 1 (high
 * half).  The words of one quad are grouped into chunks of 16 bytes (8 bytes
 * for w = 1), and chunk t of quad l sits at ((t * 32) + l) * chunk_bytes.
 */

static size_t lane_word_offset(int w, int lane, int n)
{
    int cw = (w == 1) ? 2 : 4;   /* words per chunk */
    return ((size_t)(n / cw) * 32 + lane) * (size_t)(4 * cw) + (size_t)(n % cw) * 4;
}

static uint32_t load_u32(const uint8_t *p)
{
    return (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
}

static void store_u32(uint8_t *p, uint32_t x)
{
    p[0] = (uint8_t)x; p[1] = (uint8_t)(x >> 8); p[2] = (uint8_t)(x >> 16); p[3] = (uint8_t)(x >> 24);
}

extern "C" int orc_pack_page(const orc_format *f, const orc_page *p, uint8_t *bytes)
{
    if (!packable(f) || !p || !bytes) return -1;
    size_t off = 0;
    for (int blk = 0; blk < 8; ++blk) {
        int s0 = 16 * blk;
        int g = group_of_row(f, s0);
        int kind = f->group_kind[g], bits = f->group_bits[g];
        int width[3], low[3];
        int np = planes_of(kind, bits, width, low);
        int bias = (kind == ORC_KIND_INT) ? (1 << (bits - 1)) : 0;
        for (int pl = 0; pl < np; ++pl) {
            int w = width[pl];
            uint8_t *plane = bytes + off;
            for (int lane = 0; lane < 32; ++lane) {
                for (int n = 0; n < 2 * w; ++n) {
                    uint32_t word = 0;
                    if (w == 16) {
                        int s = s0 + n / 2;
                        int j = 4 * lane + 2 * (n % 2);
                        uint32_t lo = (uint32_t)p->code[(size_t)s * 128 + j] & 0xFFFFu;
                        uint32_t hi = (uint32_t)p->code[(size_t)s * 128 + j + 1] & 0xFFFFu;
                        word = lo | (hi << 16);
                    } else {
                        int rows_per_word = 8 / w;
                        for (int sig = 0; sig < rows_per_word; ++sig) {
                            int s = s0 + n * rows_per_word + sig;
                            for (int beta = 0; beta < 4; ++beta) {
                                int j = 4 * lane + beta;
                                uint32_t u = (uint32_t)(p->code[(size_t)s * 128 + j] + bias);
                                uint32_t part = (u >> low[pl]) & ((1u << w) - 1u);
                                word |= part << (8 * beta + w * sig);
                            }
                        }
                    }
                    store_u32(plane + lane_word_offset(w, lane, n), word);
                }
            }
            off += 256 * (size_t)w;
        }
    }
    for (int s = 0; s < 128; ++s) {
        if (orc_row_kind(f, s) != ORC_KIND_INT) continue;
        store_u32(bytes + off, f32_to_bits(p->r[s]));
        off += 4;
    }
    if (f->col_scales) {
        for (int j = 0; j < 128; ++j) { store_u32(bytes + off, f32_to_bits(p->c[j])); off += 4; }
    }
    return 0;
}

extern "C" int orc_unpack_page(const orc_format *f, const uint8_t *bytes, orc_page *p)
{
    if (!packable(f) || !p || !bytes) return -1;
    size_t off = 0;
    for (int i = 0; i < 128 * 128; ++i) p->code[i] = 0;
    for (int blk = 0; blk < 8; ++blk) {
        int s0 = 16 * blk;
        int g = group_of_row(f, s0);
        int kind = f->group_kind[g], bits = f->group_bits[g];
        int width[3], low[3];
        int np = planes_of(kind, bits, width, low);
        for (int pl = 0; pl < np; ++pl) {
            int w = width[pl];
            const uint8_t *plane = bytes + off;
            for (int lane = 0; lane < 32; ++lane) {
                for (int n = 0; n < 2 * w; ++n) {
                    uint32_t word = load_u32(plane + lane_word_offset(w, lane, n));
                    if (w == 16) {
                        int s = s0 + n / 2;
                        int j = 4 * lane + 2 * (n % 2);
                        p->code[(size_t)s * 128 + j] = (int32_t)(word & 0xFFFFu);
                        p->code[(size_t)s * 128 + j + 1] = (int32_t)(word >> 16);
                    } else {
                        int rows_per_word = 8 / w;
                        for (int sig = 0; sig < rows_per_word; ++sig) {
                            int s = s0 + n * rows_per_word + sig;
                            for (int beta = 0; beta < 4; ++beta) {
                                int j = 4 * lane + beta;
                                uint32_t part = (word >> (8 * beta + w * sig)) & ((1u << w) - 1u);
                                p->code[(size_t)s * 128 + j] |= (int32_t)(part << low[pl]);
                            }
                        }
                    }
                }
            }
            off += 256 * (size_t)w;
        }
    }
    /* remove the bias from INT rows */
    for (int s = 0; s < 128; ++s) {
        if (orc_row_kind(f, s) != ORC_KIND_INT) continue;
        int bias = 1 << (f->group_bits[group_of_row(f, s)] - 1);
        for (int j = 0; j < 128; ++j) p->code[(size_t)s * 128 + j] -= bias;
    }
    for (int s = 0; s < 128; ++s) {
        if (orc_row_kind(f, s) != ORC_KIND_INT) { p->r[s] = 0.0f; continue; }
        p->r[s] = bits_to_f32(load_u32(bytes + off));
        off += 4;
    }
    for (int j = 0; j < 128; ++j) {
        if (f->col_scales) { p->c[j] = bits_to_f32(load_u32(bytes + off)); off += 4; }
        else p->c[j] = 1.0f;
    }
    return 0;
}

static int decode_step_pages(int plain, const orc_format *f, int B, int H, uint8_t *pages,
                             const int32_t *perm, const float *q, const float *k,
                             const float *v, const float *alpha, const float *beta,
                             float *o, uint64_t seed, uint32_t step,
                             long page_begin, long page_end)
{
    if (!packable(f) || B < 1 || H < 1 || !pages || !perm) return -1;
    long pb = orc_page_bytes(f);
    long n_pages = (long)B * H;
    if (page_begin < 0 || page_end > n_pages || page_begin > page_end) return -2;
    std::vector<int32_t> code(128 * 128);
    std::vector<float> r(128), c(128);
    orc_page pg = { code.data(), r.data(), c.data() };
    for (long pi = page_begin; pi < page_end; ++pi) {
        uint32_t b = (uint32_t)(pi / H), h = (uint32_t)(pi % H);
        uint8_t *bytes = pages + (size_t)pi * pb;
        orc_unpack_page(f, bytes, &pg);
        const float *al = f->gate_vector ? alpha + (size_t)pi * 128 : alpha + pi;
        step_f32(plain, f, &pg, perm + (size_t)h * 128, q + (size_t)pi * 128, k + (size_t)pi * 128,
                 v + (size_t)pi * 128, al, beta[pi], o + (size_t)pi * 128,
                 seed, step, b, h, nullptr, nullptr);
        orc_pack_page(f, &pg, bytes);
    }
    return 0;
}

extern "C" int orc_decode_step_pages(const orc_format *f, int B, int H, uint8_t *pages,
                                     const int32_t *perm, const float *q, const float *k,
                                     const float *v, const float *alpha, const float *beta,
                                     float *o, uint64_t seed, uint32_t step,
                                     long page_begin, long page_end)
{
    return decode_step_pages(0, f, B, H, pages, perm, q, k, v, alpha, beta, o, seed, step, page_begin, page_end);
}

extern "C" int orc_decode_step_pages_plain(const orc_format *f, int B, int H, uint8_t *pages,
                                           const int32_t *perm, const float *q, const float *k,
                                           const float *v, const float *alpha, const float *beta,
                                           float *o, uint64_t seed, uint32_t step,
                                           long page_begin, long page_end)
{
    return decode_step_pages(1, f, B, H, pages, perm, q, k, v, alpha, beta, o, seed, step, page_begin, page_end);
}
