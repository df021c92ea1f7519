/*
 * stq_oracle.c -- CPU oracle for the quantized gated delta-rule decode step.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  The product path
 * (the CUDA library and its Python binding) never calls it, and the two
 * share no code: this file has its own packer, unpacker, quantizer and
 * recurrence, written from the method's definition, deliberately plain and
 * slow (bit-by-bit packing, scalar loops, no blocking, no reordering).
 *
 * Source of every formula: the page "STEPQuant: When and Where Errors Matter
 * in Delta-Rule Recurrent State Quantization" (paper.rainbus.top/paper/
 * 2609.38169), cited below by its section names:
 *   [bg-state]  background, "linear attention and recurrent state":
 *               y_t = S_t^T q_t, S in R^{dk x dv}.
 *   [bg-delta]  background, "gated delta rule":
 *               S_t = (I - b_t k_t k_t^T) D_t S_{t-1} + b_t k_t v_t^T,
 *               D_t = alpha_t I (GDN) or a per-channel diagonal (KDA).
 *   [bg-quant]  background, "PTQ and symmetric uniform quantisation":
 *               Q_{b,s}(x) = s clip(round(x / s), -q_b, q_b), q_b = 2^(b-1) - 1.
 *   [bg-smooth] background, "smoothing": absmax quantisation, row factor r_i,
 *               column factor c_j.
 *   [core]      core method: reconstruction  X^_ij = r_i c_j z_ij.
 *   [steps]     method steps, online decode (the paper's Table C2):
 *               step 1 reconstruct S^_{t-1} from integer codes and scales;
 *               step 2 X_t = D_t S^ + b_t k_t (v_t^T - k_t^T D_t S^);
 *               step 3 emit y_t = X_t^T q_t before requantisation;
 *               steps 4-6 scale, quantise, pack the codes and scales back.
 *
 * Readings taken where the page is silent (each listed in the design notes):
 *   - one quantisation group per key row: s_i = a_i / q_b with
 *     a_i = max_j |X_ij / (r_i c_j)| (absmax; the row factor and column
 *     factor are frozen per-head tables);
 *   - round() is IEEE round-half-to-even; the code -2^(b-1) is never made;
 *   - scales are stored as fp32 (format 0); format 1 stores them as IEEE
 *     binary16, s16 = half(a_i / q_b) rounded to nearest even, and the codes
 *     are then rounded from mu_ij / s16 so that s16 z reconstructs them; a
 *     scale above the binary16 range is reported like a non-finite row;
 *   - raw units (the page's FP16 storage applied to a whole pool, and the
 *     fp32 control state): every row of the unit is 16 or 32 bits wide and
 *     holds the state value itself in IEEE binary16 / binary32, with no scale
 *     and no r, c factors; the step is the same recurrence, and X is rounded
 *     once (to nearest even) on store;
 *   - FP16 pivots ([steps] step 1: "pivot units are read in FP16 directly";
 *     format flag 4, a pool that mixes pivots with quantized units): a
 *     16-bit row keeps its scale slot, which holds 1, and stores
 *     mu_ij = fl32(X_ij / (r_i c_j)) rounded once to binary16 in place of
 *     the codes; it reconstructs as s_i r_i c_j mu_ij like a quantized row
 *     (with r = c = 1, the state value itself);
 *   - online column fit ([core]: c_j minimises sum_{i,j} w_i^2 (X_ij -
 *     r_i c_j z_ij)^2; [steps] steps 4-5, closed form c_j = sum_i w_i^2
 *     v_ij X_ij / sum_i w_i^2 v_ij^2 with the page's garbled v_ij read as the
 *     row's reconstruction without c, r_i s_i z_ij; format flag 8): the page
 *     carries its own dv fp32 column factors after the scales.  Each
 *     quantisation takes the codes with the page's current factors (one pass,
 *     no iteration between codes and factors), then refits every column over
 *     the unit's rows with the frozen row weights w_i and stores the new
 *     factors; a column whose codes are all zero keeps its factor.  With one
 *     absmax scale per row, r_i cancels from codes and reconstruction alike,
 *     so the row factor's online formula r_i = m_i^(1/2) w_i^(-1/2) changes
 *     nothing here and is not evaluated;
 *   - pivot rows in a fitted unit ([core]: c_j is fitted "across non-pivot
 *     rows"): the fit sums run over the non-pivot rows only, and a pivot row
 *     stores mu_ij = fl32(X_ij / r_i) without the column factor (its value
 *     must not move when the factors are refitted), reconstructing as
 *     s_i r_i mu_ij with s_i = 1;
 *   - the continuous part (reconstruction, decay, retrieval, write,
 *     readout) is computed in fp64; the quantisation decision is taken in
 *     fp32 on the fp32-rounded value mu_ij = fl32(X_ij / (r_i c_j)), with
 *     IEEE fp32 division for s_i = a_i / q_b and for mu_ij / s_i;
 *   - an all-zero row has s_i = 0 and all codes 0.
 *
 * Packed page of one (request, slot, head) unit, dk rows of dv codes:
 *   bytes [0, 4 dk)        fp32 scales s_0 .. s_{dk-1} (little-endian);
 *                          [0, 2 dk) binary16 scales in format 1; no scale
 *                          section in a raw unit
 *   then row i = 0..dk-1   dv codes of b_i bits each, dv * b_i / 8 bytes, as
 *                          b_i-bit two's complement values in the row's
 *                          little-endian bit string (bit p is bit p%8 of byte
 *                          p/8): 4- and 8-bit code j at bits [j b, (j + 1) b);
 *                          6-bit codes in groups of eight, group g (codes
 *                          8g .. 8g+7) a 48-bit string whose bits [0, 32) are
 *                          the 32-bit word at bits [32 g, 32 g + 32) and whose
 *                          bits [32, 48) are the 16-bit half at bits
 *                          [32 G + 16 g, 32 G + 16 g + 16), G = dv / 8; code
 *                          8g + p at bits [6p, 6p + 6) of its group
 *   padding up to a multiple of 128 bytes.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_NONFINITE 1
#define ORC_BADARG 2

static int q_of_bits(int b) { return (1 << (b - 1)) - 1; }

static size_t row_bytes(int dv, int b) { return (size_t)dv * (size_t)b / 8u; }

/* format flags: bit 0 binary16 scales, bit 2 FP16 pivot rows among quantized ones,
 * bit 3 per-page column factors fitted at every quantisation */
#define ORC_FMT_F16 1
#define ORC_FMT_PIVOT 4
#define ORC_FMT_FITC 8

static int fmt_ok(int fmt)
{
    return fmt >= 0 && (fmt & ~(ORC_FMT_F16 | ORC_FMT_PIVOT | ORC_FMT_FITC)) == 0;
}

/* 16 or 32 for a raw unit (its first row decides; bits_ok checks the rest), else 0 */
static int raw_width(int dk, const uint8_t *bits, int fmt)
{
    if (dk <= 0 || (fmt & ORC_FMT_PIVOT)) return 0;
    return (bits[0] == 16 || bits[0] == 32) ? bits[0] : 0;
}

/* quantized rows are 4, 6 or 8 bits (or 16, pivots, under ORC_FMT_PIVOT); a raw
 * unit has all rows at 16 or at 32 */
static int bits_ok(int dk, int dv, const uint8_t *bits, int fmt)
{
    if (!fmt_ok(fmt)) return 0;
    int raw = raw_width(dk, bits, fmt);
    for (int i = 0; i < dk; ++i) {
        int b = bits[i];
        if (raw) {
            if (b != raw) return 0;
        } else if (b != 4 && b != 6 && b != 8 && !(b == 16 && (fmt & ORC_FMT_PIVOT))) {
            return 0;
        }
        if ((dv * b) % 8 != 0 || (b == 6 && dv % 8 != 0)) return 0;
    }
    return 1;
}

/* bytes per scale: fp32, or binary16 with ORC_FMT_F16; a raw unit has none */
static size_t scale_bytes(int dk, const uint8_t *bits, int fmt)
{
    if (raw_width(dk, bits, fmt)) return 0;
    return (fmt & ORC_FMT_F16) ? 2u : 4u;
}

/* bytes of the column-factor section (fp32, after the scales) */
static size_t colf_bytes(int dv, int fmt) { return (fmt & ORC_FMT_FITC) ? 4u * (size_t)dv : 0u; }

size_t orc_page_bytes_fmt(int dk, int dv, const uint8_t *bits, int fmt)
{
    size_t n = scale_bytes(dk, bits, fmt) * (size_t)dk + colf_bytes(dv, fmt);
    for (int i = 0; i < dk; ++i) n += row_bytes(dv, bits[i]);
    return (n + 127u) / 128u * 128u;
}

size_t orc_page_bytes(int dk, int dv, const uint8_t *bits) { return orc_page_bytes_fmt(dk, dv, bits, 0); }

static size_t row_offset(int dk, int dv, const uint8_t *bits, int fmt, int i)
{
    size_t n = scale_bytes(dk, bits, fmt) * (size_t)dk + colf_bytes(dv, fmt);
    for (int t = 0; t < i; ++t) n += row_bytes(dv, bits[t]);
    return n;
}

/*
 * IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction
 * bits; exponent 0 holds zero and the subnormals f 2^-24, exponent 31 the
 * infinities and NaNs.
 */
double orc_half_to_double(uint16_t h)
{
    int sign = h >> 15, e = (h >> 10) & 31, f = h & 1023;
    double v;
    if (e == 0) v = ldexp((double)f, -24);
    else if (e == 31) v = f ? NAN : INFINITY;
    else v = ldexp((double)(1024 + f), e - 25);
    return sign ? -v : v;
}

/* x rounded once to the nearest binary16, ties to even (rint under the default rounding mode) */
uint16_t orc_double_to_half(double x)
{
    if (isnan(x)) return 0x7E00u;
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    double a = fabs(x);
    if (a < ldexp(1.0, -14)) {
        /* subnormal range: a multiple of 2^-24; 1024 units carry into the smallest normal */
        double n = rint(ldexp(a, 24));
        return (uint16_t)(sign | (uint16_t)n);
    }
    int e;
    double m = frexp(a, &e); /* a = m 2^e, m in [0.5, 1) */
    double t = rint(ldexp(m, 11)); /* 11 significant bits, in [1024, 2048] */
    if (t == 2048.0) {
        t = 1024.0;
        e += 1;
    }
    int be = e - 1 + 15; /* biased exponent of t 2^(e - 11) = (t / 1024) 2^(e - 1) */
    if (be >= 31) return (uint16_t)(sign | 0x7C00u);
    return (uint16_t)(sign | (uint16_t)(be << 10) | (uint16_t)((int)t - 1024));
}

/* bit index in a row of dv codes of bit t of code j (see the page format above) */
static int code_bit(int b, int dv, int j, int t)
{
    if (b != 6) return j * b + t;
    int g = j / 8, q = 6 * (j % 8) + t; /* bit q of group g's 48-bit string */
    return q < 32 ? 32 * g + q : 32 * (dv / 8) + 16 * g + (q - 32);
}

/* code j of a packed row of dv codes, read one bit at a time, then sign-extended */
static int32_t get_code(const uint8_t *row, int b, int dv, int j)
{
    uint32_t u = 0;
    for (int t = 0; t < b; ++t) {
        int p = code_bit(b, dv, j, t);
        u |= (uint32_t)((row[p / 8] >> (p % 8)) & 1u) << t;
    }
    if (u & (1u << (b - 1))) return (int32_t)u - (int32_t)(1u << b);
    return (int32_t)u;
}

static void put_code(uint8_t *row, int b, int dv, int j, int32_t z)
{
    uint32_t u = (uint32_t)z & ((1u << b) - 1u);
    for (int t = 0; t < b; ++t) {
        int p = code_bit(b, dv, j, t);
        if ((u >> t) & 1u) row[p / 8] = (uint8_t)(row[p / 8] | (1u << (p % 8)));
        else row[p / 8] = (uint8_t)(row[p / 8] & ~(1u << (p % 8)));
    }
}

static float get_scale(const uint8_t *page, int fmt, int i)
{
    if (fmt & ORC_FMT_F16) {
        uint16_t h;
        memcpy(&h, page + 2 * (size_t)i, 2);
        return (float)orc_half_to_double(h);
    }
    float s;
    memcpy(&s, page + 4 * (size_t)i, 4);
    return s;
}

/* stores s (format 0) or half(s) (format 1); returns the value stored, as a float */
static float put_scale(uint8_t *page, int fmt, int i, float s)
{
    if (fmt & ORC_FMT_F16) {
        uint16_t h = orc_double_to_half((double)s);
        memcpy(page + 2 * (size_t)i, &h, 2);
        return (float)orc_half_to_double(h);
    }
    memcpy(page + 4 * (size_t)i, &s, 4);
    return s;
}

/* element j of a raw row of width b (16 or 32) */
static double get_raw(const uint8_t *row, int b, int j)
{
    if (b == 16) {
        uint16_t h;
        memcpy(&h, row + 2 * (size_t)j, 2);
        return orc_half_to_double(h);
    }
    float f;
    memcpy(&f, row + 4 * (size_t)j, 4);
    return (double)f;
}

/* stores x rounded once to the row's format; returns the stored value */
static double put_raw(uint8_t *row, int b, int j, double x)
{
    if (b == 16) {
        uint16_t h = orc_double_to_half(x);
        memcpy(row + 2 * (size_t)j, &h, 2);
        return orc_half_to_double(h);
    }
    float f = (float)x;
    memcpy(row + 4 * (size_t)j, &f, 4);
    return (double)f;
}

/* column factor j of a unit: the page's own under ORC_FMT_FITC, else the frozen table */
static float col_factor(const uint8_t *page, int dk, const uint8_t *bits, int fmt, const float *c, int j)
{
    if (!(fmt & ORC_FMT_FITC)) return c[j];
    float f;
    memcpy(&f, page + scale_bytes(dk, bits, fmt) * (size_t)dk + 4 * (size_t)j, 4);
    return f;
}

static void put_col_factor(uint8_t *page, int dk, const uint8_t *bits, int fmt, int j, float f)
{
    memcpy(page + scale_bytes(dk, bits, fmt) * (size_t)dk + 4 * (size_t)j, &f, 4);
}

/* exported for the pack/unpack pins */
int32_t orc_get_code(const uint8_t *row, int b, int dv, int j) { return get_code(row, b, dv, j); }
void orc_put_code(uint8_t *row, int b, int dv, int j, int32_t z) { put_code(row, b, dv, j, z); }

/* [steps] step 1, [core]: S^_ij = s_i r_i c_j z_ij, in fp64 (a raw unit: the stored
 * value; a pivot row: z_ij is its binary16 value) */
static void reconstruct(int dk, int dv, const uint8_t *bits, const float *r, const float *c,
                        int fmt, const uint8_t *page, double *S)
{
    int raw = raw_width(dk, bits, fmt);
    for (int i = 0; i < dk; ++i) {
        const uint8_t *row = page + row_offset(dk, dv, bits, fmt, i);
        if (raw) {
            for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] = get_raw(row, raw, j);
            continue;
        }
        double s = (double)get_scale(page, fmt, i);
        int pivot_fit = bits[i] == 16 && (fmt & ORC_FMT_FITC);
        for (int j = 0; j < dv; ++j) {
            double z = bits[i] == 16 ? get_raw(row, 16, j) : (double)get_code(row, bits[i], dv, j);
            double cj = pivot_fit ? 1.0 : (double)col_factor(page, dk, bits, fmt, c, j);
            S[(size_t)i * dv + j] = s * (double)r[i] * cj * z;
        }
    }
}

/*
 * [core], [steps] steps 4-5: the weighted least-squares column factors of the
 * codes just written, c_j = sum_i w_i^2 v_ij X_ij / sum_i w_i^2 v_ij^2 with
 * v_ij = s_i r_i z_ij, in fp64, stored as fp32 (a column whose codes are all
 * zero keeps c_old).  Returns ORC_NONFINITE if a factor is not finite.
 */
static int fit_columns(int dk, int dv, const uint8_t *bits, const float *r, const float *c_old,
                       const float *w, int fmt, const double *X, uint8_t *page)
{
    int status = ORC_OK;
    for (int j = 0; j < dv; ++j) {
        double num = 0.0, den = 0.0;
        for (int i = 0; i < dk; ++i) {
            if (bits[i] == 16) continue; /* pivot rows are not part of the fit */
            const uint8_t *row = page + row_offset(dk, dv, bits, fmt, i);
            double v = (double)get_scale(page, fmt, i) * (double)r[i] * (double)get_code(row, bits[i], dv, j);
            double wi = w ? (double)w[i] : 1.0;
            num += wi * wi * v * X[(size_t)i * dv + j];
            den += wi * wi * v * v;
        }
        float cj = den > 0.0 ? (float)(num / den) : c_old[j];
        if (!isfinite(cj)) status = ORC_NONFINITE;
        put_col_factor(page, dk, bits, fmt, j, cj);
    }
    return status;
}

/*
 * [bg-quant], [bg-smooth], [core], [steps] steps 4-6: quantise X row by row
 * and write scales and codes into page.  quot (optional) receives the fp32
 * quotient mu_ij / s_i that round() is applied to (for near-tie analysis).
 * c holds the column factors the codes are taken with (the unit's current
 * ones); under ORC_FMT_FITC the page then receives refitted factors (row
 * weights w, NULL for 1).  Returns ORC_NONFINITE if a row maximum is not finite.
 */
static int requantize(int dk, int dv, const uint8_t *bits, const float *r, const float *c,
                      const float *w, int fmt, const double *X, uint8_t *page, float *quot)
{
    int status = ORC_OK;
    int raw = raw_width(dk, bits, fmt);
    if (raw) {
        /* raw unit: X rounded once to the row format; quot receives fl32(X) */
        for (int i = 0; i < dk; ++i) {
            uint8_t *row = page + row_offset(dk, dv, bits, fmt, i);
            for (int j = 0; j < dv; ++j) {
                double x = X[(size_t)i * dv + j];
                double st = put_raw(row, raw, j, x);
                if (!isfinite(st)) status = ORC_NONFINITE;
                if (quot) quot[(size_t)i * dv + j] = (float)x;
            }
        }
        return status;
    }
    float *mu = (float *)malloc(sizeof(float) * (size_t)dv);
    for (int i = 0; i < dk; ++i) {
        if (bits[i] == 16) {
            /* pivot row: scale slot 1, mu rounded once to binary16 (in a fitted unit without
             * the column factor); quot receives mu */
            uint8_t *row = page + row_offset(dk, dv, bits, fmt, i);
            put_scale(page, fmt, i, 1.0f);
            for (int j = 0; j < dv; ++j) {
                double rc = (fmt & ORC_FMT_FITC) ? (double)r[i] : (double)r[i] * (double)c[j];
                float m = (float)(X[(size_t)i * dv + j] / rc);
                double st = put_raw(row, 16, j, (double)m);
                if (!isfinite(st)) status = ORC_NONFINITE;
                if (quot) quot[(size_t)i * dv + j] = m;
            }
            continue;
        }
        int qb = q_of_bits(bits[i]);
        float a = 0.0f;
        for (int j = 0; j < dv; ++j) {
            double rc = (double)r[i] * (double)c[j];
            mu[j] = (float)(X[(size_t)i * dv + j] / rc);
            float m = fabsf(mu[j]);
            if (!(m <= a)) a = m; /* also propagates NaN */
        }
        if (!isfinite(a)) status = ORC_NONFINITE;
        float s = put_scale(page, fmt, i, a / (float)qb); /* the scale as stored */
        if (!isfinite(s)) status = ORC_NONFINITE; /* also a binary16 overflow */
        uint8_t *row = page + row_offset(dk, dv, bits, fmt, i);
        for (int j = 0; j < dv; ++j) {
            int32_t z = 0;
            float x = 0.0f;
            if (s > 0.0f && isfinite(s)) {
                x = mu[j] / s;
                float rz = rintf(x);
                if (rz > (float)qb) rz = (float)qb;
                if (rz < (float)-qb) rz = (float)-qb;
                z = (int32_t)rz;
            }
            if (quot) quot[(size_t)i * dv + j] = x;
            put_code(row, bits[i], dv, j, z);
        }
    }
    free(mu);
    if ((fmt & ORC_FMT_FITC) && fit_columns(dk, dv, bits, r, c, w, fmt, X, page) != ORC_OK) status = ORC_NONFINITE;
    return status;
}

/* fp32 state -> packed page (the quantizer applied to a given state; under
 * ORC_FMT_FITC the codes are taken with the table's factors c and the page
 * receives the refitted ones) */
int orc_quantize_unit_w(int dk, int dv, const uint8_t *bits, const float *r, const float *c,
                        const float *w, int fmt, const float *S, uint8_t *page, float *quot)
{
    if (!bits_ok(dk, dv, bits, fmt)) return ORC_BADARG;
    size_t nb = orc_page_bytes_fmt(dk, dv, bits, fmt);
    memset(page, 0, nb);
    double *X = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    for (size_t e = 0; e < (size_t)dk * dv; ++e) X[e] = (double)S[e];
    int st = requantize(dk, dv, bits, r, c, w, fmt, X, page, quot);
    free(X);
    return st;
}

int orc_quantize_unit_fmt(int dk, int dv, const uint8_t *bits, const float *r, const float *c,
                          int fmt, const float *S, uint8_t *page, float *quot)
{
    return orc_quantize_unit_w(dk, dv, bits, r, c, NULL, fmt, S, page, quot);
}

int orc_quantize_unit(int dk, int dv, const uint8_t *bits, const float *r, const float *c,
                      const float *S, uint8_t *page, float *quot)
{
    return orc_quantize_unit_fmt(dk, dv, bits, r, c, 0, S, page, quot);
}

/* packed page -> fp32 reconstruction fl32(s_i r_i c_j z_ij) (a raw unit: its values) */
int orc_dequantize_unit_fmt(int dk, int dv, const uint8_t *bits, const float *r, const float *c,
                            int fmt, const uint8_t *page, float *S)
{
    if (!bits_ok(dk, dv, bits, fmt)) return ORC_BADARG;
    double *X = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    reconstruct(dk, dv, bits, r, c, fmt, page, X);
    for (size_t e = 0; e < (size_t)dk * dv; ++e) S[e] = (float)X[e];
    free(X);
    return ORC_OK;
}

int orc_dequantize_unit(int dk, int dv, const uint8_t *bits, const float *r, const float *c,
                        const uint8_t *page, float *S)
{
    return orc_dequantize_unit_fmt(dk, dv, bits, r, c, 0, page, S);
}

/*
 * One quantized decode step of one unit ([steps] steps 1-6):
 *   S^  = reconstruct(page_in)
 *   P   = D S^,            D = diag(g)          ([bg-delta], [steps] step 2)
 *   vo  = P^T k                                 (retrieval)
 *   u   = beta (v - vo)
 *   X   = P + k u^T                             (delta write)
 *   y   = X^T q                                 ([steps] step 3, before requant)
 *   page_out = requantize(X)
 * y is returned in fp64; quot (optional, dk*dv floats) receives the fp32
 * quotients the new codes were rounded from.
 */
int orc_step_unit_w(int dk, int dv, const uint8_t *bits, const float *r, const float *c,
                    const float *w, int fmt, const uint8_t *page_in, uint8_t *page_out,
                    const float *q, const float *k, const float *v, float beta, const float *g,
                    double *y, float *quot)
{
    if (!bits_ok(dk, dv, bits, fmt)) return ORC_BADARG;
    size_t nel = (size_t)dk * dv;
    double *P = (double *)malloc(sizeof(double) * nel);
    double *vo = (double *)malloc(sizeof(double) * (size_t)dv);
    double *u = (double *)malloc(sizeof(double) * (size_t)dv);
    reconstruct(dk, dv, bits, r, c, fmt, page_in, P);
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) P[(size_t)i * dv + j] *= (double)g[i];
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += (double)k[i] * P[(size_t)i * dv + j];
        vo[j] = acc;
        u[j] = (double)beta * ((double)v[j] - acc);
    }
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) P[(size_t)i * dv + j] += (double)k[i] * u[j]; /* P is now X */
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += (double)q[i] * P[(size_t)i * dv + j];
        y[j] = acc;
    }
    /* the codes are taken with the unit's current column factors */
    float *c_now = (float *)calloc((size_t)dv, sizeof(float));
    for (int j = 0; j < dv; ++j) c_now[j] = col_factor(page_in, dk, bits, fmt, c, j);
    memset(page_out, 0, orc_page_bytes_fmt(dk, dv, bits, fmt));
    int st = requantize(dk, dv, bits, r, c_now, w, fmt, P, page_out, quot);
    free(c_now);
    for (int j = 0; j < dv; ++j)
        if (!isfinite(y[j])) st = ORC_NONFINITE;
    free(P);
    free(vo);
    free(u);
    return st;
}

int orc_step_unit_fmt(int dk, int dv, const uint8_t *bits, const float *r, const float *c,
                      int fmt, const uint8_t *page_in, uint8_t *page_out,
                      const float *q, const float *k, const float *v, float beta, const float *g,
                      double *y, float *quot)
{
    return orc_step_unit_w(dk, dv, bits, r, c, NULL, fmt, page_in, page_out, q, k, v, beta, g, y, quot);
}

int orc_step_unit(int dk, int dv, const uint8_t *bits, const float *r, const float *c,
                  const uint8_t *page_in, uint8_t *page_out,
                  const float *q, const float *k, const float *v, float beta, const float *g,
                  double *y, float *quot)
{
    return orc_step_unit_fmt(dk, dv, bits, r, c, 0, page_in, page_out, q, k, v, beta, g, y, quot);
}

/*
 * The same recurrence with quantisation off, state kept in fp64 (in place):
 *   X = D S + k (beta (v - (D S)^T k))^T,  y = X^T q,  S <- X.
 */
int orc_step_unit_f64(int dk, int dv, double *S, const float *q, const float *k,
                      const float *v, float beta, const float *g, double *y)
{
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= (double)g[i];
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += (double)k[i] * S[(size_t)i * dv + j];
        double uj = (double)beta * ((double)v[j] - acc);
        for (int i = 0; i < dk; ++i) S[(size_t)i * dv + j] += (double)k[i] * uj;
    }
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += (double)q[i] * S[(size_t)i * dv + j];
        y[j] = acc;
    }
    return ORC_OK;
}

/*
 * Many independent units at once (the CPU baseline): unit n uses head
 * head[n] of the per-head tables bits [H][dk], r [H][dk], c [H][dv];
 * its input page starts at pages_in + off_in[n], its output page at
 * pages_out + off_out[n].  q, k, v, g: [n][128]; beta: [n]; y: [n][dv].
 * Units are spread over nthreads OpenMP threads (<= 0: the runtime default).
 * Returns the number of units that reported a non-finite value.
 */
int orc_step_many(int n, int dk, int dv, const int32_t *head, const uint8_t *bits,
                  const float *r, const float *c, const uint8_t *pages_in, const int64_t *off_in,
                  uint8_t *pages_out, const int64_t *off_out, const float *q, const float *k,
                  const float *v, const float *beta, const float *g, double *y, int nthreads)
{
    int bad = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#else
    nthreads = 1;
#endif
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : bad) num_threads(nthreads)
    for (int u = 0; u < n; ++u) {
        int h = head[u];
        int st = orc_step_unit(dk, dv, bits + (size_t)h * dk, r + (size_t)h * dk,
                               c + (size_t)h * dv, pages_in + off_in[u], pages_out + off_out[u],
                               q + (size_t)u * dk, k + (size_t)u * dk, v + (size_t)u * dv, beta[u],
                               g + (size_t)u * dk, y + (size_t)u * dv, NULL);
        if (st != ORC_OK) bad += 1;
    }
    return bad;
}

/* the number of OpenMP threads orc_step_many uses when nthreads <= 0 */
int orc_default_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
