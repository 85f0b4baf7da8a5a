/*
 * w4a4_oracle.c -- plain, slow CPU oracle for the pure W4A4 group-quantized GEMM.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test suite, the smoke check of
 * __graft_entry__.py and the cpu_baseline leg of bench.py may load or call this file.
 * It shares no code, header, table or constant with the CUDA library, and the CUDA
 * library never calls it.
 *
 * What it computes (source: "APEX4: Efficient Pure W4A4 LLM Inference via Intra-SM
 * Compute Rebalancing", abstract -- a W4A4 kernel with 128-wide K-groups on both
 * operands, INT4 products dequantised per group; the quantizer details are the plainest
 * reading of that statement, listed below):
 *
 *   quantize (per row r, per K-group g of width `group`):
 *     absmax = max |x[r,k]| over the group                      (exact, inputs are fp16)
 *     s      = fp16_rne( fp32(absmax) / 7.0f )                  (IEEE fp32 division)
 *     q[r,k] = clamp( round_half_even( fp32(x) / fp32(s) ), -8, 7 ),  q = 0 when s == 0
 *   pack: byte j of a row holds k = 2j in bits 0..3 and k = 2j+1 in bits 4..7
 *         (two's-complement nibbles)
 *   group partials (effective group ge = min(ga, gw)):
 *     P[g][m][n] = sum_{k in group g} qa[m,k] * qw[n,k]         (int64)
 *   output:
 *     Y[m][n] = sum_g P[g][m][n] * sa[m, g*ge/ga] * sw[n, g*ge/gw]   (fp64, g ascending)
 *
 * Every function is a direct transcription of one of the lines above; there is no
 * blocking, fusion or reordering beyond the row loop that OpenMP splits across cores.
 * The fp16 <-> fp32 conversions are written by hand (no compiler half type), so the
 * pins in the test suite can check them against numpy's float16.
 */
#include <stdint.h>
#include <string.h>
#include <math.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- fp16 helpers */

/* fp32 -> fp16, round to nearest, ties to even; subnormals kept, overflow -> inf. */
uint16_t w4o_f32_to_f16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    uint32_t sign = (u >> 16) & 0x8000u;
    uint32_t a = u & 0x7FFFFFFFu;
    if (a >= 0x7F800000u)                      /* inf or nan */
        return (uint16_t)(sign | 0x7C00u | (a > 0x7F800000u ? 0x200u : 0u));
    if (a >= 0x477FF000u)                      /* >= 65520 rounds to inf */
        return (uint16_t)(sign | 0x7C00u);
    if (a < 0x38800000u) {                     /* below 2^-14: fp16 subnormal or zero */
        if (a < 0x33000000u)                   /* below 2^-25: rounds to zero */
            return (uint16_t)sign;
        uint32_t e = a >> 23;                  /* value = m * 2^(e-150) */
        uint32_t m = (a & 0x7FFFFFu) | 0x800000u;
        uint32_t shift = 126u - e;             /* value / 2^-24 = m >> shift */
        uint32_t q = m >> shift;
        uint32_t rem = m & ((1u << shift) - 1u);
        uint32_t half = 1u << (shift - 1u);
        if (rem > half || (rem == half && (q & 1u)))
            q++;
        return (uint16_t)(sign | q);
    }
    uint32_t e = (a >> 23) - 127u + 15u;
    uint32_t m = a & 0x7FFFFFu;
    uint32_t q = (e << 10) | (m >> 13);
    uint32_t rem = m & 0x1FFFu;
    if (rem > 0x1000u || (rem == 0x1000u && (q & 1u)))
        q++;
    return (uint16_t)(sign | q);
}

/* fp16 -> fp64 (exact). */
double w4o_f16_to_f64(uint16_t h)
{
    int sign = h >> 15;
    int e = (h >> 10) & 0x1F;
    int m = h & 0x3FF;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(m | 0x400), e - 25);
    return sign ? -v : v;
}

/* fp16 -> fp32 (exact: every fp16 value is an fp32 value). */
float w4o_f16_to_f32(uint16_t h)
{
    return (float)w4o_f16_to_f64(h);
}

/* round half to even of a finite fp32 value of small magnitude */
static int32_t rne_to_int(float t)
{
    double d = (double)t;
    double fl = floor(d);
    double frac = d - fl;
    int32_t q = (int32_t)fl;
    if (frac > 0.5 || (frac == 0.5 && (q & 1)))
        q += 1;
    return q;
}

/* ---------------------------------------------------------------- quantize + pack */

/* Scale of one group: fp16_rne(fp32(absmax) / 7). */
uint16_t w4o_group_scale(const uint16_t *x, int64_t n)
{
    float amax = 0.0f;
    for (int64_t k = 0; k < n; ++k) {
        float v = fabsf(w4o_f16_to_f32(x[k]));
        if (v > amax)
            amax = v;
    }
    volatile float q = amax / 7.0f;            /* one IEEE fp32 division */
    return w4o_f32_to_f16(q);
}

/* Quantized value of one element against the stored fp16 scale. */
int32_t w4o_quantize_one(uint16_t x, uint16_t s)
{
    float sf = w4o_f16_to_f32(s);
    if (sf == 0.0f)
        return 0;
    volatile float t = w4o_f16_to_f32(x) / sf; /* one IEEE fp32 division */
    int32_t q = rne_to_int(t);
    if (q < -8) q = -8;
    if (q > 7) q = 7;
    return q;
}

/* Quantize rows x[rows][K] (fp16 bits) per K-group of width `group` and pack.
 * packed: [rows][K/2] bytes, scales: [rows][K/group] fp16 bits.
 * Returns 0, or -1 on a shape the definition does not cover. */
int w4o_quantize_pack(const uint16_t *x, int64_t rows, int64_t K, int32_t group,
                      uint8_t *packed, uint16_t *scales)
{
    if (rows < 0 || K <= 0 || group <= 0 || K % group != 0 || K % 2 != 0 || group % 2 != 0)
        return -1;
    int64_t G = K / group;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t g = 0; g < G; ++g) {
            const uint16_t *xg = x + r * K + g * group;
            uint16_t s = w4o_group_scale(xg, group);
            scales[r * G + g] = s;
            for (int64_t k = 0; k < group; k += 2) {
                int32_t q0 = w4o_quantize_one(xg[k], s);
                int32_t q1 = w4o_quantize_one(xg[k + 1], s);
                packed[r * (K / 2) + (g * group + k) / 2] =
                    (uint8_t)((q0 & 0xF) | ((q1 & 0xF) << 4));
            }
        }
    }
    return 0;
}

/* Unpack [rows][K/2] bytes to signed int8 values [rows][K]. */
void w4o_unpack(const uint8_t *packed, int64_t rows, int64_t K, int8_t *q)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < K; ++k) {
            uint8_t b = packed[r * (K / 2) + k / 2];
            int v = (k & 1) ? (b >> 4) : (b & 0xF);
            if (v >= 8)
                v -= 16;
            q[r * K + k] = (int8_t)v;
        }
}

/* ---------------------------------------------------------------- GEMM */

static int check_groups(int64_t K, int32_t ga, int32_t gw, int32_t *ge)
{
    if (K <= 0 || ga <= 0 || gw <= 0 || K % ga || K % gw)
        return -1;
    int32_t lo = ga < gw ? ga : gw, hi = ga < gw ? gw : ga;
    if (hi % lo)
        return -1;
    *ge = lo;
    return 0;
}

/* Per-group integer partials for a list of A rows (rows == NULL: all M rows).
 * out: [K/ge][nrows][N] int64. */
int w4o_group_partials(const uint8_t *ap, const uint8_t *wp, int64_t M, int64_t N, int64_t K,
                       int32_t ga, int32_t gw, const int64_t *rows, int64_t nrows, int64_t *out)
{
    int32_t ge;
    if (check_groups(K, ga, gw, &ge))
        return -1;
    if (!rows)
        nrows = M;
    int64_t G = K / ge;
    int8_t *qw = (int8_t *)malloc((size_t)(N > 0 ? N : 1) * (size_t)K);
    if (!qw)
        return -2;
    w4o_unpack(wp, N, K, qw);
    int fail = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t m = rows ? rows[i] : i;
        int8_t *qa = (int8_t *)malloc((size_t)K);
        if (!qa) { fail = 1; continue; }
        w4o_unpack(ap + m * (K / 2), 1, K, qa);
        for (int64_t g = 0; g < G; ++g)
            for (int64_t n = 0; n < N; ++n) {
                int64_t acc = 0;
                for (int64_t k = g * ge; k < (g + 1) * ge; ++k)
                    acc += (int64_t)qa[k] * (int64_t)qw[n * K + k];
                out[(g * nrows + i) * N + n] = acc;
            }
        free(qa);
    }
    free(qw);
    return fail ? -2 : 0;
}

/* Output rows in fp64 for a list of A rows (rows == NULL: all M rows). y: [nrows][N]. */
int w4o_gemm(const uint8_t *ap, const uint16_t *sa, const uint8_t *wp, const uint16_t *sw,
             int64_t M, int64_t N, int64_t K, int32_t ga, int32_t gw,
             const int64_t *rows, int64_t nrows, double *y)
{
    int32_t ge;
    if (check_groups(K, ga, gw, &ge))
        return -1;
    if (!rows)
        nrows = M;
    int64_t G = K / ge, Ga = K / ga, Gw = K / gw;
    int8_t *qw = (int8_t *)malloc((size_t)(N > 0 ? N : 1) * (size_t)K);
    if (!qw)
        return -2;
    w4o_unpack(wp, N, K, qw);
    int fail = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t m = rows ? rows[i] : i;
        int8_t *qa = (int8_t *)malloc((size_t)K);
        if (!qa) { fail = 1; continue; }
        w4o_unpack(ap + m * (K / 2), 1, K, qa);
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t g = 0; g < G; ++g) {
                int64_t p = 0;
                for (int64_t k = g * ge; k < (g + 1) * ge; ++k)
                    p += (int64_t)qa[k] * (int64_t)qw[n * K + k];
                double s_a = w4o_f16_to_f64(sa[m * Ga + (g * ge) / ga]);
                double s_w = w4o_f16_to_f64(sw[n * Gw + (g * ge) / gw]);
                acc += (double)p * s_a * s_w;
            }
            y[i * N + n] = acc;
        }
        free(qa);
    }
    free(qw);
    return fail ? -2 : 0;
}

/* Threads the OpenMP loops above use. */
int w4o_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
