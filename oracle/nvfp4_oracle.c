/*
 * CPU oracle for NVFP4 W4A4 linear layers.  TEST INFRASTRUCTURE ONLY: it is
 * loaded by the test-suite, by the smoke check and by the benchmark's CPU
 * baseline leg, never by the library.  It shares no code, header, table or
 * constant with the CUDA path.
 *
 * What it follows ("Why Gated DeltaNet Survives 4-Bit Quantization: NVFP4 W4A4
 * for the Recurrent Half of a Hybrid 27B LLM", page summary, section
 * "Background", item 1): NVFP4 holds E2M1 4-bit values, one E4M3 scale per
 * 16-element block set to blockmax/6, and one FP32 scale per tensor.  The GEMM
 * runs on both quantized operands (W4A4, abstract; news article,
 * second paragraph), and when separately calibrated modules are served as one
 * fused GEMM, each module's own global scale governs its own output columns
 * (abstract, last sentence; "Risks and caveats").
 *
 * Readings where the pages are silent (all arithmetic FP32 round-to-nearest-
 * even, no flush-to-zero, unless stated):
 *   - global scale s_g = amax / 2688 (2688 = 6 * 448 maps the largest block's
 *     scale onto the largest E4M3 value); if that quotient is 0 (amax == 0, or
 *     so small the quotient underflows) then s_g = 1.
 *   - block scale byte sb = E4M3_rne_satfinite(bm / (6 * s_g)), two FP32
 *     operations: t = 6*s_g, then bm / t.  The effective scale
 *     decode(sb) * s_g is then about blockmax/6, the pages' rule.
 *   - se = decode(sb) * s_g; if se == 0 the whole block encodes to +0 codes.
 *     Otherwise inv = 1/se (FP32, correctly rounded; clamped to FLT_MAX when
 *     the reciprocal overflows), y = x * inv, code = E2M1_rne_satfinite(|y|)
 *     with the sign bit copied from x.
 *   - two codes per byte, the even element in the low nibble.
 * Dequantisation and the GEMM are FP64 and exact up to FP64 summation.
 *
 * Further sections, each with its own readings: the MLP glue between the two
 * W4A4 layers of a gated MLP (BF16 steps, as the kernels round), the Gated
 * DeltaNet gates of the fused input projection (FP64), and the calibrated
 * FP8 (E4M3) KV cache (FP32 product, then the E4M3 argmin).
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

/* ---------------------------------------------------------------------------
 * Element formats
 * ------------------------------------------------------------------------- */

/* E2M1 (1 sign, 2 exponent, 1 mantissa bit, bias 1, no inf/nan): magnitude of
 * codes 0..7.  Exponent field 0 is subnormal (0 and 0.5). */
static double e2m1_magnitude(int code)
{
    int e = (code >> 1) & 3, m = code & 1;
    if (e == 0) return 0.5 * m;
    return ldexp(1.0 + 0.5 * m, e - 1);
}

/* E4M3 (bias 7, the "fn" variant: 0x7f / 0xff are NaN, no inf), code 0..126. */
static double e4m3_magnitude(int code)
{
    int e = (code >> 3) & 15, m = code & 7;
    if (e == 0) return ldexp((double)m / 8.0, -6);
    return ldexp(1.0 + (double)m / 8.0, e - 7);
}

double oracle_e2m1_decode(uint8_t code)
{
    double v = e2m1_magnitude(code & 7);
    return (code & 8) ? -v : v;
}

double oracle_e4m3_decode(uint8_t code)
{
    double v = e4m3_magnitude(code & 0x7f);
    return (code & 0x80) ? -v : v;
}

/* Round-to-nearest over a value set by plain argmin; a tie goes to the code
 * whose lowest (mantissa) bit is 0.  Magnitudes at or above the largest finite
 * value saturate to it (checked first: for huge inputs the FP64 distances to
 * neighbouring grid points are no longer distinct). */
uint8_t oracle_e2m1_encode_magnitude(float a)
{
    double x = fabs((double)a);
    if (x >= 6.0) return 7;
    int best = 0;
    double best_d = fabs(x - e2m1_magnitude(0));
    for (int c = 1; c < 8; ++c) {
        double d = fabs(x - e2m1_magnitude(c));
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_d = d;
        }
    }
    return (uint8_t)best;
}

uint8_t oracle_e4m3_encode_positive(float a)
{
    double x = fabs((double)a);
    if (x >= 448.0) return 0x7e;
    int best = 0;
    double best_d = fabs(x - e4m3_magnitude(0));
    for (int c = 1; c < 127; ++c) {
        double d = fabs(x - e4m3_magnitude(c));
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_d = d;
        }
    }
    return (uint8_t)best;
}

void oracle_e2m1_encode_many(const float* y, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; ++i) {
        uint8_t c = oracle_e2m1_encode_magnitude(y[i]);
        out[i] = signbit(y[i]) ? (uint8_t)(c | 8) : c;
    }
}

void oracle_e4m3_encode_many(const float* x, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode_positive(x[i]);
}

/* ---------------------------------------------------------------------------
 * Two-level scaling
 * ------------------------------------------------------------------------- */

/* amax over a rows x cols matrix with row stride ld (elements). */
float oracle_amax(const float* x, int64_t rows, int64_t cols, int64_t ld)
{
    float amax = 0.0f;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            float a = fabsf(x[r * ld + c]);
            if (a > amax) amax = a;
        }
    return amax;
}

float oracle_global_scale_from_amax(float amax)
{
    volatile float s = amax / 2688.0f;
    if (s == 0.0f) s = 1.0f;
    return s;
}

float oracle_global_scale(const float* x, int64_t rows, int64_t cols, int64_t ld)
{
    return oracle_global_scale_from_amax(oracle_amax(x, rows, cols, ld));
}

/*
 * Quantise rows x k (k % 16 == 0) with global scale s_g.
 *   q  : rows x k/2 bytes, row-major, element 2j in the low nibble of byte j.
 *   sf : rows x k/16 scale bytes, ROW-MAJOR (the plain view; the tiled device
 *        layout is produced separately by oracle_sf_to_tiled).
 */
void oracle_quantize(const float* x, int64_t rows, int64_t k, int64_t ld, float s_g,
                     uint8_t* q, uint8_t* sf)
{
    const int64_t nb = k / 16;
    const float t = 6.0f * s_g;
    /* rows are independent: the OpenMP split changes no arithmetic */
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            const float* xb = x + r * ld + b * 16;
            float bm = 0.0f;
            for (int j = 0; j < 16; ++j) {
                float a = fabsf(xb[j]);
                if (a > bm) bm = a;
            }
            volatile float sb32 = bm / t;
            uint8_t sb = oracle_e4m3_encode_positive(sb32);
            sf[r * nb + b] = sb;
            volatile float se = (float)e4m3_magnitude(sb) * s_g;
            uint8_t codes[16];
            if (se == 0.0f) {
                memset(codes, 0, sizeof codes);
            } else {
                volatile float inv = 1.0f / se;
                if (isinf(inv)) inv = FLT_MAX;
                for (int j = 0; j < 16; ++j) {
                    volatile float y = xb[j] * inv;
                    uint8_t c = oracle_e2m1_encode_magnitude(y);
                    codes[j] = signbit(xb[j]) ? (uint8_t)(c | 8) : c;
                }
            }
            uint8_t* qb = q + r * (k / 2) + b * 8;
            for (int j = 0; j < 8; ++j)
                qb[j] = (uint8_t)(codes[2 * j] | (codes[2 * j + 1] << 4));
        }
    }
}

/* x_hat = e2m1(q) * e4m3(sb) * s_g, FP64 (exact: 2 + 4 + 24 significant bits). */
void oracle_dequantize(const uint8_t* q, const uint8_t* sf, int64_t rows, int64_t k,
                       float s_g, double* out)
{
    const int64_t nb = k / 16;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t i = 0; i < k; ++i) {
            uint8_t byte = q[r * (k / 2) + i / 2];
            uint8_t code = (i & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15);
            out[r * k + i] = oracle_e2m1_decode(code) * oracle_e4m3_decode(sf[r * nb + i / 16])
                             * (double)s_g;
        }
}

/* ---------------------------------------------------------------------------
 * Tiled scale-factor layout used by block-scaled tensor-core MMAs: atoms of
 * 128 rows x 4 scale columns (512 bytes).  Inside an atom, row r sits at
 * (r % 32) * 16 + (r / 32) * 4 and scale column c at + c.  Atoms are ordered
 * K-atom fastest, then 128-row block.  Rows pad to 128, k/16 pads to 4,
 * padding bytes are zero.
 * ------------------------------------------------------------------------- */
int64_t oracle_sf_tiled_bytes(int64_t rows, int64_t k)
{
    int64_t nb = k / 16;
    return ((rows + 127) / 128) * 128 * ((nb + 3) / 4) * 4;
}

int64_t oracle_sf_tiled_offset(int64_t row, int64_t kb, int64_t k)
{
    int64_t katoms = (k / 16 + 3) / 4;
    int64_t atom = (row / 128) * katoms + kb / 4;
    int64_t r = row % 128;
    return atom * 512 + (r % 32) * 16 + (r / 32) * 4 + (kb % 4);
}

void oracle_sf_to_tiled(const uint8_t* sf, int64_t rows, int64_t k, uint8_t* tiled)
{
    const int64_t nb = k / 16;
    memset(tiled, 0, (size_t)oracle_sf_tiled_bytes(rows, k));
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < nb; ++b)
            tiled[oracle_sf_tiled_offset(r, b, k)] = sf[r * nb + b];
}

/* ---------------------------------------------------------------------------
 * GEMM: C[m, n] = sum_k A_hat[m, k] * W_hat[n, k] in FP64 (W is N x K, the
 * nn.Linear layout).  Row-parallel with OpenMP when built with -fopenmp.
 * ------------------------------------------------------------------------- */
void oracle_gemm(const double* a, const double* w, int64_t m, int64_t n, int64_t k, double* c)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < m; ++i)
        for (int64_t j = 0; j < n; ++j) {
            double acc = 0.0;
            for (int64_t p = 0; p < k; ++p) acc += a[i * k + p] * w[j * k + p];
            c[i * n + j] = acc;
        }
}

/* ---------------------------------------------------------------------------
 * BF16 helpers and the MLP glue h = bf16(silu(g) * u), silu(x) = x / (1 + e^-x),
 * every step in FP32.
 * ------------------------------------------------------------------------- */
static float bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static uint16_t f32_to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u) return 0x7fc0;
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

void oracle_bf16_round(const float* x, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16_rne(x[i]);
}

void oracle_silu_mul_bf16(const uint16_t* g, const uint16_t* u, int64_t n, uint16_t* h)
{
    for (int64_t i = 0; i < n; ++i) {
        volatile float x = bf16_to_f32(g[i]);
        volatile float e = expf(-x);
        volatile float d = 1.0f + e;
        volatile float s = x / d;
        volatile float p = s * bf16_to_f32(u[i]);
        h[i] = f32_to_bf16_rne(p);
    }
}

/* -------------------------------------------------------------------------
 * Calibrated FP8 KV cache (abstract: calibrated FP8 KV-cache scales cost no
 * performance and ship with the recipe; Glonce article, "How to use it";
 * aiany.app, "Mechanistic notes").  The pages give no formula; the readings:
 *   - one FP32 scale per tensor (K and V each), calibrated as
 *     s = amax / 448 (448 = the largest E4M3 value; one FP32 division), or
 *     s = 1 if that quotient is 0;
 *   - stored byte = E4M3_rne_satfinite(x * inv_s), inv_s = 1 / s (FP32,
 *     correctly rounded; FLT_MAX if the reciprocal overflows), the sign bit
 *     copied from the FP32 product (so -0 and small negatives give 0x80);
 *   - the value read back is decode(byte) * s.
 * ------------------------------------------------------------------------- */
float oracle_fp8_scale_from_amax(float amax)
{
    volatile float s = amax / 448.0f;
    return s == 0.0f ? 1.0f : s;
}

void oracle_fp8_quantize(const float* x, int64_t n, float scale, uint8_t* out)
{
    volatile float inv = 1.0f / scale;
    if (isinf(inv)) inv = FLT_MAX;
    for (int64_t i = 0; i < n; ++i) {
        volatile float y = x[i] * inv;
        uint8_t c = oracle_e4m3_encode_positive(y);
        out[i] = signbit(y) ? (uint8_t)(c | 0x80) : c;
    }
}

/* -------------------------------------------------------------------------
 * Gated DeltaNet gates from the two head-wide segments a and b of the fused
 * input projection ("Why Gated DeltaNet Survives 4-Bit Quantization", page
 * summary, "Gated DeltaNet Mechanics"): the forget gate in log space
 *     g = -exp(A_log[h]) * softplus(a + dt_bias[h]),  softplus(x) = log(1 + e^x),
 * and the correction scale beta = sigmoid(b) = 1 / (1 + e^-b) (the pages name
 * beta_t but its formula is lost in the extracted text; the sigmoid of the b
 * projection is the reading taken).  FP64 throughout.
 * ------------------------------------------------------------------------- */
static double softplus64(double x)
{
    /* log(1 + e^x) without overflow: max(x, 0) + log1p(e^-|x|) */
    return (x > 0.0 ? x : 0.0) + log1p(exp(-fabs(x)));
}

void oracle_gdn_gates(const float* a, const float* b, int64_t m, int64_t heads, int64_t ld,
                      const float* A_log, const float* dt_bias, double* g, double* beta)
{
    for (int64_t r = 0; r < m; ++r)
        for (int64_t h = 0; h < heads; ++h) {
            g[r * heads + h] = -exp((double)A_log[h]) * softplus64((double)a[r * ld + h] + (double)dt_bias[h]);
            beta[r * heads + h] = 1.0 / (1.0 + exp(-(double)b[r * ld + h]));
        }
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
