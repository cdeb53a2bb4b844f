/*
 * CPU oracle for MXFP4 quantize / dequantize -- TEST INFRASTRUCTURE ONLY.
 *
 * This file is the plain, slow, obviously-correct definition that the CUDA
 * library is checked against.  It shares no code, header, table or constant
 * generator with the CUDA path.  Only tests, the smoke check and the
 * benchmark's CPU-baseline leg may load it; the product never does.
 *
 * What the pages fix (agentlenshq.com, "Transformers 4.40 performance upgrades
 * for OpenAI GPT-OSS: zero-build kernels, MXFP4 quantization, parallelism, and
 * faster loading", section "MXFP4 4-Bit Quantization / What MXFP4 Is"; the same
 * section on the zh-CN page and the E2M1 sentence of the otomatix.tech page):
 *   - each element is an E2M1 float: 1 sign bit, 2 exponent bits, 1 mantissa bit;
 *   - elements come in blocks of 32 that share one scale.
 * Readings taken where the pages are silent:
 *   - E2M1 exponent bias 1, so the magnitudes are {0, .5, 1, 1.5, 2, 3, 4, 6};
 *   - the shared scale is an E8M0 byte S meaning 2^(S-127); S = 0xFF is NaN;
 *   - scale exponent s = floor(log2(amax)) - 2 ("floor" rule, 2 being the
 *     largest E2M1 exponent) or the smallest s with amax / 2^s <= 6 ("ceil"
 *     rule), clamped to [-127, 127]; an all-zero block gets S = 0;
 *   - element codes are round-to-nearest-even of |v| / 2^s onto the E2M1 grid,
 *     saturating at 6, with the input's sign bit copied (so -0 -> code 0x8);
 *   - a block holding Inf or NaN gets S = 0xFF and all-zero codes;
 *   - two codes per byte, the even element in the low nibble; blocks run along
 *     the last (contiguous) dimension, scales stored row-major [rows, cols/32].
 * Dequantize is the exact product code_value * 2^(S-127) rounded once to bf16
 * (round-to-nearest-even; only overflow to Inf can actually round).
 *
 * Everything is computed in fp64; OpenMP only splits independent rows.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define MX_BLOCK 32

/* E2M1 magnitude of a 3-bit magnitude code (2 exponent bits e, 1 mantissa bit m),
 * bias 1: e == 0 is subnormal, m * 2^(1-1) * 1/2; otherwise 2^(e-1) * (1 + m/2). */
double oracle_e2m1_magnitude(int mag_code) {
    int e = (mag_code >> 1) & 3;
    int m = mag_code & 1;
    if (e == 0) return 0.5 * (double)m;
    return ldexp(1.0 + 0.5 * (double)m, e - 1);
}

/* Exact value of a bf16 bit pattern. */
static double bf16_value(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round an fp64 value to bf16 with round-to-nearest-even (8 significant bits,
 * normal exponents [-126, 127], subnormal quantum 2^-133, overflow to Inf). */
uint16_t oracle_f64_to_bf16(double x) {
    if (isnan(x)) return 0x7FC0;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (a == 0.0) return sign;
    if (isinf(a)) return (uint16_t)(sign | 0x7F80);
    int ex;
    frexp(a, &ex);                 /* a = f * 2^ex, f in [0.5, 1) */
    int e = ex - 1;                /* floor(log2 a) */
    if (e < -126) e = -126;        /* subnormal range keeps the quantum fixed */
    int qe = e - 7;                /* weight of the last kept significand bit */
    double q = nearbyint(ldexp(a, -qe));   /* ties to even (default mode) */
    double r = ldexp(q, qe);
    if (r >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80);
    float f = (float)r;            /* exact: r has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | ((u >> 16) & 0x7FFF));
}

void oracle_f64_to_bf16_array(const double* x, int64_t n, uint16_t* out) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f64_to_bf16(x[i]);
}

/* Round r >= 0 to the E2M1 grid with ties to even and saturation at 6.
 * The grid spacing is 0.5 on [0, 2), 1 on [2, 4) and 2 on [4, 8); rounding
 * r / spacing to the nearest integer (ties to even) and scaling back is the
 * textbook round-to-nearest-even; values past 6 saturate.  Returns the 3-bit
 * magnitude code, i.e. the index of the result in the ordered grid. */
static int e2m1_round_rne(double r) {
    double spacing = (r < 2.0) ? 0.5 : (r < 4.0 ? 1.0 : 2.0);
    double q = nearbyint(r / spacing) * spacing;
    if (q > 6.0) q = 6.0;
    for (int c = 0; c < 8; ++c)
        if (oracle_e2m1_magnitude(c) == q) return c;
    return -1; /* unreachable: q is always on the grid */
}

/* Quantize one block of 32 values (v exact, neg = sign bits). */
static void quantize_block(const double* v, const int* neg, int rule,
                           uint8_t* codes4 /* 32 codes, one per byte */, uint8_t* scale) {
    int nonfinite = 0;
    double amax = 0.0;
    for (int i = 0; i < MX_BLOCK; ++i) {
        if (!isfinite(v[i])) nonfinite = 1;
        else if (fabs(v[i]) > amax) amax = fabs(v[i]);
    }
    if (nonfinite) {
        *scale = 0xFF;
        for (int i = 0; i < MX_BLOCK; ++i) codes4[i] = 0;
        return;
    }
    int s;
    if (amax == 0.0) {
        s = -127;
    } else {
        int ex;
        frexp(amax, &ex);
        int e = ex - 1;                  /* floor(log2 amax), exact */
        s = e - 2;                       /* floor rule: 2 = top E2M1 exponent */
        if (rule == 1 && amax > ldexp(6.0, s)) s += 1;   /* ceil rule: never clip */
        if (s < -127) s = -127;
        if (s > 127) s = 127;
    }
    *scale = (uint8_t)(s + 127);
    for (int i = 0; i < MX_BLOCK; ++i) {
        double r = ldexp(fabs(v[i]), -s);    /* exact power-of-two scaling */
        int mag = e2m1_round_rne(r);
        codes4[i] = (uint8_t)((neg[i] ? 8 : 0) | mag);
    }
}

static void quantize_rows(const void* x, int is_f32, int64_t rows, int64_t cols,
                          uint8_t* codes, uint8_t* scales, int rule) {
    int64_t nb = cols / MX_BLOCK;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        double v[MX_BLOCK];
        int neg[MX_BLOCK];
        uint8_t c[MX_BLOCK];
        for (int64_t b = 0; b < nb; ++b) {
            for (int i = 0; i < MX_BLOCK; ++i) {
                int64_t idx = r * cols + b * MX_BLOCK + i;
                if (is_f32) {
                    float f = ((const float*)x)[idx];
                    v[i] = (double)f;
                    neg[i] = signbit(f) ? 1 : 0;
                } else {
                    uint16_t h = ((const uint16_t*)x)[idx];
                    v[i] = bf16_value(h);
                    neg[i] = (h >> 15) & 1;
                }
            }
            quantize_block(v, neg, rule, c, &scales[r * nb + b]);
            for (int j = 0; j < MX_BLOCK / 2; ++j)
                codes[r * (cols / 2) + b * (MX_BLOCK / 2) + j] =
                    (uint8_t)(c[2 * j] | (c[2 * j + 1] << 4));
        }
    }
}

void oracle_quantize_bf16(const uint16_t* x, int64_t rows, int64_t cols,
                          uint8_t* codes, uint8_t* scales, int rule) {
    quantize_rows(x, 0, rows, cols, codes, scales, rule);
}

void oracle_quantize_f32(const float* x, int64_t rows, int64_t cols,
                         uint8_t* codes, uint8_t* scales, int rule) {
    quantize_rows(x, 1, rows, cols, codes, scales, rule);
}

/* Exact dequantized value of element i of a row (fp64; NaN for S = 0xFF). */
static double dequant_value(const uint8_t* codes_row, const uint8_t* scales_row, int64_t i) {
    uint8_t byte = codes_row[i / 2];
    int code = (i & 1) ? (byte >> 4) : (byte & 0xF);
    uint8_t S = scales_row[i / MX_BLOCK];
    if (S == 0xFF) return NAN;
    double mag = ldexp(oracle_e2m1_magnitude(code & 7), (int)S - 127);
    return (code & 8) ? -mag : mag;
}

void oracle_dequantize_f64(const uint8_t* codes, const uint8_t* scales,
                           int64_t rows, int64_t cols, double* out) {
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t i = 0; i < cols; ++i)
            out[r * cols + i] = dequant_value(codes + r * (cols / 2),
                                              scales + r * (cols / MX_BLOCK), i);
}

void oracle_dequantize_bf16(const uint8_t* codes, const uint8_t* scales,
                            int64_t rows, int64_t cols, uint16_t* out) {
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t i = 0; i < cols; ++i)
            out[r * cols + i] = oracle_f64_to_bf16(
                dequant_value(codes + r * (cols / 2), scales + r * (cols / MX_BLOCK), i));
}
