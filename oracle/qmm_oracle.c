/*
 * qmm_oracle.c -- plain, slow CPU oracle for MLX-style group-wise affine
 * quantization (quantize / dequantize).  TEST INFRASTRUCTURE ONLY: it exists
 * to check the CUDA library and is never linked into, loaded by or called
 * from the product path.  It shares no code, header, table or constant with
 * the CUDA sources.
 *
 * What it computes, and where that comes from:
 *
 *  - Quantization works along the last axis of a tensor of rank 2 or more
 *    (EMLX.Quantization, section `quantize`): each run of group_size
 *    consecutive elements of a row forms a group with its own floating-point
 *    scale and bias (mlx-rs ops/quantization.rs, doc comments of `quantize`
 *    and `quantized_matmul`).
 *  - Each element takes `bits` bits packed into unsigned 32-bit words;
 *    with bits=4 a word holds eight codes, so the last axis shrinks by 32/bits
 *    (Emily.QuantizedWeight, section Layout).
 *  - Scales and biases have the source weight's dtype and shape
 *    (..., last_dim / group_size) (Emily.QuantizedWeight, section Layout).
 *
 * None of the documents above prints the scale/bias rule or the bit order.  The reading
 * used here (stated once, applied everywhere):
 *    bias  = min of the group,
 *    scale = (max - min) / (2^bits - 1)          (fp32, correctly rounded),
 *    s, b  = scale, bias rounded to the storage dtype (round-to-nearest-even),
 *    q     = s == 0 ? 0 : clamp(rint((w - b) / s), 0, 2^bits - 1)   (fp32),
 *    element j of a row occupies bits [j*bits, (j+1)*bits) of the row's
 *    bit stream, bit i of the stream being bit (i mod 32) of word i / 32
 *    (least-significant code first; for bits 2, 4, 8 that is bit
 *    (j mod 32/bits) * bits of word j / (32/bits); 3- and 6-bit codes may
 *    straddle two words),
 *    dequantized w = fmaf(s, q, b), then rounded to the storage dtype.
 *
 * Every floating-point step is a single IEEE operation in fp32 (build with
 * -ffp-contract=off so that no multiply-add is fused behind our back); the
 * only fused operation is the explicit fmaf of the dequantize step.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* dtype tags (the oracle's own numbering) */
#define ORC_F32 0
#define ORC_BF16 1
#define ORC_F16 2

#define ORC_OK 0
#define ORC_BAD_ARG 1

/* ---- storage dtype conversions -------------------------------------- */

static float bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16; /* bf16 is the top half of an fp32 */
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* fp32 -> bf16, round to nearest, ties to even (NaN stays NaN). */
static uint16_t f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u)
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t keep_lsb = (u >> 16) & 1u;
    u += 0x7fffu + keep_lsb;
    return (uint16_t)(u >> 16);
}

static float load_elem(const void *p, int dtype, int64_t i)
{
    switch (dtype) {
    case ORC_F32: return ((const float *)p)[i];
    case ORC_BF16: return bf16_to_f32(((const uint16_t *)p)[i]);
    default: return (float)((const _Float16 *)p)[i]; /* exact widening */
    }
}

/* Store f rounded to nearest-even in `dtype`; return the stored value. */
static float store_elem(void *p, int dtype, int64_t i, float f)
{
    switch (dtype) {
    case ORC_F32:
        ((float *)p)[i] = f;
        return f;
    case ORC_BF16: {
        uint16_t h = f32_to_bf16(f);
        ((uint16_t *)p)[i] = h;
        return bf16_to_f32(h);
    }
    default: {
        _Float16 h = (_Float16)f; /* IEEE conversion, current mode = RNE */
        ((_Float16 *)p)[i] = h;
        return (float)h;
    }
    }
}

static int check_args(int dtype, int64_t rows, int64_t cols, int group_size, int bits)
{
    if (dtype != ORC_F32 && dtype != ORC_BF16 && dtype != ORC_F16)
        return ORC_BAD_ARG;
    if (bits != 2 && bits != 3 && bits != 4 && bits != 6 && bits != 8)
        return ORC_BAD_ARG;
    if (group_size != 32 && group_size != 64 && group_size != 128)
        return ORC_BAD_ARG;
    if (rows < 0 || cols <= 0 || cols % group_size != 0)
        return ORC_BAD_ARG;
    return ORC_OK;
}

/* Store code q of element (r, c): bits [c*bits, (c+1)*bits) of row r's bit
 * stream (words zeroed beforehand); the part past bit 31 of a word goes to
 * the low bits of the next word. */
static void put_code(uint32_t *wq, int64_t words_per_row, int bits, int64_t r, int64_t c,
                     uint32_t q)
{
    const int64_t bit = c * bits;
    const int off = (int)(bit % 32);
    uint32_t *row = wq + r * words_per_row;
    row[bit / 32] |= q << off;
    if (off + bits > 32)
        row[bit / 32 + 1] |= q >> (32 - off);
}

/*
 * Quantize w[rows, cols] (row-major, dtype `dtype`) group by group along the
 * last axis.  Outputs: wq[rows, cols*bits/32] (uint32), scales and biases
 * [rows, cols/group_size] in `dtype`.
 */
int oracle_quantize(const void *w, int dtype, int64_t rows, int64_t cols,
                    int group_size, int bits,
                    uint32_t *wq, void *scales, void *biases)
{
    int rc = check_args(dtype, rows, cols, group_size, bits);
    if (rc != ORC_OK)
        return rc;
    const int64_t words_per_row = cols * bits / 32;
    const int64_t groups_per_row = cols / group_size;
    const float qmax = (float)((1u << bits) - 1u);

    memset(wq, 0, (size_t)(rows * words_per_row) * sizeof(uint32_t));

    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t g = 0; g < groups_per_row; ++g) {
            const int64_t first = r * cols + g * group_size;

            /* 1. the group's minimum and maximum */
            float lo = load_elem(w, dtype, first);
            float hi = lo;
            for (int j = 1; j < group_size; ++j) {
                float v = load_elem(w, dtype, first + j);
                if (v < lo) lo = v;
                if (v > hi) hi = v;
            }

            /* 2. scale and bias, rounded to the storage dtype */
            float scale32 = (hi - lo) / qmax;
            const int64_t sb = r * groups_per_row + g;
            float s = store_elem(scales, dtype, sb, scale32);
            float b = store_elem(biases, dtype, sb, lo);

            /* 3. codes against the stored scale and bias, then packing */
            for (int j = 0; j < group_size; ++j) {
                float v = load_elem(w, dtype, first + j);
                uint32_t q = 0;
                if (s != 0.0f) {
                    float t = rintf((v - b) / s);
                    if (t < 0.0f) t = 0.0f;
                    if (t > qmax) t = qmax;
                    q = (uint32_t)t;
                }
                const int64_t c = g * group_size + j; /* column within the row */
                put_code(wq, words_per_row, bits, r, c, q);
            }
        }
    }
    return ORC_OK;
}

/* The code of element (r, c) read back from the row's bit stream. */
static uint32_t code_at(const uint32_t *wq, int64_t words_per_row, int bits,
                        int64_t r, int64_t c)
{
    const int64_t bit = c * bits;
    const int off = (int)(bit % 32);
    const uint32_t *row = wq + r * words_per_row;
    uint32_t v = row[bit / 32] >> off;
    if (off + bits > 32)
        v |= row[bit / 32 + 1] << (32 - off);
    return v & ((1u << bits) - 1u);
}

/*
 * Dequantize: w = scale * q + bias per element (mlx-rs ops/quantization.rs,
 * `dequantize`; EMLX.Quantization, section `dequantize`).  `out_f32` gets the
 * fp32 value fmaf(s, q, b) before any rounding to the storage dtype (may be
 * NULL); `out` gets it rounded to `dtype` (may be NULL).
 */
int oracle_dequantize(const uint32_t *wq, const void *scales, const void *biases,
                      int dtype, int64_t rows, int64_t cols, int group_size,
                      int bits, void *out, float *out_f32)
{
    int rc = check_args(dtype, rows, cols, group_size, bits);
    if (rc != ORC_OK)
        return rc;
    const int64_t words_per_row = cols * bits / 32;
    const int64_t groups_per_row = cols / group_size;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t c = 0; c < cols; ++c) {
            const int64_t sb = r * groups_per_row + c / group_size;
            float s = load_elem(scales, dtype, sb);
            float b = load_elem(biases, dtype, sb);
            float q = (float)code_at(wq, words_per_row, bits, r, c);
            float v = fmaf(s, q, b);
            if (out_f32)
                out_f32[r * cols + c] = v;
            if (out)
                store_elem(out, dtype, r * cols + c, v);
        }
    }
    return ORC_OK;
}

/* Unpack the codes alone: q[rows, cols] as uint8 (for code-level checks). */
int oracle_unpack_codes(const uint32_t *wq, int64_t rows, int64_t cols, int bits,
                        uint8_t *q)
{
    if (bits != 2 && bits != 3 && bits != 4 && bits != 6 && bits != 8)
        return ORC_BAD_ARG;
    const int64_t words_per_row = cols * bits / 32;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            q[r * cols + c] = (uint8_t)code_at(wq, words_per_row, bits, r, c);
    return ORC_OK;
}

/* fp32 -> storage dtype -> fp32, RNE (used to round fp64 matmul results). */
int oracle_round_to_dtype(const float *in, int dtype, int64_t n, void *out)
{
    if (dtype != ORC_F32 && dtype != ORC_BF16 && dtype != ORC_F16)
        return ORC_BAD_ARG;
    for (int64_t i = 0; i < n; ++i)
        store_elem(out, dtype, i, in[i]);
    return ORC_OK;
}

/* ======================================================================
 * Microscaled modes (Emily.QuantizedWeight, section Microscaled modes):
 *   mxfp4  group 32, 4-bit E2M1 elements, E8M0 scale byte
 *   mxfp8  group 32, 8-bit E4M3 elements, E8M0 scale byte
 *   nvfp4  group 16, 4-bit E2M1 elements, E4M3 scale byte
 * no biases.  The pages name the formats (a fused e8m0/e4m3 scale stored as
 * u8) but give no rule; the rule here follows the published definitions:
 *   - element and scale encodings: OCP Microscaling Formats (MX) v1.0
 *     (E2M1: bias 1, magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6;  E4M3: bias 7,
 *     largest finite 448, S.1111.111 is NaN;  E8M0: 2^(E - 127));
 *   - mx scale: X = 2^(floor(log2(max |v|)) - emax_elem), emax_elem = 2 for
 *     E2M1 and 8 for E4M3, clamped to the E8M0 range; elements are v / X
 *     rounded to nearest-even and saturated to the largest finite value
 *     (OCP MX v1.0, conversion of a vector to MX);
 *   - nvfp4 scale: the block maximum is mapped to E2M1's 6:  s = max|v| / 6
 *     rounded (nearest-even, saturating) to E4M3; elements are v / s in E2M1
 *     (NVIDIA's NVFP4 block format, without the optional per-tensor scale,
 *     which the pages' calls do not pass).
 * An all-zero block gets scale byte 0 and zero elements.
 * ====================================================================== */

#define ORC_MXFP4 1
#define ORC_MXFP8 2
#define ORC_NVFP4 3

static const float e2m1_mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

static float e2m1_value(uint32_t code)
{
    float m = e2m1_mag[code & 7u];
    return (code & 8u) ? -m : m;
}

/* Nearest E2M1 value, ties to the even code (last mantissa bit 0), values
 * beyond 6 saturated to 6; the sign is kept (so -0.1 gives negative zero). */
static uint32_t e2m1_encode(float v)
{
    const uint32_t sign = signbit(v) ? 8u : 0u;
    const float a = fabsf(v);
    uint32_t c;
    if (a <= 0.25f) c = 0;        /* 0.25: tie between 0 and 0.5 -> 0 (even) */
    else if (a < 0.75f) c = 1;    /* 0.5 */
    else if (a <= 1.25f) c = 2;   /* 1.0 (0.75 and 1.25 are ties that go to it) */
    else if (a < 1.75f) c = 3;    /* 1.5 */
    else if (a <= 2.5f) c = 4;    /* 2.0 (1.75 and 2.5 go to it) */
    else if (a < 3.5f) c = 5;     /* 3.0 */
    else if (a <= 5.0f) c = 6;    /* 4.0 (3.5 and 5.0 go to it) */
    else c = 7;                   /* 6.0, and everything above */
    return sign | c;
}

static float e4m3_value(uint32_t code)
{
    const uint32_t e = (code >> 3) & 15u, m = code & 7u;
    float a;
    if (e == 15u && m == 7u) a = NAN;
    else if (e == 0u) a = ldexpf((float)m, -9);                 /* m/8 * 2^-6 */
    else a = ldexpf(1.0f + (float)m / 8.0f, (int)e - 7);
    return (code & 0x80u) ? -a : a;
}

/* Nearest E4M3 value, ties to even, saturated to +-448 (no infinities). */
static uint32_t e4m3_encode(float v)
{
    const uint32_t sign = signbit(v) ? 0x80u : 0u;
    const float a = fabsf(v);
    if (a >= 0x1.0p-6f) {
        int e2;
        frexpf(a, &e2);              /* a = f * 2^e2, f in [0.5, 1) */
        int e = e2 - 1;              /* a in [2^e, 2^(e+1)) */
        float mi = rintf(ldexpf(a, 3 - e) - 8.0f);   /* mantissa in eighths, RNE */
        if (mi == 8.0f) {
            mi = 0.0f;
            ++e;
        }
        if (e > 8 || (e == 8 && mi == 7.0f)) return sign | 0x7Eu;  /* 448 */
        return sign | ((uint32_t)(e + 7) << 3) | (uint32_t)mi;
    }
    /* subnormal range: multiples of 2^-9 (m = 8 is the smallest normal, code 8) */
    const float m = rintf(ldexpf(a, 9));
    return sign | (uint32_t)m;
}

static int mx_params(int mode, int *gs, int *bits)
{
    switch (mode) {
    case ORC_MXFP4: *gs = 32; *bits = 4; return ORC_OK;
    case ORC_MXFP8: *gs = 32; *bits = 8; return ORC_OK;
    case ORC_NVFP4: *gs = 16; *bits = 4; return ORC_OK;
    default: return ORC_BAD_ARG;
    }
}

/* Element codes of `n` values for a mode's element format (for pins). */
int oracle_encode_elements(int mode, const float *in, int64_t n, uint8_t *out)
{
    int gs, bits;
    if (mx_params(mode, &gs, &bits) != ORC_OK) return ORC_BAD_ARG;
    for (int64_t i = 0; i < n; ++i)
        out[i] = (uint8_t)(bits == 8 ? e4m3_encode(in[i]) : e2m1_encode(in[i]));
    return ORC_OK;
}

/* Value of a scale byte (E8M0 for mx modes, E4M3 for nvfp4). */
static float mx_scale_value(int mode, uint32_t s)
{
    if (mode == ORC_NVFP4) return e4m3_value(s);
    return s == 255u ? NAN : ldexpf(1.0f, (int)s - 127);   /* E8M0 0xFF is NaN */
}

int oracle_quantize_mx(const void *w, int dtype, int64_t rows, int64_t cols, int mode,
                       uint32_t *wq, uint8_t *scales)
{
    int gs, bits;
    if (mx_params(mode, &gs, &bits) != ORC_OK) return ORC_BAD_ARG;
    if (dtype != ORC_F32 && dtype != ORC_BF16 && dtype != ORC_F16) return ORC_BAD_ARG;
    if (rows < 0 || cols <= 0 || cols % gs != 0) return ORC_BAD_ARG;
    const int64_t per_word = 32 / bits;
    const int64_t words_per_row = cols / per_word;
    const int64_t groups_per_row = cols / gs;
    const int emax = bits == 8 ? 8 : 2;
    memset(wq, 0, (size_t)(rows * words_per_row) * sizeof(uint32_t));
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t g = 0; g < groups_per_row; ++g) {
            const int64_t first = r * cols + g * gs;
            float amax = 0.0f;
            for (int j = 0; j < gs; ++j) {
                float a = fabsf(load_elem(w, dtype, first + j));
                if (a > amax) amax = a;
            }
            uint32_t scode;
            float div = 0.0f;   /* nvfp4: the stored scale the elements are divided by */
            int shared = -127;  /* mx: scale exponent */
            if (mode == ORC_NVFP4) {
                scode = e4m3_encode(amax / 6.0f);
                div = e4m3_value(scode);
            } else if (amax == 0.0f) {
                scode = 0;
            } else {
                int e2;
                frexpf(amax, &e2);
                shared = (e2 - 1) - emax;          /* floor(log2 amax) - emax_elem */
                if (shared < -127) shared = -127;
                if (shared > 127) shared = 127;
                scode = (uint32_t)(shared + 127);
            }
            scales[r * groups_per_row + g] = (uint8_t)scode;
            for (int j = 0; j < gs; ++j) {
                const float v = load_elem(w, dtype, first + j);
                uint32_t q;
                if (mode == ORC_NVFP4) {
                    q = div == 0.0f ? 0u : e2m1_encode(v / div);
                } else if (amax == 0.0f) {
                    q = 0u;
                } else {
                    const float t = ldexpf(v, -shared);   /* v / X */
                    q = bits == 8 ? e4m3_encode(t) : e2m1_encode(t);
                }
                put_code(wq, words_per_row, bits, r, g * gs + j, q);
            }
        }
    }
    return ORC_OK;
}

/* w = X * element, X the value of the group's scale byte; fp32 (exact) in
 * out_f32 (may be NULL) and rounded to `dtype` in out (may be NULL). */
int oracle_dequantize_mx(const uint32_t *wq, const uint8_t *scales, int dtype, int64_t rows,
                         int64_t cols, int mode, void *out, float *out_f32)
{
    int gs, bits;
    if (mx_params(mode, &gs, &bits) != ORC_OK) return ORC_BAD_ARG;
    if (dtype != ORC_F32 && dtype != ORC_BF16 && dtype != ORC_F16) return ORC_BAD_ARG;
    if (rows < 0 || cols <= 0 || cols % gs != 0) return ORC_BAD_ARG;
    const int64_t words_per_row = cols * bits / 32;
    const int64_t groups_per_row = cols / gs;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t c = 0; c < cols; ++c) {
            const float x = mx_scale_value(mode, scales[r * groups_per_row + c / gs]);
            const uint32_t q = code_at(wq, words_per_row, bits, r, c);
            const float e = bits == 8 ? e4m3_value(q) : e2m1_value(q);
            const float v = x * e;
            if (out_f32) out_f32[r * cols + c] = v;
            if (out) store_elem(out, dtype, r * cols + c, v);
        }
    }
    return ORC_OK;
}
