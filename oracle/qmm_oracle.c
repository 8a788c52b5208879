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
 *    element j of a row sits at bit (j mod (32/bits)) * bits of word
 *    j / (32/bits)  (least-significant code first),
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
    if (bits != 2 && bits != 4 && bits != 8)
        return ORC_BAD_ARG;
    if (group_size != 32 && group_size != 64 && group_size != 128)
        return ORC_BAD_ARG;
    if (rows < 0 || cols <= 0 || cols % group_size != 0)
        return ORC_BAD_ARG;
    return ORC_OK;
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
    const int64_t per_word = 32 / bits;
    const int64_t words_per_row = cols / per_word;
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
                wq[r * words_per_row + c / per_word] |= q << ((c % per_word) * bits);
            }
        }
    }
    return ORC_OK;
}

/* The code of element (r, c) read back from the packed words. */
static uint32_t code_at(const uint32_t *wq, int64_t words_per_row, int bits,
                        int64_t r, int64_t c)
{
    const int64_t per_word = 32 / bits;
    uint32_t word = wq[r * words_per_row + c / per_word];
    return (word >> ((c % per_word) * bits)) & ((1u << bits) - 1u);
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
    if (bits != 2 && bits != 4 && bits != 8)
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
