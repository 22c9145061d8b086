/*
 * fp8q_oracle.c -- plain, single-threaded CPU oracle of the FP8 E4M3
 * quantization path (group quantization, paged KV write, |K|/|V| absmax,
 * freeze scale).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and
 * the benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA library: it is written from the
 * definitions below, element by element, in the order they are stated, with
 * no blocking, fusion or reordering.
 *
 * Sources (page title, then the item on that page):
 *  - "spark_model/layers/ops/fp8_act_quant.rs", module doc: per-token
 *    quantization in 1x128 groups of a bf16 [M, K] activation into E4M3 codes
 *    plus one fp32 scale per group; grid (M, K/128), so K is a multiple of 128.
 *  - "spark_model/layers/ops/dispatch_proj_decode.rs", DecodeW8a8Scratch::fits
 *    and decode_w8a8_quant_act: codes are rows*k bytes, scales rows*(k/128)
 *    fp32 in [M, K/128] order.
 *  - "spark_model/layers/fp8_calibration/staging.rs", Fp8KvWriteTarget and
 *    KvStaging::replay_and_release: reshape_and_cache_fp8 takes bf16 K/V rows
 *    at key_stride/value_stride elements, an int64 slot per token, one k_scale
 *    and one v_scale, and pools whose blocks are cache_stride elements apart
 *    (block_size * num_kv_heads * head_dim).
 *  - "metrale_model_layers/layers/fp8_calibration.rs", module doc and absmax:
 *    amax is max |x| over the batch; the frozen scale is amax*headroom/448.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - the group scale is max(amax, 1e-12f) / 448.0f, an IEEE fp32 division;
 *  - a code is the E4M3 rounding of the fp32 quotient x / scale (the quotient
 *    is rounded to fp32 first, then to E4M3, round-to-nearest-even, saturating
 *    to +-448; the sign of zero is kept);
 *  - a slot < 0 is skipped; a slot >= num_blocks*block_size is skipped and
 *    counted;
 *  - inside one call, a later token wins a duplicated slot;
 *  - the frozen scale is max(amax*headroom, 1e-12f) / 448.0f, the product
 *    rounded to fp32 before the division.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC.
 * Floating point is evaluated in IEEE single precision (x86-64 SSE,
 * FLT_EVAL_METHOD == 0); -ffp-contract=off forbids fused multiply-adds.
 */
#include <stdint.h>
#include <string.h>
#include <math.h>

#define ORACLE_GROUP 128

/* bf16 is the top half of an IEEE binary32: widening is a 16-bit shift and
 * is exact. */
float oracle_bf16_to_f32(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/*
 * E4M3 ("FN" flavour: 1 sign, 4 exponent bits with bias 7, 3 mantissa bits,
 * no infinities, S.1111.111 is NaN).  The finite magnitudes are
 *   subnormal:  m * 2^-9,               m = 1..7      (exponent field 0)
 *   normal:     (1 + m/8) * 2^(e - 7),  e = 1..15     (m = 7 excluded at e = 15)
 * so the largest finite magnitude is 1.75 * 2^8 = 448.
 *
 * Encoding of a binary32 y: round |y| to the nearest point of that grid, ties
 * to the even mantissa; anything that would round above 448 saturates to 448
 * (0x7E); the sign bit is copied, so -0.0 encodes as 0x80.  NaN maps to the
 * NaN code of its sign (finite inputs are a precondition of the path).
 */
uint8_t oracle_e4m3_encode(float y)
{
    uint32_t u;
    memcpy(&u, &y, sizeof u);
    const uint8_t sign = (u >> 31) ? 0x80 : 0x00;
    if (isnan(y))
        return (uint8_t)(sign | 0x7F);

    const double a = fabs((double)y); /* exact */
    /* 448 is the top of the grid.  Between 448 and the next grid point of the
     * infinite-exponent extension (480) the midpoint 464 ties to 448 (even
     * mantissa 110 against odd 111), and above it the rounding would leave
     * the finite range: both saturate. */
    if (a >= 448.0)
        return (uint8_t)(sign | 0x7E);
    if (a == 0.0)
        return sign;

    /* Spacing of the grid around a: 2^(E-3) for a in [2^E, 2^(E+1)) with
     * E >= -6; the subnormal range below 2^-6 has the fixed spacing 2^-9. */
    int e2;
    (void)frexp(a, &e2);          /* a = f * 2^e2, f in [0.5, 1) */
    int E = e2 - 1;               /* floor(log2(a)) */
    if (E < -6)
        E = -6;
    const double spacing = ldexp(1.0, E - 3);
    /* a / spacing is exact (power-of-two scaling of a double that holds a
     * float).  nearbyint rounds in the current mode, round-to-nearest with
     * ties to even. */
    const double n = nearbyint(a / spacing);
    const double v = n * spacing; /* the rounded magnitude, exact */

    if (v == 0.0)
        return sign;
    if (v < ldexp(1.0, -6)) {
        /* subnormal: v = n * 2^-9 with n = 1..7 */
        return (uint8_t)(sign | (uint8_t)n);
    }
    /* normal (a subnormal that rounded up to 2^-6 lands here too) */
    int ev;
    (void)frexp(v, &ev);
    const int Ev = ev - 1;                             /* floor(log2(v)) */
    const int mant = (int)(ldexp(v, -Ev) * 8.0) - 8;   /* 0..7 */
    const int efield = Ev + 7;                         /* 1..15 */
    return (uint8_t)(sign | (uint8_t)((efield << 3) | mant));
}

void oracle_e4m3_encode_array(const float *y, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_e4m3_encode(y[i]);
}

/* Group scale of the activation quantizer: max(amax, 1e-12) / 448 in fp32. */
float oracle_group_scale(float amax)
{
    const float floored = fmaxf(amax, 1e-12f);
    return floored / 448.0f;
}

/*
 * Per-token 1x128-group quantization of a bf16 activation.
 *   x       [m, k] bf16 bits, row r starts at x + r * x_row_stride
 *   q       [m, k] E4M3 codes, packed rows (row stride k)
 *   scales  [m, k/128] fp32, row-major
 * For each row r and group g: amax = max_j |x[r, 128g + j]| (fp32, exact);
 * s = oracle_group_scale(amax); q[r, 128g + j] = E4M3(fp32(x / s)).
 * Returns 0, or -1 if k is not a positive multiple of 128 or the stride is
 * shorter than a row.
 */
int oracle_group_quant(const uint16_t *x, int64_t m, int64_t k,
                       int64_t x_row_stride, uint8_t *q, float *scales)
{
    if (k <= 0 || k % ORACLE_GROUP != 0 || x_row_stride < k || m < 0)
        return -1;
    const int64_t groups = k / ORACLE_GROUP;
    for (int64_t r = 0; r < m; ++r) {
        for (int64_t g = 0; g < groups; ++g) {
            const uint16_t *xg = x + r * x_row_stride + g * ORACLE_GROUP;
            float amax = 0.0f;
            for (int j = 0; j < ORACLE_GROUP; ++j) {
                const float a = fabsf(oracle_bf16_to_f32(xg[j]));
                if (a > amax)
                    amax = a;
            }
            const float s = oracle_group_scale(amax);
            scales[r * groups + g] = s;
            uint8_t *qg = q + r * k + g * ORACLE_GROUP;
            for (int j = 0; j < ORACLE_GROUP; ++j) {
                const float quotient = oracle_bf16_to_f32(xg[j]) / s;
                qg[j] = oracle_e4m3_encode(quotient);
            }
        }
    }
    return 0;
}

/*
 * max |x| over `rows` rows of `row_elems` bf16 values, row r at
 * x + r * row_stride.  0 for an empty input.  This is the bf16_absmax of the
 * calibrator (the pages pass packed rows; strided rows are honoured here).
 */
float oracle_absmax(const uint16_t *x, int64_t rows, int64_t row_elems,
                    int64_t row_stride)
{
    float amax = 0.0f;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t e = 0; e < row_elems; ++e) {
            const float a = fabsf(oracle_bf16_to_f32(x[r * row_stride + e]));
            if (a > amax)
                amax = a;
        }
    }
    return amax;
}

/*
 * reshape_and_cache_fp8: quantize each token's K and V row at the per-tensor
 * scale and scatter it into the paged pools.
 *   k, v          [num_tokens, num_kv_heads, head_dim] bf16 bits; token t's
 *                 row starts at k + t * key_stride (v + t * value_stride)
 *   slot_mapping  int64 per token; slot = block * block_size + offset
 *   k_pool/v_pool E4M3 bytes; the entry of (block, offset) starts at
 *                 block * cache_stride + offset * (num_kv_heads * head_dim)
 * Tokens are written in index order.  slot < 0: skipped.  slot >= num_blocks
 * * block_size: skipped and counted.  Returns the number of such
 * out-of-range slots, or -1 on invalid sizes.
 */
int64_t oracle_kv_write(const uint16_t *k, const uint16_t *v,
                        int64_t key_stride, int64_t value_stride,
                        const int64_t *slot_mapping, int64_t num_tokens,
                        int32_t num_kv_heads, int32_t head_dim,
                        uint8_t *k_pool, uint8_t *v_pool,
                        int32_t block_size, int64_t cache_stride,
                        int64_t num_blocks, float k_scale, float v_scale)
{
    const int64_t elems = (int64_t)num_kv_heads * head_dim;
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        block_size <= 0 || num_blocks < 0 || key_stride < elems ||
        value_stride < elems || cache_stride < (int64_t)block_size * elems)
        return -1;
    const int64_t num_slots = num_blocks * block_size;
    int64_t out_of_range = 0;
    for (int64_t t = 0; t < num_tokens; ++t) {
        const int64_t slot = slot_mapping[t];
        if (slot < 0)
            continue;
        if (slot >= num_slots) {
            ++out_of_range;
            continue;
        }
        const int64_t block = slot / block_size;
        const int64_t offset = slot % block_size;
        const int64_t base = block * cache_stride + offset * elems;
        for (int64_t e = 0; e < elems; ++e) {
            const float kq = oracle_bf16_to_f32(k[t * key_stride + e]) / k_scale;
            const float vq = oracle_bf16_to_f32(v[t * value_stride + e]) / v_scale;
            k_pool[base + e] = oracle_e4m3_encode(kq);
            v_pool[base + e] = oracle_e4m3_encode(vq);
        }
    }
    return out_of_range;
}

/* Scale frozen at the end of the calibration window:
 * max(amax * headroom, 1e-12) / 448, the product rounded to fp32 first. */
float oracle_freeze_scale(float amax, float headroom)
{
    const float widened = amax * headroom;
    const float floored = fmaxf(widened, 1e-12f);
    return floored / 448.0f;
}
