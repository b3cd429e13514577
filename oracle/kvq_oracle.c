/*
 * kvq_oracle.c -- plain CPU oracle for the quantized-KV-cache hot path.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test-suite, the smoke
 * check and the CPU-baseline leg of the benchmark may load this file's
 * library.  It shares no code, header, table or constant generator with the
 * CUDA library; it is written straight from the pages it cites, in their
 * notation, with no blocking, fusion or reordering.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC
 * (no FMA contraction, no fast-math: every fp32 operation below is one IEEE
 * operation rounded to nearest-even, in the order written).
 *
 * Sources (page title, section):
 *   [P1] "大模型KV缓存量化技术：原理、优化与实践", section 2.1 (static global
 *        quantization: scale = (max - min) / (2^bits - 1)); sections 3.1
 *        (Oaken: offline thresholds, online group-shift quantization,
 *        dense-sparse encoding), 3.2.1 (threshold zones and their widths)
 *        and 3.2.2 (group shift: Delta = value - T_hi or value - T_lo,
 *        dequantized as T + Delta * scale).
 *   [P2] "大模型推理加速之KV Cache量化压缩原理与工程实现": the KV-cache size
 *        formula (2 * layers * kv_heads * head_dim * seq_len * batch * bytes);
 *        "常见问题排查" (scale clamped to at least 1e-5); INT4 asymmetric
 *        group quantization with group_size 128 or 64.
 *   [P3] "长上下文LLM推理中的KV Cache优化技术解析", section 3.2
 *        (score = q . k^T / sqrt(dim)).
 *   [P4] Cocktail page (peacm.com news 1099647): 3.1.1 (chunk search: cosine
 *        similarity, T_low / T_high from alpha and beta, FP16 / INT4 / INT2);
 *        3.1.2 (reorder chunks so equal bit-widths are contiguous);
 *        3.2.2 (group quantization quant(x) = round(x/s) + z);
 *        3.2.3 (chunked attention, merged, equal to unchunked attention).
 *   [P5] TurboQuant page (bhfrc.com news 57821): 1.2 (KV element count
 *        worked example); 2.3 (per-group scaling, dequantization inside
 *        the attention matmul).
 *   [P2'] The KV-cache page above, "主流KV Cache量化方案对比" item 1 (FP8
 *        KV cache, E4M3 or E5M2, 2x compression), item 2 (INT8 quantization
 *        with a symmetric scale amax / 127, round, clamp to [-128, 127]) and
 *        "实践中的调优建议" (dynamic quantization: the scale is computed from
 *        the current vectors at every step).
 *
 * Readings taken where the pages are silent (each one also listed in the
 * design notes):
 *   R1  "round" is round-half-to-even (rintf in the default rounding mode).
 *   R2  The 1e-5 scale floor is applied in fp32 before s is stored in fp16,
 *       and s is stored rounded toward +infinity (the smallest fp16 value
 *       not below the fp32 scale): then the stored grid still spans
 *       [min, max] in 2^b - 1 steps and every element keeps |x - x_hat|
 *       <= s/2.  Rounding s to nearest could shrink it and push the
 *       group's maximum one code past 2^b - 1.
 *   R3  Quantization divides by the stored fp16 scale, not the fp32 one.
 *   R4  z = rint(-min / s), clamped to the fp16 range, stored as fp16, NOT
 *       clamped to [0, qmax]; a zero-point of -0 is stored as +0.
 *   R5  quant(x) rounds x/s first and then adds the integer z; the result is
 *       clamped to [0, qmax].
 *   R6  Groups run along head_dim within one token row.
 *   R7  Codes are packed little-endian inside bytes: element j of a row sits
 *       in byte floor(j*b/8) at bit offset (j*b) mod 8.
 *   R8  Cocktail's garbled threshold rule reads: sim > T_high -> FP16,
 *       T_low < sim <= T_high -> INT4, sim <= T_low -> INT2; s_min and s_max
 *       are taken over the chunks of one sequence; all in fp64.
 *   R9  Reorder order: FP16 chunks, then INT4, then INT2, each class in
 *       ascending original chunk index.
 *   R14 FP8 codes are E4M3 in the variant without infinities (bias 7, three
 *       mantissa bits, largest finite 448, S.1111.111 is NaN).  Scales are
 *       dynamic and per group of G along head_dim of each token, like the
 *       integer formats: s = max(amax / 448, 1e-5) in fp32, stored in fp16
 *       rounded toward +infinity (so |x / s| <= 448), zero point 0; each
 *       code is x / s (one fp32 division) rounded to the nearest E4M3 value,
 *       ties to even, saturating at +-448; x_hat = e4m3(code) * s.
 *   R15 Symmetric INT8 ([P2'] item 2): the listing reduces the scale over
 *       head_dim of each token while its prose says per channel; the group
 *       runs along head_dim per token like every other format (G = head_dim
 *       is the listing's per-token scale).  s = max(amax / 127, 1e-5) in
 *       fp32, stored in fp16 rounded toward +infinity (R2), zero point 0;
 *       code = clamp(round(x / s), -128, 127) with one fp32 division by the
 *       stored scale (R3) and round-half-to-even (R1), stored as a two's
 *       complement byte; x_hat = code * s.  With the rounded-up scale
 *       |x / s| <= 127, so the clamp never acts; it is kept as written.
 *   R16 Per-channel K ([P2'] item 2: the Key is more sensitive to
 *       quantization error and is quantized per channel, the Value per
 *       token).  K is grouped per channel over blocks of 32 consecutive
 *       tokens of one (sequence, KV head): each channel of a block has its
 *       own (s, z), from the asymmetric formula of R1-R5 over the block's 32
 *       values of that channel.  Codes stay packed along token rows (R7);
 *       the (s, z) pairs are stored per block and channel.  Only complete
 *       blocks are quantized: the tokens of an unfinished block stay in
 *       fp16 (a separate fp16 segment) until the block is complete.  V keeps
 *       its per-token groups along head_dim (R6).
 *   R17 FP8 E5M2 ([P2'] item 1 names E5M2 beside E4M3): the format with
 *       bias 15, two mantissa bits, largest finite 57344, infinities and NaN
 *       in E = 31; the scale as R14 with 57344 for 448 (s = max(amax /
 *       57344, 1e-5), fp16 rounded up); codes the nearest E5M2 value of x /
 *       s, ties to even, saturating at +-57344 (never an infinity).
 *   R18 Oaken group-shift codec ([P1] 3.1 online phase, 3.2.1 zones,
 *       3.2.2 group shift).  The thresholds are fixed offline per plane and
 *       given as an inner scale s_in (an fp16 value) and an integer inner
 *       zero point z_in in [0, 15]: T_lo = -z_in * s_in, T_hi = (15 - z_in)
 *       * s_in, both exact in fp32, so the thresholds sit on the inner grid.
 *       The outer scale s_out > 0 and the outer width b in {5, 6, 7} are
 *       fixed offline too.  Per element v (fp16 read exactly into fp32):
 *         T_lo <= v <= T_hi: c = clamp(rint(v / s_in) + z_in, 0, 15) (the
 *           listing's quantize(value, inner_scale), with R1, R5), no
 *           outlier.  The page's inner and middle zones (both 4-bit) are
 *           this one quantizer: the listing has a single non-outer branch.
 *         v > T_hi: c = 15 and the outlier Delta = v - T_hi (one fp32
 *           subtraction) is kept as m = min(rint(Delta / s_out), 2^b - 1).
 *         v < T_lo: c = 0, Delta = v - T_lo, m = min(rint(-Delta / s_out),
 *           2^b - 1), kept as -m.
 *       Dense-sparse storage: the codes c are packed like 4-bit integer
 *       codes (R7).  A row's outliers go, in ascending dim order, to 16
 *       slots of 16 bits each (low byte the dim, high byte the signed m as
 *       a two's complement byte).  Slots after the last outlier hold 0.
 *       Outliers after the 16th are dropped, so those elements reconstruct
 *       to their threshold.  x_hat = (c - z_in) * s_in + d * s_out, where d
 *       is the element's signed slot value (0 without a slot).  For an
 *       outlier that is T_hi + m * s_out or T_lo - m * s_out: the page's
 *       dequantization T + Delta_hat.
 *
 * Code formats (the `fmt` arguments): 0 asymmetric integer codes of `bits`
 * bits (R1-R7), 1 E4M3 (R14), 2 symmetric INT8 (R15), 3 E5M2 (R17).  The
 * Oaken codec (R18) has functions of its own.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* IEEE 754 binary16 <-> binary32, written from the format definition.      */
/* ------------------------------------------------------------------------ */

/* Round an fp32 value to the nearest binary16 value, ties to even. */
uint16_t kvqo_f32_to_f16(float f)
{
    uint32_t x;
    memcpy(&x, &f, sizeof x);
    uint32_t sign = (x >> 16) & 0x8000u;
    uint32_t exp8 = (x >> 23) & 0xffu;
    uint32_t frac = x & 0x7fffffu;

    if (exp8 == 0xffu) /* infinity or NaN */
        return (uint16_t)(sign | 0x7c00u | (frac ? 0x0200u : 0u));

    int32_t e = (int32_t)exp8 - 127; /* unbiased exponent */
    if (e >= 16)                     /* |f| >= 2^16: beyond the largest finite */
        return (uint16_t)(sign | 0x7c00u);

    if (e >= -14) {
        /* normal binary16 range: keep 10 fraction bits, round the other 13 */
        uint32_t h = ((uint32_t)(e + 15) << 10) | (frac >> 13);
        uint32_t rest = frac & 0x1fffu;
        if (rest > 0x1000u || (rest == 0x1000u && (h & 1u)))
            h += 1u; /* a carry into the exponent is the correct result */
        return (uint16_t)(sign | h);
    }

    /* subnormal binary16: value = m * 2^-24, m in [0, 1023] */
    if (exp8 == 0u)
        return (uint16_t)sign; /* fp32 subnormals are far below 2^-25 */
    uint32_t full = frac | 0x800000u; /* value = full * 2^(e - 23) */
    int32_t shift = -e - 1;           /* m = full * 2^(e + 1), i.e. >> (-e-1) */
    if (shift > 24)
        return (uint16_t)sign; /* below half of the smallest subnormal */
    uint32_t m = full >> shift;
    uint32_t rest = full & ((1u << shift) - 1u);
    uint32_t half = 1u << (shift - 1);
    if (rest > half || (rest == half && (m & 1u)))
        m += 1u;
    return (uint16_t)(sign | m);
}

float kvqo_f16_to_f32(uint16_t h);

/* Round a positive finite fp32 value up to the nearest binary16 value
 * (the smallest binary16 value >= f). */
uint16_t kvqo_f32_to_f16_up(float f)
{
    uint16_t h = kvqo_f32_to_f16(f);
    if (kvqo_f16_to_f32(h) < f)
        h = (uint16_t)(h + 1u); /* next binary16 value above */
    return h;
}

float kvqo_f16_to_f32(uint16_t h)
{
    uint32_t exp5 = (h >> 10) & 0x1fu;
    uint32_t frac = h & 0x3ffu;
    float v;
    if (exp5 == 0u)
        v = ldexpf((float)frac, -24);
    else if (exp5 == 31u)
        v = frac ? NAN : INFINITY;
    else
        v = ldexpf((float)(1024u + frac), (int)exp5 - 25);
    return (h & 0x8000u) ? -v : v;
}

void kvqo_f32_to_f16_array(const float *x, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = kvqo_f32_to_f16(x[i]);
}

void kvqo_f16_to_f32_array(const uint16_t *h, int64_t n, float *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = kvqo_f16_to_f32(h[i]);
}

float kvqo_bf16_to_f32(uint16_t h)
{
    uint32_t x = (uint32_t)h << 16;
    float v;
    memcpy(&v, &x, sizeof v);
    return v;
}

/* ------------------------------------------------------------------------ */
/* Group-wise asymmetric quantization ([P4] 3.2.2, [P1] 2.1, [P2], [P5] 2.3) */
/* ------------------------------------------------------------------------ */

/* Value of the j-th input element: binary16 or bfloat16 bit patterns, both
 * read exactly into fp32. */
static float kvqo_in(const uint16_t *x, int j, int in_bf16)
{
    return in_bf16 ? kvqo_bf16_to_f32(x[j]) : kvqo_f16_to_f32(x[j]);
}

/*
 * Quantize one group x[0..G-1] (binary16 bit patterns, or bfloat16 with
 * in_bf16) to `bits`-bit codes.  Writes the G unpacked codes, and the fp16
 * bit patterns of s and z.
 */
static void kvqo_quantize_group_in(const uint16_t *x, int in_bf16, int G, int bits,
                                   uint8_t *code, uint16_t *s_out, uint16_t *z_out)
{
    const float qmax = (float)((1 << bits) - 1);

    /* min and max of the group, in fp32 (exact for fp16 and bf16 inputs) */
    float mn = kvqo_in(x, 0, in_bf16);
    float mx = mn;
    for (int j = 1; j < G; ++j) {
        float v = kvqo_in(x, j, in_bf16);
        if (v < mn)
            mn = v;
        if (v > mx)
            mx = v;
    }

    /* scale = (max - min) / (2^bits - 1), floored at 1e-5, stored fp16 (R2) */
    float s32 = (mx - mn) / qmax;
    if (s32 < 1e-5f)
        s32 = 1e-5f;
    uint16_t s16 = kvqo_f32_to_f16_up(s32);
    float s = kvqo_f16_to_f32(s16); /* R3: the stored scale is the one used */

    /* zero point z = round(-min / s) (R1, R4) */
    float zf = rintf(-mn / s) + 0.0f; /* + 0.0f turns -0 into +0 */
    if (zf > 65504.0f)
        zf = 65504.0f;
    if (zf < -65504.0f)
        zf = -65504.0f;
    uint16_t z16 = kvqo_f32_to_f16(zf);
    float z = kvqo_f16_to_f32(z16);

    /* quant(x) = round(x / s) + z, clamped to the code range (R5) */
    for (int j = 0; j < G; ++j) {
        float c = rintf(kvqo_in(x, j, in_bf16) / s) + z;
        if (c < 0.0f)
            c = 0.0f;
        if (c > qmax)
            c = qmax;
        code[j] = (uint8_t)c;
    }
    *s_out = s16;
    *z_out = z16;
}

void kvqo_quantize_group(const uint16_t *x, int G, int bits,
                         uint8_t *code, uint16_t *s_out, uint16_t *z_out)
{
    kvqo_quantize_group_in(x, 0, G, bits, code, s_out, z_out);
}

/*
 * Quantize n_rows token rows of D fp16 values, groups of G along the row
 * (R6).  codes: [n_rows][D*bits/8] packed (R7); meta: [n_rows][D/G][2]
 * binary16 (scale, zero).  bits == 16 stores the fp16 row unchanged and
 * writes no meta (the FP16 class of [P4] 3.1.1).
 */
static void kvqo_quantize_rows_in(const uint16_t *x, int in_bf16, int64_t n_rows, int D,
                                  int G, int bits, uint8_t *codes, uint16_t *meta)
{
    const int64_t row_bytes = (int64_t)D * bits / 8;
    uint8_t *tmp = (uint8_t *)malloc((size_t)G);
    for (int64_t r = 0; r < n_rows; ++r) {
        const uint16_t *xr = x + r * D;
        uint8_t *cr = codes + r * row_bytes;
        if (bits == 16) {
            memcpy(cr, xr, (size_t)row_bytes);
            continue;
        }
        memset(cr, 0, (size_t)row_bytes);
        for (int g = 0; g < D / G; ++g) {
            uint16_t s16, z16;
            kvqo_quantize_group_in(xr + g * G, in_bf16, G, bits, tmp, &s16, &z16);
            meta[(r * (D / G) + g) * 2 + 0] = s16;
            meta[(r * (D / G) + g) * 2 + 1] = z16;
            for (int j = 0; j < G; ++j) {
                int e = g * G + j; /* element index within the row */
                int bitpos = e * bits;
                cr[bitpos / 8] |= (uint8_t)(tmp[j] << (bitpos % 8));
            }
        }
    }
    free(tmp);
}

void kvqo_quantize_rows(const uint16_t *x, int64_t n_rows, int D, int G,
                        int bits, uint8_t *codes, uint16_t *meta)
{
    kvqo_quantize_rows_in(x, 0, n_rows, D, G, bits, codes, meta);
}

/* ------------------------------------------------------------------------ */
/* FP8 E4M3 ([P2'] item 1; R14), written from the format definition.       */
/* ------------------------------------------------------------------------ */

/* Value of an E4M3 code: (-1)^S * 2^(E-7) * (1 + M/8) for E >= 1, and
 * (-1)^S * 2^-6 * M/8 for E = 0; E = 15 with M = 7 is NaN. */
double kvqo_e4m3_to_f64(uint8_t c)
{
    int sgn = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp((double)(8 + m), e - 10);
    return sgn ? -v : v;
}

/* Nearest E4M3 code to an fp32 value, ties to even, magnitudes past the
 * largest finite value (448) saturated to it; NaN gives S.1111.111. */
uint8_t kvqo_f32_to_e4m3(float x)
{
    if (isnan(x))
        return 0x7F;
    uint8_t sgn = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    /* the spacing of E4M3 values around a: 2^-9 below 2^-6, else 2^(e-3) */
    int e = (a > 0.0) ? (int)floor(log2(a)) : -100;
    if (a > 0.0 && ldexp(1.0, e) > a) /* guard log2 rounding */
        e -= 1;
    if (a > 0.0 && ldexp(1.0, e + 1) <= a)
        e += 1;
    double quantum = ldexp(1.0, (e < -6 ? -6 : e) - 3);
    double r = rint(a / quantum) * quantum; /* a / quantum is exact */
    if (r > 448.0)
        r = 448.0;
    if (r == 0.0)
        return sgn;
    int re = (int)floor(log2(r));
    if (ldexp(1.0, re) > r)
        re -= 1;
    if (re < -6)
        return (uint8_t)(sgn | (uint8_t)(r / ldexp(1.0, -9))); /* subnormal */
    int m = (int)(r / ldexp(1.0, re - 3)) - 8;
    return (uint8_t)(sgn | ((re + 7) << 3) | m);
}

/* One group of G binary16 values to E4M3 codes with scale s (R14). */
static void kvqo_quantize_group_fp8_in(const uint16_t *x, int in_bf16, int G, uint8_t *code,
                                       uint16_t *s_out)
{
    float amax = 0.0f;
    for (int j = 0; j < G; ++j) {
        float v = fabsf(kvqo_in(x, j, in_bf16));
        if (v > amax)
            amax = v;
    }
    float s32 = amax / 448.0f;
    if (s32 < 1e-5f)
        s32 = 1e-5f;
    uint16_t s16 = kvqo_f32_to_f16_up(s32);
    float s = kvqo_f16_to_f32(s16);
    for (int j = 0; j < G; ++j)
        code[j] = kvqo_f32_to_e4m3(kvqo_in(x, j, in_bf16) / s);
    *s_out = s16;
}

void kvqo_quantize_group_fp8(const uint16_t *x, int G, uint8_t *code, uint16_t *s_out)
{
    kvqo_quantize_group_fp8_in(x, 0, G, code, s_out);
}

/* Token rows to E4M3 codes (one byte per element) and (s, 0) fp16 pairs per
 * group of G along the row. */
void kvqo_quantize_rows_fp8(const uint16_t *x, int64_t n_rows, int D, int G, uint8_t *codes,
                            uint16_t *meta)
{
    for (int64_t r = 0; r < n_rows; ++r)
        for (int g = 0; g < D / G; ++g) {
            uint16_t s16;
            kvqo_quantize_group_fp8(x + r * D + g * G, G, codes + r * D + g * G, &s16);
            meta[(r * (D / G) + g) * 2 + 0] = s16;
            meta[(r * (D / G) + g) * 2 + 1] = 0; /* zero point 0 */
        }
}

/* ------------------------------------------------------------------------ */
/* FP8 E5M2 ([P2'] item 1; R17), written from the format definition.       */
/* ------------------------------------------------------------------------ */

/* Value of an E5M2 code: (-1)^S * 2^(E-15) * (1 + M/4) for 1 <= E <= 30,
 * (-1)^S * 2^-14 * M/4 for E = 0; E = 31 is infinity (M = 0) or NaN. */
double kvqo_e5m2_to_f64(uint8_t c)
{
    int sgn = c >> 7, e = (c >> 2) & 31, m = c & 3;
    double v;
    if (e == 31)
        v = (m == 0) ? INFINITY : NAN;
    else if (e == 0)
        v = ldexp((double)m, -16);
    else
        v = ldexp((double)(4 + m), e - 17);
    return sgn ? -v : v;
}

/* Nearest E5M2 code to an fp32 value, ties to even, magnitudes past the
 * largest finite value (57344) saturated to it; NaN gives S.11111.11. */
uint8_t kvqo_f32_to_e5m2(float x)
{
    if (isnan(x))
        return 0x7F;
    uint8_t sgn = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    /* the spacing of E5M2 values around a: 2^-16 below 2^-14, else 2^(e-2) */
    int e = (a > 0.0) ? (int)floor(log2(a)) : -100;
    if (a > 0.0 && ldexp(1.0, e) > a) /* guard log2 rounding */
        e -= 1;
    if (a > 0.0 && ldexp(1.0, e + 1) <= a)
        e += 1;
    double quantum = ldexp(1.0, (e < -14 ? -14 : e) - 2);
    double r = rint(a / quantum) * quantum; /* a / quantum is exact */
    if (r > 57344.0)
        r = 57344.0;
    if (r == 0.0)
        return sgn;
    int re = (int)floor(log2(r));
    if (re < -14)
        return (uint8_t)(sgn | (uint8_t)(r / ldexp(1.0, -16))); /* subnormal */
    int m = (int)(r / ldexp(1.0, re - 2)) - 4;
    return (uint8_t)(sgn | ((re + 15) << 2) | m);
}

/* One group of G binary16 values to E5M2 codes with scale s (R17). */
static void kvqo_quantize_group_e5m2_in(const uint16_t *x, int in_bf16, int G, uint8_t *code,
                                       uint16_t *s_out)
{
    float amax = 0.0f;
    for (int j = 0; j < G; ++j) {
        float v = fabsf(kvqo_in(x, j, in_bf16));
        if (v > amax)
            amax = v;
    }
    float s32 = amax / 57344.0f;
    if (s32 < 1e-5f)
        s32 = 1e-5f;
    uint16_t s16 = kvqo_f32_to_f16_up(s32);
    float s = kvqo_f16_to_f32(s16);
    for (int j = 0; j < G; ++j)
        code[j] = kvqo_f32_to_e5m2(kvqo_in(x, j, in_bf16) / s);
    *s_out = s16;
}

void kvqo_quantize_group_e5m2(const uint16_t *x, int G, uint8_t *code, uint16_t *s_out)
{
    kvqo_quantize_group_e5m2_in(x, 0, G, code, s_out);
}

/* Token rows to E5M2 codes and (s, 0) fp16 pairs per group of G. */
void kvqo_quantize_rows_e5m2(const uint16_t *x, int64_t n_rows, int D, int G, uint8_t *codes,
                             uint16_t *meta)
{
    for (int64_t r = 0; r < n_rows; ++r)
        for (int g = 0; g < D / G; ++g) {
            uint16_t s16;
            kvqo_quantize_group_e5m2(x + r * D + g * G, G, codes + r * D + g * G, &s16);
            meta[(r * (D / G) + g) * 2 + 0] = s16;
            meta[(r * (D / G) + g) * 2 + 1] = 0; /* zero point 0 */
        }
}

/* Symmetric INT8 ([P2'] item 2; R15): one group of G binary16 values to
 * two's complement codes with scale s. */
static void kvqo_quantize_group_sym8_in(const uint16_t *x, int in_bf16, int G, uint8_t *code,
                                        uint16_t *s_out)
{
    float amax = 0.0f;
    for (int j = 0; j < G; ++j) {
        float v = fabsf(kvqo_in(x, j, in_bf16));
        if (v > amax)
            amax = v;
    }
    float s32 = amax / 127.0f;
    if (s32 < 1e-5f)
        s32 = 1e-5f;
    uint16_t s16 = kvqo_f32_to_f16_up(s32);
    float s = kvqo_f16_to_f32(s16);
    for (int j = 0; j < G; ++j) {
        float c = rintf(kvqo_in(x, j, in_bf16) / s);
        if (c < -128.0f)
            c = -128.0f;
        if (c > 127.0f)
            c = 127.0f;
        code[j] = (uint8_t)(int8_t)c;
    }
    *s_out = s16;
}

void kvqo_quantize_group_sym8(const uint16_t *x, int G, uint8_t *code, uint16_t *s_out)
{
    kvqo_quantize_group_sym8_in(x, 0, G, code, s_out);
}

/* Token rows to symmetric INT8 codes (one byte per element) and (s, 0) fp16
 * pairs per group of G along the row. */
void kvqo_quantize_rows_sym8(const uint16_t *x, int64_t n_rows, int D, int G, uint8_t *codes,
                             uint16_t *meta)
{
    for (int64_t r = 0; r < n_rows; ++r)
        for (int g = 0; g < D / G; ++g) {
            uint16_t s16;
            kvqo_quantize_group_sym8(x + r * D + g * G, G, codes + r * D + g * G, &s16);
            meta[(r * (D / G) + g) * 2 + 0] = s16;
            meta[(r * (D / G) + g) * 2 + 1] = 0; /* zero point 0 */
        }
}

/*
 * Token rows of D values (binary16 bit patterns, or bfloat16 with in_bf16:
 * the KV-cache page's caches hold either; both read exactly into fp32), one
 * group of G along the row, in any of the token-grouped formats: fmt 0
 * asymmetric integer codes of `bits` bits, 1 FP8 E4M3, 2 symmetric INT8,
 * 3 FP8 E5M2 (bits 8).  codes: [n_rows][D*bits/8]; meta: [n_rows][D/G][2].
 * Every format runs the arithmetic above on the fp32 values unchanged.
 */
void kvqo_quantize_rows_any(const uint16_t *x, int in_bf16, int64_t n_rows, int D, int G,
                            int bits, int fmt, uint8_t *codes, uint16_t *meta)
{
    if (fmt == 0) {
        kvqo_quantize_rows_in(x, in_bf16, n_rows, D, G, bits, codes, meta);
        return;
    }
    for (int64_t r = 0; r < n_rows; ++r)
        for (int g = 0; g < D / G; ++g) {
            uint16_t s16;
            const uint16_t *xg = x + r * D + g * G;
            uint8_t *cg = codes + r * D + g * G;
            if (fmt == 1)
                kvqo_quantize_group_fp8_in(xg, in_bf16, G, cg, &s16);
            else if (fmt == 2)
                kvqo_quantize_group_sym8_in(xg, in_bf16, G, cg, &s16);
            else
                kvqo_quantize_group_e5m2_in(xg, in_bf16, G, cg, &s16);
            meta[(r * (D / G) + g) * 2 + 0] = s16;
            meta[(r * (D / G) + g) * 2 + 1] = 0; /* zero point 0 */
        }
}

/* Oaken group-shift codec ([P1] 3.1, 3.2.2; R18): one row of D binary16
 * values to packed 4-bit codes (D / 2 bytes) and 16 outlier slots. */
#define KVQO_OAKEN_SLOTS 16

void kvqo_oaken_quantize_row_in(const uint16_t *x, int in_bf16, int D, float s_in, int z_in,
                                float s_out, int outer_bits, uint8_t *codes, uint16_t *slots)
{
    const float z = (float)z_in;
    const float t_lo = -z * s_in;
    const float t_hi = (15.0f - z) * s_in;
    const float m_max = (float)((1 << outer_bits) - 1);
    int n_slot = 0;
    memset(codes, 0, (size_t)D / 2);
    for (int i = 0; i < KVQO_OAKEN_SLOTS; ++i)
        slots[i] = 0;
    for (int j = 0; j < D; ++j) {
        const float v = kvqo_in(x, j, in_bf16); /* binary16 or bfloat16 (R19), exact */
        unsigned c;
        int outlier = 0, d = 0;
        if (v > t_hi) { /* outer zone, high side: shift by T_hi */
            const float delta = v - t_hi;
            float m = rintf(delta / s_out);
            if (m > m_max)
                m = m_max;
            c = 15;
            outlier = 1;
            d = (int)m;
        } else if (v < t_lo) { /* outer zone, low side: shift by T_lo */
            const float delta = v - t_lo;
            float m = rintf(-delta / s_out);
            if (m > m_max)
                m = m_max;
            c = 0;
            outlier = 1;
            d = -(int)m;
        } else { /* inner and middle zones: the 4-bit inner quantizer */
            float cf = rintf(v / s_in) + z;
            if (cf < 0.0f)
                cf = 0.0f;
            if (cf > 15.0f)
                cf = 15.0f;
            c = (unsigned)cf;
        }
        codes[j / 2] |= (uint8_t)(c << ((j % 2) * 4));
        if (outlier && n_slot < KVQO_OAKEN_SLOTS) {
            slots[n_slot] = (uint16_t)((unsigned)j | ((unsigned)(uint8_t)(int8_t)d << 8));
            ++n_slot;
        }
    }
}

void kvqo_oaken_quantize_row(const uint16_t *x, int D, float s_in, int z_in, float s_out,
                             int outer_bits, uint8_t *codes, uint16_t *slots)
{
    kvqo_oaken_quantize_row_in(x, 0, D, s_in, z_in, s_out, outer_bits, codes, slots);
}

void kvqo_oaken_quantize_rows_in(const uint16_t *x, int in_bf16, int64_t n_rows, int D,
                                 float s_in, int z_in, float s_out, int outer_bits,
                                 uint8_t *codes, uint16_t *slots)
{
    for (int64_t r = 0; r < n_rows; ++r)
        kvqo_oaken_quantize_row_in(x + r * D, in_bf16, D, s_in, z_in, s_out, outer_bits,
                                   codes + r * (D / 2), slots + r * KVQO_OAKEN_SLOTS);
}

void kvqo_oaken_quantize_rows(const uint16_t *x, int64_t n_rows, int D, float s_in, int z_in,
                              float s_out, int outer_bits, uint8_t *codes, uint16_t *slots)
{
    kvqo_oaken_quantize_rows_in(x, 0, n_rows, D, s_in, z_in, s_out, outer_bits, codes, slots);
}

/* x_hat = (c - z_in) * s_in + d * s_out in fp64 (R18); the dense part is the
 * threshold for an outlier, the slot adds its shifted magnitude. */
void kvqo_oaken_dequantize_rows(const uint8_t *codes, const uint16_t *slots, int64_t n_rows,
                                int D, float s_in, int z_in, float s_out, double *out)
{
    for (int64_t r = 0; r < n_rows; ++r) {
        const uint8_t *row = codes + r * (D / 2);
        double *o = out + r * D;
        for (int j = 0; j < D; ++j) {
            const unsigned c = (row[j / 2] >> ((j % 2) * 4)) & 15u;
            o[j] = ((double)c - (double)z_in) * (double)s_in;
        }
        for (int i = 0; i < KVQO_OAKEN_SLOTS; ++i) {
            const uint16_t w = slots[r * KVQO_OAKEN_SLOTS + i];
            const int j = w & 0xff;
            const int d = (int8_t)(uint8_t)(w >> 8);
            if (j < D)
                o[j] += (double)d * (double)s_out;
        }
    }
}

/* Unpack code e of a packed row (R7). */
static unsigned kvqo_code_at(const uint8_t *row, int e, int bits)
{
    int bitpos = e * bits;
    return (row[bitpos / 8] >> (bitpos % 8)) & ((1u << bits) - 1u);
}

/*
 * Dequantize n_rows packed rows: x_hat = (c - z) * s, evaluated in fp64,
 * where it is exact (|c - z| < 2^17 and s has 11 significant bits); with
 * fmt 1 the codes are E4M3 and x_hat = e4m3(c) * s (R14), with fmt 2 they
 * are two's complement bytes and x_hat = c * s (R15), with fmt 3 E5M2 and
 * x_hat = e5m2(c) * s (R17), all also exact.
 */
void kvqo_dequantize_rows(const uint8_t *codes, const uint16_t *meta,
                          int64_t n_rows, int D, int G, int bits, double *out);

void kvqo_dequantize_rows_fmt(const uint8_t *codes, const uint16_t *meta, int64_t n_rows,
                              int D, int G, int bits, int fmt, double *out)
{
    if (fmt == 1 || fmt == 2 || fmt == 3) {
        for (int64_t r = 0; r < n_rows; ++r)
            for (int e = 0; e < D; ++e) {
                double s = (double)kvqo_f16_to_f32(meta[(r * (D / G) + e / G) * 2 + 0]);
                uint8_t c = codes[r * D + e];
                double v = (fmt == 1) ? kvqo_e4m3_to_f64(c)
                           : (fmt == 3) ? kvqo_e5m2_to_f64(c) : (double)(int8_t)c;
                out[r * D + e] = v * s;
            }
        return;
    }
    kvqo_dequantize_rows(codes, meta, n_rows, D, G, bits, out);
}

void kvqo_dequantize_rows(const uint8_t *codes, const uint16_t *meta,
                          int64_t n_rows, int D, int G, int bits, double *out)
{
    const int64_t row_bytes = (int64_t)D * bits / 8;
    for (int64_t r = 0; r < n_rows; ++r) {
        const uint8_t *cr = codes + r * row_bytes;
        for (int e = 0; e < D; ++e) {
            if (bits == 16) {
                uint16_t h = (uint16_t)(cr[2 * e] | (cr[2 * e + 1] << 8));
                out[r * D + e] = (double)kvqo_f16_to_f32(h);
                continue;
            }
            int g = e / G;
            double s = (double)kvqo_f16_to_f32(meta[(r * (D / G) + g) * 2 + 0]);
            double z = (double)kvqo_f16_to_f32(meta[(r * (D / G) + g) * 2 + 1]);
            double c = (double)kvqo_code_at(cr, e, bits);
            out[r * D + e] = (c - z) * s;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Per-channel K ([P2'] item 2: the Key quantized per channel; R16)         */
/* ------------------------------------------------------------------------ */

/* One block of T token rows x [T][D] (binary16, or bfloat16 when in_bf16,
 * R19) of one (sequence, KV head): the T values of channel d form one
 * group, quantized with the asymmetric formula of R1-R5
 * (kvqo_quantize_group_in).  codes: [T][D*bits/8], packed along each token
 * row (R7); meta: [D][2], the (s, z) of each channel. */
void kvqo_quantize_block_channels_in(const uint16_t *x, int in_bf16, int T, int D, int bits,
                                     uint8_t *codes, uint16_t *meta)
{
    const int64_t row_bytes = (int64_t)D * bits / 8;
    uint16_t *col = (uint16_t *)malloc((size_t)T * sizeof(uint16_t));
    uint8_t *tmp = (uint8_t *)malloc((size_t)T);
    memset(codes, 0, (size_t)(T * row_bytes));
    for (int d = 0; d < D; ++d) {
        for (int t = 0; t < T; ++t)
            col[t] = x[(int64_t)t * D + d];
        uint16_t s16, z16;
        kvqo_quantize_group_in(col, in_bf16, T, bits, tmp, &s16, &z16);
        meta[d * 2 + 0] = s16;
        meta[d * 2 + 1] = z16;
        const int bitpos = d * bits;
        for (int t = 0; t < T; ++t)
            codes[t * row_bytes + bitpos / 8] |= (uint8_t)(tmp[t] << (bitpos % 8));
    }
    free(col);
    free(tmp);
}

/* The binary16 form of the above. */
void kvqo_quantize_block_channels(const uint16_t *x, int T, int D, int bits, uint8_t *codes,
                                  uint16_t *meta)
{
    kvqo_quantize_block_channels_in(x, 0, T, D, bits, codes, meta);
}

/* x_hat[t][d] = (c[t][d] - z_d) * s_d of one block, in fp64 (exact). */
void kvqo_dequantize_block_channels(const uint8_t *codes, const uint16_t *meta, int T, int D,
                                    int bits, double *out)
{
    const int64_t row_bytes = (int64_t)D * bits / 8;
    for (int t = 0; t < T; ++t)
        for (int d = 0; d < D; ++d) {
            double s = (double)kvqo_f16_to_f32(meta[d * 2 + 0]);
            double z = (double)kvqo_f16_to_f32(meta[d * 2 + 1]);
            double c = (double)kvqo_code_at(codes + t * row_bytes, d, bits);
            out[(int64_t)t * D + d] = (c - z) * s;
        }
}

/* ------------------------------------------------------------------------ */
/* Decode attention in fp64 ([P3] 3.2 score; [P4] 3.2.3 chunked + merge)    */
/* ------------------------------------------------------------------------ */

/*
 * One KV head serving g query heads.  q: [g][D], K, V: [L][D] (dequantized),
 * all fp64.  For each head: score_t = scale * sum_j q_j K_tj;
 * p = softmax(score) with the max subtracted; o = sum_t p_t V_t;
 * lse = log sum_t exp(score_t).  L == 0 gives o = 0, lse = -inf.
 */
void kvqo_attention(const double *q, int g, const double *K, const double *V,
                    int64_t L, int D, double scale, double *o, double *lse)
{
    double *score = (double *)malloc((size_t)(L > 0 ? L : 1) * sizeof(double));
    for (int h = 0; h < g; ++h) {
        const double *qh = q + (int64_t)h * D;
        double *oh = o + (int64_t)h * D;
        for (int j = 0; j < D; ++j)
            oh[j] = 0.0;
        if (L == 0) {
            lse[h] = -INFINITY;
            continue;
        }
        double m = -INFINITY;
        for (int64_t t = 0; t < L; ++t) {
            double acc = 0.0;
            for (int j = 0; j < D; ++j)
                acc += qh[j] * K[t * D + j];
            score[t] = scale * acc;
            if (score[t] > m)
                m = score[t];
        }
        double l = 0.0;
        for (int64_t t = 0; t < L; ++t) {
            double p = exp(score[t] - m);
            l += p;
            for (int j = 0; j < D; ++j)
                oh[j] += p * V[t * D + j];
        }
        for (int j = 0; j < D; ++j)
            oh[j] /= l;
        lse[h] = m + log(l);
    }
    free(score);
}

/*
 * The same attention computed block by block and merged by log-sum-exp:
 * tokens are cut at bounds[0] = 0 < bounds[1] < ... < bounds[n_blocks] = L.
 * Block b keeps its own max m_b, sum l_b = sum exp(score - m_b) and
 * unnormalised output u_b = sum exp(score - m_b) V.  The merge takes
 * M = max m_b, l = sum exp(m_b - M) l_b, o = sum exp(m_b - M) u_b / l,
 * lse = M + log l.  Empty blocks contribute nothing.
 */
void kvqo_attention_blocks(const double *q, int g, const double *K,
                           const double *V, int D, double scale,
                           const int64_t *bounds, int n_blocks, double *o,
                           double *lse)
{
    double *mb = (double *)malloc((size_t)n_blocks * sizeof(double));
    double *lb = (double *)malloc((size_t)n_blocks * sizeof(double));
    double *ub = (double *)malloc((size_t)n_blocks * D * sizeof(double));
    for (int h = 0; h < g; ++h) {
        const double *qh = q + (int64_t)h * D;
        for (int b = 0; b < n_blocks; ++b) {
            int64_t t0 = bounds[b], t1 = bounds[b + 1];
            double m = -INFINITY;
            for (int64_t t = t0; t < t1; ++t) {
                double acc = 0.0;
                for (int j = 0; j < D; ++j)
                    acc += qh[j] * K[t * D + j];
                if (scale * acc > m)
                    m = scale * acc;
            }
            double l = 0.0;
            for (int j = 0; j < D; ++j)
                ub[b * D + j] = 0.0;
            for (int64_t t = t0; t < t1; ++t) {
                double acc = 0.0;
                for (int j = 0; j < D; ++j)
                    acc += qh[j] * K[t * D + j];
                double p = exp(scale * acc - m);
                l += p;
                for (int j = 0; j < D; ++j)
                    ub[b * D + j] += p * V[t * D + j];
            }
            mb[b] = m;
            lb[b] = l;
        }
        double M = -INFINITY;
        for (int b = 0; b < n_blocks; ++b)
            if (lb[b] > 0.0 && mb[b] > M)
                M = mb[b];
        double l = 0.0;
        double *oh = o + (int64_t)h * D;
        for (int j = 0; j < D; ++j)
            oh[j] = 0.0;
        for (int b = 0; b < n_blocks; ++b) {
            if (lb[b] == 0.0)
                continue;
            double w = exp(mb[b] - M);
            l += w * lb[b];
            for (int j = 0; j < D; ++j)
                oh[j] += w * ub[b * D + j];
        }
        if (l == 0.0) {
            lse[h] = -INFINITY;
            continue;
        }
        for (int j = 0; j < D; ++j)
            oh[j] /= l;
        lse[h] = M + log(l);
    }
    free(mb);
    free(lb);
    free(ub);
}

/*
 * Decode attention straight from a packed cache of one (sequence, KV head):
 * each token row is dequantized ((c - z) * s in fp64) as it is read, then
 * the fp64 attention above is applied.  q16: [g][D] binary16 or bfloat16
 * bit patterns (q_is_bf16).
 */
void kvqo_attention_packed_fmt(const uint16_t *q16, int q_is_bf16, int g,
                               const uint8_t *k_codes, const uint16_t *k_meta, int k_bits,
                               const uint8_t *v_codes, const uint16_t *v_meta, int v_bits,
                               int fmt, int G, int64_t L, int D, double scale, double *o,
                               double *lse);

void kvqo_attention_packed(const uint16_t *q16, int q_is_bf16, int g,
                           const uint8_t *k_codes, const uint16_t *k_meta,
                           int k_bits, const uint8_t *v_codes,
                           const uint16_t *v_meta, int v_bits, int G,
                           int64_t L, int D, double scale, double *o,
                           double *lse)
{
    kvqo_attention_packed_fmt(q16, q_is_bf16, g, k_codes, k_meta, k_bits, v_codes, v_meta,
                              v_bits, 0, G, L, D, scale, o, lse);
}

/* The same with a code format for K and V (fmt as in the header). */
void kvqo_attention_packed_fmt(const uint16_t *q16, int q_is_bf16, int g,
                               const uint8_t *k_codes, const uint16_t *k_meta, int k_bits,
                               const uint8_t *v_codes, const uint16_t *v_meta, int v_bits,
                               int fmt, int G, int64_t L, int D, double scale, double *o,
                               double *lse)
{
    double *q = (double *)malloc((size_t)g * D * sizeof(double));
    for (int64_t i = 0; i < (int64_t)g * D; ++i)
        q[i] = q_is_bf16 ? (double)kvqo_bf16_to_f32(q16[i])
                         : (double)kvqo_f16_to_f32(q16[i]);
    double *K = (double *)malloc((size_t)(L > 0 ? L : 1) * D * sizeof(double));
    double *V = (double *)malloc((size_t)(L > 0 ? L : 1) * D * sizeof(double));
    int Gk = (k_bits == 16) ? D : G;
    int Gv = (v_bits == 16) ? D : G;
    kvqo_dequantize_rows_fmt(k_codes, k_meta, L, D, Gk, k_bits, fmt, K);
    kvqo_dequantize_rows_fmt(v_codes, v_meta, L, D, Gv, v_bits, fmt, V);
    kvqo_attention(q, g, K, V, L, D, scale, o, lse);
    free(q);
    free(K);
    free(V);
}

/* ------------------------------------------------------------------------ */
/* Cocktail chunk-level bit-width search and reorder ([P4] 3.1.1, 3.1.2)   */
/* ------------------------------------------------------------------------ */

/*
 * sim(q, c_i) = (q . c_i) / (||q|| * ||c_i||) in fp64, every sum taken in
 * index order with separate multiply and add.  T_low = s_min + (s_max -
 * s_min) * alpha, T_high = s_max - (s_max - s_min) * beta.  Class (R8):
 * 16 (FP16) if sim > T_high, 4 (INT4) if T_low < sim <= T_high, else 2.
 */
void kvqo_chunk_assign(const float *emb, const float *qemb, int n_chunks,
                       int dim, double alpha, double beta, double *sim,
                       uint8_t *bits_out)
{
    double qq = 0.0;
    for (int d = 0; d < dim; ++d)
        qq += (double)qemb[d] * (double)qemb[d];
    double nq = sqrt(qq);
    double s_min = INFINITY, s_max = -INFINITY;
    for (int i = 0; i < n_chunks; ++i) {
        const float *c = emb + (int64_t)i * dim;
        double dot = 0.0, cc = 0.0;
        for (int d = 0; d < dim; ++d) {
            dot += (double)qemb[d] * (double)c[d];
            cc += (double)c[d] * (double)c[d];
        }
        sim[i] = dot / (nq * sqrt(cc));
        if (sim[i] < s_min)
            s_min = sim[i];
        if (sim[i] > s_max)
            s_max = sim[i];
    }
    double span = s_max - s_min;
    double t_low = s_min + span * alpha;
    double t_high = s_max - span * beta;
    for (int i = 0; i < n_chunks; ++i) {
        if (sim[i] > t_high)
            bits_out[i] = 16;
        else if (sim[i] > t_low)
            bits_out[i] = 4;
        else
            bits_out[i] = 2;
    }
}

/*
 * Stable partition of chunk indices by class (R9).  perm[k] is the original
 * index of the chunk at position k of the reordered cache; counts[0..2] are
 * the numbers of FP16, INT4 and INT2 chunks.
 */
void kvqo_chunk_partition(const uint8_t *bits, int n_chunks, int32_t *perm,
                          int32_t *counts)
{
    static const uint8_t order[3] = {16, 4, 2};
    int k = 0;
    for (int c = 0; c < 3; ++c) {
        counts[c] = 0;
        for (int i = 0; i < n_chunks; ++i) {
            if (bits[i] == order[c]) {
                perm[k++] = i;
                counts[c] += 1;
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* KV-cache size ([P2] formula; [P5] 1.2 worked example)                    */
/* ------------------------------------------------------------------------ */

/* Number of cached K and V elements: 2 * layers * kv_heads * head_dim *
 * seq_len * batch. */
uint64_t kvqo_kv_elements(uint64_t layers, uint64_t kv_heads,
                          uint64_t head_dim, uint64_t seq_len, uint64_t batch)
{
    return 2u * layers * kv_heads * head_dim * seq_len * batch;
}
