/*
 * kvq_oracle.c -- plain, slow, single-threaded CPU oracle of the asymmetric
 * low-bit KV cache and of decode attention over it.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and
 * the bench's CPU-baseline leg may load or run this code.  It shares no code,
 * header, table or helper with the CUDA library; the two meet only through
 * the seeded inputs both receive.
 *
 * What it follows (pages cited by title and section):
 *  - "KV cache compression: quantization, eviction and sparse attention"
 *    (arganzheng.life), section 3.2 "KIVI": keys are quantized per channel,
 *    the range taken over a group of G tokens; values per token, the range
 *    taken over the channels; the most recent R tokens stay full precision
 *    until a whole group can be quantized, and attention is computed over
 *    both parts.  Section 3.4: paged blocks carry their own scales.
 *    Section 3.1: FP8 E4M3 with a per-head static scale.  Section 8.1: the
 *    byte count of a KV cache.
 *  - "KV Cache lab" (door4ai-lab), experiment 01: scale = (max - min) /
 *    (2^bits - 1), zero = min, every value snaps to the nearest grid line,
 *    only the integer line index is stored.
 *  - "KV cache compression" (jaedaily.cn), formulas section: the per-channel
 *    key and per-token value quantizers k^ = round((k - z)/s)*s + z, and the
 *    byte formula M_KV = 2 L H_kv n d_h b; process section: the cache has two
 *    regions, recent tokens in FP16 and the rest quantized.
 *
 * Readings where the pages leave a step open (stated here so the code can be
 * checked against them):
 *  - Quantizer arithmetic is IEEE fp32, each operation rounded on its own:
 *      scale32 = (max - min) / (2^b - 1);  s = fp16(scale32);
 *      z = fp16(min + 0.0f)  (the +0 turns -0 into +0);
 *      inv = s > 0 ? 1/s : 0;  code = clamp(rint_half_even((x - z) * inv)).
 *    The division of the formula is taken as a multiply by the reciprocal of
 *    the stored fp16 scale (oracle_encode_truediv keeps the literal division
 *    as a diagnostic).  A NaN quotient becomes code 0.
 *  - scale and zero are stored as fp16 (section 8.1 counts "FP16 x2" per
 *    group); codes are computed against the fp16-rounded scale and zero.
 *  - A constant group (max == min) gets scale 0, all codes 0, and decodes to
 *    exactly the zero point.
 *  - Residual window: n_q = G * floor(max(n - R, 0) / G) tokens are
 *    quantized and tokens [n_q, n) stay bf16 in a ring of R + G slots indexed
 *    by token mod (R + G); a group is flushed when the window reaches R + G.
 *  - Dequantized values and attention are evaluated in double.
 *  - FP8: S = amax / 448 in fp32 (1 if amax is 0); code = e4m3(x * (1/S))
 *    with round-to-nearest-even and saturation to +-448 (OCP "E4M3FN":
 *    bias 7, no infinities, S.1111.111 is NaN).  Values decode to e4m3 * S.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Scalar formats                                                            */
/* ------------------------------------------------------------------------ */

static inline uint32_t f32_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static inline float bits_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

/* bf16 is the upper half of an IEEE binary32: widening is exact. */
float oracle_bf16_to_f32(uint16_t b) { return bits_f32((uint32_t)b << 16); }

/* IEEE binary16 value of a bit pattern. */
float oracle_f16_to_f32(uint16_t h)
{
    const int sign = (h >> 15) & 1, e = (h >> 10) & 31, m = h & 1023;
    double v;
    if (e == 0) v = ldexp((double)m, -24);                  /* zero / subnormal */
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = ldexp((double)(1024 + m), e - 25);             /* (1 + m/1024) 2^(e-15) */
    return (float)(sign ? -v : v);
}

/* binary32 -> binary16, round to nearest, ties to even; overflow -> inf. */
uint16_t oracle_f32_to_f16(float f)
{
    const uint16_t sign = (f32_bits(f) >> 16) & 0x8000u;
    if (isnan(f)) return sign | 0x7E00u;
    const double a = fabs((double)f);
    /* 65520 is the midpoint between the largest finite (65504) and 2^16;
     * it rounds to the even neighbour 2^16, i.e. overflows. */
    if (a >= 65520.0) return sign | 0x7C00u;
    int e;                                   /* a in [2^e, 2^(e+1)), clamped at -14 */
    if (a < 0x1p-14) e = -14;
    else { (void)frexp(a, &e); e -= 1; }
    const double quantum = ldexp(1.0, e - 10);          /* spacing of binade e */
    double k = nearbyint(a / quantum);                  /* exact quotient, ties to even */
    if (e == -14 && k < 1024.0) return sign | (uint16_t)k;      /* subnormal or zero */
    if (k == 2048.0) { k = 1024.0; e += 1; }            /* carried into the next binade */
    return sign | (uint16_t)(((e + 15) << 10) | ((int)k - 1024));
}

/* OCP FP8 E4M3 ("FN"): bias 7, exponent 0 subnormal, S.1111.111 NaN. */
float oracle_e4m3_decode(uint8_t c)
{
    const int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) v = NAN;
    else if (e == 0) v = ldexp((double)m, -9);          /* m/8 * 2^-6 */
    else v = ldexp((double)(8 + m), e - 10);            /* (1 + m/8) 2^(e-7) */
    return (float)(sign ? -v : v);
}

/* binary32 -> E4M3, round to nearest even, saturating to +-448. */
uint8_t oracle_e4m3_encode(float y)
{
    const uint8_t sign = (f32_bits(y) >> 24) & 0x80u;
    if (isnan(y)) return 0x7Fu;
    const double a = fabs((double)y);
    if (a >= 448.0) return sign | 0x7Eu;
    int e;
    if (a < 0x1p-6) e = -6;
    else { (void)frexp(a, &e); e -= 1; }
    const double quantum = ldexp(1.0, e - 3);
    double k = nearbyint(a / quantum);
    if (e == -6 && k < 8.0) return sign | (uint8_t)k;
    if (k == 16.0) { k = 8.0; e += 1; }
    return sign | (uint8_t)(((e + 7) << 3) | ((int)k - 8));
}

/* The same encoding by exhaustive search over the 127 non-negative finite
 * codes: nearest value, ties to the even code.  Used to pin the one above. */
uint8_t oracle_e4m3_encode_bruteforce(float y)
{
    const uint8_t sign = (f32_bits(y) >> 24) & 0x80u;
    if (isnan(y)) return 0x7Fu;
    const double a = fabs((double)y);
    if (a >= 448.0) return sign | 0x7Eu;
    int best = 0;
    double best_d = INFINITY;
    for (int c = 0; c <= 0x7E; ++c) {
        const double d = fabs((double)oracle_e4m3_decode((uint8_t)c) - a);
        if (d < best_d || (d == best_d && (c & 1) == 0)) { best = c; best_d = d; }
    }
    return sign | (uint8_t)best;
}

/* ------------------------------------------------------------------------ */
/* The asymmetric min/max quantizer                                          */
/* ------------------------------------------------------------------------ */

void oracle_quant_params(float mn, float mx, int32_t bits, uint16_t *s16, uint16_t *z16)
{
    const float levels = (float)((1 << bits) - 1);
    const float scale32 = (mx - mn) / levels;
    *s16 = oracle_f32_to_f16(scale32);
    *z16 = oracle_f32_to_f16(mn + 0.0f);
}

static inline uint8_t clamp_code(float r, int32_t bits)
{
    const float top = (float)((1 << bits) - 1);
    if (!(r >= 0.0f)) return 0;          /* negative or NaN */
    if (r > top) return (uint8_t)top;
    return (uint8_t)r;
}

uint8_t oracle_encode(float x, uint16_t s16, uint16_t z16, int32_t bits)
{
    const float s = oracle_f16_to_f32(s16);
    const float z = oracle_f16_to_f32(z16);
    const float inv = (s > 0.0f) ? 1.0f / s : 0.0f;
    const float diff = x - z;
    const float t = diff * inv;
    return clamp_code(nearbyintf(t), bits);
}

/* Literal reading of round((x - z) / s): IEEE division by the stored scale. */
uint8_t oracle_encode_truediv(float x, uint16_t s16, uint16_t z16, int32_t bits)
{
    const float s = oracle_f16_to_f32(s16);
    const float z = oracle_f16_to_f32(z16);
    if (!(s > 0.0f)) return 0;
    return clamp_code(nearbyintf((x - z) / s), bits);
}

/* Quantize one set of `count` values x[i*stride] (fp32) with one scale and
 * one zero: the unit of every granularity (a K channel over a token group,
 * a V token over its channels, or anything else a check wants). */
void oracle_quantize_set(const float *x, int64_t count, int64_t stride, int32_t bits,
                         uint8_t *codes, int64_t code_stride, uint16_t *s16, uint16_t *z16)
{
    float mn = INFINITY, mx = -INFINITY;
    for (int64_t i = 0; i < count; ++i) {
        mn = fminf(mn, x[i * stride]);
        mx = fmaxf(mx, x[i * stride]);
    }
    oracle_quant_params(mn, mx, bits, s16, z16);
    for (int64_t i = 0; i < count; ++i)
        codes[i * code_stride] = oracle_encode(x[i * stride], *s16, *z16, bits);
}

/* Dequantized value code * s + z, exact in double. */
double oracle_dequant(uint8_t code, uint16_t s16, uint16_t z16)
{
    return (double)code * (double)oracle_f16_to_f32(s16) + (double)oracle_f16_to_f32(z16);
}

/* Canonical packing of one row of codes along the channel axis:
 * 4-bit: byte j holds channel 2j in bits 0-3 and channel 2j+1 in bits 4-7;
 * 2-bit: byte j holds channel 4j+i in bits 2i..2i+1. */
void oracle_pack(const uint8_t *codes, int64_t count, int32_t bits, uint8_t *out)
{
    const int per = 8 / bits;
    for (int64_t j = 0; j < count / per; ++j) {
        uint8_t byte = 0;
        for (int i = 0; i < per; ++i) byte |= (uint8_t)(codes[j * per + i] << (bits * i));
        out[j] = byte;
    }
}

void oracle_unpack(const uint8_t *packed, int64_t count, int32_t bits, uint8_t *codes)
{
    const int per = 8 / bits;
    const uint8_t mask = (uint8_t)((1 << bits) - 1);
    for (int64_t c = 0; c < count; ++c)
        codes[c] = (packed[c / per] >> (bits * (c % per))) & mask;
}

/* Bytes of a KV cache: 2 (K and V) * layers * kv heads * tokens * head_dim
 * * bytes per element, with the element size given in bits. */
int64_t oracle_kv_bytes(int64_t layers, int64_t kv_heads, int64_t tokens, int64_t head_dim,
                        int64_t bits_per_elem)
{
    return 2 * layers * kv_heads * tokens * head_dim * bits_per_elem / 8;
}

/* ------------------------------------------------------------------------ */
/* One (sequence, kv head) unit of the cache                                 */
/* ------------------------------------------------------------------------ */

typedef struct {
    int32_t bits;        /* 2 or 4 */
    int32_t D;           /* head dim */
    int32_t G;           /* K group (tokens) */
    int32_t R;           /* residual window */
    int32_t cap;         /* capacity (tokens), multiple of G */
    int32_t n;           /* tokens held */
    int32_t n_q;         /* tokens quantized */
    uint8_t *k_codes;    /* [cap][D], one code per byte */
    uint16_t *k_scale;   /* [cap/G][D] fp16 bits */
    uint16_t *k_zero;    /* [cap/G][D] fp16 bits */
    uint8_t *v_codes;    /* [cap][D] */
    uint16_t *v_scale;   /* [cap] */
    uint16_t *v_zero;    /* [cap] */
    uint16_t *k_ring;    /* [R+G][D] bf16 bits, slot = token mod (R+G) */
    uint16_t *v_ring;
    /* Mixed 2/4-bit cache (both NULL for a uniform one): the bit width of
     * every key/value group, and the class (2 or 4) of the token in every
     * window slot. */
    uint8_t *group_bits; /* [cap/G] */
    uint8_t *ring_class; /* [R+G] */
    /* Dense-and-sparse cache (all NULL otherwise): every key set (channel
     * of a group) and value set (token) holds its largest-magnitude value
     * aside, exactly (bf16 bits), with its position in the set. */
    uint16_t *k_out;     /* [cap/G][D] */
    uint8_t *k_out_idx;  /* [cap/G][D]: token within the group */
    uint16_t *v_out;     /* [cap] */
    uint8_t *v_out_idx;  /* [cap]: channel */
} oracle_unit;

/* Quantize tokens [t0, t0+G) whose K and V rows are k_rows[i*ld], v_rows[i*ld]
 * (bf16 bits): one K group (per channel) and G V tokens (per token). */
/* KVQuant's dense-and-sparse split ("KV Cache lab", door4ai-lab, after
 * experiment 03: the few extreme values are kept apart in fp16 as a sparse
 * matrix and the rest is quantized; experiment 01 shows why: one large value
 * stretches the scale of its whole set).  Reading: in every set the one
 * value of largest magnitude (the first such, on ties; NaN counts as smaller
 * than any number) is kept aside exactly
 * as its bf16 input, with its index in the set; the set's min/max and
 * codes are taken over the other values, and the kept value's own code is 0.
 * raw: the set's bf16 bits (for the kept value); x: the same as fp32.
 * Returns the kept index. */
int32_t oracle_quantize_set_sparse(const float *x, const uint16_t *raw, int64_t count, int64_t stride,
                                   int32_t bits, uint8_t *codes, int64_t code_stride, uint16_t *s16, uint16_t *z16,
                                   uint16_t *out_val)
{
    /* magnitude order for the kept value: a NaN counts below every number */
    int64_t im = 0;
    float best = isnan(x[0]) ? -1.0f : fabsf(x[0]);
    for (int64_t i = 1; i < count; ++i) {
        const float m = isnan(x[i * stride]) ? -1.0f : fabsf(x[i * stride]);
        if (m > best) { im = i; best = m; }
    }
    float mn = INFINITY, mx = -INFINITY;
    for (int64_t i = 0; i < count; ++i) {
        if (i == im) continue;
        mn = fminf(mn, x[i * stride]);
        mx = fmaxf(mx, x[i * stride]);
    }
    oracle_quant_params(mn, mx, bits, s16, z16);
    for (int64_t i = 0; i < count; ++i)
        codes[i * code_stride] = i == im ? 0 : oracle_encode(x[i * stride], *s16, *z16, bits);
    *out_val = raw[im * stride];
    return (int32_t)im;
}

static void quantize_group(oracle_unit *u, int32_t t0, const uint16_t *const *k_rows,
                           const uint16_t *const *v_rows)
{
    const int32_t D = u->D, G = u->G, g = t0 / G;
    const int32_t bits = u->group_bits ? u->group_bits[g] : u->bits;
    float col[4096];
    float row[4096];
    uint16_t rawc[4096];
    for (int32_t c = 0; c < D; ++c) {
        for (int32_t i = 0; i < G; ++i) col[i] = oracle_bf16_to_f32(k_rows[i][c]);
        if (u->k_out) {
            for (int32_t i = 0; i < G; ++i) rawc[i] = k_rows[i][c];
            u->k_out_idx[(int64_t)g * D + c] = (uint8_t)oracle_quantize_set_sparse(
                col, rawc, G, 1, bits, &u->k_codes[(int64_t)t0 * D + c], D, &u->k_scale[(int64_t)g * D + c],
                &u->k_zero[(int64_t)g * D + c], &u->k_out[(int64_t)g * D + c]);
        } else {
            oracle_quantize_set(col, G, 1, bits, &u->k_codes[(int64_t)t0 * D + c], D,
                                &u->k_scale[(int64_t)g * D + c], &u->k_zero[(int64_t)g * D + c]);
        }
    }
    for (int32_t i = 0; i < G; ++i) {
        for (int32_t c = 0; c < D; ++c) row[c] = oracle_bf16_to_f32(v_rows[i][c]);
        if (u->v_out) {
            u->v_out_idx[t0 + i] = (uint8_t)oracle_quantize_set_sparse(
                row, v_rows[i], D, 1, bits, &u->v_codes[(int64_t)(t0 + i) * D], 1, &u->v_scale[t0 + i],
                &u->v_zero[t0 + i], &u->v_out[t0 + i]);
        } else {
            oracle_quantize_set(row, D, 1, bits, &u->v_codes[(int64_t)(t0 + i) * D], 1,
                                &u->v_scale[t0 + i], &u->v_zero[t0 + i]);
        }
    }
}

static inline int32_t quantized_prefix(int32_t n, int32_t R, int32_t G)
{
    const int32_t over = n - R > 0 ? n - R : 0;
    return G * (over / G);
}

/* Fill the unit from n tokens; row t of K is k[t*ld .. t*ld+D). Returns 0,
 * or -1 if n exceeds the capacity or the group is too large. */
int32_t oracle_unit_prefill(oracle_unit *u, const uint16_t *k, const uint16_t *v, int64_t ld, int32_t n)
{
    if (n < 0 || n > u->cap || u->G > 4096 || u->D > 4096) return -1;
    const int32_t D = u->D, G = u->G, W = u->R + u->G;
    const int32_t n_q = quantized_prefix(n, u->R, G);
    const uint16_t *kr[4096], *vr[4096];
    for (int32_t t0 = 0; t0 < n_q; t0 += G) {
        for (int32_t i = 0; i < G; ++i) { kr[i] = k + (int64_t)(t0 + i) * ld; vr[i] = v + (int64_t)(t0 + i) * ld; }
        quantize_group(u, t0, kr, vr);
    }
    for (int32_t t = n_q; t < n; ++t) {
        memcpy(&u->k_ring[(int64_t)(t % W) * D], k + (int64_t)t * ld, (size_t)D * 2);
        memcpy(&u->v_ring[(int64_t)(t % W) * D], v + (int64_t)t * ld, (size_t)D * 2);
    }
    u->n = n;
    u->n_q = n_q;
    return 0;
}

/* Write one token into the window.  Returns -1 (and changes nothing) when
 * the capacity or the window is full. */
int32_t oracle_unit_append(oracle_unit *u, const uint16_t *k_tok, const uint16_t *v_tok)
{
    const int32_t W = u->R + u->G;
    if (u->n >= u->cap || u->n - u->n_q >= W) return -1;
    memcpy(&u->k_ring[(int64_t)(u->n % W) * u->D], k_tok, (size_t)u->D * 2);
    memcpy(&u->v_ring[(int64_t)(u->n % W) * u->D], v_tok, (size_t)u->D * 2);
    u->n += 1;
    return 0;
}

/* Quantize the oldest G window tokens once the window holds R + G of them.
 * Returns 1 if a group was quantized, else 0.  A mixed cache stores the
 * group at the widest class of its G tokens. */
int32_t oracle_unit_flush(oracle_unit *u)
{
    const int32_t G = u->G, W = u->R + u->G, D = u->D;
    if (u->n - u->n_q != W) return 0;
    if (u->group_bits) {
        int32_t bits = 2;
        for (int32_t i = 0; i < G; ++i)
            if (u->ring_class[(u->n_q + i) % W] == 4) bits = 4;
        u->group_bits[u->n_q / G] = (uint8_t)bits;
    }
    const uint16_t *kr[4096], *vr[4096];
    for (int32_t i = 0; i < G; ++i) {
        const int32_t slot = (u->n_q + i) % W;
        kr[i] = &u->k_ring[(int64_t)slot * D];
        vr[i] = &u->v_ring[(int64_t)slot * D];
    }
    quantize_group(u, u->n_q, kr, vr);
    u->n_q += G;
    return 1;
}

/* ------------------------------------------------------------------------ */
/* Mixed 2/4-bit cache by token class                                        */
/* ------------------------------------------------------------------------ */

/* "KV cache compression" (miraclefarms wiki), TriAxialKV: tokens are sorted
 * into classes (modality, time, meaning) and each class is kept at 2 or 4
 * bits, most tokens at 2.  Reading for a per-channel key cache: every token
 * carries a class 2 or 4 (an input); a key group, and the values of its G
 * tokens, are stored at the widest class among its tokens, so that the
 * per-channel ranges of a group share one grid.  The window keeps each
 * token's class until its group is flushed.  tok_class: [n], 2 or 4. */
int32_t oracle_unit_prefill_mixed(oracle_unit *u, const uint16_t *k, const uint16_t *v, int64_t ld, int32_t n,
                                  const uint8_t *tok_class)
{
    if (!u->group_bits || !u->ring_class) return -1;
    if (n < 0 || n > u->cap || u->G > 4096 || u->D > 4096) return -1;
    const int32_t G = u->G, W = u->R + u->G;
    const int32_t n_q = quantized_prefix(n, u->R, G);
    for (int32_t g = 0; g < n_q / G; ++g) {
        int32_t bits = 2;
        for (int32_t i = 0; i < G; ++i)
            if (tok_class[g * G + i] == 4) bits = 4;
        u->group_bits[g] = (uint8_t)bits;
    }
    for (int32_t t = n_q; t < n; ++t) u->ring_class[t % W] = tok_class[t];
    return oracle_unit_prefill(u, k, v, ld, n);
}

/* Append one token of class cls (2 or 4) to a mixed cache's window. */
int32_t oracle_unit_append_mixed(oracle_unit *u, const uint16_t *k_tok, const uint16_t *v_tok, int32_t cls)
{
    const int32_t W = u->R + u->G, slot = u->n % W;
    if (!u->ring_class) return -1;
    const int32_t rc = oracle_unit_append(u, k_tok, v_tok);
    if (rc == 0) u->ring_class[slot] = (uint8_t)cls;
    return rc;
}

/* K^ and V^ of every held token, in double: dequantized codes for [0, n_q),
 * the bf16 window for [n_q, n).  khat, vhat: [n][D]. */
void oracle_unit_materialize(const oracle_unit *u, double *khat, double *vhat)
{
    const int32_t D = u->D, G = u->G, W = u->R + u->G;
    for (int32_t t = 0; t < u->n; ++t) {
        for (int32_t c = 0; c < D; ++c) {
            double kv, vv;
            if (t < u->n_q) {
                const int64_t g = t / G;
                kv = oracle_dequant(u->k_codes[(int64_t)t * D + c], u->k_scale[g * D + c], u->k_zero[g * D + c]);
                vv = oracle_dequant(u->v_codes[(int64_t)t * D + c], u->v_scale[t], u->v_zero[t]);
                /* dense-and-sparse: the kept value replaces the dense one */
                if (u->k_out && u->k_out_idx[g * D + c] == t - g * G) kv = oracle_bf16_to_f32(u->k_out[g * D + c]);
                if (u->v_out && u->v_out_idx[t] == c) vv = oracle_bf16_to_f32(u->v_out[t]);
            } else {
                kv = oracle_bf16_to_f32(u->k_ring[(int64_t)(t % W) * D + c]);
                vv = oracle_bf16_to_f32(u->v_ring[(int64_t)(t % W) * D + c]);
            }
            khat[(int64_t)t * D + c] = kv;
            vhat[(int64_t)t * D + c] = vv;
        }
    }
}

/* Softmax attention of nh query rows q[h*q_ld..] (bf16 bits) over n rows of
 * K^ and V^ (double): out[h][c] = sum_t p_t v_t[c], p = softmax(scale * q.k_t).
 * logits: optional [nh][n] output of the scaled logits. */
void oracle_attend(const double *khat, const double *vhat, int32_t n, int32_t D,
                   const uint16_t *q, int64_t q_ld, int32_t nh, double scale,
                   double *out, double *logits_out, double *work)
{
    for (int32_t h = 0; h < nh; ++h) {
        double *lg = work;
        double mx = -INFINITY;
        for (int32_t t = 0; t < n; ++t) {
            double dot = 0.0;
            for (int32_t c = 0; c < D; ++c)
                dot += (double)oracle_bf16_to_f32(q[h * q_ld + c]) * khat[(int64_t)t * D + c];
            lg[t] = dot * scale;
            if (lg[t] > mx) mx = lg[t];
        }
        if (logits_out) memcpy(&logits_out[(int64_t)h * n], lg, (size_t)n * sizeof(double));
        double denom = 0.0;
        for (int32_t t = 0; t < n; ++t) { lg[t] = exp(lg[t] - mx); denom += lg[t]; }
        for (int32_t c = 0; c < D; ++c) {
            double acc = 0.0;
            for (int32_t t = 0; t < n; ++t) acc += lg[t] * vhat[(int64_t)t * D + c];
            out[(int64_t)h * D + c] = n > 0 ? acc / denom : 0.0;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Keys quantized before RoPE, rotated when read                             */
/* ------------------------------------------------------------------------ */

/* RoPE rotates adjacent channel pairs ("KV cache compression"
 * (arganzheng.life) section 2.1: a pairwise rotation that keeps each pair's
 * norm; "KV Cache lab", experiment 03: adjacent dimensions as a plane).
 * Reading: pair (2i, 2i+1) turns by the angle position * theta^(-2i/D),
 *   x'_2i = x_2i cos a - x_2i+1 sin a,   x'_2i+1 = x_2i sin a + x_2i+1 cos a,
 * all in double.  Row t of x [n][D] is at position pos0 + t. */
void oracle_rope_rows(double *x, int64_t n, int32_t D, double theta, int64_t pos0)
{
    for (int64_t t = 0; t < n; ++t) {
        const double pos = (double)(pos0 + t);
        for (int32_t i = 0; i < D / 2; ++i) {
            const double a = pos * pow(theta, -2.0 * (double)i / (double)D);
            const double c = cos(a), s = sin(a);
            const double x0 = x[t * D + 2 * i], x1 = x[t * D + 2 * i + 1];
            x[t * D + 2 * i] = x0 * c - x1 * s;
            x[t * D + 2 * i + 1] = x0 * s + x1 * c;
        }
    }
}

/* KVQuant's pre-RoPE key quantization (arganzheng.life section 3.3: keys
 * are quantized before RoPE, whose rotation would otherwise move the
 * outlier channels' values from token to token and widen the per-channel
 * ranges, and RoPE is applied when the keys are read).  The unit holds
 * un-rotated keys (quantized part and window alike); decode dequantizes,
 * rotates key t by its position t, and attends.  work: 2*n*D + n doubles. */
void oracle_unit_decode_rope(const oracle_unit *u, const uint16_t *q, int64_t q_ld, int32_t nh,
                             double scale, double theta, double *out, double *work)
{
    double *khat = work, *vhat = work + (int64_t)u->n * u->D, *lg = vhat + (int64_t)u->n * u->D;
    oracle_unit_materialize(u, khat, vhat);
    oracle_rope_rows(khat, u->n, u->D, theta, 0);
    oracle_attend(khat, vhat, u->n, u->D, q, q_ld, nh, scale, out, NULL, lg);
}

/* Decode attention of one unit: the nh query heads that share this kv head.
 * work: at least 2*n*D + n doubles. */
void oracle_unit_decode(const oracle_unit *u, const uint16_t *q, int64_t q_ld, int32_t nh,
                        double scale, double *out, double *work)
{
    double *khat = work, *vhat = work + (int64_t)u->n * u->D, *lg = vhat + (int64_t)u->n * u->D;
    oracle_unit_materialize(u, khat, vhat);
    oracle_attend(khat, vhat, u->n, u->D, q, q_ld, nh, scale, out, NULL, lg);
}

/* ------------------------------------------------------------------------ */
/* FP8-E4M3 cache with a static per-(kv head, K|V) scale                     */
/* ------------------------------------------------------------------------ */

/* S = amax / 448 in fp32; 1 when amax is 0 (or not finite). */
float oracle_fp8_scale(float amax)
{
    if (!(amax > 0.0f) || isinf(amax)) return 1.0f;
    return amax / 448.0f;
}

/* amax of |x| over n rows x[t*ld .. t*ld+D) (bf16 bits), folded into *amax. */
void oracle_amax_rows(const uint16_t *x, int64_t ld, int64_t n, int32_t D, float *amax)
{
    float a = *amax;
    for (int64_t t = 0; t < n; ++t)
        for (int32_t c = 0; c < D; ++c) a = fmaxf(a, fabsf(oracle_bf16_to_f32(x[t * ld + c])));
    *amax = a;
}

/* codes[t*D + c] = e4m3(x * (1/S)), inv and product each rounded in fp32. */
void oracle_fp8_encode_rows(const uint16_t *x, int64_t ld, int64_t n, int32_t D, float S, uint8_t *codes)
{
    const float inv = 1.0f / S;
    for (int64_t t = 0; t < n; ++t)
        for (int32_t c = 0; c < D; ++c) {
            const float y = oracle_bf16_to_f32(x[t * ld + c]) * inv;
            codes[t * D + c] = oracle_e4m3_encode(y);
        }
}

/* Decode attention over an FP8 unit: n tokens of codes [n][D]. */
void oracle_fp8_decode(const uint8_t *k_codes, const uint8_t *v_codes, int32_t n, int32_t D,
                       float Sk, float Sv, const uint16_t *q, int64_t q_ld, int32_t nh,
                       double scale, double *out, double *work)
{
    double *khat = work, *vhat = work + (int64_t)n * D, *lg = vhat + (int64_t)n * D;
    for (int64_t i = 0; i < (int64_t)n * D; ++i) {
        khat[i] = (double)oracle_e4m3_decode(k_codes[i]) * (double)Sk;
        vhat[i] = (double)oracle_e4m3_decode(v_codes[i]) * (double)Sv;
    }
    oracle_attend(khat, vhat, n, D, q, q_ld, nh, scale, out, NULL, lg);
}

/* ------------------------------------------------------------------------ */
/* INT8 per-token dynamic cache                                              */
/* ------------------------------------------------------------------------ */

/* "KV cache compression" (arganzheng.life), section 3.1: besides FP8 with a
 * static scale, an 8-bit KV cache can be INT8 per token with a dynamic
 * scale; its 255 levels leave the ordinary channels of a key a dozen-odd
 * levels even when one channel is 20 times larger.  Reading: every token's
 * key row and value row get their own (scale, zero) over their D channels
 * (the asymmetric min/max quantizer above at 8 bits), computed when the
 * token is written; no window.  Rows x[t*ld .. t*ld+D) (bf16 bits). */
void oracle_int8_encode_rows(const uint16_t *x, int64_t ld, int64_t n, int32_t D,
                             uint8_t *codes, uint16_t *s16, uint16_t *z16)
{
    float row[4096];
    for (int64_t t = 0; t < n; ++t) {
        for (int32_t c = 0; c < D; ++c) row[c] = oracle_bf16_to_f32(x[t * ld + c]);
        oracle_quantize_set(row, D, 1, 8, &codes[t * D], 1, &s16[t], &z16[t]);
    }
}

/* K^ and V^ of n INT8 tokens, in double: code * s_t + z_t with token t's own
 * scale and zero.  khat, vhat: [n][D]. */
void oracle_int8_materialize(const uint8_t *k_codes, const uint16_t *k_s, const uint16_t *k_z,
                             const uint8_t *v_codes, const uint16_t *v_s, const uint16_t *v_z,
                             int32_t n, int32_t D, double *khat, double *vhat)
{
    for (int32_t t = 0; t < n; ++t)
        for (int32_t c = 0; c < D; ++c) {
            khat[(int64_t)t * D + c] = oracle_dequant(k_codes[(int64_t)t * D + c], k_s[t], k_z[t]);
            vhat[(int64_t)t * D + c] = oracle_dequant(v_codes[(int64_t)t * D + c], v_s[t], v_z[t]);
        }
}

/* Decode attention over an INT8 unit of n tokens.  work: 2*n*D + n doubles. */
void oracle_int8_decode(const uint8_t *k_codes, const uint16_t *k_s, const uint16_t *k_z,
                        const uint8_t *v_codes, const uint16_t *v_s, const uint16_t *v_z,
                        int32_t n, int32_t D, const uint16_t *q, int64_t q_ld, int32_t nh,
                        double scale, double *out, double *work)
{
    double *khat = work, *vhat = work + (int64_t)n * D, *lg = vhat + (int64_t)n * D;
    oracle_int8_materialize(k_codes, k_s, k_z, v_codes, v_s, v_z, n, D, khat, vhat);
    oracle_attend(khat, vhat, n, D, q, q_ld, nh, scale, out, NULL, lg);
}

/* ------------------------------------------------------------------------ */
/* Array forms of the scalar routines (so checks can sweep many values)     */
/* ------------------------------------------------------------------------ */

void oracle_f32_to_f16_array(const float *x, int64_t n, uint16_t *out)
{ for (int64_t i = 0; i < n; ++i) out[i] = oracle_f32_to_f16(x[i]); }

void oracle_f16_to_f32_array(const uint16_t *h, int64_t n, float *out)
{ for (int64_t i = 0; i < n; ++i) out[i] = oracle_f16_to_f32(h[i]); }

void oracle_e4m3_encode_array(const float *x, int64_t n, uint8_t *out)
{ for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode(x[i]); }

void oracle_e4m3_encode_bruteforce_array(const float *x, int64_t n, uint8_t *out)
{ for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode_bruteforce(x[i]); }

void oracle_e4m3_decode_array(const uint8_t *c, int64_t n, float *out)
{ for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_decode(c[i]); }

void oracle_encode_array(const float *x, int64_t n, uint16_t s16, uint16_t z16, int32_t bits,
                         int32_t truediv, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = truediv ? oracle_encode_truediv(x[i], s16, z16, bits) : oracle_encode(x[i], s16, z16, bits);
}
