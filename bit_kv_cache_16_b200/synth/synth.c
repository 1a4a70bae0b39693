/*
 * Seeded synthetic KV / query generator shared by the tests, the bench and
 * the oracle-side checks.  It holds none of the quantization or attention
 * arithmetic: it only draws numbers and shapes them like the KV statistics
 * the pages describe (fixed outlier channels in K, heavy tokens in V, RoPE
 * applied to K).
 *
 * Random numbers are counter-based: element i of sub-stream `stream` under
 * `seed` is the i-th output of a SplitMix64 sequence whose start state is
 * derived from (seed, stream).  SplitMix64 is Vigna's published generator
 * (Steele, Lea, Flood, "Fast splittable pseudorandom number generators",
 * OOPSLA 2014; finaliser constants as published there).  A normal draw uses
 * the cosine branch of the Box-Muller transform on two consecutive uniforms,
 * evaluated in double, then rounded to fp32 and from fp32 to bf16 with
 * round-to-nearest-even.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>

#define GOLDEN_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* Start state of a sub-stream: one SplitMix64 step from seed, then one from
 * the stream id, so that neighbouring (seed, stream) pairs are unrelated. */
static inline uint64_t stream_key(uint64_t seed, uint64_t stream)
{
    return mix64(mix64(seed + GOLDEN_GAMMA) ^ (stream * GOLDEN_GAMMA + 0x632BE59BD9B4E019ULL));
}

/* i-th 64-bit output of the SplitMix64 sequence started at `key`. */
static inline uint64_t draw_u64(uint64_t key, uint64_t i)
{
    return mix64(key + (i + 1) * GOLDEN_GAMMA);
}

/* Uniform in the open interval (0, 1): 53 high bits, centred in their cell. */
static inline double draw_uniform(uint64_t key, uint64_t i)
{
    return ((double)(draw_u64(key, i) >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

static inline double draw_normal(uint64_t key, uint64_t i)
{
    const double u1 = draw_uniform(key, 2 * i);
    const double u2 = draw_uniform(key, 2 * i + 1);
    return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925286766559 * u2);
}

static inline uint16_t f32_to_bf16_rne(float f)
{
    union { float f; uint32_t u; } v = { f };
    uint32_t u = v.u;
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu))
        return (uint16_t)((u >> 16) | 0x0040u); /* keep NaN quiet */
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* ---- exported ---------------------------------------------------------- */

void synth_u64(uint64_t seed, uint64_t stream, uint64_t first, int64_t count, uint64_t *out)
{
    const uint64_t key = stream_key(seed, stream);
    for (int64_t j = 0; j < count; ++j) out[j] = draw_u64(key, first + (uint64_t)j);
}

void synth_uniform(uint64_t seed, uint64_t stream, uint64_t first, int64_t count, double *out)
{
    const uint64_t key = stream_key(seed, stream);
    for (int64_t j = 0; j < count; ++j) out[j] = draw_uniform(key, first + (uint64_t)j);
}

void synth_normal(uint64_t seed, uint64_t stream, uint64_t first, int64_t count, double *out)
{
    const uint64_t key = stream_key(seed, stream);
    for (int64_t j = 0; j < count; ++j) out[j] = draw_normal(key, first + (uint64_t)j);
}

/*
 * Fill rows of a token-major tensor out[n_tok][H][D] (bf16 bits).
 * Element (t, h, c) takes normal draw number index0 + (t*H + h)*D + c, times
 * chan_factor[h*D + c] (if given) and tok_factor[t] (if given), in double.
 * If rope_theta > 0, adjacent channel pairs (2i, 2i+1) are then rotated by
 * the angle positions[t] * rope_theta^(-2i/D), in double.  The result is
 * rounded to fp32 and then to bf16.
 */
void synth_fill_rows_bf16(uint64_t seed, uint64_t stream, uint64_t index0,
                          int64_t n_tok, int32_t H, int32_t D,
                          const double *chan_factor, const double *tok_factor,
                          double rope_theta, const int64_t *positions,
                          uint16_t *out)
{
    const uint64_t key = stream_key(seed, stream);
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n_tok; ++t) {
        double row[1024];
        for (int32_t h = 0; h < H; ++h) {
            const uint64_t base = index0 + ((uint64_t)t * (uint64_t)H + (uint64_t)h) * (uint64_t)D;
            for (int32_t c = 0; c < D; ++c) {
                double x = draw_normal(key, base + (uint64_t)c);
                if (chan_factor) x *= chan_factor[(int64_t)h * D + c];
                if (tok_factor) x *= tok_factor[t];
                row[c] = x;
            }
            if (rope_theta > 0.0) {
                const double pos = (double)positions[t];
                for (int32_t i = 0; i < D / 2; ++i) {
                    const double ang = pos * pow(rope_theta, -2.0 * (double)i / (double)D);
                    const double cs = cos(ang), sn = sin(ang);
                    const double a = row[2 * i], b = row[2 * i + 1];
                    row[2 * i] = a * cs - b * sn;
                    row[2 * i + 1] = a * sn + b * cs;
                }
            }
            uint16_t *dst = out + ((int64_t)t * H + h) * D;
            for (int32_t c = 0; c < D; ++c) dst[c] = f32_to_bf16_rne((float)row[c]);
        }
    }
}
