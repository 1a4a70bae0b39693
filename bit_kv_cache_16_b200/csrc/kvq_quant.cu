// Write side of the cache: prefill quantization, append, flush (INT2/INT4),
// and the FP8-E4M3 comparison cache.
//
// INT prefill and flush: one CTA of four warps quantizes one block of
// TB = max(G, 32) tokens of one (sequence, kv head).
//  * Warps 0 and 1 are key warps.  Lane i of key warp w owns the channel
//    pair (2p, 2p+1), p = 32w + i, for every token of a group: it reads one
//    bf16x2 word per token (a warp reads 128 contiguous bytes of a row),
//    reduces min/max over the group's tokens in packed bf16x2 form (no
//    shuffles), derives the two channels' fp16 scale/zero itself, and writes
//    one code byte (INT4) or half a byte (INT2) of each token's row.
//  * Warps 2 and 3 are value warps, one 16-token tile at a time.  Lane
//    (n, l) holds tokens 2l, 2l+1, 2l+8, 2l+9 of the tile, channels
//    [16n, 16n+16): per-token min/max is reduced in registers, then across
//    the 8 lanes that share a token with one packed (min, -max) word per
//    token; each quarter of the lanes derives one token's scale/zero and
//    hands it to the others; the lane writes its words of the tile in the
//    decode's fragment order (include/kvq.h).
// Encoding runs two values per instruction with packed fp32x2 arithmetic:
// (x - z) and (.) * inv are each rounded like the scalar IEEE operations,
// and adding 1.5 * 2^23 rounds to the nearest integer, ties to even, which
// leaves the code in the low mantissa bits.  That shortcut is taken only
// when every code of the warp's groups is known to land in [0, 2^b - 1]
// without clamping and no input is NaN (the endpoints of a group bound all
// its values, because both rounded steps are monotone); otherwise the warp
// runs the scalar encoder with explicit clamping.
#include "kvq_common.cuh"

namespace kvq {

// Rows of a token block: row(i) = base + ((start + i) mod m) * stride  (m > 0)
//                                  base + i * stride                    (m == 0)
struct RowSrc {
  const uint16_t* base;
  int64_t stride;  // in bf16 elements
  int start;
  int mod;
  __device__ __forceinline__ const uint16_t* row(int i) const {
    const int r = mod > 0 ? (start + i) % mod : i;
    return base + (int64_t)r * stride;
  }
};

struct GroupDst {
  uint8_t* k_codes;     // row of token 0 of the group; rows of RB bytes
  __half* k_meta;       // [2][128]
  uint8_t* v_tiles;     // tile 0 of the group; consecutive tiles
  __half* v_meta;       // [G][2]
  uint32_t* k_sparse;   // dense-and-sparse: [128] kept key per channel (null otherwise)
  uint32_t* v_sparse;   // dense-and-sparse: [G] kept value per token (null otherwise)
};

// ---------------------------------------------------------------------------
// Packed helpers
// ---------------------------------------------------------------------------

typedef unsigned long long u64;
constexpr u64 kRoundMagic2 = 0x4B4000004B400000ull;   // 1.5 * 2^23 in both fp32 lanes
constexpr uint32_t kPosInf2 = 0x7F807F80u;            // bf16x2 (+inf, +inf)
constexpr uint32_t kNegInf2 = 0xFF80FF80u;            // bf16x2 (-inf, -inf)

// NaN-propagating packed bf16 min/max: without NaNs they equal fminf/fmaxf,
// and a NaN anywhere shows up in the result.
__device__ __forceinline__ uint32_t bmin2_nan(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("min.NaN.bf16x2 %0, %1, %2;\n" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bmax2_nan(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.bf16x2 %0, %1, %2;\n" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ bool bf16x2_has_nan(uint32_t w) {
  return (w & 0x7FFFu) > 0x7F80u || (w & 0x7FFF0000u) > 0x7F800000u;
}

__device__ __forceinline__ u64 pack_f2(float lo, float hi) {
  u64 d;
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}

// (1.0f, 1.0f) read from constant memory: an operand the compiler cannot
// see the value of (see encode2_fast).
__constant__ u64 kOnePair = 0x3F8000003F800000ull;

// The bf16 pair w (lo, hi) -> two encoder outputs y whose low mantissa bits
// are rint_half_even((x - z) * inv) (valid when that lies in [0, 2^22)).
// The rounding add is written as t * one + magic with `one` loaded at run
// time: a plain add would let the compiler fuse the preceding multiply into
// one FMA, which rounds the exact product instead of the fp32 product t and
// so breaks exact .5 ties of t the other way.  t * 1 is exact, so the FMA
// rounds t + magic once, as the add would.
__device__ __forceinline__ void encode2_fast(uint32_t w, u64 z2, u64 inv2, u64 one2, uint32_t& ylo,
                                             uint32_t& yhi) {
  u64 x2, d, t, y;
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(x2) : "r"(w << 16), "r"(w & 0xFFFF0000u));
  asm("sub.rn.f32x2 %0, %1, %2;\n" : "=l"(d) : "l"(x2), "l"(z2));
  asm("mul.rn.f32x2 %0, %1, %2;\n" : "=l"(t) : "l"(d), "l"(inv2));
  asm("fma.rn.f32x2 %0, %1, %2, %3;\n" : "=l"(y) : "l"(t), "l"(one2), "l"(kRoundMagic2));
  asm("mov.b64 {%0, %1}, %2;\n" : "=r"(ylo), "=r"(yhi) : "l"(y));
}

// (hi << s) + lo: one shift-add that merges the low code bits of two encoder
// outputs (garbage above bit 21 + s never reaches the low byte).
__device__ __forceinline__ uint32_t shl_add(uint32_t hi, uint32_t lo, int s) { return (hi << s) + lo; }

// Codes that need no clamp: t(min) >= -1/2 and t(max) < top + 1/2 (both
// false for NaN), so every value of the set rounds into [0, top].
__device__ __forceinline__ bool clamp_free(float mn, float mx, const QParams& p, int top) {
  const float tl = __fmul_rn(__fsub_rn(mn, p.z), p.inv);
  const float th = __fmul_rn(__fsub_rn(mx, p.z), p.inv);
  return tl >= -0.5f && th < (float)top + 0.5f;
}

// ---------------------------------------------------------------------------
// Key groups: lane owns the channel pair p of G tokens
// ---------------------------------------------------------------------------


template <int BITS>
__device__ __forceinline__ void store_kcode(uint8_t* row, int p, uint32_t ylo, uint32_t yhi) {
  if (BITS == 4) {
    row[p] = (uint8_t)shl_add(yhi, ylo, 4);
  } else {
    // channels 2p, 2p+1 are the low (p even) or high (p odd) half of byte p/2
    const uint32_t nib = shl_add(yhi, ylo, 2) & 0xFu;
    const uint32_t other = __shfl_xor_sync(0xffffffffu, nib, 1);
    if ((p & 1) == 0) row[p >> 1] = (uint8_t)(nib | (other << 4));
  }
}

template <int BITS>
__device__ __forceinline__ void store_kcode_scalar(uint8_t* row, int p, uint32_t clo, uint32_t chi) {
  if (BITS == 4) {
    row[p] = (uint8_t)(clo | (chi << 4));
  } else {
    const uint32_t nib = clo | (chi << 2);
    const uint32_t other = __shfl_xor_sync(0xffffffffu, nib, 1);
    if ((p & 1) == 0) row[p >> 1] = (uint8_t)(nib | (other << 4));
  }
}

// The codes of N tokens of channel pair p (words x, clamp-free) into their
// rows.  At 2 bits a byte holds the nibbles of two lanes (channels
// 4j .. 4j+3): four tokens' nibbles travel in one word and one shuffle, and
// the even lane stores the bytes of the first two tokens, the odd lane those
// of the last two.
template <int BITS, int N>
__device__ __forceinline__ void store_keys_fast(const uint32_t (&x)[N], int p, uint8_t* codes, u64 z2, u64 inv2,
                                                u64 one2) {
  constexpr int RB = kHeadDim * BITS / 8;
  if constexpr (BITS == 4) {
#pragma unroll
    for (int i = 0; i < N; ++i) {
      uint32_t ylo, yhi;
      encode2_fast(x[i], z2, inv2, one2, ylo, yhi);
      store_kcode<BITS>(codes + (size_t)i * RB, p, ylo, yhi);
    }
  } else {
    static_assert(N % 4 == 0, "tokens in fours");
    const bool odd = p & 1;
    const int u0 = odd ? 2 : 0;
#pragma unroll
    for (int i = 0; i < N; i += 4) {
      uint32_t mine = 0u;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        uint32_t ylo, yhi;
        encode2_fast(x[i + u], z2, inv2, one2, ylo, yhi);
        mine |= (shl_add(yhi, ylo, 2) & 0xFu) << (8 * u);
      }
      const uint32_t other = __shfl_xor_sync(0xffffffffu, mine, 1);
      const uint32_t bytes = (odd ? other : mine) | ((odd ? mine : other) << 4);   // byte u: token i + u
      uint8_t* r0 = codes + (size_t)(i + u0) * RB + (p >> 1);
      r0[0] = (uint8_t)(bytes >> (8 * u0));
      r0[RB] = (uint8_t)(bytes >> (8 * u0 + 8));
    }
  }
}

// One key group of G tokens for the channel pair p of this lane.
template <int BITS, int G>
__device__ __forceinline__ void k_group(const RowSrc& src, int p, uint8_t* codes, __half* meta) {
  constexpr int CH = G < 32 ? G : 32;       // tokens held in registers at a time
  constexpr int NCH = G / CH;
  constexpr int RB = kHeadDim * BITS / 8;
  constexpr int top = (1 << BITS) - 1;
  uint32_t x[CH];
  auto load = [&](int c) {
#pragma unroll
    for (int i = 0; i < CH; ++i) x[i] = *reinterpret_cast<const uint32_t*>(src.row(c * CH + i) + 2 * p);
  };
  uint32_t mn2 = kPosInf2, mx2 = kNegInf2;
#pragma unroll 1
  for (int c = 0; c < NCH; ++c) {
    load(c);
#pragma unroll
    for (int i = 0; i < CH; ++i) {
      mn2 = bmin2_nan(mn2, x[i]);
      mx2 = bmax2_nan(mx2, x[i]);
    }
  }
  float mn[2] = {bf16_lo(mn2), bf16_hi(mn2)}, mx[2] = {bf16_lo(mx2), bf16_hi(mx2)};
  QParams qp[2];
  bool fast = !bf16x2_has_nan(mn2) && !bf16x2_has_nan(mx2);
  if (__all_sync(0xffffffffu, fast)) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      qp[e] = quant_params(mn[e], mx[e], BITS);
      fast = fast && clamp_free(mn[e], mx[e], qp[e], top);
    }
  }
  if (__all_sync(0xffffffffu, fast)) {
    const u64 z2 = pack_f2(qp[0].z, qp[1].z), inv2 = pack_f2(qp[0].inv, qp[1].inv);
    const u64 one2 = kOnePair;
#pragma unroll 1
    for (int c = 0; c < NCH; ++c) {
      if (NCH > 1) load(c);
      store_keys_fast<BITS, CH>(x, p, codes + (size_t)c * CH * RB, z2, inv2, one2);
    }
  } else {
    // exact scalar path: min/max ignoring NaN (fminf/fmaxf), clamped codes
    mn[0] = mn[1] = INFINITY;
    mx[0] = mx[1] = -INFINITY;
#pragma unroll 1
    for (int c = 0; c < NCH; ++c) {
      load(c);
#pragma unroll
      for (int i = 0; i < CH; ++i) {
        mn[0] = fminf(mn[0], bf16_lo(x[i])); mx[0] = fmaxf(mx[0], bf16_lo(x[i]));
        mn[1] = fminf(mn[1], bf16_hi(x[i])); mx[1] = fmaxf(mx[1], bf16_hi(x[i]));
      }
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) qp[e] = quant_params(mn[e], mx[e], BITS);
#pragma unroll 1
    for (int c = 0; c < NCH; ++c) {
      if (NCH > 1) load(c);
#pragma unroll
      for (int i = 0; i < CH; ++i) {
        const uint32_t clo = encode(bf16_lo(x[i]), qp[0].z, qp[0].inv, top);
        const uint32_t chi = encode(bf16_hi(x[i]), qp[1].z, qp[1].inv, top);
        store_kcode_scalar<BITS>(codes + (size_t)(c * CH + i) * RB, p, clo, chi);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int pos = kmeta_pos<BITS>(2 * p + e);
    meta[pos] = qp[e].s16;
    meta[kHeadDim + pos] = qp[e].z16;
  }
}

// One key group of G <= 32 tokens whose words (channel pair p, one per
// token) are already in registers: k_group without the loads, so that a
// caller can keep several groups' loads in flight.
template <int BITS, int G>
__device__ __forceinline__ void k_group_x(const uint32_t (&x)[G], int p, uint8_t* codes, __half* meta) {
  static_assert(G <= 32, "one register block");
  constexpr int RB = kHeadDim * BITS / 8;
  constexpr int top = (1 << BITS) - 1;
  uint32_t mn2 = kPosInf2, mx2 = kNegInf2;
#pragma unroll
  for (int i = 0; i < G; ++i) {
    mn2 = bmin2_nan(mn2, x[i]);
    mx2 = bmax2_nan(mx2, x[i]);
  }
  float mn[2] = {bf16_lo(mn2), bf16_hi(mn2)}, mx[2] = {bf16_lo(mx2), bf16_hi(mx2)};
  QParams qp[2];
  bool fast = !bf16x2_has_nan(mn2) && !bf16x2_has_nan(mx2);
  if (__all_sync(0xffffffffu, fast)) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      qp[e] = quant_params(mn[e], mx[e], BITS);
      fast = fast && clamp_free(mn[e], mx[e], qp[e], top);
    }
  }
  if (__all_sync(0xffffffffu, fast)) {
    const u64 z2 = pack_f2(qp[0].z, qp[1].z), inv2 = pack_f2(qp[0].inv, qp[1].inv);
    const u64 one2 = kOnePair;
    store_keys_fast<BITS, G>(x, p, codes, z2, inv2, one2);
  } else {
    // exact scalar path: min/max ignoring NaN (fminf/fmaxf), clamped codes
    mn[0] = mn[1] = INFINITY;
    mx[0] = mx[1] = -INFINITY;
#pragma unroll
    for (int i = 0; i < G; ++i) {
      mn[0] = fminf(mn[0], bf16_lo(x[i])); mx[0] = fmaxf(mx[0], bf16_lo(x[i]));
      mn[1] = fminf(mn[1], bf16_hi(x[i])); mx[1] = fmaxf(mx[1], bf16_hi(x[i]));
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) qp[e] = quant_params(mn[e], mx[e], BITS);
#pragma unroll
    for (int i = 0; i < G; ++i) {
      const uint32_t clo = encode(bf16_lo(x[i]), qp[0].z, qp[0].inv, top);
      const uint32_t chi = encode(bf16_hi(x[i]), qp[1].z, qp[1].inv, top);
      store_kcode_scalar<BITS>(codes + (size_t)i * RB, p, clo, chi);
    }
  }
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int pos = kmeta_pos<BITS>(2 * p + e);
    meta[pos] = qp[e].s16;
    meta[kHeadDim + pos] = qp[e].z16;
  }
}

// Dense-and-sparse order of magnitudes: a NaN counts below every number.
__device__ __forceinline__ float sparse_key(float v) { return isnan(v) ? -1.0f : fabsf(v); }

// One key group of G <= 32 tokens for the channel pair p of this lane, with
// each channel's largest-magnitude value (the first such) kept aside: its
// bf16 bits and token index go to ksp[channel], its code is 0, and the
// channel's min/max and codes are taken over the other tokens (exact scalar
// arithmetic, clamped codes).
template <int BITS, int G>
__device__ __forceinline__ void k_group_sparse(const RowSrc& src, int p, uint8_t* codes, __half* meta,
                                               uint32_t* ksp) {
  static_assert(G <= 32, "one group in registers");
  constexpr int RB = kHeadDim * BITS / 8;
  constexpr int top = (1 << BITS) - 1;
  uint32_t x[G];
#pragma unroll
  for (int i = 0; i < G; ++i) x[i] = *reinterpret_cast<const uint32_t*>(src.row(i) + 2 * p);
  uint32_t cl[G], ch[G];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    auto val = [&](int i) { return e ? bf16_hi(x[i]) : bf16_lo(x[i]); };
    int im = 0;
    float best = sparse_key(val(0));
#pragma unroll
    for (int i = 1; i < G; ++i) {
      const float m = sparse_key(val(i));
      if (m > best) { im = i; best = m; }
    }
    float mn = INFINITY, mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < G; ++i)
      if (i != im) { mn = fminf(mn, val(i)); mx = fmaxf(mx, val(i)); }
    const QParams qp = quant_params(mn, mx, BITS);
#pragma unroll
    for (int i = 0; i < G; ++i) {
      const uint32_t cd = i == im ? 0u : encode(val(i), qp.z, qp.inv, top);
      if (e) ch[i] = cd; else cl[i] = cd;
    }
    const uint32_t raw = e ? (x[im] >> 16) : (x[im] & 0xFFFFu);
    ksp[2 * p + e] = raw | ((uint32_t)im << 16);
    const int pos = kmeta_pos<BITS>(2 * p + e);
    meta[pos] = qp.s16;
    meta[kHeadDim + pos] = qp.z16;
  }
#pragma unroll
  for (int i = 0; i < G; ++i) store_kcode_scalar<BITS>(codes + (size_t)i * RB, p, cl[i], ch[i]);
}

// ---------------------------------------------------------------------------
// Value tiles: lane (n, l) holds 4 tokens x 16 channels of a 16-token tile
// ---------------------------------------------------------------------------

// One 16-token value tile.  The lane's tokens are q = 0..3 = (2l, 2l+1,
// 2l+8, 2l+9); in every tile word byte q holds token q, which is the nibble
// (INT4) or 2-bit (INT2) order of the fragment layout: position = (channel
// bits) + 2o + 4s (INT4) or + 4o + 8s (INT2) for token 8s + 2l + o, so that
// the decode's e4m3 converter turns bytes (0, 1) and (2, 3) of a word's
// split codes into the fp16 pairs of tokens (2l, 2l+1) and (2l+8, 2l+9).
template <int BITS>
__device__ __forceinline__ void v_tile(const RowSrc& src, int tile, uint8_t* vt, __half* vm,
                                       int tstride = tile_bytes(BITS)) {   // bytes from one tile to the next
  const int lane = threadIdx.x & 31;
  const int n = lane >> 2, l = lane & 3;
  const int tok[4] = {2 * l, 2 * l + 1, 2 * l + 8, 2 * l + 9};
  constexpr int top = (1 << BITS) - 1;
  uint32_t x[4][8];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint16_t* r = src.row(kTile * tile + tok[q]) + 16 * n;
    const uint4 a = *reinterpret_cast<const uint4*>(r);
    const uint4 b = *reinterpret_cast<const uint4*>(r + 8);
    x[q][0] = a.x; x[q][1] = a.y; x[q][2] = a.z; x[q][3] = a.w;
    x[q][4] = b.x; x[q][5] = b.y; x[q][6] = b.z; x[q][7] = b.w;
  }
  // per-token (min, -max) as one bf16x2 word, reduced over the 8 lanes of the token
  uint32_t mm[4];
  bool nan_free = true;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t a = x[q][0], b = x[q][0];
#pragma unroll
    for (int i = 1; i < 8; ++i) {
      a = bmin2_nan(a, x[q][i]);
      b = bmax2_nan(b, x[q][i]);
    }
    a = bmin2_nan(a, prmt(a, a, 0x1032u));           // both halves: min of the lane's 16 values
    b = bmax2_nan(b, prmt(b, b, 0x1032u));
    mm[q] = prmt(a, b ^ 0x80008000u, 0x7610u);       // (min, -max)
  }
#pragma unroll
  for (int off = 4; off < 32; off <<= 1)
#pragma unroll
    for (int q = 0; q < 4; ++q) mm[q] = bmin2_nan(mm[q], __shfl_xor_sync(0xffffffffu, mm[q], off));
#pragma unroll
  for (int q = 0; q < 4; ++q) nan_free = nan_free && !bf16x2_has_nan(mm[q]);
  if (__all_sync(0xffffffffu, nan_free)) {
    // lane (n, l) derives token q = n & 3 and passes it to the lanes that need it
    const int qm = n & 3;
    uint32_t sel = mm[0];
#pragma unroll
    for (int q = 1; q < 4; ++q) sel = qm == q ? mm[q] : sel;
    const float tmn = bf16_lo(sel), tmx = -bf16_hi(sel);
    const QParams qp = quant_params(tmn, tmx, BITS);
    const bool ok = clamp_free(tmn, tmx, qp, top);
    if (__all_sync(0xffffffffu, ok)) {
      const u64 one2 = kOnePair;
      float zq[4], iq[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        zq[q] = __shfl_sync(0xffffffffu, qp.z, 4 * q + l);
        iq[q] = __shfl_sync(0xffffffffu, qp.inv, 4 * q + l);
      }
      if (n < 4) {
        const uint32_t m = (uint32_t)__half_as_ushort(qp.s16) | ((uint32_t)__half_as_ushort(qp.z16) << 16);
        *reinterpret_cast<uint32_t*>(vm + 2 * (kTile * tile + tok[n])) = m;
      }
      // y[q][c]: encoder outputs of token q, channel c (0..15) of the lane
      if (BITS == 4) {
        uint32_t w[8];
#pragma unroll
        for (int ww = 0; ww < 8; ++ww) {
          uint32_t by[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t ylo, yhi;
            encode2_fast(x[q][ww], pack_f2(zq[q], zq[q]), pack_f2(iq[q], iq[q]), one2, ylo, yhi);
            by[q] = shl_add(yhi, ylo, 4);     // channels (2ww, 2ww+1) of token q
          }
          // byte q: token q's channels (2ww, 2ww+1)
          w[ww] = prmt(prmt(by[0], by[1], 0x0040u), prmt(by[2], by[3], 0x0040u), 0x5410u);
        }
        uint8_t* t8 = vt + (size_t)tile * tstride;
        *reinterpret_cast<uint4*>(t8 + 16 * lane) = make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4*>(t8 + 512 + 16 * lane) = make_uint4(w[4], w[5], w[6], w[7]);
      } else {
        uint32_t w[4];
#pragma unroll
        for (int ww = 0; ww < 4; ++ww) {
          uint32_t by[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t y0, y1, y2, y3;
            encode2_fast(x[q][2 * ww], pack_f2(zq[q], zq[q]), pack_f2(iq[q], iq[q]), one2, y0, y1);
            encode2_fast(x[q][2 * ww + 1], pack_f2(zq[q], zq[q]), pack_f2(iq[q], iq[q]), one2, y2, y3);
            by[q] = shl_add(shl_add(shl_add(y3, y2, 2), y1, 2), y0, 2);   // channels 4ww..4ww+3
          }
          w[ww] = prmt(prmt(by[0], by[1], 0x0040u), prmt(by[2], by[3], 0x0040u), 0x5410u);
        }
        uint8_t* t8 = vt + (size_t)tile * tstride;
        *reinterpret_cast<uint4*>(t8 + 16 * lane) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      return;
    }
  }
  // exact scalar path: per-token min/max ignoring NaN, clamped codes
  QParams qp[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float mn = INFINITY, mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      mn = fminf(mn, fminf(bf16_lo(x[q][i]), bf16_hi(x[q][i])));
      mx = fmaxf(mx, fmaxf(bf16_lo(x[q][i]), bf16_hi(x[q][i])));
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    }
    qp[q] = quant_params(mn, mx, BITS);
  }
  uint8_t* t8 = vt + (size_t)tile * tstride;
  if (BITS == 4) {
    uint32_t w[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int s = q >> 1, o = q & 1;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float val = (j & 1) ? bf16_hi(x[q][j >> 1]) : bf16_lo(x[q][j >> 1]);
        const uint32_t code = encode(val, qp[q].z, qp[q].inv, top);
        w[j >> 1] |= code << (4 * ((j & 1) + 2 * o + 4 * s));
      }
    }
    *reinterpret_cast<uint4*>(t8 + 16 * lane) = make_uint4(w[0], w[1], w[2], w[3]);
    *reinterpret_cast<uint4*>(t8 + 512 + 16 * lane) = make_uint4(w[4], w[5], w[6], w[7]);
  } else {
    uint32_t w[4] = {0, 0, 0, 0};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int s = q >> 1, o = q & 1;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float val = (j & 1) ? bf16_hi(x[q][j >> 1]) : bf16_lo(x[q][j >> 1]);
        const uint32_t code = encode(val, qp[q].z, qp[q].inv, top);
        w[j >> 2] |= code << (2 * ((j & 3) + 4 * o + 8 * s));
      }
    }
    *reinterpret_cast<uint4*>(t8 + 16 * lane) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (n == 0) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t m = (uint32_t)__half_as_ushort(qp[q].s16) | ((uint32_t)__half_as_ushort(qp[q].z16) << 16);
      *reinterpret_cast<uint32_t*>(vm + 2 * (kTile * tile + tok[q])) = m;
    }
  }
}

// One 16-token value tile with each token's largest-magnitude value (the
// first in channel order) kept aside: vsp[token] = bf16 bits | channel << 16,
// its code 0, the token's min/max and codes over the other channels (exact
// scalar arithmetic, clamped codes).  Lane (n, l) holds channels
// [16n, 16n+16) of tokens 2l, 2l+1, 2l+8, 2l+9, as in v_tile.
template <int BITS>
__device__ __forceinline__ void v_tile_sparse(const RowSrc& src, int tile, uint8_t* vt, __half* vm, uint32_t* vsp,
                                              int tstride = tile_bytes(BITS)) {
  const int lane = threadIdx.x & 31;
  const int n = lane >> 2, l = lane & 3;
  const int tok[4] = {2 * l, 2 * l + 1, 2 * l + 8, 2 * l + 9};
  constexpr int top = (1 << BITS) - 1;
  uint32_t x[4][8];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint16_t* r = src.row(kTile * tile + tok[q]) + 16 * n;
    const uint4 a = *reinterpret_cast<const uint4*>(r);
    const uint4 b = *reinterpret_cast<const uint4*>(r + 8);
    x[q][0] = a.x; x[q][1] = a.y; x[q][2] = a.z; x[q][3] = a.w;
    x[q][4] = b.x; x[q][5] = b.y; x[q][6] = b.z; x[q][7] = b.w;
  }
  QParams qp[4];
  int keep[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    // largest magnitude of the token: this lane's 16 channels, then the 8
    // lanes of the token (ties: the lower channel)
    int ch = 16 * n;
    float best = sparse_key(bf16_lo(x[q][0]));
#pragma unroll
    for (int j = 1; j < 16; ++j) {
      const float m = sparse_key((j & 1) ? bf16_hi(x[q][j >> 1]) : bf16_lo(x[q][j >> 1]));
      if (m > best) { best = m; ch = 16 * n + j; }
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, off);
      const int oc = __shfl_xor_sync(0xffffffffu, ch, off);
      if (ob > best || (ob == best && oc < ch)) { best = ob; ch = oc; }
    }
    keep[q] = ch;
    float mn = INFINITY, mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if (16 * n + j == ch) continue;
      const float v = (j & 1) ? bf16_hi(x[q][j >> 1]) : bf16_lo(x[q][j >> 1]);
      mn = fminf(mn, v);
      mx = fmaxf(mx, v);
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    }
    qp[q] = quant_params(mn, mx, BITS);
  }
  uint8_t* t8 = vt + (size_t)tile * tstride;
  if (BITS == 4) {
    uint32_t w[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int s = q >> 1, o = q & 1;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float val = (j & 1) ? bf16_hi(x[q][j >> 1]) : bf16_lo(x[q][j >> 1]);
        const uint32_t code = 16 * n + j == keep[q] ? 0u : encode(val, qp[q].z, qp[q].inv, top);
        w[j >> 1] |= code << (4 * ((j & 1) + 2 * o + 4 * s));
      }
    }
    *reinterpret_cast<uint4*>(t8 + 16 * lane) = make_uint4(w[0], w[1], w[2], w[3]);
    *reinterpret_cast<uint4*>(t8 + 512 + 16 * lane) = make_uint4(w[4], w[5], w[6], w[7]);
  } else {
    uint32_t w[4] = {0, 0, 0, 0};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int s = q >> 1, o = q & 1;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float val = (j & 1) ? bf16_hi(x[q][j >> 1]) : bf16_lo(x[q][j >> 1]);
        const uint32_t code = 16 * n + j == keep[q] ? 0u : encode(val, qp[q].z, qp[q].inv, top);
        w[j >> 2] |= code << (2 * ((j & 3) + 4 * o + 8 * s));
      }
    }
    *reinterpret_cast<uint4*>(t8 + 16 * lane) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  // the lane holding the kept channel writes the token's entry; lanes n = 0
  // write the tokens' (scale, zero)
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int j = keep[q] - 16 * n;
    if (j >= 0 && j < 16) {
      const uint32_t raw = (j & 1) ? (x[q][j >> 1] >> 16) : (x[q][j >> 1] & 0xFFFFu);
      vsp[kTile * tile + tok[q]] = raw | ((uint32_t)keep[q] << 16);
    }
  }
  if (n == 0) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t m = (uint32_t)__half_as_ushort(qp[q].s16) | ((uint32_t)__half_as_ushort(qp[q].z16) << 16);
      *reinterpret_cast<uint32_t*>(vm + 2 * (kTile * tile + tok[q])) = m;
    }
  }
}

__device__ __forceinline__ void set_err(uint32_t* err, uint32_t bit) { atomicOr(err, bit); }

// Destination of group g of (b, h); false if its page id is out of range.
__device__ __forceinline__ bool group_dst(const kvq_cache& c, int b, int h, int g, GroupDst& d) {
  const kvq_shape& s = c.shape;
  d.k_sparse = nullptr;
  d.v_sparse = nullptr;
  if (s.page_size == 0) {
    d.k_codes = (uint8_t*)c.k_codes + Addr::k_codes_unit(s, b, h) + (size_t)g * s.group * row_bytes(s.format);
    d.k_meta = (__half*)c.k_meta + Addr::k_meta_group(s, b, h, g);
    d.v_tiles = (uint8_t*)c.v_codes + Addr::v_codes_tile(s, b, h, g * (s.group / kTile));
    d.v_meta = (__half*)c.v_meta + Addr::v_meta_token(s, b, h, g * s.group);
    if (s.sparse) {
      const size_t unit = (size_t)b * s.num_kv_heads + h;
      d.k_sparse = c.k_sparse + (unit * (size_t)(s.capacity / s.group) + g) * kHeadDim;
      d.v_sparse = c.v_sparse + unit * (size_t)s.capacity + (size_t)g * s.group;
    }
    return true;
  }
  const int page = c.page_table[(size_t)b * s.max_pages_per_seq + g];
  if (page < 0 || page >= s.num_pages) return false;
  d.k_codes = (uint8_t*)c.k_codes + Addr::pg_k_codes(s, page, h);
  d.k_meta = (__half*)c.k_meta + Addr::pg_k_meta(s, page, h);
  d.v_tiles = (uint8_t*)c.v_codes + Addr::pg_v_codes(s, page, h);
  d.v_meta = (__half*)c.v_meta + Addr::pg_v_meta(s, page, h);
  return true;
}

__device__ __forceinline__ int quantized_prefix(int n, int R, int G) {
  const int over = n - R > 0 ? n - R : 0;
  return G * (over / G);
}

// Quantize one group (tokens [0, G) of ks and vs) into d with the warp
// roles of a 4-warp team (warp = 0..3 within the team).
// SPARSE: the dense-and-sparse variant (G of 16 or 32; d's sparse arrays set).
template <int BITS, int G, bool SPARSE = false>
__device__ __forceinline__ void quantize_group_cta(const RowSrc& ks, const RowSrc& vs, const GroupDst& d,
                                                   int warp = threadIdx.x >> 5, int tstride = tile_bytes(BITS)) {
  const int lane = threadIdx.x & 31;
  if constexpr (SPARSE) {
    static_assert(G <= 32, "dense-and-sparse groups are held in registers");
    if (warp < 2) k_group_sparse<BITS, G>(ks, 32 * warp + lane, d.k_codes, d.k_meta, d.k_sparse);
    else
      for (int t = warp - 2; t < G / kTile; t += 2) v_tile_sparse<BITS>(vs, t, d.v_tiles, d.v_meta, d.v_sparse);
    return;
  }
  if (warp < 2) {
    k_group<BITS, G>(ks, 32 * warp + lane, d.k_codes, d.k_meta);
  } else {
    for (int t = warp - 2; t < G / kTile; t += 2) v_tile<BITS>(vs, t, d.v_tiles, d.v_meta, tstride);
  }
}

// A group of a MIXED cache at 4 or 2 bits (the group's slots are laid out
// as INT4: key rows of a 2-bit group packed from the slot's start, value
// tiles in the first half of their 1 KB slots).
template <int G>
__device__ __forceinline__ void quantize_group_mixed(bool four, const RowSrc& ks, const RowSrc& vs, const GroupDst& d) {
  if (four) quantize_group_cta<4, G>(ks, vs, d, threadIdx.x >> 5, tile_bytes(4));
  else quantize_group_cta<2, G>(ks, vs, d, threadIdx.x >> 5, tile_bytes(4));
}

// Grid (ceil(max_len / TB), H_kv, B), 128 threads; TB = max(G, 32) tokens
// per CTA (two key groups when G = 16, one value warp per group).
// Registers are cut for 8 CTAs per SM at G = 16 and 32 (64 registers,
// some spill; more CTAs keep more of the short per-CTA loads in flight).
// Means of 20 calls: the paged ragged batch (G = 16) 1585 us at 5 CTAs,
// 1432 at 6, 1353 at 7, 1260 at 8, 1602 at 10, 1943 at 12; the 8B layer
// (G = 32) 78.0 us at 6 against 71.5 at 8, the 70B layer 134.6 against
// 124.5 (INT4) and 133.6 against 128.4 (INT2).  The dense-and-sparse
// kernel keeps 6 at G = 32 (5 or 8 were slower) and 5 at G = 16; G = 64
// and 128 keep 5 (no spill).
template <int BITS, int G, bool SPARSE>
__global__ void __launch_bounds__(128, SPARSE ? (G == 32 ? 6 : 5) : ((G == 16 || G == 32) ? 8 : 5)) prefill_int_kernel(kvq_cache c, const uint16_t* __restrict__ k,
                                                          const uint16_t* __restrict__ v,
                                                          const int32_t* __restrict__ cu, int max_len) {
  constexpr int TB = G < 32 ? 32 : G;
  const kvq_shape& s = c.shape;
  const int blk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int Ws = window_slots(s);
  const int t0 = cu[b];
  int n = cu[b + 1] - t0;
  const bool too_long = n > s.capacity || n < 0 || n > max_len;
  if (too_long) n = 0;
  const int nq = quantized_prefix(n, s.residual, G);
  if (blk == 0 && h == 0 && threadIdx.x == 0) {
    c.seq_len[b] = n;
    c.n_quant[b] = nq;
    if (too_long) set_err(c.err_word, KVQ_DEVERR_PREFILL_LEN);
  }
  const int tb0 = blk * TB;
  if (tb0 >= n) return;
  const int64_t stride = (int64_t)s.num_kv_heads * kHeadDim;
  bool page_bad = false;
  if constexpr (G == 16 && !SPARSE) {
    // the block's two 16-token groups: each key warp loads both groups'
    // words before quantizing either (twice the loads in flight); value
    // warp 2 + gi takes group gi's tile
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    GroupDst d[2];
    bool ok[2] = {false, false};
#pragma unroll
    for (int gi = 0; gi < 2; ++gi) {
      const int g = 2 * blk + gi;
      if ((g + 1) * G > nq) break;
      ok[gi] = group_dst(c, b, h, g, d[gi]);
      page_bad = page_bad || !ok[gi];
    }
    if (warp < 2) {
      const int p = 32 * warp + lane;
      uint32_t x0[16], x1[16];
      const uint16_t* r0 = k + ((int64_t)(t0 + 32 * blk) * s.num_kv_heads + h) * kHeadDim + 2 * p;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        x0[i] = ok[0] ? *reinterpret_cast<const uint32_t*>(r0 + i * stride) : 0u;
        x1[i] = ok[1] ? *reinterpret_cast<const uint32_t*>(r0 + (16 + i) * stride) : 0u;
      }
      if (ok[0]) k_group_x<BITS, 16>(x0, p, d[0].k_codes, d[0].k_meta);
      if (ok[1]) k_group_x<BITS, 16>(x1, p, d[1].k_codes, d[1].k_meta);
    } else if (ok[warp - 2]) {
      const int gi = warp - 2;
      const RowSrc vs{v + ((int64_t)(t0 + 32 * blk + 16 * gi) * s.num_kv_heads + h) * kHeadDim, stride, 0, 0};
      v_tile<BITS>(vs, 0, d[gi].v_tiles, d[gi].v_meta);
    }
  } else {
#pragma unroll 1
  for (int gi = 0; gi < TB / G; ++gi) {
    const int g = blk * (TB / G) + gi;
    if ((g + 1) * G > nq) break;
    GroupDst d;
    if (!group_dst(c, b, h, g, d)) {
      page_bad = true;
      continue;
    }
    const RowSrc ks{k + ((int64_t)(t0 + g * G) * s.num_kv_heads + h) * kHeadDim, stride, 0, 0};
    const RowSrc vs{v + ((int64_t)(t0 + g * G) * s.num_kv_heads + h) * kHeadDim, stride, 0, 0};
    if (G == 16) {
      // a 16-token group has one value tile: value warp 2 + gi takes group
      // gi's, so both value warps work while the key warps take both groups
      const int warp = threadIdx.x >> 5;
      if constexpr (SPARSE) {
        if (warp < 2) k_group_sparse<BITS, 16>(ks, 32 * warp + (threadIdx.x & 31), d.k_codes, d.k_meta, d.k_sparse);
        else if (warp - 2 == gi) v_tile_sparse<BITS>(vs, 0, d.v_tiles, d.v_meta, d.v_sparse);
      } else {
        if (warp < 2) k_group<BITS, G>(ks, 32 * warp + (threadIdx.x & 31), d.k_codes, d.k_meta);
        else if (warp - 2 == gi) v_tile<BITS>(vs, 0, d.v_tiles, d.v_meta);
      }
    } else {
      quantize_group_cta<BITS, G, SPARSE>(ks, vs, d);
    }
  }
  }
  if (page_bad && threadIdx.x == 0) set_err(c.err_word, KVQ_DEVERR_PAGE_RANGE);
  // window tokens of this block -> ring slots t mod (R + G)
  const int lo = max(tb0, nq), hi = min(tb0 + TB, n);
  uint16_t* kr = (uint16_t*)c.k_res;
  uint16_t* vr = (uint16_t*)c.v_res;
  for (int e = threadIdx.x; e < (hi - lo) * 16; e += blockDim.x) {
    const int t = lo + e / 16, piece = e % 16;
    const int64_t src = ((int64_t)(t0 + t) * s.num_kv_heads + h) * kHeadDim + piece * 8;
    const size_t dst = Addr::ring_row(s, b, h, t % Ws) + piece * 8;
    *reinterpret_cast<uint4*>(kr + dst) = *reinterpret_cast<const uint4*>(k + src);
    *reinterpret_cast<uint4*>(vr + dst) = *reinterpret_cast<const uint4*>(v + src);
  }
}

// Grid (H_kv, B), 128 threads: quantizes the oldest G window tokens of
// (b, h) when the window of sequence b holds R + G tokens.  n_quant is left
// alone here (other heads' CTAs of the sequence still read it);
// flush_commit_kernel, next on the stream, advances it.
template <int BITS, int G, bool SPARSE>
__global__ void __launch_bounds__(128) flush_int_kernel(kvq_cache c) {
  grid_dependents_launch();   // the commit kernel may be scheduled; it waits for this grid
  const kvq_shape& s = c.shape;
  const int h = blockIdx.x, b = blockIdx.y;
  const int Ws = window_slots(s);
  const int n = c.seq_len[b], nq = c.n_quant[b];
  if (n - nq != Ws) return;
  if (nq < 0 || nq + G > s.capacity || nq % G) {
    if (threadIdx.x == 0 && h == 0) set_err(c.err_word, KVQ_DEVERR_STATE);
    return;
  }
  GroupDst d;
  if (!group_dst(c, b, h, nq / G, d)) {
    if (threadIdx.x == 0) set_err(c.err_word, KVQ_DEVERR_PAGE_RANGE);
    return;
  }
  const RowSrc ks{(const uint16_t*)c.k_res + Addr::ring_row(s, b, h, 0), kHeadDim, nq % Ws, Ws};
  const RowSrc vs{(const uint16_t*)c.v_res + Addr::ring_row(s, b, h, 0), kHeadDim, nq % Ws, Ws};
  quantize_group_cta<BITS, G, SPARSE>(ks, vs, d);
}

// Grid (B), 32 threads: after flush_int_kernel, advance n_quant of every
// sequence whose window was full and whose group pages were all valid.
__global__ void flush_commit_kernel(kvq_cache c) {
  grid_dependency_wait();     // every flush CTA has read n_quant and written its group
  const kvq_shape& s = c.shape;
  const int b = blockIdx.x;
  const int G = s.group, Ws = window_slots(s);
  const int n = c.seq_len[b], nq = c.n_quant[b];
  if (n - nq != Ws || nq < 0 || nq + G > s.capacity || nq % G) return;
  bool ok = true;
  if (s.page_size != 0) {
    const int page = c.page_table[(size_t)b * s.max_pages_per_seq + nq / G];
    ok = page >= 0 && page < s.num_pages;
  }
  if (ok && threadIdx.x == 0) c.n_quant[b] = nq + G;
}

// Grid (B); block H_kv * 32 threads.  INT formats: token -> window slot
// (MIXED: cls[b], the token's class, into window_class).
__global__ void append_int_kernel(kvq_cache c, const uint16_t* __restrict__ kn, const uint16_t* __restrict__ vn,
                                  const uint8_t* __restrict__ cls) {
  const kvq_shape& s = c.shape;
  const int b = blockIdx.x;
  const int n = c.seq_len[b], nq = c.n_quant[b];
  const int Ws = window_slots(s);
  if (n >= s.capacity || n - nq >= Ws || n < nq) {
    if (threadIdx.x == 0) set_err(c.err_word, KVQ_DEVERR_APPEND_FULL);
    return;
  }
  uint16_t* kr = (uint16_t*)c.k_res;
  uint16_t* vr = (uint16_t*)c.v_res;
  for (int e = threadIdx.x; e < s.num_kv_heads * 16; e += blockDim.x) {
    const int h = e / 16, piece = e % 16;
    const size_t src = ((size_t)b * s.num_kv_heads + h) * kHeadDim + piece * 8;
    const size_t dst = Addr::ring_row(s, b, h, n % Ws) + piece * 8;
    *reinterpret_cast<uint4*>(kr + dst) = *reinterpret_cast<const uint4*>(kn + src);
    *reinterpret_cast<uint4*>(vr + dst) = *reinterpret_cast<const uint4*>(vn + src);
  }
  if (cls && threadIdx.x == 0) c.window_class[(size_t)b * Ws + n % Ws] = cls[b] == 4 ? 4 : 2;
  __syncthreads();
  if (threadIdx.x == 0) c.seq_len[b] = n + 1;
}

// Grid (H_kv, B) in clusters of (H_kv, 1): the CTAs of one sequence form a
// cluster.  Append, then flush when due, in one launch: CTA (h, b) writes the
// new token of kv head h to window slot seq_len mod (R + G); if the window
// now holds R + G tokens it quantizes the oldest G of them (the same group
// kvq_flush_group would take); after a cluster barrier (every CTA of the
// sequence has read seq_len and n_quant) CTA 0 advances seq_len and, after a
// flush, n_quant.  The states, codes and errors equal those of
// kvq_append_token followed by kvq_flush_group.
template <int BITS, int G, bool SPARSE>
__global__ void __launch_bounds__(128) append_flush_int_kernel(kvq_cache c, const uint16_t* __restrict__ kn,
                                                               const uint16_t* __restrict__ vn) {
  const kvq_shape& s = c.shape;
  const int h = blockIdx.x, b = blockIdx.y, t = threadIdx.x;
  const int Ws = window_slots(s);
  // the new token's row is loaded first: its address does not depend on the
  // state, so both loads are in flight together
  const int piece = t & 15;
  uint4 row = make_uint4(0u, 0u, 0u, 0u);
  if (t < 32)
    row = *reinterpret_cast<const uint4*>((t < 16 ? kn : vn) + ((size_t)b * s.num_kv_heads + h) * kHeadDim + piece * 8);
  const int n = c.seq_len[b], nq = c.n_quant[b];
  // append (as kvq_append_token)
  const bool appended = !(n >= s.capacity || n - nq >= Ws || n < nq);
  if (appended) {
    if (t < 32) {
      const size_t dst = Addr::ring_row(s, b, h, n % Ws) + piece * 8;
      *reinterpret_cast<uint4*>((uint16_t*)(t < 16 ? c.k_res : c.v_res) + dst) = row;
    }
  } else if (t == 0 && h == 0) {
    set_err(c.err_word, KVQ_DEVERR_APPEND_FULL);
  }
  // flush (as kvq_flush_group, on the state after the append)
  const int n1 = appended ? n + 1 : n;
  bool flushed = false;
  if (n1 - nq == Ws) {
    if (nq < 0 || nq + G > s.capacity || nq % G) {
      if (t == 0 && h == 0) set_err(c.err_word, KVQ_DEVERR_STATE);
    } else {
      GroupDst d;
      if (!group_dst(c, b, h, nq / G, d)) {
        if (t == 0) set_err(c.err_word, KVQ_DEVERR_PAGE_RANGE);
      } else {
        __syncthreads();   // the appended row is visible to the whole team
        const RowSrc ks{(const uint16_t*)c.k_res + Addr::ring_row(s, b, h, 0), kHeadDim, nq % Ws, Ws};
        const RowSrc vs{(const uint16_t*)c.v_res + Addr::ring_row(s, b, h, 0), kHeadDim, nq % Ws, Ws};
        quantize_group_cta<BITS, G, SPARSE>(ks, vs, d);
        flushed = true;   // the page is the sequence's, so every CTA of the cluster agrees
      }
    }
  }
  // every CTA of the sequence has read seq_len and n_quant before they change
  // (the reads have returned: their values decided the branches above, so a
  // relaxed arrive orders them; the ring and group writes need no ordering
  // against the state update within this launch, the next launch sees them all)
  asm volatile("barrier.cluster.arrive.relaxed.aligned;\nbarrier.cluster.wait.acquire.aligned;\n" ::: "memory");
  if (h == 0 && t == 0) {
    if (appended) c.seq_len[b] = n1;
    if (flushed) c.n_quant[b] = nq + G;
  }
}

// ---------------------------------------------------------------------------
// FP8-E4M3 cache
// ---------------------------------------------------------------------------

// Grid (ceil(max_len/64), H_kv, B): amax |x| over a 64-token chunk of one kv
// head, folded into fp8_amax[0|1][h] (non-negative floats order like their bits).
__global__ void fp8_amax_kernel(kvq_cache c, const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
                                const int32_t* __restrict__ cu, int max_len) {
  const kvq_shape& s = c.shape;
  const int h = blockIdx.y, b = blockIdx.z;
  const int t0 = cu[b];
  const int n = cu[b + 1] - t0;
  if (n > s.capacity || n < 0 || n > max_len) return;
  float ak = 0.f, av = 0.f;
  const int lo = blockIdx.x * 64, hi = min(lo + 64, n);
  for (int e = threadIdx.x; e < (hi - lo) * 16; e += blockDim.x) {
    const int t = lo + e / 16, piece = e % 16;
    const int64_t off = ((int64_t)(t0 + t) * s.num_kv_heads + h) * kHeadDim + piece * 8;
    const uint4 a = *reinterpret_cast<const uint4*>(k + off);
    const uint4 bb = *reinterpret_cast<const uint4*>(v + off);
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      ak = fmaxf(ak, fmaxf(fabsf(bf16_lo(wa[p])), fabsf(bf16_hi(wa[p]))));
      av = fmaxf(av, fmaxf(fabsf(bf16_lo(wb[p])), fabsf(bf16_hi(wb[p]))));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    ak = fmaxf(ak, __shfl_xor_sync(0xffffffffu, ak, off));
    av = fmaxf(av, __shfl_xor_sync(0xffffffffu, av, off));
  }
  if ((threadIdx.x & 31) == 0 && hi > lo) {
    atomicMax(&c.fp8_amax[h], __float_as_uint(ak));
    atomicMax(&c.fp8_amax[s.num_kv_heads + h], __float_as_uint(av));
  }
}

// FP8 value-tile byte of (token i in tile, channel ch).
__device__ __forceinline__ int fp8_vtile_offset(int i, int ch) {
  const int n = ch >> 4, j = ch & 15, l = (i & 7) >> 1, sbit = i >> 3, o = i & 1;
  const int lane = 4 * n + l;
  return 16 * lane + 512 * (j >> 2) + 4 * (j & 3) + 2 * sbit + o;
}

__device__ __forceinline__ void fp8_write_words(const kvq_cache& c, int b, int h, int t, uint2 kx, uint2 vx,
                                                float inv_k, float inv_v, int lane) {
  // lane handles channels 4*lane .. 4*lane+3 (kx, vx: their bf16 words)
  const kvq_shape& s = c.shape;
  const float kf[4] = {bf16_lo(kx.x), bf16_hi(kx.x), bf16_lo(kx.y), bf16_hi(kx.y)};
  const float vf[4] = {bf16_lo(vx.x), bf16_hi(vx.x), bf16_lo(vx.y), bf16_hi(vx.y)};
  uint32_t kw = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) kw |= e4m3_encode(__fmul_rn(kf[i], inv_k)) << (8 * i);
  uint8_t* kc = (uint8_t*)c.k_codes + Addr::k_codes_unit(s, b, h) + (size_t)t * kHeadDim;
  *reinterpret_cast<uint32_t*>(kc + 4 * lane) = kw;
  uint8_t* vt = (uint8_t*)c.v_codes + Addr::v_codes_tile(s, b, h, t / kTile);
#pragma unroll
  for (int i = 0; i < 4; ++i)
    vt[fp8_vtile_offset(t % kTile, 4 * lane + i)] = (uint8_t)e4m3_encode(__fmul_rn(vf[i], inv_v));
}

__device__ __forceinline__ void fp8_write_token(const kvq_cache& c, int b, int h, int t, const uint16_t* krow,
                                                const uint16_t* vrow, float inv_k, float inv_v, int lane) {
  fp8_write_words(c, b, h, t, *reinterpret_cast<const uint2*>(krow + 4 * lane),
                  *reinterpret_cast<const uint2*>(vrow + 4 * lane), inv_k, inv_v, lane);
}

// Grid (ceil(max_len/16), H_kv, B); block 16 warps: warp i encodes token
// 16*blockIdx.x + i (zeros for tokens past the end of the sequence).
__global__ void __launch_bounds__(512) fp8_prefill_kernel(kvq_cache c, const uint16_t* __restrict__ k,
                                                          const uint16_t* __restrict__ v,
                                                          const int32_t* __restrict__ cu, int max_len) {
  const kvq_shape& s = c.shape;
  const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int t0 = cu[b];
  int n = cu[b + 1] - t0;
  const bool too_long = n > s.capacity || n < 0 || n > max_len;
  if (too_long) n = 0;
  const float Sk = fp8_scale_from_amax(__uint_as_float(c.fp8_amax[h]));
  const float Sv = fp8_scale_from_amax(__uint_as_float(c.fp8_amax[s.num_kv_heads + h]));
  if (tile == 0 && threadIdx.x == 0) {
    if (b == 0) {
      c.fp8_scale[h] = Sk;
      c.fp8_scale[s.num_kv_heads + h] = Sv;
    }
    if (h == 0) {
      c.seq_len[b] = n;
      c.n_quant[b] = n;
      if (too_long) set_err(c.err_word, KVQ_DEVERR_PREFILL_LEN);
    }
  }
  if (tile * kTile >= n) return;
  const float inv_k = __frcp_rn(Sk), inv_v = __frcp_rn(Sv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = tile * kTile + warp;
  if (t < n) {
    const int64_t off = ((int64_t)(t0 + t) * s.num_kv_heads + h) * kHeadDim;
    fp8_write_token(c, b, h, t, k + off, v + off, inv_k, inv_v, lane);
  } else {
    uint8_t* vt = (uint8_t*)c.v_codes + Addr::v_codes_tile(s, b, h, tile);
#pragma unroll
    for (int i = 0; i < 4; ++i) vt[fp8_vtile_offset(t % kTile, 4 * lane + i)] = 0;
  }
}

// Grid (B); block H_kv warps.
__global__ void fp8_append_kernel(kvq_cache c, const uint16_t* __restrict__ kn, const uint16_t* __restrict__ vn) {
  const kvq_shape& s = c.shape;
  const int b = blockIdx.x;
  const int h = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the new rows and the head's scales do not depend on the state: their
  // loads are issued with the state's
  uint2 kx = make_uint2(0u, 0u), vx = make_uint2(0u, 0u);
  float Sk = 1.f, Sv = 1.f;
  if (h < s.num_kv_heads) {
    const size_t off = ((size_t)b * s.num_kv_heads + h) * kHeadDim;
    kx = *reinterpret_cast<const uint2*>(kn + off + 4 * lane);
    vx = *reinterpret_cast<const uint2*>(vn + off + 4 * lane);
    Sk = c.fp8_scale[h];
    Sv = c.fp8_scale[s.num_kv_heads + h];
  }
  const int n = c.seq_len[b];
  if (n >= s.capacity || n < 0) {
    if (threadIdx.x == 0) set_err(c.err_word, KVQ_DEVERR_APPEND_FULL);
    return;
  }
  if (h < s.num_kv_heads) fp8_write_words(c, b, h, n, kx, vx, __frcp_rn(Sk), __frcp_rn(Sv), lane);
  __syncthreads();
  if (threadIdx.x == 0) {
    c.seq_len[b] = n + 1;
    c.n_quant[b] = n + 1;
  }
}

// ---------------------------------------------------------------------------
// MIXED cache: INT4 or INT2 per group by the classes of its tokens
// ---------------------------------------------------------------------------

// Grid (ceil(max_len / G), H_kv, B), 128 threads: one group per CTA (G >= 32),
// stored at 4 bits if any of its tokens has class 4, else at 2; then the
// block's window tokens and their classes.  Registers are cut for 7 CTAs
// per SM (72 registers, some spill): 73.8 against 82.1 us at 5 on the 8B
// layer, no better at 8 or 10.
template <int G>
__global__ void __launch_bounds__(128, 7) prefill_mixed_kernel(kvq_cache c, const uint16_t* __restrict__ k,
                                                               const uint16_t* __restrict__ v,
                                                               const uint8_t* __restrict__ cls,
                                                               const int32_t* __restrict__ cu, int max_len) {
  static_assert(G >= 32, "one group per CTA");
  const kvq_shape& s = c.shape;
  const int g = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int Ws = window_slots(s);
  const int t0 = cu[b];
  int n = cu[b + 1] - t0;
  const bool too_long = n > s.capacity || n < 0 || n > max_len;
  if (too_long) n = 0;
  const int nq = quantized_prefix(n, s.residual, G);
  if (g == 0 && h == 0 && threadIdx.x == 0) {
    c.seq_len[b] = n;
    c.n_quant[b] = nq;
    if (too_long) set_err(c.err_word, KVQ_DEVERR_PREFILL_LEN);
  }
  const int tb0 = g * G;
  if (tb0 >= n) return;
  if ((g + 1) * G <= nq) {
    const bool four = __syncthreads_or(threadIdx.x < G && cls[t0 + tb0 + threadIdx.x] == 4) != 0;
    if (h == 0 && threadIdx.x == 0) c.group_bits[(size_t)b * (s.capacity / G) + g] = four ? 4 : 2;
    GroupDst d;
    group_dst(c, b, h, g, d);     // contiguous: always valid
    const int64_t stride = (int64_t)s.num_kv_heads * kHeadDim;
    const RowSrc ks{k + ((int64_t)(t0 + tb0) * s.num_kv_heads + h) * kHeadDim, stride, 0, 0};
    const RowSrc vs{v + ((int64_t)(t0 + tb0) * s.num_kv_heads + h) * kHeadDim, stride, 0, 0};
    quantize_group_mixed<G>(four, ks, vs, d);
  }
  // window tokens of this block -> ring slots t mod (R + G), with their classes
  const int lo = max(tb0, nq), hi = min(tb0 + G, n);
  uint16_t* kr = (uint16_t*)c.k_res;
  uint16_t* vr = (uint16_t*)c.v_res;
  for (int e = threadIdx.x; e < (hi - lo) * 16; e += blockDim.x) {
    const int t = lo + e / 16, piece = e % 16;
    const int64_t src = ((int64_t)(t0 + t) * s.num_kv_heads + h) * kHeadDim + piece * 8;
    const size_t dst = Addr::ring_row(s, b, h, t % Ws) + piece * 8;
    *reinterpret_cast<uint4*>(kr + dst) = *reinterpret_cast<const uint4*>(k + src);
    *reinterpret_cast<uint4*>(vr + dst) = *reinterpret_cast<const uint4*>(v + src);
  }
  if (h == 0)
    for (int t = lo + (int)threadIdx.x; t < hi; t += blockDim.x)
      c.window_class[(size_t)b * Ws + t % Ws] = cls[t0 + t] == 4 ? 4 : 2;
}

// Grid (H_kv, B), 128 threads: the flush of a MIXED cache (as
// flush_int_kernel), the group stored at the widest class of its G window
// tokens; flush_commit_kernel advances n_quant.
template <int G>
__global__ void __launch_bounds__(128) flush_mixed_kernel(kvq_cache c) {
  grid_dependents_launch();
  const kvq_shape& s = c.shape;
  const int h = blockIdx.x, b = blockIdx.y;
  const int Ws = window_slots(s);
  const int n = c.seq_len[b], nq = c.n_quant[b];
  if (n - nq != Ws) return;
  if (nq < 0 || nq + G > s.capacity || nq % G) {
    if (threadIdx.x == 0 && h == 0) set_err(c.err_word, KVQ_DEVERR_STATE);
    return;
  }
  const bool four =
      __syncthreads_or(threadIdx.x < G && c.window_class[(size_t)b * Ws + (nq + threadIdx.x) % Ws] == 4) != 0;
  if (h == 0 && threadIdx.x == 0) c.group_bits[(size_t)b * (s.capacity / G) + nq / G] = four ? 4 : 2;
  GroupDst d;
  group_dst(c, b, h, nq / G, d);
  const RowSrc ks{(const uint16_t*)c.k_res + Addr::ring_row(s, b, h, 0), kHeadDim, nq % Ws, Ws};
  const RowSrc vs{(const uint16_t*)c.v_res + Addr::ring_row(s, b, h, 0), kHeadDim, nq % Ws, Ws};
  quantize_group_mixed<G>(four, ks, vs, d);
}

// ---------------------------------------------------------------------------
// INT8 per-token cache: every key and value row quantized over its 128
// channels at 8 bits when it is written (no window)
// ---------------------------------------------------------------------------

// One 16-token tile of rows (key or value) of one (sequence, kv head): lane
// (n, l) holds channels [16n, 16n+16) of tokens 2l, 2l+1, 2l+8, 2l+9 of the
// tile (rows past `valid` read as zeros, which quantize to code 0, scale 0,
// zero 0).  Per-token min/max is reduced in registers, then over the 8
// lanes that share the tokens.  KEY: codes go to canonical rows (byte c =
// channel c) at codes + token * 128; otherwise to the value tile layout
// (include/kvq.h, "FP8 and INT8"), which is exactly this lane's own 64
// bytes.  meta: [16][2] fp16 (scale, zero) of the tile's tokens.
template <bool KEY>
__device__ __forceinline__ void int8_token_tile(const uint16_t* rows, int64_t stride, int valid, uint8_t* codes,
                                                __half* meta) {
  const int lane = threadIdx.x & 31;
  const int n = lane >> 2, l = lane & 3;
  const int tok[4] = {2 * l, 2 * l + 1, 2 * l + 8, 2 * l + 9};
  uint32_t x[4][8];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    if (tok[q] < valid) {
      const uint16_t* r = rows + (int64_t)tok[q] * stride + 16 * n;
      const uint4 a = *reinterpret_cast<const uint4*>(r);
      const uint4 b = *reinterpret_cast<const uint4*>(r + 8);
      x[q][0] = a.x; x[q][1] = a.y; x[q][2] = a.z; x[q][3] = a.w;
      x[q][4] = b.x; x[q][5] = b.y; x[q][6] = b.z; x[q][7] = b.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) x[q][i] = 0u;
    }
  }
  // per-token (min, -max) as one bf16x2 word, reduced over the token's 8 lanes
  uint32_t mm[4];
  bool nan_free = true;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t a = x[q][0], b = x[q][0];
#pragma unroll
    for (int i = 1; i < 8; ++i) {
      a = bmin2_nan(a, x[q][i]);
      b = bmax2_nan(b, x[q][i]);
    }
    a = bmin2_nan(a, prmt(a, a, 0x1032u));
    b = bmax2_nan(b, prmt(b, b, 0x1032u));
    mm[q] = prmt(a, b ^ 0x80008000u, 0x7610u);
  }
#pragma unroll
  for (int off = 4; off < 32; off <<= 1)
#pragma unroll
    for (int q = 0; q < 4; ++q) mm[q] = bmin2_nan(mm[q], __shfl_xor_sync(0xffffffffu, mm[q], off));
#pragma unroll
  for (int q = 0; q < 4; ++q) nan_free = nan_free && !bf16x2_has_nan(mm[q]);
  // codes of token q, channel pair ww: low bytes of cl[q][ww] (channel 2ww)
  // and ch[q][ww] (channel 2ww + 1)
  uint32_t cl[4][8], ch[4][8];
  QParams qp[4];
  bool fast = false;
  if (__all_sync(0xffffffffu, nan_free)) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float tmn = bf16_lo(mm[q]), tmx = -bf16_hi(mm[q]);
      qp[q] = quant_params(tmn, tmx, 8);
    }
    bool ok = true;
#pragma unroll
    for (int q = 0; q < 4; ++q) ok = ok && clamp_free(bf16_lo(mm[q]), -bf16_hi(mm[q]), qp[q], 255);
    fast = __all_sync(0xffffffffu, ok);
  }
  if (fast) {
    const u64 one2 = kOnePair;
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int ww = 0; ww < 8; ++ww)
        encode2_fast(x[q][ww], pack_f2(qp[q].z, qp[q].z), pack_f2(qp[q].inv, qp[q].inv), one2, cl[q][ww],
                     ch[q][ww]);
  } else {
    // exact scalar path: min/max ignoring NaN, clamped codes
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float mn = INFINITY, mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        mn = fminf(mn, fminf(bf16_lo(x[q][i]), bf16_hi(x[q][i])));
        mx = fmaxf(mx, fmaxf(bf16_lo(x[q][i]), bf16_hi(x[q][i])));
      }
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      }
      qp[q] = quant_params(mn, mx, 8);
#pragma unroll
      for (int ww = 0; ww < 8; ++ww) {
        cl[q][ww] = encode(bf16_lo(x[q][ww]), qp[q].z, qp[q].inv, 255);
        ch[q][ww] = encode(bf16_hi(x[q][ww]), qp[q].z, qp[q].inv, 255);
      }
    }
  }
  if (KEY) {
    // token q's 16 channels = 4 words of 4 codes, one 16-byte store per token
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (tok[q] >= valid) continue;
      uint32_t w[4];
#pragma unroll
      for (int m = 0; m < 4; ++m)
        w[m] = prmt(prmt(cl[q][2 * m], ch[q][2 * m], 0x0040u), prmt(cl[q][2 * m + 1], ch[q][2 * m + 1], 0x0040u),
                    0x5410u);
      *reinterpret_cast<uint4*>(codes + (size_t)tok[q] * kHeadDim + 16 * n) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  } else {
    // word j (channel 16n + j) = the codes of tokens 2l, 2l+1, 2l+8, 2l+9
    uint32_t w[16];
#pragma unroll
    for (int ww = 0; ww < 8; ++ww) {
      w[2 * ww] = prmt(prmt(cl[0][ww], cl[1][ww], 0x0040u), prmt(cl[2][ww], cl[3][ww], 0x0040u), 0x5410u);
      w[2 * ww + 1] = prmt(prmt(ch[0][ww], ch[1][ww], 0x0040u), prmt(ch[2][ww], ch[3][ww], 0x0040u), 0x5410u);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<uint4*>(codes + 16 * lane + 512 * i) = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2],
                                                                          w[4 * i + 3]);
  }
  // (scale, zero) of token q, written by lane (n = q, l) for n < 4
  if (n < 4) {
    uint32_t m = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (q == n) m = (uint32_t)__half_as_ushort(qp[q].s16) | ((uint32_t)__half_as_ushort(qp[q].z16) << 16);
    *reinterpret_cast<uint32_t*>(meta + 2 * tok[n]) = m;
  }
}

// Grid (ceil(max_len / 32), H_kv, B), 128 threads: warps 0 and 1 quantize
// the key rows of the block's two 16-token tiles, warps 2 and 3 the value
// rows.  Tokens of a sequence's last tile past its length are stored as
// code 0 with scale and zero 0.  Registers are cut for 6 CTAs per SM (80,
// some spill): 84.0 against 88.1 us at 5 on the 8B layer; 8 is slower.
__global__ void __launch_bounds__(128, 6) prefill_int8_kernel(kvq_cache c, const uint16_t* __restrict__ k,
                                                           const uint16_t* __restrict__ v,
                                                           const int32_t* __restrict__ cu, int max_len) {
  const kvq_shape& s = c.shape;
  const int blk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int t0 = cu[b];
  int n = cu[b + 1] - t0;
  const bool too_long = n > s.capacity || n < 0 || n > max_len;
  if (too_long) n = 0;
  if (blk == 0 && h == 0 && threadIdx.x == 0) {
    c.seq_len[b] = n;
    c.n_quant[b] = n;
    if (too_long) set_err(c.err_word, KVQ_DEVERR_PREFILL_LEN);
  }
  const int tile = 2 * blk + (warp & 1);
  if (tile * kTile >= n) return;
  const int valid = min(kTile, n - tile * kTile);
  const int64_t stride = (int64_t)s.num_kv_heads * kHeadDim;
  const int64_t row0 = ((int64_t)(t0 + tile * kTile) * s.num_kv_heads + h) * kHeadDim;
  if (warp < 2) {
    uint8_t* kc = (uint8_t*)c.k_codes + Addr::k_codes_unit(s, b, h) + (size_t)tile * kTile * kHeadDim;
    __half* km = (__half*)c.k_meta + Addr::k_meta_token(s, b, h, tile * kTile);
    int8_token_tile<true>(k + row0, stride, valid, kc, km);
  } else {
    uint8_t* vt = (uint8_t*)c.v_codes + Addr::v_codes_tile(s, b, h, tile);
    __half* vm = (__half*)c.v_meta + Addr::v_meta_token(s, b, h, tile * kTile);
    int8_token_tile<false>(v + row0, stride, valid, vt, vm);
  }
}

// One token row of 128 channels quantized by one warp (lane: channels
// 4 lane .. 4 lane + 3): returns the four codes in the bytes of a word and
// the (scale, zero) pair as a word.
__device__ __forceinline__ uint32_t int8_encode_words(uint2 xw, uint32_t& meta) {
  const float xf[4] = {bf16_lo(xw.x), bf16_hi(xw.x), bf16_lo(xw.y), bf16_hi(xw.y)};
  float mn = fminf(fminf(xf[0], xf[1]), fminf(xf[2], xf[3]));   // fminf/fmaxf ignore NaN
  float mx = fmaxf(fmaxf(xf[0], xf[1]), fmaxf(xf[2], xf[3]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  }
  const QParams qp = quant_params(mn, mx, 8);
  uint32_t w = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) w |= encode(xf[i], qp.z, qp.inv, 255) << (8 * i);
  meta = (uint32_t)__half_as_ushort(qp.s16) | ((uint32_t)__half_as_ushort(qp.z16) << 16);
  return w;
}

// Grid (B); block H_kv warps: warp h quantizes sequence b's new key and
// value rows of kv head h into token seq_len[b]; then seq_len and n_quant
// advance together.  The rows are loaded and encoded before the state is
// needed (only the stores depend on it), so the row and state loads are in
// flight together.
__global__ void append_int8_kernel(kvq_cache c, const uint16_t* __restrict__ kn, const uint16_t* __restrict__ vn) {
  const kvq_shape& s = c.shape;
  const int b = blockIdx.x;
  const int h = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint2 kx = make_uint2(0u, 0u), vx = make_uint2(0u, 0u);
  const size_t off = ((size_t)b * s.num_kv_heads + h) * kHeadDim;
  if (h < s.num_kv_heads) {
    kx = *reinterpret_cast<const uint2*>(kn + off + 4 * lane);
    vx = *reinterpret_cast<const uint2*>(vn + off + 4 * lane);
  }
  const int n = c.seq_len[b], nq = c.n_quant[b];
  uint32_t km = 0, vm = 0, kw = 0, vw = 0;
  if (h < s.num_kv_heads) {
    kw = int8_encode_words(kx, km);
    vw = int8_encode_words(vx, vm);
  }
  if (n >= s.capacity || n < 0 || nq != n) {
    if (threadIdx.x == 0) set_err(c.err_word, KVQ_DEVERR_APPEND_FULL);
    return;
  }
  if (h < s.num_kv_heads) {
    uint8_t* kc = (uint8_t*)c.k_codes + Addr::k_codes_unit(s, b, h) + (size_t)n * kHeadDim;
    *reinterpret_cast<uint32_t*>(kc + 4 * lane) = kw;
    uint8_t* vt = (uint8_t*)c.v_codes + Addr::v_codes_tile(s, b, h, n / kTile);
#pragma unroll
    for (int i = 0; i < 4; ++i) vt[fp8_vtile_offset(n % kTile, 4 * lane + i)] = (uint8_t)(vw >> (8 * i));
    if (lane == 0) {
      *reinterpret_cast<uint32_t*>((__half*)c.k_meta + Addr::k_meta_token(s, b, h, n)) = km;
      *reinterpret_cast<uint32_t*>((__half*)c.v_meta + Addr::v_meta_token(s, b, h, n)) = vm;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    c.seq_len[b] = n + 1;
    c.n_quant[b] = n + 1;
  }
}

// ---------------------------------------------------------------------------
// Host launchers (called by kvq_api.cu after validation)
// ---------------------------------------------------------------------------

cudaError_t launch_prefill(const kvq_cache& c, const void* k, const void* v, const int32_t* cu, int max_len,
                           cudaStream_t st) {
  const kvq_shape& s = c.shape;
  const int limit = max_len;           // longer sequences are rejected on the device
  if (max_len <= 0) max_len = 1;
  if (is_int8(s.format)) {
    dim3 g8((max_len + 2 * kTile - 1) / (2 * kTile), s.num_kv_heads, s.batch);
    prefill_int8_kernel<<<g8, 128, 0, st>>>(c, (const uint16_t*)k, (const uint16_t*)v, cu, limit);
    return cudaGetLastError();
  }
  if (is_fp8(s.format)) {
    cudaError_t e = cudaMemsetAsync(c.fp8_amax, 0, sizeof(uint32_t) * 2 * s.num_kv_heads, st);
    if (e != cudaSuccess) return e;
    dim3 ga((max_len + 63) / 64, s.num_kv_heads, s.batch);
    fp8_amax_kernel<<<ga, 128, 0, st>>>(c, (const uint16_t*)k, (const uint16_t*)v, cu, limit);
    dim3 gp((max_len + kTile - 1) / kTile, s.num_kv_heads, s.batch);
    fp8_prefill_kernel<<<gp, 32 * kTile, 0, st>>>(c, (const uint16_t*)k, (const uint16_t*)v, cu, limit);
    return cudaGetLastError();
  }
  const int TB = s.group < 32 ? 32 : s.group;
  dim3 grid((max_len + TB - 1) / TB, s.num_kv_heads, s.batch);
  const uint16_t* kk = (const uint16_t*)k;
  const uint16_t* vv = (const uint16_t*)v;
#define KVQ_PREFILL_CASE(B, GG) \
  if (s.format == B && s.group == GG && !s.sparse) prefill_int_kernel<B, GG, false><<<grid, 128, 0, st>>>(c, kk, vv, cu, limit);
#define KVQ_PREFILL_SPARSE_CASE(B, GG) \
  if (s.format == B && s.group == GG && s.sparse) prefill_int_kernel<B, GG, true><<<grid, 128, 0, st>>>(c, kk, vv, cu, limit);
  KVQ_PREFILL_CASE(4, 16) KVQ_PREFILL_CASE(4, 32) KVQ_PREFILL_CASE(4, 64) KVQ_PREFILL_CASE(4, 128)
  KVQ_PREFILL_CASE(2, 16) KVQ_PREFILL_CASE(2, 32) KVQ_PREFILL_CASE(2, 64) KVQ_PREFILL_CASE(2, 128)
  KVQ_PREFILL_SPARSE_CASE(4, 16) KVQ_PREFILL_SPARSE_CASE(4, 32) KVQ_PREFILL_SPARSE_CASE(2, 16) KVQ_PREFILL_SPARSE_CASE(2, 32)
#undef KVQ_PREFILL_CASE
#undef KVQ_PREFILL_SPARSE_CASE
  return cudaGetLastError();
}

cudaError_t launch_prefill_mixed(const kvq_cache& c, const void* k, const void* v, const uint8_t* cls,
                                 const int32_t* cu, int max_len, cudaStream_t st) {
  const kvq_shape& s = c.shape;
  const int limit = max_len;
  if (max_len <= 0) max_len = 1;
  dim3 grid((max_len + s.group - 1) / s.group, s.num_kv_heads, s.batch);
  const uint16_t* kk = (const uint16_t*)k;
  const uint16_t* vv = (const uint16_t*)v;
  if (s.group == 32) prefill_mixed_kernel<32><<<grid, 128, 0, st>>>(c, kk, vv, cls, cu, limit);
  else if (s.group == 64) prefill_mixed_kernel<64><<<grid, 128, 0, st>>>(c, kk, vv, cls, cu, limit);
  else if (s.group == 128) prefill_mixed_kernel<128><<<grid, 128, 0, st>>>(c, kk, vv, cls, cu, limit);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_append_mixed(const kvq_cache& c, const void* kn, const void* vn, const uint8_t* cls,
                                cudaStream_t st) {
  const kvq_shape& s = c.shape;
  append_int_kernel<<<s.batch, 32 * min(s.num_kv_heads, 32), 0, st>>>(c, (const uint16_t*)kn, (const uint16_t*)vn,
                                                                      cls);
  return cudaGetLastError();
}

cudaError_t launch_append(const kvq_cache& c, const void* kn, const void* vn, cudaStream_t st) {
  const kvq_shape& s = c.shape;
  if (is_fp8(s.format))
    fp8_append_kernel<<<s.batch, 32 * s.num_kv_heads, 0, st>>>(c, (const uint16_t*)kn, (const uint16_t*)vn);
  else if (is_int8(s.format))
    append_int8_kernel<<<s.batch, 32 * s.num_kv_heads, 0, st>>>(c, (const uint16_t*)kn, (const uint16_t*)vn);
  else
    append_int_kernel<<<s.batch, 32 * min(s.num_kv_heads, 32), 0, st>>>(c, (const uint16_t*)kn,
                                                                        (const uint16_t*)vn, nullptr);
  return cudaGetLastError();
}

cudaError_t launch_flush(const kvq_cache& c, cudaStream_t st);

// Append and flush in one launch (one cluster of H_kv CTAs per sequence)
// when the kv heads fit a portable cluster; otherwise the two calls.
cudaError_t launch_append_flush(const kvq_cache& c, const void* kn, const void* vn, cudaStream_t st) {
  const kvq_shape& s = c.shape;
  if (is_token_cache(s.format) || s.num_kv_heads > 8) {
    cudaError_t e = launch_append(c, kn, vn, st);
    return e != cudaSuccess ? e : launch_flush(c, st);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(s.num_kv_heads, s.batch);
  cfg.blockDim = dim3(128);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = s.num_kv_heads;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const uint16_t* k16 = (const uint16_t*)kn;
  const uint16_t* v16 = (const uint16_t*)vn;
#define KVQ_APPEND_FLUSH_CASE(B, GG, SP) \
  if (s.format == B && s.group == GG && (bool)s.sparse == SP) \
    return cudaLaunchKernelEx(&cfg, append_flush_int_kernel<B, GG, SP>, c, k16, v16);
  KVQ_APPEND_FLUSH_CASE(4, 16, false) KVQ_APPEND_FLUSH_CASE(4, 32, false) KVQ_APPEND_FLUSH_CASE(4, 64, false)
  KVQ_APPEND_FLUSH_CASE(4, 128, false) KVQ_APPEND_FLUSH_CASE(2, 16, false) KVQ_APPEND_FLUSH_CASE(2, 32, false)
  KVQ_APPEND_FLUSH_CASE(2, 64, false) KVQ_APPEND_FLUSH_CASE(2, 128, false)
  KVQ_APPEND_FLUSH_CASE(4, 16, true) KVQ_APPEND_FLUSH_CASE(4, 32, true) KVQ_APPEND_FLUSH_CASE(2, 16, true)
  KVQ_APPEND_FLUSH_CASE(2, 32, true)
#undef KVQ_APPEND_FLUSH_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_flush(const kvq_cache& c, cudaStream_t st) {
  const kvq_shape& s = c.shape;
  if (is_token_cache(s.format)) return cudaSuccess;
  dim3 grid(s.num_kv_heads, s.batch);
  if (is_mixed(s.format)) {
    if (s.group == 32) flush_mixed_kernel<32><<<grid, 128, 0, st>>>(c);
    else if (s.group == 64) flush_mixed_kernel<64><<<grid, 128, 0, st>>>(c);
    else if (s.group == 128) flush_mixed_kernel<128><<<grid, 128, 0, st>>>(c);
  }
#define KVQ_FLUSH_CASE(B, GG, SP) \
  if (s.format == B && s.group == GG && (bool)s.sparse == SP) flush_int_kernel<B, GG, SP><<<grid, 128, 0, st>>>(c);
  KVQ_FLUSH_CASE(4, 16, false) KVQ_FLUSH_CASE(4, 32, false) KVQ_FLUSH_CASE(4, 64, false) KVQ_FLUSH_CASE(4, 128, false)
  KVQ_FLUSH_CASE(2, 16, false) KVQ_FLUSH_CASE(2, 32, false) KVQ_FLUSH_CASE(2, 64, false) KVQ_FLUSH_CASE(2, 128, false)
  KVQ_FLUSH_CASE(4, 16, true) KVQ_FLUSH_CASE(4, 32, true) KVQ_FLUSH_CASE(2, 16, true) KVQ_FLUSH_CASE(2, 32, true)
#undef KVQ_FLUSH_CASE
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // the commit is launched early (programmatic dependent launch) and waits
  // on the device, which hides its launch latency behind the flush
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(s.batch);
  cfg.blockDim = dim3(32);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  pdl_attribute(attr[0]);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, flush_commit_kernel, c);
}

}  // namespace kvq
