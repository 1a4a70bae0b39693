// Decode attention over the packed cache (split-K / flash-decoding).
//
// INT2/INT4 (decode_int_kernel + decode_int_combine_kernel): a persistent
// grid of 148 x 3 CTAs of 4 warps.  The quantized 32-token chunks of all
// (sequence, kv head) units are laid end to end and warp p streams the
// slice [p C / P, (p+1) C / P) through a private ring of shared-memory
// stages filled by per-lane cp.async copies, writing one partial per unit
// it touches; the bf16 window's 16-token tiles are spread over the warps
// that share the unit.  The combine kernel merges a unit's partials.
// FP8 (decode_fp8_kernel + decode_combine_kernel): grid (splits, H_kv, B),
// kWarps warps per CTA; split s owns a contiguous range of chunks and each
// warp a sub-range, streamed through a ring filled by per-lane cp.async
// copies.
//
// Scores and the value sum run on the tensor cores (mma.sync m16n8k16, fp32
// accumulate) fed from registers:
//  * QK (INT): A = the query times the group's per-channel key scale,
//    q''[h][c] = q[h][c] 2^-a s_k[c], as fp16 hi (rows 0-7) and lo (rows
//    8-15) parts; B = the key codes as exact fp16 numbers.  An INT4 code
//    masked into a byte is the e4m3 number code * 2^-9, which the hardware
//    e4m3x2 -> f16x2 converter turns into an exact normal fp16 (the score
//    sum is scaled back by 2^9); an INT2 code OR-ed into the mantissa of
//    1024.0 is 1024 + 2^k code, and one fused multiply-add removes the
//    offset and the position factor exactly.  The zero-point term
//    sum_c q[h][c] z_k[c] is a second small MMA per group.
//  * PV (INT): transposed, O^T += V^T P'^T: A = value codes (16 channels x
//    16 tokens, INT2 and INT4 through the e4m3 converter as code * 2^-9),
//    B = P' = p[h][t] s_v[t] as fp16 hi/lo columns (the window's P' scaled
//    by 2^-9 to match; the accumulators are scaled back when a unit ends);
//    the value zero points add sum_t p[h][t] z_v[t].
//    (Codes are not fed as fp16 subnormals: measured on this tensor core,
//    sums with subnormal operands lose about 1e-6 to 1e-4 relative
//    accuracy, while normal operands stay near fp32 rounding.)
//  * FP8: e4m3 codes convert to fp16 exactly (one instruction per pair);
//    one static scale per kv head for keys and one for values.
//
// Softmax is online per warp (running max in log2 units, rescaled only when
// a chunk raises it); partials are merged across warps and splits at the end.
#include <atomic>
#include <type_traits>

#include "kvq_common.cuh"

namespace kvq {

constexpr int kWarps = 4;
constexpr int kFp8MinBlocks = 3;  // CTAs per SM the FP8 kernel's registers are cut for
constexpr int kChunk = 32;          // tokens per pipeline stage (two tiles)
constexpr int kMergeStride = 132;   // floats per (warp, head) row of the merge buffer (16-byte rows)

// Template format codes: 2, 4 = INT2/INT4 (per-channel key groups, bf16
// window); 8 = FP8-E4M3; 16 = INT8 per token (kvq_format values).
template <int FMT> struct DecodeCfg;   // kRB: bytes of codes per token row
template <> struct DecodeCfg<4> { static constexpr int kRB = 64; };
template <> struct DecodeCfg<2> { static constexpr int kRB = 32; };
template <> struct DecodeCfg<8> { static constexpr int kRB = 128; };
template <> struct DecodeCfg<16> { static constexpr int kRB = 128; };
template <> struct DecodeCfg<6> { static constexpr int kRB = 64; };   // MIXED: slots sized as INT4

template <int FMT> struct Stage {
  static constexpr int kTB = kTile * DecodeCfg<FMT>::kRB;           // one tile of codes
  static constexpr int kK = 0;                                      // 2 tiles of key rows
  static constexpr int kV = 2 * kTB;                                // 2 value tiles
  static constexpr int kVm = 4 * kTB;                               // INT: 2 x [16][2] fp16
  // INT2/4: up to 2 x [2][128] fp16 key group tables; INT8: 2 x [16][2]
  // fp16 per-token key (scale, zero)
  static constexpr int kKm = kVm + (FMT == 8 ? 0 : 128);
  static constexpr int kBytes = kKm + (FMT == 8 ? 0 : (FMT == 16 ? 128 : 1024));
};
// MIXED: a stage holds a chunk of either width, laid out as that width's
// stage (INT4 is the larger).
template <> struct Stage<6> : Stage<4> {};

constexpr int kQStashBytes = 32 * 16 * 4;   // per warp: the lanes' 16 query-pair words

// FP8 kernel: per warp a ring of kFp8Stages stages; the rings become the
// CTA's merge buffer at the end.
constexpr int kFp8Stages = 2;
constexpr int fp8_smem_bytes() { return kWarps * kFp8Stages * Stage<8>::kBytes; }
static_assert(kWarps * 8 * kMergeStride * 4 <= kWarps * kFp8Stages * Stage<8>::kBytes, "merge buffer fits the rings");

constexpr float kLn2 = 0.69314718055994531f;   // ln 2: log2 units -> natural-log units

struct DecodeArgs {
  kvq_cache c;
  const uint16_t* q;       // [B][H_q][128] bf16
  float* ws_o;             // [B][H_q][S][128]
  float* ws_ml;            // [B][H_q][S][2]
  float scale_log2;        // softmax_scale * log2(e)
  int num_splits;          // S
};

struct SoftmaxState {
  float m;        // running max (log2 units) of this thread's head
  float l;        // this thread's share of the running sum
  float z;        // this thread's share of sum p * z_v
};

__device__ __forceinline__ float quad_max(float x) {
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 1));
  return fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 2));
}
__device__ __forceinline__ float quad_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  return x + __shfl_xor_sync(0xffffffffu, x, 2);
}

// Raise the running max to cover `tmax`; rescale this warp's accumulators if
// any head's max grew.
__device__ __forceinline__ void online_max_update(float tmax, SoftmaxState& st, float (&O)[16][4]) {
  const float mnew = fmaxf(st.m, tmax);
  const bool grow = mnew > st.m;
  if (__any_sync(0xffffffffu, grow)) {
    const float alpha = (st.m == -INFINITY) ? 0.f : ex2(st.m - mnew);
    const float a = grow ? alpha : 1.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      O[j][0] *= a; O[j][1] *= a; O[j][2] *= a; O[j][3] *= a;
    }
    st.l *= a;
    st.z *= a;
    st.m = mnew;
  }
}

// Packed half / bfloat16 arithmetic through PTX (one instruction each).
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;\n" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;\n" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
// a * b - c in both halves (the negation folds into the fma's operand).
__device__ __forceinline__ uint32_t hfms2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("{\n .reg .b32 t;\n neg.f16x2 t, %3;\n fma.rn.f16x2 %0, %1, %2, t;\n}\n" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// 1024 + f*code (both halves) -> code, exactly: x/f - 1024/f in one fma
// (every value involved is an fp16 number in [1024, 2048) or a small integer).
template <int F>
__device__ __forceinline__ uint32_t unmagic(uint32_t x) {
  constexpr uint32_t lf = F == 1 ? 0 : (F == 4 ? 2 : (F == 16 ? 4 : (F == 64 ? 6 : 8)));   // log2 F
  constexpr uint32_t inv = (15u - lf) << 10;                      // 2^-lf
  constexpr uint32_t off = 0x8000u | ((25u - lf) << 10);         // -(1024 / F)
  return hfma2(x, inv | (inv << 16), off | (off << 16));
}
__device__ __forceinline__ uint32_t magic(uint32_t w, uint32_t mask) { return lop_or(w, mask, 0x64006400u); }


// Per-warp result -> shared memory; the CTA merges its warps and writes one
// split partial.  sm: kWarps * 8 * kMergeStride floats.
__device__ __forceinline__ void cta_merge_and_store(float* sm, const SoftmaxState& st, const float (&O)[16][4],
                                                   float out_scale, int gq, const DecodeArgs& A, int b, int kv,
                                                   int split) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, l = lane & 3;
  const float lsum = quad_sum(st.l);
  const float zsum = quad_sum(st.z);
  float* wo = sm + (size_t)(warp * 8 + g) * kMergeStride;
  float4* o4 = reinterpret_cast<float4*>(wo + 32 * l);
  // channel 32l + j comes from column 2l of n-tile j, 32l + 16 + j from column 2l+1
  float v0[16], v1[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    v0[j] = (O[j][0] + O[j][2]) * out_scale + zsum;
    v1[j] = (O[j][1] + O[j][3]) * out_scale + zsum;
  }
#pragma unroll
  for (int j4 = 0; j4 < 4; ++j4) {
    o4[j4] = make_float4(v0[4 * j4], v0[4 * j4 + 1], v0[4 * j4 + 2], v0[4 * j4 + 3]);
    o4[4 + j4] = make_float4(v1[4 * j4], v1[4 * j4 + 1], v1[4 * j4 + 2], v1[4 * j4 + 3]);
  }
  if (l == 0) {
    wo[128] = st.m;
    wo[129] = lsum;
  }
  __syncthreads();
  const kvq_shape& s = A.c.shape;
  for (int e = threadIdx.x; e < gq * kHeadDim; e += blockDim.x) {
    const int hh = e / kHeadDim, ch = e % kHeadDim;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm[(w * 8 + hh) * kMergeStride + 128]);
    float o = 0.f, L = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float* x = sm + (w * 8 + hh) * kMergeStride;
        const float f = ex2(x[128] - M);
        o += f * x[ch];
        L += f * x[129];
      }
    }
    const int h = kv * gq + hh;
    const size_t row = ((size_t)b * s.num_q_heads + h) * A.num_splits + split;
    A.ws_o[row * kHeadDim + ch] = o;
    if (ch == 0) {
      A.ws_ml[row * 2] = M;
      A.ws_ml[row * 2 + 1] = L;
    }
  }
}

// bf16 query of this thread's head (row g), channels [32l, 32l+32), as 16
// words of adjacent channel pairs.
__device__ __forceinline__ void load_q_words(const DecodeArgs& A, int b, int kv, int gq, uint32_t (&qw)[16]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, l = lane & 3;
  const kvq_shape& s = A.c.shape;
  if (g < gq) {
    const uint4* qr = reinterpret_cast<const uint4*>(A.q + ((size_t)b * s.num_q_heads + kv * gq + g) * kHeadDim +
                                                     32 * l);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 v = qr[i];
      qw[4 * i] = v.x; qw[4 * i + 1] = v.y; qw[4 * i + 2] = v.z; qw[4 * i + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) qw[i] = 0u;
  }
}

// Power a with max |q| over the heads of this kv head < 2^a.
__device__ __forceinline__ int q_exponent(const uint32_t (&qw)[16]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(qw[i])), fabsf(bf16_hi(qw[i]))));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  int e = 0;
  if (amax > 0.f && amax < INFINITY) frexpf(amax, &e);
  return e;
}

// q * 2^-a as fp16 pairs in the order the key fragments pair channels:
//   pair p = 2*kb + bsel holds channels (32l + c, 32l + c + step) with
//   INT4: c = 8*(p/4) + p%2 + 4*((p/2)%2), step 2;  INT2: c = 16*(p/8) + p%8,
//   step 8;  FP8: c = 2p, step 1 (adjacent channels).
template <int FMT>
__device__ __forceinline__ int qpair_channel(int p) {
  if (FMT == 4) return 8 * (p >> 2) + (p & 1) + 4 * ((p >> 1) & 1);
  if (FMT == 2) return 16 * (p >> 3) + (p & 7);
  return 2 * p;
}
template <int FMT>
__device__ __forceinline__ void q_pairs(const uint32_t (&qw)[16], float sc, uint32_t (&qi)[16]) {
  constexpr int step = FMT == 4 ? 2 : (FMT == 2 ? 8 : 1);
  float qf[32];
#pragma unroll
  for (int i = 0; i < 16; ++i) { qf[2 * i] = bf16_lo(qw[i]) * sc; qf[2 * i + 1] = bf16_hi(qw[i]) * sc; }
#pragma unroll
  for (int p = 0; p < 16; ++p) {
    const int c = qpair_channel<FMT>(p);
    qi[p] = pack_h2(qf[c], qf[c + step]);
  }
}

// ---------------------------------------------------------------------------
// Quantized chunks
// ---------------------------------------------------------------------------

// Two e4m3 bytes -> an fp16 pair, for both halves of a word (the hardware
// converter; a 4-bit code in the low bits of an e4m3 byte is the exact
// value code * 2^-9, a normal fp16).
__device__ __forceinline__ void e4m3x4_to_h2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n .reg .b16 a, b;\n mov.b32 {a, b}, %2;\n cvt.rn.f16x2.e4m3x2 %0, a;\n cvt.rn.f16x2.e4m3x2 %1, b;\n}\n"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}

// One n8 tile of key codes (this thread's slice of row g) against the A
// fragments of q'' (two independent accumulation chains).  INT4 codes come
// out as code * 2^-9 (the caller scales the sum back).
template <int FMT>
__device__ __forceinline__ void qk_ntile(const uint8_t* krow, const uint32_t (&Aq)[8][4], float (&a0)[4],
                                         float (&a1)[4]) {
  const int l = threadIdx.x & 3;
  if constexpr (FMT == 4) {
    const uint4 kw = *reinterpret_cast<const uint4*>(krow + 16 * l);
    const uint32_t w[4] = {kw.x, kw.y, kw.z, kw.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      // word j = channels 8j .. 8j+7 (nibble k = channel 8j + k): the even
      // nibbles and the odd ones, one per byte, give the channel pairs
      // (8j, 8j+2), (8j+4, 8j+6) and (8j+1, 8j+3), (8j+5, 8j+7), i.e. the
      // pairs of (kb = 2j + r/2, bsel = r%2) for registers r = 0, 2, 1, 3
      uint32_t r0, r1, r2, r3;
      e4m3x4_to_h2x2(w[j] & 0x0F0F0F0Fu, r0, r2);
      e4m3x4_to_h2x2((w[j] >> 4) & 0x0F0F0F0Fu, r1, r3);
      if (j < 2) {
        mma_f16(a0, Aq[2 * j][0], Aq[2 * j][1], Aq[2 * j][2], Aq[2 * j][3], r0, r1);
        mma_f16(a0, Aq[2 * j + 1][0], Aq[2 * j + 1][1], Aq[2 * j + 1][2], Aq[2 * j + 1][3], r2, r3);
      } else {
        mma_f16(a1, Aq[2 * j][0], Aq[2 * j][1], Aq[2 * j][2], Aq[2 * j][3], r0, r1);
        mma_f16(a1, Aq[2 * j + 1][0], Aq[2 * j + 1][1], Aq[2 * j + 1][2], Aq[2 * j + 1][3], r2, r3);
      }
    }
  } else {
    const uint2 kw = *reinterpret_cast<const uint2*>(krow + 8 * l);
    const uint32_t w[2] = {kw.x, kw.y};
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      // register s = positions (s, s+8) of word j: kb = 4j + s/2, bsel = s%2
      uint32_t r[8];
      const uint32_t w10 = w[j] >> 10;
      r[0] = unmagic<1>(magic(w[j], 0x00030003u));
      r[1] = unmagic<4>(magic(w[j], 0x000C000Cu));
      r[2] = unmagic<16>(magic(w[j], 0x00300030u));
      r[3] = unmagic<64>(magic(w[j], 0x00C000C0u));
      r[4] = unmagic<256>(magic(w[j], 0x03000300u));
      r[5] = unmagic<1>(magic(w10, 0x00030003u));
      r[6] = unmagic<4>(magic(w10, 0x000C000Cu));
      r[7] = unmagic<16>(magic(w10, 0x00300030u));
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (j == 0) mma_f16(a0, Aq[k][0], Aq[k][1], Aq[k][2], Aq[k][3], r[2 * k], r[2 * k + 1]);
        else mma_f16(a1, Aq[4 + k][0], Aq[4 + k][1], Aq[4 + k][2], Aq[4 + k][3], r[2 * k], r[2 * k + 1]);
      }
    }
  }
}

// One n8 tile of e4m3 key codes (this thread's slice of row g) against the
// query pairs qi (rows 0-7: the heads' fp16 parts; two accumulation chains).
__device__ __forceinline__ void qk_ntile_fp8(const uint8_t* krow, const uint32_t (&qi)[16], float (&a0)[4],
                                             float (&a1)[4]) {
  const int l = threadIdx.x & 3;
  const uint4* kp = reinterpret_cast<const uint4*>(krow + 32 * l);
  const uint4 k0 = kp[0], k1 = kp[1];
  const uint32_t w[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
#pragma unroll
  for (int kb = 0; kb < 8; ++kb) {
    if (kb < 4) mma_f16(a0, qi[2 * kb], 0u, qi[2 * kb + 1], 0u, e4m3x2_to_h2(w[kb]), e4m3x2_to_h2(w[kb] >> 16));
    else mma_f16(a1, qi[2 * kb], 0u, qi[2 * kb + 1], 0u, e4m3x2_to_h2(w[kb]), e4m3x2_to_h2(w[kb] >> 16));
  }
}

// One n8 tile of INT8 key codes (this thread's slice of row g: channels
// [32l, 32l+32)) against the query pairs qi (adjacent channels, rows 0-7
// the heads' fp16 q; two accumulation chains).  A code byte placed under
// 0x64 is the half 1024 + code; one fused multiply-add removes the 1024.
__device__ __forceinline__ void qk_ntile_i8(const uint8_t* krow, const uint32_t (&qi)[16], float (&a0)[4],
                                            float (&a1)[4]) {
  const int l = threadIdx.x & 3;
  const uint4* kp = reinterpret_cast<const uint4*>(krow + 32 * l);
  const uint4 k0 = kp[0], k1 = kp[1];
  const uint32_t w[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
#pragma unroll
  for (int kb = 0; kb < 8; ++kb) {
    const uint32_t b0 = unmagic<1>(prmt(w[kb], 0x64646464u, 0x4140u));   // channels 4kb, 4kb+1
    const uint32_t b1 = unmagic<1>(prmt(w[kb], 0x64646464u, 0x4342u));   // channels 4kb+2, 4kb+3
    if (kb < 4) mma_f16(a0, qi[2 * kb], 0u, qi[2 * kb + 1], 0u, b0, b1);
    else mma_f16(a1, qi[2 * kb], 0u, qi[2 * kb + 1], 0u, b0, b1);
  }
}

// One tile of e4m3 value codes (16 tokens x 128 channels, token-major rows)
// -> the 16 output n-tiles; keep masks out the codes of tokens past the end.
__device__ __forceinline__ void pv_tile_fp8(const uint8_t* vt, const uint32_t (&Ap)[4], float (&O)[16][4],
                                            uint32_t keep) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k4 = 0; k4 < 4; ++k4) {
    const uint4 v = *reinterpret_cast<const uint4*>(vt + 512 * k4 + 16 * lane);
    const uint32_t w[4] = {v.x & keep, v.y & keep, v.z & keep, v.w & keep};
#pragma unroll
    for (int jj = 0; jj < 4; ++jj)
      mma_f16(O[4 * k4 + jj], Ap[0], Ap[1], Ap[2], Ap[3], e4m3x2_to_h2(w[jj]), e4m3x2_to_h2(w[jj] >> 16));
  }
}

// FP8-E4M3 decode, grid (splits, H_kv, B), kWarps warps per CTA: split s
// owns a contiguous range of the 32-token chunks of (sequence b, kv head)
// and each warp a sub-range, streamed through a ring of per-lane cp.async
// copies.  Scores: the query heads' fp16
// parts on the A rows, e4m3 key codes converted to fp16 (exact) as B, one
// static scale per kv head; values: P (fp16 hi/lo) times e4m3 value codes.
// The CTA merges its warps and writes one split partial per query head.
__global__ void __launch_bounds__(kWarps * 32, kFp8MinBlocks) decode_fp8_kernel(DecodeArgs A) {
  extern __shared__ __align__(128) uint8_t smem[];
  using St = Stage<8>;
  constexpr int NS = kFp8Stages;
  constexpr int RB = DecodeCfg<8>::kRB;
  const kvq_cache& c = A.c;
  const kvq_shape& s = c.shape;
  const int split = blockIdx.x, kv = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, l = lane & 3;
  const int gq = s.num_q_heads / s.num_kv_heads;
  const int S = A.num_splits;
  // the combine kernel may be scheduled as soon as every CTA here runs (it
  // waits for this grid before reading the partials)
  grid_dependents_launch();

  const int n = c.seq_len[b];
  const bool bad_state = n < 0 || n > s.capacity;
  const int n_tiles = bad_state ? 0 : (n + kTile - 1) / kTile;
  const int n_chunks = (n_tiles + 1) / 2;
  const int c_begin = (int)((long long)n_chunks * split / S);
  const int c_end = (int)((long long)n_chunks * (split + 1) / S);
  const int w_begin = c_begin + (c_end - c_begin) * warp / kWarps;
  const int w_end = c_begin + (c_end - c_begin) * (warp + 1) / kWarps;
  const int n_steps = w_end - w_begin;

  uint8_t* ring = smem + (size_t)warp * NS * St::kBytes;

  // base addresses of this warp's first chunk
  const uint8_t* kc0 = (const uint8_t*)c.k_codes + Addr::k_codes_unit(s, b, kv) + (size_t)w_begin * 2 * St::kTB;
  const uint8_t* vc0 = (const uint8_t*)c.v_codes + Addr::v_codes_tile(s, b, kv, 2 * w_begin);

  // chunk w_begin + i into stage i % NS: every lane copies its 16-byte
  // pieces (cp.async, one commit group per chunk)
  auto issue = [&](int i) {
    const int st = i % NS;
    const int t0 = 2 * (w_begin + i);
    uint8_t* dst = ring + (size_t)st * St::kBytes;
    const uint8_t* gk = kc0 + (size_t)i * 2 * St::kTB;
    const uint8_t* gv = vc0 + (size_t)i * 2 * St::kTB;
    if (t0 + 2 <= n_tiles) {
      warp_copy<2 * St::kTB>(dst + St::kK, gk, lane);
      warp_copy<2 * St::kTB>(dst + St::kV, gv, lane);
    } else {
      warp_copy<St::kTB>(dst + St::kK, gk, lane);
      warp_copy<St::kTB>(dst + St::kV, gv, lane);
    }
  };
  for (int i = 0; i < NS; ++i) {
    if (i < n_steps) issue(i);
    cp_async_commit();
  }

  // ---- query setup ----
  uint32_t qw[16];
  load_q_words(A, b, kv, gq, qw);
  const int a_exp = q_exponent(qw);
  uint32_t qi[16];
  q_pairs<8>(qw, ldexpf(1.f, -a_exp), qi);
  // q16-unit dot with exact e4m3 key values -> log2 logit
  const float s_code = A.scale_log2 * ldexpf(1.f, a_exp) * c.fp8_scale[kv];
  const float out_scale = c.fp8_scale[s.num_kv_heads + kv];

  SoftmaxState st{-INFINITY, 0.f, 0.f};
  float O[16][4];
#pragma unroll
  for (int j = 0; j < 16; ++j) O[j][0] = O[j][1] = O[j][2] = O[j][3] = 0.f;

  for (int i = 0; i < n_steps; ++i) {
    const int stg = i % NS;
    cp_async_wait<NS - 1>();   // this lane's pieces of chunk i have landed
    __syncwarp();              // ... and every lane's
    const int t0 = 2 * (w_begin + i);
    const int nt = min(2, n_tiles - t0);
    const uint8_t* sbuf = ring + (size_t)stg * St::kBytes;
    float S2[2][2][2];      // [tile][n8][elem]
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
      if (tt == 0 || nt == 2) {
        const uint8_t* kt = sbuf + St::kK + tt * St::kTB;
#pragma unroll
        for (int n8 = 0; n8 < 2; ++n8) {
          float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
          qk_ntile_fp8(kt + (8 * n8 + g) * RB, qi, a0, a1);
          S2[tt][n8][0] = ((a0[0] + a1[0]) + (a0[2] + a1[2])) * s_code;
          S2[tt][n8][1] = ((a0[1] + a1[1]) + (a0[3] + a1[3])) * s_code;
        }
      } else {
        S2[1][0][0] = S2[1][0][1] = S2[1][1][0] = S2[1][1][1] = -INFINITY;
      }
    }
    // Query rows past the heads of this kv head hold zeros and only fill
    // accumulator rows that are never written out, so they need no mask.
    // Tokens past the end exist only in the last tile.
    if ((t0 + 2) * kTile > n) {
#pragma unroll
      for (int tt = 0; tt < 2; ++tt)
#pragma unroll
        for (int n8 = 0; n8 < 2; ++n8)
#pragma unroll
          for (int e = 0; e < 2; ++e)
            if ((t0 + tt) * kTile + 8 * n8 + 2 * l + e >= n) S2[tt][n8][e] = -INFINITY;
    }
    const float tmax = fmaxf(fmaxf(fmaxf(S2[0][0][0], S2[0][0][1]), fmaxf(S2[0][1][0], S2[0][1][1])),
                             fmaxf(fmaxf(S2[1][0][0], S2[1][0][1]), fmaxf(S2[1][1][0], S2[1][1][1])));
    online_max_update(quad_max(tmax), st, O);
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
      if (tt == 0 || nt == 2) {
        float p[2][2];
#pragma unroll
        for (int n8 = 0; n8 < 2; ++n8)
#pragma unroll
          for (int e = 0; e < 2; ++e) p[n8][e] = ex2(S2[tt][n8][e] - st.m);
        st.l += (p[0][0] + p[0][1]) + (p[1][0] + p[1][1]);
        uint32_t Ap[4];
        split_h2(p[0][0], p[0][1], Ap[0], Ap[1]);
        split_h2(p[1][0], p[1][1], Ap[2], Ap[3]);
        uint32_t keep = 0xFFFFFFFFu;
        const int tok0 = (t0 + tt) * kTile;
        if (tok0 + kTile > n) {
          const int tb = tok0 + 2 * l;
          keep = (tb < n ? 0x000000FFu : 0u) | (tb + 1 < n ? 0x0000FF00u : 0u) |
                 (tb + 8 < n ? 0x00FF0000u : 0u) | (tb + 9 < n ? 0xFF000000u : 0u);
        }
        pv_tile_fp8(sbuf + St::kV + tt * St::kTB, Ap, O, keep);
      }
    }
    __syncwarp();              // every lane is done with stage i % NS
    if (i + NS < n_steps) issue(i + NS);
    cp_async_commit();
  }
  cp_async_wait<0>();
  if (lane == 0 && bad_state && warp == 0 && split == 0) atomicOr(c.err_word, KVQ_DEVERR_STATE);
  __syncthreads();   // every warp is done with its ring before smem becomes the merge buffer
  cta_merge_and_store(reinterpret_cast<float*>(smem), st, O, out_scale, gq, A, b, kv, split);
}

// ---------------------------------------------------------------------------
// INT formats: values on the tensor cores with channels on the M side
// ---------------------------------------------------------------------------
//
// Scores are computed as above (query heads' hi/lo parts on the 16 rows of
// an m16n8k16 MMA, exact key codes as the B operand).  The value sum is the
// transposed product O^T += V^T P^T: the A operand holds the value codes of
// 16 channels x 16 tokens (exact fp16 integers straight from the fragment-
// ordered tile), the B operand holds P'^T = (p * s_v) for 16 tokens x 8
// columns.  With at most 4 query heads per kv head the 8 columns carry the
// heads' fp16 hi parts (columns 0-3) and lo parts (columns 4-7) so one MMA
// carries both precision terms; with 5-8 heads the columns are heads and a
// second MMA adds the lo parts.  The softmax output of a thread (head g,
// tokens 2l, 2l+1, 2l+8, 2l+9) is exactly its B fragment, so nothing is
// transposed, and the 8 accumulator tiles (32 registers) cover all 128
// channels.  p * s_v stays in natural scale: p <= 1 and s_v <= 65504 keep it
// finite in fp16, and values too small for the fp16 normal range carry an
// absolute error below 2^-25.  The same holds for the key operand q * s_k.

#ifndef KVQ_DECODE_INT_STAGES4
#define KVQ_DECODE_INT_STAGES4 2
#endif
#ifndef KVQ_DECODE_INT_STAGES2
#define KVQ_DECODE_INT_STAGES2 3
#endif
#ifndef KVQ_DECODE_INT_MIN_BLOCKS
#define KVQ_DECODE_INT_MIN_BLOCKS 3      // CTAs per SM the streaming kernel's registers are cut for
#endif
#ifndef KVQ_DECODE_INT_WARPS
#define KVQ_DECODE_INT_WARPS 4           // streaming warps per CTA
#endif
constexpr int kIntWarps = KVQ_DECODE_INT_WARPS;

template <int FMT> struct IntCfg;
template <> struct IntCfg<4> { static constexpr int kStages = KVQ_DECODE_INT_STAGES4; };
template <> struct IntCfg<2> { static constexpr int kStages = KVQ_DECODE_INT_STAGES2; };
template <> struct IntCfg<16> { static constexpr int kStages = 2; };
template <> struct IntCfg<6> { static constexpr int kStages = KVQ_DECODE_INT_STAGES4; };

// Shared memory of the streaming kernel: the warps' rings, then their query
// stashes (16-byte aligned: stage sizes are multiples of 16 bytes).  INT8
// keeps its query fragments in registers (one per unit, not per group).
// Dense-and-sparse (SP) stages also hold the kept keys of up to two groups
// (2 x 128 words) and the kept values of the chunk's 32 tokens.
constexpr int kSpStageBytes = 2 * kHeadDim * 4 + 32 * 4;
template <int FMT, bool SP = false>
__host__ __device__ constexpr int int_stage_bytes() { return Stage<FMT>::kBytes + (SP ? kSpStageBytes : 0); }
template <int FMT, bool SP = false>
__host__ __device__ constexpr int int_qstash_offset() {
  return kIntWarps * IntCfg<FMT>::kStages * int_stage_bytes<FMT, SP>();
}
template <int FMT, bool SP = false>
__host__ __device__ constexpr int decode_int_smem_bytes() {
  // MIXED keeps the query pairs in both widths' channel orders
  return int_qstash_offset<FMT, SP>() + (FMT == 16 ? 0 : (FMT == 6 ? 2 : 1) * kIntWarps * kQStashBytes);
}
// SP: after the stashes, per warp the key corrections [32 tokens][8 heads]
// and the value corrections [gq heads][128] (fp32).
// per warp: 32 tokens x kMaxHeadsPerKv heads, rows padded to an odd stride
// so that a warp's scatter over tokens spreads over the banks
constexpr int kKcStride = kMaxHeadsPerKv + 1;
constexpr int kSpKcorrBytes = 32 * kKcStride * 4;
// value corrections per warp: gq rows of 128 channels, rows 132 floats apart
// (a multiple of 4 for the float4 rescale, and heads' rows in different
// banks for the same channel)
constexpr int kVcStride = kHeadDim + 4;
inline int decode_int_sp_extra_bytes(int gq) { return kIntWarps * (kSpKcorrBytes + gq * kVcStride * 4); }
static_assert(Stage<4>::kBytes % 16 == 0 && Stage<2>::kBytes % 16 == 0 && Stage<16>::kBytes % 16 == 0,
              "cp.async destinations are 16-byte aligned");

// Key A fragments of one group: rows 0-7 = hi(q * s_k), rows 8-15 =
// lo = q * s_k - hi (exact), for the 16 channel pairs of this lane (pair
// order, include/kvq.h); returns the zero-point dot sum_c q_c z_c of the
// lane's head (raw q units).
__device__ __forceinline__ float aprep_int(const uint8_t* km_smem, const uint4* qstash, uint32_t (&Aq)[8][4]) {
  const int lane = threadIdx.x & 31, l = lane & 3;
  const uint4* km = reinterpret_cast<const uint4*>(km_smem) + 4 * l;
  uint32_t qv[16], zv[16];
#pragma unroll
  for (int v4 = 0; v4 < 4; ++v4) {
    const uint4 sv = km[v4], q = qstash[32 * v4 + lane], z = km[16 + v4];
    const uint32_t sw[4] = {sv.x, sv.y, sv.z, sv.w};
    qv[4 * v4] = q.x; qv[4 * v4 + 1] = q.y; qv[4 * v4 + 2] = q.z; qv[4 * v4 + 3] = q.w;
    zv[4 * v4] = z.x; zv[4 * v4 + 1] = z.y; zv[4 * v4 + 2] = z.z; zv[4 * v4 + 3] = z.w;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int p = 4 * v4 + k;
      const uint32_t hi = hmul2(qv[p], sw[k]);
      Aq[p >> 1][2 * (p & 1)] = hi;
      Aq[p >> 1][2 * (p & 1) + 1] = hfms2(qv[p], sw[k], hi);
    }
  }
  // every B column holds the lane's zero points, so C[g][*] = sum_c q_g[c] z[c]
  float zc[4] = {0.f, 0.f, 0.f, 0.f}, zd[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int kb = 0; kb < 4; ++kb) {
    mma_f16(zc, qv[2 * kb], 0u, qv[2 * kb + 1], 0u, zv[2 * kb], zv[2 * kb + 1]);
    mma_f16(zd, qv[2 * kb + 8], 0u, qv[2 * kb + 9], 0u, zv[2 * kb + 8], zv[2 * kb + 9]);
  }
  return zc[0] + zd[0];
}

// One 16-token value tile into the transposed accumulators.  Tile word ww
// of this lane (lane = 4g + l) holds channels 16g + 2ww (a) and 16g + 2ww + 1
// (b) of tokens 2l, 2l+1, 2l+8, 2l+9 (INT4; INT2 words hold 4 channels),
// byte q = token q, so its codes split into bytes and converted by the e4m3
// converter give the A fragment of m-tile ww directly: row g = channel a,
// row g + 8 = channel b, k = tokens.  INT2/INT4 values come out as
// code * 2^-9 (the accumulators hold 2^-9 times their sums; INT8 does not).
template <int FMT, bool WIDE>
__device__ __forceinline__ void pv_tile_int(const uint8_t* vt, uint32_t b0, uint32_t b1, uint32_t c0, uint32_t c1,
                                            float (&O)[8][4]) {
  const int lane = threadIdx.x & 31;
  if constexpr (FMT == 16) {
    // INT8: word j of this lane holds channel 16g + j of tokens 2l, 2l+1,
    // 2l+8, 2l+9 (one byte each); m-tile mt takes words 2mt (row g) and
    // 2mt + 1 (row g + 8).  A byte placed under 0x64 is the half 1024 + code.
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 v = *reinterpret_cast<const uint4*>(vt + 512 * i + 16 * lane);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int mt = 2 * i + h;
        const uint32_t wa = w[2 * h], wb = w[2 * h + 1];
        const uint32_t a0 = unmagic<1>(prmt(wa, 0x64646464u, 0x4140u));
        const uint32_t a1 = unmagic<1>(prmt(wb, 0x64646464u, 0x4140u));
        const uint32_t a2 = unmagic<1>(prmt(wa, 0x64646464u, 0x4342u));
        const uint32_t a3 = unmagic<1>(prmt(wb, 0x64646464u, 0x4342u));
        mma_f16(O[mt], a0, a1, a2, a3, b0, b1);
        if (WIDE) mma_f16(O[mt], a0, a1, a2, a3, c0, c1);
      }
    }
  } else if constexpr (FMT == 4) {
    const uint4 v0 = *reinterpret_cast<const uint4*>(vt + 16 * lane);
    const uint4 v1 = *reinterpret_cast<const uint4*>(vt + 512 + 16 * lane);
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int ww = 0; ww < 8; ++ww) {
      // low nibbles: channel a of tokens (2l, 2l+1 | 2l+8, 2l+9); high: channel b
      uint32_t a0, a1, a2, a3;
      e4m3x4_to_h2x2(w[ww] & 0x0F0F0F0Fu, a0, a2);
      e4m3x4_to_h2x2((w[ww] >> 4) & 0x0F0F0F0Fu, a1, a3);
      mma_f16(O[ww], a0, a1, a2, a3, b0, b1);
      if (WIDE) mma_f16(O[ww], a0, a1, a2, a3, c0, c1);
    }
  } else {
    const uint4 v0 = *reinterpret_cast<const uint4*>(vt + 16 * lane);
    const uint32_t w[4] = {v0.x, v0.y, v0.z, v0.w};
#pragma unroll
    for (int ww = 0; ww < 4; ++ww) {
      // word ww: channels 16g + 4ww + j at 2-bit position j + 4 (byte = token)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // channels j = 2h (row g) and 2h + 1 (row g + 8)
        uint32_t a0, a1, a2, a3;
        e4m3x4_to_h2x2((w[ww] >> (4 * h)) & 0x03030303u, a0, a2);
        e4m3x4_to_h2x2((w[ww] >> (4 * h + 2)) & 0x03030303u, a1, a3);
        mma_f16(O[2 * ww + h], a0, a1, a2, a3, b0, b1);
        if (WIDE) mma_f16(O[2 * ww + h], a0, a1, a2, a3, c0, c1);
      }
    }
  }
}

// Packed fp32 pairs (one 64-bit register pair): Blackwell issues one
// add/mul/fma for both lanes, each rounded like the scalar operation.
typedef unsigned long long f2_t;
__device__ __forceinline__ f2_t f2(float lo, float hi) {
  f2_t d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}
__device__ __forceinline__ void f2_split(f2_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ f2_t f2_add(f2_t a, f2_t b) {
  f2_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f2_t f2_mul(f2_t a, f2_t b) {
  f2_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f2_t f2_fma(f2_t a, f2_t b, f2_t c) {
  f2_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

struct IntSoftmax {
  float m;   // running max (log2 units) of head g
  float l;   // this lane's share of sum p
  float z;   // this lane's share of sum p * z_v
};

// Raise the running max of head g to cover tmax (already reduced over the
// quad); rescale l, z and the accumulator columns of heads hc0, hc0 + 1.
__device__ __forceinline__ void int_max_update(float tmax, IntSoftmax& st, float (&O)[8][4], int hc0,
                                               float* vcorr = nullptr, int gq = 0) {
  const float mnew = fmaxf(st.m, tmax);
  const bool grow = mnew > st.m;
  if (__any_sync(0xffffffffu, grow)) {
    const float a = grow ? (st.m == -INFINITY ? 0.f : ex2(st.m - mnew)) : 1.f;
    st.l *= a;
    st.z *= a;
    st.m = mnew;
    if (vcorr) {
      // dense-and-sparse value corrections share the accumulators' scale:
      // lane (g, l) rescales channels [32l, 32l+32) of head g
      const int lane = threadIdx.x & 31, g = lane >> 2, l = lane & 3;
      __syncwarp();
      if (g < gq) {
        float4* v4 = reinterpret_cast<float4*>(vcorr + g * kVcStride + 32 * l);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float4 x = v4[j];
          x.x *= a; x.y *= a; x.z *= a; x.w *= a;
          v4[j] = x;
        }
      }
      __syncwarp();
    }
    const float a0 = __shfl_sync(0xffffffffu, a, 4 * hc0), a1 = __shfl_sync(0xffffffffu, a, 4 * (hc0 + 1));
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      O[mt][0] *= a0; O[mt][1] *= a1; O[mt][2] *= a0; O[mt][3] *= a1;
    }
  }
}

// B fragments of P'^T from this lane's (hi, lo) pairs: narrow layouts take
// the hi pair (rows g < 4) or the lo pair of head g - 4 from lane ^ 16.
template <bool WIDE>
__device__ __forceinline__ void pv_operands(uint32_t hi0, uint32_t lo0, uint32_t hi1, uint32_t lo1, uint32_t& b0,
                                            uint32_t& b1, uint32_t& c0, uint32_t& c1) {
  if (WIDE) {
    b0 = hi0; b1 = hi1; c0 = lo0; c1 = lo1;
  } else {
    const uint32_t x0 = __shfl_xor_sync(0xffffffffu, lo0, 16), x1 = __shfl_xor_sync(0xffffffffu, lo1, 16);
    const bool hi_row = (threadIdx.x & 31) < 16;
    b0 = hi_row ? hi0 : x0;
    b1 = hi_row ? hi1 : x1;
    c0 = c1 = 0u;
  }
}

// 16 window tokens (bf16 ring rows) into the same state.
template <bool WIDE>
__device__ __forceinline__ void window_chunk_int(const kvq_cache& c, int b, int kv, int nq, int r, int ci,
                                                 const uint32_t (&qw)[16], int gq, float scale_log2, int hc0,
                                                 IntSoftmax& st, float (&O)[8][4]) {
  const kvq_shape& s = c.shape;
  const int lane = threadIdx.x & 31, g = lane >> 2, l = lane & 3;
  const int Ws = window_slots(s);
  const uint16_t* kr = (const uint16_t*)c.k_res + Addr::ring_row(s, b, kv, 0);
  const uint16_t* vr = (const uint16_t*)c.v_res + Addr::ring_row(s, b, kv, 0);
  float S[2][2];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    const int tk = ci * kTile + 8 * nt + g;
    uint32_t w[16];
    if (tk < r) {
      const uint4* kp = reinterpret_cast<const uint4*>(kr + (size_t)((nq + tk) % Ws) * kHeadDim + 32 * l);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 v = kp[i];
        w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) w[i] = 0u;
    }
    float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kb = 0; kb < 4; ++kb) {
      mma_bf16(a0, qw[2 * kb], 0u, qw[2 * kb + 1], 0u, w[2 * kb], w[2 * kb + 1]);
      mma_bf16(a1, qw[2 * kb + 8], 0u, qw[2 * kb + 9], 0u, w[2 * kb + 8], w[2 * kb + 9]);
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int tok = ci * kTile + 8 * nt + 2 * l + e;
      S[nt][e] = (g < gq && tok < r) ? (a0[e] + a1[e]) * scale_log2 : -INFINITY;
    }
  }
  int_max_update(quad_max(fmaxf(fmaxf(S[0][0], S[0][1]), fmaxf(S[1][0], S[1][1]))), st, O, hc0);
  const float mref = st.m == -INFINITY ? 0.f : st.m;
  float p[2][2];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) p[nt][e] = ex2(S[nt][e] - mref);
  st.l += (p[0][0] + p[0][1]) + (p[1][0] + p[1][1]);
  // the accumulators hold 2^-9 times the value sums (pv_tile_int)
  uint32_t hi0, lo0, hi1, lo1, b0, b1, c0, c1;
  split_bf2(p[0][0] * 0x1p-9f, p[0][1] * 0x1p-9f, hi0, lo0);
  split_bf2(p[1][0] * 0x1p-9f, p[1][1] * 0x1p-9f, hi1, lo1);
  pv_operands<WIDE>(hi0, lo0, hi1, lo1, b0, b1, c0, c1);
  // values: tokens 2l, 2l+1, 2l+8, 2l+9 of the chunk, channels [16g, 16g+16)
  uint32_t vw[4][8];
  const int tl[4] = {2 * l, 2 * l + 1, 2 * l + 8, 2 * l + 9};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int tk = ci * kTile + tl[q];
    if (tk < r) {
      const uint4* vp = reinterpret_cast<const uint4*>(vr + (size_t)((nq + tk) % Ws) * kHeadDim + 16 * g);
      const uint4 a = vp[0], bb = vp[1];
      vw[q][0] = a.x; vw[q][1] = a.y; vw[q][2] = a.z; vw[q][3] = a.w;
      vw[q][4] = bb.x; vw[q][5] = bb.y; vw[q][6] = bb.z; vw[q][7] = bb.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) vw[q][i] = 0u;
    }
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    const uint32_t a0 = prmt(vw[0][mt], vw[1][mt], 0x5410u), a1 = prmt(vw[0][mt], vw[1][mt], 0x7632u);
    const uint32_t a2 = prmt(vw[2][mt], vw[3][mt], 0x5410u), a3 = prmt(vw[2][mt], vw[3][mt], 0x7632u);
    mma_bf16(O[mt], a0, a1, a2, a3, b0, b1);
    if (WIDE) mma_bf16(O[mt], a0, a1, a2, a3, c0, c1);
  }
}

// ---------------------------------------------------------------------------
// Work split of the quantized part: a flat list of 32-token chunks
// ---------------------------------------------------------------------------
//
// Units u = b * H_kv + kv in order; unit u holds seq_chunks(b) chunks of its
// quantized tokens.  With Pw warps in the grid, warp p streams the chunks
// [lo(p), lo(p+1)) of the flat list, lo(p) = floor(p * C / Pw), so every warp
// gets the same number of chunks whatever the mix of sequence lengths.  A
// warp's range meets one or more units; for each it writes one partial
// (m, l, o) to slot p + u.  That map is one to one (a later warp never meets
// an earlier unit), so the slots of unit u are p_first(u) + u ..
// p_last(u) + u, with p_first/p_last the owners of its first and last chunk
// (skipping warps whose range is empty, which write nothing).

// A (seq_len, n_quant) pair no prefill, append or flush can produce.
__device__ __forceinline__ bool state_bad(const kvq_shape& s, int n, int nq) {
  if (is_int8(s.format)) return n < 0 || nq != n || n > s.capacity;
  return n < 0 || nq < 0 || nq > n || nq > s.capacity || (nq & (s.group - 1)) || n - nq > window_slots(s);
}
// 16-token tiles of a quantized part of nq tokens (INT8: the last one may
// be partial; INT2/4: nq is a whole number of groups).
__device__ __forceinline__ int quant_tiles(const kvq_shape& s, int nq) {
  return is_int8(s.format) ? (nq + kTile - 1) / kTile : nq / kTile;
}

// Chunks of sequence b's quantized part (0 for a state that fails the checks).
__device__ __forceinline__ int seq_chunks(const kvq_cache& c, int b) {
  const kvq_shape& s = c.shape;
  const int n = c.seq_len[b], nq = c.n_quant[b];
  return state_bad(s, n, nq) ? 0 : (quant_tiles(s, nq) + 1) / 2;
}

// Total chunks C of the batch (warp-uniform result).
__device__ __forceinline__ int total_chunks(const kvq_cache& c) {
  const int lane = threadIdx.x & 31;
  int sum = 0;
  for (int b0 = 0; b0 < c.shape.batch; b0 += 32) {
    int v = b0 + lane < c.shape.batch ? seq_chunks(c, b0 + lane) : 0;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    sum += v;
  }
  return sum * c.shape.num_kv_heads;
}

// The sequence b whose units hold flat chunk x, and the chunks before it
// (all warp-uniform).  b = batch when x is past the end.
__device__ __forceinline__ void find_sequence(const kvq_cache& c, int x, int& b_out, int& before) {
  const int lane = threadIdx.x & 31;
  const int H = c.shape.num_kv_heads;
  int base = 0;
  for (int b0 = 0; b0 < c.shape.batch; b0 += 32) {
    const int v = b0 + lane < c.shape.batch ? seq_chunks(c, b0 + lane) * H : 0;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    const int tot = __shfl_sync(0xffffffffu, incl, 31);
    const unsigned hit = __ballot_sync(0xffffffffu, base + incl > x);
    if (hit) {
      const int ln = __ffs(hit) - 1;
      b_out = b0 + ln;
      before = base + __shfl_sync(0xffffffffu, incl - v, ln);
      return;
    }
    base += tot;
  }
  b_out = c.shape.batch;
  before = base;
}

// floor(n / d) for 0 <= n < 2^63, 0 < d < 2^31: a 32-bit division whenever
// n fits (the common case), the 64-bit one otherwise.
__device__ __forceinline__ int floor_div(unsigned long long n, int d) {
  return (n >> 32) == 0 ? (int)((unsigned)n / (unsigned)d) : (int)(n / (unsigned)d);
}
__device__ __forceinline__ int chunk_lo(int p, int C, int Pw) {
  return floor_div((unsigned long long)(unsigned)p * (unsigned)C, Pw);
}
// The warp whose range holds flat chunk x: lo(p) <= x < lo(p + 1).
__device__ __forceinline__ int chunk_owner(int x, int C, int Pw) {
  return floor_div((unsigned long long)(unsigned)(x + 1) * (unsigned)Pw - 1ull, C);
}

// Position of a warp in the flat chunk list.
struct ChunkCursor {
  int b, kv, c;     // sequence, kv head, chunk within the unit
  int nc;           // chunks per unit of sequence b
  int nt;           // 16-token tiles of sequence b's quantized part
  int first;        // first chunk of this warp's segment in the current unit
  __device__ __forceinline__ void start(const kvq_cache& cc, int x) {
    int before;
    find_sequence(cc, x, b, before);
    nc = b < cc.shape.batch ? seq_chunks(cc, b) : 0;
    nt = b < cc.shape.batch ? quant_tiles(cc.shape, cc.n_quant[b]) : 0;
    const int local = x - before;
    kv = nc ? local / nc : 0;
    c = nc ? local - kv * nc : 0;
    first = c;
  }
  __device__ __forceinline__ void advance(const kvq_cache& cc) {
    if (++c < nc) return;
    c = 0;
    first = 0;
    if (++kv < cc.shape.num_kv_heads) return;
    kv = 0;
    do {
      ++b;
      nc = b < cc.shape.batch ? seq_chunks(cc, b) : 1;
    } while (nc == 0);
    nt = b < cc.shape.batch ? quant_tiles(cc.shape, cc.n_quant[b]) : 0;
  }
};

// Partial slots for the INT decode: (num_splits * kIntWarps + units) slots of
// gq heads x (m, l) and gq x 128 floats.
__host__ __device__ inline size_t int_slots(const kvq_shape& s, int num_splits) {
  return (size_t)num_splits * kIntWarps + (size_t)s.batch * s.num_kv_heads;
}
// Floats of the (m, l) area, rounded up so that the o area that follows it
// starts on a 256-byte boundary (it is read with 16-byte vector loads).
__host__ __device__ inline size_t int_ml_floats(const kvq_shape& s, int num_splits) {
  const size_t n = int_slots(s, num_splits) * (s.num_q_heads / s.num_kv_heads) * 2;
  return (n + 63) / 64 * 64;
}

struct IntArgs {
  kvq_cache c;
  const uint16_t* q;   // [B][H_q][128] bf16
  float* ws_o;         // [slots][gq][128]
  float* ws_ml;        // [slots][gq][2]
  float* out;          // [B][H_q][128]
  float* lse;          // [B][H_q] natural-log softmax denominators, or null
  float scale_log2;
  int num_splits;
};

// bf16 query of head (kv * gq + g), channels [32l, 32l+32), as 16 words of
// adjacent channel pairs (zeros for rows past the kv head's gq heads).
__device__ __forceinline__ void load_q_words_int(const uint16_t* q, const kvq_shape& s, int b, int kv, int gq,
                                                 uint32_t (&qw)[16]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, l = lane & 3;
  if (g < gq) {
    const uint4* qr = reinterpret_cast<const uint4*>(q + ((size_t)b * s.num_q_heads + kv * gq + g) * kHeadDim + 32 * l);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 v = qr[i];
      qw[4 * i] = v.x; qw[4 * i + 1] = v.y; qw[4 * i + 2] = v.z; qw[4 * i + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) qw[i] = 0u;
  }
}


// Grid (num_splits), kIntWarps warps; each warp streams its slice of the flat
// chunk list through a private ring of shared-memory stages filled by
// per-lane cp.async copies.
template <int FMT, bool PAGED, bool WIDE, bool ROPE, bool SP>
__global__ void __launch_bounds__(kIntWarps * 32, KVQ_DECODE_INT_MIN_BLOCKS) decode_int_kernel(IntArgs A) {
  extern __shared__ __align__(128) uint8_t smem[];
  using St = Stage<FMT>;
  constexpr int NS = IntCfg<FMT>::kStages;
  const kvq_cache& c = A.c;
  const kvq_shape& s = c.shape;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, l = lane & 3;
  const int gq = s.num_q_heads / s.num_kv_heads;
  const int hc0 = WIDE ? 2 * l : (2 * l) & 3;       // heads of this lane's accumulator columns
  constexpr bool I8 = FMT == 16;                   // INT8 per token: per-token key scales, no window
  constexpr bool MX = FMT == 6;                    // MIXED: each group at 4 or 2 bits
  const int T = I8 ? 1 : s.group / kTile;          // tiles per key group: 1, 2, 4 or 8
  // ROPE (keys stored before RoPE): the 64 pair frequencies in double, and
  // per warp the fp32 scale and zero of the current key group in channel order
  // and the rotation by 8 positions of every pair, (cos 8 theta_i, sin 8 theta_i)
  // (tables padded so that the four lane groups l = 0..3, which read pairs
  // [16l, 16l + 16) and channels [32l, 32l + 32), hit different banks:
  // pair p at p + p / 16, channel c at c + 4 (c / 32))
  __shared__ double rope_freq[ROPE ? kHeadDim / 2 + 4 : 1];
  __shared__ float2 rope_step8[ROPE ? kHeadDim / 2 + 4 : 1];
  __shared__ __align__(16) float rope_sz[ROPE ? kIntWarps * 2 * (kHeadDim + 16) : 4];
  if constexpr (ROPE) {
    if (threadIdx.x < kHeadDim / 2) {
      const double f = pow((double)s.rope_theta, -2.0 * (double)threadIdx.x / (double)kHeadDim);
      rope_freq[threadIdx.x + threadIdx.x / 16] = f;
      double sn, cs;
      sincos(8.0 * f, &sn, &cs);
      rope_step8[threadIdx.x + threadIdx.x / 16] = make_float2((float)cs, (float)sn);
    }
    __syncthreads();
  }
  // the combine kernel may start its window work as soon as every CTA here runs
  grid_dependents_launch();

  const int Pw = A.num_splits * kIntWarps;
  const int p = blockIdx.x * kIntWarps + warp;
  const int C = total_chunks(c);
  const int x0 = C ? chunk_lo(p, C, Pw) : 0, x1 = C ? chunk_lo(p + 1, C, Pw) : 0;
  const int n_steps = x1 - x0;
  if (n_steps <= 0) return;

  constexpr int SB = int_stage_bytes<FMT, SP>();     // bytes per ring stage
  uint8_t* ring = smem + (size_t)warp * NS * SB;
  uint4* qstash = reinterpret_cast<uint4*>(smem + int_qstash_offset<FMT, SP>() + warp * kQStashBytes);
  uint4* qstash2 = reinterpret_cast<uint4*>(smem + int_qstash_offset<FMT, SP>() + (kIntWarps + warp) * kQStashBytes);
  // dense-and-sparse corrections of this warp (after the stash)
  float* kcorr = reinterpret_cast<float*>(smem + decode_int_smem_bytes<FMT, SP>() + warp * kSpKcorrBytes);
  float* vcorr = reinterpret_cast<float*>(smem + decode_int_smem_bytes<FMT, SP>() + kIntWarps * kSpKcorrBytes) +
                 warp * gq * kVcStride;

  ChunkCursor ic, cc;     // issue and consume positions
  ic.start(c, x0);
  cc = ic;

  // per-unit strides of the contiguous layout, computed once (the group
  // count per unit is a run-time division)
  const size_t unit_tiles = (size_t)(s.capacity / kTile);
  const size_t unit_groups = I8 ? 0 : (size_t)(s.capacity / s.group);
  // Chunk at ic into stage i % NS: every lane copies its 16-byte pieces of
  // the key tiles, value tiles, value (scale, zero) and key group tables
  // (cp.async, one group per chunk; a chunk with a bad page id copies
  // nothing and is skipped when consumed).
  const int lgT = __ffs(T) - 1;        // T is a power of two
  auto issue = [&](int i) {
    const int st = i % NS;
    const int t0 = 2 * ic.c;
    const int nt = min(2, ic.nt - t0);
    uint8_t* dst = ring + (size_t)st * SB;
    if (PAGED) {
      const int32_t* ptab = c.page_table + (size_t)ic.b * s.max_pages_per_seq;
      int pg[2] = {0, 0};
      bool ok = true;
      for (int k = 0; k < nt; ++k) {
        pg[k] = ptab[t0 + k];
        ok = ok && pg[k] >= 0 && pg[k] < s.num_pages;
      }
      if (!ok) return;
      for (int k = 0; k < nt; ++k) {
        warp_copy<St::kTB>(dst + St::kK + k * St::kTB, (const uint8_t*)c.k_codes + Addr::pg_k_codes(s, pg[k], ic.kv), lane);
        warp_copy<St::kTB>(dst + St::kV + k * St::kTB, (const uint8_t*)c.v_codes + Addr::pg_v_codes(s, pg[k], ic.kv), lane);
        warp_copy<64>(dst + St::kVm + k * 64, (const uint8_t*)((const __half*)c.v_meta + Addr::pg_v_meta(s, pg[k], ic.kv)), lane);
        warp_copy<512>(dst + St::kKm + k * 512, (const uint8_t*)((const __half*)c.k_meta + Addr::pg_k_meta(s, pg[k], ic.kv)), lane);
      }
      return;
    }
    if constexpr (I8) {
      // key and value tiles, then the per-token (scale, zero) of both
      const size_t tile = ((size_t)ic.b * s.num_kv_heads + ic.kv) * unit_tiles + t0;
      const uint8_t* gk = (const uint8_t*)c.k_codes + tile * St::kTB;
      const uint8_t* gv = (const uint8_t*)c.v_codes + tile * St::kTB;
      const uint8_t* gvm = (const uint8_t*)c.v_meta + tile * 64;
      const uint8_t* gkm = (const uint8_t*)c.k_meta + tile * 64;
      if (nt == 2) {
        warp_copy<2 * St::kTB>(dst + St::kK, gk, lane);
        warp_copy<2 * St::kTB>(dst + St::kV, gv, lane);
        warp_copy<128>(dst + St::kVm, gvm, lane);
        warp_copy<128>(dst + St::kKm, gkm, lane);
      } else {
        warp_copy<St::kTB>(dst + St::kK, gk, lane);
        warp_copy<St::kTB>(dst + St::kV, gv, lane);
        warp_copy<64>(dst + St::kVm, gvm, lane);
        warp_copy<64>(dst + St::kKm, gkm, lane);
      }
      return;
    }
    if constexpr (MX) {
      // a group stored at 2 bits: its key rows packed at 32 bytes from the
      // group slot's start, each value tile in the first half of its slot;
      // copied into the 2-bit stage layout
      const int gi = t0 >> lgT;
      if (c.group_bits[(size_t)ic.b * unit_groups + gi] != 4) {
        using S2 = Stage<2>;
        const bool km2 = ic.c == ic.first || (t0 & (T - 1)) == 0;
        const size_t unit = (size_t)ic.b * s.num_kv_heads + ic.kv;
        const size_t tile = unit * unit_tiles + t0;
        const uint8_t* gk = (const uint8_t*)c.k_codes + unit * unit_tiles * St::kTB + (size_t)gi * s.group * 64 +
                            (size_t)(t0 * kTile - gi * s.group) * 32;
        const uint8_t* gv = (const uint8_t*)c.v_codes + tile * St::kTB;
        const uint8_t* gvm = (const uint8_t*)c.v_meta + tile * 64;
        const uint8_t* gkm = (const uint8_t*)c.k_meta + ((unit * unit_groups + gi) << 9);
        if (nt == 2) {
          warp_copy<2 * S2::kTB>(dst + S2::kK, gk, lane);
          warp_copy<S2::kTB>(dst + S2::kV, gv, lane);
          warp_copy<S2::kTB>(dst + S2::kV + S2::kTB, gv + St::kTB, lane);
          warp_copy<128>(dst + S2::kVm, gvm, lane);
        } else {
          warp_copy<S2::kTB>(dst + S2::kK, gk, lane);
          warp_copy<S2::kTB>(dst + S2::kV, gv, lane);
          warp_copy<64>(dst + S2::kVm, gvm, lane);
        }
        if (km2) warp_copy<512>(dst + S2::kKm, gkm, lane);
        return;
      }
    }
    const bool km = (T == 1) || ic.c == ic.first || (t0 & (T - 1)) == 0;
    const size_t unit = (size_t)ic.b * s.num_kv_heads + ic.kv;
    const size_t tile = unit * unit_tiles + t0;                  // 16-token tiles (codes: kTB bytes each)
    const uint8_t* gk = (const uint8_t*)c.k_codes + tile * St::kTB;
    const uint8_t* gv = (const uint8_t*)c.v_codes + tile * St::kTB;
    const uint8_t* gvm = (const uint8_t*)c.v_meta + tile * 64;
    const uint8_t* gkm = (const uint8_t*)c.k_meta + ((unit * unit_groups + (t0 >> lgT)) << 9);
    if constexpr (SP) {
      // kept keys of the chunk's group(s), copied with the group table; kept
      // values of its tokens
      const uint8_t* gks = (const uint8_t*)(c.k_sparse + ((unit * unit_groups + (t0 >> lgT)) << 7));
      const uint8_t* gvs = (const uint8_t*)(c.v_sparse + tile * kTile);
      if (km) {
        if (T == 1 && nt == 2) warp_copy<1024>(dst + St::kBytes, gks, lane);
        else warp_copy<512>(dst + St::kBytes, gks, lane);
      }
      if (nt == 2) warp_copy<128>(dst + St::kBytes + 1024, gvs, lane);
      else warp_copy<64>(dst + St::kBytes + 1024, gvs, lane);
    }
    if (nt == 2) {
      warp_copy<2 * St::kTB>(dst + St::kK, gk, lane);
      warp_copy<2 * St::kTB>(dst + St::kV, gv, lane);
      warp_copy<128>(dst + St::kVm, gvm, lane);
      if (km) {
        if (T == 1) warp_copy<1024>(dst + St::kKm, gkm, lane);
        else warp_copy<512>(dst + St::kKm, gkm, lane);
      }
    } else {
      warp_copy<St::kTB>(dst + St::kK, gk, lane);
      warp_copy<St::kTB>(dst + St::kV, gv, lane);
      warp_copy<64>(dst + St::kVm, gvm, lane);
      if (km) warp_copy<512>(dst + St::kKm, gkm, lane);
    }
  };

  for (int i = 0; i < NS; ++i) {
    if (i < n_steps) {
      issue(i);
      ic.advance(c);
    }
    cp_async_commit();
  }

  IntSoftmax st{-INFINITY, 0.f, 0.f};
  float O[8][4];
  uint32_t Aq[8][4];
  float zs = 0.f, s_mul = 0.f;
  uint32_t qi8[16];             // INT8: the unit's query pairs (adjacent channels; unused otherwise)
  float zq = 0.f;               // INT8: scale_log2 * sum_c q[g][c] (the key zero points' factor)
  int ulen = 0;                 // INT8: tokens of the unit (the last tile may be partial)
  int ub = 0, ukv = 0;          // the unit being accumulated
  bool page_bad = false;

  // Write the partial of the unit just finished (slot p + u) and clear the state.
  auto finish_unit = [&]() {
    const float lsum = quad_sum(st.l), zsum = quad_sum(st.z);
    if (!WIDE) {
#pragma unroll
      for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int k = 0; k < 4; ++k) O[mt][k] += __shfl_xor_sync(0xffffffffu, O[mt][k], 2);
    }
    if constexpr (!I8) {
      // INT2/INT4 value codes (and the window's share) were summed at 2^-9
#pragma unroll
      for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int k = 0; k < 4; ++k) O[mt][k] *= 512.f;
    }
    const float z0 = __shfl_sync(0xffffffffu, zsum, 4 * hc0), z1 = __shfl_sync(0xffffffffu, zsum, 4 * (hc0 + 1));
    const size_t slot = (size_t)p + (size_t)ub * s.num_kv_heads + ukv;
    if constexpr (SP) __syncwarp();      // every lane's value corrections are in
    if ((WIDE || l < 2) && hc0 < gq) {
      float* o0 = A.ws_o + (slot * gq + hc0) * kHeadDim + 16 * g;
      // dense-and-sparse: the kept values' share (channels 16g + 2mt, +1)
      auto vc = [&](int hd, int ch) { return SP ? vcorr[hd * kVcStride + ch] : 0.f; };
#pragma unroll
      for (int mt = 0; mt < 8; ++mt)
        *reinterpret_cast<float2*>(o0 + 2 * mt) = make_float2(O[mt][0] + z0 + vc(hc0, 16 * g + 2 * mt),
                                                               O[mt][2] + z0 + vc(hc0, 16 * g + 2 * mt + 1));
      if (hc0 + 1 < gq) {
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
          *reinterpret_cast<float2*>(o0 + kHeadDim + 2 * mt) =
              make_float2(O[mt][1] + z1 + vc(hc0 + 1, 16 * g + 2 * mt), O[mt][3] + z1 + vc(hc0 + 1, 16 * g + 2 * mt + 1));
      }
    }
    if (l == 0 && g < gq) *reinterpret_cast<float2*>(A.ws_ml + (slot * gq + g) * 2) = make_float2(st.m, lsum);
    st = IntSoftmax{-INFINITY, 0.f, 0.f};
  };
  auto start_unit = [&](int x_here) {
#pragma unroll
    for (int j = 0; j < 8; ++j) O[j][0] = O[j][1] = O[j][2] = O[j][3] = 0.f;
    if constexpr (SP) {
      __syncwarp();
      for (int i = lane; i < gq * kVcStride; i += 32) vcorr[i] = 0.f;
      for (int i = lane; i < 32 * kKcStride; i += 32) kcorr[i] = 0.f;
      __syncwarp();
    }
    ub = cc.b;
    ukv = cc.kv;
    uint32_t qw[16];
    load_q_words_int(A.q, s, ub, ukv, gq, qw);
    if constexpr (ROPE) {
      // keys are rotated in the chunk loop; the combine kernel takes the
      // windows of these units (rotated there)
      const int a_exp = q_exponent(qw);
      q_pairs<8>(qw, ldexpf(1.f, -a_exp), qi8);
      s_mul = A.scale_log2 * ldexpf(1.f, a_exp);
      return;
    }
    if constexpr (I8) {
      ulen = c.seq_len[ub];
      const int a_exp = q_exponent(qw);
      q_pairs<8>(qw, ldexpf(1.f, -a_exp), qi8);
      float qs = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) qs += bf16_lo(qw[i]) + bf16_hi(qw[i]);
      zq = A.scale_log2 * quad_sum(qs);
      s_mul = A.scale_log2 * ldexpf(1.f, a_exp);
      return;
    }
    {
      // the unit's bf16 window tiles: tile j goes to the owner of the unit's
      // chunk j * nc / tiles, spreading the tiles over the warps that share
      // the unit (every tile has exactly one owner); done while this warp's
      // first copies are in flight
      const int nq_u = cc.nt * kTile;
      const int r = c.seq_len[ub] - nq_u;
      const int x_unit = x_here - cc.c;
      const int wt = (r + kTile - 1) / kTile;
      // this warp owns chunks [x0, x1): tile j is its own iff
      // a <= floor(j nc / wt) < b, i.e. j in [ceil(a wt / nc), ceil(b wt / nc))
      const long long a = max(x0 - x_unit, 0), b = min(x1 - x_unit, cc.nc);
      const int j0 = (int)((a * wt + cc.nc - 1) / cc.nc), j1 = (int)((b * wt + cc.nc - 1) / cc.nc);
      for (int j = j0; j < j1; ++j)
        window_chunk_int<WIDE>(c, ub, ukv, nq_u, r, j, qw, gq, A.scale_log2, hc0, st, O);
    }
    const int a_exp = q_exponent(qw);
    uint32_t qi[16];
    q_pairs<MX ? 4 : FMT>(qw, ldexpf(1.f, -a_exp), qi);
    __syncwarp();
#pragma unroll
    for (int v4 = 0; v4 < 4; ++v4)
      qstash[32 * v4 + lane] = make_uint4(qi[4 * v4], qi[4 * v4 + 1], qi[4 * v4 + 2], qi[4 * v4 + 3]);
    if constexpr (MX) {
      q_pairs<2>(qw, ldexpf(1.f, -a_exp), qi);
#pragma unroll
      for (int v4 = 0; v4 < 4; ++v4)
        qstash2[32 * v4 + lane] = make_uint4(qi[4 * v4], qi[4 * v4 + 1], qi[4 * v4 + 2], qi[4 * v4 + 3]);
    }
    __syncwarp();
    s_mul = A.scale_log2 * ldexpf(1.f, a_exp);   // q16-unit dot -> log2 logit
  };

  for (int i = 0; i < n_steps; ++i) {
    if (i == 0 || cc.c == 0) {
      if (i > 0) finish_unit();
      start_unit(x0 + i);
    }
    const int stg = i % NS;
    cp_async_wait<NS - 1>();   // this lane's pieces of chunk i have landed
    __syncwarp();              // ... and every lane's
    const int t0 = 2 * cc.c;
    const int nt = min(2, cc.nt - t0);
    const uint8_t* sbuf = ring + (size_t)stg * SB;
    if (PAGED) {
      const int32_t* ptab = c.page_table + (size_t)cc.b * s.max_pages_per_seq;
      bool ok = true;
      for (int k = 0; k < nt; ++k) {
        const int pg = ptab[t0 + k];
        ok = ok && pg >= 0 && pg < s.num_pages;
      }
      if (!ok) {
        page_bad = true;
        goto next_chunk;
      }
    }
    {
      // The chunk's work for code width F (the format's own, or for a MIXED
      // cache the width its group was stored at); SF is that width's stage
      // layout and qs the query pairs in its channel order.
      auto chunk_body = [&](auto ftag) {
        constexpr int F = decltype(ftag)::value;
        using SF = Stage<F>;
        constexpr int RBF = DecodeCfg<F>::kRB;
        const uint4* qs = (MX && F == 2) ? qstash2 : qstash;
        (void)qs;                          // unused by the INT8 and pre-RoPE key paths
        const bool fresh = cc.c == cc.first || (t0 & (T - 1)) == 0;
        // scores of tile tt (the key fragments of its group must be in Aq)
        auto qk_tile = [&](int tt, float (&S)[2][2]) {
          const uint8_t* kt = sbuf + SF::kK + tt * SF::kTB;
  #pragma unroll
          for (int n8 = 0; n8 < 2; ++n8) {
            float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
            qk_ntile<F>(kt + (8 * n8 + g) * RBF, Aq, a0, a1);
            const f2_t x = f2_add(f2(a0[0], a0[1]), f2(a1[0], a1[1]));
            f2_t y = f2_add(f2(a0[2], a0[3]), f2(a1[2], a1[3]));
            y = f2_add(x, y);
            if constexpr (F == 4) y = f2_mul(y, f2(512.f, 512.f));   // INT4 codes were read as code * 2^-9
            f2_split(f2_fma(y, f2(s_mul, s_mul), f2(zs, zs)), S[n8][0], S[n8][1]);
          }
        };
        // probabilities, value zero points and the value product of tile tt
        // (INT8: tokens of the tile at or past `lim` are masked out)
        auto pv_softmax_tile = [&](int tt, const float (&S)[2][2], int lim = kTile) {
          float pr[2][2];
  #pragma unroll
          for (int n8 = 0; n8 < 2; ++n8) {
            float d0, d1;
            f2_split(f2_add(f2(S[n8][0], S[n8][1]), f2(-st.m, -st.m)), d0, d1);
            pr[n8][0] = ex2(d0);
            pr[n8][1] = ex2(d1);
          }
          st.l += (pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]);
          // (scale, zero) of tokens 2l, 2l+1 and 2l+8, 2l+9 of the tile
          const uint8_t* vm = sbuf + SF::kVm + tt * 64;
          const uint2 m0 = *reinterpret_cast<const uint2*>(vm + 8 * l);
          const uint2 m1 = *reinterpret_cast<const uint2*>(vm + 32 + 8 * l);
          // each word is one token's (scale, zero) pair: convert the halves directly
          f2_t s01 = f2(__low2float(u32_as_h2(m0.x)), __low2float(u32_as_h2(m0.y)));
          f2_t z01 = f2(__high2float(u32_as_h2(m0.x)), __high2float(u32_as_h2(m0.y)));
          f2_t s89 = f2(__low2float(u32_as_h2(m1.x)), __low2float(u32_as_h2(m1.y)));
          f2_t z89 = f2(__high2float(u32_as_h2(m1.x)), __high2float(u32_as_h2(m1.y)));
          if (F == 16 && lim < kTile) {
            // the scale and zero of tokens past the end are not data: zero them
            // so that p = 0 leaves nothing of them in the sums
            const float zero = 0.f;
            float a, b;
            f2_split(s01, a, b); s01 = f2(2 * l < lim ? a : zero, 2 * l + 1 < lim ? b : zero);
            f2_split(z01, a, b); z01 = f2(2 * l < lim ? a : zero, 2 * l + 1 < lim ? b : zero);
            f2_split(s89, a, b); s89 = f2(2 * l + 8 < lim ? a : zero, 2 * l + 9 < lim ? b : zero);
            f2_split(z89, a, b); z89 = f2(2 * l + 8 < lim ? a : zero, 2 * l + 9 < lim ? b : zero);
          }
          if constexpr (SP) {
            // kept values: o[g][c_t] += p (x_t - z_t) (their dense code is 0)
            const uint32_t* vsp = reinterpret_cast<const uint32_t*>(sbuf + St::kBytes + 1024) + tt * kTile;
            float zz[4];
            f2_split(z01, zz[0], zz[1]);
            f2_split(z89, zz[2], zz[3]);
            const int tk[4] = {2 * l, 2 * l + 1, 2 * l + 8, 2 * l + 9};
            const float pp[4] = {pr[0][0], pr[0][1], pr[1][0], pr[1][1]};
            if (g < gq) {
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const uint32_t e = vsp[tk[q]];
                atomicAdd(vcorr + g * kVcStride + (e >> 16), pp[q] * (bf16_lo(e) - zz[q]));
              }
            }
          }
          const f2_t p01 = f2(pr[0][0], pr[0][1]), p89 = f2(pr[1][0], pr[1][1]);
          float za, zb;
          f2_split(f2_fma(p01, z01, f2_mul(p89, z89)), za, zb);
          st.z += za + zb;
          float x0, x1, x8, x9;
          f2_split(f2_mul(p01, s01), x0, x1);
          f2_split(f2_mul(p89, s89), x8, x9);
          uint32_t hi0, lo0, hi1, lo1, b0, b1, c0, c1;
          split_h2(x0, x1, hi0, lo0);
          split_h2(x8, x9, hi1, lo1);
          pv_operands<WIDE>(hi0, lo0, hi1, lo1, b0, b1, c0, c1);
          pv_tile_int<F, WIDE>(sbuf + SF::kV + tt * SF::kTB, b0, b1, c0, c1, O);
        };
          // dense-and-sparse: the kept keys' share of the scores,
        // q[h][c] (k_c - z_c) for the token each channel kept (its dense
        // code is 0, i.e. z_c), gathered per (token, head) in shared memory
        auto k_sparse_fix = [&](float (&S0)[2][2], float (&S1)[2][2]) {
          if constexpr (SP) {
            const uint32_t* ksp = reinterpret_cast<const uint32_t*>(sbuf + St::kBytes);
            const __half* kmh = reinterpret_cast<const __half*>(sbuf + SF::kKm);
            const int ngroups = T == 1 ? nt : 1;     // G = 16: a group per tile; G = 32: the chunk
            const uint16_t* qrow = A.q + ((size_t)ub * s.num_q_heads + (size_t)ukv * gq) * kHeadDim;
            __syncwarp();
            for (int gi = 0; gi < ngroups; ++gi) {
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const int ch = 32 * k + lane;
                const uint32_t e = ksp[gi * kHeadDim + ch];
                const int tok = (int)(e >> 16) + kTile * gi;
                const float d = bf16_lo(e) - __half2float(kmh[gi * 2 * kHeadDim + kHeadDim + kmeta_pos<F>(ch)]);
                for (int hh = 0; hh < gq; ++hh)
                  atomicAdd(kcorr + tok * kKcStride + hh,
                            __uint_as_float((uint32_t)qrow[hh * kHeadDim + ch] << 16) * d);
              }
            }
            __syncwarp();
            if (g < gq) {
#pragma unroll
              for (int n8 = 0; n8 < 2; ++n8)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                  float* c0 = kcorr + (8 * n8 + 2 * l + e) * kKcStride + g;
                  float* c1 = kcorr + (kTile + 8 * n8 + 2 * l + e) * kKcStride + g;
                  S0[n8][e] += *c0 * A.scale_log2;
                  S1[n8][e] += *c1 * A.scale_log2;
                  *c0 = 0.f;
                  *c1 = 0.f;
                }
            }
            __syncwarp();
          }
        };
      auto chunk_max = [&](const float (&S0)[2][2], const float (&S1)[2][2]) {
          return fmaxf(fmaxf(fmaxf(S0[0][0], S0[0][1]), fmaxf(S0[1][0], S0[1][1])),
                       fmaxf(fmaxf(S1[0][0], S1[0][1]), fmaxf(S1[1][0], S1[1][1])));
        };
        float S0[2][2], S1[2][2];
        if constexpr (ROPE) {
          // Keys stored before RoPE: dequantize k^ = code * s + z in fp32,
          // turn each channel pair by its token's angle, split into fp16
          // hi + lo, and multiply with the exact fp16 query pairs (adjacent
          // channels, rows 0-7 = heads).  Lane l holds channels [32l, 32l+32)
          // = pairs [16l, 16l+16) of its token row g of every n8 tile.
          float* sz = rope_sz + warp * 2 * (kHeadDim + 16);
          if (fresh) {
            // the group's scale/zero rows (pair order) -> channel order, fp32
            const __half* km = reinterpret_cast<const __half*>(sbuf + SF::kKm);
            __syncwarp();
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int ch = 32 * k + lane;
              sz[ch + 4 * k] = __half2float(km[kmeta_pos<F>(ch)]);
              sz[kHeadDim + 16 + ch + 4 * k] = __half2float(km[kHeadDim + kmeta_pos<F>(ch)]);
            }
            __syncwarp();
          }
          float acc[2][2][4];
          uint32_t kw[2][2][4];
#pragma unroll
          for (int tt = 0; tt < 2; ++tt)
#pragma unroll
            for (int n8 = 0; n8 < 2; ++n8) {
              acc[tt][n8][0] = acc[tt][n8][1] = acc[tt][n8][2] = acc[tt][n8][3] = 0.f;
              const uint8_t* row = sbuf + SF::kK + tt * SF::kTB + (8 * n8 + g) * RBF;
              if (tt < nt) {
                if constexpr (F == 4) {
                  const uint4 v = *reinterpret_cast<const uint4*>(row + 16 * l);
                  kw[tt][n8][0] = v.x; kw[tt][n8][1] = v.y; kw[tt][n8][2] = v.z; kw[tt][n8][3] = v.w;
                } else {
                  const uint2 v = *reinterpret_cast<const uint2*>(row + 8 * l);
                  kw[tt][n8][0] = v.x; kw[tt][n8][1] = v.y; kw[tt][n8][2] = 0u; kw[tt][n8][3] = 0u;
                }
              } else {
                kw[tt][n8][0] = kw[tt][n8][1] = kw[tt][n8][2] = kw[tt][n8][3] = 0u;
              }
            }
#pragma unroll
          for (int kb = 0; kb < 8; ++kb) {
            // channels 32l + 4kb .. +3 (pairs 16l + 2kb, 16l + 2kb + 1)
            const float4 s4 = *reinterpret_cast<const float4*>(sz + 36 * l + 4 * kb);
            const float4 z4 = *reinterpret_cast<const float4*>(sz + kHeadDim + 16 + 36 * l + 4 * kb);
            // the lane's tokens are t0 * 16 + g + 8m, m = 2tt + n8: the angles of
            // m = 0 in double, each next one by a turn of 8 theta_i (fp32, ~1e-7
            // relative error per turn)
            float c0, s0, c1, s1;
            rope_cos_sin(t0 * kTile + g, rope_freq[17 * l + 2 * kb], c0, s0);
            rope_cos_sin(t0 * kTile + g, rope_freq[17 * l + 2 * kb + 1], c1, s1);
            const float2 st0 = rope_step8[17 * l + 2 * kb], st1 = rope_step8[17 * l + 2 * kb + 1];
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
              if (tt >= nt) continue;
#pragma unroll
              for (int n8 = 0; n8 < 2; ++n8) {
                if (tt + n8 > 0) {
                  const float cn0 = c0 * st0.x - s0 * st0.y, cn1 = c1 * st1.x - s1 * st1.y;
                  s0 = s0 * st0.x + c0 * st0.y;
                  s1 = s1 * st1.x + c1 * st1.y;
                  c0 = cn0;
                  c1 = cn1;
                }
                uint32_t cq;                   // the 4 codes, one per byte
                if constexpr (F == 4) {
                  const uint32_t w = kw[tt][n8][kb >> 1] >> (16 * (kb & 1));   // bytes 2kb, 2kb+1
                  cq = prmt(w & 0x0F0Fu, (w >> 4) & 0x0F0Fu, 0x5140u);          // c0, c1, c2, c3
                } else {
                  const uint32_t w = (kw[tt][n8][kb >> 2] >> (8 * (kb & 3))) & 0xFFu;   // byte kb
                  cq = (w & 3u) | ((w >> 2) & 3u) << 8 | ((w >> 4) & 3u) << 16 | ((w >> 6) & 3u) << 24;
                }
                // code byte i under the exponent of 2^23 is the float 2^23 + code:
                // one PRMT and one exact subtraction instead of an int conversion
                const float k0 = fmaf(__uint_as_float(prmt(cq, 0x4Bu, 0x4550u)) - 8388608.f, s4.x, z4.x);
                const float k1 = fmaf(__uint_as_float(prmt(cq, 0x4Bu, 0x4551u)) - 8388608.f, s4.y, z4.y);
                const float k2 = fmaf(__uint_as_float(prmt(cq, 0x4Bu, 0x4552u)) - 8388608.f, s4.z, z4.z);
                const float k3 = fmaf(__uint_as_float(prmt(cq, 0x4Bu, 0x4553u)) - 8388608.f, s4.w, z4.w);
                const float r0 = k0 * c0 - k1 * s0, r1 = k0 * s0 + k1 * c0;
                const float r2 = k2 * c1 - k3 * s1, r3 = k2 * s1 + k3 * c1;
                uint32_t h01, l01, h23, l23;
                split_h2(r0, r1, h01, l01);
                split_h2(r2, r3, h23, l23);
                mma_f16(acc[tt][n8], qi8[2 * kb], 0u, qi8[2 * kb + 1], 0u, h01, h23);
                mma_f16(acc[tt][n8], qi8[2 * kb], 0u, qi8[2 * kb + 1], 0u, l01, l23);
              }
            }
          }
#pragma unroll
          for (int n8 = 0; n8 < 2; ++n8) {
            S0[n8][0] = acc[0][n8][0] * s_mul;
            S0[n8][1] = acc[0][n8][1] * s_mul;
            S1[n8][0] = nt == 2 ? acc[1][n8][0] * s_mul : -INFINITY;
            S1[n8][1] = nt == 2 ? acc[1][n8][1] * s_mul : -INFINITY;
          }
          int_max_update(quad_max(chunk_max(S0, S1)), st, O, hc0);
          pv_softmax_tile(0, S0);
          if (nt == 2) pv_softmax_tile(1, S1);
        } else if constexpr (F == 16) {
          // scores: s_k[t] * (q . codes_t) + z_k[t] * sum_c q[c], log2 units;
          // tokens past the unit's length are masked
          auto qk_tile_i8 = [&](int tt, float (&S)[2][2]) {
            const uint8_t* kt = sbuf + SF::kK + tt * SF::kTB;
            const uint8_t* kmt = sbuf + SF::kKm + tt * 64;
            const int tok0 = (t0 + tt) * kTile;
  #pragma unroll
            for (int n8 = 0; n8 < 2; ++n8) {
              float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
              qk_ntile_i8(kt + (8 * n8 + g) * RBF, qi8, a0, a1);
              const uint2 m = *reinterpret_cast<const uint2*>(kmt + 32 * n8 + 8 * l);   // tokens 8n8 + 2l, +1
              const float d0 = (a0[0] + a1[0]) + (a0[2] + a1[2]), d1 = (a0[1] + a1[1]) + (a0[3] + a1[3]);
              float x0, x1;
              f2_split(f2_fma(f2_mul(f2(d0, d1), f2(s_mul, s_mul)),
                              f2(__low2float(u32_as_h2(m.x)), __low2float(u32_as_h2(m.y))),
                              f2_mul(f2(zq, zq), f2(__high2float(u32_as_h2(m.x)), __high2float(u32_as_h2(m.y))))),
                       x0, x1);
              const int tk = tok0 + 8 * n8 + 2 * l;
              S[n8][0] = tk < ulen ? x0 : -INFINITY;
              S[n8][1] = tk + 1 < ulen ? x1 : -INFINITY;
            }
          };
          qk_tile_i8(0, S0);
          if (nt == 2) qk_tile_i8(1, S1);
          else S1[0][0] = S1[0][1] = S1[1][0] = S1[1][1] = -INFINITY;
          int_max_update(quad_max(chunk_max(S0, S1)), st, O, hc0);
          pv_softmax_tile(0, S0, ulen - t0 * kTile);
          if (nt == 2) pv_softmax_tile(1, S1, ulen - (t0 + 1) * kTile);
        } else if (T > 1 && nt == 2) {
          // the common case: both tiles in one key group, straight-line code
          if (fresh) zs = aprep_int(sbuf + SF::kKm, qs, Aq) * s_mul;
          qk_tile(0, S0);
          qk_tile(1, S1);
          k_sparse_fix(S0, S1);
          int_max_update(quad_max(chunk_max(S0, S1)), st, O, hc0, SP ? vcorr : nullptr, gq);
          pv_softmax_tile(0, S0);
          pv_softmax_tile(1, S1);
        } else {
          // a group per tile (G = 16) or a unit's last, single tile
          if (T == 1) zs = aprep_int(sbuf + SF::kKm, qs, Aq) * s_mul;
          else if (fresh) zs = aprep_int(sbuf + SF::kKm, qs, Aq) * s_mul;
          qk_tile(0, S0);
          if (nt == 2) {
            zs = aprep_int(sbuf + SF::kKm + 512, qs, Aq) * s_mul;   // T == 1 here
            qk_tile(1, S1);
          } else {
            S1[0][0] = S1[0][1] = S1[1][0] = S1[1][1] = -INFINITY;
          }
          k_sparse_fix(S0, S1);
          int_max_update(quad_max(chunk_max(S0, S1)), st, O, hc0, SP ? vcorr : nullptr, gq);
          pv_softmax_tile(0, S0);
          if (nt == 2) pv_softmax_tile(1, S1);
        }
      };
      if constexpr (MX) {
        if (c.group_bits[(size_t)cc.b * unit_groups + (t0 >> lgT)] == 4) chunk_body(std::integral_constant<int, 4>{});
        else chunk_body(std::integral_constant<int, 2>{});
      } else {
        chunk_body(std::integral_constant<int, FMT>{});
      }
    }
  next_chunk:
    __syncwarp();              // every lane is done with stage i % NS
    if (i + NS < n_steps) {
      issue(i + NS);
      ic.advance(c);
    }
    cp_async_commit();
    if (i + 1 < n_steps) cc.advance(c);
  }
  cp_async_wait<0>();
  finish_unit();
  if (page_bad && lane == 0) atomicOr(c.err_word, KVQ_DEVERR_PAGE_RANGE);
}

// Grid (H_q, B), 256 threads: the bf16 window's share of head h of sequence
// b (fp32, read from the ring), then -- once the streaming kernel is done --
// the merge of the window with every partial slot of the unit.  Both halves
// keep many loads in flight: one thread per window token for the scores,
// 16 token lanes x 8-channel vectors for the values, and the slots split
// over 8 lanes x 32 channel quads.
constexpr int kCombineThreads = 128;

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int w = 1; w < kCombineThreads / 32; ++w) r = fmaxf(r, red[w]);
  return r;
}
__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int w = 1; w < kCombineThreads / 32; ++w) r += red[w];
  return r;
}

// Chunks before sequence b (times H_kv), sequence b's chunks, and the total,
// from one pass over the batch (warp-uniform results).
__device__ __forceinline__ void unit_offsets(const kvq_cache& c, int b, int& before, int& nc_b, int& total) {
  const int lane = threadIdx.x & 31;
  const int H = c.shape.num_kv_heads;
  int run = 0, pre = 0, mine = 0;
  for (int b0 = 0; b0 < c.shape.batch; b0 += 32) {
    const int bb = b0 + lane;
    const int v = bb < c.shape.batch ? seq_chunks(c, bb) : 0;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    if (bb == b) {
      pre = run + incl - v;
      mine = v;
    }
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
  const int src = b & 31;
  before = __shfl_sync(0xffffffffu, pre, src) * H;
  nc_b = __shfl_sync(0xffffffffu, mine, src);
  total = run * H;
}

// Grid (H_q, B, CS), 128 threads: channels [CW z, CW z + CW) of head h of
// sequence b, CW = 128 / CS (CS = 1 ... 32: more CTAs when the batch has few
// heads).  The window of a unit with no quantized chunk is computed here
// (the streaming warps take every other unit's window); then, once the
// streaming kernel is done, the unit's partial slots are merged in one pass:
// 128 / (CW / 4) slot lanes x CW / 4 channel quads, each slot lane merging
// its slots online, then a shuffle merge over the slot lanes of each quad
// (two stages when a quad has more than 32 lanes).
__global__ void __launch_bounds__(kCombineThreads, 16) decode_int_combine_kernel(IntArgs A) {
  constexpr int NT = kCombineThreads, TL = NT / 16;   // threads; window token lanes
  const int CW = kHeadDim / gridDim.z;               // channels per CTA: 128 ... 4
  const int NQ4 = CW / 4, SL = NT / NQ4;             // channel quads (32 ... 1), slot lanes (4 ... 128)
  struct WinSmem {
    float qs[kHeadDim];
    float ps[NT];
    float wsum[TL][kHeadDim];
    double freq[kHeadDim / 2];    // RoPE pair frequencies (keys stored before RoPE)
  };
  struct MergeSmem {
    float4 acc[NT];
    float lsh[NT];
    float msh[NT];
    float4 po[4];
    float pm[4], pl[4];
  };
  __shared__ __align__(16) union {
    WinSmem w;
    MergeSmem m;
  } sm;
  __shared__ float red[NT / 32];
  __shared__ __align__(16) float wout[kHeadDim];
  const kvq_cache& c = A.c;
  const kvq_shape& s = c.shape;
  const int h = blockIdx.x, b = blockIdx.y, z = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = s.num_q_heads / s.num_kv_heads, kv = h / gq, hh = h - kv * gq;
  const int Ws = window_slots(s);
  const int n = c.seq_len[b], nq = c.n_quant[b];
  const bool bad = state_bad(s, n, nq);
  if (bad && tid == 0 && h == 0 && z == 0) atomicOr(c.err_word, KVQ_DEVERR_STATE);

  // ---- the unit's chunk range (every warp computes the same) ----
  int before, nc, C;
  unit_offsets(c, b, before, nc, C);
  if (bad) nc = 0;

  // ---- window: only for units with no quantized chunk (with keys stored
  // before RoPE, for every unit: the keys are rotated here) ----
  const bool rope = s.rope_theta > 0.f;
  const int r = (bad || (nc && !rope)) ? 0 : n - nq;
  float Mw = -INFINITY, Lw = 0.f;
  if (r > 0) {
    const int vc = tid & 15, tl = tid >> 4;      // channels [8vc, 8vc+8), token lane
    float ow[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const uint16_t* qrow = A.q + ((size_t)b * s.num_q_heads + h) * kHeadDim;
    for (int i = tid; i < kHeadDim; i += NT) sm.w.qs[i] = __uint_as_float((uint32_t)qrow[i] << 16);
    if (rope && tid < kHeadDim / 2)
      sm.w.freq[tid] = pow((double)s.rope_theta, -2.0 * (double)tid / (double)kHeadDim);
    __syncthreads();
    const uint16_t* kr = (const uint16_t*)c.k_res + Addr::ring_row(s, b, kv, 0);
    const uint16_t* vr = (const uint16_t*)c.v_res + Addr::ring_row(s, b, kv, 0);
    for (int t0 = 0; t0 < r; t0 += NT) {
      float sc = -INFINITY;
      if (t0 + tid < r) {
        const uint4* kp = reinterpret_cast<const uint4*>(kr + (size_t)((nq + t0 + tid) % Ws) * kHeadDim);
        float d = 0.f;
        if (rope) {
          // key t at position nq + t0 + tid: each channel pair (2i, 2i+1) turned
          // by its angle before the dot product
          const int pos = nq + t0 + tid;
#pragma unroll 1
          for (int i0 = 0; i0 < 16; ++i0) {
            const uint4 kv = kp[i0];
            const uint32_t kw4[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int pr = 4 * i0 + j;           // pair: channels 2pr, 2pr + 1
              float cs, sn;
              rope_cos_sin(pos, sm.w.freq[pr], cs, sn);
              const float k0 = bf16_lo(kw4[j]), k1 = bf16_hi(kw4[j]);
              d = fmaf(sm.w.qs[2 * pr], k0 * cs - k1 * sn, d);
              d = fmaf(sm.w.qs[2 * pr + 1], k0 * sn + k1 * cs, d);
            }
          }
        } else {
#pragma unroll 1
          for (int i0 = 0; i0 < 16; i0 += 4) {     // 4 row vectors in flight: few registers
            uint4 kw[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) kw[i] = kp[i0 + i];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float4 qa = *reinterpret_cast<const float4*>(sm.w.qs + 8 * (i0 + i));
              const float4 qb = *reinterpret_cast<const float4*>(sm.w.qs + 8 * (i0 + i) + 4);
              d = fmaf(qa.x, bf16_lo(kw[i].x), d); d = fmaf(qa.y, bf16_hi(kw[i].x), d);
              d = fmaf(qa.z, bf16_lo(kw[i].y), d); d = fmaf(qa.w, bf16_hi(kw[i].y), d);
              d = fmaf(qb.x, bf16_lo(kw[i].z), d); d = fmaf(qb.y, bf16_hi(kw[i].z), d);
              d = fmaf(qb.z, bf16_lo(kw[i].w), d); d = fmaf(qb.w, bf16_hi(kw[i].w), d);
            }
          }
        }
        sc = d * A.scale_log2;
      }
      const float Mb = block_max(sc, red);
      const float Mn = fmaxf(Mw, Mb);
      const float alpha = Mw == -INFINITY ? 0.f : ex2(Mw - Mn);
      const float pr = sc == -INFINITY ? 0.f : ex2(sc - Mn);
      sm.w.ps[tid] = pr;
      Lw = Lw * alpha + block_sum(pr, red);     // block_sum's barriers also publish ps
#pragma unroll
      for (int k = 0; k < 8; ++k) ow[k] *= alpha;
      Mw = Mn;
      const int tn = min(NT, r - t0);
#pragma unroll 2
      for (int t = tl; t < tn; t += TL) {
        const uint4 v = *reinterpret_cast<const uint4*>(vr + (size_t)((nq + t0 + t) % Ws) * kHeadDim + 8 * vc);
        const float pt = sm.w.ps[t];
        ow[0] = fmaf(pt, bf16_lo(v.x), ow[0]); ow[1] = fmaf(pt, bf16_hi(v.x), ow[1]);
        ow[2] = fmaf(pt, bf16_lo(v.y), ow[2]); ow[3] = fmaf(pt, bf16_hi(v.y), ow[3]);
        ow[4] = fmaf(pt, bf16_lo(v.z), ow[4]); ow[5] = fmaf(pt, bf16_hi(v.z), ow[5]);
        ow[6] = fmaf(pt, bf16_lo(v.w), ow[6]); ow[7] = fmaf(pt, bf16_hi(v.w), ow[7]);
      }
      __syncthreads();   // ps is rewritten by the next block of tokens
    }
    // sum the token lanes of this CTA's channels
#pragma unroll
    for (int k = 0; k < 8; ++k) sm.w.wsum[tl][8 * vc + k] = ow[k];
    __syncthreads();
    for (int i = tid; i < CW; i += NT) {
      float o = 0.f;
#pragma unroll
      for (int t = 0; t < TL; ++t) o += sm.w.wsum[t][CW * z + i];
      wout[i] = o;
    }
    __syncthreads();   // the merge below reuses the window's shared memory
  }

  // ---- slots of the unit: their range is known before the streaming
  // kernel ends, their contents after ----
  const int x_first = before + kv * nc;
  const int Pw = A.num_splits * kIntWarps;
  const int u = b * s.num_kv_heads + kv;
  const int p_first = nc ? chunk_owner(x_first, C, Pw) : 0, p_last = nc ? chunk_owner(x_first + nc - 1, C, Pw) : -1;
  // with fewer chunks than warps some warps own no chunk and wrote no slot
  const bool sparse = C < Pw;
  auto live = [&](int pp) { return !sparse || chunk_lo(pp, C, Pw) < chunk_lo(pp + 1, C, Pw); };
  grid_dependency_wait();
  const int cq = tid % NQ4, sl = tid / NQ4;      // channels CW z + [4cq, 4cq+4), slot lane
  float Ml = -INFINITY, Lt = 0.f;
  float4 o4 = make_float4(0.f, 0.f, 0.f, 0.f);
  // this lane's slots p_first + sl + k SL, two at a time: both slots' loads
  // are issued together (no branch between them), then merged online in
  // slot order
  for (int pp0 = p_first + sl; pp0 <= p_last; pp0 += 2 * SL) {
    float2 mlv[2];
    float4 ov[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int pp = pp0 + k * SL;
      const bool ok = pp <= p_last && live(pp);
      const size_t slot = (size_t)(ok ? pp + u : u) * gq + hh;
      mlv[k] = ok ? *reinterpret_cast<const float2*>(A.ws_ml + slot * 2) : make_float2(-INFINITY, 0.f);
      ov[k] = ok ? *reinterpret_cast<const float4*>(A.ws_o + slot * kHeadDim + CW * z + 4 * cq)
                 : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float2 ml = mlv[k];
      const float4 o = ov[k];
      if (ml.x == -INFINITY) continue;
      const float mn = fmaxf(Ml, ml.x);
      const float fo = Ml == -INFINITY ? 0.f : ex2(Ml - mn), fn = ex2(ml.x - mn);
      Lt = fmaf(fn, ml.y, Lt * fo);
      o4.x = fmaf(fn, o.x, o4.x * fo); o4.y = fmaf(fn, o.y, o4.y * fo);
      o4.z = fmaf(fn, o.z, o4.z * fo); o4.w = fmaf(fn, o.w, o4.w * fo);
      Ml = mn;
    }
  }
  sm.m.acc[tid] = o4;
  sm.m.lsh[tid] = Lt;
  sm.m.msh[tid] = Ml;
  __syncthreads();

  // lanes of quad mq: thread sl * NQ4 + mq for sl < SL.  Up to 32 lanes
  // per quad merge in one warp (32 / SL quads per warp); 64 or 128 lanes
  // merge per warp first, then across the warps of the quad.
  const int span = SL <= 32 ? SL : 32;
  const int mq = SL <= 32 ? warp * (32 / SL) + lane / SL : warp / (SL / 32);
  const int ln = SL <= 32 ? lane % SL : (warp % (SL / 32)) * 32 + lane;
  float Ms, L, o[4];
  {
    const int t = ln * NQ4 + mq;
    const float m = sm.m.msh[t];
    Ms = m;
    for (int off = span / 2; off > 0; off >>= 1) Ms = fmaxf(Ms, __shfl_xor_sync(0xffffffffu, Ms, off));
    const float f = m == -INFINITY ? 0.f : ex2(m - Ms);
    const float4 a4 = sm.m.acc[t];
    L = f * sm.m.lsh[t];
    o[0] = f * a4.x; o[1] = f * a4.y; o[2] = f * a4.z; o[3] = f * a4.w;
    for (int off = span / 2; off > 0; off >>= 1) {
      L += __shfl_xor_sync(0xffffffffu, L, off);
#pragma unroll
      for (int k = 0; k < 4; ++k) o[k] += __shfl_xor_sync(0xffffffffu, o[k], off);
    }
  }
  bool writer = ln == 0;
  if (SL > 32) {
    // one partial per warp, then thread mq merges the SL / 32 warps of its quad
    if (lane == 0) {
      sm.m.pm[warp] = Ms;
      sm.m.pl[warp] = L;
      sm.m.po[warp] = make_float4(o[0], o[1], o[2], o[3]);
    }
    __syncthreads();
    writer = tid < NQ4;
    if (writer) {
      const int G = SL / 32, w0 = tid * G;
      Ms = -INFINITY;
      for (int k = 0; k < G; ++k) Ms = fmaxf(Ms, sm.m.pm[w0 + k]);
      L = 0.f;
      o[0] = o[1] = o[2] = o[3] = 0.f;
      for (int k = 0; k < G; ++k) {
        const float f = sm.m.pm[w0 + k] == -INFINITY ? 0.f : ex2(sm.m.pm[w0 + k] - Ms);
        const float4 p4 = sm.m.po[w0 + k];
        L = fmaf(f, sm.m.pl[w0 + k], L);
        o[0] = fmaf(f, p4.x, o[0]); o[1] = fmaf(f, p4.y, o[1]); o[2] = fmaf(f, p4.z, o[2]); o[3] = fmaf(f, p4.w, o[3]);
      }
    }
  }
  if (writer) {
    const int q = SL > 32 ? tid : mq;
    const float M = fmaxf(Mw, Ms);
    float4 res = make_float4(0.f, 0.f, 0.f, 0.f);
    float lse2 = -INFINITY;     // log2 of sum_t 2^(score_t), scores in log2 units
    if (M != -INFINITY) {
      const float fs = Ms == -INFINITY ? 0.f : ex2(Ms - M), fw = Mw == -INFINITY ? 0.f : ex2(Mw - M);
      const float Lm = L * fs + Lw * fw;
      if (Lm > 0.f) {
        lse2 = M + log2f(Lm);
        const float inv = 1.f / Lm;
        float4 w4 = make_float4(0.f, 0.f, 0.f, 0.f);
        if (Mw != -INFINITY) w4 = *reinterpret_cast<const float4*>(&wout[4 * q]);
        res.x = (o[0] * fs + w4.x * fw) * inv;
        res.y = (o[1] * fs + w4.y * fw) * inv;
        res.z = (o[2] * fs + w4.z * fw) * inv;
        res.w = (o[3] * fs + w4.w * fw) * inv;
      }
    }
    *reinterpret_cast<float4*>(A.out + ((size_t)b * s.num_q_heads + h) * kHeadDim + CW * z + 4 * q) = res;
    if (A.lse && z == 0 && q == 0) A.lse[(size_t)b * s.num_q_heads + h] = lse2 * kLn2;
  }
}

// Grid (B * H_q); block 128: out[b][h][c] = merge over splits; lse (if
// not null) gets the row's natural-log softmax denominator.
__global__ void decode_combine_kernel(const float* __restrict__ ws_o, const float* __restrict__ ws_ml, float* out,
                                      float* lse, int num_splits) {
  const size_t bh = blockIdx.x;
  const int ch = threadIdx.x;
  grid_dependency_wait();    // launched as a dependent of the FP8 streaming kernel
  const float* ml = ws_ml + bh * num_splits * 2;
  float M = -INFINITY;
  for (int i = 0; i < num_splits; ++i) M = fmaxf(M, ml[2 * i]);
  float o = 0.f, L = 0.f;
  if (M != -INFINITY) {
    for (int i = 0; i < num_splits; ++i) {
      const float f = ex2(ml[2 * i] - M);
      o += f * ws_o[(bh * num_splits + i) * kHeadDim + ch];
      L += f * ml[2 * i + 1];
    }
  }
  out[bh * kHeadDim + ch] = L > 0.f ? o / L : 0.f;
  if (lse && ch == 0) lse[bh] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
}

// Grid (rows); block 128: merge of `parts` partial attentions of the same
// rows over disjoint token sets (section 3.2 of the arganzheng page attends
// the window and the quantized part apart and merges them the same way):
// out = sum_p e^(lse_p - L) out_p with L = ln sum_p e^(lse_p).  A part with
// lse = -inf has no tokens; a row with no tokens anywhere gets zeros.
__global__ void __launch_bounds__(kHeadDim) merge_partials_kernel(const float* __restrict__ outs,
                                                                  const float* __restrict__ lses, int parts,
                                                                  long long rows, float* __restrict__ out,
                                                                  float* __restrict__ lse_out) {
  const long long r = blockIdx.x;
  const int ch = threadIdx.x;
  float M = -INFINITY;
  for (int p = 0; p < parts; ++p) M = fmaxf(M, lses[p * rows + r]);
  float o = 0.f, L = 0.f;
  if (M != -INFINITY) {
    for (int p = 0; p < parts; ++p) {
      const float lp = lses[p * rows + r];
      const float w = lp == -INFINITY ? 0.f : expf(lp - M);
      L += w;
      o = fmaf(w, outs[(p * rows + r) * kHeadDim + ch], o);
    }
  }
  out[r * kHeadDim + ch] = L > 0.f ? o / L : 0.f;
  if (lse_out && ch == 0) lse_out[r] = L > 0.f ? M + logf(L) : -INFINITY;
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

// Split count: about one wave of resident CTAs (three per SM), with at
// least two chunks per warp.
int decode_default_splits(const kvq_shape& s, int max_len) {
  if (!is_fp8(s.format)) {
    // one wave of the streaming kernel, fewer CTAs when the batch holds too
    // few chunks for 2 per warp (small problems are latency-bound; measured
    // against 4 per warp: 17.5 -> 15.4 us on the 512-token check, 19.5 ->
    // 17.5 us on two 2K-token sequences of the 8B layer)
    const long long chunks = (long long)s.batch * s.num_kv_heads * ((max_len + kChunk - 1) / kChunk);
    const long long want = (chunks + 2 * kIntWarps - 1) / (2 * kIntWarps);
    return (int)max(1ll, min((long long)(148 * KVQ_DECODE_INT_MIN_BLOCKS), want));
  }
  const int units = s.batch * s.num_kv_heads;
  const int slots = 148 * kFp8MinBlocks;
  const int max_chunks = max(1, (max_len + kChunk - 1) / kChunk);
  int sq = slots / units;
  sq = max(1, min(sq, max_chunks / (2 * kWarps)));
  return sq;
}

size_t decode_workspace_bytes(const kvq_shape& s, int num_splits) {
  if (!is_fp8(s.format))
    return (int_ml_floats(s, num_splits) + int_slots(s, num_splits) * (s.num_q_heads / s.num_kv_heads) * kHeadDim) *
           sizeof(float);
  return (size_t)s.batch * s.num_q_heads * num_splits * (kHeadDim + 2) * sizeof(float);
}

static cudaError_t launch_fp8(const DecodeArgs& A, cudaStream_t st) {
  constexpr int smem = fp8_smem_bytes();
  // The attribute is per device; setting it again is harmless, so a racing
  // first call from two threads only repeats the work.
  static std::atomic<unsigned long long> attr_done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !((attr_done.load(std::memory_order_relaxed) >> dev) & 1ull)) {
    e = cudaFuncSetAttribute(decode_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_done.fetch_or(1ull << dev, std::memory_order_relaxed);
  }
  const kvq_shape& s = A.c.shape;
  dim3 grid(A.num_splits, s.num_kv_heads, s.batch);
  decode_fp8_kernel<<<grid, kWarps * 32, smem, st>>>(A);
  return cudaGetLastError();
}

// Channel split CS of the combine grid (H_q, B, CS).  A CTA's 128 threads
// are 32 / CS channel quads x 4 CS slot lanes, so CS sets how many partial
// slots each lane merges: about four (a unit holds about 4 num_splits /
// units + 1 slots), which keeps the per-CTA setup and the shuffle tree over
// the slot lanes small against the merge itself; a power of two from 1 to
// 32, and no more CTAs than are resident at once (one wave).
static cudaError_t combine_split(const kvq_shape& s, int num_splits, int dev, int& cs) {
  static std::atomic<int> resident[64];   // 0 until looked up; racing lookups store the same value
  int r = dev < 64 ? resident[dev].load(std::memory_order_relaxed) : 0;
  if (r == 0) {
    int per_sm = 0, sms = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_int_combine_kernel, kCombineThreads, 0);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    r = per_sm * sms;
    if (dev < 64) resident[dev].store(r, std::memory_order_relaxed);
  }
  const long long heads = (long long)s.batch * s.num_q_heads;
  const long long units = (long long)s.batch * s.num_kv_heads;
  const long long slots_per_unit = (long long)kIntWarps * num_splits / units + 1;
  cs = 1;
  while (cs < 32 && 16ll * cs < slots_per_unit) cs <<= 1;
  while (cs > 1 && heads * cs > r) cs >>= 1;
  return cudaSuccess;
}

template <int FMT, bool PAGED, bool WIDE, bool ROPE = false, bool SP = false>
static cudaError_t launch_int_t(const IntArgs& A, cudaStream_t st) {
  const int smem = decode_int_smem_bytes<FMT, SP>() +
                   (SP ? decode_int_sp_extra_bytes(A.c.shape.num_q_heads / A.c.shape.num_kv_heads) : 0);
  static std::atomic<unsigned long long> attr_done{0};   // per device, as in launch_fp8
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !((attr_done.load(std::memory_order_relaxed) >> dev) & 1ull)) {
    e = cudaFuncSetAttribute(decode_int_kernel<FMT, PAGED, WIDE, ROPE, SP>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             decode_int_smem_bytes<FMT, SP>() + (SP ? decode_int_sp_extra_bytes(kMaxHeadsPerKv) : 0));
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_done.fetch_or(1ull << dev, std::memory_order_relaxed);
  }
  decode_int_kernel<FMT, PAGED, WIDE, ROPE, SP><<<A.num_splits, kIntWarps * 32, smem, st>>>(A);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // the combine starts early (programmatic dependent launch): its window
  // work overlaps the streaming kernel's tail, its merge waits for it
  const kvq_shape& s = A.c.shape;
  int cs = 1;
  e = combine_split(s, A.num_splits, dev, cs);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(s.num_q_heads, s.batch, cs);
  cfg.blockDim = dim3(kCombineThreads);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  pdl_attribute(attr[0]);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_int_combine_kernel, A);
}

template <int FMT>
static cudaError_t launch_int(const IntArgs& A, cudaStream_t st) {
  const kvq_shape& s = A.c.shape;
  const bool paged = s.page_size != 0, wide = s.num_q_heads / s.num_kv_heads > 4;
  if constexpr (FMT != 16 && FMT != 6) {     // INT8 and MIXED are contiguous only
    if (paged) return wide ? launch_int_t<FMT, true, true>(A, st) : launch_int_t<FMT, true, false>(A, st);
  }
  if constexpr (FMT == 2 || FMT == 4) {       // keys stored before RoPE (contiguous INT2 / INT4)
    if (s.rope_theta > 0.f)
      return wide ? launch_int_t<FMT, false, true, true>(A, st) : launch_int_t<FMT, false, false, true>(A, st);
    if (s.sparse)                             // dense-and-sparse (contiguous INT2 / INT4)
      return wide ? launch_int_t<FMT, false, true, false, true>(A, st)
                  : launch_int_t<FMT, false, false, false, true>(A, st);
  }
  return wide ? launch_int_t<FMT, false, true>(A, st) : launch_int_t<FMT, false, false>(A, st);
}

cudaError_t launch_decode(const kvq_cache& c, const void* q, float* out, float* lse, float softmax_scale, void* ws,
                          int num_splits, cudaStream_t st) {
  const kvq_shape& s = c.shape;
  const float scale_log2 = softmax_scale * 1.4426950408889634f;
  if (!is_fp8(s.format)) {
    IntArgs A;
    A.c = c;
    A.q = (const uint16_t*)q;
    A.num_splits = num_splits;
    A.ws_ml = (float*)ws;
    A.ws_o = (float*)ws + int_ml_floats(s, num_splits);
    A.out = out;
    A.lse = lse;
    A.scale_log2 = scale_log2;
    if (s.format == KVQ_FORMAT_INT8) return launch_int<16>(A, st);
    if (s.format == KVQ_FORMAT_MIXED) return launch_int<6>(A, st);
    return s.format == KVQ_FORMAT_INT4 ? launch_int<4>(A, st) : launch_int<2>(A, st);
  }
  DecodeArgs A;
  A.c = c;
  A.q = (const uint16_t*)q;
  A.num_splits = num_splits;
  A.ws_ml = (float*)ws;
  A.ws_o = (float*)ws + (size_t)s.batch * s.num_q_heads * num_splits * 2;
  A.scale_log2 = scale_log2;
  cudaError_t e = launch_fp8(A, st);
  if (e != cudaSuccess) return e;
  // programmatic dependent launch: the combine's launch overlaps the
  // streaming kernel's tail, and it waits for it on the device
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(s.batch * s.num_q_heads);
  cfg.blockDim = dim3(kHeadDim);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  pdl_attribute(attr[0]);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_combine_kernel, (const float*)A.ws_o, (const float*)A.ws_ml, out, lse,
                            num_splits);
}

cudaError_t launch_merge(const float* outs, const float* lses, int parts, long long rows, float* out, float* lse_out,
                         cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  merge_partials_kernel<<<(unsigned)rows, kHeadDim, 0, st>>>(outs, lses, parts, rows, out, lse_out);
  return cudaGetLastError();
}

}  // namespace kvq
