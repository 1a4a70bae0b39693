// Decode attention over the packed cache (split-K / flash-decoding).
//
// Grid (splits, H_kv, B); 4 warps per CTA.  A split owns a contiguous range of
// key groups of one (sequence, kv head); each warp takes every 4th group and
// streams its 16-token tiles through a private ring of shared-memory stages
// filled by 1-D bulk copies (the TMA engine) that complete on an mbarrier.
// For INT formats the last split of each (b, kv) attends to the bf16 window.
//
// Scores and the value sum run on the tensor cores (mma.sync m16n8k16, fp32
// accumulate) fed straight from registers:
//  * QK: A = the query with the group's per-channel key scale folded in,
//    q''[h][c] = q[h][c] * 2^-a * s_k[c], split into fp16 hi (rows 0-7) and
//    lo (rows 8-15) parts; B = key codes turned into exact fp16 integers.
//    The zero-point term sum_c q[h][c] z_k[c] is one more small MMA per group.
//  * PV: A = p[h][t] * s_v[t] split into fp16 hi/lo rows; B = value codes as
//    exact fp16 integers; the value zero points add sum_t p[h][t] z_v[t].
// Rows 0-7 / 8-15 hold the hi / lo parts of the (up to) 8 query heads that
// share the kv head, so one MMA carries both precision terms.
//
// Softmax is online per warp (running max in log2 units, rescaled only when
// a tile raises it); warps merge in shared memory; a combine kernel merges
// the splits.
#include "kvq_common.cuh"

namespace kvq {

constexpr int kWarps = 4;
constexpr int kMergeStride = 132;   // floats per (warp, head) row of the merge buffer: 128 + m, l, pad (16-byte rows)

template <int FMT> struct DecodeCfg;
template <> struct DecodeCfg<4> { static constexpr int kStages = 8;  static constexpr int kKBytes = 16 * 64;  static constexpr int kVBytes = 1024; };
template <> struct DecodeCfg<2> { static constexpr int kStages = 12; static constexpr int kKBytes = 16 * 32;  static constexpr int kVBytes = 512;  };
template <> struct DecodeCfg<8> { static constexpr int kStages = 6;  static constexpr int kKBytes = 16 * 128; static constexpr int kVBytes = 2048; };

template <int FMT> struct Stage {
  static constexpr int kK = 0;
  static constexpr int kV = DecodeCfg<FMT>::kKBytes;
  static constexpr int kKm = kV + DecodeCfg<FMT>::kVBytes;                 // INT only: [2][128] fp16
  static constexpr int kVm = kKm + (FMT == 8 ? 0 : 512);                    // INT only: [16][2] fp16
  static constexpr int kBytes = kVm + (FMT == 8 ? 0 : 64);
};

template <int FMT>
constexpr int decode_smem_bytes() {
  return kWarps * DecodeCfg<FMT>::kStages * (Stage<FMT>::kBytes + 8);
}

struct DecodeArgs {
  kvq_cache c;
  const uint16_t* q;       // [B][H_q][128] bf16
  float* ws_o;             // [B][H_q][S][128]
  float* ws_ml;            // [B][H_q][S][2]
  float scale_log2;        // softmax_scale * log2(e)
  int num_splits;          // S (INT: S-1 quantized splits + 1 window split)
};

struct SoftmaxState {
  float m;        // running max (log2 units) of this thread's head
  float l;        // this thread's share of the running sum
  float z;        // this thread's share of sum p * z_v
};

// Rescale the accumulators of this warp if any head's running max grew.
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

__device__ __forceinline__ float quad_max(float x) {
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 1));
  return fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 2));
}
__device__ __forceinline__ float quad_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  return x + __shfl_xor_sync(0xffffffffu, x, 2);
}

// Per-warp result -> shared memory; then the CTA merges its warps and writes
// one split partial.  sm: kWarps * 8 * kMergeStride floats.
__device__ __forceinline__ void cta_merge_and_store(float* sm, const SoftmaxState& st, const float (&O)[16][4],
                                                   float out_scale, int gq, const DecodeArgs& A, int b, int kv,
                                                   int split) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, l = lane & 3;
  const float lsum = quad_sum(st.l);
  const float zsum = quad_sum(st.z);
  float* wo = sm + (size_t)(warp * 8 + g) * kMergeStride;
  float4* o4 = reinterpret_cast<float4*>(wo + 32 * l);
#pragma unroll
  for (int j4 = 0; j4 < 4; ++j4) {
    // channels 32l + j (j < 16) come from column 2l, 32l + 16 + j from column 2l+1
    o4[j4] = make_float4(O[4 * j4][0] + O[4 * j4][2] + zsum, O[4 * j4 + 1][0] + O[4 * j4 + 1][2] + zsum,
                         O[4 * j4 + 2][0] + O[4 * j4 + 2][2] + zsum, O[4 * j4 + 3][0] + O[4 * j4 + 3][2] + zsum);
    o4[4 + j4] = make_float4(O[4 * j4][1] + O[4 * j4][3] + zsum, O[4 * j4 + 1][1] + O[4 * j4 + 1][3] + zsum,
                             O[4 * j4 + 2][1] + O[4 * j4 + 2][3] + zsum,
                             O[4 * j4 + 3][1] + O[4 * j4 + 3][3] + zsum);
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
    A.ws_o[row * kHeadDim + ch] = o * out_scale;
    if (ch == 0) {
      A.ws_ml[row * 2] = M;
      A.ws_ml[row * 2 + 1] = L;
    }
  }
}

// q of this thread's head (row g), channels [32l, 32l+32), scaled by 2^-a so
// that |q * 2^-a| <= 1; returns the fp32 values and the power a.
__device__ __forceinline__ void load_q(const DecodeArgs& A, int b, int kv, int gq, float (&qf)[32], int& a_exp) {
  const int lane = threadIdx.x & 31, g = lane >> 2, l = lane & 3;
  const kvq_shape& s = A.c.shape;
  float amax = 0.f;
  if (g < gq) {
    const uint16_t* qr = A.q + ((size_t)b * s.num_q_heads + kv * gq + g) * kHeadDim + 32 * l;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 v = *reinterpret_cast<const uint4*>(qr + 8 * i);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        qf[8 * i + 2 * p] = bf16_lo(w[p]);
        qf[8 * i + 2 * p + 1] = bf16_hi(w[p]);
      }
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(qf[i]));
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) qf[i] = 0.f;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  int e = 0;
  if (amax > 0.f && amax < INFINITY) frexpf(amax, &e);   // amax < 2^e
  a_exp = e;
}

// Natural pairing of the fp16 query: pair (kb, s) = channels 32l + 4kb + 2s, +1.
__device__ __forceinline__ void q_pairs_natural(const float (&qf)[32], float sc, uint32_t (&qn)[8][2]) {
#pragma unroll
  for (int kb = 0; kb < 8; ++kb)
#pragma unroll
    for (int s = 0; s < 2; ++s) qn[kb][s] = pack_h2(qf[4 * kb + 2 * s] * sc, qf[4 * kb + 2 * s + 1] * sc);
}

// Pairing that matches the key-code unpack order.
//  INT4: pair (kb, s) = channels 32l + 8(kb/2) + 2(kb%2) + s, +4
//  INT2: pair (kb, s) = channels 32l + 16(kb/4) + 2(kb%4) + s, +8
template <int BITS>
__device__ __forceinline__ int kpair_first(int kb, int s) {
  return BITS == 4 ? 8 * (kb >> 1) + 2 * (kb & 1) + s : 16 * (kb >> 2) + 2 * (kb & 3) + s;
}
template <int BITS>
__device__ __forceinline__ void q_pairs_kcode(const float (&qf)[32], float sc, uint32_t (&qi)[8][2]) {
  constexpr int step = BITS == 4 ? 4 : 8;
#pragma unroll
  for (int kb = 0; kb < 8; ++kb)
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const int c = kpair_first<BITS>(kb, s);
      qi[kb][s] = pack_h2(qf[c] * sc, qf[c + step] * sc);
    }
}

// ---------------------------------------------------------------------------
// Quantized tiles (INT2 / INT4 / FP8)
// ---------------------------------------------------------------------------

template <int FMT, bool PAGED>
__device__ __forceinline__ void decode_quantized(const DecodeArgs& A, uint8_t* smem, int b, int kv, int split) {
  using Cfg = DecodeCfg<FMT>;
  using St = Stage<FMT>;
  constexpr int NS = Cfg::kStages;
  constexpr bool INT = FMT != 8;
  const kvq_cache& c = A.c;
  const kvq_shape& s = c.shape;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, l = lane & 3;
  const int gq = s.num_q_heads / s.num_kv_heads;

  const int n = c.seq_len[b];
  const int nq = INT ? c.n_quant[b] : n;
  const int G = INT ? s.group : kTile;
  const int T = G / kTile;                               // tiles per group
  int n_groups = INT ? (nq > 0 ? nq / G : 0) : (n + kTile - 1) / kTile;
  bool bad_state = n < 0 || nq < 0 || nq > n || nq > s.capacity || (INT && nq % G);
  if (bad_state) n_groups = 0;
  const int qsplits = INT ? A.num_splits - 1 : A.num_splits;
  const int per = (n_groups + qsplits - 1) / max(qsplits, 1);
  const int g_begin = min(split * per, n_groups), g_end = min(g_begin + per, n_groups);
  // this warp's groups: g_begin + warp + kWarps*k
  const int my_groups = g_end - g_begin > warp ? (g_end - g_begin - warp + kWarps - 1) / kWarps : 0;
  const int n_steps = my_groups * T;

  uint8_t* ring = smem + (size_t)warp * NS * St::kBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)kWarps * NS * St::kBytes) + warp * NS;

  // page / unit addressing of tile t of group gi
  auto tile_src = [&](int gi, int t, const uint8_t*& kc, const uint8_t*& vc, const __half*& km,
                      const __half*& vm) -> bool {
    if (!PAGED) {
      kc = (const uint8_t*)c.k_codes + Addr::k_codes_unit(s, b, kv) + ((size_t)gi * G + t * kTile) * row_bytes(FMT);
      vc = (const uint8_t*)c.v_codes + Addr::v_codes_tile(s, b, kv, gi * T + t);
      if (INT) {
        km = (const __half*)c.k_meta + Addr::k_meta_group(s, b, kv, gi);
        vm = (const __half*)c.v_meta + Addr::v_meta_token(s, b, kv, gi * G + t * kTile);
      }
      return true;
    }
    const int page = c.page_table[(size_t)b * s.max_pages_per_seq + gi];
    if (page < 0 || page >= s.num_pages) return false;
    kc = (const uint8_t*)c.k_codes + Addr::pg_k_codes(s, page, kv);
    vc = (const uint8_t*)c.v_codes + Addr::pg_v_codes(s, page, kv);
    if (INT) {
      km = (const __half*)c.k_meta + Addr::pg_k_meta(s, page, kv);
      vm = (const __half*)c.v_meta + Addr::pg_v_meta(s, page, kv);
    }
    return true;
  };

  auto issue = [&](int i) {   // lane 0 only
    const int st = i % NS;
    const int gi = g_begin + warp + kWarps * (i / T), t = i % T;
    const uint8_t *kc = nullptr, *vc = nullptr;
    const __half *km = nullptr, *vm = nullptr;
    uint8_t* dst = ring + (size_t)st * St::kBytes;
    if (!tile_src(gi, t, kc, vc, km, vm)) {
      asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(&bars[st])) : "memory");
      return;
    }
    uint32_t bytes = Cfg::kKBytes + Cfg::kVBytes;
    if (INT) bytes += 64 + (t == 0 ? 512 : 0);
    mbar_expect_tx(&bars[st], bytes);
    bulk_g2s(dst + St::kK, kc, Cfg::kKBytes, &bars[st]);
    bulk_g2s(dst + St::kV, vc, Cfg::kVBytes, &bars[st]);
    if (INT) {
      bulk_g2s(dst + St::kVm, vm, 64, &bars[st]);
      if (t == 0) bulk_g2s(dst + St::kKm, km, 512, &bars[st]);
    }
  };

  if (lane == 0) {
    for (int i = 0; i < NS; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
  }
  __syncwarp();
  if (lane == 0)
    for (int i = 0; i < min(NS, n_steps); ++i) issue(i);

  // ---- per-CTA query setup ----
  float qf[32];
  int a_exp;
  load_q(A, b, kv, gq, qf, a_exp);
  const float sc = ldexpf(1.f, -a_exp);
  uint32_t qn[8][2];
  q_pairs_natural(qf, sc, qn);
  uint32_t qi[8][2];
  if constexpr (INT) q_pairs_kcode<FMT>(qf, sc, qi);
  float s_mul = A.scale_log2 * ldexpf(1.f, a_exp);      // acc * s_mul = logit in log2 units
  float out_scale = 1.f;
  if constexpr (!INT) {
    s_mul *= c.fp8_scale[kv];
    out_scale = c.fp8_scale[s.num_kv_heads + kv];
  }

  SoftmaxState st{-INFINITY, 0.f, 0.f};
  float O[16][4];
#pragma unroll
  for (int j = 0; j < 16; ++j) O[j][0] = O[j][1] = O[j][2] = O[j][3] = 0.f;
  uint32_t Aq[8][4];          // A fragments of q'' for the current group (INT)
  float zterm = 0.f;
  bool timed_out = false, page_bad = false;
  int stall_step = 0;

  for (int i = 0; i < n_steps; ++i) {
    const int stg = i % NS;
    const uint32_t phase = (uint32_t)(i / NS) & 1u;
    const bool arrived = mbar_wait_bounded(&bars[stg], phase);
    if (!__all_sync(0xffffffffu, arrived)) { timed_out = true; stall_step = i; break; }
    const int gi = g_begin + warp + kWarps * (i / T), t = i % T;
    const uint8_t* sbuf = ring + (size_t)stg * St::kBytes;
    bool valid = true;
    if (PAGED) {
      const int page = c.page_table[(size_t)b * s.max_pages_per_seq + gi];
      valid = page >= 0 && page < s.num_pages;
    }
    if (!valid) {
      page_bad = true;
    } else {
      // ---- per-group A-prep (INT): q'' = q16 * s_k, hi/lo; zero-point term ----
      if constexpr (INT) {
        if (t == 0) {
          const uint4* kmv = reinterpret_cast<const uint4*>(sbuf + St::kKm) + 4 * l;  // scale row, channels 32l..
          uint32_t skw[16], zkw[16];
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            const uint4 a = kmv[v4], z = kmv[16 + v4];
            skw[4 * v4] = a.x; skw[4 * v4 + 1] = a.y; skw[4 * v4 + 2] = a.z; skw[4 * v4 + 3] = a.w;
            zkw[4 * v4] = z.x; zkw[4 * v4 + 1] = z.y; zkw[4 * v4 + 2] = z.z; zkw[4 * v4 + 3] = z.w;
          }
          constexpr int half_step = FMT == 4 ? 2 : 4;     // words between a channel and its partner
#pragma unroll
          for (int kb = 0; kb < 8; ++kb) {
#pragma unroll
            for (int sb = 0; sb < 2; ++sb) {
              const int u = kpair_first<FMT>(kb, sb);       // local channel of the pair's first element
              const uint32_t sel = (u & 1) ? 0x7632u : 0x5410u;
              const uint32_t skp = prmt(skw[u >> 1], skw[(u >> 1) + half_step], sel);
              const __half2 hi = __hmul2(u32_as_h2(qi[kb][sb]), u32_as_h2(skp));
              const __half2 lo = __hfma2(u32_as_h2(qi[kb][sb]), u32_as_h2(skp), __hneg2(hi));
              Aq[kb][2 * sb] = h2_as_u32(hi);
              Aq[kb][2 * sb + 1] = h2_as_u32(lo);
            }
          }
          float zc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int kb = 0; kb < 8; ++kb) mma_f16(zc, qn[kb][0], 0u, qn[kb][1], 0u, zkw[2 * kb], zkw[2 * kb + 1]);
          zterm = zc[0];
        }
      }
      // ---- QK: two n8 tiles of 8 tokens ----
      float S[2][2];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        const uint8_t* krow = sbuf + St::kK + (size_t)(8 * nt + g) * (Cfg::kKBytes / kTile);
        if constexpr (FMT == 4) {
          const uint4 kw = *reinterpret_cast<const uint4*>(krow + 16 * l);
          const uint32_t w[4] = {kw.x, kw.y, kw.z, kw.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint32_t bq[4];
            unpack_int4_word(w[j], bq);
            mma_f16(acc, Aq[2 * j][0], Aq[2 * j][1], Aq[2 * j][2], Aq[2 * j][3], bq[0], bq[1]);
            mma_f16(acc, Aq[2 * j + 1][0], Aq[2 * j + 1][1], Aq[2 * j + 1][2], Aq[2 * j + 1][3], bq[2], bq[3]);
          }
        } else if constexpr (FMT == 2) {
          const uint2 kw = *reinterpret_cast<const uint2*>(krow + 8 * l);
          const uint32_t w[2] = {kw.x, kw.y};
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            uint32_t bq[8];
            unpack_int2_word(w[j], bq);
#pragma unroll
            for (int r = 0; r < 4; ++r)
              mma_f16(acc, Aq[4 * j + r][0], Aq[4 * j + r][1], Aq[4 * j + r][2], Aq[4 * j + r][3], bq[2 * r],
                      bq[2 * r + 1]);
          }
        } else {
          const uint4* kp = reinterpret_cast<const uint4*>(krow + 32 * l);
          const uint4 k0 = kp[0], k1 = kp[1];
          const uint32_t w[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
#pragma unroll
          for (int kb = 0; kb < 8; ++kb)
            mma_f16(acc, qn[kb][0], 0u, qn[kb][1], 0u, e4m3x2_to_h2(w[kb]), e4m3x2_to_h2(w[kb] >> 16));
        }
        S[nt][0] = (acc[0] + acc[2] + zterm) * s_mul;
        S[nt][1] = (acc[1] + acc[3] + zterm) * s_mul;
      }
      // masks: padded head rows; FP8 tokens past the end
      const int tok0 = (gi * T + t) * kTile;
      bool tail = false;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const bool dead = g >= gq || (!INT && tok0 + 8 * nt + 2 * l + e >= n);
          if (dead) S[nt][e] = -INFINITY;
        }
      if constexpr (!INT) tail = tok0 + kTile > n;

      const float tmax = quad_max(fmaxf(fmaxf(S[0][0], S[0][1]), fmaxf(S[1][0], S[1][1])));
      online_max_update(tmax, st, O);
      const float mref = st.m == -INFINITY ? 0.f : st.m;
      float p[2][2];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) p[nt][e] = ex2(S[nt][e] - mref);
      st.l += (p[0][0] + p[0][1]) + (p[1][0] + p[1][1]);

      uint32_t Ap[4];
      if constexpr (INT) {
        // per-token value scale/zero of tokens 2l, 2l+1 (nt 0) and 8+2l, 9+2l (nt 1)
        const uint2 m0 = *reinterpret_cast<const uint2*>(sbuf + St::kVm + 4 * (2 * l));
        const uint2 m1 = *reinterpret_cast<const uint2*>(sbuf + St::kVm + 4 * (8 + 2 * l));
        const float2 sz00 = __half22float2(u32_as_h2(m0.x)), sz01 = __half22float2(u32_as_h2(m0.y));
        const float2 sz10 = __half22float2(u32_as_h2(m1.x)), sz11 = __half22float2(u32_as_h2(m1.y));
        st.z += p[0][0] * sz00.y + p[0][1] * sz01.y + p[1][0] * sz10.y + p[1][1] * sz11.y;
        split_h2(p[0][0] * sz00.x, p[0][1] * sz01.x, Ap[0], Ap[1]);
        split_h2(p[1][0] * sz10.x, p[1][1] * sz11.x, Ap[2], Ap[3]);
      } else {
        split_h2(p[0][0], p[0][1], Ap[0], Ap[1]);
        split_h2(p[1][0], p[1][1], Ap[2], Ap[3]);
      }
      // ---- PV: 16 n8 tiles of output channels ----
      const uint8_t* vt = sbuf + St::kV;
      if constexpr (FMT == 4) {
        const uint4 v0 = *reinterpret_cast<const uint4*>(vt + 16 * lane);
        const uint4 v1 = *reinterpret_cast<const uint4*>(vt + 512 + 16 * lane);
        const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int ww = 0; ww < 8; ++ww) {
          uint32_t bv[4];
          unpack_int4_word(w[ww], bv);
          mma_f16(O[2 * ww], Ap[0], Ap[1], Ap[2], Ap[3], bv[0], bv[1]);
          mma_f16(O[2 * ww + 1], Ap[0], Ap[1], Ap[2], Ap[3], bv[2], bv[3]);
        }
      } else if constexpr (FMT == 2) {
        const uint4 v0 = *reinterpret_cast<const uint4*>(vt + 16 * lane);
        const uint32_t w[4] = {v0.x, v0.y, v0.z, v0.w};
#pragma unroll
        for (int ww = 0; ww < 4; ++ww) {
          uint32_t bv[8];
          unpack_int2_word(w[ww], bv);
#pragma unroll
          for (int r = 0; r < 4; ++r) mma_f16(O[4 * ww + r], Ap[0], Ap[1], Ap[2], Ap[3], bv[2 * r], bv[2 * r + 1]);
        }
      } else {
        // token validity of this thread's four value tokens (only the last tile can be partial)
        uint32_t keep = 0xFFFFFFFFu;
        if (tail) {
          const int tb = tok0 + 2 * l;
          keep = (tb < n ? 0x000000FFu : 0u) | (tb + 1 < n ? 0x0000FF00u : 0u) |
                 (tb + 8 < n ? 0x00FF0000u : 0u) | (tb + 9 < n ? 0xFF000000u : 0u);
        }
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const uint4 v = *reinterpret_cast<const uint4*>(vt + 512 * k4 + 16 * lane);
          const uint32_t w[4] = {v.x & keep, v.y & keep, v.z & keep, v.w & keep};
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
            mma_f16(O[4 * k4 + jj], Ap[0], Ap[1], Ap[2], Ap[3], e4m3x2_to_h2(w[jj]), e4m3x2_to_h2(w[jj] >> 16));
        }
      }
    }
    __syncwarp();
    if (lane == 0 && i + NS < n_steps) {
      fence_proxy_async_smem();
      issue(i + NS);
    }
  }
  if (timed_out && lane == 0) {
    // steps stall_step .. stall_step+NS-1 may still have copies in flight:
    // let them land (bounded) before the CTA's shared memory goes away
    for (int k = stall_step; k < min(stall_step + NS, n_steps); ++k)
      (void)mbar_wait_bounded(&bars[k % NS], (uint32_t)(k / NS) & 1u);
    atomicOr(c.err_word, KVQ_DEVERR_WAIT_TIMEOUT);
  }
  if (lane == 0) {
    if (page_bad) atomicOr(c.err_word, KVQ_DEVERR_PAGE_RANGE);
    if (bad_state && warp == 0 && split == 0) atomicOr(c.err_word, KVQ_DEVERR_STATE);
  }
  __syncthreads();   // all warps done with their rings before smem is reused for the merge
  cta_merge_and_store(reinterpret_cast<float*>(smem), st, O, out_scale, gq, A, b, kv, split);
}

// ---------------------------------------------------------------------------
// The bf16 window (INT formats): tokens [n_quant, seq_len) in ring slots
// ---------------------------------------------------------------------------

__device__ __forceinline__ void decode_window(const DecodeArgs& A, uint8_t* smem, int b, int kv, int split) {
  const kvq_cache& c = A.c;
  const kvq_shape& s = c.shape;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, l = lane & 3;
  const int gq = s.num_q_heads / s.num_kv_heads;
  const int Ws = window_slots(s);
  const int n = c.seq_len[b], nq = c.n_quant[b];
  int r = n - nq;
  if (r < 0 || r > Ws || nq < 0) r = 0;

  // bf16 query, natural pairs (kb, s) = channels 32l + 4kb + 2s, +1 (unscaled)
  uint32_t qb[8][2];
  if (g < gq) {
    const uint16_t* qr = A.q + ((size_t)b * s.num_q_heads + kv * gq + g) * kHeadDim + 32 * l;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 v = *reinterpret_cast<const uint4*>(qr + 8 * i);
      qb[2 * i][0] = v.x; qb[2 * i][1] = v.y; qb[2 * i + 1][0] = v.z; qb[2 * i + 1][1] = v.w;
    }
  } else {
#pragma unroll
    for (int kb = 0; kb < 8; ++kb) qb[kb][0] = qb[kb][1] = 0u;
  }
  SoftmaxState st{-INFINITY, 0.f, 0.f};
  float O[16][4];
#pragma unroll
  for (int j = 0; j < 16; ++j) O[j][0] = O[j][1] = O[j][2] = O[j][3] = 0.f;
  const uint16_t* kr = (const uint16_t*)c.k_res + Addr::ring_row(s, b, kv, 0);
  const uint16_t* vr = (const uint16_t*)c.v_res + Addr::ring_row(s, b, kv, 0);
  const int chunks = (r + kTile - 1) / kTile;
  for (int ci = warp; ci < chunks; ci += kWarps) {
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
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kb = 0; kb < 8; ++kb) mma_bf16(acc, qb[kb][0], 0u, qb[kb][1], 0u, w[2 * kb], w[2 * kb + 1]);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int tok = ci * kTile + 8 * nt + 2 * l + e;
        S[nt][e] = (g < gq && tok < r) ? acc[e] * A.scale_log2 : -INFINITY;
      }
    }
    const float tmax = quad_max(fmaxf(fmaxf(S[0][0], S[0][1]), fmaxf(S[1][0], S[1][1])));
    online_max_update(tmax, st, O);
    const float mref = st.m == -INFINITY ? 0.f : st.m;
    float p[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) p[nt][e] = ex2(S[nt][e] - mref);
    st.l += (p[0][0] + p[0][1]) + (p[1][0] + p[1][1]);
    uint32_t Ap[4];
    split_bf2(p[0][0], p[0][1], Ap[0], Ap[1]);
    split_bf2(p[1][0], p[1][1], Ap[2], Ap[3]);
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
    for (int j = 0; j < 16; ++j) {
      const uint32_t sel = (j & 1) ? 0x7632u : 0x5410u;
      const uint32_t b0 = prmt(vw[0][j >> 1], vw[1][j >> 1], sel);
      const uint32_t b1 = prmt(vw[2][j >> 1], vw[3][j >> 1], sel);
      mma_bf16(O[j], Ap[0], Ap[1], Ap[2], Ap[3], b0, b1);
    }
  }
  __syncthreads();
  cta_merge_and_store(reinterpret_cast<float*>(smem), st, O, 1.f, gq, A, b, kv, split);
}

template <int FMT, bool PAGED>
__global__ void __launch_bounds__(kWarps * 32) decode_split_kernel(DecodeArgs A) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int split = blockIdx.x, kv = blockIdx.y, b = blockIdx.z;
  if (FMT != 8 && split == A.num_splits - 1) decode_window(A, smem, b, kv, split);
  else decode_quantized<FMT, PAGED>(A, smem, b, kv, split);
}

// Grid (B * H_q); block 128: out[b][h][c] = merge over splits.
__global__ void decode_combine_kernel(const float* __restrict__ ws_o, const float* __restrict__ ws_ml, float* out,
                                      int num_splits) {
  const size_t bh = blockIdx.x;
  const int ch = threadIdx.x;
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
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

int decode_default_splits(const kvq_shape& s, int max_len) {
  const int units = s.batch * s.num_kv_heads;
  const int G = eff_group(s);
  const int max_groups = max(1, (max_len + G - 1) / G);
  const int target = 148 * 4;                      // CTAs: about two waves at two CTAs per SM
  int sq = (target + units - 1) / units;
  sq = max(1, min(sq, (max_groups + 1) / 2));      // at least ~2 groups per split
  return is_fp8(s.format) ? sq : sq + 1;           // + the window split
}

size_t decode_workspace_bytes(const kvq_shape& s, int num_splits) {
  return (size_t)s.batch * s.num_q_heads * num_splits * (kHeadDim + 2) * sizeof(float);
}

template <int FMT, bool PAGED>
static cudaError_t launch_decode_t(const DecodeArgs& A, cudaStream_t st) {
  constexpr int smem = decode_smem_bytes<FMT>();
  // The attribute is per device; setting it again is harmless, so a racing
  // first call from two threads only repeats the work.
  static unsigned long long attr_done = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !((attr_done >> dev) & 1ull)) {
    e = cudaFuncSetAttribute(decode_split_kernel<FMT, PAGED>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_done |= 1ull << dev;
  }
  const kvq_shape& s = A.c.shape;
  dim3 grid(A.num_splits, s.num_kv_heads, s.batch);
  decode_split_kernel<FMT, PAGED><<<grid, kWarps * 32, smem, st>>>(A);
  return cudaGetLastError();
}

cudaError_t launch_decode(const kvq_cache& c, const void* q, float* out, float softmax_scale, void* ws,
                          int num_splits, cudaStream_t st) {
  const kvq_shape& s = c.shape;
  DecodeArgs A;
  A.c = c;
  A.q = (const uint16_t*)q;
  A.num_splits = num_splits;
  A.ws_ml = (float*)ws;
  A.ws_o = (float*)ws + (size_t)s.batch * s.num_q_heads * num_splits * 2;
  A.scale_log2 = softmax_scale * 1.4426950408889634f;
  cudaError_t e;
  const bool paged = s.page_size != 0;
  switch (s.format) {
    case KVQ_FORMAT_INT4: e = paged ? launch_decode_t<4, true>(A, st) : launch_decode_t<4, false>(A, st); break;
    case KVQ_FORMAT_INT2: e = paged ? launch_decode_t<2, true>(A, st) : launch_decode_t<2, false>(A, st); break;
    default: e = launch_decode_t<8, false>(A, st); break;
  }
  if (e != cudaSuccess) return e;
  decode_combine_kernel<<<s.batch * s.num_q_heads, kHeadDim, 0, st>>>(A.ws_o, A.ws_ml, out, num_splits);
  return cudaGetLastError();
}

}  // namespace kvq
