// Write side of the cache: prefill quantization, append, flush (INT2/INT4),
// and the FP8-E4M3 comparison cache.
//
// Key groups: one CTA team of G/16 warps quantizes one group of G tokens of
// one (sequence, kv head).  Each lane loads 16-byte pieces (8 channels) of 8
// token rows, reduces min/max per channel over the group with warp shuffles,
// derives fp16 scale/zero, and writes canonical packed rows.  The same warps
// then quantize the group's value tokens, one 16-token tile per warp, with
// min/max per token reduced over the 8 lanes that share the token, and write
// the tile in the decode's fragment order (include/kvq.h).
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
};

// Key half of a group: warp `wq` of `nw` = G/16 warps.
template <int BITS>
__device__ __forceinline__ void quantize_k_group(int wq, int G, const RowSrc& src, const GroupDst& dst) {
  const int lane = threadIdx.x & 31;
  const int nw = G / kTile;
  const int CW = kHeadDim / nw;          // channels of this warp
  const int LP = CW / 8;                 // lanes per token row
  const int TS = 32 / LP;                // token stride
  const int li = lane % LP, lt = lane / LP;
  const int c0 = wq * CW + li * 8;
  uint4 v[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) v[k] = *reinterpret_cast<const uint4*>(src.row(lt + TS * k) + c0);
  float mn[8], mx[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) { mn[c] = INFINITY; mx[c] = -INFINITY; }
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const float a = bf16_lo(w[p]), b = bf16_hi(w[p]);
      mn[2 * p] = fminf(mn[2 * p], a); mx[2 * p] = fmaxf(mx[2 * p], a);
      mn[2 * p + 1] = fminf(mn[2 * p + 1], b); mx[2 * p + 1] = fmaxf(mx[2 * p + 1], b);
    }
  }
  for (int off = LP; off < 32; off <<= 1) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      mn[c] = fminf(mn[c], __shfl_xor_sync(0xffffffffu, mn[c], off));
      mx[c] = fmaxf(mx[c], __shfl_xor_sync(0xffffffffu, mx[c], off));
    }
  }
  QParams qp[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) qp[c] = quant_params(mn[c], mx[c], BITS);
  // Key scale/zero rows in pair order (include/kvq.h): the decode reads
  // each half2 word as the pair of channels one fragment register holds.
  uint32_t sh[8], zh[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    sh[c] = __half_as_ushort(qp[c].s16);
    zh[c] = __half_as_ushort(qp[c].z16);
  }
  if (BITS == 4) {
    // channels u' = r + 4*h2 of this 8-channel block go to half 2r + h2
    if (lt == 0) {
      uint32_t s[4], z[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        s[r] = sh[r] | (sh[r + 4] << 16);
        z[r] = zh[r] | (zh[r + 4] << 16);
      }
      *reinterpret_cast<uint4*>(dst.k_meta + c0) = make_uint4(s[0], s[1], s[2], s[3]);
      *reinterpret_cast<uint4*>(dst.k_meta + kHeadDim + c0) = make_uint4(z[0], z[1], z[2], z[3]);
    }
  } else {
    // a 16-channel block pairs channel s' with s'+8 in half2 word s'; the
    // lane holding channels [c0, c0+8) of an even block half trades values
    // with its neighbour (which holds c0+8 ..)
    uint32_t ps[8], pz[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      ps[c] = __shfl_xor_sync(0xffffffffu, sh[c], 1);
      pz[c] = __shfl_xor_sync(0xffffffffu, zh[c], 1);
    }
    if (lt == 0 && (li & 1) == 0) {
      uint32_t s[8], z[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        s[k] = sh[k] | (ps[k] << 16);
        z[k] = zh[k] | (pz[k] << 16);
      }
      uint4* sd = reinterpret_cast<uint4*>(dst.k_meta + c0);
      uint4* zd = reinterpret_cast<uint4*>(dst.k_meta + kHeadDim + c0);
      sd[0] = make_uint4(s[0], s[1], s[2], s[3]);
      sd[1] = make_uint4(s[4], s[5], s[6], s[7]);
      zd[0] = make_uint4(z[0], z[1], z[2], z[3]);
      zd[1] = make_uint4(z[4], z[5], z[6], z[7]);
    }
  }
  constexpr int RB = kHeadDim * BITS / 8;
  constexpr int top = (1 << BITS) - 1;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
    uint32_t packed = 0;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const uint32_t a = encode(bf16_lo(w[p]), qp[2 * p].z, qp[2 * p].inv, top);
      const uint32_t b = encode(bf16_hi(w[p]), qp[2 * p + 1].z, qp[2 * p + 1].inv, top);
      packed |= (a << (BITS * 2 * p)) | (b << (BITS * (2 * p + 1)));
    }
    uint8_t* row = dst.k_codes + (size_t)(lt + TS * k) * RB;
    if (BITS == 4) *reinterpret_cast<uint32_t*>(row + c0 / 2) = packed;
    else *reinterpret_cast<uint16_t*>(row + c0 / 4) = (uint16_t)packed;
  }
}

// Value half of a group: warp `wq` quantizes tile wq (tokens 16wq..16wq+15).
template <int BITS>
__device__ __forceinline__ void quantize_v_tile(int wq, const RowSrc& src, const GroupDst& dst) {
  const int lane = threadIdx.x & 31;
  const int n = lane >> 2, l = lane & 3;
  const int tok[4] = {2 * l, 2 * l + 1, 2 * l + 8, 2 * l + 9};   // (s, o) = (0,0) (0,1) (1,0) (1,1)
  uint32_t x[4][8];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint16_t* r = src.row(kTile * wq + tok[q]) + 16 * n;
    const uint4 a = *reinterpret_cast<const uint4*>(r);
    const uint4 b = *reinterpret_cast<const uint4*>(r + 8);
    x[q][0] = a.x; x[q][1] = a.y; x[q][2] = a.z; x[q][3] = a.w;
    x[q][4] = b.x; x[q][5] = b.y; x[q][6] = b.z; x[q][7] = b.w;
  }
  QParams qp[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float mn = INFINITY, mx = -INFINITY;
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      mn = fminf(mn, fminf(bf16_lo(x[q][p]), bf16_hi(x[q][p])));
      mx = fmaxf(mx, fmaxf(bf16_lo(x[q][p]), bf16_hi(x[q][p])));
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    }
    qp[q] = quant_params(mn, mx, BITS);
  }
  constexpr int top = (1 << BITS) - 1;
  uint8_t* tile = dst.v_tiles + (size_t)wq * tile_bytes(BITS);
  if (BITS == 4) {
    uint32_t w[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int s = q >> 1, o = q & 1;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float val = (j & 1) ? bf16_hi(x[q][j >> 1]) : bf16_lo(x[q][j >> 1]);
        const uint32_t code = encode(val, qp[q].z, qp[q].inv, top);
        const int p = (j & 1) + 2 * s + 4 * o;
        w[j >> 1] |= code << (4 * p);
      }
    }
    *reinterpret_cast<uint4*>(tile + 16 * lane) = make_uint4(w[0], w[1], w[2], w[3]);
    *reinterpret_cast<uint4*>(tile + 512 + 16 * lane) = make_uint4(w[4], w[5], w[6], w[7]);
  } else {
    uint32_t w[4] = {0, 0, 0, 0};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int s = q >> 1, o = q & 1;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float val = (j & 1) ? bf16_hi(x[q][j >> 1]) : bf16_lo(x[q][j >> 1]);
        const uint32_t code = encode(val, qp[q].z, qp[q].inv, top);
        const int p = (j & 3) + 4 * s + 8 * o;
        w[j >> 2] |= code << (2 * p);
      }
    }
    *reinterpret_cast<uint4*>(tile + 16 * lane) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (n == 0) {
    uint32_t m[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      m[q] = (uint32_t)__half_as_ushort(qp[q].s16) | ((uint32_t)__half_as_ushort(qp[q].z16) << 16);
    __half* vm = dst.v_meta + 2 * (kTile * wq);
    *reinterpret_cast<uint2*>(vm + 2 * (2 * l)) = make_uint2(m[0], m[1]);
    *reinterpret_cast<uint2*>(vm + 2 * (2 * l + 8)) = make_uint2(m[2], m[3]);
  }
}

template <int BITS>
__device__ __forceinline__ void quantize_group(int wq, int G, const RowSrc& ks, const RowSrc& vs,
                                               const GroupDst& dst) {
  quantize_k_group<BITS>(wq, G, ks, dst);
  quantize_v_tile<BITS>(wq, vs, dst);
}

__device__ __forceinline__ void set_err(uint32_t* err, uint32_t bit) { atomicOr(err, bit); }

// Destination of group g of (b, h); false if its page id is out of range.
__device__ __forceinline__ bool group_dst(const kvq_cache& c, int b, int h, int g, GroupDst& d) {
  const kvq_shape& s = c.shape;
  if (s.page_size == 0) {
    d.k_codes = (uint8_t*)c.k_codes + Addr::k_codes_unit(s, b, h) + (size_t)g * s.group * row_bytes(s.format);
    d.k_meta = (__half*)c.k_meta + Addr::k_meta_group(s, b, h, g);
    d.v_tiles = (uint8_t*)c.v_codes + Addr::v_codes_tile(s, b, h, g * (s.group / kTile));
    d.v_meta = (__half*)c.v_meta + Addr::v_meta_token(s, b, h, g * s.group);
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

// Grid (ceil(max_len/G), H_kv, B); block G/16 warps.
template <int BITS>
__global__ void __launch_bounds__(256) prefill_int_kernel(kvq_cache c, const uint16_t* __restrict__ k,
                                                          const uint16_t* __restrict__ v,
                                                          const int32_t* __restrict__ cu) {
  const kvq_shape& s = c.shape;
  const int g = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int G = s.group, Ws = window_slots(s);
  const int t0 = cu[b];
  int n = cu[b + 1] - t0;
  const bool too_long = n > s.capacity || n < 0;
  if (too_long) n = 0;
  const int nq = quantized_prefix(n, s.residual, G);
  if (g == 0 && h == 0 && threadIdx.x == 0) {
    c.seq_len[b] = n;
    c.n_quant[b] = nq;
    if (too_long) set_err(c.err_word, KVQ_DEVERR_PREFILL_LEN);
  }
  const int64_t stride = (int64_t)s.num_kv_heads * kHeadDim;
  const int wq = threadIdx.x >> 5;
  if (g * G < nq) {
    GroupDst d;
    if (!group_dst(c, b, h, g, d)) {
      if (threadIdx.x == 0) set_err(c.err_word, KVQ_DEVERR_PAGE_RANGE);
      return;
    }
    const RowSrc ks{k + ((int64_t)(t0 + g * G) * s.num_kv_heads + h) * kHeadDim, stride, 0, 0};
    const RowSrc vs{v + ((int64_t)(t0 + g * G) * s.num_kv_heads + h) * kHeadDim, stride, 0, 0};
    quantize_group<BITS>(wq, G, ks, vs, d);
  } else {
    // window tokens [max(gG, nq), min((g+1)G, n)) -> ring slots t mod (R+G)
    const int lo = max(g * G, nq), hi = min((g + 1) * G, n);
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
}

// Grid (B); block (kv heads per pass) * G/16 warps.  Quantizes the oldest G
// window tokens of every kv head of sequence b when the window is full.
template <int BITS>
__global__ void __launch_bounds__(512) flush_int_kernel(kvq_cache c, int heads_per_pass) {
  const kvq_shape& s = c.shape;
  const int b = blockIdx.x;
  const int G = s.group, Ws = window_slots(s);
  const int n = c.seq_len[b], nq = c.n_quant[b];
  if (n - nq != Ws) return;
  if (nq < 0 || nq + G > s.capacity || nq % G) {
    if (threadIdx.x == 0) set_err(c.err_word, KVQ_DEVERR_STATE);
    return;
  }
  const int team = G / kTile;
  const int warp = threadIdx.x >> 5;
  const int hsub = warp / team, wq = warp % team;
  bool page_ok = true;
  for (int h0 = 0; h0 < s.num_kv_heads; h0 += heads_per_pass) {
    const int h = h0 + hsub;
    if (hsub < heads_per_pass && h < s.num_kv_heads) {
      GroupDst d;
      if (group_dst(c, b, h, nq / G, d)) {
        const RowSrc ks{(const uint16_t*)c.k_res + Addr::ring_row(s, b, h, 0), kHeadDim, nq % Ws, Ws};
        const RowSrc vs{(const uint16_t*)c.v_res + Addr::ring_row(s, b, h, 0), kHeadDim, nq % Ws, Ws};
        quantize_group<BITS>(wq, G, ks, vs, d);
      } else {
        page_ok = false;
      }
    }
  }
  __syncthreads();
  const int bad = __syncthreads_or(!page_ok);
  if (threadIdx.x == 0) {
    if (bad) set_err(c.err_word, KVQ_DEVERR_PAGE_RANGE);
    else c.n_quant[b] = nq + G;
  }
}

// Grid (B); block H_kv * 32 threads.  INT formats: token -> window slot.
__global__ void append_int_kernel(kvq_cache c, const uint16_t* __restrict__ kn, const uint16_t* __restrict__ vn) {
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
  __syncthreads();
  if (threadIdx.x == 0) c.seq_len[b] = n + 1;
}

// ---------------------------------------------------------------------------
// FP8-E4M3 cache
// ---------------------------------------------------------------------------

// Grid (ceil(max_len/64), H_kv, B): amax |x| over a 64-token chunk of one kv
// head, folded into fp8_amax[0|1][h] (non-negative floats order like their bits).
__global__ void fp8_amax_kernel(kvq_cache c, const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
                                const int32_t* __restrict__ cu) {
  const kvq_shape& s = c.shape;
  const int h = blockIdx.y, b = blockIdx.z;
  const int t0 = cu[b];
  const int n = cu[b + 1] - t0;
  if (n > s.capacity || n < 0) return;
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

__device__ __forceinline__ void fp8_write_token(const kvq_cache& c, int b, int h, int t, const uint16_t* krow,
                                                const uint16_t* vrow, float inv_k, float inv_v, int lane) {
  // lane handles channels 4*lane .. 4*lane+3
  const kvq_shape& s = c.shape;
  const uint2 kx = *reinterpret_cast<const uint2*>(krow + 4 * lane);
  const uint2 vx = *reinterpret_cast<const uint2*>(vrow + 4 * lane);
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

// Grid (ceil(max_len/16), H_kv, B); block 16 warps: warp i encodes token
// 16*blockIdx.x + i (zeros for tokens past the end of the sequence).
__global__ void __launch_bounds__(512) fp8_prefill_kernel(kvq_cache c, const uint16_t* __restrict__ k,
                                                          const uint16_t* __restrict__ v,
                                                          const int32_t* __restrict__ cu) {
  const kvq_shape& s = c.shape;
  const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int t0 = cu[b];
  int n = cu[b + 1] - t0;
  const bool too_long = n > s.capacity || n < 0;
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
  const int n = c.seq_len[b];
  if (n >= s.capacity || n < 0) {
    if (threadIdx.x == 0) set_err(c.err_word, KVQ_DEVERR_APPEND_FULL);
    return;
  }
  const int h = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (h < s.num_kv_heads) {
    const float Sk = c.fp8_scale[h], Sv = c.fp8_scale[s.num_kv_heads + h];
    const size_t off = ((size_t)b * s.num_kv_heads + h) * kHeadDim;
    fp8_write_token(c, b, h, n, kn + off, vn + off, __frcp_rn(Sk), __frcp_rn(Sv), lane);
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
  if (max_len <= 0) max_len = 1;
  if (is_fp8(s.format)) {
    cudaError_t e = cudaMemsetAsync(c.fp8_amax, 0, sizeof(uint32_t) * 2 * s.num_kv_heads, st);
    if (e != cudaSuccess) return e;
    dim3 ga((max_len + 63) / 64, s.num_kv_heads, s.batch);
    fp8_amax_kernel<<<ga, 128, 0, st>>>(c, (const uint16_t*)k, (const uint16_t*)v, cu);
    dim3 gp((max_len + kTile - 1) / kTile, s.num_kv_heads, s.batch);
    fp8_prefill_kernel<<<gp, 32 * kTile, 0, st>>>(c, (const uint16_t*)k, (const uint16_t*)v, cu);
    return cudaGetLastError();
  }
  dim3 grid((max_len + s.group - 1) / s.group, s.num_kv_heads, s.batch);
  const int threads = 32 * (s.group / kTile);
  if (s.format == KVQ_FORMAT_INT4)
    prefill_int_kernel<4><<<grid, threads, 0, st>>>(c, (const uint16_t*)k, (const uint16_t*)v, cu);
  else
    prefill_int_kernel<2><<<grid, threads, 0, st>>>(c, (const uint16_t*)k, (const uint16_t*)v, cu);
  return cudaGetLastError();
}

cudaError_t launch_append(const kvq_cache& c, const void* kn, const void* vn, cudaStream_t st) {
  const kvq_shape& s = c.shape;
  if (is_fp8(s.format))
    fp8_append_kernel<<<s.batch, 32 * s.num_kv_heads, 0, st>>>(c, (const uint16_t*)kn, (const uint16_t*)vn);
  else
    append_int_kernel<<<s.batch, 32 * min(s.num_kv_heads, 32), 0, st>>>(c, (const uint16_t*)kn,
                                                                        (const uint16_t*)vn);
  return cudaGetLastError();
}

cudaError_t launch_flush(const kvq_cache& c, cudaStream_t st) {
  const kvq_shape& s = c.shape;
  if (is_fp8(s.format)) return cudaSuccess;
  const int team = s.group / kTile;
  const int per_pass = max(1, min(s.num_kv_heads, 16 / team));   // at most 512 threads
  const int threads = 32 * team * per_pass;
  if (s.format == KVQ_FORMAT_INT4) flush_int_kernel<4><<<s.batch, threads, 0, st>>>(c, per_pass);
  else flush_int_kernel<2><<<s.batch, threads, 0, st>>>(c, per_pass);
  return cudaGetLastError();
}

}  // namespace kvq
