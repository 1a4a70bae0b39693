// Internal helpers of libkvq (device code for sm_100a).  Nothing here is part
// of the C ABI; include/kvq.h is.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kvq.h"

namespace kvq {

constexpr int kHeadDim = 128;
constexpr int kTile = 16;              // tokens per value tile (and per page)
constexpr int kMaxGroup = 128;         // largest supported key group
constexpr int kMaxHeadsPerKv = 8;      // query heads per kv head handled by one CTA

// ---------------------------------------------------------------------------
// Shape-derived sizes (host and device)
// ---------------------------------------------------------------------------

__host__ __device__ inline bool is_fp8(int format) { return format == KVQ_FORMAT_FP8_E4M3; }
__host__ __device__ inline bool is_int8(int format) { return format == KVQ_FORMAT_INT8; }
// Formats that quantize every token when it is written (no window, n_quant == seq_len).
__host__ __device__ inline bool is_token_cache(int format) { return is_fp8(format) || is_int8(format); }
// MIXED: INT4 or INT2 per group; its regions are laid out (sized) as INT4.
__host__ __device__ inline bool is_mixed(int format) { return format == KVQ_FORMAT_MIXED; }
__host__ __device__ inline int row_bytes(int format) {       // packed bytes per token row
  return is_token_cache(format) ? kHeadDim : (is_mixed(format) ? kHeadDim / 2 : kHeadDim * format / 8);
}
__host__ __device__ inline int tile_bytes(int format) { return kTile * row_bytes(format); }
__host__ __device__ inline int window_slots(const kvq_shape& s) {
  return is_token_cache(s.format) ? 0 : s.residual + s.group;
}
__host__ __device__ inline int eff_group(const kvq_shape& s) { return is_token_cache(s.format) ? kTile : s.group; }

// Per-(b, kv) unit addressing of the cache regions.  For the paged layout the
// caller resolves the physical page first.
struct Addr {
  // contiguous layout
  __host__ __device__ static size_t k_codes_unit(const kvq_shape& s, int b, int h) {
    return ((size_t)b * s.num_kv_heads + h) * (size_t)s.capacity * row_bytes(s.format);
  }
  __host__ __device__ static size_t k_meta_group(const kvq_shape& s, int b, int h, int g) {  // in halves
    return (((size_t)b * s.num_kv_heads + h) * (size_t)(s.capacity / s.group) + g) * 2 * kHeadDim;
  }
  __host__ __device__ static size_t v_codes_tile(const kvq_shape& s, int b, int h, int tile) {
    return (((size_t)b * s.num_kv_heads + h) * (size_t)(s.capacity / kTile) + tile) * tile_bytes(s.format);
  }
  __host__ __device__ static size_t v_meta_token(const kvq_shape& s, int b, int h, int t) {  // in halves
    return (((size_t)b * s.num_kv_heads + h) * (size_t)s.capacity + t) * 2;
  }
  // INT8: per-token key (scale, zero), the same shape as the value table
  __host__ __device__ static size_t k_meta_token(const kvq_shape& s, int b, int h, int t) {  // in halves
    return v_meta_token(s, b, h, t);
  }
  __host__ __device__ static size_t ring_row(const kvq_shape& s, int b, int h, int slot) {  // in bf16 elems
    return (((size_t)b * s.num_kv_heads + h) * (size_t)window_slots(s) + slot) * kHeadDim;
  }
  // paged layout: one page holds one tile / group of 16 tokens
  __host__ __device__ static size_t pg_k_codes(const kvq_shape& s, int page, int h) {
    return ((size_t)page * s.num_kv_heads + h) * (size_t)tile_bytes(s.format);
  }
  __host__ __device__ static size_t pg_k_meta(const kvq_shape& s, int page, int h) {  // halves
    return ((size_t)page * s.num_kv_heads + h) * 2 * kHeadDim;
  }
  __host__ __device__ static size_t pg_v_codes(const kvq_shape& s, int page, int h) {
    return ((size_t)page * s.num_kv_heads + h) * (size_t)tile_bytes(s.format);
  }
  __host__ __device__ static size_t pg_v_meta(const kvq_shape& s, int page, int h) {  // halves
    return ((size_t)page * s.num_kv_heads + h) * 2 * kTile;
  }
};

// Position of channel c in a key scale/zero row (the decode's pair order,
// include/kvq.h).
template <int BITS>
__host__ __device__ __forceinline__ int kmeta_pos(int c) {
  if (BITS == 4) {   // u = 8J + (r & 1) + 4 (r >> 1) + 2h (r < 4, h < 2) stored at 8J + 2r + h
    const int u = c & 31, J = u >> 3, v = u & 7, h = (v >> 1) & 1, r = (v & 1) + 2 * (v >> 2);
    return (c & ~31) + 8 * J + 2 * r + h;
  } else {           // u = 16J + r + 8h (r < 8) stored at 16J + 2r + h
    const int u = c & 31, J = u >> 4, r = u & 7, h = (u >> 3) & 1;
    return (c & ~31) + 16 * J + 2 * r + h;
  }
}

// RoPE angle of pair i at position pos, reduced to [-pi, pi] in double
// (freq = theta^(-2i/128) in double), then its cosine and sine in fp32
// (the fast sine/cosine are accurate to about 2^-21 on [-pi, pi]).
__device__ __forceinline__ void rope_cos_sin(int pos, double freq, float& c, float& s) {
  const double a = (double)pos * freq;
  const double k = rint(a * 0.15915494309189533577);        // 1 / (2 pi)
  const double r = fma(-k, 6.28318530717958647692, a);       // a - 2 pi k
  __sincosf((float)r, &s, &c);
}

// ---------------------------------------------------------------------------
// The encoder: IEEE fp32 steps, each rounded on its own (no contraction)
// ---------------------------------------------------------------------------

struct QParams {
  __half s16, z16;
  float z, inv;
};

__device__ __forceinline__ QParams quant_params(float mn, float mx, int bits) {
  QParams p;
  const float levels = (float)((1 << bits) - 1);
  const float scale32 = __fdiv_rn(__fsub_rn(mx, mn), levels);
  p.s16 = __float2half_rn(scale32);
  p.z16 = __float2half_rn(__fadd_rn(mn, 0.0f));   // -0 -> +0
  const float s = __half2float(p.s16);
  p.z = __half2float(p.z16);
  p.inv = (s > 0.0f) ? __frcp_rn(s) : 0.0f;
  return p;
}

__device__ __forceinline__ uint32_t encode(float x, float z, float inv, int top) {
  const float t = __fmul_rn(__fsub_rn(x, z), inv);
  int r = __float2int_rn(t);                       // ties to even; NaN -> 0
  r = r < 0 ? 0 : (r > top ? top : r);
  return (uint32_t)r;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ---------------------------------------------------------------------------
// FP8 E4M3 (static scale)
// ---------------------------------------------------------------------------

__device__ __forceinline__ float fp8_scale_from_amax(float amax) {
  if (!(amax > 0.0f) || isinf(amax)) return 1.0f;
  return __fdiv_rn(amax, 448.0f);
}

__device__ __forceinline__ uint32_t e4m3_encode(float y) {
  return (uint32_t)__nv_cvt_float_to_fp8(y, __NV_SATFINITE, __NV_E4M3);
}

// ---------------------------------------------------------------------------
// Tensor-core fragments (mma.sync m16n8k16, fp32 accumulate)
// ---------------------------------------------------------------------------

__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// Two f32 -> f16x2 (lo in bits 0-15), round to nearest even.
__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  return h2_as_u32(__floats2half2_rn(lo, hi));
}
__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Split two fp32 values into fp16 hi and lo parts: x ~= hi + lo, ~22 bits.
__device__ __forceinline__ void split_h2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(x0, x1);
  const float2 hf = __half22float2(h);
  hi = h2_as_u32(h);
  lo = pack_h2(x0 - hf.x, x1 - hf.y);
}
__device__ __forceinline__ void split_bf2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const float2 hf = __bfloat1622float2(h);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = pack_bf2(x0 - hf.x, x1 - hf.y);
}

// Codes -> exact fp16 pairs.  OR-ing a code into the mantissa of 1024.0
// (0x6400) gives the half 1024 + code exactly; subtracting 1024 leaves the
// code.  Codes sitting higher in the half give 1024 + 2^k * code, undone by
// one fused multiply-add (exact: every value stays in [1024, 2048)).
__device__ __forceinline__ uint32_t lop_or(uint32_t a, uint32_t mask, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;\n" : "=r"(d) : "r"(a), "r"(mask), "r"(c));  // (a & mask) | c
  return d;
}

// Two e4m3 codes (bits 0-7, 8-15 of v) -> exact f16x2.
__device__ __forceinline__ uint32_t e4m3x2_to_h2(uint32_t v16) {
  __half2_raw r = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(v16 & 0xFFFFu), __NV_E4M3);
  return (uint32_t)r.x | ((uint32_t)r.y << 16);
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;\n" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start before the previous kernel on the stream ends;
// grid_dependency_wait() blocks until that kernel has finished and its
// memory is visible, grid_dependents_launch() lets the dependent start early.
// ---------------------------------------------------------------------------

__device__ __forceinline__ void grid_dependents_launch() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }

// Launch attribute set for a dependent kernel (see above).
inline void pdl_attribute(cudaLaunchAttribute& a) {
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = 1;
}

// ---------------------------------------------------------------------------
// Global -> shared copies: per-lane cp.async of 16-byte pieces in commit
// groups; the hardware tracks each thread's groups, so no wait spins.
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// cp.async of 16-byte pieces: lane l copies pieces l, l + 32, ... of the
// BYTES at src (BYTES a multiple of 16; both addresses 16-byte aligned).
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }
template <int BYTES>
__device__ __forceinline__ void warp_copy(uint8_t* dst, const uint8_t* src, int lane) {
  static_assert(BYTES % 16 == 0, "16-byte pieces");
#pragma unroll
  for (int off = 0; off < BYTES; off += 512)
    if (off + 16 * lane < BYTES) cp_async16(dst + off + 16 * lane, src + off + 16 * lane);
}

}  // namespace kvq
