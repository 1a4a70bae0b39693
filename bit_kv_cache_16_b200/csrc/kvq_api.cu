// C ABI of libkvq: host-side validation, buffer sizes and launches.  Every
// entry point checks its arguments before enqueuing anything.
#include <string.h>

#include "kvq_common.cuh"

namespace kvq {
cudaError_t launch_prefill(const kvq_cache& c, const void* k, const void* v, const int32_t* cu, int max_len,
                           cudaStream_t st);
cudaError_t launch_append(const kvq_cache& c, const void* kn, const void* vn, cudaStream_t st);
cudaError_t launch_flush(const kvq_cache& c, cudaStream_t st);
cudaError_t launch_append_flush(const kvq_cache& c, const void* kn, const void* vn, cudaStream_t st);
cudaError_t launch_prefill_mixed(const kvq_cache& c, const void* k, const void* v, const uint8_t* cls,
                                 const int32_t* cu, int max_len, cudaStream_t st);
cudaError_t launch_append_mixed(const kvq_cache& c, const void* kn, const void* vn, const uint8_t* cls,
                                cudaStream_t st);
cudaError_t launch_decode(const kvq_cache& c, const void* q, float* out, float* lse, float softmax_scale, void* ws,
                          int num_splits, cudaStream_t st);
cudaError_t launch_merge(const float* outs, const float* lses, int parts, long long rows, float* out, float* lse_out,
                         cudaStream_t st);
int decode_default_splits(const kvq_shape& s, int max_len);
size_t decode_workspace_bytes(const kvq_shape& s, int num_splits);
}  // namespace kvq

using namespace kvq;

namespace {

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

kvq_status check_shape(const kvq_shape* s) {
  if (!s) return KVQ_ERR_INVALID_ARG;
  if (s->format != KVQ_FORMAT_INT2 && s->format != KVQ_FORMAT_INT4 && s->format != KVQ_FORMAT_FP8_E4M3 &&
      s->format != KVQ_FORMAT_INT8 && s->format != KVQ_FORMAT_MIXED)
    return KVQ_ERR_INVALID_ARG;
  if (s->batch <= 0 || s->num_q_heads <= 0 || s->num_kv_heads <= 0 || s->head_dim <= 0 || s->capacity < 0)
    return KVQ_ERR_INVALID_ARG;
  if (s->head_dim != kHeadDim) return KVQ_ERR_UNSUPPORTED;
  if (s->num_q_heads % s->num_kv_heads) return KVQ_ERR_SHAPE;
  if (s->num_q_heads / s->num_kv_heads > kMaxHeadsPerKv) return KVQ_ERR_UNSUPPORTED;
  if (s->batch > 65535 || s->num_kv_heads > 65535) return KVQ_ERR_UNSUPPORTED;
  const bool fp8 = is_token_cache(s->format);     // FP8 and INT8: every token quantized on write
  if (!fp8) {
    if (s->group <= 0 || s->residual < 0) return KVQ_ERR_INVALID_ARG;
    // power-of-two groups of 16 to 128 tokens
    if (s->group < kTile || s->group > kMaxGroup || (s->group & (s->group - 1))) return KVQ_ERR_UNSUPPORTED;
  }
  // a mixed cache's 32-token decode chunks lie within one group
  if (is_mixed(s->format) && s->group < 32) return KVQ_ERR_UNSUPPORTED;
  if (s->page_size != 0) {
    if (s->page_size != kTile) return KVQ_ERR_UNSUPPORTED;
    if (fp8 || is_mixed(s->format)) return KVQ_ERR_UNSUPPORTED;
    if (s->group != kTile) return KVQ_ERR_SHAPE;   // the key group is aligned to the page
    if (s->max_pages_per_seq <= 0 || s->num_pages <= 0) return KVQ_ERR_INVALID_ARG;
    if (s->capacity != s->max_pages_per_seq * kTile) return KVQ_ERR_SHAPE;
  } else {
    if (s->capacity % (fp8 ? kTile : s->group)) return KVQ_ERR_SHAPE;
  }
  if ((int64_t)s->capacity > (1ll << 30)) return KVQ_ERR_UNSUPPORTED;
  if (!(s->rope_theta >= 0.0f) || isinf(s->rope_theta)) return KVQ_ERR_INVALID_ARG;
  if (s->rope_theta > 0.0f &&
      (s->page_size != 0 || (s->format != KVQ_FORMAT_INT2 && s->format != KVQ_FORMAT_INT4) || s->group < 32))
    return KVQ_ERR_UNSUPPORTED;       // keys rotated at read: contiguous INT2 / INT4, groups of 32 or more
  if (s->sparse != 0 && s->sparse != 1) return KVQ_ERR_INVALID_ARG;
  if (s->sparse && (s->page_size != 0 || (s->format != KVQ_FORMAT_INT2 && s->format != KVQ_FORMAT_INT4) ||
                    s->group > 32 || s->rope_theta > 0.0f))
    return KVQ_ERR_UNSUPPORTED;       // dense-and-sparse: contiguous INT2 / INT4, groups of 16 or 32
  return KVQ_OK;
}

kvq_status region_bytes(const kvq_shape& s, kvq_region r, size_t* out) {
  const bool fp8 = s.format == KVQ_FORMAT_FP8_E4M3, i8 = s.format == KVQ_FORMAT_INT8;
  const bool paged = s.page_size != 0;
  const size_t B = s.batch, H = s.num_kv_heads, cap = s.capacity, D = kHeadDim;
  const size_t RB = row_bytes(s.format), TB = tile_bytes(s.format);
  const size_t P = paged ? (size_t)s.num_pages : 0;
  size_t n = 0;
  switch (r) {
    case KVQ_REGION_K_CODES: n = paged ? P * H * TB : B * H * cap * RB; break;
    case KVQ_REGION_K_META:
      n = fp8 ? 0 : (i8 ? B * H * cap * 2 * 2 : (paged ? P * H * 2 * D * 2 : B * H * (cap / s.group) * 2 * D * 2));
      break;
    case KVQ_REGION_V_CODES: n = paged ? P * H * TB : B * H * (cap / kTile) * TB; break;
    case KVQ_REGION_V_META: n = fp8 ? 0 : (paged ? P * H * kTile * 2 * 2 : B * H * cap * 2 * 2); break;
    case KVQ_REGION_K_RES:
    case KVQ_REGION_V_RES: n = (fp8 || i8) ? 0 : B * H * (size_t)(s.residual + s.group) * D * 2; break;
    case KVQ_REGION_SEQ_LEN:
    case KVQ_REGION_N_QUANT: n = B * sizeof(int32_t); break;
    case KVQ_REGION_PAGE_TABLE: n = paged ? B * (size_t)s.max_pages_per_seq * sizeof(int32_t) : 0; break;
    case KVQ_REGION_FP8_SCALE: n = fp8 ? 2 * H * sizeof(float) : 0; break;
    case KVQ_REGION_FP8_AMAX: n = fp8 ? 2 * H * sizeof(uint32_t) : 0; break;
    case KVQ_REGION_ERR_WORD: n = sizeof(uint32_t); break;
    case KVQ_REGION_GROUP_BITS: n = is_mixed(s.format) ? B * (cap / s.group) : 0; break;
    case KVQ_REGION_WINDOW_CLASS: n = is_mixed(s.format) ? B * (size_t)(s.residual + s.group) : 0; break;
    case KVQ_REGION_K_SPARSE: n = s.sparse ? B * H * (cap / s.group) * D * 4 : 0; break;
    case KVQ_REGION_V_SPARSE: n = s.sparse ? B * H * cap * 4 : 0; break;
    default: return KVQ_ERR_INVALID_ARG;
  }
  *out = n;
  return KVQ_OK;
}

// Every region the format uses must be non-null and 16-byte aligned.
kvq_status check_cache(const kvq_cache* c) {
  if (!c) return KVQ_ERR_INVALID_ARG;
  kvq_status st = check_shape(&c->shape);
  if (st != KVQ_OK) return st;
  const kvq_shape& s = c->shape;
  const bool fp8 = s.format == KVQ_FORMAT_FP8_E4M3, i8 = s.format == KVQ_FORMAT_INT8;
  const void* need[] = {c->k_codes, c->v_codes, c->seq_len, c->n_quant, c->err_word};
  for (const void* p : need) {
    if (!p) return KVQ_ERR_INVALID_ARG;
    if (!aligned16(p)) return KVQ_ERR_ALIGNMENT;
  }
  if (i8) {
    const void* need_i8[] = {c->k_meta, c->v_meta};
    for (const void* p : need_i8) {
      if (!p) return KVQ_ERR_INVALID_ARG;
      if (!aligned16(p)) return KVQ_ERR_ALIGNMENT;
    }
  } else if (!fp8) {
    const void* need_int[] = {c->k_meta, c->v_meta, c->k_res, c->v_res};
    for (const void* p : need_int) {
      if (!p) return KVQ_ERR_INVALID_ARG;
      if (!aligned16(p)) return KVQ_ERR_ALIGNMENT;
    }
    if (s.sparse) {
      const void* need_sp[] = {c->k_sparse, c->v_sparse};
      for (const void* p : need_sp) {
        if (!p) return KVQ_ERR_INVALID_ARG;
        if (!aligned16(p)) return KVQ_ERR_ALIGNMENT;
      }
    }
    if (is_mixed(s.format)) {
      const void* need_mx[] = {c->group_bits, c->window_class};
      for (const void* p : need_mx) {
        if (!p) return KVQ_ERR_INVALID_ARG;
        if (!aligned16(p)) return KVQ_ERR_ALIGNMENT;
      }
    }
  } else {
    if (!c->fp8_scale || !c->fp8_amax) return KVQ_ERR_INVALID_ARG;
    if (!aligned16(c->fp8_scale) || !aligned16(c->fp8_amax)) return KVQ_ERR_ALIGNMENT;
  }
  if (s.page_size != 0) {
    if (!c->page_table) return KVQ_ERR_INVALID_ARG;
    if (!aligned16(c->page_table)) return KVQ_ERR_ALIGNMENT;
  }
  return KVQ_OK;
}

kvq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA; }

}  // namespace

extern "C" {

kvq_status kvq_buffer_bytes(const kvq_shape* shape, kvq_region region, size_t* bytes) {
  if (!bytes) return KVQ_ERR_INVALID_ARG;
  kvq_status st = check_shape(shape);
  if (st != KVQ_OK) return st;
  return region_bytes(*shape, region, bytes);
}

kvq_status kvq_quantize_prefill(kvq_cache* cache, const void* k_bf16, const void* v_bf16,
                                const int32_t* cu_seqlens_dev, int32_t max_len, kvq_stream_t stream) {
  kvq_status st = check_cache(cache);
  if (st != KVQ_OK) return st;
  if (is_mixed(cache->shape.format)) return KVQ_ERR_INVALID_ARG;   // needs the token classes
  if (!k_bf16 || !v_bf16 || !cu_seqlens_dev || max_len < 0) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(k_bf16) || !aligned16(v_bf16) || ((uintptr_t)cu_seqlens_dev & 3u)) return KVQ_ERR_ALIGNMENT;
  if (max_len > cache->shape.capacity) max_len = cache->shape.capacity;   // longer sequences are rejected on device
  return from_cuda(launch_prefill(*cache, k_bf16, v_bf16, cu_seqlens_dev, max_len, (cudaStream_t)stream));
}

kvq_status kvq_append_token(kvq_cache* cache, const void* k_new_bf16, const void* v_new_bf16,
                            kvq_stream_t stream) {
  kvq_status st = check_cache(cache);
  if (st != KVQ_OK) return st;
  if (is_mixed(cache->shape.format)) return KVQ_ERR_INVALID_ARG;
  if (!k_new_bf16 || !v_new_bf16) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(k_new_bf16) || !aligned16(v_new_bf16)) return KVQ_ERR_ALIGNMENT;
  if (is_token_cache(cache->shape.format) && cache->shape.num_kv_heads > 32) return KVQ_ERR_UNSUPPORTED;
  return from_cuda(launch_append(*cache, k_new_bf16, v_new_bf16, (cudaStream_t)stream));
}

kvq_status kvq_flush_group(kvq_cache* cache, kvq_stream_t stream) {
  kvq_status st = check_cache(cache);
  if (st != KVQ_OK) return st;
  return from_cuda(launch_flush(*cache, (cudaStream_t)stream));
}

kvq_status kvq_append_flush(kvq_cache* cache, const void* k_new_bf16, const void* v_new_bf16,
                            kvq_stream_t stream) {
  kvq_status st = check_cache(cache);
  if (st != KVQ_OK) return st;
  if (is_mixed(cache->shape.format)) return KVQ_ERR_INVALID_ARG;
  if (!k_new_bf16 || !v_new_bf16) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(k_new_bf16) || !aligned16(v_new_bf16)) return KVQ_ERR_ALIGNMENT;
  if (is_token_cache(cache->shape.format) && cache->shape.num_kv_heads > 32) return KVQ_ERR_UNSUPPORTED;
  return from_cuda(launch_append_flush(*cache, k_new_bf16, v_new_bf16, (cudaStream_t)stream));
}

kvq_status kvq_quantize_prefill_mixed(kvq_cache* cache, const void* k_bf16, const void* v_bf16,
                                      const uint8_t* token_class_dev, const int32_t* cu_seqlens_dev,
                                      int32_t max_len, kvq_stream_t stream) {
  kvq_status st = check_cache(cache);
  if (st != KVQ_OK) return st;
  if (!is_mixed(cache->shape.format)) return KVQ_ERR_INVALID_ARG;
  if (!k_bf16 || !v_bf16 || !cu_seqlens_dev || !token_class_dev || max_len < 0) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(k_bf16) || !aligned16(v_bf16) || ((uintptr_t)cu_seqlens_dev & 3u)) return KVQ_ERR_ALIGNMENT;
  if (max_len > cache->shape.capacity) max_len = cache->shape.capacity;
  return from_cuda(launch_prefill_mixed(*cache, k_bf16, v_bf16, token_class_dev, cu_seqlens_dev, max_len,
                                        (cudaStream_t)stream));
}

kvq_status kvq_append_token_mixed(kvq_cache* cache, const void* k_new_bf16, const void* v_new_bf16,
                                  const uint8_t* token_class_dev, kvq_stream_t stream) {
  kvq_status st = check_cache(cache);
  if (st != KVQ_OK) return st;
  if (!is_mixed(cache->shape.format)) return KVQ_ERR_INVALID_ARG;
  if (!k_new_bf16 || !v_new_bf16 || !token_class_dev) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(k_new_bf16) || !aligned16(v_new_bf16)) return KVQ_ERR_ALIGNMENT;
  return from_cuda(launch_append_mixed(*cache, k_new_bf16, v_new_bf16, token_class_dev, (cudaStream_t)stream));
}

kvq_status kvq_append_flush_mixed(kvq_cache* cache, const void* k_new_bf16, const void* v_new_bf16,
                                  const uint8_t* token_class_dev, kvq_stream_t stream) {
  kvq_status st = kvq_append_token_mixed(cache, k_new_bf16, v_new_bf16, token_class_dev, stream);
  if (st != KVQ_OK) return st;
  return from_cuda(launch_flush(*cache, (cudaStream_t)stream));
}

int32_t kvq_decode_default_splits(const kvq_cache* cache, int32_t max_len) {
  if (check_shape(cache ? &cache->shape : nullptr) != KVQ_OK) return 0;
  return decode_default_splits(cache->shape, max_len < 1 ? 1 : max_len);
}

size_t kvq_decode_workspace_bytes(const kvq_cache* cache, int32_t num_splits, int32_t max_len) {
  if (!cache || check_shape(&cache->shape) != KVQ_OK || num_splits < 0) return 0;
  if (num_splits == 0) num_splits = decode_default_splits(cache->shape, max_len < 1 ? 1 : max_len);
  return decode_workspace_bytes(cache->shape, num_splits);
}

}  // extern "C"

namespace kvq {
// Every check of the decode entry points except those on the workspace:
// the cache, q, out, lse, the scale and the split count (0 resolved to the
// library's choice, returned in *splits).  Shared by the entry point with a
// caller workspace and by the allocation-free one, so both return the same
// status for the same bad argument.
kvq_status decode_validate(const kvq_cache* cache, const void* q_bf16, const float* out, const float* lse,
                           float softmax_scale, int32_t num_splits, int32_t max_len, int32_t* splits) {
  kvq_status st = check_cache(cache);
  if (st != KVQ_OK) return st;
  if (!q_bf16 || !out || num_splits < 0 || max_len < 0) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(q_bf16) || !aligned16(out)) return KVQ_ERR_ALIGNMENT;
  if (lse && !aligned16(lse)) return KVQ_ERR_ALIGNMENT;
  if (!(softmax_scale == softmax_scale)) return KVQ_ERR_INVALID_ARG;
  if (num_splits == 0) num_splits = decode_default_splits(cache->shape, max_len < 1 ? 1 : max_len);
  if (num_splits < 1 || num_splits > 65535) return KVQ_ERR_INVALID_ARG;
  *splits = num_splits;
  return KVQ_OK;
}
}  // namespace kvq

extern "C" {

static kvq_status decode_checked(const kvq_cache* cache, const void* q_bf16, float* out, float* lse,
                                 float softmax_scale, void* workspace, size_t ws_bytes, int32_t num_splits,
                                 int32_t max_len, kvq_stream_t stream) {
  int32_t splits = 0;
  kvq_status st = decode_validate(cache, q_bf16, out, lse, softmax_scale, num_splits, max_len, &splits);
  if (st != KVQ_OK) return st;
  if (!workspace) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return KVQ_ERR_ALIGNMENT;
  if (ws_bytes < decode_workspace_bytes(cache->shape, splits)) return KVQ_ERR_WORKSPACE;
  return from_cuda(
      launch_decode(*cache, q_bf16, out, lse, softmax_scale, workspace, splits, (cudaStream_t)stream));
}

kvq_status kvq_decode_attention(const kvq_cache* cache, const void* q_bf16, float* out, float softmax_scale,
                                void* workspace, size_t ws_bytes, int32_t num_splits, int32_t max_len,
                                kvq_stream_t stream) {
  return decode_checked(cache, q_bf16, out, nullptr, softmax_scale, workspace, ws_bytes, num_splits, max_len, stream);
}

kvq_status kvq_decode_attention_lse(const kvq_cache* cache, const void* q_bf16, float* out, float* lse,
                                    float softmax_scale, void* workspace, size_t ws_bytes, int32_t num_splits,
                                    int32_t max_len, kvq_stream_t stream) {
  if (!lse) return KVQ_ERR_INVALID_ARG;
  return decode_checked(cache, q_bf16, out, lse, softmax_scale, workspace, ws_bytes, num_splits, max_len, stream);
}

kvq_status kvq_merge_partials(const float* outs, const float* lses, int32_t parts, int64_t rows, float* out,
                              float* lse_out, kvq_stream_t stream) {
  if (!outs || !lses || !out || parts < 1 || rows < 0) return KVQ_ERR_INVALID_ARG;
  if (rows > 0x7fffffffll) return KVQ_ERR_UNSUPPORTED;
  if (!aligned16(outs) || !aligned16(lses) || !aligned16(out) || (lse_out && !aligned16(lse_out)))
    return KVQ_ERR_ALIGNMENT;
  return from_cuda(launch_merge(outs, lses, parts, rows, out, lse_out, (cudaStream_t)stream));
}

kvq_status kvq_read_error(const kvq_cache* cache, uint32_t* flags, kvq_stream_t stream) {
  if (!cache || !flags || !cache->err_word) return KVQ_ERR_INVALID_ARG;
  uint32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, cache->err_word, sizeof(v), cudaMemcpyDeviceToHost, (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return KVQ_ERR_CUDA;
  *flags = v;
  return KVQ_OK;
}

const char* kvq_status_string(kvq_status status) {
  switch (status) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_INVALID_ARG: return "invalid argument";
    case KVQ_ERR_SHAPE: return "inconsistent shape";
    case KVQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case KVQ_ERR_ALIGNMENT: return "device pointer not 16-byte aligned";
    case KVQ_ERR_WORKSPACE: return "workspace too small";
    case KVQ_ERR_CUDA: return "CUDA launch failed";
  }
  return "unknown status";
}

const char* kvq_version(void) { return "0.1.0"; }

}  // extern "C"
