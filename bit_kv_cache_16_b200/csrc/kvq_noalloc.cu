// Allocation-free decode entry point.
//
// kvq_decode_attention needs a caller-provided workspace for the per-split
// partial results.  Some callers cannot provide one: code that runs where
// cudaMalloc is forbidden or unsafe (inside a custom allocator's own
// callbacks, in a plugin whose host framework owns all device memory and
// exposes no allocation hook, or on a latency path that must never touch
// the driver's allocator).  kvq_decode_attention_noalloc serves them: it
// runs the same decode kernels, with the partials kept in a fixed array in
// the library's own device memory (kvq_noalloc_scratch below), and
// allocates nothing.
//
// Costs and rules of that array:
//  * Its size is fixed at KVQ_NOALLOC_SCRATCH_BYTES (8 MiB), and every GPU
//    on which the library is loaded holds it until the process exits.
//  * Every call on a device shares it and it keeps the last call's
//    contents.  Nothing in it needs to start at zero: the decode writes
//    every partial before the combine pass reads it.
//  * Calls whose work overlaps on the GPU (different streams, or different
//    host threads without ordering) race on the array and corrupt each
//    other's results; order such calls on one stream.
//  * The first call on each device looks up the array's device address
//    (cudaGetSymbolAddress) with that device current; make that first call
//    before capturing the stream into a CUDA graph.
#include <mutex>

#include "kvq_common.cuh"

namespace kvq {
size_t decode_workspace_bytes(const kvq_shape& s, int num_splits);
kvq_status decode_validate(const kvq_cache* cache, const void* q_bf16, const float* out, const float* lse,
                           float softmax_scale, int32_t num_splits, int32_t max_len, int32_t* splits);
}  // namespace kvq

namespace {

constexpr size_t kScratchBytes = 8u << 20;   // KVQ_NOALLOC_SCRATCH_BYTES
static_assert(kScratchBytes == (size_t)KVQ_NOALLOC_SCRATCH_BYTES, "header and library disagree");

// The split partials of kvq_decode_attention_noalloc.  In host code this
// name is only a handle for the runtime; its device address comes from
// cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char kvq_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once
// per device).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, kvq_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" kvq_status kvq_decode_attention_noalloc(const kvq_cache* cache, const void* q_bf16, float* out,
                                                   float softmax_scale, int32_t num_splits, int32_t max_len,
                                                   kvq_stream_t stream) {
  // The same checks, in the same order, as kvq_decode_attention (so a bad
  // argument gives the same status from both), then the scratch size.
  int32_t splits = 0;
  const kvq_status st = kvq::decode_validate(cache, q_bf16, out, nullptr, softmax_scale, num_splits, max_len, &splits);
  if (st != KVQ_OK) return st;
  const size_t need = kvq::decode_workspace_bytes(cache->shape, splits);
  if (need > kScratchBytes) return KVQ_ERR_WORKSPACE;   // the shape needs more than the fixed array holds
  void* ws = nullptr;
  if (scratch_address(&ws) != cudaSuccess) return KVQ_ERR_CUDA;
  return kvq_decode_attention(cache, q_bf16, out, softmax_scale, ws, kScratchBytes, splits, max_len, stream);
}
