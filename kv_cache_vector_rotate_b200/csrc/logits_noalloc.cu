// tq_logits_noalloc: the fused-logits call for callers that cannot allocate
// device memory at the point of the call.
//
// Who needs it: a serving loop whose device memory is an arena carved up once
// at start-up, a host framework or plugin interface that owns every device
// allocation and hands an operator no workspace, or code that must not call
// cudaMalloc / cudaFree on its hot path because those calls can block or
// synchronize the device.  tq_logits needs a small workspace (the rotated,
// sketched query fragments); this entry point takes it from a file-scope
// device array instead of from the caller.
//
// Limits and rules (also stated in include/tq.h):
//  * the array holds kScratchBytes = 1 MiB on every device that loads the
//    library, for as long as the process lives;
//  * a request whose workspace would exceed it is rejected with TQ_EINVAL
//    before anything is launched;
//  * every call on a device shares the one array, so calls that overlap on
//    the GPU (different streams without ordering) race -- order them;
//  * nothing in the array needs clearing: each call overwrites all of the
//    scratch it reads;
//  * the first call on a device looks up the array's device address with
//    cudaGetSymbolAddress (with that device current) and keeps it.
// Nothing here allocates: no cudaMalloc, cudaFree or allocating library call.

#include <mutex>

#include "tq_internal.cuh"

namespace {

constexpr size_t kScratchBytes = size_t(1) << 20;
constexpr int kMaxDevices = 128;

// In host code this name is only a host-side stand-in for the device array;
// its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_logits_scratch[kScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

tq_status scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return tq::cuda_fail(e, "tq_logits_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return tq::fail(TQ_EUNSUPPORTED, "tq_logits_noalloc: device ordinal too large");
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_logits_scratch);   // the current device is `dev`
    if (e != cudaSuccess) return tq::cuda_fail(e, "tq_logits_noalloc: cudaGetSymbolAddress");
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return TQ_OK;
}

}  // namespace

extern "C" tq_status tq_logits_noalloc(const tq_codebook* cb, const tq_cache* cache, const void* q,
                                       tq_dtype dtype, int64_t batch, int32_t n_q_heads,
                                       const int32_t* ctx_len, int64_t max_ctx, float* out,
                                       int64_t out_stride, void* stream) {
  if (!cb || !cache) return tq::fail(TQ_EINVAL, "tq_logits_noalloc: codebook / cache is NULL");
  const size_t need = tq_logits_workspace_bytes(cb, batch, cache->n_kv_heads, n_q_heads);
  if (need > kScratchBytes)
    return tq::fail(TQ_EINVAL, "tq_logits_noalloc: this request needs " + std::to_string(need) +
                                   " bytes of scratch; the static scratch holds " +
                                   std::to_string(kScratchBytes));
  void* scratch = nullptr;
  tq_status s = scratch_address(&scratch);
  if (s != TQ_OK) return s;
  return tq_logits(cb, cache, q, dtype, batch, n_q_heads, ctx_len, max_ctx, out, out_stride, scratch,
                   kScratchBytes, stream);
}

extern "C" size_t tq_logits_noalloc_scratch_bytes(void) { return kScratchBytes; }
