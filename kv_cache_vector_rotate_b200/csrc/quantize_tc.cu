// Quantize-and-append on the tcgen05 tensor cores (placeholder until the
// tensor-core kernel lands: every call is served by the CUDA-core kernel).
#include "tq_internal.cuh"

namespace tq {

tq_status launch_quantize_tc(const tq_codebook*, const void*, tq_dtype, int64_t, int, int64_t,
                             const int32_t*, const CacheView&, cudaStream_t, bool* handled) {
  *handled = false;
  return TQ_OK;
}

}  // namespace tq
