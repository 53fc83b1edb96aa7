// Fused decode attention kernels for 1-bit keys (all value widths).
#include "attend_fused.cuh"

namespace tq {

tq_status launch_attend_fused_k1(const tqd::AttendParams& p, int vbits, int E, int F, int lines, cudaStream_t st) {
  return launch_attend_fused_kb<1>(p, vbits, E, F, lines, st);
}

}  // namespace tq
