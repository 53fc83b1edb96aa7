// Fused decode attention kernels for 2-bit keys (all value widths).
#include "attend_fused.cuh"

namespace tq {

tq_status launch_attend_fused_k2(const tqd::AttendParams& p, int vbits, int E, int F, int lines, cudaStream_t st) {
  return launch_attend_fused_kb<2>(p, vbits, E, F, lines, st);
}

}  // namespace tq
