// Attention kernels for head_dim 64 and 128 QJL bits (every code width and
// head map; see tq_attend.cuh).
#include "tq_attend.cuh"

namespace tq {

att::AttendFn attend_pick_64_128(int bw, int b_theta, int G, int mode, int* smem) {
  return att::attend_fn_dm<64, 128>(bw, b_theta, G, mode, smem);
}

}  // namespace tq
