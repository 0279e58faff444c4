// tcgen05 / TMEM / TMA branch-attention kernels for sm_100a.
#include "internal.cuh"

namespace ba {

bool sm100_available() { return false; }

ba_status launch_fwd_sm100(const AttnParams &, cudaStream_t) {
  set_error("tcgen05 forward kernel not built");
  return BA_ERR_UNSUPPORTED;
}

ba_status launch_bwd_sm100(const AttnParams &, cudaStream_t) {
  set_error("tcgen05 backward kernel not built");
  return BA_ERR_UNSUPPORTED;
}

}  // namespace ba
