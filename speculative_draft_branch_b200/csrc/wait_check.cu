// Device self-check of the failure-detection path: one thread waits, with the
// bounded mbarrier wait every tcgen05 kernel uses, on a barrier that is
// either arrived on first (the wait completes) or never arrived on (the wait
// gives up after its limit and reports through the plan's device-timeout
// word, as a kernel whose wait gave up does).  Nothing traps or faults; the
// thread returns either way and the context stays usable.
#include <cstdint>

#include "internal.cuh"
#include "sm100.cuh"

namespace ba {
namespace {

using namespace sm100;

// Bit of the device-timeout word this check sets (the attention kernels use
// the low bits for their own wait sites).
constexpr int kWaitCheckSite = 15;

__global__ void __launch_bounds__(1) wait_check_kernel(int *status, int arrive) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  mbar_fence_init();
  abort_flag = 0;
  if (arrive) mbar_arrive(b);
  // phase 0 completes on the single arrival; without it the wait runs out
  mbar_wait(b, 0, &abort_flag, status + 1, kWaitCheckSite);
}

}  // namespace
}  // namespace ba

extern "C" ba_status ba_wait_check(void *plan_ws, int32_t arrive, ba_stream_t stream) {
  using namespace ba;
  if (!plan_ws) {
    set_error("ba_wait_check: plan workspace is NULL");
    return BA_ERR_INVALID_ARG;
  }
  if (reinterpret_cast<uintptr_t>(plan_ws) % 16 != 0) {
    set_error("ba_wait_check: plan workspace must be 16-byte aligned");
    return BA_ERR_MISALIGNED;
  }
  if (arrive != 0 && arrive != 1) {
    set_error("ba_wait_check: arrive must be 0 or 1 (got %d)", arrive);
    return BA_ERR_INVALID_ARG;
  }
  // the status words sit at offset 0 of the plan workspace
  wait_check_kernel<<<1, 1, 0, (cudaStream_t)stream>>>(static_cast<int *>(plan_ws), arrive);
  count_launches(1);
  return cuda_check(cudaGetLastError(), "wait_check launch");
}
