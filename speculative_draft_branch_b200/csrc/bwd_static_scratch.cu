// Backward pass for callers that cannot allocate device memory.
//
// Some host programs own every byte of device memory themselves, for example
// a serving or training process that reserves its whole HBM budget in its own
// pool at start-up, or a plugin whose host forbids allocation once it is
// running.  Such callers cannot cudaMalloc the backward workspace that
// branch_attn_bwd asks for.  This entry point runs the same backward with its
// scratch (D = rowsum(dO * O), the per-query records and the fp32 dQ
// accumulator) placed in a file-scope device array instead, so it allocates
// nothing.
//
// The array is a module global: every GPU that loads this library holds
// kStaticScratchBytes of it until the process exits.  All calls on a device
// share that one array and it keeps whatever the last call left in it; the
// backward rewrites D and the records on every call, and the fused backward
// zeroes its dQ accumulator before it sums into it, so nothing has to be
// cleared in between.  Two calls whose kernels overlap on the GPU (different
// streams without ordering) race on the array.
#include <mutex>

#include "internal.cuh"

namespace ba {
namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB per device

// Host code may only name this array to ask the runtime for its device
// address; the name itself is a host-side stand-in, not a device pointer.
static __device__ __align__(256) unsigned char g_bwd_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_addr[kMaxDevices] = {};
void *g_ctx[kMaxDevices] = {};  // the context g_addr[dev] was looked up in

using CtxGetCurrentFn = int (*)(void **);

// The driver's cuCtxGetCurrent, found through the runtime (the library links
// no driver library); null if the driver does not provide it.
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// Device address of the scratch array on the current device, looked up with
// that device current once per device context and cached.  The cache is keyed
// on the context as well as the device ordinal, so after a device reset (a new
// primary context) the address is looked up again instead of reusing one that
// belonged to the destroyed context.
ba_status scratch_address(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_check(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) {
    set_error("device %d outside the supported range for the static scratch", dev);
    return BA_ERR_UNSUPPORTED;
  }
  CtxGetCurrentFn get = ctx_get_current();
  if (!get) {
    set_error("cuCtxGetCurrent unavailable: cannot key the static scratch address on a context");
    return BA_ERR_CUDA;
  }
  void *ctx = nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (get(&ctx) != 0 || !ctx || !g_addr[dev] || g_ctx[dev] != ctx) {
    // the runtime call binds the device's primary context to this thread if
    // none is current yet; the context is read again after it
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_bwd_scratch);
    if (e != cudaSuccess) return cuda_check(e, "cudaGetSymbolAddress(static backward scratch)");
    if (get(&ctx) != 0 || !ctx) {
      set_error("no CUDA context is current after the static scratch lookup");
      return BA_ERR_CUDA;
    }
    g_addr[dev] = p;
    g_ctx[dev] = ctx;
  }
  *out = g_addr[dev];
  return BA_OK;
}

}  // namespace
}  // namespace ba

extern "C" ba_status branch_attn_bwd_static_scratch(
    const ba_problem *p, const void *plan_ws, const void *q_m, const void *k_m,
    const void *v_m, const void *q_b, const void *k_b, const void *v_b, const void *o_m,
    const void *o_b, const float *lse_m, const float *lse_b, const void *do_m,
    const void *do_b, void *dq_m, void *dk_m, void *dv_m, void *dq_b, void *dk_b, void *dv_b,
    ba_stream_t stream) {
  size_t need = 0;
  ba_status st = ba_workspace_size(p, nullptr, nullptr, &need);
  if (st != BA_OK) return st;
  if (need > ba::kStaticScratchBytes) {
    ba::set_error(
        "problem needs %zu bytes of backward scratch but the static scratch holds %zu bytes "
        "(at most about %zu fp32 dQ values); use branch_attn_bwd with a caller-provided "
        "workspace for larger problems",
        need, ba::kStaticScratchBytes, ba::kStaticScratchBytes / 4);
    return BA_ERR_WORKSPACE_TOO_SMALL;
  }
  void *scratch = nullptr;
  st = ba::scratch_address(&scratch);
  if (st != BA_OK) return st;
  return branch_attn_bwd(p, plan_ws, scratch, ba::kStaticScratchBytes, q_m, k_m, v_m, q_b, k_b,
                         v_b, o_m, o_b, lse_m, lse_b, do_m, do_b, dq_m, dk_m, dv_m, dq_b, dk_b,
                         dv_b, stream);
}
