// One training step on host buffers: upload, plan, forward, backward,
// download, with the copies overlapped against the kernels.
//
// The step needs every input before the forward and produces every output
// after the backward, so within one call only two overlaps exist: dO (used
// by the backward alone) uploads while the forward runs, and O / LSE
// (final after the forward) download while the backward runs.  The larger
// gain is across calls: uploads and downloads run on two library streams,
// so the upload of the next step (issued on another stream with its own
// staging area) proceeds while this step downloads, using both directions
// of the host link at once.
#include <mutex>

#include "internal.cuh"

namespace ba {
namespace {

constexpr int kMaxDevices = 64;

struct CopyStreams {
  cudaStream_t up = nullptr, down = nullptr;
  cudaEvent_t start = nullptr, in_fwd = nullptr, in_bwd = nullptr, fwd = nullptr,
              bwd = nullptr, done = nullptr;
};

std::mutex g_mu;
CopyStreams g_streams[kMaxDevices];

void destroy(CopyStreams &c) {
  for (cudaStream_t s : {c.up, c.down})
    if (s) cudaStreamDestroy(s);
  for (cudaEvent_t ev : {c.start, c.in_fwd, c.in_bwd, c.fwd, c.bwd, c.done})
    if (ev) cudaEventDestroy(ev);
}

// Created all at once on first use per device: a partly created set is
// destroyed and never published, so a later call retries from scratch.
ba_status copy_streams(int dev, CopyStreams **out) {
  CopyStreams &c = g_streams[dev];
  if (!c.up) {
    CopyStreams n;
    cudaError_t e = cudaStreamCreateWithFlags(&n.up, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&n.down, cudaStreamNonBlocking);
    cudaEvent_t *evs[6] = {&n.start, &n.in_fwd, &n.in_bwd, &n.fwd, &n.bwd, &n.done};
    for (cudaEvent_t *ev : evs)
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
    if (e != cudaSuccess) {
      destroy(n);
      return cuda_check(e, "creating the copy streams and events");
    }
    c = n;
  }
  *out = &c;
  return BA_OK;
}

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// Byte sizes of the tensors of a step, in staging order.
struct StepSizes {
  size_t plan, fwd, bwd, cu, anchor, depth;
  size_t q_m, kv_m, q_b, kv_b, lse_m, lse_b;
};

ba_status step_sizes(const ba_problem *p, StepSizes *s) {
  ba_status st = ba_workspace_size(p, &s->plan, &s->fwd, &s->bwd);
  if (st != BA_OK) return st;
  const size_t d = (size_t)p->head_dim;
  s->cu = 4 * ((size_t)p->n_seqs + 1);
  s->anchor = 4 * (size_t)p->n_branches;
  s->depth = 4 * (size_t)p->n_branches;
  s->q_m = 2 * (size_t)p->n_main * p->hq * d;
  s->kv_m = 2 * (size_t)p->n_main * p->hkv * d;
  s->q_b = 2 * (size_t)p->n_branch_tokens * p->hq * d;
  s->kv_b = 2 * (size_t)p->n_branch_tokens * p->hkv * d;
  s->lse_m = 4 * (size_t)p->n_main * p->hq;
  s->lse_b = 4 * (size_t)p->n_branch_tokens * p->hq;
  return BA_OK;
}

// Staging layout: plan, forward and backward workspaces, metadata, the eight
// inputs (q k v main, q k v branch, dO main, dO branch), O and LSE (main,
// branch), the six gradients (dq dk dv main, dq dk dv branch); every region
// starts on a 256-byte boundary.
size_t staging_bytes_for(const StepSizes &s) {
  const size_t parts[] = {s.plan, s.fwd, s.bwd, s.cu, s.anchor, s.depth,
                          s.q_m, s.kv_m, s.kv_m, s.q_b, s.kv_b, s.kv_b, s.q_m, s.q_b,
                          s.q_m, s.q_b, s.lse_m, s.lse_b,
                          s.q_m, s.kv_m, s.kv_m, s.q_b, s.kv_b, s.kv_b};
  size_t total = 0;
  for (size_t x : parts) total += up256(x);
  return total;
}

}  // namespace
}  // namespace ba

extern "C" ba_status ba_step_host_workspace_size(const ba_problem *p, size_t *bytes) {
  if (!p || !bytes) {
    ba::set_error("ba_step_host_workspace_size: null argument");
    return BA_ERR_INVALID_ARG;
  }
  ba::StepSizes s;
  ba_status st = ba::step_sizes(p, &s);
  if (st != BA_OK) return st;
  *bytes = ba::staging_bytes_for(s);
  return BA_OK;
}

extern "C" ba_status branch_attn_step_host(
    const ba_problem *p, void *staging, size_t staging_bytes, const void *q_m,
    const void *k_m, const void *v_m, const void *q_b, const void *k_b, const void *v_b,
    const void *do_m, const void *do_b, void *o_m, void *o_b, float *lse_m, float *lse_b,
    void *dq_m, void *dk_m, void *dv_m, void *dq_b, void *dk_b, void *dv_b,
    ba_stream_t stream_arg) {
  using namespace ba;
  if (!p || !staging) {
    set_error("branch_attn_step_host: null problem or staging");
    return BA_ERR_INVALID_ARG;
  }
  StepSizes s;
  ba_status st = step_sizes(p, &s);
  if (st != BA_OK) return st;
  const size_t need = staging_bytes_for(s);
  if (staging_bytes < need) {
    set_error("branch_attn_step_host: staging holds %zu bytes, the step needs %zu",
              staging_bytes, need);
    return BA_ERR_WORKSPACE_TOO_SMALL;
  }
  if (reinterpret_cast<uintptr_t>(staging) % 256 != 0) {
    set_error("branch_attn_step_host: staging must be 256-byte aligned");
    return BA_ERR_MISALIGNED;
  }
  const bool has_m = p->n_main > 0, has_b = p->n_branch_tokens > 0;
  if (!p->cu_seqlens || (p->n_branches > 0 && (!p->branch_anchor || !p->branch_depth)) ||
      (has_m && (!q_m || !k_m || !v_m || !do_m || !o_m || !lse_m || !dq_m || !dk_m || !dv_m)) ||
      (has_b && (!q_b || !k_b || !v_b || !do_b || !o_b || !lse_b || !dq_b || !dk_b || !dv_b))) {
    set_error("branch_attn_step_host: null host buffer for a non-empty tensor");
    return BA_ERR_INVALID_ARG;
  }

  // carve the staging area
  char *cur = static_cast<char *>(staging);
  auto take = [&](size_t bytes) {
    char *r = cur;
    cur += up256(bytes);
    return r;
  };
  void *plan_ws = take(s.plan), *fwd_ws = take(s.fwd), *bwd_ws = take(s.bwd);
  int32_t *d_cu = reinterpret_cast<int32_t *>(take(s.cu));
  int32_t *d_anchor = reinterpret_cast<int32_t *>(take(s.anchor));
  int32_t *d_depth = reinterpret_cast<int32_t *>(take(s.depth));
  char *d_q_m = take(s.q_m), *d_k_m = take(s.kv_m), *d_v_m = take(s.kv_m);
  char *d_q_b = take(s.q_b), *d_k_b = take(s.kv_b), *d_v_b = take(s.kv_b);
  char *d_do_m = take(s.q_m), *d_do_b = take(s.q_b);
  char *d_o_m = take(s.q_m), *d_o_b = take(s.q_b);
  float *d_lse_m = reinterpret_cast<float *>(take(s.lse_m));
  float *d_lse_b = reinterpret_cast<float *>(take(s.lse_b));
  char *d_dq_m = take(s.q_m), *d_dk_m = take(s.kv_m), *d_dv_m = take(s.kv_m);
  char *d_dq_b = take(s.q_b), *d_dk_b = take(s.kv_b), *d_dv_b = take(s.kv_b);

  ba_problem pd = *p;
  pd.cu_seqlens = d_cu;
  pd.branch_anchor = d_anchor;
  pd.branch_depth = d_depth;

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_check(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) {
    set_error("device %d outside the supported range", dev);
    return BA_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  CopyStreams *c = nullptr;
  if ((st = copy_streams(dev, &c)) != BA_OK) return st;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_arg);

  auto h2d = [&](void *dst, const void *src, size_t bytes) {
    return bytes ? cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, c->up) : cudaSuccess;
  };
  auto d2h = [&](void *dst, const void *src, size_t bytes) {
    return bytes ? cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToHost, c->down)
                 : cudaSuccess;
  };
  // Once a copy is queued it reads or writes the caller's host buffers.  An
  // error after that point waits for every copy already queued on the two
  // copy streams before returning, so the caller may reuse its buffers as soon
  // as the call has returned, whatever the outcome.
  bool queued = false;
  auto settle = [&](ba_status st_err) {
    if (queued) {
      cudaStreamSynchronize(c->up);
      cudaStreamSynchronize(c->down);
    }
    return st_err;
  };
#define BA_TRY(x)                                                  \
  do {                                                             \
    cudaError_t e_ = (x);                                          \
    if (e_ != cudaSuccess) return settle(cuda_check(e_, #x));      \
  } while (0)
#define BA_TRY_ST(x)                     \
  do {                                   \
    ba_status s_ = (x);                  \
    if (s_ != BA_OK) return settle(s_);  \
  } while (0)

  // uploads wait for the caller's earlier work on `stream` (which may still
  // read this staging area)
  BA_TRY(cudaEventRecord(c->start, stream));
  BA_TRY(cudaStreamWaitEvent(c->up, c->start, 0));
  queued = true;
  BA_TRY(h2d(d_cu, p->cu_seqlens, s.cu));
  BA_TRY(h2d(d_anchor, p->branch_anchor, s.anchor));
  BA_TRY(h2d(d_depth, p->branch_depth, s.depth));
  BA_TRY(h2d(d_q_m, q_m, s.q_m));
  BA_TRY(h2d(d_k_m, k_m, s.kv_m));
  BA_TRY(h2d(d_v_m, v_m, s.kv_m));
  BA_TRY(h2d(d_q_b, q_b, s.q_b));
  BA_TRY(h2d(d_k_b, k_b, s.kv_b));
  BA_TRY(h2d(d_v_b, v_b, s.kv_b));
  BA_TRY(cudaEventRecord(c->in_fwd, c->up));
  BA_TRY(h2d(d_do_m, do_m, s.q_m));
  BA_TRY(h2d(d_do_b, do_b, s.q_b));
  BA_TRY(cudaEventRecord(c->in_bwd, c->up));

  BA_TRY(cudaStreamWaitEvent(stream, c->in_fwd, 0));
  BA_TRY_ST(ba_plan(&pd, plan_ws, s.plan, stream_arg));
  BA_TRY_ST(branch_attn_fwd(&pd, plan_ws, fwd_ws, s.fwd, d_q_m, d_k_m, d_v_m, d_q_b, d_k_b,
                            d_v_b, d_o_m, d_o_b, d_lse_m, d_lse_b, stream_arg));
  BA_TRY(cudaEventRecord(c->fwd, stream));
  BA_TRY(cudaStreamWaitEvent(stream, c->in_bwd, 0));
  BA_TRY_ST(branch_attn_bwd(&pd, plan_ws, bwd_ws, s.bwd, d_q_m, d_k_m, d_v_m, d_q_b, d_k_b,
                            d_v_b, d_o_m, d_o_b, d_lse_m, d_lse_b, d_do_m, d_do_b, d_dq_m,
                            d_dk_m, d_dv_m, d_dq_b, d_dk_b, d_dv_b, stream_arg));
  BA_TRY(cudaEventRecord(c->bwd, stream));

  BA_TRY(cudaStreamWaitEvent(c->down, c->fwd, 0));
  BA_TRY(d2h(o_m, d_o_m, s.q_m));
  BA_TRY(d2h(o_b, d_o_b, s.q_b));
  BA_TRY(d2h(lse_m, d_lse_m, s.lse_m));
  BA_TRY(d2h(lse_b, d_lse_b, s.lse_b));
  BA_TRY(cudaStreamWaitEvent(c->down, c->bwd, 0));
  BA_TRY(d2h(dq_m, d_dq_m, s.q_m));
  BA_TRY(d2h(dk_m, d_dk_m, s.kv_m));
  BA_TRY(d2h(dv_m, d_dv_m, s.kv_m));
  BA_TRY(d2h(dq_b, d_dq_b, s.q_b));
  BA_TRY(d2h(dk_b, d_dk_b, s.kv_b));
  BA_TRY(d2h(dv_b, d_dv_b, s.kv_b));
  BA_TRY(cudaEventRecord(c->done, c->down));
  BA_TRY(cudaStreamWaitEvent(stream, c->done, 0));
#undef BA_TRY
#undef BA_TRY_ST
  return BA_OK;
}
