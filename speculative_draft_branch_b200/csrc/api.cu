// C ABI of libbranch_attn: host-side validation, workspace layout and kernel
// dispatch.  The declarations and their contracts are in branch_attn.h.
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "internal.cuh"

namespace ba {

namespace {
thread_local char g_err[1024] = "";
std::atomic<int> g_family{0};
std::atomic<int64_t> g_launches{0};
std::atomic<void *> g_ev_start[3] = {nullptr, nullptr, nullptr};
std::atomic<void *> g_ev_stop[3] = {nullptr, nullptr, nullptr};

void record_event(int which, bool start, cudaStream_t s) {
  void *ev = start ? g_ev_start[which].load() : g_ev_stop[which].load();
  if (ev) cudaEventRecord((cudaEvent_t)ev, s);
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

constexpr int64_t kMaxRows = int64_t(1) << 28;  // main or branch tokens per call
}  // namespace

const char *set_error(const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return g_err;
}

void count_launches(int n) { g_launches.fetch_add(n); }

ba_status cuda_check(cudaError_t e, const char *what) {
  if (e == cudaSuccess) return BA_OK;
  set_error("%s: %s", what, cudaGetErrorString(e));
  return BA_ERR_CUDA;
}

namespace {

ba_status validate_problem(const ba_problem *p, bool need_index_ptrs) {
  if (!p) { set_error("problem is NULL"); return BA_ERR_INVALID_ARG; }
  if (p->n_seqs < 1) { set_error("n_seqs must be >= 1 (got %d)", p->n_seqs); return BA_ERR_INVALID_ARG; }
  if (p->n_main < 1 || p->n_main > kMaxRows) {
    set_error("n_main must be in [1, 2^28] (got %d)", p->n_main);
    return BA_ERR_INVALID_ARG;
  }
  if (p->n_seqs > p->n_main) {
    set_error("n_seqs (%d) exceeds n_main (%d)", p->n_seqs, p->n_main);
    return BA_ERR_INVALID_ARG;
  }
  if (p->n_branches < 0 || p->n_branch_tokens < 0 || p->n_branch_tokens > kMaxRows) {
    set_error("branch counts out of range (n_branches %d, n_branch_tokens %d)", p->n_branches,
              p->n_branch_tokens);
    return BA_ERR_INVALID_ARG;
  }
  if ((int64_t)p->n_branch_tokens < p->n_branches ||
      (int64_t)p->n_branch_tokens > (int64_t)kMaxDepth * p->n_branches) {
    set_error("n_branch_tokens (%d) must lie in [n_branches, 64 n_branches] (n_branches %d)",
              p->n_branch_tokens, p->n_branches);
    return BA_ERR_INVALID_ARG;
  }
  if (p->hq < 1 || p->hkv < 1 || p->hq % p->hkv != 0 || p->hq > 1024) {
    set_error("head counts invalid (hq %d, hkv %d): need hq %% hkv == 0", p->hq, p->hkv);
    return BA_ERR_INVALID_ARG;
  }
  if (p->head_dim != 64 && p->head_dim != 128) {
    set_error("head_dim %d not supported (64 or 128)", p->head_dim);
    return BA_ERR_UNSUPPORTED;
  }
  if (p->mask < BA_MASK_TTT_CAUSAL || p->mask > BA_MASK_BLOCK_CAUSAL) {
    set_error("unknown mask kind %d", p->mask);
    return BA_ERR_INVALID_ARG;
  }
  if (p->zigzag_C < 1 || p->zigzag_C > 64) {
    set_error("zigzag_C must be in [1, 64] (got %d)", p->zigzag_C);
    return BA_ERR_INVALID_ARG;
  }
  if (!(p->scale > 0.f) || !std::isfinite(p->scale)) {
    set_error("scale must be finite and > 0");
    return BA_ERR_INVALID_ARG;
  }
  if (need_index_ptrs) {
    if (!p->cu_seqlens || (p->n_branches > 0 && (!p->branch_anchor || !p->branch_depth))) {
      set_error("index array pointer is NULL");
      return BA_ERR_INVALID_ARG;
    }
    if (!aligned(p->cu_seqlens, 4) || !aligned(p->branch_anchor, 4) ||
        !aligned(p->branch_depth, 4)) {
      set_error("index arrays must be 4-byte aligned");
      return BA_ERR_MISALIGNED;
    }
  }
  return BA_OK;
}

void plan_layout(const ba_problem &p, ba_plan_layout *L) {
  std::memset(L, 0, sizeof(*L));
  L->n_qtiles_main = (int32_t)cdiv64(p.n_main, kTileM);
  L->n_qtiles_branch = (int32_t)cdiv64(p.n_branch_tokens, kTileM);
  L->n_kv_main = (int32_t)cdiv64(p.n_main, kTileN);
  L->n_kv_branch = (int32_t)cdiv64(p.n_branch_tokens, kTileN);
  const int64_t n_qt = L->n_qtiles_main + L->n_qtiles_branch;
  const int64_t n_kv = L->n_kv_main + L->n_kv_branch;
  const int64_t rows = (int64_t)p.n_main + p.n_branch_tokens;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  L->off_status = take(16);
  L->off_cu_branch = take(4 * ((size_t)p.n_branches + 1));
  L->off_branch_seq = take(4 * (size_t)p.n_branches);
  L->off_row_iv = take(16 * (size_t)rows);
  L->off_qtile = take(24 * (size_t)n_qt);
  L->off_kv_main = take(16 * (size_t)L->n_kv_main);
  L->off_kv_branch = take(8 * (size_t)L->n_kv_branch);
  L->off_fwd_order = take(4 * (size_t)n_qt);
  L->off_bwd_order = take(4 * (size_t)n_kv);
  L->off_fwd_cost = take(4 * (size_t)n_qt);
  L->off_bwd_cost = take(4 * (size_t)n_kv);
  L->off_zz_tiles = take(p.zigzag_C > 1 ? 16 * (size_t)p.zigzag_C * n_qt : 0);
  L->off_key_iv = take(16 * (size_t)rows);
  L->off_bwd_prefix = take(4 * (size_t)n_kv);
  L->total_bytes = off;
}

PlanView plan_view(const ba_plan_layout &L, const void *ws) {
  char *b = reinterpret_cast<char *>(const_cast<void *>(ws));
  PlanView v;
  v.status = reinterpret_cast<int32_t *>(b + L.off_status);
  v.cu_branch = reinterpret_cast<int32_t *>(b + L.off_cu_branch);
  v.branch_seq = reinterpret_cast<int32_t *>(b + L.off_branch_seq);
  v.row_iv = reinterpret_cast<int32_t *>(b + L.off_row_iv);
  v.qtile = reinterpret_cast<int32_t *>(b + L.off_qtile);
  v.kv_main = reinterpret_cast<int32_t *>(b + L.off_kv_main);
  v.kv_branch = reinterpret_cast<int32_t *>(b + L.off_kv_branch);
  v.fwd_order = reinterpret_cast<int32_t *>(b + L.off_fwd_order);
  v.bwd_order = reinterpret_cast<int32_t *>(b + L.off_bwd_order);
  v.fwd_cost = reinterpret_cast<int32_t *>(b + L.off_fwd_cost);
  v.bwd_cost = reinterpret_cast<int32_t *>(b + L.off_bwd_cost);
  v.zz_tiles = reinterpret_cast<int32_t *>(b + L.off_zz_tiles);
  v.key_iv = reinterpret_cast<int32_t *>(b + L.off_key_iv);
  v.bwd_prefix = reinterpret_cast<int32_t *>(b + L.off_bwd_prefix);
  return v;
}

size_t fwd_ws_bytes(const ba_problem &p) {
  if (p.zigzag_C <= 1) return 0;
  const size_t rows = (size_t)p.n_main + p.n_branch_tokens;
  return align_up(4 * rows * p.hq * p.head_dim, 256) + align_up(4 * rows * p.hq, 256);
}

size_t rows_padded(const ba_problem &p) {
  return align_up((size_t)p.n_main, 128) + align_up((size_t)p.n_branch_tokens, 128);
}

// Backward workspace, three regions at 256-byte offsets:
//   D        [Hq, rows] fp32, rowsum(dO * O)
//   records  [2][Hq][rows padded to 128 per kind] float4 {LSE log2 e, D, key lo, key hi}
//   dQ acc   [rows, Hq, d] fp32 (the fused backward's dQ accumulator)
size_t bwd_d_bytes(const ba_problem &p) {
  return align_up(4 * ((size_t)p.n_main + p.n_branch_tokens) * p.hq, 256);
}
size_t bwd_rec_bytes(const ba_problem &p) { return align_up(8 * rows_padded(p) * p.hq, 256); }
size_t bwd_ws_bytes(const ba_problem &p) {
  const size_t rows = (size_t)p.n_main + p.n_branch_tokens;
  return bwd_d_bytes(p) + bwd_rec_bytes(p) + align_up(4 * rows * p.hq * p.head_dim, 256);
}

AttnParams make_params(const ba_problem &p, const ba_plan_layout &L, const void *plan_ws) {
  AttnParams a;
  std::memset(&a, 0, sizeof(a));
  a.plan = plan_view(L, plan_ws);
  a.cu_seqlens = p.cu_seqlens;
  a.n_main = p.n_main;
  a.n_bt = p.n_branch_tokens;
  a.n_seqs = p.n_seqs;
  a.hq = p.hq;
  a.hkv = p.hkv;
  a.head_dim = p.head_dim;
  a.mask = p.mask;
  a.n_qt_main = L.n_qtiles_main;
  a.n_qt = L.n_qtiles_main + L.n_qtiles_branch;
  a.n_kt = L.n_kv_main;
  a.n_bkt = L.n_kv_branch;
  a.scale = p.scale;
  a.scale_log2 = p.scale * 1.4426950408889634f;
  a.zz_step = -1;
  a.zz_C = p.zigzag_C;
  a.ring = 0;
  a.n_keys_m = p.n_main;
  {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    a.n_sms = sms > 0 ? sms : 148;
  }
  return a;
}

ba_status check_tensor(const void *ptr, bool needed, const char *name) {
  if (!needed) return BA_OK;
  if (!ptr) { set_error("%s is NULL", name); return BA_ERR_INVALID_ARG; }
  if (!aligned(ptr, 16)) { set_error("%s is not 16-byte aligned", name); return BA_ERR_MISALIGNED; }
  return BA_OK;
}

ba_status check_f32(const void *ptr, bool needed, const char *name) {
  if (!needed) return BA_OK;
  if (!ptr) { set_error("%s is NULL", name); return BA_ERR_INVALID_ARG; }
  if (!aligned(ptr, 4)) { set_error("%s is not 4-byte aligned", name); return BA_ERR_MISALIGNED; }
  return BA_OK;
}

ba_status check_plan_ws(const void *plan_ws) {
  if (!plan_ws) { set_error("plan workspace is NULL"); return BA_ERR_INVALID_ARG; }
  if (!aligned(plan_ws, 16)) { set_error("plan workspace must be 16-byte aligned"); return BA_ERR_MISALIGNED; }
  return BA_OK;
}


#define BA_TRY(expr)                   \
  do {                                 \
    ba_status _s = (expr);             \
    if (_s != BA_OK) return _s;        \
  } while (0)

}  // namespace
}  // namespace ba

using namespace ba;

extern "C" {

ba_status ba_workspace_size(const ba_problem *p, size_t *plan_bytes, size_t *fwd_bytes,
                            size_t *bwd_bytes) {
  BA_TRY(validate_problem(p, false));
  ba_plan_layout L;
  plan_layout(*p, &L);
  if (plan_bytes) *plan_bytes = L.total_bytes;
  if (fwd_bytes) *fwd_bytes = fwd_ws_bytes(*p);
  if (bwd_bytes) *bwd_bytes = bwd_ws_bytes(*p);
  return BA_OK;
}

ba_status ba_plan_layout_query(const ba_problem *p, ba_plan_layout *out) {
  BA_TRY(validate_problem(p, false));
  if (!out) { set_error("out is NULL"); return BA_ERR_INVALID_ARG; }
  plan_layout(*p, out);
  return BA_OK;
}

ba_status ba_plan(const ba_problem *p, void *plan_ws, size_t plan_bytes, ba_stream_t stream) {
  BA_TRY(validate_problem(p, true));
  BA_TRY(check_plan_ws(plan_ws));
  ba_plan_layout L;
  plan_layout(*p, &L);
  if (plan_bytes < L.total_bytes) {
    set_error("plan workspace too small: %zu < %zu bytes", plan_bytes, L.total_bytes);
    return BA_ERR_WORKSPACE_TOO_SMALL;
  }
  return launch_plan(*p, L, plan_view(L, plan_ws), (cudaStream_t)stream);
}

ba_status ba_plan_status(const void *plan_ws, ba_stream_t stream, int32_t *status_out) {
  BA_TRY(check_plan_ws(plan_ws));
  int32_t words[2] = {0, 0};
  BA_TRY(cuda_check(cudaMemcpyAsync(words, plan_ws, sizeof(words), cudaMemcpyDeviceToHost,
                                    (cudaStream_t)stream),
                    "ba_plan_status copy"));
  BA_TRY(cuda_check(cudaStreamSynchronize((cudaStream_t)stream), "ba_plan_status sync"));
  if (status_out) *status_out = words[0];
  if (words[0] != 0) {
    set_error("plan content checks failed (status 0x%x)", words[0]);
    return BA_ERR_BAD_METADATA;
  }
  if (words[1] != 0) {
    set_error("a bounded device-side wait gave up (sites 0x%x)", words[1]);
    return BA_ERR_DEVICE_TIMEOUT;
  }
  return BA_OK;
}

ba_status branch_attn_fwd(const ba_problem *p, const void *plan_ws, void *fwd_ws,
                          size_t fwd_bytes, const void *q_m, const void *k_m, const void *v_m,
                          const void *q_b, const void *k_b, const void *v_b, void *o_m,
                          void *o_b, float *lse_m, float *lse_b, ba_stream_t stream) {
  BA_TRY(validate_problem(p, true));
  BA_TRY(check_plan_ws(plan_ws));
  const bool br = p->n_branch_tokens > 0;
  BA_TRY(check_tensor(q_m, true, "q_m"));
  BA_TRY(check_tensor(k_m, true, "k_m"));
  BA_TRY(check_tensor(v_m, true, "v_m"));
  BA_TRY(check_tensor(o_m, true, "o_m"));
  BA_TRY(check_tensor(q_b, br, "q_b"));
  BA_TRY(check_tensor(k_b, br, "k_b"));
  BA_TRY(check_tensor(v_b, br, "v_b"));
  BA_TRY(check_tensor(o_b, br, "o_b"));
  BA_TRY(check_f32(lse_m, true, "lse_m"));
  BA_TRY(check_f32(lse_b, br, "lse_b"));
  const size_t need = fwd_ws_bytes(*p);
  if (need > 0) {
    BA_TRY(check_tensor(fwd_ws, true, "fwd_ws"));
    if (fwd_bytes < need) {
      set_error("forward workspace too small: %zu < %zu bytes", fwd_bytes, need);
      return BA_ERR_WORKSPACE_TOO_SMALL;
    }
  }
  ba_plan_layout L;
  plan_layout(*p, &L);
  AttnParams a = make_params(*p, L, plan_ws);
  a.q_m = (const __nv_bfloat16 *)q_m; a.k_m = (const __nv_bfloat16 *)k_m;
  a.v_m = (const __nv_bfloat16 *)v_m; a.q_b = (const __nv_bfloat16 *)q_b;
  a.k_b = (const __nv_bfloat16 *)k_b; a.v_b = (const __nv_bfloat16 *)v_b;
  a.o_m = (__nv_bfloat16 *)o_m; a.o_b = (__nv_bfloat16 *)o_b;
  a.lse_m = lse_m; a.lse_b = lse_b;
  cudaStream_t s = (cudaStream_t)stream;
  auto launch = [&](const AttnParams &x) { return launch_fwd_sm100(x, s); };
  if (p->zigzag_C <= 1) {
    record_event(0, true, s);
    ba_status st = launch(a);
    record_event(0, false, s);
    return st;
  }
  const size_t rows = (size_t)p->n_main + p->n_branch_tokens;
  a.zz_o = reinterpret_cast<float *>(fwd_ws);
  a.zz_lse = reinterpret_cast<float *>(reinterpret_cast<char *>(fwd_ws) +
                                       align_up(4 * rows * p->hq * p->head_dim, 256));
  // ring steps 0..C-1 over the main keys, then the rank-local branch pass,
  // each merged into the running (O, l) by the LSE rule
  record_event(0, true, s);
  for (int step = 0; step <= p->zigzag_C; ++step) {
    a.zz_step = step;
    BA_TRY(launch(a));
  }
  record_event(0, false, s);
  return BA_OK;
}

ba_status branch_attn_bwd(const ba_problem *p, const void *plan_ws, void *bwd_ws,
                          size_t bwd_bytes, const void *q_m, const void *k_m, const void *v_m,
                          const void *q_b, const void *k_b, const void *v_b, const void *o_m,
                          const void *o_b, const float *lse_m, const float *lse_b,
                          const void *do_m, const void *do_b, void *dq_m, void *dk_m,
                          void *dv_m, void *dq_b, void *dk_b, void *dv_b, ba_stream_t stream) {
  BA_TRY(validate_problem(p, true));
  BA_TRY(check_plan_ws(plan_ws));
  const bool br = p->n_branch_tokens > 0;
  const void *need_main[] = {q_m, k_m, v_m, o_m, do_m, dq_m, dk_m, dv_m};
  const char *names_main[] = {"q_m", "k_m", "v_m", "o_m", "do_m", "dq_m", "dk_m", "dv_m"};
  for (int i = 0; i < 8; ++i) BA_TRY(check_tensor(need_main[i], true, names_main[i]));
  const void *need_br[] = {q_b, k_b, v_b, o_b, do_b, dq_b, dk_b, dv_b};
  const char *names_br[] = {"q_b", "k_b", "v_b", "o_b", "do_b", "dq_b", "dk_b", "dv_b"};
  for (int i = 0; i < 8; ++i) BA_TRY(check_tensor(need_br[i], br, names_br[i]));
  BA_TRY(check_f32(lse_m, true, "lse_m"));
  BA_TRY(check_f32(lse_b, br, "lse_b"));
  BA_TRY(check_tensor(bwd_ws, true, "bwd_ws"));
  const size_t need = bwd_ws_bytes(*p);
  if (bwd_bytes < need) {
    set_error("backward workspace too small: %zu < %zu bytes", bwd_bytes, need);
    return BA_ERR_WORKSPACE_TOO_SMALL;
  }
  ba_plan_layout L;
  plan_layout(*p, &L);
  AttnParams a = make_params(*p, L, plan_ws);
  a.q_m = (const __nv_bfloat16 *)q_m; a.k_m = (const __nv_bfloat16 *)k_m;
  a.v_m = (const __nv_bfloat16 *)v_m; a.q_b = (const __nv_bfloat16 *)q_b;
  a.k_b = (const __nv_bfloat16 *)k_b; a.v_b = (const __nv_bfloat16 *)v_b;
  a.o_m = (__nv_bfloat16 *)o_m; a.o_b = (__nv_bfloat16 *)o_b;
  a.lse_m = const_cast<float *>(lse_m); a.lse_b = const_cast<float *>(lse_b);
  a.do_m = (const __nv_bfloat16 *)do_m; a.do_b = (const __nv_bfloat16 *)do_b;
  a.dk_m = (__nv_bfloat16 *)dk_m; a.dv_m = (__nv_bfloat16 *)dv_m;
  a.dk_b = (__nv_bfloat16 *)dk_b; a.dv_b = (__nv_bfloat16 *)dv_b;
  char *ws = reinterpret_cast<char *>(bwd_ws);
  a.d_all = reinterpret_cast<const float *>(ws);
  a.rec = reinterpret_cast<float *>(ws + bwd_d_bytes(*p));
  a.dq_acc = reinterpret_cast<float *>(ws + bwd_d_bytes(*p) + bwd_rec_bytes(*p));
  a.n_main_pad = (int32_t)align_up((size_t)p->n_main, 128);
  a.rows_pad = (int32_t)rows_padded(*p);
  a.dq_out_m = (__nv_bfloat16 *)dq_m;
  a.dq_out_b = (__nv_bfloat16 *)dq_b;
  cudaStream_t s = (cudaStream_t)stream;
  // family 0: the split backward (dK/dV kernel + dQ kernel, both writing bf16
  // directly; deterministic); family 1: one fused kernel accumulating dQ in
  // fp32 (the preprocess zeroes the accumulator, a last pass converts it)
  const bool fused = g_family.load() == 1 && sm100_fused_bwd_available();
  a.zero_dq_acc = fused ? 1 : 0;
  record_event(2, true, s);
  BA_TRY(launch_bwd_preprocess(a, s));
  record_event(2, false, s);
  record_event(1, true, s);
  BA_TRY(fused ? launch_bwd_fused_sm100(a, s) : launch_bwd_sm100(a, s));
  if (fused) BA_TRY(launch_dq_convert(a, (__nv_bfloat16 *)dq_m, (__nv_bfloat16 *)dq_b, s));
  record_event(1, false, s);
  return BA_OK;
}

// ---- zigzag ring across ranks ---------------------------------------------

ba_status ba_zigzag_shard(const int32_t *cu, int32_t n_seqs, const int32_t *anchor,
                          const int32_t *depth, int32_t n_branches, int32_t C, int32_t shard,
                          int32_t *n_main_local, int32_t *n_branches_local,
                          int32_t *n_branch_tokens_local, int32_t *cu_local,
                          int32_t *anchor_local, int32_t *depth_local, int32_t *main_rows,
                          int32_t *branch_rows) {
  if (!cu || n_seqs < 1 || n_branches < 0 || (n_branches > 0 && (!anchor || !depth))) {
    set_error("ba_zigzag_shard: cu_seqlens, anchors and depths are required (host arrays)");
    return BA_ERR_INVALID_ARG;
  }
  if (C < 1 || C > 64 || shard < 0 || shard >= C) {
    set_error("ba_zigzag_shard: need 1 <= C <= 64 and 0 <= shard < C (C %d, shard %d)", C, shard);
    return BA_ERR_INVALID_ARG;
  }
  if (!n_main_local || !n_branches_local || !n_branch_tokens_local) {
    set_error("ba_zigzag_shard: the three count pointers are required");
    return BA_ERR_INVALID_ARG;
  }
  if (cu[0] != 0) {
    set_error("ba_zigzag_shard: cu_seqlens[0] must be 0");
    return BA_ERR_INVALID_ARG;
  }
  for (int s = 0; s < n_seqs; ++s) {
    const int64_t L = (int64_t)cu[s + 1] - cu[s];
    if (L < 2 * C) {
      set_error("ba_zigzag_shard: sequence %d holds %lld tokens, fewer than 2C = %d", s,
                (long long)L, 2 * C);
      return L < 1 ? BA_ERR_INVALID_ARG : BA_ERR_UNSUPPORTED;
    }
  }
  // chunk k of sequence s: [cu[s] + floor(kL/2C), cu[s] + floor((k+1)L/2C))
  auto chunk = [&](int s, int k, int64_t *a, int64_t *b) {
    const int64_t L = (int64_t)cu[s + 1] - cu[s];
    *a = cu[s] + (k * L) / (2 * C);
    *b = cu[s] + ((k + 1) * L) / (2 * C);
  };
  int64_t nm = 0, nb = 0, nbt = 0;
  if (cu_local) cu_local[0] = 0;
  int b = 0;          // branches are sorted by anchor
  int64_t brow = 0;   // first branch row of branch b
  for (int s = 0; s < n_seqs; ++s) {
    for (int piece = 0; piece < 2; ++piece) {
      int64_t a0, a1;
      chunk(s, piece == 0 ? shard : 2 * C - 1 - shard, &a0, &a1);
      // main rows a0..a1-1 become local rows nm .. nm + (a1 - a0) - 1
      while (b < n_branches && anchor[b] < a0) brow += depth[b++];
      int bb = b;
      int64_t bbrow = brow;
      while (bb < n_branches && anchor[bb] < a1) {
        if (anchor[bb] < a0) {  // anchors must be sorted
          set_error("ba_zigzag_shard: branch anchors must be non-decreasing");
          return BA_ERR_INVALID_ARG;
        }
        if (anchor_local) anchor_local[nb] = (int32_t)(nm + (anchor[bb] - a0));
        if (depth_local) depth_local[nb] = depth[bb];
        for (int j = 0; j < depth[bb]; ++j)
          if (branch_rows) branch_rows[nbt + j] = (int32_t)(bbrow + j);
        nbt += depth[bb];
        bbrow += depth[bb];
        ++nb;
        ++bb;
      }
      if (main_rows)
        for (int64_t r = a0; r < a1; ++r) main_rows[nm + (r - a0)] = (int32_t)r;
      nm += a1 - a0;
    }
    if (cu_local) cu_local[s + 1] = (int32_t)nm;
  }
  *n_main_local = (int32_t)nm;
  *n_branches_local = (int32_t)nb;
  *n_branch_tokens_local = (int32_t)nbt;
  return BA_OK;
}

ba_status ba_ring_workspace_size(const ba_problem *local, int32_t C, size_t *plan_bytes,
                                 size_t *acc_bytes) {
  BA_TRY(validate_problem(local, false));
  if (C < 1 || C > 64) {
    set_error("ring size C must be in [1, 64] (got %d)", C);
    return BA_ERR_INVALID_ARG;
  }
  ba_plan_layout L;
  plan_layout(*local, &L);
  const size_t rows = (size_t)local->n_main + local->n_branch_tokens;
  if (plan_bytes) *plan_bytes = L.total_bytes;
  if (acc_bytes)
    *acc_bytes = align_up(4 * rows * local->hq * local->head_dim, 256) +
                 align_up(4 * rows * local->hq, 256);
  return BA_OK;
}

namespace {
ba_status check_ring(const ba_problem *local, int32_t C, int32_t step, bool allow_last) {
  BA_TRY(validate_problem(local, true));
  if (local->zigzag_C != 1) {
    set_error("the shard-local problem must have zigzag_C = 1 (the ring size is passed apart)");
    return BA_ERR_INVALID_ARG;
  }
  if (C < 1 || C > 64 || step < 0 || step > (allow_last ? C : C - 1)) {
    set_error("ring: need 1 <= C <= 64 and 0 <= step < C (C %d, step %d)", C, step);
    return BA_ERR_INVALID_ARG;
  }
  return BA_OK;
}

ba_status ring_acc(const ba_problem *local, int32_t C, void *acc_ws, size_t acc_bytes,
                   AttnParams *a) {
  size_t need = 0;
  BA_TRY(ba_ring_workspace_size(local, C, nullptr, &need));
  BA_TRY(check_tensor(acc_ws, true, "acc_ws"));
  if (acc_bytes < need) {
    set_error("ring accumulator too small: %zu < %zu bytes", acc_bytes, need);
    return BA_ERR_WORKSPACE_TOO_SMALL;
  }
  const size_t rows = (size_t)local->n_main + local->n_branch_tokens;
  a->zz_o = reinterpret_cast<float *>(acc_ws);
  a->zz_lse = reinterpret_cast<float *>(reinterpret_cast<char *>(acc_ws) +
                                        align_up(4 * rows * local->hq * local->head_dim, 256));
  return BA_OK;
}
}  // namespace

ba_status ba_ring_plan(const ba_problem *local, int32_t C, int32_t shard, int32_t step,
                       const int32_t *cu_global, const int32_t *cu_visit, void *plan_ws,
                       size_t plan_bytes, ba_stream_t stream) {
  BA_TRY(check_ring(local, C, step, false));
  if (shard < 0 || shard >= C) {
    set_error("ring: shard %d outside [0, %d)", shard, C);
    return BA_ERR_INVALID_ARG;
  }
  BA_TRY(check_plan_ws(plan_ws));
  ba_plan_layout L;
  plan_layout(*local, &L);
  if (plan_bytes < L.total_bytes) {
    set_error("plan workspace too small: %zu < %zu bytes", plan_bytes, L.total_bytes);
    return BA_ERR_WORKSPACE_TOO_SMALL;
  }
  if (step == 0) return launch_plan(*local, L, plan_view(L, plan_ws), (cudaStream_t)stream);
  if (!cu_global || !cu_visit || !aligned(cu_global, 4) || !aligned(cu_visit, 4)) {
    set_error("ring plan: cu_global and cu_visit must be 4-byte aligned device arrays");
    return cu_global && cu_visit ? BA_ERR_MISALIGNED : BA_ERR_INVALID_ARG;
  }
  const int j = ((shard - step) % C + C) % C;
  return launch_ring_plan(*local, L, plan_view(L, plan_ws), cu_global, cu_visit, C, shard, j,
                          (cudaStream_t)stream);
}

ba_status branch_attn_ring_step(const ba_problem *local, int32_t C, int32_t step,
                                const void *plan_ws, void *acc_ws, size_t acc_bytes,
                                int32_t n_main_visit, const void *q_m, const void *k_m_visit,
                                const void *v_m_visit, const void *q_b, ba_stream_t stream) {
  BA_TRY(check_ring(local, C, step, false));
  BA_TRY(check_plan_ws(plan_ws));
  if (n_main_visit < 1 || n_main_visit > kMaxRows) {
    set_error("n_main_visit must be in [1, 2^28] (got %d)", n_main_visit);
    return BA_ERR_INVALID_ARG;
  }
  const bool br = local->n_branch_tokens > 0;
  BA_TRY(check_tensor(q_m, true, "q_m"));
  BA_TRY(check_tensor(k_m_visit, true, "k_m_visit"));
  BA_TRY(check_tensor(v_m_visit, true, "v_m_visit"));
  BA_TRY(check_tensor(q_b, br, "q_b"));
  ba_plan_layout L;
  plan_layout(*local, &L);
  AttnParams a = make_params(*local, L, plan_ws);
  BA_TRY(ring_acc(local, C, acc_ws, acc_bytes, &a));
  a.ring = 1;
  a.zz_step = step;
  a.zz_C = C;
  a.n_keys_m = n_main_visit;
  a.q_m = (const __nv_bfloat16 *)q_m;
  a.k_m = (const __nv_bfloat16 *)k_m_visit;
  a.v_m = (const __nv_bfloat16 *)v_m_visit;
  a.q_b = (const __nv_bfloat16 *)q_b;
  cudaStream_t s = (cudaStream_t)stream;
  record_event(0, true, s);
  ba_status st = launch_fwd_sm100(a, s);
  record_event(0, false, s);
  return st;
}

ba_status branch_attn_ring_finish(const ba_problem *local, int32_t C, const void *plan_ws,
                                  void *acc_ws, size_t acc_bytes, const void *q_m,
                                  const void *q_b, const void *k_b, const void *v_b, void *o_m,
                                  void *o_b, float *lse_m, float *lse_b, ba_stream_t stream) {
  BA_TRY(check_ring(local, C, C, true));
  BA_TRY(check_plan_ws(plan_ws));
  const bool br = local->n_branch_tokens > 0;
  BA_TRY(check_tensor(q_m, true, "q_m"));
  BA_TRY(check_tensor(o_m, true, "o_m"));
  BA_TRY(check_tensor(q_b, br, "q_b"));
  BA_TRY(check_tensor(k_b, br, "k_b"));
  BA_TRY(check_tensor(v_b, br, "v_b"));
  BA_TRY(check_tensor(o_b, br, "o_b"));
  BA_TRY(check_f32(lse_m, true, "lse_m"));
  BA_TRY(check_f32(lse_b, br, "lse_b"));
  ba_plan_layout L;
  plan_layout(*local, &L);
  AttnParams a = make_params(*local, L, plan_ws);
  BA_TRY(ring_acc(local, C, acc_ws, acc_bytes, &a));
  a.ring = 1;
  a.zz_step = C;
  a.zz_C = C;
  a.q_m = (const __nv_bfloat16 *)q_m;
  a.q_b = (const __nv_bfloat16 *)q_b;
  a.k_b = (const __nv_bfloat16 *)k_b;
  a.v_b = (const __nv_bfloat16 *)v_b;
  a.o_m = (__nv_bfloat16 *)o_m;
  a.o_b = (__nv_bfloat16 *)o_b;
  a.lse_m = lse_m;
  a.lse_b = lse_b;
  cudaStream_t s = (cudaStream_t)stream;
  record_event(0, true, s);
  ba_status st = launch_fwd_sm100(a, s);
  record_event(0, false, s);
  return st;
}

ba_status lse_merge(int64_t rows, int32_t heads, int32_t head_dim, int32_t o_is_fp32,
                    const void *o_a, const float *lse_a, const void *o_b, const float *lse_b,
                    void *o_out, float *lse_out, ba_stream_t stream) {
  if (rows < 0 || heads < 1) {
    set_error("lse_merge: rows must be >= 0 and heads >= 1 (rows %lld, heads %d)",
              (long long)rows, heads);
    return BA_ERR_INVALID_ARG;
  }
  if (head_dim != 64 && head_dim != 128) {
    set_error("lse_merge: head_dim %d not supported (64 or 128)", head_dim);
    return BA_ERR_UNSUPPORTED;
  }
  if (rows == 0) return BA_OK;
  BA_TRY(check_tensor(o_a, true, "o_a"));
  BA_TRY(check_tensor(o_b, true, "o_b"));
  BA_TRY(check_tensor(o_out, true, "o_out"));
  BA_TRY(check_f32(lse_a, true, "lse_a"));
  BA_TRY(check_f32(lse_b, true, "lse_b"));
  BA_TRY(check_f32(lse_out, true, "lse_out"));
  return launch_lse_merge(rows, heads, head_dim, o_is_fp32 ? 1 : 0, o_a, lse_a, o_b, lse_b,
                          o_out, lse_out, (cudaStream_t)stream);
}

ba_status ba_exp2_check(const float *x, float *y_fma, float *y_hw, int64_t n, ba_stream_t stream) {
  if (n < 0) {
    set_error("ba_exp2_check: n must be >= 0");
    return BA_ERR_INVALID_ARG;
  }
  if (n == 0) return BA_OK;
  BA_TRY(check_f32(x, true, "x"));
  BA_TRY(check_f32(y_fma, true, "y_fma"));
  BA_TRY(check_f32(y_hw, true, "y_hw"));
  return launch_exp2_check(x, y_fma, y_hw, n, (cudaStream_t)stream);
}

ba_status ba_set_kernel_family(int32_t family) {
  if (family < 0 || family > 1) {
    set_error("unknown kernel family %d", family);
    return BA_ERR_INVALID_ARG;
  }
  g_family.store(family);
  return BA_OK;
}

int32_t ba_get_kernel_family(void) { return g_family.load(); }

ba_status ba_set_kernel_events(int32_t which, void *start_event, void *stop_event) {
  if (which < 0 || which > 2) {
    set_error("ba_set_kernel_events: which must be 0 (forward), 1 (backward) or 2 (preprocess)");
    return BA_ERR_INVALID_ARG;
  }
  g_ev_start[which].store(start_event);
  g_ev_stop[which].store(stop_event);
  return BA_OK;
}

int64_t ba_launch_count(void) { return g_launches.load(); }

const char *ba_last_error(void) { return g_err; }

const char *ba_version(void) { return "branch_attn 0.1 (sm_100a)"; }

}  // extern "C"
