// Internal declarations shared by the translation units of libbranch_attn.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "branch_attn.h"

namespace ba {

constexpr int kTileM = BA_TILE_M;  // query rows per tile
constexpr int kTileN = BA_TILE_N;  // key rows per tile
constexpr int kMaxDepth = 64;

// Plan workspace views, resolved from a ba_plan_layout.
struct PlanView {
  int32_t *status;
  int32_t *cu_branch;
  int32_t *branch_seq;
  int32_t *row_iv;     // [(N + Nb) * 4]
  int32_t *qtile;      // [n_qt * 6]
  int32_t *kv_main;    // [n_kt * 4]
  int32_t *kv_branch;  // [n_bkt * 2]
  int32_t *fwd_order;
  int32_t *bwd_order;
  int32_t *fwd_cost;
  int32_t *bwd_cost;
  int32_t *zz_tiles;   // [C * n_qt * 4] or null
  int32_t *key_iv;     // [(N + Nb) * 4]
  int32_t *bwd_prefix; // [n_kt + n_bkt] bwd_cost summed over the key tiles ranked before
};

// Everything an attention kernel needs; device pointers only.
struct AttnParams {
  const __nv_bfloat16 *q_m, *k_m, *v_m, *q_b, *k_b, *v_b;
  __nv_bfloat16 *o_m, *o_b;
  float *lse_m, *lse_b;
  // backward
  const __nv_bfloat16 *do_m, *do_b;
  const float *d_all;         // D [Hq, N + Nb]
  float *dq_acc;              // [(N + Nb), Hq, d] fp32
  __nv_bfloat16 *dk_m, *dv_m, *dk_b, *dv_b;
  __nv_bfloat16 *dq_out_m, *dq_out_b;  // dQ written directly (tcgen05 backward)
  int32_t zero_dq_acc;                  // preprocess clears dq_acc
  // per-query backward records (tcgen05 backward), 8 B per (q head, padded
  // row); main rows at [0, n_main_pad), branch rows after.  Each 128-row
  // block of a head is 256 words: LSE * log2(e) [128], then D [128]
  // (rec_block below), so one 16-byte load gives four consecutive queries.
  float *rec;
  int32_t n_main_pad, rows_pad;
  // zigzag partial output (fp32 O accumulator [(N+Nb), Hq, d], LSE [Hq, N+Nb])
  float *zz_o;
  float *zz_lse;
  int32_t zz_step;            // ring step, -1 = monolithic, C = branch-local pass
  int32_t zz_C;
  // ring mode (zigzag context parallelism across ranks): the plan holds this
  // step's main-key intervals in row_iv (x, y) and tile ranges in qtile[0..3];
  // step C takes the branch-local keys (row_iv z, w; qtile[4..5])
  int32_t ring;
  int32_t n_keys_m;           // main key rows (the visiting shard's in ring mode, else n_main)
  int32_t n_sms;              // streaming multiprocessors of the device (launch-order bands)
  const int32_t *cu_seqlens;
  PlanView plan;
  int32_t n_main, n_bt;       // main / branch token counts
  int32_t n_seqs;
  int32_t hq, hkv, head_dim;
  int32_t mask;
  int32_t n_qt_main, n_qt;    // query tiles (main, total)
  int32_t n_kt, n_bkt;        // key tiles (main, branch)
  float scale;
  float scale_log2;           // scale * log2(e)
};

const char *set_error(const char *fmt, ...);
void count_launches(int n);
ba_status cuda_check(cudaError_t e, const char *what);

ba_status launch_plan(const ba_problem &p, const ba_plan_layout &L, const PlanView &v,
                      cudaStream_t s);
ba_status launch_ring_plan(const ba_problem &p, const ba_plan_layout &L, const PlanView &v,
                           const int32_t *cu_glob, const int32_t *cu_vis, int C, int q, int j,
                           cudaStream_t s);
ba_status launch_lse_merge(int64_t rows, int heads, int d, int fp32, const void *oa,
                           const float *la, const void *ob, const float *lb, void *oo,
                           float *lo, cudaStream_t s);
ba_status launch_bwd_preprocess(const AttnParams &a, cudaStream_t s);
ba_status launch_dq_convert(const AttnParams &a, __nv_bfloat16 *dq_m, __nv_bfloat16 *dq_b,
                            cudaStream_t s);
ba_status launch_zz_finalize(const AttnParams &a, cudaStream_t s);

// tcgen05 / TMEM / TMA kernels
ba_status launch_fwd_sm100(const AttnParams &a, cudaStream_t s);
ba_status launch_bwd_sm100(const AttnParams &a, cudaStream_t s);
bool sm100_fused_bwd_available();
ba_status launch_bwd_fused_sm100(const AttnParams &a, cudaStream_t s);
ba_status launch_exp2_check(const float *x, float *y_fma, float *y_mufu, int64_t n,
                            cudaStream_t s);

__host__ __device__ inline int64_t cdiv64(int64_t a, int64_t b) { return (a + b - 1) / b; }

// First word of the 128-row record block holding padded row pr of q head h;
// field f of that row is at + f + (pr % 128).
constexpr int kRecLse = 0, kRecD = 128;
__host__ __device__ inline int64_t rec_block(int64_t h, int32_t rows_pad, int64_t pr) {
  return (h * rows_pad + (pr & ~(int64_t)127)) * 2;
}

}  // namespace ba
