// Fused backward of branch attention on the tcgen05 tensor cores (sm_100a):
// one kernel computes all five tile products of the backward,
//   S^T = K Q^T,  dP^T = V dO^T,  dV += P^T dO,  dK += dS^T Q,  dQ = dS K,
// with P = exp(S - l) recomputed from the merged LSE l written by the forward
// (so the main-prefix and branch-local parts of a branch query share one
// softmax normalisation, as the merge rule of "Online Draft Co-Training",
// technical-contribution section, makes them) and dS = P (dP - D),
// D = rowsum(dO O).
//
// CTA = (128-key tile from the plan's backward order, kv head g).  It walks
// every 128-row query tile of every q head of the group that sees the tile
// (the same walk as the split dK/dV kernel), keeping dK and dV in TMEM for
// the whole walk.  Each chunk's dQ partial (this key tile's contribution to
// the 128 query rows) is summed into an fp32 accumulator in global memory;
// a final pass scales it and converts it to bf16.
//
// 576 threads: warp 0 TMA producer, warp 1 MMA issuer (one thread), warps
// 2-17 elementwise, four threads per key row (row r = TMEM lane, quarter qq
// of the 128 queries).  TMEM (512 columns):
//   dK [0, D)  dV [D, 2D)  SP [2D, 2D + 128)  QB [2D + 128, 2D + 256)
// SP holds S^T(c), then dP^T(c) once every thread has S^T(c) in registers,
// then P^T(c) (bf16 pairs, written by each thread over the dP^T columns it
// read), the TMEM A operand of dV(c).  QB holds dQ(c) until it is summed out.
// Shared memory: K, V, two-deep Q and dO rings, dS^T (one tile, 128 B
// swizzle: the K-major A operand of dK and the MN-major A operand of dQ) and
// the chunk's per-query records {l log2 e, D, key lo, key hi}.
//
// Issue order of chunk c: dV(c), S^T(c+1), dK(c), dQ(c), dP^T(c+1).  The
// elementwise threads of chunk c take S^T(c) (exp phase), then sum dQ(c-1)
// out of QB, then take dP^T(c) and write P^T(c), dS^T(c); the tensor core
// meanwhile runs dK(c-1), dQ(c-1) and dP^T(c).
#include "attn_sm100_common.cuh"

namespace ba {
namespace {

using namespace sm100;

constexpr int kFThreads = 576;
constexpr int kFElem = kFThreads - 64;  // elementwise threads

template <int D>
struct FusedSmem {
  bf16 k[128 * D];                 // D/64 boxes of [128 rows][64], 16 KB each
  bf16 v[128 * D];
  bf16 q[2][kQc * D];
  bf16 dout[2][kQc * D];
  bf16 ds[128 * kQc];              // dS^T: two boxes [128 keys][64 queries]
  alignas(16) float rec[2 * kQc];  // LSE log2 [128], D [128]
  int4 rec_chunk;                   // {no mask needed, branch query tile, first query row}
  uint64_t bar_kv;
  uint64_t bar_q_full[2], bar_q_empty[2];
  uint64_t bar_do_full[2], bar_do_empty[2];
  uint64_t bar_rec_full;
  uint64_t bar_s_full, bar_s_read, bar_dp_full, bar_pds, bar_dq_full;
  uint64_t bar_acc, bar_drain;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ void red_add_v4(float *p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};\n" ::"l"(p), "f"(a), "f"(b),
               "f"(c), "f"(d)
               : "memory");
}

template <int D>
__global__ void __launch_bounds__(kFThreads, 1)
    bwd_fused_sm100_kernel(const AttnParams a, const __grid_constant__ DkvMaps tm) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  FusedSmem<D> &sm = *reinterpret_cast<FusedSmem<D> *>(smem_raw);
  if (a.plan.status[0] != 0) return;
  int *status_word = a.plan.status + 1;
  // the 128-byte swizzled tiles need 1024-byte aligned shared memory; the
  // layout has no room for padding, so refuse (status bit 14) instead
  if ((smem_u32(smem_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicOr(status_word, 1 << 14);
    return;
  }

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int item = a.plan.bwd_order[blockIdx.x / a.hkv];
  const int g = blockIdx.x % a.hkv;
  const bool main_kv = item < a.n_kt;
  const int kt = main_kv ? item : item - a.n_kt;
  const int key0 = kt * 128;
  const int n_keys = main_kv ? a.n_main : a.n_bt;
  const ChunkWalk cw = make_walk(a, main_kv, kt, g);
  const int total = cw.grp * (cw.n_t0 + cw.n_t1);
  volatile int *abort_flag = &sm.abort_flag;

  const uint32_t b_kv = smem_u32(&sm.bar_kv), b_rec = smem_u32(&sm.bar_rec_full);
  const uint32_t b_s = smem_u32(&sm.bar_s_full), b_sr = smem_u32(&sm.bar_s_read);
  const uint32_t b_dp = smem_u32(&sm.bar_dp_full), b_pds = smem_u32(&sm.bar_pds);
  const uint32_t b_dq = smem_u32(&sm.bar_dq_full), b_acc = smem_u32(&sm.bar_acc);
  const uint32_t b_drain = smem_u32(&sm.bar_drain);
  if (threadIdx.x == 0) {
    mbar_init(b_kv, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&sm.bar_q_full[s]), 1);
      mbar_init(smem_u32(&sm.bar_q_empty[s]), 1);
      mbar_init(smem_u32(&sm.bar_do_full[s]), 1);
      mbar_init(smem_u32(&sm.bar_do_empty[s]), 1);
    }
    mbar_init(b_rec, 1);
    mbar_init(b_s, 1);
    mbar_init(b_sr, kFElem);
    mbar_init(b_dp, 1);
    mbar_init(b_pds, kFElem);
    mbar_init(b_dq, 1);
    mbar_init(b_acc, 1);
    mbar_init(b_drain, 1);
    sm.abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(&sm.tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const uint32_t t_dk = tmem, t_dv = tmem + D, t_sp = tmem + 2 * D, t_qb = tmem + 2 * D + 128;
  // records of this CTA's key kind: main-key intervals or branch-local ones

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    if (total > 0) {
      mbar_expect_tx(b_kv, 2 * 128 * D * 2);
      const CUtensorMap *km = main_kv ? &tm.t.k_m : &tm.t.k_b;
      const CUtensorMap *vm = main_kv ? &tm.t.v_m : &tm.t.v_b;
#pragma unroll
      for (int x = 0; x < D / 64; ++x) {
        tma_load_3d(smem_u32(sm.k) + x * 16384, km, b_kv, x * 64, g, key0);
        tma_load_3d(smem_u32(sm.v) + x * 16384, vm, b_kv, x * 64, g, key0);
      }
    }
    int q_issued = 0, do_issued = 0, rec_issued = 0;
    for (int c = 0; c < total; ++c) {
      int h, tile, nrows;
      bool is_main_q;
      cw.at(c, a, h, is_main_q, tile, nrows);
      const int row0 = tile * kQc;
      const int st = c & 1;
      if (c >= 2 && !mbar_wait(smem_u32(&sm.bar_q_empty[st]), ((c >> 1) - 1) & 1, abort_flag,
                               status_word, 1))
        break;
      const uint32_t qbar = smem_u32(&sm.bar_q_full[st]);
      mbar_expect_tx(qbar, kQc * D * 2);
      const CUtensorMap *qm = is_main_q ? &tm.t.q_m : &tm.t.q_b;
#pragma unroll
      for (int x = 0; x < D / 64; ++x)
        tma_load_3d(smem_u32(sm.q[st]) + x * 16384, qm, qbar, x * 64, h, row0);
      ++q_issued;
      if (c >= 2 && !mbar_wait(smem_u32(&sm.bar_do_empty[st]), ((c >> 1) - 1) & 1, abort_flag,
                               status_word, 1))
        break;
      const uint32_t dbar = smem_u32(&sm.bar_do_full[st]);
      mbar_expect_tx(dbar, kQc * D * 2);
      const CUtensorMap *dm = is_main_q ? &tm.do_m : &tm.do_b;
#pragma unroll
      for (int x = 0; x < D / 64; ++x)
        tma_load_3d(smem_u32(sm.dout[st]) + x * 16384, dm, dbar, x * 64, h, row0);
      ++do_issued;
      // the single record buffer is free once chunk c-1's elementwise work is done
      if (c >= 1 && !mbar_wait(b_pds, (c - 1) & 1, abort_flag, status_word, 1)) break;
      // a chunk whose every query sees every key of this tile needs no mask;
      // the flag is published by the arrive below, with the records
      bool full = false;
      if (main_kv) {
        const int32_t *qt =
            a.plan.qtile + (int64_t)(is_main_q ? tile : a.n_qt_main + tile) * 6;
        full = nrows == kQc && kt >= qt[1] && kt < qt[2];
      }
      sm.rec_chunk = make_int4(full ? 1 : 0, is_main_q ? 0 : 1, row0, 0);
      mbar_expect_tx(b_rec, kQc * 8);
      const int64_t prow = (is_main_q ? 0 : a.n_main_pad) + row0;
      bulk_load(smem_u32(sm.rec), a.rec + rec_block(h, a.rows_pad, prow), kQc * 8, b_rec);
      ++rec_issued;
    }
    // no copy may still be writing shared memory when the CTA exits
    for (int c = (q_issued > 2 ? q_issued - 2 : 0); c < q_issued; ++c)
      mbar_wait_drain(smem_u32(&sm.bar_q_full[c & 1]), (c >> 1) & 1, status_word, 2);
    for (int c = (do_issued > 2 ? do_issued - 2 : 0); c < do_issued; ++c)
      mbar_wait_drain(smem_u32(&sm.bar_do_full[c & 1]), (c >> 1) & 1, status_word, 2);
    if (rec_issued > 0) mbar_wait_drain(b_rec, (rec_issued - 1) & 1, status_word, 2);
    if (total > 0) mbar_wait_drain(b_kv, 0, status_word, 2);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_s = idesc_bf16(128, kQc, false, false);   // S^T, dP^T
    constexpr uint32_t idesc_g = idesc_bf16(128, D, false, true);      // dV, dK
    constexpr uint32_t idesc_q = idesc_bf16(128, D, true, true);       // dQ
    bool ok = total == 0 || mbar_wait(b_kv, 0, abort_flag, status_word, 3);
    const uint64_t kd_k = sdesc(smem_u32(sm.k), 16, 1024);        // K, K-major (A of S^T)
    const uint64_t vd_k = sdesc(smem_u32(sm.v), 16, 1024);        // V, K-major (A of dP^T)
    const uint64_t kd_mn = sdesc(smem_u32(sm.k), 16384, 1024);    // K, MN-major (B of dQ)
    const uint64_t dsd_k = sdesc(smem_u32(sm.ds), 16, 1024);      // dS^T, K-major (A of dK)
    const uint64_t dsd_mn = sdesc(smem_u32(sm.ds), 16384, 1024);  // dS, MN-major (A of dQ)
    // An mbarrier wait in this thread holds it until the MMAs it queued are
    // (nearly) done, so each chunk waits at two points only: before dV(c)
    // (P^T / dS^T of c, and Q(c+1) for S^T(c+1)) and before dP^T(c+1).
    auto wait_q = [&](int c) -> bool {
      return mbar_wait(smem_u32(&sm.bar_q_full[c & 1]), (c >> 1) & 1, abort_flag, status_word, 5);
    };
    auto issue_s = [&](int c) {
      const int st = c & 1;
      const uint64_t qd = sdesc(smem_u32(sm.q[st]), 16, 1024);
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
        mma_bf16(t_sp, desc_at(kd_k, off), desc_at(qd, off), idesc_s, k > 0 ? 1u : 0u);
      }
      mma_commit(b_s);
    };
    auto issue_dp = [&](int c) -> bool {
      const int st = c & 1;
      // S^T(c) has left SP for the elementwise threads' registers
      if (!mbar_wait(b_sr, c & 1, abort_flag, status_word, 6) ||
          !mbar_wait(smem_u32(&sm.bar_do_full[st]), (c >> 1) & 1, abort_flag, status_word, 5))
        return false;
      tc_fence_after();
      const uint64_t dd = sdesc(smem_u32(sm.dout[st]), 16, 1024);
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
        mma_bf16(t_sp, desc_at(vd_k, off), desc_at(dd, off), idesc_s, k > 0 ? 1u : 0u);
      }
      mma_commit(b_dp);
      return true;
    };
    if (ok && total > 0) {
      ok = wait_q(0);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        ok = issue_dp(0);
      }
    }
    for (int c = 0; ok && c < total; ++c) {
      // P^T(c) in SP, dS^T(c) in shared memory, dQ(c-1) out of QB; Q(c+1) loaded
      if (!mbar_wait(b_pds, c & 1, abort_flag, status_word, 4) ||
          (c + 1 < total && !wait_q(c + 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int st = c & 1;
      const uint32_t acc = c > 0 ? 1u : 0u;
      // dV += P^T dO: P^T from TMEM (K-step k = queries 16k.., at SP + 32 (k/2) + 8 (k%2)),
      // dO MN-major (16 query rows of 128 B per K-step)
      const uint64_t dd = sdesc(smem_u32(sm.dout[st]), 16384, 1024);
#pragma unroll
      for (int k = 0; k < kQc / 16; ++k)
        mma_bf16_ts(t_dv, t_sp + (k >> 1) * 32 + (k & 1) * 8, desc_at(dd, k * 2048), idesc_g,
                    (acc | (uint32_t)k) ? 1u : 0u);
      mma_commit(smem_u32(&sm.bar_do_empty[st]));
      // S^T(c+1) over SP: the MMAs of this thread run in order, so dV(c) has
      // read P^T(c) before it is overwritten
      if (c + 1 < total) issue_s(c + 1);
      // dK += dS^T Q: dS^T K-major from shared memory, Q MN-major
      const uint64_t qd = sdesc(smem_u32(sm.q[st]), 16384, 1024);
#pragma unroll
      for (int k = 0; k < kQc / 16; ++k) {
        const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
        mma_bf16(t_dk, desc_at(dsd_k, off), desc_at(qd, k * 2048), idesc_g,
                 (acc | (uint32_t)k) ? 1u : 0u);
      }
      mma_commit(smem_u32(&sm.bar_q_empty[st]));
      // dQ = dS K: dS (queries x keys) is dS^T read MN-major, K MN-major;
      // K-step k = keys 16k.. (16 rows of 128 B in both operands)
#pragma unroll
      for (int k = 0; k < 128 / 16; ++k)
        mma_bf16(t_qb, desc_at(dsd_mn, k * 2048), desc_at(kd_mn, k * 2048), idesc_q,
                 k > 0 ? 1u : 0u);
      mma_commit(b_dq);
      if (c + 1 < total && !issue_dp(c + 1)) {
        ok = false;
        break;
      }
    }
    if (ok && total > 0) mma_commit(b_acc);
    // nothing may still write TMEM or read shared memory when the CTA exits
    mma_commit(b_drain);
    mbar_wait_drain(b_drain, 0, status_word, 2);
  } else if (warp >= 2) {
    // ------------------------------------------------------------ elementwise (4 threads / key)
    const int qq = (warp - 2) >> 2;   // query quarter: [32 qq, 32 qq + 32)
    const int row = (warp & 3) * 32 + lane;
    const int key = key0 + row;
    const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
    const float sl2 = a.scale_log2;
    constexpr int kDqCols = D / 4;    // dQ columns this thread sums out of QB
    const uint32_t ds_row = smem_u32(sm.ds) + (qq >> 1) * 16384 + row * 128;
    // the query rows that see this key: main rows [x, y), branch rows [z, w)
    int4 kiv = make_int4(0, 0, 0, 0);
    if (key < n_keys)
      kiv = reinterpret_cast<const int4 *>(a.plan.key_iv)[(main_kv ? 0 : a.n_main) + key];
    bool ok = true;
    // sums dQ(c) (query row `row` of chunk c, columns [qq D/4, (qq+1) D/4)) into
    // the fp32 accumulator
    auto drain_dq = [&](int c) -> bool {
      if (!__all_sync(0xffffffffu, mbar_wait(b_dq, c & 1, abort_flag, status_word, 11)))
        return false;
      tc_fence_after();
      int h, tile, nrows;
      bool is_main_q;
      cw.at(c, a, h, is_main_q, tile, nrows);
      uint32_t o[kDqCols];
      if constexpr (kDqCols == 32) tmem_ld32(t_qb + lane_addr + qq * kDqCols, o);
      else tmem_ld16(t_qb + lane_addr + qq * kDqCols, o);
      tc_wait_ld();
      tc_fence_before();
      if (row < nrows) {
        const int64_t grow = (is_main_q ? 0 : a.n_main) + (int64_t)tile * kQc + row;
        float *dst = a.dq_acc + (grow * a.hq + h) * D + qq * kDqCols;
#pragma unroll
        for (int e = 0; e < kDqCols / 4; ++e)
          red_add_v4(dst + 4 * e, __uint_as_float(o[4 * e]), __uint_as_float(o[4 * e + 1]),
                     __uint_as_float(o[4 * e + 2]), __uint_as_float(o[4 * e + 3]));
      }
      return true;
    };
    for (int c = 0; c < total; ++c) {
      // ---- exp phase: S^T(c) -> P
      if (!__all_sync(0xffffffffu, mbar_wait(b_s, c & 1, abort_flag, status_word, 7))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float p[32];
      tmem_ld32(t_sp + lane_addr + qq * 32, reinterpret_cast<uint32_t *>(p));
      tc_wait_ld();
      tc_fence_before();
      mbar_arrive(b_sr);
      if (!__all_sync(0xffffffffu, mbar_wait(b_rec, c & 1, abort_flag, status_word, 8))) {
        ok = false;
        break;
      }
      // this quarter's 32 queries of each record field, four per 16-byte load
      const float4 *r_lse = reinterpret_cast<const float4 *>(sm.rec + kRecLse + qq * 32);
      const float4 *r_d = reinterpret_cast<const float4 *>(sm.rec + kRecD + qq * 32);
      const int4 ch = sm.rec_chunk;
      if (!ch.x) {
        // queries q of this quarter with lo <= q < hi see the key
        const int base = ch.z + qq * 32;
        const int lo = (ch.y ? kiv.z : kiv.x) - base, hi = (ch.y ? kiv.w : kiv.y) - base;
#pragma unroll
        for (int q = 0; q < 32; ++q)
          if (q < lo || q >= hi) p[q] = kNegInf;
      }
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) {
        const float4 l = r_lse[q4];
        p[4 * q4] = ex2(fmaf(p[4 * q4], sl2, -l.x));
        p[4 * q4 + 1] = ex2(fmaf(p[4 * q4 + 1], sl2, -l.y));
        p[4 * q4 + 2] = ex2(fmaf(p[4 * q4 + 2], sl2, -l.z));
        p[4 * q4 + 3] = ex2(fmaf(p[4 * q4 + 3], sl2, -l.w));
      }
      uint32_t pk[16];
#pragma unroll
      for (int q = 0; q < 32; q += 2) pk[q / 2] = pack_bf16(p[q], p[q + 1]);
      // ---- dQ(c-1) out of QB (its product ran during the exp phase); after
      // this, dK(c-1) and dQ(c-1) have also finished reading dS^T(c-1)
      if (c > 0 && !drain_dq(c - 1)) {
        ok = false;
        break;
      }
      // ---- dS phase: dP^T(c) -> P^T(c) into SP, dS^T(c) into shared memory
      if (!__all_sync(0xffffffffu, mbar_wait(b_dp, c & 1, abort_flag, status_word, 9))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t col = t_sp + lane_addr + qq * 32;
      float dp[32];
      tmem_ld32(col, reinterpret_cast<uint32_t *>(dp));
      tc_wait_ld();
      tmem_st16(col, pk);
      uint32_t dk2[16];
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) {
        const float4 dd = r_d[q4];
        dk2[2 * q4] = pack_bf16(p[4 * q4] * (dp[4 * q4] - dd.x), p[4 * q4 + 1] * (dp[4 * q4 + 1] - dd.y));
        dk2[2 * q4 + 1] =
            pack_bf16(p[4 * q4 + 2] * (dp[4 * q4 + 2] - dd.z), p[4 * q4 + 3] * (dp[4 * q4 + 3] - dd.w));
      }
      // row `row` of dS^T, queries [32 qq, 32 qq + 32): 16-byte chunks
      // (qq & 1) * 4 + e of the row, placed by the 128-byte swizzle
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t chunk = (uint32_t)(((qq & 1) * 4 + e) ^ (row & 7));
        st_shared_v4(ds_row + chunk * 16, dk2[4 * e], dk2[4 * e + 1], dk2[4 * e + 2],
                     dk2[4 * e + 3]);
      }
      tc_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(b_pds);
    }
    if (ok && total > 0 && !drain_dq(total - 1)) ok = false;
    if (ok && total > 0 &&
        !__all_sync(0xffffffffu, mbar_wait(b_acc, 0, abort_flag, status_word, 10)))
      ok = false;
    tc_fence_after();
    // epilogue: each of the four threads of a key row stores a quarter of dK and dV
    constexpr int kCols = D / 4;
    const bool valid = key < n_keys;
    bf16 *dkg = (main_kv ? a.dk_m : a.dk_b) + ((int64_t)key * a.hkv + g) * D + qq * kCols;
    bf16 *dvg = (main_kv ? a.dv_m : a.dv_b) + ((int64_t)key * a.hkv + g) * D + qq * kCols;
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      const uint32_t src = (part == 0 ? t_dk : t_dv) + qq * kCols + lane_addr;
      const float mul = part == 0 ? a.scale : 1.f;
      bf16 *dst = part == 0 ? dkg : dvg;
      uint32_t o[kCols];
      if (ok && total > 0) {
        if constexpr (kCols == 32) tmem_ld32(src, o);
        else tmem_ld16(src, o);
        tc_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < kCols; ++e) o[e] = 0u;
      }
      if (!valid) continue;
      uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
      for (int e = 0; e < kCols / 8; ++e)
        d4[e] = make_uint4(
            pack_bf16(__uint_as_float(o[8 * e]) * mul, __uint_as_float(o[8 * e + 1]) * mul),
            pack_bf16(__uint_as_float(o[8 * e + 2]) * mul, __uint_as_float(o[8 * e + 3]) * mul),
            pack_bf16(__uint_as_float(o[8 * e + 4]) * mul, __uint_as_float(o[8 * e + 5]) * mul),
            pack_bf16(__uint_as_float(o[8 * e + 6]) * mul, __uint_as_float(o[8 * e + 7]) * mul));
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, 512);
}

template <int D>
ba_status launch_fused(const AttnParams &a, const DkvMaps &maps, cudaStream_t s) {
  const int64_t grid = (int64_t)(a.n_kt + a.n_bkt) * a.hkv;
  if (grid <= 0) return BA_OK;
  const size_t smem = sizeof(FusedSmem<D>);
  static_assert(sizeof(FusedSmem<D>) <= 232448, "fused backward exceeds 227 KB of shared memory");
  cudaError_t e = cudaFuncSetAttribute(bwd_fused_sm100_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return cuda_check(e, "bwd_fused_sm100_kernel smem");
  bwd_fused_sm100_kernel<D><<<(unsigned)grid, kFThreads, smem, s>>>(a, maps);
  count_launches(1);
  return cuda_check(cudaGetLastError(), "bwd_fused_sm100_kernel launch");
}

}  // namespace

bool sm100_fused_bwd_available() { return true; }

ba_status launch_bwd_fused_sm100(const AttnParams &a, cudaStream_t s) {
  const int d = a.head_dim;
  DkvMaps m;
  ba_status st;
  const bool br = a.n_bt > 0;
#define BA_MAP(dst, ptr, rows, heads)                                              \
  if ((st = make_tensor_map(&(dst), ptr, rows, heads, d, 128)) != BA_OK) return st;
  BA_MAP(m.t.q_m, a.q_m, a.n_main, a.hq)
  BA_MAP(m.t.k_m, a.k_m, a.n_main, a.hkv)
  BA_MAP(m.t.v_m, a.v_m, a.n_main, a.hkv)
  BA_MAP(m.do_m, a.do_m, a.n_main, a.hq)
  if (br) {
    BA_MAP(m.t.q_b, a.q_b, a.n_bt, a.hq)
    BA_MAP(m.t.k_b, a.k_b, a.n_bt, a.hkv)
    BA_MAP(m.t.v_b, a.v_b, a.n_bt, a.hkv)
    BA_MAP(m.do_b, a.do_b, a.n_bt, a.hq)
  } else {
    m.t.q_b = m.t.q_m; m.t.k_b = m.t.k_m; m.t.v_b = m.t.v_m; m.do_b = m.do_m;
  }
#undef BA_MAP
  return d == 64 ? launch_fused<64>(a, m, s) : launch_fused<128>(a, m, s);
}

}  // namespace ba
