// Branch attention on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// Forward kernel: one CTA per (query tile of 128 rows, q head), 8 warps.
//   warp 0      TMA producer: Q once, then 3-stage rings of 128-key K tiles
//               and V tiles (K is refilled as soon as S has read it)
//   warp 1      MMA issuer (one thread): S_j = Q K_j^T into TMEM (two S
//               buffers, so S_{j+1} runs while tile j is in softmax), then
//               O += P_j V_j with P read from TMEM and O accumulating there
//   warp 2      TMEM allocation (512 columns: S0, S1, O, P0, P1)
//   warps 4-7   softmax, one thread per query row (= TMEM lane): reads its S
//               row, masks it with the row's key interval, keeps the running
//               max / sum, writes P (bf16 pairs) back to TMEM, and rescales
//               its O row only when the running max grew by more than 2^8.
// Key tiles come from the plan: the main key tiles of the query tile, then
// (branch tiles) the branch-local key rows.  Folding each tile's partial into
// the running (O, l) is the online-softmax merge; the branch-local tiles come
// last, so their fold is the paper's merge of (O_b, l_b) into (O_m, l_m)
// ("Online Draft Co-Training", technical-contribution section).  The epilogue
// normalises O and writes the LSE, or, on the zigzag ring path, merges the
// step's partial into an fp32 accumulator by the same rule.
#include <cudaTypedefs.h>

#include <mutex>

#include "attn_sm100_common.cuh"

namespace ba {

// ---- host: tensor maps -------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [rows, heads, d] bf16 -> 3-D map (d, heads, rows), box (64, 1, box_rows), 128-byte swizzle.
ba_status make_tensor_map(CUtensorMap *m, const void *ptr, int64_t rows, int heads, int d,
                          int box_rows) {
  auto fn = encode_fn();
  if (!fn) {
    set_error("cuTensorMapEncodeTiled unavailable");
    return BA_ERR_CUDA;
  }
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)heads * d * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("cuTensorMapEncodeTiled failed (%d)", (int)r);
    return BA_ERR_CUDA;
  }
  return BA_OK;
}


namespace {

using namespace sm100;

constexpr float kRescaleThreshold = 8.0f;  // log2 units

// ---- device ---------------------------------------------------------------------
constexpr int kFwdStages = 3;

template <int D>
struct FwdSmem {
  bf16 q[128 * D];              // D/64 boxes of [128 rows][64], 16 KB each
  bf16 k[kFwdStages][128 * D];
  bf16 v[kFwdStages][128 * D];
  uint64_t bar_q;
  uint64_t bar_k_full[kFwdStages], bar_k_empty[kFwdStages];
  uint64_t bar_v_full[kFwdStages], bar_v_empty[kFwdStages];
  uint64_t bar_s_full[2], bar_s_empty[2];
  uint64_t bar_p_full[2];
  uint64_t bar_o_done;
  uint64_t bar_o_final;  // one phase: the last PV product has landed in O
  uint64_t bar_drain;    // one phase: every MMA the issuer queued has completed
  uint32_t tmem_base;
  int abort_flag;
};

// TMEM columns: S double-buffered at 0 and 128, O at 256, P (bf16 pairs)
// double-buffered at 384 and 448.
template <int D>
__global__ void __launch_bounds__(256, 1)
    fwd_sm100_kernel(const AttnParams a, const __grid_constant__ TensorMaps tm) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  FwdSmem<D> &sm = *reinterpret_cast<FwdSmem<D> *>(smem_raw + (((raw + 1023) & ~1023u) - raw));
  if (a.plan.status[0] != 0) return;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int item = blockIdx.x;
  const int t = a.plan.fwd_order[item / a.hq];
  const int h = item % a.hq;
  const int g = h / (a.hq / a.hkv);
  const bool is_main = t < a.n_qt_main;
  const int tt = is_main ? t : t - a.n_qt_main;
  const int rows_total = is_main ? a.n_main : a.n_bt;
  const int row0 = tt * 128;
  const int nrows = min(128, rows_total - row0);
  const int row_off = is_main ? 0 : a.n_main;
  const TileSegs segs = make_segs(a, t, is_main);
  const int total = segs.total;
  int *status_word = a.plan.status + 1;
  volatile int *abort_flag = &sm.abort_flag;

  const uint32_t b_q = smem_u32(&sm.bar_q), b_o = smem_u32(&sm.bar_o_done);
  const uint32_t b_final = smem_u32(&sm.bar_o_final);
  if (threadIdx.x == 0) {
    mbar_init(b_q, 1);
    for (int s = 0; s < kFwdStages; ++s) {
      mbar_init(smem_u32(&sm.bar_k_full[s]), 1);
      mbar_init(smem_u32(&sm.bar_k_empty[s]), 1);
      mbar_init(smem_u32(&sm.bar_v_full[s]), 1);
      mbar_init(smem_u32(&sm.bar_v_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&sm.bar_s_full[s]), 1);
      mbar_init(smem_u32(&sm.bar_s_empty[s]), 128);
      mbar_init(smem_u32(&sm.bar_p_full[s]), 128);
    }
    mbar_init(b_o, 1);
    mbar_init(b_final, 1);
    mbar_init(smem_u32(&sm.bar_drain), 1);
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
  const uint32_t t_o = tmem + 256;
  auto t_p = [&](int b) { return tmem + 384 + b * 64; };

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    const CUtensorMap *qmap = is_main ? &tm.q_m : &tm.q_b;
    if (total > 0) {
      mbar_expect_tx(b_q, 128 * D * 2);
#pragma unroll
      for (int x = 0; x < D / 64; ++x)
        tma_load_3d(smem_u32(sm.q) + x * 16384, qmap, b_q, x * 64, h, row0);
    }
    int issued_k = 0, issued_v = 0;
    for (int j = 0; j < total; ++j) {
      const int st = j % kFwdStages;
      const uint32_t ph = ((j / kFwdStages) - 1) & 1;
      int key0, kind;
      bool full;
      segs.locate(j, key0, kind, full);
      if (j >= kFwdStages &&
          !mbar_wait(smem_u32(&sm.bar_k_empty[st]), ph, abort_flag, status_word, 1))
        break;
      const uint32_t kb = smem_u32(&sm.bar_k_full[st]);
      mbar_expect_tx(kb, 128 * D * 2);
#pragma unroll
      for (int x = 0; x < D / 64; ++x)
        tma_load_3d(smem_u32(sm.k[st]) + x * 16384, kind == 2 ? &tm.k_b : &tm.k_m, kb, x * 64, g,
                    key0);
      ++issued_k;
      if (j >= kFwdStages &&
          !mbar_wait(smem_u32(&sm.bar_v_empty[st]), ph, abort_flag, status_word, 1))
        break;
      const uint32_t vb = smem_u32(&sm.bar_v_full[st]);
      mbar_expect_tx(vb, 128 * D * 2);
#pragma unroll
      for (int x = 0; x < D / 64; ++x)
        tma_load_3d(smem_u32(sm.v[st]) + x * 16384, kind == 2 ? &tm.v_b : &tm.v_m, vb, x * 64, g,
                    key0);
      ++issued_v;
    }
    // on abort: let the loads already issued land before the CTA exits
    for (int j = (issued_k > kFwdStages ? issued_k - kFwdStages : 0); j < issued_k; ++j)
      mbar_wait_drain(smem_u32(&sm.bar_k_full[j % kFwdStages]), (j / kFwdStages) & 1, status_word, 2);
    for (int j = (issued_v > kFwdStages ? issued_v - kFwdStages : 0); j < issued_v; ++j)
      mbar_wait_drain(smem_u32(&sm.bar_v_full[j % kFwdStages]), (j / kFwdStages) & 1, status_word, 2);
    if (total > 0) mbar_wait_drain(b_q, 0, status_word, 2);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_qk = idesc_bf16(128, 128, false, false);
    constexpr uint32_t idesc_pv = idesc_bf16(128, D, false, true);
    bool ok = total == 0 || mbar_wait(b_q, 0, abort_flag, status_word, 3);
    const uint32_t q_s = smem_u32(sm.q);
    auto issue_pv = [&](int i) -> bool {
      const int pb = i & 1, st = i % kFwdStages;
      if (!mbar_wait(smem_u32(&sm.bar_v_full[st]), (i / kFwdStages) & 1, abort_flag, status_word,
                     4) ||
          !mbar_wait(smem_u32(&sm.bar_p_full[pb]), (i >> 1) & 1, abort_flag, status_word, 4))
        return false;
      tc_fence_after();
      const uint64_t vd = sdesc(smem_u32(sm.v[st]), 16384, 1024);
      // O += P V: P (bf16 pairs) from TMEM, V as an MN-major operand
#pragma unroll
      for (int k = 0; k < 8; ++k)
        mma_bf16_ts(t_o, t_p(pb) + k * 8, desc_at(vd, k * 2048), idesc_pv,
                    (i > 0 || k > 0) ? 1u : 0u);
      mma_commit(b_o);
      mma_commit(smem_u32(&sm.bar_v_empty[st]));
      return true;
    };
    for (int j = 0; ok && j < total; ++j) {
      const int st = j % kFwdStages, sb = j & 1;
      if (!mbar_wait(smem_u32(&sm.bar_k_full[st]), (j / kFwdStages) & 1, abort_flag, status_word,
                     5) ||
          (j >= 2 && !mbar_wait(smem_u32(&sm.bar_s_empty[sb]), ((j - 2) >> 1) & 1, abort_flag,
                                status_word, 6))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint64_t qd = sdesc(q_s, 16, 1024), kd = sdesc(smem_u32(sm.k[st]), 16, 1024);
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
        mma_bf16(tmem + sb * 128, desc_at(qd, off), desc_at(kd, off), idesc_qk, k > 0 ? 1u : 0u);
      }
      mma_commit(smem_u32(&sm.bar_s_full[sb]));
      mma_commit(smem_u32(&sm.bar_k_empty[st]));
      if (j >= 1 && !issue_pv(j - 1)) {
        ok = false;
        break;
      }
    }
    if (ok && total > 0 && issue_pv(total - 1)) mma_commit(b_final);
    // nothing may still write TMEM when it is freed, aborted or not
    mma_commit(smem_u32(&sm.bar_drain));
    mbar_wait_drain(smem_u32(&sm.bar_drain), 0, status_word, 2);
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int row = threadIdx.x - 128;
    const bool valid = row < nrows;
    const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
    int lo[3] = {0, 0, 0}, hi[3] = {-1, -1, -1};
    const int zz = a.zz_step;
    if (valid) {
      const int4 iv = reinterpret_cast<const int4 *>(a.plan.row_iv)[row_off + row0 + row];
      if (a.ring) {
        // ring mode: this step's main interval, or the branch-local one last
        if (zz < a.zz_C) { lo[0] = iv.x; hi[0] = iv.y; }
        else { lo[2] = iv.z; hi[2] = iv.w; }
      } else if (zz < 0 || zz == a.zz_C) {
        lo[0] = iv.x; hi[0] = iv.y;
        lo[2] = iv.z; hi[2] = iv.w;
      }
      if (!a.ring && zz >= 0 && zz < a.zz_C) {
        int s_lo = 0, s_hi = a.n_seqs;
        while (s_lo < s_hi) {
          const int mid = (s_lo + s_hi + 1) >> 1;
          if (a.cu_seqlens[mid] <= iv.x) s_lo = mid; else s_hi = mid - 1;
        }
        const int64_t L = a.cu_seqlens[s_lo + 1] - iv.x;
        const int64_t pos = iv.y - iv.x;
        const int C = a.zz_C;
        const int c = (int)((2 * C * (pos + 1) - 1) / L);
        const int shard = c < C ? c : 2 * C - 1 - c;
        const int jw = ((shard - zz) % C + C) % C;
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          const int ch = w == 0 ? jw : 2 * C - 1 - jw;
          lo[w] = max(iv.x + (int)((ch * L) / (2 * C)), iv.x);
          hi[w] = min(iv.x + (int)(((ch + 1) * L) / (2 * C)) - 1, iv.y);
        }
      }
    }
    // running max (log2 units, possibly stale by < 2^8) and sum
    float m_used = kNegInf, l = 0.f;
    bool ok = true;
    const float sl2 = a.scale_log2;
    for (int j = 0; j < total; ++j) {
      const int sb = j & 1;
      // warp-uniform decisions: tcgen05.ld / st below are warp-collective
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.bar_s_full[sb]), (j >> 1) & 1,
                                             abort_flag, status_word, 7))) {
        ok = false;
        break;
      }
      tc_fence_after();
      int key0, kind;
      bool full;
      segs.locate(j, key0, kind, full);
      const int clo = kind == 0 ? lo[0] : (kind == 1 ? lo[1] : lo[2]);
      const int chi = kind == 0 ? hi[0] : (kind == 1 ? hi[1] : hi[2]);
      float s[128];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tmem_ld32(tmem + lane_addr + sb * 128 + c * 32, reinterpret_cast<uint32_t *>(s) + c * 32);
      tc_wait_ld();
      tc_fence_before();
      mbar_arrive(smem_u32(&sm.bar_s_empty[sb]));
      // mask (raw scores; the positive scale is applied after the max)
      if (!(full && valid)) {
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const int key = key0 + c;
          if (key < clo || key > chi) s[c] = kNegInf;
        }
      }
      float mx4[4] = {kNegInf, kNegInf, kNegInf, kNegInf};
#pragma unroll
      for (int c = 0; c < 128; c += 4) {
#pragma unroll
        for (int e = 0; e < 4; ++e) mx4[e] = fmaxf(mx4[e], s[c + e]);
      }
      const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * sl2;
      const float m_new = fmaxf(m_used, mx);
      const bool need = m_new > m_used + kRescaleThreshold;
      const float alpha = need ? ex2(m_used - m_new) : 1.f;
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        // O holds PV_{j-1}: wait for it, then scale the rows that need it in
        // TMEM (the whole warp takes part; other lanes scale by 1)
        if (!__all_sync(0xffffffffu, mbar_wait(b_o, (j - 1) & 1, abort_flag, status_word, 8))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(t_o + lane_addr + c * 32, o);
          tc_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(t_o + lane_addr + c * 32, o);
        }
        tc_wait_st();
      }
      if (need) {
        l *= alpha;
        m_used = m_new;
      }
      const float msub = m_used == kNegInf ? 0.f : m_used;
      // P = 2^(scale log2(e) s - m), packed to bf16 pairs in place
      uint32_t *pk = reinterpret_cast<uint32_t *>(s);
      float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 128; c += 4) {
        float pv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          pv[e] = ex2(fmaf(s[c + e], sl2, -msub));
          l4[e] += pv[e];
        }
        pk[c / 2] = pack_bf16(pv[0], pv[1]);
        pk[c / 2 + 1] = pack_bf16(pv[2], pv[3]);
      }
      l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
      // P buffer sb was last read by PV_{j-2}, which completed before S_j
      tmem_st32(t_p(sb) + lane_addr, pk);
      tmem_st32(t_p(sb) + lane_addr + 32, pk + 32);
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&sm.bar_p_full[sb]));
    }
    // the epilogue may lag o_done by two phases, so it waits on its own
    // one-phase barrier instead of a parity of o_done
    if (ok && total > 0 &&
        !__all_sync(0xffffffffu, mbar_wait(b_final, 0, abort_flag, status_word, 9)))
      ok = false;
    tc_fence_after();

    // ------------------------------------------------------------ epilogue
    const bool empty = !(l > 0.f) || m_used == kNegInf;
    float lse = empty ? kNegInf : (m_used + __log2f(l)) * kLn2;
    const float inv = empty ? 0.f : 1.f / l;
    const bool final_out = zz < 0 || zz == a.zz_C;
    float wa = 0.f, wb = 1.f;
    float *acc = nullptr;
    if (zz >= 0 && valid) {
      const int64_t all_rows = (int64_t)a.n_main + a.n_bt;
      const int64_t grow = row_off + row0 + row;
      acc = a.zz_o + (grow * a.hq + h) * D;
      float *accl = a.zz_lse + (int64_t)h * all_rows + grow;
      float lnew = lse;
      if (zz > 0) {
        const float la = *accl;
        const float mm = fmaxf(la, lse);
        if (mm == kNegInf) {
          lnew = kNegInf; wa = 0.f; wb = 0.f;
        } else {
          lnew = mm + logf(expf(la - mm) + expf(lse - mm));
          wa = expf(la - lnew);
          wb = expf(lse - lnew);
        }
      }
      if (!final_out) *accl = lnew;
      lse = lnew;
    }
    bf16 *og = (is_main ? a.o_m : a.o_b) + ((int64_t)(row0 + row) * a.hq + h) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      if (ok && total > 0) {
        tmem_ld32(t_o + lane_addr + c * 32, o);
        tc_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = 0u;
      }
      if (!valid) continue;
      float f[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(o[e]) * inv;
      if (zz >= 0) {
        float4 *ap = reinterpret_cast<float4 *>(acc + c * 32);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float4 prev = zz > 0 ? ap[e] : make_float4(0.f, 0.f, 0.f, 0.f);
          f[4 * e + 0] = wa * prev.x + wb * f[4 * e + 0];
          f[4 * e + 1] = wa * prev.y + wb * f[4 * e + 1];
          f[4 * e + 2] = wa * prev.z + wb * f[4 * e + 2];
          f[4 * e + 3] = wa * prev.w + wb * f[4 * e + 3];
          if (!final_out) ap[e] = make_float4(f[4 * e], f[4 * e + 1], f[4 * e + 2], f[4 * e + 3]);
        }
      }
      if (final_out) {
        uint4 *dst = reinterpret_cast<uint4 *>(og + c * 32);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          dst[e] = make_uint4(pack_bf16(f[8 * e], f[8 * e + 1]), pack_bf16(f[8 * e + 2], f[8 * e + 3]),
                              pack_bf16(f[8 * e + 4], f[8 * e + 5]),
                              pack_bf16(f[8 * e + 6], f[8 * e + 7]));
      }
    }
    if (valid && final_out)
      (is_main ? a.lse_m : a.lse_b)[(int64_t)h * rows_total + row0 + row] = lse;
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, 512);
}

// ============================================================================
// Two-head forward: the CTA takes two q heads of one kv group for the same
// query tile.  Both share every K / V tile.  Two softmax warpgroups (A, B)
// alternate with the tensor core:
//   S_A(0) S_B(0) | PV_A(0) S_A(1) PV_B(0) S_B(1) | PV_A(1) S_A(2) PV_B(1) ...
// so one group's softmax overlaps the other group's MMAs.  TMEM: S_A, S_B,
// O_A, O_B; each P (bf16 pairs) is written over the S it came from.  PV_X(j-1)
// is issued before S_X(j), so when a softmax thread sees S_X(j) its O row is
// stable and can be rescaled without a further wait.
// ============================================================================
constexpr int kFwd2Stages = 2;

template <int D>
struct Fwd2Smem {
  bf16 q[2][128 * D];
  bf16 k[kFwd2Stages][128 * D];
  bf16 v[kFwd2Stages][128 * D];
  uint64_t bar_q;
  uint64_t bar_k_full[kFwd2Stages], bar_k_empty[kFwd2Stages];
  uint64_t bar_v_full[kFwd2Stages], bar_v_empty[kFwd2Stages];
  uint64_t bar_s_full[2], bar_p_full[2];
  uint64_t bar_o_final;
  uint64_t bar_drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
__global__ void __launch_bounds__(384, 1)
    fwd2_sm100_kernel(const AttnParams a, const __grid_constant__ TensorMaps tm) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  Fwd2Smem<D> &sm = *reinterpret_cast<Fwd2Smem<D> *>(smem_raw + (((raw + 1023) & ~1023u) - raw));
  if (a.plan.status[0] != 0) return;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int pairs = a.hq / 2;
  const int t = a.plan.fwd_order[blockIdx.x / pairs];
  const int h0 = 2 * (blockIdx.x % pairs);
  const int g = h0 / (a.hq / a.hkv);
  const bool is_main = t < a.n_qt_main;
  const int tt = is_main ? t : t - a.n_qt_main;
  const int rows_total = is_main ? a.n_main : a.n_bt;
  const int row0 = tt * 128;
  const int nrows = min(128, rows_total - row0);
  const int row_off = is_main ? 0 : a.n_main;
  const TileSegs segs = make_segs(a, t, is_main);
  const int total = segs.total;
  int *status_word = a.plan.status + 1;
  volatile int *abort_flag = &sm.abort_flag;

  const uint32_t b_q = smem_u32(&sm.bar_q), b_final = smem_u32(&sm.bar_o_final);
  if (threadIdx.x == 0) {
    mbar_init(b_q, 1);
    for (int s = 0; s < kFwd2Stages; ++s) {
      mbar_init(smem_u32(&sm.bar_k_full[s]), 1);
      mbar_init(smem_u32(&sm.bar_k_empty[s]), 1);
      mbar_init(smem_u32(&sm.bar_v_full[s]), 1);
      mbar_init(smem_u32(&sm.bar_v_empty[s]), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(smem_u32(&sm.bar_s_full[x]), 1);
      mbar_init(smem_u32(&sm.bar_p_full[x]), 128);
    }
    mbar_init(b_final, 1);
    mbar_init(smem_u32(&sm.bar_drain), 1);
    sm.abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&sm.tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  auto t_s = [&](int x) { return tmem + x * 128; };
  auto t_o = [&](int x) { return tmem + 256 + x * 128; };

  // warpgroup 0 (producer, MMA issuer, two idle warps) hands registers to
  // the two softmax warpgroups: 128 x 56 + 256 x 208 = 60416 <= 384 x 168
  if (warp < 4) {
    regs_dec<56>();
  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    const CUtensorMap *qmap = is_main ? &tm.q_m : &tm.q_b;
    if (total > 0) {
      mbar_expect_tx(b_q, 2 * 128 * D * 2);
#pragma unroll
      for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem_u32(sm.q[x]) + c * 16384, qmap, b_q, c * 64, h0 + x, row0);
    }
    int issued_k = 0, issued_v = 0;
    for (int j = 0; j < total; ++j) {
      const int st = j % kFwd2Stages;
      const uint32_t ph = ((j / kFwd2Stages) - 1) & 1;
      int key0, kind;
      bool full;
      segs.locate(j, key0, kind, full);
      if (j >= kFwd2Stages &&
          !mbar_wait(smem_u32(&sm.bar_k_empty[st]), ph, abort_flag, status_word, 1))
        break;
      const uint32_t kb = smem_u32(&sm.bar_k_full[st]);
      mbar_expect_tx(kb, 128 * D * 2);
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        tma_load_3d(smem_u32(sm.k[st]) + c * 16384, kind == 2 ? &tm.k_b : &tm.k_m, kb, c * 64, g,
                    key0);
      ++issued_k;
      if (j >= kFwd2Stages &&
          !mbar_wait(smem_u32(&sm.bar_v_empty[st]), ph, abort_flag, status_word, 1))
        break;
      const uint32_t vb = smem_u32(&sm.bar_v_full[st]);
      mbar_expect_tx(vb, 128 * D * 2);
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        tma_load_3d(smem_u32(sm.v[st]) + c * 16384, kind == 2 ? &tm.v_b : &tm.v_m, vb, c * 64, g,
                    key0);
      ++issued_v;
    }
    for (int j = (issued_k > kFwd2Stages ? issued_k - kFwd2Stages : 0); j < issued_k; ++j)
      mbar_wait_drain(smem_u32(&sm.bar_k_full[j % kFwd2Stages]), (j / kFwd2Stages) & 1, status_word, 2);
    for (int j = (issued_v > kFwd2Stages ? issued_v - kFwd2Stages : 0); j < issued_v; ++j)
      mbar_wait_drain(smem_u32(&sm.bar_v_full[j % kFwd2Stages]), (j / kFwd2Stages) & 1, status_word, 2);
    if (total > 0) mbar_wait_drain(b_q, 0, status_word, 2);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_qk = idesc_bf16(128, 128, false, false);
    constexpr uint32_t idesc_pv = idesc_bf16(128, D, false, true);
    bool ok = total == 0 || mbar_wait(b_q, 0, abort_flag, status_word, 3);
    auto issue_s = [&](int x, int j) -> bool {
      const int st = j % kFwd2Stages;
      if (x == 0 &&
          !mbar_wait(smem_u32(&sm.bar_k_full[st]), (j / kFwd2Stages) & 1, abort_flag, status_word, 5))
        return false;
      tc_fence_after();
      const uint64_t qd = sdesc(smem_u32(sm.q[x]), 16, 1024);
      const uint64_t kd = sdesc(smem_u32(sm.k[st]), 16, 1024);
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
        mma_bf16(t_s(x), desc_at(qd, off), desc_at(kd, off), idesc_qk, k > 0 ? 1u : 0u);
      }
      mma_commit(smem_u32(&sm.bar_s_full[x]));
      if (x == 1) mma_commit(smem_u32(&sm.bar_k_empty[st]));
      return true;
    };
    auto issue_pv = [&](int x, int i) -> bool {
      const int st = i % kFwd2Stages;
      if ((x == 0 && !mbar_wait(smem_u32(&sm.bar_v_full[st]), (i / kFwd2Stages) & 1, abort_flag,
                                status_word, 4)) ||
          !mbar_wait(smem_u32(&sm.bar_p_full[x]), i & 1, abort_flag, status_word, 4))
        return false;
      tc_fence_after();
      const uint64_t vd = sdesc(smem_u32(sm.v[st]), 16384, 1024);
#pragma unroll
      for (int k = 0; k < 8; ++k)
        mma_bf16_ts(t_o(x), t_s(x) + k * 8, desc_at(vd, k * 2048), idesc_pv,
                    (i > 0 || k > 0) ? 1u : 0u);
      if (x == 1) mma_commit(smem_u32(&sm.bar_v_empty[st]));
      return true;
    };
    if (ok && total > 0) ok = issue_s(0, 0) && issue_s(1, 0);
    for (int j = 0; ok && j < total; ++j) {
      // P_X(j) must be consumed before S_X(j+1) overwrites it: issue order
      ok = issue_pv(0, j) && (j + 1 >= total || issue_s(0, j + 1)) && issue_pv(1, j) &&
           (j + 1 >= total || issue_s(1, j + 1));
    }
    if (ok && total > 0) mma_commit(b_final);
    mma_commit(smem_u32(&sm.bar_drain));
    mbar_wait_drain(smem_u32(&sm.bar_drain), 0, status_word, 2);
  }
  } else {
    regs_inc<208>();
    // ------------------------------------------------------------ softmax A / B
    const int x = (warp - 4) / 4;  // 0 = head h0 (warps 4-7), 1 = head h0 + 1 (warps 8-11)
    const int h = h0 + x;
    const int row = (warp & 3) * 32 + lane;  // TMEM lane quarter = warp % 4
    const bool valid = row < nrows;
    const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
    int lo[3] = {0, 0, 0}, hi[3] = {-1, -1, -1};
    const int zz = a.zz_step;
    if (valid) {
      const int4 iv = reinterpret_cast<const int4 *>(a.plan.row_iv)[row_off + row0 + row];
      if (a.ring) {
        // ring mode: this step's main interval, or the branch-local one last
        if (zz < a.zz_C) { lo[0] = iv.x; hi[0] = iv.y; }
        else { lo[2] = iv.z; hi[2] = iv.w; }
      } else if (zz < 0 || zz == a.zz_C) {
        lo[0] = iv.x; hi[0] = iv.y;
        lo[2] = iv.z; hi[2] = iv.w;
      }
      if (!a.ring && zz >= 0 && zz < a.zz_C) {
        int s_lo = 0, s_hi = a.n_seqs;
        while (s_lo < s_hi) {
          const int mid = (s_lo + s_hi + 1) >> 1;
          if (a.cu_seqlens[mid] <= iv.x) s_lo = mid; else s_hi = mid - 1;
        }
        const int64_t L = a.cu_seqlens[s_lo + 1] - iv.x;
        const int64_t pos = iv.y - iv.x;
        const int C = a.zz_C;
        const int c = (int)((2 * C * (pos + 1) - 1) / L);
        const int shard = c < C ? c : 2 * C - 1 - c;
        const int jw = ((shard - zz) % C + C) % C;
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          const int ch = w == 0 ? jw : 2 * C - 1 - jw;
          lo[w] = max(iv.x + (int)((ch * L) / (2 * C)), iv.x);
          hi[w] = min(iv.x + (int)(((ch + 1) * L) / (2 * C)) - 1, iv.y);
        }
      }
    }
    const uint32_t b_s = smem_u32(&sm.bar_s_full[x]), b_p = smem_u32(&sm.bar_p_full[x]);
    const uint32_t ts = t_s(x) + lane_addr, to = t_o(x) + lane_addr;
    float m_used = kNegInf, l = 0.f;
    bool ok = true;
    const float sl2 = a.scale_log2;
    for (int j = 0; j < total; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(b_s, j & 1, abort_flag, status_word, 7))) {
        ok = false;
        break;
      }
      tc_fence_after();
      int key0, kind;
      bool full;
      segs.locate(j, key0, kind, full);
      const int clo = kind == 0 ? lo[0] : (kind == 1 ? lo[1] : lo[2]);
      const int chi = kind == 0 ? hi[0] : (kind == 1 ? hi[1] : hi[2]);
      float s[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(ts + c * 32, reinterpret_cast<uint32_t *>(s) + c * 32);
      tc_wait_ld();
      if (!(full && valid)) {
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const int key = key0 + c;
          if (key < clo || key > chi) s[c] = kNegInf;
        }
      }
      float mx4[4] = {kNegInf, kNegInf, kNegInf, kNegInf};
#pragma unroll
      for (int c = 0; c < 128; c += 8) {
#pragma unroll
        for (int e = 0; e < 4; ++e) mx4[e] = fmax3(mx4[e], s[c + e], s[c + 4 + e]);
      }
      const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * sl2;
      const float m_new = fmaxf(m_used, mx);
      const bool need = m_new > m_used + kRescaleThreshold;
      const float alpha = need ? ex2(m_used - m_new) : 1.f;
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        // PV_X(j-1) was issued before S_X(j) and has completed: O is stable
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(to + c * 32, o);
          tc_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(to + c * 32, o);
        }
      }
      if (need) {
        l *= alpha;
        m_used = m_new;
      }
      const float msub = m_used == kNegInf ? 0.f : m_used;
      // P = 2^(s sl2 - m), packed to bf16 pairs in place, written over the
      // first 64 columns of this head's S (all of S is in registers now)
      uint32_t *pk = reinterpret_cast<uint32_t *>(s);
      // scale and shift, and the row sums, on fp32 pairs
      const uint64_t sl2x2 = f2_pack(sl2, sl2), negm = f2_pack(-msub, -msub);
      uint64_t l01 = f2_pack(0.f, 0.f), l23 = f2_pack(0.f, 0.f);
#pragma unroll
      for (int c = 0; c < 128; c += 4) {
        float pv[4], x[4];
        f2_unpack(f2_fma(f2_pack(s[c], s[c + 1]), sl2x2, negm), x[0], x[1]);
        f2_unpack(f2_fma(f2_pack(s[c + 2], s[c + 3]), sl2x2, negm), x[2], x[3]);
#pragma unroll
        for (int e = 0; e < 4; ++e) pv[e] = ex2(x[e]);
        l01 = f2_add(l01, f2_pack(pv[0], pv[1]));
        l23 = f2_add(l23, f2_pack(pv[2], pv[3]));
        pk[c / 2] = pack_bf16(pv[0], pv[1]);
        pk[c / 2 + 1] = pack_bf16(pv[2], pv[3]);
      }
      tmem_st32(ts, pk);
      tmem_st32(ts + 32, pk + 32);
      float l4[4];
      f2_unpack(l01, l4[0], l4[1]);
      f2_unpack(l23, l4[2], l4[3]);
      l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(b_p);
    }
    if (ok && total > 0 &&
        !__all_sync(0xffffffffu, mbar_wait(b_final, 0, abort_flag, status_word, 9)))
      ok = false;
    tc_fence_after();

    // ------------------------------------------------------------ epilogue
    const bool empty = !(l > 0.f) || m_used == kNegInf;
    float lse = empty ? kNegInf : (m_used + __log2f(l)) * kLn2;
    const float inv = empty ? 0.f : 1.f / l;
    const bool final_out = zz < 0 || zz == a.zz_C;
    float wa = 0.f, wb = 1.f;
    float *acc = nullptr;
    if (zz >= 0 && valid) {
      const int64_t all_rows = (int64_t)a.n_main + a.n_bt;
      const int64_t grow = row_off + row0 + row;
      acc = a.zz_o + (grow * a.hq + h) * D;
      float *accl = a.zz_lse + (int64_t)h * all_rows + grow;
      float lnew = lse;
      if (zz > 0) {
        const float la = *accl;
        const float mm = fmaxf(la, lse);
        if (mm == kNegInf) {
          lnew = kNegInf; wa = 0.f; wb = 0.f;
        } else {
          lnew = mm + logf(expf(la - mm) + expf(lse - mm));
          wa = expf(la - lnew);
          wb = expf(lse - lnew);
        }
      }
      if (!final_out) *accl = lnew;
      lse = lnew;
    }
    bf16 *og = (is_main ? a.o_m : a.o_b) + ((int64_t)(row0 + row) * a.hq + h) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      if (ok && total > 0) {
        tmem_ld32(to + c * 32, o);
        tc_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = 0u;
      }
      if (!valid) continue;
      float f[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(o[e]) * inv;
      if (zz >= 0) {
        float4 *ap = reinterpret_cast<float4 *>(acc + c * 32);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float4 prev = zz > 0 ? ap[e] : make_float4(0.f, 0.f, 0.f, 0.f);
          f[4 * e + 0] = wa * prev.x + wb * f[4 * e + 0];
          f[4 * e + 1] = wa * prev.y + wb * f[4 * e + 1];
          f[4 * e + 2] = wa * prev.z + wb * f[4 * e + 2];
          f[4 * e + 3] = wa * prev.w + wb * f[4 * e + 3];
          if (!final_out) ap[e] = make_float4(f[4 * e], f[4 * e + 1], f[4 * e + 2], f[4 * e + 3]);
        }
      }
      if (final_out) {
        uint4 *dst = reinterpret_cast<uint4 *>(og + c * 32);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          dst[e] = make_uint4(pack_bf16(f[8 * e], f[8 * e + 1]), pack_bf16(f[8 * e + 2], f[8 * e + 3]),
                              pack_bf16(f[8 * e + 4], f[8 * e + 5]),
                              pack_bf16(f[8 * e + 6], f[8 * e + 7]));
      }
    }
    if (valid && final_out)
      (is_main ? a.lse_m : a.lse_b)[(int64_t)h * rows_total + row0 + row] = lse;
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

__global__ void exp2_check_kernel(const float *x, float *y_fma, float *y_mufu, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    y_fma[i] = exp2_fma(x[i]);
    y_mufu[i] = ex2(x[i]);
  }
}

}  // namespace

ba_status launch_exp2_check(const float *x, float *y_fma, float *y_mufu, int64_t n,
                            cudaStream_t s) {
  if (n <= 0) return BA_OK;
  const int64_t blocks = (n + 255) / 256;
  exp2_check_kernel<<<(unsigned)(blocks < 4096 ? blocks : 4096), 256, 0, s>>>(x, y_fma, y_mufu, n);
  count_launches(1);
  return cuda_check(cudaGetLastError(), "exp2_check_kernel launch");
}


ba_status launch_fwd_sm100(const AttnParams &a, cudaStream_t s) {
  TensorMaps tm = {};
  const int d = a.head_dim;
  ba_status st;
  // a ring step reads only the visiting shard's main K/V; the ring's last
  // step only the local branch K/V; maps that a launch never reads alias one
  // that it does
  const bool need_main_kv = !(a.ring && a.zz_step == a.zz_C);
  const bool need_branch_kv = a.n_bt > 0 && !(a.ring && a.zz_step < a.zz_C);
  if ((st = make_tensor_map(&tm.q_m, a.q_m, a.n_main, a.hq, d, 128)) != BA_OK) return st;
  if (a.n_bt > 0) {
    if ((st = make_tensor_map(&tm.q_b, a.q_b, a.n_bt, a.hq, d, 128)) != BA_OK) return st;
  } else {
    tm.q_b = tm.q_m;
  }
  if (need_main_kv) {
    if ((st = make_tensor_map(&tm.k_m, a.k_m, a.n_keys_m, a.hkv, d, 128)) != BA_OK) return st;
    if ((st = make_tensor_map(&tm.v_m, a.v_m, a.n_keys_m, a.hkv, d, 128)) != BA_OK) return st;
  }
  if (need_branch_kv) {
    if ((st = make_tensor_map(&tm.k_b, a.k_b, a.n_bt, a.hkv, d, 128)) != BA_OK) return st;
    if ((st = make_tensor_map(&tm.v_b, a.v_b, a.n_bt, a.hkv, d, 128)) != BA_OK) return st;
  }
  if (!need_main_kv) { tm.k_m = tm.k_b; tm.v_m = tm.v_b; }
  if (!need_branch_kv) { tm.k_b = tm.k_m; tm.v_b = tm.v_m; }
  const int64_t grid = (int64_t)a.n_qt * a.hq;
  if (grid == 0) return BA_OK;
  cudaError_t e;
  if ((a.hq / a.hkv) % 2 == 0) {
    // two heads of one kv group per CTA
    const int64_t grid2 = (int64_t)a.n_qt * (a.hq / 2);
    if (d == 64) {
      const size_t smem = sizeof(Fwd2Smem<64>) + 1024;
      e = cudaFuncSetAttribute(fwd2_sm100_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem);
      if (e != cudaSuccess) return cuda_check(e, "fwd2_sm100_kernel<64> smem");
      fwd2_sm100_kernel<64><<<(unsigned)grid2, 384, smem, s>>>(a, tm);
    } else {
      const size_t smem = sizeof(Fwd2Smem<128>) + 1024;
      e = cudaFuncSetAttribute(fwd2_sm100_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem);
      if (e != cudaSuccess) return cuda_check(e, "fwd2_sm100_kernel<128> smem");
      fwd2_sm100_kernel<128><<<(unsigned)grid2, 384, smem, s>>>(a, tm);
    }
    count_launches(1);
    return cuda_check(cudaGetLastError(), "fwd2_sm100_kernel launch");
  }
  if (d == 64) {
    const size_t smem = sizeof(FwdSmem<64>) + 1024;
    e = cudaFuncSetAttribute(fwd_sm100_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return cuda_check(e, "fwd_sm100_kernel<64> smem");
    fwd_sm100_kernel<64><<<(unsigned)grid, 256, smem, s>>>(a, tm);
  } else {
    const size_t smem = sizeof(FwdSmem<128>) + 1024;
    e = cudaFuncSetAttribute(fwd_sm100_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return cuda_check(e, "fwd_sm100_kernel<128> smem");
    fwd_sm100_kernel<128><<<(unsigned)grid, 256, smem, s>>>(a, tm);
  }
  count_launches(1);
  return cuda_check(cudaGetLastError(), "fwd_sm100_kernel launch");
}


}  // namespace ba
