// Backward of branch attention on the tcgen05 tensor cores (sm_100a).
//
// Given the merged LSE l of every query (written by the forward) and
// D = rowsum(dO * O), every visible (query i, key k) pair has
//   P_ik = exp(scale q_i.k_k - l_i),  dS_ik = P_ik (dO_i.v_k - D_i),
// and the gradients are dV_k = sum_i P_ik dO_i, dK_k = scale sum_i dS_ik q_i,
// dQ_i = scale sum_k dS_ik k_k.  P is recomputed from the merged LSE, so the
// main-prefix and branch-local parts of a branch query share one softmax
// normalisation, as the paper's merge rule makes them
// ("Online Draft Co-Training", technical-contribution section).
//
// Two kernels, neither with atomics:
//   dq_sm100_kernel    query-stationary (one CTA per 128-row query tile and q
//                      head, the forward's work order): per key tile S and dP
//                      into TMEM, dS by 512 threads (four per row) written back
//                      to TMEM as bf16, dQ += dS K (A operand from TMEM)
//                      accumulated in TMEM; K and V come through separate
//                      rings so V is refilled as soon as dP is done.  S / dP
//                      and dQ are issued by two threads, so waiting for one
//                      stream's inputs never holds back the other's MMAs.
//   dkdv_sm100_kernel  key-stationary (one CTA per 128-row key tile and kv
//                      head, the plan's backward work order): over every
//                      128-row query tile of every q head of the group that
//                      visits the tile, S^T = K Q^T and dP^T = V dO^T into
//                      TMEM (N = 128: the tensor cores' full rate), P^T and
//                      dS^T written over dP^T as bf16, dV += P^T dO and
//                      dK += dS^T Q (A operands from TMEM) accumulated in TMEM
//                      for the whole walk.  Q (three deep) and dO (two deep)
//                      come through separate rings, each freed by the product
//                      that reads it last; per-query records {LSE, D} arrive by
//                      bulk copy with dO; each key thread masks with the plan's
//                      range of query rows that see its key.
#include "attn_sm100_common.cuh"

namespace ba {
namespace {

using namespace sm100;

// ============================================================================
// dQ kernel
// ============================================================================
constexpr int kDqKStages = 3;  // K is read twice (S, then dQ): deeper ring
constexpr int kDqVStages = 2;  // V is free as soon as dP is computed

template <int D>
struct DqSmem {
  bf16 q[128 * D];
  bf16 dout[128 * D];
  bf16 k[kDqKStages][128 * D];
  bf16 v[kDqVStages][128 * D];
  uint64_t bar_qdo;
  uint64_t bar_k_full[kDqKStages], bar_k_empty[kDqKStages];
  uint64_t bar_v_full[kDqVStages], bar_v_empty[kDqVStages];
  uint64_t bar_sdp_full, bar_sdp_empty;
  uint64_t bar_ds_full[2];  // one per dS buffer: the dS threads may run a tile ahead
  uint64_t bar_dq_done[2];  // dQ(i) has read dS buffer i % 2
  uint64_t bar_dq_final;
  uint64_t bar_drain[2];    // per issuing thread: its queued MMAs have completed
  uint32_t tmem_base;
  int abort_flag;
};

struct DqMaps {
  TensorMaps t;
  CUtensorMap do_m, do_b;
};

// TMEM columns: S [0, 128), dP [128, 256), dQ [256, 256 + D), dS (bf16 pairs)
// double-buffered at 384 and 448.  608 threads: warp 0 producer, warp 1 S / dP
// issuer, warp 2 TMEM owner and dQ issuer, warps 3-18 dS, four threads per
// query row (warp w reaches TMEM lanes 32 (w % 4) .., key quarter
// (w - 3) / 4 of the tile).
constexpr int kDqThreads = 608;
constexpr int kDqElem = kDqThreads - 96;

template <int D>
__global__ void __launch_bounds__(kDqThreads, 1)
    dq_sm100_kernel(const AttnParams a, const __grid_constant__ DqMaps tm) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  DqSmem<D> &sm = *reinterpret_cast<DqSmem<D> *>(smem_raw + (((raw + 1023) & ~1023u) - raw));
  if (a.plan.status[0] != 0) return;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int t = a.plan.fwd_order[blockIdx.x / a.hq];
  const int h = blockIdx.x % a.hq;
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

  const uint32_t b_qdo = smem_u32(&sm.bar_qdo);
  const uint32_t b_sdp_full = smem_u32(&sm.bar_sdp_full), b_sdp_empty = smem_u32(&sm.bar_sdp_empty);
  const uint32_t b_final = smem_u32(&sm.bar_dq_final);
  if (threadIdx.x == 0) {
    mbar_init(b_qdo, 1);
    for (int s = 0; s < kDqKStages; ++s) {
      mbar_init(smem_u32(&sm.bar_k_full[s]), 1);
      mbar_init(smem_u32(&sm.bar_k_empty[s]), 1);
    }
    for (int s = 0; s < kDqVStages; ++s) {
      mbar_init(smem_u32(&sm.bar_v_full[s]), 1);
      mbar_init(smem_u32(&sm.bar_v_empty[s]), 1);
    }
    mbar_init(b_sdp_full, 1);
    mbar_init(b_sdp_empty, kDqElem);
    mbar_init(smem_u32(&sm.bar_ds_full[0]), kDqElem);
    mbar_init(smem_u32(&sm.bar_ds_full[1]), kDqElem);
    mbar_init(smem_u32(&sm.bar_dq_done[0]), 1);
    mbar_init(smem_u32(&sm.bar_dq_done[1]), 1);
    mbar_init(b_final, 1);
    mbar_init(smem_u32(&sm.bar_drain[0]), 1);
    mbar_init(smem_u32(&sm.bar_drain[1]), 1);
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
  const uint32_t t_s = tmem, t_dp = tmem + 128, t_dq = tmem + 256;
  auto t_ds = [&](int b) { return tmem + 384 + b * 64; };

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    if (total > 0) {
      mbar_expect_tx(b_qdo, 2 * 128 * D * 2);
      const CUtensorMap *qm = is_main ? &tm.t.q_m : &tm.t.q_b;
      const CUtensorMap *dm = is_main ? &tm.do_m : &tm.do_b;
#pragma unroll
      for (int x = 0; x < D / 64; ++x) {
        tma_load_3d(smem_u32(sm.q) + x * 16384, qm, b_qdo, x * 64, h, row0);
        tma_load_3d(smem_u32(sm.dout) + x * 16384, dm, b_qdo, x * 64, h, row0);
      }
    }
    int issued_k = 0, issued_v = 0;
    for (int j = 0; j < total; ++j) {
      int key0, kind;
      bool full;
      segs.locate(j, key0, kind, full);
      const int ks = j % kDqKStages, vs = j % kDqVStages;
      if (j >= kDqKStages && !mbar_wait(smem_u32(&sm.bar_k_empty[ks]),
                                        ((j / kDqKStages) - 1) & 1, abort_flag, status_word, 1))
        break;
      const uint32_t kb = smem_u32(&sm.bar_k_full[ks]);
      mbar_expect_tx(kb, 128 * D * 2);
#pragma unroll
      for (int x = 0; x < D / 64; ++x)
        tma_load_3d(smem_u32(sm.k[ks]) + x * 16384, kind == 2 ? &tm.t.k_b : &tm.t.k_m, kb, x * 64,
                    g, key0);
      ++issued_k;
      if (j >= kDqVStages && !mbar_wait(smem_u32(&sm.bar_v_empty[vs]),
                                        ((j / kDqVStages) - 1) & 1, abort_flag, status_word, 1))
        break;
      const uint32_t vb = smem_u32(&sm.bar_v_full[vs]);
      mbar_expect_tx(vb, 128 * D * 2);
#pragma unroll
      for (int x = 0; x < D / 64; ++x)
        tma_load_3d(smem_u32(sm.v[vs]) + x * 16384, kind == 2 ? &tm.t.v_b : &tm.t.v_m, vb, x * 64,
                    g, key0);
      ++issued_v;
    }
    for (int j = (issued_k > kDqKStages ? issued_k - kDqKStages : 0); j < issued_k; ++j)
      mbar_wait_drain(smem_u32(&sm.bar_k_full[j % kDqKStages]), (j / kDqKStages) & 1, status_word, 2);
    for (int j = (issued_v > kDqVStages ? issued_v - kDqVStages : 0); j < issued_v; ++j)
      mbar_wait_drain(smem_u32(&sm.bar_v_full[j % kDqVStages]), (j / kDqVStages) & 1, status_word, 2);
    if (total > 0) mbar_wait_drain(b_qdo, 0, status_word, 2);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ S / dP issuer
    // Two issuing threads: this one issues S and dP of each key tile, warp 2
    // the dQ products.  An mbarrier wait holds the thread that executes it
    // until the MMAs it has queued are done, so one issuer waiting for dS
    // would keep the next tile's S / dP out of the tensor pipe (and waiting
    // for the next K / V would hold back dQ); split, each waits only on its
    // own inputs.
    constexpr uint32_t idesc_s = idesc_bf16(128, 128, false, false);
    const uint64_t qd0 = sdesc(smem_u32(sm.q), 16, 1024), dod0 = sdesc(smem_u32(sm.dout), 16, 1024);
    bool ok = total == 0 || mbar_wait(b_qdo, 0, abort_flag, status_word, 3);
    for (int j = 0; ok && j < total; ++j) {
      const int ks = j % kDqKStages, vs = j % kDqVStages;
      if (!mbar_wait(smem_u32(&sm.bar_k_full[ks]), (j / kDqKStages) & 1, abort_flag, status_word,
                     5) ||
          !mbar_wait(smem_u32(&sm.bar_v_full[vs]), (j / kDqVStages) & 1, abort_flag, status_word,
                     5) ||
          (j >= 1 && !mbar_wait(b_sdp_empty, (j - 1) & 1, abort_flag, status_word, 6))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint64_t kd = sdesc(smem_u32(sm.k[ks]), 16, 1024);
      const uint64_t vd = sdesc(smem_u32(sm.v[vs]), 16, 1024);
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
        mma_bf16(t_s, desc_at(qd0, off), desc_at(kd, off), idesc_s, k > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
        mma_bf16(t_dp, desc_at(dod0, off), desc_at(vd, off), idesc_s, k > 0 ? 1u : 0u);
      }
      mma_commit(b_sdp_full);
      mma_commit(smem_u32(&sm.bar_v_empty[vs]));
    }
    mma_commit(smem_u32(&sm.bar_drain[0]));
    mbar_wait_drain(smem_u32(&sm.bar_drain[0]), 0, status_word, 2);
  } else if (warp == 2 && lane == 0) {
    // ------------------------------------------------------------ dQ issuer
    // dQ(i) += dS(i) K(i).  K(i) is released here: S(i) read it before the
    // dS threads could finish tile i.
    constexpr uint32_t idesc_dq = idesc_bf16(128, D, false, true);
    bool ok = true;
    for (int i = 0; ok && i < total; ++i) {
      if (!mbar_wait(smem_u32(&sm.bar_ds_full[i & 1]), (i >> 1) & 1, abort_flag, status_word, 4)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint64_t kd = sdesc(smem_u32(sm.k[i % kDqKStages]), 16384, 1024);
#pragma unroll
      for (int k = 0; k < 8; ++k)
        mma_bf16_ts(t_dq, t_ds(i & 1) + k * 8, desc_at(kd, k * 2048), idesc_dq,
                    (i > 0 || k > 0) ? 1u : 0u);
      mma_commit(smem_u32(&sm.bar_k_empty[i % kDqKStages]));
      mma_commit(smem_u32(&sm.bar_dq_done[i & 1]));
    }
    if (ok && total > 0) mma_commit(b_final);
    mma_commit(smem_u32(&sm.bar_drain[1]));
    mbar_wait_drain(smem_u32(&sm.bar_drain[1]), 0, status_word, 2);
  } else if (warp >= 3) {
    // ------------------------------------------------------------ dS (4 threads / row)
    const int qq = (warp - 3) >> 2;  // key quarter [32 qq, 32 qq + 32) of each tile
    const int row = (warp & 3) * 32 + lane;
    const bool valid = row < nrows;
    const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
    int lo0 = 0, hi0 = -1, lo2 = 0, hi2 = -1;
    float lse2 = 0.f, dd = 0.f;
    if (valid) {
      const int4 iv = reinterpret_cast<const int4 *>(a.plan.row_iv)[row_off + row0 + row];
      lo0 = iv.x; hi0 = iv.y; lo2 = iv.z; hi2 = iv.w;
      lse2 = (is_main ? a.lse_m : a.lse_b)[(int64_t)h * rows_total + row0 + row] * kLog2e;
      dd = a.d_all[(int64_t)h * ((int64_t)a.n_main + a.n_bt) + row_off + row0 + row];
    }
    bool ok = true;
    for (int j = 0; j < total; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(b_sdp_full, j & 1, abort_flag, status_word, 7))) {
        ok = false;
        break;
      }
      tc_fence_after();
      int key0, kind;
      bool full;
      segs.locate(j, key0, kind, full);
      const int clo = kind == 2 ? lo2 : lo0, chi = kind == 2 ? hi2 : hi0;
      float s[32], dp[32];
      tmem_ld32(t_s + lane_addr + qq * 32, reinterpret_cast<uint32_t *>(s));
      tmem_ld32(t_dp + lane_addr + qq * 32, reinterpret_cast<uint32_t *>(dp));
      tc_wait_ld();
      tc_fence_before();
      mbar_arrive(b_sdp_empty);
      const int kbase = key0 + qq * 32;
      // masked scores -> -inf only on partial tiles, then P = 2^(s sl2 - l2)
      // branch-free; dS packed to bf16 pairs in place (entry c/2 after c, c+1)
      if (!(full && valid)) {
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int key = kbase + c;
          if (key < clo || key > chi) s[c] = kNegInf;
        }
      }
      const float sl2 = a.scale_log2;
      const uint64_t sl2x2 = f2_pack(sl2, sl2), nl2 = f2_pack(-lse2, -lse2), dd2 = f2_pack(dd, dd);
      uint32_t *pk = reinterpret_cast<uint32_t *>(dp);
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        float x0, x1, d0, d1;
        f2_unpack(f2_fma(f2_pack(s[c], s[c + 1]), sl2x2, nl2), x0, x1);
        f2_unpack(f2_mul(f2_pack(ex2(x0), ex2(x1)), f2_sub(f2_pack(dp[c], dp[c + 1]), dd2)), d0, d1);
        pk[c / 2] = pack_bf16(d0, d1);
      }
      // dS buffer j&1 was last read by dQ_{j-2}
      if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.bar_dq_done[j & 1]),
                                                      ((j - 2) >> 1) & 1, abort_flag,
                                                      status_word, 8))) {
        ok = false;
        break;
      }
      tc_fence_after();
      tmem_st16(t_ds(j & 1) + lane_addr + qq * 16, pk);
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&sm.bar_ds_full[j & 1]));
    }
    if (ok && total > 0 &&
        !__all_sync(0xffffffffu, mbar_wait(b_final, 0, abort_flag, status_word, 9)))
      ok = false;
    tc_fence_after();
    // each of the four threads of a row stores a quarter of its dQ
    constexpr int kCols = D / 4;
    bf16 *dst = (is_main ? a.dq_out_m : a.dq_out_b) + ((int64_t)(row0 + row) * a.hq + h) * D +
                qq * kCols;
    uint32_t o[kCols];
    if (ok && total > 0) {
      if constexpr (kCols == 32) tmem_ld32(t_dq + lane_addr + qq * kCols, o);
      else tmem_ld16(t_dq + lane_addr + qq * kCols, o);
      tc_wait_ld();
    } else {
#pragma unroll
      for (int e = 0; e < kCols; ++e) o[e] = 0u;
    }
    if (valid) {
      uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
      for (int e = 0; e < kCols / 8; ++e)
        d4[e] = make_uint4(
            pack_bf16(__uint_as_float(o[8 * e]) * a.scale, __uint_as_float(o[8 * e + 1]) * a.scale),
            pack_bf16(__uint_as_float(o[8 * e + 2]) * a.scale,
                      __uint_as_float(o[8 * e + 3]) * a.scale),
            pack_bf16(__uint_as_float(o[8 * e + 4]) * a.scale,
                      __uint_as_float(o[8 * e + 5]) * a.scale),
            pack_bf16(__uint_as_float(o[8 * e + 6]) * a.scale,
                      __uint_as_float(o[8 * e + 7]) * a.scale));
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) {
    __syncwarp();  // lane 0 comes back from the dQ issuer's loop
    tmem_dealloc(tmem, 512);
  }
}

// ============================================================================
// dK / dV kernel
// ============================================================================
// Q(c + 1) is read by S^T(c + 1), issued right after dV(c); Q(c - 1), whose
// stage it would take in a two-deep ring, is freed only by dK(c - 1): three deep.
constexpr int kQStages = 3;
constexpr int kDoStages = 2;  // dO + records ring (freed once dK of the chunk, after its dS work, is issued)

template <int D>
struct DkvSmem {
  bf16 k[128 * D];
  bf16 v[128 * D];
  bf16 q[kQStages][kQc * D];      // D/64 boxes of [128 rows][64], 16 KB each
  bf16 dout[kDoStages][kQc * D];
  alignas(16) float rec[kDoStages][2 * kQc];  // LSE log2 [128], D [128]
  int4 chunk[kDoStages];          // {no mask needed, branch query tile, first query row}
  uint64_t bar_kv;
  uint64_t bar_q_full[kQStages], bar_q_empty[kQStages];
  uint64_t bar_do_full[kDoStages], bar_do_empty[kDoStages];
  uint64_t bar_s_full, bar_dp_full, bar_p_ready, bar_ds_ready;
  uint64_t bar_acc_done;
  uint64_t bar_drain;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(DkvSmem<128>) <= 232448, "dK/dV kernel exceeds 227 KB of shared memory");

// TMEM columns: dK [0, D), dV [D, 2D), X = S^T at 2D, Y = dP^T at 2D + 128
// (128 columns each).  Four threads per key row, one per query quarter
// [32 qq, 32 qq + 32) (16 warps; warp w reaches TMEM lanes 32 (w % 4) ..).
// Each thread writes only over the 32 columns of X and Y it has read itself:
// P^T (bf16 pairs, 16 columns) over its S^T quarter in X as soon as the
// exponentials are done, dS^T over its dP^T quarter in Y once dP^T is there.
// K-step k (queries 16k..16k+15) of the dV product reads P^T at
// X + 32 (k / 2) + 8 (k % 2), that of the dK product dS^T at the same offset
// in Y.  So dV(c) waits only for the exponentials of chunk c, not for dP^T(c)
// and the dS work: issue order per chunk dV(c), S^T(c+1), dK(c), dP^T(c+1),
// and the dS work of chunk c runs under dV(c) and S^T(c+1).
// 576 threads: warp 0 producer, warp 1 MMA issuer, warps 2-17 P^T / dS^T.
constexpr int kDkvThreads = 576;
constexpr int kDkvElem = kDkvThreads - 64;   // P^T / dS^T threads

template <int D>
__global__ void __launch_bounds__(kDkvThreads, 1)
    dkdv_sm100_kernel(const AttnParams a, const __grid_constant__ DkvMaps tm) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  DkvSmem<D> &sm = *reinterpret_cast<DkvSmem<D> *>(smem_raw);
  if (a.plan.status[0] != 0) return;
  int *status_word = a.plan.status + 1;
  // the 128-byte swizzled tiles need 1024-byte aligned shared memory; the
  // layout has no room for padding, so refuse (status bit 14) instead
  if ((smem_u32(smem_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicOr(status_word, 1 << 14);
    return;
  }

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // Launch order: the plan's longest-first key tiles in bands of one CTA per
  // SM.  A band runs kv group by kv group, so that a wave is one kv group's
  // key tiles, which walk the same q heads' query tiles and share their Q /
  // dO tiles in L2.  That starts the band's longest walk of the last kv group
  // after the walk ahead of the band and (hkv-1)/hkv of the band's own, spread
  // over the SMs; where it would then end more than a quarter past the
  // launch's balanced end (hkv * walk / n_sms), the band keeps the kv groups
  // of a key tile side by side instead, longest walks first.
  const int n_items = a.n_kt + a.n_bkt;
  const int band = a.n_sms;
  const int per_band = band * a.hkv;
  const int b0 = (int)(blockIdx.x / per_band) * band;       // first item of this band
  const int width = min(band, n_items - b0);                  // items in this band
  const int in_band = (int)(blockIdx.x % per_band);
  const int64_t walk = a.plan.status[2];
  const int64_t ahead = a.plan.bwd_prefix[b0];
  const int64_t next = b0 + 1 < n_items ? a.plan.bwd_prefix[b0 + 1] : walk;
  const int64_t end = b0 + width < n_items ? a.plan.bwd_prefix[b0 + width] : walk;
  const int item_g = a.plan.bwd_order[b0 + in_band % width];
  const int item_k = a.plan.bwd_order[b0 + in_band / a.hkv];
  const int64_t finish = a.hkv * ahead + (a.hkv - 1) * (end - ahead) + (int64_t)a.n_sms * (next - ahead);
  const bool by_group = 4 * finish <= 5 * (int64_t)a.hkv * walk;
  const int g = by_group ? in_band / width : in_band % a.hkv;
  const int item = by_group ? item_g : item_k;
  const bool main_kv = item < a.n_kt;
  const int kt = main_kv ? item : item - a.n_kt;
  const int key0 = kt * 128;
  const int n_keys = main_kv ? a.n_main : a.n_bt;
  const ChunkWalk cw = make_walk(a, main_kv, kt, g);
  const int total = cw.grp * (cw.n_t0 + cw.n_t1);
  volatile int *abort_flag = &sm.abort_flag;

  const uint32_t b_kv = smem_u32(&sm.bar_kv), b_acc = smem_u32(&sm.bar_acc_done);
  const uint32_t b_s = smem_u32(&sm.bar_s_full), b_pr = smem_u32(&sm.bar_p_ready);
  const uint32_t b_dp = smem_u32(&sm.bar_dp_full), b_dsr = smem_u32(&sm.bar_ds_ready);
  if (threadIdx.x == 0) {
    mbar_init(b_kv, 1);
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(smem_u32(&sm.bar_q_full[s]), 1);
      mbar_init(smem_u32(&sm.bar_q_empty[s]), 1);
    }
    for (int s = 0; s < kDoStages; ++s) {
      mbar_init(smem_u32(&sm.bar_do_full[s]), 1);
      mbar_init(smem_u32(&sm.bar_do_empty[s]), 1);
    }
    mbar_init(b_s, 1);
    mbar_init(b_pr, kDkvElem);
    mbar_init(b_dp, 1);
    mbar_init(b_dsr, kDkvElem);
    mbar_init(b_acc, 1);
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
  const uint32_t t_dk = tmem, t_dv = tmem + D, t_x = tmem + 2 * D, t_y = tmem + 2 * D + 128;

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
    int q_issued = 0, do_issued = 0;
    for (int c = 0; c < total; ++c) {
      int h, tile, nrows;
      bool is_main_q;
      cw.at(c, a, h, is_main_q, tile, nrows);
      const int row0 = tile * kQc;
      const int st = c % kQStages, ds = c % kDoStages;
      if (c >= kQStages &&
          !mbar_wait(smem_u32(&sm.bar_q_empty[st]), ((c / kQStages) - 1) & 1, abort_flag,
                     status_word, 1))
        break;
      const uint32_t qbar = smem_u32(&sm.bar_q_full[st]);
      mbar_expect_tx(qbar, kQc * D * 2);
      const CUtensorMap *qm = is_main_q ? &tm.t.q_m : &tm.t.q_b;
#pragma unroll
      for (int x = 0; x < D / 64; ++x)
        tma_load_3d(smem_u32(sm.q[st]) + x * 16384, qm, qbar, x * 64, h, row0);
      ++q_issued;
      if (c >= kDoStages &&
          !mbar_wait(smem_u32(&sm.bar_do_empty[ds]), ((c / kDoStages) - 1) & 1, abort_flag,
                     status_word, 1))
        break;
      // a chunk whose every query sees every key of this tile needs no mask;
      // the chunk's description travels with the stage (published by the
      // arrive below)
      bool full = false;
      if (main_kv) {
        const int32_t *qt =
            a.plan.qtile + (int64_t)(is_main_q ? tile : a.n_qt_main + tile) * 6;
        full = nrows == kQc && kt >= qt[1] && kt < qt[2];
      }
      sm.chunk[ds] = make_int4(full ? 1 : 0, is_main_q ? 0 : 1, row0, 0);
      const uint32_t dbar = smem_u32(&sm.bar_do_full[ds]);
      mbar_expect_tx(dbar, kQc * D * 2 + kQc * 8);
      const CUtensorMap *dm = is_main_q ? &tm.do_m : &tm.do_b;
#pragma unroll
      for (int x = 0; x < D / 64; ++x)
        tma_load_3d(smem_u32(sm.dout[ds]) + x * 16384, dm, dbar, x * 64, h, row0);
      const int64_t prow = (is_main_q ? 0 : a.n_main_pad) + row0;
      bulk_load(smem_u32(sm.rec[ds]), a.rec + rec_block(h, a.rows_pad, prow), kQc * 8, dbar);
      ++do_issued;
    }
    // no copy may still be writing shared memory when the CTA exits
    for (int c = (q_issued > kQStages ? q_issued - kQStages : 0); c < q_issued; ++c)
      mbar_wait_drain(smem_u32(&sm.bar_q_full[c % kQStages]), (c / kQStages) & 1, status_word, 2);
    for (int c = (do_issued > kDoStages ? do_issued - kDoStages : 0); c < do_issued; ++c)
      mbar_wait_drain(smem_u32(&sm.bar_do_full[c % kDoStages]), (c / kDoStages) & 1, status_word, 2);
    if (total > 0) mbar_wait_drain(b_kv, 0, status_word, 2);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    // Issue order per chunk c: dV(c), S^T(c+1), dK(c), dP^T(c+1).  S^T(c+1)
    // overwrites X after dV(c) has read P^T(c) from it, dP^T(c+1) overwrites Y
    // after dK(c) has read dS^T(c): tcgen05 MMAs issued by one thread run in
    // order.  Waits are grouped (a wait in this thread holds it until its
    // queued MMAs are nearly done): before dV(c) for P^T(c) and Q(c+1),
    // before dK(c) for dS^T(c) and dO(c+1).
    constexpr uint32_t idesc_s = idesc_bf16(128, kQc, false, false);
    constexpr uint32_t idesc_g = idesc_bf16(128, D, false, true);
    bool ok = total == 0 || mbar_wait(b_kv, 0, abort_flag, status_word, 3);
    const uint64_t kd0 = sdesc(smem_u32(sm.k), 16, 1024), vd0 = sdesc(smem_u32(sm.v), 16, 1024);
    auto wait_q = [&](int c) -> bool {
      return mbar_wait(smem_u32(&sm.bar_q_full[c % kQStages]), (c / kQStages) & 1, abort_flag,
                       status_word, 5);
    };
    auto wait_do = [&](int c) -> bool {
      return mbar_wait(smem_u32(&sm.bar_do_full[c % kDoStages]), (c / kDoStages) & 1, abort_flag,
                       status_word, 5);
    };
    auto issue_s = [&](int c) {
      const uint64_t qd = sdesc(smem_u32(sm.q[c % kQStages]), 16, 1024);
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
        mma_bf16(t_x, desc_at(kd0, off), desc_at(qd, off), idesc_s, k > 0 ? 1u : 0u);
      }
      mma_commit(b_s);
    };
    auto issue_dp = [&](int c) {
      const uint64_t dd = sdesc(smem_u32(sm.dout[c % kDoStages]), 16, 1024);
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
        mma_bf16(t_y, desc_at(vd0, off), desc_at(dd, off), idesc_s, k > 0 ? 1u : 0u);
      }
      mma_commit(b_dp);
    };
    if (ok && total > 0) {
      ok = wait_q(0) && wait_do(0);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        issue_dp(0);
      }
    }
    for (int c = 0; ok && c < total; ++c) {
      const int st = c % kQStages, ds = c % kDoStages;
      const uint32_t acc = c > 0 ? 1u : 0u;
      // B operands MN-major: K = 16 queries per step (16 rows of 128 B), the
      // two 64-column halves of D one 16 KB box apart
      if (!mbar_wait(b_pr, c & 1, abort_flag, status_word, 4) || (c + 1 < total && !wait_q(c + 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint64_t dd = sdesc(smem_u32(sm.dout[ds]), 16384, 1024);
      // dV += P^T dO (P^T from X)
#pragma unroll
      for (int k = 0; k < kQc / 16; ++k)
        mma_bf16_ts(t_dv, t_x + (k >> 1) * 32 + (k & 1) * 8, desc_at(dd, k * 2048), idesc_g,
                    (acc | (uint32_t)k) ? 1u : 0u);
      if (c + 1 < total) issue_s(c + 1);
      if (!mbar_wait(b_dsr, c & 1, abort_flag, status_word, 6) ||
          (c + 1 < total && !wait_do(c + 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint64_t qd = sdesc(smem_u32(sm.q[st]), 16384, 1024);
      // dK += dS^T Q (dS^T from Y)
#pragma unroll
      for (int k = 0; k < kQc / 16; ++k)
        mma_bf16_ts(t_dk, t_y + (k >> 1) * 32 + (k & 1) * 8, desc_at(qd, k * 2048), idesc_g,
                    (acc | (uint32_t)k) ? 1u : 0u);
      mma_commit(smem_u32(&sm.bar_q_empty[st]));
      // the dO stage also holds chunk c's records, read by the dS work that
      // ds_ready(c) waited for: free it only now (dV(c) ran before in order)
      mma_commit(smem_u32(&sm.bar_do_empty[ds]));
      if (c + 1 < total) issue_dp(c + 1);
    }
    if (ok && total > 0) mma_commit(b_acc);
    mma_commit(smem_u32(&sm.bar_drain));
    mbar_wait_drain(smem_u32(&sm.bar_drain), 0, status_word, 2);
  } else if (warp >= 2) {
    // ------------------------------------------------------------ P^T, dS^T (4 threads / key)
    const int qq = (warp - 2) >> 2;   // query quarter: [32 qq, 32 qq + 32)
    const int row = (warp & 3) * 32 + lane;
    const int key = key0 + row;
    const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
    const float sl2 = a.scale_log2;
    // the query rows that see this key: main rows [x, y), branch rows [z, w)
    int4 kiv = make_int4(0, 0, 0, 0);
    if (key < n_keys)
      kiv = reinterpret_cast<const int4 *>(a.plan.key_iv)[(main_kv ? 0 : a.n_main) + key];
    bool ok = true;
    for (int c = 0; c < total; ++c) {
      const int ds = c % kDoStages;
      if (!__all_sync(0xffffffffu, mbar_wait(b_s, c & 1, abort_flag, status_word, 7))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t colx = t_x + lane_addr + qq * 32, coly = t_y + lane_addr + qq * 32;
      float p[32];
      tmem_ld32(colx, reinterpret_cast<uint32_t *>(p));
      tc_wait_ld();
      // the records come with dO
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.bar_do_full[ds]), (c / kDoStages) & 1,
                                             abort_flag, status_word, 8))) {
        ok = false;
        break;
      }
      // this quarter's 32 queries of each record field, four per 16-byte load
      const float4 *r_lse = reinterpret_cast<const float4 *>(sm.rec[ds] + kRecLse + qq * 32);
      const float4 *r_d = reinterpret_cast<const float4 *>(sm.rec[ds] + kRecD + qq * 32);
      const int4 ch = sm.chunk[ds];
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
      // P^T over this thread's own S^T columns: dV(c) may start now
      uint32_t pk[16];
#pragma unroll
      for (int q = 0; q < 32; q += 2) pk[q / 2] = pack_bf16(p[q], p[q + 1]);
      tmem_st16(colx, pk);
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(b_pr);
      if (!__all_sync(0xffffffffu, mbar_wait(b_dp, c & 1, abort_flag, status_word, 9))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float dp[32];
      tmem_ld32(coly, reinterpret_cast<uint32_t *>(dp));
      tc_wait_ld();
      uint32_t dk2[16];
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) {
        const float4 dd = r_d[q4];
        float d[4];
        f2_unpack(f2_mul(f2_pack(p[4 * q4], p[4 * q4 + 1]),
                         f2_sub(f2_pack(dp[4 * q4], dp[4 * q4 + 1]), f2_pack(dd.x, dd.y))),
                  d[0], d[1]);
        f2_unpack(f2_mul(f2_pack(p[4 * q4 + 2], p[4 * q4 + 3]),
                         f2_sub(f2_pack(dp[4 * q4 + 2], dp[4 * q4 + 3]), f2_pack(dd.z, dd.w))),
                  d[2], d[3]);
        dk2[2 * q4] = pack_bf16(d[0], d[1]);
        dk2[2 * q4 + 1] = pack_bf16(d[2], d[3]);
      }
      tmem_st16(coly, dk2);
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(b_dsr);
    }
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

template <typename K, typename M>
ba_status launch_kernel(K kernel, size_t smem, int64_t grid, int threads, const AttnParams &a,
                        const M &maps, cudaStream_t s, const char *name) {
  if (grid <= 0) return BA_OK;
  cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return cuda_check(e, name);
  kernel<<<(unsigned)grid, threads, smem, s>>>(a, maps);
  count_launches(1);
  return cuda_check(cudaGetLastError(), name);
}

}  // namespace


ba_status launch_bwd_sm100(const AttnParams &a, cudaStream_t s) {
  const int d = a.head_dim;
  TensorMaps t;
  ba_status st;
  const bool br = a.n_bt > 0;
#define BA_MAP(dst, ptr, rows, heads, box)                                      \
  if ((st = make_tensor_map(&(dst), ptr, rows, heads, d, box)) != BA_OK) return st;
  BA_MAP(t.q_m, a.q_m, a.n_main, a.hq, 128)
  BA_MAP(t.k_m, a.k_m, a.n_main, a.hkv, 128)
  BA_MAP(t.v_m, a.v_m, a.n_main, a.hkv, 128)
  if (br) {
    BA_MAP(t.q_b, a.q_b, a.n_bt, a.hq, 128)
    BA_MAP(t.k_b, a.k_b, a.n_bt, a.hkv, 128)
    BA_MAP(t.v_b, a.v_b, a.n_bt, a.hkv, 128)
  } else {
    t.q_b = t.q_m; t.k_b = t.k_m; t.v_b = t.v_m;
  }
  DqMaps dqm;
  dqm.t = t;
  BA_MAP(dqm.do_m, a.do_m, a.n_main, a.hq, 128)
  if (br) { BA_MAP(dqm.do_b, a.do_b, a.n_bt, a.hq, 128) } else { dqm.do_b = dqm.do_m; }
  DkvMaps kvm;
  kvm.t = t;
  kvm.do_m = dqm.do_m;
  kvm.do_b = dqm.do_b;
#undef BA_MAP
  const int64_t grid_dq = (int64_t)a.n_qt * a.hq;
  const int64_t grid_kv = (int64_t)(a.n_kt + a.n_bkt) * a.hkv;
  if (d == 64) {
    if ((st = launch_kernel(dkdv_sm100_kernel<64>, sizeof(DkvSmem<64>), grid_kv, kDkvThreads, a,
                            kvm, s, "dkdv_sm100_kernel<64>")) != BA_OK)
      return st;
    return launch_kernel(dq_sm100_kernel<64>, sizeof(DqSmem<64>) + 1024, grid_dq, kDqThreads, a, dqm, s,
                         "dq_sm100_kernel<64>");
  }
  if ((st = launch_kernel(dkdv_sm100_kernel<128>, sizeof(DkvSmem<128>), grid_kv, kDkvThreads, a,
                          kvm, s, "dkdv_sm100_kernel<128>")) != BA_OK)
    return st;
  return launch_kernel(dq_sm100_kernel<128>, sizeof(DqSmem<128>) + 1024, grid_dq, kDqThreads, a, dqm, s,
                       "dq_sm100_kernel<128>");
}

}  // namespace ba
