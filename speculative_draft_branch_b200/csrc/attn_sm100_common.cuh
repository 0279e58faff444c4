// Pieces shared by the tcgen05 forward and backward kernels: the TMA tensor
// maps of the six Q/K/V tensors and the walk over a query tile's key tiles.
#pragma once

#include "internal.cuh"
#include "sm100.cuh"

namespace ba {

using bf16 = __nv_bfloat16;
constexpr float kNegInf = -INFINITY;
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;

struct TensorMaps {
  CUtensorMap q_m, q_b, k_m, v_m, k_b, v_b;
};

// [rows, heads, d] bf16 tensor -> TMA map with boxes of 64 elements x 1 head
// x box_rows rows, 128-byte swizzle (rows past the end read as zero).
ba_status make_tensor_map(CUtensorMap *m, const void *ptr, int64_t rows, int heads, int d,
                          int box_rows);

struct Seg {
  int key0, n, kind, full_b, full_e;
};

// Up to three key segments of a query tile, walked in order.  Kept as three
// named members (never an array indexed at run time), so the walk stays in
// registers instead of local memory.
struct TileSegs {
  Seg s0, s1, s2;
  int total;
  __device__ __forceinline__ void locate(int it, int &key0, int &kind, bool &full) const {
    int sub = it;
    Seg g = s0;
    if (sub >= s0.n) {
      sub -= s0.n;
      g = s1;
      if (sub >= s1.n) {
        sub -= s1.n;
        g = s2;
      }
    }
    key0 = g.key0 + sub * 128;
    kind = g.kind;
    full = kind == 0 && key0 >= g.full_b && key0 + 128 <= g.full_e;
  }
  __device__ __forceinline__ void push(const Seg &g, int &n) {
    if (n == 0) s0 = g;
    else if (n == 1) s1 = g;
    else s2 = g;
    ++n;
  }
};

__device__ __forceinline__ TileSegs make_segs(const AttnParams &a, int t, bool is_main) {
  TileSegs ts;
  const Seg none = {0, 0, 2, 0, 0};
  ts.s0 = none; ts.s1 = none; ts.s2 = none;
  int n = 0;
  const int32_t *qt = a.plan.qtile + (int64_t)t * 6;
  const int zz = a.zz_step;
  if (zz < 0 || (a.ring && zz < a.zz_C)) {
    const int k0 = qt[0] * 128, k1 = min(qt[3] * 128, a.n_keys_m);
    if (k1 > k0) ts.push({k0, (k1 - k0 + 127) / 128, 0, qt[1] * 128, qt[2] * 128}, n);
  } else if (zz < a.zz_C) {
    const int32_t *z = a.plan.zz_tiles + ((int64_t)zz * a.n_qt + t) * 4;
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      const int k0 = z[2 * w] * 128, k1 = min(z[2 * w + 1] * 128, a.n_keys_m);
      if (k1 > k0) ts.push({k0, (k1 - k0 + 127) / 128, w, 0, 0}, n);
    }
  }
  if (!is_main && (zz < 0 || zz == a.zz_C)) {
    const int b0 = qt[4], b1 = qt[5];
    if (b1 > b0) ts.push({b0, (b1 - b0 + 127) / 128, 2, 0, 0}, n);
  }
  ts.total = ts.s0.n + ts.s1.n + ts.s2.n;
  return ts;
}

// ---- key-stationary backward walk -------------------------------------------
constexpr int kQc = 128;  // query rows per chunk: N of the S^T / dP^T products

struct DkvMaps {
  TensorMaps t;
  CUtensorMap do_m, do_b;
};

// Chunk c of a CTA's walk: query tile step s = c / grp, q head g grp + c % grp.
// The tile steps merge the CTA's main q tiles and branch q tiles, each taken
// from the last down, interleaved in proportion to their counts.  Every CTA
// of a sequence then starts on the same (highest) tiles and moves through
// them at the same pace, so the Q / dO tiles one CTA loads are still in L2
// when the CTAs of the other key tiles of that sequence ask for them.
struct ChunkWalk {
  int n_t0, n_t1, t0, t1, grp, g;
  __device__ __forceinline__ void at(int c, const AttnParams &a, int &h, bool &is_main_q,
                                     int &tile, int &nrows) const {
    const int s = c / grp;
    h = g * grp + (c - s * grp);
    const int n = n_t0 + n_t1;
    const int m0 = (int)((int64_t)s * n_t0 / n);
    const int m1 = (int)((int64_t)(s + 1) * n_t0 / n);
    is_main_q = m1 > m0;
    tile = is_main_q ? t0 + n_t0 - 1 - m0 : t1 + n_t1 - 1 - (s - m0);
    const int rows = is_main_q ? a.n_main : a.n_bt;
    nrows = max(0, min(kQc, rows - tile * kQc));
  }
};

// The CTA's walk for (key tile item of the plan's backward order, kv head g).
__device__ __forceinline__ ChunkWalk make_walk(const AttnParams &a, bool main_kv, int kt, int g) {
  ChunkWalk cw;
  cw.grp = a.hq / a.hkv;
  cw.g = g;
  if (main_kv) {
    const int32_t *r = a.plan.kv_main + (int64_t)kt * 4;
    cw.t0 = r[0]; cw.n_t0 = r[1] - r[0]; cw.t1 = r[2]; cw.n_t1 = r[3] - r[2];
  } else {
    const int32_t *r = a.plan.kv_branch + (int64_t)kt * 2;
    cw.t0 = 0; cw.n_t0 = 0; cw.t1 = r[0]; cw.n_t1 = r[1] - r[0];
  }
  return cw;
}

}  // namespace ba
