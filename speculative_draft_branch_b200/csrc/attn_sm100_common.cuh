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

struct TileSegs {
  Seg s[3];
  int total;
  __device__ __forceinline__ void locate(int it, int &key0, int &kind, bool &full) const {
    int si = 0, sub = it;
    if (sub >= s[0].n) {
      sub -= s[0].n;
      si = 1;
      if (sub >= s[1].n) {
        sub -= s[1].n;
        si = 2;
      }
    }
    const Seg g = si == 0 ? s[0] : (si == 1 ? s[1] : s[2]);
    key0 = g.key0 + sub * 128;
    kind = g.kind;
    full = kind == 0 && key0 >= g.full_b && key0 + 128 <= g.full_e;
  }
};

__device__ __forceinline__ TileSegs make_segs(const AttnParams &a, int t, bool is_main) {
  TileSegs ts;
  int n = 0;
  const int32_t *qt = a.plan.qtile + (int64_t)t * 6;
  const int zz = a.zz_step;
  if (zz < 0) {
    const int k0 = qt[0] * 128, k1 = min(qt[3] * 128, a.n_main);
    ts.s[n++] = {k0, (k1 - k0 + 127) / 128, 0, qt[1] * 128, qt[2] * 128};
  } else if (zz < a.zz_C) {
    const int32_t *z = a.plan.zz_tiles + ((int64_t)zz * a.n_qt + t) * 4;
    for (int w = 0; w < 2; ++w) {
      const int k0 = z[2 * w] * 128, k1 = min(z[2 * w + 1] * 128, a.n_main);
      if (k1 > k0) ts.s[n++] = {k0, (k1 - k0 + 127) / 128, w, 0, 0};
    }
  }
  if (!is_main && (zz < 0 || zz == a.zz_C)) {
    const int b0 = qt[4], b1 = qt[5];
    if (b1 > b0) ts.s[n++] = {b0, (b1 - b0 + 127) / 128, 2, 0, 0};
  }
  for (int i = n; i < 3; ++i) ts.s[i] = {0, 0, 2, 0, 0};
  ts.total = ts.s[0].n + ts.s[1].n + ts.s[2].n;
  return ts;
}

}  // namespace ba
