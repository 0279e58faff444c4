// Branch attention with warp-level mma.sync (m16n8k16, bf16 -> fp32): the
// pre-Blackwell tensor-core path, kept as a second, independent
// implementation next to the tcgen05 kernels.
//
// Forward: one CTA per (query tile of 128 rows, q head); 8 warps x 16 rows.
// Keys are visited in 64-row sub-tiles: the main key tiles the plan lists
// for the query tile, then (branch tiles only) the branch-local key rows.
// Each sub-tile's partial (O, l) is folded into the running one by the
// online-softmax rule; the branch-local keys come last, so their fold is the
// paper's merge of (O_b, l_b) into (O_m, l_m) (technical-contribution section).
//
// Backward: one CTA per (key tile of 128 rows, kv head); 8 warps x 16 keys.
// It loops over the q heads of the group and over every query tile that
// visits the key tile, recomputes P from the merged LSE, accumulates dK/dV in
// registers and adds dQ into an fp32 buffer with atomics.
#include "internal.cuh"

namespace ba {
namespace {

using bf16 = __nv_bfloat16;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
  const int sz = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(sz));
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src, bool valid) {
  const int sz = valid ? 4 : 0;
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(dst), "l"(src), "r"(sz));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n"); }
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;\n" ::: "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t r[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t r[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float c[4], const uint32_t a[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, "
      "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// Byte offset of 16-byte chunk `ch` of row `row` in a tile whose rows are
// D bf16 wide; the chunk index is XOR-swizzled with the row (mod 8) so that
// ldmatrix over 8 consecutive rows hits 8 distinct bank groups.
template <int D>
__device__ __forceinline__ uint32_t swz(int row, int ch) {
  return (uint32_t)(row * (D * 2) + ((ch ^ (row & 7)) << 4));
}

// Copy `ROWS` rows x D of head `head` of a [tokens, heads, D] tensor into a
// swizzled smem tile; rows at or beyond `limit` are zero-filled.
template <int ROWS, int D, int NT>
__device__ __forceinline__ void load_tile(uint32_t sbase, const bf16 *g, int64_t row0,
                                          int64_t limit, int heads, int head) {
  constexpr int kChunks = D / 8;
  for (int i = threadIdx.x; i < ROWS * kChunks; i += NT) {
    const int r = i / kChunks, ch = i % kChunks;
    const int64_t gr = row0 + r;
    const bool ok = gr >= 0 && gr < limit;
    const bf16 *src = g + (ok ? ((gr * heads + head) * D + ch * 8) : 0);
    cp_async16(sbase + swz<D>(r, ch), src, ok);
  }
}

constexpr float kNegInf = -INFINITY;
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;

// ============================================================================
// Forward
// ============================================================================
template <int D>
struct FwdMmaSmem {
  bf16 q[128 * D];
  bf16 k[2][64 * D];
  bf16 v[2][64 * D];
};

// A segment of key sub-tiles visited with one kind of per-row interval.
struct Seg {
  int key0;      // first key row (main or branch row space)
  int n;         // number of 64-row sub-tiles
  int kind;      // 0/1: main keys with interval 0/1, 2: branch-local keys
  int full_b, full_e;  // key rows [full_b, full_e) need no mask (kind 0 only)
};

template <int D>
__global__ void __launch_bounds__(256, 1) fwd_mma_kernel(const AttnParams a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  FwdMmaSmem<D> &sm = *reinterpret_cast<FwdMmaSmem<D> *>(smem_raw);
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
  const int row_off = is_main ? 0 : a.n_main;  // offset in the all-rows arrays
  const bf16 *qg = is_main ? a.q_m : a.q_b;
  const int32_t *qt = a.plan.qtile + (int64_t)t * 6;

  // ---- segments ----
  Seg seg[3];
  int nseg = 0;
  const int zz = a.zz_step;
  if (zz < 0) {
    const int kb = qt[0], fb = qt[1], fe = qt[2], ke = qt[3];
    const int k0 = kb * 128, k1 = min(ke * 128, a.n_main);
    seg[nseg++] = {k0, (k1 - k0 + 63) / 64, 0, fb * 128, fe * 128};
  } else if (zz < a.zz_C) {
    const int32_t *z = a.plan.zz_tiles + ((int64_t)zz * a.n_qt + t) * 4;
    for (int w = 0; w < 2; ++w) {
      const int k0 = z[2 * w] * 128, k1 = min(z[2 * w + 1] * 128, a.n_main);
      if (k1 > k0) seg[nseg++] = {k0, (k1 - k0 + 63) / 64, w, 0, 0};
    }
  }
  if (!is_main && (zz < 0 || zz == a.zz_C)) {
    const int b0 = qt[4], b1 = qt[5];
    if (b1 > b0) seg[nseg++] = {b0, (b1 - b0 + 63) / 64, 2, 0, 0};
  }
  for (int i = nseg; i < 3; ++i) seg[i] = {0, 0, 2, 0, 0};
  const int total = seg[0].n + seg[1].n + seg[2].n;

  // ---- per-thread rows and their key intervals ----
  const int ra = warp * 16 + lane / 4, rb = ra + 8;
  int lo[2][3], hi[2][3];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int r = i == 0 ? ra : rb;
#pragma unroll
    for (int k = 0; k < 3; ++k) { lo[i][k] = 0; hi[i][k] = -1; }
    if (r < nrows) {
      const int4 iv = reinterpret_cast<const int4 *>(a.plan.row_iv)[row_off + row0 + r];
      if (zz < 0 || zz == a.zz_C) {
        lo[i][0] = iv.x; hi[i][0] = iv.y;
        lo[i][2] = iv.z; hi[i][2] = iv.w;
      }
      if (zz >= 0 && zz < a.zz_C) {
        // ring-step windows: chunks j and 2C-1-j of the row's sequence, j =
        // (shard(row) - step) mod C, intersected with the causal interval
        int s_lo = 0, s_hi = a.n_seqs;
        while (s_lo < s_hi) {  // sequence with cu[s] == iv.x
          const int mid = (s_lo + s_hi + 1) >> 1;
          if (a.cu_seqlens[mid] <= iv.x) s_lo = mid; else s_hi = mid - 1;
        }
        const int64_t L = a.cu_seqlens[s_lo + 1] - iv.x;
        const int64_t pos = iv.y - iv.x;
        const int C = a.zz_C;
        const int c = (int)((2 * C * (pos + 1) - 1) / L);
        const int shard = c < C ? c : 2 * C - 1 - c;
        const int j = ((shard - zz) % C + C) % C;
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          const int ch = w == 0 ? j : 2 * C - 1 - j;
          lo[i][w] = max(iv.x + (int)((ch * L) / (2 * C)), iv.x);
          hi[i][w] = min(iv.x + (int)(((ch + 1) * L) / (2 * C)) - 1, iv.y);
        }
      }
    }
  }

  auto seg_of = [&](int it, int &si, int &sub) {
    si = 0;
    sub = it;
    if (sub >= seg[0].n) { sub -= seg[0].n; si = 1;
      if (sub >= seg[1].n) { sub -= seg[1].n; si = 2; } }
  };
  auto issue_kv = [&](int it) {
    int si, sub;
    seg_of(it, si, sub);
    const Seg sg = si == 0 ? seg[0] : (si == 1 ? seg[1] : seg[2]);
    const int key0 = sg.key0 + sub * 64;
    const bool loc = sg.kind == 2;
    const bf16 *kg = loc ? a.k_b : a.k_m;
    const bf16 *vg = loc ? a.v_b : a.v_m;
    const int64_t lim = loc ? a.n_bt : a.n_main;
    const int buf = it & 1;
    load_tile<64, D, 256>(smem_u32(sm.k[buf]), kg, key0, lim, a.hkv, g);
    load_tile<64, D, 256>(smem_u32(sm.v[buf]), vg, key0, lim, a.hkv, g);
  };

  load_tile<128, D, 256>(smem_u32(sm.q), qg, row0, rows_total, a.hq, h);
  if (total > 0) issue_kv(0);
  cp_async_commit();
  cp_async_wait_all();
  __syncthreads();

  uint32_t qf[D / 16][4];
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const int r = warp * 16 + (lane % 8) + 8 * ((lane / 8) & 1);
    ldsm_x4(qf[kk], smem_u32(sm.q) + swz<D>(r, 2 * kk + lane / 16));
  }

  float o[D / 8][4];
#pragma unroll
  for (int j = 0; j < D / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m[2] = {kNegInf, kNegInf}, l[2] = {0.f, 0.f};

  for (int it = 0; it < total; ++it) {
    if (it > 0) {
      cp_async_wait_all();
      __syncthreads();
    }
    if (it + 1 < total) {
      issue_kv(it + 1);
      cp_async_commit();
    }
    int si, sub;
    seg_of(it, si, sub);
    const Seg sg = si == 0 ? seg[0] : (si == 1 ? seg[1] : seg[2]);
    const int key0 = sg.key0 + sub * 64;
    const int kind = sg.kind;
    const bool full = kind == 0 && key0 >= sg.full_b && key0 + 64 <= sg.full_e;
    // this sub-tile's per-row interval (register selects, no local memory)
    int clo[2], chi[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      clo[i] = kind == 0 ? lo[i][0] : (kind == 1 ? lo[i][1] : lo[i][2]);
      chi[i] = kind == 0 ? hi[i][0] : (kind == 1 ? hi[i][1] : hi[i][2]);
    }
    const uint32_t kb = smem_u32(sm.k[it & 1]), vb = smem_u32(sm.v[it & 1]);

    float s[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int jp = 0; jp < 4; ++jp) {
        uint32_t b[4];
        const int kr = 16 * jp + (lane % 8) + 8 * (lane / 16);
        ldsm_x4(b, kb + swz<D>(kr, 2 * kk + ((lane / 8) & 1)));
        mma16816(s[2 * jp], qf[kk], b[0], b[1]);
        mma16816(s[2 * jp + 1], qf[kk], b[2], b[3]);
      }
    }
    // scale to log2 domain, mask, row max
    float mx[2] = {kNegInf, kNegInf};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = e >> 1;
        float x = s[j][e] * a.scale_log2;
        if (!full) {
          const int key = key0 + 8 * j + 2 * (lane % 4) + (e & 1);
          if (key < clo[i] || key > chi[i]) x = kNegInf;
        }
        s[j][e] = x;
        mx[i] = fmaxf(mx[i], x);
      }
    }
    float alpha[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 1));
      mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 2));
      const float mn = fmaxf(m[i], mx[i]);
      const float mu = mn == kNegInf ? 0.f : mn;
      alpha[i] = exp2f(m[i] - mu);
      m[i] = mn;
      mx[i] = mu;  // reuse as the subtracted max
    }
    float rs[2] = {0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float p = exp2f(s[j][e] - mx[e >> 1]);
        s[j][e] = p;
        rs[e >> 1] += p;
      }
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) l[i] = l[i] * alpha[i] + rs[i];
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
      o[j][0] *= alpha[0]; o[j][1] *= alpha[0];
      o[j][2] *= alpha[1]; o[j][3] *= alpha[1];
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t pa[4];
      pa[0] = pack2(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack2(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int dn = 0; dn < D / 16; ++dn) {
        uint32_t b[4];
        const int vr = 16 * kk + (lane % 8) + 8 * ((lane / 8) & 1);
        ldsm_x4_t(b, vb + swz<D>(vr, 2 * dn + lane / 16));
        mma16816(o[2 * dn], pa, b[0], b[1]);
        mma16816(o[2 * dn + 1], pa, b[2], b[3]);
      }
    }
  }

  // ---- epilogue: normalise, LSE ----
  float lse[2], inv[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    l[i] += __shfl_xor_sync(0xffffffffu, l[i], 1);
    l[i] += __shfl_xor_sync(0xffffffffu, l[i], 2);
    const bool empty = m[i] == kNegInf || l[i] <= 0.f;
    lse[i] = empty ? kNegInf : (m[i] + log2f(l[i])) * kLn2;
    inv[i] = empty ? 0.f : 1.f / l[i];
  }
#pragma unroll
  for (int j = 0; j < D / 8; ++j) {
    o[j][0] *= inv[0]; o[j][1] *= inv[0];
    o[j][2] *= inv[1]; o[j][3] *= inv[1];
  }

  const bool final_out = zz < 0 || zz == a.zz_C;
  if (zz >= 0) {
    // ring-step partial: merge into the fp32 accumulator (step 0 initialises);
    // the branch-local pass merges last and writes the final outputs below
    const int64_t all_rows = (int64_t)a.n_main + a.n_bt;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int r = i == 0 ? ra : rb;
      const bool valid = r < nrows;
      const int64_t grow = row_off + row0 + (valid ? r : 0);
      float *acc = a.zz_o + (grow * a.hq + h) * D;
      float *accl = a.zz_lse + (int64_t)h * all_rows + grow;
      // lane 0 of the quad owns the row's LSE: it reads and later writes it
      float la = kNegInf;
      if (zz > 0 && valid && (lane % 4) == 0) la = *accl;
      la = __shfl_sync(0xffffffffu, la, lane & ~3);
      float wa = 0.f, wb = 1.f, lnew = lse[i];
      if (zz > 0) {
        const float mm = fmaxf(la, lse[i]);
        if (mm == kNegInf) { lnew = kNegInf; wa = 0.f; wb = 0.f; }
        else {
          lnew = mm + logf(expf(la - mm) + expf(lse[i] - mm));
          wa = expf(la - lnew);
          wb = expf(lse[i] - lnew);
        }
      }
      if (valid) {
#pragma unroll
        for (int j = 0; j < D / 8; ++j) {
          const int col = 8 * j + 2 * (lane % 4);
          float2 prev = zz > 0 ? *reinterpret_cast<float2 *>(acc + col) : make_float2(0.f, 0.f);
          float2 nv;
          nv.x = wa * prev.x + wb * o[j][2 * i];
          nv.y = wa * prev.y + wb * o[j][2 * i + 1];
          o[j][2 * i] = nv.x;
          o[j][2 * i + 1] = nv.y;
          if (!final_out) *reinterpret_cast<float2 *>(acc + col) = nv;
        }
        if (!final_out && (lane % 4) == 0) *accl = lnew;
      }
      lse[i] = lnew;
    }
  }
  if (!final_out) return;

  // final outputs: stage O through the (no longer used) Q tile, 16 B stores
  bf16 *og = is_main ? a.o_m : a.o_b;
  float *lg = is_main ? a.lse_m : a.lse_b;
  const uint32_t qs = smem_u32(sm.q);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int r = i == 0 ? ra : rb;
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
      const uint32_t addr = qs + swz<D>(r, j) + 4 * (lane % 4);
      const uint32_t v = pack2(o[j][2 * i], o[j][2 * i + 1]);
      asm volatile("st.shared.b32 [%0], %1;\n" ::"r"(addr), "r"(v));
    }
    if ((lane % 4) == 0 && r < nrows) lg[(int64_t)h * rows_total + row0 + r] = lse[i];
  }
  __syncwarp();
  constexpr int kChunks = D / 8;
  for (int i = lane; i < 16 * kChunks; i += 32) {
    const int r = warp * 16 + i / kChunks, ch = i % kChunks;
    if (r >= nrows) continue;
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(qs + swz<D>(r, ch)));
    *reinterpret_cast<uint4 *>(og + ((int64_t)(row0 + r) * a.hq + h) * D + ch * 8) = v;
  }
}

// ============================================================================
// Backward
// ============================================================================
constexpr int kQC = 64;  // query rows per backward chunk

template <int D>
struct BwdMmaSmem {
  bf16 k[128 * D];
  bf16 v[128 * D];
  bf16 q[2][kQC * D];
  bf16 dout[2][kQC * D];
  bf16 ds[128 * kQC];       // dS^T [key][q]
  float lse[2][kQC];        // log2-domain LSE of each query row
  float dd[2][kQC];         // D = rowsum(dO * O)
  int4 iv[2][kQC];          // key intervals of each query row
};

template <int D>
__global__ void __launch_bounds__(256, 1) bwd_mma_kernel(const AttnParams a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  BwdMmaSmem<D> &sm = *reinterpret_cast<BwdMmaSmem<D> *>(smem_raw);
  if (a.plan.status[0] != 0) return;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int item = a.plan.bwd_order[blockIdx.x / a.hkv];
  const int g = blockIdx.x % a.hkv;
  const int grp = a.hq / a.hkv;
  const bool main_kv = item < a.n_kt;
  const int kt = main_kv ? item : item - a.n_kt;
  const int key0 = kt * 128;
  const int n_keys = main_kv ? a.n_main : a.n_bt;
  const bf16 *kg = main_kv ? a.k_m : a.k_b;
  const bf16 *vg = main_kv ? a.v_m : a.v_b;
  int tr[2][2];  // query-tile ranges: [part][begin/end]; part 0 main, 1 branch
  if (main_kv) {
    const int32_t *r = a.plan.kv_main + (int64_t)kt * 4;
    tr[0][0] = r[0]; tr[0][1] = r[1]; tr[1][0] = r[2]; tr[1][1] = r[3];
  } else {
    const int32_t *r = a.plan.kv_branch + (int64_t)kt * 2;
    tr[0][0] = 0; tr[0][1] = 0; tr[1][0] = r[0]; tr[1][1] = r[1];
  }
  const int n_t0 = tr[0][1] - tr[0][0], n_t1 = tr[1][1] - tr[1][0];
  const int per_head = 2 * (n_t0 + n_t1);
  const int total = grp * per_head;
  const int64_t all_rows = (int64_t)a.n_main + a.n_bt;

  struct Chunk {
    int h, is_main_q, tile, row0, nrows;
  };
  auto chunk_of = [&](int c) {
    Chunk ck;
    const int hh = c / per_head, rem = c % per_head;
    const int ti = rem / 2, half = rem % 2;
    ck.h = g * grp + hh;
    ck.is_main_q = ti < n_t0;
    const int tile = ck.is_main_q ? tr[0][0] + ti : tr[1][0] + (ti - n_t0);
    ck.tile = tile;
    const int rows = ck.is_main_q ? a.n_main : a.n_bt;
    ck.row0 = tile * 128 + half * kQC;
    ck.nrows = max(0, min(kQC, rows - ck.row0));
    return ck;
  };
  auto issue_chunk = [&](int c) {
    const Chunk ck = chunk_of(c);
    const int buf = c & 1;
    const int rows = ck.is_main_q ? a.n_main : a.n_bt;
    load_tile<kQC, D, 256>(smem_u32(sm.q[buf]), ck.is_main_q ? a.q_m : a.q_b, ck.row0, rows,
                           a.hq, ck.h);
    load_tile<kQC, D, 256>(smem_u32(sm.dout[buf]), ck.is_main_q ? a.do_m : a.do_b, ck.row0,
                           rows, a.hq, ck.h);
    const int tid = threadIdx.x;
    const int roff = ck.is_main_q ? 0 : a.n_main;
    if (tid < kQC) {
      const bool ok = tid < ck.nrows;
      const float *src = (ck.is_main_q ? a.lse_m : a.lse_b) +
                         (ok ? (int64_t)ck.h * rows + ck.row0 + tid : 0);
      cp_async4(smem_u32(&sm.lse[buf][tid]), src, ok);
    } else if (tid < 2 * kQC) {
      const int r = tid - kQC;
      const bool ok = r < ck.nrows;
      const float *src = a.d_all + (ok ? (int64_t)ck.h * all_rows + roff + ck.row0 + r : 0);
      cp_async4(smem_u32(&sm.dd[buf][r]), src, ok);
    } else if (tid < 3 * kQC) {
      const int r = tid - 2 * kQC;
      const bool ok = r < ck.nrows;
      const int32_t *src = a.plan.row_iv + (ok ? (roff + ck.row0 + r) * 4 : 0);
      cp_async16(smem_u32(&sm.iv[buf][r]), src, ok);
    }
  };

  load_tile<128, D, 256>(smem_u32(sm.k), kg, key0, n_keys, a.hkv, g);
  load_tile<128, D, 256>(smem_u32(sm.v), vg, key0, n_keys, a.hkv, g);
  if (total > 0) issue_chunk(0);
  cp_async_commit();

  float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
  for (int j = 0; j < D / 8; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) { dk[j][e] = 0.f; dv[j][e] = 0.f; }

  const uint32_t ks = smem_u32(sm.k), vs = smem_u32(sm.v);
  const int kr_a = warp * 16 + lane / 4;  // this thread's key rows in the tile
  for (int c = 0; c < total; ++c) {
    cp_async_wait_all();
    __syncthreads();
    if (c + 1 < total) {
      issue_chunk(c + 1);
      cp_async_commit();
    }
    const Chunk ck = chunk_of(c);
    if (ck.nrows == 0) continue;  // uniform across the block
    const int buf = c & 1;
    const uint32_t qs = smem_u32(sm.q[buf]), dos = smem_u32(sm.dout[buf]);
    bool full = false;
    if (main_kv) {
      const int32_t *qt = a.plan.qtile +
                          (int64_t)(ck.is_main_q ? ck.tile : a.n_qt_main + ck.tile) * 6;
      full = kt >= qt[1] && kt < qt[2];
    }
    // S^T = K Q^T and dP^T = V dO^T (16 keys x 64 queries per warp)
    float st[8][4], dpt[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) { st[j][e] = 0.f; dpt[j][e] = 0.f; }
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t ka[4], va[4];
      const int ar = warp * 16 + (lane % 8) + 8 * ((lane / 8) & 1);
      ldsm_x4(ka, ks + swz<D>(ar, 2 * kk + lane / 16));
      ldsm_x4(va, vs + swz<D>(ar, 2 * kk + lane / 16));
#pragma unroll
      for (int jp = 0; jp < 4; ++jp) {
        uint32_t b[4];
        const int qr = 16 * jp + (lane % 8) + 8 * (lane / 16);
        ldsm_x4(b, qs + swz<D>(qr, 2 * kk + ((lane / 8) & 1)));
        mma16816(st[2 * jp], ka, b[0], b[1]);
        mma16816(st[2 * jp + 1], ka, b[2], b[3]);
        ldsm_x4(b, dos + swz<D>(qr, 2 * kk + ((lane / 8) & 1)));
        mma16816(dpt[2 * jp], va, b[0], b[1]);
        mma16816(dpt[2 * jp + 1], va, b[2], b[3]);
      }
    }
    // P^T = exp(S^T - LSE) masked; dS^T = P^T (dP^T - D)
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int q = 8 * j + 2 * (lane % 4) + (e & 1);
        const int key = key0 + kr_a + 8 * (e >> 1);
        const int4 iv = sm.iv[buf][q];
        const int klo = main_kv ? iv.x : iv.z, khi = main_kv ? iv.y : iv.w;
        const bool vis = q < ck.nrows && (full || (key >= klo && key <= khi));
        const float p = vis ? exp2f(st[j][e] * a.scale_log2 - sm.lse[buf][q] * kLog2e) : 0.f;
        st[j][e] = p;
        dpt[j][e] = p * (dpt[j][e] - sm.dd[buf][q]);
      }
    }
    // dV += P^T dO ; dK += dS^T Q   (k = 64 queries)
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t pa[4], sa[4];
      pa[0] = pack2(st[2 * kk][0], st[2 * kk][1]);
      pa[1] = pack2(st[2 * kk][2], st[2 * kk][3]);
      pa[2] = pack2(st[2 * kk + 1][0], st[2 * kk + 1][1]);
      pa[3] = pack2(st[2 * kk + 1][2], st[2 * kk + 1][3]);
      sa[0] = pack2(dpt[2 * kk][0], dpt[2 * kk][1]);
      sa[1] = pack2(dpt[2 * kk][2], dpt[2 * kk][3]);
      sa[2] = pack2(dpt[2 * kk + 1][0], dpt[2 * kk + 1][1]);
      sa[3] = pack2(dpt[2 * kk + 1][2], dpt[2 * kk + 1][3]);
#pragma unroll
      for (int dn = 0; dn < D / 16; ++dn) {
        uint32_t b[4];
        const int qr = 16 * kk + (lane % 8) + 8 * ((lane / 8) & 1);
        ldsm_x4_t(b, dos + swz<D>(qr, 2 * dn + lane / 16));
        mma16816(dv[2 * dn], pa, b[0], b[1]);
        mma16816(dv[2 * dn + 1], pa, b[2], b[3]);
        ldsm_x4_t(b, qs + swz<D>(qr, 2 * dn + lane / 16));
        mma16816(dk[2 * dn], sa, b[0], b[1]);
        mma16816(dk[2 * dn + 1], sa, b[2], b[3]);
      }
    }
    // dS^T to smem (bf16, [128 keys][64 q], 8 chunks per row)
    const uint32_t dss = smem_u32(sm.ds);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int row = kr_a + 8 * i;
        const uint32_t addr = dss + swz<kQC>(row, j) + 4 * (lane % 4);
        asm volatile("st.shared.b32 [%0], %1;\n" ::"r"(addr),
                     "r"(pack2(dpt[j][2 * i], dpt[j][2 * i + 1])));
      }
    }
    __syncthreads();
    // dQ[64 x D] = dS K: warp -> 16 query rows x D/2 columns
    {
      const int qb = 16 * (warp % 4), cb = (warp / 4) * (D / 2);
      float dq[D / 16][4];
#pragma unroll
      for (int j = 0; j < D / 16; ++j) dq[j][0] = dq[j][1] = dq[j][2] = dq[j][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {  // 128 keys
        uint32_t af[4];
        const int krow = 16 * kk + (lane % 8) + 8 * (lane / 16);
        ldsm_x4_t(af, dss + swz<kQC>(krow, qb / 8 + ((lane / 8) & 1)));
#pragma unroll
        for (int dn = 0; dn < D / 32; ++dn) {
          uint32_t b[4];
          const int kr2 = 16 * kk + (lane % 8) + 8 * ((lane / 8) & 1);
          ldsm_x4_t(b, ks + swz<D>(kr2, cb / 8 + 2 * dn + lane / 16));
          mma16816(dq[2 * dn], af, b[0], b[1]);
          mma16816(dq[2 * dn + 1], af, b[2], b[3]);
        }
      }
      const int roff = ck.is_main_q ? 0 : a.n_main;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int q = qb + lane / 4 + 8 * i;
        if (q >= ck.nrows) continue;
        float *dst = a.dq_acc + ((int64_t)(roff + ck.row0 + q) * a.hq + ck.h) * D + cb +
                     2 * (lane % 4);
#pragma unroll
        for (int j = 0; j < D / 16; ++j) {
          atomicAdd(reinterpret_cast<float2 *>(dst + 8 * j),
                    make_float2(dq[j][2 * i], dq[j][2 * i + 1]));
        }
      }
    }
  }

  // ---- epilogue: dK (scaled), dV as bf16 through smem ----
  __syncthreads();
  bf16 *dkg = main_kv ? a.dk_m : a.dk_b;
  bf16 *dvg = main_kv ? a.dv_m : a.dv_b;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int row = kr_a + 8 * i;
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
      const uint32_t off = swz<D>(row, j) + 4 * (lane % 4);
      asm volatile("st.shared.b32 [%0], %1;\n" ::"r"(ks + off),
                   "r"(pack2(dk[j][2 * i] * a.scale, dk[j][2 * i + 1] * a.scale)));
      asm volatile("st.shared.b32 [%0], %1;\n" ::"r"(vs + off),
                   "r"(pack2(dv[j][2 * i], dv[j][2 * i + 1])));
    }
  }
  __syncwarp();
  constexpr int kChunks = D / 8;
  for (int i = lane; i < 16 * kChunks; i += 32) {
    const int r = warp * 16 + i / kChunks, ch = i % kChunks;
    const int64_t key = key0 + r;
    if (key >= n_keys) continue;
    uint4 x, y;
    asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(x.x), "=r"(x.y), "=r"(x.z), "=r"(x.w)
                 : "r"(ks + swz<D>(r, ch)));
    asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(y.x), "=r"(y.y), "=r"(y.z), "=r"(y.w)
                 : "r"(vs + swz<D>(r, ch)));
    const int64_t off = (key * a.hkv + g) * D + ch * 8;
    *reinterpret_cast<uint4 *>(dkg + off) = x;
    *reinterpret_cast<uint4 *>(dvg + off) = y;
  }
}

template <typename K>
ba_status launch_with_smem(K kernel, size_t smem, int64_t grid, const AttnParams &a,
                           cudaStream_t s, const char *name) {
  if (grid <= 0) return BA_OK;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return cuda_check(e, name);
  kernel<<<(unsigned)grid, 256, smem, s>>>(a);
  count_launches(1);
  return cuda_check(cudaGetLastError(), name);
}

}  // namespace

ba_status launch_fwd_mma(const AttnParams &a, cudaStream_t s) {
  const int64_t grid = (int64_t)a.n_qt * a.hq;
  if (a.head_dim == 64)
    return launch_with_smem(fwd_mma_kernel<64>, sizeof(FwdMmaSmem<64>), grid, a, s,
                            "fwd_mma_kernel<64>");
  return launch_with_smem(fwd_mma_kernel<128>, sizeof(FwdMmaSmem<128>), grid, a, s,
                          "fwd_mma_kernel<128>");
}

ba_status launch_bwd_mma(const AttnParams &a, cudaStream_t s) {
  const int64_t grid = (int64_t)(a.n_kt + a.n_bkt) * a.hkv;
  if (a.head_dim == 64)
    return launch_with_smem(bwd_mma_kernel<64>, sizeof(BwdMmaSmem<64>), grid, a, s,
                            "bwd_mma_kernel<64>");
  return launch_with_smem(bwd_mma_kernel<128>, sizeof(BwdMmaSmem<128>), grid, a, s,
                          "bwd_mma_kernel<128>");
}

}  // namespace ba
