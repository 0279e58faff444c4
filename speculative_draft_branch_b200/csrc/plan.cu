// Plan kernels: device-side validation of the index arrays and the tile
// metadata that drives tile skipping in the attention kernels.
//
// Which keys a query sees is fixed by the paper's method-detail section (a
// branch query reads the causal main prefix up to its anchor and its own
// branch; a main query reads its causal prefix).  The metadata below turns
// that into per-row key intervals and per-tile key-tile ranges.
#include "internal.cuh"

namespace ba {
namespace {

__device__ __forceinline__ void flag(int32_t *status, int bit) { atomicOr(status, bit); }

// largest i in [0, n) with a[i] <= x (a non-decreasing, a[0] <= x)
__device__ __forceinline__ int upper_index(const int32_t *a, int n, int32_t x) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (a[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ---- K1: validation + exclusive scan of branch depths (one block) ---------
constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) plan_scan_kernel(
    const int32_t *cu, const int32_t *anchor, const int32_t *depth, int n_seqs, int n_main,
    int n_br, int n_bt, int32_t *status, int32_t *cu_branch) {
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t bad;
  const int tid = threadIdx.x;
  if (tid == 0) { status[0] = 0; status[1] = 0; status[2] = 0; status[3] = 0; bad = 0; }
  __syncthreads();
  int local_bad = 0;
  // cu_seqlens checks
  for (int i = tid; i <= n_seqs; i += kScanThreads) {
    int32_t c = cu[i];
    if (i == 0 && c != 0) local_bad |= BA_META_CU_START;
    if (i > 0 && c <= cu[i - 1]) local_bad |= BA_META_CU_ORDER;
    if (i == n_seqs && c != n_main) local_bad |= BA_META_CU_TOTAL;
  }
  // anchors and depths
  for (int b = tid; b < n_br; b += kScanThreads) {
    int32_t a = anchor[b];
    if (a < 0 || a >= n_main) local_bad |= BA_META_ANCHOR_RANGE;
    if (b > 0 && a < anchor[b - 1]) local_bad |= BA_META_ANCHOR_ORDER;
    int32_t d = depth[b];
    if (d < 1 || d > kMaxDepth) local_bad |= BA_META_DEPTH_RANGE;
  }
  // exclusive scan in contiguous chunks (depth clamped so the sum stays sane)
  const int per = (n_br + kScanThreads - 1) / kScanThreads;
  const int b0 = min(tid * per, n_br), b1 = min(b0 + per, n_br);
  int64_t sum = 0;
  for (int b = b0; b < b1; ++b) sum += min(max(depth[b], 0), kMaxDepth);
  int32_t s32 = (int32_t)sum;
  const int lane = tid & 31, wid = tid >> 5;
  int32_t incl = s32;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    int32_t w = warp_sums[lane];
    int32_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int32_t y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    warp_sums[lane] = wi - w;  // exclusive warp offsets
  }
  __syncthreads();
  int32_t run = warp_sums[wid] + incl - s32;
  for (int b = b0; b < b1; ++b) {
    cu_branch[b] = run;
    run += min(max(depth[b], 0), kMaxDepth);
  }
  if (tid == kScanThreads - 1) {
    cu_branch[n_br] = run;  // total
    if (run != n_bt) local_bad |= BA_META_DEPTH_TOTAL;
  }
  if (local_bad) atomicOr(&bad, local_bad);
  __syncthreads();
  if (tid == 0 && bad) flag(status, bad);
}

// ---- K2: per-branch sequence, per-row key intervals ----------------------
__global__ void plan_rows_kernel(const int32_t *cu, const int32_t *anchor, int n_seqs,
                                 int n_main, int n_br, int mask, const int32_t *status,
                                 const int32_t *cu_branch, int32_t *branch_seq,
                                 int32_t *row_iv) {
  if (status[0] != 0) return;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n_main) {
    int r = (int)i;
    int s = upper_index(cu, n_seqs + 1, r);
    int4 v = make_int4(cu[s], r, 0, -1);
    reinterpret_cast<int4 *>(row_iv)[r] = v;
  }
  if (i < n_br) {
    int b = (int)i;
    int a = anchor[b];
    int s = upper_index(cu, n_seqs + 1, a);
    branch_seq[b] = s;
    int r0 = cu_branch[b], r1 = cu_branch[b + 1];
    for (int r = r0; r < r1; ++r) {
      int hi = (mask == BA_MASK_BLOCK_BIDIR) ? (r1 - 1) : r;
      reinterpret_cast<int4 *>(row_iv)[n_main + r] = make_int4(cu[s], a, r0, hi);
    }
  }
}

// ---- per key row: the query rows that see it ------------------------------
// Query rows of one kind (main rows, branch rows) have non-decreasing lower
// and upper key bounds (packed order; anchors non-decreasing), so the rows
// that see key k are one range: from the first row whose upper bound reaches
// k to the first row whose lower bound passes it.
__device__ int first_row_at_least(const int32_t *row_iv, int base, int n, int field, int k) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (row_iv[(int64_t)(base + mid) * 4 + field] >= k) hi = mid;
    else lo = mid + 1;
  }
  return lo;
}

__device__ int2 rows_seeing(const int32_t *row_iv, int base, int n, int f_lo, int f_hi, int k) {
  const int b = first_row_at_least(row_iv, base, n, f_hi, k);
  const int e = first_row_at_least(row_iv, base, n, f_lo, k + 1);
  return b < e ? make_int2(b, e) : make_int2(0, 0);
}

__global__ void plan_key_iv_kernel(int n_main, int n_bt, const int32_t *status,
                                   const int32_t *row_iv, int32_t *key_iv) {
  if (status[0] != 0) return;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)n_main + n_bt) return;
  int2 m = make_int2(0, 0), b;
  if (i < n_main) {
    m = rows_seeing(row_iv, 0, n_main, 0, 1, (int)i);
    b = rows_seeing(row_iv, n_main, n_bt, 0, 1, (int)i);
  } else {
    b = rows_seeing(row_iv, n_main, n_bt, 2, 3, (int)(i - n_main));
  }
  reinterpret_cast<int4 *>(key_iv)[i] = make_int4(m.x, m.y, b.x, b.y);
}

// ---- K3: per query tile key ranges ----------------------------------------
__global__ void plan_tiles_kernel(int n_main, int n_bt, int n_br, int n_qt_main, int n_qt,
                                  const int32_t *status, const int32_t *cu_branch,
                                  const int32_t *row_iv, int32_t *qtile, int32_t *fwd_cost) {
  if (status[0] != 0) return;
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= n_qt) return;
  const bool is_main = t < n_qt_main;
  const int tt = is_main ? t : t - n_qt_main;
  const int rows = is_main ? n_main : n_bt;
  const int off = is_main ? 0 : n_main;
  const int r0 = tt * kTileM, r1 = min(r0 + kTileM, rows) - 1;
  const int4 f = reinterpret_cast<const int4 *>(row_iv)[off + r0];
  const int4 l = reinterpret_cast<const int4 *>(row_iv)[off + r1];
  const int seq_start = f.x, a_lo = f.y, a_hi = l.y;
  const bool same_seq = f.x == l.x;
  const int kv_begin = seq_start / kTileN;
  const int kv_end = a_hi / kTileN + 1;
  int fb = (seq_start + kTileN - 1) / kTileN;
  int fe = (a_lo + 1) / kTileN;
  if (!same_seq || fb >= fe) { fb = kv_begin; fe = kv_begin; }
  int bl_b = 0, bl_e = 0;
  if (!is_main) {
    bl_b = f.z;  // cu_branch[b_lo]
    // b_hi: branch whose rows contain r1
    int lo = 0, hi = n_br - 1;
    while (lo < hi) {
      int mid = (lo + hi + 1) >> 1;
      if (cu_branch[mid] <= r1) lo = mid; else hi = mid - 1;
    }
    bl_e = cu_branch[lo + 1];
  }
  int32_t *q = qtile + (int64_t)t * 6;
  q[0] = kv_begin; q[1] = fb; q[2] = fe; q[3] = kv_end; q[4] = bl_b; q[5] = bl_e;
  fwd_cost[t] = (kv_end - kv_begin) + (bl_e - bl_b + kTileN - 1) / kTileN;
}

// first t in [lo, hi) with key(t) > x, for key non-decreasing; hi if none
template <int FIELD>
__device__ __forceinline__ int first_greater(const int32_t *qtile, int lo, int hi, int x) {
  while (lo < hi) {
    int mid = (lo + hi) >> 1;
    if (qtile[(int64_t)mid * 6 + FIELD] > x) hi = mid; else lo = mid + 1;
  }
  return lo;
}

// ---- K4: per key tile query-tile ranges (backward) -------------------------
__global__ void plan_kv_kernel(int n_bt, int n_qt_main, int n_qt, int n_kt, int n_bkt,
                               int32_t *status, const int32_t *qtile, int32_t *kv_main,
                               int32_t *kv_branch, int32_t *bwd_cost) {
  if (status[0] != 0) return;
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  int cost = 0;
  if (k < n_kt) {
    int out[4];
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      const int lo = part == 0 ? 0 : n_qt_main, hi = part == 0 ? n_qt_main : n_qt;
      int t1 = first_greater<3>(qtile, lo, hi, k);      // first with kv_end > k
      int t2 = first_greater<0>(qtile, lo, hi, k) - 1;  // last with kv_begin <= k
      if (t1 <= t2) { out[2 * part] = t1 - lo; out[2 * part + 1] = t2 + 1 - lo; }
      else { out[2 * part] = 0; out[2 * part + 1] = 0; }
    }
    int32_t *o = kv_main + (int64_t)k * 4;
    o[0] = out[0]; o[1] = out[1]; o[2] = out[2]; o[3] = out[3];
    cost = (out[1] - out[0]) + (out[3] - out[2]);
    bwd_cost[k] = cost;
  } else if (k < n_kt + n_bkt) {
    const int kb = k - n_kt;
    const int key_lo = kb * kTileN, key_hi = min(key_lo + kTileN, n_bt);
    int t1 = first_greater<5>(qtile, n_qt_main, n_qt, key_lo);          // bl_end > key_lo
    int t2 = first_greater<4>(qtile, n_qt_main, n_qt, key_hi - 1) - 1;  // bl_begin < key_hi
    int b = 0, e = 0;
    if (t1 <= t2) { b = t1 - n_qt_main; e = t2 + 1 - n_qt_main; }
    kv_branch[(int64_t)kb * 2] = b;
    kv_branch[(int64_t)kb * 2 + 1] = e;
    cost = e - b;
    bwd_cost[k] = cost;
  }
  // status word 2: the backward's whole walk (query tiles over all key tiles)
  cost = __reduce_add_sync(0xffffffffu, cost);
  if ((threadIdx.x & 31) == 0 && cost) atomicAdd(status + 2, cost);
}

// ---- K5: stable order by decreasing cost (rank by counting) ---------------
// prefix (optional): at each position of the order, the cost summed over the
// entries ranked before it.
constexpr int kRankThreads = 256;
__global__ void __launch_bounds__(kRankThreads) plan_rank_kernel(const int32_t *status,
                                                                 const int32_t *cost, int n,
                                                                 int32_t *order, int32_t *prefix) {
  if (status[0] != 0) return;
  __shared__ int32_t sc[kRankThreads];
  const int i = blockIdx.x * kRankThreads + threadIdx.x;
  const int ci = i < n ? cost[i] : 0;
  int rank = 0, ahead = 0;
  for (int base = 0; base < n; base += kRankThreads) {
    __syncthreads();
    int j = base + threadIdx.x;
    sc[threadIdx.x] = j < n ? cost[j] : INT32_MIN;
    __syncthreads();
    const int lim = min(kRankThreads, n - base);
    for (int u = 0; u < lim; ++u) {
      int cu_ = sc[u];
      int j2 = base + u;
      const bool before = (cu_ > ci) || (cu_ == ci && j2 < i);
      rank += before;
      ahead += before ? cu_ : 0;
    }
  }
  if (i < n) {
    order[rank] = i;
    if (prefix) prefix[rank] = ahead;
  }
}

// ---- K6: zigzag ring-step key-tile ranges ----------------------------------
// Row windows at ring step s: the row's chunk c (of its own position, or its
// anchor's) lies in shard i = c < C ? c : 2C-1-c; it reads the main keys of
// shard j = (i - s) mod C, i.e. chunks j and 2C-1-j of the same sequence,
// intersected with its causal interval.
__device__ __forceinline__ void zz_row_windows(const int32_t *cu, int n_seqs, int C, int step,
                                               int seq_start, int hi_key, int lo_key,
                                               int w[4]) {
  const int s = upper_index(cu, n_seqs + 1, seq_start);
  const int64_t L = cu[s + 1] - seq_start;
  const int64_t pos = hi_key - seq_start;  // own position / anchor position
  const int c = (int)((2 * C * (pos + 1) - 1) / L);
  const int shard = c < C ? c : 2 * C - 1 - c;
  const int j = ((shard - step) % C + C) % C;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int ch = k == 0 ? j : 2 * C - 1 - j;
    int a = seq_start + (int)((ch * L) / (2 * C));
    int b = seq_start + (int)(((ch + 1) * L) / (2 * C)) - 1;
    a = max(a, lo_key);
    b = min(b, hi_key);
    w[2 * k] = a;
    w[2 * k + 1] = b;  // empty when b < a
  }
}

__global__ void plan_zz_kernel(const int32_t *cu, int n_seqs, int C, int n_main, int n_bt,
                               int n_qt_main, int n_qt, const int32_t *status,
                               const int32_t *row_iv, int32_t *zz) {
  if (status[0] != 0) return;
  const int64_t gi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (gi >= (int64_t)C * n_qt) return;
  const int step = (int)(gi / n_qt), t = (int)(gi % n_qt);
  const bool is_main = t < n_qt_main;
  const int tt = is_main ? t : t - n_qt_main;
  const int rows = is_main ? n_main : n_bt;
  const int off = is_main ? 0 : n_main;
  const int r0 = tt * kTileM, r1 = min(r0 + kTileM, rows);
  int lo0 = INT32_MAX, hi0 = -1, lo1 = INT32_MAX, hi1 = -1;
  for (int r = r0; r < r1; ++r) {
    int4 iv = reinterpret_cast<const int4 *>(row_iv)[off + r];
    int w[4];
    zz_row_windows(cu, n_seqs, C, step, iv.x, iv.y, iv.x, w);
    if (w[1] >= w[0]) { lo0 = min(lo0, w[0]); hi0 = max(hi0, w[1]); }
    if (w[3] >= w[2]) { lo1 = min(lo1, w[2]); hi1 = max(hi1, w[3]); }
  }
  int32_t *o = zz + gi * 4;
  o[0] = hi0 >= 0 ? lo0 / kTileN : 0;
  o[1] = hi0 >= 0 ? hi0 / kTileN + 1 : 0;
  o[2] = hi1 >= 0 ? lo1 / kTileN : 0;
  o[3] = hi1 >= 0 ? hi1 / kTileN + 1 : 0;
}

// ---- ring steps (zigzag context parallelism across ranks) -----------------
// A rank holding shard q keeps chunks q and 2C-1-q of every sequence (chunk k
// of a sequence of length L covers positions [floor(kL/2C), floor((k+1)L/2C)))
// as one packed problem, in position order.  Against the main keys of another
// shard j (held in the same shard-local order by the rank it came from), a
// chunk of keys is either wholly before a query's position or wholly after it:
//   j < q: every query of the sequence sees shard j's first chunk (chunk j);
//   j > q: queries in the second chunk (2C-1-q) see all of shard j's keys of
//          the sequence, queries in the first chunk none.
// A branch query takes its anchor's chunk (the anchor is a main position).
// Step 0 (j = q) is the causal plan of the shard-local problem itself.
__device__ __forceinline__ int chunk_len(int64_t L, int C, int k) {
  return (int)(((k + 1) * L) / (2 * C) - (k * L) / (2 * C));
}

__device__ __forceinline__ int2 ring_interval(const int32_t *cu_loc, const int32_t *cu_glob,
                                              const int32_t *cu_vis, int n_seqs, int C, int q,
                                              int j, int local_row) {
  const int s = upper_index(cu_loc, n_seqs + 1, local_row);
  const int pos = local_row - cu_loc[s];
  const int64_t L = cu_glob[s + 1] - cu_glob[s];
  const bool second = pos >= chunk_len(L, C, q);
  const int lo = cu_vis[s];
  int hi;
  if (j < q) hi = lo + chunk_len(L, C, j) - 1;
  else hi = second ? cu_vis[s + 1] - 1 : lo - 1;
  return make_int2(lo, hi);
}

__global__ void plan_ring_rows_kernel(const int32_t *cu_loc, const int32_t *cu_glob,
                                      const int32_t *cu_vis, const int32_t *anchor, int n_seqs,
                                      int n_main, int n_br, int C, int q, int j,
                                      const int32_t *status, const int32_t *cu_branch,
                                      int32_t *row_iv) {
  if (status[0] != 0) return;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n_main) {
    const int2 v = ring_interval(cu_loc, cu_glob, cu_vis, n_seqs, C, q, j, (int)i);
    reinterpret_cast<int4 *>(row_iv)[i] = make_int4(v.x, v.y, 0, -1);
  }
  if (i < n_br) {
    const int b = (int)i;
    const int2 v = ring_interval(cu_loc, cu_glob, cu_vis, n_seqs, C, q, j, anchor[b]);
    for (int r = cu_branch[b]; r < cu_branch[b + 1]; ++r)
      reinterpret_cast<int4 *>(row_iv)[n_main + r] = make_int4(v.x, v.y, 0, -1);
  }
}

// Per query tile: the key tiles any row sees, and those every row sees whole.
__global__ void plan_ring_tiles_kernel(int n_main, int n_bt, int n_qt_main, int n_qt,
                                       const int32_t *status, const int32_t *row_iv,
                                       int32_t *qtile, int32_t *fwd_cost) {
  if (status[0] != 0) return;
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= n_qt) return;
  const bool is_main = t < n_qt_main;
  const int tt = is_main ? t : t - n_qt_main;
  const int rows = is_main ? n_main : n_bt;
  const int off = is_main ? 0 : n_main;
  const int r0 = tt * kTileM, r1 = min(r0 + kTileM, rows);
  int lo_min = INT32_MAX, hi_max = -1, lo_max = -1, hi_min = INT32_MAX;
  bool every = r1 - r0 == kTileM;
  for (int r = r0; r < r1; ++r) {
    const int4 iv = reinterpret_cast<const int4 *>(row_iv)[off + r];
    if (iv.y >= iv.x) {
      lo_min = min(lo_min, iv.x); hi_max = max(hi_max, iv.y);
      lo_max = max(lo_max, iv.x); hi_min = min(hi_min, iv.y);
    } else {
      every = false;
    }
  }
  int kb = 0, ke = 0, fb = 0, fe = 0;
  if (hi_max >= 0) {
    kb = lo_min / kTileN;
    ke = hi_max / kTileN + 1;
    fb = (lo_max + kTileN - 1) / kTileN;
    fe = (hi_min + 1) / kTileN;
    if (!every || fb >= fe) { fb = kb; fe = kb; }
  }
  int32_t *o = qtile + (int64_t)t * 6;
  o[0] = kb; o[1] = fb; o[2] = fe; o[3] = ke; o[4] = 0; o[5] = 0;
  fwd_cost[t] = ke - kb;
}

}  // namespace

ba_status launch_ring_plan(const ba_problem &p, const ba_plan_layout &L, const PlanView &v,
                           const int32_t *cu_glob, const int32_t *cu_vis, int C, int q, int j,
                           cudaStream_t s) {
  const int n_qt = L.n_qtiles_main + L.n_qtiles_branch;
  plan_scan_kernel<<<1, kScanThreads, 0, s>>>(p.cu_seqlens, p.branch_anchor, p.branch_depth,
                                              p.n_seqs, p.n_main, p.n_branches,
                                              p.n_branch_tokens, v.status, v.cu_branch);
  ba_status st = cuda_check(cudaGetLastError(), "plan_scan_kernel launch");
  if (st != BA_OK) return st;
  const int64_t nrow = p.n_main > p.n_branches ? p.n_main : p.n_branches;
  plan_ring_rows_kernel<<<(unsigned)cdiv64(nrow, 256), 256, 0, s>>>(
      p.cu_seqlens, cu_glob, cu_vis, p.branch_anchor, p.n_seqs, p.n_main, p.n_branches, C, q, j,
      v.status, v.cu_branch, v.row_iv);
  plan_ring_tiles_kernel<<<(unsigned)cdiv64(n_qt, 128), 128, 0, s>>>(
      p.n_main, p.n_branch_tokens, L.n_qtiles_main, n_qt, v.status, v.row_iv, v.qtile,
      v.fwd_cost);
  plan_rank_kernel<<<(unsigned)cdiv64(n_qt, kRankThreads), kRankThreads, 0, s>>>(
      v.status, v.fwd_cost, n_qt, v.fwd_order, nullptr);
  count_launches(4);
  return cuda_check(cudaGetLastError(), "ring plan kernels launch");
}

ba_status launch_plan(const ba_problem &p, const ba_plan_layout &L, const PlanView &v,
                      cudaStream_t s) {
  const int n_qt = L.n_qtiles_main + L.n_qtiles_branch;
  plan_scan_kernel<<<1, kScanThreads, 0, s>>>(p.cu_seqlens, p.branch_anchor, p.branch_depth,
                                              p.n_seqs, p.n_main, p.n_branches,
                                              p.n_branch_tokens, v.status, v.cu_branch);
  ba_status st = cuda_check(cudaGetLastError(), "plan_scan_kernel launch");
  if (st != BA_OK) return st;
  const int64_t nrow = p.n_main > p.n_branches ? p.n_main : p.n_branches;
  plan_rows_kernel<<<(unsigned)cdiv64(nrow, 256), 256, 0, s>>>(
      p.cu_seqlens, p.branch_anchor, p.n_seqs, p.n_main, p.n_branches, p.mask, v.status,
      v.cu_branch, v.branch_seq, v.row_iv);
  plan_tiles_kernel<<<(unsigned)cdiv64(n_qt, 128), 128, 0, s>>>(
      p.n_main, p.n_branch_tokens, p.n_branches, L.n_qtiles_main, n_qt, v.status,
      v.cu_branch, v.row_iv, v.qtile, v.fwd_cost);
  const int n_kv = L.n_kv_main + L.n_kv_branch;
  plan_kv_kernel<<<(unsigned)cdiv64(n_kv, 128), 128, 0, s>>>(
      p.n_branch_tokens, L.n_qtiles_main, n_qt, L.n_kv_main, L.n_kv_branch, v.status,
      v.qtile, v.kv_main, v.kv_branch, v.bwd_cost);
  plan_rank_kernel<<<(unsigned)cdiv64(n_qt, kRankThreads), kRankThreads, 0, s>>>(
      v.status, v.fwd_cost, n_qt, v.fwd_order, nullptr);
  plan_rank_kernel<<<(unsigned)cdiv64(n_kv, kRankThreads), kRankThreads, 0, s>>>(
      v.status, v.bwd_cost, n_kv, v.bwd_order, v.bwd_prefix);
  const int64_t n_keys = (int64_t)p.n_main + p.n_branch_tokens;
  plan_key_iv_kernel<<<(unsigned)cdiv64(n_keys, 256), 256, 0, s>>>(
      p.n_main, p.n_branch_tokens, v.status, v.row_iv, v.key_iv);
  count_launches(7);
  if (p.zigzag_C > 1) {
    count_launches(1);
    const int64_t n = (int64_t)p.zigzag_C * n_qt;
    plan_zz_kernel<<<(unsigned)cdiv64(n, 128), 128, 0, s>>>(
        p.cu_seqlens, p.n_seqs, p.zigzag_C, p.n_main, p.n_branch_tokens, L.n_qtiles_main,
        n_qt, v.status, v.row_iv, v.zz_tiles);
  }
  return cuda_check(cudaGetLastError(), "plan kernels launch");
}

}  // namespace ba
