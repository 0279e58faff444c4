// Streaming (HBM-bound) kernels: the standalone online-softmax merge, the
// backward preprocess D = rowsum(dO * O), and the dQ fp32 -> bf16 convert.
// All use 16-byte vector accesses and a grid of (SM count x resident blocks)
// that strides over the work: the merge and the convert take one row-head
// per group of lanes, the preprocess one row per lane (32 rows of one head
// per warp, so that its per-head outputs are written in contiguous runs).
#include "internal.cuh"

namespace ba {
namespace {

__device__ __forceinline__ void unpack8(const uint4 &u, float f[8]) {
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

__device__ __forceinline__ uint4 pack8(const float f[8]) {
  uint4 u;
  __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
  return u;
}

int grid_for(int64_t groups, int groups_per_block) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t need = cdiv64(groups, groups_per_block);
  int64_t cap = (int64_t)sms * 8;
  return (int)(need < cap ? (need > 0 ? need : 1) : cap);
}

// ---- online-softmax merge --------------------------------------------------
// l = log(e^{l_a} + e^{l_b}), O = e^{l_a - l} O_a + e^{l_b - l} O_b, with
// m = max(l_a, l_b) subtracted first; an empty side (-inf) has weight 0.
template <bool FP32, int D>
__global__ void __launch_bounds__(256) lse_merge_kernel(int64_t rows, int heads,
                                                        const void *oa, const float *la,
                                                        const void *ob, const float *lb,
                                                        void *oo, float *lo) {
  constexpr int kElems = FP32 ? 4 : 8;       // elements per 16-byte access
  constexpr int kLanes = D / kElems;         // lanes per row-head
  constexpr int kPerWarp = 32 / kLanes;      // row-heads per warp pass
  const int lane = threadIdx.x % kLanes;
  const int64_t total = rows * heads;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
  // warp-uniform trip count: every lane of a warp runs the same iterations
  for (int64_t w = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
       w * kPerWarp < total; w += warps) {
    const int64_t g = w * kPerWarp + (threadIdx.x % 32) / kLanes;
    const bool active = g < total;
    float l = 0.f;
    int64_t li = 0;
    if (active) {
      const int64_t row = g / heads;
      const int h = (int)(g % heads);
      li = (int64_t)h * rows + row;
      const float a = la[li], b = lb[li];
      const float m = fmaxf(a, b);
      float wa, wb;
      if (m == -INFINITY) {
        l = -INFINITY; wa = 0.f; wb = 0.f;
      } else {
        const float ea = expf(a - m), eb = expf(b - m);
        l = m + logf(ea + eb);
        wa = expf(a - l);
        wb = expf(b - l);
      }
      const int64_t base = g * D + lane * kElems;
      if (FP32) {
        float4 x = reinterpret_cast<const float4 *>(oa)[base / 4];
        float4 y = reinterpret_cast<const float4 *>(ob)[base / 4];
        float4 z;
        z.x = wa * x.x + wb * y.x; z.y = wa * x.y + wb * y.y;
        z.z = wa * x.z + wb * y.z; z.w = wa * x.w + wb * y.w;
        reinterpret_cast<float4 *>(oo)[base / 4] = z;
      } else {
        float x[8], y[8], z[8];
        unpack8(reinterpret_cast<const uint4 *>(oa)[base / 8], x);
        unpack8(reinterpret_cast<const uint4 *>(ob)[base / 8], y);
#pragma unroll
        for (int i = 0; i < 8; ++i) z[i] = wa * x[i] + wb * y[i];
        reinterpret_cast<uint4 *>(oo)[base / 8] = pack8(z);
      }
    }
    // all lanes of the group have read lse_a before it is overwritten (in-place
    // accumulation aliases lse_out with lse_a)
    __syncwarp();
    if (active && lane == 0) lo[li] = l;
  }
}

// ---- backward preprocess ---------------------------------------------------
// D[h, row] = sum_d dO[row, h, d] * O[row, h, d] (fp32 accumulate), rows =
// main rows then branch rows, and the per-query records the backward reads
// {l log2 e, D}, laid out as two arrays of 128 per 128-row block.
// A warp takes 32 consecutive rows of one head, one lane per row: each lane
// streams its row's 2 d bf16 of O and dO (16-byte loads, all issued before
// the products), and the warp's writes of D and of each record field are
// 128-byte contiguous runs.  When the backward accumulates dQ in fp32 the
// accumulator of the same row-head is zeroed in the same pass.
template <int D>
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(AttnParams a) {
  constexpr int kVec = D / 8;  // 16-byte vectors per row-head
  if (a.plan.status[0] != 0) return;
  const int64_t rows = (int64_t)a.n_main + a.n_bt;
  const int64_t blocks32 = (rows + 31) / 32;
  const int64_t tasks = blocks32 * a.hq;
  const int lane = threadIdx.x % 32;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
  for (int64_t w = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32; w < tasks;
       w += warps) {
    const int h = (int)(w % a.hq);
    const int64_t row = (w / a.hq) * 32 + lane;
    if (row >= rows) continue;
    const bool is_main = row < a.n_main;
    const int64_t r = is_main ? row : row - a.n_main;
    const int64_t off = (r * a.hq + h) * D;
    const uint4 *o4 = reinterpret_cast<const uint4 *>((is_main ? a.o_m : a.o_b) + off);
    const uint4 *d4 = reinterpret_cast<const uint4 *>((is_main ? a.do_m : a.do_b) + off);
    uint4 ov[kVec], dv[kVec];
#pragma unroll
    for (int i = 0; i < kVec; ++i) {
      ov[i] = o4[i];
      dv[i] = d4[i];
    }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < kVec; ++i) {
      float x[8], y[8];
      unpack8(ov[i], x);
      unpack8(dv[i], y);
#pragma unroll
      for (int e = 0; e < 8; ++e) s = fmaf(x[e], y[e], s);
    }
    if (a.zero_dq_acc) {
      float4 *dq = reinterpret_cast<float4 *>(a.dq_acc + (row * a.hq + h) * D);
#pragma unroll
      for (int i = 0; i < D / 4; ++i) dq[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const_cast<float *>(a.d_all)[(int64_t)h * rows + row] = s;
    const float l2 = (is_main ? a.lse_m : a.lse_b)[(int64_t)h * (is_main ? a.n_main : a.n_bt) + r] *
                     1.4426950408889634f;
    const int64_t pr = (is_main ? 0 : a.n_main_pad) + r;
    float *r0 = a.rec + rec_block(h, a.rows_pad, pr) + (pr & 127);
    r0[kRecLse] = l2;
    r0[kRecD] = s;
  }
  // padding rows of the records (no query sees a key through them)
  const int pad_m = a.n_main_pad - a.n_main;
  const int pad_b = a.rows_pad - a.n_main_pad - a.n_bt;
  const int64_t n_pad = (int64_t)(pad_m + pad_b) * a.hq;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_pad;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int per = pad_m + pad_b;
    const int64_t kh = i / per;
    const int j = (int)(i % per);
    const int64_t pr = j < pad_m ? a.n_main + j : a.n_main_pad + a.n_bt + (j - pad_m);
    float *rp = a.rec + rec_block(kh, a.rows_pad, pr) + (pr & 127);
    rp[kRecLse] = 0.f;
    rp[kRecD] = 0.f;
  }
}

// ---- dQ convert: dq = scale * dq_acc, fp32 -> bf16 -------------------------
__global__ void __launch_bounds__(256) dq_convert_kernel(const float *acc, int64_t n_main_elems,
                                                         int64_t n_total_elems, float scale,
                                                         int32_t const *status,
                                                         __nv_bfloat16 *dq_m,
                                                         __nv_bfloat16 *dq_b) {
  if (status[0] != 0) return;
  const int64_t n8 = n_total_elems / 8;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float4 u = reinterpret_cast<const float4 *>(acc)[2 * i];
    const float4 v = reinterpret_cast<const float4 *>(acc)[2 * i + 1];
    float f[8] = {u.x * scale, u.y * scale, u.z * scale, u.w * scale,
                  v.x * scale, v.y * scale, v.z * scale, v.w * scale};
    const int64_t e = i * 8;
    uint4 packed = pack8(f);
    if (e < n_main_elems) reinterpret_cast<uint4 *>(dq_m)[e / 8] = packed;
    else reinterpret_cast<uint4 *>(dq_b)[(e - n_main_elems) / 8] = packed;
  }
}

}  // namespace

ba_status launch_lse_merge(int64_t rows, int heads, int d, int fp32, const void *oa,
                           const float *la, const void *ob, const float *lb, void *oo,
                           float *lo, cudaStream_t s) {
  const int64_t groups = rows * heads;
  if (groups == 0) return BA_OK;
#define BA_MERGE_LAUNCH(F, DD)                                                       \
  {                                                                                  \
    constexpr int lanes = DD / ((F) ? 4 : 8);                                        \
    lse_merge_kernel<F, DD><<<grid_for(groups, 256 / lanes), 256, 0, s>>>(           \
        rows, heads, oa, la, ob, lb, oo, lo);                                        \
  }
  if (fp32 && d == 64) BA_MERGE_LAUNCH(true, 64)
  else if (fp32 && d == 128) BA_MERGE_LAUNCH(true, 128)
  else if (!fp32 && d == 64) BA_MERGE_LAUNCH(false, 64)
  else BA_MERGE_LAUNCH(false, 128)
#undef BA_MERGE_LAUNCH
  count_launches(1);
  return cuda_check(cudaGetLastError(), "lse_merge launch");
}

ba_status launch_bwd_preprocess(const AttnParams &a, cudaStream_t s) {
  // one warp task per 32 rows of one head; 8 warps per block
  const int64_t tasks = (((int64_t)a.n_main + a.n_bt + 31) / 32) * a.hq;
  if (a.head_dim == 64)
    bwd_preprocess_kernel<64><<<grid_for(tasks, 8), 256, 0, s>>>(a);
  else
    bwd_preprocess_kernel<128><<<grid_for(tasks, 8), 256, 0, s>>>(a);
  count_launches(1);
  return cuda_check(cudaGetLastError(), "bwd_preprocess launch");
}

ba_status launch_dq_convert(const AttnParams &a, __nv_bfloat16 *dq_m, __nv_bfloat16 *dq_b,
                            cudaStream_t s) {
  const int64_t per_row = (int64_t)a.hq * a.head_dim;
  const int64_t n_main_elems = (int64_t)a.n_main * per_row;
  const int64_t n_total = ((int64_t)a.n_main + a.n_bt) * per_row;
  dq_convert_kernel<<<grid_for(n_total / 8, 256), 256, 0, s>>>(
      a.dq_acc, n_main_elems, n_total, a.scale, a.plan.status, dq_m, dq_b);
  count_launches(1);
  return cuda_check(cudaGetLastError(), "dq_convert launch");
}

}  // namespace ba
