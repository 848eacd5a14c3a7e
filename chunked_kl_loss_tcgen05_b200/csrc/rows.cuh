// Per-row kernels around the GEMMs: valid-row count, teacher preparation,
// cross-CTA log-sum-exp merge with the per-row KL, and the final mean.
#pragma once

#include <climits>

#include "gemm.cuh"

namespace fckl {

constexpr int ROW_WARPS = 8;  // rows per 256-thread block in the warp-per-row kernels
constexpr int K_MAX = 256;

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// N_valid = #rows with row_mask != 0 (N when there is no mask).  One block.
__global__ void __launch_bounds__(1024) k_count_valid(const uint8_t* __restrict__ mask, long long N,
                                                      DeviceCtl* ctl) {
  __shared__ int red[32];
  int c = 0;
  if (mask == nullptr) {
    c = threadIdx.x == 0 ? (int)N : 0;
  } else {
    for (long long i = threadIdx.x; i < N; i += blockDim.x) c += mask[i] != 0;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x < 32) {
    c = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if (threadIdx.x == 0) ctl->n_valid = c;
  }
}

// Teacher side of one chunk, one warp per row: p = softmax(topk_logit / T)
// over the K cached logits, sum_k p_k log p_k, the (id, p) pairs sorted by id,
// and for every vocab tile of 256 columns the position of its first id in the
// sorted list (tstart, NT + 1 entries per row), so that a GEMM epilogue finds
// the cached ids of its tile with one load.  Ids outside [0, V) are recorded
// as an error and replaced by INT_MAX, which no vocab column matches.
__global__ void __launch_bounds__(ROW_WARPS * 32)
    k_prep_teacher(const int32_t* __restrict__ ids, const float* __restrict__ lg,
                   const uint8_t* __restrict__ mask, int rows_c, int K, int V, int NT,
                   float invT, int* __restrict__ sid, float* __restrict__ sp,
                   float* __restrict__ zs, uint16_t* __restrict__ tstart,
                   float* __restrict__ plogp, DeviceCtl* ctl) {
  __shared__ int s_ids[ROW_WARPS][K_MAX];
  __shared__ int s_sorted[ROW_WARPS][K_MAX];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * ROW_WARPS + warp;
  if (row >= rows_c) return;  // warp-uniform
  const bool keep = mask == nullptr || mask[row] != 0;
  float t[K_MAX / 32];
  int id[K_MAX / 32];
  float m = -INFINITY;
  bool bad_val = false, bad_id = false;
#pragma unroll
  for (int i = 0; i < K_MAX / 32; ++i) {
    const int k = lane + 32 * i;
    t[i] = -INFINITY;
    id[i] = INT_MAX;
    if (k < K) {
      const float x = lg[(size_t)row * K + k];
      int d = ids[(size_t)row * K + k];
      if (isnan(x) || x == INFINITY) bad_val = true;
      if (d < 0 || d >= V) { bad_id = true; d = INT_MAX; }
      t[i] = x * invT;
      id[i] = d;
      s_ids[warp][k] = d;
      m = fmaxf(m, t[i]);
    }
  }
  m = warp_max(m);
  bad_val = __any_sync(0xffffffffu, bad_val);
  bad_id = __any_sync(0xffffffffu, bad_id);
  if (keep && lane == 0) {
    if (bad_id) atomicOr(&ctl->err, kErrBadIndex);
    if (bad_val || !(m > -INFINITY)) atomicOr(&ctl->err, kErrBadTeacher);
  }
  const float ms = (m > -INFINITY && m < INFINITY) ? m : 0.f;
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < K_MAX / 32; ++i)
    if (lane + 32 * i < K) s += expf(t[i] - ms);
  s = warp_sum(s);
  const float lse = s > 0.f ? ms + logf(s) : INFINITY;
  float p[K_MAX / 32];
  float pl = 0.f;
#pragma unroll
  for (int i = 0; i < K_MAX / 32; ++i) {
    p[i] = 0.f;
    if (lane + 32 * i < K) {
      p[i] = expf(t[i] - lse);
      if (p[i] > 0.f) pl += p[i] * (t[i] - lse);
    }
  }
  pl = warp_sum(pl);
  __syncwarp();
#pragma unroll
  for (int i = 0; i < K_MAX / 32; ++i) {
    const int k = lane + 32 * i;
    if (k < K) {
      int rk = 0;
      for (int j = 0; j < K; ++j) {
        const int o = s_ids[warp][j];
        rk += (o < id[i]) || (o == id[i] && j < k);
      }
      sid[(size_t)row * K + rk] = id[i];
      sp[(size_t)row * K + rk] = p[i];
      zs[(size_t)row * K + rk] = 0.f;
      s_sorted[warp][rk] = id[i];
    }
  }
  __syncwarp();
  for (int vt = lane; vt <= NT; vt += 32) {  // lower bound of vt * 256 in the sorted ids
    const long long key = (long long)vt * BN;
    int lo = 0, hi = K;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if ((long long)s_sorted[warp][mid] < key) lo = mid + 1; else hi = mid;
    }
    tstart[(size_t)row * (NT + 1) + vt] = (uint16_t)lo;
  }
  if (lane == 0) plogp[row] = pl;
}

// Merge the per-vocab-tile (max, sum) partials of each row into its
// log-sum-exp (log2 domain, kept for the backward epilogue) and form the row
// loss  l_r = sum_k p_k log p_k - sum_k p_k (z_k / T - LSE_r),  0 for masked rows.
__global__ void __launch_bounds__(ROW_WARPS * 32)
    k_merge_loss(const float2* __restrict__ partials, int NT, int rows_c, int K, float invT,
                 const float* __restrict__ zs, const float* __restrict__ sp,
                 const float* __restrict__ plogp, const uint8_t* __restrict__ mask,
                 float* __restrict__ lse2_out, float* __restrict__ row_loss) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * ROW_WARPS + warp;
  if (row >= rows_c) return;
  const float2* pr = partials + (size_t)row * NT;
  float M = -INFINITY;
  for (int t = lane; t < NT; t += 32) M = fmaxf(M, pr[t].x);
  M = warp_max(M);
  float S = 0.f;
  for (int t = lane; t < NT; t += 32) {
    const float2 q = pr[t];
    if (q.x > -INFINITY) S += q.y * exp2f(q.x - M);
  }
  S = warp_sum(S);
  const float L2 = M + log2f(S);
  const float lse = L2 * 0.69314718055994530942f;
  float acc = 0.f;
  for (int k = lane; k < K; k += 32) {
    const float pk = sp[(size_t)row * K + k];
    if (pk > 0.f) acc += pk * fmaf(zs[(size_t)row * K + k], invT, -lse);
  }
  acc = warp_sum(acc);
  if (lane == 0) {
    const bool keep = mask == nullptr || mask[row] != 0;
    lse2_out[row] = L2;
    row_loss[row] = keep ? plogp[row] - acc : 0.f;
  }
}

// loss = sum(row_loss) / N_valid, fp64 accumulation in a fixed order.
__global__ void __launch_bounds__(1024) k_finalize(const float* __restrict__ row_loss, long long N,
                                                   const DeviceCtl* ctl, float* loss) {
  __shared__ double red[1024];
  double s = 0.0;
  for (long long i = threadIdx.x; i < N; i += blockDim.x) s += (double)row_loss[i];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = blockDim.x >> 1; w > 0; w >>= 1) {
    if ((int)threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const int n = ctl->n_valid;
    *loss = n > 0 ? (float)(red[0] / (double)n) : 0.f;
  }
}

}  // namespace fckl
