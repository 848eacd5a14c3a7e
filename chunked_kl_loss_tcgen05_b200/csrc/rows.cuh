// Per-row kernels around the GEMMs: valid-row count, teacher preparation,
// cross-CTA log-sum-exp merge with the per-row KL, and the final mean.
#pragma once

#include <climits>

#include <cuda_bf16.h>

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
__device__ __forceinline__ int warp_sum_int(int x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// N_valid = #rows with row_mask != 0 (N when there is no mask), or the
// caller's total (> 0) when the rows are one shard of a larger batch.  One block.
__global__ void __launch_bounds__(1024) k_count_valid(const uint8_t* __restrict__ mask, long long N,
                                                      int total, DeviceCtl* ctl) {
  pdl_wait();
  pdl_trigger();
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
    if (threadIdx.x == 0) ctl->n_valid = total > 0 ? total : c;
  }
}

// N_valid for a row list: entries in [0, N) count; negative entries are
// padding and are skipped; entries >= N are reported as bad indices.  One block.
__global__ void __launch_bounds__(1024) k_count_list(const int32_t* __restrict__ rows, long long n,
                                                     long long N, int total, DeviceCtl* ctl) {
  pdl_wait();
  pdl_trigger();
  __shared__ int red[32];
  int c = 0;
  bool bad = false;
  for (long long i = threadIdx.x; i < n; i += blockDim.x) {
    const int r = rows[i];
    c += (r >= 0 && r < N);
    bad |= r >= N;
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(&ctl->err, kErrBadIndex);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x < 32) {
    c = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if (threadIdx.x == 0) ctl->n_valid = total > 0 ? total : c;
  }
}

// dW = 0 when the call compacted no row (then no dW launch writes it);
// otherwise nothing.
__global__ void k_zero_if_no_valid(float4* __restrict__ out, long long n4, const DeviceCtl* ctl) {
  pdl_trigger();  // the dW GEMM after it may start its main loop
  pdl_wait();
  if (ctl->n_rows > 0) return;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4;
       i += (long long)gridDim.x * blockDim.x)
    out[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// Gather the listed rows of one chunk (block i copies list entry i): hidden
// row -> hst[i] (bf16, 16-byte vectors), teacher ids/logits -> idst/lgst[i],
// mst[i] = 1.  Entries outside [0, N) give a zero row with mst[i] = 0.
// When the row count n is read on the device (fewer rows than the launch's
// blocks), blocks n .. n+63 zero their staged hidden row and, if dlz is given,
// their dlogits row (dl_u4 16-byte words each): the dW GEMM reads whole blocks
// of 64 rows, and the rows past n that its last block covers must be zero.
__global__ void __launch_bounds__(128)
    k_gather_rows(const int32_t* __restrict__ list, RowCount rc, long long N, int H, int K,
                  const __nv_bfloat16* __restrict__ hidden, const int32_t* __restrict__ ids,
                  const float* __restrict__ lg, __nv_bfloat16* __restrict__ hst,
                  int32_t* __restrict__ idst, float* __restrict__ lgst, uint8_t* __restrict__ mst,
                  uint4* __restrict__ dlz, long long dl_u4) {
  pdl_wait();
  pdl_trigger();
  const int i = blockIdx.x;
  const int n = rc.get();
  if (i >= n) {
    if (i >= n + 64) return;
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    uint4* hrow = reinterpret_cast<uint4*>(hst + (size_t)i * H);
    for (int j = threadIdx.x; j < H / 8; j += blockDim.x) hrow[j] = zero;
    if (dlz != nullptr)
      for (long long j = threadIdx.x; j < dl_u4; j += blockDim.x) dlz[(size_t)i * dl_u4 + j] = zero;
    return;
  }
  const int r = list[i];
  const bool ok = r >= 0 && r < N;
  const uint4* src = reinterpret_cast<const uint4*>(hidden + (size_t)(ok ? r : 0) * H);
  uint4* dst = reinterpret_cast<uint4*>(hst + (size_t)i * H);
  for (int j = threadIdx.x; j < H / 8; j += blockDim.x)
    dst[j] = ok ? src[j] : make_uint4(0u, 0u, 0u, 0u);
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    idst[(size_t)i * K + k] = ok ? ids[(size_t)r * K + k] : 0;
    lgst[(size_t)i * K + k] = ok ? lg[(size_t)r * K + k] : 0.f;
  }
  if (threadIdx.x == 0) mst[i] = ok ? 1 : 0;
}

// Order-preserving map of a float to uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t float_key(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Exclusive block-wide prefix sum of one int per thread (blockDim.x = 1024).
__device__ __forceinline__ int block_exclusive_scan(int v, int* sh, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < (int)(blockDim.x >> 5) ? sh[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    sh[lane] = w;  // inclusive warp totals
  }
  __syncthreads();
  const int before = (warp > 0 ? sh[warp - 1] : 0) + x - v;
  *total = sh[(blockDim.x >> 5) - 1];
  __syncthreads();
  return before;
}

// Row indices of the valid rows (row_mask != 0), ascending, into list[0, n),
// n into ctl->n_rows and N_v (n, or the caller's global total when > 0) into
// ctl->n_valid, in two passes over kCompactBlocks blocks: block b owns rows
// [b*R, (b+1)*R) (R a multiple of 4096).  Pass 1 counts each block's valid
// rows into ctl->block_count[b]; pass 2 starts block b at the sum of the
// counts before it and writes its rows 4096 at a time (thread t takes 4
// consecutive rows; a block-wide prefix sum gives every thread its position).
__global__ void __launch_bounds__(1024) k_compact_count(const uint8_t* __restrict__ mask,
                                                        long long N, long long R, DeviceCtl* ctl) {
  pdl_wait();
  pdl_trigger();
  __shared__ int red[32];
  const long long r0 = blockIdx.x * R, r1 = (r0 + R < N) ? r0 + R : N;
  int c = 0;
  for (long long i = r0 + threadIdx.x; i < r1; i += blockDim.x) c += mask[i] != 0;
  c = warp_sum_int(c);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x < 32) {
    c = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0;
    c = warp_sum_int(c);
    if (threadIdx.x == 0) ctl->block_count[blockIdx.x] = c;
  }
}

__global__ void __launch_bounds__(1024) k_compact_write(const uint8_t* __restrict__ mask,
                                                        long long N, long long R, int total,
                                                        int32_t* __restrict__ list,
                                                        DeviceCtl* ctl) {
  pdl_wait();
  pdl_trigger();
  __shared__ int sh[32];
  __shared__ int s_base, s_total;
  if (threadIdx.x == 0) {
    int before = 0, all = 0;
    for (int b = 0; b < (int)gridDim.x; ++b) {
      const int cb = ctl->block_count[b];
      before += b < (int)blockIdx.x ? cb : 0;
      all += cb;
    }
    s_base = before;
    s_total = all;
  }
  __syncthreads();
  int base = s_base;
  const long long r0 = blockIdx.x * R, r1 = (r0 + R < N) ? r0 + R : N;
  for (long long t0 = r0; t0 < r1; t0 += 4 * (long long)blockDim.x) {
    const long long i0 = t0 + 4 * (long long)threadIdx.x;
    int f = 0;  // bit k: row i0 + k is valid
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (i0 + k < r1 && mask[i0 + k] != 0) f |= 1 << k;
    int tile_total;
    int pos = base + block_exclusive_scan(__popc(f), sh, &tile_total);
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (f & (1 << k)) list[pos++] = (int32_t)(i0 + k);
    base += tile_total;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    ctl->n_rows = s_total;
    ctl->n_valid = total > 0 ? total : s_total;
  }
}

// Top-n rows by score among valid rows (row_mask != 0, or all), one block:
// an MSB-first radix select (8 bits per pass) finds the n-th largest key, then
// every row above it and the lowest-index rows equal to it are written to
// rows_out in ascending row order.  n = min(n_select, valid rows); the rest of
// rows_out[0, n_select) is set to -1 and *count_out = n.
__global__ void __launch_bounds__(1024)
    k_select_top_rows(const float* __restrict__ score, const uint8_t* __restrict__ mask,
                      long long N, long long n_select, int32_t* __restrict__ rows_out,
                      int32_t* __restrict__ count_out) {
  __shared__ int hist[256];
  __shared__ int sh[32];
  __shared__ uint32_t s_prefix, s_need;
  const int tid = threadIdx.x;
  // number of valid rows
  int cnt = 0;
  for (long long i = tid; i < N; i += blockDim.x) cnt += (mask == nullptr || mask[i] != 0);
  int nvalid = 0;
  block_exclusive_scan(cnt, sh, &nvalid);
  const long long n = n_select < nvalid ? n_select : nvalid;
  uint32_t prefix = 0, need = (uint32_t)n;  // need: how many keys >= threshold still to take
  if (n > 0) {
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      const uint32_t hi_mask = pass == 0 ? 0u : (0xFFFFFFFFu << (32 - 8 * pass));
      for (int b = tid; b < 256; b += blockDim.x) hist[b] = 0;
      __syncthreads();
      for (long long i = tid; i < N; i += blockDim.x) {
        if (mask != nullptr && mask[i] == 0) continue;
        const uint32_t k = float_key(score[i]);
        if ((k & hi_mask) == (prefix & hi_mask)) atomicAdd(&hist[(k >> shift) & 255u], 1);
      }
      __syncthreads();
      if (tid == 0) {
        uint32_t acc = 0;
        int b = 255;
        for (; b > 0; --b) {  // walk bins from the largest digit down
          if (acc + (uint32_t)hist[b] >= need) break;
          acc += (uint32_t)hist[b];
        }
        s_prefix = prefix | ((uint32_t)b << shift);
        s_need = need - acc;
      }
      __syncthreads();
      prefix = s_prefix;
      need = s_need;
      __syncthreads();
    }
  }
  // prefix = threshold key; need = how many rows equal to it are taken.
  const long long per = (N + blockDim.x - 1) / blockDim.x;
  const long long i0 = tid * per, i1 = (i0 + per < N) ? i0 + per : N;
  int n_gt = 0, n_eq = 0;
  if (n > 0)
    for (long long i = i0; i < i1; ++i) {
      if (mask != nullptr && mask[i] == 0) continue;
      const uint32_t k = float_key(score[i]);
      n_gt += k > prefix;
      n_eq += k == prefix;
    }
  int tot;
  const int eq_before = block_exclusive_scan(n_eq, sh, &tot);
  int take_eq = 0;
  if (eq_before < (int)need) take_eq = min(n_eq, (int)need - eq_before);
  const int out_before = block_exclusive_scan(n_gt + take_eq, sh, &tot);
  if (n > 0) {
    int pos = out_before, eq_seen = 0;
    for (long long i = i0; i < i1; ++i) {
      if (mask != nullptr && mask[i] == 0) continue;
      const uint32_t k = float_key(score[i]);
      bool take = k > prefix;
      if (k == prefix) take = eq_seen++ < take_eq;
      if (take && pos < n_select) rows_out[pos++] = (int32_t)i;
    }
  }
  for (long long j = n + tid; j < n_select; j += blockDim.x) rows_out[j] = -1;
  if (tid == 0) *count_out = (int32_t)n;
}

// Teacher side of one chunk, one warp per row: the teacher probabilities of
// the K cache entries (softmax of topk_logit / T, or given weights
// normalised), the (id, p) pairs sorted by id, sum p~ log p~ over the distinct
// ids (entries with the same id add into one class), and for every vocab tile
// of 256 columns the position of its first id in the sorted list (tstart,
// NT + 1 entries per row), so that a GEMM epilogue finds the cached ids of its
// tile with one load.  Ids outside [0, V) are recorded as an error and replaced
// by INT_MAX, which no vocab column matches.  When dH_row0 is given, the warp
// also zeroes its row of dH (H floats), which the chunk's dH GEMM reduce-adds
// into.
// Everything lives in registers (entry k of the row in slot k / 32 of lane
// k % 32) and warp shuffles; the kernel uses no shared memory, so its blocks fit
// beside a running GEMM's CTAs.  One pass over the K entries gives each entry
// its rank in (id, position) order, the summed probability of its id, whether
// it is the first entry of its id, and the largest id ranked before it (for
// the tile starts).
__global__ void __launch_bounds__(ROW_WARPS * 32)
    k_prep_teacher(const int32_t* __restrict__ ids, const float* __restrict__ lg,
                   const uint8_t* __restrict__ mask, RowCount rc, int K, int V, int NT,
                   float invT, bool probs, int* __restrict__ sid, float* __restrict__ sp,
                   float* __restrict__ zs, uint16_t* __restrict__ tstart,
                   float* __restrict__ plogp, DeviceCtl* ctl, float* __restrict__ dH_row0,
                   int H) {
  constexpr int S = K_MAX / 32;  // slots per lane
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * ROW_WARPS + warp;
  if (row >= rc.get()) return;  // warp-uniform
  if (dH_row0 != nullptr) {  // the dH GEMM of this chunk reduce-adds into zeroed rows
    float4* z = reinterpret_cast<float4*>(dH_row0 + (size_t)row * H);
    for (int j = lane; j < H / 4; j += 32) z[j] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const bool keep = mask == nullptr || mask[row] != 0;
  const int nslots = (K + 31) / 32;  // warp-uniform
  float t[S];
  int id[S];
  float m = -INFINITY;
  bool bad_val = false, bad_id = false;
#pragma unroll
  for (int i = 0; i < S; ++i) {
    const int k = lane + 32 * i;
    t[i] = probs ? 0.f : -INFINITY;
    id[i] = INT_MAX;
    if (k < K) {
      const float x = lg[(size_t)row * K + k];
      int d = ids[(size_t)row * K + k];
      if (probs) {
        if (!(x >= 0.f) || x == INFINITY) bad_val = true;  // negative, NaN or +inf weight
        t[i] = (x >= 0.f && x < INFINITY) ? x : 0.f;
      } else {
        if (isnan(x) || x == INFINITY) bad_val = true;
        t[i] = x * invT;
      }
      if (d < 0 || d >= V) { bad_id = true; d = INT_MAX; }
      id[i] = d;
      m = fmaxf(m, t[i]);
    }
  }
  m = warp_max(m);
  bad_val = __any_sync(0xffffffffu, bad_val);
  bad_id = __any_sync(0xffffffffu, bad_id);
  float p[S];
  if (probs) {
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < S; ++i) s += t[i];
    s = warp_sum(s);
    if (!(s > 0.f)) bad_val = true;
    const float inv = s > 0.f ? 1.f / s : 0.f;
#pragma unroll
    for (int i = 0; i < S; ++i) p[i] = t[i] * inv;
  } else {
    if (!(m > -INFINITY)) bad_val = true;
    const float ms = (m > -INFINITY && m < INFINITY) ? m : 0.f;
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < S; ++i)
      if (lane + 32 * i < K) s += expf(t[i] - ms);
    s = warp_sum(s);
    const float lse = s > 0.f ? ms + logf(s) : INFINITY;
#pragma unroll
    for (int i = 0; i < S; ++i) p[i] = (lane + 32 * i < K) ? expf(t[i] - lse) : 0.f;
  }
  if (keep && lane == 0) {
    if (bad_id) atomicOr(&ctl->err, kErrBadIndex);
    if (bad_val) atomicOr(&ctl->err, kErrBadTeacher);
  }
  // One pass over the entries j (broadcast slot by slot): for each own entry i,
  // rank = #{j : (id_j, j) < (id_i, i)}, P = sum of p_j with id_j == id_i,
  // first = no j < i has id_j == id_i, prev = the largest id_j ranked before i.
  int rk[S], prev[S];
  float P[S];
  bool first[S];
#pragma unroll
  for (int i = 0; i < S; ++i) { rk[i] = 0; prev[i] = -1; P[i] = 0.f; first[i] = true; }
#pragma unroll
  for (int js = 0; js < S; ++js) {
    if (js >= nslots) break;
    for (int l0 = 0; l0 < 32; l0 += 4) {
      if (js * 32 + l0 >= K) break;  // warp-uniform
      int idj[4];
      float pj[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {  // four independent broadcasts in flight
        idj[u] = __shfl_sync(0xffffffffu, id[js], l0 + u);
        pj[u] = __shfl_sync(0xffffffffu, p[js], l0 + u);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = js * 32 + l0 + u;
        if (j >= K) break;  // warp-uniform
#pragma unroll
        for (int i = 0; i < S; ++i) {
          if (i >= nslots) break;  // warp-uniform: only the slots that hold entries
          const int k = lane + 32 * i;
          const bool before = idj[u] < id[i] || (idj[u] == id[i] && j < k);
          rk[i] += before ? 1 : 0;
          prev[i] = before ? max(prev[i], idj[u]) : prev[i];
          const bool same = idj[u] == id[i];
          P[i] += same ? pj[u] : 0.f;
          first[i] = first[i] && !(same && j < k);
        }
      }
    }
  }
  float pl = 0.f;
  uint16_t* ts = tstart + (size_t)row * (NT + 1);
#pragma unroll
  for (int i = 0; i < S; ++i) {
    const int k = lane + 32 * i;
    if (k >= K) continue;
    sid[(size_t)row * K + rk[i]] = id[i];
    sp[(size_t)row * K + rk[i]] = p[i];
    zs[(size_t)row * K + rk[i]] = 0.f;
    if (first[i] && P[i] > 0.f) pl += P[i] * logf(P[i]);
    // tiles vt with prev < vt * 256 <= id start at this entry; the last entry
    // also starts every tile after its own (at K)
    const long long lo = rk[i] == 0 ? 0 : (long long)prev[i] / BN + 1;
    const long long hi = min((long long)NT, (long long)id[i] / BN);
    for (long long vt = lo; vt <= hi; ++vt) ts[vt] = (uint16_t)rk[i];
    if (rk[i] == K - 1)
      for (long long vt = (long long)id[i] / BN + 1; vt <= NT; ++vt) ts[vt] = (uint16_t)K;
  }
  pl = warp_sum(pl);
  if (lane == 0) plogp[row] = pl;
}

// Merge the per-vocab-tile (max, sum) partials of each row into its
// log-sum-exp (log2 domain, kept for the backward epilogue) and form the row
// loss  l_r = sum_k p_k log p_k - sum_k p_k (z_k / T - LSE_r),  0 for masked rows.
// The row loss goes to row_loss[row], or -- for gathered rows -- to
// row_loss[out_rows[row]] (entries outside [0, N) are skipped).
__global__ void __launch_bounds__(ROW_WARPS * 32)
    k_merge_loss(const float2* __restrict__ partials, int NT, RowCount rc, int K, float invT,
                 const float* __restrict__ zs, const float* __restrict__ sp,
                 const float* __restrict__ plogp, const uint8_t* __restrict__ mask,
                 float* __restrict__ lse2_out, float* __restrict__ row_loss,
                 const int32_t* __restrict__ out_rows, long long N) {
  pdl_trigger();  // the recompute GEMM after it may start its main loop
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * ROW_WARPS + warp;
  if (row >= rc.get()) return;
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
    const float l = keep ? plogp[row] - acc : 0.f;
    if (out_rows == nullptr) {
      row_loss[row] = l;
    } else {
      const int r = out_rows[row];
      if (r >= 0 && r < N) row_loss[r] = l;
    }
  }
}

// Student entropy per row from the per-tile (max, sum, weighted sum) partials:
// with a = z log2(e) / T, S = sum 2^(a - M), U = sum 2^(a - M) a and
// LSE2 = M + log2 S, H(q) = -sum q ln q = ln2 * (LSE2 - U / S) nats.
// Masked rows get 0.
__global__ void __launch_bounds__(ROW_WARPS * 32)
    k_merge_entropy(const float2* __restrict__ partials, const float* __restrict__ upart, int NT,
                    RowCount rc, const uint8_t* __restrict__ mask, float* __restrict__ entropy) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * ROW_WARPS + warp;
  if (row >= rc.get()) return;
  const float2* pr = partials + (size_t)row * NT;
  const float* pu = upart + (size_t)row * NT;
  float M = -INFINITY;
  for (int t = lane; t < NT; t += 32) M = fmaxf(M, pr[t].x);
  M = warp_max(M);
  float S = 0.f, U = 0.f;
  for (int t = lane; t < NT; t += 32) {
    const float2 q = pr[t];
    if (q.x > -INFINITY) {
      const float f = exp2f(q.x - M);
      S += q.y * f;
      U += pu[t] * f;
    }
  }
  S = warp_sum(S);
  U = warp_sum(U);
  if (lane == 0) {
    const bool keep = mask == nullptr || mask[row] != 0;
    entropy[row] = keep ? 0.69314718055994530942f * (M + log2f(S) - U / S) : 0.f;
  }
}

// loss = sum(row_loss) / N_valid, fp64 accumulation in a fixed order.
__global__ void __launch_bounds__(1024) k_finalize(const float* __restrict__ row_loss, long long N,
                                                   const DeviceCtl* ctl, float* loss) {
  pdl_wait();
  pdl_trigger();
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
