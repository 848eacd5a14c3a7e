// The four GEMM epilogues of the fused chunked KL loss.  In every epilogue a
// thread owns one accumulator row (TMEM lane) and walks the tile's 256
// columns 32 at a time.
//
//   EpiLse      forward:  z = h W^T tile -> online (max, sum 2^(a - max)) of
//               a = z log2(e) / T over the row's vocab tiles, plus a gather of
//               z at the row's cached teacher ids.  Nothing of the tile is
//               written; one (max, sum) partial per row per vocab segment.
//   EpiDlogits  backward: recomputed z tile -> q - p~ (0 for masked rows and
//               for columns >= V), rounded once to bf16, stored to the chunk's
//               dlogits block.
//   EpiDH       dH[rows, :] += alpha * (dlogits W) partial (split-K), fp32.
//   EpiDW       dW (+)= alpha * (dlogits^T h), fp32 read-modify-write.
// alpha = 1 / (T * N_valid) is applied here so the bf16 operand stays O(1).
#pragma once

#include <cuda_bf16.h>
#include <climits>

#include "gemm.cuh"

namespace fckl {

__device__ __forceinline__ int lower_bound_ids(const int* a, int n, int key) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(a + mid) < key) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// Warp-convergent TMEM load (tcgen05.ld must be executed by the whole warp).
__device__ __forceinline__ void tmem_ld32_conv(uint32_t taddr, float (&v)[32]) {
  __syncwarp();
  tmem_ld32(taddr, v);
}

struct EpiLse {
  struct Params {
    int rows_c;      // valid rows of this chunk
    int V, K, Smax;
    float scale2;    // log2(e) / T
    const int* sid;  // [rows_c, K] ids sorted ascending (invalid ids -> INT_MAX)
    float* zs;       // [rows_c, K] gathered z, same order as sid
    float2* partials;  // [RB][Smax][128] (max, sum) in the log2 domain
  };
  struct State {
    float m, s;
    int cur, nid;
  };
  static __device__ void init(const Params&, State& st) {
    st.m = -INFINITY; st.s = 0.f; st.cur = 0; st.nid = INT_MAX;
  }
  static __device__ void tile(const Params& p, State& st, const Work& w, uint32_t taddr, int r) {
    const int row = w.mb * BM + r;
    const bool rv = row < p.rows_c;
    const int* rid = p.sid + (size_t)(rv ? row : 0) * p.K;
    const int col0 = w.nb * BN;
    if (w.seg_begin) {
      st.m = -INFINITY;
      st.s = 0.f;
      if (rv) {
        st.cur = lower_bound_ids(rid, p.K, col0);
        st.nid = st.cur < p.K ? __ldg(rid + st.cur) : INT_MAX;
      }
    }
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      float v[32];
      tmem_ld32_conv(taddr + (uint32_t)(c * 32), v);
      if (!rv) continue;
      const int base = col0 + c * 32;
      while (st.nid < base + 32) {  // gather z at cached ids in this 32-column slice
        const int j = st.nid - base;
        float z = 0.f;
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) z = (jj == j) ? v[jj] : z;
        p.zs[(size_t)row * p.K + st.cur] = z;
        ++st.cur;
        st.nid = st.cur < p.K ? __ldg(rid + st.cur) : INT_MAX;
      }
      float cm = -INFINITY;
      if (base + 32 <= p.V) {
#pragma unroll
        for (int j = 0; j < 32; ++j) { v[j] *= p.scale2; cm = fmaxf(cm, v[j]); }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          v[j] = (base + j < p.V) ? v[j] * p.scale2 : -INFINITY;
          cm = fmaxf(cm, v[j]);
        }
      }
      if (cm == -INFINITY) continue;
      const float nm = fmaxf(st.m, cm);
      float acc = 0.f;
#pragma unroll
      for (int j = 0; j < 32; ++j) acc += exp2f(v[j] - nm);
      st.s = st.s * exp2f(st.m - nm) + acc;
      st.m = nm;
    }
    if (w.seg_end && rv)
      p.partials[((size_t)w.mb * p.Smax + w.split) * BM + r] = make_float2(st.m, st.s);
  }
  static __device__ void finish(const Params&, State&) {}
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&b);
}

struct EpiDlogits {
  struct Params {
    int rows_c, V, Vp, K;
    float scale2;          // log2(e) / T
    const float* lse2;     // [rows_c] log2-domain log-sum-exp of z / T
    const int* sid;        // [rows_c, K] sorted ids
    const float* sp;       // [rows_c, K] teacher probabilities, same order
    const uint8_t* mask;   // chunk rows, or nullptr
    __nv_bfloat16* dlog;   // [rows_c, Vp]
  };
  struct State {
    int cur, nid;
  };
  static __device__ void init(const Params&, State& st) { st.cur = 0; st.nid = INT_MAX; }
  static __device__ void tile(const Params& p, State& st, const Work& w, uint32_t taddr, int r) {
    const int row = w.mb * BM + r;
    const bool rv = row < p.rows_c;
    const bool keep = rv && (p.mask == nullptr || p.mask[row] != 0);
    const int* rid = p.sid + (size_t)(rv ? row : 0) * p.K;
    const float* rp = p.sp + (size_t)(rv ? row : 0) * p.K;
    const float lse = keep ? p.lse2[row] : 0.f;
    const int col0 = w.nb * BN;
    if (w.seg_begin && keep) {
      st.cur = lower_bound_ids(rid, p.K, col0);
      st.nid = st.cur < p.K ? __ldg(rid + st.cur) : INT_MAX;
    }
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      float v[32];
      tmem_ld32_conv(taddr + (uint32_t)(c * 32), v);
      const int base = col0 + c * 32;
      if (!rv || base >= p.Vp) continue;
      if (keep) {
        if (base + 32 <= p.V) {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = exp2f(fmaf(v[j], p.scale2, -lse));
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = (base + j < p.V) ? exp2f(fmaf(v[j], p.scale2, -lse)) : 0.f;
        }
        while (st.nid < base + 32) {  // subtract the teacher mass at cached ids
          const int j = st.nid - base;
          const float pv = __ldg(rp + st.cur);
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) v[jj] = (jj == j) ? v[jj] - pv : v[jj];
          ++st.cur;
          st.nid = st.cur < p.K ? __ldg(rid + st.cur) : INT_MAX;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = 0.f;
      }
      uint4* dst = reinterpret_cast<uint4*>(p.dlog + (size_t)row * p.Vp + base);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (base + 8 * i < p.Vp) {
          uint4 o;
          o.x = pack_bf16x2(v[8 * i + 0], v[8 * i + 1]);
          o.y = pack_bf16x2(v[8 * i + 2], v[8 * i + 3]);
          o.z = pack_bf16x2(v[8 * i + 4], v[8 * i + 5]);
          o.w = pack_bf16x2(v[8 * i + 6], v[8 * i + 7]);
          dst[i] = o;
        }
      }
    }
  }
  static __device__ void finish(const Params&, State&) {}
};

struct EpiDH {
  struct Params {
    int rows_c, H;
    float invT;
    const DeviceCtl* ctl;
    float* dH;  // chunk rows: [rows_c, H]
  };
  struct State {
    float alpha;
  };
  static __device__ void init(const Params& p, State& st) {
    const int n = p.ctl->n_valid;
    st.alpha = n > 0 ? p.invT / (float)n : 0.f;
  }
  static __device__ void tile(const Params& p, State& st, const Work& w, uint32_t taddr, int r) {
    const int row = w.mb * BM + r;
    const bool rv = row < p.rows_c;
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      float v[32];
      tmem_ld32_conv(taddr + (uint32_t)(c * 32), v);
      if (!rv) continue;
      const int col = w.nb * BN + c * 32;
      float* dst = p.dH + (size_t)row * p.H + col;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (col + 4 * i < p.H)
          atomicAdd(reinterpret_cast<float4*>(dst + 4 * i),
                    make_float4(st.alpha * v[4 * i], st.alpha * v[4 * i + 1],
                                st.alpha * v[4 * i + 2], st.alpha * v[4 * i + 3]));
      }
    }
  }
  static __device__ void finish(const Params&, State&) {}
};

struct EpiDW {
  struct Params {
    int V, H;
    float invT;
    int accumulate;  // 0: overwrite (first chunk), 1: add
    const DeviceCtl* ctl;
    float* dW;       // [V, H]
  };
  struct State {
    float alpha;
  };
  static __device__ void init(const Params& p, State& st) {
    const int n = p.ctl->n_valid;
    st.alpha = n > 0 ? p.invT / (float)n : 0.f;
  }
  static __device__ void tile(const Params& p, State& st, const Work& w, uint32_t taddr, int r) {
    const int vr = w.mb * BM + r;
    const bool rv = vr < p.V;
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      float v[32];
      tmem_ld32_conv(taddr + (uint32_t)(c * 32), v);
      if (!rv) continue;
      const int col = w.nb * BN + c * 32;
      float4* dst = reinterpret_cast<float4*>(p.dW + (size_t)vr * p.H + col);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (col + 4 * i < p.H) {
          float4 o = p.accumulate ? dst[i] : make_float4(0.f, 0.f, 0.f, 0.f);
          o.x = fmaf(st.alpha, v[4 * i + 0], o.x);
          o.y = fmaf(st.alpha, v[4 * i + 1], o.y);
          o.z = fmaf(st.alpha, v[4 * i + 2], o.z);
          o.w = fmaf(st.alpha, v[4 * i + 3], o.w);
          dst[i] = o;
        }
      }
    }
  }
  static __device__ void finish(const Params&, State&) {}
};

}  // namespace fckl
