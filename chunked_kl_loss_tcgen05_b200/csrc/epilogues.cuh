// The four GEMM epilogues of the fused chunked KL loss.  In every epilogue a
// thread owns one accumulator row (TMEM lane) and walks the tile's 256
// columns 32 at a time.
//
//   EpiLse      forward:  z = h W^T tile -> (max, sum 2^(a - max)) of
//               a = z log2(e) / T over the tile's 256 vocab columns, plus a
//               gather of z at the row's cached teacher ids that fall in the
//               tile.  Nothing of the tile is written; one (max, sum) partial
//               per row per vocab tile.
//   EpiDlogits  backward: recomputed z tile -> q - p~ (0 for masked rows,
//               for rows past the launch's rows and for columns >= V),
//               rounded once to bf16, staged in shared memory and
//               TMA-stored to the chunk's dlogits block.
//   EpiDH       dH[rows, :] += alpha * (dlogits W) partial (split-K): fp32
//               tile staged in shared memory, TMA reduce-add into dH (or,
//               for gathered rows, vector reductions into the caller's rows).
//   EpiDW       dW (+)= alpha * (dlogits^T h): TMA store (first chunk) or
//               TMA reduce-add (later chunks), so the fp32 read-modify-write
//               of dW happens in L2, coalesced and off the epilogue threads.
// alpha = 1 / (T * N_valid) is applied here so the bf16 operand stays O(1).
//
// Staging layout (EpiDlogits / EpiDH / EpiDW): each epilogue warp owns two
// 4 KB buffers (double buffering against the TMA engine).  A buffer holds the
// warp's 32 rows x 128 bytes in the TMA 128-byte swizzle: the 16-byte chunk j
// of row r sits at r * 128 + ((j ^ (r & 7)) * 16), which also makes the
// per-thread row writes bank-conflict free.
#pragma once

#include <cuda_bf16.h>
#include <climits>

#include "gemm.cuh"

namespace fckl {

// Warp-convergent TMEM load (tcgen05.ld must be executed by the whole warp).
__device__ __forceinline__ void tmem_ld32_conv(uint32_t taddr, float (&v)[32]) {
  __syncwarp();
  tmem_ld32(taddr, v);
}

// kGather: gather z at the cached teacher ids (loss path).
// kEntropy: also accumulate sum 2^(a - max) * a per tile, so that the merge can
// form the student entropy H(q) = ln2 * (LSE2 - U / S) (student-entropy pass).
template <bool kGather, bool kEntropy>
struct EpiLseT {
  static constexpr uint32_t kSmemBytes = 0;
  static constexpr bool kUsesMapC = false;
  struct Params {
    int V, K, NT;
    float scale2;             // log2(e) / T
    const int* sid;           // [rows_c, K] ids sorted ascending (invalid ids -> INT_MAX)
    const uint16_t* tstart;   // [rows_c, NT + 1] first sorted position of each vocab tile
    float* zs;                // [rows_c, K] gathered z, same order as sid
    float2* partials;         // [rows_c, NT] (max, sum) in the log2 domain
    float* upart;             // [rows_c, NT] sum 2^(a - max) * a (kEntropy only)
  };
  struct State {};
  static __device__ void init(const Params&, State&, uint8_t*, int) {}
  static __device__ void tile(const Params& p, State&, const Work& w, uint32_t taddr, int r,
                              const CUtensorMap*, int, int) {
    const int row = w.m0 + r;
    const bool rv = row < w.rows;
    const int* rid = p.sid + (size_t)(rv ? row : 0) * p.K;
    int cur = 0, nid = INT_MAX;
    if (kGather && rv) {
      cur = __ldg(p.tstart + (size_t)row * (p.NT + 1) + w.nt);
      nid = cur < p.K ? __ldg(rid + cur) : INT_MAX;
    }
    float m = -INFINITY, s = 0.f, u = 0.f;
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      float v[32];
      tmem_ld32_conv(taddr + (uint32_t)(c * 32), v);
      if (!rv) continue;
      const int base = w.n0 + c * 32;
      if (kGather) {
        while (nid < base + 32) {  // gather z at cached ids in this 32-column slice
          const int j = nid - base;
          float z = 0.f;
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) z = (jj == j) ? v[jj] : z;
          p.zs[(size_t)row * p.K + cur] = z;
          ++cur;
          nid = cur < p.K ? __ldg(rid + cur) : INT_MAX;
        }
      }
      // Max over the raw logits first (scale2 > 0 keeps the order), then one
      // FMA per element forms a - max inside the exp2.
      const bool full = base + 32 <= p.V;
      if (!full) {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = (base + j < p.V) ? v[j] : -INFINITY;
      }
      float cz = v[0];
#pragma unroll
      for (int j = 1; j < 32; ++j) cz = fmaxf(cz, v[j]);
      if (cz == -INFINITY) continue;
      const float nm = fmaxf(m, cz * p.scale2);
      const float rescale = ex2_approx(m - nm);
      float acc = 0.f, uacc = 0.f;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float a = v[j] * p.scale2;
        const float e = ex2_approx(fmaf(v[j], p.scale2, -nm));
        acc += e;
        if (kEntropy) uacc += (full || e > 0.f) ? e * a : 0.f;
      }
      s = s * rescale + acc;
      if (kEntropy) u = u * rescale + uacc;
      m = nm;
    }
    if (rv) {
      p.partials[(size_t)row * p.NT + w.nt] = make_float2(m, s);
      if (kEntropy) p.upart[(size_t)row * p.NT + w.nt] = u;
    }
  }
  static __device__ void finish(const Params&, State&, int) {}
};
using EpiLse = EpiLseT<true, false>;
using EpiEntropy = EpiLseT<false, true>;

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&b);
}

// Swizzled position of 16-byte chunk j of this lane's row in a staging buffer.
__device__ __forceinline__ uint4* stage_chunk(uint8_t* buf, int lane, int j) {
  return reinterpret_cast<uint4*>(buf + lane * 128 + ((j ^ (lane & 7)) << 4));
}

// Wait until the staging buffer about to be refilled is no longer read by the
// TMA store issued two slices ago (only the issuing lane can wait on it).
__device__ __forceinline__ void stage_acquire(int lane) {
  if (lane == 0) bulk_wait_read<1>();
  __syncwarp();
}
// Publish this warp's staged rows to the TMA engine.
__device__ __forceinline__ void stage_release() {
  fence_async_smem();
  __syncwarp();
}

struct EpiDlogits {
  static constexpr uint32_t kSmemBytes = 4 * 2 * 4096;
  static constexpr bool kUsesMapC = true;  // map C: dlogits [rows, V] bf16, box {64, 32}
  struct Params {
    int V, K, NT;
    float scale2;             // log2(e) / T
    const float* lse2;        // [rows_c] log2-domain log-sum-exp of z / T
    const int* sid;           // [rows_c, K] sorted ids
    const uint16_t* tstart;   // [rows_c, NT + 1] first sorted position of each vocab tile
    const float* sp;          // [rows_c, K] teacher probabilities, same order
    const uint8_t* mask;      // chunk rows, or nullptr
    int store_rows;           // rows of the store map (the chunk's row capacity)
  };
  struct State {
    int cur, nid, n;
    uint8_t* buf;
  };
  static __device__ void init(const Params&, State& st, uint8_t* smem_warp, int) {
    st.cur = 0; st.nid = INT_MAX; st.n = 0; st.buf = smem_warp;
  }
  // q - p~ for one 32-column slice in place (v holds raw z on entry).
  static __device__ __forceinline__ void slice(const Params& p, State& st, float (&v)[32],
                                               int base, bool keep, float lse, const int* rid,
                                               const float* rp) {
    if (!keep) {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = 0.f;
      return;
    }
    if (base + 32 <= p.V) {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = ex2_approx(fmaf(v[j], p.scale2, -lse));
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        v[j] = (base + j < p.V) ? ex2_approx(fmaf(v[j], p.scale2, -lse)) : 0.f;
    }
    while (st.nid < base + 32) {  // subtract the teacher mass at cached ids
      const int j = st.nid - base;
      const float pv = __ldg(rp + st.cur);
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) v[jj] = (jj == j) ? v[jj] - pv : v[jj];
      ++st.cur;
      st.nid = st.cur < p.K ? __ldg(rid + st.cur) : INT_MAX;
    }
  }
  static __device__ void tile(const Params& p, State& st, const Work& w, uint32_t taddr, int r,
                              const CUtensorMap* mapC, int quarter, int lane) {
    const int row = w.m0 + r;
    const bool rv = row < w.rows;
    const bool keep = rv && (p.mask == nullptr || p.mask[row] != 0);
    const int* rid = p.sid + (size_t)(rv ? row : 0) * p.K;
    const float* rp = p.sp + (size_t)(rv ? row : 0) * p.K;
    const float lse = keep ? p.lse2[row] : 0.f;
    const int col0 = w.n0;
    const int y = w.m0 + quarter * 32;
    // Slabs of 32 rows are stored up to the launch's rows rounded up to 64
    // (rows past the last row hold zeros: the dW GEMM reads whole 64-row
    // blocks), never starting outside the store map.
    const int y_end = min((w.rows + 63) & ~63, p.store_rows);
    st.nid = INT_MAX;
    if (keep) {
      st.cur = __ldg(p.tstart + (size_t)row * (p.NT + 1) + w.nt);
      st.nid = st.cur < p.K ? __ldg(rid + st.cur) : INT_MAX;
    }
#pragma unroll 1
    for (int s = 0; s < BN / 64; ++s) {
      const int base = col0 + s * 64;
      float v0[32], v1[32];
      tmem_ld32_conv(taddr + (uint32_t)(s * 64), v0);
      tmem_ld32_conv(taddr + (uint32_t)(s * 64 + 32), v1);
      slice(p, st, v0, base, keep, lse, rid, rp);
      slice(p, st, v1, base + 32, keep, lse, rid, rp);
      uint8_t* buf = st.buf + (st.n & 1) * 4096;
      stage_acquire(lane);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        *stage_chunk(buf, lane, j) = make_uint4(pack_bf16x2(v0[8 * j], v0[8 * j + 1]),
                                                pack_bf16x2(v0[8 * j + 2], v0[8 * j + 3]),
                                                pack_bf16x2(v0[8 * j + 4], v0[8 * j + 5]),
                                                pack_bf16x2(v0[8 * j + 6], v0[8 * j + 7]));
#pragma unroll
      for (int j = 0; j < 4; ++j)
        *stage_chunk(buf, lane, 4 + j) = make_uint4(pack_bf16x2(v1[8 * j], v1[8 * j + 1]),
                                                    pack_bf16x2(v1[8 * j + 2], v1[8 * j + 3]),
                                                    pack_bf16x2(v1[8 * j + 4], v1[8 * j + 5]),
                                                    pack_bf16x2(v1[8 * j + 6], v1[8 * j + 7]));
      stage_release();
      if (lane == 0) {  // one group per slice, empty when the slice lies outside the map
        if (base < p.V && y < y_end) tma_store_2d(mapC, smem_u32(buf), base, y);
        bulk_commit();
      }
      ++st.n;
    }
  }
  static __device__ void finish(const Params&, State&, int lane) {
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }
};

// Shared staging of alpha * accumulator, one 32-column fp32 slice at a time,
// written to global memory by TMA (store or reduce-add).
template <bool kReduce>
__device__ __forceinline__ void stage_fp32_slices(uint8_t* bufs, int& n, uint32_t taddr,
                                                  float alpha, const CUtensorMap* map, int x0,
                                                  int x_end, int y, bool y_ok, int lane) {
#pragma unroll 1
  for (int c = 0; c < BN / 32; ++c) {
    float v[32];
    tmem_ld32_conv(taddr + (uint32_t)(c * 32), v);
    uint8_t* buf = bufs + (n & 1) * 4096;
    stage_acquire(lane);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *stage_chunk(buf, lane, j) =
          make_uint4(__float_as_uint(alpha * v[4 * j]), __float_as_uint(alpha * v[4 * j + 1]),
                     __float_as_uint(alpha * v[4 * j + 2]), __float_as_uint(alpha * v[4 * j + 3]));
    stage_release();
    const int x = x0 + c * 32;
    if (lane == 0) {  // one group per slice, empty when the slice lies outside the map
      if (x < x_end && y_ok) {
        if (kReduce) tma_reduce_add_2d(map, smem_u32(buf), x, y);
        else tma_store_2d(map, smem_u32(buf), x, y);
      }
      bulk_commit();
    }
    ++n;
  }
}

// dH of gathered rows goes straight to the caller's dH rows: the staged slice
// is read back 4 rows x 128 bytes per warp instruction and added with vector
// reductions at dH + out_rows[row] * H (rows outside [0, N) are skipped).
__device__ __forceinline__ void reduce_slice_to_rows(const uint8_t* buf, int lane, int y_local,
                                                     int rows, const int32_t* out_rows,
                                                     long long N, float* out, int H, int x) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int rr = i * 4 + (lane >> 3), ch = lane & 7;
    const int row = y_local + rr;
    if (row >= rows || x + ch * 4 >= H) continue;
    const int r = __ldg(out_rows + row);
    if (r < 0 || r >= N) continue;
    const uint4 q = *reinterpret_cast<const uint4*>(buf + rr * 128 + ((ch ^ (rr & 7)) << 4));
    float* dst = out + (size_t)r * H + x + ch * 4;
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst),
                 "f"(__uint_as_float(q.x)), "f"(__uint_as_float(q.y)), "f"(__uint_as_float(q.z)),
                 "f"(__uint_as_float(q.w))
                 : "memory");
  }
}

struct EpiDH {
  static constexpr uint32_t kSmemBytes = 4 * 2 * 4096;
  static constexpr bool kUsesMapC = true;  // map C: dH chunk rows [rows, H] fp32, box {32, 32}
  struct Params {
    int H;
    float invT;
    const DeviceCtl* ctl;
    // Gathered rows: the caller's row of each chunk row (nullptr: the chunk's
    // rows are contiguous rows of dH and map C covers them), the caller's dH
    // and its row count.
    const int32_t* out_rows;
    float* out;
    long long N;
  };
  struct State {
    float alpha;
    int n;
    uint8_t* buf;
  };
  static __device__ void init(const Params& p, State& st, uint8_t* smem_warp, int) {
    const int nv = p.ctl->n_valid;
    st.alpha = nv > 0 ? p.invT / (float)nv : 0.f;
    st.n = 0;
    st.buf = smem_warp;
  }
  static __device__ void tile(const Params& p, State& st, const Work& w, uint32_t taddr, int,
                              const CUtensorMap* mapC, int quarter, int lane) {
    const int y = w.m0 + quarter * 32;
    if (p.out_rows == nullptr) {
      stage_fp32_slices<true>(st.buf, st.n, taddr, st.alpha, mapC, w.n0, p.H, y, y < w.rows, lane);
      return;
    }
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      float v[32];
      tmem_ld32_conv(taddr + (uint32_t)(c * 32), v);
      if (y >= w.rows) continue;
      uint8_t* buf = st.buf;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        *stage_chunk(buf, lane, j) =
            make_uint4(__float_as_uint(st.alpha * v[4 * j]), __float_as_uint(st.alpha * v[4 * j + 1]),
                       __float_as_uint(st.alpha * v[4 * j + 2]), __float_as_uint(st.alpha * v[4 * j + 3]));
      __syncwarp();
      reduce_slice_to_rows(buf, lane, y, w.rows, p.out_rows, p.N, p.out, p.H, w.n0 + c * 32);
      __syncwarp();
    }
  }
  static __device__ void finish(const Params&, State&, int lane) {
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }
};

struct EpiDW {
  static constexpr uint32_t kSmemBytes = 4 * 2 * 4096;
  static constexpr bool kUsesMapC = true;  // map C: dW [V, H] fp32, box {32, 32}
  struct Params {
    int V, H;
    float invT;
    int accumulate;  // 0: overwrite (first chunk), 1: add
    const DeviceCtl* ctl;
  };
  struct State {
    float alpha;
    int n;
    uint8_t* buf;
  };
  static __device__ void init(const Params& p, State& st, uint8_t* smem_warp, int) {
    const int nv = p.ctl->n_valid;
    st.alpha = nv > 0 ? p.invT / (float)nv : 0.f;
    st.n = 0;
    st.buf = smem_warp;
  }
  static __device__ void tile(const Params& p, State& st, const Work& w, uint32_t taddr, int,
                              const CUtensorMap* mapC, int quarter, int lane) {
    const int y = w.m0 + quarter * 32;
    if (p.accumulate)
      stage_fp32_slices<true>(st.buf, st.n, taddr, st.alpha, mapC, w.n0, p.H, y, y < p.V, lane);
    else
      stage_fp32_slices<false>(st.buf, st.n, taddr, st.alpha, mapC, w.n0, p.H, y, y < p.V, lane);
  }
  static __device__ void finish(const Params&, State&, int lane) {
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }
};

}  // namespace fckl
