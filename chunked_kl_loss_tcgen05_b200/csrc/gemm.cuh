// Persistent, warp-specialised tcgen05 GEMM core shared by the four GEMMs of
// the fused chunked KL loss.
//
//   warp 0      TMA producer: one elected thread streams 64-wide k-blocks of A
//               and B into a ring of shared-memory stages (128B swizzle).
//   warp 1      allocates 512 TMEM columns (two 128x256 fp32 accumulators) and
//               one elected thread issues tcgen05.mma (M=128, N=256, K=16).
//   warps 2-5   epilogue: tcgen05.ld the finished accumulator (thread = row),
//               run the kernel-specific epilogue, release the accumulator.
//
// Double-buffered accumulators let the epilogue of tile i overlap the
// main loop of tile i+1.  Every wait is bounded (see ptx.cuh).
//
// Operand majors (bf16, row-major global tensors):
//   A K-major  : A[m, k] contiguous in k  -> TMA box {64 k, 128 m}
//   A MN-major : A[m, k] contiguous in m  -> two TMA boxes {64 m, 64 k}
//   B K-major  : B[n, k] contiguous in k  -> TMA box {64 k, 256 n}
//   B MN-major : B[n, k] contiguous in n  -> four TMA boxes {64 n, 64 k}
#pragma once

#include "ptx.cuh"

namespace fckl {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr uint32_t A_STAGE_BYTES = BM * BK * 2;  // 16 KB
constexpr uint32_t B_STAGE_BYTES = BN * BK * 2;  // 32 KB
constexpr uint32_t STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
constexpr uint32_t TMEM_COLS = 512;
constexpr int GEMM_THREADS = 192;
// Dynamic shared memory: 1 KB alignment slack, the operand stages, the
// epilogue's staging area (Epi::kSmemBytes, split evenly over the 4 epilogue
// warps) and 256 bytes of barriers.
template <class Epi>
constexpr size_t gemm_smem_bytes() {
  return 1024 + (size_t)STAGES * STAGE_BYTES + Epi::kSmemBytes + 256;
}

// Wait-site codes recorded on timeout (diagnostics only).
enum : uint32_t {
  SITE_PROD_EMPTY = 1, SITE_MMA_TEMPTY = 2, SITE_MMA_FULL = 3, SITE_EPI_TFULL = 4,
  SITE_DRAIN_MMA = 5, SITE_DRAIN_TMA = 6
};

struct Work {
  int mb, nb;      // tile coordinates: rows [mb*128, +128), cols [nb*256, +256)
  int kb0, kb1;    // k-blocks [kb0, kb1) of 64
  int split;       // partial-result slot (vocab-split kernels)
  bool seg_begin;  // first tile of a run of consecutive vocab tiles of one row block
  bool seg_end;    // last tile of that run
};

// Scheduling arguments (one struct for every scheduler).
struct SchedArgs {
  long long total;  // linear schedule: RB * NT tiles; unit schedules: number of units
  int NT;           // tiles along n per row block (linear) / n tiles (unit schedules)
  int KB;           // k-blocks of the full reduction
  int S;            // split-K factor (split-K schedule)
  int tiles;        // output tiles (split-K schedule)
};

// Linear schedule over (row block, vocab tile), row-block-major; CTA i owns the
// contiguous range [i*T/G, (i+1)*T/G).  Tiles of one row block that fall in one
// CTA form a segment, whose per-row partial statistics land in slot `split`.
__host__ __device__ inline long long lin_begin(long long i, long long total, long long G) {
  return i * total / G;
}
// The CTA whose range contains tile x.
__host__ __device__ inline long long lin_owner(long long x, long long total, long long G) {
  return ((x + 1) * G + total - 1) / total - 1;
}

struct SchedLinear {
  long long t, t_beg, t_end, total;
  int NT, KB, G, cta;
  __device__ void init(const SchedArgs& a, int cta_, int G_) {
    total = a.total; NT = a.NT; KB = a.KB; G = G_; cta = cta_;
    t_beg = lin_begin(cta, total, G);
    t_end = lin_begin(cta + 1, total, G);
    t = t_beg;
  }
  __device__ bool next(Work& w) {
    if (t >= t_end) return false;
    const int rb = (int)(t / NT);
    const int vt = (int)(t - (long long)rb * NT);
    w.mb = rb; w.nb = vt; w.kb0 = 0; w.kb1 = KB;
    w.seg_begin = (t == t_beg) || (vt == 0);
    w.seg_end = (t + 1 == t_end) || (vt == NT - 1);
    w.split = cta - (int)lin_owner((long long)rb * NT, total, G);
    ++t;
    return true;
  }
};

// Split-K over the reduction dimension: units ordered k-segment-major so that
// all CTAs read the same k-slab of both operands at about the same time (the
// slab stays in L2).  CTA i takes units i, i+G, i+2G, ...
struct SchedSplitK {
  long long u, total;
  int G, tiles, NT, KB, S;
  __device__ void init(const SchedArgs& a, int cta, int G_) {
    total = a.total; tiles = a.tiles; NT = a.NT; KB = a.KB; S = a.S; G = G_; u = cta;
  }
  __device__ bool next(Work& w) {
    if (u >= total) return false;
    const int ks = (int)(u / tiles);
    const int tile = (int)(u - (long long)ks * tiles);
    w.mb = tile / NT; w.nb = tile - w.mb * NT;
    w.kb0 = (int)((long long)ks * KB / S);
    w.kb1 = (int)((long long)(ks + 1) * KB / S);
    w.split = ks; w.seg_begin = true; w.seg_end = true;
    u += G;
    return true;
  }
};

// Whole-K output tiles, CTA i takes tiles i, i+G, ...; consecutive tiles share
// the same m block (same A panel).
struct SchedTiles {
  long long u, total;
  int G, NT, KB;
  __device__ void init(const SchedArgs& a, int cta, int G_) {
    total = a.total; NT = a.NT; KB = a.KB; G = G_; u = cta;
  }
  __device__ bool next(Work& w) {
    if (u >= total) return false;
    w.mb = (int)(u / NT); w.nb = (int)(u - (long long)w.mb * NT);
    w.kb0 = 0; w.kb1 = KB; w.split = 0; w.seg_begin = true; w.seg_end = true;
    u += G;
    return true;
  }
};

struct CtlArgs {
  DeviceCtl* ctl;
  uint64_t timeout_ns;
  int debug_skip_commit;  // >0: the MMA thread omits its first accumulator-ready commit
};

template <class Sched, class Epi, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmC, const typename Epi::Params ep,
                const SchedArgs sa, const CtlArgs ca) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_STAGE_BYTES;
  uint8_t* sEpi = smem + STAGES * STAGE_BYTES;  // 1 KB aligned
  uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + Epi::kSmemBytes);
  uint64_t* full = bars;                // [STAGES]  TMA -> MMA
  uint64_t* empty = bars + STAGES;      // [STAGES]  MMA -> TMA
  uint64_t* tfull = bars + 2 * STAGES;  // [2]       MMA -> epilogue
  uint64_t* tempty = tfull + 2;         // [2]       epilogue -> MMA
  uint64_t* drain = tempty + 2;         // [1]       MMA drain at exit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&tfull[a]), 1);
      mbar_init(smem_u32(&tempty[a]), 4);
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0u;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (Epi::kUsesMapC) tma_prefetch_desc(&tmC);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtx wc{ca.timeout_ns, ca.ctl, abort_flag};

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      Sched sch;
      sch.init(sa, blockIdx.x, gridDim.x);
      Work w;
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0;  // bit s: stage s has been armed at least once
      uint32_t last_parity = 0;  // bit s: parity of the last armed phase of stage s
      bool ok = true;
      while (ok && sch.next(w)) {
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!wait_phase(smem_u32(&empty[stage]), phase ^ 1u, wc, SITE_PROD_EMPTY)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&full[stage]);
          mbar_arrive_expect_tx(fb, STAGE_BYTES);
          armed |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          const uint32_t a_dst = smem_u32(sA + stage * A_STAGE_BYTES);
          const uint32_t b_dst = smem_u32(sB + stage * B_STAGE_BYTES);
          const int k0 = kb * BK;
          if (!A_MN) {
            tma_load_2d(a_dst, &tmA, fb, k0, w.mb * BM);
          } else {
            tma_load_2d(a_dst, &tmA, fb, w.mb * BM, k0);
            tma_load_2d(a_dst + 8192, &tmA, fb, w.mb * BM + 64, k0);
          }
          if (!B_MN) {
            tma_load_2d(b_dst, &tmB, fb, k0, w.nb * BN);
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) tma_load_2d(b_dst + j * 8192, &tmB, fb, w.nb * BN + 64 * j, k0);
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // Let every copy this thread started land before the CTA can exit.
      for (int s = 0; s < STAGES; ++s)
        if (armed & (1u << s)) drain_phase(smem_u32(&full[s]), (last_parity >> s) & 1u, wc, SITE_DRAIN_TMA);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      Sched sch;
      sch.init(sa, blockIdx.x, gridDim.x);
      Work w;
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, A_MN, B_MN);
      bool ok = true;
      int skip = ca.debug_skip_commit;
      while (ok && sch.next(w)) {
        if (!wait_phase(smem_u32(&tempty[acc]), acc_phase ^ 1u, wc, SITE_MMA_TEMPTY)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!wait_phase(smem_u32(&full[stage]), phase, wc, SITE_MMA_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * A_STAGE_BYTES);
          const uint32_t b_base = smem_u32(sB + stage * B_STAGE_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = A_MN ? sw128_desc(a_base + k * 2048, 8192, 1024)
                                     : sw128_desc(a_base + k * 32, 16, 1024);
            const uint64_t bd = B_MN ? sw128_desc(b_base + k * 2048, 8192, 1024)
                                     : sw128_desc(b_base + k * 32, 16, 1024);
            umma_bf16(d_tmem, ad, bd, idesc, (kb > w.kb0 || k > 0) ? 1u : 0u);
          }
          umma_commit(smem_u32(&empty[stage]));  // frees the stage once these MMAs finish
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if (skip > 0) {
          --skip;  // fault-injection knob: this accumulator is never announced
        } else {
          umma_commit(smem_u32(&tfull[acc]));
        }
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      // Wait for every MMA this thread issued before TMEM can be released.
      umma_commit(smem_u32(drain));
      drain_phase(smem_u32(drain), 0, wc, SITE_DRAIN_MMA);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes [32*quarter, +32) belong to this warp
    const int r = quarter * 32 + lane;
    Sched sch;
    sch.init(sa, blockIdx.x, gridDim.x);
    Work w;
    int acc = 0;
    uint32_t acc_phase = 0;
    typename Epi::State st;
    Epi::init(ep, st, sEpi + quarter * (Epi::kSmemBytes / 4), lane);
    while (sch.next(w)) {
      bool ok = true;
      if (lane == 0) ok = wait_phase(smem_u32(&tfull[acc]), acc_phase, wc, SITE_EPI_TFULL);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
      Epi::tile(ep, st, w, taddr, r, &tmC, quarter, lane);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tempty[acc]));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    Epi::finish(ep, st, lane);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
}

}  // namespace fckl
