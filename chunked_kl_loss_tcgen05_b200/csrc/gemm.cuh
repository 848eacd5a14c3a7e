// Persistent, warp-specialised tcgen05 GEMM core shared by the four GEMMs of
// the fused chunked KL loss, run on CTA pairs (clusters of 2).
//
// One work unit is a 256 x 256 output tile computed by a CTA pair with
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16 per instruction):
//   * CTA r (r = 0, 1) stages rows [128 r, +128) of A and columns
//     [128 r, +128) of B in its own shared memory (128-byte swizzle); no
//     multicast copies are used;
//   * the even CTA's single MMA thread issues the MMAs for the pair; each CTA's
//     TMEM receives the fp32 accumulator of its own 128 rows x 256 columns;
//   * each CTA's epilogue reads its own TMEM.
//
// Warp roles in every CTA (192 threads):
//   warp 0      TMA producer (one thread): waits for a free stage, loads this
//               CTA's A and B halves; the completion of both CTAs' copies is
//               counted on the even CTA's "full" barrier.
//   warp 1      allocates 512 TMEM columns (two accumulators) for the pair; in
//               the even CTA one thread issues the MMAs, frees stages in both
//               CTAs and announces finished accumulators to both CTAs with
//               multicast tcgen05.commit.
//   warps 2-5   epilogue: tcgen05.ld (thread = row), kernel-specific epilogue,
//               then release the accumulator on the even CTA's barrier.
// Double-buffered accumulators overlap the epilogue of one tile with the main
// loop of the next.  Every wait is bounded (see ptx.cuh).
//
// Operand majors (bf16, row-major global tensors), per CTA and stage:
//   A K-major  : A[m, k] contiguous in k  -> TMA box {64 k, 128 m}
//   A MN-major : A[m, k] contiguous in m  -> one 3-D box {64 m, 64 k, 2 chunks}
//                (or two 2-D boxes {64 m, 64 k} when m's extent is not a
//                multiple of 64)
//   B K-major  : B[n, k] contiguous in k  -> TMA box {64 k, 128 n}
//   B MN-major : B[n, k] contiguous in n  -> as A MN-major
// A last column tile of at most 128 columns may run as N = 128 MMAs (each CTA
// stages 64 columns of B); see SchedArgs::narrow_tail.
#pragma once

#include <climits>

#include "ptx.cuh"

namespace fckl {

constexpr int PM = 256;  // rows of a pair tile
constexpr int CM = 128;  // rows per CTA
constexpr int BN = 256;  // columns of a tile
constexpr int BK = 64;   // k-block
constexpr uint32_t A_HALF_BYTES = CM * BK * 2;        // 16 KB
constexpr uint32_t B_HALF_BYTES = (BN / 2) * BK * 2;  // 16 KB
constexpr uint32_t PSTAGE_BYTES = A_HALF_BYTES + B_HALF_BYTES;
constexpr uint32_t TMEM_COLS = 512;
constexpr int GEMM_THREADS = 192;
constexpr size_t SMEM_LIMIT = 232448;  // opt-in dynamic shared memory per CTA on sm_100

// Dynamic shared memory: 1 KB alignment slack, the operand stages, the
// epilogue's staging area (Epi::kSmemBytes, split over the 4 epilogue warps)
// and 256 bytes of barriers.  As many stages as fit.
template <class Epi>
__host__ __device__ constexpr int pair_stages() {
  return (int)((SMEM_LIMIT - 1024 - 256 - Epi::kSmemBytes) / PSTAGE_BYTES);
}
template <class Epi>
__host__ __device__ constexpr size_t pair_smem_bytes() {
  return 1024 + (size_t)pair_stages<Epi>() * PSTAGE_BYTES + Epi::kSmemBytes + 256;
}

// Wait-site codes recorded on timeout (diagnostics only).
enum : uint32_t {
  SITE_PROD_EMPTY = 1, SITE_MMA_TEMPTY = 2, SITE_MMA_FULL = 3, SITE_EPI_TFULL = 4,
  SITE_DRAIN_MMA = 5, SITE_DRAIN_TMA = 6
};

// Rows a launch covers: a host value, or -- when the rows are the compacted
// valid rows of a masked call, whose number only the device knows --
// clamp(ctl->n_rows - row0, 0, cap), read when the kernel starts (the count is
// written by an earlier kernel on the same stream).
struct RowCount {
  int fixed;  // >= 0: this many rows; < 0: read from ctl
  const DeviceCtl* ctl;
  int row0, cap;
  __device__ __forceinline__ int get() const {
    if (fixed >= 0) return fixed;
    const int r = ctl->n_rows - row0;
    return r < 0 ? 0 : (r > cap ? cap : r);
  }
};

struct Work {
  int mt, nt;    // pair tile: rows [mt*256, +256), columns [nt*256, +256)
  int kb0, kb1;  // k-blocks [kb0, kb1) of 64
  int rev;       // 1: walk the k-blocks from kb1 - 1 down to kb0
  int m0, n0;    // this CTA's first row (mt*256 + 128*rank) and the first column
  int rows;      // rows of the launch (row-tiled kernels: rows >= rows are padding)
};

enum SchedKind : int {
  SCHED_VOCAB_MAJOR = 0,  // units (vocab tile nt, row tile mt), mt fastest; full K
  SCHED_SPLIT_K = 1,      // units (k segment, output tile), k segment slowest
  SCHED_TILES = 2,        // units (mt, nt), nt fastest; K = the launch's rows
};

struct SchedArgs {
  int kind;
  int NT;      // vocab tiles (SCHED_VOCAB_MAJOR) / column tiles (SCHED_SPLIT_K, SCHED_TILES)
  int KB;      // k-blocks of the reduction (SCHED_VOCAB_MAJOR, SCHED_SPLIT_K)
  int S;       // split-K factor (SCHED_SPLIT_K); 0: chosen on the device from the row count
  int MT;      // row tiles of M (SCHED_TILES: M is the vocabulary)
  RowCount rc; // the launch's rows: M of the first two kinds, K of SCHED_TILES
  // MN-major operands: 1 = the map is 3-D {64, k, MN/64}, so that one box
  // brings both 64-wide column chunks of a CTA's half tile; 0 = two 2-D boxes.
  int a3d, b3d;
  int mt0;     // SCHED_TILES: first row tile of the launch (launches over a slice of M)
  // 1: the last column tile holds at most 128 columns, so it runs as an
  // N = 128 MMA (each CTA of the pair stages 64 columns of B) instead of 256.
  int narrow_tail;
  // Programmatic dependent launch.  0: every thread waits for the preceding
  // kernel before touching global memory, then lets the next kernel launch.
  // 1: the operands were complete before the preceding kernel launched, so the
  // producer and the MMA issuer start at once (overlapping the tail of the
  // kernels before) and only the epilogue waits; the next kernel may launch
  // right away (it waits for this one before touching memory).
  int early;
  // SCHED_SPLIT_K: order of the output tiles inside a k segment.  0: column
  // tile fastest (the pairs running at once cover few row tiles and every
  // column tile: A re-read little, B once per wave); 1: row tile fastest (the
  // reverse); 2: chosen when the kernel starts -- row tile fastest when the
  // launch's rows are at most its columns, so that the smaller operand is the
  // one re-read.
  int tile_order;
  // SCHED_SPLIT_K: 1 = serpentine k order -- units of odd waves walk their
  // k segment backwards, so they start on the k-blocks the wave before them
  // touched last, which are still in L2 (the operand every wave re-reads is
  // then served mostly from L2 instead of DRAM).
  int serpentine;
};

__device__ __forceinline__ bool narrow_unit(const SchedArgs& a, const Work& w) {
  return a.narrow_tail && w.nt == a.NT - 1;
}

// Split-K factor for `tiles` output tiles of KB k-blocks on `slots` CTA pairs:
// minimise waves * (k-blocks per unit + a fixed cost of 6 per unit).  Used on
// the device when the row count (hence the tile count) is only known there;
// the host applies the same model when it knows the rows.
__device__ __forceinline__ int choose_split_dev(int tiles, int KB, int slots) {
  if (tiles <= 0 || KB <= 0) return 1;
  int best = 1;
  long long best_cost = LLONG_MAX;
  const int smax = KB < 128 ? KB : 128;
  for (int S = 1; S <= smax; ++S) {
    const long long waves = ((long long)tiles * S + slots - 1) / slots;
    const long long cost = waves * ((KB + S - 1) / S + 6);
    if (cost < best_cost) { best_cost = cost; best = S; }
  }
  return best;
}

// Cluster c of G takes units c, c+G, c+2G, ...  In every order above, the
// clusters running at the same moment touch a narrow band of the streamed
// operand, so it is read from DRAM about once and reused from L2.
struct PairSched {
  long long u, total;
  SchedArgs a;
  int G, rows, MT, tiles, KB;
  // S_dev: the split factor the CTA chose on the device (used when a.S == 0).
  __device__ void init(const SchedArgs& args, int cluster, int nclusters, int S_dev) {
    a = args; G = nclusters; u = cluster;
    if (a.kind == SCHED_SPLIT_K && a.S == 0) a.S = S_dev;
    rows = a.rc.get();
    const int row_tiles = (rows + PM - 1) / PM;
    if (a.kind == SCHED_VOCAB_MAJOR) {
      MT = row_tiles; KB = a.KB; tiles = MT * a.NT; total = (long long)tiles;
    } else if (a.kind == SCHED_SPLIT_K) {
      MT = row_tiles; KB = a.KB; tiles = MT * a.NT; total = (long long)tiles * a.S;
      if (a.tile_order == 2) a.tile_order = rows <= a.NT * BN ? 1 : 0;
    } else {
      MT = a.MT; KB = (rows + BK - 1) / BK; tiles = MT * a.NT;
      total = rows > 0 ? (long long)tiles : 0;
    }
  }
  __device__ bool next(Work& w) {
    if (u >= total) return false;
    if (a.kind == SCHED_VOCAB_MAJOR) {
      w.nt = (int)(u / MT);
      w.mt = (int)(u - (long long)w.nt * MT);
      w.kb0 = 0; w.kb1 = KB; w.rev = 0;
    } else if (a.kind == SCHED_SPLIT_K) {
      const int ks = (int)(u / tiles);
      const int tile = (int)(u - (long long)ks * tiles);
      if (a.tile_order == 1) {
        w.nt = tile / MT; w.mt = tile - w.nt * MT;
      } else {
        w.mt = tile / a.NT; w.nt = tile - w.mt * a.NT;
      }
      w.kb0 = (int)((long long)ks * KB / a.S);
      w.kb1 = (int)((long long)(ks + 1) * KB / a.S);
      w.rev = a.serpentine ? (int)((u / G) & 1) : 0;  // odd waves walk backwards
    } else {
      const int t = (int)(u / a.NT);
      w.nt = (int)(u - (long long)t * a.NT);
      w.mt = a.mt0 + t;
      w.kb0 = 0; w.kb1 = KB; w.rev = 0;
    }
    w.rows = rows;
    u += G;
    return true;
  }
};

struct CtlArgs {
  DeviceCtl* ctl;
  uint64_t timeout_ns;
  int debug_skip_commit;  // >0: the MMA thread omits its first accumulator-ready commit
};

template <class Epi, bool A_MN, bool B_MN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GEMM_THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmC, const typename Epi::Params ep,
                     const SchedArgs sa, const CtlArgs ca) {
  constexpr int STAGES = pair_stages<Epi>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sA = smem;                                  // [STAGES][16 KB]
  uint8_t* sB = smem + STAGES * A_HALF_BYTES;          // [STAGES][16 KB]
  uint8_t* sEpi = smem + STAGES * PSTAGE_BYTES;        // 1 KB aligned
  uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + Epi::kSmemBytes);
  uint64_t* full = bars;                 // [STAGES]  TMA (both CTAs) -> MMA   (even CTA's used)
  uint64_t* empty = bars + STAGES;       // [STAGES]  MMA -> TMA               (each CTA's own)
  uint64_t* tfull = bars + 2 * STAGES;   // [2]       MMA -> epilogue          (each CTA's own)
  uint64_t* tempty = tfull + 2;          // [2]       epilogues -> MMA         (even CTA's used)
  uint64_t* drain = tempty + 2;          // [1]       MMA drain at exit        (even CTA's used)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  uint32_t* abort_flag = tmem_slot + 1;
  int* split_slot = reinterpret_cast<int*>(abort_flag + 1);

  // A launch over no rows (a chunk past the last compacted row) has no work:
  // both CTAs of every pair see the same count and leave before setting up
  // barriers or TMEM (still waiting for the kernel ahead, so that completion
  // keeps implying the completion of everything before).
  if (sa.rc.get() <= 0) {
    pdl_wait();
    pdl_trigger();
    return;
  }
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster = blockIdx.x >> 1;
  const int nclusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&tfull[a]), 1);
      mbar_init(smem_u32(&tempty[a]), 8);  // 4 epilogue warps in each CTA of the pair
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0u;
    // Split-K factor chosen here when only the device knows the rows; every
    // role (and both CTAs of the pair, from the same inputs) uses this value.
    *split_slot = (sa.kind == SCHED_SPLIT_K && sa.S == 0)
                      ? choose_split_dev(((sa.rc.get() + PM - 1) / PM) * sa.NT, sa.KB, nclusters)
                      : sa.S;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (Epi::kUsesMapC) tma_prefetch_desc(&tmC);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // barriers of both CTAs initialised before any remote use
  tc_fence_after();
  if (!sa.early) pdl_wait();
  pdl_trigger();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtx wc{ca.timeout_ns, ca.ctl, abort_flag};

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      PairSched sch;
      sch.init(sa, cluster, nclusters, *split_slot);
      Work w;
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, last_parity = 0;  // even CTA: which full phases it armed
      bool ok = true;
      while (ok && sch.next(w)) {
        const int a_row = w.mt * PM + (int)rank * CM;
        const int b_col = w.nt * BN + (int)rank * (narrow_unit(sa, w) ? 64 : BN / 2);
        for (int i = 0; i < w.kb1 - w.kb0; ++i) {
          const int kb = w.rev ? w.kb1 - 1 - i : w.kb0 + i;
          if (!wait_phase(smem_u32(&empty[stage]), phase ^ 1u, wc, SITE_PROD_EMPTY)) {
            ok = false;
            break;
          }
          const uint32_t fb_local = smem_u32(&full[stage]);
          if (leader) {
            mbar_arrive_expect_tx(fb_local, 2 * PSTAGE_BYTES);
            armed |= 1u << stage;
            last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          }
          const uint32_t fb = mapa_shared(fb_local, 0);
          const uint32_t a_dst = smem_u32(sA + stage * A_HALF_BYTES);
          const uint32_t b_dst = smem_u32(sB + stage * B_HALF_BYTES);
          const int k0 = kb * BK;
          if (!A_MN) {
            tma_load_2d_pair(a_dst, &tmA, fb, k0, a_row);
          } else if (sa.a3d) {
            tma_load_3d_pair(a_dst, &tmA, fb, 0, k0, a_row >> 6);
          } else {
            tma_load_2d_pair(a_dst, &tmA, fb, a_row, k0);
            tma_load_2d_pair(a_dst + 8192, &tmA, fb, a_row + 64, k0);
          }
          if (!B_MN) {
            tma_load_2d_pair(b_dst, &tmB, fb, k0, b_col);
          } else if (sa.b3d) {
            tma_load_3d_pair(b_dst, &tmB, fb, 0, k0, b_col >> 6);
          } else {
            tma_load_2d_pair(b_dst, &tmB, fb, b_col, k0);
            tma_load_2d_pair(b_dst + 8192, &tmB, fb, b_col + 64, k0);
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (leader) {
        // Every copy counted on an armed phase has landed before the pair can exit.
        for (int s = 0; s < STAGES; ++s)
          if (armed & (1u << s))
            drain_phase(smem_u32(&full[s]), (last_parity >> s) & 1u, wc, SITE_DRAIN_TMA);
      } else if (!ok) {
        __nanosleep(20000);  // aborted: give copies already issued time to land
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (leader && lane == 0) {
      PairSched sch;
      sch.init(sa, cluster, nclusters, *split_slot);
      Work w;
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      constexpr uint32_t idesc_full = idesc_bf16_f32(PM, BN, A_MN, B_MN);
      constexpr uint32_t idesc_narrow = idesc_bf16_f32(PM, 128, A_MN, B_MN);
      bool ok = true;
      int skip = ca.debug_skip_commit;
      while (ok && sch.next(w)) {
        if (!wait_phase(smem_u32(&tempty[acc]), acc_phase ^ 1u, wc, SITE_MMA_TEMPTY)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        const uint32_t idesc = narrow_unit(sa, w) ? idesc_narrow : idesc_full;
        for (int i = 0; i < w.kb1 - w.kb0; ++i) {  // k order is the producer's
          if (!wait_phase(smem_u32(&full[stage]), phase, wc, SITE_MMA_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * A_HALF_BYTES);
          const uint32_t b_base = smem_u32(sB + stage * B_HALF_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = A_MN ? sw128_desc(a_base + k * 2048, 8192, 1024)
                                     : sw128_desc(a_base + k * 32, 16, 1024);
            const uint64_t bd = B_MN ? sw128_desc(b_base + k * 2048, 8192, 1024)
                                     : sw128_desc(b_base + k * 32, 16, 1024);
            umma_bf16_pair(d_tmem, ad, bd, idesc, (i > 0 || k > 0) ? 1u : 0u);
          }
          umma_commit_pair(smem_u32(&empty[stage]), 0x3);  // frees the stage in both CTAs
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if (skip > 0) {
          --skip;  // fault-injection knob: this accumulator is never announced
        } else {
          umma_commit_pair(smem_u32(&tfull[acc]), 0x3);
        }
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      // Every MMA issued by this thread is complete before TMEM is released
      // (a pair with no unit -- a launch over zero device-counted rows -- issued none).
      if ((long long)cluster < sch.total) {
        umma_commit_pair(smem_u32(drain), 0x1);
        drain_phase(smem_u32(drain), 0, wc, SITE_DRAIN_MMA);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes [32*quarter, +32) belong to this warp
    const int r = quarter * 32 + lane;
    PairSched sch;
    sch.init(sa, cluster, nclusters, *split_slot);
    Work w;
    int acc = 0;
    uint32_t acc_phase = 0;
    if (sa.early) pdl_wait();  // the epilogue reads and writes what earlier kernels produce
    typename Epi::State st;
    Epi::init(ep, st, sEpi + quarter * (Epi::kSmemBytes / 4), lane);
    while (sch.next(w)) {
      bool ok = true;
      // A tile's main loop lasts tens of microseconds: the epilogue polls its
      // accumulator-ready barrier every 2 us (measured ~0.5-0.9% faster steps
      // under the power cap than polling back to back).
      if (lane == 0) ok = wait_phase(smem_u32(&tfull[acc]), acc_phase, wc, SITE_EPI_TFULL, 2000);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      tc_fence_after();
      w.m0 = w.mt * PM + (int)rank * CM;
      w.n0 = w.nt * BN;
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
      Epi::tile(ep, st, w, taddr, r, &tmC, quarter, lane);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    Epi::finish(ep, st, lane);
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // neither CTA releases TMEM or exits while the pair still uses it
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, TMEM_COLS);
}

}  // namespace fckl
