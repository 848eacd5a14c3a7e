// Host side of libfckl: argument checks, workspace layout, tensor maps and the
// chunk scheduler that enqueues the kernels of every chunk on the caller's
// stream.  The library allocates no memory.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "fckl.h"
#include "epilogues.cuh"
#include "gemm.cuh"
#include "ptx.cuh"
#include "rows.cuh"

using namespace fckl;

namespace {

constexpr size_t kAlign = 256;
constexpr int kMaxDevices = 64;

// Rows one dW GEMM reduces over at least when the library picks the chunk:
// below ~4096 rows per launch the fp32 read-modify-write of dW (V*H*8 bytes
// per launch) measurably slows the dW GEMM (-10% at 2048, -30% at 1024 rows).
constexpr long long kAutoDwRows = 4096;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline long long cdiv(long long a, long long b) { return (a + b - 1) / b; }

struct Layout {
  long long N, H, V, K, C, Vp, nchunks, NT;
  long long G;  // chunks per dW group: dlogits of G chunks feed one dW GEMM
  size_t off_rowloss, off_sid, off_sp, off_zs, off_tstart, off_plogp, off_lse2, off_part,
      off_upart, off_hstage, off_idstage, off_lgstage, off_mstage, off_list, off_dlog, total;
};

bool valid_problem(const fckl_problem* p) {
  if (p == nullptr) return false;
  if (p->N < 1 || p->H < 1 || p->V < 1 || p->K < 1 || p->chunk < 0) return false;
  if (!(std::isfinite(p->T) && p->T > 0.f)) return false;
  if (p->N > INT32_MAX || p->H > INT32_MAX || p->V > INT32_MAX) return false;
  if (p->teacher != FCKL_TEACHER_LOGITS && p->teacher != FCKL_TEACHER_PROBS) return false;
  if (p->n_valid_total < 0 || p->n_valid_total > INT32_MAX) return false;
  if (p->dw_rows < 0 || p->dw_rows > INT32_MAX) return false;
  return true;
}

bool supported_problem(const fckl_problem* p) {
  return p->K <= FCKL_K_MAX && p->K <= p->V && p->H % 8 == 0;
}

long long resolve_chunk(const fckl_problem* p) {
  const long long Vp = align_up((size_t)p->V, 64);
  long long C = p->chunk;
  if (C == 0) {
    // 1 GiB of bf16 dlogits: at V = 128K a 4096-row chunk, deep enough that
    // one dW read-modify-write (V*H*8 bytes) per chunk stays well under the
    // chunk's dW tensor-core time, with few launches (and tail waves).
    const long long budget = 1024ll << 20;
    C = budget / (Vp * 2) / 128 * 128;
    C = std::max(C, 128ll);
    C = std::min(C, (long long)align_up((size_t)p->N, 64));
  }
  return std::min<long long>(C, p->N);
}

// full = false: the forward-loss-only layout (no dlogits, no entropy or
// row-list buffers), used by the allocation-free entry point.
Layout make_layout(const fckl_problem* p, bool full = true) {
  Layout L{};
  L.N = p->N; L.H = p->H; L.V = p->V; L.K = p->K;
  // dlogits rows are padded to a multiple of 64 columns (zeros in the pad), so
  // the dW GEMM can read them as whole 64-column chunks.
  L.Vp = (long long)align_up((size_t)p->V, 64);
  L.C = resolve_chunk(p);
  L.nchunks = cdiv(L.N, L.C);
  // The dW GEMM reduces over the rows of its dlogits block, and each launch
  // reads and writes dW once (fp32, V*H*8 bytes).  With the caller's chunk
  // every chunk runs its own dW GEMM, so the workspace holds one chunk of
  // dlogits; dw_rows groups chunks so that one dW launch covers at least
  // dw_rows rows, at the cost of keeping the group's dlogits live together.
  // The automatic chunk groups to kAutoDwRows rows unless dw_rows says otherwise.
  const long long dw = p->dw_rows > 0 ? p->dw_rows : (p->chunk == 0 ? kAutoDwRows : 0);
  L.G = std::min<long long>(L.nchunks, std::max<long long>(1, cdiv(dw, L.C)));
  L.NT = cdiv(L.V, BN);
  size_t off = align_up(sizeof(DeviceCtl), kAlign);
  auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, kAlign); return o; };
  const size_t C = (size_t)L.C;
  L.off_rowloss = take((size_t)L.N * 4);
  L.off_sid = take(C * L.K * 4);
  L.off_sp = take(C * L.K * 4);
  L.off_zs = take(C * L.K * 4);
  L.off_tstart = take(C * (L.NT + 1) * 2);
  L.off_plogp = take(C * 4);
  L.off_lse2 = take(C * 4);
  L.off_part = take(C * L.NT * sizeof(float2));
  L.off_upart = take(full ? C * L.NT * 4 : 0);
  // Row-list calls gather their rows into these staging buffers.
  // two buffers of a group's gathered hidden rows (alternating by group)
  L.off_hstage = take(full ? 2 * (size_t)L.G * C * L.H * 2 : 0);
  L.off_idstage = take(full ? C * L.K * 4 : 0);
  L.off_lgstage = take(full ? C * L.K * 4 : 0);
  L.off_mstage = take(full ? C : 0);
  L.off_list = take(full ? (size_t)L.N * 4 : 0);  // valid rows of a masked call, compacted
  L.off_dlog = take(full ? (size_t)L.G * C * L.Vp * 2 : 0);
  L.total = off;
  return L;
}

// ---------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 2-D map (bf16 or fp32): inner (contiguous) extent, outer extent, outer
// stride in bytes, box {box_inner, box_outer}, 128-byte swizzle, zero fill out
// of bounds.
bool make_map(CUtensorMap* m, const void* base, long long inner, long long outer,
              long long stride_bytes, int box_inner, int box_outer, bool fp32 = false) {
  EncodeTiledFn enc = get_encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  cuuint64_t strides[1] = {(cuuint64_t)stride_bytes};
  cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_outer};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
             const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D view of a row-major bf16 [outer, inner] matrix (inner % 64 == 0) for
// MN-major operand loads: dims {64, outer, inner / 64}, strides {row pitch,
// 128 B}; a box {64, box_outer, 2} brings two adjacent 64-wide column chunks,
// stored chunk after chunk in shared memory exactly as two 2-D boxes would be.
bool make_map_mn3(CUtensorMap* m, const void* base, long long inner, long long outer,
                  long long stride_bytes, int box_outer) {
  EncodeTiledFn enc = get_encode_fn();
  if (enc == nullptr || inner % 64 != 0) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)outer, (cuuint64_t)(inner / 64)};
  cuuint64_t strides[2] = {(cuuint64_t)stride_bytes, 128};
  cuuint32_t box[3] = {64, (cuuint32_t)box_outer, 2};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// MN-major operand map: the 3-D form when the column count allows it and the
// driver accepts it (sets *is3d), else the 2-D form with 64-column boxes.
bool make_map_mn(CUtensorMap* m, const void* base, long long inner, long long outer,
                 long long stride_bytes, int* is3d) {
  *is3d = 0;
  if (inner % 64 == 0 && make_map_mn3(m, base, inner, outer, stride_bytes, BK)) {
    *is3d = 1;
    return true;
  }
  return make_map(m, base, inner, outer, stride_bytes, 64, BK);
}

// ---------------------------------------------------------------- device info
struct DeviceInfo {
  bool ready = false;
  bool ok = false;
  int sms = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

template <class Epi, bool A_MN, bool B_MN>
bool set_smem_attr() {
  return cudaFuncSetAttribute(gemm_pair_kernel<Epi, A_MN, B_MN>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)pair_smem_bytes<Epi>()) == cudaSuccess;
}

const DeviceInfo* device_info() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    d.ready = true;
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    d.ok = major == 10 && minor == 0 && d.sms > 0;
    if (d.ok) {
      d.ok = set_smem_attr<EpiLse, false, false>() && set_smem_attr<EpiDlogits, false, false>() &&
             set_smem_attr<EpiDH, false, true>() && set_smem_attr<EpiDW, true, true>() &&
             set_smem_attr<EpiEntropy, false, false>();
    }
  }
  return &d;
}

// ---------------------------------------------------------------- knobs
uint64_t wait_timeout_ns() {
  const char* s = std::getenv("FCKL_WAIT_TIMEOUT_MS");
  long long ms = s ? std::atoll(s) : 2000;
  if (ms < 1) ms = 1;
  if (ms > 60000) ms = 60000;
  return (uint64_t)ms * 1000000ull;
}
int debug_skip_commit() {
  const char* s = std::getenv("FCKL_DEBUG_SKIP_ARRIVE");
  return (s && std::atoi(s) > 0) ? 1 : 0;
}
// Tile order of the dH GEMM's split-K units (SchedArgs::tile_order; default 2,
// chosen on the device; FCKL_DH_ORDER = 0 or 1 fixes it, for measurements).
int dh_tile_order() {
  const char* s = std::getenv("FCKL_DH_ORDER");
  const int v = s ? std::atoi(s) : 2;
  return (v == 0 || v == 1) ? v : 2;
}
// Serpentine k order of the dH GEMM's split-K units (FCKL_DH_SERPENTINE=0
// turns it off, for measurements).
int dh_serpentine() {
  const char* s = std::getenv("FCKL_DH_SERPENTINE");
  return (s && std::atoi(s) == 0) ? 0 : 1;
}
// Programmatic dependent launch for the kernels of a call (FCKL_NO_PDL=1 turns
// it off: every kernel then starts after the previous one has completed).
bool pdl_enabled() {
  const char* s = std::getenv("FCKL_NO_PDL");
  return !(s && std::atoi(s) > 0);
}

// Launches `kernel` on `st`, with programmatic stream serialization when
// `pdl`: the kernel may start once every CTA of the previous kernel has
// called pdl_trigger() (or exited); it calls pdl_wait() before it touches what
// that kernel produces.  Kernels with compile-time cluster dimensions keep them.
template <typename... KArgs, typename... Args>
cudaError_t launch(bool pdl, void (*kernel)(KArgs...), int grid, int block, size_t smem,
                   cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3((unsigned)block, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------- profiling
enum Kind {
  K_COUNT, K_PREP, K_FWD, K_MERGE, K_BWD, K_DH, K_DW, K_FINAL, K_ENT, K_ENT_MERGE, K_GATHER,
  K_SCATTER, K_SELECT, K_ZERO_DW, K_NKINDS
};
const char* const kKindName[K_NKINDS] = {
    "count_valid", "prep_teacher", "fwd_logits_lse", "merge_loss", "bwd_dlogits",
    "dH_gemm",     "dW_gemm",      "finalize",       "entropy_gemm", "merge_entropy",
    "gather_rows", "scatter_rows", "select_rows", "zero_dw"};
struct ProfRec {
  int kind;
  cudaEvent_t a, b;
  double flops, bytes;
};
struct Profiler {
  bool on = false;
  uint32_t mask = 0xFFFFFFFFu;
  std::vector<ProfRec> recs;
  std::vector<cudaEvent_t> pool;
  size_t used = 0;
  cudaEvent_t next() {
    if (used == pool.size()) {
      cudaEvent_t e = nullptr;
      if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
      pool.push_back(e);
    }
    return pool[used++];
  }
};
Profiler g_prof;

struct ProfScope {
  int kind;
  cudaStream_t st;
  double flops, bytes;
  cudaEvent_t a = nullptr;
  ProfScope(int k, cudaStream_t s, double f, double b) : kind(k), st(s), flops(f), bytes(b) {
    if (g_prof.on && ((g_prof.mask >> k) & 1u) && (a = g_prof.next()) != nullptr)
      cudaEventRecord(a, st);
  }
  ~ProfScope() {
    if (!g_prof.on || a == nullptr) return;
    cudaEvent_t b = g_prof.next();
    if (b == nullptr) return;
    cudaEventRecord(b, st);
    g_prof.recs.push_back(ProfRec{kind, a, b, flops, bytes});
  }
};

// Split-K factor for dH: minimise waves * (k-blocks per unit + fixed cost),
// with `slots` CTA pairs working at once.  (Capping the k-segment to keep it
// L2-resident cut DRAM reads but made the kernel slower: more, shorter units.)
int choose_split(long long tiles, long long KB, int slots) {
  int best = 1;
  double best_cost = 1e300;
  const long long smax = std::min<long long>(KB, 512);
  for (long long S = 1; S <= smax; ++S) {
    const long long units = tiles * S;
    const double waves = (double)cdiv(units, slots);
    const double cost = waves * ((double)cdiv(KB, S) + 6.0);
    if (cost < best_cost - 1e-9) { best_cost = cost; best = (int)S; }
  }
  return best;
}

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

enum class Mode { kFwd, kFwdBwd, kEntropy };

// Everything one library call asks for.  rows == nullptr: the rows are
// 0..N-1 (row_mask optional); otherwise the call covers the n_rows listed
// rows (negative entries are skipped) and gathers them chunk by chunk.
struct Request {
  Mode mode = Mode::kFwd;
  const fckl_problem* prob = nullptr;
  const void* hidden = nullptr;
  const void* W = nullptr;
  const int32_t* topk_idx = nullptr;
  const float* topk_logit = nullptr;
  const uint8_t* row_mask = nullptr;
  const int32_t* rows = nullptr;
  long long n_rows = 0;
  float* loss = nullptr;
  float* row_loss = nullptr;
  float* dH = nullptr;
  float* dW = nullptr;
  float* entropy = nullptr;
  void* workspace = nullptr;
  size_t ws_bytes = 0;
  void* stream = nullptr;
  bool full_layout = true;
  // Host-input calls: ready[0] marks the row mask copied to the device,
  // ready[1 + c] the rows chunk c reads; the chunk waits for it on the stream.
  const cudaEvent_t* ready = nullptr;
  // Sliced dW: the last dW launch runs as n_slices launches over consecutive
  // vocabulary ranges; slice_events[i] is recorded after slice i and
  // slice_rows[i..i+1] receives its dW row range.
  int n_slices = 0;
  cudaEvent_t const* slice_events = nullptr;
  int64_t* slice_rows = nullptr;
};

// Per device: the library's second stream, on which the next chunk's gather
// and teacher prep run while the current chunk's dH GEMM runs on the caller's
// stream, and a pool of events for the hand-overs (created on first use, kept
// until the process exits).  Calls that use it are serialised while they
// enqueue.  FCKL_ONE_STREAM=1 keeps everything on the caller's stream.
struct RowStream {
  std::mutex mu;
  cudaStream_t rs = nullptr;
  std::vector<cudaEvent_t> ev;
};
RowStream g_rs[kMaxDevices];

bool two_streams_enabled() {
  const char* s = std::getenv("FCKL_ONE_STREAM");
  return !(s && std::atoi(s) > 0);
}

fckl_status run(const Request& q) {
  const fckl_problem* prob = q.prob;
  const bool bwd = q.mode == Mode::kFwdBwd;
  const bool ent = q.mode == Mode::kEntropy;
  const bool user_list = q.rows != nullptr;
  if (!valid_problem(prob)) return FCKL_ERR_INVALID_ARG;
  if (!q.hidden || !q.W || !aligned(q.hidden, 16) || !aligned(q.W, 16)) return FCKL_ERR_INVALID_ARG;
  if (ent) {
    if (!q.entropy || !aligned(q.entropy, 4)) return FCKL_ERR_INVALID_ARG;
  } else {
    if (!q.topk_idx || !q.topk_logit || !q.loss) return FCKL_ERR_INVALID_ARG;
    if (!aligned(q.topk_idx, 4) || !aligned(q.topk_logit, 4) || !aligned(q.loss, 4) ||
        (q.row_loss && !aligned(q.row_loss, 4)))
      return FCKL_ERR_INVALID_ARG;
  }
  if (bwd && (!q.dH || !q.dW || !aligned(q.dH, 16) || !aligned(q.dW, 16)))
    return FCKL_ERR_INVALID_ARG;
  if (user_list && (q.n_rows < 1 || q.n_rows > INT32_MAX || !aligned(q.rows, 4)))
    return FCKL_ERR_INVALID_ARG;
  if (!supported_problem(prob)) return FCKL_ERR_UNSUPPORTED;
  const Layout L = make_layout(prob, q.full_layout);
  if (q.workspace == nullptr || !aligned(q.workspace, kAlign) || q.ws_bytes < L.total)
    return FCKL_ERR_WORKSPACE;
  const DeviceInfo* dev = device_info();
  if (dev == nullptr || !dev->ok) return FCKL_ERR_UNSUPPORTED;
  if (get_encode_fn() == nullptr) return FCKL_ERR_CUDA;

  // How the rows are fed to the chunk pipeline:
  //   direct  : rows 0..N-1 in place (no mask, the entropy pass, or the
  //             forward-only layout of the allocation-free entry point);
  //   listed  : the caller's row list, gathered chunk by chunk;
  //   compact : a masked call -- the valid rows are compacted on the device and
  //             gathered, so masked rows cost no GEMM work; the row count of
  //             each chunk is read on the device.
  const bool compact = !ent && !user_list && q.row_mask != nullptr && q.full_layout;
  const bool list = user_list || compact;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(q.stream);
  uint8_t* ws = static_cast<uint8_t*>(q.workspace);
  DeviceCtl* ctl = reinterpret_cast<DeviceCtl*>(ws);
  float* rl = q.row_loss ? q.row_loss : reinterpret_cast<float*>(ws + L.off_rowloss);
  int* sid = reinterpret_cast<int*>(ws + L.off_sid);
  float* sp = reinterpret_cast<float*>(ws + L.off_sp);
  float* zs = reinterpret_cast<float*>(ws + L.off_zs);
  uint16_t* tstart = reinterpret_cast<uint16_t*>(ws + L.off_tstart);
  float* plogp = reinterpret_cast<float*>(ws + L.off_plogp);
  float* lse2 = reinterpret_cast<float*>(ws + L.off_lse2);
  float2* part = reinterpret_cast<float2*>(ws + L.off_part);
  float* upart = reinterpret_cast<float*>(ws + L.off_upart);
  __nv_bfloat16* hstage = reinterpret_cast<__nv_bfloat16*>(ws + L.off_hstage);
  int32_t* idstage = reinterpret_cast<int32_t*>(ws + L.off_idstage);
  float* lgstage = reinterpret_cast<float*>(ws + L.off_lgstage);
  uint8_t* mstage = ws + L.off_mstage;
  int32_t* clist = reinterpret_cast<int32_t*>(ws + L.off_list);
  __nv_bfloat16* dlog = reinterpret_cast<__nv_bfloat16*>(ws + L.off_dlog);
  const int32_t* rowlist = user_list ? q.rows : clist;

  const int H = (int)L.H, V = (int)L.V, K = (int)L.K;
  const float invT = 1.0f / prob->T;
  const float scale2 = 1.4426950408889634f / prob->T;
  CtlArgs ca{ctl, wait_timeout_ns(), debug_skip_commit()};
  const bool pdl = pdl_enabled();
  // Launch with programmatic dependent launch; a failed launch ends the call.
#define FCKL_LAUNCH(kernel, grid, block, smem, ...)                                   \
  do {                                                                                 \
    if (launch(pdl, kernel, (int)(grid), (int)(block), (size_t)(smem), st, __VA_ARGS__) != \
        cudaSuccess)                                                                   \
      return FCKL_ERR_CUDA;                                                            \
  } while (0)

  if (cudaMemsetAsync(ctl, 0, sizeof(DeviceCtl), st) != cudaSuccess) return FCKL_ERR_CUDA;
  if (q.ready && cudaStreamWaitEvent(st, q.ready[0], 0) != cudaSuccess) return FCKL_ERR_CUDA;
  if (!ent) {
    ProfScope ps(K_COUNT, st, 0.0,
                 user_list ? q.n_rows * 4.0 : (q.row_mask ? L.N * (compact ? 5.0 : 1.0) : 0.0));
    if (user_list)
      FCKL_LAUNCH(k_count_list, 1, 1024, 0, q.rows, (long long)q.n_rows, (long long)L.N,
                  (int)prob->n_valid_total, ctl);
    else if (compact)
    {
      // two passes over at most kCompactBlocks blocks of R rows (R % 4096 == 0)
      const long long R = std::max<long long>(4096, cdiv(cdiv(L.N, kCompactBlocks), 4096) * 4096);
      const int nb = (int)cdiv(L.N, R);
      FCKL_LAUNCH(k_compact_count, nb, 1024, 0, q.row_mask, (long long)L.N, R, ctl);
      FCKL_LAUNCH(k_compact_write, nb, 1024, 0, q.row_mask, (long long)L.N, R,
                  (int)prob->n_valid_total, clist, ctl);
    }
    else
      FCKL_LAUNCH(k_count_valid, 1, 1024, 0, q.row_mask, (long long)L.N,
                  (int)prob->n_valid_total, ctl);
  }
  // The profiler's flop and byte counts follow the rows a launch really
  // processes; for a compacted call it reads their number back once (profiling
  // only -- the normal path never waits on the device).
  long long prof_rows = -1;
  if (compact && g_prof.on) {
    int32_t n = 0;
    if (cudaMemcpyAsync(&n, &ctl->n_rows, sizeof(n), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
      return FCKL_ERR_CUDA;
    prof_rows = n;
  }
  if (list) {  // rows that are not processed get zero row loss and zero dH
    if (cudaMemsetAsync(rl, 0, (size_t)L.N * 4, st) != cudaSuccess) return FCKL_ERR_CUDA;
    if (bwd && cudaMemsetAsync(q.dH, 0, (size_t)L.N * L.H * 4, st) != cudaSuccess)
      return FCKL_ERR_CUDA;
  }

  CUtensorMap mapW_k, mapW_mn, mapdW;
  if (!make_map(&mapW_k, q.W, L.H, L.V, L.H * 2, BK, BN / 2)) return FCKL_ERR_CUDA;
  int w3d = 0;
  if (bwd && !make_map_mn(&mapW_mn, q.W, L.H, L.V, L.H * 2, &w3d)) return FCKL_ERR_CUDA;
  if (bwd && !make_map(&mapdW, q.dW, L.H, L.V, L.H * 4, 32, 32, true)) return FCKL_ERR_CUDA;

  const int pairs = std::max(1, dev->sms / 2);  // CTA pairs that run at once
  const long long NT = L.NT;
  const long long KBh = cdiv(L.H, BK);
  const long long NTh = cdiv(L.H, BN);
  const long long KBv = cdiv(L.V, BK);
  // dH and dW tile the hidden dimension by 256; a last tile of at most 128
  // columns (e.g. H = 2880) runs as a half-width MMA.
  const int narrow_h = (L.H % BN != 0 && L.H % BN <= 128) ? 1 : 0;
  const long long R = user_list ? q.n_rows : L.N;  // rows (or list entries), upper bound
  const long long nchunks = cdiv(R, L.C);
  const long long G = std::min<long long>(nchunks, L.G);
  auto grid_for = [&](long long units) {
    return (int)(2 * std::max<long long>(1, std::min<long long>(pairs, units)));
  };
  // Rows of the chunk starting at row0 (at most cap): a host number, or read on
  // the device for compacted calls.
  auto rows_of = [&](long long row0, long long cap) {
    return compact ? RowCount{-1, ctl, (int)row0, (int)cap} : RowCount{(int)cap, ctl, 0, 0};
  };
  // One chunk's rows and where they come from: the caller's rows directly,
  // or the staging buffers the listed / compacted rows are gathered into.
  // Staged hidden rows alternate between two buffers (by dW group), so that
  // the next chunk can be gathered while the current group's dW GEMM still
  // reads its rows.
  struct ChunkIO {
    long long row0;
    int cap;              // rows of the chunk (upper bound if compact)
    RowCount rc;
    double nr;            // rows processed, as far as the host knows (profiling figures)
    long long MT;
    int row_blocks;
    const void* h;
    const int32_t* ids;
    const float* lg;
    const uint8_t* mask;
    float* rl;               // row loss of the chunk's first row; with out_rows, of row 0
    float* dH;               // dH of the chunk's first row; nullptr with out_rows
    const int32_t* out_rows; // gathered rows: the caller's row of each chunk row
    __nv_bfloat16* dlog;     // this chunk's rows in the group's dlogits block
  };
  auto hslot = [&](long long c) {
    return hstage + (size_t)(((c / G) & 1) * G + c % G) * L.C * L.H;
  };
  auto chunk_io = [&](long long c) {
    ChunkIO io;
    io.row0 = c * L.C;
    io.cap = (int)std::min(L.C, R - io.row0);
    io.rc = rows_of(io.row0, io.cap);
    io.nr = prof_rows < 0 ? (double)io.cap
                          : (double)std::max(0LL, std::min<long long>(io.cap, prof_rows - io.row0));
    io.MT = cdiv(io.cap, PM);
    io.row_blocks = (int)cdiv(io.cap, ROW_WARPS);
    if (list) {
      // row losses and dH rows go straight to the caller's rows (dH was zeroed
      // at the start of the call)
      io.h = hslot(c); io.ids = idstage; io.lg = lgstage; io.rl = rl; io.dH = nullptr;
      io.out_rows = rowlist + io.row0;
      io.mask = compact ? nullptr : mstage;  // compacted rows are all valid
    } else {
      io.out_rows = nullptr;
      io.h = static_cast<const uint8_t*>(q.hidden) + (size_t)io.row0 * L.H * 2;
      io.ids = q.topk_idx ? q.topk_idx + io.row0 * K : nullptr;
      io.lg = q.topk_logit ? q.topk_logit + io.row0 * K : nullptr;
      io.mask = q.row_mask ? q.row_mask + io.row0 : nullptr;
      io.rl = rl + io.row0;
      io.dH = bwd ? q.dH + io.row0 * L.H : nullptr;
    }
    io.dlog = dlog + (size_t)(c % G) * L.C * L.Vp;
    return io;
  };
  // What chunk c needs before its forward GEMM: its host-input piece, its
  // gathered rows (listed and compacted calls) and the teacher preparation
  // (which, for rows that are not gathered, also zeroes the chunk's dH rows
  // for the dH GEMM's reduce-adds).
  auto stage_in = [&](long long c, const ChunkIO& io, cudaStream_t ss) -> fckl_status {
    cudaStream_t st = ss;  // the launches below go to this stream
    if (q.ready && cudaStreamWaitEvent(st, q.ready[1 + c], 0) != cudaSuccess) return FCKL_ERR_CUDA;
    if (list) {
      // A compacted chunk zeroes the dlogits rows just past its last valid row
      // (the dW GEMM reads whole 64-row blocks, which may reach into the next
      // chunk's slot of the group).  The first chunk of a group leaves this to
      // its recompute GEMM, because the previous group's dW GEMM may still be
      // reading that slot when the gather runs.
      uint4* dlz = (bwd && compact && c % G != 0) ? reinterpret_cast<uint4*>(io.dlog) : nullptr;
      ProfScope ps(K_GATHER, st, 0.0, io.nr * (L.H * 4.0 + K * 16.0 + 5.0));
      FCKL_LAUNCH(k_gather_rows, io.cap, 128, 0, rowlist + io.row0, io.rc, (long long)L.N, H, K,
                  static_cast<const __nv_bfloat16*>(q.hidden), q.topk_idx, q.topk_logit,
                  static_cast<__nv_bfloat16*>(const_cast<void*>(io.h)), idstage, lgstage, mstage,
                  dlz, (long long)(L.Vp / 8));
    }
    if (!ent) {
      ProfScope ps(K_PREP, st, 0.0, io.nr * K * 20.0 + io.nr * (NT + 1) * 2.0);
      FCKL_LAUNCH(k_prep_teacher, io.row_blocks, ROW_WARPS * 32, 0, io.ids, io.lg, io.mask, io.rc,
                  K, V, (int)NT, invT, prob->teacher == FCKL_TEACHER_PROBS, sid, sp, zs, tstart,
                  plogp, ctl, io.dH, H);
    }
    return FCKL_OK;
  };

  // Backward calls of several chunks run the next chunk's gather and teacher
  // prep on the library's second stream, between the recompute GEMM and the
  // dW GEMM of the current chunk: the teacher buffers are free once the
  // recompute GEMM is done, and the gathered rows go to the other buffer.
  std::unique_lock<std::mutex> rs_lock;
  RowStream* rsd = nullptr;
  if (bwd && nchunks > 1 && two_streams_enabled()) {
    int dev_id = 0;
    if (cudaGetDevice(&dev_id) != cudaSuccess || dev_id < 0 || dev_id >= kMaxDevices)
      return FCKL_ERR_CUDA;
    rsd = &g_rs[dev_id];
    rs_lock = std::unique_lock<std::mutex>(rsd->mu);
    if (rsd->rs == nullptr &&
        cudaStreamCreateWithFlags(&rsd->rs, cudaStreamNonBlocking) != cudaSuccess) {
      rsd->rs = nullptr;
      return FCKL_ERR_CUDA;
    }
    while ((long long)rsd->ev.size() < 2 * nchunks) {
      cudaEvent_t e = nullptr;
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return FCKL_ERR_CUDA;
      rsd->ev.push_back(e);
    }
  }

  ChunkIO io = chunk_io(0);
  if (const fckl_status s0 = stage_in(0, io, st); s0 != FCKL_OK) return s0;
  for (long long c = 0; c < nchunks; ++c) {
    const bool more = c + 1 < nchunks;
    CUtensorMap mapH_k;
    if (!make_map(&mapH_k, io.h, L.H, io.cap, L.H * 2, BK, CM)) return FCKL_ERR_CUDA;
    // Forward units are vocab-major so that concurrent pairs share W tiles.
    SchedArgs sa_v{SCHED_VOCAB_MAJOR, (int)NT, (int)KBh, 1, 0, io.rc, 0, 0};
    const int Gv = grid_for(io.MT * NT);
    const double gemm_flops = 2.0 * io.nr * (double)L.V * (double)L.H;

    if (ent) {  // student entropy: forward GEMM with the entropy epilogue, then merge
      EpiEntropy::Params pe{V, 1, (int)NT, scale2, nullptr, nullptr, nullptr, part, upart};
      {
        ProfScope ps(K_ENT, st, gemm_flops, 2.0 * (io.nr + (double)L.V) * L.H + io.nr * NT * 12.0);
        FCKL_LAUNCH((gemm_pair_kernel<EpiEntropy, false, false>), Gv, GEMM_THREADS,
                    pair_smem_bytes<EpiEntropy>(), mapH_k, mapW_k, mapW_k, pe, sa_v, ca);
      }
      {
        ProfScope ps(K_ENT_MERGE, st, 0.0, io.nr * NT * 12.0 + io.nr * 5.0);
        FCKL_LAUNCH(k_merge_entropy, io.row_blocks, ROW_WARPS * 32, 0, (const float2*)part,
                    (const float*)upart, (int)NT, io.rc, io.mask, q.entropy + io.row0);
      }
      if (more) {
        io = chunk_io(c + 1);
        if (const fckl_status s1 = stage_in(c + 1, io, st); s1 != FCKL_OK) return s1;
      }
      continue;
    }

    // Forward: the main loop reads h and W only, complete before the kernel
    // ahead of it launched (the gather ran before the teacher prep), so it
    // starts at once -- possibly over the tail of the previous chunk's dW
    // GEMM -- and only the epilogue waits.
    SchedArgs sa_f = sa_v;
    sa_f.early = 1;
    EpiLse::Params pf{V, K, (int)NT, scale2, sid, tstart, zs, part, nullptr};
    CtlArgs ca_f = ca;
    ca_f.debug_skip_commit = (c == 0) ? ca.debug_skip_commit : 0;
    {
      ProfScope ps(K_FWD, st, gemm_flops, 2.0 * (io.nr + (double)L.V) * L.H + io.nr * NT * 8.0);
      FCKL_LAUNCH((gemm_pair_kernel<EpiLse, false, false>), Gv, GEMM_THREADS,
                  pair_smem_bytes<EpiLse>(), mapH_k, mapW_k, mapW_k, pf, sa_f, ca_f);
    }
    {
      ProfScope ps(K_MERGE, st, 0.0, io.nr * K * 8.0 + io.nr * NT * 8.0 + io.nr * 13.0);
      FCKL_LAUNCH(k_merge_loss, io.row_blocks, ROW_WARPS * 32, 0, (const float2*)part, (int)NT,
                  io.rc, K, invT, (const float*)zs, (const float*)sp, (const float*)plogp, io.mask,
                  lse2, io.rl, io.out_rows, (long long)L.N);
    }
    if (!bwd) {
      if (more) {
        io = chunk_io(c + 1);
        if (const fckl_status s1 = stage_in(c + 1, io, st); s1 != FCKL_OK) return s1;
      }
      continue;
    }

    // Backward 1: recompute the tiles and form bf16 dlogits = q - p~.  Its
    // operands (h, W) were complete before the kernel ahead of it launched, so
    // its main loop starts at once and only its epilogue waits for the merge.
    // Rows past the chunk's last row, up to the next multiple of 64 (within
    // the chunk), are stored as zeros for the dW GEMM's last 64-row block.
    EpiDlogits::Params pb{V, K, (int)NT, scale2, lse2, sid, tstart, sp, io.mask, io.cap};
    SchedArgs sa_b = sa_v;
    sa_b.early = 1;
    CUtensorMap mapD_st;
    // The store map spans the padded width: the pad columns receive zeros.
    if (!make_map(&mapD_st, io.dlog, L.Vp, io.cap, L.Vp * 2, 64, 32)) return FCKL_ERR_CUDA;
    {
      ProfScope ps(K_BWD, st, gemm_flops, 2.0 * (io.nr + (double)L.V) * L.H + 2.0 * io.nr * L.V);
      FCKL_LAUNCH((gemm_pair_kernel<EpiDlogits, false, false>), Gv, GEMM_THREADS,
                  pair_smem_bytes<EpiDlogits>(), mapH_k, mapW_k, mapD_st, pb, sa_b, ca);
    }
    if (rsd != nullptr && more) {  // next chunk's gather + prep on the second stream
      const ChunkIO nxt = chunk_io(c + 1);
      if (cudaEventRecord(rsd->ev[2 * c], st) != cudaSuccess ||
          cudaStreamWaitEvent(rsd->rs, rsd->ev[2 * c], 0) != cudaSuccess)
        return FCKL_ERR_CUDA;
      if (const fckl_status s1 = stage_in(c + 1, nxt, rsd->rs); s1 != FCKL_OK) return s1;
      if (cudaEventRecord(rsd->ev[2 * c + 1], rsd->rs) != cudaSuccess) return FCKL_ERR_CUDA;
    }

    // Backward 2: dH[rows] = alpha * dlogits W; A = dlogits (K-major), B = W (MN-major),
    // reduce-added into the rows k_prep_teacher zeroed.
    CUtensorMap mapD_k, mapD_mn, mapH_mn, mapdH;
    if (!make_map(&mapD_k, io.dlog, L.V, io.cap, L.Vp * 2, BK, CM)) return FCKL_ERR_CUDA;
    // (gathered rows are added to the caller's rows without a map; the map
    // then spans all of dH and is not used)
    if (io.out_rows ? !make_map(&mapdH, q.dH, L.H, L.N, L.H * 4, 32, 32, true)
                    : !make_map(&mapdH, io.dH, L.H, io.cap, L.H * 4, 32, 32, true))
      return FCKL_ERR_CUDA;
    const long long tiles_h = io.MT * NTh;
    // A compacted chunk's row count is only known on the device: the kernel
    // picks the split there (S = 0) and the launch covers every pair.
    const int S = compact ? 0 : choose_split(tiles_h, KBv, pairs);
    SchedArgs sa_h{SCHED_SPLIT_K, (int)NTh, (int)KBv, S, 0, io.rc, 0, w3d, 0, narrow_h, 0,
                   dh_tile_order(), dh_serpentine()};
    EpiDH::Params ph{H, invT, ctl, io.out_rows, q.dH, (long long)L.N};
    {
      ProfScope ps(K_DH, st, gemm_flops,
                   2.0 * io.nr * (double)L.V + 2.0 * (double)L.V * L.H + 4.0 * io.nr * L.H);
      FCKL_LAUNCH((gemm_pair_kernel<EpiDH, false, true>),
                  S > 0 ? grid_for(tiles_h * S) : 2 * pairs, GEMM_THREADS, pair_smem_bytes<EpiDH>(),
                  mapD_k, mapW_mn, mapdH, ph, sa_h, ca);
    }
    const ChunkIO cur = io;
    // The next chunk's gather and teacher prep go ahead of this group's dW
    // GEMM, so that the next forward GEMM can follow the dW GEMM directly
    // (on the second stream they ran beside this chunk's dH GEMM).
    if (more) {
      io = chunk_io(c + 1);
      if (rsd != nullptr) {
        if (cudaStreamWaitEvent(st, rsd->ev[2 * c + 1], 0) != cudaSuccess) return FCKL_ERR_CUDA;
      } else if (const fckl_status s1 = stage_in(c + 1, io, st); s1 != FCKL_OK) {
        return s1;
      }
    }

    // Backward 3, once per group of G chunks (or at the last chunk):
    // dW (+)= alpha * dlogits^T h over the group's rows; A = dlogits^T, B = h
    // (both MN-major).
    if ((c + 1) % G != 0 && more) continue;
    const long long g0 = c / G * G;  // first chunk of the group
    const long long grow0 = g0 * L.C;
    const int gcap = (int)(cur.row0 + cur.cap - grow0);
    const void* h_g = list ? static_cast<const void*>(hslot(g0))
                           : static_cast<const uint8_t*>(q.hidden) + (size_t)grow0 * L.H * 2;
    int d3d = 0, h3d = 0;
    if (!make_map_mn(&mapD_mn, dlog, L.Vp, gcap, L.Vp * 2, &d3d)) return FCKL_ERR_CUDA;
    if (!make_map_mn(&mapH_mn, h_g, L.H, gcap, L.H * 2, &h3d)) return FCKL_ERR_CUDA;
    const long long MTv = cdiv(L.V, PM);
    EpiDW::Params pw{V, H, invT, g0 > 0 ? 1 : 0, ctl};
    if (compact && g0 == 0) {  // with no valid row no dW launch below writes dW
      ProfScope ps(K_ZERO_DW, st, 0.0, 0.0);
      FCKL_LAUNCH(k_zero_if_no_valid, 2 * pairs, 256, 0, reinterpret_cast<float4*>(q.dW),
                  (long long)(L.V * L.H / 4), (const DeviceCtl*)ctl);
    }
    // One launch over all vocabulary tiles, or -- for the last group of a
    // sliced call -- one launch per slice, each followed by its event.
    const bool sliced = q.n_slices > 0 && !more;
    const long long ns = sliced ? std::min<long long>(q.n_slices, MTv) : 1;
    const double gr = prof_rows < 0
                          ? (double)gcap
                          : (double)std::max(0LL, std::min<long long>(gcap, prof_rows - grow0));
    for (long long i = 0; i < ns; ++i) {
      const long long mt0 = i * MTv / ns, mt1 = (i + 1) * MTv / ns;
      const long long v0 = mt0 * PM, v1 = std::min<long long>(L.V, mt1 * PM);
      // The dW main loop reads only dlogits and h, complete before the kernel
      // ahead of it launched: it starts at once, the epilogue waits.
      SchedArgs sa_w{SCHED_TILES, (int)NTh, 0, 1, (int)(mt1 - mt0), rows_of(grow0, gcap), d3d, h3d,
                     (int)mt0, narrow_h, 1};
      {
        const double vs = (double)(v1 - v0);
        ProfScope ps(K_DW, st, 2.0 * gr * vs * (double)L.H,
                     2.0 * gr * vs + 2.0 * gr * L.H * ns + (g0 > 0 ? 8.0 : 4.0) * vs * L.H);
        FCKL_LAUNCH((gemm_pair_kernel<EpiDW, true, true>), grid_for((mt1 - mt0) * NTh),
                    GEMM_THREADS, pair_smem_bytes<EpiDW>(), mapD_mn, mapH_mn, mapdW, pw, sa_w, ca);
      }
      if (sliced) {
        if (cudaEventRecord(q.slice_events[i], st) != cudaSuccess) return FCKL_ERR_CUDA;
        q.slice_rows[i] = v0;
        q.slice_rows[i + 1] = v1;
      }
    }
    if (sliced) {  // slices beyond the vocabulary tiles are empty
      for (long long i = ns; i < q.n_slices; ++i) {
        if (cudaEventRecord(q.slice_events[i], st) != cudaSuccess) return FCKL_ERR_CUDA;
        q.slice_rows[i + 1] = L.V;
      }
    }
  }
  if (!ent) {
    ProfScope ps(K_FINAL, st, 0.0, (double)L.N * 4.0);
    FCKL_LAUNCH(k_finalize, 1, 1024, 0, (const float*)rl, (long long)L.N, (const DeviceCtl*)ctl,
                q.loss);
  }
#undef FCKL_LAUNCH
  if (cudaGetLastError() != cudaSuccess) return FCKL_ERR_CUDA;
  return FCKL_OK;
}

// ---------------------------------------------------------------- no-alloc forward
// Library-owned scratch for fckl_fwd_noalloc.  Every GPU that loads the
// library keeps this array resident until the process exits.
constexpr size_t kStaticScratchBytes = 32ull << 20;
__device__ __align__(256) uint8_t g_fwd_scratch[kStaticScratchBytes];

struct StaticScratch {
  bool ready = false;
  void* ptr = nullptr;
};
StaticScratch g_scratch[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of g_fwd_scratch on the current device.  In host code the
// symbol is only a host-side stand-in, so the address is looked up once per
// device with that device current.
void* static_scratch() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  StaticScratch& s = g_scratch[dev];
  if (!s.ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fwd_scratch) != cudaSuccess || p == nullptr) return nullptr;
    s.ptr = p;
    s.ready = true;
  }
  return s.ptr;
}

// Device-side error bits of the control block -> fckl_status, for callers
// that have no workspace to hand to fckl_check().
__global__ void k_export_status(const DeviceCtl* ctl, int32_t* status_out) {
  const uint32_t e = ctl->err;
  *status_out = (e & kErrTimeout)     ? (int32_t)FCKL_ERR_TIMEOUT
                : (e & kErrBadIndex)  ? (int32_t)FCKL_ERR_BAD_INDEX
                : (e & kErrBadTeacher) ? (int32_t)FCKL_ERR_BAD_TEACHER
                                       : (int32_t)FCKL_OK;
}

}  // namespace

// ---------------------------------------------------------------- host inputs
// Per device: a copy stream and a pool of events for the host-input entry
// point (created on first use, kept until the process exits).
struct HostIO {
  std::mutex mu;
  cudaStream_t cs = nullptr;
  std::vector<cudaEvent_t> ev;
};
HostIO g_hio[kMaxDevices];

// Device copies of the host inputs, after the regular workspace.
struct HostLayout {
  size_t off_hidden, off_ids, off_lg, off_mask, off_loss, total;
};
HostLayout make_host_layout(const fckl_problem* p) {
  HostLayout h{};
  size_t off = make_layout(p).total;
  auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, kAlign); return o; };
  h.off_hidden = take((size_t)p->N * p->H * 2);
  h.off_ids = take((size_t)p->N * p->K * 4);
  h.off_lg = take((size_t)p->N * p->K * 4);
  h.off_mask = take((size_t)p->N);
  h.off_loss = take(4);
  h.total = off;
  return h;
}

// Host rows [0, end[c]) hold every row chunk c reads: with a mask, chunk c
// takes the valid rows numbered [c*C, (c+1)*C) (in row order), so end[c] is one
// past the last of them; the piece that reaches the last valid row runs to N.
std::vector<long long> piece_ends(const uint8_t* mask, long long N, long long C) {
  const long long nchunks = cdiv(N, C);
  std::vector<long long> end(nchunks, N);
  if (mask == nullptr) {
    for (long long c = 0; c < nchunks; ++c) end[c] = std::min(N, (c + 1) * C);
    return end;
  }
  long long seen = 0, c = 0;
  for (long long i = 0; i < N && c < nchunks; ++i) {
    if (mask[i] == 0) continue;
    if (++seen == (c + 1) * C) end[c++] = i + 1;
  }
  if (c < nchunks) end[c] = N;  // the chunk holding the last valid row (or none)
  return end;
}

extern "C" {

fckl_status fckl_fwd_noalloc(const fckl_problem* prob, const void* hidden, const void* W,
                             const int32_t* topk_idx, const float* topk_logit,
                             const uint8_t* row_mask, float* loss, float* row_loss,
                             int32_t* device_status, void* stream) {
  if (!valid_problem(prob)) return FCKL_ERR_INVALID_ARG;
  if (!supported_problem(prob)) return FCKL_ERR_UNSUPPORTED;
  if (device_status && !aligned(device_status, 4)) return FCKL_ERR_INVALID_ARG;
  fckl_problem q = *prob;
  long long C = resolve_chunk(prob);
  // The caller's chunk, or the automatic one; if its scratch does not fit
  // (automatic chunk only), the largest multiple of PM rows below it that fits.
  for (;;) {
    q.chunk = C;
    if (make_layout(&q, false).total <= kStaticScratchBytes) break;
    if (prob->chunk != 0) return FCKL_ERR_WORKSPACE;
    C = (C - 1) / PM * PM;
    if (C < PM) return FCKL_ERR_WORKSPACE;
  }
  void* scratch = static_scratch();
  if (scratch == nullptr) return FCKL_ERR_CUDA;
  Request rq;
  rq.mode = Mode::kFwd;
  rq.prob = &q;
  rq.hidden = hidden; rq.W = W; rq.topk_idx = topk_idx; rq.topk_logit = topk_logit;
  rq.row_mask = row_mask; rq.loss = loss; rq.row_loss = row_loss;
  rq.workspace = scratch; rq.ws_bytes = kStaticScratchBytes; rq.stream = stream;
  rq.full_layout = false;
  const fckl_status st = run(rq);
  if (st != FCKL_OK || device_status == nullptr) return st;
  k_export_status<<<1, 1, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const DeviceCtl*>(scratch), device_status);
  return cudaGetLastError() == cudaSuccess ? FCKL_OK : FCKL_ERR_CUDA;
}


size_t fckl_workspace_bytes(const fckl_problem* prob) {
  if (!valid_problem(prob) || !supported_problem(prob)) return 0;
  return make_layout(prob).total;
}

int64_t fckl_resolved_chunk(const fckl_problem* prob) {
  if (!valid_problem(prob) || !supported_problem(prob)) return -1;
  return resolve_chunk(prob);
}

fckl_status fckl_fwd(const fckl_problem* prob, const void* hidden, const void* W,
                     const int32_t* topk_idx, const float* topk_logit, const uint8_t* row_mask,
                     float* loss, float* row_loss, void* workspace, size_t workspace_bytes,
                     void* stream) {
  Request q;
  q.mode = Mode::kFwd;
  q.prob = prob; q.hidden = hidden; q.W = W; q.topk_idx = topk_idx; q.topk_logit = topk_logit;
  q.row_mask = row_mask; q.loss = loss; q.row_loss = row_loss;
  q.workspace = workspace; q.ws_bytes = workspace_bytes; q.stream = stream;
  return run(q);
}

fckl_status fckl_fwd_bwd(const fckl_problem* prob, const void* hidden, const void* W,
                         const int32_t* topk_idx, const float* topk_logit,
                         const uint8_t* row_mask, float* loss, float* row_loss, float* dH,
                         float* dW, void* workspace, size_t workspace_bytes, void* stream) {
  Request q;
  q.mode = Mode::kFwdBwd;
  q.prob = prob; q.hidden = hidden; q.W = W; q.topk_idx = topk_idx; q.topk_logit = topk_logit;
  q.row_mask = row_mask; q.loss = loss; q.row_loss = row_loss; q.dH = dH; q.dW = dW;
  q.workspace = workspace; q.ws_bytes = workspace_bytes; q.stream = stream;
  return run(q);
}

fckl_status fckl_fwd_bwd_sliced(const fckl_problem* prob, const void* hidden, const void* W,
                                const int32_t* topk_idx, const float* topk_logit,
                                const uint8_t* row_mask, float* loss, float* row_loss, float* dH,
                                float* dW, void* workspace, size_t workspace_bytes, void* stream,
                                int32_t n_slices, void* const* slice_events,
                                int64_t* slice_rows) {
  if (n_slices < 1 || n_slices > 4096 || slice_events == nullptr || slice_rows == nullptr)
    return FCKL_ERR_INVALID_ARG;
  for (int32_t i = 0; i < n_slices; ++i)
    if (slice_events[i] == nullptr) return FCKL_ERR_INVALID_ARG;
  Request q;
  q.mode = Mode::kFwdBwd;
  q.prob = prob; q.hidden = hidden; q.W = W; q.topk_idx = topk_idx; q.topk_logit = topk_logit;
  q.row_mask = row_mask; q.loss = loss; q.row_loss = row_loss; q.dH = dH; q.dW = dW;
  q.workspace = workspace; q.ws_bytes = workspace_bytes; q.stream = stream;
  q.n_slices = n_slices;
  q.slice_events = reinterpret_cast<cudaEvent_t const*>(slice_events);
  q.slice_rows = slice_rows;
  slice_rows[0] = 0;
  return run(q);
}

size_t fckl_host_workspace_bytes(const fckl_problem* prob) {
  if (!valid_problem(prob) || !supported_problem(prob)) return 0;
  return make_host_layout(prob).total;
}

fckl_status fckl_fwd_bwd_host(const fckl_problem* prob, const void* hidden_host, const void* W,
                              const int32_t* topk_idx_host, const float* topk_logit_host,
                              const uint8_t* row_mask_host, float* loss_host, float* dH, float* dW,
                              void* workspace, size_t workspace_bytes, void* stream) {
  if (!valid_problem(prob)) return FCKL_ERR_INVALID_ARG;
  if (!hidden_host || !topk_idx_host || !topk_logit_host || !loss_host)
    return FCKL_ERR_INVALID_ARG;
  if (!supported_problem(prob)) return FCKL_ERR_UNSUPPORTED;
  const HostLayout HL = make_host_layout(prob);
  if (workspace == nullptr || !aligned(workspace, kAlign) || workspace_bytes < HL.total)
    return FCKL_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FCKL_ERR_CUDA;
  const long long N = prob->N, H = prob->H, K = prob->K;
  const long long C = resolve_chunk(prob);
  const long long nchunks = cdiv(N, C);
  const std::vector<long long> end = piece_ends(row_mask_host, N, C);

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* hid = ws + HL.off_hidden;
  int32_t* ids = reinterpret_cast<int32_t*>(ws + HL.off_ids);
  float* lg = reinterpret_cast<float*>(ws + HL.off_lg);
  uint8_t* mask = row_mask_host ? ws + HL.off_mask : nullptr;
  float* loss_dev = reinterpret_cast<float*>(ws + HL.off_loss);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  HostIO& io = g_hio[dev];
  std::lock_guard<std::mutex> lk(io.mu);
  if (io.cs == nullptr && cudaStreamCreateWithFlags(&io.cs, cudaStreamNonBlocking) != cudaSuccess) {
    io.cs = nullptr;
    return FCKL_ERR_CUDA;
  }
  while ((long long)io.ev.size() < nchunks + 2) {
    cudaEvent_t e = nullptr;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return FCKL_ERR_CUDA;
    io.ev.push_back(e);
  }
  // The copies start after the work already on the caller's stream (which may
  // still read the device copies of a previous call).
  auto ok = [](cudaError_t e) { return e == cudaSuccess; };
  if (!ok(cudaEventRecord(io.ev[0], st)) || !ok(cudaStreamWaitEvent(io.cs, io.ev[0], 0)))
    return FCKL_ERR_CUDA;
  if (mask && !ok(cudaMemcpyAsync(mask, row_mask_host, (size_t)N, cudaMemcpyHostToDevice, io.cs)))
    return FCKL_ERR_CUDA;
  if (!ok(cudaEventRecord(io.ev[1], io.cs))) return FCKL_ERR_CUDA;
  long long r0 = 0;
  for (long long c = 0; c < nchunks; ++c) {
    const long long r1 = end[c];
    if (r1 > r0) {
      const size_t n = (size_t)(r1 - r0);
      if (!ok(cudaMemcpyAsync(hid + (size_t)r0 * H * 2,
                              static_cast<const uint8_t*>(hidden_host) + (size_t)r0 * H * 2,
                              n * H * 2, cudaMemcpyHostToDevice, io.cs)) ||
          !ok(cudaMemcpyAsync(ids + (size_t)r0 * K, topk_idx_host + (size_t)r0 * K, n * K * 4,
                              cudaMemcpyHostToDevice, io.cs)) ||
          !ok(cudaMemcpyAsync(lg + (size_t)r0 * K, topk_logit_host + (size_t)r0 * K, n * K * 4,
                              cudaMemcpyHostToDevice, io.cs)))
        return FCKL_ERR_CUDA;
      r0 = r1;
    }
    if (!ok(cudaEventRecord(io.ev[2 + c], io.cs))) return FCKL_ERR_CUDA;
  }
  Request q;
  q.mode = Mode::kFwdBwd;
  q.prob = prob; q.hidden = hid; q.W = W; q.topk_idx = ids; q.topk_logit = lg;
  q.row_mask = mask; q.loss = loss_dev; q.dH = dH; q.dW = dW;
  q.workspace = workspace; q.ws_bytes = workspace_bytes; q.stream = stream;
  q.ready = io.ev.data() + 1;
  const fckl_status s = run(q);
  if (s != FCKL_OK) {
    cudaStreamWaitEvent(st, io.ev[1 + nchunks], 0);  // leave no copy running past the call
    return s;
  }
  if (!ok(cudaMemcpyAsync(loss_host, loss_dev, 4, cudaMemcpyDeviceToHost, st)))
    return FCKL_ERR_CUDA;
  return FCKL_OK;
}

fckl_status fckl_fwd_bwd_rows(const fckl_problem* prob, const void* hidden, const void* W,
                              const int32_t* topk_idx, const float* topk_logit,
                              const int32_t* rows, int64_t n_rows, float* loss, float* row_loss,
                              float* dH, float* dW, void* workspace, size_t workspace_bytes,
                              void* stream) {
  if (rows == nullptr || (dH == nullptr) != (dW == nullptr)) return FCKL_ERR_INVALID_ARG;
  Request q;
  q.mode = dH ? Mode::kFwdBwd : Mode::kFwd;
  q.prob = prob; q.hidden = hidden; q.W = W; q.topk_idx = topk_idx; q.topk_logit = topk_logit;
  q.rows = rows; q.n_rows = n_rows;
  q.loss = loss; q.row_loss = row_loss; q.dH = dH; q.dW = dW;
  q.workspace = workspace; q.ws_bytes = workspace_bytes; q.stream = stream;
  return run(q);
}

fckl_status fckl_student_entropy(const fckl_problem* prob, const void* hidden, const void* W,
                                 const uint8_t* row_mask, float* row_entropy, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  if (prob == nullptr) return FCKL_ERR_INVALID_ARG;
  fckl_problem p1 = *prob;  // the teacher does not take part: K is ignored
  p1.K = 1;
  Request q;
  q.mode = Mode::kEntropy;
  q.prob = &p1; q.hidden = hidden; q.W = W; q.row_mask = row_mask; q.entropy = row_entropy;
  q.workspace = workspace; q.ws_bytes = workspace_bytes; q.stream = stream;
  return run(q);
}

fckl_status fckl_select_top_rows(const float* score, const uint8_t* row_mask, int64_t N,
                                 int64_t n_select, int32_t* rows_out, int32_t* count_out,
                                 void* stream) {
  if (!score || !rows_out || !count_out || N < 1 || N > INT32_MAX || n_select < 1 ||
      n_select > N || !aligned(score, 4) || !aligned(rows_out, 4) || !aligned(count_out, 4))
    return FCKL_ERR_INVALID_ARG;
  const DeviceInfo* dev = device_info();
  if (dev == nullptr || !dev->ok) return FCKL_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  {
    ProfScope ps(K_SELECT, st, 0.0, N * 5.0 * 4 + n_select * 4.0);
    k_select_top_rows<<<1, 1024, 0, st>>>(score, row_mask, N, n_select, rows_out, count_out);
  }
  return cudaGetLastError() == cudaSuccess ? FCKL_OK : FCKL_ERR_CUDA;
}

fckl_status fckl_check(void* workspace, void* stream) {
  if (workspace == nullptr) return FCKL_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint32_t err = 0;
  if (cudaMemcpyAsync(&err, workspace, sizeof(err), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return FCKL_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return FCKL_ERR_CUDA;
  if (err & kErrTimeout) return FCKL_ERR_TIMEOUT;
  if (err & kErrBadIndex) return FCKL_ERR_BAD_INDEX;
  if (err & kErrBadTeacher) return FCKL_ERR_BAD_TEACHER;
  return FCKL_OK;
}

void fckl_profile_begin(uint32_t kind_mask) {
  g_prof.on = true;
  g_prof.mask = kind_mask ? kind_mask : 0xFFFFFFFFu;
  g_prof.recs.clear();
  g_prof.used = 0;
}

int fckl_profile_end(fckl_kernel_stat* stats, int max_stats) {
  g_prof.on = false;
  int order[K_NKINDS];
  int nkinds = 0;
  fckl_kernel_stat acc[K_NKINDS];
  std::memset(acc, 0, sizeof(acc));
  int slot[K_NKINDS];
  for (int k = 0; k < K_NKINDS; ++k) slot[k] = -1;
  for (const ProfRec& r : g_prof.recs) {
    if (cudaEventSynchronize(r.b) != cudaSuccess) return -1;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) return -1;
    if (slot[r.kind] < 0) {
      slot[r.kind] = nkinds;
      order[nkinds++] = r.kind;
    }
    fckl_kernel_stat& a = acc[slot[r.kind]];
    a.launches += 1;
    a.total_ms += ms;
    a.flops += r.flops;
    a.bytes += r.bytes;
  }
  for (int i = 0; i < nkinds && i < max_stats && stats; ++i) {
    stats[i] = acc[i];
    std::strncpy(stats[i].name, kKindName[order[i]], sizeof(stats[i].name) - 1);
    stats[i].name[sizeof(stats[i].name) - 1] = 0;
  }
  g_prof.recs.clear();
  g_prof.used = 0;
  return nkinds;
}

const char* fckl_status_string(fckl_status s) {
  switch (s) {
    case FCKL_OK: return "FCKL_OK";
    case FCKL_ERR_INVALID_ARG: return "FCKL_ERR_INVALID_ARG";
    case FCKL_ERR_UNSUPPORTED: return "FCKL_ERR_UNSUPPORTED";
    case FCKL_ERR_WORKSPACE: return "FCKL_ERR_WORKSPACE";
    case FCKL_ERR_BAD_INDEX: return "FCKL_ERR_BAD_INDEX";
    case FCKL_ERR_BAD_TEACHER: return "FCKL_ERR_BAD_TEACHER";
    case FCKL_ERR_TIMEOUT: return "FCKL_ERR_TIMEOUT";
    case FCKL_ERR_CUDA: return "FCKL_ERR_CUDA";
  }
  return "FCKL_ERR_UNKNOWN";
}

}  // extern "C"
