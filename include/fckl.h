/*
 * fckl.h -- fused chunked forward-KL distillation loss on B200 (sm_100a).
 *
 * The operation (notation of the library):
 *   rows r = 0..N-1 are the flattened batch x sequence positions; a row is valid
 *   when row_mask[r] != 0 (all rows when row_mask is NULL); N_v = #valid rows.
 *   z_r   = W h_r                         student logits over the vocabulary V
 *   q     = softmax(z_r / T)              over all V
 *   p     = softmax(topk_logit[r,:] / T)  over the K cached teacher ids, zero
 *                                         elsewhere (or given weights, see
 *                                         fckl_teacher_format)
 *   p~_v  = sum_{k: topk_idx[r,k] = v} p_k the dense teacher over V
 *   l_r   = sum_v p~_v (log p~_v - log q_v)  forward KL(p~ || q); with distinct
 *                                         ids = sum_k p_k (log p_k - log q[id_k])
 *   loss  = (1/N_v) sum_{valid r} l_r                      (0 when N_v = 0)
 *   dH_r  = dlogits_r W,  dW = sum_r dlogits_r^T h_r,
 *   dlogits_r = (q - p~) / (T N_v),  p~_v = sum_{k: topk_idx[r,k] = v} p_k,
 *   and dlogits_r = 0 for masked rows.
 *
 * Passages this implements:
 *   - "[논문리뷰] Efficient Knowledge Distillation for LLMs: Offline Top-K Logits
 *     and a Fused Chunked KL Loss", section 1 (Key Terms): the output projection
 *     is folded into the loss and the sequence is processed chunk by chunk, so
 *     the full-vocabulary logit tensor is never created; section 3: memory is
 *     linear in the sequence length.
 *   - aibase.it write-up "Knowledge Distillation 비용 줄이기", section
 *     "offline top-K logits 방식": the teacher is a per-position top-K cache of
 *     token ids and logits (top-100); section "chunked KL loss가 하는 일": per
 *     chunk, project hidden states to logits, add to the loss, discard, and
 *     recompute the chunk in the backward pass.
 *   - LLM Primer ch.6 "프루닝과 지식 증류", section 6.2: forward KL between the
 *     temperature-softened teacher and student.
 *   The pages give no formula for the gradient scale; this library applies no
 *   T^2 factor (the gradients are those of `loss` itself, upstream grad 1).
 *
 * Common conventions for every entry point:
 *   - Array pointers are DEVICE pointers into memory the caller owns (except
 *     the host inputs of fckl_fwd_bwd_host).  The library allocates no device
 *     memory; between calls it keeps only a per-device cache of kernel
 *     attributes, the copy stream and events of fckl_fwd_bwd_host, a second
 *     stream and events for the next chunk's row preparation (below), the
 *     profiler's events and the static scratch of fckl_fwd_noalloc.
 *   - Forward+backward calls of more than one chunk run the next chunk's row
 *     gather and teacher preparation on that library-owned stream, beside the
 *     current chunk's dH GEMM; it forks from and joins back into `stream` with
 *     events, so the call stays ordered on `stream` (and can be captured in a
 *     CUDA graph from it).  Calls that use it are serialised while they enqueue.
 *     FCKL_ONE_STREAM=1 in the environment keeps all work on `stream`;
 *     FCKL_NO_PDL=1 launches the kernels without programmatic dependent launch.
 *   - Arrays are dense and row-major.  hidden, W, dH and dW must start on a
 *     16-byte boundary (TMA), the others on a 4-byte boundary:
 *       hidden     bf16  [N, H]      (raw bfloat16 bit patterns)
 *       W          bf16  [V, H]
 *       topk_idx   int32 [N, K]      ids in [0, V); order within a row is free
 *       topk_logit fp32  [N, K]      may hold -inf (probability 0); not all -inf
 *       row_mask   uint8 [N] or NULL
 *       loss       fp32  scalar
 *       row_loss   fp32  [N] or NULL (per-row l_r, 0 for masked rows)
 *       dH         fp32  [N, H]      overwritten
 *       dW         fp32  [V, H]      overwritten
 *     A pointer carries no length: each array must hold the elements listed
 *     (a shorter buffer is read or written past its end).  The PyTorch helpers
 *     of the binding check tensor shapes before they call the library.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     asynchronous on that stream; the workspace must not be shared by calls
 *     that can overlap.
 *   - Errors that the host can see (null pointers, bad sizes, misalignment,
 *     T <= 0 or not finite, K > FCKL_K_MAX, H % 8 != 0, workspace too small)
 *     are returned before anything is enqueued.  Errors only the device can see
 *     (an id outside [0, V), a teacher row with no finite logit, an exhausted
 *     bounded wait) are recorded in the workspace and reported by fckl_check().
 */
#ifndef FCKL_H_
#define FCKL_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FCKL_K_MAX 256

typedef enum {
  FCKL_OK = 0,
  FCKL_ERR_INVALID_ARG = 1,   /* null pointer, size <= 0, misaligned, T not > 0 */
  FCKL_ERR_UNSUPPORTED = 2,   /* K > FCKL_K_MAX, H % 8 != 0, no sm_100 device   */
  FCKL_ERR_WORKSPACE = 3,     /* workspace NULL or smaller than required        */
  FCKL_ERR_BAD_INDEX = 4,     /* device: a topk_idx entry outside [0, V)        */
  FCKL_ERR_BAD_TEACHER = 5,   /* device: a valid row whose K logits are NaN,
                                 +inf, or all -inf                               */
  FCKL_ERR_TIMEOUT = 6,       /* device: a bounded wait inside a kernel ran out */
  FCKL_ERR_CUDA = 7           /* a CUDA runtime call or launch failed           */
} fckl_status;

/* Problem description.  chunk = rows per chunk (0 = automatic: the largest
 * multiple of 128 rows whose bf16 dlogits block [chunk, V] fits in 1 GiB,
 * capped at N rounded up to 64).  Every chunk runs its own dW GEMM by
 * default, so the workspace holds one chunk's bf16 dlogits and the live
 * device bytes are O(chunk * V) of workspace plus the caller's O(N * H)
 * activations and gradients and O(V * H) weights and dW -- the memory bound of
 * the chunked loss ("[논문리뷰] Efficient Knowledge Distillation for LLMs",
 * section 3; aibase.it write-up "Knowledge Distillation 비용 줄이기", section
 * "chunked KL loss가 하는 일").  dw_rows > chunk groups ceil(dw_rows / chunk)
 * consecutive chunks into one dW GEMM (at most all of them): fewer
 * read-modify-writes of the fp32 dW (V * H * 8 bytes each) for small chunks,
 * at the price of a workspace holding the whole group's dlogits.  With
 * chunk = 0 and dw_rows = 0 the library also picks the grouping: at least
 * 4096 rows per dW GEMM (e.g. two automatic 2560-row chunks at V = 201,088). */
typedef struct {
  int64_t N;        /* rows (batch * sequence)                  */
  int64_t H;        /* hidden size                              */
  int64_t V;        /* vocabulary size                          */
  int32_t K;        /* cached teacher entries per row           */
  float T;          /* temperature (> 0)                        */
  int64_t chunk;    /* rows per chunk, 0 = auto                 */
  int32_t teacher;  /* fckl_teacher_format of topk_logit        */
  int64_t n_valid_total; /* 0: N_v = the valid rows of this call;
                            > 0: N_v used for the mean and the gradient
                            scale, e.g. the valid rows of all data-parallel
                            ranks, each rank passing its own row shard */
  int64_t dw_rows;  /* 0: one dW GEMM per chunk (automatic chunk: at
                       least 4096 rows); > 0: each dW GEMM reduces over at
                       least this many rows (chunks grouped; see above).
                       0 <= dw_rows <= INT32_MAX */
} fckl_problem;

/* What the teacher cache holds in topk_logit [N, K]:
 *   FCKL_TEACHER_LOGITS  the top-K teacher logits; p = softmax(topk_logit / T)
 *                        over the row's K entries ("offline top-K logits 방식").
 *   FCKL_TEACHER_PROBS   non-negative class weights of sampled sparse targets
 *                        (RS-KD, "기술 요약: 선택적 지식 증류의 재고", 방법론);
 *                        p = topk_logit / sum(topk_logit) over the row, and T
 *                        applies to the student only.  A valid row whose
 *                        weights are negative, not finite or all zero is
 *                        reported as FCKL_ERR_BAD_TEACHER.
 * In both formats entries with the same id add into one class of the teacher
 * distribution p~ (the dense teacher grid), so ids may repeat. */
typedef enum { FCKL_TEACHER_LOGITS = 0, FCKL_TEACHER_PROBS = 1 } fckl_teacher_format;

/* Bytes of device workspace fckl_fwd / fckl_fwd_bwd / fckl_fwd_bwd_rows /
 * fckl_student_entropy need for `prob` (0 when the problem is invalid): the
 * per-chunk teacher and log-sum-exp buffers, the bf16 dlogits of one chunk
 * (of one dW group when dw_rows, or the automatic chunk, groups chunks), two
 * chunks' staged hidden rows, N floats of row loss, N int32
 * of compacted row list and the staging buffers that row-list and masked
 * calls gather into.  Pure host arithmetic; needs no GPU. */
size_t fckl_workspace_bytes(const fckl_problem* prob);

/* The chunk size the library will use for `prob` (resolves chunk = 0), or -1
 * when the problem is invalid.  Pure host arithmetic. */
int64_t fckl_resolved_chunk(const fckl_problem* prob);

/* Forward only: loss (and optionally row_loss).  Per chunk: teacher softmax
 * over the K cached logits, the fused projection z = h W^T on the tensor cores
 * with a full-vocabulary online log-sum-exp and a gather of z at the cached
 * ids (the [chunk, V] logit tile is never written), then the per-row KL.
 * With a row_mask, the valid rows are first compacted on the device and
 * gathered chunk by chunk, so masked rows cost no GEMM work (row_loss is 0
 * there).  Cost: 2*H*V flops per valid row. */
fckl_status fckl_fwd(const fckl_problem* prob, const void* hidden, const void* W,
                     const int32_t* topk_idx, const float* topk_logit,
                     const uint8_t* row_mask, float* loss, float* row_loss,
                     void* workspace, size_t workspace_bytes, void* stream);

/* Forward + backward: loss, row_loss (optional), dH and dW (fp32, overwritten).
 * Per chunk, after the forward steps above: recompute the logit tile, form
 * bf16 dlogits = q - p~ (masked rows 0) in the GEMM epilogue, then
 * dH_chunk = (1/(T N_v)) dlogits W and dW += (1/(T N_v)) dlogits^T h_chunk on
 * the tensor cores with fp32 accumulation; masked rows are skipped as in
 * fckl_fwd (their dH rows are 0).  Cost: 8*H*V flops per valid row. */
fckl_status fckl_fwd_bwd(const fckl_problem* prob, const void* hidden, const void* W,
                         const int32_t* topk_idx, const float* topk_logit,
                         const uint8_t* row_mask, float* loss, float* row_loss,
                         float* dH, float* dW,
                         void* workspace, size_t workspace_bytes, void* stream);

/* fckl_fwd_bwd with the dW write-out exposed slice by slice, so that a caller
 * can reduce finished parts of dW across ranks while the rest is computed
 * (row-sharded data parallelism: the dW all-reduce overlaps the last dW GEMM).
 * The last dW launch runs as min(n_slices, ceil(V/256)) launches over
 * consecutive vocabulary ranges; after the launch that finishes dW rows
 * [slice_rows[i], slice_rows[i+1]) the call records slice_events[i] (a
 * cudaEvent_t of the caller, on the current device) on `stream`.  Slices past
 * the vocabulary tiles are empty (their event is recorded after the last one).
 * slice_rows (host, n_slices + 1 entries) is filled before the call returns;
 * slice_rows[0] = 0 and slice_rows[n_slices] = V.  The dW rows of slice i are
 * final once event i has fired; everything else (loss, dH) is as in
 * fckl_fwd_bwd, complete in stream order after the call's work.
 * 1 <= n_slices <= 4096, every event non-NULL, else FCKL_ERR_INVALID_ARG.
 * (An addition of this library for multi-GPU use; the pages run on one GPU.) */
fckl_status fckl_fwd_bwd_sliced(const fckl_problem* prob, const void* hidden, const void* W,
                                const int32_t* topk_idx, const float* topk_logit,
                                const uint8_t* row_mask, float* loss, float* row_loss, float* dH,
                                float* dW, void* workspace, size_t workspace_bytes, void* stream,
                                int32_t n_slices, void* const* slice_events,
                                int64_t* slice_rows);

/* Bytes of device workspace fckl_fwd_bwd_host needs: the fckl_workspace_bytes
 * layout followed by device copies of hidden, topk_idx, topk_logit, row_mask
 * and the loss.  0 when the problem is invalid. */
size_t fckl_host_workspace_bytes(const fckl_problem* prob);

/* Forward + backward with the per-step inputs in HOST memory: hidden [N,H]
 * bf16, topk_idx [N,K], topk_logit [N,K] and row_mask [N] (or NULL) are host
 * pointers; W stays a device pointer (the student's resident output
 * projection); dH and dW are device outputs as in fckl_fwd_bwd; the loss is
 * copied to the host scalar *loss_host at the end of the call's work on
 * `stream`.  (An addition of this library: the pages feed the loss from
 * activations already on the GPU and a teacher cache read from storage.)
 *   - The inputs go to the device in chunk-sized pieces on a copy stream of the
 *     library's own (one per device, created on first use), so the copy of
 *     chunk c+1 overlaps the kernels of chunk c; each chunk waits on the
 *     caller's stream only for its own piece.  With a row mask, the call reads
 *     the host mask once on the host to place the piece boundaries.
 *   - Host buffers must stay valid and unchanged until the stream has passed
 *     the call; page-locked (pinned) memory keeps the copies asynchronous.
 *   - The device copies live in the workspace (fckl_host_workspace_bytes), so
 *     the call allocates no device memory.  Calls from several host threads
 *     are serialised while they enqueue.
 * Errors as fckl_fwd_bwd; device-side errors come back through fckl_check. */
fckl_status fckl_fwd_bwd_host(const fckl_problem* prob, const void* hidden_host, const void* W,
                              const int32_t* topk_idx_host, const float* topk_logit_host,
                              const uint8_t* row_mask_host, float* loss_host, float* dH, float* dW,
                              void* workspace, size_t workspace_bytes, void* stream);

/* Forward only (loss and optional row_loss), like fckl_fwd, but without a
 * workspace argument: the call allocates nothing and takes no memory from the
 * caller beyond its inputs and outputs.  It is meant for callers that cannot
 * call cudaMalloc or hand out scratch buffers -- for example code running
 * inside a host framework whose own allocator owns all device memory and
 * forbids side allocations, or a plugin whose interface passes only the
 * tensors it computes on.  (The pages describe no such entry point; it is an
 * addition of this library.)
 *   - Scratch lives in a 32 MiB file-scope __device__ array of the library;
 *     every GPU that loads the library holds it until the process exits.
 *   - The first call on a device looks up that array's device address with
 *     the device current (one cudaGetSymbolAddress per device); make that
 *     first call before any stream capture on the device.
 *   - The scratch holds N floats of per-row loss plus the per-chunk teacher
 *     and log-sum-exp buffers.  With prob->chunk = 0 the call takes the
 *     automatic chunk (see fckl_problem) if its scratch fits, else the largest
 *     multiple of 256 rows below it whose scratch fits; an explicit chunk that
 *     does not fit, or a problem for which even 256 rows do not fit, returns
 *     FCKL_ERR_WORKSPACE before anything is enqueued.
 *   - All calls share the one array and each call re-initialises what must
 *     start at zero; calls that can overlap on the GPU (other streams, other
 *     host threads) race on it and must be serialised by the caller.
 *   - device_status (device int32, may be NULL) receives, in stream order, the
 *     device-side status of this call (FCKL_OK, FCKL_ERR_BAD_INDEX,
 *     FCKL_ERR_BAD_TEACHER or FCKL_ERR_TIMEOUT) -- the role fckl_check() plays
 *     for the workspace entry points.
 * Other arguments, layouts and host-side errors are those of fckl_fwd. */
fckl_status fckl_fwd_noalloc(const fckl_problem* prob, const void* hidden, const void* W,
                             const int32_t* topk_idx, const float* topk_logit,
                             const uint8_t* row_mask, float* loss, float* row_loss,
                             int32_t* device_status, void* stream);

/* ----------------------------------------------------------------------------
 * Position selection by student entropy (the selective-distillation method of
 * "기술 요약: 선택적 지식 증류(Selective Knowledge Distillation)의 재고", sections
 * 방법론 (SE-KD: supervise the top-k% positions by student entropy H(q_t)) and
 * 효율성 최적화 (chunked entropy computation; a selective LM head that
 * computes logits and gradients only at the selected positions)).
 * ------------------------------------------------------------------------- */

/* Student entropy H(q_r) = -sum_v q_v ln q_v (nats), q = softmax(W h_r / T), for
 * every row, written to row_entropy [N] (0 for masked rows).  Computed chunk by
 * chunk in the epilogue of the projection GEMM: the logits are never stored.
 * prob->K and the teacher arrays take no part (K is ignored).  Uses the same
 * workspace as fckl_fwd_bwd.  Cost: 2*H*V flops per row. */
fckl_status fckl_student_entropy(const fckl_problem* prob, const void* hidden, const void* W,
                                 const uint8_t* row_mask, float* row_entropy, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* The n_select rows with the largest score (e.g. row_entropy) among the valid
 * rows (row_mask != 0, or all rows when NULL), written to rows_out in
 * ascending row order; ties at the threshold go to the lower row index.  If
 * fewer than n_select rows are valid, all valid rows are written and the rest
 * of rows_out[0, n_select) is set to -1.  *count_out (device int32) receives
 * the number of rows written.  Scores must not be NaN.  Device pointers;
 * 1 <= n_select <= N.  One kernel, no workspace. */
fckl_status fckl_select_top_rows(const float* score, const uint8_t* row_mask, int64_t N,
                                 int64_t n_select, int32_t* rows_out, int32_t* count_out,
                                 void* stream);

/* Loss and gradients over a list of rows only (a selective LM head): rows is a
 * device int32 [n_rows] of distinct row indices in [0, N); negative entries are
 * skipped (so the padded output of fckl_select_top_rows can be passed as is).
 * The listed rows are gathered chunk by chunk, so the GEMM work scales with
 * the number of listed rows, not with N.  Results equal fckl_fwd_bwd with
 * row_mask = the indicator of the listed rows: loss = mean over listed rows,
 * row_loss and dH rows of unlisted rows are 0, dW sums over listed rows.
 * dH = dW = NULL computes the loss only.  hidden/topk arrays are the full
 * [N, ...] arrays; the workspace is fckl_workspace_bytes(prob).  An entry >= N
 * is reported by fckl_check as FCKL_ERR_BAD_INDEX and skipped. */
fckl_status fckl_fwd_bwd_rows(const fckl_problem* prob, const void* hidden, const void* W,
                              const int32_t* topk_idx, const float* topk_logit,
                              const int32_t* rows, int64_t n_rows, float* loss, float* row_loss,
                              float* dH, float* dW, void* workspace, size_t workspace_bytes,
                              void* stream);

/* Synchronises `stream`, then returns the first device-side error recorded in
 * `workspace` by the last call that used it (FCKL_OK if none), or
 * FCKL_ERR_CUDA if the stream reports a CUDA error. */
fckl_status fckl_check(void* workspace, void* stream);

/* Static, human-readable name of a status code. */
const char* fckl_status_string(fckl_status status);

/* Optional per-kernel timing for measurement tools.  Between
 * fckl_profile_begin(mask) and fckl_profile_end(), every kernel the library
 * launches whose kind is selected by `mask` (bit i = kind i of the list below;
 * 0 selects every kind) is bracketed by two CUDA events recorded on the
 * call's stream (events are created on first use and reused; no device
 * memory is allocated).  Event records between kernels cost time, so select
 * only the kinds you need while timing a whole call.  fckl_profile_end()
 * synchronises those events, stops recording and writes up to `max_stats`
 * per-kernel summaries (one per kind, in first-launch order); it returns how
 * many kinds were seen, or -1 on a CUDA error.  Recording is process-wide and
 * not thread-safe.
 * A masked call's flop and byte figures count the rows it processes (its
 * valid rows); to know their number it reads one integer back from the device
 * once per call while recording is on.
 * Kinds: 0 count_valid, 1 prep_teacher, 2 fwd_logits_lse, 3 merge_loss,
 *        4 bwd_dlogits, 5 dH_gemm, 6 dW_gemm, 7 finalize, 8 entropy_gemm,
 *        9 merge_entropy, 10 gather_rows, 11 scatter_rows (reserved: gathered
 *        rows write their results in place, no kernel of this kind runs),
 *        12 select_rows, 13 zero_dw. */
typedef struct {
  char name[32];     /* kernel kind, e.g. "fwd_logits_lse" */
  int64_t launches;  /* launches recorded */
  double total_ms;   /* sum of event-timed durations */
  double flops;      /* algorithmic flops of those launches (GEMMs: 2*M*N*K) */
  double bytes;      /* algorithmic HBM bytes of those launches (compulsory
                        reads + writes of operands and outputs) */
} fckl_kernel_stat;

void fckl_profile_begin(uint32_t kind_mask);
int fckl_profile_end(fckl_kernel_stat* stats, int max_stats);

#ifdef __cplusplus
}
#endif

#endif /* FCKL_H_ */
