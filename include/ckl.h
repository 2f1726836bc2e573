/*
 * ckl.h -- C ABI of libckl.so, the fused chunked KL-distillation loss on
 * NVIDIA B200 (sm_100a).
 *
 * The method: Multiverse Computing, "Efficient Knowledge Distillation for
 * LLMs: Offline Top-K Logits and a Fused Chunked KL Loss".  The teacher runs
 * once and its top-K tokens per position are cached as (token id, log-prob)
 * pairs ("Дистилляция LLM на одной GPU: offline-кэш и chunked KL loss",
 * section «Два приёма»).  The loss projects the student's hidden states to
 * logits one chunk of the sequence at a time, folds the chunk into a running
 * loss and drops it; the backward recomputes each chunk, so no [T, V] logit
 * grid is ever held and memory grows linearly with T ("LLMのための効率的な
 * 知識蒸留...", section "2つのシステム変更").
 *
 * The pages do not print the formula.  This library computes the forward KL
 * of the renormalised teacher top-K against the full-vocabulary student
 * softmax, averaged over the positions that count:
 *
 *   z_tv  = sum_j H[t,j] W[v,j]            lse_t = log sum_v exp(z_tv)
 *   p_tk  = softmax_k(topk_logp[t,:])      (renormalised over the K entries)
 *   KL_t  = sum_k p_tk (log p_tk - z_{t,idx_tk} + lse_t)
 *   loss  = sum_t m_t KL_t / N,  N = sum_t m_t  (loss = 0 when N = 0)
 *   dL/dz_tv = (g m_t / N) (exp(z_tv - lse_t) - sum_k p_tk [idx_tk = v])
 *   dH = (dL/dz) W,  dW = (dL/dz)^T H
 *
 * Conventions for every call:
 *  - Layout: every array is row-major and contiguous.  bf16 arrays are passed
 *    as uint16_t bit patterns.  Pointers are DEVICE pointers owned by the
 *    caller unless stated otherwise; the library allocates nothing and keeps
 *    nothing between calls (it only caches per-device properties such as the
 *    SM count).
 *  - Sizes: T >= 0 tokens, d >= 8 with d % 8 == 0 (16-byte rows for the TMA
 *    unit), V >= 1, 1 <= K <= 2048, chunk >= 1.  T, d and V are below 2^31.
 *  - Alignment: H, W, dH, dW and the workspace must be 16-byte aligned.
 *  - Errors detectable on the host (null pointer, bad size, misalignment,
 *    small workspace) return a status before anything is enqueued.  A
 *    failed launch returns CKL_ERR_CUDA.  Errors that depend on the data
 *    (a teacher id outside [0, V), a teacher row with no finite log-prob, a
 *    NaN or +inf log-prob, a device wait that ran out of time) are recorded
 *    in a status word inside the workspace; read it with
 *    ckl_read_device_status.  Outputs are unspecified when it is non-zero.
 *  - Asynchrony: calls enqueue work on `stream` (a cudaStream_t; NULL = the
 *    legacy default stream) and return without waiting.
 *  - Concurrency: calls that share a workspace must not overlap on the GPU.
 */
#ifndef CKL_H_
#define CKL_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CKL_API __attribute__((visibility("default")))
#else
#define CKL_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every entry point. */
typedef enum ckl_status {
  CKL_OK = 0,
  CKL_ERR_INVALID_ARG = 1, /* null pointer, size out of range, misalignment */
  CKL_ERR_UNSUPPORTED = 2, /* no sm_100 device, or K above 2048 */
  CKL_ERR_WORKSPACE = 3,   /* workspace smaller than ckl_workspace_bytes() */
  CKL_ERR_CUDA = 4,        /* a CUDA runtime/driver call or launch failed */
  CKL_ERR_BAD_INDEX = 5,   /* device: a teacher id outside [0, V) */
  CKL_ERR_BAD_LOGP = 6,    /* device: NaN/+inf log-prob, or a row with none finite */
  CKL_ERR_TIMEOUT = 7,     /* device: a bounded wait inside a kernel ran out */
  CKL_ERR_TOPK_TIES = 8,   /* device: too many logits tie at a row's K-th value */
  CKL_ERR_DUP_INDEX = 9    /* a teacher id repeated within a row (ckl_find_duplicate_ids) */
} ckl_status;

/* Kernel ids written by the optional launch trace. */
enum {
  CKL_KERNEL_PREP = 1,        /* teacher cache check, renormalisation, sort, N */
  CKL_KERNEL_FWD_GEMM = 2,    /* logit GEMM + online log-sum-exp + teacher gather */
  CKL_KERNEL_FWD_COMBINE = 3, /* merge vocabulary splits: lse, KL, masked mean */
  CKL_KERNEL_BWD_DZ = 4,      /* logit recompute + dZ = softmax - scatter(p) */
  CKL_KERNEL_BWD_DHDW = 5,    /* dH = s dZ W and dW += s dZ^T H for one chunk */
  CKL_KERNEL_OTHER = 6,
  CKL_KERNEL_TOPK = 7,        /* teacher top-K cache producer */
  CKL_KERNEL_SP_GEMM = 8,     /* single pass: one chunk's logit GEMM, stores fp32 z too */
  CKL_KERNEL_SP_ROWS = 9      /* single pass: lse, loss terms and dZ from the stored z */
};

/*
 * Optional per-launch trace (tracing / profiling aid).  When a non-NULL
 * trace is passed, the library records events[2 i] before and events[2 i + 1]
 * after its i-th kernel launch on `stream`, writes kernel_id[i], and bumps
 * `count`, for as long as count < capacity.  The events are cudaEvent_t
 * handles created by the caller; the library never creates or destroys them.
 * Only the library's own kernels are traced (not memsets).
 */
typedef struct ckl_trace {
  int32_t capacity;   /* in:  launch slots available */
  int32_t count;      /* in/out: launches recorded so far */
  void** events;      /* in:  [2 * capacity] cudaEvent_t */
  int32_t* kernel_id; /* out: [capacity] CKL_KERNEL_* */
} ckl_trace;

/*
 * Workspace bytes needed by ckl_forward / ckl_backward for these sizes.
 * Linear in T: per token K*8 (sorted teacher pairs) + 4 (sum p log p) +
 * 64*16 (vocabulary-split partials) + 8/256 bytes, plus, independent of T
 * once T > chunk, a chunk x V bf16 buffer for dZ (min(chunk, T) rows of
 * round_up(V, 64) entries), and for the blocked backward (ckl_backward_plan)
 * a transposed copy of up to R rows of H (d x R bf16) and an fp32 partial dH
 * of R rows (R x d fp32), R = min(round_up(sqrt(chunk V), 256), the rows of
 * 48 MiB of H) or 0 when T <= chunk, and a 256-byte header.  Returns 0 for
 * sizes outside the supported range.
 */
CKL_API size_t ckl_workspace_bytes(int64_t T, int64_t d, int64_t V, int32_t K, int64_t chunk);

/*
 * The blocking ckl_backward uses for these sizes (host only, no device work):
 * plan[0] = rows per row chunk (Cr), plan[1] = vocabulary columns per slab
 * (Sv, a multiple of 256 when plan[2] > 1), plan[2] = slabs per row chunk.
 * The pages' schedule is one chunk of rows x all V at a time (plan =
 * {min(chunk, T), round_up(V, 64), 1}).  When the batch spans several chunks
 * the library may instead take taller row chunks swept in vocabulary slabs,
 * with Cr x Sv <= min(chunk, T) x round_up(V, 64) (the same dZ buffer): dW is
 * then re-added once per tall row chunk instead of once per chunk, and a
 * partial fp32 dH (Cr x d, in the workspace) is added once per slab; it is
 * chosen when that moves fewer bytes.  Returns CKL_ERR_INVALID_ARG for sizes
 * outside the supported range or a NULL plan.
 */
CKL_API int ckl_backward_plan(int64_t T, int64_t d, int64_t V, int32_t K, int64_t chunk,
                              int64_t* plan);

/*
 * Forward: the mean KL over the positions that count, and lse for EVERY row
 * (masked rows too).  The pages' forward pass: hidden states are projected
 * to logits a piece at a time and each piece is folded into the running
 * loss and dropped ("Дистилляция LLM на одной GPU: offline-кэш и chunked KL
 * loss", section «Два приёма»); here the pieces are 128 x 256 tensor-core
 * tiles whose epilogue keeps an online log-sum-exp and gathers the teacher
 * ids, so no logit is ever stored.
 *   H          [T, d] bf16  student hidden states
 *   W          [V, d] bf16  output head
 *   topk_idx   [T, K] int32 cached teacher token ids (repeats allowed; each
 *                           entry is its own term of the sum over k)
 *   topk_logp  [T, K] fp32  cached teacher log-probs (any offset per row;
 *                           renormalised over K; -inf = probability 0)
 *   mask       [T]    uint8 non-zero = position counts; NULL = all count
 *   chunk                   rows per backward step (sets the dZ buffer size;
 *                           the forward holds no per-chunk logits at all)
 *   loss       [1]    fp32  out
 *   lse        [T]    fp32  out: log-sum-exp of each row's logits
 *   workspace               >= ckl_workspace_bytes(T, d, V, K, chunk) bytes
 *   stream                  cudaStream_t
 *   trace                   optional launch trace, may be NULL
 */
CKL_API int ckl_forward(const uint16_t* H, const uint16_t* W, const int32_t* topk_idx,
                const float* topk_logp, const uint8_t* mask, int64_t T, int64_t d, int64_t V,
                int32_t K, int64_t chunk, float* loss, float* lse, void* workspace,
                size_t workspace_bytes, void* stream, ckl_trace* trace);

/*
 * Backward by recomputation: the backward rebuilds each chunk's logits
 * instead of keeping them ("LLMのための効率的な知識蒸留...", section
 * "2つのシステム変更"), and the logit gradient is the closed form the paper
 * mentions ("Tối ưu hóa chi phí chưng cất tri thức ...", closing paragraph,
 * after "Mô hình học sinh thu được").  One block at a time, each block's
 * logits are rebuilt from H and W, turned into the unscaled logit gradient
 * dZ = exp(z - lse) - scatter(p) (0 on rows that do not count), stored as
 * bf16 in the workspace (at most chunk x V entries), then fed to two
 * tensor-core GEMMs: dH_c = s dZ_c W and dW (+)= s dZ_c^T H_c, with
 * s = g / N.  A block is one chunk of rows x all V (the pages' schedule) or,
 * when that moves fewer bytes, a taller row chunk x a vocabulary slab of the
 * same size (ckl_backward_plan reports which); the results are the same up
 * to fp32 summation order.
 *   lse        [T]    fp32  from ckl_forward on the same inputs
 *   grad_loss  [1]    fp32  upstream gradient g (device); NULL = 1
 *   dH         [T, d] bf16  out (fp32 accumulation, rounded once)
 *   dW         [V, d] fp32  out: overwritten when accumulate_dW == 0, else
 *                           the gradient is added to its contents
 * Other arguments as in ckl_forward.  The workspace need not hold anything
 * from the forward; the teacher cache is prepared again.
 */
CKL_API int ckl_backward(const uint16_t* H, const uint16_t* W, const int32_t* topk_idx,
                 const float* topk_logp, const uint8_t* mask, int64_t T, int64_t d, int64_t V,
                 int32_t K, int64_t chunk, const float* lse, const float* grad_loss,
                 uint16_t* dH, float* dW, int32_t accumulate_dW, void* workspace,
                 size_t workspace_bytes, void* stream, ckl_trace* trace);

/*
 * Single-pass forward + backward (the loss is the only consumer of the
 * logits, and g is known before the forward runs).
 *
 * The pages measure the fused method's backward projection as its extra cost
 * at 8K context ("Tối ưu hóa chi phí chưng cất tri thức ...", section "Điều
 * này thay đổi những gì trong thực tế"; "LLMのための効率的な知識蒸留", table
 * in "パフォーマンスとメモリのベンチマーク": fused chunked slower than
 * forward-chunked).  This entry point drops the recompute: per chunk of rows
 * it runs the logit GEMM once, storing the chunk's fp32 logits (chunk x V)
 * beside the online log-sum-exp, turns them into dZ once lse is known, and
 * feeds dZ to the same dH / dW GEMMs as ckl_backward, once per group of up
 * to four chunks (so dW is read and written once per group).  6 d V FLOP per
 * token instead of 8 d V, for chunk x V x 4 more workspace bytes (the fp32
 * logits) and a dZ buffer of up to 4 chunks x V bf16.  Results equal
 * ckl_forward followed by ckl_backward up to rounding (lse may differ in the
 * last bits: the vocabulary is split differently per chunk).
 *   grad_loss  [1]    fp32  upstream gradient g (device); NULL = 1
 *   loss, lse               as in ckl_forward
 *   dH, dW, accumulate_dW   as in ckl_backward
 *   workspace               >= ckl_single_pass_workspace_bytes(...) bytes
 * Other arguments as in ckl_forward.
 */
CKL_API size_t ckl_single_pass_workspace_bytes(int64_t T, int64_t d, int64_t V, int32_t K,
                                               int64_t chunk);
CKL_API int ckl_forward_backward(const uint16_t* H, const uint16_t* W, const int32_t* topk_idx,
                                 const float* topk_logp, const uint8_t* mask, int64_t T,
                                 int64_t d, int64_t V, int32_t K, int64_t chunk,
                                 const float* grad_loss, float* loss, float* lse, uint16_t* dH,
                                 float* dW, int32_t accumulate_dW, void* workspace,
                                 size_t workspace_bytes, void* stream, ckl_trace* trace);

/*
 * ckl_backward with a host callback for overlapping the gradient exchange of
 * data-parallel training (no counterpart in the pages, which run on one GPU).
 * on_dw_ready(v_begin, v_end, user) is called on the calling host thread,
 * in increasing v order, as soon as the launches that write dW rows
 * [v_begin, v_end) for the last time have been ENQUEUED on `stream` (not
 * completed): work the callback orders after them on `stream` (an event, a
 * collective on a stream that waits for `stream`) sees those rows final while
 * the rest of the backward keeps running.  The ranges partition [0, V):
 * one per vocabulary slab when the backward is sliced (ckl_backward_plan),
 * else one for all of V after the last chunk.  The callback must not call
 * into this library.  on_dw_ready may be NULL (then this is ckl_backward).
 */
typedef void (*ckl_dw_ready_fn)(int64_t v_begin, int64_t v_end, void* user);
CKL_API int ckl_backward_ex(const uint16_t* H, const uint16_t* W, const int32_t* topk_idx,
                            const float* topk_logp, const uint8_t* mask, int64_t T, int64_t d,
                            int64_t V, int32_t K, int64_t chunk, const float* lse,
                            const float* grad_loss, uint16_t* dH, float* dW,
                            int32_t accumulate_dW, void* workspace, size_t workspace_bytes,
                            void* stream, ckl_trace* trace, ckl_dw_ready_fn on_dw_ready,
                            void* user);

/*
 * fp32 inputs (the pages' fp32 case): the same loss and gradients with H and
 * W in fp32, multiplied on the tensor cores as tf32 (tcgen05 kind::tf32,
 * fp32 accumulation; 10-bit mantissa products).  dH is fp32 (like H); dZ is
 * held in fp32, so the workspace (ckl_workspace_bytes_f32) holds 4 bytes per
 * dZ entry instead of 2.  Arguments, layouts, status and error behaviour as
 * in ckl_forward / ckl_backward, with float in place of bf16.
 */
CKL_API size_t ckl_workspace_bytes_f32(int64_t T, int64_t d, int64_t V, int32_t K,
                                       int64_t chunk);
CKL_API int ckl_forward_f32(const float* H, const float* W, const int32_t* topk_idx,
                            const float* topk_logp, const uint8_t* mask, int64_t T, int64_t d,
                            int64_t V, int32_t K, int64_t chunk, float* loss, float* lse,
                            void* workspace, size_t workspace_bytes, void* stream,
                            ckl_trace* trace);
CKL_API int ckl_backward_f32(const float* H, const float* W, const int32_t* topk_idx,
                             const float* topk_logp, const uint8_t* mask, int64_t T, int64_t d,
                             int64_t V, int32_t K, int64_t chunk, const float* lse,
                             const float* grad_loss, float* dH, float* dW,
                             int32_t accumulate_dW, void* workspace, size_t workspace_bytes,
                             void* stream, ckl_trace* trace);

/*
 * Self-test of the kernels' bounded waits (failure detection without a GPU
 * fault; no counterpart in the pages).  Launches one CTA on `stream` that
 * waits, with the same time-bounded mbarrier wait every kernel uses, on a
 * barrier nothing arrives on.  After limit_ns (1 ms .. 4 s) the wait gives
 * up, CKL_DEV_TIMEOUT is recorded in the status word at the start of
 * `workspace` (>= 256 bytes, 16-byte aligned), and the kernel returns: the
 * context stays usable.  ckl_read_device_status(workspace, ...) then returns
 * CKL_ERR_TIMEOUT.  Returns CKL_ERR_INVALID_ARG for a bad limit or workspace.
 */
CKL_API int ckl_selftest_wait_timeout(int64_t limit_ns, void* workspace, size_t workspace_bytes,
                                      void* stream);

/*
 * Vocabulary-parallel loss: the head is split by rows over g GPUs, rank r
 * holding W_shard = W[v_begin, v_end) (the output projection of a model
 * whose vocabulary is sharded, so that no GPU holds all of W or dW).  The
 * pages run one GPU and say that the fused loss let a GPT-OSS-20B
 * distillation shrink from four nodes to one ("Tối ưu hóa chi phí chưng cất
 * tri thức ...", section "Mở rộng quy mô đến độ dài ngữ cảnh dài"); this is
 * the split a larger head takes when it does not fit one GPU.  Every rank
 * holds all T rows of H and of the teacher cache; ids are global, in [0, V).
 *
 * ckl_forward_vocab_shard: prep + logit GEMM over this shard's columns;
 *   writes row_partials [T, 4] fp32 (16-byte aligned): per row, (m, s, pz, 0)
 *   with m = max over the shard of z log2(e), s = sum over the shard of
 *   2^(z log2(e) - m), pz = sum of p_k z over the teacher ids inside the
 *   shard.  Workspace: ckl_workspace_bytes(T, d, v_end - v_begin, K, chunk).
 * ckl_combine_vocab_shards: gathered [g, T, 4] = every rank's row_partials
 *   in rank order (an all-gather); writes lse [T] and the loss, exactly as
 *   ckl_forward does from its vocabulary splits.  Uses the sum p log p and N
 *   that ckl_forward_vocab_shard left in `workspace` (same T, K).
 * ckl_backward_vocab_shard: recomputes this shard's logits with the global
 *   lse; writes dH_partial [T, d] fp32 = this shard's share of dH (sum it
 *   over the ranks, then round with ckl_dh_to_bf16) and dW_shard
 *   [v_end - v_begin, d] fp32 (store, or add when accumulate_dW), which is
 *   final: it needs no exchange.
 * ckl_dh_to_bf16: dst[i] = bf16(src[i]), round to nearest even, n % 4 == 0,
 *   src 16-byte and dst 8-byte aligned.
 * Sizes, alignment and errors as in ckl_forward / ckl_backward, plus
 * CKL_ERR_INVALID_ARG unless 0 <= v_begin < v_end <= V.
 */
CKL_API int ckl_forward_vocab_shard(const uint16_t* H, const uint16_t* W_shard,
                                    const int32_t* topk_idx, const float* topk_logp,
                                    const uint8_t* mask, int64_t T, int64_t d, int64_t V,
                                    int64_t v_begin, int64_t v_end, int32_t K, int64_t chunk,
                                    float* row_partials, void* workspace, size_t workspace_bytes,
                                    void* stream, ckl_trace* trace);
CKL_API int ckl_combine_vocab_shards(const float* gathered, int32_t g, const uint8_t* mask,
                                     int64_t T, int32_t K, float* loss, float* lse,
                                     void* workspace, size_t workspace_bytes, void* stream,
                                     ckl_trace* trace);
CKL_API int ckl_backward_vocab_shard(const uint16_t* H, const uint16_t* W_shard,
                                     const int32_t* topk_idx, const float* topk_logp,
                                     const uint8_t* mask, int64_t T, int64_t d, int64_t V,
                                     int64_t v_begin, int64_t v_end, int32_t K, int64_t chunk,
                                     const float* lse, const float* grad_loss, float* dH_partial,
                                     float* dW_shard, int32_t accumulate_dW, void* workspace,
                                     size_t workspace_bytes, void* stream, ckl_trace* trace);
CKL_API int ckl_dh_to_bf16(const float* src, uint16_t* dst, int64_t n, void* stream);

/*
 * Data-parallel training over T (no counterpart in the pages, which run on
 * one GPU): each rank holds its own rows of the batch and all of W, and the
 * loss is the mean over the positions that count on every rank.
 *
 * ckl_dp_local_stats: after ckl_forward on this rank's rows with
 * `workspace`, writes (device memory, 8-byte aligned, fp64)
 *   stats[0] = stats[2] = sum over this rank's counted positions of KL_t,
 *   stats[1] = stats[3] = N_r, the number of those positions.
 * The step then sums stats[0..1] over the ranks (an all-reduce of two
 * doubles) and keeps stats[2..3] as they are.
 *
 * ckl_dp_finish: from the summed stats[0..1] and this rank's N_r (stats[3]),
 * writes loss = stats[0] / stats[1] (0 when no position counts on any rank)
 * and grad_local = g N_r / N (fp32, device; g = *grad_loss, NULL = 1; 0 when
 * N = 0).  ckl_backward on this rank with grad_loss = grad_local scales by
 * g / N, so its dH rows are final and its dW is this rank's share of the
 * gradient; summing dW over the ranks gives the global dW.
 * Both enqueue one tiny kernel on `stream` and return CKL_ERR_INVALID_ARG for
 * null or misaligned pointers.
 */
CKL_API int ckl_dp_local_stats(const void* workspace, double* stats, void* stream);
CKL_API int ckl_dp_finish(const double* stats, const float* grad_loss, float* loss,
                          float* grad_local, void* stream);

/*
 * Reads the device status word of the last call that used `workspace`:
 * synchronises `stream`, copies the word to *device_status (a host pointer)
 * and returns the matching ckl_status (CKL_OK when the word is 0).
 */
CKL_API int ckl_read_device_status(const void* workspace, void* stream, int32_t* device_status);

/*
 * The offline teacher cache ("Дистилляция LLM на одной GPU: offline-кэш и
 * chunked KL loss", section «Два приёма»: the teacher runs once and its 100
 * most likely tokens per position are kept).  From the teacher's logits,
 * writes per row the K most likely token ids, ordered by descending logit
 * (equal logits: smaller id first), and their log-probabilities under the
 * full-vocabulary softmax, z_v - log sum_u exp z_u.
 *   teacher_logits [T, V] bf16  device, row-major, finite values
 *   topk_idx       [T, K] int32 out
 *   topk_logp      [T, K] fp32  out
 *   device_status  [1]    int32 device memory or NULL: zeroed, then
 *                               bit 8 is set when a row has more than
 *                               2048 elements at or above its K-th largest
 *                               logit (ties at that value; the row's output
 *                               is then unspecified)
 * Requires 1 <= K <= min(V, 2048).  Needs no workspace.  Enqueued on
 * `stream`.  ckl_status_string(CKL_ERR_TOPK_TIES) names the device error.
 */
CKL_API int ckl_topk_cache(const uint16_t* teacher_logits, int64_t T, int64_t V, int32_t K,
                           int32_t* topk_idx, float* topk_logp, int32_t* device_status,
                           void* stream);

/*
 * Optional duplicate-id check of a teacher cache.  The pages' cache keeps
 * each position's 100 most likely tokens ("Дистилляция LLM на одной GPU:
 * offline-кэш и chunked KL loss", section «Два приёма»), so its ids are
 * distinct; ckl_forward / ckl_backward take a repeated id literally (its
 * log-probs' renormalised p are summed at that token).  A caller whose policy
 * is to refuse repeats runs this check first and treats a row >= 0 as
 * CKL_ERR_DUP_INDEX.
 *   topk_idx        [T, K] int32 device, row-major
 *   first_dup_row   [1]    int32 device out: the smallest row holding some id
 *                                more than once, or -1 when every row's ids
 *                                are distinct
 * Requires 1 <= K <= 2048.  Needs no workspace; one small kernel enqueued on
 * `stream` (the result is ready when the stream reaches it).  Returns
 * CKL_ERR_INVALID_ARG for a null or misaligned pointer or a bad size,
 * CKL_ERR_UNSUPPORTED for K above 2048.
 */
CKL_API int ckl_find_duplicate_ids(const int32_t* topk_idx, int64_t T, int32_t K,
                                   int32_t* first_dup_row, void* stream);

/* Static, human-readable text for a status code. */
CKL_API const char* ckl_status_string(int32_t status);

/* Library version: major * 10000 + minor * 100 + patch. */
CKL_API int32_t ckl_version(void);

/*
 * Forward without a caller-supplied workspace.
 *
 * The paper has no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory: a plugin or extension whose host
 * runtime owns every device allocation and hands the plugin only its input
 * and output pointers, or code on a latency-critical path where a device
 * allocation (which may synchronise the device) is not allowed.  Such a
 * caller cannot provide the workspace that ckl_forward needs.
 *
 * Same inputs and outputs as ckl_forward (there is no `chunk`: the forward
 * never holds per-chunk logits).  The scratch lives in one library-owned
 * static device buffer of CKL_STATIC_SCRATCH_BYTES, present on every GPU
 * that loads the library until the process exits.  A problem fits when
 *   256 + r(8 K T) + r(4 T) + r(1024 T) + r(8 ceil(T / 256))
 *       <= CKL_STATIC_SCRATCH_BYTES,   r(x) = x rounded up to a multiple of 256
 * (the sorted teacher pairs, sum p log p, the vocabulary-split partials and
 * the loss's block sums), whatever the GPU: T <= 18 355 at K = 100.  Larger
 * problems return CKL_ERR_WORKSPACE before anything is enqueued, and before
 * any CUDA call.  Nothing is allocated: no cudaMalloc, no cudaFree.  The
 * results are those of ckl_forward on the same inputs (the same launches).
 *
 * On each device, the first call looks up the buffer's device address
 * (cudaGetSymbolAddress) with that device current, and keeps it with the
 * CUDA context it was looked up in; a call in another context of that device
 * (after cudaDeviceReset) looks it up again.  Make the first call on a
 * device before any stream capture begins.  Every call on a device shares
 * the one buffer, which keeps the previous call's contents (the call clears
 * what must start at zero): calls that overlap on the GPU -- on different
 * streams, or from different host threads -- race and give wrong results.
 *
 *   device_status  [1] int32, device memory, may be NULL: receives the
 *                  device status word of this call (CKL_DEV bits: 1 = bad
 *                  teacher id, 2 = bad log-prob, 4 = timed-out wait; 0 = ok)
 */
#define CKL_STATIC_SCRATCH_BYTES (32u << 20)
CKL_API int ckl_forward_static_scratch(const uint16_t* H, const uint16_t* W,
                                       const int32_t* topk_idx, const float* topk_logp,
                                       const uint8_t* mask, int64_t T, int64_t d, int64_t V,
                                       int32_t K, float* loss, float* lse, int32_t* device_status,
                                       void* stream);

#ifdef __cplusplus
}
#endif

#endif /* CKL_H_ */
