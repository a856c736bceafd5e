/*
 * ckl.h -- fused, chunked top-K forward-KL distillation loss (C ABI).
 *
 * The operation is the "Full Chunked KL" loss of "Chunked KL loss, running
 * Knowledge Distillation locally in less <6GB VRAM" (README: the three methods
 * and the formula section). A student's last hidden states H (T x d) and LM-head
 * weight W (V x d) give logits z = H W^T; a teacher is cached as its top-K
 * logits per position (the author's forum post: the cache keeps the 100 largest
 * teacher logits of each position). Per token
 *
 *     l_t = sum_{v in S} P_v log P_v - sum_{v in S} P_v z_v + M * logsumexp(z)
 *
 * with S the cached ids, p = softmax of the cached logits, P_v the probability of
 * id v (slots that repeat an id add up), M = sum p (1, or 0 when every cached
 * logit is -inf). Only logsumexp spans the vocabulary. The loss is the mean of
 * l_t over unmasked tokens (N = number of tokens with mask != 0; loss and
 * gradients are 0 when N = 0). Gradients use the closed form
 * dl_t/dz_v = M softmax(z)_v - P_v:
 *     dH = (mask/N) G W,    dW = sum_t (mask_t/N) G_t^T H_t.
 * The T x V logit tensor is never stored: the logits are produced tile by tile
 * on the tensor cores, chunk tokens at a time, and reduced to the log-normaliser
 * in the tile's epilogue (the README's fused variant, which folds the output
 * projection into the loss and never keeps the logits of the whole sequence).
 * For the analytic gradient the default keeps exp(z - r) of the current chunk in
 * the chunk-bounded gradient buffer, r a per-row reference logit, and applies the
 * one factor per row that turns it into the gradient where dH and dW are formed;
 * the README's design, which forms the chunk's logits again in the backward pass,
 * is ckl_set_recompute(h, 1).
 *
 * Conventions for every entry point:
 *  - All matrices are dense, row-major, contiguous. H is T x d, W is V x d,
 *    topk_idx and topk_logit are T x K, mask is T bytes, dH is T x d, dW is V x d.
 *  - "device" pointers are CUDA device memory of the handle's device; the caller
 *    owns every buffer. The library allocates no device memory during a call
 *    (ckl_fwd_bwd_from_host creates a stream and events on its first use).
 *  - H, W, dH have the handle's dtype (CKL_F32: float; CKL_BF16: bfloat16 bits).
 *    dW, topk_logit, loss and the per-token outputs are float32; topk_idx is int32.
 *  - H, W, dH, dW, topk_idx, topk_logit must be 16-byte aligned; the workspace
 *    256-byte aligned. mask has no alignment requirement.
 *  - stream is a cudaStream_t (NULL = legacy default stream); all work is
 *    enqueued on it in order (ckl_fwd_bwd_from_host adds its copies on a stream
 *    of the handle, ordered after the work already on `stream`). A handle must
 *    not be used by two calls at once.
 *  - Errors found on the host (bad sizes, null or misaligned pointers, a small
 *    workspace) return before anything is enqueued. Errors found on the device
 *    (a teacher id outside [0, V), a pipeline wait that exceeded its bound) set a
 *    status word in the handle; the kernels skip the offending access and never
 *    trap. The status is returned by the synchronising calls (loss_host != NULL,
 *    ckl_sync_status). The outputs of a call that reports an error are undefined.
 */
#ifndef CKL_H
#define CKL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct ckl_ctx* ckl_handle;

typedef enum {
  CKL_OK = 0,
  CKL_ERR_INVALID_ARG = 1,  /* null pointer, negative or inconsistent size */
  CKL_ERR_UNSUPPORTED = 2,  /* a size the kernels do not handle (d % 8 != 0, K > 1024, ...) */
  CKL_ERR_WORKSPACE = 3,    /* workspace null, misaligned or smaller than ckl_workspace_bytes */
  CKL_ERR_INDEX_RANGE = 4,  /* device: a topk_idx entry outside [0, V) */
  CKL_ERR_CUDA = 5,         /* a CUDA runtime call failed (no device, launch failure, ...) */
  CKL_ERR_TIMEOUT = 6,      /* device: a pipeline wait exceeded its bound; the kernel gave up */
  CKL_ERR_ALIGNMENT = 7,    /* a pointer is not aligned as stated above */
  CKL_ERR_INTERNAL = 8,     /* device: an internal consistency check failed */
  CKL_ERR_COLLECTIVE = 9    /* a caller-supplied collective returned nonzero */
} ckl_status;

typedef enum { CKL_F32 = 0, CKL_BF16 = 1 } ckl_dtype;

/* Create a handle for one LM head shape on one device.
 * device: CUDA ordinal. dtype: type of H, W, dH. V, d, K: vocabulary size, hidden
 * size, cached entries per token (1 <= K <= 1024, d % 8 == 0, V >= 1).
 * max_chunk: the largest chunk any call will use (>= 1).
 * On success *out holds the handle (release with ckl_destroy). The handle owns
 * a few bytes of device memory (status word, counters) and a pinned host word. */
ckl_status ckl_create(ckl_handle* out, int device, ckl_dtype dtype, int64_t V, int64_t d,
                      int64_t K, int64_t max_chunk);

/* Release a handle and what it owns. NULL is accepted. */
ckl_status ckl_destroy(ckl_handle h);

/* Short English description of a status code (static storage). */
const char* ckl_status_str(ckl_status s);

/* Bytes of device workspace a call with T tokens and this chunk needs. The size
 * is O(T) for per-token values plus O(chunk * V) for the gradient tile of one
 * chunk, never O(T * V). */
ckl_status ckl_workspace_bytes(ckl_handle h, int64_t T, int64_t chunk, size_t* bytes);

/* Loss, dH and dW in one call (forward and backward fused).
 * Inputs (device): H, W, topk_idx, topk_logit; mask may be NULL (all tokens count).
 * T >= 0 tokens, processed `chunk` tokens at a time (1 <= chunk <= max_chunk).
 * Outputs (device): loss (1 float), dH (T x d, overwritten), dW (V x d float32,
 * overwritten, not accumulated). token_lse and token_loss (T floats each, device)
 * are optional: logsumexp(z_t) and l_t per token (l_t is reported for masked
 * tokens too; they are left out of the mean).
 * loss_host: if non-NULL, the call waits for the stream, stores the loss there
 * and returns the device-detected status; otherwise the call only enqueues work
 * and returns CKL_OK once it is enqueued. */
ckl_status ckl_fwd_bwd(ckl_handle h, const void* H, const void* W, const int32_t* topk_idx,
                       const float* topk_logit, const uint8_t* mask, int64_t T, int64_t chunk,
                       float* loss, void* dH, float* dW, float* token_lse, float* token_loss,
                       void* workspace, size_t workspace_bytes, void* stream, float* loss_host);

/* Forward only: the loss (and optional per-token values) without gradients, for
 * evaluation. Same arguments and rules as ckl_fwd_bwd. */
ckl_status ckl_forward(ckl_handle h, const void* H, const void* W, const int32_t* topk_idx,
                       const float* topk_logit, const uint8_t* mask, int64_t T, int64_t chunk,
                       float* loss, float* token_lse, float* token_loss, void* workspace,
                       size_t workspace_bytes, void* stream, float* loss_host);

/* ckl_fwd_bwd with the per-step inputs in HOST memory: copies H_host, idx_host,
 * logit_host and mask_host (may be NULL) into the caller's device buffers H_dev,
 * idx_dev, logit_dev, mask_dev, runs the fused loss, copies the loss back to
 * *loss_host and waits. The copies run chunk by chunk (one cudaMemcpyAsync per
 * tensor per chunk, the mask first) on a stream the handle creates on first use,
 * after the work already enqueued on `stream`; chunk c's kernels wait for chunk
 * c's copies only, so the next chunk crosses the bus while this one computes.
 * Host buffers should be pinned for the copies to be asynchronous. W stays on the
 * device. Returns the device-detected status; on an error no copy is still
 * running when the call returns. */
ckl_status ckl_fwd_bwd_from_host(ckl_handle h, const void* H_host, const int32_t* idx_host,
                                 const float* logit_host, const uint8_t* mask_host, void* H_dev,
                                 int32_t* idx_dev, float* logit_dev, uint8_t* mask_dev,
                                 const void* W, int64_t T, int64_t chunk, float* loss, void* dH,
                                 float* dW, void* workspace, size_t workspace_bytes, void* stream,
                                 float* loss_host);

/* Forward-only loss that allocates nothing, for callers that may not call
 * cudaMalloc: code embedded in a runtime that owns all device memory through its
 * own arena or caching allocator, and latency-critical loops that cannot afford
 * the device-wide synchronisation of cudaMalloc / cudaFree. (The source pages
 * have no counterpart: this is a deployment variant of ckl_forward.)
 * No handle is involved, since ckl_create allocates. The forward workspace and
 * the device status word live in one file-scope device array of 32 MiB that
 * every GPU which loads this library keeps until the process exits. A call whose
 * T and chunk need more than that (32 MiB minus 256 bytes, as
 * ckl_workspace_bytes would size the forward pass) is rejected with
 * CKL_ERR_WORKSPACE before anything is enqueued. At V = 201088 and K = 100 a
 * 2048-token chunk needs about 21 MiB plus 8 bytes per token of T.
 * The first call on a device looks up the array's device address, the SM count
 * and the TMA descriptor encoder for that device (with the device current); make
 * that first call before any stream capture. Every call shares the array and
 * clears the status word it needs; calls that overlap on the GPU (different
 * streams or host threads) race on the array and must not be issued.
 * Arguments are those of ckl_create (device, dtype, V, d, K) followed by those
 * of ckl_forward without the workspace; chunk has no max_chunk bound other than
 * the scratch size. loss_host is required (NULL gives CKL_ERR_INVALID_ARG): with
 * no handle there is no later ckl_sync_status, and the next call clears the
 * shared status word, so every call waits for its stream, stores the loss in
 * *loss_host (pageable memory is fine) and returns the device-detected status
 * (CKL_ERR_INDEX_RANGE for a teacher id outside [0, V), ...).
 * The cached device address of the array stays valid for the life of the
 * process's CUDA context on that device: after cudaDeviceReset on a device this
 * entry point must not be called on it again in the same process. */
ckl_status ckl_forward_static(int device, ckl_dtype dtype, int64_t V, int64_t d, int64_t K,
                              const void* H, const void* W, const int32_t* topk_idx,
                              const float* topk_logit, const uint8_t* mask, int64_t T,
                              int64_t chunk, float* loss, float* token_lse, float* token_loss,
                              void* stream, float* loss_host);

/* Teacher top-K cache builder: the offline half of the method ("Efficient
 * Knowledge Distillation for LLMs: Offline Top-K Logits and a Fused Chunked KL
 * Loss", abstract; the author's forum post: the teacher runs once and each
 * position keeps its 100 largest logits). For a handle made with the TEACHER's
 * shape (V, d = teacher hidden size, K = cache width; bf16 only, K <= V):
 * H (T x d, device) holds the teacher's last hidden states and W (V x d,
 * device) its LM head. Writes, per token, the K largest logits of H_t W^T
 * (fp32, from a bf16 x bf16 -> fp32 contraction) to topk_logit (T x K) and their
 * ids to topk_idx (T x K), in descending order of logit; equal logits in
 * ascending id order. These are exactly the topk_idx / topk_logit inputs of
 * ckl_fwd_bwd. Processed `chunk` tokens at a time (1 <= chunk <= max_chunk) with
 * two tensor-core passes over the logits (best per 256-column tile, then the
 * candidates at least as good as the K-th best tile best) and a per-token
 * selection; the workspace is ckl_topk_workspace_bytes bytes (about
 * chunk * min(V, 256 K) * 8 bytes). wait != 0: wait for the stream and return
 * the device-detected status. */
ckl_status ckl_topk_workspace_bytes(ckl_handle h, int64_t T, int64_t chunk, size_t* bytes);
ckl_status ckl_topk_cache(ckl_handle h, const void* H, const void* W, int64_t T, int64_t chunk,
                          int32_t* topk_idx, float* topk_logit, void* workspace,
                          size_t workspace_bytes, void* stream, int wait);

/* ---- Vocabulary-parallel loss (tensor parallelism over the LM head) ----
 *
 * The benchmark on the page "Chunked KL loss, running Knowledge Distillation
 * locally in less <6GB VRAM" runs its losses tensor-parallel (options table,
 * `--tp`) without describing the split; this is the split of the LM head by
 * vocabulary rows. The ranks of a group hold the same tokens (H, ids, logits,
 * mask) and disjoint, contiguous row ranges of W: this rank holds rows
 * [v0, v0 + V) of the full V_total x d head, V being its handle's V. Per chunk,
 * each rank reduces its own logits to per-token (max, sum of exp, sum of p z at
 * the cached ids inside its rows); the group all-gathers those triples and every
 * rank merges them in rank order, so lse, the per-token losses and the loss are
 * the same on every rank, bit for bit. dH = sum over ranks of G_r W_r is summed
 * in fp32 by an all-reduce per chunk; dW_r = G_r^T H stays on its rank.
 * The library calls no collective library itself: the caller supplies the two
 * collectives (NCCL, torch.distributed, MPI, ...). Each must be ordered on the
 * `stream` it is given (enqueued there, or complete when it returns) and return
 * 0 on success. Every rank makes the same sequence of collective calls, one
 * all-gather per chunk and one all-reduce per chunk (T = 0: none). After a
 * kernel failure the remaining collectives are still made (the group stays
 * matched) and the call returns CKL_ERR_CUDA; after a collective returns
 * nonzero no further collective is called and the call returns
 * CKL_ERR_COLLECTIVE. Argument errors are returned before any collective.
 * bf16 handles only; world = 1 gives the result of ckl_fwd_bwd. */
typedef int (*ckl_all_gather_fn)(void* user, const float* send, float* recv, int64_t count,
                                 void* stream);  /* recv: world x count floats, rank-major */
typedef int (*ckl_all_reduce_sum_fn)(void* user, float* buf, int64_t count,
                                     void* stream);  /* in place, element-wise sum */
typedef struct {
  int32_t world;   /* ranks in the group (>= 1) */
  int32_t rank;    /* this rank (0 <= rank < world) */
  int64_t V_total; /* full vocabulary size: ids are checked against it */
  int64_t v0;      /* first vocabulary row held by this rank (v0 + V <= V_total) */
  ckl_all_gather_fn all_gather;
  ckl_all_reduce_sum_fn all_reduce_sum;
  void* user;      /* passed back to both functions */
} ckl_vocab_group;

/* Workspace of ckl_fwd_bwd_vocab_parallel: ckl_workspace_bytes plus
 * chunk * (16 (world + 1) + 4 d) bytes for the exchanged statistics and dH. */
ckl_status ckl_vp_workspace_bytes(ckl_handle h, int32_t world, int64_t T, int64_t chunk,
                                  size_t* bytes);
/* As ckl_fwd_bwd with W_shard (V x d, this rank's rows) and dW_shard (V x d
 * fp32); H, ids, logits, mask, loss, dH, token_lse and token_loss as there
 * (full-vocabulary values, identical on every rank). */
ckl_status ckl_fwd_bwd_vocab_parallel(ckl_handle h, const ckl_vocab_group* group, const void* H,
                                      const void* W_shard, const int32_t* topk_idx,
                                      const float* topk_logit, const uint8_t* mask, int64_t T,
                                      int64_t chunk, float* loss, void* dH, float* dW_shard,
                                      float* token_lse, float* token_loss, void* workspace,
                                      size_t workspace_bytes, void* stream, float* loss_host);

/* Loss only (no dH, dW), vocabulary split over ranks: one all-gather per chunk
 * and no all-reduce (all_reduce_sum may be NULL). Loss, token_lse and
 * token_loss as in ckl_fwd_bwd_vocab_parallel; the workspace of
 * ckl_vp_workspace_bytes is enough. */
ckl_status ckl_forward_vocab_parallel(ckl_handle h, const ckl_vocab_group* group, const void* H,
                                      const void* W_shard, const int32_t* topk_idx,
                                      const float* topk_logit, const uint8_t* mask, int64_t T,
                                      int64_t chunk, float* loss, float* token_lse,
                                      float* token_loss, void* workspace,
                                      size_t workspace_bytes, void* stream, float* loss_host);

/* Self-test of the device-side failure detection (the pages have no counterpart):
 * one thread waits, with the bounded wait every pipeline kernel uses, on a barrier
 * that nothing arrives at. The call waits for it and returns CKL_ERR_TIMEOUT when
 * the bound fired as designed (4e9 SM cycles: about 2 s at the maximum clock,
 * longer at lower clocks), with the cycles waited in *cycles (may be NULL); any
 * other status means the mechanism failed. The status word is cleared and the
 * handle stays usable. */
ckl_status ckl_selftest_wait_bound(ckl_handle h, void* stream, int64_t* cycles);

/* The top-K cache builder for a teacher whose LM head is split by vocabulary rows
 * over a group (ckl_vocab_group as above; this handle's V = the rank's rows, and
 * K <= V). Each rank builds the K best of its own rows per chunk; the group
 * all-gathers the (logit, global id) pairs (one all-gather per chunk, world x
 * chunk x K x 8 bytes; all_reduce_sum is not used and may be NULL) and every rank
 * selects the final K of the world * K candidates, so every rank gets the cache
 * ckl_topk_cache would give one rank holding all of W, bit for bit. Workspace:
 * ckl_topk_vp_workspace_bytes. Errors and matched collectives as in
 * ckl_fwd_bwd_vocab_parallel. */
ckl_status ckl_topk_vp_workspace_bytes(ckl_handle h, int32_t world, int64_t T, int64_t chunk,
                                       size_t* bytes);
ckl_status ckl_topk_cache_vocab_parallel(ckl_handle h, const ckl_vocab_group* group, const void* H,
                                         const void* W_shard, int64_t T, int64_t chunk,
                                         int32_t* topk_idx, float* topk_logit, void* workspace,
                                         size_t workspace_bytes, void* stream, int wait);

/* Wait for `stream` and return the device-detected status of the calls enqueued
 * on it since the last synchronising call (clears it). */
ckl_status ckl_sync_status(ckl_handle h, void* stream);

/* bf16 handles only: choose how the backward pass obtains exp(z - lse).
 * recompute = 1: the logits are formed a second time on the tensor cores from H
 * and W, as the README's fused variant does (executed work 8 T V d).
 * recompute = 0 (default): the forward contraction also writes exp(z - r) in bf16
 * into the chunk x V gradient buffer, r the student's logit at the token's best
 * cached teacher id (a tile whose largest logit lies more than 2^32 above r keeps
 * its own maximum, and its row is rescaled by a repair pass); the factor
 * (mask/N) M exp(r - lse) is applied per row in the dH reduction and to the hidden
 * states dW contracts with (a scaled copy the dH contraction writes; executed work
 * 6 T V d, no pass over the buffer). lse
 * and the loss are the same, bit for bit, in both modes; the gradients agree to
 * their bf16 rounding. Memory is the same in both modes. fp32 handles always
 * recompute. */
ckl_status ckl_set_recompute(ckl_handle h, int recompute);

/* Number of kernels the handle has launched since it was created. */
int64_t ckl_launch_count(ckl_handle h);

/* Per-kernel timing. When enabled, each kernel launch is bracketed by CUDA
 * events on the launching stream (a pool of `max_launches` event pairs is
 * created here; launches past that are not timed). Two kernels of the bf16
 * backward run behind a contraction as dependent launches and are timed inside
 * its range: the next chunk's teacher kernel inside "dh_gemm", the chunk's dH
 * split reduction inside "dw_gemm" (an event between the two launches would
 * serialise them). */
ckl_status ckl_profile_enable(ckl_handle h, int enable, int max_launches);

typedef struct {
  char name[32];      /* kernel name */
  int64_t launches;   /* timed launches */
  double total_ms;    /* sum of event-measured durations */
  double flops;       /* algorithmic FLOPs of those launches (tensor-core contractions) */
  double bytes;       /* algorithmic DRAM bytes of those launches (memory-bound kernels) */
} ckl_kernel_stat;

/* Wait for the recorded events, fold them into per-kernel totals and clear the
 * record. Fills up to max_stats entries; *n_stats receives the number of kernels. */
ckl_status ckl_profile_collect(ckl_handle h, ckl_kernel_stat* stats, int max_stats, int* n_stats);

#ifdef __cplusplus
}
#endif

#endif /* CKL_H */
