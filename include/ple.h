/*
 * ple.h -- C ABI of libple, a B200 (sm_100a) implementation of the hashed
 * n-gram ("PLE" / Engram) embedding lookup of Qwen3.8-Flash-Next.
 *
 * The operations follow the NeMo AutoModel API page
 * "nemo_automodel.components.models.qwen3_8_flash_next.engram":
 *   - class Qwen3_8_FlashNextNGramEmbedding (docstring and parameters):
 *     heads grouped by n-gram order, context reset after EOS, signed int64
 *     wrapping hash, positive remainder per head prime, global head offsets;
 *   - _shift_right_after_eos / _hash_input_ids: context never crosses an EOS
 *     or a packed-segment boundary; rows of shape [batch, seq, ngram_heads];
 *   - _lookup_ngram_ids / forward: gather of the rows, heads concatenated;
 *   - Qwen3_8_FlashNextOwnerShardedEmbedding with process_group=None: one
 *     local table holding every global row, no collectives; its backward is
 *     the embedding's row-wise gradient accumulation.
 *
 * The page leaves the combine unprinted.  This library defines, for token t
 * of a packed sequence and order m = 2..ngram_size,
 *     ctx_0 = tok[t];  ctx_k = tok[t-k] if position t-k lies in t's packed
 *     sequence and no EOS token sits in positions [t-k, t-1], else 0;
 *     h_m = sum_{k<m} ctx_k * mults[k]            (int64, wrapping);
 *     row[t, j] = offsets[j] + ((h_m % primes[j]) + primes[j]) % primes[j]
 * for head j of order m = 2 + j / heads_per_ngram.  Packed sequences are
 * given by cu_seqlens (int32 [num_seqs + 1], cu_seqlens[0] = 0,
 * cu_seqlens[num_seqs] = num_tokens, non-decreasing); a batch of B padded
 * rows of length S is cu_seqlens = {0, S, 2S, ...}.
 *
 * Conventions for every entry point:
 *   - every tensor pointer is DEVICE memory owned by the caller; the library
 *     never allocates on a call path (the grad scatter takes a caller
 *     workspace); a plan owns only its host copy of the small constants;
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream); calls are asynchronous on it; only ple_status synchronises;
 *   - synchronous errors (bad arguments, alignment, workspace size, launch
 *     failure) are returned; nothing is launched when one is returned;
 *   - asynchronous errors found by kernels (a row id outside the table,
 *     malformed cu_seqlens, a bounded wait that ran out) never trap: the
 *     kernel zeroes or skips the affected output, sets a bit in the status
 *     word of the call's plan (on the device it runs on) and carries on;
 *     ple_status reports and clears that word.
 *   - layouts are dense row-major; int64 rows; tables [num_rows, head_dim].
 */
#ifndef PLE_H_
#define PLE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PLE_OK = 0,
  PLE_ERR_INVALID_ARG = 1,   /* null pointer, bad size, bad constants */
  PLE_ERR_UNSUPPORTED = 2,   /* a limit of this library (see each entry) */
  PLE_ERR_ALIGNMENT = 3,     /* pointer or row size not 16-byte aligned */
  PLE_ERR_WORKSPACE = 4,     /* workspace missing or smaller than required */
  PLE_ERR_CUDA = 5,          /* CUDA runtime error; see ple_last_cuda_error */
  PLE_ERR_BAD_ROW = 6,       /* async: a row id outside [0, num_rows) */
  PLE_ERR_BAD_SEQLENS = 7,   /* async: cu_seqlens not 0..num_tokens, or decreasing */
  PLE_ERR_TIMEOUT = 8        /* async: a bounded wait between the blocks of a kernel ran out */
} ple_status_t;

/* Element types.  PLE_F8E4M3 is a table type only: OCP FP8 E4M3 codes
 * (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; no infinities,
 * S.1111.111 is NaN): the official checkpoint's weights are FP8 ("Feat/qwen38
 * flash next" pull request, Summary), and no scale format is given there, so
 * the codes are widened unscaled.  A lookup of such a table
 * writes bf16: every finite E4M3 value is exactly a bf16 value, so the
 * widening is exact; a NaN code gives the quiet bf16 NaN with the code's
 * sign (0x7FC0 or 0xFFC0). */
typedef enum { PLE_F32 = 0, PLE_BF16 = 1, PLE_F8E4M3 = 2 } ple_dtype_t;

/* Hash and table description (constructor parameters of
 * Qwen3_8_FlashNextNGramEmbedding and Qwen3_8_FlashNextEngramTableConfig). */
typedef struct {
  int32_t ngram_size;       /* largest order incl. the current token; 2..8 */
  int32_t heads_per_ngram;  /* heads per order; H = (ngram_size-1)*heads_per_ngram <= 64 */
  int64_t eos_id;           /* raw token id after which context resets */
  const int64_t* mults;     /* HOST [ngram_size] signed multipliers */
  const int64_t* primes;    /* HOST [H] per-head modulus, 2 <= p <= 2^62 */
  const int64_t* offsets;   /* HOST [H] first global row of each head */
  int64_t num_rows;         /* table rows; every [offset, offset+prime) inside, disjoint */
  int32_t head_dim;         /* values per row, D */
  ple_dtype_t table_dtype;  /* element type of the table; lookup output is the same
                               type, except bf16 for a PLE_F8E4M3 table */
} ple_params_t;

typedef struct ple_plan ple_plan_t;

/* Validate the parameters and precompute the per-head remainder constants.
 * Host only: touches no GPU.  Errors: PLE_ERR_INVALID_ARG (null pointers,
 * ngram_size outside 2..8, heads_per_ngram < 1, a prime < 2 or > 2^62, a
 * negative offset, a head range outside [0, num_rows) or overlapping
 * another), PLE_ERR_UNSUPPORTED (H > 64, or 4095 plans already alive: each
 * holds one async status word), PLE_ERR_ALIGNMENT (head_dim * element size
 * not a multiple of 16 bytes).  On success *out owns a plan that
 * ple_plan_destroy frees; destroy a plan only once its calls have completed
 * (its status word goes to the next plan created). */
ple_status_t ple_plan_create(const ple_params_t* params, ple_plan_t** out);
void ple_plan_destroy(ple_plan_t* plan);
int32_t ple_plan_num_heads(const ple_plan_t* plan);

/* Rows of every (token, head): rows[t*H + j], int64 [num_tokens, H]
 * (_hash_input_ids).  tokens: int64 [num_tokens]; cu_seqlens: int32
 * [num_seqs + 1].  num_tokens == 0 is a no-op.  Errors: PLE_ERR_INVALID_ARG
 * (null pointer, negative size, num_seqs < 1 with num_tokens > 0),
 * PLE_ERR_ALIGNMENT (tokens or rows not 8-byte aligned), PLE_ERR_CUDA.
 * Async: PLE_ERR_BAD_SEQLENS (rows are still written, each token using the
 * sequence a binary search of the given array assigns it). */
ple_status_t ple_hash(const ple_plan_t* plan, const int64_t* tokens, int64_t num_tokens,
                      const int32_t* cu_seqlens, int32_t num_seqs, int64_t* rows, void* stream);

/* Hash fused with the gather (forward of Qwen3_8_FlashNextNGramEmbedding):
 * out[t, j, :] = table[row[t, j], :], out [num_tokens, H, head_dim] in the
 * table dtype, bf16 for an E4M3 table (= [tokens, H * head_dim] with heads
 * concatenated).  The copy (and the E4M3 widening) is exact.  rows_out, if not NULL, receives the int64 [num_tokens, H] rows
 * (to feed ple_grad_scatter).  table and out must be 16-byte aligned.
 * Errors as ple_hash. */
ple_status_t ple_lookup(const ple_plan_t* plan, const int64_t* tokens, int64_t num_tokens,
                        const int32_t* cu_seqlens, int32_t num_seqs, const void* table, void* out,
                        int64_t* rows_out, void* stream);

/* Global-slice lookup (_forward_global_slice of Qwen3_8_FlashNextNGramEmbedding):
 * the packed tokens are num_tokens / row_len rows of row_len tokens (a
 * replicated [batch, global_sequence] batch); every row is hashed with its
 * complete context (so a shard keeps the tokens before it and the EOS resets
 * at its boundary), and only positions [start, end) of each row are looked
 * up: out [B, end - start, H, head_dim], rows_out (nullable) [B, end - start, H].
 * cu_seqlens describes the packed segments of the whole stream (they must not
 * cross row boundaries for the rows to be independent).  Errors as
 * ple_lookup, plus PLE_ERR_INVALID_ARG unless row_len >= 1 divides
 * num_tokens and 0 <= start <= end <= row_len.  An empty slice is a no-op. */
ple_status_t ple_lookup_slice(const ple_plan_t* plan, const int64_t* tokens, int64_t num_tokens,
                              const int32_t* cu_seqlens, int32_t num_seqs, int64_t row_len, int64_t start,
                              int64_t end, const void* table, void* out, int64_t* rows_out, void* stream);

/* Gather precomputed rows (_lookup_ngram_ids): out[i, :] = table[rows[i], :]
 * for i < num_hits, out in the lookup's output type (bf16 for an E4M3
 * table).  A row outside [0, num_rows) yields a zero output row and the
 * async PLE_ERR_BAD_ROW.  table and out 16-byte aligned. */
ple_status_t ple_gather(const ple_plan_t* plan, const int64_t* rows, int64_t num_hits, const void* table,
                        void* out, void* stream);

/* Workspace bytes ple_grad_scatter needs for num_hits hits (0 for 0). */
size_t ple_grad_scatter_workspace_bytes(const ple_plan_t* plan, int64_t num_hits);

/* Deterministic table gradient (the embedding's backward):
 *   table_grad[r, :] = table_grad[r, :] + S_r   for every row r hit,
 * where S_r sums grad_out[i, :] (widened to fp32) over the hits i with
 * rows[i] == r in this fixed order: hits in ascending i, cut into chunks of
 * 32 consecutive hits; each chunk summed left to right from its first
 * element; the chunk sums summed left to right from the first; one final
 * add into table_grad.  The result is bit-identical run to run.
 * rows int64 [num_hits]; grad_out [num_hits, head_dim] of grad_dtype;
 * table_grad fp32 [num_rows, head_dim], accumulated into (the caller zeroes
 * it for a fresh gradient).  Every add is the IEEE fp32 add, subnormals
 * included (the device's fp32 reductions flush subnormals, so sums below
 * 2^-100 in magnitude are added by the row's owner with a load and a store):
 * nothing else may write table_grad while the call runs (two calls that
 * overlap on the GPU must not share a table_grad).  Hits whose row is
 * outside [0, num_rows) are dropped and raise the async PLE_ERR_BAD_ROW.  table_grad and grad_out
 * 16-byte aligned; workspace 256-byte aligned.  Errors: PLE_ERR_WORKSPACE,
 * PLE_ERR_UNSUPPORTED (head_dim > 256, num_rows >= 2^32 - 1 or num_hits >= 2^31),
 * PLE_ERR_INVALID_ARG, PLE_ERR_ALIGNMENT, PLE_ERR_CUDA. */
ple_status_t ple_grad_scatter(const ple_plan_t* plan, const int64_t* rows, int64_t num_hits,
                              const void* grad_out, ple_dtype_t grad_dtype, float* table_grad,
                              void* workspace, size_t workspace_bytes, void* stream);

/* ple_grad_scatter in two halves, for callers that want the row sort out of
 * the backward's critical path.  The sort depends only on the rows, not on
 * grad_out, so ple_grad_prepare can run as soon as the rows exist (for
 * instance on a second stream beside the forward gather, hashing the tokens
 * with ple_hash), and ple_grad_apply later folds grad_out in the prepared
 * order.  Together they compute exactly ple_grad_scatter (same order, same
 * bits).  The workspace (ple_grad_scatter_workspace_bytes for num_hits)
 * carries the prepared state: leave it untouched between the two calls, pass
 * the same plan and num_hits, and use one prepare for one apply (the apply
 * consumes counters the prepare cleared).  Errors as ple_grad_scatter, each
 * call checking its own arguments. */
ple_status_t ple_grad_prepare(const ple_plan_t* plan, const int64_t* rows, int64_t num_hits, void* workspace,
                              size_t workspace_bytes, void* stream);
ple_status_t ple_grad_apply(const ple_plan_t* plan, int64_t num_hits, const void* grad_out, ple_dtype_t grad_dtype,
                            float* table_grad, void* workspace, size_t workspace_bytes, void* stream);

/* Same sums by fp32 atomic adds, one per hit and column: no workspace and
 * no fixed order (results can differ in the last bits run to run).  A speed
 * reference for the deterministic path; same argument rules. */
ple_status_t ple_grad_scatter_atomic(const ple_plan_t* plan, const int64_t* rows, int64_t num_hits,
                                     const void* grad_out, ple_dtype_t grad_dtype, float* table_grad,
                                     void* stream);

/* The same deterministic gradient as ple_grad_scatter, for callers that
 * cannot provide a workspace: serving processes whose device memory is
 * reserved up front and may not grow while requests run, plugin hosts that
 * forbid calls to the CUDA allocator, or hot loops where cudaMalloc could
 * synchronise the device.  No counterpart on the source pages: it is a service
 * of this library.  Nothing is allocated by anyone: the kernels use a fixed
 * scratch area of ple_grad_scatter_noalloc_scratch_bytes() (32 MiB) that the
 * library holds in the device memory of every GPU that loads it, until the
 * process exits.  Sizes whose workspace (ple_grad_scatter_workspace_bytes)
 * exceeds that area are rejected with PLE_ERR_WORKSPACE before anything is
 * launched; use ple_grad_scatter with a caller workspace for them.  The first
 * call on a device (and the first after the device's context changed, e.g.
 * after cudaDeviceReset) looks up the scratch area's device address (make
 * that first call before any stream capture).  All calls share the one area, so
 * calls that overlap on the GPU (other streams, other host threads) race and
 * must be serialised by the caller; each call clears what must start at zero.
 * Other arguments, errors and results as ple_grad_scatter. */
ple_status_t ple_grad_scatter_noalloc(const ple_plan_t* plan, const int64_t* rows, int64_t num_hits,
                                      const void* grad_out, ple_dtype_t grad_dtype, float* table_grad,
                                      void* stream);

/* Bytes of the fixed scratch area ple_grad_scatter_noalloc works in. */
size_t ple_grad_scatter_noalloc_scratch_bytes(void);

/* ---- Host-memory tier ----------------------------------------------------------
 * The table stays in pinned host memory and the rows a batch touches are
 * brought to the GPU ahead of its lookup: the CPU offload of the n-gram table
 * with asynchronous prefetch ("add native Qwen3.8 Flash Next" pull request,
 * Summary and Overview: ngram_embedding_cpu_offload).
 *
 * ple_prefetch hashes the batch exactly as ple_hash, then, for the distinct
 * rows of its num_tokens * H hits in ascending order:
 *   uniq_rows[u] = the u-th distinct row (-1 for a row outside the table),
 *   cache[u, :] = host_table[uniq_rows[u], :] (raw copy in the table dtype),
 *   slots[t*H + j] = u for every hit of that row, *num_unique = the count.
 * Every distinct row is read once over the host link, with 16-byte loads
 * from the mapped host memory.  host_table: [num_rows, head_dim] in host
 * memory the device can read (pinned: cudaHostAlloc / cudaHostRegister on a
 * system with unified addressing; device or managed memory also works);
 * pageable memory is rejected with PLE_ERR_INVALID_ARG.  cache [cache_rows,
 * head_dim] table dtype and uniq_rows int64 [cache_rows] on the device,
 * cache_rows >= num_tokens * H (room for every hit); slots int64
 * [num_tokens, H]; num_unique: one int64 in device memory.  host_table and
 * cache 16-byte aligned, workspace (ple_prefetch_workspace_bytes) 256-byte
 * aligned.  Run it on a side stream for the next batch to overlap the copy
 * with the current batch's compute.  num_tokens == 0 writes *num_unique = 0.
 * Errors as ple_hash, plus PLE_ERR_WORKSPACE, PLE_ERR_ALIGNMENT,
 * PLE_ERR_UNSUPPORTED (num_tokens * H >= 2^31). */
size_t ple_prefetch_workspace_bytes(const ple_plan_t* plan, int64_t num_tokens);
ple_status_t ple_prefetch(const ple_plan_t* plan, const int64_t* tokens, int64_t num_tokens, const int32_t* cu_seqlens,
                          int32_t num_seqs, const void* host_table, void* cache, int64_t cache_rows, int64_t* slots,
                          int64_t* uniq_rows, int64_t* num_unique, void* workspace, size_t workspace_bytes,
                          void* stream);

/* The lookup of a prefetched batch: out[i, :] = cache[slots[i], :] (bf16 for
 * an E4M3 table), as ple_gather with the cache for the table; a slot outside
 * [0, cache_rows) yields a zero row and the async PLE_ERR_BAD_ROW. */
ple_status_t ple_gather_cache(const ple_plan_t* plan, const int64_t* slots, int64_t num_hits, const void* cache,
                              int64_t cache_rows, void* out, void* stream);

/* The backward of a prefetched batch: the deterministic gradient of
 * ple_grad_scatter with the slots for rows, summed into cache_grad fp32
 * [cache_rows, head_dim] (accumulated into); row u of cache_grad is the
 * gradient of table row uniq_rows[u], to be applied on the host.  Same
 * summation order, workspace (ple_grad_scatter_workspace_bytes) and errors as
 * ple_grad_scatter, with cache_rows as the row bound. */
ple_status_t ple_grad_scatter_cache(const ple_plan_t* plan, const int64_t* slots, int64_t num_hits, const void* grad_out,
                                    ple_dtype_t grad_dtype, float* cache_grad, int64_t cache_rows, void* workspace,
                                    size_t workspace_bytes, void* stream);

/* ---- The PLE layer's short convolution --------------------------------------
 * Segment-aware causal dilated depthwise convolution over packed tokens
 * (Qwen3_8_FlashNextPLELayer._causal_short_conv and _segmented_conv, NeMo
 * AutoModel engram API page; conv_kernel_size K, default 4, and
 * short_conv_dilation = ngram_size): every packed segment is convolved as if
 * it started a fresh row, with (K-1)*dilation zeros of history ahead of it:
 *   y[t, c] = bias[c] + sum_{k=0}^{K-1} w[c, k] * x[t - dilation*(K-1-k), c],
 * a tap before the first position of t's segment reading zero.
 * x, y: [num_tokens, channels] row-major, dtype PLE_BF16 or PLE_F32 (both the
 * same), 16-byte aligned, channels * element size a multiple of 16 bytes;
 * weight fp32 [channels, K] (the depthwise Conv1d weight [C, 1, K]);
 * bias fp32 [channels] or NULL.  Arithmetic in fp32 (one fused multiply-add
 * per tap, taps in ascending k after the bias), rounded to the output type.
 * cu_seqlens int32 [num_seqs + 1] as for ple_lookup.  num_tokens == 0 is a
 * no-op.  Errors: PLE_ERR_INVALID_ARG (null pointer, K < 1, dilation < 1,
 * other dtype), PLE_ERR_UNSUPPORTED (K > 8, channels > 2^24), PLE_ERR_ALIGNMENT,
 * PLE_ERR_CUDA; async PLE_ERR_BAD_SEQLENS (outputs still written, every
 * access inside the tensors). */
ple_status_t ple_conv_forward(const void* x, ple_dtype_t dtype, int64_t num_tokens, int64_t channels,
                              const int32_t* cu_seqlens, int32_t num_seqs, const float* weight, int32_t kernel_size,
                              int32_t dilation, const float* bias, void* y, void* stream);

/* Workspace bytes ple_conv_backward needs for dweight / dbias (0 for 0 tokens). */
size_t ple_conv_backward_workspace_bytes(int64_t num_tokens, int64_t channels, int32_t kernel_size);

/* Gradients of ple_conv_forward for the output gradient dy (same layout and
 * dtype as x):
 *   dx[t, c] = sum_k w[c, k] * dy[t + dilation*(K-1-k), c] over taps that stay
 *              inside t's segment (overwritten; NULL to skip);
 *   dweight[c, k] += sum_t dy[t, c] * x[t - dilation*(K-1-k), c] (taps inside
 *              the segment), dbias[c] += sum_t dy[t, c] (fp32, accumulated
 *              into; NULL to skip).
 * The sums over tokens have a fixed order, so results are bit-identical run
 * to run: the tokens are cut into consecutive chunks (256 tokens, or 512
 * when ceil(num_tokens / 512) * ceil(channels / 512) >= 592; more when that
 * would exceed 1024 chunks); each chunk's sum starts from +0 and adds its tokens
 * residue class by residue class modulo the dilation (the class of the
 * chunk's first token first), each class in ascending token order (fused
 * multiply-add for dweight); the chunk sums are added in chunk order
 * starting from the first; one final add into dweight / dbias.  dx and the
 * parameter gradients come out with the same bits whether they are asked
 * for together (one sweep) or separately.
 * workspace (16-byte aligned, ple_conv_backward_workspace_bytes) is needed
 * only for dweight or dbias.  Errors as ple_conv_forward, plus
 * PLE_ERR_WORKSPACE. */
ple_status_t ple_conv_backward(const void* dy, const void* x, ple_dtype_t dtype, int64_t num_tokens, int64_t channels,
                               const int32_t* cu_seqlens, int32_t num_seqs, const float* weight, int32_t kernel_size,
                               int32_t dilation, void* dx, float* dweight, float* dbias, void* workspace,
                               size_t workspace_bytes, void* stream);

/* Async status of the calls made with `plan` on the current device: runs
 * one small kernel on `stream` that atomically takes (reads and zeroes) the
 * plan's status word, waits for it, and returns PLE_OK if no kernel of the
 * plan flagged anything since the last take, otherwise the lowest-numbered
 * flagged error.  Taken in stream order: flags of kernels queued on
 * `stream` before the call are included, and a flag that a kernel on
 * another stream raises while the take runs is either in this result or
 * left for the next call, never lost (this replaces the pages' device
 * asserts and symmetric validation).  Each plan has a word of its own (at
 * most 4095 plans live at once; ple_plan_create returns
 * PLE_ERR_UNSUPPORTED beyond), so one plan's ple_status leaves the others'
 * flags alone.  plan == NULL takes every word of the device at once: the
 * flags of all plans and of the calls that take no plan (the short
 * convolution).  Synchronises `stream` (the only call that does); not for
 * use inside a stream capture.  A plan's word is cleared, in stream order,
 * by the plan's first call on each device (a destroyed plan's unread flags
 * are not inherited); a plan about to be used from several host threads on
 * several streams should make one call on each device first, so that this
 * clear cannot land after another stream's kernel has raised a flag.
 * Device addresses are looked up again after the current context changes
 * (cudaDeviceReset). */
ple_status_t ple_status(const ple_plan_t* plan, void* stream);

/* Text for a status code (static storage). */
const char* ple_strerror(ple_status_t status);

/* cudaError_t of the last PLE_ERR_CUDA returned on the calling thread. */
int ple_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* PLE_H_ */
