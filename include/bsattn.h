/*
 * bsattn.h -- C ABI of the B200 (sm_100a) block-sparse attention library.
 *
 * The library computes the attention forward pass
 *     O = softmax(scale * Q K^T + M) V
 * where M removes (a) the key blocks that a static 0/1 block mask zeroes out
 * ("块稀疏Attention实战", section 2.1: a zero block takes no part in QK,
 * softmax or PV; section 3.3: the tiling loop checks each block before loading
 * K) and (b) the key tiles that the BLASST rule skips ("BLASST: Dynamic
 * Blocked Attention Sparsity via Softmax Thresholding", section 3.1 and
 * Algorithm 1): inside the online softmax, key tiles of a query tile are
 * visited in ascending order, and a tile is skipped -- no exp, no row sum, no
 * P*V -- when, for every valid row of the query tile, the tile's row max is
 * below the running row max (taken over all earlier visited tiles, skipped or
 * not) plus ln(lambda).  The output is the exact softmax over the keys of the
 * executed tiles.
 *
 * Conventions shared by every entry point:
 *  - Tensors are dense and row-major.  Q is [B, Hq, N, d], K and V are
 *    [B, Hkv, N, d], O is [B, Hq, N, d], all bf16; LSE is [B, Hq, N] fp32
 *    (natural log of the softmax denominator of the scaled scores).
 *  - GQA ("Attention 的七十二变", section 5.3-5.4): query head h reads KV head
 *    h / (Hq / Hkv).
 *  - All pointers are device pointers unless stated otherwise.  The caller
 *    allocates and owns every buffer; no call allocates device memory.  One
 *    fixed reservation comes with the library itself: loading it places the
 *    32 MiB scratch array of bsattn_fwd_decode_noalloc on every device that
 *    uses the library, for the life of the process.  Between calls the
 *    library keeps only per-device caches (kernel attributes, the host-buffer
 *    prefill's streams and events, the scratch array's address).
 *  - Every call is asynchronous on `stream`.  The return value reports only
 *    host-side validation and launch errors; nothing is launched when it is
 *    not BSATTN_OK.  Errors found on the device (a pipeline wait that ran out
 *    of time, an index capacity overflow) are written to the optional device
 *    word `d_status`, which the caller sets to 0 beforehand; the library only
 *    ever writes a nonzero code there.
 *  - lambda = 0 turns the dynamic skip off; lambda must lie in [0, 1].
 */
#ifndef BSATTN_H_
#define BSATTN_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BSATTN_OK = 0,
  BSATTN_ERR_INVALID_ARG = -1,   /* null pointer, bad size or lambda outside [0, 1] */
  BSATTN_ERR_UNSUPPORTED = -2,   /* d or block not in {64, 128}, or no sm_100 device */
  BSATTN_ERR_ALIGNMENT = -3,     /* a tensor pointer is not 16-byte aligned */
  BSATTN_ERR_CAPACITY = -4,      /* index or workspace too small */
  BSATTN_ERR_CUDA = -5,          /* a CUDA runtime/driver call failed */
  BSATTN_ERR_DEVICE_TIMEOUT = -6 /* (device status only) a pipeline wait timed out */
} bsattn_status;

/* Human-readable name of a status code; never NULL. */
const char *bsattn_status_string(int status);

/* Library version as major * 10000 + minor * 100 + patch. */
int bsattn_version(void);

/*
 * bsattn_debug_set -- test hook, process-wide.  wait_limit_ns bounds every
 * pipeline wait inside the kernels (default 2 s); when one runs out the kernel
 * stops, drains its own copies, frees its tensor memory and reports
 * BSATTN_ERR_DEVICE_TIMEOUT through d_status.  inject_stall != 0 makes the
 * prefill kernels withhold their query tile from the tensor core, and the
 * backward kernels their resident tiles, so that the limit is reached on
 * purpose.  Returns BSATTN_ERR_INVALID_ARG for
 * wait_limit_ns <= 0.
 */
int bsattn_debug_set(long long wait_limit_ns, int inject_stall);

/*
 * bsattn_debug_exp2 -- test hook: d_y[i] = 2^d_x[i] for i < n through the
 * exponential that the prefill kernels run on the FMA and integer pipes for
 * part of a kept tile's columns (range reduction to floor(x) and a fraction,
 * a cubic for 2^fraction, the integer part added to the exponent field).
 * d_x and d_y are device buffers of n floats owned by the caller; the call is
 * asynchronous on `stream`.  Relative error below 1e-4 for x in [-126, 64);
 * exactly 0 for x <= -127 and x = -inf.  n < 0, n > 2^32 or a NULL buffer
 * with n > 0 give BSATTN_ERR_INVALID_ARG.
 */
int bsattn_debug_exp2(const float *d_x, float *d_y, int64_t n, cudaStream_t stream);

/*
 * bsattn_debug_trace -- debugging aid, process-wide, present only in a
 * library built with -DBSATTN_TRACE.  The shipped library has no trace
 * markers compiled into its kernels: there n = 0 returns BSATTN_OK (and sets
 * *host_view to NULL when given), n > 0 returns BSATTN_ERR_UNSUPPORTED and
 * allocates nothing.  In a trace build, n > 0 allocates n int32 of mapped,
 * pinned host memory (zeroed), returns its host address in *host_view and
 * makes the one-query-tile prefill kernel record progress there, readable while
 * a kernel is still running: slot 16 + CTA index holds the stage a CTA reached
 * (1 entered, 2 set up, 3 finished, 4 tensor memory freed; 13/14 the same
 * after a timed-out wait), slots 8..17 the warps of CTA 0 that have left
 * their role's loop (one-query-tile prefill kernel); n = 0 frees the buffer
 * and turns tracing off.  Negative n or a NULL host_view with n > 0 give
 * BSATTN_ERR_INVALID_ARG in both builds.
 */
int bsattn_debug_trace(int n, int32_t **host_view);

/*
 * bsattn_build_index -- block mask -> per-query-block CSR lists.
 *
 * Follows "块稀疏Attention实战" section 2.3 (keep the mask as an index of its
 * non-zero blocks) in the form the prefill kernel walks: for mask head h and
 * query block i, the key blocks j with mask[h][i][j] != 0, ascending; when
 * `causal` is set, only those with j * k_block <= (i + 1) * q_block - 1.
 *
 *   d_mask      uint8 [mask_heads][nq_blocks][nk_blocks], nonzero = keep
 *   d_row_ptr   int32 [mask_heads][nq_blocks + 1]: absolute offsets into
 *               d_col_idx (head h's rows follow head h-1's)
 *   d_col_idx   int32 [col_capacity]
 *   d_nnz       int32 [mask_heads]: kept blocks per mask head (always written)
 *   d_row_order int32 [mask_heads][nq_blocks] or NULL: for each mask head the
 *               query blocks ordered by decreasing row length (ties in
 *               ascending order); bsattn_fwd_prefill uses it to start the
 *               longest rows first
 *
 * When the kept blocks exceed col_capacity, no col_idx entry past the
 * capacity is written and *d_status (if given) receives BSATTN_ERR_CAPACITY;
 * row_ptr and nnz still describe the full index.  A capacity of
 * mask_heads * nq_blocks * nk_blocks can never overflow.
 */
int bsattn_build_index(const uint8_t *d_mask, int mask_heads, int nq_blocks, int nk_blocks,
                       int q_block, int k_block, int causal, int32_t *d_row_ptr,
                       int32_t *d_col_idx, int64_t col_capacity, int32_t *d_nnz,
                       int32_t *d_row_order, int32_t *d_status, cudaStream_t stream);

/*
 * bsattn_fwd_prefill -- block-sparse attention over a whole sequence.
 *
 * Query tiles and key tiles are both `block` tokens (64 or 128); d is 64 or
 * 128.  Query tile i of head h visits, in ascending order, the key tiles of
 * CSR row i of mask head (mask_heads == 1 ? 0 : h) -- or every key tile when
 * row_ptr is NULL -- restricted to j <= i when causal.  Inside a visited tile
 * keys past N and (causal) keys after the query are masked element by
 * element.  With lambda > 0 each visited tile is tested by the BLASST rule
 * (all valid rows must pass).  Query rows past N are neither written nor part
 * of the vote.
 *
 *   q, k, v, o      bf16, 16-byte aligned, shapes as in the conventions above
 *   lse             fp32 [B][Hq][N] or NULL
 *   scale           softmax scale applied to Q K^T (e.g. 1/sqrt(d))
 *   row_ptr/col_idx CSR from bsattn_build_index (q_block = k_block = block),
 *                   or row_ptr = NULL for every tile
 *   row_order       the builder's longest-first row order, or NULL; only the
 *                   order in which query tiles are scheduled depends on it
 *                   (BSATTN_ERR_INVALID_ARG when given without row_ptr)
 *   tile_status     uint8 [B][Hq][nq][nk] or NULL; the call first clears it,
 *                   then writes 1 for each visited-and-skipped tile and 2 for
 *                   each executed tile (0 = not visited)
 *   d_status        int32 device word or NULL (see conventions)
 *
 * A query row with no executed key gets O = 0 and LSE = -inf.
 */
int bsattn_fwd_prefill(const void *q, const void *k, const void *v, void *o, float *lse,
                       int B, int Hq, int Hkv, int N, int d, int block, float scale, int causal,
                       float lambda, const int32_t *row_ptr, const int32_t *col_idx,
                       const int32_t *row_order, int mask_heads, uint8_t *tile_status,
                       int32_t *d_status, cudaStream_t stream);

/* Option bits of bsattn_fwd_prefill_ex. */
#define BSATTN_PREFILL_REVERSE 0x1u
#define BSATTN_PREFILL_SKIP_V 0x2u

/*
 * bsattn_fwd_prefill_ex -- bsattn_fwd_prefill with option bits; flags = 0 is
 * exactly bsattn_fwd_prefill.  Unknown bits give BSATTN_ERR_INVALID_ARG.
 *
 * BSATTN_PREFILL_REVERSE: every query tile visits its key tiles in descending
 * order instead of ascending.  This is the block-row reordering of "BLASST:
 * Dynamic Blocked Attention Sparsity via Softmax Thresholding" (ablation
 * study, Figure 8): the tiles nearest the query (the local window, which
 * usually holds the largest scores) then set the running max first, and the
 * farther tiles are tested against it.  The skip decisions -- and so O, LSE
 * and tile_status -- are those of the reversed order; with lambda = 0 only
 * the summation order changes.
 *
 * d_seq_lens: NULL, or int32 [B] in device memory: sequence b holds
 * d_seq_lens[b] valid tokens (values are clamped to [0, N]), the rest of its
 * N positions are padding ("块稀疏Attention实战" section 5.2: pad a batch to its
 * longest sequence and mask the padding keys).  Keys at or past the length
 * take no part, key tiles wholly past it are not visited, and query rows past
 * it are padding: they do not vote and get O = 0 and LSE = -inf.  Every
 * sequence's result equals that of the sequence alone at its own length.
 *
 * BSATTN_PREFILL_SKIP_V: a V tile is loaded only when some query tile that
 * shares it executes it, instead of for every visited tile.  Results are
 * unchanged.  The BLASST page's prefill kernel loads every V tile (section
 * 4.1: bandwidth is not the bottleneck, and a load issued after the decision
 * cannot hide its latency) and names this as the option for memory-bound
 * cases; it halves the bytes of a skipped step and delays every executed one.
 */
int bsattn_fwd_prefill_ex(const void *q, const void *k, const void *v, void *o, float *lse,
                          int B, int Hq, int Hkv, int N, int d, int block, float scale,
                          int causal, float lambda, const int32_t *row_ptr,
                          const int32_t *col_idx, const int32_t *row_order, int mask_heads,
                          uint8_t *tile_status, const int32_t *d_seq_lens, unsigned flags,
                          int32_t *d_status, cudaStream_t stream);

/*
 * bsattn_fwd_prefill_host -- bsattn_fwd_prefill for inputs in host memory,
 * with the transfers overlapped with the kernels.  The pages have no
 * counterpart of this entry point: it serves callers that keep Q, K and V on
 * the host, for whom the copies in and out take longer than the attention.
 *
 * The batch is cut into chunks of one sequence and kv_heads_per_chunk KV
 * heads (with their query heads); each chunk is copied host -> device on an
 * internal stream, computed by bsattn_fwd_prefill on `stream` once its copies
 * have landed, and its O copied device -> host on a second internal stream,
 * so copies in, kernels and copies out of different chunks run at once.  With
 * one KV head per chunk and an even group of at least 4 query heads, the
 * first and the last chunk run as pieces of 2 query heads (the first piece
 * brings the KV head's K and V), which shortens the two ends the copies in
 * cannot hide.  The call only enqueues work: `stream` completes after the
 * last copy out.
 *
 *   h_q, h_k, h_v   host inputs, layouts as in bsattn_fwd_prefill; page-locked
 *                   (cudaHostAlloc / pinned) for the copies to overlap
 *   h_o             host output [B][Hq][N][d] bf16
 *   d_q, d_k, d_v, d_o  device staging of the full tensors' sizes, owned by
 *                   the caller; their contents are overwritten
 *   row_ptr, col_idx, row_order, mask_heads   as in bsattn_fwd_prefill (device
 *                   memory; per-head masks are sliced per chunk)
 *   kv_heads_per_chunk  divides Hkv; 1 gives the finest overlap
 *
 * The caller must not touch the host or staging buffers before `stream`
 * completes.  The first call on a device creates two streams and a ring of
 * events for it, kept until the process exits.  No LSE or tile status is
 * produced.  Errors as in bsattn_fwd_prefill, plus BSATTN_ERR_INVALID_ARG for
 * a chunk size that does not divide Hkv.  Every argument check (and the
 * compute-capability check) comes before any copy is enqueued.  If a later
 * step fails part-way (a copy or a chunk's launch), `stream` is still made to
 * wait for everything already queued on the internal streams before the error
 * is returned, so the caller may reuse its buffers once `stream` completes.
 */
int bsattn_fwd_prefill_host(const void *h_q, const void *h_k, const void *h_v, void *h_o,
                            void *d_q, void *d_k, void *d_v, void *d_o, int B, int Hq, int Hkv,
                            int N, int d, int block, float scale, int causal, float lambda,
                            const int32_t *row_ptr, const int32_t *col_idx,
                            const int32_t *row_order, int mask_heads, int kv_heads_per_chunk,
                            int32_t *d_status, cudaStream_t stream);

/*
 * bsattn_decode_workspace_size -- bytes of scratch bsattn_fwd_decode needs:
 * per (batch, query head, split) d fp32 partial outputs plus the split's
 * running max and row sum.
 */
size_t bsattn_decode_workspace_size(int B, int Hq, int d, int num_splits);

/*
 * bsattn_fwd_decode -- one query token per sequence against a KV cache,
 * split-KV with a combine step.
 *
 * The query tile of (batch b, KV head g) is the Hq/Hkv query heads that share
 * the KV head (their V tile is shared, so it is skipped only when all of them
 * pass).  The ceil(L / block) key tiles are cut into num_splits contiguous
 * chunks of ceil(T / num_splits) tiles; each chunk runs the BLASST visit and
 * test with its own running max starting at -inf (the pages do not define
 * split-KV; this is the reading this library implements), streaming each K
 * tile and loading a V tile only when the tile is executed.  A combine kernel
 * then merges the chunks exactly (log-sum-exp).
 *
 *   q           bf16 [B][Hq][d];  k, v bf16 [B][Hkv][L][d]
 *   o           bf16 [B][Hq][d];  lse fp32 [B][Hq] or NULL
 *   causal      accepted and ignored: the single query is the last position
 *   workspace   device scratch of at least bsattn_decode_workspace_size(...)
 *               bytes, 16-byte aligned, owned by the caller
 *   tile_status uint8 [B][Hkv][T] or NULL (cleared, then 1 skipped / 2 executed)
 *
 * Supported GQA groups Hq/Hkv: 1..16, with key tiles of 64 or 128 tokens
 * (one tensor-core kernel); anything else gives BSATTN_ERR_UNSUPPORTED.
 */
int bsattn_fwd_decode(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                      int Hq, int Hkv, int L, int d, int block, float scale, int causal,
                      float lambda, int num_splits, void *workspace, size_t workspace_bytes,
                      uint8_t *tile_status, int32_t *d_status, cudaStream_t stream);

/* Option bits of bsattn_fwd_decode_ex. */
#define BSATTN_DECODE_SINK_SEED 0x1u

/*
 * bsattn_fwd_decode_ex -- bsattn_fwd_decode with option bits; flags = 0 is
 * exactly bsattn_fwd_decode.  Unknown bits give BSATTN_ERR_INVALID_ARG.
 *
 * BSATTN_DECODE_SINK_SEED: every split but the first starts its running max
 * from the row max of key tile 0 -- the tile that holds the attention sink --
 * instead of -inf.  The split scores tile 0 for this (one more K tile read per
 * split) without visiting or executing it; tile_status and the result count
 * tile 0 only in the first split.  A later split can then skip tiles that the
 * sink dominates, where a split starting at -inf must execute its first tile
 * and test the rest against its own, smaller maxima.  (The pages define no
 * split-KV; this variant keeps their skip rule and only changes the starting
 * value of each split's running max.)
 *
 * d_seq_lens: NULL, or int32 [B] in device memory: cache b holds d_seq_lens[b]
 * valid tokens (clamped to [0, L]); keys past it take no part, and the
 * num_splits splits cut that cache's own ceil(len / block) tiles, so every
 * sequence's result equals that of its cache alone.  A zero length gives
 * O = 0 and LSE = -inf.
 */
int bsattn_fwd_decode_ex(const void *q, const void *k, const void *v, void *o, float *lse,
                         int B, int Hq, int Hkv, int L, int d, int block, float scale, int causal,
                         float lambda, int num_splits, void *workspace, size_t workspace_bytes,
                         uint8_t *tile_status, const int32_t *d_seq_lens, unsigned flags,
                         int32_t *d_status, cudaStream_t stream);

/*
 * bsattn_fwd_decode_noalloc -- bsattn_fwd_decode for callers that cannot
 * allocate device memory.  The pages have no counterpart of this entry point.
 *
 * Some callers cannot call cudaMalloc at all: code inside a host framework
 * that owns all device memory and hands extensions only their input and
 * output buffers (an inference engine with one pre-planned memory arena, for
 * instance), or latency-critical service paths where an allocation's cost and
 * possible failure are not acceptable.  They cannot provide the decode
 * workspace, so this variant uses a scratch array inside the library: a
 * file-scope device array of 32 MiB, held on every GPU that loads the library
 * until the process exits.  The call itself allocates nothing.
 *
 * Arguments, layouts and results are those of bsattn_fwd_decode without the
 * workspace.  Checks come in this order: NULL q/k/v/o, non-positive sizes or
 * Hq % Hkv != 0 give BSATTN_ERR_INVALID_ARG; then problems whose split
 * outputs need more than 32 MiB (bsattn_decode_workspace_size(B, Hq, d,
 * num_splits) > 33554432) give BSATTN_ERR_CAPACITY; then every other check of
 * bsattn_fwd_decode.  Nothing runs on a rejected call.
 *
 * The first call in each CUDA context (in practice: on each device, with that
 * device current) looks up the scratch array's device address and caches it
 * under the context's unique id, so make that call before any stream capture.
 * A later context on the same device (after cudaDeviceReset) looks it up
 * again.  Every call shares the one scratch array, which keeps the last
 * call's contents; no part of it needs to start at zero.  Calls whose kernels
 * may overlap on the GPU (unordered streams) race on it and must be
 * serialised.
 */
int bsattn_fwd_decode_noalloc(const void *q, const void *k, const void *v, void *o, float *lse,
                              int B, int Hq, int Hkv, int L, int d, int block, float scale,
                              int causal, float lambda, int num_splits, uint8_t *tile_status,
                              int32_t *d_status, cudaStream_t stream);

/*
 * bsattn_bwd_prefill_workspace_size -- bytes of scratch bsattn_bwd_prefill
 * needs: two fp32 values (D and LSE in base 2) per query row, padded to
 * whole query tiles.
 */
size_t bsattn_bwd_prefill_workspace_size(int B, int Hq, int N, int block);

/*
 * bsattn_bwd_prefill -- gradients of bsattn_fwd_prefill for sparsity-aware
 * training ("BLASST: Dynamic Blocked Attention Sparsity via Softmax
 * Thresholding", section 3.3: fine-tuning runs the forward with the skip, and
 * the blocks it skipped receive no gradient because they were never
 * computed).  With the forward's executed tiles held fixed, the forward is the
 * softmax attention over their keys, and this is its exact gradient:
 *   P = exp(scale Q K^T - LSE), D = rowsum(dO * O), dS = P (dO V^T - D),
 *   dV = P^T dO, dK = scale dS^T Q, dQ = scale dS K,
 * summed over the executed tiles only; keys in tiles that no query tile
 * executed get dK = dV = 0.
 *
 *   q, k, v, o      the forward's inputs and output (bf16, layouts as there)
 *   dout            dL/dO, bf16 [B][Hq][N][d]
 *   lse             the forward's LSE, fp32 [B][Hq][N] (required)
 *   tile_status     the forward's tile status, uint8 [B][Hq][nq][nk]
 *                   (required; only tiles marked 2, executed, take part)
 *   dq              bf16 [B][Hq][N][d];  dk, dv bf16 [B][Hkv][N][d] (written)
 *   causal, d_seq_lens  as in the forward call
 *   workspace       device scratch of bsattn_bwd_prefill_workspace_size bytes,
 *                   16-byte aligned, owned by the caller
 *
 * block must be 128 and d 64 or 128 (else BSATTN_ERR_UNSUPPORTED).  Three
 * kernels run on `stream`: per-row statistics, then dK/dV (one CTA per key
 * tile, accumulating over the GQA group's query heads) and dQ (one CTA per
 * query tile); each output tile has a single writer, no atomics.
 */
int bsattn_bwd_prefill(const void *q, const void *k, const void *v, const void *o,
                       const void *dout, const float *lse, const uint8_t *tile_status, void *dq,
                       void *dk, void *dv, int B, int Hq, int Hkv, int N, int d, int block,
                       float scale, int causal, const int32_t *d_seq_lens, void *workspace,
                       size_t workspace_bytes, int32_t *d_status, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BSATTN_H_ */
