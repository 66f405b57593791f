/*
 * seer.h -- C ABI of libseer: SeerAttention-R's gated block-sparse GQA decode
 * step on NVIDIA B200 (sm_100a).
 *
 * Sources, cited by page and section:
 *   [CP] "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning"
 *        (chapterpal.com summary): Knowl 1-2 (AttnGate), Knowl 5 (K
 *        Compression Cache, token budget and threshold), Knowl 6 (block-sparse
 *        flash decoding on a (batch, heads_kv, num_split) grid), Knowl 14
 *        (PagedAttention support).
 *   [PN] "Sparse Attention Adaptation for Long Reasoning" (papernotes.org
 *        notes): key designs 1, 2 and 4.
 *
 * One decode step of one attention layer is
 *     seer_kcomp_update -> seer_gate_score -> seer_select_blocks -> seer_sparse_decode
 * or, with the first three fused into one launch,
 *     seer_decode_plan -> seer_sparse_decode
 * or, the whole step in one launch,
 *     seer_decode_step
 *
 * Conventions shared by every call
 *   - The caller owns all memory.  The library never allocates or frees.
 *   - Every pointer argument named "device" is a CUDA device pointer on the
 *     current device; arguments of type seer_dims_t* / seer_kv_t* are HOST
 *     pointers read during the call only.
 *   - Every call only enqueues kernels on `stream` (a cudaStream_t, NULL =
 *     legacy default stream) and returns without synchronising the host.
 *   - Sequence lengths L_b (`seqlens`) count the tokens in the cache,
 *     including the token being decoded.  nfull_b = floor(L_b / b) full
 *     blocks; block nfull_b is partial when L_b mod b != 0.
 *   - bf16 tensors are IEEE bfloat16.  Query head i belongs to KV head
 *     floor(i / g), g = Hq / Hkv.
 *   - Device pointers must be 16-byte aligned.
 *   - Supported shapes: head_dim in {64, 128}; block_size in {64, 128};
 *     gate_dim in {64, 128}; 1 <= g <= 8; max_blocks <= 8192.  Anything else
 *     returns SEER_ERR_UNSUPPORTED before any work is enqueued.
 *   - On a non-OK status nothing has been enqueued (argument errors) or the
 *     launch failed (SEER_ERR_CUDA); seer_last_error() gives the reason.
 *   - Anomalies that only the device can see (a block index outside
 *     [0, ceil(L_b/b)), a page id outside the pool, a count above the
 *     capacity, a pipeline wait that timed out) never trap: the kernel skips
 *     the offending work and ORs a SEER_DEVERR_* bit into *err_word when the
 *     call was given one.
 */
#ifndef SEER_H
#define SEER_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SEER_OK = 0,
  SEER_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned pointer or stride */
  SEER_ERR_UNSUPPORTED = 2, /* shape outside the supported set above */
  SEER_ERR_CAPACITY = 3,    /* index tensor width too small for the selection mode */
  SEER_ERR_CUDA = 4         /* a CUDA runtime/driver call failed */
} seer_status;

/* Bits ORed into the optional device error word. */
#define SEER_DEVERR_BLOCK_INDEX 1  /* selected block index outside [0, ceil(L/b)) */
#define SEER_DEVERR_PAGE_INDEX 2   /* block_table entry outside [0, num_pages) */
#define SEER_DEVERR_COUNT 4        /* block count above capacity */
#define SEER_DEVERR_TIMEOUT 8      /* a pipeline wait exceeded its bound */

typedef enum { SEER_KV_CONTIGUOUS = 0, SEER_KV_PAGED = 1 } seer_kv_layout;

/*
 * A K or V cache (bf16).  head_dim elements of one token are contiguous.
 *   SEER_KV_CONTIGUOUS: element (b, h, t, c) at data + b*stride_b + h*stride_h + t*stride_t + c,
 *     t < num_tokens (the cache's token capacity).
 *   SEER_KV_PAGED (PagedAttention-style [CP Knowl 14], page size == block_size):
 *     token t of sequence b lives in page p = block_table[b*max_pages_per_seq + t/block_size]
 *     at data + p*stride_b + h*stride_h + (t % block_size)*stride_t + c, p < num_pages.
 * Strides are in elements; stride_t, stride_h and stride_b must be multiples of 8
 * (16 bytes) for the TMA tile loads.
 */
typedef struct {
  int32_t layout;             /* seer_kv_layout */
  const void* data;           /* device, bf16 */
  int64_t stride_b;           /* contiguous: per sequence; paged: per page */
  int64_t stride_h;           /* per KV head */
  int64_t stride_t;           /* per token */
  int64_t num_tokens;         /* contiguous: token capacity per (b, h); paged: ignored */
  int64_t num_pages;          /* paged: pages in the pool; contiguous: ignored */
  const int32_t* block_table; /* paged: device int32 [B, max_pages_per_seq]; contiguous: NULL */
  int32_t max_pages_per_seq;  /* paged: row length of block_table */
} seer_kv_t;

/* Problem shape shared by all calls of one layer. */
typedef struct {
  int32_t batch;        /* B */
  int32_t num_q_heads;  /* Hq */
  int32_t num_kv_heads; /* Hkv (Hq must be a multiple) */
  int32_t head_dim;     /* d */
  int32_t gate_dim;     /* d_gate: AttnGate hidden size per KV head [CP Knowl 1] */
  int32_t block_size;   /* b: sparse block = pooling kernel/stride = page size */
  int32_t max_blocks;   /* row length of kcomp and logits; must cover ceil(L_b/b) for every b */
  float rope_base;      /* RoPE base inside the gate (e.g. 1e6) */
  float softmax_scale;  /* attention scale; 0 selects 1/sqrt(head_dim) */
} seer_dims_t;

/*
 * seer_kcomp_update -- K Compression Cache maintenance [CP Knowl 5; PN design 2, 4].
 *
 * For every sequence b and KV head h and every block n with
 * valid_blocks[b, h] <= n < floor(seqlens[b] / b):
 *   p = [max | min | avg] over the b pre-RoPE keys of block n (per channel, 3d values)
 *   kcomp[b, h, n, :] = bf16( RoPE_{n*b}( W_k[h] . p ) )      (RoPE rotate-half, theta_i = base^(-2i/d_gate))
 * then valid_blocks[b, h] = floor(seqlens[b] / b).  Entries below valid_blocks[b, h] are not
 * touched, so calling this every decode step recomputes a block exactly once, when it
 * fills; valid_blocks = 0 rebuilds the whole cache (prefill).
 *
 *   k_nope        pre-RoPE key cache (see seer_kv_t); may alias the attention K cache
 *   seqlens       device int32 [B]
 *   valid_blocks  device int32 [B, Hkv] (cache fill count per sequence and KV head), read then written
 *   w_k           device bf16 [Hkv, d_gate, 3*d]  (no bias)
 *   kcomp         device bf16 [B, Hkv, max_blocks, d_gate]
 * One launch: a cluster of 8 CTAs per (b, h) shares its new blocks.
 */
seer_status seer_kcomp_update(const seer_dims_t* dims, const seer_kv_t* k_nope,
                              const int32_t* seqlens, int32_t* valid_blocks, const void* w_k,
                              void* kcomp, void* stream);

/*
 * seer_kcomp_append -- the same cache update from running block statistics, one appended
 * token per sequence and call [CP Knowl 2, Knowl 5: an entry is built from the b keys of one
 * finished block, so their per-channel max, min and sum are all it needs].
 *
 * Each sequence b has just appended token t = seqlens[b] - 1 (seqlens after the append;
 * seqlens[b] <= 0: nothing appended, nothing done).  With n = floor(t / b), i = t mod b and
 * x = k_new[b, h, :]:
 *   i == 0:  state[b, h] = (x, x, x)                                   (the block restarts)
 *   i  > 0:  state[b, h] = (max(state.max, x), min(state.min, x), state.sum + x)
 *   i == b-1 (the token completes block n):
 *            kcomp[b, h, n, :] = bf16( RoPE_{n*b}( W_k[h] . [max | min | sum/b] ) )
 *            valid_blocks[b, h] = n + 1
 * which equals what seer_kcomp_update computes for block n from the K cache (fp32 sums).  The
 * completing call requires valid_blocks[b, h] == n and n < max_blocks; otherwise it writes
 * no entry and ORs SEER_DEVERR_COUNT into *err_word.  No pre-RoPE copy of the context is needed:
 * the state is 3*d fp32 per (b, h).
 *
 *   k_new         device bf16 [B, Hkv, d]: the pre-RoPE keys of the appended tokens
 *   seqlens       device int32 [B] (after the append)
 *   state         device fp32 [B, Hkv, 3, d] (running max, min, sum; seer_kcomp_state_bytes);
 *                 read and written.  A sequence that continues mid-block must have it primed
 *                 by seer_kcomp_state_init; one at a block boundary needs nothing.
 *   valid_blocks  device int32 [B, Hkv], read and advanced
 *   w_k, kcomp    as seer_kcomp_update
 *   err_word      device int32 or NULL (SEER_DEVERR_* bits ORed in)
 * One CTA per (b, h).  Calls must be made in token order, one per appended token.
 */
size_t seer_kcomp_state_bytes(const seer_dims_t* dims);
seer_status seer_kcomp_append(const seer_dims_t* dims, const void* k_new, const int32_t* seqlens,
                              float* state, int32_t* valid_blocks, const void* w_k, void* kcomp,
                              int32_t* err_word, void* stream);

/*
 * seer_kcomp_state_init -- prime the running block statistics of seer_kcomp_append from the
 * key cache [CP Knowl 5: the entry of the block in progress is built once it is full]: for every (b, h), the per-channel max, min and sum of the pre-RoPE keys of tokens
 * [floor(L_b / b) * b, L_b) (the current, incomplete block; empty at a block boundary:
 * -inf, +inf, 0).  Reads at most b - 1 keys per (b, h).  Page or capacity errors set
 * SEER_DEVERR_PAGE_INDEX / SEER_DEVERR_COUNT in *err_word and leave the empty statistics.
 *
 *   k_nope   pre-RoPE key cache (see seer_kv_t)
 *   seqlens  device int32 [B]
 *   state    device fp32 [B, Hkv, 3, d], written
 */
seer_status seer_kcomp_state_init(const seer_dims_t* dims, const seer_kv_t* k_nope,
                                  const int32_t* seqlens, float* state, int32_t* err_word,
                                  void* stream);

/*
 * seer_gate_score -- AttnGate block logits [CP Knowl 1-2; PN design 1].
 *
 *   Q_gate[b, h] = RoPE_{L_b - 1}( W_q[h] . concat_j q_nope[b, h*g + j, :] )   (fp32, not rounded)
 *   logits[b, h, n] = <Q_gate[b, h], kcomp[b, h, n]> / sqrt(d_gate)   for n < floor(L_b / b)
 *   logits[b, h, n] = -inf                                             for floor(L_b/b) <= n < max_blocks
 * softmax over n of the logits is the gate score S.
 *
 *   q_nope      device bf16 [B, Hq, d]  (pre-RoPE query of the current token)
 *   w_q         device bf16 [Hkv, d_gate, g*d]  (one projection per KV head, no bias)
 *   kcomp       device bf16 [B, Hkv, max_blocks, d_gate]
 *   seqlens     device int32 [B]
 *   logits      device fp32 [B, Hkv, max_blocks]  (written)
 *   q_gate_out  device fp32 [B, Hkv, d_gate] or NULL
 */
seer_status seer_gate_score(const seer_dims_t* dims, const void* q_nope, const void* w_q,
                            const void* kcomp, const int32_t* seqlens, float* logits,
                            float* q_gate_out, void* stream);

#define SEER_SELECT_TOPK 0
#define SEER_SELECT_THRESHOLD 1
#define SEER_SELECT_TOPP 2

/*
 * seer_select_blocks -- logits -> block index lists [CP Knowl 5, Knowl 14].
 *
 * Per (b, h), over the nfull = floor(L_b/b) full blocks:
 *   SEER_SELECT_TOPK:      k = ceil(token_budget / b); the min(k, nfull) blocks with the largest
 *                          logits, ties to the lower block index.  Capacity >= k + 1.
 *   SEER_SELECT_THRESHOLD: S = softmax(logits[0:nfull]); blocks with S > tau (strict).
 *                          Capacity >= max_blocks.  S and the comparison are evaluated in fp64.
 *   SEER_SELECT_TOPP:      fewest blocks, in descending S order (ties to the lower index),
 *                          whose S-sum reaches tau (used as p).  Capacity >= max_blocks.
 * In every mode the partial block nfull is appended when L_b mod b != 0.
 * Output rows list the chosen indices ascending, then -1 up to `capacity`.
 *
 *   logits     device fp32 [B, Hkv, max_blocks]
 *   seqlens    device int32 [B]
 *   block_idx  device int32 [B, Hkv, capacity]  (written)
 *   block_cnt  device int32 [B, Hkv]            (written)
 */
seer_status seer_select_blocks(const seer_dims_t* dims, const float* logits,
                               const int32_t* seqlens, int32_t mode, int32_t token_budget,
                               float tau, int32_t* block_idx, int32_t* block_cnt,
                               int32_t capacity, void* stream);

/*
 * seer_decode_plan -- seer_kcomp_update + seer_gate_score + seer_select_blocks in one launch
 * [CP Knowl 1-2, Knowl 5, as those three calls].
 *
 * Same arguments and results as the three calls made in that order, with these differences:
 *   valid_blocks  NULL skips the cache update (the cache must then be current already)
 *   logits_out    device fp32 [B, Hkv, max_blocks] or NULL (the logits stay on chip)
 * One cluster of 4 CTAs per (b, h): the cache rows of newly full blocks, the gate logits
 * (shared through distributed shared memory) and the selection never leave the cluster.
 */
seer_status seer_decode_plan(const seer_dims_t* dims, const seer_kv_t* k_nope, const int32_t* seqlens,
                             int32_t* valid_blocks, const void* w_k, void* kcomp, const void* q_nope,
                             const void* w_q, float* logits_out, float* q_gate_out, int32_t mode,
                             int32_t token_budget, float tau, int32_t* block_idx, int32_t* block_cnt,
                             int32_t capacity, void* stream);

/*
 * A split count for the pages' (num_split, Hkv, B) grid [CP Knowl 6] that fills one wave of the
 * SMs (host heuristic, no device reads).  seer_sparse_decode uses its own one-wave schedules when given
 * num_split == 0 or -1; pass this value to get the grid schedule instead.
 */
int32_t seer_sparse_decode_auto_split(const seer_dims_t* dims, int32_t capacity);

/*
 * Workspace bytes seer_sparse_decode needs for `num_split` [CP Knowl 6: the split partials and
 * their log-sum-exp combine]: one arrival counter per (b, h) plus fp32 partial outputs and LSEs -- 2 slots per CTA of the one-wave schedules (num_split 0, -1),
 * num_split slots per (b, h) for the grid schedule, none for num_split == 1.  The counters must
 * be zero before the first call (e.g. allocate zero-filled); every completed call leaves them
 * zero again.
 */
size_t seer_sparse_decode_workspace_bytes(const seer_dims_t* dims, int32_t capacity,
                                          int32_t num_split);

/*
 * seer_sparse_decode -- block-sparse flash decoding + split LSE combine [CP Knowl 6; PN design 4].
 *
 * For each query head i of KV head h (GQA group shares the list [PN design 1]):
 *   T = union over the first block_cnt[b, h] entries n of block_idx[b, h, :] of tokens
 *       [n*b, min((n+1)*b, L_b))
 *   out[b, i] = sum_{t in T} softmax_t(scale * q[b,i] . K[b,h,t]) V[b,h,t]
 *   lse_out[b, i] = log sum_{t in T} exp(scale * q[b,i] . K[b,h,t])   (-inf, out = 0 when T is empty)
 * Schedules:
 *   num_split >= 1: the pages' grid (num_split, Hkv, B); each list is split into slices of
 *     ceil(capacity / num_split) positions (the split size comes from the index tensor width,
 *     max_selected_blocks, not from the sequence length).
 *   num_split == 0: balanced -- the concatenation of all lists is cut into equal contiguous
 *     ranges, one per CTA of a grid with one CTA per SM slot.
 *   num_split == -1: capacity -- as balanced, but every list counts as `capacity` positions
 *     (those at or past block_cnt are skipped), so the ranges need no scan of the counts and the
 *     first tiles are requested one round trip after the launch's inputs are ready.  Best when
 *     the counts are at or near the capacity (top-k with a fixed budget); with short lists the
 *     skipped positions leave CTAs idle.
 * Both one-wave schedules require batch*Hkv <= 4096 and batch*Hkv*capacity < 2^30.
 * In all, a (b, h) computed by several CTAs is merged (LSE combine) by the last of them.
 *
 *   q          device bf16 [B, Hq, d]  (post-RoPE query, as the model uses it)
 *   k, v       K and V caches (see seer_kv_t)
 *   block_idx  device int32 [B, Hkv, capacity]; block_cnt device int32 [B, Hkv]
 *   seqlens    device int32 [B]
 *   num_split  0 = balanced, -1 = capacity, >= 1 = grid schedule; must match the workspace size
 *   workspace  device, >= seer_sparse_decode_workspace_bytes(dims, capacity, num_split) bytes
 *   out        device bf16 [B, Hq, d]
 *   lse_out    device fp32 [B, Hq] or NULL
 *   err_word   device int32 or NULL (SEER_DEVERR_* bits ORed in)
 * Calls on the same workspace must not overlap on the GPU.
 */
seer_status seer_sparse_decode(const seer_dims_t* dims, const void* q, const seer_kv_t* k,
                               const seer_kv_t* v, const int32_t* block_idx,
                               const int32_t* block_cnt, const int32_t* seqlens,
                               int32_t capacity, int32_t num_split, void* workspace,
                               size_t workspace_bytes, void* out, float* lse_out,
                               int32_t* err_word, void* stream);

/*
 * seer_decode_step -- the whole decode step in one launch: seer_decode_plan followed by
 * seer_sparse_decode with the capacity schedule (num_split == -1) [CP Knowl 1-2, Knowl 5,
 * Knowl 6, as those calls].
 *
 * Arguments are those of seer_decode_plan (k_nope .. capacity) followed by those of
 * seer_sparse_decode (q, k, v, workspace .. err_word); results are the same: the cache rows and
 * fill counts, the optional logits / Q_gate, the block lists and counts, out and lse_out.
 *   workspace  device, >= seer_decode_step_workspace_bytes(dims, capacity) bytes, 16-byte
 *              aligned; its first B*Hkv int32 are per-row ready flags and the next section holds
 *              the decode's arrival counters: both must be zero before the first call (allocate
 *              zero-filled), and every completed call leaves them zero.  After a call that set
 *              SEER_DEVERR_TIMEOUT, zero the workspace again before the next call.
 * One CTA per SM in clusters of two: each cluster first plans the rows whose lists start in its
 * two ranges (cache update, gate, selection, as seer_decode_plan), publishes each list with a
 * per-row flag, then every CTA streams its range, waiting only for the rows it reads.  Requires
 * every CTA of the grid to be resident at once (the grid is sized from the co-resident cluster
 * count; each wait is bounded and reports SEER_DEVERR_TIMEOUT).
 * Returns SEER_ERR_UNSUPPORTED when the shape has no fused kernel (see
 * seer_decode_step_supported); use seer_decode_plan + seer_sparse_decode then.
 * seer_decode_step_supported returns 1 when the current device runs this shape and selection
 * mode fused (no device work), else 0.
 * Calls on the same workspace must not overlap on the GPU.
 */
size_t seer_decode_step_workspace_bytes(const seer_dims_t* dims, int32_t capacity);
int32_t seer_decode_step_supported(const seer_dims_t* dims, int32_t mode, int32_t capacity);
seer_status seer_decode_step(const seer_dims_t* dims, const seer_kv_t* k_nope, const int32_t* seqlens,
                             int32_t* valid_blocks, const void* w_k, void* kcomp, const void* q_nope,
                             const void* w_q, float* logits_out, float* q_gate_out, int32_t mode,
                             int32_t token_budget, float tau, int32_t* block_idx, int32_t* block_cnt,
                             int32_t capacity, const void* q, const seer_kv_t* k, const seer_kv_t* v,
                             void* workspace, size_t workspace_bytes, void* out, float* lse_out,
                             int32_t* err_word, void* stream);

/*
 * seer_sparse_decode_noalloc -- seer_sparse_decode for callers that cannot allocate.
 *
 * The pages have no counterpart to this call; it is an interface convenience.  Callers that
 * must not call cudaMalloc -- an engine that reserved all free device memory for its KV pool
 * before serving, a plugin whose host owns every allocation, a hot loop that cannot afford
 * cudaMalloc's implicit device synchronisation -- pass only inputs and outputs here.  The
 * split partials and arrival counters live in a fixed 8 MiB scratch array inside the library
 * image (held by every GPU that loads the library until the process exits).
 *
 * Arguments and results are those of seer_sparse_decode without workspace/workspace_bytes.
 * Returns SEER_ERR_CAPACITY when the chosen split count needs more scratch than 8 MiB
 * (seer_sparse_decode_workspace_bytes > 8388608).  Every argument check of seer_sparse_decode
 * runs first: on any non-OK status nothing at all is enqueued.
 * The first call on a device looks up the scratch's device address (cudaGetSymbolAddress) with
 * that device current and keeps it for the life of the process; make that first call before any
 * stream capture, and make no call after cudaDeviceReset.  Each call clears the arrival counters
 * with an async memset on `stream`.  All calls on a device share the scratch: calls that overlap
 * on the GPU race and must be serialised by the caller.  Allocates nothing.
 */
seer_status seer_sparse_decode_noalloc(const seer_dims_t* dims, const void* q, const seer_kv_t* k,
                                       const seer_kv_t* v, const int32_t* block_idx,
                                       const int32_t* block_cnt, const int32_t* seqlens,
                                       int32_t capacity, int32_t num_split, void* out,
                                       float* lse_out, int32_t* err_word, void* stream);

/*
 * seer_gate_truth -- decode ground-truth block scores from full attention [CP Knowl 3]: the
 * target the AttnGate is distilled towards, usable in its place ("oracle" selection).
 *
 * For each (b, h) with L = seqlens[b] and nblk = ceil(L / block_size) (capped at max_blocks):
 *   p_j[t]  = softmax_t(scale * q[b, h*g+j] . K[b, h, t]) over t < L, for the g heads j of the group
 *   raw[n]  = max_j max_{t in block n, t < L} p_j[t]                     (n < nblk)
 *   scores[b, h, n] = raw[n] / sum_n' raw[n'] for n < nblk, 0 for n >= nblk (all 0 when L = 0)
 *   log_scores[b, h, n] = log(scores[b, h, n]) (-inf where 0), if log_scores is not NULL:
 *     top-k or threshold selection on these (seer_select_blocks) picks blocks by ground truth.
 * Unlike the gate, the partial last block is scored too.
 *
 *   q           device bf16 [B, Hq, d] (the attention query: post-RoPE)
 *   k           the attention K cache (see seer_kv_t)
 *   seqlens     device int32 [B]
 *   scores      device fp32 [B, Hkv, max_blocks]; log_scores the same or NULL
 *   workspace   device, >= seer_gate_truth_workspace_bytes(dims) bytes, 16-byte aligned; its
 *               first B*Hkv int32 are arrival counters that must be zero before the first call
 *               (every completed call leaves them zero)
 *   err_word    device int32 or NULL (SEER_DEVERR_* bits ORed in)
 * Reads all of K once (HBM-bound).  Calls on the same workspace must not overlap on the GPU.
 */
size_t seer_gate_truth_workspace_bytes(const seer_dims_t* dims);
seer_status seer_gate_truth(const seer_dims_t* dims, const void* q, const seer_kv_t* k,
                            const int32_t* seqlens, float* scores, float* log_scores,
                            void* workspace, size_t workspace_bytes, int32_t* err_word,
                            void* stream);

/*
 * seer_prefill_gt -- causal attention over whole sequences with the block-level target of every
 * query position beside the output, extracted inside the attention forward [CP Knowl 3, Knowl 4]:
 * per key tile (one block of b keys) each query row's maximum pre-softmax score r is kept, and
 * once the row's final maximum m and normaliser l are known the block's score is exp(r - m) / l.
 *
 * For sequence b, query head i = h*g + j of KV head h and position t < L_b = seqlens[b]:
 *   out[b, i, t] = sum_{u <= t} softmax_u(scale * q[b, i, t] . K[b, h, u]) V[b, h, u]
 *   lse_out[b, i, t] = log sum_{u <= t} exp(scale * q[b, i, t] . K[b, h, u])
 *   gt[b, h, t, n] = G[n] / sum_n' G[n'],   G[n] = max_j max_{u in block n, u <= t} softmax_u(...)
 *                    for n <= t / b, and 0 for t / b < n < max_blocks
 * i.e. row t of gt is the decode target (seer_gate_truth) of query position t.  Rows t >= L_b
 * are not written, and q, K and V rows at positions >= L_b are never used (they may hold
 * anything, NaN included).
 *
 *   q          device bf16 [B, Hq, max_len, d]
 *   max_len    row capacity of q / out / lse_out / gt (>= every seqlens[b]; max_blocks*b >= max_len)
 *   k, v       contiguous K / V caches (see seer_kv_t) holding >= seqlens[b] tokens; longer
 *              sequences are cut to the caches' capacity and SEER_DEVERR_COUNT is set
 *   seqlens    device int32 [B]
 *   out        device bf16 [B, Hq, max_len, d]
 *   lse_out    device fp32 [B, Hq, max_len] or NULL
 *   gt         device fp32 [B, Hkv, max_len, max_blocks]
 *   workspace  device, >= seer_prefill_gt_workspace_bytes(dims, max_len) bytes (each query row's
 *              per-block score maxima, fp32 [B, Hq, max_blocks, max_len], then each row's log2
 *              normaliser, fp32 [B, Hq, max_len]), 16-byte aligned
 *   err_word   device int32 or NULL (SEER_DEVERR_* bits ORed in)
 * head_dim 128 with g in {1, 2, 4, 8}: the tcgen05 / TMEM forward (one CTA per 128 / g positions of
 * the group's g heads, KV head, sequence), then a bandwidth-bound kernel forming the targets (two
 * launches).  Other shapes: the warp-level mma forward, one CTA per (16 * floor(8 / g) positions,
 * KV head, sequence), targets formed in its epilogue.  The group's query heads share every K/V
 * tile.  Paged caches: SEER_ERR_UNSUPPORTED.
 */
size_t seer_prefill_gt_workspace_bytes(const seer_dims_t* dims, int32_t max_len);
seer_status seer_prefill_gt(const seer_dims_t* dims, const void* q, int32_t max_len,
                            const seer_kv_t* k, const seer_kv_t* v, const int32_t* seqlens,
                            void* out, float* lse_out, float* gt, void* workspace,
                            size_t workspace_bytes, int32_t* err_word, void* stream);

/*
 * Bounded waits of the sparse decode (seer_sparse_decode, seer_sparse_decode_noalloc and the
 * decode launch of the two-launch step).  No passage defines these: they are part of the
 * library's own error behaviour (a wait that runs out reports SEER_DEVERR_TIMEOUT and the kernel
 * returns, so the context stays usable).
 *
 * seer_set_wait_limit: the bound of every copy and hand-off wait of those kernels, in SM clock
 *   cycles, process-wide, taken at each launch.  0 restores the default (2e9 cycles, about one
 *   second).  Values outside [SEER_WAIT_LIMIT_MIN, SEER_WAIT_LIMIT_MAX]: SEER_ERR_INVALID_ARG
 *   and the bound is left as it was.  A small bound can make a healthy launch report a timeout.
 * seer_get_wait_limit: the bound in force.
 * seer_set_debug_flags: process-wide debug switches taken at each launch; 0 turns them off.
 *   SEER_DEBUG_STARVE_COPIES: the decode's producer issues no copy and arms no barrier, so the
 *   first wait of every CTA runs out; the launch writes no output, reports SEER_DEVERR_TIMEOUT and
 *   leaves the workspace's split counters zero.  For tests of the timeout path only.  Unknown
 *   bits: SEER_ERR_INVALID_ARG.  (The one-launch step, seer_decode_step, ignores the switch.)
 * After a launch that reported SEER_DEVERR_TIMEOUT for any other reason, zero the workspace
 * (seer_sparse_decode's split counters) before the next call.
 */
#define SEER_WAIT_LIMIT_MIN 1000LL
#define SEER_WAIT_LIMIT_MAX 100000000000LL
#define SEER_DEBUG_STARVE_COPIES 1
seer_status seer_set_wait_limit(int64_t cycles);
int64_t seer_get_wait_limit(void);
seer_status seer_set_debug_flags(int32_t flags);

/* Thread-local text describing the last non-OK status returned on this thread. */
const char* seer_last_error(void);

/* Library version string. */
const char* seer_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SEER_H */
