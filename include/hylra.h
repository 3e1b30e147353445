/*
 * hylra.h - C ABI of the HyLRA decode-attention library (B200, sm_100a).
 *
 * Method: "HyLRA: Hybrid Layer Reuse Attention for Efficient Long-Context
 * Inference" (gist.science technical summary of arXiv 2602.00777), cited as
 * "HyLRA summary" with its section numbers.
 *
 *   §2.3 Hybrid Inference Strategy: during decoding, a sensitive ("reset")
 *        layer runs standard full attention and extracts top-k indices that
 *        are passed forward; a tolerant ("reuse") layer reuses the indices of
 *        the preceding reset layer and restricts attention to that subset of
 *        the KV cache.                     -> hylra_decode_full, hylra_decode_reuse,
 *                                             hylra_decode_step
 *   §2.4 Block-level Sparsity: selection works on fixed 128-token blocks.
 *   §2.4 Index-Guided Offloading: a cache in host memory sends only the
 *        reused blocks across the host link.
 *                                          -> hylra_gather_blocks,
 *                                             hylra_decode_reuse_staged,
 *                                             hylra_decode_step_offload
 *   §2.2 Offline policy: a lower-triangular overlap matrix M of top-k indices
 *        between source and target layers, and a dynamic program over states
 *        (i, j) with reset jumps and vertical moves gated by theta.
 *                                          -> hylra_similarity, hylra_dp_policy,
 *                                             hylra_overlap_counts,
 *                                             hylra_similarity_from_counts
 *   §4   The Jump3 baseline (a reset every third layer).
 *                                          -> hylra_static_policy
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  * Every call returns an int status: HYLRA_OK (0) or a negative
 *    hylra_error_t.  Bad arguments are detected on the host before anything
 *    is launched; nothing is written in that case.
 *  * Device entry points are asynchronous on the caller's stream.  They never
 *    allocate, never synchronise and keep no state between calls; the caller
 *    owns every buffer.  Data problems found on the device (a sequence length
 *    beyond the cache, a block index out of range, a duplicate index) never
 *    trap: the kernel skips the offending work and sets a bit in the status
 *    word of the workspace, read with hylra_read_status.
 *  * Shapes: B sequences, Hq query heads, Hkv KV heads (r = Hq / Hkv in
 *    1..8; q-head g reads KV head g / r), head_dim d = 128, block = 128 tokens.
 *    n_b = seqlens[b], NB_b = ceil(n_b / 128), k' = min(k, NB_b).
 *  * q: [B][Hq][d] (bf16 or fp32, see dtype), out: [B][Hq][d] fp32.
 *  * K, V: dense [B][Hkv][kv_capacity][d] (kv_capacity > 0), or packed
 *    [Hkv][total_tokens][d] with sequence b at rows seq_offsets[b] ..
 *    seq_offsets[b] + n_b - 1 of every KV-head plane (kv_capacity == 0).
 *    Device pointers must be 16-byte aligned.
 *  * top-k indices: int32 [B][Hkv][k], in rank order (largest block
 *    attention mass first, lower block index first among equal fp32 scores);
 *    slots k'..k-1 hold -1.
 *  * One workspace may be used by one stream at a time.  It must be zeroed
 *    once (hylra_workspace_init) before its first use; every call leaves it
 *    ready for the next one.
 */
#ifndef HYLRA_H_
#define HYLRA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* hylra_stream_t;

#define HYLRA_BLOCK_TOKENS 128
#define HYLRA_HEAD_DIM 128
#define HYLRA_MAX_GROUP 8          /* largest Hq / Hkv                      */
#define HYLRA_MAX_BATCH 1024
#define HYLRA_MAX_TOPK 1024
#define HYLRA_MAX_SEQLEN 262144    /* 2048 blocks per sequence              */

typedef enum {
  HYLRA_OK = 0,
  HYLRA_ERR_INVALID = -1,      /* null pointer, bad size, misaligned pointer   */
  HYLRA_ERR_UNSUPPORTED = -2,  /* d != 128, block != 128, r > 8, limits above  */
  HYLRA_ERR_CUDA = -3,         /* a CUDA runtime/driver call failed            */
  HYLRA_ERR_WORKSPACE = -4     /* workspace smaller than hylra_workspace_bytes */
} hylra_error_t;

typedef enum { HYLRA_BF16 = 0, HYLRA_FP32 = 1 } hylra_dtype_t;

/* Bits of the device status word (hylra_read_status). */
#define HYLRA_STATUS_BAD_SEQLEN 0x1u   /* n_b < 0, > max_seqlen, or beyond the cache: sequence skipped */
#define HYLRA_STATUS_BAD_INDEX 0x2u    /* reuse index outside [0, NB_b) (and not -1): block skipped    */
#define HYLRA_STATUS_DUP_INDEX 0x4u    /* a block index appears twice in one reuse list               */
#define HYLRA_STATUS_NONFINITE 0x8u    /* a non-finite block score was met (treated as 0)             */
#define HYLRA_STATUS_TIMEOUT 0x10u     /* a bounded wait inside a kernel gave up                      */

typedef struct hylra_shape {
  int32_t batch;         /* B, 1..HYLRA_MAX_BATCH                                        */
  int32_t num_q_heads;   /* Hq                                                           */
  int32_t num_kv_heads;  /* Hkv; Hq % Hkv == 0 and Hq / Hkv <= HYLRA_MAX_GROUP          */
  int32_t head_dim;      /* must be 128                                                   */
  int32_t block_size;    /* must be 128 (HyLRA summary §2.4)                              */
  int32_t topk;          /* k, 1..HYLRA_MAX_TOPK                                          */
  int32_t dtype;         /* hylra_dtype_t of q, K and V                                   */
  int32_t max_seqlen;    /* upper bound on every seqlens[b]; sizes the workspace          */
  int64_t kv_capacity;   /* dense: rows per (b, KV head) plane (>= max_seqlen); 0: packed */
  int64_t total_tokens;  /* packed: rows per KV-head plane; ignored when dense           */
  const int64_t* seq_offsets; /* packed: device int64 [B]; ignored when dense            */
} hylra_shape_t;

/* Bytes of workspace the decode calls need for this shape on the current
 * device (it depends on the device's SM count).  Host only. */
int hylra_workspace_bytes(const hylra_shape_t* shape, size_t* bytes);

/* Zero a workspace (async cudaMemsetAsync on stream).  Needed once. */
int hylra_workspace_init(void* workspace, size_t bytes, hylra_stream_t stream);

/* Reset layer (HyLRA summary §2.3 "Sensitive Layers"): full single-query
 * GQA attention over every cached token, plus the per-KV-head top-k of the
 * 128-token blocks ranked by attention probability mass (summed over the r
 * q-heads of the KV head).  seqlens: device int32 [B].  out: device fp32
 * [B][Hq][d].  topk_out: device int32 [B][Hkv][k].  A sequence with n_b == 0
 * gets a zero output and all -1 indices. */
int hylra_decode_full(const hylra_shape_t* shape, const void* q, const void* K,
                      const void* V, const int32_t* seqlens, float* out,
                      int32_t* topk_out, void* workspace, size_t workspace_bytes,
                      hylra_stream_t stream);

/* Reuse layer (HyLRA summary §2.3 "Tolerant Layers"): attention restricted
 * to the blocks listed in topk_in (device int32 [B][Hkv][k], as written by
 * hylra_decode_full of an earlier layer), softmax renormalised over those
 * tokens.  Only slots 0..k'-1 are read; -1 entries are skipped; an empty
 * selection gives a zero output.  seqlens masks a partial last block. */
int hylra_decode_reuse(const hylra_shape_t* shape, const void* q, const void* K,
                       const void* V, const int32_t* seqlens, const int32_t* topk_in,
                       float* out, void* workspace, size_t workspace_bytes,
                       hylra_stream_t stream);

/* One decode step over num_layers layers (HyLRA summary §2.3): layer l runs
 * hylra_decode_full when policy[l] == 1 (writing topk + l*B*Hkv*k) and
 * hylra_decode_reuse when policy[l] == 0 (reading the slot of the most recent
 * reset layer).  policy[0] must be 1.  q, K, V, out: HOST arrays of
 * num_layers DEVICE pointers.  topk: device int32 [num_layers][B][Hkv][k];
 * slots of reuse layers are left untouched.  Capturable in a CUDA graph.
 * Layers are ordered as in a model, where a layer's query and its newest
 * K/V row are computed from the previous layer's output: layer l > 0 reads
 * q[l] and the block holding each sequence's newest token only after layer
 * l-1's kernels have completed (its kernels are launched early, as
 * programmatic dependents, and may only stage older K/V blocks before
 * that).  The step time is thus a sum of per-layer latencies. */
int hylra_decode_step(const hylra_shape_t* shape, int32_t num_layers,
                      const uint8_t* policy, const void* const* q,
                      const void* const* K, const void* const* V,
                      const int32_t* seqlens, float* const* out, int32_t* topk,
                      void* workspace, size_t workspace_bytes, hylra_stream_t stream);

/* Index-guided offloading (HyLRA summary §2.4 "Index-Guided Offloading":
 * when the KV cache exceeds device memory, the reused indices name the only
 * blocks a tolerant layer needs, so only those cross the host link).
 *
 * A host-resident cache has the same layout as a device cache (dense or
 * packed, bf16) but lives in pinned host memory the device can address
 * (cudaHostAlloc / cudaHostRegister with mapping; on systems with unified
 * addressing the host pointer itself is passed).  The staging cache is a
 * device buffer [B][Hkv][k][128][d] bf16 (hylra_stage_bytes each for K and
 * V); its slot e of (b, h) holds block topk_in[b][h][e]. */

/* Bytes of one staging cache (K or V) for this shape.  bf16 only. */
int hylra_stage_bytes(const hylra_shape_t* shape, size_t* bytes);

/* Copy the blocks listed in topk_in (device int32 [B][Hkv][k]; slots
 * 0..k'-1, -1 and out-of-range entries skipped) from the host-resident
 * K_host / V_host into the staging caches K_stage / V_stage (device); only
 * a block's valid rows are copied.  Asynchronous on stream. */
int hylra_gather_blocks(const hylra_shape_t* shape, const void* K_host, const void* V_host,
                        const int32_t* seqlens, const int32_t* topk_in, void* K_stage,
                        void* V_stage, hylra_stream_t stream);

/* hylra_decode_reuse over staging caches written by hylra_gather_blocks with
 * the same topk_in: same result as hylra_decode_reuse on the original cache. */
int hylra_decode_reuse_staged(const hylra_shape_t* shape, const void* q, const void* K_stage,
                              const void* V_stage, const int32_t* seqlens,
                              const int32_t* topk_in, float* out, void* workspace,
                              size_t workspace_bytes, hylra_stream_t stream);

/* hylra_decode_step where offloaded[l] == 1 marks a reuse layer whose K[l],
 * V[l] are host-resident.  K_stage and V_stage (device) each hold TWO
 * staging slots of hylra_stage_bytes; the offloaded layers use them in turn.
 * A second stream owned by the library (one per host thread and device,
 * created by the thread's first call, which should therefore not be inside a
 * stream capture) prefetches: each offloaded layer's reused blocks cross the
 * host link as soon as the indices it reuses exist (its reset layer is done)
 * and its slot is free (the offloaded layer two before it is done), while
 * the layers run.  The block holding each sequence's newest token is copied
 * again after the preceding layer (in a model that layer writes the newest
 * row), then the layer runs on its slot.  `stream` waits for the second
 * stream at the end; capturable in a CUDA graph.  Reset layers must be
 * device-resident (HYLRA_ERR_INVALID otherwise).  offloaded: HOST uint8
 * [num_layers].  bf16 only. */
int hylra_decode_step_offload(const hylra_shape_t* shape, int32_t num_layers,
                              const uint8_t* policy, const void* const* q,
                              const void* const* K, const void* const* V,
                              const uint8_t* offloaded, const int32_t* seqlens,
                              float* const* out, int32_t* topk, void* K_stage, void* V_stage,
                              void* workspace, size_t workspace_bytes, hylra_stream_t stream);

/* The same step with the per-step inputs and outputs in HOST memory:
 * q_host [num_layers][B][Hq][d] is copied to q_dev (same shape, device) and
 * out_dev [num_layers][B][Hq][d] fp32 to out_host and topk_dev
 * [num_layers][B][Hkv][k] to topk_host (either host pointer may be NULL to
 * skip that copy).  The copies overlap the layers: they run on a second
 * stream owned by the library (one per host thread and device, created by
 * the thread's first call, which should therefore not be inside a stream
 * capture), with event dependencies on `stream`, which has waited for all of
 * them when the call's work on it completes.  Host buffers should be pinned
 * for asynchronous copies.  Returns after enqueueing; synchronise the stream
 * before reading the host outputs. */
int hylra_decode_step_host(const hylra_shape_t* shape, int32_t num_layers,
                           const uint8_t* policy, const void* q_host, void* q_dev,
                           const void* const* K, const void* const* V,
                           const int32_t* seqlens, float* out_dev, float* out_host,
                           int32_t* topk_dev, int32_t* topk_host, void* workspace,
                           size_t workspace_bytes, hylra_stream_t stream);

/* Overlap matrix (HyLRA summary §2.2 "Similarity Matrix Construction").
 * topk: HOST int32 [num_layers][num_sets][k] index sets from a profiling run
 * in which every layer is a reset layer (num_sets = profiled steps x B x Hkv),
 * -1 padded.  M: HOST double [num_layers][num_layers], row = target layer t,
 * column = source layer s <= t: M[t][s] = sum_u |I_s(u) & I_t(u)| /
 * sum_u |I_t(u)| (pooled overlap ratio).  Diagonal 1 (0 for a layer with no
 * valid sets); upper triangle 0.  Synchronous. */
int hylra_similarity(int32_t num_layers, int32_t num_sets, int32_t k,
                     const int32_t* topk, double* M);

/* The two integer sums behind hylra_similarity (same topk argument):
 * inter: HOST int64 [num_layers][num_layers], inter[t][s] =
 * sum_u |I_s(u) & I_t(u)| for s <= t (0 above the diagonal); total: HOST
 * int64 [num_layers], total[t] = sum_u |I_t(u)|.  Both are sums over the
 * index sets, so the counts of disjoint groups of sets (for example the KV
 * heads profiled on different GPUs) add up exactly to the counts of all of
 * them; hylra_similarity_from_counts then gives the same M as
 * hylra_similarity over all the sets, bit for bit.  Synchronous. */
int hylra_overlap_counts(int32_t num_layers, int32_t num_sets, int32_t k,
                         const int32_t* topk, int64_t* inter, int64_t* total);

/* M[t][s] = inter[t][s] / total[t] for s <= t (0 where total[t] == 0, and
 * above the diagonal); counts as written by hylra_overlap_counts (or their
 * sums over groups of sets).  HYLRA_ERR_INVALID for counts no set of index
 * lists can give (negative, inter[t][s] > total[t], nonzero above the
 * diagonal).  Synchronous. */
int hylra_similarity_from_counts(int32_t num_layers, const int64_t* inter,
                                 const int64_t* total, double* M);

/* Token-level profiling (HyLRA summary §2.2 "Similarity Matrix Construction"
 * speaks of top-k *token* indices; the decode path selects 128-token blocks,
 * §2.4).  A reset layer exactly as hylra_decode_full (out and topk_out are
 * written the same way), plus the attention mass of every cached token
 * summed over the r q-heads of its KV head: scores[b][h][t] =
 * sum_g p_{g,t} for t < n_b, 0 for n_b <= t < max_seqlen.  scores: device
 * fp32 [B][Hkv][max_seqlen].  For profiling runs (CUDA cores, two extra
 * kernels that re-read K), not for the decode step.  B * Hkv <= 65535. */
int hylra_token_scores(const hylra_shape_t* shape, const void* q, const void* K,
                       const void* V, const int32_t* seqlens, float* out,
                       int32_t* topk_out, float* scores, void* workspace,
                       size_t workspace_bytes, hylra_stream_t stream);

/* Top-k entries of each of num_lists score lists (host): scores HOST fp32
 * [num_lists][n], lengths HOST int32 [num_lists] (entries 0..lengths[u]-1 of
 * list u are valid; NULL: all n), topk HOST int32 [num_lists][k]: indices in
 * rank order (score descending, lower index first among equal scores),
 * padded with -1.  Scores must be finite and >= 0 (HYLRA_ERR_INVALID
 * otherwise, nothing written).  With hylra_token_scores' output this gives
 * the token-level index sets; hylra_similarity takes them as it takes block
 * sets.  Synchronous. */
int hylra_token_topk(int32_t num_lists, int32_t n, const float* scores,
                     const int32_t* lengths, int32_t k, int32_t* topk);

/* Policy (HyLRA summary §2.2 "Dynamic Programming").  States (i, j): layer j
 * uses the indices of reset layer i; layer 0 is a reset.  Reset jump
 * (i, j) -> (j+1, j+1); vertical move (i, j) -> (i, j+1) allowed when
 * M[j+1][i] > theta (strict), adding M[j+1][i] to the cumulative similarity.
 * Optimum: fewest resets, then largest cumulative similarity (summed in layer
 * order), then the lexicographically smallest policy with reuse < reset.
 * policy: HOST uint8 [num_layers] (1 = reset, 0 = reuse).  num_resets and
 * cum_similarity may be NULL.  Synchronous. */
int hylra_dp_policy(int32_t num_layers, const double* M, double theta,
                    uint8_t* policy, int32_t* num_resets, double* cum_similarity);

/* Static policy (HyLRA summary §4 "Results": the Jump3 baseline, "a static
 * variant with fixed jump steps"; read as a reset every `period` layers,
 * Jump3 = period 3): policy[l] = 1 when l % period == 0, else 0, for
 * l < num_layers.  policy: HOST uint8 [num_layers]; num_resets may be NULL.
 * period >= 1.  Synchronous; no similarity threshold is applied. */
int hylra_static_policy(int32_t num_layers, int32_t period, uint8_t* policy,
                        int32_t* num_resets);

/* hylra_decode_full without a caller-supplied workspace.  The paper has no
 * counterpart: this exists for callers that cannot allocate device memory
 * when they call (a process that reserved all free device memory up front,
 * code that must not call cudaMalloc because it synchronises the device, or
 * a binding with nowhere to keep a workspace alive).  It allocates nothing:
 * its scratch is an 8 MiB array compiled into the library, present on every
 * device that loads the library until the process exits.
 *  - Same arguments, layouts and results as hylra_decode_full; shapes whose
 *    workspace (hylra_workspace_bytes) exceeds 8 MiB return
 *    HYLRA_ERR_WORKSPACE before anything is launched.
 *  - status_out: optional DEVICE uint32 that receives the call's status word
 *    (HYLRA_STATUS_* bits); NULL to skip.
 *  - The first call on a device looks up the scratch's device address; make
 *    that first call before any stream capture on that device.
 *  - Every call on a device shares the one scratch array: calls that can
 *    overlap on the GPU (other streams, other host threads) race; serialise
 *    them, e.g. on one stream. */
int hylra_decode_full_noalloc(const hylra_shape_t* shape, const void* q, const void* K,
                              const void* V, const int32_t* seqlens, float* out,
                              int32_t* topk_out, uint32_t* status_out, hylra_stream_t stream);

/* Failure detection.  Every wait inside the kernels (for a TMA copy, a
 * pipeline stage, a peer CTA's data) gives up after a limit of SM clocks,
 * 2^31 (about a second) by default; the kernel then stops issuing copies,
 * waits (bounded) for the copies it already issued, finishes without trusting
 * the data it did not get, and sets HYLRA_STATUS_TIMEOUT in the workspace
 * status word (hylra_read_status).  Its outputs are then meaningless; the
 * workspace, cleared with hylra_read_status(..., clear = 1), serves the next
 * call as before.  This sets the limit for launches made after the call
 * (process-wide; a CUDA graph keeps the limit it was captured with);
 * cycles <= 0 restores the default.  A short limit makes a watchdog fire on a
 * healthy GPU: tests use that to exercise the path.  Always HYLRA_OK. */
int hylra_set_wait_limit(int64_t cycles);

/* Copy the workspace status word to *status (synchronises the stream); when
 * clear != 0 the word is reset to 0 afterwards. */
int hylra_read_status(void* workspace, uint32_t* status, int clear,
                      hylra_stream_t stream);

/* Static string for a hylra_error_t value. */
const char* hylra_strerror(int err);

/* Library version, e.g. 100 for 0.1.0. */
int hylra_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HYLRA_H_ */
