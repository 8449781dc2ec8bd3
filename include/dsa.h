/*
 * dsa.h -- C ABI of libdsa: DSA-style sparse attention on NVIDIA B200 (sm_100a).
 *
 * The path has three steps, each one call, all sharing one batch descriptor
 * (dsa_batch_t) so that index selection and attention resolve tokens through
 * the same block table ("Day-0 Adaptation: Running Trillion-Parameter Models
 * on Domestic AI Accelerators", 3.1 Index Selection Operator: selection and
 * attention share the block-mapping semantics; 3.2 KV Cache Layout: paged
 * cache, block table from logical to physical blocks):
 *
 *   dsa_indexer_scores       I(t,s) = sum_j w[t,j] * ReLU(qI[t,j] . kI[s]) for s <= pos(t)
 *   dsa_topk                 the k best s per query row (ties -> lower s), ascending
 *   dsa_sparse_attn_prefill  softmax attention of every head over the selected rows
 *   dsa_sparse_attn_decode   the same, specialised for one query row per sequence
 *   dsa_cache_append         writes the batch's new tokens into the paged pools (FP8 keys)
 *
 * ("Day-0 Adaptation for LLMs: Implementing Sparse Attention and Low-Precision
 * Weights", III.1 Index Selection Path and the decode sketch: score -> topk ->
 * gather -> attention; III.3 and "Engineering Practices for Day-0 Adaptation of
 * Million-Token Context Models on Domestic AI Chips", Four Key Layers 3:
 * separate prefill and decode paths.)
 *
 * Around them: dsa_indexer_scores_append (the cache append fused into the indexer's first kernel); two
 * approximate selection variants, block-granular (dsa_block_scores, dsa_expand_blocks) and decode index
 * reuse (dsa_reuse_candidates, dsa_indexer_scores_at, dsa_gather_positions), both ending in dsa_topk;
 * the steps of context-parallel decode across GPUs (dsa_cp_*); and a self-test of the bounded device
 * waits (dsa_selftest_wait_timeout).
 *
 * Conventions shared by every call
 * --------------------------------
 * Ownership: the caller owns every buffer.  Pointers inside dsa_batch_t and all
 *   tensor arguments are DEVICE pointers (cudaMalloc'd or equivalent) unless a
 *   parameter says otherwise.  The library allocates no memory and keeps no
 *   state beyond cached device attributes; calls are thread-safe.
 * Asynchrony: every compute call only enqueues work on `stream` (a cudaStream_t
 *   passed as void*; NULL is the legacy default stream) and returns without
 *   synchronising the host.  Outputs are valid once the stream reaches them.
 *   Kernels are launched with programmatic dependent launch: one may be scheduled
 *   while the preceding work on the stream finishes, but it touches no global
 *   memory until that work has completed, so stream order holds as usual.
 * Errors: argument errors are detected on the host before anything is enqueued
 *   and return DSA_ERR_INVALID_ARG / DSA_ERR_UNSUPPORTED / DSA_ERR_WORKSPACE with
 *   nothing written.  A failed launch returns DSA_ERR_CUDA.  Kernels never spin
 *   without bound: a device wait that runs out sets a bit in the workspace status
 *   word, which dsa_read_device_status() reports as DSA_ERR_TIMEOUT.  No C++
 *   exception crosses this ABI.  dsa_last_error() returns a one-line description
 *   of the last failure on the calling thread.
 * Rows: query rows are packed sequence after sequence; sequence b owns rows
 *   cu_q[b] .. cu_q[b+1]-1, which are its LAST n_b = cu_q[b+1]-cu_q[b] tokens:
 *   row cu_q[b]+i sits at absolute position pos = seq_lens[b] - n_b + i and may
 *   attend to positions 0..pos (its own entry is already in the cache).
 *   A sequence may own no rows (n_b == 0) anywhere in the batch.  An empty batch
 *   (total_q == 0) is a no-op: every compute call checks the descriptor and returns
 *   DSA_OK without enqueueing anything or needing a device; its data pointers may
 *   then be NULL.
 * Paged cache: token s of sequence b lives in physical block
 *   block_table[b * max_blocks_per_seq + s / page_size], slot s % page_size.
 *   Only entries for s < seq_lens[b] are read.
 *
 * Supported shapes (others return DSA_ERR_UNSUPPORTED):
 *   MLA path    : bf16 q / latent cache, H = 128, Dqk = 576, Dv = 512, V = the first
 *                 512 entries of each latent row (v_pool NULL); FP8 e4m3 indexer with
 *                 Hi = 64, Di = 128 and a per-token fp32 key scale; page_size 64.
 *   fp32 path   : f32 everything, H <= 16, Dqk <= 128, Dv <= 128 with a separate
 *                 V cache, Hi <= 16, Di <= 128, no key scale; page_size 64.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DSA_API __attribute__((visibility("default")))
#else
#define DSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,   /* NULL where a buffer is required, bad sizes, misaligned strides */
  DSA_ERR_UNSUPPORTED = 2,   /* valid request outside the shapes/dtypes listed above */
  DSA_ERR_WORKSPACE = 3,     /* ws_bytes smaller than dsa_workspace_size() */
  DSA_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed */
  DSA_ERR_DEVICE_CHECK = 5,  /* a kernel found an out-of-range block id or index */
  DSA_ERR_TIMEOUT = 6        /* a bounded device wait ran out (kernel gave up, outputs invalid) */
} dsa_status_t;

typedef enum { DSA_F32 = 0, DSA_BF16 = 1, DSA_FP8_E4M3 = 2 } dsa_dtype_t;

typedef enum {
  DSA_OP_INDEXER = 0,
  DSA_OP_TOPK = 1,
  DSA_OP_ATTN_PREFILL = 2,
  DSA_OP_ATTN_DECODE = 3,
  DSA_OP_CACHE_APPEND = 4,
  DSA_OP_INDEXER_TOPK = 5
} dsa_op_t;

/* Batch descriptor shared by every call.  The three host integers at the end are
 * upper bounds the caller already knows; they size grids without a device->host
 * read.  They must hold: total_q == cu_q[num_seqs], max_q_per_seq >= every n_b,
 * max_seq_len >= every seq_lens[b]. */
typedef struct {
  int32_t num_seqs;            /* B >= 1 */
  int32_t page_size;           /* tokens per block: 64 */
  int32_t num_blocks;          /* physical blocks in each pool */
  int32_t max_blocks_per_seq;  /* row stride of block_table */
  const int32_t *block_table;  /* device [num_seqs, max_blocks_per_seq], values in [0, num_blocks) */
  const int32_t *seq_lens;     /* device [num_seqs], cached tokens including the query rows' own */
  const int32_t *cu_q;         /* device [num_seqs + 1], cu_q[0] = 0, non-decreasing */
  int32_t total_q;             /* host: cu_q[num_seqs] */
  int32_t max_q_per_seq;       /* host: >= max_b (cu_q[b+1] - cu_q[b]) */
  int32_t max_seq_len;         /* host: >= max_b seq_lens[b] */
} dsa_batch_t;

/* Bytes of workspace `op` needs for this batch.  k = top-k count, H / Dv = attention
 * heads and value width (ignored by INDEXER and TOPK).  The workspace is caller-owned
 * device memory, 256-byte aligned, reused freely between calls on one stream; calls
 * that may run concurrently need separate workspaces. */
DSA_API dsa_status_t dsa_workspace_size(dsa_op_t op, const dsa_batch_t *b, int32_t k, int32_t H, int32_t Dv,
                                size_t *bytes);

/* Indexer scores ("Day-0 Adaptation for LLMs ...", III.1 Index Selection Path; V keeps
 * index scoring at BF16/FP32: products of the FP8 inputs are exact, accumulation and the
 * result are fp32).
 *   q_idx   [total_q, Hi, Di] of q_dt (DSA_FP8_E4M3 or DSA_F32)
 *   w       [total_q, Hi] f32 per-head weights (any sign)
 *   k_idx_pool [num_blocks, page_size, Di] of k_dt (same dtype as q_dt)
 *   k_scale_pool [num_blocks, page_size] f32 > 0, required for FP8 keys, NULL for f32
 *   scores  [total_q, ld_scores] f32 output; ld_scores >= max_seq_len, multiple of 4.
 * Writes scores[row, s] = kS[s] * sum_j w[row,j] * max(0, sum_d qI[row,j,d] * kI8[s,d])
 * for s = 0..pos(row); entries s > pos(row) are left untouched. */
DSA_API dsa_status_t dsa_indexer_scores(const void *q_idx, dsa_dtype_t q_dt, const float *w,
                                const void *k_idx_pool, dsa_dtype_t k_dt, const float *k_scale_pool,
                                int32_t Hi, int32_t Di, const dsa_batch_t *b,
                                float *scores, int64_t ld_scores,
                                void *ws, size_t ws_bytes, void *stream);

/* Top-k selection ("Day-0 Adaptation for LLMs ...", III.1: top-k over long sequences;
 * decode sketch idx = topk(score, k)).  For each row, with n = pos(row) + 1 candidates
 * scores[row, 0..n): if n <= k every position is selected, else the first k positions
 * of the order (score descending, position ascending).  -0 and +0 compare equal; scores
 * must be finite.  Output idx [total_q, k] int32: selected positions in ascending
 * order, padded with -1.  The selection is exact (fp32 keys compared as integers). */
DSA_API dsa_status_t dsa_topk(const float *scores, int64_t ld_scores, const dsa_batch_t *b, int32_t k,
                      int32_t *idx, void *ws, size_t ws_bytes, void *stream);

/* Indexer scores and top-k selection in one call, the selection fused into the scoring ("Day-0 Adaptation:
 * Running Trillion-Parameter Models on Domestic AI Accelerators", 3.1 Index Selection Operator: scoring,
 * threshold filtering and index gathering in one operator so that the scores are not walked repeatedly in
 * global memory; "Engineering Practices ...", Four Key Layers 1).  Same arguments and results as
 * dsa_indexer_scores followed by dsa_topk: scores[row, s] for s <= pos(row) as dsa_indexer_scores writes
 * them (kept, so callers may reuse them), and idx [total_q, k] as dsa_topk defines it (bit for bit the same
 * selection).  For the e4m3 indexer, the scoring kernel also counts the leading 11 bits of every score's
 * order-preserving key per row (a 2048-bin histogram in the workspace), so the selection starts from the
 * threshold digit and reads each row's scores once, keeping only the keys at or above it.  The f32 indexer
 * takes the same selection kernel, which then counts the leading digit itself first.
 * Batches of at most 16 rows whose longest row has 262,144 candidates or more first gather each row's
 * survivors (keys at or above the threshold digit) over all SMs, then finish one row per CTA.
 * Workspace: dsa_workspace_size(DSA_OP_INDEXER_TOPK) (the indexer's plus 8 KB per query row, plus 640 KB of
 * survivor slots for such long-row batches); its status word also reports a selection that ran past its
 * shared-memory capacity (DSA_ERR_DEVICE_CHECK; cannot happen with a histogram written by this call). */
DSA_API dsa_status_t dsa_indexer_topk(const void *q_idx, dsa_dtype_t q_dt, const float *w, const void *k_idx_pool,
                                      dsa_dtype_t k_dt, const float *k_scale_pool, int32_t Hi, int32_t Di,
                                      const dsa_batch_t *b, int32_t k, float *scores, int64_t ld_scores, int32_t *idx,
                                      void *ws, size_t ws_bytes, void *stream);

/* Allocation-free top-k: the selection of dsa_topk ("Day-0 Adaptation for LLMs ...", III.1: top-k over
 * long sequences; decode sketch idx = topk(score, k)) with arguments and output as there, but no
 * workspace.  The source pages have no allocation-free variant; this entry point exists for callers
 * that cannot allocate device memory for a workspace -- code that runs where cudaMalloc is not allowed
 * or not wanted (a plugin or custom operator handed only a stream, a framework whose memory is owned
 * by its own pool, a latency-critical path that must not trigger an allocation and its implicit device
 * synchronisation).  Same selection and output as dsa_topk, but its scratch is a fixed device array
 * inside the library (about 2.3 MB per device, held until the process exits) instead of a caller
 * workspace.  Limits: total_q <= 256 rows and max_seq_len <= 1,048,576 candidates; larger batches return
 * DSA_ERR_UNSUPPORTED with nothing enqueued.  The first call on a device looks up the array's device
 * address (cudaGetSymbolAddress) and caches it for that device's current context; make that first call
 * outside any stream capture.  After a device reset (cudaDeviceReset) the next call finds a new context
 * and looks the address up again, so that call, too, should come before any capture.  All calls share
 * the one array, so calls whose GPU work overlaps (different streams, concurrent host threads) race on
 * it; serialise them on one stream.  The selection kernels report no device status, so there is no
 * status word to read back.  Allocates nothing: no cudaMalloc/cudaFree. */
DSA_API dsa_status_t dsa_topk_noalloc(const float *scores, int64_t ld_scores, const dsa_batch_t *b, int32_t k,
                                      int32_t *idx, void *stream);

/* Sparse attention, prefill / any batch ("Day-0 Adaptation for LLMs ...", decode sketch:
 * gather the selected KV and run exact attention; "Day-0 Model Adaptation Depends on the
 * Compute Software Stack", Operator Library Abstraction: query, key-value pairs and index
 * list in, context vector out).  For every row and head h:
 *   z_i = softmax_scale * q[row,h,:Dqk] . K[idx_i]   over valid idx_i (>= 0)
 *   out[row,h,:] = sum_i exp(z_i - m) V[idx_i] / sum_i exp(z_i - m),  m = max z
 *   lse[row,h]   = m + ln(sum_i exp(z_i - m))            (natural log; -inf if no idx)
 * K[s] = kv_pool row of token s (first Dqk entries); V[s] = first Dv entries of the
 * same row when v_pool is NULL, else the v_pool row.
 *   q       [total_q, H, Dqk] of dt;  kv_pool [num_blocks, page_size, Dqk] of dt
 *   v_pool  NULL (MLA) or [num_blocks, page_size, Dv] of dt
 *   idx     [total_q, k] int32 logical positions in [0, seq_len) or -1 (skipped)
 *   out     [total_q, H, Dv] of dt (bf16 for the MLA path);  lse [total_q, H] f32 or NULL */
DSA_API dsa_status_t dsa_sparse_attn_prefill(const void *q, dsa_dtype_t dt, const void *kv_pool, const void *v_pool,
                                     int32_t H, int32_t Dqk, int32_t Dv, float softmax_scale,
                                     const int32_t *idx, int32_t k, const dsa_batch_t *b,
                                     void *out, float *lse, void *ws, size_t ws_bytes, void *stream);

/* Sparse attention, decode: same contract as dsa_sparse_attn_prefill, for batches where
 * every sequence has exactly one query row (cu_q[b] = b); splits each row's key set over
 * several CTAs and merges the partial results (log-sum-exp combine), as the pages' prefill
 * unit does across KV blocks ("Engineering Practices ...", Four Key Layers 3).  A batch
 * with total_q != num_seqs returns DSA_ERR_INVALID_ARG. */
DSA_API dsa_status_t dsa_sparse_attn_decode(const void *q, dsa_dtype_t dt, const void *kv_pool, const void *v_pool,
                                    int32_t H, int32_t Dqk, int32_t Dv, float softmax_scale,
                                    const int32_t *idx, int32_t k, const dsa_batch_t *b,
                                    void *out, float *lse, void *ws, size_t ws_bytes, void *stream);

/* Cache append ("Engineering Practices ...", Four Key Layers 3: the decode step writes the
 * new token into the KV cache; Four Key Layers 2: the block table places it; "Day-0
 * Adaptation for LLMs ...", III.1: FP8 indexer keys).  Every query row of the batch is a new
 * token, at the position the other calls give it (row cu_q[b] + i is token
 * seq_lens[b] - n_b + i of sequence b, so seq_lens already counts the new tokens).  For each:
 *   kv_pool[token]      = kv_new[row]                         (576 bf16, copied bit for bit)
 *   k_scale_pool[token] = max_d |k_new[row, d]| / 448          (fp32; 1 if that is 0)
 *   k_idx_pool[token,d] = E4M3(k_new[row, d] / scale)          (fp32 quotient, round to nearest
 *                                                                even, saturating at +-448)
 *   kv_new      [total_q, Dqk] of kv_dt;   k_new [total_q, Di] of k_dt (f32 or bf16, finite)
 *   kv_pool     [num_blocks, page_size, Dqk];  k_idx_pool [num_blocks, page_size, Di] e4m3;
 *   k_scale_pool [num_blocks, page_size] f32
 * Supported: kv_dt bf16 with Dqk = 576, Di = 128 (the MLA path's pools).  kv_new, k_new,
 * kv_pool and k_idx_pool 16-byte aligned.  The workspace only carries the status word
 * (dsa_workspace_size(DSA_OP_CACHE_APPEND) = 256 bytes): a block id outside [0, num_blocks)
 * or a position outside the block table leaves that token unwritten and is reported by
 * dsa_read_device_status as DSA_ERR_DEVICE_CHECK.  Two rows that map to the same token race. */
DSA_API dsa_status_t dsa_cache_append(const void *kv_new, dsa_dtype_t kv_dt, const void *k_new, dsa_dtype_t k_dt,
                                      int32_t Dqk, int32_t Di, const dsa_batch_t *b, void *kv_pool,
                                      void *k_idx_pool, float *k_scale_pool, void *ws, size_t ws_bytes,
                                      void *stream);

/* Synchronises `stream`, then reads and clears the status word at the start of a
 * workspace used by the calls above: DSA_OK, DSA_ERR_TIMEOUT or DSA_ERR_DEVICE_CHECK. */
DSA_API dsa_status_t dsa_read_device_status(void *ws, void *stream);

/* Block-granular selection ("Day-0 Adaptation: Running Trillion-Parameter Models on Domestic AI
 * Accelerators", 3.1: the selection operator's top-k counts key-value blocks).  A variant of the
 * token-granular path, approximate by design:
 * dsa_block_scores: for every query row, blk_scores[row, p] = max over the causal tokens s of page p
 *   (s <= pos(row)) of scores[row, s], for p < ceil((pos + 1) / page_size), and blk_lens[row] = that page
 *   count.  blk_scores [total_q, ld_blk] f32 (ld_blk >= pages of max_seq_len, multiple of 4, 16-byte
 *   aligned), blk_lens [total_q] int32.
 * dsa_topk over blk_scores, with a batch of total_q sequences of blk_lens[row] candidates (one query row
 *   each, cu_q = 0..total_q), keeps kb pages per row, ties to the lower page.
 * dsa_expand_blocks: idx[row, i*page_size + j] = blk_idx[row, i]*page_size + j when blk_idx[row, i] is a
 *   page of the row and that position is <= pos(row), else -1.  idx [total_q, kb*page_size] feeds either
 *   attention call with k = kb*page_size. */
DSA_API dsa_status_t dsa_block_scores(const float *scores, int64_t ld_scores, const dsa_batch_t *b, float *blk_scores,
                                      int64_t ld_blk, int32_t *blk_lens, void *stream);
DSA_API dsa_status_t dsa_expand_blocks(const int32_t *blk_idx, int32_t kb, const dsa_batch_t *b, int32_t *idx,
                                       void *stream);

/* Cache append fused with the indexer ("Engineering Practices ...", Four Key Layers 3: the decode step
 * merges the KV cache update into its sparse-attention launches): dsa_cache_append's writes (new tokens'
 * latent rows and quantised indexer keys, same arguments and layouts) and then dsa_indexer_scores over
 * the updated pools, in one call.  For batches of up to 256 query rows the append runs inside the
 * indexer's first kernel; larger batches get a separate append launch ahead of it.  The workspace is the
 * indexer's (dsa_workspace_size(DSA_OP_INDEXER)); its status word also reports the append's bad block ids. */
DSA_API dsa_status_t dsa_indexer_scores_append(const void *kv_new, dsa_dtype_t kv_dt, const void *k_new,
                                               dsa_dtype_t k_new_dt, void *kv_pool, const void *q_idx, dsa_dtype_t q_dt,
                                               const float *w, void *k_idx_pool, dsa_dtype_t k_dt, float *k_scale_pool,
                                               int32_t Hi, int32_t Di, const dsa_batch_t *b, float *scores,
                                               int64_t ld_scores, void *ws, size_t ws_bytes, void *stream);

/* Decode index reuse ("Day-0 Adaptation: Running Trillion-Parameter Models on Domestic AI Accelerators",
 * 3.3: the decode path maintains its indices incrementally and reuses the previous step's result).  A
 * variant of the full selection, approximate by design, for decode batches (one row per sequence):
 * dsa_reuse_candidates: cand[row, j] = prev_idx[row, j] for j < k (entries >= prev_lens[row] become -1),
 *   then prev_lens[row] + (j - k) for the positions added since, -1 past the row's position.  cand
 *   [T, k + max_new]; a row with more than max_new new positions is reported by dsa_read_device_status
 *   as DSA_ERR_DEVICE_CHECK (its extra positions are not candidates).
 * dsa_indexer_scores_at: cand_scores[row, j] = the indexer score I(row, cand[row, j]) (same definition
 *   as dsa_indexer_scores), -inf for -1 or positions past the row.  e4m3 indexer, Hi = 64, Di = 128.
 * dsa_topk over cand_scores (a batch of T sequences of m candidates, one query row each; m a multiple of
 *   4) keeps k slots, ties to the earlier slot (the lower position).
 * dsa_gather_positions: idx[row, j] = cand[row, sel[row, j]] (-1 for -1), for either attention call. */
DSA_API dsa_status_t dsa_reuse_candidates(const int32_t *prev_idx, int32_t k, const int32_t *prev_lens, int32_t max_new,
                                          const dsa_batch_t *b, int32_t *cand, void *ws, size_t ws_bytes, void *stream);
DSA_API dsa_status_t dsa_indexer_scores_at(const void *q_idx, dsa_dtype_t q_dt, const float *w, const void *k_idx_pool,
                                           dsa_dtype_t k_dt, const float *k_scale_pool, int32_t Hi, int32_t Di,
                                           const dsa_batch_t *b, const int32_t *cand, int32_t m, float *cand_scores,
                                           void *ws, size_t ws_bytes, void *stream);
DSA_API dsa_status_t dsa_gather_positions(const int32_t *sel, int32_t k, const int32_t *cand, int32_t m, int32_t T,
                                          int32_t *idx, void *stream);

/* Context-parallel decode ("Engineering Practices ...", Four Key Layers 3: partial attention over
 * disjoint key sets merged by a log-sum-exp reduction, here across GPUs).  Every sequence of a decode
 * batch (one query row per sequence, T rows) is spread over G ranks, rank r holding the contiguous token
 * range [lo[t], hi[t]) of row t's sequence, ranks in ascending order of their ranges.  Each rank runs
 * dsa_indexer_scores and dsa_topk on a batch of its own ranges (local positions), then:
 *
 * dsa_cp_candidates: cand_score[t, j] = scores[t, idx[t, j]], cand_gidx[t, j] = idx[t, j] + offsets[t]
 *   (offsets = lo); idx entries outside [0, ld_scores) give (-inf, -1).  All arrays [T, k], device.
 * After an all-gather of both into [G, T, k]:
 * dsa_cp_rows: rows[t, r*k + j] = g_score[r, t, j], rows [T, ld_rows], ld_rows >= G*k.  dsa_topk over these
 *   rows (a batch of T sequences of G*k candidates, one query row each) picks the global top-k; ties go
 *   to the lower candidate position, which is the lower global position.
 * dsa_cp_select_local: local_idx[t, j] = g - lo[t] where g = g_gidx[p / k, t, p % k] for p = sel[t, j],
 *   if lo[t] <= g < hi[t], else -1.  dsa_sparse_attn_decode over local_idx gives this rank's o_r, lse_r.
 * After an all-gather of those into part_out [G, T, H, Dv] (bf16) and part_lse [G, T, H]:
 * dsa_cp_merge: lse = log sum_r exp(lse_r), out = sum_r exp(lse_r - lse) o_r in fp32, stored as bf16;
 *   ranks with lse_r = -inf contribute nothing; lse may be NULL.
 * Each call only enqueues; T = 0 returns DSA_OK at once. */
DSA_API dsa_status_t dsa_cp_candidates(const float *scores, int64_t ld_scores, const int32_t *idx, int32_t T, int32_t k,
                                       const int32_t *offsets, float *cand_score, int32_t *cand_gidx, void *stream);
DSA_API dsa_status_t dsa_cp_rows(const float *g_score, int32_t G, int32_t T, int32_t k, float *rows, int64_t ld_rows,
                                 void *stream);
DSA_API dsa_status_t dsa_cp_select_local(const int32_t *sel, const int32_t *g_gidx, int32_t G, int32_t T, int32_t k,
                                         const int32_t *lo, const int32_t *hi, int32_t *local_idx, void *stream);
DSA_API dsa_status_t dsa_cp_merge(const void *part_out, dsa_dtype_t dt, const float *part_lse, int32_t G, int32_t T,
                                  int32_t H, int32_t Dv, void *out, float *lse, void *stream);

/* Self-test of the bounded device waits: enqueues one kernel whose thread waits on an mbarrier that
 * nothing completes, through the wait routine every tensor-core kernel uses, with a budget of
 * `budget_cycles` SM cycles (1 .. 4e9; the kernels' own budget is 8e9).  The wait gives up, sets the
 * timeout bit of the workspace status word (ws: at least 256 bytes, 256-byte aligned) and the kernel
 * returns, so dsa_read_device_status(ws) then reports DSA_ERR_TIMEOUT and the context stays usable.
 * No GPU fault is involved. */
DSA_API dsa_status_t dsa_selftest_wait_timeout(uint64_t budget_cycles, void *ws, size_t ws_bytes, void *stream);

DSA_API const char *dsa_status_string(dsa_status_t s);
DSA_API const char *dsa_last_error(void);

/* Number of kernels this library has launched in the process so far (all devices, all
 * threads).  Lets a caller count the library's launches over a region of its own code. */
DSA_API uint64_t dsa_launch_count(void);

/* Library version, "major.minor.patch". */
DSA_API const char *dsa_version(void);

#ifdef __cplusplus
}
#endif
#endif /* DSA_H_ */
