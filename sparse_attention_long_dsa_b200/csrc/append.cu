// Appending new tokens to the paged cache.
//
// Every query row of the batch is a new token of its sequence: row cu_q[b] + i sits at position
// seq_lens[b] - n_b + i, the same convention the indexer, top-k and attention use, so one batch
// descriptor covers the whole decode step ("Engineering Practices for Day-0 Adaptation of
// Million-Token Context Models on Domestic AI Chips", Four Key Layers 3: the decode step writes the
// new token into the KV cache; Four Key Layers 2: the block table places it in its block).
//
// Per token: the 576-entry bf16 latent row is copied into the latent pool, and the 128-entry indexer
// key is stored as FP8 E4M3 with one fp32 scale ("Day-0 Adaptation for LLMs: Implementing Sparse
// Attention and Low-Precision Weights", III.1: low-precision index scoring):
//   scale = max|k| / 448 (1 when that is 0),  code_d = e4m3_rn_satfinite(k_d / scale),
// both divisions IEEE fp32 (append.cuh).  One warp per token; the work is a few hundred bytes per token, so
// the kernel is bound by launch latency for a decode batch and by HBM for a prefill chunk.
#include "append.cuh"

namespace dsa {

constexpr int kAppendWarps = 8;

__global__ void __launch_bounds__(kAppendWarps * 32)
cache_append_kernel(AppendArgs a, BatchView bv, int T, uint32_t *status) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * kAppendWarps + (threadIdx.x >> 5);
  if (row >= T) return;                                   // whole warps leave together
  append_token_warp(a, bv, row, lane, status);
}

dsa_status_t cache_append_launch(const void *kv_new, const void *k_new, bool k_bf16, const dsa_batch_t *b,
                                 void *kv_pool, void *kI_pool, float *kS_pool, void *ws, cudaStream_t stream) {
  const int T = b->total_q;
  const int grid = (T + kAppendWarps - 1) / kAppendWarps;
  const AppendArgs a{(const uint4 *)kv_new, k_new, k_bf16 ? 1 : 0, (uint4 *)kv_pool, (uint32_t *)kI_pool, kS_pool};
  DSA_LAUNCH_PDL("cache_append_kernel", cache_append_kernel, dim3(grid), dim3(kAppendWarps * 32), 0, stream, a,
                 view_of(b), T, (uint32_t *)ws);
  return DSA_OK;
}

}  // namespace dsa
