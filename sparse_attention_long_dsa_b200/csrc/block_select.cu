// Block-granular selection: the variant whose top-k counts key-value blocks ("Day-0 Adaptation: Running
// Trillion-Parameter Models on Domestic AI Accelerators", 3.1 Index Selection Operator).
//
// From the indexer's token scores, a page's score is the largest score among its causal tokens; the usual
// top-k then keeps kb pages per query row (a batch whose "sequences" are the rows' page lists), and each
// kept page expands to its token positions for the attention call:
//   block_scores_kernel  one CTA per query row, a warp per page: two coalesced loads per lane, warp max;
//                        also the row's page count (the block batch's sequence length);
//   expand_kernel        one CTA per query row: entry i*64 + j is page_i*64 + j when that position is
//                        causal (<= the row's position), else -1.
// Both read or write a few bytes per candidate and are bound by launch latency at decode sizes.
#include "common.cuh"

namespace dsa {

constexpr int kBlkThreads = 256;

__global__ void __launch_bounds__(kBlkThreads)
block_scores_kernel(const float *__restrict__ scores, int64_t ld, BatchView bv, float *__restrict__ blk,
                    int64_t ld_blk, int32_t *__restrict__ blk_lens) {
  pdl_wait();
  pdl_trigger();
  const int row = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  int b;
  const int pos = pos_of_row_warp(bv, row, &b);      // every warp finds the row's position itself
  const int nb = pos / 64 + 1;
  if (threadIdx.x == 0) blk_lens[row] = nb;
  const float *sr = scores + (int64_t)row * ld;
  for (int p = warp; p < nb; p += nw) {
    const int s0 = 64 * p + lane, s1 = s0 + 32;
    float m = s0 <= pos ? __ldg(sr + s0) : -INFINITY;
    if (s1 <= pos) m = fmaxf(m, __ldg(sr + s1));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) blk[(int64_t)row * ld_blk + p] = m;
  }
}

__global__ void __launch_bounds__(kBlkThreads)
expand_kernel(const int32_t *__restrict__ blk_idx, int kb, BatchView bv, int32_t *__restrict__ idx) {
  pdl_wait();
  pdl_trigger();
  __shared__ int s_pos;
  const int row = blockIdx.x;
  if (threadIdx.x < 32) {
    int b;
    const int pos = pos_of_row_warp(bv, row, &b);
    if (threadIdx.x == 0) s_pos = pos;
  }
  __syncthreads();
  const int pos = s_pos, n = kb * 64;
  const int32_t *br = blk_idx + (int64_t)row * kb;
  int32_t *out = idx + (int64_t)row * n;
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    const int pg = __ldg(br + e / 64);
    const bool ok = pg >= 0 && pg <= pos / 64;               // a page of this row (others read as -1)
    const int s = ok ? 64 * pg + (e & 63) : -1;
    out[e] = (ok && s <= pos) ? s : -1;
  }
}

dsa_status_t block_scores_launch(const float *scores, int64_t ld, const dsa_batch_t *b, float *blk, int64_t ld_blk,
                                 int32_t *blk_lens, cudaStream_t stream) {
  DSA_LAUNCH_PDL("block_scores_kernel", block_scores_kernel, dim3(b->total_q), dim3(kBlkThreads), 0, stream, scores, ld,
                 view_of(b), blk, ld_blk, blk_lens);
  return DSA_OK;
}

dsa_status_t expand_blocks_launch(const int32_t *blk_idx, int kb, const dsa_batch_t *b, int32_t *idx,
                                  cudaStream_t stream) {
  DSA_LAUNCH_PDL("expand_kernel", expand_kernel, dim3(b->total_q), dim3(kBlkThreads), 0, stream, blk_idx, kb,
                 view_of(b), idx);
  return DSA_OK;
}

}  // namespace dsa
