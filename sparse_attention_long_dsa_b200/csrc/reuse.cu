// Decode index reuse: a decode step that keeps an earlier selection instead of scoring the whole context
// ("Day-0 Adaptation: Running Trillion-Parameter Models on Domestic AI Accelerators", 3.3: the decode path
// maintains its indices incrementally and reuses the previous step's result).
//
// The candidates of a query row are the earlier selection (made when its sequence held prev_len tokens)
// followed by every position added since, prev_len .. pos.  They are scored by the indexer's definition at
// those positions only, the usual top-k keeps k of them (ties to the earlier slot, which is the lower
// position: the earlier selection is ascending and all of it precedes the new positions), and the kept
// slots map back to positions:
//   reuse_candidates_kernel  one CTA per row: the candidate list [T, k + max_new]
//   indexer_at_kernel        CTAs of (row, candidate block): the row's 64 x 128 FP8 query decoded once into
//                            shared memory (rows padded to 129 floats: conflict-free), a warp per candidate
//                            decodes its 128-byte key, each lane owns two heads, warp sum of the weighted
//                            ReLUs, times the key's scale; -inf for empty slots and positions past the row
//   gather_positions_kernel  kept slot -> position
// The scores are fp32 sums of exact FP8 products, in another order than the tensor-core indexer's.
#include <cuda_fp8.h>

#include "common.cuh"

namespace dsa {

constexpr int kReuseThreads = 256;
constexpr int kReuseCandsPerCta = 64;
constexpr int kReuseQStride = 129;

__global__ void __launch_bounds__(kReuseThreads)
reuse_candidates_kernel(const int32_t *__restrict__ prev_idx, int k, const int32_t *__restrict__ prev_lens,
                        int max_new, BatchView bv, int32_t *__restrict__ cand, uint32_t *status) {
  pdl_wait();
  pdl_trigger();
  __shared__ int s_pos;
  const int row = blockIdx.x, m = k + max_new;
  if (threadIdx.x < 32) {
    int b;
    const int pos = pos_of_row_warp(bv, row, &b);
    if (threadIdx.x == 0) s_pos = pos;
  }
  __syncthreads();
  const int pos = s_pos, plen = __ldg(prev_lens + row);
  if (threadIdx.x == 0 && (plen < 0 || pos - plen + 1 > max_new)) set_status(status, kStatusBadIndex);
  int32_t *out = cand + (int64_t)row * m;
  for (int j = threadIdx.x; j < m; j += blockDim.x) {
    int v;
    if (j < k) {
      v = __ldg(prev_idx + (int64_t)row * k + j);
      if (v >= plen) v = -1;                            // an earlier selection holds only earlier positions
    } else {
      v = plen + (j - k);
      if (plen < 0 || v > pos) v = -1;
    }
    out[j] = v;
  }
}

__global__ void __launch_bounds__(kReuseThreads)
indexer_at_kernel(const uint8_t *__restrict__ qI, const float *__restrict__ w, const uint8_t *__restrict__ kpool,
                  const float *__restrict__ kscale, BatchView bv, const int32_t *__restrict__ cand, int m,
                  float *__restrict__ out, uint32_t *status) {
  pdl_wait();
  pdl_trigger();
  __shared__ float sq[64 * kReuseQStride];
  __shared__ float sw[64];
  __shared__ float skey[kReuseThreads / 32][128];
  __shared__ int s_pos, s_seq;
  const int row = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x < 32) {
    int b;
    const int pos = pos_of_row_warp(bv, row, &b);
    if (threadIdx.x == 0) {
      s_pos = pos;
      s_seq = b;
    }
  }
  const uint8_t *qr = qI + (int64_t)row * 64 * 128;
  for (int i = threadIdx.x; i < 64 * 128; i += blockDim.x) {
    const __nv_fp8_e4m3 c = *reinterpret_cast<const __nv_fp8_e4m3 *>(qr + i);
    sq[(i >> 7) * kReuseQStride + (i & 127)] = float(c);
  }
  if (threadIdx.x < 64) sw[threadIdx.x] = __ldg(w + (int64_t)row * 64 + threadIdx.x);
  __syncthreads();
  const int pos = s_pos, b = s_seq;
  const int j0 = blockIdx.x * kReuseCandsPerCta;
  const int j1 = min(m, j0 + kReuseCandsPerCta);
  for (int j = j0 + warp; j < j1; j += kReuseThreads / 32) {
    const int s = __ldg(cand + (int64_t)row * m + j);
    int64_t pr = -1;
    if (s >= 0 && s <= pos) {
      pr = phys_row(bv, b, s);
      if (pr < 0 && lane == 0) set_status(status, kStatusBadIndex);
    }
    float score = -INFINITY;
    if (pr >= 0) {                                        // warp-uniform
      const uint32_t codes = __ldg(reinterpret_cast<const uint32_t *>(kpool + pr * 128) + lane);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint8_t byte = (uint8_t)(codes >> (8 * e));
        skey[warp][4 * lane + e] = float(*reinterpret_cast<const __nv_fp8_e4m3 *>(&byte));
      }
      __syncwarp();
      float d0 = 0.f, d1 = 0.f;
      const float *q0 = sq + lane * kReuseQStride, *q1 = sq + (lane + 32) * kReuseQStride;
#pragma unroll 8
      for (int d = 0; d < 128; ++d) {
        const float kv = skey[warp][d];
        d0 = fmaf(q0[d], kv, d0);
        d1 = fmaf(q1[d], kv, d1);
      }
      float part = sw[lane] * fmaxf(d0, 0.f) + sw[lane + 32] * fmaxf(d1, 0.f);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
      score = __ldg(kscale + pr) * part;
      __syncwarp();
    }
    if (lane == 0) out[(int64_t)row * m + j] = score;
  }
}

__global__ void __launch_bounds__(kReuseThreads)
gather_positions_kernel(const int32_t *__restrict__ sel, int k, const int32_t *__restrict__ cand, int m, int T,
                        int32_t *__restrict__ idx) {
  pdl_wait();
  pdl_trigger();
  const int64_t n = (int64_t)T * k;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / k;
    const int p = __ldg(sel + i);
    idx[i] = (p >= 0 && p < m) ? __ldg(cand + t * m + p) : -1;
  }
}

dsa_status_t reuse_candidates_launch(const int32_t *prev_idx, int k, const int32_t *prev_lens, int max_new,
                                     const dsa_batch_t *b, int32_t *cand, void *ws, cudaStream_t stream) {
  DSA_LAUNCH_PDL("reuse_candidates_kernel", reuse_candidates_kernel, dim3(b->total_q), dim3(kReuseThreads), 0, stream,
                 prev_idx, k, prev_lens, max_new, view_of(b), cand, (uint32_t *)ws);
  return DSA_OK;
}

dsa_status_t indexer_at_launch(const uint8_t *qI, const float *w, const uint8_t *kpool, const float *kscale,
                               const dsa_batch_t *b, const int32_t *cand, int m, float *out, void *ws,
                               cudaStream_t stream) {
  const dim3 grid((unsigned)((m + kReuseCandsPerCta - 1) / kReuseCandsPerCta), (unsigned)b->total_q);
  DSA_LAUNCH_PDL("indexer_at_kernel", indexer_at_kernel, grid, dim3(kReuseThreads), 0, stream, qI, w, kpool, kscale,
                 view_of(b), cand, m, out, (uint32_t *)ws);
  return DSA_OK;
}

dsa_status_t gather_positions_launch(const int32_t *sel, int k, const int32_t *cand, int m, int T, int32_t *idx,
                                     cudaStream_t stream) {
  const int64_t n = (int64_t)T * k;
  const int grid = (int)std::min<int64_t>(65535, (n + kReuseThreads - 1) / kReuseThreads);
  DSA_LAUNCH_PDL("gather_positions_kernel", gather_positions_kernel, dim3(grid < 1 ? 1 : grid), dim3(kReuseThreads), 0,
                 stream, sel, k, cand, m, T, idx);
  return DSA_OK;
}

}  // namespace dsa
