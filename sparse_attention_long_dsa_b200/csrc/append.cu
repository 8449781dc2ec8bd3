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
// both divisions IEEE fp32.  One warp per token; the work is a few hundred bytes per token, so the
// kernel is bound by launch latency for a decode batch and by HBM for a prefill chunk.
#include <cuda_fp8.h>

#include "common.cuh"

namespace dsa {

constexpr int kAppendWarps = 8;
constexpr int kAppendKvVec = 576 * 2 / 16;       // 16-byte vectors in one latent row: 72

// the 4 key elements 4*lane .. 4*lane+3 as fp32
__device__ __forceinline__ void load_key4(const void *keys, bool bf16, int64_t row, int lane, float v[4]) {
  if (bf16) {
    const uint2 u = __ldg(reinterpret_cast<const uint2 *>(keys) + row * 32 + lane);
    v[0] = __uint_as_float(u.x << 16);
    v[1] = __uint_as_float(u.x & 0xFFFF0000u);
    v[2] = __uint_as_float(u.y << 16);
    v[3] = __uint_as_float(u.y & 0xFFFF0000u);
  } else {
    const float4 f = __ldg(reinterpret_cast<const float4 *>(keys) + row * 32 + lane);
    v[0] = f.x;
    v[1] = f.y;
    v[2] = f.z;
    v[3] = f.w;
  }
}

__global__ void __launch_bounds__(kAppendWarps * 32)
cache_append_kernel(const uint4 *__restrict__ kv_new, const void *__restrict__ k_new, int k_bf16, BatchView bv,
                    int T, uint4 *__restrict__ kv_pool, uint32_t *__restrict__ kI_pool, float *__restrict__ kS_pool,
                    uint32_t *status) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * kAppendWarps + (threadIdx.x >> 5);
  if (row >= T) return;                                   // whole warps leave together
  int b;
  const int pos = pos_of_row_warp(bv, row, &b);
  if (pos < 0 || pos >= bv.max_blocks_per_seq * bv.page_size) {
    if (lane == 0) set_status(status, kStatusBadIndex);
    return;
  }
  const int64_t pr = phys_row(bv, b, pos);
  if (pr < 0) {
    if (lane == 0) set_status(status, kStatusBadIndex);
    return;
  }

  // latent row: a straight 1152-byte copy
  const uint4 *src = kv_new + (int64_t)row * kAppendKvVec;
  uint4 *dst = kv_pool + pr * kAppendKvVec;
  for (int i = lane; i < kAppendKvVec; i += 32) dst[i] = __ldg(src + i);

  // indexer key: per-token scale from the warp's max |k|, then round-to-nearest saturating E4M3
  float v[4];
  load_key4(k_new, k_bf16 != 0, row, lane, v);
  float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  float scale = amax / 448.0f;
  if (scale == 0.0f) scale = 1.0f;
  uint32_t packed = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __nv_fp8_storage_t c = __nv_cvt_float_to_fp8(v[e] / scale, __NV_SATFINITE, __NV_E4M3);
    packed |= (uint32_t)c << (8 * e);
  }
  kI_pool[pr * 32 + lane] = packed;
  if (lane == 0) kS_pool[pr] = scale;
}

dsa_status_t cache_append_launch(const void *kv_new, const void *k_new, bool k_bf16, const dsa_batch_t *b,
                                 void *kv_pool, void *kI_pool, float *kS_pool, void *ws, cudaStream_t stream) {
  const int T = b->total_q;
  const int grid = (T + kAppendWarps - 1) / kAppendWarps;
  DSA_LAUNCH_PDL("cache_append_kernel", cache_append_kernel, dim3(grid), dim3(kAppendWarps * 32), 0, stream,
                 (const uint4 *)kv_new, k_new, k_bf16 ? 1 : 0, view_of(b), T, (uint4 *)kv_pool, (uint32_t *)kI_pool,
                 kS_pool, (uint32_t *)ws);
  return DSA_OK;
}

}  // namespace dsa
