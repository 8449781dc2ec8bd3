// Appending one new token to the paged cache, by one warp (shared by the standalone append kernel and
// the indexer's first kernel when the two are fused).
//
// The token is query row `row` of the batch, at the position the other steps give it.  Its 576-entry bf16
// latent row is copied into the latent pool; its 128-entry indexer key (f32 or bf16) is stored as E4M3 codes
// with one fp32 scale:  scale = max|k| / 448 (1 when that is 0), code_d = e4m3_rn_satfinite(k_d / scale),
// both divisions IEEE fp32.  A position outside the block table or a block id outside the pool leaves the
// token unwritten and raises the bad-index bit of the status word.
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"

namespace dsa {

struct AppendArgs {
  const uint4 *kv_new;      // [T, 72] 16-byte vectors of the bf16 latent rows
  const void *k_new;        // [T, 128] f32 or bf16 indexer keys
  int k_bf16;
  uint4 *kv_pool;           // [num_blocks * 64, 72]
  uint32_t *kI_pool;        // [num_blocks * 64, 32] (4 codes per word)
  float *kS_pool;           // [num_blocks * 64]
};

constexpr int kAppendKvVec = 576 * 2 / 16;

__device__ __forceinline__ void append_key4(const void *keys, bool bf16, int64_t row, int lane, float v[4]) {
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

// every lane of the warp calls this with the same row
__device__ __forceinline__ void append_token_warp(const AppendArgs &a, const BatchView &bv, int row, int lane,
                                                  uint32_t *status) {
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
  const uint4 *src = a.kv_new + (int64_t)row * kAppendKvVec;
  uint4 *dst = a.kv_pool + pr * kAppendKvVec;
  for (int i = lane; i < kAppendKvVec; i += 32) dst[i] = __ldg(src + i);
  float v[4];
  append_key4(a.k_new, a.k_bf16 != 0, row, lane, v);
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
  a.kI_pool[pr * 32 + lane] = packed;
  if (lane == 0) a.kS_pool[pr] = scale;
}

}  // namespace dsa
