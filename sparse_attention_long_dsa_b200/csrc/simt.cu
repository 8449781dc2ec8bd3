// CUDA-core kernels: the fp32 path (small head counts and dims, exact fp32 arithmetic).
//
// indexer_simt_kernel : scores[row, s] = kS[s] * sum_j w[row,j] * max(0, qI[row,j,:] . kI[s,:])
//                       one thread per candidate token, the row's indexer query staged in smem.
// attn_simt_kernel    : softmax attention of HG heads of one row over its selected tokens, in
//                       chunks of 32 tokens with a running max / sum (online softmax, the
//                       per-tile accumulation of the pages' tile sketch made exact: "Day-0
//                       Adaptation for LLMs: Implementing Sparse Attention and Low-Precision
//                       Weights", II tile-level sparse attention skeleton).
#include "common.cuh"

namespace dsa {

constexpr int kIdxSimtTile = 128;
constexpr int kIdxSimtMaxD = 128;

template <typename TQ>
__device__ __forceinline__ float load_val(const TQ *p, int64_t i);
template <>
__device__ __forceinline__ float load_val<float>(const float *p, int64_t i) { return __ldg(p + i); }

template <typename TQ>
__global__ void __launch_bounds__(kIdxSimtTile)
indexer_simt_kernel(const TQ *__restrict__ qI, const float *__restrict__ w, const TQ *__restrict__ kpool,
                    const float *__restrict__ kscale, int Hi, int Di, BatchView bv, float *__restrict__ scores,
                    int64_t ld) {
  extern __shared__ float qs[];          // [Hi * Di] then w [Hi]
  float *wsm = qs + Hi * Di;
  const int row = blockIdx.x;
  int b;
  const int n = pos_of_row(bv, row, &b) + 1;
  const int s0 = blockIdx.y * kIdxSimtTile;
  if (s0 >= n) return;
  for (int i = threadIdx.x; i < Hi * Di; i += blockDim.x) qs[i] = load_val<TQ>(qI, (int64_t)row * Hi * Di + i);
  for (int i = threadIdx.x; i < Hi; i += blockDim.x) wsm[i] = __ldg(w + (int64_t)row * Hi + i);
  __syncthreads();
  const int s = s0 + threadIdx.x;
  if (s >= n) return;
  const int64_t pr = phys_row(bv, b, s);
  if (pr < 0) return;
  float kv[kIdxSimtMaxD];
#pragma unroll
  for (int d = 0; d < kIdxSimtMaxD; ++d) kv[d] = d < Di ? load_val<TQ>(kpool, pr * Di + d) : 0.f;
  float acc = 0.f;
  for (int j = 0; j < Hi; ++j) {
    const float *qj = qs + j * Di;
    float dot = 0.f;
#pragma unroll
    for (int d = 0; d < kIdxSimtMaxD; ++d)
      if (d < Di) dot = fmaf(qj[d], kv[d], dot);
    acc = fmaf(wsm[j], fmaxf(dot, 0.f), acc);
  }
  if (kscale) acc *= __ldg(kscale + pr);
  scores[(int64_t)row * ld + s] = acc;
}

// ------------------------------------------------------------------------------------------------
constexpr int kAttnSimtHG = 8;        // heads per CTA
constexpr int kAttnSimtChunk = 32;    // tokens per chunk
constexpr int kAttnSimtMaxDv = 512;

template <typename T>
__device__ __forceinline__ void store_val(T *p, int64_t i, float v);
template <>
__device__ __forceinline__ void store_val<float>(float *p, int64_t i, float v) { p[i] = v; }

template <typename T>
__global__ void __launch_bounds__(256)
attn_simt_kernel(const T *__restrict__ q, const T *__restrict__ kv, const T *__restrict__ vpool, int H, int Dqk,
                 int Dv, float scale, const int32_t *__restrict__ idx, int k, BatchView bv, T *__restrict__ out,
                 float *__restrict__ lse) {
  extern __shared__ float sm[];
  const int KS = Dqk + 1;                                   // odd stride: conflict-free column reads
  float *qs = sm;                                           // [HG][Dqk]
  float *Ks = qs + kAttnSimtHG * Dqk;                       // [chunk][Dqk+1]
  float *Vs = Ks + kAttnSimtChunk * KS;                     // [chunk][Dv]
  float *ps = Vs + kAttnSimtChunk * Dv;                     // [HG][chunk]
  __shared__ int64_t rows[kAttnSimtChunk];

  const int row = blockIdx.x;
  const int h0 = blockIdx.y * kAttnSimtHG;
  const int nh = min(kAttnSimtHG, H - h0);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int b;
  pos_of_row(bv, row, &b);
  const int seq_len = __ldg(bv.seq_lens + b);
  for (int i = tid; i < kAttnSimtHG * Dqk; i += blockDim.x) {
    int h = i / Dqk, d = i % Dqk;
    qs[i] = h < nh ? load_val<T>(q, ((int64_t)row * H + h0 + h) * Dqk + d) : 0.f;
  }
  const int nO = (Dv + 31) / 32;
  float o[kAttnSimtMaxDv / 32];
#pragma unroll
  for (int j = 0; j < kAttnSimtMaxDv / 32; ++j) o[j] = 0.f;
  float m = -INFINITY, l = 0.f;
  const int32_t *irow = idx + (int64_t)row * k;

  for (int c0 = 0; c0 < k; c0 += kAttnSimtChunk) {
    __syncthreads();
    if (tid < kAttnSimtChunk) {
      int64_t pr = -1;
      if (c0 + tid < k) {
        int s = __ldg(irow + c0 + tid);
        if (s >= 0 && s < seq_len) pr = phys_row(bv, b, s);
      }
      rows[tid] = pr;
    }
    __syncthreads();
    for (int i = tid; i < kAttnSimtChunk * Dqk; i += blockDim.x) {
      int r = i / Dqk, d = i % Dqk;
      int64_t pr = rows[r];
      Ks[r * KS + d] = pr >= 0 ? load_val<T>(kv, pr * Dqk + d) : 0.f;
    }
    for (int i = tid; i < kAttnSimtChunk * Dv; i += blockDim.x) {
      int r = i / Dv, d = i % Dv;
      int64_t pr = rows[r];
      float v = 0.f;
      if (pr >= 0) v = vpool ? load_val<T>(vpool, pr * Dv + d) : load_val<T>(kv, pr * Dqk + d);
      Vs[r * Dv + d] = v;
    }
    __syncthreads();
    if (warp < nh) {
      const float *qh = qs + warp * Dqk;
      const float *kr = Ks + lane * KS;
      float z = 0.f;
      for (int d = 0; d < Dqk; ++d) z = fmaf(qh[d], kr[d], z);
      const bool valid = rows[lane] >= 0;
      z = valid ? z * scale : -INFINITY;
      float cm = z;
#pragma unroll
      for (int off = 16; off; off >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, off));
      const float mn = fmaxf(m, cm);
      float p = 0.f, alpha = 1.f;
      if (mn != -INFINITY) {
        p = valid ? expf(z - mn) : 0.f;
        alpha = m == -INFINITY ? 0.f : expf(m - mn);
      }
      float ls = p;
#pragma unroll
      for (int off = 16; off; off >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, off);
      l = l * alpha + ls;
      m = mn;
      ps[warp * kAttnSimtChunk + lane] = p;
      __syncwarp();
      const float *pw = ps + warp * kAttnSimtChunk;
#pragma unroll
      for (int j = 0; j < kAttnSimtMaxDv / 32; ++j) {
        if (j < nO) {
          const int dv = lane + 32 * j;
          float acc = o[j] * alpha;
          if (dv < Dv)
            for (int r = 0; r < kAttnSimtChunk; ++r) acc = fmaf(pw[r], Vs[r * Dv + dv], acc);
          o[j] = acc;
        }
      }
    }
  }
  if (warp < nh) {
    const int h = h0 + warp;
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int j = 0; j < kAttnSimtMaxDv / 32; ++j) {
      const int dv = lane + 32 * j;
      if (j < nO && dv < Dv) store_val<T>(out, ((int64_t)row * H + h) * Dv + dv, o[j] * inv);
    }
    if (lse && lane == 0) lse[(int64_t)row * H + h] = l > 0.f ? m + logf(l) : -INFINITY;
  }
}

// ------------------------------------------------------------------------------------------------
// host launchers
// ------------------------------------------------------------------------------------------------
dsa_status_t indexer_simt_launch(const void *qI, dsa_dtype_t dt, const float *w, const void *kpool,
                                 const float *kscale, int Hi, int Di, const dsa_batch_t *b, float *scores,
                                 int64_t ld, cudaStream_t stream) {
  BatchView bv = view_of(b);
  dim3 grid(b->total_q, (b->max_seq_len + kIdxSimtTile - 1) / kIdxSimtTile);
  size_t smem = (size_t)(Hi * Di + Hi) * 4;
  (void)dt;   // the e4m3 indexer runs on the tensor cores (indexer_tc.cu)
  cudaFuncSetAttribute(indexer_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  indexer_simt_kernel<float><<<grid, kIdxSimtTile, smem, stream>>>((const float *)qI, w, (const float *)kpool,
                                                                   kscale, Hi, Di, bv, scores, ld);
  DSA_LAUNCH_CHECK("indexer_simt_kernel");
  return DSA_OK;
}

dsa_status_t attn_simt_launch(const void *q, dsa_dtype_t dt, const void *kv, const void *v, int H, int Dqk, int Dv,
                              float scale, const int32_t *idx, int k, const dsa_batch_t *b, void *out, float *lse,
                              cudaStream_t stream) {
  BatchView bv = view_of(b);
  dim3 grid(b->total_q, (H + kAttnSimtHG - 1) / kAttnSimtHG);
  size_t smem = (size_t)(kAttnSimtHG * Dqk + kAttnSimtChunk * (Dqk + 1) + kAttnSimtChunk * Dv +
                         kAttnSimtHG * kAttnSimtChunk) * 4;
  (void)dt;   // the bf16 MLA path runs on the tensor cores (attn_mla_tc.cu)
  cudaFuncSetAttribute(attn_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  attn_simt_kernel<float><<<grid, 256, smem, stream>>>((const float *)q, (const float *)kv, (const float *)v, H, Dqk,
                                                       Dv, scale, idx, k, bv, (float *)out, lse);
  DSA_LAUNCH_CHECK("attn_simt_kernel");
  return DSA_OK;
}

}  // namespace dsa
