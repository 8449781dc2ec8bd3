// Context-parallel decode: the small steps around the three calls when every sequence's tokens are spread
// over G ranks, rank r holding the contiguous range [lo_b, hi_b) of sequence b.
//
// Each rank scores and selects over its own range (the indexer and top-k as usual, on a batch whose
// sequences are its ranges), then:
//   candidates   its local top-k as (score, global position) pairs, padding as (-inf, -1);
//   rows         after an all-gather [G][T][k], each query row's G*k candidates laid out contiguously;
//   (top-k)      the usual top-k over those rows: the k best candidates, ties to the lower candidate
//                position, which is the lower global position because ranks hold ascending ranges and
//                each rank's list is ascending;
//   select_local the winners that fall in this rank's range, as local positions (others -1);
//   (attention)  the usual decode attention over them: o_r and lse_r over this rank's part of the set;
//   merge        after an all-gather, o = sum_r exp(lse_r - lse) o_r with lse = log sum_r exp(lse_r).
// Every token of the global top-k is in its own rank's local top-k (fewer than k tokens of any range beat
// the global k-th score, and a range keeps its lowest-positioned ties), so the set equals the single-GPU
// selection.  The merge is the cross-block reduction of split attention ("Engineering Practices for
// Day-0 Adaptation of Million-Token Context Models on Domestic AI Chips", Four Key Layers 3), taken
// across GPUs.  All four kernels are plain elementwise / row passes; none waits on another CTA.
#include "common.cuh"

namespace dsa {

constexpr int kCpThreads = 256;

__global__ void __launch_bounds__(kCpThreads)
cp_candidates_kernel(const float *__restrict__ scores, int64_t ld, const int32_t *__restrict__ idx, int T, int k,
                     const int32_t *__restrict__ offsets, float *__restrict__ cand_score,
                     int32_t *__restrict__ cand_gidx) {
  pdl_wait();
  pdl_trigger();
  const int64_t n = (int64_t)T * k;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int t = (int)(i / k);
    const int s = __ldg(idx + i);
    const bool ok = s >= 0 && s < ld;
    cand_score[i] = ok ? __ldg(scores + (int64_t)t * ld + s) : -INFINITY;
    cand_gidx[i] = ok ? s + __ldg(offsets + t) : -1;
  }
}

__global__ void __launch_bounds__(kCpThreads)
cp_rows_kernel(const float *__restrict__ g_score, int G, int T, int k, float *__restrict__ rows, int64_t ld_rows) {
  pdl_wait();
  pdl_trigger();
  const int64_t gk = (int64_t)G * k, n = (int64_t)T * gk;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / gk, p = i % gk, r = p / k, j = p % k;
    rows[t * ld_rows + p] = __ldg(g_score + (r * T + t) * k + j);
  }
}

__global__ void __launch_bounds__(kCpThreads)
cp_select_local_kernel(const int32_t *__restrict__ sel, const int32_t *__restrict__ g_gidx, int G, int T, int k,
                       const int32_t *__restrict__ lo, const int32_t *__restrict__ hi, int32_t *__restrict__ local) {
  pdl_wait();
  pdl_trigger();
  const int64_t n = (int64_t)T * k, gk = (int64_t)G * k;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / k;
    const int p = __ldg(sel + i);
    int g = -1;
    if (p >= 0 && p < gk) g = __ldg(g_gidx + (((int64_t)(p / k)) * T + t) * k + (p % k));
    const int l = __ldg(lo + t), h = __ldg(hi + t);
    local[i] = (g >= 0 && g >= l && g < h) ? g - l : -1;
  }
}

// one CTA per (row, head), Dv / 4 threads, four values each
__global__ void __launch_bounds__(256)
cp_merge_kernel(const __nv_bfloat16 *__restrict__ part_out, const float *__restrict__ part_lse, int G, int T, int H,
                int Dv, __nv_bfloat16 *__restrict__ out, float *__restrict__ lse) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x, h = blockIdx.y, d = 4 * threadIdx.x;
  const int64_t th = (int64_t)t * H + h, TH = (int64_t)T * H;
  float mx = -INFINITY;
  for (int r = 0; r < G; ++r) mx = fmaxf(mx, __ldg(part_lse + r * TH + th));
  float tot = 0.f;
  for (int r = 0; r < G; ++r) {
    const float l = __ldg(part_lse + r * TH + th);
    if (l != -INFINITY) tot += expf(l - mx);
  }
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  if (tot > 0.f) {
    for (int r = 0; r < G; ++r) {
      const float l = __ldg(part_lse + r * TH + th);
      if (l == -INFINITY) continue;
      const float wgt = expf(l - mx) / tot;
      const uint2 u = __ldg(reinterpret_cast<const uint2 *>(part_out + (r * TH + th) * Dv + d));
      acc[0] += wgt * __uint_as_float(u.x << 16);
      acc[1] += wgt * __uint_as_float(u.x & 0xFFFF0000u);
      acc[2] += wgt * __uint_as_float(u.y << 16);
      acc[3] += wgt * __uint_as_float(u.y & 0xFFFF0000u);
    }
  }
  const __nv_bfloat162 b0 = __floats2bfloat162_rn(acc[0], acc[1]), b1 = __floats2bfloat162_rn(acc[2], acc[3]);
  uint2 w;
  w.x = *reinterpret_cast<const uint32_t *>(&b0);
  w.y = *reinterpret_cast<const uint32_t *>(&b1);
  *reinterpret_cast<uint2 *>(out + th * Dv + d) = w;
  if (lse && threadIdx.x == 0) lse[th] = tot > 0.f ? mx + logf(tot) : -INFINITY;
}

static int cp_grid(int64_t n) {
  const int64_t g = (n + kCpThreads - 1) / kCpThreads;
  return (int)(g < 1 ? 1 : (g > 65535 ? 65535 : g));
}

dsa_status_t cp_candidates_launch(const float *scores, int64_t ld, const int32_t *idx, int T, int k,
                                  const int32_t *offsets, float *cand_score, int32_t *cand_gidx, cudaStream_t stream) {
  DSA_LAUNCH_PDL("cp_candidates_kernel", cp_candidates_kernel, dim3(cp_grid((int64_t)T * k)), dim3(kCpThreads), 0,
                 stream, scores, ld, idx, T, k, offsets, cand_score, cand_gidx);
  return DSA_OK;
}

dsa_status_t cp_rows_launch(const float *g_score, int G, int T, int k, float *rows, int64_t ld_rows,
                            cudaStream_t stream) {
  DSA_LAUNCH_PDL("cp_rows_kernel", cp_rows_kernel, dim3(cp_grid((int64_t)T * G * k)), dim3(kCpThreads), 0, stream,
                 g_score, G, T, k, rows, ld_rows);
  return DSA_OK;
}

dsa_status_t cp_select_local_launch(const int32_t *sel, const int32_t *g_gidx, int G, int T, int k, const int32_t *lo,
                                    const int32_t *hi, int32_t *local, cudaStream_t stream) {
  DSA_LAUNCH_PDL("cp_select_local_kernel", cp_select_local_kernel, dim3(cp_grid((int64_t)T * k)), dim3(kCpThreads), 0,
                 stream, sel, g_gidx, G, T, k, lo, hi, local);
  return DSA_OK;
}

dsa_status_t cp_merge_launch(const void *part_out, const float *part_lse, int G, int T, int H, int Dv, void *out,
                             float *lse, cudaStream_t stream) {
  DSA_LAUNCH_PDL("cp_merge_kernel", cp_merge_kernel, dim3(T, H), dim3(Dv / 4), 0, stream,
                 (const __nv_bfloat16 *)part_out, part_lse, G, T, H, Dv, (__nv_bfloat16 *)out, lse);
  return DSA_OK;
}

}  // namespace dsa
