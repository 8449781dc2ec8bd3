// Streaming threshold selection: the k best positions of each query row (score descending, position
// ascending), written in ascending position order.
//
// The selection operator the pages describe fuses scoring, threshold filtering and index gathering so that
// the scores are not walked over and over in global memory ("Day-0 Adaptation: Running Trillion-Parameter
// Models on Domestic AI Accelerators", 3.1 Index Selection Operator; "Engineering Practices for Day-0
// Adaptation of Million-Token Context Models on Domestic AI Chips", Four Key Layers 1: row-grouped
// selection with shared-memory buffering and vector loads).  Here the indexer's epilogue counts, for every
// row, the leading 11 bits of each score's order-preserving key (a 2048-bin histogram), so this kernel
// knows the threshold digit before it reads a single score.  It then streams the row once and keeps only
// the survivors -- keys whose digit is at or above the threshold digit, about k plus the threshold bin --
// in shared memory, finishes the selection on those, and writes the result.
//
// Per row a cluster of C CTAs (C = 1 .. 16) takes contiguous slices; every CTA keeps the same selection state
// (fixed key bits: prefix P under mask M; `above` keys strictly above the prefix; `need` still to take from the
// prefix's bin of `bin_cnt` keys).  A digit is fixed from a row histogram that every CTA holds a copy of: each
// CTA adds the non-zero bins of its slice's histogram into every CTA's copy (distributed shared memory
// atomics, then one cluster barrier).  While the survivors would not fit in the capacity, a counting pass over
// the slice fixes the next digit (11, 11 then 10 bits).  When every bit is fixed, keys equal to the threshold
// are kept in position order up to `need` (the slices before take theirs first), so the survivors always fit.
// The storing pass compacts each slice's survivors in position order; the remaining digits are fixed on the
// survivors the same way (stopping as soon as the prefix's bin holds exactly the keys still needed); then each
// slice writes its selected positions, offset by the counts of the slices before it, stored into the later
// CTAs before a barrier.  No CTA reads another's shared memory.  Without a histogram (plain scores) the first
// counting pass fixes the leading digit.  Very long rows in small batches collect their survivors over every SM
// first (select_gather_kernel, below), and one CTA per row goes on from them.
#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstdlib>

#include "tc.cuh"

namespace dsa {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelBins = 2048;
constexpr int kSelPerThread = 8;                        // keys per thread per tile (2 x float4)
constexpr int kSelTile = kSelThreads * kSelPerThread;   // 4096 keys
constexpr int kSelBatch = 2;                            // tiles whose loads are issued together
constexpr int kSelVec = kSelPerThread / 4;
constexpr int kSelMaxCluster = 16;

struct SelArgs {
  const float *scores;
  int64_t ld;
  BatchView bv;
  int k;
  int32_t *idx;
  const uint32_t *hist;    // [T][2048] leading-digit counts of each row's causal keys, or nullptr
  int cap;                 // survivors a CTA can hold (shared memory)
  uint32_t *status;
  // survivors already collected by select_gather_kernel (one CTA per row then), or nullptr
  const uint32_t *surv_key;
  const int32_t *surv_pos;
  const uint32_t *surv_cnt;
  int surv_ctas, surv_q;
};

// Very long rows (a million-token decode): one cluster of CTAs per row would leave most of the GPU idle, so the
// survivors are first collected by select_gather_kernel over every SM -- each of G CTAs takes one range of the
// row and keeps, in position order, the keys whose leading digit is at or above the threshold digit, up to
// kSelSurvQ of them -- and select_stream_kernel (one CTA per row) goes on from those.
constexpr int kSelLongRow = 262144;     // rows at least this long (in the batch's longest) take the gather
constexpr int kSelLongMaxRows = 16;     // ... for batches of at most this many rows
constexpr int kSelLongCtas = 160;       // gather CTAs over the batch (at most; the workspace is sized for it)
constexpr int kSelSurvQ = 512;          // survivors one gather CTA keeps (a range holding more: the row is streamed)

size_t select_long_ws_bytes(int total_q, int max_seq_len) {
  if (max_seq_len < kSelLongRow || total_q > kSelLongMaxRows || total_q < 1) return 0;
  const size_t slots = (size_t)kSelLongCtas * kSelSurvQ;
  return (slots * 8 + 255) / 256 * 256 + ((size_t)kSelLongCtas * 4 + 255) / 256 * 256;
}

// shared memory (u32 words): survivors (key, position) [cap], the slice histogram, two row histograms
// (alternating passes), scan scratch, the earlier slices' equal-key counts (full case) and final counts
constexpr int kSelFixedWords = 3 * kSelBins + 64 + kSelMaxCluster + 2 * kSelMaxCluster;
size_t select_smem_bytes(int cap) { return ((size_t)2 * cap + kSelFixedWords) * 4; }

__device__ __forceinline__ uint32_t sel_cl_nranks() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void sel_cl_red_add(const uint32_t *p, uint32_t rank, uint32_t v) {
  asm volatile("red.shared::cluster.add.u32 [%0], %1;" ::"r"(tc::map_to_rank(tc::smem_u32(p), rank)), "r"(v) : "memory");
}
__device__ __forceinline__ void sel_cl_st(const uint32_t *p, uint32_t rank, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(tc::map_to_rank(tc::smem_u32(p), rank)), "r"(v) : "memory");
}
// split cluster barrier (aligned forms: the warp is made converged first)
__device__ __forceinline__ void sel_cl_arrive() {
  __syncwarp();
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void sel_cl_wait() {
  __syncwarp();
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Bin holding the need-th key counted from the top of hist[0..nb) (1 <= need <= the total), and the count of
// keys in higher bins.  Two levels: warp w sums the w-th group of nb / 16 bins from the top, then warp 0 scans the
// 16 group sums and the chosen group's bins (nb / 512 per lane, the lane's own ones in order).  Every thread of
// the block calls it; two block barriers.
__device__ void sel_find_bin(const uint32_t *hist, int nb, uint32_t need, uint32_t *tmp, int *s_bin,
                             uint32_t *s_above) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gsz = nb / kSelWarps;                          // 128 or 64
  if (threadIdx.x == 0) {                                  // (a consistent histogram always overwrites these)
    *s_bin = 0;
    *s_above = 0u;
  }
  {
    const int g0 = nb - (warp + 1) * gsz;
    uint32_t s = 0;
    for (int j = lane; j < gsz; j += 32) s += hist[g0 + j];
    s = __reduce_add_sync(0xffffffffu, s);
    if (lane == 0) tmp[warp] = s;
  }
  __syncthreads();
  if (warp == 0) {
    const uint32_t gs = lane < kSelWarps ? tmp[lane] : 0u;
    uint32_t incl = gs;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int gw = __ffs(__ballot_sync(0xffffffffu, incl - gs < need && incl >= need)) - 1;
    const uint32_t above = __shfl_sync(0xffffffffu, incl - gs, gw < 0 ? 0 : gw);
    const uint32_t want = need - above;
    const int per = gsz >> 5;                              // 4 or 2 bins per lane, from the group's top down
    const int hi = nb - (gw < 0 ? 0 : gw) * gsz - 1 - per * lane;
    uint32_t loc = 0;
    for (int e = 0; e < per; ++e) loc += hist[hi - e];
    uint32_t incl2 = loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl2, o);
      if (lane >= o) incl2 += y;
    }
    uint32_t run = incl2 - loc;
    if (gw >= 0 && run < want && incl2 >= want) {
      for (int e = 0; e < per; ++e) {
        const uint32_t c = hist[hi - e];
        if (run + c >= want) {
          *s_bin = hi - e;
          *s_above = above + run;
          break;
        }
        run += c;
      }
    }
  }
  __syncthreads();
}

// A tile of kSelTile keys is 16 warp segments of 32 x kSelPerThread in position order; in its segment a lane
// holds the keys at 128 v + 4 lane + j (v < kSelPerThread / 4, j = 0..3), read as coalesced float4 loads.
// key[4 v + j]; valid bit 4 v + j is clear for positions at or past m.
__device__ __forceinline__ int sel_elem(int base, int v, int j) {
  return base + (int)(threadIdx.x >> 5) * (32 * kSelPerThread) + 128 * v + 4 * (int)(threadIdx.x & 31) + j;
}
// Loads are issued for a whole batch of tiles before any value is used (a load followed at once by its use
// would cost a memory round trip per vector), and a batch's loads are issued before the previous batch is
// processed.  Positions at or past m read as 0 and are marked invalid at conversion.
struct SelRaw {
  float4 f[kSelBatch][kSelVec];
};
__device__ __forceinline__ void sel_issue(const float *src, int m, int base, SelRaw &raw) {
#pragma unroll
  for (int t = 0; t < kSelBatch; ++t)
#pragma unroll
    for (int v = 0; v < kSelVec; ++v) {
      const int i0 = sel_elem(base + t * kSelTile, v, 0);
      if (i0 + 4 <= m) {
        raw.f[t][v] = __ldg(reinterpret_cast<const float4 *>(src + i0));
      } else {
        raw.f[t][v].x = i0 < m ? __ldg(src + i0) : 0.f;
        raw.f[t][v].y = i0 + 1 < m ? __ldg(src + i0 + 1) : 0.f;
        raw.f[t][v].z = i0 + 2 < m ? __ldg(src + i0 + 2) : 0.f;
        raw.f[t][v].w = i0 + 3 < m ? __ldg(src + i0 + 3) : 0.f;
      }
    }
}
__device__ __forceinline__ void sel_convert(const SelRaw &raw, int t, int m, int base, uint32_t (&key)[kSelPerThread],
                                            uint32_t &valid) {
  valid = 0u;
#pragma unroll
  for (int v = 0; v < kSelVec; ++v) {
    const int i0 = sel_elem(base, v, 0);
    const float fv[4] = {raw.f[t][v].x, raw.f[t][v].y, raw.f[t][v].z, raw.f[t][v].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const bool in = i0 + j < m;
      key[4 * v + j] = in ? ordered_key(fv[j]) : 0u;
      valid |= (in ? 1u : 0u) << (4 * v + j);
    }
  }
}

// Ordered positions of flagged items in a tile laid out as sel_elem describes: flags bit 4 v + j.  Returns, for
// each v, the count of flagged items before (v, lane, 0) in the tile (pre[v]), and the tile's total; `wsum`
// holds 16 words of shared scratch.  One __syncthreads inside, one more before wsum is reused.
__device__ __forceinline__ uint32_t sel_tile_prefix(uint32_t flags, uint32_t (&pre)[kSelPerThread / 4], uint32_t *wsum) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t run = 0u;
#pragma unroll
  for (int v = 0; v < kSelPerThread / 4; ++v) {
    const uint32_t cnt = __popc((flags >> (4 * v)) & 0xFu);
    uint32_t incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    pre[v] = run + incl - cnt;
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) wsum[warp] = run;
  __syncthreads();
  uint32_t before = 0u, total = 0u;
#pragma unroll
  for (int w = 0; w < kSelWarps; ++w) {
    const uint32_t x = wsum[w];
    before += w < warp ? x : 0u;
    total += x;
  }
#pragma unroll
  for (int v = 0; v < kSelPerThread / 4; ++v) pre[v] += before;
  return total;
}

// the row's length: one round of loads for a batch of one query row per sequence (the row is its sequence)
__device__ __forceinline__ int sel_row_len(const BatchView &bv, int row) {
  int sc0 = 0, sc1 = 0, ssl = 0;
  if (row < bv.num_seqs) {
    sc0 = __ldg(bv.cu_q + row);
    sc1 = __ldg(bv.cu_q + row + 1);
    ssl = __ldg(bv.seq_lens + row);
  }
  const int b = seq_of_row_warp(bv.cu_q, bv.num_seqs, row);
  if (b == row) return ssl - (sc1 - sc0) + (row - sc0) + 1;
  const int c0 = __ldg(bv.cu_q + b), c1 = __ldg(bv.cu_q + b + 1);
  return __ldg(bv.seq_lens + b) - (c1 - c0) + (row - c0) + 1;
}

struct GatherArgs {
  const float *scores;
  int64_t ld;
  BatchView bv;
  int k;
  const uint32_t *hist;
  uint32_t *surv_key;      // [T][G][kSelSurvQ]
  int32_t *surv_pos;
  uint32_t *surv_cnt;      // [T][G]: survivors of each range (more than kSelSurvQ: not all kept)
  int G;
};

__global__ void __launch_bounds__(kSelThreads, 1) select_gather_kernel(const GatherArgs a) {
  pdl_wait();
  pdl_trigger();
  __shared__ __align__(16) uint32_t lh[kSelBins];
  __shared__ uint32_t tmp[64];
  __shared__ int s_bin;
  __shared__ uint32_t s_above;
  const int row = blockIdx.x / a.G, g = blockIdx.x % a.G;
  const int tid = threadIdx.x;
  const int n = sel_row_len(a.bv, row);
  if (n <= a.k) return;                                    // (the selection writes such rows itself)
  const int per = ((n + a.G - 1) / a.G + 3) & ~3;
  const int lo = min(n, g * per), m = min(n, lo + per) - lo;
  const float *src = a.scores + (int64_t)row * a.ld + lo;
  // the threshold digit, as the selection will find it
  const uint4 *hr = reinterpret_cast<const uint4 *>(a.hist + (int64_t)row * kSelBins);
  reinterpret_cast<uint4 *>(lh)[tid] = __ldcg(hr + tid);
  __syncthreads();
  if (tid == 0) {
    s_bin = 0;
    s_above = 0u;
  }
  sel_find_bin(lh, kSelBins, (uint32_t)a.k, tmp, &s_bin, &s_above);
  const uint32_t P = (uint32_t)s_bin << 21, M = 0xFFE00000u;
  uint32_t *sk = a.surv_key + ((int64_t)row * a.G + g) * kSelSurvQ;
  int32_t *sp = a.surv_pos + ((int64_t)row * a.G + g) * kSelSurvQ;
  uint32_t stored = 0u;
  SelRaw nxt;
  if (m > 0) sel_issue(src, m, 0, nxt);
#pragma unroll 1
  for (int bb = 0; bb < m; bb += kSelBatch * kSelTile) {
    const SelRaw cur = nxt;
    if (bb + kSelBatch * kSelTile < m) sel_issue(src, m, bb + kSelBatch * kSelTile, nxt);
#pragma unroll
    for (int t = 0; t < kSelBatch; ++t) {
      const int base = bb + t * kSelTile;
      if (base >= m) break;                                // (m is the same for the whole block)
      uint32_t kc[kSelPerThread], vc;
      sel_convert(cur, t, m, base, kc, vc);
      uint32_t keep = 0u;
#pragma unroll
      for (int e = 0; e < kSelPerThread; ++e)
        if (((vc >> e) & 1u) && (kc[e] & M) >= P) keep |= 1u << e;
      uint32_t pre[kSelPerThread / 4];
      const uint32_t tot = sel_tile_prefix(keep, pre, tmp);
#pragma unroll
      for (int v = 0; v < kSelPerThread / 4; ++v) {
        uint32_t off = stored + pre[v];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if ((keep >> (4 * v + j)) & 1u) {
            if (off < (uint32_t)kSelSurvQ) {
              sk[off] = kc[4 * v + j];
              sp[off] = lo + sel_elem(base, v, j);
            }
            ++off;
          }
      }
      stored += tot;
      __syncthreads();
    }
  }
  if (tid == 0) a.surv_cnt[row * a.G + g] = stored;
}

// kGathered: the survivors may come from select_gather_kernel (an instance of its own, so that the code for it
// costs the other launches no registers)
template <bool kGathered>
__global__ void __launch_bounds__(kSelThreads, kGathered ? 1 : 2) select_stream_kernel(const SelArgs a) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) uint32_t sm[];
  const uint32_t cap = (uint32_t)a.cap;
  uint32_t *skey = sm;
  int32_t *spos = reinterpret_cast<int32_t *>(sm + cap);
  uint32_t *lh = sm + 2 * cap;                 // this slice's histogram of the current digit
  uint32_t *gh0 = lh + kSelBins;               // row histograms, even / odd pushed passes
  uint32_t *tmp = gh0 + 2 * kSelBins;
  uint32_t *eq_in = tmp + 64;                  // [c]: equal keys in slice c (full case), stored by CTA c
  uint32_t *cnt_in = eq_in + kSelMaxCluster;   // [2c], [2c + 1]: (keys > T, keys == T) among slice c's survivors
  __shared__ int s_bin;
  __shared__ uint32_t s_above, s_flag;

  const uint32_t C = sel_cl_nranks(), r = tc::cluster_ctarank();
  const int row = blockIdx.x / (int)C;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // the row's length: one round of loads for a batch of one query row per sequence (the row is its sequence)
  int n;
  {
    int sc0 = 0, sc1 = 0, ssl = 0;
    if (row < a.bv.num_seqs) {
      sc0 = __ldg(a.bv.cu_q + row);
      sc1 = __ldg(a.bv.cu_q + row + 1);
      ssl = __ldg(a.bv.seq_lens + row);
    }
    const int b = seq_of_row_warp(a.bv.cu_q, a.bv.num_seqs, row);
    if (b == row) {
      n = ssl - (sc1 - sc0) + (row - sc0) + 1;
    } else {
      const int c0 = __ldg(a.bv.cu_q + b), c1 = __ldg(a.bv.cu_q + b + 1);
      n = __ldg(a.bv.seq_lens + b) - (c1 - c0) + (row - c0) + 1;
    }
  }
  int32_t *out = a.idx + (int64_t)row * a.k;
  // (every branch on n, on the row histograms and on the selection state is taken by the whole cluster)
  if (n <= a.k) {
    if (r == 0)
      for (int j = tid; j < a.k; j += kSelThreads) out[j] = j < n ? j : -1;
    return;
  }
  const int per = ((n + (int)C - 1) / (int)C + 3) & ~3;
  const int lo = min(n, (int)r * per), m = min(n, lo + per) - lo;
  const float *src = a.scores + (int64_t)row * a.ld + lo;

  // both row histograms start empty before any CTA adds into them; the barrier publishing that is waited on
  // just before the first push
  for (int i = tid; i < 2 * kSelBins; i += kSelThreads) gh0[i] = 0u;
  bool wait_pending = false;
  if (C > 1) {
    sel_cl_arrive();
    wait_pending = true;
  }
  int pushes = 0;
  // this slice's histogram lh[0..nb) -> the row histogram (every CTA's copy); returns it
  auto row_hist = [&](int nb) -> uint32_t * {
    uint32_t *gh = gh0 + (pushes & 1) * kSelBins;
    if (C > 1) {
      if (wait_pending) {
        sel_cl_wait();
        wait_pending = false;
      }
      for (int i = tid; i < nb; i += kSelThreads) {
        const uint32_t v = lh[i];
        if (v != 0u)
          for (uint32_t c = 0; c < C; ++c) sel_cl_red_add(gh + i, c, v);
      }
      sel_cl_arrive();
      sel_cl_wait();
    } else {
      for (int i = tid; i < nb; i += kSelThreads) gh[i] = lh[i];
      __syncthreads();
    }
    ++pushes;
    return gh;
  };
  // done with a row histogram: cleared for the pass after next (peers add into it only after the next barrier)
  auto release_row_hist = [&](uint32_t *gh, int nb) {
    __syncthreads();
    for (int i = tid; i < nb; i += kSelThreads) gh[i] = 0u;
  };

  uint32_t P = 0u, M = 0u, above = 0u, need = (uint32_t)a.k, bin_cnt = (uint32_t)n, local_eq = 0u;
  int shift = 32;
  if (a.hist != nullptr) {
    // the leading digit from the indexer's row histogram (read by every CTA of the cluster)
    const uint4 *hr = reinterpret_cast<const uint4 *>(a.hist + (int64_t)row * kSelBins);
    static_assert(kSelBins == 4 * kSelThreads, "one 16-byte load per thread");
    reinterpret_cast<uint4 *>(lh)[tid] = __ldcg(hr + tid);
    __syncthreads();
    sel_find_bin(lh, kSelBins, need, tmp, &s_bin, &s_above);
    P = (uint32_t)s_bin << 21;
    M = 0xFFE00000u;
    above = s_above;
    need -= s_above;
    bin_cnt = lh[s_bin];
    shift = 21;
    __syncthreads();
  }
  // survivors collected over the whole GPU (one CTA per row here): every range's list, in range order, is the
  // row's survivors in position order -- when every range kept all of its own and they add up
  bool gathered = false;
  uint32_t stored = 0u;                // survivors in shared memory (block-uniform)
  if (kGathered && a.surv_cnt != nullptr && shift == 21 && above + bin_cnt <= cap) {
    const int G = a.surv_ctas;
    const uint32_t c = tid < G ? __ldcg(a.surv_cnt + row * G + tid) : 0u;
    const bool fits = __syncthreads_and(c <= (uint32_t)a.surv_q) != 0;
    uint32_t tot;
    const uint32_t off = block_exclusive_scan(c, tmp, &tot);
    if (fits && tot == above + bin_cnt) {
      uint32_t *offs = lh;                     // offs[g]: first survivor of range g in the row's list
      if (tid < G) offs[tid] = off;
      __syncthreads();
      // thread t copies entries t, t + 512, ... of the concatenated lists, finding each entry's range by a binary
      // search over the offsets; a batch of entries' loads all go out before any is stored
      constexpr int kCopy = 4;
      const uint32_t *gk0 = a.surv_key + (int64_t)row * G * a.surv_q;
      const int32_t *gp0 = a.surv_pos + (int64_t)row * G * a.surv_q;
      for (uint32_t i0 = tid; i0 < tot; i0 += kCopy * kSelThreads) {
        uint32_t kv[kCopy];
        int32_t pv[kCopy];
#pragma unroll
        for (int q = 0; q < kCopy; ++q) {
          const uint32_t i = i0 + q * kSelThreads;
          if (i < tot) {
            int lo_g = 0, hi_g = G - 1;              // last range whose offset is <= i
            while (lo_g < hi_g) {
              const int mid = (lo_g + hi_g + 1) >> 1;
              if (offs[mid] <= i) lo_g = mid; else hi_g = mid - 1;
            }
            const int64_t src_i = (int64_t)lo_g * a.surv_q + (i - offs[lo_g]);
            kv[q] = __ldcg(gk0 + src_i);
            pv[q] = __ldcg(gp0 + src_i);
          }
        }
#pragma unroll
        for (int q = 0; q < kCopy; ++q) {
          const uint32_t i = i0 + q * kSelThreads;
          if (i < tot) {
            skey[i] = kv[q];
            spos[i] = pv[q];
          }
        }
      }
      stored = tot;
      gathered = true;
    }
    __syncthreads();
  }
  // ------------------------------------------------------------------ counting passes over the slice
#pragma unroll 1
  while (!gathered && shift > 0 && (shift == 32 || above + bin_cnt > cap)) {
    const int nbits = shift == 10 ? 10 : 11;
    const int nshift = shift - nbits;
    const int nb = 1 << nbits;
    for (int i = tid; i < nb; i += kSelThreads) lh[i] = 0u;
    __syncthreads();
    SelRaw nxt;
    if (m > 0) sel_issue(src, m, 0, nxt);
#pragma unroll 1
    for (int bb = 0; bb < m; bb += kSelBatch * kSelTile) {
      const SelRaw cur = nxt;
      if (bb + kSelBatch * kSelTile < m) sel_issue(src, m, bb + kSelBatch * kSelTile, nxt);
#pragma unroll
      for (int t = 0; t < kSelBatch; ++t) {
        uint32_t kc[kSelPerThread], vc;
        sel_convert(cur, t, m, bb + t * kSelTile, kc, vc);
#pragma unroll
        for (int e = 0; e < kSelPerThread; ++e)
          if (((vc >> e) & 1u) && (kc[e] & M) == P) atomicAdd(&lh[(kc[e] >> nshift) & (uint32_t)(nb - 1)], 1u);
      }
    }
    __syncthreads();
    uint32_t *gh = row_hist(nb);
    sel_find_bin(gh, nb, need, tmp, &s_bin, &s_above);
    P |= (uint32_t)s_bin << nshift;
    M |= (uint32_t)(nb - 1) << nshift;
    above += s_above;
    need -= s_above;
    bin_cnt = gh[s_bin];
    local_eq = lh[s_bin];
    shift = nshift;
    release_row_hist(gh, nb);
  }
  const bool full = shift == 0;      // P is the exact threshold key; take `need` of the keys equal to it

  // full case: keys equal to the threshold in the slices before this one come first in position order
  uint32_t eq_before = 0u;
  if (full && C > 1) {
    if (tid > (int)r && tid < (int)C) sel_cl_st(eq_in + r, (uint32_t)tid, local_eq);
    sel_cl_arrive();
    sel_cl_wait();
    for (uint32_t c = 0; c < r; ++c) eq_before += eq_in[c];
  }

  // ------------------------------------------------------------------ storing pass: ordered survivors
  if (tid == 0) s_flag = 0u;
  if (!gathered) {
    SelRaw nxt;
    if (m > 0) sel_issue(src, m, 0, nxt);
#pragma unroll 1
    for (int bb = 0; bb < m; bb += kSelBatch * kSelTile) {
      // a batch's tiles come from one set of loads; the next batch's loads go out before its first tile
      const SelRaw cur = nxt;
      if (bb + kSelBatch * kSelTile < m) sel_issue(src, m, bb + kSelBatch * kSelTile, nxt);
#pragma unroll
    for (int t = 0; t < kSelBatch; ++t) {
      const int base = bb + t * kSelTile;
      if (base >= m) break;                     // (m is the same for the whole block)
      uint32_t kc[kSelPerThread], vc;
      sel_convert(cur, t, m, base, kc, vc);
      uint32_t keep = 0u, eq = 0u;
#pragma unroll
      for (int e = 0; e < kSelPerThread; ++e) {
        const uint32_t km = kc[e] & M;
        if ((vc >> e) & 1u) {
          if (km > P) keep |= 1u << e;
          else if (km == P) eq |= 1u << e;
        }
      }
      uint32_t pre[kSelPerThread / 4];
      if (full) {
        // equal keys taken in position order: the first `need` of the row
        const uint32_t eq_tot = sel_tile_prefix(eq, pre, tmp);
#pragma unroll
        for (int v = 0; v < kSelPerThread / 4; ++v) {
          uint32_t rank_eq = eq_before + pre[v];
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if ((eq >> (4 * v + j)) & 1u) {
              if (rank_eq < need) keep |= 1u << (4 * v + j);
              ++rank_eq;
            }
        }
        eq_before += eq_tot;
        __syncthreads();
      } else {
        keep |= eq;
      }
      const uint32_t tot = sel_tile_prefix(keep, pre, tmp);
#pragma unroll
      for (int v = 0; v < kSelPerThread / 4; ++v) {
        uint32_t off = stored + pre[v];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if ((keep >> (4 * v + j)) & 1u) {
            if (off < cap) {
              skey[off] = kc[4 * v + j];
              spos[off] = lo + sel_elem(base, v, j);
            } else {
              s_flag = 1u;
            }
            ++off;
          }
      }
      stored += tot;
      __syncthreads();
    }
    }
  }
  if (stored > cap) stored = cap;
  if (s_flag && tid == 0) set_status(a.status, kStatusBadIndex);

  // ------------------------------------------------------------------ remaining digits, on the survivors
  // (a slice's survivors hold every key of its slice in the prefix's bin, so their histograms are the slice's)
#pragma unroll 1
  while (shift > 0 && bin_cnt != need) {
    const int nbits = shift == 10 ? 10 : 11;
    const int nshift = shift - nbits;
    const int nb = 1 << nbits;
    for (int i = tid; i < nb; i += kSelThreads) lh[i] = 0u;
    __syncthreads();
    for (uint32_t i = tid; i < stored; i += kSelThreads) {
      const uint32_t kv = skey[i];
      if ((kv & M) == P) atomicAdd(&lh[(kv >> nshift) & (uint32_t)(nb - 1)], 1u);
    }
    __syncthreads();
    uint32_t *gh = row_hist(nb);
    sel_find_bin(gh, nb, need, tmp, &s_bin, &s_above);
    P |= (uint32_t)s_bin << nshift;
    M |= (uint32_t)(nb - 1) << nshift;
    above += s_above;
    need -= s_above;
    bin_cnt = gh[s_bin];
    shift = nshift;
    release_row_hist(gh, nb);
  }

  // ------------------------------------------------------------------ ordered write of the selection
  // Survivors in tiles of 16 warp segments of 256, lane l of a segment holding entries 32 e + l (e = 0..7):
  // every survivor above the prefix is taken, and the first `need` of the row equal to it (the slices before
  // this one first).  A first sweep counts this slice's (above, equal) survivors for the later CTAs.
  const uint32_t lt_mask = (1u << lane) - 1u;
  uint32_t gt_loc = 0u, eq_loc = 0u;
  for (uint32_t i = tid; i < stored; i += kSelThreads) {
    const uint32_t km = skey[i] & M;
    gt_loc += km > P;
    eq_loc += km == P;
  }
  gt_loc = __reduce_add_sync(0xffffffffu, gt_loc);
  eq_loc = __reduce_add_sync(0xffffffffu, eq_loc);
  if (lane == 0) {
    tmp[warp] = gt_loc;
    tmp[kSelWarps + warp] = eq_loc;
  }
  __syncthreads();
  uint32_t gt_tot = 0u, eq_tot = 0u;
#pragma unroll
  for (int w = 0; w < kSelWarps; ++w) {
    gt_tot += tmp[w];
    eq_tot += tmp[kSelWarps + w];
  }
  uint32_t out_base = 0u, eq_seen = 0u;
  if (C > 1) {
    if (wait_pending) {
      sel_cl_wait();
      wait_pending = false;
    }
    if (tid > (int)r && tid < (int)C) {
      sel_cl_st(cnt_in + 2 * r, (uint32_t)tid, gt_tot);
      sel_cl_st(cnt_in + 2 * r + 1, (uint32_t)tid, eq_tot);
    }
    sel_cl_arrive();
    sel_cl_wait();
    for (uint32_t c = 0; c < r; ++c) {
      const uint32_t g = cnt_in[2 * c], e = cnt_in[2 * c + 1];
      out_base += g + (need > eq_seen ? min(e, need - eq_seen) : 0u);
      eq_seen += e;
    }
  }
  __syncthreads();
  uint32_t written = out_base;
  // every key of the prefix's bin is taken (the usual end of the digit passes): when every survivor of this slice
  // is above or in the bin, the survivors are the slice's output as they stand, in position order
  const bool all_eq = bin_cnt == need;
  if (all_eq && gt_tot + eq_tot == stored) {
    for (uint32_t i = tid; i < stored; i += kSelThreads)
      if (out_base + i < (uint32_t)a.k) out[out_base + i] = spos[i];
    written = out_base + stored;
    stored = 0u;                                        // (nothing left for the general write below)
  }
#pragma unroll 1
  for (uint32_t base = 0; base < stored; base += kSelThreads * 8) {
    const uint32_t i0 = base + (uint32_t)warp * 256u + (uint32_t)lane;
    uint32_t gtb[8], eqb[8], seg_eq = 0u;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint32_t i = i0 + 32u * e;
      const uint32_t km = i < stored ? (skey[i] & M) : 0u;
      gtb[e] = __ballot_sync(0xffffffffu, i < stored && km > P);
      eqb[e] = __ballot_sync(0xffffffffu, i < stored && km == P);
      seg_eq += __popc(eqb[e]);
    }
    if (lane == 0) tmp[warp] = seg_eq;
    __syncthreads();
    uint32_t eq_before_seg = eq_seen, eq_tile = 0u;
#pragma unroll
    for (int w = 0; w < kSelWarps; ++w) {
      eq_before_seg += w < warp ? tmp[w] : 0u;
      eq_tile += tmp[w];
    }
    uint32_t selb[8], seg_sel = 0u, run_eq = eq_before_seg;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint32_t my_rank = run_eq + __popc(eqb[e] & lt_mask);
      const bool take = ((eqb[e] >> lane) & 1u) && my_rank < need;
      selb[e] = gtb[e] | __ballot_sync(0xffffffffu, take);
      run_eq += __popc(eqb[e]);
      seg_sel += __popc(selb[e]);
    }
    eq_seen += eq_tile;
    __syncthreads();
    if (lane == 0) tmp[warp] = seg_sel;
    __syncthreads();
    uint32_t off = written, sel_tile = 0u;
#pragma unroll
    for (int w = 0; w < kSelWarps; ++w) {
      off += w < warp ? tmp[w] : 0u;
      sel_tile += tmp[w];
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if ((selb[e] >> lane) & 1u) {
        const uint32_t o = off + __popc(selb[e] & lt_mask);
        if (o < (uint32_t)a.k) out[o] = spos[i0 + 32u * e];
      }
      off += __popc(selb[e]);
    }
    written += sel_tile;
    __syncthreads();
  }
  // a consistent histogram always yields exactly k over the row; the last slice pads defensively otherwise
  if (r == C - 1) {
    for (uint32_t j = written + tid; j < (uint32_t)a.k; j += kSelThreads) out[j] = -1;
    if (written != (uint32_t)a.k && tid == 0) set_status(a.status, kStatusBadIndex);
  }
}

// ------------------------------------------------------------------------------------------------ host
// Survivor capacity: room for k plus the threshold bin of a typical row; at least k (so that the fully
// resolved threshold always fits) and at most what leaves two CTAs per SM possible for small k.
static int select_cap(int k) {
  int cap = std::max(2 * k, 8192);
  return std::min(cap, 24576);
}

// CTAs per row: enough to spread few rows over the SMs (half of them busy at most, so rows of a batch with
// many rows run one CTA each), no slice under 4096 keys, at most 16.  Measured on the decode batch (32 rows of
// 4K-32K keys): 4 CTAs per row select in about half the time of one.
static int select_cluster(int T, int max_seq_len, int num_sms) {
  int C = 1;
  while (C < 16 && (int64_t)T * C * 2 <= (int64_t)num_sms && (int64_t)max_seq_len >= (int64_t)C * 2 * 4096) C *= 2;
  return C;
}

// Largest cluster (16, 8, 4, 2 or 1 CTAs) the device can place at the largest shared-memory footprint; found
// once per device (threads racing on the first call compute the same value).
static int select_max_cluster(int num_sms) {
  static std::atomic<int> cached[kMaxDevices];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) dev = -1;
  int c = dev >= 0 ? cached[dev].load(std::memory_order_relaxed) : 0;
  if (c > 0) return c;
  const size_t smem = select_smem_bytes(select_cap(16384));
  cudaFuncSetAttribute(select_stream_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  cudaFuncSetAttribute(select_stream_kernel<false>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  for (c = 16; c > 1; c /= 2) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)c);
    cfg.blockDim = dim3(kSelThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = (unsigned)c;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, select_stream_kernel<false>, &cfg) == cudaSuccess && n >= 1) break;
    cudaGetLastError();
  }
  (void)num_sms;
  if (dev >= 0) cached[dev].store(c, std::memory_order_relaxed);
  return c;
}

dsa_status_t select_launch(const float *scores, int64_t ld, const dsa_batch_t *b, int k, int32_t *idx,
                           const uint32_t *hist, uint32_t *status, void *long_ws, cudaStream_t stream, int num_sms) {
  SelArgs a{};
  a.scores = scores;
  a.ld = ld;
  a.bv = view_of(b);
  a.k = k;
  a.idx = idx;
  a.hist = hist;
  a.cap = select_cap(k);
  a.status = status;
  const size_t smem = select_smem_bytes(a.cap);
  int C = std::min(select_cluster(b->total_q, b->max_seq_len, num_sms), select_max_cluster(num_sms));
  if (hist != nullptr && long_ws != nullptr && select_long_ws_bytes(b->total_q, b->max_seq_len) > 0) {
    // very long rows: the survivors are collected over every SM first, then one CTA per row goes on
    GatherArgs ga{};
    ga.scores = scores;
    ga.ld = ld;
    ga.bv = a.bv;
    ga.k = k;
    ga.hist = hist;
    ga.G = std::max(1, std::min(num_sms, kSelLongCtas) / b->total_q);
    const size_t slots = (size_t)kSelLongCtas * kSelSurvQ;
    ga.surv_key = (uint32_t *)long_ws;
    ga.surv_pos = (int32_t *)((uint32_t *)long_ws + slots);
    ga.surv_cnt = (uint32_t *)((char *)long_ws + (slots * 8 + 255) / 256 * 256);
    DSA_LAUNCH_PDL("select_gather_kernel", select_gather_kernel, dim3(b->total_q * ga.G), dim3(kSelThreads), 0, stream,
                   ga);
    a.surv_key = ga.surv_key;
    a.surv_pos = ga.surv_pos;
    a.surv_cnt = ga.surv_cnt;
    a.surv_ctas = ga.G;
    a.surv_q = kSelSurvQ;
    C = 1;
  }
  const bool gathered = a.surv_cnt != nullptr;
  cudaFuncSetAttribute(gathered ? select_stream_kernel<true> : select_stream_kernel<false>,
                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(b->total_q * C));
  cfg.blockDim = dim3(kSelThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)C;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t le = gathered ? cudaLaunchKernelEx(&cfg, select_stream_kernel<true>, a)
                                  : cudaLaunchKernelEx(&cfg, select_stream_kernel<false>, a);
  if (le != cudaSuccess) {
    set_error("select_stream_kernel: %s", cudaGetErrorString(le));
    return DSA_ERR_CUDA;
  }
  DSA_LAUNCH_CHECK("select_stream_kernel");
  return DSA_OK;
}

}  // namespace dsa
