// Exact per-row top-k over fp32 indexer scores (radix select in shared memory).
//
// Selection order: score descending, token position ascending (the lower position wins a tie;
// -0 == +0).  Scores are compared as order-preserving u32 keys, so the selection is exact.
// The k-th key T is found digit by digit (11 + 11 + 10 bits) with shared-memory histograms; every
// key > T is selected plus the lowest-positioned keys == T until k are taken.  The passes stop early once
// the threshold digit's bin holds exactly the keys still needed (keys are then compared on the digits
// fixed so far).  The result is
// written in ascending position order by a block-wide ordered compaction, so no sort is needed.
//
// Rows are grouped by row, buffered in shared memory and read with 16-byte vector loads, the
// structure the pages credit for their index-selection speed-up ("Engineering Practices for
// Day-0 Adaptation of Million-Token Context Models on Domestic AI Chips", Four Key Layers 1).
//
// Two regimes:
//   A) n <= C * kTopkSmemCap candidates: a cluster of C CTAs per row (C = 1, 2, 4 or 8: more when there
//      are few rows, so that the rows fill the GPU, and as many as the longest row needs, at most 2 for
//      a large batch), each CTA staging one contiguous slice of the row in shared memory.  Every digit
//      pass builds slice histograms whose non-zero bins each CTA adds into every CTA's copy of the row
//      histogram (distributed shared memory atomics, then one cluster barrier); the ordered write offsets
//      each slice by the counts of the slices before it, stored into the later CTAs.  One launch.
//   B) longer rows (a million-token decode): the row is split into segments of kTopkSeg keys over
//      a persistent grid; each digit pass is one launch whose CTAs add segment histograms into a
//      per-row global histogram, and the last CTA of a row to finish (atomic counter, no waiting)
//      picks the digit.  Then a count launch and an ordered-write launch.  No CTA ever waits for
//      another.
#include <algorithm>
#include <mutex>

#include <cuda.h>

#include "common.cuh"

namespace dsa {

constexpr int kTopkSmemCap = 49152;
constexpr int kTopkThreadsA = 1024;
constexpr int kTopkSeg = 8192;
constexpr int kTopkThreadsB = 512;
constexpr int kRadixBins = 2048;

struct TopkRowState {
  uint32_t prefix, pmask, k_rem, done;
};

// Workspace layout for regime B (after the 256-byte header):
//   [0]            u32 long-row count
//   [64 ..)        i32 long-row list [total_q]
//   state          TopkRowState [total_q]
//   hist           u32 [total_q][2048]
//   segcnt         uint2 [total_q][max_segs]   (gt, eq) per segment
struct TopkWs {
  uint32_t *count;
  int32_t *list;
  TopkRowState *state;
  uint32_t *hist;
  uint2 *segcnt;
  int max_segs;
};

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline int topk_max_segs(int max_seq_len) { return (max_seq_len + kTopkSeg - 1) / kTopkSeg; }

size_t topk_workspace_bytes(int total_q, int max_seq_len) {
  size_t bytes = kWsHeader;
  if (max_seq_len <= kTopkSmemCap) return bytes;
  size_t off = 64 + align_up((size_t)total_q * 4, 256);
  off += align_up((size_t)total_q * sizeof(TopkRowState), 256);
  off += align_up((size_t)total_q * kRadixBins * 4, 256);
  off += align_up((size_t)total_q * topk_max_segs(max_seq_len) * sizeof(uint2), 256);
  return bytes + off;
}

static TopkWs topk_ws_view(void *ws, int total_q, int max_seq_len) {
  char *p = (char *)ws + kWsHeader;
  TopkWs w;
  w.count = (uint32_t *)p;
  w.list = (int32_t *)(p + 64);
  size_t off = 64 + align_up((size_t)total_q * 4, 256);
  w.state = (TopkRowState *)(p + off);
  off += align_up((size_t)total_q * sizeof(TopkRowState), 256);
  w.hist = (uint32_t *)(p + off);
  off += align_up((size_t)total_q * kRadixBins * 4, 256);
  w.segcnt = (uint2 *)(p + off);
  w.max_segs = topk_max_segs(max_seq_len);
  return w;
}

// Threshold digit: among bins taken in descending order, the bin where the running count first
// reaches k_rem.  Returns the bin and the count of keys in higher bins.  All threads participate.
__device__ void find_threshold_bin(const uint32_t *hist, int nbins, uint32_t k_rem, uint32_t *tmp,
                                   int *s_bin, uint32_t *s_above) {
  const int per = (nbins + blockDim.x - 1) / blockDim.x;
  const int d0 = threadIdx.x * per;
  uint32_t local = 0;
  for (int d = d0; d < d0 + per && d < nbins; ++d) local += hist[nbins - 1 - d];
  uint32_t before = block_exclusive_scan(local, tmp, nullptr);
  uint32_t run = before;
  for (int d = d0; d < d0 + per && d < nbins; ++d) {
    uint32_t c = hist[nbins - 1 - d];
    if (run < k_rem && run + c >= k_rem) {
      *s_bin = nbins - 1 - d;
      *s_above = run;
    }
    run += c;
  }
  __syncthreads();
}

// The same for a block of at least 32 warps, in two levels: warp w sums the w-th group of nbins / 32 bins
// from the top, then warp 0 scans the 32 group sums, and scans the chosen group's bins (one or two per lane).
// Two block barriers.  Needs 1 <= k_rem <= the histogram's total (so one bin qualifies).
__device__ void find_threshold_bin_w32(const uint32_t *hist, int nbins, uint32_t k_rem, uint32_t *tmp,
                                       int *s_bin, uint32_t *s_above) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gsz = nbins >> 5;                                  // bins per group: 64 or 32
  if (warp < 32) {
    const int g0 = nbins - (warp + 1) * gsz;
    uint32_t s = 0;
    for (int j = lane; j < gsz; j += 32) s += hist[g0 + j];
    s = __reduce_add_sync(0xffffffffu, s);
    if (lane == 0) tmp[warp] = s;
  }
  __syncthreads();
  if (warp == 0) {
    // groups from the top: lane l holds group l; exactly one group holds the k_rem-th key
    const uint32_t gs = tmp[lane];
    uint32_t incl = gs;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int gw = __ffs(__ballot_sync(0xffffffffu, incl - gs < k_rem && incl >= k_rem)) - 1;
    const uint32_t above = __shfl_sync(0xffffffffu, incl - gs, gw);
    const uint32_t need = k_rem - above;
    // the group's bins from the top: lane l takes the per = gsz / 32 bins below top - per * l
    const int per = gsz >> 5;
    const int hi = nbins - gw * gsz - 1 - per * lane;
    const uint32_t c0 = hist[hi], c1 = per == 2 ? hist[hi - 1] : 0u;
    const uint32_t loc = c0 + c1;
    uint32_t incl2 = loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl2, o);
      if (lane >= o) incl2 += y;
    }
    const uint32_t excl2 = incl2 - loc;
    if (excl2 < need && incl2 >= need) {
      if (excl2 + c0 >= need) {
        *s_bin = hi;
        *s_above = above + excl2;
      } else {
        *s_bin = hi - 1;
        *s_above = above + excl2 + c0;
      }
    }
  }
  __syncthreads();
}

// keys[0..len) = the ordered keys of src[0..len) (src 16-byte aligned).  Each thread issues up to kV 16-byte
// loads before it converts any of them: a load followed at once by its use would cost a memory round trip
// per vector.
template <int kV>
__device__ __forceinline__ void stage_keys(const float *__restrict__ src, int len, uint32_t *keys) {
  const int l4 = len >> 2, bs = blockDim.x;
  const float4 *src4 = reinterpret_cast<const float4 *>(src);
  for (int i0 = threadIdx.x; i0 < l4; i0 += kV * bs) {
    float4 v[kV];
#pragma unroll
    for (int q = 0; q < kV; ++q)
      if (i0 + q * bs < l4) v[q] = __ldg(src4 + i0 + q * bs);
#pragma unroll
    for (int q = 0; q < kV; ++q)
      if (i0 + q * bs < l4)
        reinterpret_cast<uint4 *>(keys)[i0 + q * bs] =
            make_uint4(ordered_key(v[q].x), ordered_key(v[q].y), ordered_key(v[q].z), ordered_key(v[q].w));
  }
  for (int i = 4 * l4 + threadIdx.x; i < len; i += bs) keys[i] = ordered_key(__ldg(src + i));
}

// ------------------------------------------------------------------------------------------------
// Regime A
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cl_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cl_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
// red.shared::cluster.add of v to the u32 at the same shared-memory location in CTA `rank` of the cluster
__device__ __forceinline__ void cl_red_add(const void *p, uint32_t rank, uint32_t v) {
  uint32_t a = (uint32_t)__cvta_generic_to_shared(p), ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
  asm volatile("red.shared::cluster.add.u32 [%0], %1;" ::"r"(ra), "r"(v) : "memory");
}
__device__ __forceinline__ void cl_st(const void *p, uint32_t rank, uint32_t v) {
  uint32_t a = (uint32_t)__cvta_generic_to_shared(p), ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(ra), "r"(v) : "memory");
}
// (aligned forms: the warp is made converged first, as they require)
__device__ __forceinline__ void cl_arrive() {
  __syncwarp();
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cl_wait() {
  __syncwarp();
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// shared memory of a regime-A CTA: the slice histogram, two row histograms (alternating passes), scan scratch,
// the slices' counts for the ordered write (pairs, up to 16 CTAs), then the slice's keys
constexpr int kTopkMaxCluster = 16;
constexpr int kTopkSmemFixedU32 = 3 * kRadixBins + 64 + 2 * kTopkMaxCluster;

// Every access to another CTA's shared memory is a push (an add or a store) issued before a cluster barrier
// that the receiver waits on: the row histogram of a pass is the sum of the slice histograms' non-zero bins,
// added into every CTA's copy; the ordered write's offsets come from counts stored into the later CTAs.  No
// CTA reads a peer's shared memory, so none has to wait for its peers before it exits.
__global__ void __launch_bounds__(kTopkThreadsA, 2)
topk_rows_smem_kernel(const float *__restrict__ scores, int64_t ld, BatchView bv, int k,
                      int32_t *__restrict__ idx, TopkWs lw, int register_long) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) uint32_t sm[];
  uint32_t *hist = sm;                                   // this slice
  uint32_t *tmp = sm + 3 * kRadixBins;
  uint32_t *cnts = tmp + 64;                             // (keys > T, keys == T) of the slice of each rank
  uint32_t *keys = sm + kTopkSmemFixedU32;
  __shared__ int s_bin;
  __shared__ uint32_t s_above;

  const uint32_t C = cl_size(), r = cl_rank();
  const int row = blockIdx.x / (int)C;
  const int tid = threadIdx.x, bs = blockDim.x;
  // the row's length: one round of loads for a batch of one query row per sequence (the row is its
  // sequence: its entries are loaded beside the search's), two otherwise
  int n;
  {
    int sc0 = 0, sc1 = 0, ssl = 0;
    if (row < bv.num_seqs) {
      sc0 = __ldg(bv.cu_q + row);
      sc1 = __ldg(bv.cu_q + row + 1);
      ssl = __ldg(bv.seq_lens + row);
    }
    const int b = seq_of_row_warp(bv.cu_q, bv.num_seqs, row);
    if (b == row) {
      n = ssl - (sc1 - sc0) + (row - sc0) + 1;
    } else {
      const int c0 = __ldg(bv.cu_q + b), c1 = __ldg(bv.cu_q + b + 1);
      n = __ldg(bv.seq_lens + b) - (c1 - c0) + (row - c0) + 1;
    }
  }
  int32_t *out = idx + (int64_t)row * k;

  // (every branch below depends on n only, so all CTAs of a cluster take it together)
  if (n > (int)C * kTopkSmemCap) {
    // long row: hand it to regime B, initialise its state and histogram
    if (register_long && r == 0) {
      if (tid == 0) {
        uint32_t slot = atomicAdd(lw.count, 1u);
        lw.list[slot] = row;
        lw.state[row] = TopkRowState{0u, 0u, (uint32_t)k, 0u};
      }
      for (int i = tid; i < kRadixBins; i += bs) lw.hist[(int64_t)row * kRadixBins + i] = 0u;
    }
    return;
  }
  if (n <= k) {
    if (r == 0)
      for (int j = tid; j < k; j += bs) out[j] = j < n ? j : -1;
    return;
  }

  // both row histograms start empty before any peer adds into them: the barrier that publishes the clearing
  // is waited on just before the first push, so the slice load and histogram run meanwhile
  for (int i = tid; i < 2 * kRadixBins; i += bs) sm[kRadixBins + i] = 0u;
  if (C > 1) cl_arrive();

  // this CTA's slice [lo, lo + m): a multiple of 4 keys long, so 16-byte loads stay aligned
  const int slice = ((n + (int)C - 1) / (int)C + 3) & ~3;
  const int lo = min(n, (int)r * slice), m = min(n, lo + slice) - lo;
  stage_keys<2>(scores + (int64_t)row * ld + lo, m, keys);
  __syncthreads();

  uint32_t prefix = 0u, pmask = 0u, k_rem = (uint32_t)k;
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const int nb = pass == 2 ? 1024 : 2048;
    uint32_t *ghist = sm + kRadixBins * (1 + (pass & 1));   // the row histogram of this pass (even / odd)
    for (int i = tid; i < nb; i += bs) hist[i] = 0u;
    __syncthreads();
    for (int i = tid; i < m; i += bs) {
      uint32_t u = keys[i];
      if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & (nb - 1)], 1u);
    }
    __syncthreads();
    if (C > 1) {
      // add the slice's non-zero bins into every CTA's row histogram; the barrier completes the row histograms
      if (pass == 0) cl_wait();
      for (int i = tid; i < nb; i += bs) {
        const uint32_t v = hist[i];
        if (v != 0u)
          for (uint32_t c = 0; c < C; ++c) cl_red_add(ghist + i, c, v);
      }
      cl_arrive();
      cl_wait();
    } else {
      for (int i = tid; i < nb; i += bs) ghist[i] = hist[i];
      __syncthreads();
    }
    find_threshold_bin_w32(ghist, nb, k_rem, tmp, &s_bin, &s_above);
    prefix |= (uint32_t)s_bin << shift;
    pmask |= (uint32_t)(nb - 1) << shift;
    k_rem -= s_above;
    // every key of the threshold bin is taken: no finer digit can change the selection, so the keys are
    // compared on the digits fixed so far (the same row histogram in every CTA of the cluster: they all stop)
    const bool last = ghist[s_bin] == k_rem;
    __syncthreads();
    // this row histogram takes the adds of pass + 2, which peers make only after the next pass's barrier,
    // which this CTA reaches after clearing it
    for (int i = tid; i < nb; i += bs) ghist[i] = 0u;
    if (last) break;
  }
  const uint32_t T = prefix;

  // ordered compaction: each thread owns a contiguous range of the slice; the slice's output offset is
  // the selection of the slices before it (every key > T, keys == T in position order up to k_rem)
  const int per = (m + bs - 1) / bs;
  const int tlo = min(m, tid * per), thi = min(m, tlo + per);
  uint32_t gt = 0, eq = 0;
  for (int i = tlo; i < thi; ++i) {
    uint32_t u = keys[i] & pmask;
    gt += u > T;
    eq += u == T;
  }
  // both counts in one scan: (gt << 16) | eq never carries, a slice holding at most kTopkSmemCap < 65536 keys
  uint32_t tot;
  const uint32_t before = block_exclusive_scan((gt << 16) | eq, tmp, &tot);
  const uint32_t gt_tot = tot >> 16, eq_tot = tot & 0xFFFFu;
  uint32_t eq_before = before & 0xFFFFu;
  const uint32_t gt_before = before >> 16;
  uint32_t out_base = 0u, eq_base = 0u;
  if (C > 1) {
    // this slice's counts go to the CTAs after it
    if (tid > (int)r && tid < (int)C) {
      cl_st(cnts + 2 * r, (uint32_t)tid, gt_tot);
      cl_st(cnts + 2 * r + 1, (uint32_t)tid, eq_tot);
    }
    cl_arrive();
    cl_wait();
    for (uint32_t c = 0; c < r; ++c) {
      const uint32_t g = cnts[2 * c], e = cnts[2 * c + 1];
      const uint32_t take = k_rem > eq_base ? min(e, k_rem - eq_base) : 0u;
      out_base += g + take;
      eq_base += e;
    }
  }
  eq_before += eq_base;
  const uint32_t take_eq = k_rem > eq_before ? min(eq, k_rem - eq_before) : 0u;
  // equal keys taken before this thread, in this slice
  const uint32_t eq_taken_slice = min(eq_before, k_rem) - min(eq_base, k_rem);
  uint32_t off = out_base + gt_before + eq_taken_slice;
  uint32_t e = 0;
  for (int i = tlo; i < thi; ++i) {
    uint32_t u = keys[i] & pmask;
    bool sel = u > T;
    if (u == T) { sel = e < take_eq; ++e; }
    if (sel && off < (uint32_t)k) out[off++] = lo + i;
  }
}

// ------------------------------------------------------------------------------------------------
// Regime B (persistent over (long row, segment) items)
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ bool long_item(const TopkWs &w, const BatchView &bv, int item, int *row, int *seg,
                                          int *n, int *nseg) {
  const int r_i = item / w.max_segs;
  *seg = item % w.max_segs;
  *row = w.list[r_i];
  int b;
  *n = pos_of_row_warp(bv, *row, &b) + 1;
  *nseg = (*n + kTopkSeg - 1) / kTopkSeg;
  return *seg < *nseg;
}

// stage one segment's keys in shared memory; returns its length
__device__ int stage_segment(const float *__restrict__ scores, int64_t ld, int row, int seg, int n, uint32_t *keys) {
  const int lo = seg * kTopkSeg;
  const int len = min(kTopkSeg, n - lo);
  stage_keys<4>(scores + (int64_t)row * ld + lo, len, keys);
  __syncthreads();
  return len;
}

__global__ void __launch_bounds__(kTopkThreadsB)
topk_long_hist_kernel(const float *__restrict__ scores, int64_t ld, BatchView bv, TopkWs w, int pass) {
  pdl_wait();
  pdl_trigger();
  __shared__ __align__(16) uint32_t keys[kTopkSeg];
  __shared__ uint32_t hist[kRadixBins];
  __shared__ uint32_t tmp[64];
  __shared__ int s_bin, s_last;
  __shared__ uint32_t s_above;
  const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
  const int nb = pass == 2 ? 1024 : 2048;
  const int items = (int)(*w.count) * w.max_segs;
  for (int item = blockIdx.x; item < items; item += gridDim.x) {
    int row, seg, n, nseg;
    if (!long_item(w, bv, item, &row, &seg, &n, &nseg)) continue;
    const TopkRowState st = w.state[row];
    const int len = stage_segment(scores, ld, row, seg, n, keys);
    for (int i = threadIdx.x; i < nb; i += blockDim.x) hist[i] = 0u;
    __syncthreads();
    for (int i = threadIdx.x; i < len; i += blockDim.x) {
      uint32_t u = keys[i];
      if ((u & st.pmask) == st.prefix) atomicAdd(&hist[(u >> shift) & (nb - 1)], 1u);
    }
    __syncthreads();
    uint32_t *gh = w.hist + (int64_t)row * kRadixBins;
    for (int i = threadIdx.x; i < nb; i += blockDim.x)
      if (hist[i]) atomicAdd(gh + i, hist[i]);
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(&w.state[row].done, 1u) == (uint32_t)(nseg - 1);
    __syncthreads();
    if (s_last) {
      __threadfence();
      for (int i = threadIdx.x; i < nb; i += blockDim.x) {
        hist[i] = __ldcg(gh + i);
        gh[i] = 0u;
      }
      __syncthreads();
      find_threshold_bin(hist, nb, st.k_rem, tmp, &s_bin, &s_above);
      if (threadIdx.x == 0) {
        TopkRowState ns;
        ns.prefix = st.prefix | ((uint32_t)s_bin << shift);
        ns.pmask = st.pmask | ((uint32_t)(nb - 1) << shift);
        ns.k_rem = st.k_rem - s_above;
        ns.done = 0u;
        w.state[row] = ns;
      }
    }
    __syncthreads();
  }
}

__global__ void __launch_bounds__(kTopkThreadsB)
topk_long_count_kernel(const float *__restrict__ scores, int64_t ld, BatchView bv, TopkWs w) {
  pdl_wait();
  pdl_trigger();
  __shared__ __align__(16) uint32_t keys[kTopkSeg];
  __shared__ uint32_t tmp[64];
  const int items = (int)(*w.count) * w.max_segs;
  for (int item = blockIdx.x; item < items; item += gridDim.x) {
    int row, seg, n, nseg;
    if (!long_item(w, bv, item, &row, &seg, &n, &nseg)) continue;
    const uint32_t T = w.state[row].prefix;
    const int len = stage_segment(scores, ld, row, seg, n, keys);
    uint32_t gt = 0, eq = 0;
    for (int i = threadIdx.x; i < len; i += blockDim.x) {
      gt += keys[i] > T;
      eq += keys[i] == T;
    }
    uint32_t tg, te;
    block_exclusive_scan(gt, tmp, &tg);
    block_exclusive_scan(eq, tmp, &te);
    if (threadIdx.x == 0) w.segcnt[(int64_t)row * w.max_segs + seg] = make_uint2(tg, te);
    __syncthreads();
  }
}

__global__ void __launch_bounds__(kTopkThreadsB)
topk_long_write_kernel(const float *__restrict__ scores, int64_t ld, BatchView bv, TopkWs w, int k,
                       int32_t *__restrict__ idx) {
  pdl_wait();
  pdl_trigger();
  __shared__ __align__(16) uint32_t keys[kTopkSeg];
  __shared__ uint32_t tmp[64];
  __shared__ uint32_t s_gt_before, s_eq_before;
  const int items = (int)(*w.count) * w.max_segs;
  for (int item = blockIdx.x; item < items; item += gridDim.x) {
    int row, seg, n, nseg;
    if (!long_item(w, bv, item, &row, &seg, &n, &nseg)) continue;
    const TopkRowState st = w.state[row];
    const uint32_t T = st.prefix, k_rem = st.k_rem;
    // counts of the earlier segments of this row
    uint32_t g = 0, e = 0;
    for (int s = threadIdx.x; s < seg; s += blockDim.x) {
      uint2 c = w.segcnt[(int64_t)row * w.max_segs + s];
      g += c.x;
      e += c.y;
    }
    uint32_t tg, te;
    block_exclusive_scan(g, tmp, &tg);
    block_exclusive_scan(e, tmp, &te);
    if (threadIdx.x == 0) { s_gt_before = tg; s_eq_before = te; }
    const int len = stage_segment(scores, ld, row, seg, n, keys);   // syncs
    const uint32_t seg_gt_before = s_gt_before, seg_eq_before = s_eq_before;
    const int per = (len + blockDim.x - 1) / blockDim.x;
    const int lo = min(len, (int)threadIdx.x * per), hi = min(len, lo + per);
    uint32_t gt = 0, eq = 0;
    for (int i = lo; i < hi; ++i) {
      gt += keys[i] > T;
      eq += keys[i] == T;
    }
    const uint32_t eq_before = seg_eq_before + block_exclusive_scan(eq, tmp, nullptr);
    const uint32_t take_eq = k_rem > eq_before ? min(eq, k_rem - eq_before) : 0u;
    // selected before this thread = every gt of earlier segments + the eq ones taken there
    const uint32_t eq_taken_before_seg = min(seg_eq_before, k_rem);
    uint32_t off = seg_gt_before + eq_taken_before_seg + block_exclusive_scan(gt + take_eq, tmp, nullptr);
    int32_t *out = idx + (int64_t)row * k;
    uint32_t c = 0;
    const int base = seg * kTopkSeg;
    for (int i = lo; i < hi; ++i) {
      uint32_t u = keys[i];
      bool sel = u > T;
      if (u == T) { sel = c < take_eq; ++c; }
      if (sel && off < (uint32_t)k) out[off++] = base + i;
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------------------------------------
// host entry
// ------------------------------------------------------------------------------------------------
dsa_status_t topk_launch(const float *scores, int64_t ld, const dsa_batch_t *b, int k, int32_t *idx, void *ws,
                         cudaStream_t stream, int num_sms) {
  BatchView bv = view_of(b);
  // cluster size: enough CTAs per row to fill the GPU when there are few rows, then enough for the longest
  // row to fit in the cluster's shared memory.  Regime B suits a handful of very long rows; a large batch
  // of rows just past one CTA's capacity (a prefill chunk deep in a long prompt) is far cheaper here.
  // With many rows the length-driven growth stops at 2 CTAs, since every CTA then takes the shared memory
  // of the longest slice and fewer rows run at once; the rare longer rows of such a batch go to regime B.
  int C = 1;
  while (C < 8 && (int64_t)b->total_q * C * 2 <= num_sms) C *= 2;
  const int c_len_max = (int64_t)b->total_q * 2 > num_sms ? 2 : 8;
  while (C < c_len_max && (int64_t)b->max_seq_len > (int64_t)C * kTopkSmemCap) C *= 2;
  const bool has_long = (int64_t)b->max_seq_len > (int64_t)C * kTopkSmemCap;
  TopkWs lw{};
  if (has_long) {
    lw = topk_ws_view(ws, b->total_q, b->max_seq_len);
    if (cudaMemsetAsync(lw.count, 0, 4, stream) != cudaSuccess) {
      set_error("topk: cudaMemsetAsync failed");
      return DSA_ERR_CUDA;
    }
  }
  const int slice_max = std::min(kTopkSmemCap, ((b->max_seq_len + C - 1) / C + 3) & ~3);
  const size_t smem = (size_t)(kTopkSmemFixedU32 + std::max(slice_max, 4)) * 4;
  cudaFuncSetAttribute(topk_rows_smem_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  cudaFuncSetAttribute(topk_rows_smem_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(b->total_q * C));
    cfg.blockDim = dim3(kTopkThreadsA);
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
    const int reg_long = has_long ? 1 : 0;
    const cudaError_t le = cudaLaunchKernelEx(&cfg, topk_rows_smem_kernel, scores, ld, bv, k, idx, lw, reg_long);
    if (le != cudaSuccess) {
      set_error("topk_rows_smem_kernel: %s", cudaGetErrorString(le));
      return DSA_ERR_CUDA;
    }
    DSA_LAUNCH_CHECK("topk_rows_smem_kernel");
  }
  if (has_long) {
    const int grid = max(num_sms * 4, topk_max_segs(b->max_seq_len));   // one segment per CTA per row
    for (int pass = 0; pass < 3; ++pass) {
      DSA_LAUNCH_PDL("topk_long_hist_kernel", topk_long_hist_kernel, dim3(grid), dim3(kTopkThreadsB), 0, stream, scores,
                     ld, bv, lw, pass);
    }
    DSA_LAUNCH_PDL("topk_long_count_kernel", topk_long_count_kernel, dim3(grid), dim3(kTopkThreadsB), 0, stream, scores,
                   ld, bv, lw);
    DSA_LAUNCH_PDL("topk_long_write_kernel", topk_long_write_kernel, dim3(grid), dim3(kTopkThreadsB), 0, stream, scores,
                   ld, bv, lw, k, idx);
  }
  return DSA_OK;
}

// ------------------------------------------------------------------------------------------------
// Allocation-free variant.  Its scratch (long-row histograms, row states, segment counts and the status
// header) is one file-scope device array, sized for at most kNoAllocMaxRows query rows and rows of at
// most kNoAllocMaxSeqLen candidates.  Every device that loads the library holds it until the process
// exits.  Host code must not hand the array's host-side name to a kernel: it is only a stand-in there,
// so the device address is looked up with cudaGetSymbolAddress once per device (and context) and cached.
// ------------------------------------------------------------------------------------------------
constexpr int kNoAllocMaxRows = 256;
constexpr int kNoAllocMaxSeqLen = 1 << 20;
constexpr size_t al256c(size_t x) { return (x + 255) / 256 * 256; }
constexpr size_t kNoAllocBytes =
    kWsHeader + 64 + al256c((size_t)kNoAllocMaxRows * 4) + al256c((size_t)kNoAllocMaxRows * sizeof(TopkRowState)) +
    al256c((size_t)kNoAllocMaxRows * kRadixBins * 4) +
    al256c((size_t)kNoAllocMaxRows * ((kNoAllocMaxSeqLen + kTopkSeg - 1) / kTopkSeg) * sizeof(uint2));

static __device__ __align__(256) unsigned char g_topk_scratch[kNoAllocBytes];

// Device address of the array in the current context.  Looked up once per device and context: a device
// reset (or any other teardown of the context) unloads the module, and the array's address in the new
// context may differ, so the cached address is keyed on the context's unique ID as well.
struct ScratchAddr {
  unsigned long long ctx_id;
  void *ptr;
};
static ScratchAddr g_topk_scratch_addr[kMaxDevices];
static std::mutex g_topk_scratch_mu;

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

// unique ID of the calling thread's current context (0 if there is none or the driver cannot say)
static unsigned long long current_ctx_id() {
  static const CtxGetCurrentFn get_cur = []() -> CtxGetCurrentFn {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    return cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
                   q == cudaDriverEntryPointSuccess ? (CtxGetCurrentFn)p : nullptr;
  }();
  static const CtxGetIdFn get_id = []() -> CtxGetIdFn {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    return cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
                   q == cudaDriverEntryPointSuccess ? (CtxGetIdFn)p : nullptr;
  }();
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_cur && get_id && get_cur(&ctx) == CUDA_SUCCESS && ctx != nullptr && get_id(ctx, &id) == CUDA_SUCCESS) return id;
  return 0;
}

static dsa_status_t topk_scratch_address(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    set_error("dsa_topk_noalloc: no current CUDA device");
    return DSA_ERR_CUDA;
  }
  // the runtime makes the device's primary context current on its first call above
  const unsigned long long ctx = current_ctx_id();
  std::lock_guard<std::mutex> g(g_topk_scratch_mu);
  ScratchAddr &c = g_topk_scratch_addr[dev];
  if (c.ptr == nullptr || ctx == 0 || c.ctx_id != ctx) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_topk_scratch);
    if (e != cudaSuccess || p == nullptr) {
      set_error("dsa_topk_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
      return DSA_ERR_CUDA;
    }
    c.ptr = p;
    c.ctx_id = ctx;
  }
  *out = c.ptr;
  return DSA_OK;
}

dsa_status_t topk_noalloc_launch(const float *scores, int64_t ld, const dsa_batch_t *b, int k, int32_t *idx,
                                 cudaStream_t stream, int num_sms) {
  if (b->total_q > kNoAllocMaxRows || b->max_seq_len > kNoAllocMaxSeqLen ||
      topk_workspace_bytes(b->total_q, b->max_seq_len) > kNoAllocBytes) {
    set_error("dsa_topk_noalloc: batch exceeds the built-in scratch (at most %d rows of at most %d candidates; "
              "got %d rows, max_seq_len %d)", kNoAllocMaxRows, kNoAllocMaxSeqLen, b->total_q, b->max_seq_len);
    return DSA_ERR_UNSUPPORTED;
  }
  void *scratch = nullptr;
  dsa_status_t st = topk_scratch_address(&scratch);
  if (st != DSA_OK) return st;
  return topk_launch(scores, ld, b, k, idx, scratch, stream, num_sms);
}

}  // namespace dsa
