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
// Per row a cluster of C CTAs (C = 1 .. 16) takes contiguous slices.  State shared by the cluster: the
// fixed key bits (prefix P under mask M), the count `above` of keys strictly above the prefix, the number
// `need` still to take from the prefix's bin, and that bin's size.  While the survivors would not fit in
// the capacity, one more streaming pass histograms the next digit (11, 11 then 10 bits) among keys in the
// bin, summed over the cluster through distributed shared memory.  When every bit is fixed, keys equal to
// the threshold are kept in position order up to `need`, so the survivors are then exactly k.  The storing
// pass compacts survivors in position order; rank 0 collects the other slices' survivors after its own,
// resolves the remaining bits on them and emits every survivor above the threshold plus the first `need`
// equal ones.  Without a histogram (plain scores) the first pass counts the leading digit itself.
#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstdlib>

#include "tc.cuh"

namespace dsa {

constexpr int kSelThreads = 512;
constexpr int kSelBins = 2048;
constexpr int kSelPerThread = 8;                        // keys per thread per tile (2 x float4)
constexpr int kSelTile = kSelThreads * kSelPerThread;   // 4096 keys

struct SelArgs {
  const float *scores;
  int64_t ld;
  BatchView bv;
  int k;
  int32_t *idx;
  const uint32_t *hist;    // [T][2048] leading-digit counts of each row's causal keys, or nullptr
  int cap;                 // survivors a CTA can hold (shared memory)
  uint32_t *status;
};

// shared memory: survivors (key, position) [cap], two local histograms, the cluster histogram, scan scratch,
// per-CTA counts read by the other CTAs of the cluster
constexpr int kSelFixedWords = 3 * kSelBins + 64 + 8;
size_t select_smem_bytes(int cap) { return ((size_t)2 * cap + kSelFixedWords) * 4; }

__device__ __forceinline__ uint32_t sel_cl_nranks() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
// u32 at the same shared-memory location in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t sel_cl_ld(const void *p, uint32_t rank) {
  const uint32_t ra = tc::map_to_rank(tc::smem_u32(p), rank);
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(ra) : "memory");
  return v;
}

// Bin holding the need-th key counted from the top of hist[0..nb) (need >= 1, at most the total).  Returns
// it in *s_bin and the count of keys in higher bins in *s_above.  Every thread of the block calls this (a
// block scan over per-thread runs of bins in descending order).
__device__ void sel_find_bin(const uint32_t *hist, int nb, uint32_t need, uint32_t *tmp, int *s_bin,
                             uint32_t *s_above) {
  const int per = (nb + kSelThreads - 1) / kSelThreads;
  const int d0 = threadIdx.x * per;                    // position in descending bin order
  if (threadIdx.x == 0) {                              // (a consistent histogram always overwrites these)
    *s_bin = 0;
    *s_above = 0u;
  }
  uint32_t local = 0;
  for (int d = d0; d < d0 + per && d < nb; ++d) local += hist[nb - 1 - d];
  uint32_t run = block_exclusive_scan(local, tmp, nullptr);
  for (int d = d0; d < d0 + per && d < nb; ++d) {
    const uint32_t c = hist[nb - 1 - d];
    if (run < need && run + c >= need) {
      *s_bin = nb - 1 - d;
      *s_above = run;
    }
    run += c;
  }
  __syncthreads();
}

// A tile of kSelTile keys is 16 warp segments of 32 x kSelPerThread in position order; in its segment a lane
// holds the keys at 128 v + 4 lane + j (v < kSelPerThread / 4, j = 0..3), read as coalesced float4 loads.
// key[4 v + j]; valid bit 4 v + j is clear for positions at or past m.
__device__ __forceinline__ int sel_elem(int base, int v, int j) {
  return base + (int)(threadIdx.x >> 5) * (32 * kSelPerThread) + 128 * v + 4 * (int)(threadIdx.x & 31) + j;
}
__device__ __forceinline__ void sel_load_tile(const float *src, int m, int base, uint32_t (&key)[kSelPerThread],
                                              uint32_t &valid) {
  valid = 0u;
#pragma unroll
  for (int v = 0; v < kSelPerThread / 4; ++v) {
    const int i0 = sel_elem(base, v, 0);
    if (i0 + 4 <= m) {
      const float4 f = __ldg(reinterpret_cast<const float4 *>(src + i0));
      key[4 * v] = ordered_key(f.x);
      key[4 * v + 1] = ordered_key(f.y);
      key[4 * v + 2] = ordered_key(f.z);
      key[4 * v + 3] = ordered_key(f.w);
      valid |= 0xFu << (4 * v);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const bool in = i0 + j < m;
        key[4 * v + j] = in ? ordered_key(__ldg(src + i0 + j)) : 0u;
        valid |= (in ? 1u : 0u) << (4 * v + j);
      }
    }
  }
}

// Ordered positions of flagged items in a tile laid out as sel_elem describes: flags bit 4 v + j.  Returns, for
// each v, the count of flagged items before (v, lane, 0) in the tile (pre[v]), and the tile's total; `wsum`
// holds 32 words of shared scratch.  One __syncthreads inside, one more before wsum is reused.
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
  for (int w = 0; w < kSelThreads / 32; ++w) {
    const uint32_t x = wsum[w];
    before += w < warp ? x : 0u;
    total += x;
  }
#pragma unroll
  for (int v = 0; v < kSelPerThread / 4; ++v) pre[v] += before;
  return total;
}

__global__ void __launch_bounds__(kSelThreads) select_stream_kernel(const SelArgs a) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) uint32_t sm[];
  uint32_t *skey = sm;
  int32_t *spos = reinterpret_cast<int32_t *>(sm + a.cap);
  uint32_t *lh[2] = {sm + 2 * a.cap, sm + 2 * a.cap + kSelBins};
  uint32_t *gh = sm + 2 * a.cap + 2 * kSelBins;
  uint32_t *tmp = gh + kSelBins;
  uint32_t *info = tmp + 64;           // [0] survivors stored, [1] keys equal to the final prefix in this slice
  __shared__ int s_bin;
  __shared__ uint32_t s_above, s_flag;

  const uint32_t C = sel_cl_nranks(), r = tc::cluster_ctarank();
  const int row = blockIdx.x / (int)C;
  const int tid = threadIdx.x;
  int b;
  const int n = pos_of_row_warp(a.bv, row, &b) + 1;
  int32_t *out = a.idx + (int64_t)row * a.k;
  // (every branch on n is taken by the whole cluster)
  if (n <= a.k) {
    if (r == 0)
      for (int j = tid; j < a.k; j += kSelThreads) out[j] = j < n ? j : -1;
    return;
  }
  const int per = ((n + (int)C - 1) / (int)C + 3) & ~3;
  const int lo = min(n, (int)r * per), m = min(n, lo + per) - lo;
  const float *src = a.scores + (int64_t)row * a.ld + lo;
  const uint32_t cap = (uint32_t)a.cap;

  uint32_t P = 0u, M = 0u, above = 0u, need = (uint32_t)a.k, bin_cnt = (uint32_t)n, local_eq = 0u;
  int shift = 32;
  // the slice's first tile is read while the threshold digit is found
  uint32_t key0[kSelPerThread], valid0;
  sel_load_tile(src, m, 0, key0, valid0);
  if (a.hist != nullptr) {
    const uint32_t *hr = a.hist + (int64_t)row * kSelBins;
    for (int i = tid; i < kSelBins; i += kSelThreads) gh[i] = __ldcg(hr + i);
    __syncthreads();
    sel_find_bin(gh, kSelBins, need, tmp, &s_bin, &s_above);
    P = (uint32_t)s_bin << 21;
    M = 0xFFE00000u;
    above = s_above;
    need -= s_above;
    bin_cnt = gh[s_bin];
    shift = 21;
    __syncthreads();
  }
  // ------------------------------------------------------------------ counting passes (next digit)
  int pass = 0;
#pragma unroll 1
  while (shift > 0 && (shift == 32 || above + bin_cnt > cap)) {
    const int nbits = shift == 10 ? 10 : 11;
    const int nshift = shift - nbits;
    const int nb = 1 << nbits;
    uint32_t *h = lh[pass & 1];
    for (int i = tid; i < nb; i += kSelThreads) h[i] = 0u;
    __syncthreads();
    for (int base = 0; base < m; base += kSelTile) {
      uint32_t key[kSelPerThread], valid;
      sel_load_tile(src, m, base, key, valid);
#pragma unroll
      for (int e = 0; e < kSelPerThread; ++e)
        if (((valid >> e) & 1u) && (key[e] & M) == P) atomicAdd(&h[(key[e] >> nshift) & (uint32_t)(nb - 1)], 1u);
    }
    __syncthreads();
    if (C > 1) {
      tc::cluster_sync();
      for (int i = tid; i < nb; i += kSelThreads) {
        uint32_t sum = 0u;
        for (uint32_t c = 0; c < C; ++c) sum += sel_cl_ld(h + i, c);
        gh[i] = sum;
      }
    } else {
      for (int i = tid; i < nb; i += kSelThreads) gh[i] = h[i];
    }
    __syncthreads();
    sel_find_bin(gh, nb, need, tmp, &s_bin, &s_above);
    P |= (uint32_t)s_bin << nshift;
    M |= (uint32_t)(nb - 1) << nshift;
    above += s_above;
    need -= s_above;
    bin_cnt = gh[s_bin];
    local_eq = h[s_bin];
    shift = nshift;
    ++pass;
    __syncthreads();
  }
  const bool full = shift == 0;      // P is the exact threshold key; take `need` of the keys equal to it

  // keys equal to the threshold in lower-ranked slices (full case: they come first in position order)
  uint32_t eq_before = 0u;
  if (full && C > 1) {
    if (tid == 0) info[1] = local_eq;
    tc::cluster_sync();
    for (uint32_t c = 0; c < r; ++c) eq_before += sel_cl_ld(info + 1, c);
  }

  // ------------------------------------------------------------------ storing pass: ordered survivors
  uint32_t stored = 0u;                // survivors written so far (block-uniform)
  if (tid == 0) s_flag = 0u;
  uint32_t kn[kSelPerThread], vn = 0u;  // the next tile, loaded while this one is compacted
#pragma unroll 1
  for (int base = 0; base < m; base += kSelTile) {
    uint32_t key[kSelPerThread], valid;
#pragma unroll
    for (int e = 0; e < kSelPerThread; ++e) key[e] = base == 0 ? key0[e] : kn[e];
    valid = base == 0 ? valid0 : vn;
    if (base + kSelTile < m) sel_load_tile(src, m, base + kSelTile, kn, vn);
    uint32_t keep = 0u, eq = 0u;
#pragma unroll
    for (int e = 0; e < kSelPerThread; ++e) {
      const uint32_t km = key[e] & M;
      if ((valid >> e) & 1u) {
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
            skey[off] = key[4 * v + j];
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
  if (stored > cap) stored = cap;
  __syncthreads();
  if (s_flag && tid == 0) set_status(a.status, kStatusBadIndex);

  // ------------------------------------------------------------------ rank 0 collects the cluster's survivors
  if (C > 1) {
    if (tid == 0) info[0] = stored;
    tc::cluster_sync();                          // every slice's survivors are in place
    if (r == 0) {
      // the other slices' counts, their offsets after this slice's survivors, then every piece in one round
      uint32_t *offs = lh[0];                    // (free here) offs[c] = first slot of slice c, offs[C] = end
      if (tid == 0) {
        uint32_t total = stored;
        offs[0] = 0u;
        for (uint32_t c = 1; c < C; ++c) {
          const uint32_t cnt = sel_cl_ld(info, c);
          offs[c] = total;
          total += cnt;
        }
        offs[C] = total;
        if (total > cap) set_status(a.status, kStatusBadIndex);
      }
      __syncthreads();
      const uint32_t end = min(offs[C], cap);
      for (uint32_t i = stored + tid; i < end; i += kSelThreads) {
        uint32_t c = 1;
        while (c + 1 < C && offs[c + 1] <= i) ++c;
        const uint32_t j = i - offs[c];
        uint32_t kv, pv;
        asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(kv) : "r"(tc::map_to_rank(tc::smem_u32(skey + j), c)) : "memory");
        asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(pv) : "r"(tc::map_to_rank(tc::smem_u32(spos + j), c)) : "memory");
        skey[i] = kv;
        spos[i] = (int32_t)pv;
      }
      stored = end;
    }
    tc::cluster_sync();                          // rank 0 has read every other slice
    if (r != 0) return;
  }
  __syncthreads();

  // ------------------------------------------------------------------ remaining digits on the survivors
#pragma unroll 1
  while (shift > 0) {
    const int nbits = shift == 10 ? 10 : 11;
    const int nshift = shift - nbits;
    const int nb = 1 << nbits;
    uint32_t *h = lh[0];
    for (int i = tid; i < nb; i += kSelThreads) h[i] = 0u;
    __syncthreads();
    for (uint32_t i = tid; i < stored; i += kSelThreads) {
      const uint32_t kv = skey[i];
      if ((kv & M) == P) atomicAdd(&h[(kv >> nshift) & (uint32_t)(nb - 1)], 1u);
    }
    __syncthreads();
    sel_find_bin(h, nb, need, tmp, &s_bin, &s_above);
    P |= (uint32_t)s_bin << nshift;
    M |= (uint32_t)(nb - 1) << nshift;
    above += s_above;
    need -= s_above;
    shift = nshift;
    __syncthreads();
  }
  // P is now the k-th key: emit every survivor above it and the first `need` equal to it, in order
  // survivors in tiles of 16 warp segments of 256, lane l of a segment holding entries 32 e + l (e = 0..7)
  uint32_t written = 0u, eq_seen = 0u;
  const int lane = tid & 31, warp = tid >> 5;
  const uint32_t lt_mask = (1u << lane) - 1u;
#pragma unroll 1
  for (uint32_t base = 0; base < stored; base += kSelThreads * 8) {
    const uint32_t i0 = base + (uint32_t)warp * 256u + (uint32_t)lane;
    uint32_t gtb[8], eqb[8], seg_eq = 0u;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint32_t i = i0 + 32u * e;
      const uint32_t kv = i < stored ? skey[i] : 0u;
      gtb[e] = __ballot_sync(0xffffffffu, i < stored && kv > P);
      eqb[e] = __ballot_sync(0xffffffffu, i < stored && kv == P);
      seg_eq += __popc(eqb[e]);
    }
    // equal keys in position order: the first `need` of all survivors are taken
    if (lane == 0) tmp[warp] = seg_eq;
    __syncthreads();
    uint32_t eq_before_seg = eq_seen, eq_tile = 0u;
    for (int w = 0; w < kSelThreads / 32; ++w) {
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
    for (int w = 0; w < kSelThreads / 32; ++w) {
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
  // a consistent histogram always yields exactly k; pad defensively otherwise
  for (uint32_t j = written + tid; j < (uint32_t)a.k; j += kSelThreads) out[j] = -1;
  if (written != (uint32_t)a.k && tid == 0) set_status(a.status, kStatusBadIndex);
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
  cudaFuncSetAttribute(select_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  cudaFuncSetAttribute(select_stream_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
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
    if (cudaOccupancyMaxActiveClusters(&n, select_stream_kernel, &cfg) == cudaSuccess && n >= 1) break;
    cudaGetLastError();
  }
  (void)num_sms;
  if (dev >= 0) cached[dev].store(c, std::memory_order_relaxed);
  return c;
}

dsa_status_t select_launch(const float *scores, int64_t ld, const dsa_batch_t *b, int k, int32_t *idx,
                           const uint32_t *hist, uint32_t *status, cudaStream_t stream, int num_sms) {
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
  const int C = std::min(select_cluster(b->total_q, b->max_seq_len, num_sms), select_max_cluster(num_sms));
  cudaFuncSetAttribute(select_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
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
  const cudaError_t le = cudaLaunchKernelEx(&cfg, select_stream_kernel, a);
  if (le != cudaSuccess) {
    set_error("select_stream_kernel: %s", cudaGetErrorString(le));
    return DSA_ERR_CUDA;
  }
  DSA_LAUNCH_CHECK("select_stream_kernel");
  return DSA_OK;
}

}  // namespace dsa
