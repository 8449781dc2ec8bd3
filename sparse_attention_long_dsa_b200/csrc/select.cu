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
constexpr int kSelPerThread = 16;                       // consecutive keys per thread per tile (4 x float4)
constexpr int kSelTile = kSelThreads * kSelPerThread;   // 8192 keys

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
// it in *s_bin and the count of keys in higher bins in *s_above.  Every thread of the block calls this.
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

// keys of the slice tile starting at `base` (kSelPerThread consecutive per thread); positions past m get
// valid = false
__device__ __forceinline__ void sel_load_tile(const float *src, int m, int base, uint32_t (&key)[kSelPerThread],
                                              uint32_t &valid) {
  const int i0 = base + threadIdx.x * kSelPerThread;
  valid = 0u;
  if (i0 + kSelPerThread <= m) {
#pragma unroll
    for (int v = 0; v < kSelPerThread / 4; ++v) {
      const float4 f = __ldg(reinterpret_cast<const float4 *>(src + i0) + v);
      key[4 * v] = ordered_key(f.x);
      key[4 * v + 1] = ordered_key(f.y);
      key[4 * v + 2] = ordered_key(f.z);
      key[4 * v + 3] = ordered_key(f.w);
    }
    valid = 0xFFFFu;
  } else {
#pragma unroll
    for (int e = 0; e < kSelPerThread; ++e) {
      const bool in = i0 + e < m;
      key[e] = in ? ordered_key(__ldg(src + i0 + e)) : 0u;
      valid |= (in ? 1u : 0u) << e;
    }
  }
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
  const int n = pos_of_row(a.bv, row, &b) + 1;
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
#pragma unroll 1
  for (int base = 0; base < m; base += kSelTile) {
    uint32_t key[kSelPerThread], valid;
    sel_load_tile(src, m, base, key, valid);
    uint32_t keep = 0u, eq = 0u;
#pragma unroll
    for (int e = 0; e < kSelPerThread; ++e) {
      const uint32_t km = key[e] & M;
      if ((valid >> e) & 1u) {
        if (km > P) keep |= 1u << e;
        else if (km == P) eq |= 1u << e;
      }
    }
    if (full) {
      // equal keys taken in position order: the first `need` of the row
      uint32_t eq_tot;
      const uint32_t eq_ex = block_exclusive_scan(__popc(eq), tmp, &eq_tot);
      uint32_t rank_eq = eq_before + eq_ex;
#pragma unroll
      for (int e = 0; e < kSelPerThread; ++e)
        if ((eq >> e) & 1u) {
          if (rank_eq < need) keep |= 1u << e;
          ++rank_eq;
        }
      eq_before += eq_tot;
    } else {
      keep |= eq;
    }
    uint32_t tot;
    uint32_t off = stored + block_exclusive_scan(__popc(keep), tmp, &tot);
    const int i0 = base + tid * kSelPerThread;
#pragma unroll
    for (int e = 0; e < kSelPerThread; ++e)
      if ((keep >> e) & 1u) {
        if (off < cap) {
          skey[off] = key[e];
          spos[off] = lo + i0 + e;
        } else {
          s_flag = 1u;
        }
        ++off;
      }
    stored += tot;
  }
  if (stored > cap) stored = cap;
  __syncthreads();
  if (s_flag && tid == 0) set_status(a.status, kStatusBadIndex);

  // ------------------------------------------------------------------ rank 0 collects the cluster's survivors
  if (C > 1) {
    if (tid == 0) info[0] = stored;
    tc::cluster_sync();                          // every slice's survivors are in place
    if (r == 0) {
      uint32_t total = stored;
      for (uint32_t c = 1; c < C; ++c) {
        const uint32_t cnt = sel_cl_ld(info, c);
        const uint32_t take = total + cnt <= cap ? cnt : cap - total;
        if (take < cnt && tid == 0) set_status(a.status, kStatusBadIndex);
        const uint32_t kaddr = tc::map_to_rank(tc::smem_u32(skey), c);
        const uint32_t paddr = tc::map_to_rank(tc::smem_u32(spos), c);
        for (uint32_t i = tid; i < take; i += kSelThreads) {
          uint32_t kv, pv;
          asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(kv) : "r"(kaddr + 4 * i) : "memory");
          asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(pv) : "r"(paddr + 4 * i) : "memory");
          skey[total + i] = kv;
          spos[total + i] = (int32_t)pv;
        }
        total += take;
      }
      stored = total;
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
  uint32_t written = 0u, eq_seen = 0u;
#pragma unroll 1
  for (uint32_t base = 0; base < stored; base += kSelTile) {
    const uint32_t i0 = base + tid * kSelPerThread;
    uint32_t gt = 0u, eq = 0u;
#pragma unroll
    for (int e = 0; e < kSelPerThread; ++e) {
      if (i0 + e < stored) {
        const uint32_t kv = skey[i0 + e];
        if (kv > P) gt |= 1u << e;
        else if (kv == P) eq |= 1u << e;
      }
    }
    uint32_t eq_tot;
    uint32_t rank_eq = eq_seen + block_exclusive_scan(__popc(eq), tmp, &eq_tot);
    uint32_t sel = gt;
#pragma unroll
    for (int e = 0; e < kSelPerThread; ++e)
      if ((eq >> e) & 1u) {
        if (rank_eq < need) sel |= 1u << e;
        ++rank_eq;
      }
    eq_seen += eq_tot;
    uint32_t tot;
    uint32_t off = written + block_exclusive_scan(__popc(sel), tmp, &tot);
#pragma unroll
    for (int e = 0; e < kSelPerThread; ++e)
      if ((sel >> e) & 1u) {
        if (off < (uint32_t)a.k) out[off] = spos[i0 + e];
        ++off;
      }
    written += tot;
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

// CTAs per row: enough to spread few rows over the SMs (two per SM), no slice under 2048 keys, at most 16.
static int select_cluster(int T, int max_seq_len, int num_sms) {
  int C = 1;
  while (C < 16 && (int64_t)T * C * 2 * 2 <= (int64_t)num_sms * 2 && (int64_t)max_seq_len >= (int64_t)C * 2 * 4096)
    C *= 2;
  return C;
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
  cudaFuncSetAttribute(select_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  cudaFuncSetAttribute(select_stream_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  int C = select_cluster(b->total_q, b->max_seq_len, num_sms);
  for (;; C /= 2) {
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
    if (C > 1) {
      // a cluster that cannot be placed is not launched: fall back to a smaller one
      int nclusters = 0;
      if (cudaOccupancyMaxActiveClusters(&nclusters, select_stream_kernel, &cfg) != cudaSuccess || nclusters < 1) {
        cudaGetLastError();
        continue;
      }
    }
    const cudaError_t le = cudaLaunchKernelEx(&cfg, select_stream_kernel, a);
    if (le != cudaSuccess) {
      set_error("select_stream_kernel: %s", cudaGetErrorString(le));
      return DSA_ERR_CUDA;
    }
    DSA_LAUNCH_CHECK("select_stream_kernel");
    return DSA_OK;
  }
}

}  // namespace dsa
