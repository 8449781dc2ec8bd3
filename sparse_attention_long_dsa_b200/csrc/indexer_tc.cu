// FP8 indexer scores on the 5th-generation tensor cores (tcgen05, sm_100a).
//
//   scores[row, s] = kS[s] * sum_j w[row, j] * max(0, sum_d qI[row, j, d] * kI8[s, d]),  s <= pos(row)
//
// ("Day-0 Adaptation for LLMs: Implementing Sparse Attention and Low-Precision Weights", III.1:
// the lightweight indexer scores each query against every historical token, at higher precision
// than attention.  The FP8 products are exact and accumulate in fp32; the scorer's form is the one
// this library takes for the pages' open "indexer(q, kv_meta)".)  kS is factored out of the ReLU,
// which is exact because kS > 0 and ReLU is positively homogeneous.
//
// Contraction per tile: D[128 keys, 64*R] = K[128 keys, 128] x Q[64*R, 128]^T with R <= 4 query
// rows of one sequence sharing the keys (prefill / chunked prefill) or R = 1 (decode).  Keys are the
// M dimension so that each TMEM lane holds one key and the weighted ReLU sum over heads is a
// per-thread reduction with no shuffles.  A 128-key tile is two 64-token pages fetched by TMA through
// the block table (128-byte swizzle, the layout the MMA descriptor reads).
//
// Warp roles (416 threads, persistent, one CTA per SM):
//   warps 0,6-8  TMA producers: key tiles into an 8-stage ring (round-robin over the four warps); warp 0
//                also loads the query rows + weights of each row group
//   warp 1       allocates 512 TMEM columns; lane 0 issues 4 MMAs (K = 32 each) per tile into one of two
//                256-column accumulators and commits them to the ring / accumulator barriers
//   warps 2..5,  epilogue, two groups taking alternate tiles (one accumulator each): tcgen05.ld 64 heads per
//   9..12        row, ReLU, weight, sum, key scale, causal store
// Work units are (row group, key tile) pairs in group order, split evenly over the CTAs; a one-CTA
// plan kernel enumerates the groups and their tile counts in the workspace first.
#include <algorithm>

#include "append.cuh"
#include "tc.cuh"

namespace dsa {

constexpr int kIdxTile = 128;
constexpr int kIdxRows = 4;
constexpr int kIdxStages = 8;
constexpr int kIdxThreads = 416;                  // warps 0, 6-8 TMA, 1 MMA, 2-5 and 9-12 epilogue
constexpr int kIdxEpiThreads = 256;               // two epilogue groups of four warps
constexpr int kIdxHi = 64, kIdxDi = 128;
constexpr uint32_t kIdxTileBytes = kIdxTile * kIdxDi;         // 16 KB
constexpr uint32_t kIdxPageBytes = 64 * kIdxDi;               // 8 KB
constexpr uint32_t kIdxBSlotBytes = kIdxRows * kIdxHi * kIdxDi;  // 32 KB
constexpr uint32_t kIdxWSlotBytes = kIdxRows * kIdxHi * 4;       // 1 KB
// Leading-digit histograms for the selection step: per row of a group, 2048 bins of the top 11 bits of each
// score's order-preserving key, as 16-bit counters packed in pairs; flushed to global memory (adds of the
// non-zero bins) when the group changes and before a counter could pass 65535 (511 tiles of 128 keys).
constexpr int kIdxHistBins = 2048;
constexpr int kIdxHistFlushTiles = 511;
// Decode batches (one query row per sequence, so row g is sequence g and a group is one row) of up to this
// many rows are planned inside the main kernel: each CTA scans the rows' tile counts into shared memory,
// with no plan kernel in front and no chain of dependent plan reads before its first copy.
constexpr int kIdxInlinePlanMax = 1024;

// ------------------------------------------------------------------------------------------------ plan
// workspace (after the header): int32 [0] = G, [1] = U, then arrays
struct IdxPlanView {
  int32_t *hdr;
  int32_t *seq_goff;      // [num_seqs + 1]
  int32_t *g_row0;        // [total_q]
  int32_t *g_nrows;       // [total_q]
  int32_t *g_seq;         // [total_q]
  int32_t *tile_prefix;   // [total_q + 1]
};

static size_t al256(size_t x) { return (x + 255) / 256 * 256; }

size_t indexer_workspace_bytes(int num_seqs, int total_q) {
  return kWsHeader + 256 + al256((size_t)(num_seqs + 1) * 4) + 3 * al256((size_t)total_q * 4) +
         al256((size_t)(total_q + 1) * 4);
}

static IdxPlanView plan_view(void *ws, int num_seqs, int total_q) {
  char *p = (char *)ws + kWsHeader;
  IdxPlanView v;
  v.hdr = (int32_t *)p;
  p += 256;
  v.seq_goff = (int32_t *)p;
  p += al256((size_t)(num_seqs + 1) * 4);
  v.g_row0 = (int32_t *)p;
  p += al256((size_t)total_q * 4);
  v.g_nrows = (int32_t *)p;
  p += al256((size_t)total_q * 4);
  v.g_seq = (int32_t *)p;
  p += al256((size_t)total_q * 4);
  v.tile_prefix = (int32_t *)p;
  return v;
}

// the plan, by one CTA of 1024 threads (tmp: 64 words of scan scratch, s_carry: one shared word)
__device__ __forceinline__ void indexer_plan_body(const BatchView &bv, const IdxPlanView &pv, uint32_t *tmp,
                                                  uint32_t &s_carry) {
  const int tid = threadIdx.x;
  if (tid == 0) s_carry = 0;
  __syncthreads();
  // groups per sequence -> seq_goff (exclusive prefix)
  for (int base = 0; base < bv.num_seqs; base += blockDim.x) {
    const int b = base + tid;
    uint32_t g = 0;
    if (b < bv.num_seqs) {
      const int nb = __ldg(bv.cu_q + b + 1) - __ldg(bv.cu_q + b);
      g = (nb + kIdxRows - 1) / kIdxRows;
    }
    uint32_t tot;
    const uint32_t ex = block_exclusive_scan(g, tmp, &tot);
    if (b < bv.num_seqs) pv.seq_goff[b] = (int)(s_carry + ex);
    __syncthreads();
    if (tid == 0) s_carry += tot;
    __syncthreads();
  }
  const int G = (int)s_carry;
  if (tid == 0) pv.seq_goff[bv.num_seqs] = G;
  __syncthreads();
  if (tid == 0) s_carry = 0;
  __syncthreads();
  // per group: rows, sequence, tile count -> tile_prefix
  for (int base = 0; base < G; base += blockDim.x) {
    const int gi = base + tid;
    uint32_t tiles = 0;
    if (gi < G) {
      int lo = 0, hi = bv.num_seqs - 1;            // last b with seq_goff[b] <= gi
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pv.seq_goff[mid] <= gi) lo = mid; else hi = mid - 1;
      }
      const int b = lo;
      const int g = gi - pv.seq_goff[b];
      const int c0 = __ldg(bv.cu_q + b), nb = __ldg(bv.cu_q + b + 1) - c0;
      const int nrows = min(kIdxRows, nb - g * kIdxRows);
      const int pos_last = __ldg(bv.seq_lens + b) - nb + g * kIdxRows + nrows - 1;
      tiles = (uint32_t)(pos_last / kIdxTile + 1);
      pv.g_row0[gi] = c0 + g * kIdxRows;
      pv.g_nrows[gi] = nrows;
      pv.g_seq[gi] = b;
    }
    uint32_t tot;
    const uint32_t ex = block_exclusive_scan(tiles, tmp, &tot);
    if (gi < G) pv.tile_prefix[gi] = (int)(s_carry + ex);
    __syncthreads();
    if (tid == 0) s_carry += tot;
    __syncthreads();
  }
  if (tid == 0) {
    pv.tile_prefix[G] = (int)s_carry;
    pv.hdr[0] = G;
    pv.hdr[1] = (int)s_carry;
  }
}

__global__ void __launch_bounds__(1024) indexer_plan_kernel(BatchView bv, IdxPlanView pv) {
  __shared__ uint32_t tmp[64];
  __shared__ uint32_t s_carry;
  pdl_wait();
  pdl_trigger();
  indexer_plan_body(bv, pv, tmp, s_carry);
}

// The plan (CTA 0) and, over the whole grid, the zeroing of the rows' leading-digit histograms that the
// main kernel's epilogue accumulates for the selection step (hist_words u32, a multiple of 4).
__global__ void __launch_bounds__(1024) indexer_prep_kernel(BatchView bv, IdxPlanView pv, uint32_t *hist,
                                                            int64_t hist_words, int do_plan) {
  __shared__ uint32_t tmp[64];
  __shared__ uint32_t s_carry;
  pdl_wait();
  pdl_trigger();
  uint4 *h4 = reinterpret_cast<uint4 *>(hist);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < hist_words / 4; i += (int64_t)gridDim.x * blockDim.x)
    h4[i] = make_uint4(0u, 0u, 0u, 0u);
  if (do_plan && blockIdx.x == 0) indexer_plan_body(bv, pv, tmp, s_carry);
}

// The decode step's cache update fused into its first kernel: the 32 warps append the batch's new tokens
// (one warp per token, append.cuh), then the CTA builds the plan.  The indexer's main kernel, which reads
// the new keys, starts its work only once this kernel has completed.
constexpr int kIdxFusedAppendMaxRows = 256;

__global__ void __launch_bounds__(1024) indexer_plan_append_kernel(BatchView bv, IdxPlanView pv, AppendArgs app, int T,
                                                                   uint32_t *status) {
  __shared__ uint32_t tmp[64];
  __shared__ uint32_t s_carry;
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int row = warp; row < T; row += 32) append_token_warp(app, bv, row, lane, status);
  indexer_plan_body(bv, pv, tmp, s_carry);
}

// ------------------------------------------------------------------------------------------------ main
struct IdxSmem {
  uint64_t full[kIdxStages], empty[kIdxStages];
  uint64_t bfull[2], bempty[2];
  uint64_t tfull[2], tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

// position of unit u: group index and tile within the group
// (tile_prefix is in global memory, or in shared memory for the in-kernel decode plan: plain loads)
__device__ __forceinline__ void unit_locate(const int32_t *tile_prefix, int G, int u, int *gi, int *t) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tile_prefix[mid] <= u) lo = mid; else hi = mid - 1;
  }
  *gi = lo;
  *t = u - tile_prefix[lo];
}

// kHist: the epilogue also counts each row's leading-digit histogram (the fused selection); without it the
// kernel is compiled with none of that code.
template <bool kHist>
__global__ void __launch_bounds__(kIdxThreads, 1)
indexer_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                  const float *__restrict__ kscale, const float *__restrict__ w, BatchView bv, IdxPlanView pv,
                  float *__restrict__ scores, int64_t ld, uint32_t *status, uint32_t *__restrict__ hist,
                  int inline_plan) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t *sA = smem;                                             // kIdxStages x 16 KB
  uint8_t *sB = sA + kIdxStages * kIdxTileBytes;                  // 2 x 32 KB
  float *sW = (float *)(sB + 2 * kIdxBSlotBytes);                 // 2 x 1 KB
  float *sKS = sW + 2 * (kIdxWSlotBytes / 4);                     // kIdxStages x 128 key scales
  uint32_t *sHist = (uint32_t *)(sKS + kIdxStages * kIdxTile);    // kIdxRows x 2048 16-bit counters
  int32_t *sTP = (int32_t *)(sHist + kIdxRows * (kIdxHistBins / 2));   // in-kernel plan: tile prefix
  int32_t *sSL = sTP + kIdxInlinePlanMax + 4;                          // in-kernel plan: sequence lengths
  IdxSmem *S = (IdxSmem *)(sSL + kIdxInlinePlanMax);
  __shared__ uint32_t s_scan[64];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kIdxStages; ++i) {
      tc::mbar_init(tc::smem_u32(&S->full[i]), 1);
      tc::mbar_init(tc::smem_u32(&S->empty[i]), 1 + 4);      // MMA commit + the tile's 4 epilogue warps (key scales)
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(tc::smem_u32(&S->bfull[i]), 1);
      tc::mbar_init(tc::smem_u32(&S->bempty[i]), 1 + 8);     // MMA commit + both epilogue groups
      tc::mbar_init(tc::smem_u32(&S->tfull[i]), 1);
      tc::mbar_init(tc::smem_u32(&S->tempty[i]), 4);
    }
    tc::mbar_init(tc::smem_u32(&S->drain), 1);
    S->abort = 0;
    tc::fence_barrier_init();
    tc::prefetch_tmap(&tm_k);
    tc::prefetch_tmap(&tm_q);
  }
  if (warp == 1) {
    tc::tmem_alloc(tc::smem_u32(&S->tmem_base), 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = S->tmem_base;
  volatile int *abort = &S->abort;
  // the plan (and the inputs) come from earlier work on the stream
  pdl_wait();
  pdl_trigger();
  int G, U;
  const int32_t *tp;
  if (inline_plan) {
    // row g = sequence g, one group per row: its tiles cover keys 0 .. seq_lens[g] - 1
    G = bv.num_seqs;
    uint32_t carry = 0;
    for (int base = 0; base < G; base += kIdxThreads) {
      const int g = base + (int)threadIdx.x;
      const int sl = g < G ? __ldg(bv.seq_lens + g) : 1;
      const uint32_t tiles = g < G ? (uint32_t)((sl - 1) / kIdxTile + 1) : 0u;
      uint32_t tot;
      const uint32_t ex = block_exclusive_scan(tiles, s_scan, &tot);
      if (g < G) {
        sTP[g] = (int)(carry + ex);
        sSL[g] = sl;
      }
      carry += tot;
    }
    if (threadIdx.x == 0) sTP[G] = (int)carry;
    __syncthreads();
    U = (int)carry;
    tp = sTP;
  } else {
    G = pv.hdr[0];
    U = pv.hdr[1];
    tp = pv.tile_prefix;
  }
  auto g_seq = [&](int g) { return inline_plan ? g : pv.g_seq[g]; };
  auto g_row0 = [&](int g) { return inline_plan ? g : pv.g_row0[g]; };
  auto g_nrows = [&](int g) { return inline_plan ? 1 : pv.g_nrows[g]; };
  const int u0 = (int)(((int64_t)blockIdx.x * U) / gridDim.x);
  const int u1 = (int)(((int64_t)(blockIdx.x + 1) * U) / gridDim.x);

  if (u0 < u1) {
    if (warp == 0 || (warp >= 6 && warp <= 8)) {
      // ------------------------------------------------------------------ TMA producers (4 warps)
      // Key tiles are spread over four producer warps (a tile's stage is fixed by its position, so each
      // warp owns two of the eight stages): the copy engine takes several warps' copies at once.  Each
      // warp looks up the block-table entries of its next 32 tiles in one memory round trip.  Warp 0 also
      // loads the query rows + weights of every row group, in order.
      const int pw = warp == 0 ? 0 : warp - 5;              // 0..3
      uint32_t issued = 0, last_par = 0;                    // stages this warp filled / parity of last fill
      uint32_t b_issued = 0, b_last_par = 0;
      bool ok = true;
      // ---- row-group (B operand) loads, warp 0: all groups of the range in order, ahead of the tiles
      auto load_group = [&](int gj, int nbg) -> bool {
        const int bslot = nbg & 1;
        const uint32_t use = (uint32_t)(nbg >> 1);
        if (!tc::mbar_wait(tc::smem_u32(&S->bempty[bslot]), (use & 1u) ^ 1u, abort, status)) return false;
        const int row0 = g_row0(gj), nr = g_nrows(gj);
        const uint32_t bar = tc::smem_u32(&S->bfull[bslot]);
        tc::mbar_expect_tx(bar, (uint32_t)nr * (kIdxHi * kIdxDi + kIdxHi * 4));
        for (int q = 0; q < nr; ++q) {
          tc::tma_load_2d(tc::smem_u32(sB + bslot * kIdxBSlotBytes + q * kIdxHi * kIdxDi), &tm_q, 0, (row0 + q) * kIdxHi,
                          bar);
          tc::bulk_load(tc::smem_u32(sW + bslot * (kIdxWSlotBytes / 4) + q * kIdxHi), w + (int64_t)(row0 + q) * kIdxHi,
                        kIdxHi * 4, bar);
        }
        b_issued |= 1u << bslot;
        b_last_par = (b_last_par & ~(1u << bslot)) | ((use & 1u) << bslot);
        return true;
      };
      int g_next = 0, g_cur = -1, g_count = 0, g_last = -1;   // warp 0: groups loaded so far
      if (pw == 0) {
        int t0;
        unit_locate(tp, G, u0, &g_next, &t0);
        unit_locate(tp, G, u1 - 1, &g_last, &t0);
      }
      const int mine = (u1 - u0 - pw + 3) / 4;              // tiles of this warp: u0 + pw + 4 m
      for (int mb = 0; mb < mine && ok; mb += 32) {
        // ---- lane l describes tile m = mb + l of this warp
        const int m = mb + lane;
        const int u = u0 + pw + 4 * m;
        int gi = 0, t = 0, blk0 = -1, blk1 = -1;
        if (m < mine) {
          unit_locate(tp, G, u, &gi, &t);
          const int b = g_seq(gi);
          int pos_last;
          if (inline_plan) {
            pos_last = sSL[b] - 1;                          // one query row per sequence, at its last position
          } else {
            const int c0 = __ldg(bv.cu_q + b), nbq = __ldg(bv.cu_q + b + 1) - c0;
            pos_last = __ldg(bv.seq_lens + b) - nbq + (g_row0(gi) - c0) + g_nrows(gi) - 1;
          }
          const int pages = pos_last / 64 + 1;
          const int32_t *btr = bv.block_table + (int64_t)b * bv.max_blocks_per_seq;
          blk0 = __ldg(btr + 2 * t);
          if (2 * t + 1 < pages) blk1 = __ldg(btr + 2 * t + 1);
          if ((unsigned)blk0 >= (unsigned)bv.num_blocks) { set_status(status, kStatusBadIndex); blk0 = -1; }
          if (2 * t + 1 < pages && (unsigned)blk1 >= (unsigned)bv.num_blocks) {
            set_status(status, kStatusBadIndex);
            blk1 = -1;
          }
        }
        const int n = min(32, mine - mb);
        for (int j = 0; j < n; ++j) {
          const int gj = __shfl_sync(0xffffffffu, gi, j);
          const int b0 = __shfl_sync(0xffffffffu, blk0, j);
          const int b1 = __shfl_sync(0xffffffffu, blk1, j);
          if (lane == 0) {
            // warp 0 keeps the group loads at least up to the group of its current tile
            if (pw == 0)
              while (ok && g_cur < gj) {
                ok = load_group(g_next, g_count);
                g_cur = g_next++;
                ++g_count;
              }
            const int q = (mb + j) * 4 + pw;                // position of the tile in this CTA's range
            const int stage = q % kIdxStages;
            const uint32_t phase = (uint32_t)(q / kIdxStages) & 1u;
            if (ok) ok = tc::mbar_wait(tc::smem_u32(&S->empty[stage]), phase ^ 1u, abort, status);
            if (ok) {
              const uint32_t bar = tc::smem_u32(&S->full[stage]);
              const uint32_t bytes = (b0 >= 0 ? kIdxPageBytes + 256u : 0u) + (b1 >= 0 ? kIdxPageBytes + 256u : 0u);
              if (bytes) {
                tc::mbar_expect_tx(bar, bytes);
                const uint32_t a_dst = tc::smem_u32(sA + stage * kIdxTileBytes);
                const uint32_t k_dst = tc::smem_u32(sKS + stage * kIdxTile);
                if (b0 >= 0) {
                  tc::tma_load_2d(a_dst, &tm_k, 0, b0 * 64, bar);
                  tc::bulk_load(k_dst, kscale + (int64_t)b0 * 64, 256, bar);
                }
                if (b1 >= 0) {
                  tc::tma_load_2d(a_dst + kIdxPageBytes, &tm_k, 0, b1 * 64, bar);
                  tc::bulk_load(k_dst + 256, kscale + (int64_t)b1 * 64, 256, bar);
                }
              } else {
                tc::mbar_arrive(bar);
              }
              issued |= 1u << stage;
              last_par = (last_par & ~(1u << stage)) | (phase << stage);
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
        }
      }
      if (lane == 0 && pw == 0)      // groups of the range not reached by warp 0's own tiles
        while (ok && g_cur < g_last) {
          ok = load_group(g_next, g_count);
          g_cur = g_next++;
          ++g_count;
        }
      // never leave with copies in flight: wait for the last fill of every stage / slot this warp issued
      if (lane == 0) {
        for (int s2 = 0; s2 < kIdxStages; ++s2)
          if (issued & (1u << s2)) {
            volatile int no_abort = 0;
            tc::mbar_wait(tc::smem_u32(&S->full[s2]), (last_par >> s2) & 1u, &no_abort, status);
          }
        for (int s2 = 0; s2 < 2; ++s2)
          if (b_issued & (1u << s2)) {
            volatile int no_abort = 0;
            tc::mbar_wait(tc::smem_u32(&S->bfull[s2]), (b_last_par >> s2) & 1u, &no_abort, status);
          }
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------------ MMA issuer (whole warp, one elected lane issues)
      int gi, t;
      unit_locate(tp, G, u0, &gi, &t);
      int stage = 0, acc = 0, nb_groups = 0, bslot = 0, cur = -1;
      uint32_t phase = 0, acc_phase = 0;
      for (int u = u0; u < u1; ++u) {
        if (gi != cur) {
          bslot = nb_groups & 1;
          if (!tc::mbar_wait_w(tc::smem_u32(&S->bfull[bslot]), (uint32_t)(nb_groups >> 1) & 1u, abort, status)) break;
          ++nb_groups;
          cur = gi;
        }
        if (!tc::mbar_wait_w(tc::smem_u32(&S->tempty[acc]), acc_phase ^ 1u, abort, status)) break;
        tc::fence_after_sync();
        if (!tc::mbar_wait_w(tc::smem_u32(&S->full[stage]), phase, abort, status)) break;
        const int nr = g_nrows(gi);
        const uint32_t idesc = tc::make_idesc(0, 0, 128, 64 * nr, false, false);
        const uint32_t a0 = tc::smem_u32(sA + stage * kIdxTileBytes);
        const uint32_t b0 = tc::smem_u32(sB + bslot * kIdxBSlotBytes);
#pragma unroll
        for (int k = 0; k < kIdxDi / 32; ++k) {
          tc::mma_f8f6f4_w(tmem + acc * 256, tc::desc_sw128(a0 + 32 * k, 1024), tc::desc_sw128(b0 + 32 * k, 1024), idesc,
                         k > 0 ? 1u : 0u);
        }
        tc::mma_commit_w(tc::smem_u32(&S->empty[stage]));
        tc::mma_commit_w(tc::smem_u32(&S->tfull[acc]));
        const bool last_of_group = (t + 1 == tp[gi + 1] - tp[gi]) || (u + 1 == u1);
        if (last_of_group) tc::mma_commit_w(tc::smem_u32(&S->bempty[bslot]));
        if (++stage == kIdxStages) { stage = 0; phase ^= 1u; }
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        if (++t == tp[gi + 1] - tp[gi]) { ++gi; t = 0; }
      }
      // every MMA issued by this thread has completed before TMEM is released
      tc::mma_commit_w(tc::smem_u32(&S->drain));
      volatile int no_abort = 0;
      tc::mbar_wait_w(tc::smem_u32(&S->drain), 0, &no_abort, status);
    } else if ((warp >= 2 && warp < 6) || warp >= 9) {
      // ------------------------------------------------------------------ epilogue (two groups of 4 warps)
      // Group eg (warps 2-5: 0, warps 9-12: 1) takes the tiles of even / odd position in the CTA's range, which
      // are exactly the tiles the MMA accumulates into TMEM accumulator eg: the weighted ReLU sums of two tiles
      // run at once.  Both groups walk every unit to keep the row-group bookkeeping: each waits for every row
      // group's query rows and releases them once it is past the group's last tile.
      const int quad = warp & 3;                 // TMEM lane quadrant this warp may access
      const int key_local = quad * 32 + lane;
      const int eg = warp >= 9 ? 1 : 0;
      const int et = (warp >= 9 ? warp - 5 : warp - 2) * 32 + lane;   // 0..255 over the two groups
      // With histograms on, the eight warps meet at named barrier 1 around every flush, so the loop never
      // leaves early then: after a timeout the waits return at once and the remaining units pass through
      // without touching TMEM or global memory.
      if constexpr (kHist) {
        for (int j = et; j < kIdxRows * (kIdxHistBins / 2); j += kIdxEpiThreads) sHist[j] = 0u;
        tc::named_bar_sync(1, kIdxEpiThreads);
      }
      int gi, t;
      unit_locate(tp, G, u0, &gi, &t);
      int nb_groups = 0, bslot = 0, cur = -1, span = 0;
      uint32_t acc_phase = 0;                    // phase of accumulator eg
      int b = 0, row0 = 0, nr = 0, pos0 = 0;
      bool ok = true;
      // adds this CTA's counts of the current group's rows to their global histograms and clears them
      auto flush = [&]() {
        tc::named_bar_sync(1, kIdxEpiThreads);
        for (int q = 0; q < nr; ++q) {
          uint32_t *hg = hist + (int64_t)(row0 + q) * kIdxHistBins;
          uint32_t *hs = sHist + q * (kIdxHistBins / 2);
          for (int j = et; j < kIdxHistBins / 2; j += kIdxEpiThreads) {
            const uint32_t v = hs[j];
            if (v != 0u) {
              if (ok) {
                if (v & 0xFFFFu) atomicAdd(hg + 2 * j, v & 0xFFFFu);
                if (v >> 16) atomicAdd(hg + 2 * j + 1, v >> 16);
              }
              hs[j] = 0u;
            }
          }
        }
        tc::named_bar_sync(1, kIdxEpiThreads);
        span = 0;
      };
      // this group is done with the current row group's query rows and weights
      auto release_group = [&]() {
        __syncwarp();
        if (lane == 0 && ok) tc::mbar_arrive(tc::smem_u32(&S->bempty[bslot]));
      };
      for (int u = u0; u < u1; ++u) {
        const bool mine = ((u - u0) & 1) == eg;
        if (gi != cur) {
          if (cur >= 0) {
            if (kHist) flush();
            release_group();
          }
          bslot = nb_groups & 1;
          ok = __all_sync(0xffffffffu, tc::mbar_wait(tc::smem_u32(&S->bfull[bslot]), (uint32_t)(nb_groups >> 1) & 1u, abort,
                                                     status)) && ok;
          if (!kHist && !ok) break;
          ++nb_groups;
          cur = gi;
          b = g_seq(gi);
          row0 = g_row0(gi);
          nr = g_nrows(gi);
          if (inline_plan) {
            pos0 = sSL[b] - 1;
          } else {
            const int c0 = __ldg(bv.cu_q + b);
            pos0 = __ldg(bv.seq_lens + b) - (__ldg(bv.cu_q + b + 1) - c0) + (row0 - c0);
          }
        } else if (kHist && span == kIdxHistFlushTiles) {
          flush();
        }
        if (mine) {
          const int s = t * kIdxTile + key_local;
          // the TMEM loads below are warp-collective: the warp takes them together or not at all
          ok = __all_sync(0xffffffffu, tc::mbar_wait(tc::smem_u32(&S->tfull[eg]), acc_phase, abort, status)) && ok;
          if (!kHist && !ok) break;
          if (ok) {
            tc::fence_after_sync();
            // the tile's key scales arrived with it; the stage's fill has completed (the MMA consumed it), the
            // wait below returns at once and orders the bulk copy before these reads
            const int stage = (u - u0) % kIdxStages;
            tc::mbar_wait(tc::smem_u32(&S->full[stage]), (uint32_t)((u - u0) / kIdxStages) & 1u, abort, status);
            const float ks = sKS[stage * kIdxTile + key_local];
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(tc::smem_u32(&S->empty[stage]));
            const float *wq = sW + bslot * (kIdxWSlotBytes / 4);
            const uint32_t tbase = tmem + ((uint32_t)(quad * 32) << 16) + eg * 256;
            uint32_t dig[kIdxRows];             // leading digits of this thread's scores (bit 31: none)
#pragma unroll
            for (int q = 0; q < kIdxRows; ++q) {
              dig[q] = 0x80000000u;
              if (q >= nr) continue;
              float v0[32], v1[32];
              tc::tmem_ld32(tbase + q * 64, v0);
              tc::tmem_ld32(tbase + q * 64 + 32, v1);
              tc::tmem_wait_ld();
              const float *wr = wq + q * kIdxHi;
              float a0 = 0.f, a1 = 0.f;
#pragma unroll
              for (int h = 0; h < 32; h += 2) {
                a0 = fmaf(wr[h], fmaxf(v0[h], 0.f), a0);
                a1 = fmaf(wr[h + 1], fmaxf(v0[h + 1], 0.f), a1);
              }
#pragma unroll
              for (int h = 0; h < 32; h += 2) {
                a0 = fmaf(wr[32 + h], fmaxf(v1[h], 0.f), a0);
                a1 = fmaf(wr[33 + h], fmaxf(v1[h + 1], 0.f), a1);
              }
              if (s <= pos0 + q) {
                const float sc = (a0 + a1) * ks;
                scores[(int64_t)(row0 + q) * ld + s] = sc;
                if constexpr (kHist) dig[q] = ordered_key(sc) >> 21;
              }
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(tc::smem_u32(&S->tempty[eg]));
            if constexpr (kHist) {
              // counted after the accumulator is handed back (an arrive orders every earlier memory operation
              // of the warp before it, so adds in front of it would hold the tensor core up)
#pragma unroll
              for (int q = 0; q < kIdxRows; ++q)
                if (dig[q] != 0x80000000u) {
                  const uint32_t addr = tc::smem_u32(&sHist[q * (kIdxHistBins / 2) + (dig[q] >> 1)]);
                  asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(addr), "r"((dig[q] & 1u) ? 0x10000u : 1u) : "memory");
                }
            }
          }
          acc_phase ^= 1u;
        }
        ++span;
        if (++t == tp[gi + 1] - tp[gi]) { ++gi; t = 0; }
      }
      if (cur >= 0) {
        if (kHist) flush();
        release_group();
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------------------------------ host
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn() {
  // looked up once, thread-safely (function-local static initialisation)
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return (EncodeTiledFn)p;
    return nullptr;
  }();
  return fn;
}

// 2-D byte matrix [rows, 128] read in boxes of 64 rows x 128 bytes with the 128-byte swizzle
static bool make_rows128_map(CUtensorMap *m, const void *base, uint64_t rows) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {128, rows};
  cuuint64_t strides[1] = {128};
  cuuint32_t box[2] = {128, 64};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static size_t indexer_tc_smem() {
  return 1024 + kIdxStages * kIdxTileBytes + 2 * kIdxBSlotBytes + 2 * kIdxWSlotBytes + kIdxStages * kIdxTile * 4 +
         kIdxRows * (kIdxHistBins / 2) * 4 + (kIdxInlinePlanMax + 4) * 4 + kIdxInlinePlanMax * 4 + sizeof(IdxSmem);
}

size_t indexer_hist_bytes(int total_q) { return al256((size_t)total_q * kIdxHistBins * 4); }

dsa_status_t cache_append_launch(const void *kv_new, const void *k_new, bool k_bf16, const dsa_batch_t *b,
                                 void *kv_pool, void *kI_pool, float *kS_pool, void *ws, cudaStream_t stream);

dsa_status_t indexer_tc_launch(const uint8_t *qI, const float *w, const uint8_t *kpool, const float *kscale,
                               const dsa_batch_t *b, float *scores, int64_t ld, void *ws, cudaStream_t stream,
                               int num_sms, const AppendArgs *app, uint32_t *hist) {
  BatchView bv = view_of(b);
  IdxPlanView pv = plan_view(ws, b->num_seqs, b->total_q);
  CUtensorMap tm_k, tm_q;
  if (!make_rows128_map(&tm_k, kpool, (uint64_t)b->num_blocks * 64) ||
      !make_rows128_map(&tm_q, qI, (uint64_t)b->total_q * kIdxHi)) {
    set_error("indexer: cuTensorMapEncodeTiled failed");
    return DSA_ERR_CUDA;
  }
  const int inline_plan =
      b->total_q == b->num_seqs && b->max_q_per_seq == 1 && b->num_seqs <= kIdxInlinePlanMax ? 1 : 0;
  if (app != nullptr && hist == nullptr && b->total_q <= kIdxFusedAppendMaxRows) {
    DSA_LAUNCH_PDL("indexer_plan_append_kernel", indexer_plan_append_kernel, dim3(1), dim3(1024), 0, stream, bv, pv,
                   *app, b->total_q, (uint32_t *)ws);
  } else {
    if (app != nullptr) {
      const dsa_status_t st = cache_append_launch(app->kv_new, app->k_new, app->k_bf16 != 0, b, app->kv_pool,
                                                  app->kI_pool, app->kS_pool, ws, stream);
      if (st != DSA_OK) return st;
    }
    if (hist != nullptr) {
      // the histograms are cleared here, a stream step ahead of the kernel that adds into them
      const int64_t words = (int64_t)b->total_q * kIdxHistBins;
      const int grid = (int)std::min<int64_t>(num_sms, std::max<int64_t>(1, words / (4 * 1024 * 4)));
      DSA_LAUNCH_PDL("indexer_prep_kernel", indexer_prep_kernel, dim3(grid), dim3(1024), 0, stream, bv, pv, hist, words,
                     inline_plan ? 0 : 1);
    } else if (!inline_plan) {
      DSA_LAUNCH_PDL("indexer_plan_kernel", indexer_plan_kernel, dim3(1), dim3(1024), 0, stream, bv, pv);
    }
  }
  const size_t smem = indexer_tc_smem();
  if (hist != nullptr) {
    cudaFuncSetAttribute(indexer_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    DSA_LAUNCH_PDL("indexer_tc_kernel", indexer_tc_kernel<true>, dim3(num_sms), dim3(kIdxThreads), smem, stream, tm_k,
                   tm_q, kscale, w, bv, pv, scores, ld, (uint32_t *)ws, hist, inline_plan);
  } else {
    cudaFuncSetAttribute(indexer_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    DSA_LAUNCH_PDL("indexer_tc_kernel", indexer_tc_kernel<false>, dim3(num_sms), dim3(kIdxThreads), smem, stream, tm_k,
                   tm_q, kscale, w, bv, pv, scores, ld, (uint32_t *)ws, hist, inline_plan);
  }
  return DSA_OK;
}

}  // namespace dsa
