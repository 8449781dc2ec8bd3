// Sparse MLA attention on tcgen05 tensor cores, one CTA pair (cluster of 2) per query row.
//
// For one query row with 128 heads, latent rows of 576 bf16 (the first 512 are also the values) and
// up to k selected token positions:
//   z[h, i] = scale * q[h, :] . K[idx_i],   o[h, :] = sum_i softmax_i(z[h, :]) V[idx_i],   lse[h]
// ("Day-0 Adaptation for LLMs: Implementing Sparse Attention and Low-Precision Weights", decode sketch:
// gather the selected KV, exact attention over it; "Engineering Practices for Day-0 Adaptation of
// Million-Token Context Models on Domestic AI Chips", Four Key Layers 3: prefill processes query
// tokens in parallel units, decode prefetches the next KV block with asynchronous copies while the
// current one is computed, partial results are merged by a cross-block reduction.)
//
// Work split of a CTA pair (rank r = 0, 1) over chunks of 96 selected tokens:
//   * each CTA gathers ITS 48 tokens of the chunk (tokens 48r..48r+47), all 576 dims, into a chunk buffer
//     [9 dim blocks][48 tokens][128 B] (128-byte swizzle), by TMA gather4 through the block table;
//   * QK^T  : M = 128 heads (rank r holds heads 64r..64r+63 of q), N = 96 tokens (48 from each CTA),
//             K = 576; each CTA gets S for its 64 heads x all 96 tokens in TMEM;
//   * swap  : the values each CTA needs for P V are 256 of the 512 value dims of all 96 tokens; its own
//             tokens already hold them, the peer's tokens are fetched from the peer's chunk buffer over
//             distributed shared memory (dim blocks 0-3 of rank 1's tokens <-> dim blocks 4-7 of rank 0's
//             tokens, in place), so every token row crosses the copy engine once per pair;
//   * softmax: 4 warps per CTA, one (head, 48-token half) per thread, running max shared with the partner
//             thread, exp2, P (bf16) into smem; O is rescaled in TMEM only when the running max grows by
//             more than 2^8 (exact: the final division uses the same reference max);
//   * P V   : M = 128 heads, N = 512 values as two N = 256 MMAs (rank r supplies values 256r..256r+255),
//             K = 96 tokens; O (64 heads x 512 fp32 per CTA) stays in TMEM, 256 columns.
// Every MMA is issued by one thread of rank 0 for the pair (cta_group::2).  Chunk buffers are double
// buffered; rank 1's buffer completions are relayed to rank 0's barriers by one thread.  Token positions
// that are -1 (or out of range) are zero-filled by the copy engine and masked.
//
// Units: prefill = one row (all its chunks); decode = (row, split) pairs whose partial (o, lse) are
// merged by attn_combine_kernel.  Rows are taken longest-first (reverse order) round-robin over pairs.
#include <algorithm>
#include <cstdio>
#include <cstdlib>

#include "tc.cuh"

namespace dsa {

constexpr int kAttH = 128, kAttD = 576, kAttDv = 512;
constexpr int kAttChunk = 96;                    // tokens per chunk (48 per CTA)
constexpr int kAttHalf = kAttChunk / 2;
constexpr int kAttThreads = 320;                 // warps 0-3 softmax, 4-7 gather, 8 MMA, 9 relay
constexpr uint32_t kAttBlkBytes = kAttHalf * 128;                // one dim block of a CTA's 48 tokens: 6 KB
constexpr uint32_t kAttBufBytes = 9 * kAttBlkBytes;              // 54 KB
constexpr uint32_t kAttQBytes = 9 * 8192;
constexpr uint32_t kAttPBytes = 16384;           // [2 token blocks of 64][64 heads][128 B]
constexpr uint32_t kTmemO = 0, kTmemS = 256;     // O: 256 columns; S: two buffers of 48 columns
constexpr float kRescaleLog2 = 8.0f;
constexpr int kPrefetchAhead = 2;                // chunks of L2 prefetch ahead of the gather

struct AttSmem {
  uint64_t buf_full[2];             // local: TMA bytes of this CTA's half of a chunk (4 producer warps)
  uint64_t pair_full[2];            // rank 0: 2 relays
  uint64_t buf_empty[2];            // MMA commit to both CTAs after P V of the chunk
  uint64_t q_full, pair_q_full, q_empty;
  uint64_t s_full[2];               // MMA commit to both CTAs
  uint64_t xchg[2];                 // the peer's 4 softmax warps finished reading this CTA's buffer
  uint64_t p_full;                  // rank 0: 8 softmax warps (swap written + P written)
  uint64_t pv_done;                 // MMA commit to both CTAs, once per chunk
  uint64_t o_empty;                 // rank 0: 8 softmax warps after the epilogue read O
  uint64_t drain;
  uint64_t mask_full[4], mask_empty[4];   // validity masks of upcoming chunks (gather -> softmax)
  uint32_t tmem_base;
  int abort;
  uint32_t mask[4][4];              // 3 ballot words per chunk (tokens 0-31, 32-63, 64-95)
  float xm[2][128];
  float xl[2][128];
  int32_t phys[2][kAttChunk];
};

struct AttArgs {
  const __nv_bfloat16 *q;       // [T, 128, 576]
  const __nv_bfloat16 *kv;      // [NB*64, 576]
  const int32_t *idx;           // [T, k]
  int k;
  BatchView bv;
  const int32_t *neff;          // [T] 1 + last valid idx position
  int T, splits;                // splits = 1: prefill units (one per row)
  float scale_log2;             // softmax_scale * log2(e)
  __nv_bfloat16 *out;           // [T, 128, 512] (splits == 1)
  float *lse;                   // [T, 128] or nullptr (splits == 1)
  float *part_o;                // [T*splits, 128, 512] (splits > 1)
  float *part_lse;              // [T*splits, 128]
  uint32_t *status;
};

__device__ __forceinline__ void unit_of(const AttArgs &a, int u, int *row, int *cb, int *ce) {
  if (a.splits == 1) {
    *row = a.T - 1 - u;
    const int n = __ldg(a.neff + *row);
    *cb = 0;
    *ce = (n + kAttChunk - 1) / kAttChunk;
  } else {
    *row = u / a.splits;
    const int s = u % a.splits;
    const int n = __ldg(a.neff + *row);
    const int nch = (n + kAttChunk - 1) / kAttChunk;
    *cb = (s * nch) / a.splits;
    *ce = ((s + 1) * nch) / a.splits;
  }
}

__device__ __forceinline__ int num_units(const AttArgs &a) { return a.T * a.splits; }

// ------------------------------------------------------------------------------------------------ plan
// neff[row] = 1 + largest j with a usable idx[row, j] (0 if none); flags positions outside [0, seq_len).
// One warp per row; every lane reads 16-byte vectors, all of them issued before any is used.
__global__ void attn_plan_kernel(const int32_t *__restrict__ idx, int k, BatchView bv, int T, int32_t *neff,
                                 uint32_t *status) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= T) return;
  int b;
  pos_of_row(bv, warp, &b);
  const int seq_len = __ldg(bv.seq_lens + b);
  int last = -1;
  bool bad = false;
  const int32_t *ir = idx + (int64_t)warp * k;
  const bool vec = (k & 3) == 0 && (((uintptr_t)ir) & 15) == 0;
  if (vec) {
    const int k4 = k >> 2;
    for (int base = 0; base < k4; base += 32 * 8) {
      int4 v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int j4 = base + e * 32 + lane;
        v[e] = j4 < k4 ? __ldg(reinterpret_cast<const int4 *>(ir) + j4) : make_int4(-1, -1, -1, -1);
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int j = 4 * (base + e * 32 + lane);
        const int vals[4] = {v[e].x, v[e].y, v[e].z, v[e].w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (vals[c] >= 0 && vals[c] < seq_len) last = max(last, j + c);
          else if (vals[c] >= seq_len) bad = true;
        }
      }
    }
  } else {
    for (int j = lane; j < k; j += 32) {
      const int s = __ldg(ir + j);
      if (s >= 0 && s < seq_len) last = j;
      else if (s >= seq_len) bad = true;
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
  bad = __any_sync(0xffffffffu, bad);
  if (lane == 0) {
    neff[warp] = last + 1;
    if (bad) set_status(status, kStatusBadIndex);
  }
}

// ------------------------------------------------------------------------------------------------ main
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kAttThreads, 1)
    attn_mla_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv, const AttArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t *sQ = smem;                                  // [9 dim blocks][64 heads][128 B]
  uint8_t *sBuf = sQ + kAttQBytes;                     // 2 x [9 dim blocks][48 tokens][128 B]
  uint8_t *sP = sBuf + 2 * kAttBufBytes;               // [2 token blocks][64 heads][128 B]
  AttSmem *S = (AttSmem *)(sP + kAttPBytes);

  const uint32_t rank = tc::cluster_ctarank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int U = num_units(a);

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(tc::smem_u32(&S->buf_full[i]), 4);
      tc::mbar_init(tc::smem_u32(&S->pair_full[i]), 2);
      tc::mbar_init(tc::smem_u32(&S->buf_empty[i]), 1);
      tc::mbar_init(tc::smem_u32(&S->s_full[i]), 1);
      tc::mbar_init(tc::smem_u32(&S->xchg[i]), 4);
    }
    tc::mbar_init(tc::smem_u32(&S->q_full), 1);
    tc::mbar_init(tc::smem_u32(&S->pair_q_full), 2);
    tc::mbar_init(tc::smem_u32(&S->q_empty), 1);
    tc::mbar_init(tc::smem_u32(&S->p_full), 8);
    tc::mbar_init(tc::smem_u32(&S->pv_done), 1);
    tc::mbar_init(tc::smem_u32(&S->o_empty), 8);
    tc::mbar_init(tc::smem_u32(&S->drain), 1);
    for (int i = 0; i < 4; ++i) {
      tc::mbar_init(tc::smem_u32(&S->mask_full[i]), 1);
      tc::mbar_init(tc::smem_u32(&S->mask_empty[i]), 4);
    }
    S->abort = 0;
    tc::fence_barrier_init();
    tc::prefetch_tmap(&tm_q);
    tc::prefetch_tmap(&tm_kv);
  }
  if (warp == 8) {
    tc::tmem_alloc2(tc::smem_u32(&S->tmem_base), 512);
    tc::tmem_relinquish2();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::cluster_sync();
  tc::fence_after_sync();
  const uint32_t tmem = S->tmem_base;
  volatile int *abort = &S->abort;
  uint32_t *status = a.status;

  if (warp >= 4 && warp < 8) {
    // ====================================================================== gather (128 threads)
    // q by one tiled TMA per dim block; this CTA's 48 tokens of every chunk by TMA gather4 (4 rows x 128
    // bytes per instruction, 128-byte swizzle applied by the copy engine), warp w taking dim blocks w, w+4
    // (and 8 for warp 0).  Loops holding the named barrier never break: after a timeout every wait returns
    // at once and the copies are skipped, so all 128 threads still meet at the barriers and the teardown.
    const int t = threadIdx.x - 128, pw = t >> 5;
    const int oob_row = a.bv.num_blocks * 64;           // outside the map: the copy engine fills zeros
    uint32_t v = 0, g = 0;
    // L2 prefetch cursor, kPrefetchAhead chunks ahead of the chunk being gathered: each CTA prefetches the
    // full latent rows of its own 48 tokens (and the next unit's q when the cursor enters it)
    int pf_u = pair, pf_c = 0, pf_row = -1, pf_cb = 0, pf_nch = 0, pf_seq = 0;
    const int32_t *pf_btr = nullptr;
    auto pf_enter = [&](int uu) {
      for (; uu < U; uu += npairs) {
        int r2, cb2, ce2;
        unit_of(a, uu, &r2, &cb2, &ce2);
        if (ce2 > cb2) {
          int b2;
          pos_of_row(a.bv, r2, &b2);
          pf_u = uu; pf_c = 0; pf_row = r2; pf_cb = cb2; pf_nch = ce2 - cb2;
          pf_seq = __ldg(a.bv.seq_lens + b2);
          pf_btr = a.bv.block_table + (int64_t)b2 * a.bv.max_blocks_per_seq;
          if (t < 64) tc::prefetch_l2(a.q + ((int64_t)r2 * kAttH + 64 * rank + t) * kAttD, kAttD * 2);
          return;
        }
      }
      pf_u = U;
    };
    auto pf_step = [&]() {
      if (pf_u >= U) return;
      if (t < kAttHalf) {
        const int j = (pf_cb + pf_c) * kAttChunk + kAttHalf * (int)rank + t;
        if (j < a.k) {
          const int s = __ldg(a.idx + (int64_t)pf_row * a.k + j);
          if (s >= 0 && s < pf_seq) {
            const int blk = __ldg(pf_btr + (s >> 6));
            if ((unsigned)blk < (unsigned)a.bv.num_blocks)
              tc::prefetch_l2(a.kv + ((int64_t)blk * 64 + (s & 63)) * kAttD, kAttD * 2);
          }
        }
      }
      if (++pf_c == pf_nch) pf_enter(pf_u + npairs);
    };
    pf_enter(pair);
    for (int d = 0; d < kPrefetchAhead; ++d) pf_step();
    for (int u = pair; u < U; u += npairs) {
      int row, cb, ce;
      unit_of(a, u, &row, &cb, &ce);
      const int nch = ce - cb;
      if (nch <= 0) continue;
      int b;
      pos_of_row(a.bv, row, &b);
      const int seq_len = __ldg(a.bv.seq_lens + b);
      const int32_t *btr = a.bv.block_table + (int64_t)b * a.bv.max_blocks_per_seq;
      if (t == 0) {
        const bool ok = v == 0 || tc::mbar_wait_cl(tc::smem_u32(&S->q_empty), (v - 1) & 1u, abort, status);
        if (ok) {
          const uint32_t bar = tc::smem_u32(&S->q_full);
          tc::mbar_expect_tx(bar, kAttQBytes);
          for (int d = 0; d < 9; ++d)
            tc::tma_load_2d(tc::smem_u32(sQ + d * 8192), &tm_q, d * 64, row * kAttH + 64 * (int)rank, bar);
        }
      }
      for (int i = 0; i < nch; ++i, ++g) {
        const uint32_t bi = g & 1u, use = g >> 1;
        pf_step();
        // token positions of the chunk -> physical rows (-1: masked); validity words go to the softmax
        const uint32_t mslot = g & 3u;
        const bool m_ok = __all_sync(0xffffffffu, tc::mbar_wait(tc::smem_u32(&S->mask_empty[mslot]),
                                                                ((g >> 2) & 1u) ^ 1u, abort, status));
        tc::named_bar_sync(1, 128);
        {
          int32_t pr = -1;
          const int j = (cb + i) * kAttChunk + t;
          if (t < kAttChunk && j < a.k) {
            const int s = __ldg(a.idx + (int64_t)row * a.k + j);
            if (s >= 0 && s < seq_len) {
              const int blk = __ldg(btr + (s >> 6));
              if ((unsigned)blk < (unsigned)a.bv.num_blocks) pr = blk * 64 + (s & 63);
              else set_status(status, kStatusBadIndex);
            }
          }
          if (t < kAttChunk) S->phys[bi][t] = pr;
          const unsigned bits = __ballot_sync(0xffffffffu, pr >= 0);
          if (lane == 0 && m_ok && pw < 3) S->mask[mslot][pw] = bits;
        }
        tc::named_bar_sync(1, 128);
        if (t == 0) tc::mbar_arrive(tc::smem_u32(&S->mask_full[mslot]));
        // this warp's dim blocks of this CTA's 48 tokens, into chunk buffer bi
        const int nblk = pw == 0 ? 3 : 2;
        bool ok = true;
        if (lane == 0) {
          ok = tc::mbar_wait_cl(tc::smem_u32(&S->buf_empty[bi]), (use & 1u) ^ 1u, abort, status);
          if (ok) tc::mbar_expect_tx(tc::smem_u32(&S->buf_full[bi]), (uint32_t)nblk * kAttBlkBytes);
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (ok && lane < kAttHalf / 4) {
          const int32_t *ph = S->phys[bi] + kAttHalf * (int)rank + 4 * lane;
          int r4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) r4[e] = ph[e] >= 0 ? ph[e] : oob_row;
          for (int m = 0; m < nblk; ++m) {
            const int d = pw + 4 * m;
            tc::tma_gather4(tc::smem_u32(sBuf + bi * kAttBufBytes + d * kAttBlkBytes + 4 * lane * 128), &tm_kv, d * 64,
                            r4[0], r4[1], r4[2], r4[3], tc::smem_u32(&S->buf_full[bi]));
          }
        }
      }
      ++v;
    }
  } else if (warp == 9) {
    // ====================================================================== relay (lane 0)
    if (lane == 0) {
      const uint32_t peer_pair_full = tc::map_to_rank(tc::smem_u32(&S->pair_full[0]), 0);
      const uint32_t peer_pair_q = tc::map_to_rank(tc::smem_u32(&S->pair_q_full), 0);
      uint32_t v = 0, g = 0;
      bool ok = true;
      for (int u = pair; u < U && ok; u += npairs) {
        int row, cb, ce;
        unit_of(a, u, &row, &cb, &ce);
        const int nch = ce - cb;
        if (nch <= 0) continue;
        if (!tc::mbar_wait(tc::smem_u32(&S->q_full), v & 1u, abort, status)) break;
        tc::fence_proxy_async();
        tc::mbar_arrive_cluster(peer_pair_q);
        for (int i = 0; i < nch; ++i, ++g) {
          if (!tc::mbar_wait(tc::smem_u32(&S->buf_full[g & 1u]), (g >> 1) & 1u, abort, status)) { ok = false; break; }
          tc::fence_proxy_async();
          tc::mbar_arrive_cluster(peer_pair_full + (g & 1u) * 8);
        }
        ++v;
      }
    }
  } else if (warp == 8) {
    // ====================================================================== MMA issuer (rank 0, lane 0)
    if (rank == 0 && lane == 0) {
      const uint32_t idesc_qk = tc::make_idesc(1, 1, 128, kAttChunk, false, false);
      const uint32_t idesc_pv = tc::make_idesc(1, 1, 128, 256, false, true);
      const uint16_t both = 3;
      const uint32_t qbase = tc::smem_u32(sQ), pbase = tc::smem_u32(sP);
      uint32_t v = 0, g = 0;
      bool ok = true;
      auto pv = [&](uint32_t gc, bool first) -> bool {
        if (!tc::mbar_wait_cl(tc::smem_u32(&S->p_full), gc & 1u, abort, status)) return false;
        if (first && v > 0 && !tc::mbar_wait_cl(tc::smem_u32(&S->o_empty), (v - 1) & 1u, abort, status)) return false;
        tc::fence_after_sync();
        const uint32_t base = tc::smem_u32(sBuf + (gc & 1u) * kAttBufBytes);
        for (int p = 0; p < 2; ++p)
          for (int kh = 0; kh < 2; ++kh)
#pragma unroll
            for (int ks = 0; ks < kAttHalf / 16; ++ks) {
              const int kg = (kAttHalf / 16) * kh + ks;          // 16-token step within the chunk
              const uint64_t ad = tc::desc_sw128(pbase + (kg >> 2) * 8192 + (kg & 3) * 32, 1024);
              const uint64_t bd =
                  tc::desc_sw128_lbo(base + (4 * kh + 2 * p) * kAttBlkBytes + ks * 2048, kAttBlkBytes, 1024);
              tc::mma_bf16_pair(tmem + kTmemO + 128 * p, ad, bd, idesc_pv, (first && kg == 0) ? 0u : 1u);
            }
        tc::mma_commit_pair(tc::smem_u32(&S->buf_empty[gc & 1u]), both);
        tc::mma_commit_pair(tc::smem_u32(&S->pv_done), both);
        return true;
      };
      for (int u = pair; u < U && ok; u += npairs) {
        int row, cb, ce;
        unit_of(a, u, &row, &cb, &ce);
        const int nch = ce - cb;
        if (nch <= 0) continue;
        if (!tc::mbar_wait_cl(tc::smem_u32(&S->pair_q_full), v & 1u, abort, status)) break;
        tc::fence_after_sync();
        const uint32_t g0 = g;
        for (int i = 0; i < nch; ++i) {
          if (!tc::mbar_wait_cl(tc::smem_u32(&S->pair_full[g & 1u]), (g >> 1) & 1u, abort, status)) { ok = false; break; }
          tc::fence_after_sync();
          const uint32_t base = tc::smem_u32(sBuf + (g & 1u) * kAttBufBytes);
          const uint32_t sb = tmem + kTmemS + kAttHalf * (g & 1u);
          for (int d = 0; d < 9; ++d) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = tc::desc_sw128(qbase + d * 8192 + kk * 32, 1024);
              const uint64_t bd = tc::desc_sw128(base + d * kAttBlkBytes + kk * 32, 1024);
              tc::mma_bf16_pair(sb, ad, bd, idesc_qk, (d == 0 && kk == 0) ? 0u : 1u);
            }
          }
          tc::mma_commit_pair(tc::smem_u32(&S->s_full[g & 1u]), both);
          if (i == nch - 1) tc::mma_commit_pair(tc::smem_u32(&S->q_empty), both);
          ++g;
          if (i > 0 && !pv(g0 + i - 1, i - 1 == 0)) { ok = false; break; }
        }
        if (ok && !pv(g0 + nch - 1, nch == 1)) ok = false;
        ++v;
      }
      tc::mma_commit_pair_local(tc::smem_u32(&S->drain));
      volatile int no_abort = 0;
      tc::mbar_wait(tc::smem_u32(&S->drain), 0, &no_abort, status);
    }
  } else {
    // ====================================================================== swap + softmax + epilogue
    // Like the gather role, these loops never break (they hold named barrier 2): after a timeout the
    // waits return at once and the remaining chunks run through without touching TMEM or memory.
    const int L = threadIdx.x;                 // TMEM lane
    const int h = L & 63, half = L >> 6;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const uint32_t p_full_r0 = tc::map_to_rank(tc::smem_u32(&S->p_full), 0);
    const uint32_t o_empty_r0 = tc::map_to_rank(tc::smem_u32(&S->o_empty), 0);
    const uint32_t peer_buf = tc::map_to_rank(tc::smem_u32(sBuf), rank ^ 1u);
    const uint32_t peer_xchg = tc::map_to_rank(tc::smem_u32(&S->xchg[0]), rank ^ 1u);
    // the swap moves the value dims this CTA needs from the peer's tokens: rank 0 takes dim blocks 0-3 of
    // rank 1's tokens into its blocks 4-7; rank 1 takes dim blocks 4-7 of rank 0's tokens into its blocks 0-3
    const uint32_t src_off = (rank == 0 ? 0u : 4u) * kAttBlkBytes, dst_off = (rank == 0 ? 4u : 0u) * kAttBlkBytes;
    constexpr int kSwapVec = 4 * kAttBlkBytes / 16 / 128;       // 16-byte vectors per thread
    uint32_t g = 0, v = 0;
    for (int u = pair; u < U; u += npairs) {
      int row, cb, ce;
      unit_of(a, u, &row, &cb, &ce);
      const int nch = ce - cb;
      const int head = 64 * (int)rank + h;
      if (nch <= 0) {
        // nothing selected: o = 0, lse = -inf
        if (a.splits == 1) {
          __nv_bfloat16 *o = a.out + ((int64_t)row * kAttH + head) * kAttDv + 256 * half;
          for (int c = 0; c < 256; c += 8) *reinterpret_cast<uint4 *>(o + c) = make_uint4(0, 0, 0, 0);
          if (a.lse && half == 0) a.lse[(int64_t)row * kAttH + head] = -INFINITY;
        } else {
          float *o = a.part_o + ((int64_t)u * kAttH + head) * kAttDv + 256 * half;
          for (int c = 0; c < 256; c += 4) *reinterpret_cast<float4 *>(o + c) = make_float4(0.f, 0.f, 0.f, 0.f);
          if (half == 0) a.part_lse[(int64_t)u * kAttH + head] = -INFINITY;
        }
        continue;
      }
      float m_run = -INFINITY, l_run = 0.f, l_exact = 0.f;
      for (int i = 0; i < nch; ++i, ++g) {
        const uint32_t bi = g & 1u;
        // validity of this thread's 48 tokens, published by the gather warps
        const uint32_t mslot = g & 3u;
        const bool m_ok = __all_sync(0xffffffffu, tc::mbar_wait(tc::smem_u32(&S->mask_full[mslot]),
                                                                (g >> 2) & 1u, abort, status));
        uint64_t valid = 0;
        if (m_ok) {
          const uint64_t w0 = S->mask[mslot][0], w1 = S->mask[mslot][1], w2 = S->mask[mslot][2];
          valid = half == 0 ? (w0 | (w1 << 32)) : ((w1 >> 16) | (w2 << 16));
          valid &= (1ull << kAttHalf) - 1ull;
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(tc::smem_u32(&S->mask_empty[mslot]));
        const bool have_s =
            __all_sync(0xffffffffu, tc::mbar_wait_cl(tc::smem_u32(&S->s_full[bi]), (g >> 1) & 1u, abort, status));
        tc::fence_after_sync();
        // ---- swap over distributed shared memory: read the peer's values, hand-shake, write them here
        {
          uint4 sw[kSwapVec];
#pragma unroll
          for (int m = 0; m < kSwapVec; ++m)
            sw[m] = have_s ? tc::ld_dsmem16(peer_buf + bi * kAttBufBytes + src_off + (L + 128 * m) * 16)
                           : make_uint4(0, 0, 0, 0);
          __syncwarp();
          if (lane == 0) tc::mbar_arrive_cluster(peer_xchg + bi * 8);
          const bool got = __all_sync(0xffffffffu, tc::mbar_wait_cl(tc::smem_u32(&S->xchg[bi]), (g >> 1) & 1u, abort, status));
          if (have_s && got) {
#pragma unroll
            for (int m = 0; m < kSwapVec; ++m)
              *reinterpret_cast<uint4 *>(sBuf + bi * kAttBufBytes + dst_off + (L + 128 * m) * 16) = sw[m];
          }
        }
        // ---- S for this thread's head and 48 tokens
        float sv[kAttHalf];
        {
          float t0[32], t1[16];
          const uint32_t sa = tmem + lane_base + kTmemS + kAttHalf * bi;
          tc::tmem_ld32(sa, t0);
          tc::tmem_ld16(sa + 32, t1);
          tc::tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) sv[c] = t0[c];
#pragma unroll
          for (int c = 0; c < 16; ++c) sv[32 + c] = t1[c];
        }
        if (!have_s) valid = 0;
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < kAttHalf; ++c) {
          sv[c] = ((valid >> c) & 1ull) ? sv[c] * a.scale_log2 : -INFINITY;
          mx = fmaxf(mx, sv[c]);
        }
        const float mloc = fmaxf(m_run, mx);
        S->xm[g & 1u][L] = mloc;
        tc::named_bar_sync(2, 128);
        const float m_new = fmaxf(mloc, S->xm[g & 1u][L ^ 64]);
        // P V of the previous chunk must be finished before O is touched or P is overwritten
        bool pv_ok = true;
        if (i > 0) {
          pv_ok = tc::mbar_wait_cl(tc::smem_u32(&S->pv_done), (g - 1) & 1u, abort, status);
          tc::fence_after_sync();
        }
        pv_ok = __all_sync(0xffffffffu, pv_ok);
        if (i == 0) {
          m_run = m_new;
        } else {
          // TMEM loads/stores are warp-collective: the warp rescales if any of its rows needs it,
          // rows that do not keep their reference max (alpha = 1)
          const bool want = m_new > m_run + kRescaleLog2;
          if (__any_sync(0xffffffffu, want)) {
            const float alpha = want ? tc::ex2(m_run - m_new) : 1.f;
            if (pv_ok) {
              for (int cc = 0; cc < 8; ++cc) {
                float ov[32];
                tc::tmem_ld32(tmem + lane_base + kTmemO + 32 * cc, ov);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) ov[e] *= alpha;
                tc::tmem_st32(tmem + lane_base + kTmemO + 32 * cc, ov);
              }
              tc::tmem_wait_st();
            }
            if (want) {
              l_run *= alpha;
              l_exact *= alpha;
              m_run = m_new;
            }
          }
        }
        // P = exp2(z - m) in bf16 into the 128-byte-swizzled A operand: row h, tokens 48*half + [0, 48).
        // l_run sums the rounded P (what the MMA multiplies) and normalises O; l_exact gives lse.
        if (pv_ok) {
          float lsum = 0.f, lex = 0.f;
#pragma unroll
          for (int c = 0; c < kAttHalf / 8; ++c) {
            uint32_t w4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int t0 = 8 * c + 2 * e;
              const float p0 = ((valid >> t0) & 1ull) ? tc::ex2(sv[t0] - m_run) : 0.f;
              const float p1 = ((valid >> (t0 + 1)) & 1ull) ? tc::ex2(sv[t0 + 1] - m_run) : 0.f;
              const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
              const float2 pr = __bfloat1622float2(pb);
              lsum += pr.x + pr.y;
              lex += p0 + p1;
              w4[e] = *reinterpret_cast<const uint32_t *>(&pb);
            }
            const int kc = (kAttHalf / 8) * half + c;              // 8-token chunk within the 96 tokens
            *reinterpret_cast<uint4 *>(sP + (kc >> 3) * 8192 + h * 128 + (((kc & 7) ^ (h & 7)) << 4)) =
                make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
          l_run += lsum;
          l_exact += lex;
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive_cluster(p_full_r0);
      }
      // ---- epilogue: wait for the last P V, normalise, store
      const bool o_ok =
          __all_sync(0xffffffffu, tc::mbar_wait_cl(tc::smem_u32(&S->pv_done), (g - 1) & 1u, abort, status));
      tc::fence_after_sync();
      S->xl[0][L] = l_run;
      S->xl[1][L] = l_exact;
      tc::named_bar_sync(2, 128);
      const float l_tot = l_run + S->xl[0][L ^ 64];
      const float l_ex = l_exact + S->xl[1][L ^ 64];
      const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
      const float lse_v = l_ex > 0.f ? (m_run + __log2f(l_ex)) * 0.69314718055994531f : -INFINITY;
      if (o_ok) {
        if (a.splits == 1) {
          __nv_bfloat16 *o = a.out + ((int64_t)row * kAttH + head) * kAttDv + 256 * half;
          for (int cc = 0; cc < 8; ++cc) {
            float ov[32];
            tc::tmem_ld32(tmem + lane_base + kTmemO + 32 * cc, ov);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint4 w;
              __nv_bfloat162 b0 = __floats2bfloat162_rn(ov[e] * inv, ov[e + 1] * inv);
              __nv_bfloat162 b1 = __floats2bfloat162_rn(ov[e + 2] * inv, ov[e + 3] * inv);
              __nv_bfloat162 b2 = __floats2bfloat162_rn(ov[e + 4] * inv, ov[e + 5] * inv);
              __nv_bfloat162 b3 = __floats2bfloat162_rn(ov[e + 6] * inv, ov[e + 7] * inv);
              w.x = *reinterpret_cast<uint32_t *>(&b0);
              w.y = *reinterpret_cast<uint32_t *>(&b1);
              w.z = *reinterpret_cast<uint32_t *>(&b2);
              w.w = *reinterpret_cast<uint32_t *>(&b3);
              *reinterpret_cast<uint4 *>(o + 32 * cc + e) = w;
            }
          }
          if (a.lse && half == 0) a.lse[(int64_t)row * kAttH + head] = lse_v;
        } else {
          float *o = a.part_o + ((int64_t)u * kAttH + head) * kAttDv + 256 * half;
          for (int cc = 0; cc < 8; ++cc) {
            float ov[32];
            tc::tmem_ld32(tmem + lane_base + kTmemO + 32 * cc, ov);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4 *>(o + 32 * cc + e) =
                  make_float4(ov[e] * inv, ov[e + 1] * inv, ov[e + 2] * inv, ov[e + 3] * inv);
          }
          if (half == 0) a.part_lse[(int64_t)u * kAttH + head] = lse_v;
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive_cluster(o_empty_r0);
      ++v;
    }
  }

  // ---- teardown: every role is done; MMAs drained; peers done with our barriers, buffers and TMEM
  tc::fence_before_sync();
  __syncthreads();
  tc::cluster_sync();
  if (warp == 8) {
    tc::fence_after_sync();
    tc::tmem_dealloc2(tmem, 512);
  }
}

// ------------------------------------------------------------------------------------------------ combine
// out[row, h, :] = sum_s exp(lse_s - lse) o_s,  lse = log sum_s exp(lse_s)   (splits of one row)
__global__ void __launch_bounds__(128) attn_combine_kernel(const float *__restrict__ part_o,
                                                           const float *__restrict__ part_lse, int splits,
                                                           __nv_bfloat16 *__restrict__ out, float *__restrict__ lse) {
  const int row = blockIdx.x, h = blockIdx.y;
  float mx = -INFINITY;
  for (int s = 0; s < splits; ++s) mx = fmaxf(mx, __ldg(part_lse + ((int64_t)row * splits + s) * kAttH + h));
  float tot = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float l = __ldg(part_lse + ((int64_t)row * splits + s) * kAttH + h);
    tot += l == -INFINITY ? 0.f : __expf(l - mx);
  }
  const int dv = threadIdx.x * 4;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (tot > 0.f) {
    for (int s = 0; s < splits; ++s) {
      const float l = __ldg(part_lse + ((int64_t)row * splits + s) * kAttH + h);
      if (l == -INFINITY) continue;
      const float wgt = __expf(l - mx) / tot;
      const float4 o = __ldg(reinterpret_cast<const float4 *>(part_o + (((int64_t)row * splits + s) * kAttH + h) * kAttDv + dv));
      acc.x += wgt * o.x;
      acc.y += wgt * o.y;
      acc.z += wgt * o.z;
      acc.w += wgt * o.w;
    }
  }
  __nv_bfloat162 b0 = __floats2bfloat162_rn(acc.x, acc.y), b1 = __floats2bfloat162_rn(acc.z, acc.w);
  uint2 w;
  w.x = *reinterpret_cast<uint32_t *>(&b0);
  w.y = *reinterpret_cast<uint32_t *>(&b1);
  *reinterpret_cast<uint2 *>(out + ((int64_t)row * kAttH + h) * kAttDv + dv) = w;
  if (lse && threadIdx.x == 0) lse[(int64_t)row * kAttH + h] = tot > 0.f ? mx + __logf(tot) : -INFINITY;
}

// ------------------------------------------------------------------------------------------------ host
static size_t al256b(size_t x) { return (x + 255) / 256 * 256; }

// Decode splits are sized for the B200's 148 SMs (74 CTA pairs); the same figure sizes the workspace.
constexpr int kAttPairsForSplits = 74;

int attn_decode_splits(int T, int k) {
  const int pairs = kAttPairsForSplits;
  const int chunks = (k + kAttChunk - 1) / kAttChunk;
  int s = T > 0 ? pairs / T : 1;
  return s < 1 ? 1 : (s > chunks ? chunks : s);
}

size_t attn_workspace_bytes(int T, int k, bool decode) {
  size_t bytes = kWsHeader + al256b((size_t)T * 4);
  if (decode) {
    const int s = attn_decode_splits(T, k);
    if (s > 1) bytes += al256b((size_t)T * s * kAttH * kAttDv * 4) + al256b((size_t)T * s * kAttH * 4);
  }
  return bytes;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn();

// bf16 matrix [rows, 576] read in boxes of `box_rows` rows x 64 columns (128 bytes) with the 128-byte swizzle
static bool make_bf16_rows_map(CUtensorMap *m, const void *base, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kAttD, rows};
  cuuint64_t strides[1] = {(cuuint64_t)kAttD * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static size_t attn_smem_bytes() { return 1024 + kAttQBytes + 2 * kAttBufBytes + kAttPBytes + sizeof(AttSmem); }

dsa_status_t attn_mla_launch(const void *q, const void *kv, const int32_t *idx, int k, float softmax_scale,
                             const dsa_batch_t *b, void *out, float *lse, void *ws, bool decode, cudaStream_t stream,
                             int num_sms) {
  AttArgs a{};
  a.q = (const __nv_bfloat16 *)q;
  a.kv = (const __nv_bfloat16 *)kv;
  a.idx = idx;
  a.k = k;
  a.bv = view_of(b);
  a.T = b->total_q;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.status = (uint32_t *)ws;
  char *p = (char *)ws + kWsHeader;
  a.neff = (const int32_t *)p;
  int32_t *neff = (int32_t *)p;
  p += al256b((size_t)a.T * 4);
  a.splits = decode ? attn_decode_splits(a.T, k) : 1;
  if (a.splits > 1) {
    a.part_o = (float *)p;
    p += al256b((size_t)a.T * a.splits * kAttH * kAttDv * 4);
    a.part_lse = (float *)p;
  } else {
    a.out = (__nv_bfloat16 *)out;
    a.lse = lse;
  }
  CUtensorMap tm_q, tm_kv;
  if (!make_bf16_rows_map(&tm_q, q, (uint64_t)a.T * kAttH, 64) ||
      !make_bf16_rows_map(&tm_kv, kv, (uint64_t)b->num_blocks * 64, 1)) {
    set_error("attention: cuTensorMapEncodeTiled failed");
    return DSA_ERR_CUDA;
  }
  attn_plan_kernel<<<(a.T + 3) / 4, 128, 0, stream>>>(idx, k, a.bv, a.T, neff, a.status);
  DSA_LAUNCH_CHECK("attn_plan_kernel");
  const size_t smem = attn_smem_bytes();
  cudaFuncSetAttribute(attn_mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  // persistent grid: as many CTA pairs as can be resident at once
  static int max_pairs = 0;
  if (max_pairs == 0) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.gridDim = dim3(num_sms & ~1);
    cfg.blockDim = dim3(kAttThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, attn_mla_kernel, &cfg) != cudaSuccess || n < 1) {
      cudaGetLastError();
      n = num_sms / 2;
    }
    max_pairs = std::min(n, num_sms / 2);
    if (getenv("DSA_VERBOSE")) fprintf(stderr, "[libdsa] attention: %d resident CTA pairs\n", max_pairs);
  }
  const int units = a.T * a.splits;
  const int pairs = std::min(max_pairs, units);
  attn_mla_kernel<<<2 * pairs, kAttThreads, smem, stream>>>(tm_q, tm_kv, a);
  DSA_LAUNCH_CHECK("attn_mla_kernel");
  if (a.splits > 1) {
    attn_combine_kernel<<<dim3(a.T, kAttH), 128, 0, stream>>>(a.part_o, a.part_lse, a.splits, (__nv_bfloat16 *)out,
                                                               lse);
    DSA_LAUNCH_CHECK("attn_combine_kernel");
  }
  return DSA_OK;
}

}  // namespace dsa
