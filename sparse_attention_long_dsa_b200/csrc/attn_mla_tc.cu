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
// Work split of a CTA pair (rank r = 0, 1) over chunks of 64 selected tokens:
//   * resolve: one warp turns token positions into physical cache rows (block table) and publishes the
//              validity mask of the chunk, up to four chunks ahead (KV rows are not prefetched into L2:
//              prefetches share the copy engine with the gathers and slowed them);
//   * gather : each CTA gathers ITS 32 tokens of the chunk (tokens 32r..32r+31), all 576 dims, into one
//              of three chunk buffers [9 dim blocks][32 tokens][128 B] (128-byte swizzle), by TMA gather4;
//   * QK^T   : M = 128 heads (rank r holds heads 64r..64r+63 of q), N = 64 tokens (32 from each CTA),
//              K = 576; each CTA gets S for its 64 heads x all 64 tokens in TMEM;
//   * cross  : the values each CTA needs for P V are 256 of the 512 value dims of all 64 tokens; its own
//              tokens already hold them, the peer's 32 tokens' half (16 KB, which the peer's copy engine pulls
//              through L2 at the same time) is loaded into registers by four warps a chunk ahead and stored
//              into the dim blocks QK^T no longer needs once it has run (rank 0: blocks 4-7 <- dims 0-255 of
//              rank 1's tokens; rank 1: blocks 0-3 <- dims 256-511 of rank 0's tokens).  HBM carries each row
//              once per pair (the peer's half is an L2 hit); each CTA writes only its own shared memory;
//   * softmax: 4 warps per CTA, one (head, 32-token half) per thread, running max shared with the partner
//              thread, exp2, P (bf16) into one of two P buffers; O is rescaled in TMEM only when the
//              running max grows by more than 2^8 (exact: the final division uses the same reference max);
//   * P V    : M = 128 heads, N = 512 values as two N = 256 MMAs (rank r supplies values 256r..256r+255),
//              K = 64 tokens; O (64 heads x 512 fp32 per CTA) stays in TMEM, 256 columns.
// Every MMA is issued by rank 0's MMA warp for the pair (cta_group::2).  Both CTAs' copies of a chunk (and
// of q) complete on rank 0's barriers (.cta_group::2 TMA), so rank 0 sees one barrier per operand.  Token
// positions that are -1 (or out of range) are zero-filled by the copy engine and masked.
//
// Units: prefill = one row (all its chunks); decode = (row, split) pairs whose partial (o, lse) are
// merged by attn_combine_kernel.  Rows are taken longest-first (reverse order) round-robin over pairs.
#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstdlib>

#include "tc.cuh"

namespace dsa {

constexpr int kAttH = 128, kAttD = 576, kAttDv = 512;
constexpr int kAttChunk = 64;                    // tokens per chunk (32 per CTA)
constexpr int kAttHalf = kAttChunk / 2;
constexpr int kAttNBuf = 3;                      // chunk buffers
constexpr int kAttRing = 4;                      // resolved chunks (physical rows + masks) in flight
constexpr int kAttThreads = 512;                 // warpgroups: softmax, gather, cross, (MMA, -, resolve, -)
constexpr int kAttWarpMMA = 12, kAttWarpResolve = 14;
// registers per thread after the split: 128 x (224 + 96 + 96 + 96) = 65536
constexpr uint32_t kAttRegsSoftmax = 224, kAttRegsGather = 96, kAttRegsCross = 96, kAttRegsMisc = 96;
constexpr uint32_t kAttBlkBytes = kAttHalf * 128;                // one dim block of a CTA's 32 tokens: 4 KB
constexpr uint32_t kAttBufBytes = 9 * kAttBlkBytes;              // 36 KB
constexpr uint32_t kAttQBytes = 9 * 8192;
constexpr uint32_t kAttPBytes = 8192;            // one P buffer: [64 heads][64 tokens] bf16, 128-byte rows
constexpr uint32_t kTmemO = 0, kTmemS = 256;     // O: 256 columns; S: two buffers of 32 columns
constexpr float kRescaleLog2 = 8.0f;

struct AttSmem {
  uint64_t buf_full[kAttNBuf];      // rank 0: TMA bytes of both CTAs' halves of a chunk (4 gather warps expect)
  uint64_t buf_empty[kAttNBuf];     // MMA commit to both CTAs after P V of the chunk
  uint64_t v_ready[kAttNBuf];       // rank 0: 8 cross warps (both CTAs) stored the peer's values
  uint64_t q_full, q_empty;         // q_full: rank 0, both CTAs' q bytes
  uint64_t s_full[2];               // MMA commit to both CTAs
  uint64_t p_full[2];               // rank 0: 8 softmax warps wrote P
  uint64_t pv_done[2];              // MMA commit to both CTAs, per P buffer
  uint64_t o_empty;                 // rank 0: 8 softmax warps after the epilogue read O
  uint64_t drain;
  uint64_t phys_full[kAttRing], phys_empty[kAttRing];   // resolve -> gather
  uint64_t mask_full[kAttRing], mask_empty[kAttRing];   // resolve -> softmax
  uint32_t tmem_base;
  int abort;
  uint32_t mask[kAttRing][2];       // ballot words of a chunk (tokens 0-31, 32-63)
  float xm[2][128];
  float xl[128];
  int32_t phys[kAttRing][kAttChunk];
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

// Walks the chunks of the units a CTA pair owns (units pair, pair + npairs, ...), skipping empty units.
// Used by whole warps (the sequence lookup is warp-cooperative).
struct ChunkCursor {
  int u, row, j, ce, seq;
  bool first;                   // j is the first chunk of its unit
  const int32_t *btr;           // block-table row of the unit's sequence

  __device__ __forceinline__ void seek(const AttArgs &a, int uu, int npairs) {
    const int U = num_units(a);
    for (; uu < U; uu += npairs) {
      int r, cb, ce2;
      unit_of(a, uu, &r, &cb, &ce2);
      if (ce2 > cb) {
        int b;
        pos_of_row_warp(a.bv, r, &b);
        u = uu; row = r; j = cb; ce = ce2; first = true;
        seq = __ldg(a.bv.seq_lens + b);
        btr = a.bv.block_table + (int64_t)b * a.bv.max_blocks_per_seq;
        return;
      }
    }
    u = U;
  }
  __device__ __forceinline__ void next(const AttArgs &a, int npairs) {
    if (++j == ce) seek(a, u + npairs, npairs);
    else first = false;
  }
  __device__ __forceinline__ bool done(const AttArgs &a) const { return u >= num_units(a); }
};

// ------------------------------------------------------------------------------------------------ plan
// neff[row] = 1 + largest j with a usable idx[row, j] (0 if none); flags positions outside [0, seq_len).
// One 256-thread CTA per row; every thread reads 16-byte vectors, all of them issued before any is used.
constexpr int kAttPlanThreads = 256;
__global__ void __launch_bounds__(kAttPlanThreads) attn_plan_kernel(const int32_t *__restrict__ idx, int k, BatchView bv,
                                                                   int T, int32_t *neff, uint32_t *status) {
  __shared__ int s_last[kAttPlanThreads / 32];
  __shared__ int s_bad[kAttPlanThreads / 32];
  pdl_wait();
  pdl_trigger();
  const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // the row's sequence length: the warp-wide search, with the entry of sequence `row` loaded beside it (a batch
  // of one query row per sequence, where the row is its sequence, needs no second round)
  const int spec = row < bv.num_seqs ? __ldg(bv.seq_lens + row) : 0;
  const int b = seq_of_row_warp(bv.cu_q, bv.num_seqs, row);
  const int seq_len = b == row ? spec : __ldg(bv.seq_lens + b);
  int last = -1;
  bool bad = false;
  const int32_t *ir = idx + (int64_t)row * k;
  const bool vec = (k & 3) == 0 && (((uintptr_t)ir) & 15) == 0;
  if (vec) {
    const int k4 = k >> 2;
    for (int base = 0; base < k4; base += kAttPlanThreads * 4) {
      int4 v[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j4 = base + e * kAttPlanThreads + tid;
        v[e] = j4 < k4 ? __ldg(reinterpret_cast<const int4 *>(ir) + j4) : make_int4(-1, -1, -1, -1);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = 4 * (base + e * kAttPlanThreads + tid);
        const int vals[4] = {v[e].x, v[e].y, v[e].z, v[e].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (vals[q] >= 0 && vals[q] < seq_len) last = max(last, j + q);
          else if (vals[q] >= seq_len) bad = true;
        }
      }
    }
  } else {
    for (int j = tid; j < k; j += kAttPlanThreads) {
      const int sj = __ldg(ir + j);
      if (sj >= 0 && sj < seq_len) last = j;
      else if (sj >= seq_len) bad = true;
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
  bad = __any_sync(0xffffffffu, bad);
  if (lane == 0) {
    s_last[warp] = last;
    s_bad[warp] = bad;
  }
  __syncthreads();
  if (tid == 0) {
    int m = -1, any = 0;
    for (int w = 0; w < kAttPlanThreads / 32; ++w) {
      m = max(m, s_last[w]);
      any |= s_bad[w];
    }
    neff[row] = m + 1;
    if (any) set_status(status, kStatusBadIndex);
  }
  (void)T;
}

// ------------------------------------------------------------------------------------------------ main
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kAttThreads, 1)
    attn_mla_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv, const AttArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t *sQ = smem;                                  // [9 dim blocks][64 heads][128 B]
  uint8_t *sBuf = sQ + kAttQBytes;                     // 3 x [9 dim blocks][32 tokens][128 B]
  uint8_t *sP = sBuf + kAttNBuf * kAttBufBytes;        // 2 x [64 heads][64 tokens] bf16; epilogue staging
  AttSmem *S = (AttSmem *)(sP + 2 * kAttPBytes);

  const uint32_t rank = tc::cluster_ctarank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int U = num_units(a);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kAttNBuf; ++i) {
      tc::mbar_init(tc::smem_u32(&S->buf_full[i]), 4);
      tc::mbar_init(tc::smem_u32(&S->buf_empty[i]), 1);
      tc::mbar_init(tc::smem_u32(&S->v_ready[i]), 8);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(tc::smem_u32(&S->s_full[i]), 1);
      tc::mbar_init(tc::smem_u32(&S->p_full[i]), 8);
      tc::mbar_init(tc::smem_u32(&S->pv_done[i]), 1);
    }
    tc::mbar_init(tc::smem_u32(&S->q_full), 1);
    tc::mbar_init(tc::smem_u32(&S->q_empty), 1);
    tc::mbar_init(tc::smem_u32(&S->o_empty), 8);
    tc::mbar_init(tc::smem_u32(&S->drain), 1);
    for (int i = 0; i < kAttRing; ++i) {
      tc::mbar_init(tc::smem_u32(&S->phys_full[i]), 1);
      tc::mbar_init(tc::smem_u32(&S->phys_empty[i]), 8);
      tc::mbar_init(tc::smem_u32(&S->mask_full[i]), 1);
      tc::mbar_init(tc::smem_u32(&S->mask_empty[i]), 4);
    }
    S->abort = 0;
    tc::fence_barrier_init();
    tc::prefetch_tmap(&tm_q);
    tc::prefetch_tmap(&tm_kv);
  }
  if (warp == kAttWarpMMA) {
    tc::tmem_alloc2(tc::smem_u32(&S->tmem_base), 512);
    tc::tmem_relinquish2();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::cluster_sync();
  tc::fence_after_sync();
  // Each role starts by moving registers: the softmax warpgroup takes them from the three data-movement
  // warpgroups (every warp of a warpgroup executes the same setmaxnreg).
#define ATT_REGS_DEC(n) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(n))
#define ATT_REGS_INC() asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kAttRegsSoftmax))
  const uint32_t tmem = S->tmem_base;
  volatile int *abort = &S->abort;
  uint32_t *status = a.status;
  // inputs (q, idx, neff, the cache) come from earlier work on the stream
  pdl_wait();
  pdl_trigger();

  if (warp == kAttWarpResolve) {
    // ====================================================================== resolve (32 threads)
    ATT_REGS_DEC(kAttRegsMisc);
    // Chunk c of this pair: token positions -> physical rows (ring slot c % kAttRing, -1 = masked) and two
    // validity words; on entering a unit this CTA's 64 q rows are prefetched into L2.
    // The idx loads of chunk c + 1 are in flight while the block-table loads of chunk c resolve.
    ChunkCursor cur, nxt;
    cur.seek(a, pair, npairs);
    auto load_idx = [&](const ChunkCursor &cc, int (&s)[2]) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int j = cc.j * kAttChunk + 32 * e + lane;
        s[e] = (!cc.done(a) && j < a.k) ? __ldg(a.idx + (int64_t)cc.row * a.k + j) : -1;
      }
    };
    int s_cur[2];
    load_idx(cur, s_cur);
    nxt = cur;
    if (!nxt.done(a)) nxt.next(a, npairs);
    for (uint32_t c = 0; !cur.done(a); ++c) {
      int s_nxt[2];
      load_idx(nxt, s_nxt);
      if (cur.first) {
        const __nv_bfloat16 *qr = a.q + ((int64_t)cur.row * kAttH + 64 * (int)rank) * kAttD;
        tc::prefetch_l2(qr + (int64_t)lane * kAttD, kAttD * 2);
        tc::prefetch_l2(qr + (int64_t)(lane + 32) * kAttD, kAttD * 2);
      }
      int32_t pr[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        pr[e] = -1;
        const int s = s_cur[e];
        if (s >= 0 && s < cur.seq) {
          const int blk = __ldg(cur.btr + (s >> 6));
          if ((unsigned)blk < (unsigned)a.bv.num_blocks) pr[e] = blk * 64 + (s & 63);
          else set_status(status, kStatusBadIndex);
        }
      }
      const uint32_t w0 = __ballot_sync(0xffffffffu, pr[0] >= 0), w1 = __ballot_sync(0xffffffffu, pr[1] >= 0);
      const uint32_t slot = c % kAttRing, ph = ((c / kAttRing) & 1u) ^ 1u;
      const bool ok = __all_sync(0xffffffffu, tc::mbar_wait(tc::smem_u32(&S->phys_empty[slot]), ph, abort, status) &&
                                                  tc::mbar_wait(tc::smem_u32(&S->mask_empty[slot]), ph, abort, status));
      if (ok) {
        S->phys[slot][lane] = pr[0];
        S->phys[slot][32 + lane] = pr[1];
        if (lane == 0) {
          S->mask[slot][0] = w0;
          S->mask[slot][1] = w1;
        }
      }
      __syncwarp();
      if (lane == 0) {
        tc::mbar_arrive(tc::smem_u32(&S->phys_full[slot]));
        tc::mbar_arrive(tc::smem_u32(&S->mask_full[slot]));
      }
      cur = nxt;
      s_cur[0] = s_nxt[0];
      s_cur[1] = s_nxt[1];
      if (!nxt.done(a)) nxt.next(a, npairs);
    }
  } else if (warp >= 4 && warp < 8) {
    // ====================================================================== gather (128 threads)
    ATT_REGS_DEC(kAttRegsGather);
    // Chunk c: this CTA's 32 tokens by TMA gather4 (4 rows x 128 bytes per instruction, 128-byte swizzle
    // applied by the copy engine), warp w taking dim blocks w, w+4 (and 8 for warp 0); q by one tiled TMA
    // per dim block when a unit starts.  The loop never breaks: after a timeout every wait returns at once
    // and the copies are skipped.
    const int t = threadIdx.x - 128, pw = t >> 5;
    const int oob_row = a.bv.num_blocks * 64;           // outside the map: the copy engine fills zeros
    const uint32_t buf_full_r0 = tc::map_to_rank(tc::smem_u32(&S->buf_full[0]), 0);
    const uint32_t q_full_r0 = tc::map_to_rank(tc::smem_u32(&S->q_full), 0);
    ChunkCursor pc;
    pc.seek(a, pair, npairs);
    uint32_t v = 0;
    auto load_q = [&](int qrow) {
      if (rank == 0) tc::mbar_expect_tx(tc::smem_u32(&S->q_full), 2u * kAttQBytes);
      for (int d = 0; d < 9; ++d)
        tc::tma_load_2d_pair(tc::smem_u32(sQ + d * 8192), &tm_q, d * 64, qrow * kAttH + 64 * (int)rank, q_full_r0);
    };
    // the first unit's q needs no wait: fetch it before the first chunk's rows
    if (!pc.done(a) && t == 0) load_q(pc.row);
    for (uint32_t c = 0; !pc.done(a); ++c) {
      const uint32_t b = c % kAttNBuf, use = c / kAttNBuf, slot = c % kAttRing;
      const int nblk = pw == 0 ? 3 : 2;
      bool ok = __all_sync(0xffffffffu, tc::mbar_wait(tc::smem_u32(&S->phys_full[slot]), (c / kAttRing) & 1u, abort, status));
      if (lane == 0 && ok) {
        ok = tc::mbar_wait_cl(tc::smem_u32(&S->buf_empty[b]), (use & 1u) ^ 1u, abort, status);
        // rank 0 expects the bytes of this warp's dim blocks from both CTAs
        if (ok && rank == 0) tc::mbar_expect_tx(tc::smem_u32(&S->buf_full[b]), 2u * (uint32_t)nblk * kAttBlkBytes);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (ok && lane < kAttHalf / 4) {
        const int32_t *ph = S->phys[slot] + kAttHalf * (int)rank + 4 * lane;
        int r4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) r4[e] = ph[e] >= 0 ? ph[e] : oob_row;
        for (int m = 0; m < nblk; ++m) {
          const int d = pw + 4 * m;
          tc::tma_gather4_pair(tc::smem_u32(sBuf + b * kAttBufBytes + d * kAttBlkBytes + 4 * lane * 128), &tm_kv, d * 64,
                               r4[0], r4[1], r4[2], r4[3], buf_full_r0 + b * 8);
        }
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(tc::smem_u32(&S->phys_empty[slot]));
      if (pc.first) {
        // later units: q is overwritten once the previous unit's last QK^T has run
        if (t == 0 && v > 0 && tc::mbar_wait_cl(tc::smem_u32(&S->q_empty), (v - 1) & 1u, abort, status)) load_q(pc.row);
        ++v;
      }
      pc.next(a, npairs);
    }
  } else if (warp >= 8 && warp < 12) {
    // ====================================================================== cross (128 threads)
    ATT_REGS_DEC(kAttRegsCross);
    // Chunk c: the peer's 32 tokens' half of the values (rank 0 takes dims 0-255, rank 1 dims 256-511),
    // 16 bytes per load, a warp reading one 512-byte row segment per step, into registers; once QK^T of the
    // chunk has run they are stored with the 128-byte swizzle into the dim blocks it no longer needs
    // (rank 0: 4-7, rank 1: 0-3).  Masked tokens store zeros.
    const int t = threadIdx.x - 256;
    const uint32_t dst_blk0 = rank == 0 ? 4u : 0u;
    const int dim0 = rank == 0 ? 0 : 256;
    constexpr int kCrossVec = 4 * kAttBlkBytes / 16 / 128;      // 16-byte loads per thread
    const uint32_t v_ready_r0 = tc::map_to_rank(tc::smem_u32(&S->v_ready[0]), 0);
    uint32_t c = 0;
    for (int u = pair; u < U; u += npairs) {
      int row, cb, ce;
      unit_of(a, u, &row, &cb, &ce);
      for (int i = 0; i < ce - cb; ++i, ++c) {
        const uint32_t b = c % kAttNBuf, slot = c % kAttRing;
        const bool ok = __all_sync(0xffffffffu, tc::mbar_wait(tc::smem_u32(&S->phys_full[slot]), (c / kAttRing) & 1u, abort, status));
        const int32_t *ph = S->phys[slot] + kAttHalf * (int)(rank ^ 1u);
        uint4 val[kCrossVec];
#pragma unroll
        for (int m = 0; m < kCrossVec; ++m) {
          const int idx = t + 128 * m, r = idx >> 5, cq = idx & 31;
          const int pr = ph[r];
          val[m] = (ok && pr >= 0) ? __ldg(reinterpret_cast<const uint4 *>(a.kv + (int64_t)pr * kAttD + dim0 + cq * 8))
                                   : make_uint4(0, 0, 0, 0);
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(tc::smem_u32(&S->phys_empty[slot]));
        // QK^T of the chunk has read this CTA's buffer
        const bool have = __all_sync(0xffffffffu, tc::mbar_wait_cl(tc::smem_u32(&S->s_full[c & 1u]), (c >> 1) & 1u, abort, status));
        if (have) {
          uint8_t *base = sBuf + b * kAttBufBytes + dst_blk0 * kAttBlkBytes;
#pragma unroll
          for (int m = 0; m < kCrossVec; ++m) {
            const int idx = t + 128 * m, r = idx >> 5, cq = idx & 31;
            *reinterpret_cast<uint4 *>(base + (cq >> 3) * kAttBlkBytes + r * 128 + (((cq & 7) ^ (r & 7)) << 4)) = val[m];
          }
        }
        tc::fence_proxy_async();
        __syncwarp();
        if (lane == 0) {
          if (rank == 0) tc::mbar_arrive(tc::smem_u32(&S->v_ready[b]));
          else tc::mbar_arrive_remote(v_ready_r0 + b * 8);
        }
      }
    }
  } else if (warp == kAttWarpMMA) {
    // ====================================================================== MMA issuer (rank 0, whole warp)
    ATT_REGS_DEC(kAttRegsMisc);
    // The warp runs the loop uniformly and one elected lane issues each MMA and commit.  Descriptors are a
    // base descriptor plus the byte offset / 16 (the address field cannot carry: shared memory < 256 KB).
    if (rank == 0) {
      const uint32_t idesc_qk = tc::make_idesc(1, 1, 128, kAttChunk, false, false);
      const uint32_t idesc_pv = tc::make_idesc(1, 1, 128, 256, false, true);
      const uint16_t both = 3;
      const uint64_t q_desc = tc::desc_sw128(tc::smem_u32(sQ), 1024);
      const uint64_t p_desc = tc::desc_sw128(tc::smem_u32(sP), 1024);
      const uint64_t kv_desc = tc::desc_sw128(tc::smem_u32(sBuf), 1024);
      const uint64_t v_desc = tc::desc_sw128_lbo(tc::smem_u32(sBuf), kAttBlkBytes, 1024);
      uint32_t v = 0, c = 0;
      bool ok = true;
      auto pv = [&](uint32_t cc, bool first) -> bool {
        const uint32_t b = cc % kAttNBuf, pb = cc & 1u;
        if (!tc::mbar_wait_cl_w(tc::smem_u32(&S->p_full[pb]), (cc >> 1) & 1u, abort, status)) return false;
        if (!tc::mbar_wait_cl_w(tc::smem_u32(&S->v_ready[b]), (cc / kAttNBuf) & 1u, abort, status)) return false;
        if (first && v > 0 && !tc::mbar_wait_cl_w(tc::smem_u32(&S->o_empty), (v - 1) & 1u, abort, status)) return false;
        tc::fence_after_sync();
        const uint64_t pa = p_desc + ((pb * kAttPBytes) >> 4), vb = v_desc + ((b * kAttBufBytes) >> 4);
        // per half p of the values: K steps of 16 tokens = kh (token half, 4 dim blocks apart) x ks (16 rows)
        static_assert(kAttHalf == 32, "two 16-token steps per token half");
        constexpr int kS = (16 * 128) >> 4, kH = (4 * kAttBlkBytes) >> 4;
#pragma unroll
        for (int p = 0; p < 2; ++p)
          tc::mma_bf16_pair_x4_w<kS, kH, kH + kS>(tmem + kTmemO + 128 * p, pa, vb + ((2 * p * kAttBlkBytes) >> 4), idesc_pv,
                                                  first ? 0u : 1u);
        tc::mma_commit_pair_w(tc::smem_u32(&S->buf_empty[b]), both);
        tc::mma_commit_pair_w(tc::smem_u32(&S->pv_done[pb]), both);
        return true;
      };
      for (int u = pair; u < U && ok; u += npairs) {
        int row, cb, ce;
        unit_of(a, u, &row, &cb, &ce);
        const int nch = ce - cb;
        if (nch <= 0) continue;
        if (!tc::mbar_wait_cl_w(tc::smem_u32(&S->q_full), v & 1u, abort, status)) break;
        tc::fence_after_sync();
        const uint32_t c0 = c;
        for (int i = 0; i < nch; ++i) {
          const uint32_t b = c % kAttNBuf;
          if (!tc::mbar_wait_cl_w(tc::smem_u32(&S->buf_full[b]), (c / kAttNBuf) & 1u, abort, status)) { ok = false; break; }
          tc::fence_after_sync();
          const uint64_t kb = kv_desc + ((b * kAttBufBytes) >> 4);
          const uint32_t sb = tmem + kTmemS + kAttHalf * (c & 1u);
          tc::mma_qk36_pair_w<kAttBlkBytes>(sb, q_desc, kb, idesc_qk);
          tc::mma_commit_pair_w(tc::smem_u32(&S->s_full[c & 1u]), both);
          if (i == nch - 1) tc::mma_commit_pair_w(tc::smem_u32(&S->q_empty), both);
          ++c;
          if (i > 0 && !pv(c0 + i - 1, i - 1 == 0)) { ok = false; break; }
        }
        if (ok && !pv(c0 + nch - 1, nch == 1)) ok = false;
        ++v;
      }
      tc::mma_commit_pair_local_w(tc::smem_u32(&S->drain));
      volatile int no_abort = 0;
      __all_sync(0xffffffffu, tc::mbar_wait(tc::smem_u32(&S->drain), 0, &no_abort, status));
    }
  } else if (warp >= 4) {
    ATT_REGS_DEC(kAttRegsMisc);                // the spare warps of the last warpgroup
  } else {
    // ====================================================================== softmax + epilogue (warps 0-3)
    ATT_REGS_INC();
    // The loops never break (they hold named barrier 2): after a timeout the waits return at once and the
    // remaining chunks run through without touching TMEM or memory.
    const int L = threadIdx.x;                 // TMEM lane
    const int h = L & 63, half = L >> 6;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const uint32_t p_full_r0 = tc::map_to_rank(tc::smem_u32(&S->p_full[0]), 0);
    const uint32_t o_empty_r0 = tc::map_to_rank(tc::smem_u32(&S->o_empty), 0);
    uint32_t c = 0;
    for (int u = pair; u < U; u += npairs) {
      int row, cb, ce;
      unit_of(a, u, &row, &cb, &ce);
      const int nch = ce - cb;
      const int head = 64 * (int)rank + h;
      if (nch <= 0) {
        // nothing selected: o = 0, lse = -inf
        if (a.splits == 1) {
          __nv_bfloat16 *o = a.out + ((int64_t)row * kAttH + head) * kAttDv + 256 * half;
          for (int e = 0; e < 256; e += 8) *reinterpret_cast<uint4 *>(o + e) = make_uint4(0, 0, 0, 0);
          if (a.lse && half == 0) a.lse[(int64_t)row * kAttH + head] = -INFINITY;
        } else {
          float *o = a.part_o + ((int64_t)u * kAttH + head) * kAttDv + 256 * half;
          for (int e = 0; e < 256; e += 4) *reinterpret_cast<float4 *>(o + e) = make_float4(0.f, 0.f, 0.f, 0.f);
          if (half == 0) a.part_lse[(int64_t)u * kAttH + head] = -INFINITY;
        }
        continue;
      }
      float m_run = -INFINITY, l_run = 0.f;
      for (int i = 0; i < nch; ++i, ++c) {
        // validity of this thread's 32 tokens
        const uint32_t slot = c % kAttRing;
        const bool m_ok = __all_sync(0xffffffffu, tc::mbar_wait(tc::smem_u32(&S->mask_full[slot]),
                                                                (c / kAttRing) & 1u, abort, status));
        uint32_t valid = m_ok ? S->mask[slot][half] : 0u;
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(tc::smem_u32(&S->mask_empty[slot]));
        const bool have_s =
            __all_sync(0xffffffffu, tc::mbar_wait_cl(tc::smem_u32(&S->s_full[c & 1u]), (c >> 1) & 1u, abort, status));
        tc::fence_after_sync();
        float sv[kAttHalf];
        tc::tmem_ld32(tmem + lane_base + kTmemS + kAttHalf * (c & 1u), sv);
        tc::tmem_wait_ld();
        if (!have_s) valid = 0u;
        float mx = -INFINITY;
#pragma unroll
        for (int e = 0; e < kAttHalf; ++e) {
          sv[e] = ((valid >> e) & 1u) ? sv[e] * a.scale_log2 : -INFINITY;
          mx = fmaxf(mx, sv[e]);
        }
        const float mloc = fmaxf(m_run, mx);
        S->xm[c & 1u][L] = mloc;
        tc::named_bar_sync(2, 128);
        const float m_new = fmaxf(mloc, S->xm[c & 1u][L ^ 64]);
        bool pv_ok = true;
        if (i == 0) {
          m_run = m_new;
        } else {
          // TMEM loads/stores are warp-collective: the warp rescales if any of its rows needs it,
          // rows that do not keep their reference max (alpha = 1).  P V of the previous chunk must
          // have finished before O is touched.
          const bool want = m_new > m_run + kRescaleLog2;
          if (__any_sync(0xffffffffu, want)) {
            const uint32_t cp = c - 1;
            pv_ok = __all_sync(0xffffffffu, tc::mbar_wait_cl(tc::smem_u32(&S->pv_done[cp & 1u]), (cp >> 1) & 1u, abort, status));
            tc::fence_after_sync();
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
              m_run = m_new;
            }
          }
        }
        // this chunk's P buffer was last read by P V of chunk c - 2
        if (c >= 2)
          pv_ok = __all_sync(0xffffffffu, tc::mbar_wait_cl(tc::smem_u32(&S->pv_done[c & 1u]), ((c >> 1) & 1u) ^ 1u, abort,
                                                           status)) && pv_ok;
        // P = exp2(z - m) in bf16 into the 128-byte-swizzled A operand: row h, tokens 32*half + [0, 32);
        // masked tokens hold -inf and give 0.  l_run sums the unrounded P.
        if (pv_ok) {
          const float m_use = m_run == -INFINITY ? 0.f : m_run;
          uint8_t *pbuf = sP + (c & 1u) * kAttPBytes + h * 128;
          float lsum = 0.f;
#pragma unroll
          for (int q8 = 0; q8 < kAttHalf / 8; ++q8) {
            uint32_t w4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int t0 = 8 * q8 + 2 * e;
              const float p0 = tc::ex2(sv[t0] - m_use), p1 = tc::ex2(sv[t0 + 1] - m_use);
              lsum += p0 + p1;
              const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
              w4[e] = *reinterpret_cast<const uint32_t *>(&pb);
            }
            const int kc = (kAttHalf / 8) * half + q8;             // 8-token group within the 64 tokens
            *reinterpret_cast<uint4 *>(pbuf + (((kc & 7) ^ (h & 7)) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
          l_run += lsum;
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) {
          if (rank == 0) tc::mbar_arrive(tc::smem_u32(&S->p_full[c & 1u]));
          else tc::mbar_arrive_remote(p_full_r0 + (c & 1u) * 8);
        }
      }
      // ---- epilogue: wait for the last P V, normalise, store through a per-warp staging tile
      const uint32_t cl = c - 1;
      const bool o_ok =
          __all_sync(0xffffffffu, tc::mbar_wait_cl(tc::smem_u32(&S->pv_done[cl & 1u]), (cl >> 1) & 1u, abort, status));
      tc::fence_after_sync();
      S->xl[L] = l_run;
      tc::named_bar_sync(2, 128);
      const float l_tot = l_run + S->xl[L ^ 64];
      const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
      const float lse_v = l_tot > 0.f ? (m_run + __log2f(l_tot)) * 0.69314718055994531f : -INFINITY;
      if (o_ok) {
        // both P buffers are free once the last P V finished: each warp stages a 32 x 32 fp32 tile
        // (row = lane, 16-byte group j at j ^ (row & 7)) and writes whole 128-byte row segments
        float *stg = reinterpret_cast<float *>(sP) + warp * 1024;
        const int head0 = 64 * (int)rank + 32 * (warp & 1), col0 = 256 * (warp >> 1);
        for (int cc = 0; cc < 8; ++cc) {
          float ov[32];
          tc::tmem_ld32(tmem + lane_base + kTmemO + 32 * cc, ov);
          tc::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<float4 *>(stg + lane * 32 + 4 * (j ^ (lane & 7))) =
                make_float4(ov[4 * j] * inv, ov[4 * j + 1] * inv, ov[4 * j + 2] * inv, ov[4 * j + 3] * inv);
          __syncwarp();
          if (a.splits == 1) {
#pragma unroll
            for (int it = 0; it < 4; ++it) {
              const int r = 8 * it + (lane >> 2), j0 = 2 * (lane & 3);
              const float4 f0 = *reinterpret_cast<const float4 *>(stg + r * 32 + 4 * (j0 ^ (r & 7)));
              const float4 f1 = *reinterpret_cast<const float4 *>(stg + r * 32 + 4 * ((j0 + 1) ^ (r & 7)));
              __nv_bfloat162 b0 = __floats2bfloat162_rn(f0.x, f0.y), b1 = __floats2bfloat162_rn(f0.z, f0.w);
              __nv_bfloat162 b2 = __floats2bfloat162_rn(f1.x, f1.y), b3 = __floats2bfloat162_rn(f1.z, f1.w);
              uint4 w;
              w.x = *reinterpret_cast<uint32_t *>(&b0);
              w.y = *reinterpret_cast<uint32_t *>(&b1);
              w.z = *reinterpret_cast<uint32_t *>(&b2);
              w.w = *reinterpret_cast<uint32_t *>(&b3);
              *reinterpret_cast<uint4 *>(a.out + ((int64_t)row * kAttH + head0 + r) * kAttDv + col0 + 32 * cc + 4 * j0) = w;
            }
          } else {
#pragma unroll
            for (int it = 0; it < 8; ++it) {
              const int r = 4 * it + (lane >> 3), j = lane & 7;
              *reinterpret_cast<float4 *>(a.part_o + ((int64_t)u * kAttH + head0 + r) * kAttDv + col0 + 32 * cc + 4 * j) =
                  *reinterpret_cast<const float4 *>(stg + r * 32 + 4 * (j ^ (r & 7)));
            }
          }
          __syncwarp();
        }
        if (half == 0) {
          if (a.splits == 1) {
            if (a.lse) a.lse[(int64_t)row * kAttH + head] = lse_v;
          } else {
            a.part_lse[(int64_t)u * kAttH + head] = lse_v;
          }
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0) tc::mbar_arrive(tc::smem_u32(&S->o_empty));
        else tc::mbar_arrive_remote(o_empty_r0);
      }
    }
  }

  // ---- teardown: every role is done; MMAs drained; peers done with our barriers, buffers and TMEM
  tc::fence_before_sync();
  __syncthreads();
  tc::cluster_sync();
  if (warp == kAttWarpMMA) {
    tc::fence_after_sync();
    tc::tmem_dealloc2(tmem, 512);
  }
#undef ATT_REGS_DEC
#undef ATT_REGS_INC
}

// ------------------------------------------------------------------------------------------------ combine
// out[row, h, :] = sum_s exp(lse_s - lse) o_s,  lse = log sum_s exp(lse_s)   (splits of one row)
// Up to kCombineRegSplits splits: their lse values and partial outputs are loaded in one round.  More splits (a
// single long row spread over many CTA pairs): every split's lse goes to shared memory (one load per thread)
// and the partial outputs come in batches of kCombineRegSplits, each batch's loads issued before the previous
// batch is summed.  Either way the sums run over the splits in order; a split with lse = -inf wrote zeros and
// gets weight 0.
constexpr int kCombineRegSplits = 8;
constexpr int kCombineMaxSplits = 128;           // >= the largest split count (74 CTA pairs)
__device__ __forceinline__ void combine_issue(const float *po, int splits, int s0, float4 (&o)[kCombineRegSplits]) {
#pragma unroll
  for (int j = 0; j < kCombineRegSplits; ++j)
    o[j] = s0 + j < splits ? __ldg(reinterpret_cast<const float4 *>(po + (int64_t)(s0 + j) * kAttH * kAttDv))
                           : make_float4(0.f, 0.f, 0.f, 0.f);
}
__global__ void __launch_bounds__(128) attn_combine_many_kernel(const float *__restrict__ part_o,
                                                                const float *__restrict__ part_lse, int splits,
                                                                __nv_bfloat16 *__restrict__ out, float *__restrict__ lse) {
  __shared__ float s_l[kCombineMaxSplits];
  pdl_wait();
  pdl_trigger();
  const int row = blockIdx.x, h = blockIdx.y;
  const float *pl = part_lse + (int64_t)row * splits * kAttH + h;
  const int dv = threadIdx.x * 4;
  const float *po = part_o + ((int64_t)row * splits * kAttH + h) * kAttDv + dv;
  {
    float4 nxt[kCombineRegSplits];
    combine_issue(po, splits, 0, nxt);
    for (int s = threadIdx.x; s < splits; s += blockDim.x) s_l[s] = __ldg(pl + (int64_t)s * kAttH);
    __syncthreads();
    float mx = -INFINITY;
    for (int s = 0; s < splits; ++s) mx = fmaxf(mx, s_l[s]);
    float tot = 0.f;
    for (int s = 0; s < splits; ++s) tot += s_l[s] == -INFINITY ? 0.f : __expf(s_l[s] - mx);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (tot > 0.f) {
      for (int s0 = 0; s0 < splits; s0 += kCombineRegSplits) {
        float4 cur[kCombineRegSplits];
#pragma unroll
        for (int j = 0; j < kCombineRegSplits; ++j) cur[j] = nxt[j];
        if (s0 + kCombineRegSplits < splits) combine_issue(po, splits, s0 + kCombineRegSplits, nxt);
#pragma unroll
        for (int j = 0; j < kCombineRegSplits; ++j) {
          const int s = s0 + j;
          if (s >= splits || s_l[s] == -INFINITY) continue;
          const float wgt = __expf(s_l[s] - mx) / tot;
          acc.x += wgt * cur[j].x;
          acc.y += wgt * cur[j].y;
          acc.z += wgt * cur[j].z;
          acc.w += wgt * cur[j].w;
        }
      }
    }
    __nv_bfloat162 b0 = __floats2bfloat162_rn(acc.x, acc.y), b1 = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 w;
    w.x = *reinterpret_cast<uint32_t *>(&b0);
    w.y = *reinterpret_cast<uint32_t *>(&b1);
    *reinterpret_cast<uint2 *>(out + ((int64_t)row * kAttH + h) * kAttDv + dv) = w;
    if (lse && threadIdx.x == 0) lse[(int64_t)row * kAttH + h] = tot > 0.f ? mx + __logf(tot) : -INFINITY;
  }
}
__global__ void __launch_bounds__(128) attn_combine_kernel(const float *__restrict__ part_o,
                                                           const float *__restrict__ part_lse, int splits,
                                                           __nv_bfloat16 *__restrict__ out, float *__restrict__ lse) {
  pdl_wait();
  pdl_trigger();
  const int row = blockIdx.x, h = blockIdx.y;
  const float *pl = part_lse + (int64_t)row * splits * kAttH + h;
  const int dv = threadIdx.x * 4;
  const float *po = part_o + ((int64_t)row * splits * kAttH + h) * kAttDv + dv;
  float lreg[kCombineRegSplits];
  float4 o[kCombineRegSplits];
#pragma unroll
  for (int s = 0; s < kCombineRegSplits; ++s) {
    lreg[s] = s < splits ? __ldg(pl + (int64_t)s * kAttH) : -INFINITY;
    o[s] = s < splits ? __ldg(reinterpret_cast<const float4 *>(po + (int64_t)s * kAttH * kAttDv))
                      : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  float mx = -INFINITY;
#pragma unroll
  for (int s = 0; s < kCombineRegSplits; ++s) mx = fmaxf(mx, lreg[s]);
  for (int s = kCombineRegSplits; s < splits; ++s) mx = fmaxf(mx, __ldg(pl + (int64_t)s * kAttH));
  float tot = 0.f;
#pragma unroll
  for (int s = 0; s < kCombineRegSplits; ++s)
    if (s < splits) tot += lreg[s] == -INFINITY ? 0.f : __expf(lreg[s] - mx);
  for (int s = kCombineRegSplits; s < splits; ++s) {
    const float l = __ldg(pl + (int64_t)s * kAttH);
    tot += l == -INFINITY ? 0.f : __expf(l - mx);
  }
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (tot > 0.f) {
#pragma unroll
    for (int s = 0; s < kCombineRegSplits; ++s) {
      if (s >= splits || lreg[s] == -INFINITY) continue;
      const float wgt = __expf(lreg[s] - mx) / tot;
      acc.x += wgt * o[s].x;
      acc.y += wgt * o[s].y;
      acc.z += wgt * o[s].z;
      acc.w += wgt * o[s].w;
    }
    for (int s = kCombineRegSplits; s < splits; ++s) {
      const float l = __ldg(pl + (int64_t)s * kAttH);
      if (l == -INFINITY) continue;
      const float wgt = __expf(l - mx) / tot;
      const float4 os = __ldg(reinterpret_cast<const float4 *>(po + (int64_t)s * kAttH * kAttDv));
      acc.x += wgt * os.x;
      acc.y += wgt * os.y;
      acc.z += wgt * os.z;
      acc.w += wgt * os.w;
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

static size_t attn_smem_bytes() {
  return 1024 + kAttQBytes + kAttNBuf * kAttBufBytes + 2 * kAttPBytes + sizeof(AttSmem);
}

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
  DSA_LAUNCH_PDL("attn_plan_kernel", attn_plan_kernel, dim3(a.T), dim3(kAttPlanThreads), 0, stream, idx, k, a.bv, a.T,
                 neff, a.status);
  const size_t smem = attn_smem_bytes();
  cudaFuncSetAttribute(attn_mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  // persistent grid: as many CTA pairs as can be resident at once (found once per device; threads that race
  // on the first call compute the same number)
  static std::atomic<int> resident_pairs[kMaxDevices];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) dev = -1;
  int max_pairs = dev >= 0 ? resident_pairs[dev].load(std::memory_order_relaxed) : 0;
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
    if (dev >= 0) resident_pairs[dev].store(max_pairs, std::memory_order_relaxed);
    if (getenv("DSA_VERBOSE")) fprintf(stderr, "[libdsa] attention: %d resident CTA pairs\n", max_pairs);
  }
  const int units = a.T * a.splits;
  const int pairs = std::min(max_pairs, units);
  DSA_LAUNCH_PDL("attn_mla_kernel", attn_mla_kernel, dim3(2 * pairs), dim3(kAttThreads), smem, stream, tm_q, tm_kv, a);
  if (a.splits > 1) {
    if (a.splits <= kCombineRegSplits) {
      DSA_LAUNCH_PDL("attn_combine_kernel", attn_combine_kernel, dim3(a.T, kAttH), dim3(128), 0, stream,
                     (const float *)a.part_o, (const float *)a.part_lse, a.splits, (__nv_bfloat16 *)out, lse);
    } else {
      static_assert(kAttPairsForSplits <= kCombineMaxSplits, "every split's lse fits in shared memory");
      DSA_LAUNCH_PDL("attn_combine_many_kernel", attn_combine_many_kernel, dim3(a.T, kAttH), dim3(128), 0, stream,
                     (const float *)a.part_o, (const float *)a.part_lse, a.splits, (__nv_bfloat16 *)out, lse);
    }
  }
  return DSA_OK;
}

}  // namespace dsa
