// sm_100a building blocks for the tensor-core kernels: mbarriers with bounded waits, TMA and
// bulk copies, and tcgen05 (TMEM allocation, MMA issue/commit, TMEM loads).  Inline PTX only.
#pragma once

#include <cuda.h>
#include "common.cuh"

namespace dsa {
namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

// ------------------------------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: gives up after ~`budget` SM cycles (several seconds at B200 clocks), or as soon as
// another role has raised `abort`.  On giving up it raises `abort` and the workspace timeout bit.
constexpr long long kWaitBudget = 8000000000LL;

__device__ __forceinline__ bool mbar_wait_for(uint32_t bar, uint32_t parity, volatile int *abort, uint32_t *status,
                                              long long budget) {
  if (mbar_try_wait(bar, parity)) return true;
  if (*abort) return false;
  const long long t0 = clock64();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 0u) {
      if (*abort) return false;
      if (clock64() - t0 > budget) {
        *abort = 1;
        set_status(status, kStatusTimeout);
        return false;
      }
    }
  }
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort, uint32_t *status) {
  return mbar_wait_for(bar, parity, abort, status, kWaitBudget);
}

// ------------------------------------------------------------------------------------------ copies
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int c0, int c1, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
// CTA-pair forms (.cta_group::2, no multicast): the data lands in this CTA's shared memory and the
// completion bytes are counted on `bar`, a shared::cluster address that may be the barrier of either CTA
// of the pair (the peer's, to gather both halves of an operand on the MMA-issuing CTA's barrier).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, int c0, int c1, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.cta_group::2 "
      "[%0], [%1, {%3, %4}], [%2];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_gather4_pair(uint32_t dst, const CUtensorMap *map, int col, int r0, int r1, int r2,
                                                 int r3, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes.cta_group::2 "
      "[%0], [%1, {%2, %3, %4, %5, %6}], [%7];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(col), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}
// bring `bytes` (multiple of 16) of global memory into L2 without waiting for it
__device__ __forceinline__ void prefetch_l2(const void *src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------------------------------------------ tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 bits, 32 consecutive columns -> 32 registers per thread
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// ------------------------------------------------------------------------------------------ descriptors
// Shared-memory matrix descriptor, K-major operand stored with the 128-byte swizzle: rows of 128 bytes,
// 8-row atoms of 1024 bytes stacked at stride `sbo` bytes; the leading offset is unused for this mode.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;                              // leading byte offset (ignored for SW128 K-major)
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;          // stride byte offset
  d |= (uint64_t)1u << 46;                              // descriptor version (sm_100)
  d |= (uint64_t)2u << 61;                              // layout: 128-byte swizzle
  return d;
}

// Shared-memory matrix descriptor with explicit leading and stride offsets (both in bytes).
__device__ __forceinline__ uint64_t desc_sw128_lbo(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

// Instruction descriptor: dense MMA, fp32 accumulator, both operands K-major unless flagged.
//   kind::f8f6f4 with e4m3 inputs: a_fmt = b_fmt = 0;  kind::f16 with bf16 inputs: a_fmt = b_fmt = 1.
__host__ __device__ constexpr uint32_t make_idesc(uint32_t a_fmt, uint32_t b_fmt, int M, int N, bool a_mn_major,
                                                  bool b_mn_major) {
  return (1u << 4)                                   // D format: f32
         | (a_fmt << 7) | (b_fmt << 10)              // A / B formats
         | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16)
         | ((uint32_t)(N >> 3) << 17)                // N / 8
         | ((uint32_t)(M >> 4) << 24);               // M / 16
}

// ------------------------------------------------------------------------------------------ clusters
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// address of the same shared-memory location in CTA `rank` of this cluster
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
// Arrive on a barrier of the other CTA of the pair with the default (release, CTA-scope) semantics, the
// form CTA-pair pipelines use for consumer/producer signals: cheap (tens of cycles) where a cluster-scope
// release waits for every memory operation the SM has in flight.  Data written to this CTA's shared memory
// for the tensor cores is published with fence.proxy.async before the arrive.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cl(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// bounded wait with cluster-scope acquire (for barriers that receive arrivals from the peer CTA)
__device__ __forceinline__ bool mbar_wait_cl(uint32_t bar, uint32_t parity, volatile int *abort, uint32_t *status) {
  if (mbar_try_wait_cl(bar, parity)) return true;
  if (*abort) return false;
  const long long t0 = clock64();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait_cl(bar, parity)) return true;
    if ((i & 255u) == 0u) {
      if (*abort) return false;
      if (clock64() - t0 > kWaitBudget) {
        *abort = 1;
        set_status(status, kStatusTimeout);
        return false;
      }
    }
  }
}

__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ------------------------------------------------------------------------------------------ tcgen05, CTA pairs
__device__ __forceinline__ void tmem_alloc2(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish2() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// MMA issue, warp-wide forms: every lane of the warp executes the call with the same operands and one
// elected lane issues.  Warp-uniform issuing code keeps the operands in uniform registers; issuing from a
// single divergent thread cost about 60 cycles per tcgen05.mma, several MMAs per inline-asm block with
// immediate descriptor offsets about 18.
//
// Four MMAs of a CTA pair issued by one elected lane in one block: A advances by one 16-element K step
// (32 bytes) per MMA, B by the descriptor-unit offsets B1, B2, B3 (bytes / 16).  Only the first MMA may
// start a fresh accumulator (`accumulate` = 0); the other three accumulate.
template <int B1, int B2, int B3>
__device__ __forceinline__ void mma_bf16_pair_x4_w(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                   uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e, t;\n\t.reg .b64 a1, a2, a3, b1, b2, b3;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 t, 0, 0;\n\t"
      "add.u64 a1, %1, 2;\n\tadd.u64 a2, %1, 4;\n\tadd.u64 a3, %1, 6;\n\t"
      "add.u64 b1, %2, %5;\n\tadd.u64 b2, %2, %6;\n\tadd.u64 b3, %2, %7;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], a1, b1, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], a2, b2, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], a3, b3, %3, t;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "n"(B1), "n"(B2), "n"(B3)
      : "memory");
}
// The 36 MMAs of a QK^T chunk (9 dim blocks x 4 K steps) in one block issued by one elected lane: A (q)
// advances 8192 bytes per dim block, B (the chunk buffer) kBBlk bytes, both 32 bytes per K step; the
// first MMA starts a fresh accumulator, the rest accumulate.  Descriptor offsets are immediates (bytes/16).
template <int kBBlk>
__device__ __forceinline__ void mma_qk36_pair_w(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc) {
  static_assert(kBBlk == 4096, "immediates below assume 4 KB dim blocks");
  asm volatile(
      "{\n\t.reg .pred e, t, f;\n\t.reg .b64 ra, rb;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.eq.b32 t, 0, 0;\n\t"
      "setp.ne.b32 f, 0, 0;\n\t"
      "add.u64 ra, %1, 0;\n\tadd.u64 rb, %2, 0;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, f;\n\t"
      "add.u64 ra, %1, 2;\n\tadd.u64 rb, %2, 2;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 4;\n\tadd.u64 rb, %2, 4;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 6;\n\tadd.u64 rb, %2, 6;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 512;\n\tadd.u64 rb, %2, 256;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 514;\n\tadd.u64 rb, %2, 258;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 516;\n\tadd.u64 rb, %2, 260;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 518;\n\tadd.u64 rb, %2, 262;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 1024;\n\tadd.u64 rb, %2, 512;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 1026;\n\tadd.u64 rb, %2, 514;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 1028;\n\tadd.u64 rb, %2, 516;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 1030;\n\tadd.u64 rb, %2, 518;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 1536;\n\tadd.u64 rb, %2, 768;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 1538;\n\tadd.u64 rb, %2, 770;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 1540;\n\tadd.u64 rb, %2, 772;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 1542;\n\tadd.u64 rb, %2, 774;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 2048;\n\tadd.u64 rb, %2, 1024;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 2050;\n\tadd.u64 rb, %2, 1026;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 2052;\n\tadd.u64 rb, %2, 1028;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 2054;\n\tadd.u64 rb, %2, 1030;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 2560;\n\tadd.u64 rb, %2, 1280;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 2562;\n\tadd.u64 rb, %2, 1282;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 2564;\n\tadd.u64 rb, %2, 1284;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 2566;\n\tadd.u64 rb, %2, 1286;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 3072;\n\tadd.u64 rb, %2, 1536;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 3074;\n\tadd.u64 rb, %2, 1538;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 3076;\n\tadd.u64 rb, %2, 1540;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 3078;\n\tadd.u64 rb, %2, 1542;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 3584;\n\tadd.u64 rb, %2, 1792;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 3586;\n\tadd.u64 rb, %2, 1794;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 3588;\n\tadd.u64 rb, %2, 1796;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 3590;\n\tadd.u64 rb, %2, 1798;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 4096;\n\tadd.u64 rb, %2, 2048;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 4098;\n\tadd.u64 rb, %2, 2050;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 4100;\n\tadd.u64 rb, %2, 2052;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "add.u64 ra, %1, 4102;\n\tadd.u64 rb, %2, 2054;\n\t@e tcgen05.mma.cta_group::2.kind::f16 [%0], ra, rb, %3, t;\n\t"
      "}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc)
      : "memory");
}
__device__ __forceinline__ void mma_commit_pair_w(uint32_t bar, uint16_t cta_mask) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;\n\t}"
      ::"r"(bar), "h"(cta_mask)
      : "memory");
}
__device__ __forceinline__ void mma_commit_pair_local_w(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
      : "memory");
}
__device__ __forceinline__ void mma_f8f6f4_w(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_commit_w(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
      : "memory");
}
__device__ __forceinline__ bool mbar_wait_w(uint32_t bar, uint32_t parity, volatile int *abort, uint32_t *status) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, status));
}
// warp-uniform bounded wait: true only if the wait succeeded for every lane
__device__ __forceinline__ bool mbar_wait_cl_w(uint32_t bar, uint32_t parity, volatile int *abort, uint32_t *status) {
  return __all_sync(0xffffffffu, mbar_wait_cl(bar, parity, abort, status));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
      ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])),
        "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
        "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
        "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])),
        "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
        "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])),
        "r"(__float_as_uint(v[23])), "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])),
        "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])),
        "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

}  // namespace tc
}  // namespace dsa
