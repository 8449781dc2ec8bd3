// Shared device helpers for libdsa (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "dsa.h"

namespace dsa {

// ---------------------------------------------------------------------------------------------
// workspace status word: every workspace starts with a 256-byte header whose first u32 collects
// error bits set by kernels (bounded waits that ran out, out-of-range ids).
// ---------------------------------------------------------------------------------------------
constexpr size_t kWsHeader = 256;
constexpr int kMaxDevices = 64;        // per-device host caches are indexed by the CUDA device ordinal
constexpr uint32_t kStatusTimeout = 1u;
constexpr uint32_t kStatusBadIndex = 2u;

__device__ __forceinline__ void set_status(uint32_t *status, uint32_t bit) {
  if (status) atomicOr(status, bit);
}

// ---------------------------------------------------------------------------------------------
// batch helpers
// ---------------------------------------------------------------------------------------------
struct BatchView {
  const int32_t *block_table;
  const int32_t *seq_lens;
  const int32_t *cu_q;
  int32_t num_seqs, page_size, max_blocks_per_seq, num_blocks;
};

inline BatchView view_of(const dsa_batch_t *b) {
  return BatchView{b->block_table, b->seq_lens, b->cu_q, b->num_seqs, b->page_size, b->max_blocks_per_seq,
                   b->num_blocks};
}

// sequence of query row `row` (largest b with cu_q[b] <= row), by binary search
__device__ __forceinline__ int seq_of_row(const int32_t *cu_q, int num_seqs, int row) {
  int lo = 0, hi = num_seqs - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu_q + mid) <= row) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// absolute position of a query row: rows of sequence b are its last n_b tokens
__device__ __forceinline__ int pos_of_row(const BatchView &bv, int row, int *seq_out) {
  int b = seq_of_row(bv.cu_q, bv.num_seqs, row);
  int c0 = __ldg(bv.cu_q + b), c1 = __ldg(bv.cu_q + b + 1);
  *seq_out = b;
  return __ldg(bv.seq_lens + b) - (c1 - c0) + (row - c0);
}

// seq_of_row for a whole warp (every lane calls it with the same row and gets the same result): each
// round the 32 lanes test 32 evenly spaced entries of cu_q at once, so a batch of up to 33 sequences
// needs one round of loads instead of a chain of dependent ones.  cu_q is non-decreasing, so the lanes
// whose entry is <= row form a prefix of the warp.
__device__ __forceinline__ int seq_of_row_warp(const int32_t *cu_q, int num_seqs, int row) {
  const int lane = threadIdx.x & 31;
  int lo = 0, hi = num_seqs - 1;       // the answer lies in [lo, hi]
  while (lo < hi) {
    const int step = (hi - lo + 31) / 32;
    const int i = lo + 1 + lane * step;
    const bool le = i <= hi && __ldg(cu_q + i) <= row;
    const unsigned m = __ballot_sync(0xffffffffu, le);
    if (m == 0u) {
      hi = lo;
    } else {
      const int last = 31 - __clz(m);
      lo = lo + 1 + last * step;
      hi = min(hi, lo + step - 1);
    }
  }
  return lo;
}
__device__ __forceinline__ int pos_of_row_warp(const BatchView &bv, int row, int *seq_out) {
  int b = seq_of_row_warp(bv.cu_q, bv.num_seqs, row);
  int c0 = __ldg(bv.cu_q + b), c1 = __ldg(bv.cu_q + b + 1);
  *seq_out = b;
  return __ldg(bv.seq_lens + b) - (c1 - c0) + (row - c0);
}

// physical row (block * page + slot) of logical token s of sequence b; -1 if the block id is bad
__device__ __forceinline__ int64_t phys_row(const BatchView &bv, int b, int s) {
  int blk = __ldg(bv.block_table + (int64_t)b * bv.max_blocks_per_seq + s / bv.page_size);
  if ((unsigned)blk >= (unsigned)bv.num_blocks) return -1;
  return (int64_t)blk * bv.page_size + (s % bv.page_size);
}

// Programmatic dependent launch: every kernel of the path is launched so that it may start while the
// previous kernel of the stream finishes.  pdl_wait() blocks until the previous grid has completed and its
// memory is visible, and must precede every global-memory access of the kernel (reads of inputs that the
// previous kernel may produce, writes that it may still read); pdl_trigger() lets the next kernel launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// fp32 -> unsigned key whose integer order is the float order (-0 folded onto +0)
__device__ __forceinline__ uint32_t ordered_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float e4m3_to_float(uint8_t v) {
  __nv_fp8_e4m3 x;
  x.__x = v;
  return float(x);
}

// ---------------------------------------------------------------------------------------------
// block-wide exclusive scan (blockDim.x multiple of 32, <= 1024); `tmp` holds 33 u32 in smem
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t *tmp, uint32_t *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t t = lane < nwarps ? tmp[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < nwarps) tmp[lane] = t;       // inclusive warp totals
    if (lane == 31) tmp[32] = t;
  }
  __syncthreads();
  uint32_t base = warp > 0 ? tmp[warp - 1] : 0u;
  if (total) *total = tmp[32];
  uint32_t r = base + x - v;
  __syncthreads();
  return r;
}

}  // namespace dsa

// ---------------------------------------------------------------------------------------------
// host-side launch helpers (declared here, defined in dsa_api.cu)
// ---------------------------------------------------------------------------------------------
namespace dsa {
void set_error(const char *fmt, ...);
void count_launch();
}

#include <utility>
namespace dsa {
// launch with programmatic stream serialization (see pdl_wait / pdl_trigger)
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}
}  // namespace dsa

// launch a kernel with launch_pdl and fail the calling entry point on a launch error
#define DSA_LAUNCH_PDL(what, kernel, grid, block, smem, stream, ...)                    \
  do {                                                                                   \
    cudaError_t le_ = ::dsa::launch_pdl(kernel, grid, block, smem, stream, __VA_ARGS__); \
    if (le_ != cudaSuccess) {                                                            \
      ::dsa::set_error("%s: %s", what, cudaGetErrorString(le_));                         \
      return DSA_ERR_CUDA;                                                               \
    }                                                                                    \
    DSA_LAUNCH_CHECK(what);                                                              \
  } while (0)

#define DSA_LAUNCH_CHECK(what)                                                 \
  do {                                                                         \
    ::dsa::count_launch();                                                     \
    cudaError_t e_ = cudaGetLastError();                                       \
    if (e_ != cudaSuccess) {                                                   \
      ::dsa::set_error("%s: %s", what, cudaGetErrorString(e_));                \
      return DSA_ERR_CUDA;                                                     \
    }                                                                          \
  } while (0)
