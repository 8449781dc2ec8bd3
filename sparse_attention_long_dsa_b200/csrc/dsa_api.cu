// C ABI of libdsa: argument validation, workspace sizing and kernel dispatch.
// Every check runs on the host before anything is enqueued; see include/dsa.h for the contract.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>

#include "append.cuh"
#include "common.cuh"

namespace dsa {

// kernels (defined in the other translation units)
dsa_status_t topk_launch(const float *scores, int64_t ld, const dsa_batch_t *b, int k, int32_t *idx, void *ws,
                         cudaStream_t stream, int num_sms);
size_t topk_workspace_bytes(int total_q, int max_seq_len);
dsa_status_t topk_noalloc_launch(const float *scores, int64_t ld, const dsa_batch_t *b, int k, int32_t *idx,
                                 cudaStream_t stream, int num_sms);
dsa_status_t indexer_simt_launch(const void *qI, dsa_dtype_t dt, const float *w, const void *kpool,
                                 const float *kscale, int Hi, int Di, const dsa_batch_t *b, float *scores,
                                 int64_t ld, cudaStream_t stream);
dsa_status_t indexer_tc_launch(const uint8_t *qI, const float *w, const uint8_t *kpool, const float *kscale,
                               const dsa_batch_t *b, float *scores, int64_t ld, void *ws, cudaStream_t stream,
                               int num_sms, const AppendArgs *app, uint32_t *hist);
size_t indexer_workspace_bytes(int num_seqs, int total_q);
size_t indexer_hist_bytes(int total_q);
dsa_status_t select_launch(const float *scores, int64_t ld, const dsa_batch_t *b, int k, int32_t *idx,
                           const uint32_t *hist, uint32_t *status, void *long_ws, cudaStream_t stream, int num_sms);
size_t select_long_ws_bytes(int total_q, int max_seq_len);
dsa_status_t attn_mla_launch(const void *q, const void *kv, const int32_t *idx, int k, float softmax_scale,
                             const dsa_batch_t *b, void *out, float *lse, void *ws, bool decode, cudaStream_t stream,
                             int num_sms);
size_t attn_workspace_bytes(int T, int k, bool decode);
dsa_status_t cache_append_launch(const void *kv_new, const void *k_new, bool k_bf16, const dsa_batch_t *b,
                                 void *kv_pool, void *kI_pool, float *kS_pool, void *ws, cudaStream_t stream);
dsa_status_t selftest_wait_launch(long long budget, void *ws, cudaStream_t stream);
dsa_status_t reuse_candidates_launch(const int32_t *prev_idx, int k, const int32_t *prev_lens, int max_new,
                                     const dsa_batch_t *b, int32_t *cand, void *ws, cudaStream_t stream);
dsa_status_t indexer_at_launch(const uint8_t *qI, const float *w, const uint8_t *kpool, const float *kscale,
                               const dsa_batch_t *b, const int32_t *cand, int m, float *out, void *ws,
                               cudaStream_t stream);
dsa_status_t gather_positions_launch(const int32_t *sel, int k, const int32_t *cand, int m, int T, int32_t *idx,
                                     cudaStream_t stream);
dsa_status_t block_scores_launch(const float *scores, int64_t ld, const dsa_batch_t *b, float *blk, int64_t ld_blk,
                                 int32_t *blk_lens, cudaStream_t stream);
dsa_status_t expand_blocks_launch(const int32_t *blk_idx, int kb, const dsa_batch_t *b, int32_t *idx,
                                  cudaStream_t stream);
dsa_status_t cp_candidates_launch(const float *scores, int64_t ld, const int32_t *idx, int T, int k,
                                  const int32_t *offsets, float *cand_score, int32_t *cand_gidx, cudaStream_t stream);
dsa_status_t cp_rows_launch(const float *g_score, int G, int T, int k, float *rows, int64_t ld_rows,
                            cudaStream_t stream);
dsa_status_t cp_select_local_launch(const int32_t *sel, const int32_t *g_gidx, int G, int T, int k, const int32_t *lo,
                                    const int32_t *hi, int32_t *local, cudaStream_t stream);
dsa_status_t cp_merge_launch(const void *part_out, const float *part_lse, int G, int T, int H, int Dv, void *out,
                             float *lse, cudaStream_t stream);
dsa_status_t attn_simt_launch(const void *q, dsa_dtype_t dt, const void *kv, const void *v, int H, int Dqk, int Dv,
                              float scale, const int32_t *idx, int k, const dsa_batch_t *b, void *out, float *lse,
                              cudaStream_t stream);

static thread_local char g_err[512] = "";
static std::atomic<uint64_t> g_launches{0};

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

void set_error(const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
}

struct DeviceInfo {
  int num_sms = 0;
  int cc_major = 0, cc_minor = 0;
};
static DeviceInfo g_dev[kMaxDevices];
static std::mutex g_dev_mu;

// Current device's attributes; fails unless it is an sm_100 part (B200).
static dsa_status_t current_device(DeviceInfo *out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    set_error("no current CUDA device");
    return DSA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> g(g_dev_mu);
  if (g_dev[dev].num_sms == 0) {
    DeviceInfo d;
    if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
      set_error("cudaDeviceGetAttribute failed");
      return DSA_ERR_CUDA;
    }
    g_dev[dev] = d;
  }
  *out = g_dev[dev];
  if (out->cc_major != 10 || out->cc_minor != 0) {
    set_error("libdsa is built for sm_100a (B200); current device is sm_%d%d", out->cc_major, out->cc_minor);
    return DSA_ERR_UNSUPPORTED;
  }
  return DSA_OK;
}

#define CHECK_ARG(cond, ...)          \
  do {                                \
    if (!(cond)) {                    \
      set_error(__VA_ARGS__);         \
      return DSA_ERR_INVALID_ARG;     \
    }                                 \
  } while (0)

#define CHECK_SUP(cond, ...)          \
  do {                                \
    if (!(cond)) {                    \
      set_error(__VA_ARGS__);         \
      return DSA_ERR_UNSUPPORTED;     \
    }                                 \
  } while (0)

static dsa_status_t check_batch(const dsa_batch_t *b) {
  CHECK_ARG(b != nullptr, "batch descriptor is NULL");
  CHECK_ARG(b->num_seqs >= 1, "num_seqs must be >= 1 (got %d)", b->num_seqs);
  CHECK_SUP(b->page_size == 64, "page_size must be 64 (got %d)", b->page_size);
  CHECK_ARG(b->num_blocks >= 1 && b->max_blocks_per_seq >= 1, "num_blocks and max_blocks_per_seq must be >= 1");
  CHECK_ARG(b->block_table && b->seq_lens && b->cu_q, "block_table, seq_lens and cu_q are required");
  CHECK_ARG(b->total_q >= 0, "total_q must be >= 0");
  CHECK_ARG(b->max_seq_len >= 1 && b->max_q_per_seq >= 0, "max_seq_len must be >= 1");
  CHECK_ARG(b->max_q_per_seq <= b->max_seq_len, "max_q_per_seq (%d) exceeds max_seq_len (%d)", b->max_q_per_seq,
            b->max_seq_len);
  CHECK_ARG((int64_t)b->total_q <= (int64_t)b->num_seqs * b->max_q_per_seq,
            "total_q (%d) exceeds num_seqs * max_q_per_seq", b->total_q);
  CHECK_ARG((int64_t)b->max_seq_len <= (int64_t)b->max_blocks_per_seq * b->page_size,
            "max_seq_len (%d) exceeds max_blocks_per_seq * page_size", b->max_seq_len);
  return DSA_OK;
}

static dsa_status_t check_ws(void *ws, size_t ws_bytes, size_t need) {
  if (ws == nullptr || ws_bytes < need) {
    set_error("workspace of %zu bytes given, %zu needed", ws == nullptr ? (size_t)0 : ws_bytes, need);
    return DSA_ERR_WORKSPACE;
  }
  CHECK_ARG(((uintptr_t)ws & 255) == 0, "workspace must be 256-byte aligned");
  return DSA_OK;
}

static bool is_mla_attn(dsa_dtype_t dt, int H, int Dqk, int Dv, const void *v) {
  return dt == DSA_BF16 && H == 128 && Dqk == 576 && Dv == 512 && v == nullptr;
}
static bool is_f32_attn(dsa_dtype_t dt, int H, int Dqk, int Dv, const void *v) {
  return dt == DSA_F32 && H >= 1 && H <= 16 && Dqk >= 1 && Dqk <= 128 && Dv >= 1 && Dv <= 128 && v != nullptr;
}

// the fused scores + selection call: the indexer's workspace, then the rows' leading-digit histograms
static size_t indexer_topk_ws_bytes(const dsa_batch_t *b) {
  return indexer_workspace_bytes(b->num_seqs, b->total_q) + indexer_hist_bytes(b->total_q) +
         select_long_ws_bytes(b->total_q, b->max_seq_len);
}

static size_t attn_ws_bytes(const dsa_batch_t *b, int k, int H, int Dv, bool decode) {
  return H == 128 && Dv == 512 ? attn_workspace_bytes(b->total_q, k, decode) : kWsHeader;
}

}  // namespace dsa

using namespace dsa;

extern "C" {

const char *dsa_version(void) { return "0.1.0"; }

uint64_t dsa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char *dsa_last_error(void) { return g_err; }

const char *dsa_status_string(dsa_status_t s) {
  switch (s) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case DSA_ERR_WORKSPACE: return "workspace too small";
    case DSA_ERR_CUDA: return "CUDA error";
    case DSA_ERR_DEVICE_CHECK: return "device-side index check failed";
    case DSA_ERR_TIMEOUT: return "bounded device wait ran out";
  }
  return "unknown status";
}

dsa_status_t dsa_workspace_size(dsa_op_t op, const dsa_batch_t *b, int32_t k, int32_t H, int32_t Dv,
                                size_t *bytes) {
  if (bytes == nullptr) {
    set_error("bytes is NULL");
    return DSA_ERR_INVALID_ARG;
  }
  dsa_status_t st = check_batch(b);
  if (st != DSA_OK) return st;
  switch (op) {
    case DSA_OP_INDEXER: *bytes = indexer_workspace_bytes(b->num_seqs, b->total_q); return DSA_OK;
    case DSA_OP_TOPK: *bytes = topk_workspace_bytes(b->total_q, b->max_seq_len); return DSA_OK;
    case DSA_OP_ATTN_PREFILL: *bytes = attn_ws_bytes(b, k, H, Dv, false); return DSA_OK;
    case DSA_OP_ATTN_DECODE: *bytes = attn_ws_bytes(b, k, H, Dv, true); return DSA_OK;
    case DSA_OP_CACHE_APPEND: *bytes = kWsHeader; return DSA_OK;
    case DSA_OP_INDEXER_TOPK: *bytes = indexer_topk_ws_bytes(b); return DSA_OK;
  }
  set_error("unknown op %d", (int)op);
  return DSA_ERR_INVALID_ARG;
}

dsa_status_t dsa_indexer_scores(const void *q_idx, dsa_dtype_t q_dt, const float *w, const void *k_idx_pool,
                                dsa_dtype_t k_dt, const float *k_scale_pool, int32_t Hi, int32_t Di,
                                const dsa_batch_t *b, float *scores, int64_t ld_scores, void *ws, size_t ws_bytes,
                                void *stream) {
  dsa_status_t st = check_batch(b);
  if (st != DSA_OK) return st;
  if (b->total_q == 0) return DSA_OK;   // empty batch: nothing to enqueue, data pointers may be NULL
  CHECK_ARG(q_idx && w && k_idx_pool && scores, "q_idx, w, k_idx_pool and scores are required");
  CHECK_ARG(q_dt == k_dt, "query and key dtypes differ");
  CHECK_ARG(ld_scores >= b->max_seq_len && ld_scores % 4 == 0,
            "ld_scores (%lld) must be >= max_seq_len and a multiple of 4", (long long)ld_scores);
  CHECK_ARG(((uintptr_t)scores & 15) == 0, "scores must be 16-byte aligned");
  const bool mla = q_dt == DSA_FP8_E4M3 && Hi == 64 && Di == 128;
  const bool f32 = q_dt == DSA_F32 && Hi >= 1 && Hi <= 16 && Di >= 1 && Di <= 128;
  CHECK_SUP(mla || f32, "indexer supports e4m3 with Hi=64, Di=128 or f32 with Hi<=16, Di<=128");
  CHECK_ARG(mla ? k_scale_pool != nullptr : k_scale_pool == nullptr,
            "k_scale_pool is required for e4m3 keys and must be NULL for f32 keys");
  CHECK_ARG((((uintptr_t)q_idx | (uintptr_t)w | (uintptr_t)k_idx_pool | (uintptr_t)k_scale_pool) & 15) == 0,
            "q_idx, w, k_idx_pool and k_scale_pool must be 16-byte aligned");
  if ((st = check_ws(ws, ws_bytes, indexer_workspace_bytes(b->num_seqs, b->total_q))) != DSA_OK) return st;
  DeviceInfo dev;
  if ((st = current_device(&dev)) != DSA_OK) return st;
  if (mla)
    return indexer_tc_launch((const uint8_t *)q_idx, w, (const uint8_t *)k_idx_pool, k_scale_pool, b, scores,
                             ld_scores, ws, (cudaStream_t)stream, dev.num_sms, nullptr, nullptr);
  return indexer_simt_launch(q_idx, q_dt, w, k_idx_pool, k_scale_pool, Hi, Di, b, scores, ld_scores,
                             (cudaStream_t)stream);
}

dsa_status_t dsa_topk(const float *scores, int64_t ld_scores, const dsa_batch_t *b, int32_t k, int32_t *idx,
                      void *ws, size_t ws_bytes, void *stream) {
  dsa_status_t st = check_batch(b);
  if (st != DSA_OK) return st;
  if (b->total_q == 0) return DSA_OK;   // empty batch: nothing to enqueue, data pointers may be NULL
  CHECK_ARG(scores && idx, "scores and idx are required");
  CHECK_SUP(k >= 1 && k <= 16384, "k must be in [1, 16384] (got %d)", k);
  CHECK_ARG(ld_scores >= b->max_seq_len && ld_scores % 4 == 0,
            "ld_scores (%lld) must be >= max_seq_len and a multiple of 4", (long long)ld_scores);
  CHECK_ARG(((uintptr_t)scores & 15) == 0, "scores must be 16-byte aligned");
  if ((st = check_ws(ws, ws_bytes, topk_workspace_bytes(b->total_q, b->max_seq_len))) != DSA_OK) return st;
  DeviceInfo dev;
  if ((st = current_device(&dev)) != DSA_OK) return st;
  return topk_launch(scores, ld_scores, b, k, idx, ws, (cudaStream_t)stream, dev.num_sms);
}

dsa_status_t dsa_indexer_topk(const void *q_idx, dsa_dtype_t q_dt, const float *w, const void *k_idx_pool,
                              dsa_dtype_t k_dt, const float *k_scale_pool, int32_t Hi, int32_t Di, const dsa_batch_t *b,
                              int32_t k, float *scores, int64_t ld_scores, int32_t *idx, void *ws, size_t ws_bytes,
                              void *stream) {
  dsa_status_t st = check_batch(b);
  if (st != DSA_OK) return st;
  if (b->total_q == 0) return DSA_OK;   // empty batch: nothing to enqueue, data pointers may be NULL
  CHECK_ARG(q_idx && w && k_idx_pool && scores && idx, "q_idx, w, k_idx_pool, scores and idx are required");
  CHECK_ARG(q_dt == k_dt, "query and key dtypes differ");
  CHECK_SUP(k >= 1 && k <= 16384, "k must be in [1, 16384] (got %d)", k);
  CHECK_ARG(ld_scores >= b->max_seq_len && ld_scores % 4 == 0,
            "ld_scores (%lld) must be >= max_seq_len and a multiple of 4", (long long)ld_scores);
  CHECK_ARG(((uintptr_t)scores & 15) == 0, "scores must be 16-byte aligned");
  const bool mla = q_dt == DSA_FP8_E4M3 && Hi == 64 && Di == 128;
  const bool f32 = q_dt == DSA_F32 && Hi >= 1 && Hi <= 16 && Di >= 1 && Di <= 128;
  CHECK_SUP(mla || f32, "indexer supports e4m3 with Hi=64, Di=128 or f32 with Hi<=16, Di<=128");
  CHECK_ARG(mla ? k_scale_pool != nullptr : k_scale_pool == nullptr,
            "k_scale_pool is required for e4m3 keys and must be NULL for f32 keys");
  CHECK_ARG((((uintptr_t)q_idx | (uintptr_t)w | (uintptr_t)k_idx_pool | (uintptr_t)k_scale_pool) & 15) == 0,
            "q_idx, w, k_idx_pool and k_scale_pool must be 16-byte aligned");
  if ((st = check_ws(ws, ws_bytes, indexer_topk_ws_bytes(b))) != DSA_OK) return st;
  DeviceInfo dev;
  if ((st = current_device(&dev)) != DSA_OK) return st;
  if (mla) {
    uint32_t *hist = (uint32_t *)((char *)ws + indexer_workspace_bytes(b->num_seqs, b->total_q));
    st = indexer_tc_launch((const uint8_t *)q_idx, w, (const uint8_t *)k_idx_pool, k_scale_pool, b, scores, ld_scores,
                           ws, (cudaStream_t)stream, dev.num_sms, nullptr, hist);
    if (st != DSA_OK) return st;
    void *long_ws = select_long_ws_bytes(b->total_q, b->max_seq_len) > 0
                        ? (void *)((char *)hist + indexer_hist_bytes(b->total_q))
                        : nullptr;
    return select_launch(scores, ld_scores, b, k, idx, hist, (uint32_t *)ws, long_ws, (cudaStream_t)stream,
                         dev.num_sms);
  }
  // fp32 indexer (CUDA cores): the selection counts the leading digit itself
  st = indexer_simt_launch(q_idx, q_dt, w, k_idx_pool, k_scale_pool, Hi, Di, b, scores, ld_scores, (cudaStream_t)stream);
  if (st != DSA_OK) return st;
  return select_launch(scores, ld_scores, b, k, idx, nullptr, (uint32_t *)ws, nullptr, (cudaStream_t)stream,
                       dev.num_sms);
}

dsa_status_t dsa_topk_noalloc(const float *scores, int64_t ld_scores, const dsa_batch_t *b, int32_t k,
                              int32_t *idx, void *stream) {
  dsa_status_t st = check_batch(b);
  if (st != DSA_OK) return st;
  if (b->total_q == 0) return DSA_OK;   // empty batch: nothing to enqueue, data pointers may be NULL
  CHECK_ARG(scores && idx, "scores and idx are required");
  CHECK_SUP(k >= 1 && k <= 16384, "k must be in [1, 16384] (got %d)", k);
  CHECK_ARG(ld_scores >= b->max_seq_len && ld_scores % 4 == 0,
            "ld_scores (%lld) must be >= max_seq_len and a multiple of 4", (long long)ld_scores);
  CHECK_ARG(((uintptr_t)scores & 15) == 0, "scores must be 16-byte aligned");
  DeviceInfo dev;
  if ((st = current_device(&dev)) != DSA_OK) return st;
  return topk_noalloc_launch(scores, ld_scores, b, k, idx, (cudaStream_t)stream, dev.num_sms);
}

static dsa_status_t attn_common(bool decode, const void *q, dsa_dtype_t dt, const void *kv_pool, const void *v_pool,
                                int32_t H, int32_t Dqk, int32_t Dv, float softmax_scale, const int32_t *idx,
                                int32_t k, const dsa_batch_t *b, void *out, float *lse, void *ws, size_t ws_bytes,
                                void *stream) {
  dsa_status_t st = check_batch(b);
  if (st != DSA_OK) return st;
  if (b->total_q == 0) return DSA_OK;   // empty batch: nothing to enqueue, data pointers may be NULL
  CHECK_ARG(q && kv_pool && idx && out, "q, kv_pool, idx and out are required");
  CHECK_ARG(k >= 1, "k must be >= 1");
  CHECK_ARG(softmax_scale == softmax_scale && softmax_scale > 0.f && softmax_scale < 1e30f,
            "softmax_scale must be finite and positive");
  const bool mla = is_mla_attn(dt, H, Dqk, Dv, v_pool);
  const bool f32 = is_f32_attn(dt, H, Dqk, Dv, v_pool);
  CHECK_SUP(mla || f32,
            "attention supports bf16 MLA (H=128, Dqk=576, Dv=512, V inside the latent row) or f32 with "
            "H<=16, Dqk<=128, Dv<=128 and a separate V cache");
  if (decode) CHECK_ARG(b->total_q == b->num_seqs && b->max_q_per_seq == 1,
                        "decode needs exactly one query row per sequence");
  CHECK_ARG((((uintptr_t)q | (uintptr_t)kv_pool | (uintptr_t)out) & 15) == 0,
            "q, kv_pool and out must be 16-byte aligned");
  if ((st = check_ws(ws, ws_bytes, attn_ws_bytes(b, k, H, Dv, decode))) != DSA_OK) return st;
  DeviceInfo dev;
  if ((st = current_device(&dev)) != DSA_OK) return st;
  if (mla)
    return attn_mla_launch(q, kv_pool, idx, k, softmax_scale, b, out, lse, ws, decode, (cudaStream_t)stream,
                           dev.num_sms);
  return attn_simt_launch(q, dt, kv_pool, v_pool, H, Dqk, Dv, softmax_scale, idx, k, b, out, lse,
                          (cudaStream_t)stream);
}

dsa_status_t dsa_sparse_attn_prefill(const void *q, dsa_dtype_t dt, const void *kv_pool, const void *v_pool, int32_t H,
                                     int32_t Dqk, int32_t Dv, float softmax_scale, const int32_t *idx, int32_t k,
                                     const dsa_batch_t *b, void *out, float *lse, void *ws, size_t ws_bytes,
                                     void *stream) {
  return attn_common(false, q, dt, kv_pool, v_pool, H, Dqk, Dv, softmax_scale, idx, k, b, out, lse, ws, ws_bytes,
                     stream);
}

dsa_status_t dsa_sparse_attn_decode(const void *q, dsa_dtype_t dt, const void *kv_pool, const void *v_pool, int32_t H,
                                    int32_t Dqk, int32_t Dv, float softmax_scale, const int32_t *idx, int32_t k,
                                    const dsa_batch_t *b, void *out, float *lse, void *ws, size_t ws_bytes,
                                    void *stream) {
  return attn_common(true, q, dt, kv_pool, v_pool, H, Dqk, Dv, softmax_scale, idx, k, b, out, lse, ws, ws_bytes,
                     stream);
}

dsa_status_t dsa_cache_append(const void *kv_new, dsa_dtype_t kv_dt, const void *k_new, dsa_dtype_t k_dt, int32_t Dqk,
                              int32_t Di, const dsa_batch_t *b, void *kv_pool, void *k_idx_pool, float *k_scale_pool,
                              void *ws, size_t ws_bytes, void *stream) {
  dsa_status_t st = check_batch(b);
  if (st != DSA_OK) return st;
  if (b->total_q == 0) return DSA_OK;   // empty batch: nothing to enqueue, data pointers may be NULL
  CHECK_ARG(kv_new && k_new && kv_pool && k_idx_pool && k_scale_pool,
            "kv_new, k_new, kv_pool, k_idx_pool and k_scale_pool are required");
  CHECK_SUP(kv_dt == DSA_BF16 && Dqk == 576 && Di == 128 && (k_dt == DSA_F32 || k_dt == DSA_BF16),
            "cache append supports bf16 latent rows of 576 and f32 or bf16 indexer keys of 128");
  CHECK_ARG((((uintptr_t)kv_new | (uintptr_t)k_new | (uintptr_t)kv_pool | (uintptr_t)k_idx_pool) & 15) == 0 &&
                ((uintptr_t)k_scale_pool & 3) == 0,
            "kv_new, k_new, kv_pool and k_idx_pool must be 16-byte aligned, k_scale_pool 4-byte aligned");
  if ((st = check_ws(ws, ws_bytes, kWsHeader)) != DSA_OK) return st;
  DeviceInfo dev;
  if ((st = current_device(&dev)) != DSA_OK) return st;
  return cache_append_launch(kv_new, k_new, k_dt == DSA_BF16, b, kv_pool, k_idx_pool, k_scale_pool, ws,
                             (cudaStream_t)stream);
}

dsa_status_t dsa_selftest_wait_timeout(uint64_t budget_cycles, void *ws, size_t ws_bytes, void *stream) {
  CHECK_ARG(budget_cycles >= 1 && budget_cycles <= 4000000000ull,
            "budget_cycles must be in [1, 4e9] (got %llu)", (unsigned long long)budget_cycles);
  dsa_status_t st = check_ws(ws, ws_bytes, kWsHeader);
  if (st != DSA_OK) return st;
  DeviceInfo dev;
  if ((st = current_device(&dev)) != DSA_OK) return st;
  return selftest_wait_launch((long long)budget_cycles, ws, (cudaStream_t)stream);
}

dsa_status_t dsa_indexer_scores_append(const void *kv_new, dsa_dtype_t kv_dt, const void *k_new, dsa_dtype_t k_new_dt,
                                       void *kv_pool, const void *q_idx, dsa_dtype_t q_dt, const float *w,
                                       void *k_idx_pool, dsa_dtype_t k_dt, float *k_scale_pool, int32_t Hi, int32_t Di,
                                       const dsa_batch_t *b, float *scores, int64_t ld_scores, void *ws,
                                       size_t ws_bytes, void *stream) {
  dsa_status_t st = check_batch(b);
  if (st != DSA_OK) return st;
  if (b->total_q == 0) return DSA_OK;   // empty batch: nothing to enqueue, data pointers may be NULL
  CHECK_ARG(kv_new && k_new && kv_pool && q_idx && w && k_idx_pool && k_scale_pool && scores,
            "kv_new, k_new, kv_pool, q_idx, w, k_idx_pool, k_scale_pool and scores are required");
  CHECK_SUP(kv_dt == DSA_BF16 && (k_new_dt == DSA_F32 || k_new_dt == DSA_BF16) && q_dt == DSA_FP8_E4M3 &&
                k_dt == DSA_FP8_E4M3 && Hi == 64 && Di == 128,
            "the fused append supports the MLA path: bf16 latent rows, f32 or bf16 new keys, e4m3 indexer 64 x 128");
  CHECK_ARG(ld_scores >= b->max_seq_len && ld_scores % 4 == 0,
            "ld_scores (%lld) must be >= max_seq_len and a multiple of 4", (long long)ld_scores);
  CHECK_ARG((((uintptr_t)kv_new | (uintptr_t)k_new | (uintptr_t)kv_pool | (uintptr_t)q_idx | (uintptr_t)w |
              (uintptr_t)k_idx_pool | (uintptr_t)k_scale_pool | (uintptr_t)scores) & 15) == 0,
            "every buffer must be 16-byte aligned");
  if ((st = check_ws(ws, ws_bytes, indexer_workspace_bytes(b->num_seqs, b->total_q))) != DSA_OK) return st;
  DeviceInfo dev;
  if ((st = current_device(&dev)) != DSA_OK) return st;
  const AppendArgs app{(const uint4 *)kv_new, k_new, k_new_dt == DSA_BF16 ? 1 : 0, (uint4 *)kv_pool,
                       (uint32_t *)k_idx_pool, k_scale_pool};
  return indexer_tc_launch((const uint8_t *)q_idx, w, (const uint8_t *)k_idx_pool, k_scale_pool, b, scores, ld_scores,
                           ws, (cudaStream_t)stream, dev.num_sms, &app, nullptr);
}

dsa_status_t dsa_reuse_candidates(const int32_t *prev_idx, int32_t k, const int32_t *prev_lens, int32_t max_new,
                                  const dsa_batch_t *b, int32_t *cand, void *ws, size_t ws_bytes, void *stream) {
  dsa_status_t st = check_batch(b);
  if (st != DSA_OK) return st;
  if (b->total_q == 0) return DSA_OK;   // empty batch: nothing to enqueue, data pointers may be NULL
  CHECK_ARG(b->total_q == b->num_seqs && b->max_q_per_seq == 1, "index reuse takes decode batches (one row per sequence)");
  CHECK_ARG(k >= 1 && max_new >= 0 && (int64_t)k + max_new <= 1 << 24, "k >= 1, max_new >= 0, k + max_new <= 2^24");
  CHECK_ARG(prev_idx && prev_lens && cand, "prev_idx, prev_lens and cand are required");
  if ((st = check_ws(ws, ws_bytes, kWsHeader)) != DSA_OK) return st;
  DeviceInfo dev;
  if ((st = current_device(&dev)) != DSA_OK) return st;
  return reuse_candidates_launch(prev_idx, k, prev_lens, max_new, b, cand, ws, (cudaStream_t)stream);
}

dsa_status_t dsa_indexer_scores_at(const void *q_idx, dsa_dtype_t q_dt, const float *w, const void *k_idx_pool,
                                   dsa_dtype_t k_dt, const float *k_scale_pool, int32_t Hi, int32_t Di,
                                   const dsa_batch_t *b, const int32_t *cand, int32_t m, float *cand_scores, void *ws,
                                   size_t ws_bytes, void *stream) {
  dsa_status_t st = check_batch(b);
  if (st != DSA_OK) return st;
  if (b->total_q == 0) return DSA_OK;   // empty batch: nothing to enqueue, data pointers may be NULL
  CHECK_SUP(q_dt == DSA_FP8_E4M3 && k_dt == DSA_FP8_E4M3 && Hi == 64 && Di == 128,
            "scores at positions support the e4m3 indexer with Hi = 64, Di = 128");
  CHECK_ARG(m >= 1, "m must be >= 1");
  CHECK_ARG(q_idx && w && k_idx_pool && k_scale_pool && cand && cand_scores, "every pointer is required");
  CHECK_ARG(((uintptr_t)k_idx_pool & 15) == 0, "k_idx_pool must be 16-byte aligned");
  if ((st = check_ws(ws, ws_bytes, kWsHeader)) != DSA_OK) return st;
  DeviceInfo dev;
  if ((st = current_device(&dev)) != DSA_OK) return st;
  return indexer_at_launch((const uint8_t *)q_idx, w, (const uint8_t *)k_idx_pool, k_scale_pool, b, cand, m, cand_scores,
                           ws, (cudaStream_t)stream);
}

dsa_status_t dsa_gather_positions(const int32_t *sel, int32_t k, const int32_t *cand, int32_t m, int32_t T,
                                  int32_t *idx, void *stream) {
  CHECK_ARG(T >= 0 && k >= 1 && m >= 1, "T >= 0, k and m >= 1");
  if (T == 0) return DSA_OK;
  CHECK_ARG(sel && cand && idx, "sel, cand and idx are required");
  DeviceInfo dev;
  dsa_status_t st;
  if ((st = current_device(&dev)) != DSA_OK) return st;
  return gather_positions_launch(sel, k, cand, m, T, idx, (cudaStream_t)stream);
}

dsa_status_t dsa_block_scores(const float *scores, int64_t ld_scores, const dsa_batch_t *b, float *blk_scores,
                              int64_t ld_blk, int32_t *blk_lens, void *stream) {
  dsa_status_t st = check_batch(b);
  if (st != DSA_OK) return st;
  if (b->total_q == 0) return DSA_OK;   // empty batch: nothing to enqueue, data pointers may be NULL
  CHECK_ARG(scores && blk_scores && blk_lens, "scores, blk_scores and blk_lens are required");
  CHECK_ARG(ld_scores >= b->max_seq_len, "ld_scores (%lld) must be >= max_seq_len", (long long)ld_scores);
  CHECK_ARG(ld_blk >= (b->max_seq_len + b->page_size - 1) / b->page_size && ld_blk % 4 == 0,
            "ld_blk (%lld) must be >= the pages of max_seq_len and a multiple of 4", (long long)ld_blk);
  CHECK_ARG(((uintptr_t)blk_scores & 15) == 0, "blk_scores must be 16-byte aligned");
  DeviceInfo dev;
  if ((st = current_device(&dev)) != DSA_OK) return st;
  return block_scores_launch(scores, ld_scores, b, blk_scores, ld_blk, blk_lens, (cudaStream_t)stream);
}

dsa_status_t dsa_expand_blocks(const int32_t *blk_idx, int32_t kb, const dsa_batch_t *b, int32_t *idx, void *stream) {
  dsa_status_t st = check_batch(b);
  if (st != DSA_OK) return st;
  if (b->total_q == 0) return DSA_OK;   // empty batch: nothing to enqueue, data pointers may be NULL
  CHECK_ARG(kb >= 1 && (int64_t)kb * b->page_size <= 1 << 20, "kb must be >= 1 with kb * page_size <= 2^20");
  CHECK_ARG(blk_idx && idx, "blk_idx and idx are required");
  DeviceInfo dev;
  if ((st = current_device(&dev)) != DSA_OK) return st;
  return expand_blocks_launch(blk_idx, kb, b, idx, (cudaStream_t)stream);
}

dsa_status_t dsa_cp_candidates(const float *scores, int64_t ld_scores, const int32_t *idx, int32_t T, int32_t k,
                               const int32_t *offsets, float *cand_score, int32_t *cand_gidx, void *stream) {
  CHECK_ARG(T >= 0 && k >= 1 && ld_scores >= 1, "T must be >= 0, k and ld_scores >= 1");
  if (T == 0) return DSA_OK;
  CHECK_ARG(scores && idx && offsets && cand_score && cand_gidx, "scores, idx, offsets, cand_score and cand_gidx are required");
  DeviceInfo dev;
  dsa_status_t st;
  if ((st = current_device(&dev)) != DSA_OK) return st;
  return cp_candidates_launch(scores, ld_scores, idx, T, k, offsets, cand_score, cand_gidx, (cudaStream_t)stream);
}

dsa_status_t dsa_cp_rows(const float *g_score, int32_t G, int32_t T, int32_t k, float *rows, int64_t ld_rows,
                         void *stream) {
  CHECK_ARG(G >= 1 && T >= 0 && k >= 1, "G and k must be >= 1, T >= 0");
  CHECK_ARG(ld_rows >= (int64_t)G * k, "ld_rows (%lld) must be >= G * k", (long long)ld_rows);
  if (T == 0) return DSA_OK;
  CHECK_ARG(g_score && rows, "g_score and rows are required");
  DeviceInfo dev;
  dsa_status_t st;
  if ((st = current_device(&dev)) != DSA_OK) return st;
  return cp_rows_launch(g_score, G, T, k, rows, ld_rows, (cudaStream_t)stream);
}

dsa_status_t dsa_cp_select_local(const int32_t *sel, const int32_t *g_gidx, int32_t G, int32_t T, int32_t k,
                                 const int32_t *lo, const int32_t *hi, int32_t *local_idx, void *stream) {
  CHECK_ARG(G >= 1 && T >= 0 && k >= 1, "G and k must be >= 1, T >= 0");
  CHECK_ARG((int64_t)G * k <= 0x7FFFFFFF, "G * k must fit in int32");
  if (T == 0) return DSA_OK;
  CHECK_ARG(sel && g_gidx && lo && hi && local_idx, "sel, g_gidx, lo, hi and local_idx are required");
  DeviceInfo dev;
  dsa_status_t st;
  if ((st = current_device(&dev)) != DSA_OK) return st;
  return cp_select_local_launch(sel, g_gidx, G, T, k, lo, hi, local_idx, (cudaStream_t)stream);
}

dsa_status_t dsa_cp_merge(const void *part_out, dsa_dtype_t dt, const float *part_lse, int32_t G, int32_t T, int32_t H,
                          int32_t Dv, void *out, float *lse, void *stream) {
  CHECK_ARG(G >= 1 && T >= 0 && H >= 1 && H <= 65535, "G and H must be >= 1 (H <= 65535), T >= 0");
  CHECK_SUP(dt == DSA_BF16 && Dv >= 4 && Dv <= 1024 && Dv % 4 == 0,
            "merge supports bf16 partial outputs with Dv a multiple of 4 in [4, 1024]");
  if (T == 0) return DSA_OK;
  CHECK_ARG(part_out && part_lse && out, "part_out, part_lse and out are required");
  CHECK_ARG((((uintptr_t)part_out | (uintptr_t)out) & 7) == 0, "part_out and out must be 8-byte aligned");
  DeviceInfo dev;
  dsa_status_t st;
  if ((st = current_device(&dev)) != DSA_OK) return st;
  return cp_merge_launch(part_out, part_lse, G, T, H, Dv, out, lse, (cudaStream_t)stream);
}

dsa_status_t dsa_read_device_status(void *ws, void *stream) {
  if (ws == nullptr) {
    set_error("workspace is NULL");
    return DSA_ERR_INVALID_ARG;
  }
  uint32_t word = 0;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess ||
      cudaMemcpy(&word, ws, 4, cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemset(ws, 0, 4) != cudaSuccess) {
    set_error("reading the device status word failed: %s", cudaGetErrorString(cudaGetLastError()));
    return DSA_ERR_CUDA;
  }
  if (word & kStatusTimeout) {
    set_error("a bounded device wait ran out (status 0x%x)", word);
    return DSA_ERR_TIMEOUT;
  }
  if (word & kStatusBadIndex) {
    set_error("a kernel met an out-of-range block id or index (status 0x%x)", word);
    return DSA_ERR_DEVICE_CHECK;
  }
  return DSA_OK;
}

}  // extern "C"
