// kin_api.cu -- the extern "C" boundary of libkin.so: argument checks,
// workspace layout, launch-shape heuristics and launches.
// Semantics of every call are documented in include/kin.h.
#include <atomic>
#include <mutex>
#include <cmath>

#include "kin_internal.cuh"

#define KIN_EXPORT extern "C" __attribute__((visibility("default")))

namespace {

using namespace kin;

constexpr int kTargetSMs = 148;  // B200 SM count, used only to shape grids
constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

int nbcap_of(const kin_dims& d) { return (d.max_seq_len + d.block_size - 1) / d.block_size; }
int pairs_of(const kin_dims& d) { return d.batch * d.num_kv_heads; }

#ifndef KIN_ATTN_CHUNK_TOKENS
#define KIN_ATTN_CHUNK_TOKENS 768
#endif

// Kept blocks per attention CTA: KIN_ATTN_CHUNK_TOKENS tokens (768 -> 384 KB
// of K+V), fewer when the grid would hold fewer than 2 CTAs per SM.
int attn_chunk_blocks(const kin_dims& d, int k) {
  const int k_eff = k < nbcap_of(d) ? k : nbcap_of(d);
  const int by_tokens = KIN_ATTN_CHUNK_TOKENS / d.block_size > 0 ? KIN_ATTN_CHUNK_TOKENS / d.block_size : 1;
  const int64_t by_grid = (int64_t)k_eff * pairs_of(d) / (2 * kTargetSMs);
  int ch = by_tokens;
  if (by_grid < ch) ch = by_grid > 0 ? (int)by_grid : 1;
  const int cap = kMaxItemTiles / (d.block_size / kTileTokens);  // tiles per item <= 64
  return ch < cap ? ch : cap;
}

int attn_max_chunks(const kin_dims& d, int k) {
  const int k_eff = k < nbcap_of(d) ? k : nbcap_of(d);
  const int ch = attn_chunk_blocks(d, k);
  return (k_eff + ch - 1) / ch;
}

struct WsLayout {
  size_t attn_counters, scores, partials, total;
};

WsLayout ws_layout(const kin_dims& d, int k) {
  WsLayout w;
  const size_t pairs = (size_t)pairs_of(d);
  const size_t g = (size_t)(d.num_q_heads / d.num_kv_heads);
  size_t off = 0;
  w.attn_counters = off;
  off = align_up(off + pairs * sizeof(uint32_t));
  w.scores = off;
  off = align_up(off + pairs * (size_t)nbcap_of(d) * sizeof(float));
  w.partials = off;
  off = align_up(off + pairs * (size_t)attn_max_chunks(d, k) * g * kPartStride * sizeof(float));
  w.total = off;
  return w;
}

kin_status check_ws(const kin_dims& d, int k, void* ws, size_t ws_bytes, WsLayout* out) {
  *out = ws_layout(d, k);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0) return KIN_ERR_WORKSPACE;
  if (ws_bytes < out->total) return KIN_ERR_WORKSPACE;
  return KIN_OK;
}

kin_status from_cuda(cudaError_t e) { return e == cudaSuccess ? KIN_OK : KIN_ERR_CUDA; }

PageTable contiguous() {
  PageTable pt;
  pt.table = nullptr;
  pt.max_blocks = 0;
  pt.num_pages = 0;
  return pt;
}

// A page pool [num_pages][Hkv][bs][D] bf16 and its table [B][ceil(Lcap / bs)].
kin_status check_pages(const kin_dims& d, const void* pool, int32_t num_pages, const int32_t* table,
                       PageTable* out) {
  if (!pool || !table || num_pages < 1) return KIN_ERR_INVALID_ARG;
  if (!aligned16(pool)) return KIN_ERR_INVALID_ARG;
  out->table = table;
  out->max_blocks = nbcap_of(d);
  out->num_pages = num_pages;
  return KIN_OK;
}

}  // namespace

namespace kin {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

kin_status check_dims(const kin_dims* d) {
  if (!d) return KIN_ERR_INVALID_ARG;
  if (d->batch < 1 || d->num_kv_heads < 1 || d->num_q_heads < 1 || d->max_seq_len < 1)
    return KIN_ERR_INVALID_ARG;
  if (d->num_q_heads % d->num_kv_heads != 0) return KIN_ERR_INVALID_ARG;
  if (d->head_dim != kHeadDim) return KIN_ERR_INVALID_ARG;
  const int bs = d->block_size;
  if (bs != 16 && bs != 32 && bs != 64 && bs != 128) return KIN_ERR_INVALID_ARG;
  if (d->num_q_heads / d->num_kv_heads > kMaxGroup) return KIN_ERR_CAPACITY;
  if ((d->max_seq_len + bs - 1) / bs > kMaxBlocksPerSeq) return KIN_ERR_CAPACITY;
  if ((int64_t)d->batch * d->num_kv_heads * d->max_seq_len >= (int64_t)1 << 31) return KIN_ERR_CAPACITY;
  return KIN_OK;
}

constexpr int kMaxDevices = 64;

int device_sm_count() {
  // per device, written once with the same value by whichever thread gets there first
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return kTargetSMs;
  int n = dev < kMaxDevices ? cache[dev].load(std::memory_order_relaxed) : 0;
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) return kTargetSMs;
    if (dev < kMaxDevices) cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

cudaError_t ensure_smem_limit(const void* kernel, int slot, size_t bytes) {
  // slot: a small per-kernel index.  The kernel's limit only ever grows: it
  // is read and raised under one lock, so a thread never lowers it under
  // another thread's launch, and the cache (the limit last seen, per slot and
  // device) never exceeds the limit in force.
  // slots in use: 0, 2, 3, then 8, 9, 10, then 12, 13, 14 block top-k (256,
  // 512, 1024 threads; plain, refining, refining per page), 1 attention, 4
  // means update, 5 token top-k, 6 token logits
  static std::atomic<size_t> done[16][kMaxDevices];
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool cached = dev >= 0 && dev < kMaxDevices && slot >= 0 && slot < 16;
  if (cached && done[slot][dev].load(std::memory_order_acquire) >= bytes) return cudaSuccess;
  std::lock_guard<std::mutex> lock(mu);
  cudaFuncAttributes attr;
  e = cudaFuncGetAttributes(&attr, kernel);
  if (e != cudaSuccess) return e;
  size_t limit = attr.maxDynamicSharedSizeBytes > 0 ? (size_t)attr.maxDynamicSharedSizeBytes : 0;
  if (limit < bytes) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    limit = bytes;
  }
  if (cached) done[slot][dev].store(limit, std::memory_order_release);
  return cudaSuccess;
}

}  // namespace kin

KIN_EXPORT const char* kin_status_string(kin_status s) {
  switch (s) {
    case KIN_OK: return "KIN_OK";
    case KIN_ERR_INVALID_ARG: return "KIN_ERR_INVALID_ARG";
    case KIN_ERR_WORKSPACE: return "KIN_ERR_WORKSPACE";
    case KIN_ERR_CAPACITY: return "KIN_ERR_CAPACITY";
    case KIN_ERR_CUDA: return "KIN_ERR_CUDA";
    case KIN_ERR_DEVICE_DATA: return "KIN_ERR_DEVICE_DATA";
    case KIN_ERR_TIMEOUT: return "KIN_ERR_TIMEOUT";
  }
  return "KIN_ERR_UNKNOWN";
}

KIN_EXPORT size_t kin_workspace_bytes(const kin_dims* dims, int32_t k_blocks) {
  if (check_dims(dims) != KIN_OK || k_blocks < 2) return 0;
  return ws_layout(*dims, k_blocks).total;
}

KIN_EXPORT size_t kin_dual_means_bytes(const kin_dims* dims) {
  if (check_dims(dims) != KIN_OK) return 0;
  const int64_t rows = (int64_t)dims->batch * dims->num_kv_heads * nbcap_of(*dims);
  return (size_t)rows * (kHeadDim * 4 + kHeadDim * 2 + 4);
}

KIN_EXPORT size_t kin_dual_page_means_bytes(const kin_dims* dims, int32_t num_pages) {
  if (check_dims(dims) != KIN_OK || num_pages < 1) return 0;
  const int64_t rows = (int64_t)num_pages * dims->num_kv_heads;
  return (size_t)rows * (kHeadDim * 4 + kHeadDim * 2 + 4);
}

namespace {

kin_status means_build(const kin_dims* dims, const void* k_rows, const PageTable& pt, const int32_t* seq_lens,
                       void* block_means, int means_bf16, int32_t* dev_status, void* stream, int per_page = 0) {
  MeansBuildParams p{};  // every field not set below is zero or null
  p.means_per_page = per_page;
  p.k_cache = static_cast<const __nv_bfloat16*>(k_rows);
  p.seq_lens = seq_lens;
  p.means = block_means;
  p.means_bf16 = means_bf16;
  p.dev_status = dev_status;
  p.pages = pt;
  p.B = dims->batch;
  p.Hkv = dims->num_kv_heads;
  p.Lcap = dims->max_seq_len;
  p.bs = dims->block_size;
  p.nbcap = nbcap_of(*dims);
  p.mean_rows = per_page ? (int64_t)pt.num_pages * p.Hkv : (int64_t)p.B * p.Hkv * p.nbcap;
  return from_cuda(launch_means_build(p, static_cast<cudaStream_t>(stream)));
}

kin_status means_update(const kin_dims* dims, void* k_rows, void* v_rows, const PageTable& pt,
                        void* block_means, int means_bf16, int32_t* seq_lens, const void* k_new,
                        const void* v_new, int32_t n_new, int32_t* dev_status, void* stream, int per_page = 0) {
  MeansUpdateParams p{};
  p.means_per_page = per_page;
  p.k_cache = static_cast<__nv_bfloat16*>(k_rows);
  p.v_cache = static_cast<__nv_bfloat16*>(v_rows);
  p.means = block_means;
  p.means_bf16 = means_bf16;
  p.seq_lens = seq_lens;
  p.k_new = static_cast<const __nv_bfloat16*>(k_new);
  p.v_new = static_cast<const __nv_bfloat16*>(v_new);
  p.dev_status = dev_status;
  p.pages = pt;
  p.B = dims->batch;
  p.Hkv = dims->num_kv_heads;
  p.Lcap = dims->max_seq_len;
  p.bs = dims->block_size;
  p.nbcap = nbcap_of(*dims);
  p.mean_rows = per_page ? (int64_t)pt.num_pages * p.Hkv : (int64_t)p.B * p.Hkv * p.nbcap;
  p.n_new = n_new;
  return from_cuda(launch_means_update(p, static_cast<cudaStream_t>(stream)));
}

kin_status check_update_count(const kin_dims* dims, int32_t n_new) {
  if (n_new < 0) return KIN_ERR_INVALID_ARG;
  if (n_new > dims->max_seq_len) return KIN_ERR_CAPACITY;
  return KIN_OK;
}

kin_status check_update_args(const void* k_rows, const void* v_rows, const void* block_means,
                             const int32_t* seq_lens, const void* k_new, const void* v_new) {
  if (!k_rows || !v_rows || !block_means || !seq_lens || !k_new || !v_new) return KIN_ERR_INVALID_ARG;
  if (!aligned16(k_rows) || !aligned16(v_rows) || !aligned16(block_means) || !aligned16(k_new) ||
      !aligned16(v_new))
    return KIN_ERR_INVALID_ARG;
  return KIN_OK;
}

}  // namespace

KIN_EXPORT kin_status kin_block_means_build(const kin_dims* dims, const void* k_cache,
                                            const int32_t* seq_lens, float* block_means,
                                            int32_t* dev_status, void* stream) {
  KIN_NVTX_RANGE();
  kin_status st = check_dims(dims);
  if (st != KIN_OK) return st;
  if (!k_cache || !seq_lens || !block_means) return KIN_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(block_means)) return KIN_ERR_INVALID_ARG;
  return means_build(dims, k_cache, contiguous(), seq_lens, block_means, 0, dev_status, stream);
}

KIN_EXPORT kin_status kin_block_means_build_paged(const kin_dims* dims, const void* k_pages, int32_t num_pages,
                                                  const int32_t* block_table, const int32_t* seq_lens,
                                                  float* block_means, int32_t* dev_status, void* stream) {
  KIN_NVTX_RANGE();
  kin_status st = check_dims(dims);
  if (st != KIN_OK) return st;
  PageTable pt;
  st = check_pages(*dims, k_pages, num_pages, block_table, &pt);
  if (st != KIN_OK) return st;
  if (!seq_lens || !block_means || !aligned16(block_means)) return KIN_ERR_INVALID_ARG;
  return means_build(dims, k_pages, pt, seq_lens, block_means, 0, dev_status, stream);
}

KIN_EXPORT kin_status kin_block_means_update(const kin_dims* dims, void* k_cache, void* v_cache,
                                             float* block_means, int32_t* seq_lens,
                                             const void* k_new, const void* v_new, int32_t n_new,
                                             int32_t* dev_status, void* stream) {
  KIN_NVTX_RANGE();
  kin_status st = check_dims(dims);
  if (st != KIN_OK) return st;
  st = check_update_count(dims, n_new);
  if (st != KIN_OK || n_new == 0) return st;
  st = check_update_args(k_cache, v_cache, block_means, seq_lens, k_new, v_new);
  if (st != KIN_OK) return st;
  return means_update(dims, k_cache, v_cache, contiguous(), block_means, 0, seq_lens, k_new, v_new, n_new,
                      dev_status, stream);
}

KIN_EXPORT kin_status kin_block_means_update_paged(const kin_dims* dims, void* k_pages, void* v_pages,
                                                   int32_t num_pages, const int32_t* block_table,
                                                   float* block_means, int32_t* seq_lens, const void* k_new,
                                                   const void* v_new, int32_t n_new, int32_t* dev_status,
                                                   void* stream) {
  KIN_NVTX_RANGE();
  kin_status st = check_dims(dims);
  if (st != KIN_OK) return st;
  st = check_update_count(dims, n_new);
  if (st != KIN_OK || n_new == 0) return st;
  PageTable pt;
  st = check_pages(*dims, k_pages, num_pages, block_table, &pt);
  if (st != KIN_OK) return st;
  st = check_update_args(k_pages, v_pages, block_means, seq_lens, k_new, v_new);
  if (st != KIN_OK) return st;
  return means_update(dims, k_pages, v_pages, pt, block_means, 0, seq_lens, k_new, v_new, n_new, dev_status,
                      stream);
}

namespace {

kin_status topk_select(const kin_dims* dims, const void* q, const void* block_means, int means_bf16,
                       const int32_t* seq_lens, int32_t k_blocks, int32_t* sel_idx, int32_t* sel_cnt,
                       void* workspace, size_t ws_bytes, int32_t* dev_status, void* stream,
                       const PageTable* mpages = nullptr) {
  if (k_blocks < 2) return KIN_ERR_INVALID_ARG;
  if (!q || !block_means || !seq_lens || !sel_idx || !sel_cnt) return KIN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(block_means)) return KIN_ERR_INVALID_ARG;
  WsLayout w;
  kin_status st = check_ws(*dims, k_blocks, workspace, ws_bytes, &w);
  if (st != KIN_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  SelectParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.means = block_means;
  p.means_bf16 = means_bf16;
  p.refine = 0;
  p.means_f32 = nullptr;
  p.radii = nullptr;
  if (means_bf16 == 2) {  // dual: scan the bf16 rows, rescore from the fp32 rows
    const int64_t rows = mpages ? (int64_t)mpages->num_pages * dims->num_kv_heads
                                : (int64_t)dims->batch * dims->num_kv_heads * nbcap_of(*dims);
    const float* f = static_cast<const float*>(block_means);
    p.means = f + rows * kHeadDim;
    p.means_bf16 = 1;
    p.refine = 1;
    p.means_f32 = f;
    p.radii = f + rows * (kHeadDim + kHeadDim / 2);
  }
  p.mpages = mpages ? *mpages : contiguous();
  p.seq_lens = seq_lens;
  p.sel_idx = sel_idx;
  p.sel_cnt = sel_cnt;
  p.scores = reinterpret_cast<float*>(ws + w.scores);
  p.dev_status = dev_status;
  p.B = dims->batch;
  p.Hkv = dims->num_kv_heads;
  p.Hq = dims->num_q_heads;
  p.g = dims->num_q_heads / dims->num_kv_heads;
  p.bs = dims->block_size;
  p.Lcap = dims->max_seq_len;
  p.nbcap = nbcap_of(*dims);
  p.k = k_blocks;
  p.score_scale = 1.0f / std::sqrt((float)kHeadDim);
  return from_cuda(launch_select(p, static_cast<cudaStream_t>(stream)));
}

// means_dtype as a kernel flag (0 fp32, 1 bf16, 2 dual); -1 for an unknown value
int means_flag(int32_t means_dtype) {
  const int32_t t = means_dtype & ~KIN_MEANS_PER_PAGE;
  return t == KIN_MEANS_F32 ? 0 : t == KIN_MEANS_BF16 ? 1 : t == KIN_MEANS_DUAL ? 2 : -1;
}
int per_page_flag(int32_t means_dtype) { return (means_dtype & KIN_MEANS_PER_PAGE) ? 1 : 0; }

// A NULL table selects the contiguous cache (num_pages ignored).
kin_status layout_of(const kin_dims& d, const void* k_rows, int32_t num_pages, const int32_t* block_table,
                     PageTable* pt) {
  if (!block_table) {
    *pt = contiguous();
    return KIN_OK;
  }
  return check_pages(d, k_rows, num_pages, block_table, pt);
}

}  // namespace

KIN_EXPORT kin_status kin_block_topk_select(const kin_dims* dims, const void* q, const float* block_means,
                                            const int32_t* seq_lens, int32_t k_blocks, int32_t* sel_idx,
                                            int32_t* sel_cnt, void* workspace, size_t ws_bytes,
                                            int32_t* dev_status, void* stream) {
  KIN_NVTX_RANGE();
  kin_status st = check_dims(dims);
  if (st != KIN_OK) return st;
  return topk_select(dims, q, block_means, 0, seq_lens, k_blocks, sel_idx, sel_cnt, workspace, ws_bytes,
                     dev_status, stream);
}

KIN_EXPORT kin_status kin_block_topk_select_ex(const kin_dims* dims, const void* q, const void* block_means,
                                               int32_t means_dtype, const int32_t* seq_lens, int32_t k_blocks,
                                               int32_t* sel_idx, int32_t* sel_cnt, void* workspace,
                                               size_t ws_bytes, int32_t* dev_status, void* stream) {
  KIN_NVTX_RANGE();
  kin_status st = check_dims(dims);
  if (st != KIN_OK) return st;
  const int bf = means_flag(means_dtype);
  if (bf < 0 || per_page_flag(means_dtype)) return KIN_ERR_INVALID_ARG;  // per-page means need the table
  return topk_select(dims, q, block_means, bf, seq_lens, k_blocks, sel_idx, sel_cnt, workspace, ws_bytes,
                     dev_status, stream);
}

KIN_EXPORT kin_status kin_block_topk_select_paged(const kin_dims* dims, const void* q, const void* page_means,
                                                  int32_t means_dtype, int32_t num_pages,
                                                  const int32_t* block_table, const int32_t* seq_lens,
                                                  int32_t k_blocks, int32_t* sel_idx, int32_t* sel_cnt,
                                                  void* workspace, size_t ws_bytes, int32_t* dev_status,
                                                  void* stream) {
  KIN_NVTX_RANGE();
  kin_status st = check_dims(dims);
  if (st != KIN_OK) return st;
  const int bf = means_flag(means_dtype);
  if (bf < 0) return KIN_ERR_INVALID_ARG;
  PageTable pt;
  st = check_pages(*dims, page_means, num_pages, block_table, &pt);
  if (st != KIN_OK) return st;
  return topk_select(dims, q, page_means, bf, seq_lens, k_blocks, sel_idx, sel_cnt, workspace, ws_bytes,
                     dev_status, stream, &pt);
}

KIN_EXPORT kin_status kin_block_means_build_ex(const kin_dims* dims, const void* k_rows, int32_t num_pages,
                                               const int32_t* block_table, const int32_t* seq_lens,
                                               void* block_means, int32_t means_dtype, int32_t* dev_status,
                                               void* stream) {
  KIN_NVTX_RANGE();
  kin_status st = check_dims(dims);
  if (st != KIN_OK) return st;
  const int bf = means_flag(means_dtype);
  if (bf < 0) return KIN_ERR_INVALID_ARG;
  if (!k_rows || !seq_lens || !block_means) return KIN_ERR_INVALID_ARG;
  if (!aligned16(k_rows) || !aligned16(block_means)) return KIN_ERR_INVALID_ARG;
  PageTable pt;
  st = layout_of(*dims, k_rows, num_pages, block_table, &pt);
  if (st != KIN_OK) return st;
  const int pp = per_page_flag(means_dtype);
  if (pp && !block_table) return KIN_ERR_INVALID_ARG;
  return means_build(dims, k_rows, pt, seq_lens, block_means, bf, dev_status, stream, pp);
}

KIN_EXPORT kin_status kin_block_means_update_ex(const kin_dims* dims, void* k_rows, void* v_rows,
                                                int32_t num_pages, const int32_t* block_table,
                                                void* block_means, int32_t means_dtype, int32_t* seq_lens,
                                                const void* k_new, const void* v_new, int32_t n_new,
                                                int32_t* dev_status, void* stream) {
  KIN_NVTX_RANGE();
  kin_status st = check_dims(dims);
  if (st != KIN_OK) return st;
  const int bf = means_flag(means_dtype);
  if (bf < 0) return KIN_ERR_INVALID_ARG;
  st = check_update_count(dims, n_new);
  if (st != KIN_OK || n_new == 0) return st;
  st = check_update_args(k_rows, v_rows, block_means, seq_lens, k_new, v_new);
  if (st != KIN_OK) return st;
  PageTable pt;
  st = layout_of(*dims, k_rows, num_pages, block_table, &pt);
  if (st != KIN_OK) return st;
  const int pp = per_page_flag(means_dtype);
  if (pp && !block_table) return KIN_ERR_INVALID_ARG;
  return means_update(dims, k_rows, v_rows, pt, block_means, bf, seq_lens, k_new, v_new, n_new, dev_status,
                      stream, pp);
}

namespace {

kin_status sparse_decode_attn(const kin_dims* dims, const void* q, const void* k_rows, const void* v_rows,
                              const PageTable& pt, const int32_t* seq_lens, const int32_t* sel_idx,
                              const int32_t* sel_cnt, int32_t k_blocks, float softmax_scale, void* out,
                              float* lse, void* workspace, size_t ws_bytes, int32_t* dev_status, void* stream) {
  if (k_blocks < 2) return KIN_ERR_INVALID_ARG;
  if (!q || !k_rows || !v_rows || !seq_lens || !sel_idx || !sel_cnt || !out) return KIN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_rows) || !aligned16(v_rows) || !aligned16(out)) return KIN_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale) || std::isinf(softmax_scale)) return KIN_ERR_INVALID_ARG;
  WsLayout w;
  kin_status st = check_ws(*dims, k_blocks, workspace, ws_bytes, &w);
  if (st != KIN_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  AttnParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_cache = static_cast<const __nv_bfloat16*>(k_rows);
  p.v_cache = static_cast<const __nv_bfloat16*>(v_rows);
  p.seq_lens = seq_lens;
  p.sel_idx = sel_idx;
  p.sel_cnt = sel_cnt;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.partials = reinterpret_cast<float*>(ws + w.partials);
  p.counters = reinterpret_cast<uint32_t*>(ws + w.attn_counters);
  p.dev_status = dev_status;
  p.pages = pt;
  p.B = dims->batch;
  p.Hkv = dims->num_kv_heads;
  p.Hq = dims->num_q_heads;
  p.g = dims->num_q_heads / dims->num_kv_heads;
  p.bs = dims->block_size;
  p.Lcap = dims->max_seq_len;
  p.k = k_blocks;
  p.chunk_blocks = attn_chunk_blocks(*dims, k_blocks);
  p.max_chunks = attn_max_chunks(*dims, k_blocks);
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)kHeadDim);
  p.scale_log2 = scale * 1.4426950408889634f;
  const int num_items = pairs_of(*dims) * p.max_chunks;
  return from_cuda(launch_attn(p, num_items, static_cast<cudaStream_t>(stream)));
}

}  // namespace

KIN_EXPORT kin_status kin_sparse_decode_attn(const kin_dims* dims, const void* q, const void* k_cache,
                                             const void* v_cache, const int32_t* seq_lens,
                                             const int32_t* sel_idx, const int32_t* sel_cnt,
                                             int32_t k_blocks, float softmax_scale, void* out, float* lse,
                                             void* workspace, size_t ws_bytes, int32_t* dev_status,
                                             void* stream) {
  KIN_NVTX_RANGE();
  kin_status st = check_dims(dims);
  if (st != KIN_OK) return st;
  return sparse_decode_attn(dims, q, k_cache, v_cache, contiguous(), seq_lens, sel_idx, sel_cnt, k_blocks,
                            softmax_scale, out, lse, workspace, ws_bytes, dev_status, stream);
}

KIN_EXPORT kin_status kin_sparse_decode_attn_paged(const kin_dims* dims, const void* q, const void* k_pages,
                                                   const void* v_pages, int32_t num_pages,
                                                   const int32_t* block_table, const int32_t* seq_lens,
                                                   const int32_t* sel_idx, const int32_t* sel_cnt,
                                                   int32_t k_blocks, float softmax_scale, void* out,
                                                   float* lse, void* workspace, size_t ws_bytes,
                                                   int32_t* dev_status, void* stream) {
  KIN_NVTX_RANGE();
  kin_status st = check_dims(dims);
  if (st != KIN_OK) return st;
  PageTable pt;
  st = check_pages(*dims, k_pages, num_pages, block_table, &pt);
  if (st != KIN_OK) return st;
  return sparse_decode_attn(dims, q, k_pages, v_pages, pt, seq_lens, sel_idx, sel_cnt, k_blocks,
                            softmax_scale, out, lse, workspace, ws_bytes, dev_status, stream);
}

// ------------------------------------------------------------ token top-k
namespace {

constexpr int kTokenKeyCap = 32768;  // the token top-k keeps keys in shared memory up to this length

struct TokenWs {
  size_t logits, keys, sel, cnt, total;
};

TokenWs token_ws_layout(const kin_dims& d, int kt) {
  const size_t rows = (size_t)d.batch * d.num_q_heads;
  TokenWs w;
  size_t off = 0;
  w.logits = off;
  off = align_up(off + rows * (size_t)d.max_seq_len * sizeof(float));
  w.keys = off;
  if (d.max_seq_len > kTokenKeyCap) off = align_up(off + rows * (size_t)d.max_seq_len * sizeof(uint32_t));
  w.sel = off;
  off = align_up(off + rows * (size_t)kt * sizeof(int32_t));
  w.cnt = off;
  off = align_up(off + rows * sizeof(int32_t));
  w.total = off;
  return w;
}

}  // namespace

KIN_EXPORT size_t kin_token_topk_workspace_bytes(const kin_dims* dims, int32_t k_tokens) {
  if (check_dims(dims) != KIN_OK || k_tokens < 1) return 0;
  return token_ws_layout(*dims, k_tokens).total;
}

KIN_EXPORT kin_status kin_token_topk_decode_attn(const kin_dims* dims, const void* q, const void* k_cache,
                                                 const void* v_cache, const int32_t* seq_lens, int32_t k_tokens,
                                                 float softmax_scale, void* out, float* lse, int32_t* sel_tokens,
                                                 void* workspace, size_t ws_bytes, int32_t* dev_status,
                                                 void* stream) {
  KIN_NVTX_RANGE();
  kin_status st = check_dims(dims);
  if (st != KIN_OK) return st;
  if (k_tokens < 1) return KIN_ERR_INVALID_ARG;
  if (!q || !k_cache || !v_cache || !seq_lens || !out) return KIN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out)) return KIN_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale) || std::isinf(softmax_scale)) return KIN_ERR_INVALID_ARG;
  if ((int64_t)dims->batch * dims->num_q_heads * dims->max_seq_len >= (int64_t)1 << 31) return KIN_ERR_CAPACITY;
  const TokenWs w = token_ws_layout(*dims, k_tokens);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0 || ws_bytes < w.total)
    return KIN_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  TokenParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_cache = static_cast<const __nv_bfloat16*>(k_cache);
  p.v_cache = static_cast<const __nv_bfloat16*>(v_cache);
  p.seq_lens = seq_lens;
  p.logits = reinterpret_cast<float*>(ws + w.logits);
  p.key_scratch = reinterpret_cast<uint32_t*>(ws + w.keys);
  p.sel = sel_tokens ? sel_tokens : reinterpret_cast<int32_t*>(ws + w.sel);
  p.cnt = reinterpret_cast<int32_t*>(ws + w.cnt);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.dev_status = dev_status;
  p.B = dims->batch;
  p.Hkv = dims->num_kv_heads;
  p.Hq = dims->num_q_heads;
  p.g = dims->num_q_heads / dims->num_kv_heads;
  p.Lcap = dims->max_seq_len;
  p.kt = k_tokens;
  p.scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)kHeadDim);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_token_logits(p, s);
  if (e == cudaSuccess) e = launch_token_topk(p, s);
  if (e == cudaSuccess) e = launch_token_attn(p, s);
  return from_cuda(e);
}
