// kin_noalloc.cu -- kin_block_topk_select_noalloc: the block top-k select
// for callers that cannot allocate device memory.
//
// Who needs it: code that runs inside a host whose device memory is planned
// up front and owned by someone else (an inference runtime with a fixed
// memory plan, a plugin or extension that may not call cudaMalloc, a
// real-time decode loop that must never touch the allocator), or that has no
// way to create and keep a workspace buffer before its first call.  Such a
// caller still owns its inputs and outputs; only the scratch memory moves
// into the library.
//
// How: the per-block scores the select writes between its scan and its top-k
// live in a file-scope device array of fixed size (KIN_NOALLOC_SCRATCH_FLOATS
// floats, 8 MiB), which every GPU that loads libkin.so keeps until the
// process exits.  Host code cannot hand the array's name to a kernel (on the
// host it is only a stand-in for the device symbol), so the first call on
// each device looks up the array's device address with cudaGetSymbolAddress,
// with that device current, and caches it.  That first call is therefore the
// set-up call and should run before any stream capture begins.  Nothing in
// the array needs to start at zero: every score the top-k reads is written by
// the scan of the same call.  All calls share the one array, so calls whose
// kernels overlap on a GPU (two streams, or two threads) race on it.
#include <atomic>
#include "kin_internal.cuh"

#define KIN_EXPORT extern "C" __attribute__((visibility("default")))

namespace {

using namespace kin;

static __device__ __align__(256) float g_select_scratch[KIN_NOALLOC_SCRATCH_FLOATS];

constexpr int kMaxDevicesNoAlloc = 64;

// Device address of g_select_scratch on the current device (nullptr on error).
float* scratch_on_current_device(cudaError_t* err) {
  // per device, written once with the same address by whichever thread gets there first
  static std::atomic<float*> cache[kMaxDevicesNoAlloc];
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  const bool cached = dev >= 0 && dev < kMaxDevicesNoAlloc;
  if (cached) {
    float* c = cache[dev].load(std::memory_order_relaxed);
    if (c) return c;
  }
  void* ptr = nullptr;
  *err = cudaGetSymbolAddress(&ptr, g_select_scratch);
  if (*err != cudaSuccess || !ptr) return nullptr;
  if (cached) cache[dev].store(static_cast<float*>(ptr), std::memory_order_relaxed);
  return static_cast<float*>(ptr);
}

}  // namespace

KIN_EXPORT kin_status kin_block_topk_select_noalloc(const kin_dims* dims, const void* q,
                                                    const float* block_means, const int32_t* seq_lens,
                                                    int32_t k_blocks, int32_t* sel_idx,
                                                    int32_t* sel_cnt, int32_t* dev_status,
                                                    void* stream) {
  KIN_NVTX_RANGE();
  kin_status st = check_dims(dims);
  if (st != KIN_OK) return st;
  if (k_blocks < 2) return KIN_ERR_INVALID_ARG;
  if (!q || !block_means || !seq_lens || !sel_idx || !sel_cnt) return KIN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(block_means)) return KIN_ERR_INVALID_ARG;
  const int bs = dims->block_size;
  const int nbcap = (dims->max_seq_len + bs - 1) / bs;
  const int64_t need = (int64_t)dims->batch * dims->num_kv_heads * nbcap;  // one score per block
  if (need > (int64_t)KIN_NOALLOC_SCRATCH_FLOATS) return KIN_ERR_CAPACITY;
  cudaError_t err = cudaSuccess;
  float* scratch = scratch_on_current_device(&err);
  if (!scratch) return KIN_ERR_CUDA;

  SelectParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.means = block_means;
  p.means_bf16 = 0;
  p.refine = 0;  // fp32 means: the plain select (no dual-means refinement)
  p.means_f32 = nullptr;
  p.radii = nullptr;
  p.mpages.table = nullptr;  // logical means
  p.mpages.max_blocks = 0;
  p.mpages.num_pages = 0;
  p.seq_lens = seq_lens;
  p.sel_idx = sel_idx;
  p.sel_cnt = sel_cnt;
  p.scores = scratch;
  p.dev_status = dev_status;
  p.B = dims->batch;
  p.Hkv = dims->num_kv_heads;
  p.Hq = dims->num_q_heads;
  p.g = dims->num_q_heads / dims->num_kv_heads;
  p.bs = bs;
  p.Lcap = dims->max_seq_len;
  p.nbcap = nbcap;
  p.k = k_blocks;
  p.score_scale = 1.0f / sqrtf((float)kHeadDim);
  return launch_select(p, static_cast<cudaStream_t>(stream)) == cudaSuccess ? KIN_OK : KIN_ERR_CUDA;
}
