// kin_internal.cuh -- shared device helpers and launch-parameter structs of
// libkin.so (sm_100a).  Not part of the public ABI (see include/kin.h).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kin.h"

// NVTX ranges around every launching kin_* call (header-only NVTX3; a no-op
// unless a profiler is attached).  -DKIN_NVTX=0 compiles them out.
#ifndef KIN_NVTX
#define KIN_NVTX 1
#endif
#if KIN_NVTX
#include <nvtx3/nvToolsExt.h>
#endif

namespace kin {

// Scoped NVTX range named after the entry point (host code).
struct NvtxRange {
  explicit NvtxRange(const char* name) {
#if KIN_NVTX
    nvtxRangePushA(name);
#else
    (void)name;
#endif
  }
  ~NvtxRange() {
#if KIN_NVTX
    nvtxRangePop();
#endif
  }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
#define KIN_NVTX_RANGE() ::kin::NvtxRange kin_nvtx_range_(__func__)

constexpr int kHeadDim = 128;
constexpr int kMaxGroup = 8;
constexpr int kMaxBlocksPerSeq = 32768;
constexpr int kTileTokens = 16;  // tokens per attention tile (one m16 MMA row block)
constexpr int kMaxItemTiles = 64;  // attention tiles per work item (chunk of kept blocks)
// floats per (chunk, query head) attention partial: o[D], max, sum, 2 pad
// (a multiple of 4, so every record starts on a 16-byte boundary)
constexpr int kPartStride = kHeadDim + 4;

// ----------------------------------------------------------------- status
__device__ __forceinline__ void set_status(int32_t* st, int32_t code) {
  if (st) atomicCAS(st, 0, code);
}

// ---------------------------------------------------- order-preserving keys
// Maps fp32 bits to uint32 so that unsigned order == float order.
__device__ __forceinline__ uint32_t float_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------- programmatic dependent launch
// Kernels of a step are launched with programmatic stream serialization: a
// kernel may be scheduled while its predecessor drains, and waits here (a
// hardware dependency wait, not a spin) before touching the predecessor's
// results; each kernel signals once its own results are written.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
// An L2 prefetch hint: moves no data into the program's view of memory, so
// it may run before pdl_wait (a line that a predecessor later writes is
// simply fetched again).  The address must lie inside an allocation.
__device__ __forceinline__ void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }
// Where a kernel lets the next one launch.  griddepcontrol.wait returns
// only once every prerequisite grid has completed and its memory is visible,
// so the signal's place never changes results, only overlap: with
// KIN_PDL_EARLY 1 a kernel signals right after its own wait, and the next
// kernel's CTAs are scheduled onto free SM slots while this grid runs (they
// sit in their wait); with 0 it signals as its CTAs finish.
#ifndef KIN_PDL_EARLY
#define KIN_PDL_EARLY 1
#endif
__device__ __forceinline__ void pdl_trigger_early() {
  if (KIN_PDL_EARLY) pdl_trigger();
}
__device__ __forceinline__ void pdl_trigger_late() {
  if (!KIN_PDL_EARLY) pdl_trigger();
}

// ------------------------------------------------------------- cp.async
// 16-byte async copy global -> shared; src_bytes 0 writes zeros and reads nothing.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Invalidates one 128-byte L2 line (128-byte aligned address) without writing it back: for
// scratch whose contents are no longer needed, so it costs no DRAM write.
__device__ __forceinline__ void discard_l2_line(const void* p) {
  asm volatile("discard.global.L2 [%0], 128;" ::"l"(p) : "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// -------------------------------------------------- PTX: warp-level MMA path
__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                            uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                                  uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}

// D = A(16x16 bf16, row) * B(16x8 bf16, col) + C (fp32)
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// ---------------------------------------------------------- KV addressing
// Where the K/V rows of a logical block live.  table == NULL: the contiguous
// cache [B][Hkv][Lcap][D].  Otherwise a page pool [num_pages][Hkv][bs][D]
// (the page is one KV block; a head's rows of a page are contiguous) and
// table[b * max_blocks + i] is the page of sequence b's logical block i.
struct PageTable {
  const int32_t* table;
  int max_blocks;
  int num_pages;
};

// Element offset of row r (0 <= r < bs) of logical block blk of pair (b, h),
// or -1 when the block's page index lies outside the pool.
__device__ __forceinline__ int64_t kv_row_offset(const PageTable& pt, int b, int h, int Hkv, int Lcap,
                                                 int bs, int blk, int r) {
  if (!pt.table) return (((int64_t)b * Hkv + h) * Lcap + (int64_t)blk * bs + r) * kHeadDim;
  const int page = __ldg(pt.table + (int64_t)b * pt.max_blocks + blk);
  if (page < 0 || page >= pt.num_pages) return -1;
  return (((int64_t)page * Hkv + h) * bs + r) * kHeadDim;
}

// ---------------------------------------------------------- launch params
// Block means are fp32 rows of D (the default), or bf16 rows (means_bf16:
// each fp32 mean rounded to nearest even), [B][Hkv][nbcap][D] either way.
__device__ __forceinline__ void store_mean_row(void* means, int means_bf16, int64_t row, int lane, float4 m) {
  if (means_bf16) {
    uint2 v;
    v.x = pack_bf16x2(m.x, m.y);
    v.y = pack_bf16x2(m.z, m.w);
    reinterpret_cast<uint2*>(means)[row * (kHeadDim / 4) + lane] = v;
  } else {
    reinterpret_cast<float4*>(means)[row * (kHeadDim / 4) + lane] = m;
  }
}

// Dual block means (KIN_MEANS_DUAL; kernel flag 2): one buffer holding the
// fp32 rows [rows][D], then the same means rounded to bf16 [rows][D], then
// each row's error radius [rows] (fp32), rows = the logical mean rows.  A
// select scans the bf16 rows and rescores from the fp32 rows only the blocks
// that its error bound cannot place.  The radius of row m with bf16 rounding
// b (d = m - b, exact in fp32) is an upper bound on
//   |d|_2 + 2^-19 |m|_2 + 2^-60,
// rounded up: (1 + 2^-12) |d|_2 + 2^-18 |m|_2 + 2^-59 (the norms' fp32
// sums of 128 squares are within 2^-20 relative, and underflow of the
// squares loses less than 2^-60 from a norm).  Warp-wide: lane l holds dims
// 4l..4l+3 of the row.
__device__ __forceinline__ float bf16_residual(float x) {
  return x - __bfloat162float(__float2bfloat16_rn(x));
}

__device__ __forceinline__ void store_mean_row_dual(void* means, int64_t rows, int64_t row, int lane, float4 m) {
  float* f = reinterpret_cast<float*>(means);
  reinterpret_cast<float4*>(f)[row * (kHeadDim / 4) + lane] = m;
  uint2 v;
  v.x = pack_bf16x2(m.x, m.y);
  v.y = pack_bf16x2(m.z, m.w);
  reinterpret_cast<uint2*>(f + rows * kHeadDim)[row * (kHeadDim / 4) + lane] = v;
  const float4 d = make_float4(bf16_residual(m.x), bf16_residual(m.y), bf16_residual(m.z), bf16_residual(m.w));
  float mm = m.x * m.x, dd = d.x * d.x;
  mm = fmaf(m.y, m.y, mm);
  dd = fmaf(d.y, d.y, dd);
  mm = fmaf(m.z, m.z, mm);
  dd = fmaf(d.z, d.z, dd);
  mm = fmaf(m.w, m.w, mm);
  dd = fmaf(d.w, d.w, dd);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    mm += __shfl_xor_sync(0xffffffffu, mm, off);
    dd += __shfl_xor_sync(0xffffffffu, dd, off);
  }
  if (lane == 0) {
    const float rad = __fadd_ru(__fadd_ru(__fmul_ru(__fsqrt_ru(dd), 0x1.001p0f), __fmul_ru(__fsqrt_ru(mm), 0x1p-18f)),
                                0x1p-59f);
    f[rows * (kHeadDim + kHeadDim / 2) + row] = rad;
  }
}

// A mean row in the layout the flag names (0 fp32, 1 bf16, 2 dual).
__device__ __forceinline__ void store_mean(void* means, int flag, int64_t rows, int64_t row, int lane, float4 m) {
  if (flag == 2)
    store_mean_row_dual(means, rows, row, lane, m);
  else
    store_mean_row(means, flag, row, lane, m);
}

// Row of block i of pair (b, h) in the block-means array: logical
// [B][Hkv][nbcap][D], or per page [num_pages][Hkv][D] (means_per_page: the
// mean of a page's rows, shared by every sequence whose table maps a block
// to that page).  -1 for a page index outside the pool.
__device__ __forceinline__ int64_t means_row_index(const PageTable& pt, int means_per_page, int b, int h, int Hkv,
                                                   int nbcap, int i) {
  if (!means_per_page) return ((int64_t)b * Hkv + h) * nbcap + i;
  const int page = __ldg(pt.table + (int64_t)b * pt.max_blocks + i);
  if (page < 0 || page >= pt.num_pages) return -1;
  return (int64_t)page * Hkv + h;
}

struct MeansBuildParams {
  const __nv_bfloat16* k_cache;  // contiguous cache or page pool (see PageTable)
  const int32_t* seq_lens;
  void* means;
  int means_bf16;              // 0 fp32, 1 bf16, 2 dual
  int64_t mean_rows;           // rows of the logical layout (the dual layout's stride)
  int means_per_page;            // means [num_pages][Hkv][D] (needs a page table)
  int32_t* dev_status;
  PageTable pages;
  int B, Hkv, Lcap, bs, nbcap;
};

struct MeansUpdateParams {
  __nv_bfloat16* k_cache;
  __nv_bfloat16* v_cache;
  void* means;
  int means_bf16;              // 0 fp32, 1 bf16, 2 dual
  int64_t mean_rows;
  int means_per_page;
  int32_t* seq_lens;
  const __nv_bfloat16* k_new;
  const __nv_bfloat16* v_new;
  int32_t* dev_status;
  PageTable pages;
  int B, Hkv, Lcap, bs, nbcap, n_new;
};

struct SelectParams {
  const __nv_bfloat16* q;
  const void* means;
  int means_bf16;
  PageTable mpages;     // table != NULL: means per page [num_pages][Hkv][D], found through the table
  const int32_t* seq_lens;
  int32_t* sel_idx;
  int32_t* sel_cnt;
  float* scores;        // workspace [B*Hkv][nbcap]
  int32_t* dev_status;
  int B, Hkv, Hq, g, bs, Lcap, nbcap, k;
  float score_scale;
  // dual means: the scan reads the bf16 rows (means), the top-k rescores
  // from the fp32 rows the blocks that the rows' error radii cannot place
  int refine;
  const float* means_f32;  // [B*Hkv][nbcap][D]
  const float* radii;      // [B*Hkv][nbcap]
};

struct AttnParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k_cache;
  const __nv_bfloat16* v_cache;
  const int32_t* seq_lens;
  const int32_t* sel_idx;
  const int32_t* sel_cnt;
  __nv_bfloat16* out;
  float* lse;
  float* partials;      // workspace [B*Hkv][max_chunks][g][kPartStride]
  uint32_t* counters;   // workspace [B*Hkv], zero between calls
  int32_t* dev_status;
  PageTable pages;
  int B, Hkv, Hq, g, bs, Lcap, k, chunk_blocks, max_chunks;
  float scale_log2;     // softmax_scale * log2(e)
};

// Token-level top-k attention: every logit of every query head, a top-k of
// tokens per head, attention over the kept tokens.
struct TokenParams {
  const __nv_bfloat16* q;        // [B][Hq][D]
  const __nv_bfloat16* k_cache;  // [B][Hkv][Lcap][D]
  const __nv_bfloat16* v_cache;
  const int32_t* seq_lens;
  float* logits;                 // workspace [B][Hq][Lcap]: scale * q . K_t
  uint32_t* key_scratch;         // workspace [B][Hq][Lcap] when Lcap exceeds the shared-memory key cap
  int32_t* sel;                  // [B][Hq][kt] kept token indices, ascending, -1 padded
  int32_t* cnt;                  // [B][Hq]
  __nv_bfloat16* out;            // [B][Hq][D]
  float* lse;                    // [B][Hq] or NULL
  int32_t* dev_status;
  int B, Hkv, Hq, g, Lcap, kt;
  float scale;                   // softmax scale (natural log base)
};

// Launch with programmatic stream serialization (see pdl_wait).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Host-side argument checks shared by every entry point: the problem
// dimensions every kernel supports, and 16-byte alignment of a pointer.
kin_status check_dims(const kin_dims* d);
bool aligned16(const void* p);

// Per-device facts the launchers need, cached after the first query (a
// device's SM count never changes; racing first calls store the same value).
int device_sm_count();
// Raises a kernel's dynamic shared memory limit once per device.
cudaError_t ensure_smem_limit(const void* kernel, int slot, size_t bytes);

// Launchers (one per kernel family); return the launch error.
cudaError_t launch_means_build(const MeansBuildParams& p, cudaStream_t s);
cudaError_t launch_means_update(const MeansUpdateParams& p, cudaStream_t s);
cudaError_t launch_select(const SelectParams& p, cudaStream_t s);
cudaError_t launch_attn(const AttnParams& p, int num_items, cudaStream_t s);
cudaError_t launch_token_logits(const TokenParams& p, cudaStream_t s);
cudaError_t launch_token_topk(const TokenParams& p, cudaStream_t s);
cudaError_t launch_token_attn(const TokenParams& p, cudaStream_t s);

}  // namespace kin
