/*
 * kin.h -- C ABI of the B200 (sm_100a) block top-k sparse decode attention
 * library libkin.so.
 *
 * The method: for every sequence b and KV head h of a decode batch, keep one
 * mean key per fixed-size KV block, score each block against the GQA query
 * group, keep the top-k blocks (the first block and the block holding the
 * newest token always among them), and run softmax(q K^T / sqrt(d)) V over
 * the tokens of the kept blocks only.
 *   - "Kinetics: Memory-Aware Test-Time Scaling", Architecture Overview
 *     (block-level top-k sparsity) and Implementation, BlockTopKAttention
 *     (1/sqrt(head_dim) scaling, mean over a block, top-k over blocks,
 *     softmax then the weighted sum of V).
 *   - "Kinetics: Rethinking Test-Time Scaling Law", author response Q4
 *     "KV block size and grouping strategy" (KV budget = block size x number
 *     of top-k blocks, e.g. (16, 64), (32, 32), (64, 16)) and response Q3
 *     (decode batches with ragged KV lengths).
 * Readings where the pages are silent: the block summary is the mean key of
 * the block's valid tokens; a group's block score is the sum over its query
 * heads; the budget k counts the two forced blocks; ties go to the lower
 * block index; query head j reads KV head j / (Hq / Hkv).
 *
 * Conventions shared by every call
 *  - All tensor pointers are caller-owned DEVICE memory (e.g. PyTorch
 *    tensors), C-contiguous, 16-byte aligned.  The library never allocates,
 *    frees or synchronises; every call is asynchronous on `stream` (a
 *    cudaStream_t; NULL means the legacy default stream).
 *  - Layouts (bf16 = 2-byte bfloat16):
 *      q            [B][Hq][D]            bf16
 *      k_cache/v_cache [B][Hkv][Lcap][D]  bf16  (Lcap = dims.max_seq_len)
 *      block_means  [B][Hkv][NBcap][D]    fp32  (NBcap = ceil(Lcap / bs))
 *      seq_lens     [B]                   int32 (valid tokens per sequence)
 *      sel_idx      [B][Hkv][k]           int32 ascending, -1 padded
 *      sel_cnt      [B][Hkv]              int32
 *      out          [B][Hq][D]            bf16
 *      lse          [B][Hq]               fp32  natural-log log-sum-exp
 *  - The host checks every argument it can before launching and returns a
 *    status; after launching it returns KIN_ERR_CUDA if the launch failed.
 *  - Data that only the device can see (a sequence length outside
 *    [1, Lcap], a block index outside [0, nb)) makes the kernel skip that
 *    item and write the status code into *dev_status (first error wins) when
 *    dev_status is not NULL.  Kernels never trap and never wait on other
 *    CTAs or kernels: a split-K merge is run by the last chunk to arrive
 *    (counted with an atomic), so nothing spins.
 *  - No C++ exception crosses this boundary; the library keeps no state
 *    between calls other than what the caller's buffers hold (except the
 *    scratch array of kin_block_topk_select_noalloc, described there, and
 *    per-device caches of device properties and kernel shared-memory
 *    limits, kept with atomics and a lock).  Calls may come from several
 *    host threads at once, each with its own buffers and workspace.
 *  - Every call that launches kernels opens an NVTX range named after the
 *    call for its host-side duration (NVTX3, header-only: it costs nothing
 *    measurable unless a profiler is attached; built with -DKIN_NVTX=0 the
 *    ranges are compiled out).
 *  - Limits: head_dim == 128; Hq % Hkv == 0 with 1 <= Hq/Hkv <= 8;
 *    block_size in {16, 32, 64, 128}; ceil(Lcap / bs) <= 32768;
 *    B * Hkv * Lcap < 2^31.
 */
#ifndef KIN_H
#define KIN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KIN_OK = 0,
  KIN_ERR_INVALID_ARG = 1,  /* null pointer, bad dimension, k < 2, misaligned */
  KIN_ERR_WORKSPACE = 2,    /* workspace NULL, too small or misaligned */
  KIN_ERR_CAPACITY = 3,     /* a size beyond a documented limit */
  KIN_ERR_CUDA = 4,         /* a CUDA runtime/driver call or launch failed */
  KIN_ERR_DEVICE_DATA = 5,  /* (device) bad seq_len / block index: item skipped */
  KIN_ERR_TIMEOUT = 6       /* reserved for a bounded device wait; no kernel waits today */
} kin_status;

typedef struct {
  int32_t batch;         /* B */
  int32_t num_kv_heads;  /* Hkv */
  int32_t num_q_heads;   /* Hq, a multiple of Hkv */
  int32_t head_dim;      /* D, must be 128 */
  int32_t block_size;    /* bs, tokens per KV block: 16, 32, 64 or 128 */
  int32_t max_seq_len;   /* Lcap, cache capacity in tokens per sequence */
} kin_dims;

/* Human-readable name of a status code (static string, never NULL). */
const char* kin_status_string(kin_status s);

/* Bytes of scratch the select and attention calls need for budget k_blocks
 * (one buffer serves both calls: each uses its own disjoint region).  Returns
 * 0 if the dims are invalid.  The buffer must be 256-byte aligned and filled
 * with zeros before its first use; every call leaves its completion counters
 * at zero again, so the same buffer can be reused by later calls on the same
 * stream without re-zeroing.  Calls that share one workspace must not run
 * concurrently. */
size_t kin_workspace_bytes(const kin_dims* dims, int32_t k_blocks);

/* Block means of a prefilled cache: for every (b, h) and block
 * i < ceil(seq_lens[b] / bs), block_means[b][h][i][:] = mean of K rows
 * i*bs .. min((i+1)*bs, seq_lens[b]) - 1, summed in fp32 in token order and
 * divided by the number of valid rows.  Blocks at or beyond the length are
 * left untouched.  Reads k_cache; writes block_means.  This is the prefill
 * counterpart of kin_block_means_update (the same definition applied to
 * every block at once). */
kin_status kin_block_means_build(const kin_dims* dims, const void* k_cache,
                                 const int32_t* seq_lens, float* block_means,
                                 int32_t* dev_status, void* stream);

/* Append n_new tokens to every sequence and refresh the block means they
 * touch.  For each b with L0 = seq_lens[b] (read on the device):
 * k_new[b][h][r] / v_new[b][h][r] ([B][Hkv][n_new][D] bf16) are written to
 * cache rows L0 + r; the mean of every block that holds one of those rows is
 * recomputed from all its valid rows (fp32, token order, divided by the
 * count); then seq_lens[b] = L0 + n_new.  A sequence with L0 < 0 or
 * L0 + n_new > Lcap is skipped and flagged KIN_ERR_DEVICE_DATA.
 * seq_lens is device memory, read and written.  n_new == 0 is a no-op. */
kin_status kin_block_means_update(const kin_dims* dims, void* k_cache, void* v_cache,
                                  float* block_means, int32_t* seq_lens,
                                  const void* k_new, const void* v_new, int32_t n_new,
                                  int32_t* dev_status, void* stream);

/* Group-summed block scores then exact block top-k.  For pair (b, h) with
 * nb = ceil(seq_lens[b] / bs):
 *   s_i = (1/sqrt(D)) * sum_{j < g} q[b][h*g + j] . block_means[b][h][i],
 * computed in fp32 from the fp32 means.
 * If k_blocks >= nb, all nb blocks are kept.  Otherwise blocks 0 and nb-1
 * are kept and the other k_blocks - 2 are the best of 1..nb-2 by
 * (s descending, index ascending).  sel_idx[b][h][:] receives the kept
 * indices ascending followed by -1 padding to k_blocks; sel_cnt[b][h] the
 * count.  k_blocks < 2 is KIN_ERR_INVALID_ARG.  A sequence whose length is
 * outside [1, Lcap] gets sel_cnt 0 and is flagged KIN_ERR_DEVICE_DATA.
 * workspace: see kin_workspace_bytes. */
kin_status kin_block_topk_select(const kin_dims* dims, const void* q, const float* block_means,
                                 const int32_t* seq_lens, int32_t k_blocks, int32_t* sel_idx,
                                 int32_t* sel_cnt, void* workspace, size_t ws_bytes,
                                 int32_t* dev_status, void* stream);

/* Split-K flash-decode over the selected blocks, then a log-sum-exp merge.
 * For query head j of pair (b, h = j / g), over the tokens t < seq_lens[b]
 * of the blocks sel_idx[b][h][0 .. sel_cnt[b][h]-1]:
 *   z_t = softmax_scale * q[b][j] . K_t,
 *   out[b][j] = sum_t e^{z_t - max z} V_t / sum_t e^{z_t - max z}   (bf16, RNE),
 *   lse[b][j] = max z + ln sum_t e^{z_t - max z}                  (fp32).
 * softmax_scale <= 0 selects 1/sqrt(D).  lse may be NULL.  Work is split
 * into chunks of selected blocks whose partial (o, max, sum) are merged by
 * the last chunk to finish (no extra launch).  A pair with sel_cnt 0 gets
 * out = 0 and lse = -inf.  A block index outside [0, nb) is skipped and
 * flagged KIN_ERR_DEVICE_DATA.  k_blocks is the sel_idx row stride.
 * workspace: see kin_workspace_bytes. */
kin_status kin_sparse_decode_attn(const kin_dims* dims, const void* q, const void* k_cache,
                                  const void* v_cache, const int32_t* seq_lens,
                                  const int32_t* sel_idx, const int32_t* sel_cnt,
                                  int32_t k_blocks, float softmax_scale, void* out, float* lse,
                                  void* workspace, size_t ws_bytes, int32_t* dev_status,
                                  void* stream);

/* ------------------------------------------------------------------------
 * Paged KV cache.  Ragged, growing decode batches are served from a pool of
 * fixed-size pages ("Kinetics: Rethinking Test-Time Scaling Law", response
 * Q3: the FlashInfer backend partitions ragged lengths into pages).  Here a
 * page is one KV block (page size = dims.block_size):
 *     k_pages, v_pages  [num_pages][Hkv][bs][D]  bf16  (a head's rows of a
 *                       page are contiguous: 4 KB at bs 16)
 *     block_table       [B][NBcap] int32, NBcap = ceil(dims.max_seq_len / bs);
 *                       block_table[b][i] is the page holding logical block
 *                       i (tokens i*bs .. i*bs+bs-1) of sequence b.
 * Only the entries of blocks a call touches are read: blocks below
 * ceil(seq_len / bs) (and, for an append, the blocks the new tokens land
 * in, which the caller must have mapped beforehand).  Block means stay in
 * the logical layout [B][Hkv][NBcap][D], so kin_block_topk_select and its
 * workspace serve both layouts unchanged, and every result equals the
 * contiguous call's on the same logical cache, bit for bit.
 * A page index outside [0, num_pages) is device-only bad data: the block (or
 * tile, or appended row) is skipped and KIN_ERR_DEVICE_DATA is flagged.
 * num_pages < 1 or a NULL table is KIN_ERR_INVALID_ARG.  Everything else,
 * including dims.max_seq_len (the per-sequence capacity), is as in the
 * contiguous calls above. */
kin_status kin_block_means_build_paged(const kin_dims* dims, const void* k_pages, int32_t num_pages,
                                       const int32_t* block_table, const int32_t* seq_lens,
                                       float* block_means, int32_t* dev_status, void* stream);

kin_status kin_block_means_update_paged(const kin_dims* dims, void* k_pages, void* v_pages,
                                        int32_t num_pages, const int32_t* block_table, float* block_means,
                                        int32_t* seq_lens, const void* k_new, const void* v_new,
                                        int32_t n_new, int32_t* dev_status, void* stream);

kin_status kin_sparse_decode_attn_paged(const kin_dims* dims, const void* q, const void* k_pages,
                                        const void* v_pages, int32_t num_pages, const int32_t* block_table,
                                        const int32_t* seq_lens, const int32_t* sel_idx,
                                        const int32_t* sel_cnt, int32_t k_blocks, float softmax_scale,
                                        void* out, float* lse, void* workspace, size_t ws_bytes,
                                        int32_t* dev_status, void* stream);

/* ------------------------------------------------------------------------
 * Extended calls: block means in bf16, either KV layout.
 *
 * bf16 block means halve the bytes the select streams (a NEXT variant: the
 * contiguous calls above keep fp32 means, whose scores stay within the
 * method's 1e-4 near-tie band).  A bf16 mean is the fp32 mean of the calls
 * above rounded to nearest even; scores are then computed in fp32 from the
 * widened bf16 values.  block_means is [B][Hkv][NBcap][D] of the given
 * dtype; the same buffer must be passed to the build/update and the select.
 * block_table NULL selects the contiguous cache [B][Hkv][Lcap][D] (then
 * num_pages is ignored); otherwise k_rows / v_rows are the page pool of the
 * paged calls.  An unknown means_dtype is KIN_ERR_INVALID_ARG.  Otherwise
 * arguments, semantics and errors are those of kin_block_means_build,
 * kin_block_means_update (and their paged forms) and kin_block_topk_select. */
typedef enum { KIN_MEANS_F32 = 0, KIN_MEANS_BF16 = 1, KIN_MEANS_DUAL = 2 } kin_means_dtype;
/* KIN_MEANS_DUAL: one buffer of kin_dual_means_bytes(dims) bytes (16-byte
 * aligned) holding the fp32 means [B][Hkv][NBcap][D], then the same means
 * rounded to bf16 [B][Hkv][NBcap][D], then each mean row's error radius
 * [B][Hkv][NBcap] (fp32: an upper bound on |m - bf16(m)|_2 + 2^-19 |m|_2 +
 * 2^-60 for the row's fp32 mean m); the build/update calls write all three.
 * The select over it returns exactly the selection of the fp32 means (the
 * same indices as kin_block_topk_select on the fp32 part, bit for bit)
 * while it streams the bf16 copy: the scan scores every block from its
 * bf16 mean, each score s~ is within e = (1/sqrt(D)) |q_group|_2 rho (to a
 * factor 1 + 2^-10 and an underflow margin) of the fp32 score, rho being
 * the row's radius (Cauchy-Schwarz on the rounding residual; the 2^-19
 * |m|_2 term covers the fp32 rounding of both scores), a block whose
 * s~ + e is below the k-th largest s~ - e cannot be kept, one whose s~ - e
 * is above the k-th largest s~ + e is kept, and only the band between is
 * rescored from its fp32 rows with the fp32 scan's own arithmetic before
 * the exact top-k.  The sizes are 0 for invalid dims (or num_pages < 1).
 * Stored per page
 * (KIN_MEANS_DUAL | KIN_MEANS_PER_PAGE, with a block table), the same three
 * arrays hold one row per (page, KV head): [num_pages][Hkv][D] fp32, then
 * bf16, then [num_pages][Hkv] radii, in a buffer of
 * kin_dual_page_means_bytes(dims, num_pages) bytes, read by
 * kin_block_topk_select_paged (a page index outside the pool is flagged as
 * for the other means and its block scored from a zero row). */
size_t kin_dual_means_bytes(const kin_dims* dims);
size_t kin_dual_page_means_bytes(const kin_dims* dims, int32_t num_pages);
/* OR-ed into means_dtype of the build/update calls (with a block table):
 * block means per page, [num_pages][Hkv][D], read by
 * kin_block_topk_select_paged below. */
#define KIN_MEANS_PER_PAGE 0x100

kin_status kin_block_means_build_ex(const kin_dims* dims, const void* k_rows, int32_t num_pages,
                                    const int32_t* block_table, const int32_t* seq_lens, void* block_means,
                                    int32_t means_dtype, int32_t* dev_status, void* stream);

kin_status kin_block_means_update_ex(const kin_dims* dims, void* k_rows, void* v_rows, int32_t num_pages,
                                     const int32_t* block_table, void* block_means, int32_t means_dtype,
                                     int32_t* seq_lens, const void* k_new, const void* v_new, int32_t n_new,
                                     int32_t* dev_status, void* stream);

kin_status kin_block_topk_select_ex(const kin_dims* dims, const void* q, const void* block_means,
                                    int32_t means_dtype, const int32_t* seq_lens, int32_t k_blocks,
                                    int32_t* sel_idx, int32_t* sel_cnt, void* workspace, size_t ws_bytes,
                                    int32_t* dev_status, void* stream);

/* ------------------------------------------------------------------------
 * Shared-prompt (Best-of-N) reuse.  N samples of one prompt share the
 * prompt's KV, which is read once for all of them ("Kinetics: Rethinking
 * Test-Time Scaling Law", response W3: prompt sharing lets different
 * requests access the same KV memory at decoding time).  With the paged
 * calls, each sample's block table maps the prompt's blocks to the same
 * pages; with block means per page (KIN_MEANS_PER_PAGE in the build/update
 * calls), the prompt's means are stored once too.  This select reads the
 * per-page means through the table:
 *   page_means  [num_pages][Hkv][D], fp32 or bf16 (means_dtype, without the
 *               per-page flag), or dual means per page (KIN_MEANS_DUAL: the
 *               fp32 selection read from the bf16 rows, see above); block i
 *               of (b, h) is page_means[block_table[b][i]][h].
 * A page shared by several sequences must hold full blocks (bs valid rows)
 * in each of them, so its mean is the same for all.  Results equal those
 * of the select over logical means of the same blocks, bit for bit.  A page
 * index outside the pool zeroes that block's score and flags
 * KIN_ERR_DEVICE_DATA.  Other arguments and errors: kin_block_topk_select. */
kin_status kin_block_topk_select_paged(const kin_dims* dims, const void* q, const void* page_means,
                                       int32_t means_dtype, int32_t num_pages, const int32_t* block_table,
                                       const int32_t* seq_lens, int32_t k_blocks, int32_t* sel_idx,
                                       int32_t* sel_cnt, void* workspace, size_t ws_bytes, int32_t* dev_status,
                                       void* stream);

/* ------------------------------------------------------------------------
 * Token-level top-k attention (the variant the block method is compared
 * with: "Kinetics: Rethinking Test-Time Scaling Law", response Q2, Fig. 8's
 * TopK attention; TopK attention keeps the keys and values with the highest
 * attention scores).  For query head j of sequence b, over the tokens
 * t < seq_lens[b] of the contiguous cache:
 *   z_t = softmax_scale * q[b][j] . K_t            (every token: a dense K pass)
 *   S   = the k_tokens tokens with the largest z_t (ties to the lower index,
 *         nothing forced; every token when k_tokens >= seq_lens[b])
 *   out[b][j] = sum_{t in S} e^{z_t - max z} V_t / sum_{t in S} e^{z_t - max z}
 *   lse[b][j] = max z + ln sum_{t in S} e^{z_t - max z}      (max over S)
 * Each query head selects its own tokens (a GQA group does not share them).
 * sel_tokens ([B][Hq][k_tokens] int32, ascending, -1 padded) receives S when
 * not NULL.  softmax_scale <= 0 selects 1/sqrt(D); lse may be NULL.  A bad
 * length gets out = 0, lse = -inf and flags KIN_ERR_DEVICE_DATA.  Scratch:
 * kin_token_topk_workspace_bytes (256-byte aligned; no zeroing needed; the
 * fp32 logits of every token of every query head live there).  k_tokens < 1
 * is KIN_ERR_INVALID_ARG; B * Hq * max_seq_len must stay below 2^31. */
size_t kin_token_topk_workspace_bytes(const kin_dims* dims, int32_t k_tokens);

kin_status kin_token_topk_decode_attn(const kin_dims* dims, const void* q, const void* k_cache,
                                      const void* v_cache, const int32_t* seq_lens, int32_t k_tokens,
                                      float softmax_scale, void* out, float* lse, int32_t* sel_tokens,
                                      void* workspace, size_t ws_bytes, int32_t* dev_status, void* stream);

/* ------------------------------------------------------------------------
 * Allocation-free variant of kin_block_topk_select (the pages describe no
 * counterpart; it exists for callers, not for the method).
 *
 * For callers that cannot allocate device memory: code running under a host
 * that plans and owns all device memory up front (a runtime with a fixed
 * memory plan, a plugin that may not call cudaMalloc, a decode loop that
 * must never reach the allocator), or that has no workspace to pass.  It
 * computes exactly what kin_block_topk_select computes, with the same
 * kernels, but keeps its scratch (one fp32 score per block) in a fixed array
 * inside libkin.so: KIN_NOALLOC_SCRATCH_FLOATS floats (8 MiB) that every
 * GPU which loads the library holds until the process exits.
 *  - Requires batch * num_kv_heads * ceil(max_seq_len / block_size) <=
 *    KIN_NOALLOC_SCRATCH_FLOATS, else KIN_ERR_CAPACITY (nothing launched).
 *  - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *  - The first call on each device is a one-time set-up (it looks up the
 *    array's device address) and should come before any stream capture.
 *  - Every call shares the one array, which keeps the last call's contents;
 *    nothing in it needs to start at zero.  Calls whose kernels overlap on
 *    the GPU (other streams, other threads) race on it: serialize them.
 * Arguments, layouts and errors are those of kin_block_topk_select, without
 * the workspace. */
#define KIN_NOALLOC_SCRATCH_FLOATS (1 << 21)
kin_status kin_block_topk_select_noalloc(const kin_dims* dims, const void* q, const float* block_means,
                                         const int32_t* seq_lens, int32_t k_blocks, int32_t* sel_idx,
                                         int32_t* sel_cnt, int32_t* dev_status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* KIN_H */
