/*
 * mla_decode.h -- C ABI of a B200 (sm_100a) paged MLA decode attention library.
 *
 * Operation (one latent KV head, "FlashMLA 在 Hopper GPU 上的 MHA 内核调度优化解析",
 * section 计算边界特性与优化方向抉择): every cached token is one row of d_k = 576
 * values; it is the key, and its first d_v = 512 values are the value.  For
 * request b with L_b cached tokens, query row (s, h):
 *     z_j   = softmax_scale * q[b,s,h,:] . K_j          (j visible)
 *     out   = sum_j exp(z_j) V_j / sum_j exp(z_j)
 *     lse   = ln sum_j exp(z_j)
 * Tokens live in 64-token pages addressed through a block table
 * ("FlashMLA: 高性能GPU注意力机制计算库" walk-through, section 项目主要功能:
 * paged KV cache, block size 64, BF16 and FP16).  With causal != 0 and s_q > 1,
 * query position s (0-based) sees keys j <= L_b - s_q + s (bottom-right
 * alignment); a row that sees no key gets out = 0 and lse = -inf.
 *
 * The work is split across the SMs by a tile scheduler (same walk-through,
 * section 6. SM资源调度优化; hotdry page section 辅助优化：可编程依赖启动与瓦片调度),
 * computed by a split-KV kernel, and the pieces of a request that was split are
 * merged by their log-sum-exp in a combine kernel launched with programmatic
 * dependent launch (same hotdry section; "DeepSeek开源FlashMLA全解析" 2.1 item 4,
 * 结果融合).
 *
 * Conventions for every call:
 *  - Pointers named "device" are CUDA device pointers on the current device;
 *    the caller owns every buffer.  The library allocates and frees nothing on
 *    these paths and keeps only a per-device cache of SM counts and kernel
 *    attributes.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls only
 *    enqueue work; none synchronises except mla_read_device_status and
 *    mla_static_ws_read_device_status.
 *  - Return value: MLA_OK (0) or an mla_status code.  Arguments are checked on
 *    the host before anything is enqueued; a failed check enqueues nothing.
 *    A failed CUDA launch returns MLA_ERR_CUDA and mla_last_cuda_error() gives
 *    the cudaError_t (per thread).
 *  - Device data (lengths, block table) is trusted for shape but bounds-checked
 *    in the kernels: a page index outside [0, num_pages) is replaced by page 0
 *    and MLA_DEVERR_PAGE_INDEX is OR-ed into the workspace's error word; a
 *    pipeline wait that exceeds ~2 s sets MLA_DEVERR_TIMEOUT and the kernel
 *    returns.  Kernels never trap.
 */
#ifndef MLA_DECODE_H_
#define MLA_DECODE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MLA_HEAD_DIM_K 576
#define MLA_HEAD_DIM_V 512
#define MLA_PAGE_SIZE 64
#define MLA_META_INTS 8
#define MLA_FIXED_OVERHEAD_BLOCKS 3

#define MLA_DEVERR_TIMEOUT 1
#define MLA_DEVERR_PAGE_INDEX 2
#define MLA_DEVERR_APPEND_POS 4 /* a request had fewer cached tokens than new ones */

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned pointer */
  MLA_ERR_UNSUPPORTED = 2, /* valid but outside what the kernels handle */
  MLA_ERR_WORKSPACE = 3,   /* workspace smaller than mla_get_workspace_size */
  MLA_ERR_CUDA = 4         /* a CUDA runtime call failed; see mla_last_cuda_error */
} mla_status;

typedef enum { MLA_BF16 = 0, MLA_FP16 = 1 } mla_dtype;

/*
 * FP8 cache ("云上AI推理新突破：FlashMLA赋能DeepSeek-V2-Lite提速16%", section
 * 3. 动态精度缩放; "DeepSeek开源FlashMLA全解析", section 1.2 计算模式创新): OR-ed
 * into the dtype argument of the decode, split-KV, combine and append calls
 * (MLA_BF16 | MLA_KV_FP8_E5M2, MLA_FP16 | MLA_KV_FP8_E5M2), it says that
 * kcache holds float8 e5m2 values, one byte each ([num_pages, 64, 1, 576]
 * bytes, 16-B aligned); q, kv_new and out keep the base dtype.  The decode
 * casts q to e5m2 (round to nearest even; finite values beyond 57344
 * saturate), forms q.K from the 8-bit values with fp32 accumulation, runs the
 * softmax in fp32, rounds P to fp16 and multiplies it by V widened to fp16
 * (exact).  The append casts each new value to e5m2 the same way.  Kernel
 * variants (mla_set_kernel_variant) do not apply: up to 32 query rows one CTA
 * per partition takes them; above that, two CTAs per tile of 128 rows, each
 * for half of the 512 output values.
 */
#define MLA_KV_FP8_E5M2 0x100

/* Human-readable name of a status code (static string). */
const char* mla_status_string(int status);

/* cudaError_t of the last failed CUDA call made by this thread (0 if none). */
int mla_last_cuda_error(void);

/* Library version as major*10000 + minor*100 + patch. */
int mla_version(void);

/*
 * Split-KV kernel variants.  Every variant computes the same result (within
 * rounding); they differ in how the work maps onto the SMs.
 *   MLA_KERNEL_AUTO              the default: the one-CTA few-row kernel for
 *                                s_q * h_q <= 32, the row-tile kernel above
 *   MLA_KERNEL_FEW_ROWS_ONE_CTA  rows <= 32: one CTA per partition loads whole
 *                                pages (three 72 KB stages)
 *   MLA_KERNEL_FEW_ROWS_PAIR     rows <= 32: a cluster of two CTAs per
 *                                partition, each loading and contracting half
 *                                of every page's columns and exchanging the
 *                                partial scores (five 36 KB stages per CTA)
 *   MLA_KERNEL_ROW_TILE_PAIR     any rows: a cluster of two CTAs per
 *                                partition and 128-row tile, each owning half
 *                                of the output columns
 */
#define MLA_KERNEL_AUTO 0
#define MLA_KERNEL_FEW_ROWS_ONE_CTA 1
#define MLA_KERNEL_FEW_ROWS_PAIR 2
#define MLA_KERNEL_ROW_TILE_PAIR 3

/*
 * Process-wide choice of the split-KV kernel variant for the calls that follow
 * (for tuning studies; the default, MLA_KERNEL_AUTO, needs no call).  The
 * partition count depends on the variant, so call mla_get_num_sm_parts and
 * mla_get_metadata again after changing it.  A forward call whose rows exceed
 * what the chosen variant handles returns MLA_ERR_UNSUPPORTED.
 * Returns MLA_ERR_INVALID_ARG for an unknown variant.  Host only.
 */
int mla_set_kernel_variant(int variant);

/* The variant (MLA_KERNEL_FEW_ROWS_ONE_CTA .. MLA_KERNEL_ROW_TILE_PAIR) a call
 * with `rows` = s_q * h_q would run now, or -1 if none can.  Host only. */
int mla_get_kernel_variant(int rows);

/*
 * Number of scheduler partitions for `rows` = s_q * h_q query rows per request
 * on `device` under the current kernel variant: one per SM for the one-CTA
 * few-row kernel, one per co-resident CTA pair for the few-row pair kernel,
 * and the co-resident CTA pairs divided by the number of 128-row tiles for the
 * row-tile kernel.  Host only; it queries the device's SM
 * count and cluster occupancy once and caches it.  rows must be in [1, 1024].
 */
int mla_get_num_sm_parts(int device, int rows, int* num_sm_parts);

/*
 * Bytes of workspace mla_decode_fwd needs for this batch, row count and
 * partition count: a 256-byte error header, then per-chunk fp32 lse partials
 * [batch + num_sm_parts, rows] and fp32 output partials
 * [batch + num_sm_parts, rows, 512].  The first 256 bytes must be zero before
 * the first call (they accumulate device error bits until the caller clears
 * them).  Host only.
 */
int mla_get_workspace_size(int batch, int rows, int num_sm_parts, size_t* bytes);

/*
 * mla_get_num_sm_parts for a given dtype argument: with MLA_KV_FP8_E5M2 set,
 * the e5m2-cache kernels run one CTA per SM: num_sm_parts = SMs for up to 32
 * query rows, SMs / (2 * ceil(rows / 128)) above (at least 1); without it, the
 * same as mla_get_num_sm_parts.  Any num_sm_parts >= 1 gives correct
 * results; this one fills the GPU once.
 */
int mla_get_num_sm_parts_dtype(int device, int rows, int dtype, int* num_sm_parts);

/*
 * Tile scheduler ("FlashMLA: 高性能GPU注意力机制计算库", section 6. SM资源调度优化).
 *   cache_seqlens        device int32 [batch]: cached tokens per request (>= 0)
 *   batch                1 .. 16384
 *   rows                 s_q * h_q (used only to validate against num_sm_parts)
 *   num_sm_parts         from mla_get_num_sm_parts
 *   tile_sched_metadata  device int32 [num_sm_parts, 8], written: per partition
 *                        begin_req, begin_block, end_req, end_block (exclusive,
 *                        lexicographic over (request, 64-token block)),
 *                        begin_split, 0, 0, 0
 *   num_splits           device int32 [batch + 1], written: prefix sums of the
 *                        number of chunks each request is cut into
 * Blocks n_b = ceil(L_b / 64).  Requests are laid end to end on a line of
 * units (F = MLA_FIXED_OVERHEAD_BLOCKS = 3 units of fixed overhead, then one
 * unit per block); with the share S = ceil(sum_{n_b>0}(n_b + F) / P),
 * partition p owns units [p*S, (p+1)*S), so its work (blocks + F per piece)
 * is at most S + F, the walk-through's
 * ceil_div(total, num_sm_parts) + fixed overhead.
 * Enqueues one single-CTA kernel on `stream` (data-parallel: prefix sums and
 * one binary search per partition) as a programmatic dependent launch: it may
 * start while the previous kernel in the stream finishes, reads cache_seqlens
 * right away, and writes its two outputs only after that kernel has completed.
 * So cache_seqlens must be final before the previous kernel lets dependents
 * start early (kernels that do not use programmatic dependent launch let them
 * start only when they complete; this library's combine kernel lets them
 * start at once and never writes cache_seqlens).
 */
int mla_get_metadata(const int32_t* cache_seqlens, int batch, int rows, int num_sm_parts,
                     int32_t* tile_sched_metadata, int32_t* num_splits, void* stream);

/*
 * Decode forward: split-KV kernel, then the log-sum-exp combine kernel, each a
 * programmatic dependent launch of the kernel before it (it sets up while that
 * kernel finishes and waits for it before reading anything it wrote).
 *   q                 device [batch, s_q, h_q, 576], dtype, contiguous, 16-B aligned
 *   kcache            device [num_pages, 64, 1, 576], dtype, contiguous, 16-B aligned
 *   num_pages         pages in kcache (>= 1)
 *   block_table       device int32 [batch, block_table_stride]; entry p of
 *                     request b is the page holding its tokens 64p .. 64p+63
 *   block_table_stride  elements between rows of block_table (>= 1)
 *   cache_seqlens     device int32 [batch], the same values given to mla_get_metadata
 *   batch, s_q, h_q   s_q * h_q in [1, 1024]
 *   dtype             MLA_BF16 or MLA_FP16 (q, kcache and out share it), optionally
 *                     | MLA_KV_FP8_E5M2 (kcache holds e5m2 bytes; see above)
 *   softmax_scale     multiplies q.k (finite)
 *   causal            0 or 1 (see the header comment)
 *   tile_sched_metadata, num_splits, num_sm_parts   from mla_get_metadata
 *   workspace         device, >= mla_get_workspace_size bytes, 256-B aligned
 *   out               device [batch, s_q, h_q, 512], dtype, 16-B aligned (written)
 *   lse               device fp32 [batch, h_q, s_q] (written; note heads before
 *                     query positions)
 * Calls that overlap on the GPU must not share a workspace.
 */
int mla_decode_fwd(const void* q, const void* kcache, int64_t num_pages, const int32_t* block_table,
                   int64_t block_table_stride, const int32_t* cache_seqlens, int batch, int s_q, int h_q,
                   int dtype, float softmax_scale, int causal, const int32_t* tile_sched_metadata,
                   const int32_t* num_splits, int num_sm_parts, void* workspace, size_t workspace_bytes,
                   void* out, float* lse, void* stream);

/*
 * Append of the s_q new tokens' latent rows to the paged cache, the step that
 * precedes the decode ("FlashMLA: 高性能GPU注意力机制计算库", section 项目主要功能:
 * paged cache of 64-token blocks).
 *   kv_new            device [batch, s_q, 576], dtype, contiguous, 16-B aligned:
 *                     the new tokens' rows (key = all 576 values, value = the
 *                     first 512)
 *   kcache            device [num_pages, 64, 1, 576], written in place
 *   cache_seqlens     device int32 [batch]: L_b, counting the new tokens, so
 *                     new token s goes to position L_b - s_q + s, i.e. page
 *                     block_table[b, (L_b - s_q + s) / 64], slot (.. % 64)
 *   workspace         device, >= 256 bytes, 256-B aligned: its error word gets
 *                     MLA_DEVERR_PAGE_INDEX (page outside [0, num_pages); the
 *                     row is skipped) or MLA_DEVERR_APPEND_POS (L_b < s_q; the
 *                     rows without a position are skipped)
 * Every other argument as in mla_decode_fwd.  Rows of different requests must
 * not share a slot.  Enqueues one kernel as a programmatic dependent launch: it
 * sets up while the previous kernel in the stream finishes and writes nothing
 * before that kernel has completed.
 */
int mla_append_kv(const void* kv_new, void* kcache, int64_t num_pages, const int32_t* block_table,
                  int64_t block_table_stride, const int32_t* cache_seqlens, int batch, int s_q, int dtype,
                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * The decode step fused with the append: mla_append_kv, then the split-KV and
 * combine kernels of mla_decode_fwd, each a programmatic dependent launch of
 * the one before on `stream` (the split-KV kernel reads pages only after the
 * append has completed).  Arguments as in mla_decode_fwd and mla_append_kv;
 * kcache is written.  Checks run before anything is enqueued.
 */
int mla_decode_fwd_append(const void* q, const void* kv_new, void* kcache, int64_t num_pages,
                          const int32_t* block_table, int64_t block_table_stride, const int32_t* cache_seqlens,
                          int batch, int s_q, int h_q, int dtype, float softmax_scale, int causal,
                          const int32_t* tile_sched_metadata, const int32_t* num_splits, int num_sm_parts,
                          void* workspace, size_t workspace_bytes, void* out, float* lse, void* stream);

/*
 * The two stages of mla_decode_fwd, exposed for timing and testing; same
 * arguments and checks.  mla_splitkv_fwd writes out/lse of every request that
 * was not cut and the partials of the others; mla_combine_fwd merges the
 * partials (lse = ln sum_c exp(lse_c), out = sum_c exp(lse_c - lse) o_c) and
 * writes zeros / -inf for requests with no cached token.  mla_combine_fwd uses
 * programmatic dependent launch, so it may start while the split-KV kernel
 * drains; it waits for it before reading partials.
 */
int mla_splitkv_fwd(const void* q, const void* kcache, int64_t num_pages, const int32_t* block_table,
                    int64_t block_table_stride, const int32_t* cache_seqlens, int batch, int s_q, int h_q,
                    int dtype, float softmax_scale, int causal, const int32_t* tile_sched_metadata,
                    const int32_t* num_splits, int num_sm_parts, void* workspace, size_t workspace_bytes,
                    void* out, float* lse, void* stream);
int mla_combine_fwd(const int32_t* cache_seqlens, int batch, int s_q, int h_q, int dtype,
                    const int32_t* num_splits, int num_sm_parts, void* workspace, size_t workspace_bytes,
                    void* out, float* lse, void* stream);

/*
 * Decode forward for callers that cannot allocate device memory where they
 * run it -- e.g. a serving loop whose GPU memory is reserved up front by
 * another allocator, or code that must not call cudaMalloc because it may
 * synchronise the device -- and so have no workspace to pass.  The pages
 * describe no counterpart; this is a convenience of this library.
 * Same arguments, checks and results as mla_decode_fwd, minus the workspace:
 * the partials go to a 32 MiB scratch array built into the library (every GPU
 * that loads the library keeps it until the process exits).  Calls needing
 * more than 32 MiB of workspace (mla_get_workspace_size) return
 * MLA_ERR_WORKSPACE without launching; allocates nothing (no cudaMalloc,
 * cudaFree or allocating library call).  The first call on a device looks up
 * the scratch array's device address (cudaGetSymbolAddress) and caches it;
 * make that first call before any stream capture.  All calls share the one
 * scratch array, which keeps the previous call's contents (its error header is
 * cleared at the start of every call), so calls that may overlap on the GPU --
 * on different streams, or on the same device from different threads without
 * ordering -- race and must not be issued.  The cached address assumes the
 * device is not reset (cudaDeviceReset) while the library stays loaded.
 * Device-side errors of a call go to the scratch's error header:
 * mla_static_ws_read_device_status reads them until the next call clears it.
 */
int mla_decode_fwd_static_ws(const void* q, const void* kcache, int64_t num_pages, const int32_t* block_table,
                             int64_t block_table_stride, const int32_t* cache_seqlens, int batch, int s_q,
                             int h_q, int dtype, float softmax_scale, int causal,
                             const int32_t* tile_sched_metadata, const int32_t* num_splits, int num_sm_parts,
                             void* out, float* lse, void* stream);

/*
 * Companion of mla_decode_fwd_static_ws (no counterpart in the pages either):
 * copies the error word (MLA_DEVERR_* bits) and the first offending page index
 * of the built-in scratch on the current device to host `flags[2]`, i.e. the
 * device status of the last mla_decode_fwd_static_ws call on that device;
 * synchronises `stream`.  Does not clear them.
 */
int mla_static_ws_read_device_status(void* stream, int32_t* flags);

/*
 * Test hook for the kernels' bounded waits (no counterpart in the pages; never
 * needed in production).  With enable = 1, every split-KV launch that follows
 * (from any thread of the process) leaves out one software arrival -- the
 * "query rows are in tensor memory" signal of the partition's first chunk -- so
 * the pipeline stage waiting for it gives up after its wait limit, records
 * MLA_DEVERR_TIMEOUT in the workspace's error word and the kernel returns
 * (its outputs are then undefined).  wait_cycles > 0 sets the limit of every
 * pipeline wait in SM clock cycles for those launches (0 = the default of about
 * 2 s).  mla_test_withhold_q_ready(0, 0) restores normal operation.
 * Returns MLA_ERR_INVALID_ARG for enable outside {0, 1} or wait_cycles < 0.
 */
int mla_test_withhold_q_ready(int enable, long long wait_cycles);

/*
 * Copy the workspace's error word (MLA_DEVERR_* bits) and the first offending
 * page index to host `flags[2]`; synchronises `stream`.  Does not clear them.
 */
int mla_read_device_status(const void* workspace, void* stream, int32_t* flags);

#ifdef __cplusplus
}
#endif

#endif /* MLA_DECODE_H_ */
