// Append of the new tokens' latent rows to the paged cache, the step that
// precedes a decode ("FlashMLA: 高性能GPU注意力机制计算库", section 项目主要功能:
// the KV cache is paged, 64 tokens per block, addressed through a block table).
//
// cache_seqlens[b] = L counts the s_q new tokens of request b, so new token s
// (0-based) is cache position j = L - s_q + s: page block_table[b][j / 64],
// slot j % 64.  Each 576-wide row (1152 bytes) is copied by one warp with
// 16-byte stores (72 of them: 2 or 3 per lane).
//
// Launched as a programmatic dependent of the kernel before it in the stream
// (normally the tile scheduler): it may start early, but it waits for that
// kernel -- and so, through the chain, for the previous decode's kernels that
// read the cache -- before it reads or writes anything.  The split-KV kernel
// that follows is its programmatic dependent and waits for it before loading
// pages.
//
// Device data is bounds-checked: a page index outside [0, num_pages) or a
// position below 0 (L < s_q) skips the row and sets MLA_DEVERR_PAGE_INDEX /
// MLA_DEVERR_APPEND_POS in the error word.
#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace mla {
namespace append {

constexpr int kWarps = 4;
constexpr int kRowVec = kDK * 2 / 16;  // 72 16-byte pieces per row

__global__ void __launch_bounds__(kWarps * 32)
    append_kernel(const uint4* __restrict__ kv_new, uint4* __restrict__ kcache, int64_t num_pages,
                  const int32_t* __restrict__ block_table, int64_t bt_stride, const int32_t* __restrict__ seqlens,
                  int batch, int s_q, int* err) {
  ptx::pdl_launch_dependents();  // the split-KV kernel may set up now; it waits for this grid
  ptx::pdl_wait_primary();
  const int lane = threadIdx.x & 31;
  const int64_t rows = static_cast<int64_t>(batch) * s_q;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5); row < rows; row += nwarps) {
    const int b = static_cast<int>(row / s_q);
    const int s = static_cast<int>(row % s_q);
    const int pos = seqlens[b] - s_q + s;
    if (pos < 0) {
      if (lane == 0) atomicOr(err, kDevErrAppendPos);
      continue;
    }
    const int page = block_table[static_cast<int64_t>(b) * bt_stride + pos / kPage];
    if (page < 0 || static_cast<int64_t>(page) >= num_pages) {
      if (lane == 0) {
        atomicOr(err, kDevErrPage);
        atomicCAS(err + 1, 0, page == 0 ? -1 : page);
      }
      continue;
    }
    const uint4* src = kv_new + row * kRowVec;
    uint4* dst = kcache + (static_cast<int64_t>(page) * kPage + pos % kPage) * kRowVec;
#pragma unroll
    for (int i = lane; i < kRowVec; i += 32) dst[i] = __ldg(src + i);
  }
}

// Same rows and positions; each new value (bf16 or fp16) is cast to e5m2 (nearest even,
// saturating) and the row is stored as 576 bytes (72 8-byte stores per warp).
template <bool kBF16>
__global__ void __launch_bounds__(kWarps * 32)
    append_fp8_kernel(const uint4* __restrict__ kv_new, uint2* __restrict__ kcache, int64_t num_pages,
                      const int32_t* __restrict__ block_table, int64_t bt_stride, const int32_t* __restrict__ seqlens,
                      int batch, int s_q, int* err) {
  ptx::pdl_launch_dependents();
  ptx::pdl_wait_primary();
  const int lane = threadIdx.x & 31;
  const int64_t rows = static_cast<int64_t>(batch) * s_q;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5); row < rows; row += nwarps) {
    const int b = static_cast<int>(row / s_q);
    const int s = static_cast<int>(row % s_q);
    const int pos = seqlens[b] - s_q + s;
    if (pos < 0) {
      if (lane == 0) atomicOr(err, kDevErrAppendPos);
      continue;
    }
    const int page = block_table[static_cast<int64_t>(b) * bt_stride + pos / kPage];
    if (page < 0 || static_cast<int64_t>(page) >= num_pages) {
      if (lane == 0) {
        atomicOr(err, kDevErrPage);
        atomicCAS(err + 1, 0, page == 0 ? -1 : page);
      }
      continue;
    }
    const uint4* src = kv_new + row * kRowVec;
    uint2* dst = kcache + (static_cast<int64_t>(page) * kPage + pos % kPage) * kRowVec;
#pragma unroll
    for (int i = lane; i < kRowVec; i += 32) {
      const uint4 d = __ldg(src + i);
      dst[i] = make_uint2(ptx::cast4_e5m2<kBF16>(d.x, d.y), ptx::cast4_e5m2<kBF16>(d.z, d.w));
    }
  }
}

}  // namespace append

cudaError_t launch_append_fp8(bool bf16, const void* kv_new, void* kcache, int64_t num_pages,
                              const int32_t* block_table, int64_t bt_stride, const int32_t* seqlens, int batch,
                              int s_q, int* err, cudaStream_t stream) {
  const int64_t rows = static_cast<int64_t>(batch) * s_q;
  int64_t blocks = (rows + append::kWarps - 1) / append::kWarps;
  if (blocks > 2048) blocks = 2048;  // grid-stride loop beyond 8192 rows
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(append::kWarps * 32);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const uint4* src = static_cast<const uint4*>(kv_new);
  uint2* dst = static_cast<uint2*>(kcache);
  if (bf16)
    return cudaLaunchKernelEx(&cfg, append::append_fp8_kernel<true>, src, dst, num_pages, block_table, bt_stride,
                              seqlens, batch, s_q, err);
  return cudaLaunchKernelEx(&cfg, append::append_fp8_kernel<false>, src, dst, num_pages, block_table, bt_stride,
                            seqlens, batch, s_q, err);
}

cudaError_t launch_append(const void* kv_new, void* kcache, int64_t num_pages, const int32_t* block_table,
                          int64_t bt_stride, const int32_t* seqlens, int batch, int s_q, int* err,
                          cudaStream_t stream) {
  const int64_t rows = static_cast<int64_t>(batch) * s_q;
  int64_t blocks = (rows + append::kWarps - 1) / append::kWarps;
  if (blocks > 2048) blocks = 2048;  // grid-stride loop beyond 8192 rows
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(append::kWarps * 32);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, append::append_kernel, static_cast<const uint4*>(kv_new),
                            static_cast<uint4*>(kcache), num_pages, block_table, bt_stride, seqlens, batch, s_q,
                            err);
}

}  // namespace mla
