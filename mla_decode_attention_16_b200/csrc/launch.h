// Host-side launchers of the CUDA path (defined next to each kernel).
#pragma once

#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace mla {

int splitkv_smem_bytes();
int splitkv_threads();
const void* splitkv_kernel_ptr(bool bf16);
// qrmap: 32-column boxes (64-byte swizzle) of q's columns 512..575; kmap: 64-column boxes (128-byte
// swizzle) of the cache; krmap: 32-column boxes (64-byte swizzle) of the cache.
cudaError_t launch_splitkv(bool bf16, const void* q, const CUtensorMap& qrmap, const CUtensorMap& kmap,
                           const CUtensorMap& krmap, const DecodeParams& p, cudaStream_t stream);
// Few-row kernel (s_q * h_q <= kNarrowMaxRows): one CTA per partition.
constexpr int kNarrowMaxRows = 32;
int narrow_rows_padded(int rows);
int narrow_smem_bytes(int np);
const void* narrow_kernel_ptr(bool bf16, int np);
cudaError_t launch_splitkv_narrow(bool bf16, const void* q, const CUtensorMap& kmap, const DecodeParams& p,
                                  cudaStream_t stream);
// Few-row kernel on a CTA pair (s_q * h_q <= kNarrowMaxRows): one cluster of 2 CTAs per partition.
int npair_smem_bytes(int np);
const void* npair_kernel_ptr(bool bf16, int np);
cudaError_t launch_splitkv_npair(bool bf16, const void* q, const CUtensorMap& kmap, const CUtensorMap& krmap,
                                 const DecodeParams& p, cudaStream_t stream);
// Split-KV kernel over an e5m2 cache, any row count: one CTA per (partition, 32-row tile).
// kmap: 128-column boxes (128-byte swizzle); krmap: the 64 columns 512..575 (64-byte swizzle).
int fp8_row_tiles(int rows);
int fp8_smem_bytes(int np);
const void* fp8_kernel_ptr(bool bf16, int np);
cudaError_t launch_splitkv_fp8(bool bf16, const void* q, const CUtensorMap& kmap, const CUtensorMap& krmap,
                               const DecodeParams& p, cudaStream_t stream);
// Split-KV kernel over an e5m2 cache for s_q * h_q > 32: two CTAs (value halves) per 128-row tile.
int fp8_rt_tiles(int rows);
int fp8_rt_smem_bytes();
const void* fp8_rt_kernel_ptr(bool bf16);
cudaError_t launch_splitkv_fp8_rt(bool bf16, const void* q, const CUtensorMap& kmap, const CUtensorMap& krmap,
                                  const DecodeParams& p, cudaStream_t stream);
cudaError_t launch_combine(bool bf16, const DecodeParams& p, cudaStream_t stream);
// Copies kv_new [batch, s_q, 576] into cache positions L_b - s_q + s (programmatic dependent launch).
cudaError_t launch_append(const void* kv_new, void* kcache, int64_t num_pages, const int32_t* block_table,
                          int64_t bt_stride, const int32_t* seqlens, int batch, int s_q, int* err,
                          cudaStream_t stream);
// Same positions as launch_append; kv_new (bf16 or fp16) is cast to e5m2 bytes (nearest even, saturating).
cudaError_t launch_append_fp8(bool bf16, const void* kv_new, void* kcache, int64_t num_pages,
                              const int32_t* block_table, int64_t bt_stride, const int32_t* seqlens, int batch,
                              int s_q, int* err, cudaStream_t stream);
int metadata_smem_bytes(int batch, int num_parts);
constexpr int kMaxParts = 1024;  // partitions the metadata kernel stages in shared memory
const void* metadata_kernel_ptr();
cudaError_t launch_metadata(const int32_t* seqlens, int batch, int num_parts, int32_t* meta, int32_t* num_splits,
                            cudaStream_t stream);
// Records a cudaError_t for mla_last_cuda_error() (per thread).
void set_last_cuda_error(int err);
// Every host-side check mla_decode_fwd makes, with nothing enqueued: MLA_OK or the status that
// mla_decode_fwd would return for these arguments before launching anything.
int check_decode_args(const void* q, const void* kcache, int64_t num_pages, const int32_t* block_table,
                      int64_t block_table_stride, const int32_t* cache_seqlens, int batch, int s_q, int h_q,
                      int dtype, float softmax_scale, int causal, const int32_t* tile_sched_metadata,
                      const int32_t* num_splits, int num_sm_parts, void* workspace, size_t workspace_bytes,
                      void* out, float* lse);

}  // namespace mla
