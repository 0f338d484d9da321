// Shapes, workspace layout and launch-parameter structs shared by the host
// API and the kernels of the CUDA path.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "mla_decode.h"

namespace mla {

constexpr int kDK = MLA_HEAD_DIM_K;       // 576: latent row = key
constexpr int kDV = MLA_HEAD_DIM_V;       // 512: first 512 columns = value
constexpr int kPage = MLA_PAGE_SIZE;      // 64 tokens per page = one key block
constexpr int kMetaInts = MLA_META_INTS;  // ints per scheduler partition
constexpr int kFixedOverhead = MLA_FIXED_OVERHEAD_BLOCKS;
constexpr int kTileRows = 128;            // query rows per MMA tile
constexpr int kMaxRows = 1024;            // s_q * h_q supported (8 row tiles)
constexpr int kMaxBatch = 16384;          // metadata kernel keeps lengths in smem

// Default limit of every pipeline wait in the kernels: ~2 s at 1.9 GHz.
constexpr long long kDefaultWaitCycles = 4000000000LL;

// Device-side error bits (sticky, OR-ed into the first word of the workspace).
constexpr int kDevErrTimeout = MLA_DEVERR_TIMEOUT;
constexpr int kDevErrPage = MLA_DEVERR_PAGE_INDEX;
constexpr int kDevErrAppendPos = MLA_DEVERR_APPEND_POS;

// Workspace: [ error words | lse partials | o partials ], each 256-B aligned.
constexpr size_t kWsHeader = 256;
__host__ __device__ inline size_t ws_align(size_t x) { return (x + 255) & ~size_t(255); }
__host__ __device__ inline size_t ws_max_chunks(int batch, int parts) { return size_t(batch) + size_t(parts); }
__host__ __device__ inline size_t ws_lse_offset() { return kWsHeader; }
__host__ __device__ inline size_t ws_o_offset(int batch, int rows, int parts) {
  return ws_align(kWsHeader + ws_max_chunks(batch, parts) * size_t(rows) * sizeof(float));
}
__host__ __device__ inline size_t ws_bytes(int batch, int rows, int parts) {
  return ws_o_offset(batch, rows, parts) + ws_max_chunks(batch, parts) * size_t(rows) * kDV * sizeof(float);
}

struct DecodeParams {
  const int32_t* block_table;
  int64_t block_table_stride;
  int64_t num_pages;
  const int32_t* cache_seqlens;
  const int32_t* meta;
  const int32_t* num_splits;
  void* out;        // [b, s_q, h_q, 512] in the input dtype
  float* lse;       // [b, h_q, s_q]
  float* lse_acc;   // [chunks, rows]
  float* o_acc;     // [chunks, rows, 512]
  int* err;         // sticky error word
  int batch, s_q, h_q, rows, m_tiles, num_parts;
  int causal;
  float scale_log2;  // softmax_scale * log2(e)
  long long wait_cycles;  // limit of every pipeline wait, in SM clock cycles
  int withhold_q_ready;   // test hook: 1 = the first chunk's "Q ready" arrival is never made
};

// Walks a partition's blocks in order: chunk after chunk (one chunk = the
// partition's blocks of one request), block after block.
struct Walk {
  int br, bk, er, ek;     // the partition's range from the scheduler
  int req, blk, lo, hi, n;
  int L;                  // cached tokens of the request
  int chunk;              // chunk index within the partition
  bool valid;

  __device__ __forceinline__ void seek(const DecodeParams& p, int from) {
    for (int r = from; r < p.batch && (r < er || (r == er && ek > 0)); ++r) {
      L = p.cache_seqlens[r];
      n = (L + kPage - 1) / kPage;
      lo = (r == br) ? bk : 0;
      hi = (r == er) ? ek : n;
      if (hi > lo) {
        req = r;
        blk = lo;
        valid = true;
        return;
      }
    }
    valid = false;
  }
  __device__ __forceinline__ void init(const DecodeParams& p, const int* meta) {
    br = meta[0];
    bk = meta[1];
    er = meta[2];
    ek = meta[3];
    chunk = 0;
    seek(p, br);
  }
  __device__ __forceinline__ void next(const DecodeParams& p) {
    if (++blk < hi) return;
    ++chunk;
    seek(p, req + 1);
  }
  // to the first block of the partition's next chunk
  __device__ __forceinline__ void next_chunk(const DecodeParams& p) {
    ++chunk;
    seek(p, req + 1);
  }
  __device__ __forceinline__ bool first() const { return blk == lo; }
  __device__ __forceinline__ bool last() const { return blk == hi - 1; }
};

}  // namespace mla
