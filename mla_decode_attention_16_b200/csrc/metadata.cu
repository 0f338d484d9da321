// Tile scheduler ("FlashMLA: 高性能GPU注意力机制计算库", section 6. SM资源调度优化;
// "FlashMLA 在 Hopper GPU 上的 MHA 内核调度优化解析", 辅助优化：可编程依赖启动与瓦片调度).
//
// Every request is n_b = ceil(L_b / 64) blocks of 64 tokens and each piece of
// a request costs a fixed overhead F = 5 blocks (loading Q, filling the
// pipeline, writing partials, merging).  The num_sm_parts partitions each get
// quota = ceil(sum_{n_b > 0}(n_b + F) / num_sm_parts) + F and take requests in
// order; a request whose remaining blocks plus F exceed what is left of the
// quota is cut (the partition takes left - F blocks if that is positive) and
// continues in the next partition.  The last partition takes whatever is left.
//
// One CTA: the lengths are staged in shared memory with coalesced loads, the
// total is a block reduction, then one thread walks the requests (a few cycles
// per request) and writes the [num_sm_parts, 8] table and the [batch + 1]
// chunk-count prefix sums.
#include "common.cuh"
#include "launch.h"

namespace mla {
namespace metadata {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) metadata_kernel(const int32_t* __restrict__ seqlens, int batch,
                                                            int num_parts, int32_t* __restrict__ meta,
                                                            int32_t* __restrict__ num_splits) {
  extern __shared__ int s_blocks[];
  __shared__ long long s_partial[kThreads / 32];
  long long local = 0;
  for (int i = threadIdx.x; i < batch; i += kThreads) {
    const int L = seqlens[i];
    const int n = L > 0 ? (L + kPage - 1) / kPage : 0;
    s_blocks[i] = n;
    if (n > 0) local += n + kFixedOverhead;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) local += __shfl_xor_sync(0xffffffffu, local, o);
  if ((threadIdx.x & 31) == 0) s_partial[threadIdx.x >> 5] = local;
  __syncthreads();
  if (threadIdx.x != 0) return;

  long long total = 0;
  for (int w = 0; w < kThreads / 32; ++w) total += s_partial[w];
  const long long quota = total > 0 ? (total + num_parts - 1) / num_parts + kFixedOverhead : 0;

  int r = 0, k = 0, split = 0, chunks = 0;
  num_splits[0] = 0;
  for (int part = 0; part < num_parts; ++part) {
    const int begin_r = r, begin_k = k, begin_split = split;
    long long left = quota;
    const bool last = part == num_parts - 1;
    while (r < batch) {
      const int n = s_blocks[r];
      if (n == 0) {
        num_splits[r + 1] = chunks;
        ++r;
        continue;
      }
      const long long need = static_cast<long long>(n - k) + kFixedOverhead;
      if (need <= left || last) {
        left -= need;
        chunks += split + 1;
        num_splits[r + 1] = chunks;
        ++r;
        k = 0;
        split = 0;
      } else {
        const long long take = left - kFixedOverhead;
        if (take > 0) {
          k += static_cast<int>(take);
          ++split;
        }
        break;
      }
    }
    int32_t* row = meta + part * kMetaInts;
    row[0] = begin_r;
    row[1] = begin_k;
    row[2] = r;
    row[3] = k;
    row[4] = begin_split;
    row[5] = 0;
    row[6] = 0;
    row[7] = 0;
  }
}

}  // namespace metadata

int metadata_smem_bytes(int batch) { return batch * static_cast<int>(sizeof(int)); }
const void* metadata_kernel_ptr() { return reinterpret_cast<const void*>(&metadata::metadata_kernel); }

cudaError_t launch_metadata(const int32_t* seqlens, int batch, int num_parts, int32_t* meta, int32_t* num_splits,
                            cudaStream_t stream) {
  metadata::metadata_kernel<<<1, metadata::kThreads, metadata_smem_bytes(batch), stream>>>(seqlens, batch, num_parts,
                                                                                            meta, num_splits);
  return cudaGetLastError();
}

}  // namespace mla
