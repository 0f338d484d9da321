// Tile scheduler ("FlashMLA: 高性能GPU注意力机制计算库", section 6. SM资源调度优化;
// "FlashMLA 在 Hopper GPU 上的 MHA 内核调度优化解析", 辅助优化：可编程依赖启动与瓦片调度).
//
// Every request is n_b = ceil(L_b / 64) blocks of 64 tokens, and each piece of
// work on a request costs a fixed overhead of F = 3 blocks (Q load, pipeline
// fill, epilogue, merge; on B200 a second piece in a partition measured about
// one block of extra time, and F = 3 gave the shortest memory-bound launches
// of F = 1, 3, 5, 8, 12).  The requests are laid end to end on a line of
// units -- F overhead units, then one unit per block -- and partition p of P
// owns the units [p*S, (p+1)*S) with the share S = ceil(total / P), so block k
// of request b belongs to partition (cum_b + F + k) / S.  A partition's work is
// its blocks plus F per piece; only its first piece can have its overhead
// units in the previous partition, so the work is at most S + F, which is the
// pages' per-partition quota ceil_div(total, num_sm_parts) + fixed overhead.
//
// Everything is data-parallel (one CTA of 1024 threads): two block-wide
// prefix sums (units per request, pieces per request) and one binary search
// per partition boundary, instead of a walk whose length grows with
// batch + partitions.
#include "common.cuh"
#include "launch.h"

namespace mla {
namespace metadata {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;

// Exclusive prefix sum over v[0..n) in place (block-wide, all threads call it); returns the total.
template <typename T>
__device__ long long block_exclusive_scan(T* v, int n, long long* warp_tot) {
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  const int per = (n + kThreads - 1) / kThreads;
  const int lo = min(n, t * per), hi = min(n, lo + per);
  long long s = 0;
  for (int i = lo; i < hi; ++i) s += v[i];
  long long incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[w] = incl;
  __syncthreads();
  if (w == 0) {
    long long wt = warp_tot[lane];
    long long wi = wt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    warp_tot[lane] = wi - wt;  // exclusive offset of each warp
    if (lane == 31) warp_tot[kWarps] = wi;
  }
  __syncthreads();
  long long run = warp_tot[w] + incl - s;
  for (int i = lo; i < hi; ++i) {
    const long long x = v[i];
    v[i] = static_cast<T>(run);
    run += x;
  }
  const long long total = warp_tot[kWarps];
  __syncthreads();
  return total;
}

__global__ void __launch_bounds__(kThreads, 1) metadata_kernel(const int32_t* __restrict__ seqlens, int batch,
                                                            int num_parts, int32_t* __restrict__ meta,
                                                            int32_t* __restrict__ num_splits) {
  // smem: unit offset of each request (cum, int64) [batch + 1], then blocks / pieces per request (int32)
  extern __shared__ long long s_dyn[];
  long long* s_cum = s_dyn;
  int* s_cnt = reinterpret_cast<int*>(s_dyn + batch + 1);
  __shared__ long long s_warp[kWarps + 1];
  // the split-KV kernel that follows may start its prologue now; it waits for this grid before reading
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // This kernel is itself launched as a programmatic dependent (normally of the previous decode's
  // combine kernel): it reads only the lengths before the wait below, and writes its outputs, which
  // the previous decode's kernels read, only after it.

  for (int i = threadIdx.x; i < batch; i += kThreads) {
    const int L = seqlens[i];
    const int n = L > 0 ? L / kPage + (L % kPage != 0) : 0;
    s_cum[i] = n > 0 ? static_cast<long long>(n) + kFixedOverhead : 0;
    s_cnt[i] = n;  // blocks, replaced by pieces below
  }
  __syncthreads();
  const long long total = block_exclusive_scan(s_cum, batch, s_warp);
  const long long share = total > 0 ? (total + num_parts - 1) / num_parts : 0;

  for (int i = threadIdx.x; i < batch; i += kThreads) {
    const long long n = s_cnt[i];
    long long pieces = 0;
    if (n > 0) {
      const long long first = s_cum[i] + kFixedOverhead;  // unit of block 0
      pieces = (first + n - 1) / share - first / share + 1;
    }
    s_cnt[i] = static_cast<int>(pieces);
  }
  __syncthreads();
  const long long total_pieces = block_exclusive_scan(s_cnt, batch, s_warp);
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the previous kernels in the stream are done
  for (int i = threadIdx.x; i < batch; i += kThreads) num_splits[i] = s_cnt[i];
  if (threadIdx.x == 0) num_splits[batch] = static_cast<int32_t>(total_pieces);

  // partition boundaries: unit x -> (last request with cum <= x, blocks of it before x), or (batch, 0)
  auto locate = [&](long long x) -> int2 {
    if (share == 0 || x >= total) return make_int2(batch, 0);
    int lo = 0, hi = batch - 1;  // largest r with s_cum[r] <= x (s_cum[0] = 0 <= x)
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_cum[mid] <= x)
        lo = mid;
      else
        hi = mid - 1;
    }
    const long long off = x - s_cum[lo] - kFixedOverhead;
    return make_int2(lo, off > 0 ? static_cast<int>(off) : 0);
  };
  for (int part = threadIdx.x; part < num_parts; part += kThreads) {
    const int2 b = locate(static_cast<long long>(part) * share);
    const int2 e = locate(static_cast<long long>(part + 1) * share);
    int bsplit = 0;
    if (b.y > 0) bsplit = part - static_cast<int>((s_cum[b.x] + kFixedOverhead) / share);
    int4* row = reinterpret_cast<int4*>(meta + part * kMetaInts);
    row[0] = make_int4(b.x, b.y, e.x, e.y);
    row[1] = make_int4(bsplit, 0, 0, 0);
  }
}

}  // namespace metadata

int metadata_smem_bytes(int batch, int num_parts) {
  (void)num_parts;
  return (batch + 1) * static_cast<int>(sizeof(long long) + sizeof(int));
}
const void* metadata_kernel_ptr() { return reinterpret_cast<const void*>(&metadata::metadata_kernel); }

cudaError_t launch_metadata(const int32_t* seqlens, int batch, int num_parts, int32_t* meta, int32_t* num_splits,
                            cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(metadata::kThreads);
  cfg.dynamicSmemBytes = metadata_smem_bytes(batch, num_parts);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, metadata::metadata_kernel, seqlens, batch, num_parts, meta, num_splits);
}

}  // namespace mla
