// Log-sum-exp combine of split-KV partials ("DeepSeek开源FlashMLA全解析", 2.1
// item 4 结果融合; "FlashMLA 在 Hopper GPU 上的 MHA 内核调度优化解析",
// 辅助优化：可编程依赖启动与瓦片调度: the combine kernel runs under programmatic
// dependent launch behind splitkv_mla, with no host synchronisation).
//
// For request b cut into C > 1 chunks, query row r:
//     lse = ln sum_c exp(lse_c),  out = sum_c exp(lse_c - lse) * o_c.
// Requests with C == 1 were written by the split-KV kernel; requests with no
// cached token (C == 0) get out = 0, lse = -inf here.
//
// One warp per query row, 128-bit loads: lane t reads columns 4t + 128k
// (k = 0..3) of each chunk's 512-wide fp32 row, so a warp reads 512 contiguous
// bytes per instruction.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cmath>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace mla {
namespace combine {

constexpr int kWarps = 4;

template <bool kBF16>
__device__ __forceinline__ void store4(void* out, int64_t idx, float a, float b, float c, float d) {
  if constexpr (kBF16) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
    uint2 v;
    v.x = *reinterpret_cast<uint32_t*>(&lo);
    v.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(out) + idx) = v;
  } else {
    __half2 lo = __floats2half2_rn(a, b), hi = __floats2half2_rn(c, d);
    uint2 v;
    v.x = *reinterpret_cast<uint32_t*>(&lo);
    v.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(reinterpret_cast<__half*>(out) + idx) = v;
  }
}

template <bool kBF16>
__global__ void __launch_bounds__(kWarps * 32) combine_kernel(const DecodeParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int row = blockIdx.x * kWarps + warp;
  const int R = p.rows;
  // The next kernel in the stream (normally the next decode's scheduler, which waits for this grid
  // before writing anything this one reads) may launch now.
  ptx::pdl_launch_dependents();
  // Everything read here (partials, and num_splits from the scheduler two launches back, which the
  // split-KV kernel itself waited for) is complete and visible once the split-KV grid is.
  ptx::pdl_wait_primary();
  const int c0 = p.num_splits[b];
  const int nc = p.num_splits[b + 1] - c0;
  if (row >= R || nc == 1) return;

  const int s = row / p.h_q, h = row % p.h_q;
  const int64_t out_row = (static_cast<int64_t>(b) * R + row) * kDV;
  float* lse_out = p.lse + static_cast<int64_t>(b) * R + h * p.s_q + s;

  float mx = -INFINITY;
  for (int c = 0; c < nc; ++c) mx = fmaxf(mx, p.lse_acc[static_cast<int64_t>(c0 + c) * R + row]);
  if (nc == 0 || mx == -INFINITY) {
#pragma unroll
    for (int k = 0; k < 4; ++k) store4<kBF16>(p.out, out_row + 4 * lane + 128 * k, 0.f, 0.f, 0.f, 0.f);
    if (lane == 0) *lse_out = -INFINITY;
    return;
  }
  float sum = 0.f;
  for (int c = 0; c < nc; ++c) sum += expf(p.lse_acc[static_cast<int64_t>(c0 + c) * R + row] - mx);
  const float lse = mx + logf(sum);

  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  for (int c = 0; c < nc; ++c) {
    const int64_t cr = static_cast<int64_t>(c0 + c) * R + row;
    const float w = expf(p.lse_acc[cr] - lse);
    const float4* src = reinterpret_cast<const float4*>(p.o_acc + cr * kDV);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float4 v = src[lane + 32 * k];
      acc[4 * k + 0] += w * v.x;
      acc[4 * k + 1] += w * v.y;
      acc[4 * k + 2] += w * v.z;
      acc[4 * k + 3] += w * v.w;
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k)
    store4<kBF16>(p.out, out_row + 4 * lane + 128 * k, acc[4 * k], acc[4 * k + 1], acc[4 * k + 2], acc[4 * k + 3]);
  if (lane == 0) *lse_out = lse;
}

}  // namespace combine

cudaError_t launch_combine(bool bf16, const DecodeParams& p, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((p.rows + combine::kWarps - 1) / combine::kWarps, p.batch);
  cfg.blockDim = dim3(combine::kWarps * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (bf16) return cudaLaunchKernelEx(&cfg, combine::combine_kernel<true>, p);
  return cudaLaunchKernelEx(&cfg, combine::combine_kernel<false>, p);
}

}  // namespace mla
