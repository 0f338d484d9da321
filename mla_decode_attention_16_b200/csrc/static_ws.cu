// mla_decode_fwd_static_ws: the decode forward without a caller-provided
// workspace.
//
// Some callers cannot allocate device memory at the point where they run the
// decode: a serving loop whose GPU memory is reserved up front by another
// allocator and cannot hand a raw buffer through this interface, or code that
// must not call cudaMalloc because cudaMalloc may synchronise the device and
// stall every stream.  For them the split-KV partials live in a fixed scratch
// array compiled into this library instead of in a workspace they pass in.
//
// The array below is a file-scope __device__ variable: every GPU that loads
// the library holds kStaticScratchBytes of it until the process exits.  Host
// code must not hand `g_static_scratch` to a kernel directly -- on the host that
// name is only a stand-in for the device variable (a kernel given it faults or,
// where the GPU can reach host memory, silently works on the wrong memory).
// The device address is looked up once per device with cudaGetSymbolAddress
// while that device is current, and that address is what the kernels receive.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "common.cuh"
#include "launch.h"
#include "mla_decode.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB per device
constexpr int kMaxScratchDevices = 64;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxScratchDevices] = {};

// Device address of the scratch array on the current device (looked up on the
// first call for that device, then cached).
int scratch_on_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    mla::set_last_cuda_error(static_cast<int>(e));
    return MLA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxScratchDevices) return MLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || p == nullptr) {
      mla::set_last_cuda_error(static_cast<int>(e != cudaSuccess ? e : cudaErrorInvalidSymbol));
      return MLA_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MLA_OK;
}

}  // namespace

extern "C" int mla_decode_fwd_static_ws(const void* q, const void* kcache, int64_t num_pages,
                                        const int32_t* block_table, int64_t block_table_stride,
                                        const int32_t* cache_seqlens, int batch, int s_q, int h_q, int dtype,
                                        float softmax_scale, int causal, const int32_t* tile_sched_metadata,
                                        const int32_t* num_splits, int num_sm_parts, void* out, float* lse,
                                        void* stream) {
  if (s_q < 1 || h_q < 1) return MLA_ERR_INVALID_ARG;
  if (static_cast<long long>(s_q) * h_q > mla::kMaxRows) return MLA_ERR_UNSUPPORTED;
  size_t need = 0;
  int rc = mla_get_workspace_size(batch, s_q * h_q, num_sm_parts, &need);
  if (rc != MLA_OK) return rc;
  if (need > kStaticScratchBytes) return MLA_ERR_WORKSPACE;  // larger than the built-in scratch
  void* scratch = nullptr;
  if ((rc = scratch_on_current_device(&scratch)) != MLA_OK) return rc;
  // Every check the forward makes runs before the header is cleared, so a rejected call enqueues
  // nothing (and leaves the error word of an earlier call untouched).
  rc = mla::check_decode_args(q, kcache, num_pages, block_table, block_table_stride, cache_seqlens, batch, s_q,
                              h_q, dtype, softmax_scale, causal, tile_sched_metadata, num_splits, num_sm_parts,
                              scratch, kStaticScratchBytes, out, lse);
  if (rc != MLA_OK) return rc;
  // The scratch keeps whatever the previous call left.  Only the error header
  // must start at zero; every partial is written before it is read.
  cudaError_t e = cudaMemsetAsync(scratch, 0, mla::kWsHeader, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    mla::set_last_cuda_error(static_cast<int>(e));
    return MLA_ERR_CUDA;
  }
  return mla_decode_fwd(q, kcache, num_pages, block_table, block_table_stride, cache_seqlens, batch, s_q, h_q,
                        dtype, softmax_scale, causal, tile_sched_metadata, num_splits, num_sm_parts, scratch,
                        kStaticScratchBytes, out, lse, stream);
}

extern "C" int mla_static_ws_read_device_status(void* stream, int32_t* flags) {
  if (!flags) return MLA_ERR_INVALID_ARG;
  void* scratch = nullptr;
  int rc = scratch_on_current_device(&scratch);
  if (rc != MLA_OK) return rc;
  return mla_read_device_status(scratch, stream, flags);
}
