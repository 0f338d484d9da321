// C ABI of the paged MLA decode library (declarations and the contract of
// every call are in include/mla_decode.h).
//
// Host side only: argument checks, workspace carving, TMA descriptor encoding
// (the driver's cuTensorMapEncodeTiled, reached through
// cudaGetDriverEntryPoint so the library needs no -lcuda), and the launches.
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "launch.h"
#include "mla_decode.h"

namespace {

using namespace mla;

thread_local int g_last_cuda_error = 0;

int cuda_fail(cudaError_t e) {
  g_last_cuda_error = static_cast<int>(e);
  return MLA_ERR_CUDA;
}

struct DeviceInfo {
  bool ready = false;
  int sms = 0;
  int pairs = 0;   // co-resident clusters of 2 CTAs of the 128-row-tile kernel
  int npairs = 0;  // co-resident clusters of 2 CTAs of the few-row pair kernel
};
constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mutex;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// Test hook (mla_test_withhold_q_ready): read by every launch that follows.
std::atomic<int> g_withhold_q_ready{0};
// Kernel variant (mla_set_kernel_variant); MLA_KERNEL_AUTO picks by row count.
std::atomic<int> g_variant{MLA_KERNEL_AUTO};

// The split-KV kernel a call with `rows` = s_q * h_q query rows runs under `variant`
// (MLA_KERNEL_AUTO resolved), or -1 if that variant cannot take so many rows.
int kernel_for(int rows, int variant) {
  if (variant == MLA_KERNEL_AUTO) return rows <= kNarrowMaxRows ? MLA_KERNEL_FEW_ROWS_ONE_CTA : MLA_KERNEL_ROW_TILE_PAIR;
  if (variant != MLA_KERNEL_ROW_TILE_PAIR && rows > kNarrowMaxRows) return -1;
  return variant;
}
std::atomic<long long> g_wait_cycles{0};

int ensure_encode() {
  if (g_encode) return MLA_OK;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess) return cuda_fail(e);
  if (q != cudaDriverEntryPointSuccess || fn == nullptr) return cuda_fail(cudaErrorSymbolNotFound);
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return MLA_OK;
}

// One-time per-device setup: kernel attributes, SM count, cluster occupancy.
int ensure_device(int device) {
  if (device < 0 || device >= kMaxDevices) return MLA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo& d = g_dev[device];
  if (d.ready) return MLA_OK;
  int prev = 0;
  cudaError_t e = cudaGetDevice(&prev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (prev != device && (e = cudaSetDevice(device)) != cudaSuccess) return cuda_fail(e);
  int rc = MLA_OK;
  do {
    int major = 0, minor = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, device)) != cudaSuccess) {
      rc = cuda_fail(e);
      break;
    }
    if (major != 10 || minor != 0) {  // built for sm_100a only
      rc = MLA_ERR_UNSUPPORTED;
      break;
    }
    for (int bf = 0; bf < 2; ++bf) {
      const void* k = splitkv_kernel_ptr(bf == 1);
      if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, splitkv_smem_bytes())) !=
          cudaSuccess) {
        rc = cuda_fail(e);
        break;
      }
    }
    if (rc != MLA_OK) break;
    for (int bf = 0; bf < 2 && rc == MLA_OK; ++bf) {
      for (int np : {16, 32}) {
        if ((e = cudaFuncSetAttribute(narrow_kernel_ptr(bf == 1, np), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      narrow_smem_bytes(np))) != cudaSuccess) {
          rc = cuda_fail(e);
          break;
        }
      }
    }
    if (rc != MLA_OK) break;
    for (int bf = 0; bf < 2 && rc == MLA_OK; ++bf) {
      for (int np : {16, 32}) {
        if ((e = cudaFuncSetAttribute(fp8_kernel_ptr(bf == 1, np), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      fp8_smem_bytes(np))) != cudaSuccess) {
          rc = cuda_fail(e);
          break;
        }
      }
      if (rc == MLA_OK &&
          (e = cudaFuncSetAttribute(fp8_rt_kernel_ptr(bf == 1), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    fp8_rt_smem_bytes())) != cudaSuccess)
        rc = cuda_fail(e);
    }
    if (rc != MLA_OK) break;
    if ((e = cudaFuncSetAttribute(metadata_kernel_ptr(), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  metadata_smem_bytes(kMaxBatch, kMaxParts))) != cudaSuccess) {
      rc = cuda_fail(e);
      break;
    }
    for (int bf = 0; bf < 2 && rc == MLA_OK; ++bf) {
      for (int np : {16, 32}) {
        if ((e = cudaFuncSetAttribute(npair_kernel_ptr(bf == 1, np), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      npair_smem_bytes(np))) != cudaSuccess) {
          rc = cuda_fail(e);
          break;
        }
      }
    }
    if (rc != MLA_OK) break;
    // co-resident clusters of 2 CTAs of a kernel (fallback: the pair count implied by the SM count)
    auto clusters_of = [&](const void* kernel, int smem, int threads) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * 512);
      cfg.blockDim = dim3(threads);
      cfg.dynamicSmemBytes = smem;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      cudaError_t ce = cudaOccupancyMaxActiveClusters(&n, kernel, &cfg);
      if (ce != cudaSuccess || n <= 0) {
        (void)cudaGetLastError();
        n = d.sms / 2;
      }
      return n;
    };
    const int clusters = clusters_of(splitkv_kernel_ptr(true), splitkv_smem_bytes(), splitkv_threads());
    d.npairs = clusters_of(npair_kernel_ptr(true, 32), npair_smem_bytes(32), splitkv_threads());
    d.pairs = clusters;
    d.ready = true;
  } while (false);
  if (prev != device) cudaSetDevice(prev);
  return rc;
}

int current_device(int* dev) {
  cudaError_t e = cudaGetDevice(dev);
  return e == cudaSuccess ? MLA_OK : cuda_fail(e);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_rows(int s_q, int h_q) {
  if (s_q < 1 || h_q < 1) return MLA_ERR_INVALID_ARG;
  if (static_cast<long long>(s_q) * h_q > kMaxRows) return MLA_ERR_UNSUPPORTED;
  return MLA_OK;
}

// Box of box_cols x box_rows elements of q viewed as [rows_total, 576]; box_cols * 2 bytes must
// equal the swizzle span (64 columns with 128-byte swizzle, 32 with 64-byte swizzle).
int encode_2d_q(CUtensorMap* map, const void* q, int64_t rows_total, int box_rows, int box_cols,
                CUtensorMapSwizzle swizzle, bool bf16) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kDK), static_cast<cuuint64_t>(rows_total)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kDK) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                        const_cast<void*>(q), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    g_last_cuda_error = static_cast<int>(r);
    return MLA_ERR_CUDA;
  }
  return MLA_OK;
}

// Box of box_cols columns x one 64-token page of the cache viewed as [pages, 64, 576].
int encode_3d_k(CUtensorMap* map, const void* kc, int64_t num_pages, int box_cols, CUtensorMapSwizzle swizzle,
                bool bf16) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kDK), static_cast<cuuint64_t>(kPage),
                              static_cast<cuuint64_t>(num_pages)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kDK) * 2, static_cast<cuuint64_t>(kDK) * 2 * kPage};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(kPage), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                        const_cast<void*>(kc), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    g_last_cuda_error = static_cast<int>(r);
    return MLA_ERR_CUDA;
  }
  return MLA_OK;
}

// Box of box_cols columns x one 64-token page of an e5m2 cache viewed as [pages, 64, 576] bytes.
int encode_3d_k8(CUtensorMap* map, const void* kc, int64_t num_pages, int box_cols, CUtensorMapSwizzle swizzle) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kDK), static_cast<cuuint64_t>(kPage),
                              static_cast<cuuint64_t>(num_pages)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kDK), static_cast<cuuint64_t>(kDK) * kPage};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(kPage), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(kc), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    g_last_cuda_error = static_cast<int>(r);
    return MLA_ERR_CUDA;
  }
  return MLA_OK;
}

bool valid_dtype(int dtype) {
  const int base = dtype & ~MLA_KV_FP8_E5M2;
  return base == MLA_BF16 || base == MLA_FP16;
}
bool is_bf16(int dtype) { return (dtype & ~MLA_KV_FP8_E5M2) == MLA_BF16; }
bool is_kv8(int dtype) { return (dtype & MLA_KV_FP8_E5M2) != 0; }

// Shared checks + parameter packing of the forward calls.
int prepare(const int32_t* cache_seqlens, int batch, int s_q, int h_q, int dtype, int causal,
            const int32_t* meta, const int32_t* num_splits, int num_sm_parts, void* workspace,
            size_t workspace_bytes, void* out, float* lse, float softmax_scale, DecodeParams* p) {
  if (!cache_seqlens || !meta || !num_splits || !workspace || !out || !lse) return MLA_ERR_INVALID_ARG;
  if (batch < 1 || num_sm_parts < 1) return MLA_ERR_INVALID_ARG;
  if (batch > kMaxBatch) return MLA_ERR_UNSUPPORTED;
  int rc = check_rows(s_q, h_q);
  if (rc != MLA_OK) return rc;
  if (!valid_dtype(dtype)) return MLA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return MLA_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return MLA_ERR_INVALID_ARG;
  if (!aligned16(out) || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MLA_ERR_INVALID_ARG;
  const int rows = s_q * h_q;
  if (workspace_bytes < ws_bytes(batch, rows, num_sm_parts)) return MLA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p->cache_seqlens = cache_seqlens;
  p->meta = meta;
  p->num_splits = num_splits;
  p->out = out;
  p->lse = lse;
  p->err = reinterpret_cast<int*>(ws);
  p->lse_acc = reinterpret_cast<float*>(ws + ws_lse_offset());
  p->o_acc = reinterpret_cast<float*>(ws + ws_o_offset(batch, rows, num_sm_parts));
  p->batch = batch;
  p->s_q = s_q;
  p->h_q = h_q;
  p->rows = rows;
  p->m_tiles = (rows + kTileRows - 1) / kTileRows;
  p->num_parts = num_sm_parts;
  p->causal = causal;
  p->scale_log2 = softmax_scale * 1.4426950408889634f;
  const long long wc = g_wait_cycles.load();
  p->wait_cycles = wc > 0 ? wc : kDefaultWaitCycles;
  p->withhold_q_ready = g_withhold_q_ready.load();
  p->block_table = nullptr;
  p->block_table_stride = 0;
  p->num_pages = 0;
  return MLA_OK;
}

// Checks of the arguments only the split-KV kernel reads.
int check_cache_args(const void* q, const void* kcache, int64_t num_pages, const int32_t* block_table,
                     int64_t block_table_stride) {
  if (!q || !kcache || !block_table) return MLA_ERR_INVALID_ARG;
  if (num_pages < 1 || block_table_stride < 1) return MLA_ERR_INVALID_ARG;
  if (num_pages > (int64_t(1) << 31) - 1) return MLA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(kcache)) return MLA_ERR_INVALID_ARG;
  return MLA_OK;
}

int splitkv_impl(const void* q, const void* kcache, int64_t num_pages, const int32_t* block_table,
                 int64_t block_table_stride, const DecodeParams& base, int dtype, cudaStream_t stream) {
  int rc = check_cache_args(q, kcache, num_pages, block_table, block_table_stride);
  if (rc != MLA_OK) return rc;
  int dev = 0;
  rc = current_device(&dev);
  if (rc != MLA_OK) return rc;
  if ((rc = ensure_device(dev)) != MLA_OK) return rc;
  if ((rc = ensure_encode()) != MLA_OK) return rc;
  const bool bf16 = is_bf16(dtype);
  CUtensorMap qrmap, kmap, krmap;
  DecodeParams p = base;
  p.block_table = block_table;
  p.block_table_stride = block_table_stride;
  p.num_pages = num_pages;
  cudaError_t e;
  if (is_kv8(dtype)) {  // e5m2 cache: 128-column boxes (128-byte swizzle) + the 64 columns 512..575
    if ((rc = encode_3d_k8(&kmap, kcache, num_pages, 128, CU_TENSOR_MAP_SWIZZLE_128B)) != MLA_OK) return rc;
    if ((rc = encode_3d_k8(&krmap, kcache, num_pages, 64, CU_TENSOR_MAP_SWIZZLE_64B)) != MLA_OK) return rc;
    e = base.rows <= kNarrowMaxRows ? launch_splitkv_fp8(bf16, q, kmap, krmap, p, stream)
                                    : launch_splitkv_fp8_rt(bf16, q, kmap, krmap, p, stream);
    return e == cudaSuccess ? MLA_OK : cuda_fail(e);
  }
  const int kernel = kernel_for(base.rows, g_variant.load());
  if (kernel < 0) return MLA_ERR_UNSUPPORTED;
  if ((rc = encode_3d_k(&kmap, kcache, num_pages, 64, CU_TENSOR_MAP_SWIZZLE_128B, bf16)) != MLA_OK) return rc;
  if (kernel != MLA_KERNEL_FEW_ROWS_ONE_CTA) {  // the pair kernels split the columns 512..575 in 32-column boxes
    if ((rc = encode_3d_k(&krmap, kcache, num_pages, 32, CU_TENSOR_MAP_SWIZZLE_64B, bf16)) != MLA_OK) return rc;
  }
  if (kernel == MLA_KERNEL_ROW_TILE_PAIR) {  // ... and the row-tile kernel loads those of q by TMA too
    if ((rc = encode_2d_q(&qrmap, q, static_cast<int64_t>(base.batch) * base.rows, kTileRows, 32,
                          CU_TENSOR_MAP_SWIZZLE_64B, bf16)) != MLA_OK)
      return rc;
  }
  if (kernel == MLA_KERNEL_FEW_ROWS_ONE_CTA)
    e = launch_splitkv_narrow(bf16, q, kmap, p, stream);
  else if (kernel == MLA_KERNEL_FEW_ROWS_PAIR)
    e = launch_splitkv_npair(bf16, q, kmap, krmap, p, stream);
  else
    e = launch_splitkv(bf16, q, qrmap, kmap, krmap, p, stream);
  return e == cudaSuccess ? MLA_OK : cuda_fail(e);
}

}  // namespace

namespace mla {
void set_last_cuda_error(int err) { g_last_cuda_error = err; }

int check_decode_args(const void* q, const void* kcache, int64_t num_pages, const int32_t* block_table,
                      int64_t block_table_stride, const int32_t* cache_seqlens, int batch, int s_q, int h_q,
                      int dtype, float softmax_scale, int causal, const int32_t* tile_sched_metadata,
                      const int32_t* num_splits, int num_sm_parts, void* workspace, size_t workspace_bytes,
                      void* out, float* lse) {
  DecodeParams p;
  int rc = prepare(cache_seqlens, batch, s_q, h_q, dtype, causal, tile_sched_metadata, num_splits, num_sm_parts,
                   workspace, workspace_bytes, out, lse, softmax_scale, &p);
  if (rc != MLA_OK) return rc;
  return check_cache_args(q, kcache, num_pages, block_table, block_table_stride);
}
}  // namespace mla

extern "C" {

const char* mla_status_string(int status) {
  switch (status) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
    case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    default: return "MLA_ERR_UNKNOWN";
  }
}

int mla_last_cuda_error(void) { return g_last_cuda_error; }

int mla_version(void) { return 210; }

int mla_set_kernel_variant(int variant) {
  if (variant < MLA_KERNEL_AUTO || variant > MLA_KERNEL_ROW_TILE_PAIR) return MLA_ERR_INVALID_ARG;
  g_variant.store(variant);
  return MLA_OK;
}

int mla_get_kernel_variant(int rows) {
  if (rows < 1 || rows > kMaxRows) return -1;
  return kernel_for(rows, g_variant.load());
}

int mla_test_withhold_q_ready(int enable, long long wait_cycles) {
  if (enable != 0 && enable != 1) return MLA_ERR_INVALID_ARG;
  if (wait_cycles < 0) return MLA_ERR_INVALID_ARG;
  g_withhold_q_ready.store(enable);
  g_wait_cycles.store(wait_cycles);
  return MLA_OK;
}


int mla_get_num_sm_parts(int device, int rows, int* num_sm_parts) {
  if (!num_sm_parts || rows < 1) return MLA_ERR_INVALID_ARG;
  if (rows > kMaxRows) return MLA_ERR_UNSUPPORTED;
  int rc = ensure_device(device);
  if (rc != MLA_OK) return rc;
  const int kernel = kernel_for(rows, g_variant.load());
  if (kernel < 0) return MLA_ERR_UNSUPPORTED;
  if (kernel == MLA_KERNEL_FEW_ROWS_ONE_CTA) {  // one CTA per SM
    *num_sm_parts = g_dev[device].sms > 0 ? g_dev[device].sms : 1;
    return MLA_OK;
  }
  if (kernel == MLA_KERNEL_FEW_ROWS_PAIR) {  // one CTA pair per partition
    *num_sm_parts = g_dev[device].npairs > 0 ? g_dev[device].npairs : 1;
    return MLA_OK;
  }
  const int m_tiles = (rows + kTileRows - 1) / kTileRows;
  const int parts = g_dev[device].pairs / m_tiles;
  *num_sm_parts = parts > 0 ? parts : 1;
  return MLA_OK;
}

int mla_get_num_sm_parts_dtype(int device, int rows, int dtype, int* num_sm_parts) {
  if (!valid_dtype(dtype)) return MLA_ERR_INVALID_ARG;
  if (!is_kv8(dtype)) return mla_get_num_sm_parts(device, rows, num_sm_parts);
  if (!num_sm_parts || rows < 1) return MLA_ERR_INVALID_ARG;
  if (rows > kMaxRows) return MLA_ERR_UNSUPPORTED;
  int rc = ensure_device(device);
  if (rc != MLA_OK) return rc;
  // one CTA per SM: up to 32 rows one per partition, above that two per 128-row tile
  const int per_part = rows <= kNarrowMaxRows ? 1 : 2 * fp8_rt_tiles(rows);
  const int parts = g_dev[device].sms / per_part;
  *num_sm_parts = parts > 0 ? parts : 1;
  return MLA_OK;
}

int mla_get_workspace_size(int batch, int rows, int num_sm_parts, size_t* bytes) {
  if (!bytes || batch < 1 || rows < 1 || num_sm_parts < 1) return MLA_ERR_INVALID_ARG;
  if (batch > kMaxBatch || rows > kMaxRows) return MLA_ERR_UNSUPPORTED;
  *bytes = ws_bytes(batch, rows, num_sm_parts);
  return MLA_OK;
}

int mla_get_metadata(const int32_t* cache_seqlens, int batch, int rows, int num_sm_parts,
                     int32_t* tile_sched_metadata, int32_t* num_splits, void* stream) {
  if (!cache_seqlens || !tile_sched_metadata || !num_splits) return MLA_ERR_INVALID_ARG;
  if (batch < 1 || rows < 1 || num_sm_parts < 1) return MLA_ERR_INVALID_ARG;
  if (batch > kMaxBatch || rows > kMaxRows || num_sm_parts > kMaxParts) return MLA_ERR_UNSUPPORTED;
  int dev = 0;
  int rc = current_device(&dev);
  if (rc != MLA_OK) return rc;
  if ((rc = ensure_device(dev)) != MLA_OK) return rc;
  cudaError_t e = launch_metadata(cache_seqlens, batch, num_sm_parts, tile_sched_metadata, num_splits,
                                  static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MLA_OK : cuda_fail(e);
}

int mla_splitkv_fwd(const void* q, const void* kcache, int64_t num_pages, const int32_t* block_table,
                    int64_t block_table_stride, const int32_t* cache_seqlens, int batch, int s_q, int h_q,
                    int dtype, float softmax_scale, int causal, const int32_t* tile_sched_metadata,
                    const int32_t* num_splits, int num_sm_parts, void* workspace, size_t workspace_bytes,
                    void* out, float* lse, void* stream) {
  DecodeParams p;
  int rc = prepare(cache_seqlens, batch, s_q, h_q, dtype, causal, tile_sched_metadata, num_splits, num_sm_parts,
                   workspace, workspace_bytes, out, lse, softmax_scale, &p);
  if (rc != MLA_OK) return rc;
  return splitkv_impl(q, kcache, num_pages, block_table, block_table_stride, p, dtype,
                      static_cast<cudaStream_t>(stream));
}

int mla_combine_fwd(const int32_t* cache_seqlens, int batch, int s_q, int h_q, int dtype,
                    const int32_t* num_splits, int num_sm_parts, void* workspace, size_t workspace_bytes,
                    void* out, float* lse, void* stream) {
  DecodeParams p;
  // the scheduler table is not read by the combine; any non-null pointer passes the shared check
  int rc = prepare(cache_seqlens, batch, s_q, h_q, dtype, 0, num_splits, num_splits, num_sm_parts, workspace,
                   workspace_bytes, out, lse, 1.0f, &p);
  if (rc != MLA_OK) return rc;
  cudaError_t e = launch_combine(is_bf16(dtype), p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MLA_OK : cuda_fail(e);
}

int mla_decode_fwd(const void* q, const void* kcache, int64_t num_pages, const int32_t* block_table,
                   int64_t block_table_stride, const int32_t* cache_seqlens, int batch, int s_q, int h_q,
                   int dtype, float softmax_scale, int causal, const int32_t* tile_sched_metadata,
                   const int32_t* num_splits, int num_sm_parts, void* workspace, size_t workspace_bytes,
                   void* out, float* lse, void* stream) {
  DecodeParams p;
  int rc = prepare(cache_seqlens, batch, s_q, h_q, dtype, causal, tile_sched_metadata, num_splits, num_sm_parts,
                   workspace, workspace_bytes, out, lse, softmax_scale, &p);
  if (rc != MLA_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = splitkv_impl(q, kcache, num_pages, block_table, block_table_stride, p, dtype, st)) != MLA_OK) return rc;
  cudaError_t e = launch_combine(is_bf16(dtype), p, st);
  return e == cudaSuccess ? MLA_OK : cuda_fail(e);
}

int mla_append_kv(const void* kv_new, void* kcache, int64_t num_pages, const int32_t* block_table,
                  int64_t block_table_stride, const int32_t* cache_seqlens, int batch, int s_q, int dtype,
                  void* workspace, size_t workspace_bytes, void* stream) {
  if (!kv_new || !kcache || !block_table || !cache_seqlens || !workspace) return MLA_ERR_INVALID_ARG;
  if (batch < 1 || s_q < 1 || num_pages < 1 || block_table_stride < 1) return MLA_ERR_INVALID_ARG;
  if (batch > kMaxBatch || s_q > kMaxRows) return MLA_ERR_UNSUPPORTED;
  if (num_pages > (int64_t(1) << 31) - 1) return MLA_ERR_UNSUPPORTED;
  if (!valid_dtype(dtype)) return MLA_ERR_INVALID_ARG;
  if (!aligned16(kv_new) || !aligned16(kcache) || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return MLA_ERR_INVALID_ARG;
  if (workspace_bytes < kWsHeader) return MLA_ERR_WORKSPACE;
  cudaError_t e = is_kv8(dtype)
                      ? launch_append_fp8(is_bf16(dtype), kv_new, kcache, num_pages, block_table, block_table_stride,
                                          cache_seqlens, batch, s_q, static_cast<int*>(workspace),
                                          static_cast<cudaStream_t>(stream))
                      : launch_append(kv_new, kcache, num_pages, block_table, block_table_stride, cache_seqlens,
                                      batch, s_q, static_cast<int*>(workspace), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MLA_OK : cuda_fail(e);
}

int mla_decode_fwd_append(const void* q, const void* kv_new, void* kcache, int64_t num_pages,
                          const int32_t* block_table, int64_t block_table_stride, const int32_t* cache_seqlens,
                          int batch, int s_q, int h_q, int dtype, float softmax_scale, int causal,
                          const int32_t* tile_sched_metadata, const int32_t* num_splits, int num_sm_parts,
                          void* workspace, size_t workspace_bytes, void* out, float* lse, void* stream) {
  int rc = check_decode_args(q, kcache, num_pages, block_table, block_table_stride, cache_seqlens, batch, s_q, h_q,
                             dtype, softmax_scale, causal, tile_sched_metadata, num_splits, num_sm_parts, workspace,
                             workspace_bytes, out, lse);
  if (rc != MLA_OK) return rc;
  if (!kv_new || !aligned16(kv_new)) return MLA_ERR_INVALID_ARG;
  int dev = 0;
  if ((rc = current_device(&dev)) != MLA_OK) return rc;
  if ((rc = ensure_device(dev)) != MLA_OK) return rc;
  if ((rc = ensure_encode()) != MLA_OK) return rc;
  if ((rc = mla_append_kv(kv_new, kcache, num_pages, block_table, block_table_stride, cache_seqlens, batch, s_q,
                          dtype, workspace, workspace_bytes, stream)) != MLA_OK)
    return rc;
  return mla_decode_fwd(q, kcache, num_pages, block_table, block_table_stride, cache_seqlens, batch, s_q, h_q,
                        dtype, softmax_scale, causal, tile_sched_metadata, num_splits, num_sm_parts, workspace,
                        workspace_bytes, out, lse, stream);
}

int mla_read_device_status(const void* workspace, void* stream, int32_t* flags) {
  if (!workspace || !flags) return MLA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(flags, workspace, 2 * sizeof(int32_t), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  return e == cudaSuccess ? MLA_OK : cuda_fail(e);
}

}  // extern "C"
