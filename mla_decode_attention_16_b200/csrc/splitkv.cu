// Split-KV MLA decode kernel for sm_100a.
//
// What it computes: for each chunk (request, range of 64-token blocks) that the
// tile scheduler gave to this partition, the attention of one 128-row tile of
// query rows (row = s * h_q + h) over the chunk's keys, with an online softmax
// ("FlashMLA 在 Hopper GPU 上的 MHA 内核调度优化解析", 跷跷板调度的数学重构: the
// running-max rescaling is exactly the standard softmax), writing out/lse for
// a request computed in one piece and (o, lse) partials otherwise
// (辅助优化：可编程依赖启动与瓦片调度: splitkv + combine).
//
// B200 design (the pages' Hopper seesaw split of O over two warpgroups is
// prior art; here the accumulators live in TMEM):
//  * A CTA pair (cluster of 2) owns one 128-row tile.  A 128 x 512 fp32 output
//    would fill all 512 TMEM columns of an SM, so CTA c keeps only its half
//    O[:, 256c : 256c+256] (256 columns) and computes PV for that half.
//  * The 576-deep Q.K^T contraction is split between the pair, so no MMA work
//    is duplicated: CTA c contracts columns 256c .. 256c+255 plus its half of
//    the 64 columns 512..575 (32 columns each).  The fp32 partial scores of a
//    64-key block go to the peer through distributed shared memory (st.async
//    completing on the peer's mbarrier); both CTAs then hold the same full
//    scores and run the same softmax, so their two O halves stay consistent.
//  * Each CTA TMA-loads 5 column boxes (64 cols = 128 B, 128-byte swizzle) of
//    Q and of every page: boxes at columns 256c + {0,64,128,192} and 512.  The
//    first four are also this CTA's V half (V = first 512 columns of K).
//  * Warp roles: warp 0 lane 0 = TMA producer; warp 1 = TMEM owner, lane 0
//    issues every tcgen05.mma; warps 4-7 = softmax / O correction / epilogue,
//    one thread per query row (TMEM lane quadrant = warp % 4).
//  * S = Q.K^T (M=128, N=64, K=16 x 18 steps, both operands K-major in smem);
//    O += P.V (M=128, N=256, K=16 x 4 steps, P from TMEM, V MN-major in smem).
//  * exp2 with log2(e) folded into the scale ("FlashMLA: 高性能GPU注意力机制计算库",
//    4. Softmax数值稳定性优化).
//  * EVICT_FIRST L2 policy on the page loads (细粒度流水线与缓存优化).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cmath>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace mla {
namespace splitkv {

using namespace ptx;

constexpr int kThreads = 256;
constexpr int kBlockN = kPage;              // keys per pipeline step
constexpr int kBoxes = 5;                   // column boxes per CTA
constexpr int kQBox = kTileRows * 128;      // 16 KB
constexpr int kKBox = kBlockN * 128;        // 8 KB
constexpr int kQBytes = kBoxes * kQBox;     // 80 KB
constexpr int kStageBytes = kBoxes * kKBox; // 40 KB
constexpr int kStages = 2;
constexpr int kXWarp = 32 * kBlockN * 4;    // 8 KB: 32 rows x 64 fp32 partial scores
constexpr int kXBytes = 4 * kXWarp;
constexpr int kQkSteps = 18;                // 288 contraction columns / 16

constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQBytes;
constexpr int kOffX = kOffK + kStages * kStageBytes;
constexpr int kOffBar = kOffX + kXBytes;

enum Bar {
  kKvFull = 0,
  kKvEmpty = kKvFull + kStages,
  kQFull = kKvEmpty + kStages,
  kQEmpty,
  kSFull,
  kSEmpty = kSFull + 2,
  kPFull = kSEmpty + 2,
  kPEmpty = kPFull + 2,
  kODone = kPEmpty + 2,  // one phase per PV: the O correction waits for the previous PV
  kOFinal,               // one phase per chunk: the epilogue waits for the chunk's last PV
  kOEmpty,
  kXFull,
  kXEmpty = kXFull + 4,
  kDrain = kXEmpty + 4,  // MMA thread: all of its tcgen05 ops have completed
  kNumBars
};
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemUsed = kOffMisc + 16;
constexpr int kSmemBytes = kSmemUsed + 1024;  // slack to align the base to 1024 B

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;    // 256 columns
constexpr uint32_t kColS = 256;  // 2 x 64 columns
constexpr uint32_t kColP = 384;  // 2 x 32 columns (16-bit pairs)

__device__ __forceinline__ int box_col(int i, int crank) { return i < 4 ? 256 * crank + 64 * i : 512; }

// The running maximum used as the exponent reference moves only when a new
// score exceeds it by more than 2^8 (log2 units): the exponentials then stay
// <= 256 (exact in fp32 and representable in bf16/fp16), O and the row sum are
// rescaled far less often, and the final out = O / l is unchanged because both
// always share the same reference.
constexpr float kRescaleThreshold = 8.0f;



template <bool kBF16>
__device__ __forceinline__ uint32_t pack2(float a, float b) {
  if constexpr (kBF16) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
  } else {
    __half2 v = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
  }
}

template <bool kBF16>
__global__ void __launch_bounds__(kThreads, 1)
    splitkv_pair_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                        const DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + kOffBar + 8 * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t crank = cluster_ctarank();
  const uint32_t peer = crank ^ 1u;
  const int pair = blockIdx.x >> 1;
  const int part = pair / p.m_tiles;
  const int mtile = pair % p.m_tiles;
  const int* meta = p.meta + part * kMetaInts;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      uint32_t cnt = 1;
      if (i == kSEmpty || i == kSEmpty + 1 || i == kPFull || i == kPFull + 1 || i == kOEmpty) cnt = 4;
      mbar_init(bar(i), cnt);
    }
    *abort_flag = 0;
    for (int w = 0; w < 4; ++w) mbar_arrive_expect_tx(bar(kXFull + w), kXWarp);  // arm phase 0
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 32 * 2) {
    prefetch_tmap(&qmap);
    prefetch_tmap(&kmap);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // launched as a programmatic dependent of the previous kernel in the stream (normally the
  // scheduler): everything above overlapped it; nothing it wrote is read before this wait
  pdl_wait_primary();
  if (threadIdx.x == 0) pdl_launch_dependents();

  const int br = meta[0], bk = meta[1], er = meta[2], ek = meta[3], bs = meta[4];
  const int R = p.rows;
  int* err = p.err;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t evict_first = policy_evict_first();
      uint32_t it = 0, chunk = 0;
      for (int req = br; req < p.batch && (req < er || (req == er && ek > 0)); ++req) {
        const int L = p.cache_seqlens[req];
        const int n = (L + kPage - 1) / kPage;
        const int lo = (req == br) ? bk : 0;
        const int hi = (req == er) ? ek : n;
        if (hi <= lo) continue;
        mbar_wait(bar(kQEmpty), (chunk & 1) ^ 1, abort_flag, err, kDevErrTimeout);
        mbar_arrive_expect_tx(bar(kQFull), kQBytes);
        const int row0 = req * R + mtile * kTileRows;
        for (int i = 0; i < kBoxes; ++i)
          tma_load_2d(sbase + kOffQ + i * kQBox, &qmap, bar(kQFull), box_col(i, crank), row0);
        const int32_t* bt = p.block_table + static_cast<int64_t>(req) * p.block_table_stride;
        for (int blk = lo; blk < hi; ++blk, ++it) {
          if (*abort_flag) break;
          const int st = it % kStages;
          mbar_wait(bar(kKvEmpty + st), ((it / kStages) & 1) ^ 1, abort_flag, err, kDevErrTimeout);
          int page = bt[blk];
          if (page < 0 || static_cast<int64_t>(page) >= p.num_pages) {
            atomicOr(err, kDevErrPage);
            atomicCAS(err + 1, 0, page == 0 ? -1 : page);
            page = 0;
          }
          MLA_TR(kTrProd, it);
          mbar_arrive_expect_tx(bar(kKvFull + st), kStageBytes);
          for (int i = 0; i < kBoxes; ++i)
            tma_load_3d_hint(sbase + kOffK + st * kStageBytes + i * kKBox, &kmap, bar(kKvFull + st),
                             box_col(i, crank), 0, page, evict_first);
        }
        ++chunk;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_f16(kBF16, kTileRows, kBlockN, false, false);
      constexpr uint32_t idesc_pv = idesc_f16(kBF16, kTileRows, 256, false, true);
      uint32_t it = 0, chunk = 0;
      auto issue_pv = [&](uint32_t itp, int jjp, bool last) {
        const int st = itp % kStages;
        const int b = itp & 1;
        if (jjp == 0) mbar_wait(bar(kOEmpty), (chunk & 1) ^ 1, abort_flag, err, kDevErrTimeout);
        mbar_wait(bar(kPFull + b), (itp >> 1) & 1, abort_flag, err, kDevErrTimeout);
        tc_fence_after();
        MLA_TR(kTrPv, itp);
        const uint32_t vbase = sbase + kOffK + st * kStageBytes;
        for (int kk = 0; kk < kBlockN / 16; ++kk) {
          // V rows 16kk..16kk+15: 8-key groups 1024 B apart, 64-column boxes 8 KB apart
          const uint64_t bdesc = smem_desc_sw128(vbase + kk * 2048, kKBox, 1024);
          umma_ts(tmem + kColO, tmem + kColP + 32 * b + 8 * kk, bdesc, idesc_pv, (jjp > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(bar(kKvEmpty + st));
        umma_commit(bar(kPEmpty + b));
        umma_commit(bar(kODone));
        if (last) umma_commit(bar(kOFinal));
      };
      for (int req = br; req < p.batch && (req < er || (req == er && ek > 0)); ++req) {
        const int L = p.cache_seqlens[req];
        const int n = (L + kPage - 1) / kPage;
        const int lo = (req == br) ? bk : 0;
        const int hi = (req == er) ? ek : n;
        if (hi <= lo) continue;
        const int nb = hi - lo;
        mbar_wait(bar(kQFull), chunk & 1, abort_flag, err, kDevErrTimeout);
        tc_fence_after();
        if (*abort_flag) break;
        for (int jj = 0; jj < nb; ++jj) {
          const uint32_t itc = it + jj;
          const int st = itc % kStages;
          const int b = itc & 1;
          mbar_wait(bar(kKvFull + st), (itc / kStages) & 1, abort_flag, err, kDevErrTimeout);
          mbar_wait(bar(kSEmpty + b), ((itc >> 1) & 1) ^ 1, abort_flag, err, kDevErrTimeout);
          tc_fence_after();
          MLA_TR(kTrQk, itc);
          const uint32_t kbase = sbase + kOffK + st * kStageBytes;
          for (int s = 0; s < kQkSteps; ++s) {
            const int box = s < 16 ? s / 4 : 4;
            const int kk = s < 16 ? s % 4 : 2 * static_cast<int>(crank) + (s - 16);
            const uint64_t adesc = smem_desc_sw128(sbase + kOffQ + box * kQBox + kk * 32, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(kbase + box * kKBox + kk * 32, 16, 1024);
            umma_ss(tmem + kColS + 64 * b, adesc, bdesc, idesc_qk, s > 0 ? 1u : 0u);
          }
          umma_commit(bar(kSFull + b));
          if (jj == nb - 1) umma_commit(bar(kQEmpty));
          if (jj > 0) issue_pv(itc - 1, jj - 1, false);
        }
        issue_pv(it + nb - 1, nb - 1, true);
        it += nb;
        ++chunk;
      }
      umma_commit(bar(kDrain));
      mbar_wait_drain(bar(kDrain), 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax / correction / epilogue
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const int row_g = mtile * kTileRows + row;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    float* xrow = reinterpret_cast<float*>(smem + kOffX + q4 * kXWarp + lane * (kBlockN * 4));
    const uint32_t xrow_remote = mapa(smem_u32(xrow), peer);
    const uint32_t xfull_remote = mapa(bar(kXFull + q4), peer);
    const uint32_t xempty_remote = mapa(bar(kXEmpty + q4), peer);
    const int sw = lane & 15;
    // a warp whose 32 rows are all padding (rows >= s_q * h_q) keeps the
    // barrier protocol but skips the math; its peer warp skips the same way
    const bool active = mtile * kTileRows + q4 * 32 < R;
    uint32_t it = 0, chunk = 0;
    for (int req = br; req < p.batch && (req < er || (req == er && ek > 0)); ++req) {
      const int L = p.cache_seqlens[req];
      const int n = (L + kPage - 1) / kPage;
      const int lo = (req == br) ? bk : 0;
      const int hi = (req == er) ? ek : n;
      if (hi <= lo) continue;
      const int nb = hi - lo;
      int limit = 0;
      if (row_g < R) {
        limit = p.causal ? L - (p.s_q - 1 - row_g / p.h_q) : L;
        limit = limit < 0 ? 0 : limit;
      }
      float m = -INFINITY, l = 0.f;  // m: exponent reference (log2 units), l: row sum relative to it
      for (int jj = 0; jj < nb; ++jj) {
        const uint32_t itc = it + jj;
        const int b = itc & 1;
        float x[64];
        mbar_wait(bar(kSFull + b), (itc >> 1) & 1, abort_flag, err, kDevErrTimeout);
        __syncwarp();  // reconverge before the warp-collective tcgen05.ld
        tc_fence_after();
        if (lane == 0) MLA_TR(kTrSmS, itc);
        if (active) {
          uint32_t r0[32], r1[32];
          tmem_ld32(t_lane + kColS + 64 * b, r0);
          tmem_ld32(t_lane + kColS + 64 * b + 32, r1);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            x[c] = __uint_as_float(r0[c]);
            x[32 + c] = __uint_as_float(r1[c]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kSEmpty + b));
        if (!active) {
          mbar_wait(bar(kPEmpty + b), ((itc >> 1) & 1) ^ 1, abort_flag, err, kDevErrTimeout);
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(kPFull + b));
          continue;
        }

        // exchange partial scores with the peer CTA (same rows, other half of the contraction)
        mbar_wait<true>(bar(kXEmpty + q4), (itc & 1) ^ 1, abort_flag, err, kDevErrTimeout);
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4) {
          const int pos = c4 ^ sw;
          st_async_v4(xrow_remote + pos * 16, xfull_remote, x[4 * c4], x[4 * c4 + 1], x[4 * c4 + 2], x[4 * c4 + 3]);
        }
        mbar_wait<true>(bar(kXFull + q4), itc & 1, abort_flag, err, kDevErrTimeout);
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4) {
          const int pos = c4 ^ sw;
          const float4 y = *reinterpret_cast<const float4*>(xrow + pos * 4);
          x[4 * c4] += y.x;
          x[4 * c4 + 1] += y.y;
          x[4 * c4 + 2] += y.z;
          x[4 * c4 + 3] += y.w;
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive_expect_tx(bar(kXFull + q4), kXWarp);  // arm the next phase first
          mbar_arrive_cluster(xempty_remote);               // then let the peer send again
          MLA_TR(kTrSmX, itc);
        }

        // online softmax in log2 units
        const int kbase = (lo + jj) * kBlockN;
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float t = (kbase + c < limit) ? x[c] * p.scale_log2 : -INFINITY;
          x[c] = t;
          mx = fmaxf(mx, t);
        }
        bool resc = false;
        float alpha = 1.f;
        if (mx > m + kRescaleThreshold) {  // also true when m is still -inf and a key is visible
          if (m > -INFINITY) {
            resc = true;
            alpha = ex2(m - mx);
          }
          m = mx;
        }
        const float base = (m == -INFINITY) ? 0.f : m;
        float sum = 0.f;
        uint32_t pk[32];
#pragma unroll
        for (int c2 = 0; c2 < 32; ++c2) {
          const float p0 = ex2(x[2 * c2] - base);
          const float p1 = ex2(x[2 * c2 + 1] - base);
          sum += p0 + p1;
          pk[c2] = pack2<kBF16>(p0, p1);
        }
        l = l * alpha + sum;

        mbar_wait(bar(kPEmpty + b), ((itc >> 1) & 1) ^ 1, abort_flag, err, kDevErrTimeout);
        __syncwarp();
        tc_fence_after();
        tmem_st32(t_lane + kColP + 32 * b, pk);
        if (__any_sync(0xffffffffu, resc && jj > 0)) {
          // O holds PV of blocks before this one (jj == 0 is overwritten by its own PV)
          mbar_wait(bar(kODone), (itc - 1) & 1, abort_flag, err, kDevErrTimeout);
          __syncwarp();
          tc_fence_after();
#pragma unroll 1
          for (int k = 0; k < 8; ++k) {
            uint32_t o[32];
            tmem_ld32(t_lane + kColO + 32 * k, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(t_lane + kColO + 32 * k, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          MLA_TR(kTrSmP, itc);
          mbar_arrive(bar(kPFull + b));
        }
      }

      // epilogue: normalise this CTA's O half and write it
      mbar_wait(bar(kOFinal), chunk & 1, abort_flag, err, kDevErrTimeout);
      __syncwarp();
      tc_fence_after();
      if (active) {
        const bool whole = (lo == 0 && hi == n);
        const int split_idx = (req == br) ? bs : 0;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const float lse_v = l > 0.f ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
        const int64_t chunk_row = whole ? 0 : (static_cast<int64_t>(p.num_splits[req] + split_idx) * R + row_g);
#pragma unroll 1
        for (int k = 0; k < 8; ++k) {
          uint32_t o[32];
          tmem_ld32(t_lane + kColO + 32 * k, o);
          tmem_wait_ld();
          if (row_g < R) {
            const int col = static_cast<int>(crank) * 256 + 32 * k;
            if (whole) {
              uint4* dst = reinterpret_cast<uint4*>(
                  reinterpret_cast<uint16_t*>(p.out) + (static_cast<int64_t>(req) * R + row_g) * kDV + col);
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                uint4 w;
                w.x = pack2<kBF16>(__uint_as_float(o[8 * v + 0]) * inv, __uint_as_float(o[8 * v + 1]) * inv);
                w.y = pack2<kBF16>(__uint_as_float(o[8 * v + 2]) * inv, __uint_as_float(o[8 * v + 3]) * inv);
                w.z = pack2<kBF16>(__uint_as_float(o[8 * v + 4]) * inv, __uint_as_float(o[8 * v + 5]) * inv);
                w.w = pack2<kBF16>(__uint_as_float(o[8 * v + 6]) * inv, __uint_as_float(o[8 * v + 7]) * inv);
                dst[v] = w;
              }
            } else {
              float4* dst = reinterpret_cast<float4*>(p.o_acc + chunk_row * kDV + col);
#pragma unroll
              for (int v = 0; v < 8; ++v)
                dst[v] = make_float4(__uint_as_float(o[4 * v]) * inv, __uint_as_float(o[4 * v + 1]) * inv,
                                     __uint_as_float(o[4 * v + 2]) * inv, __uint_as_float(o[4 * v + 3]) * inv);
            }
          }
        }
        if (crank == 0 && row_g < R) {
          if (whole) {
            const int s = row_g / p.h_q, h = row_g % p.h_q;
            p.lse[static_cast<int64_t>(req) * R + h * p.s_q + s] = lse_v;
          } else {
            p.lse_acc[chunk_row] = lse_v;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kOEmpty));
      it += nb;
      ++chunk;
    }
  }

  // ------------------------------------------------------------ teardown
  __syncwarp();  // lanes of the producer / MMA warps rejoin their elected lane
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer may still be writing into this CTA's shared memory until here
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace splitkv

int splitkv_smem_bytes() { return splitkv::kSmemBytes; }

const void* splitkv_kernel_ptr(bool bf16) {
  return bf16 ? reinterpret_cast<const void*>(&splitkv::splitkv_pair_kernel<true>)
              : reinterpret_cast<const void*>(&splitkv::splitkv_pair_kernel<false>);
}

cudaError_t launch_splitkv(bool bf16, const CUtensorMap& qmap, const CUtensorMap& kmap, const DecodeParams& p,
                           cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * p.num_parts * p.m_tiles);  // one cluster of 2 CTAs per (partition, row tile)
  cfg.blockDim = dim3(splitkv::kThreads);
  cfg.dynamicSmemBytes = splitkv::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (bf16) return cudaLaunchKernelEx(&cfg, splitkv::splitkv_pair_kernel<true>, qmap, kmap, p);
  return cudaLaunchKernelEx(&cfg, splitkv::splitkv_pair_kernel<false>, qmap, kmap, p);
}

}  // namespace mla
