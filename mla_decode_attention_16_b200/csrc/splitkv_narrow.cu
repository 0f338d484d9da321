// Split-KV MLA decode kernel for requests with few query rows (s_q * h_q <= 32).
//
// Same computation as the pair kernel (splitkv.cu): per chunk of 64-token
// pages, scores, online softmax ("FlashMLA 在 Hopper GPU 上的 MHA 内核调度优化解析",
// 跷跷板调度的数学重构: rescaled accumulation equals the plain softmax), PV,
// and out/lse or fp32 partials for the combine (辅助优化：可编程依赖启动与瓦片调度).
//
// With <= 32 query rows the decode is bound by HBM (the cost model of
// 计算边界特性与优化方向抉择: intensity ~ 2 * h_q * s_q FLOP/B), so the goal is
// to stream pages at full bandwidth with one CTA per SM and no traffic between
// SMs.  Per 64-token page:
//   S [rows x 64 keys] = Q . K^T       (M = 128 lanes, A = Q resident in TMEM,
//                                       B = the page's key box in smem; 36 MMAs)
//   O [rows x 512]    += P . V         (weight-stationary MMA, M = 32 rows,
//                                       N = 256 values per half, A = P in smem,
//                                       B = MN-major view of the page's first 8
//                                       column boxes; 8 MMAs)
// Every tcgen05.mma up to N = 128 costs the same ~70 cycles, so the instruction
// count bounds this kernel: the M = 32 form does P.V in 8 instructions of ~87
// cycles where 4 tiles of transposed M = 128 products take 16 of ~82.  With
// M = 32 the output sits in 128 TMEM columns over all four lane quadrants
// (lane r of quadrant q: row r, values 256h + 64q .. +63 of half h).
// TMEM: O 128 columns, S 64 columns, Q 288 columns (576 16-bit values per
// row).  Q of even chunks lives in lane quadrant 0 and of odd chunks in
// quadrant 1, so the next chunk's Q is written while the current chunk runs
// (the Q.K^T MMA computes all 128 lanes; rows outside the current quadrant are
// ignored).
//
// Roles (384 threads): warp 0 lane 0 issues the page loads and the P.V MMAs,
// whichever is ready first; warp 1 TMEM owner, lane 0 issues the Q.K^T MMAs;
// warps 4-7: warp 4 + (chunk & 1) runs the softmax of a chunk (one thread per
// query row), all four rescale O when a row's exponent reference moves; warps
// 8-11 write each chunk's epilogue, and warps 8 / 9 load Q for even / odd
// chunks.  With one thread issuing both products, a page's P.V had to wait
// behind the next page's Q.K^T, holding the page's 72 KB stage that much
// longer; with P.V on its own issuer it goes as soon as P is written
// (tcgen05.commit tracks the issuing thread's own MMAs, so each issuer commits
// its own barriers).  The load thread polls both queues without blocking, so a
// free stage is refilled at once and no softmax warp stalls to issue MMAs.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cmath>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace mla {
namespace narrow {

using namespace ptx;

constexpr int kThreads = 384;
constexpr int kBoxes = kDK / 64;              // 9 column boxes of 64 columns (128 B)
constexpr int kKBox = kPage * 128;            // 8 KB: one page x 64 columns
constexpr int kStageBytes = kBoxes * kKBox;   // 72 KB: one page
constexpr int kStages = 3;
constexpr int kQCols = kDK / 2;               // 288 TMEM columns of packed 16-bit pairs
constexpr float kRescaleThreshold = 8.0f;     // see splitkv.cu

enum Bar {
  kKvFull = 0,
  kKvEmpty = kKvFull + kStages,
  kQFull = kKvEmpty + kStages,  // [2] Q rows of a chunk parity written to TMEM
  kQEmpty = kQFull + 2,         // [2] last Q.K^T of a chunk of that parity completed
  kSFull = kQEmpty + 2,
  kSEmpty,
  kPFull,                       // [2]
  kPEmpty = kPFull + 2,         // [2]
  kODone = kPEmpty + 2,         // one phase per PV
  kOFinal,                      // [2] one phase per chunk using that O buffer
  kOEmpty = kOFinal + 2,        // [2] epilogue finished reading that O buffer
  kStats = kOEmpty + 2,         // [2] row sums / reference maxima of a chunk parity in smem
  kDrain = kStats + 2,          // Q.K^T issuer's tensor-core work drained
  kDrainPV,                     // P.V issuer's tensor-core work drained
  kNumBars
};

template <int NP>
struct Layout {
  static constexpr int kOBufs = 1;
  static constexpr int kOffK = 0;
  static constexpr int kOffP = kOffK + kStages * kStageBytes;  // 1024-aligned
  static constexpr int kPBytes = 32 * 128;                     // P: 32 rows (M of the P.V MMA) x 64 keys
  static constexpr int kOffRed = kOffP + 2 * kPBytes;
  // floats: alpha [2][NP], flag [2], row sums [2][NP], reference max [2][NP]
  static constexpr int kRedFloats = 2 * NP + 2 + 2 * NP + 2 * NP;
  static constexpr int kOffBar = (kOffRed + kRedFloats * 4 + 7) / 8 * 8;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 8 + sizeof(WaitCtl) + 1024;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColO = 0;     // O: 2 halves of 256 values x 64 columns (see umma_ws_ss)
  static constexpr uint32_t kColS = kColO + kOBufs * 128;
  static constexpr uint32_t kColQ = kColS + kPage;
  static_assert(kColQ + kQCols <= kTmemCols, "TMEM budget");
};

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

// One chunk of a partition: blocks [lo, hi) of request req (n blocks in all).
struct Chunk {
  int req, lo, hi, n, L, split;
};

// Next non-empty chunk at or after request `req` of the partition (req advanced past it).
__device__ __forceinline__ bool next_chunk(const DecodeParams& p, int br, int bk, int er, int ek, int bs, int& req,
                                           Chunk& c) {
  for (; req < p.batch && (req < er || (req == er && ek > 0)); ++req) {
    const int L = p.cache_seqlens[req];
    const int n = (L + kPage - 1) / kPage;
    const int lo = (req == br) ? bk : 0;
    const int hi = (req == er) ? ek : n;
    if (hi <= lo) continue;
    c = Chunk{req, lo, hi, n, L, req == br ? bs : 0};
    ++req;
    return true;
  }
  return false;
}

template <bool kBF16, int NP>
__global__ void __launch_bounds__(kThreads, 1)
    splitkv_narrow_kernel(const void* __restrict__ qptr, const __grid_constant__ CUtensorMap kmap,
                          const DecodeParams p) {
  using Lay = Layout<NP>;
  constexpr int kOBufs = Lay::kOBufs;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + Lay::kOffBar + 8 * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kOffMisc);
  WaitCtl* wctl = reinterpret_cast<WaitCtl*>(smem + Lay::kOffMisc + 8);
  float* s_alpha = reinterpret_cast<float*>(smem + Lay::kOffRed);          // [2][NP]
  volatile int* s_flag = reinterpret_cast<volatile int*>(s_alpha + 2 * NP);  // [2]
  float* s_lsum = s_alpha + 2 * NP + 2;                                   // [2][NP]
  float* s_mref = s_lsum + 2 * NP;                                        // [2][NP]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int part = blockIdx.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      const bool four = i == kPFull || i == kPFull + 1 || i == kOEmpty || i == kOEmpty + 1;
      mbar_init(bar(i), four ? 4u : 1u);
    }
    wctl->abort = 0;
    wctl->limit = p.wait_cycles;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), Lay::kTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 64) prefetch_tmap(&kmap);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // launched as a programmatic dependent of the previous kernel in the stream (normally the
  // scheduler): the prologue above overlapped it; nothing it wrote is read before this wait
  pdl_wait_primary();
  if (threadIdx.x == 0) pdl_launch_dependents();

  const int* meta = p.meta + part * kMetaInts;
  const int br = meta[0], bk = meta[1], er = meta[2], ek = meta[3], bs = meta[4];
  const int R = p.rows;
  int* err = p.err;

  // O[:, 256h ..] += P[:, 16kk ..] . V[16kk .., 256h ..] for page itp (chunk-relative index jjp of
  // chunk `chunk`), issued by the load thread once the four softmax warps have released P.  A = P (32
  // rows, K-major), B = V (MN-major view of the page's column boxes 4h .. 4h+3, 8 KB apart; 16 keys
  // = 2 x 1 KB).  Its commit also frees the page stage: the page's Q.K^T, issued by the other
  // thread, completed before its softmax could write P.
  auto issue_pv = [&](uint32_t itp, int jjp, bool last, uint32_t chunk) {
    constexpr uint32_t idesc_pv = idesc_f16(kBF16, 32, 256, false, true);
    const int st = itp % kStages;
    const int b = itp & 1;
    const int ob = chunk % kOBufs;
    if (jjp == 0) mbar_wait(bar(kOEmpty + ob), ((chunk / kOBufs) & 1) ^ 1, wctl, err, kDevErrTimeout);
    mbar_wait(bar(kPFull + b), (itp >> 1) & 1, wctl, err, kDevErrTimeout);
    tc_fence_after();
    const uint32_t kst = sbase + Lay::kOffK + st * kStageBytes;
    const uint32_t pbuf = sbase + Lay::kOffP + b * Lay::kPBytes;
    const uint32_t dcol = tmem + Lay::kColO + ob * 128;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int kk = 0; kk < kPage / 16; ++kk) {
        const uint64_t adesc = smem_desc_sw128(pbuf + kk * 32, 16, 1024);
        const uint64_t bdesc = smem_desc_sw128(kst + (4 * h) * kKBox + kk * 2048, kKBox, 1024);
        umma_ws_ss(dcol + 64 * h, adesc, bdesc, idesc_pv, (jjp > 0 || kk > 0) ? 1u : 0u);
      }
    }
    umma_commit(bar(kKvEmpty + st));
    umma_commit(bar(kPEmpty + b));
    umma_commit(bar(kODone));
    if (last) umma_commit(bar(kOFinal + ob));
  };

  if (warp == 0) {
    // ------------------------------------------------------------ page loads and P.V issue
    if (lane == 0) {
      const uint64_t evict_first = policy_evict_first();
      Walk wl, wp;
      wl.init(p, meta);
      wp = wl;
      uint32_t tl = 0, tp = 0;
      auto pv_ready = [&]() {
        // the same O-buffer phase that issue_pv waits for
        if (wp.first() && !mbar_test_wait(bar(kOEmpty + wp.chunk % kOBufs), ((wp.chunk / kOBufs) & 1) ^ 1))
          return false;
        return mbar_test_wait(bar(kPFull + (tp & 1)), (tp >> 1) & 1);
      };
      auto issue_load = [&]() {
        const int st = tl % kStages;
        int page = p.block_table[static_cast<int64_t>(wl.req) * p.block_table_stride + wl.blk];
        if (page < 0 || static_cast<int64_t>(page) >= p.num_pages) {
          atomicOr(err, kDevErrPage);
          atomicCAS(err + 1, 0, page == 0 ? -1 : page);
          page = 0;
        }
        mbar_arrive_expect_tx(bar(kKvFull + st), kStageBytes);
        for (int i = 0; i < kBoxes; ++i)
          tma_load_3d_hint(sbase + Lay::kOffK + st * kStageBytes + i * kKBox, &kmap, bar(kKvFull + st), 64 * i, 0,
                           page, evict_first);
        wl.next(p);
        ++tl;
      };
      long long idle_since = clock64();
      uint32_t polls = 0;
      while (wp.valid) {
        if (wl.valid && mbar_test_wait(bar(kKvEmpty + tl % kStages), ((tl / kStages) & 1) ^ 1)) {
          issue_load();
        } else if (tp < tl && pv_ready()) {
          issue_pv(tp, wp.first() ? 0 : 1, wp.last(), static_cast<uint32_t>(wp.chunk));
          wp.next(p);
          ++tp;
        } else {
          if ((++polls & 15u) == 0) {
            if (aborted(wctl)) break;
            if (clock64() - idle_since > wctl->limit) {
              raise_abort(wctl);
              atomicOr(err, kDevErrTimeout);
              break;
            }
          }
          continue;
        }
        idle_since = clock64();
      }
      // Before the CTA can exit, every page load issued above must have landed and every P.V
      // issued here must have completed: bounded waits, abort or not (a phase already consumed
      // has completed, so the wait returns at once; only an abort leaves one pending).
      for (uint32_t j = tl > kStages ? tl - kStages : 0; j < tl; ++j)
        mbar_wait_drain(bar(kKvFull + j % kStages), (j / kStages) & 1, wctl->limit);
      umma_commit(bar(kDrainPV));
      mbar_wait_drain(bar(kDrainPV), 0, wctl->limit);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ Q.K^T issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_f16(kBF16, 128, kPage, false, false);
      uint32_t it = 0, chunk = 0;
      int cur = br;
      Chunk ch;
      while (!aborted(wctl) && next_chunk(p, br, bk, er, ek, bs, cur, ch)) {
        const int nb = ch.hi - ch.lo;
        const int qpar = chunk & 1;
        mbar_wait(bar(kQFull + qpar), (chunk >> 1) & 1, wctl, err, kDevErrTimeout);
        tc_fence_after();
        for (int jj = 0; jj < nb; ++jj) {
          const uint32_t itc = it + jj;
          const int st = itc % kStages;
          mbar_wait(bar(kKvFull + st), (itc / kStages) & 1, wctl, err, kDevErrTimeout);
          mbar_wait(bar(kSEmpty), (itc & 1) ^ 1, wctl, err, kDevErrTimeout);
          tc_fence_after();
          const uint32_t kst = sbase + Lay::kOffK + st * kStageBytes;
          // fully unrolled: the descriptors become constants plus the stage base, which keeps this
          // single issuing thread -- the kernel's bottleneck -- at ~1 MMA per tcgen05.mma slot
#pragma unroll
          for (int i = 0; i < kBoxes; ++i) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const int s = 4 * i + kk;
              const uint64_t bdesc = smem_desc_sw128(kst + i * kKBox + kk * 32, 16, 1024);
              umma_ts(tmem + Lay::kColS, tmem + Lay::kColQ + 8 * s, bdesc, idesc_qk, s > 0 ? 1u : 0u);
            }
          }
          umma_commit(bar(kSFull));
          if (jj == nb - 1) umma_commit(bar(kQEmpty + qpar));
        }
        it += nb;
        ++chunk;
      }
      umma_commit(bar(kDrain));
      mbar_wait_drain(bar(kDrain), 0, wctl->limit);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ softmax (one warp per chunk) + O rescale + P.V issue
    const int q4 = warp & 3;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const int r = lane;
    // With 16 query rows, lanes r and r + 16 share row r: the Q loader writes every row into both
    // halves of its lane quadrant, so S holds each row twice and each lane takes 32 of its 64 keys
    // (half the work and registers of one lane per row); the row's maximum and sum combine over
    // the pair with one shuffle each.
    constexpr int kSplit = NP == 16 ? 2 : 1;
    constexpr int kKeys = kPage / kSplit;  // keys per lane
    const int row = kSplit == 2 ? (lane & 15) : lane;
    const int half = kSplit == 2 ? (lane >> 4) : 0;
    uint32_t it = 0, chunk = 0;
    int cur = br;
    Chunk ch;
    while (next_chunk(p, br, bk, er, ek, bs, cur, ch)) {
      const int nb = ch.hi - ch.lo;
      const int par = chunk & 1;
      const bool smx = q4 == par;  // warp 4 for even chunks, warp 5 for odd ones (lane quadrant = parity)
      const int ob = chunk % kOBufs;
      int limit = 0;
      if (smx && row < R) {
        limit = p.causal ? ch.L - (p.s_q - 1 - row / p.h_q) : ch.L;
        limit = limit < 0 ? 0 : limit;
      }
      float m = -INFINITY, l = 0.f;
      for (int jj = 0; jj < nb; ++jj) {
        const uint32_t itc = it + jj;
        const int b = itc & 1;
        if (smx) {
          mbar_wait(bar(kSFull), itc & 1, wctl, err, kDevErrTimeout);
          __syncwarp();
          tc_fence_after();
          float x[kKeys];
          {
            // tcgen05.ld takes one column address for the whole warp: every lane loads both
            // 32-column halves and keeps its own (all 64 columns when a lane owns a whole row)
            uint32_t v0[32], v1[32];
            tmem_ld32(t_lane + Lay::kColS, v0);
            tmem_ld32(t_lane + Lay::kColS + 32, v1);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              if constexpr (kKeys == 64) {
                x[c] = __uint_as_float(v0[c]);
                x[32 + c] = __uint_as_float(v1[c]);
              } else {
                x[c] = __uint_as_float(half ? v1[c] : v0[c]);
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(kSEmpty));

          const int kbase = (ch.lo + jj) * kPage + kKeys * half;
          float mx = -INFINITY;
#pragma unroll
          for (int c = 0; c < kKeys; ++c) {
            const float t = (kbase + c < limit) ? x[c] * p.scale_log2 : -INFINITY;
            x[c] = t;
            mx = fmaxf(mx, t);
          }
          if constexpr (kSplit == 2) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
          bool resc = false;
          float alpha = 1.f;
          if (mx > m + kRescaleThreshold) {
            if (m > -INFINITY && jj > 0) {
              resc = true;
              alpha = ex2(m - mx);
            }
            m = mx;
          }
          const float base = (m == -INFINITY) ? 0.f : m;
          float sum = 0.f;
          uint32_t pk[kKeys / 2];
#pragma unroll
          for (int c2 = 0; c2 < kKeys / 2; ++c2) {
            const float p0 = ex2(x[2 * c2] - base);
            const float p1 = ex2(x[2 * c2 + 1] - base);
            sum += p0 + p1;
            pk[c2] = pack2<kBF16>(p0, p1);
          }
          l = l * alpha + sum;  // this lane's keys of the row
          const bool any_resc = __any_sync(0xffffffffu, resc);
          if (half == 0 && row < NP) s_alpha[b * NP + row] = alpha;
          if (lane == 0) s_flag[b] = any_resc ? 1 : 0;
          mbar_wait(bar(kPEmpty + b), ((itc >> 1) & 1) ^ 1, wctl, err, kDevErrTimeout);
          if (row < NP) {
            // P row: 64 keys = 128 bytes, 16-byte chunks XOR-swizzled by row (128-byte swizzle);
            // this lane's keys are chunks (kKeys / 8) * half ..
            uint8_t* prow = smem + Lay::kOffP + b * Lay::kPBytes + row * 128;
#pragma unroll
            for (int k = 0; k < kKeys / 8; ++k)
              *reinterpret_cast<uint4*>(prow + ((((kKeys / 8) * half + k) ^ (row & 7)) << 4)) =
                  make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
          }
          fence_proxy_async_smem();  // P is read by the tensor core (async proxy)
        }
        named_bar_sync(1, 128);
        if (s_flag[b] && jj > 0) {
          mbar_wait(bar(kODone), (itc - 1) & 1, wctl, err, kDevErrTimeout);
          __syncwarp();
          tc_fence_after();
          // lane r of every quadrant holds row r: 64 columns of each half of its values
          const float a = r < NP ? s_alpha[b * NP + r] : 1.f;
#pragma unroll 1
          for (int c32 = 0; c32 < 4; ++c32) {
            uint32_t o[32];
            const uint32_t col = Lay::kColO + ob * 128 + 32 * c32;
            tmem_ld32(t_lane + col, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * a);
            tmem_st32(t_lane + col, o);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kPFull + b));
      }
      if (smx) {
        // this stats slot was last used by chunk - 2; with two O buffers its epilogue may still
        // be reading it (with one buffer the MMA order already guarantees it finished)
        if (kOBufs == 2 && chunk >= 2)
          mbar_wait(bar(kOEmpty + par), ((chunk >> 1) & 1) ^ 1, wctl, err, kDevErrTimeout);
        float lrow = l;
        if constexpr (kSplit == 2) lrow += __shfl_xor_sync(0xffffffffu, l, 16);
        if (half == 0 && row < NP) {
          s_lsum[par * NP + row] = lrow;
          s_mref[par * NP + row] = m;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kStats + par));
      }
      it += nb;
      ++chunk;
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ Q loads (warps 8 / 9) and epilogue (8-11)
    const int q4 = warp & 3;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const int r = lane;
    auto load_q = [&](const Chunk& c, uint32_t idx) {
      // Q rows of chunk idx into lane quadrant idx & 1 (this warp's quadrant)
      mbar_wait(bar(kQEmpty + (idx & 1)), ((idx >> 1) & 1) ^ 1, wctl, err, kDevErrTimeout);
      __syncwarp();
      tc_fence_after();
      // with 16 rows, lanes r and r + 16 both hold row r (see the softmax)
      const int qr = NP == 16 ? (r & 15) : r;
      const uint4* qrow = reinterpret_cast<const uint4*>(
          reinterpret_cast<const uint16_t*>(qptr) + (static_cast<int64_t>(c.req) * R + (qr < R ? qr : 0)) * kDK);
#pragma unroll 1
      for (int c32 = 0; c32 < kQCols / 32; ++c32) {
        uint32_t w[32];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          uint4 d = make_uint4(0, 0, 0, 0);
          if (qr < R) d = __ldg(qrow + c32 * 8 + v);
          w[4 * v] = d.x;
          w[4 * v + 1] = d.y;
          w[4 * v + 2] = d.z;
          w[4 * v + 3] = d.w;
        }
        tmem_st32(t_lane + Lay::kColQ + 32 * c32, w);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && !(p.withhold_q_ready && idx == 0)) mbar_arrive(bar(kQFull + (idx & 1)));
    };
    auto epilogue = [&](const Chunk& c, uint32_t idx) {
      const int ob = idx % kOBufs;
      const int par = idx & 1;
      mbar_wait(bar(kOFinal + ob), (idx / kOBufs) & 1, wctl, err, kDevErrTimeout);
      mbar_wait(bar(kStats + par), (idx >> 1) & 1, wctl, err, kDevErrTimeout);
      __syncwarp();
      tc_fence_after();
      const bool whole = (c.lo == 0 && c.hi == c.n);
      const int64_t chunk0 = whole ? 0 : static_cast<int64_t>(p.num_splits[c.req] + c.split) * R;
      const float* ls = s_lsum + par * NP;
      // lane r of quadrant q4 holds row r, values 256h + 64 q4 + (0..63) of each half h
      const float lr = r < NP ? ls[r] : 0.f;
      const float inv = lr > 0.f ? 1.f / lr : 0.f;
#pragma unroll 1
      for (int c32 = 0; c32 < 4; ++c32) {
        uint32_t o[32];
        tmem_ld32(t_lane + Lay::kColO + ob * 128 + 32 * c32, o);
        tmem_wait_ld();
        if (r < R) {
          const int d = (c32 >> 1) * 256 + q4 * 64 + (c32 & 1) * 32;
          if (whole) {
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.out) +
                                                  (static_cast<int64_t>(c.req) * R + r) * kDV + d);
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
            float4* dst = reinterpret_cast<float4*>(p.o_acc + (chunk0 + r) * kDV + d);
#pragma unroll
            for (int v = 0; v < 8; ++v)
              dst[v] = make_float4(__uint_as_float(o[4 * v]) * inv, __uint_as_float(o[4 * v + 1]) * inv,
                                   __uint_as_float(o[4 * v + 2]) * inv, __uint_as_float(o[4 * v + 3]) * inv);
          }
        }
      }
      if (q4 == 0 && r < R) {
        const float lr = ls[r];
        const float lse_v = lr > 0.f ? (s_mref[par * NP + r] + log2f(lr)) * 0.69314718055994531f : -INFINITY;
        if (whole) {
          const int s = r / p.h_q, h = r % p.h_q;
          p.lse[static_cast<int64_t>(c.req) * R + h * p.s_q + s] = lse_v;
        } else {
          p.lse_acc[chunk0 + r] = lse_v;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kOEmpty + ob));
    };
    int cur = br;
    Chunk ch, nx;
    bool have = next_chunk(p, br, bk, er, ek, bs, cur, ch);
    if (have && q4 == 0) load_q(ch, 0);
    uint32_t chunk = 0;
    while (have) {
      const bool more = next_chunk(p, br, bk, er, ek, bs, cur, nx);
      if (more && q4 == static_cast<int>((chunk + 1) & 1)) load_q(nx, chunk + 1);  // overlaps this chunk
      epilogue(ch, chunk);
      ch = nx;
      have = more;
      ++chunk;
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Lay::kTmemCols);
  }
}

template <int NP>
const void* kernel_ptr(bool bf16) {
  return bf16 ? reinterpret_cast<const void*>(&splitkv_narrow_kernel<true, NP>)
              : reinterpret_cast<const void*>(&splitkv_narrow_kernel<false, NP>);
}

}  // namespace narrow

int narrow_rows_padded(int rows) { return rows <= 16 ? 16 : 32; }

int narrow_smem_bytes(int np) {
  return np == 16 ? narrow::Layout<16>::kSmemBytes : narrow::Layout<32>::kSmemBytes;
}

const void* narrow_kernel_ptr(bool bf16, int np) {
  return np == 16 ? narrow::kernel_ptr<16>(bf16) : narrow::kernel_ptr<32>(bf16);
}

cudaError_t launch_splitkv_narrow(bool bf16, const void* q, const CUtensorMap& kmap, const DecodeParams& p,
                                  cudaStream_t stream) {
  const int np = narrow_rows_padded(p.rows);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.num_parts);
  cfg.blockDim = dim3(narrow::kThreads);
  cfg.dynamicSmemBytes = narrow_smem_bytes(np);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (np == 16) {
    if (bf16) return cudaLaunchKernelEx(&cfg, narrow::splitkv_narrow_kernel<true, 16>, q, kmap, p);
    return cudaLaunchKernelEx(&cfg, narrow::splitkv_narrow_kernel<false, 16>, q, kmap, p);
  }
  if (bf16) return cudaLaunchKernelEx(&cfg, narrow::splitkv_narrow_kernel<true, 32>, q, kmap, p);
  return cudaLaunchKernelEx(&cfg, narrow::splitkv_narrow_kernel<false, 32>, q, kmap, p);
}

}  // namespace mla
