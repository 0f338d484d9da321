// Split-KV MLA decode kernel for few query rows (s_q * h_q <= 32) on a CTA pair.
//
// Same computation as the other split-KV kernels: per chunk of 64-token pages,
// scores, online softmax ("FlashMLA 在 Hopper GPU 上的 MHA 内核调度优化解析",
// 跷跷板调度的数学重构: the rescaled accumulation equals the plain softmax), P.V,
// and out/lse or fp32 partials for the combine (辅助优化：可编程依赖启动与瓦片调度).
//
// With <= 32 rows the decode is bound by HBM (intensity ~ 2 * h_q * s_q FLOP/B,
// section 计算边界特性与优化方向抉择), and what keeps the page stream from
// running at full bandwidth on one SM is how long a 72 KB page stays in shared
// memory: from its arrival through its 36 Q.K^T and 8 P.V instructions, which
// are issue-bound (~60 cycles each), so few pages fit in flight.  Here a
// cluster of two CTAs shares every page:
//  * CTA c loads only its half of each page -- columns 256c .. 256c+255 (four
//    64-column boxes, 128-byte swizzle; also its half of V) and 512+32c ..
//    +31 (one 32-column box, 64-byte swizzle): 36 KB, five page stages.
//  * It contracts Q.K^T over those 288 columns (16 + 2 tcgen05.mma, M = 128
//    lanes holding the query rows, N = 64 keys, A = its 288 Q columns resident
//    in TMEM) and sends the partial scores of its rows (64 fp32 each) to the
//    peer with st.async straight from registers, one block ahead.
//  * Both CTAs add own + peer partial -- the same two fp32 values in either
//    order, so the sum is the same bits on both sides -- and run the identical
//    online softmax, so each has the same P, running maximum and row sum
//    without exchanging any of them.  Within a CTA four warps share a block,
//    16 keys each: Q is written to all four TMEM lane quadrants, so every
//    quadrant holds a copy of the rows' scores and warp 4 + q reads keys
//    16q .. 16q+15 from its own quadrant; the four combine their row maxima
//    through shared memory once per block.
//  * CTA c accumulates O[:, 256c .. 256c+255] with the weight-stationary
//    tcgen05.mma (M = 32 rows, N = 256, 4 per page; A = P in shared memory,
//    B = the MN-major view of its four V boxes) and writes that half of out.
// Per page and CTA: 18 + 4 MMAs and 36 KB of shared memory, half of what one
// SM alone needs, so twice the pages are in flight per byte of stage.
//
// TMEM: O 2 x 64 columns (one buffer per chunk parity), S 3 x 64, Q 144 (the
// chunk's rows in every lane quadrant: lane 32q + r holds row r).  The next
// chunk's Q is written once the current chunk's last Q.K^T has completed (its
// rows are prefetched into L1 before that).
//
// Roles (384 threads): warp 0 lane 0 TMA producer; warp 1 TMEM owner, lane 0
// issues every tcgen05.mma, P.V first when ready (it frees a page stage),
// Q.K^T up to three blocks ahead; warps 4-7, one thread per query row and 16
// keys: send partial scores, softmax, O rescale of their quadrant; warps 8-11
// load Q (each into its own quadrant) and write each chunk's epilogue.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cmath>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace mla {
namespace npair {

using namespace ptx;

constexpr int kThreads = 384;
constexpr int kKBox = kPage * 128;               // 8 KB: 64 keys x 64 columns (128-byte swizzle)
constexpr int kKrBox = kPage * 64;               // 4 KB: 64 keys x 32 columns (64-byte swizzle)
constexpr int kStageBytes = 4 * kKBox + kKrBox;  // 36 KB: this CTA's 288 columns of a page
constexpr int kStages = 5;
constexpr int kSBufs = 3;
constexpr int kPBytes = 32 * 128;                // P: 32 rows (M of the P.V MMA) x 64 keys, 16-bit
constexpr float kRescaleThreshold = 8.0f;        // see splitkv.cu

enum Bar {
  kKvFull = 0,
  kKvEmpty = kKvFull + kStages,
  kQFull = kKvEmpty + kStages,  // 4 warps: the chunk's Q rows written to TMEM, one phase per chunk
  kQEmpty,                      // the chunk's last Q.K^T completed, one phase per chunk
  kSFull,                       // [kSBufs]
  kSEmpty = kSFull + kSBufs,    // [kSBufs] 4 warps
  kXFull = kSEmpty + kSBufs,    // [2] receive slot: the peer's partial scores of a block landed
  kXEmpty = kXFull + 2,         // [2] 4 warps of the peer consumed what this CTA sent into that slot
  kPFull = kXEmpty + 2,         // [2] 4 warps
  kPEmpty = kPFull + 2,         // [2]
  kODone = kPEmpty + 2,         // one phase per P.V
  kOFinal,                      // [2] one phase per chunk using that O buffer
  kOEmpty = kOFinal + 2,        // [2] 4 warps: the epilogue read that O buffer
  kStats = kOEmpty + 2,         // [2] row sums / reference maxima of a chunk parity in smem
  kDrain = kStats + 2,
  kNumBars
};

template <int NP>
struct Layout {
  static constexpr int kOffK = 0;
  static constexpr int kOffP = kOffK + kStages * kStageBytes;  // 1024-aligned
  static constexpr int kRcvSlot = NP * kPage * 4;              // NP rows x 64 fp32 partial scores
  static constexpr int kOffRcv = kOffP + 2 * kPBytes;
  static constexpr int kOffRed = kOffRcv + 2 * kRcvSlot;
  // floats: block maxima [2][4 warps][NP], partial row sums [4][NP], row sums [2][NP], reference max [2][NP]
  static constexpr int kRedFloats = 8 * NP + 4 * NP + 2 * NP + 2 * NP;
  static constexpr int kOffBar = (kOffRed + kRedFloats * 4 + 7) / 8 * 8;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 8 + static_cast<int>(sizeof(WaitCtl)) + 1024;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColO = 0;                       // 2 buffers x 64 columns (see umma_ws_ss)
  static constexpr uint32_t kColS = kColO + 2 * 64;          // kSBufs x 64
  static constexpr uint32_t kColQ = kColS + kSBufs * kPage;  // 128 + 16 columns of 16-bit pairs
  static_assert(kColQ + 144 <= kTmemCols, "TMEM budget");
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

template <bool kBF16, int NP>
__global__ void __launch_bounds__(kThreads, 1)
    splitkv_npair_kernel(const void* __restrict__ qptr, const __grid_constant__ CUtensorMap kmap,
                         const __grid_constant__ CUtensorMap krmap, const DecodeParams p) {
  using Lay = Layout<NP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + Lay::kOffBar + 8 * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kOffMisc);
  WaitCtl* wctl = reinterpret_cast<WaitCtl*>(smem + Lay::kOffMisc + 8);
  float* s_max = reinterpret_cast<float*>(smem + Lay::kOffRed);  // [2][4][NP]
  float* s_lpart = s_max + 8 * NP;                                // [4][NP]
  float* s_lsum = s_lpart + 4 * NP;                               // [2][NP]
  float* s_mref = s_lsum + 2 * NP;                                // [2][NP]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t crank = cluster_ctarank();
  const uint32_t peer = crank ^ 1u;
  const int part = blockIdx.x >> 1;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      const bool four = i == kPFull || i == kPFull + 1 || i == kOEmpty || i == kOEmpty + 1 || i == kQFull ||
                        (i >= kSEmpty && i < kSEmpty + kSBufs) || i == kXEmpty || i == kXEmpty + 1;
      mbar_init(bar(i), four ? 4u : 1u);
    }
    wctl->abort = 0;
    wctl->limit = p.wait_cycles;
    for (int i = 0; i < 2; ++i) mbar_arrive_expect_tx(bar(kXFull + i), Lay::kRcvSlot);  // arm phase 0
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), Lay::kTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 64) {
    prefetch_tmap(&kmap);
    prefetch_tmap(&krmap);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers are initialised before either sends to the other
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // launched as a programmatic dependent of the previous kernel in the stream (normally the
  // scheduler): the prologue above overlapped it; nothing it wrote is read before this wait
  pdl_wait_primary();
  if (threadIdx.x == 0) pdl_launch_dependents();

  const int* meta = p.meta + part * kMetaInts;
  const int R = p.rows;
  int* err = p.err;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (this CTA's half of each page)
    if (lane == 0) {
      const uint64_t evict_first = policy_evict_first();
      Walk w;
      w.init(p, meta);
      auto page_of = [&](const Walk& x) {
        return x.valid ? p.block_table[static_cast<int64_t>(x.req) * p.block_table_stride + x.blk] : 0;
      };
      int page_next = page_of(w);
      uint32_t it = 0;
      for (; w.valid && !aborted(wctl); ++it) {
        const int st = it % kStages;
        int page = page_next;
        Walk nx = w;
        nx.next(p);
        page_next = page_of(nx);  // the next block's page index is read while this stage frees up
        if (!mbar_wait(bar(kKvEmpty + st), ((it / kStages) & 1) ^ 1, wctl, err, kDevErrTimeout)) break;
        if (page < 0 || static_cast<int64_t>(page) >= p.num_pages) {
          atomicOr(err, kDevErrPage);
          atomicCAS(err + 1, 0, page == 0 ? -1 : page);
          page = 0;
        }
        mbar_arrive_expect_tx(bar(kKvFull + st), kStageBytes);
        const uint32_t dst = sbase + Lay::kOffK + st * kStageBytes;
        for (int i = 0; i < 4; ++i)  // columns 256c + 64i .. (also this CTA's V half)
          tma_load_3d_hint(dst + i * kKBox, &kmap, bar(kKvFull + st), 256 * crank + 64 * i, 0, page, evict_first);
        tma_load_3d_hint(dst + 4 * kKBox, &krmap, bar(kKvFull + st), 512 + 32 * crank, 0, page, evict_first);
        w = nx;
      }
      // Before the CTA can exit, every page load issued above must have landed: wait (bounded, abort
      // or not) for the last phase of each stage.  A phase the MMA warp already consumed has
      // completed, so the wait returns at once; only an abort leaves one pending.
      for (uint32_t j = it > kStages ? it - kStages : 0; j < it; ++j)
        mbar_wait_drain(bar(kKvFull + j % kStages), (j / kStages) & 1, wctl->limit);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_f16(kBF16, 128, kPage, false, false);
      constexpr uint32_t idesc_pv = idesc_f16(kBF16, 32, 256, false, true);
      Walk wq, wp;
      wq.init(p, meta);
      wp = wq;
      uint32_t tq = 0, tp = 0;
      // Inputs of the next Q.K^T (the chunk's Q, the page, a free score buffer) / the next P.V (P,
      // and for a chunk's first block the epilogue having read that O buffer) are complete.  No
      // phase tested here can run a full phase ahead: its producer waits on this thread's work.
      auto qk_ready = [&]() {
        if (wq.first() && !mbar_test_wait(bar(kQFull), wq.chunk & 1)) return false;
        return mbar_test_wait(bar(kKvFull + tq % kStages), (tq / kStages) & 1) &&
               mbar_test_wait(bar(kSEmpty + tq % kSBufs), ((tq / kSBufs) & 1) ^ 1);
      };
      auto pv_ready = [&]() {
        if (wp.first() && !mbar_test_wait(bar(kOEmpty + (wp.chunk & 1)), ((wp.chunk >> 1) & 1) ^ 1)) return false;
        return mbar_test_wait(bar(kPFull + (tp & 1)), (tp >> 1) & 1);
      };
      auto issue_qk = [&]() {
        const int st = tq % kStages;
        const int sb = tq % kSBufs;
        tc_fence_after();
        const uint32_t kb = sbase + Lay::kOffK + st * kStageBytes;
        const uint32_t dS = tmem + Lay::kColS + kPage * sb;
#pragma unroll
        for (int s = 0; s < 16; ++s) {  // columns 256c .. 256c+255
          const uint64_t bdesc = smem_desc_sw128(kb + (s >> 2) * kKBox + (s & 3) * 32, 16, 1024);
          umma_ts(dS, tmem + Lay::kColQ + 8 * s, bdesc, idesc_qk, s > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {  // columns 512 + 32c .. 512 + 32c + 31
          const uint64_t bdesc = smem_desc_sw64(kb + 4 * kKBox + i * 32, 16, 512);
          umma_ts(dS, tmem + Lay::kColQ + 128 + 8 * i, bdesc, idesc_qk, 1u);
        }
        umma_commit(bar(kSFull + sb));
        if (wq.last()) umma_commit(bar(kQEmpty));
        wq.next(p);
        ++tq;
      };
      auto issue_pv = [&]() {
        const int st = tp % kStages;
        const int pb = tp & 1;
        const int ob = wp.chunk & 1;
        tc_fence_after();
        const uint32_t vb = sbase + Lay::kOffK + st * kStageBytes;
        const uint32_t pbuf = sbase + Lay::kOffP + pb * kPBytes;
#pragma unroll
        for (int kk = 0; kk < kPage / 16; ++kk) {
          // O[:, 256c ..] += P[:, 16kk ..] . V[16kk .., 256c ..]: A = P (32 rows, K-major), B = V
          // (MN-major view of the four column boxes, 8 KB apart; 16 keys = 2 x 1 KB)
          const uint64_t adesc = smem_desc_sw128(pbuf + kk * 32, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(vb + kk * 2048, kKBox, 1024);
          umma_ws_ss(tmem + Lay::kColO + 64 * ob, adesc, bdesc, idesc_pv, (!wp.first() || kk > 0) ? 1u : 0u);
        }
        umma_commit(bar(kKvEmpty + st));
        umma_commit(bar(kPEmpty + pb));
        umma_commit(bar(kODone));
        if (wp.last()) umma_commit(bar(kOFinal + ob));
        wp.next(p);
        ++tp;
      };
      long long idle_since = clock64();
      uint32_t polls = 0;
      while (wp.valid) {
        if (tp < tq && pv_ready()) {
          issue_pv();
        } else if (wq.valid && tq < tp + kSBufs && qk_ready()) {
          issue_qk();
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
      umma_commit(bar(kDrain));
      mbar_wait_drain(bar(kDrain), 0, wctl->limit);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ score exchange, softmax, O rescale
    // Warp 4 + q takes keys 16q .. 16q+15 of every block for all the rows, from its quadrant's copy.
    const int q4 = warp & 3;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const int r = lane;
    const int kc = 16 * q4;
    // false once one of this thread's waits gave up (the CTA is aborting): from then on it sends
    // nothing to the peer and arrives on no barrier that waits for bytes, so nothing is left in
    // flight into the peer's shared memory and no barrier phase is over-arrived
    bool live = true;

    // Block u's partial scores of this CTA, this warp's 16 keys of every row -> the peer's receive
    // slot u & 1.  A row is 16 pieces of 16 bytes; piece j sits at j ^ (r & 7), so the eight lanes
    // of a quarter-warp reading one piece hit eight different bank groups.
    auto send = [&](uint32_t u) {
      const int sb = u % kSBufs;
      live &= mbar_wait(bar(kSFull + sb), (u / kSBufs) & 1, wctl, err, kDevErrTimeout);
      if (!__all_sync(0xffffffffu, live)) return;  // reconverged, and the same for every lane
      tc_fence_after();
      uint32_t v[16];
      tmem_ld16(t_lane + Lay::kColS + kPage * sb + kc, v);
      tmem_wait_ld();
      bool free_slot = true;
      if (lane == 0) free_slot = mbar_wait<true>(bar(kXEmpty + (u & 1)), ((u >> 1) & 1) ^ 1, wctl, err, kDevErrTimeout);
      live &= __shfl_sync(0xffffffffu, free_slot, 0);
      if (live && r < NP) {
        const uint32_t dst = mapa(sbase + Lay::kOffRcv + (u & 1) * Lay::kRcvSlot + r * (kPage * 4), peer);
        const uint32_t rb = mapa(bar(kXFull + (u & 1)), peer);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          st_async_v4(dst + (((4 * q4 + j) ^ (r & 7)) << 4), rb, __uint_as_float(v[4 * j]),
                      __uint_as_float(v[4 * j + 1]), __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
      }
    };

    Walk wt;
    wt.init(p, meta);
    if (wt.valid) send(0);
    float m = -INFINITY;  // exponent reference of the current chunk (log2 units), the same in every warp
    float lq = 0.f;       // row sum over this warp's keys, relative to m
    for (uint32_t t = 0; wt.valid; ++t) {
      Walk wn = wt;
      wn.next(p);
      const int par = wt.chunk & 1;
      const int slot = t & 1;
      const int sb = t % kSBufs;
      if (wn.valid) send(t + 1);  // the peer gets block t + 1 a block early

      // ---- block t: own partial + the peer's (same sum on both CTAs), then release both buffers
      live &= mbar_wait<true>(bar(kXFull + slot), (t >> 1) & 1, wctl, err, kDevErrTimeout);
      live &= mbar_wait(bar(kSFull + sb), (t / kSBufs) & 1, wctl, err, kDevErrTimeout);
      __syncwarp();
      tc_fence_after();
      float x[16];
      {
        uint32_t a[16];
        tmem_ld16(t_lane + Lay::kColS + kPage * sb + kc, a);
        tmem_wait_ld();
        const uint8_t* rrow = smem + Lay::kOffRcv + slot * Lay::kRcvSlot + (r < NP ? r : 0) * (kPage * 4);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float4 v = *reinterpret_cast<const float4*>(rrow + (((4 * q4 + j) ^ (r & 7)) << 4));
          x[4 * j] = __uint_as_float(a[4 * j]) + v.x;
          x[4 * j + 1] = __uint_as_float(a[4 * j + 1]) + v.y;
          x[4 * j + 2] = __uint_as_float(a[4 * j + 2]) + v.z;
          x[4 * j + 3] = __uint_as_float(a[4 * j + 3]) + v.w;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar(kSEmpty + sb));  // Q.K^T of block t + 3 may overwrite the scores
        // every lane used what it read from the receive slot before the warp barrier: arm the
        // slot's next phase (once, after a completed phase -- arming one still waiting for bytes
        // would over-arrive), then release this warp's part of it to the peer (a relaxed arrive
        // issued after x[15])
        if (live) {
          if (q4 == 0) mbar_arrive_expect_tx(bar(kXFull + slot), Lay::kRcvSlot);
          mbar_arrive_cluster_relaxed_after(mapa(bar(kXEmpty + slot), peer), x[15]);
        }
      }

      // ---- online softmax in log2 units (the same instructions on the same values as the peer)
      if (wt.first()) {
        m = -INFINITY;
        lq = 0.f;
      }
      int limit = 0;
      if (r < R) {
        limit = p.causal ? wt.L - (p.s_q - 1 - r / p.h_q) : wt.L;
        limit = limit < 0 ? 0 : limit;
      }
      const int kbase = wt.blk * kPage + kc;
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float v = (kbase + c < limit) ? x[c] * p.scale_log2 : -INFINITY;
        x[c] = v;
        mx = fmaxf(mx, v);
      }
      float* smx = s_max + slot * 4 * NP;
      if (r < NP) smx[q4 * NP + r] = mx;
      named_bar_sync(1, 128);
      if (r < NP) mx = fmaxf(fmaxf(smx[r], smx[NP + r]), fmaxf(smx[2 * NP + r], smx[3 * NP + r]));
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
      uint32_t pk[8];
#pragma unroll
      for (int c2 = 0; c2 < 8; ++c2) {
        const float p0 = ex2(x[2 * c2] - base);
        const float p1 = ex2(x[2 * c2 + 1] - base);
        sum += p0 + p1;
        pk[c2] = pack2<kBF16>(p0, p1);
      }
      lq = lq * alpha + sum;
      // P buffer `slot` was last read by the P.V of block t - 2
      live &= mbar_wait(bar(kPEmpty + slot), ((t >> 1) & 1) ^ 1, wctl, err, kDevErrTimeout);
      {
        // P row r: 64 keys = 128 bytes, 16-byte chunks XOR-swizzled by row (128-byte swizzle);
        // this warp's keys are chunks 2q and 2q + 1
        uint8_t* prow = smem + Lay::kOffP + slot * kPBytes + r * 128;
        *reinterpret_cast<uint4*>(prow + (((2 * q4) ^ (r & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *reinterpret_cast<uint4*>(prow + (((2 * q4 + 1) ^ (r & 7)) << 4)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
      }
      fence_proxy_async_smem();  // P is read by the tensor core (async proxy)
      if (__any_sync(0xffffffffu, resc)) {
        // a row's reference moved (never on a chunk's first block): O must first hold the chunk's
        // blocks up to t - 1; lane r of this quadrant holds row r, 64 of this CTA's 256 values
        live &= mbar_wait(bar(kODone), (t - 1) & 1, wctl, err, kDevErrTimeout);
        __syncwarp();
        tc_fence_after();
#pragma unroll 1
        for (int c32 = 0; c32 < 2; ++c32) {
          uint32_t o[32];
          const uint32_t col = Lay::kColO + 64 * par + 32 * c32;
          tmem_ld32(t_lane + col, o);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
          tmem_st32(t_lane + col, o);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kPFull + slot));
      if (wt.last()) {
        // row sums of the four warps, added in a fixed order (the same bits in both CTAs); this
        // chunk's stats slot was last used by chunk - 2, whose epilogue must have read it
        if (r < NP) s_lpart[q4 * NP + r] = lq;
        named_bar_sync(1, 128);
        if (q4 == 0) {
          if (wt.chunk >= 2)
            live &= mbar_wait(bar(kOEmpty + par), ((wt.chunk >> 1) & 1) ^ 1, wctl, err, kDevErrTimeout);
          if (r < NP) {
            s_lsum[par * NP + r] = (s_lpart[r] + s_lpart[NP + r]) + (s_lpart[2 * NP + r] + s_lpart[3 * NP + r]);
            s_mref[par * NP + r] = m;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(kStats + par));
        }
      }
      wt = wn;
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ Q loads (warps 8 / 9) and epilogue (8-11)
    const int q4 = warp & 3;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const int r = lane;
    auto load_q = [&](const Walk& c, uint32_t idx) {
      // this CTA's 288 Q columns of the chunk's rows into this warp's lane quadrant, once the
      // previous chunk's last Q.K^T has read the old ones (the row is requested into L1 before)
      const uint4* qrow = reinterpret_cast<const uint4*>(
          reinterpret_cast<const uint16_t*>(qptr) + (static_cast<int64_t>(c.req) * R + (r < R ? r : 0)) * kDK);
      if (r < R) {
#pragma unroll
        for (int k = 0; k < 4; ++k) prefetch_l1(qrow + 32 * crank + 8 * k);
        prefetch_l1(qrow + 64 + 4 * crank);
      }
      if (idx > 0) mbar_wait(bar(kQEmpty), (idx - 1) & 1, wctl, err, kDevErrTimeout);
      __syncwarp();
      tc_fence_after();
#pragma unroll 1
      for (int c32 = 0; c32 < 4; ++c32) {  // columns 256c + 64 c32 .. +63
        uint32_t w[32];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          uint4 d = make_uint4(0, 0, 0, 0);
          if (r < R) d = __ldg(qrow + 32 * crank + 8 * c32 + v);
          w[4 * v] = d.x;
          w[4 * v + 1] = d.y;
          w[4 * v + 2] = d.z;
          w[4 * v + 3] = d.w;
        }
        tmem_st32(t_lane + Lay::kColQ + 32 * c32, w);
      }
      {
        uint32_t w[16];  // columns 512 + 32c .. +31
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          uint4 d = make_uint4(0, 0, 0, 0);
          if (r < R) d = __ldg(qrow + 64 + 4 * crank + v);
          w[4 * v] = d.x;
          w[4 * v + 1] = d.y;
          w[4 * v + 2] = d.z;
          w[4 * v + 3] = d.w;
        }
        tmem_st16(t_lane + Lay::kColQ + 128, w);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && !(p.withhold_q_ready && idx == 0 && q4 == 0)) mbar_arrive(bar(kQFull));
    };
    auto epilogue = [&](const Walk& c, uint32_t idx) {
      const int ob = idx & 1;
      mbar_wait(bar(kOFinal + ob), (idx >> 1) & 1, wctl, err, kDevErrTimeout);
      mbar_wait(bar(kStats + ob), (idx >> 1) & 1, wctl, err, kDevErrTimeout);
      __syncwarp();
      tc_fence_after();
      const bool whole = (c.lo == 0 && c.hi == c.n);
      const int split = (c.req == c.br) ? meta[4] : 0;
      const int64_t chunk0 = whole ? 0 : static_cast<int64_t>(p.num_splits[c.req] + split) * R;
      const float* ls = s_lsum + ob * NP;
      // lane r of quadrant q4 holds row r, this CTA's values 64 q4 .. 64 q4 + 63
      const float lr = r < NP ? ls[r] : 0.f;
      const float inv = lr > 0.f ? 1.f / lr : 0.f;
#pragma unroll 1
      for (int c32 = 0; c32 < 2; ++c32) {
        uint32_t o[32];
        tmem_ld32(t_lane + Lay::kColO + 64 * ob + 32 * c32, o);
        tmem_wait_ld();
        if (r < R) {
          const int d = 256 * static_cast<int>(crank) + 64 * q4 + 32 * c32;
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
      if (crank == 0 && q4 == 0 && r < R) {
        const float lse_v = lr > 0.f ? (s_mref[ob * NP + r] + log2f(lr)) * 0.69314718055994531f : -INFINITY;
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
    Walk c;
    c.init(p, meta);
    if (c.valid) load_q(c, 0);
    for (uint32_t idx = 0; c.valid; ++idx) {
      Walk nx = c;
      nx.next_chunk(p);
      if (nx.valid) load_q(nx, idx + 1);  // as soon as this chunk's Q.K^T are done
      epilogue(c, idx);
      c = nx;
    }
  }

  // ------------------------------------------------------------ teardown
  __syncwarp();  // lanes of the producer / MMA warps rejoin their elected lane
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer may still be sending into this CTA's shared memory until here
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Lay::kTmemCols);
  }
}

template <int NP>
const void* kernel_ptr(bool bf16) {
  return bf16 ? reinterpret_cast<const void*>(&splitkv_npair_kernel<true, NP>)
              : reinterpret_cast<const void*>(&splitkv_npair_kernel<false, NP>);
}

}  // namespace npair

int npair_smem_bytes(int np) {
  return np == 16 ? npair::Layout<16>::kSmemBytes : npair::Layout<32>::kSmemBytes;
}

const void* npair_kernel_ptr(bool bf16, int np) {
  return np == 16 ? npair::kernel_ptr<16>(bf16) : npair::kernel_ptr<32>(bf16);
}

cudaError_t launch_splitkv_npair(bool bf16, const void* q, const CUtensorMap& kmap, const CUtensorMap& krmap,
                                 const DecodeParams& p, cudaStream_t stream) {
  const int np = narrow_rows_padded(p.rows);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * p.num_parts);  // one cluster of 2 CTAs per partition
  cfg.blockDim = dim3(npair::kThreads);
  cfg.dynamicSmemBytes = npair_smem_bytes(np);
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
  if (np == 16) {
    if (bf16) return cudaLaunchKernelEx(&cfg, npair::splitkv_npair_kernel<true, 16>, q, kmap, krmap, p);
    return cudaLaunchKernelEx(&cfg, npair::splitkv_npair_kernel<false, 16>, q, kmap, krmap, p);
  }
  if (bf16) return cudaLaunchKernelEx(&cfg, npair::splitkv_npair_kernel<true, 32>, q, kmap, krmap, p);
  return cudaLaunchKernelEx(&cfg, npair::splitkv_npair_kernel<false, 32>, q, kmap, krmap, p);
}

}  // namespace mla
