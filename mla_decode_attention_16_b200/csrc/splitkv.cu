// Split-KV MLA decode kernel for sm_100a, for s_q * h_q > 32 query rows.
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
//  * A 128 x 512 fp32 output tile alone fills the 512 TMEM columns of an SM, so
//    a CTA pair (cluster of 2) owns one 128-row tile: CTA c keeps O[:, 256c :
//    256c+256] and computes PV for that half.
//  * The 576-deep Q.K^T contraction is split too, so no MMA work is
//    duplicated: CTA c contracts columns 256c .. 256c+255 (its V half) plus the
//    32 columns 512 + 32c ..  Those 256 main columns of Q stay in TMEM for the
//    whole chunk (A operand from TMEM); the 32 others come from a
//    shared-memory box.
//  * The softmax of a 64-key block is split between the pair by key: CTA c
//    exponentiates keys 32c .. 32c+31 of every row.  It sends its partial
//    scores of the other 32 keys to the peer, rounded to 24 bits (sign,
//    exponent, 15 mantissa bits) and written by each thread straight from
//    registers into the peer's shared memory (three 16-byte st.async that
//    complete on the peer's mbarrier; bulk copies measured slower here, as they
//    queue in the copy engine behind the page loads), and receives the peer's
//    partials of its own keys.  The two CTAs share each row's block maximum (distributed
//    shared memory stores) so they keep the same exponent reference, and each
//    copies the P of its keys into the peer's P, so both P.V products see the
//    whole block; the row sums are added at the end of a chunk.
//  * The score exchange runs one block ahead: while block t's maximum travels,
//    each softmax warp sends its partial of block t+1.  A warp signals "slot
//    consumed" with a relaxed arrive whose input depends on every word it read
//    (a cluster-scope release there cost ~1000 cycles per block).
//  * Each CTA TMA-loads, per page, four 64-column boxes (128-byte swizzle) at
//    columns 256c + 64i -- also this CTA's V half -- and one 32-column box
//    (64-byte swizzle) at 512 + 32c: 36 KB per page, four page stages, so the
//    HBM latency of a page load hides behind three blocks of work; EVICT_FIRST
//    L2 policy on page loads (细粒度流水线与缓存优化).
//  * P goes to shared memory as four K-major tiles of 16 keys with 32-byte
//    swizzle (the A operand of the four K = 16 steps of PV), so the piece one
//    warp writes -- 32 rows x 16 keys -- is one contiguous kilobyte that a
//    single bulk copy puts into the peer's P; V is the MN-major B operand read
//    straight from the page tile.
//  * Roles: warp 0 lane 0 TMA producer; warp 1 TMEM owner, lane 0 issues every
//    tcgen05.mma (Q.K^T two blocks ahead of P.V); warps 4-11 two per TMEM lane
//    quadrant, one thread per (query row, 16 of its CTA's 32 keys): Q into
//    TMEM, score exchange, softmax (exp2 with log2(e) folded into the scale,
//    "FlashMLA: 高性能GPU注意力机制计算库" 4. Softmax数值稳定性优化), O correction,
//    epilogue.  The four threads of a row (two per CTA) agree on its maximum
//    and keep separate partial row sums, added at the end of a chunk.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cmath>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace mla {
namespace splitkv {

using namespace ptx;

constexpr int kThreads = 384;
constexpr int kBlockN = kPage;              // keys per pipeline step
constexpr int kQrBox = kTileRows * 64;     // 8 KB: 128 rows x 32 columns (64-byte swizzle)
constexpr int kKBox = kBlockN * 128;        // 8 KB: 64 keys x 64 columns (128-byte swizzle)
constexpr int kKrBox = kBlockN * 64;        // 4 KB: 64 keys x 32 columns (64-byte swizzle)
constexpr int kStageBytes = 4 * kKBox + kKrBox;  // 36 KB
constexpr int kStages = 4;
constexpr int kPTile = kTileRows * 32;      // 4 KB: P of 16 keys x 128 rows (16-bit, 32-byte swizzle)
constexpr int kPBytes = 4 * kPTile;         // 16 KB: the block's 64 keys
constexpr int kSmWarps = 8;                 // softmax warps: 4 lane quadrants x 2 key quarters
constexpr int kOwnN = kBlockN / 4;          // 16 keys per softmax thread
constexpr int kRowWords = kOwnN * 3 / 4;    // 12 words: 16 scores at 24 bits
constexpr int kRowBytes = kRowWords * 4;    // 48
constexpr int kXWarp = 32 * kRowBytes;      // 1.5 KB per warp and direction
constexpr int kXBytes = kSmWarps * kXWarp;  // 12 KB
constexpr int kSlotFloats = 2 * 2 * 2 * kTileRows;  // row values: [parity][source CTA][key quarter][row]

constexpr int kOffQR = 0;                               // this CTA's 32 of Q's columns 512..575
constexpr int kOffK = kOffQR + kQrBox;                  // page stages
constexpr int kOffP = kOffK + kStages * kStageBytes;    // P
constexpr int kOffRcv = kOffP + kPBytes;                // the peer's partial scores [8 warps]
constexpr int kOffRed = kOffRcv + kXBytes;              // row maxima / sums of both CTAs
static_assert(kOffK % 1024 == 0 && kStageBytes % 1024 == 0 && kOffP % 1024 == 0, "swizzle atom alignment");
constexpr int kOffBar = kOffRed + kSlotFloats * 4;

enum Bar {
  kKvFull = 0,
  kKvEmpty = kKvFull + kStages,
  kQrFull = kKvEmpty + kStages,  // Q column box 512..575 landed (TMA), one phase per chunk
  kQtFull,                       // Q main columns written to TMEM (8 warps), one phase per chunk
  kQEmpty,                       // the chunk's last Q.K^T completed
  kSFull,                        // [2]
  kSEmpty = kSFull + 2,          // [2], 8 warps
  kPFull = kSEmpty + 2,          // 8 warps + the peer's copies of its P, one phase per block
  kPEmpty,                       // one phase per P.V
  kOFinal,                       // one phase per chunk: its last P.V completed
  kOEmpty,                       // 8 warps, one phase per chunk
  kXFull,                        // [8 warps]: the peer's partial landed
  kXEmpty = kXFull + kSmWarps,   // [8 warps]: the peer consumed what this CTA sent
  kXchg = kXEmpty + kSmWarps,    // [4 quadrants][2 parities]: the row values of both CTAs are in
  kPeerFree = kXchg + 8,         // [8 warps]: the peer's P.V of the previous block completed
  kDrain = kPeerFree + kSmWarps,
  kNumBars
};
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemUsed = kOffMisc + 8 + sizeof(WaitCtl);
constexpr int kSmemBytes = kSmemUsed + 1024;  // slack to align the base to 1024 B
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;    // 256 columns: this CTA's half of O
constexpr uint32_t kColS = 256;  // 2 x 64 columns: partial scores
constexpr uint32_t kColQ = 384;  // 128 columns: Q columns 256c .. 256c+255 (16-bit pairs)
static_assert(kColQ + 128 == kTmemCols, "TMEM budget");

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
    splitkv_pair_kernel(const void* __restrict__ qptr, const __grid_constant__ CUtensorMap qrmap,
                        const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap krmap,
                        const DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + kOffBar + 8 * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  WaitCtl* wctl = reinterpret_cast<WaitCtl*>(smem + kOffMisc + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t crank = cluster_ctarank();
  const uint32_t peer = crank ^ 1u;
  const int pair = blockIdx.x >> 1;
  const int part = pair / p.m_tiles;
  const int mtile = pair % p.m_tiles;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      const bool eight = i == kQtFull || i == kSEmpty || i == kSEmpty + 1 || i == kPFull || i == kOEmpty;
      const bool two = i >= kXchg && i < kXchg + 8;
      mbar_init(bar(i), eight ? static_cast<uint32_t>(kSmWarps) : two ? 2u : 1u);
    }
    wctl->abort = 0;
    wctl->limit = p.wait_cycles;
    for (int i = 0; i < kSmWarps; ++i) mbar_arrive_expect_tx(bar(kXFull + i), kXWarp);  // arm phase 0
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 32 * 2) {
    prefetch_tmap(&qrmap);
    prefetch_tmap(&kmap);
    prefetch_tmap(&krmap);
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

  const int* meta = p.meta + part * kMetaInts;
  const int R = p.rows;
  int* err = p.err;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t evict_first = policy_evict_first();
      Walk w;
      w.init(p, meta);
      auto page_of = [&](const Walk& x) {
        return x.valid ? p.block_table[static_cast<int64_t>(x.req) * p.block_table_stride + x.blk] : 0;
      };
      int page_next = page_of(w);
      uint32_t it = 0;
      int q_chunks = 0;  // Q column boxes requested so far (one per chunk)
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
        const uint32_t dst = sbase + kOffK + st * kStageBytes;
        for (int i = 0; i < 4; ++i)  // columns 256c + 64i .. (also this CTA's V half)
          tma_load_3d_hint(dst + i * kKBox, &kmap, bar(kKvFull + st), 256 * crank + 64 * i, 0, page, evict_first);
        tma_load_3d_hint(dst + 4 * kKBox, &krmap, bar(kKvFull + st), 512 + 32 * crank, 0, page, evict_first);
        if (w.first()) {
          // the chunk's Q columns 512 + 32c .., once the previous chunk's last Q.K^T has read the old ones
          if (mbar_wait(bar(kQEmpty), (w.chunk & 1) ^ 1, wctl, err, kDevErrTimeout)) {
            mbar_arrive_expect_tx(bar(kQrFull), kQrBox);
            tma_load_2d(sbase + kOffQR, &qrmap, bar(kQrFull), 512 + 32 * crank, w.req * R + mtile * kTileRows);
            ++q_chunks;
          }
        }
        w = nx;
      }
      // Before the CTA can exit, every TMA load issued above must have landed: wait (bounded, abort
      // or not) for the last phase of each stage and of the Q box.  A phase the MMA warp already
      // consumed has completed, so the wait returns at once; only an abort leaves one pending.
      for (uint32_t j = it > kStages ? it - kStages : 0; j < it; ++j)
        mbar_wait_drain(bar(kKvFull + j % kStages), (j / kStages) & 1, wctl->limit);
      if (q_chunks > 0) mbar_wait_drain(bar(kQrFull), (q_chunks - 1) & 1, wctl->limit);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_f16(kBF16, kTileRows, kBlockN, false, false);
      constexpr uint32_t idesc_pv = idesc_f16(kBF16, kTileRows, 256, false, true);
      Walk wq, wp;
      wq.init(p, meta);
      wp = wq;
      uint32_t tq = 0, tp = 0;
      // Inputs of the next Q.K^T (chunk's Q, the page, a free score buffer) / the next P.V (P, and
      // for a chunk's first block the epilogue having read O) are complete.  Each barrier phase
      // tested here cannot run a full phase ahead: its producer waits on this thread's earlier work.
      auto qk_ready = [&]() {
        if (wq.first() && !(mbar_test_wait(bar(kQrFull), wq.chunk & 1) && mbar_test_wait(bar(kQtFull), wq.chunk & 1)))
          return false;
        return mbar_test_wait(bar(kKvFull + tq % kStages), (tq / kStages) & 1) &&
               mbar_test_wait(bar(kSEmpty + (tq & 1)), ((tq >> 1) & 1) ^ 1);
      };
      auto pv_ready = [&]() {
        if (wp.first() && !mbar_test_wait(bar(kOEmpty), (wp.chunk & 1) ^ 1)) return false;
        return mbar_test_wait(bar(kPFull), tp & 1);
      };
      auto issue_qk = [&]() {
        const int st = tq % kStages;
        const int b = tq & 1;
        tc_fence_after();
        const uint32_t kbase = sbase + kOffK + st * kStageBytes;
        const uint32_t dS = tmem + kColS + 64 * b;
#pragma unroll
        for (int s = 0; s < 16; ++s) {  // main columns: Q from TMEM
          const uint64_t bdesc = smem_desc_sw128(kbase + (s >> 2) * kKBox + (s & 3) * 32, 16, 1024);
          umma_ts(dS, tmem + kColQ + 8 * s, bdesc, idesc_qk, s > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {  // this CTA's 32 of the columns 512..575: Q from shared memory
          const uint64_t adesc = smem_desc_sw64(sbase + kOffQR + i * 32, 16, 512);
          const uint64_t bdesc = smem_desc_sw64(kbase + 4 * kKBox + i * 32, 16, 512);
          umma_ss(dS, adesc, bdesc, idesc_qk, 1u);
        }
        umma_commit(bar(kSFull + b));
        if (wq.last()) umma_commit(bar(kQEmpty));
        wq.next(p);
        ++tq;
      };
      auto issue_pv = [&]() {
        const int st = tp % kStages;
        tc_fence_after();
        const uint32_t vbase = sbase + kOffK + st * kStageBytes;
#pragma unroll
        for (int kk = 0; kk < kBlockN / 16; ++kk) {
          // P keys 16kk.. (tile kk: K-major, 128 rows of 32 bytes); V rows 16kk.. (MN-major: 64-column
          // boxes 8 KB apart)
          const uint64_t adesc = smem_desc_sw32(sbase + kOffP + kk * kPTile, 16, 256);
          const uint64_t bdesc = smem_desc_sw128(vbase + kk * 2048, kKBox, 1024);
          umma_ss(tmem + kColO, adesc, bdesc, idesc_pv, (!wp.first() || kk > 0) ? 1u : 0u);
        }
        umma_commit(bar(kKvEmpty + st));
        umma_commit(bar(kPEmpty));
        if (wp.last()) umma_commit(bar(kOFinal));
        wp.next(p);
        ++tp;
      };
      // Whichever is ready first: a P.V frees its page stage, so it goes before a ready Q.K^T;
      // Q.K^T may be issued up to three blocks ahead of P.V (the two score buffers bound it too).  A bounded wait covers the
      // time nothing is ready.
      long long idle_since = clock64();
      uint32_t polls = 0;
      while (wp.valid) {
        if (tp < tq && pv_ready()) {
          issue_pv();
        } else if (wq.valid && tq < tp + 3 && qk_ready()) {
          issue_qk();
        } else {
          if ((++polls & 15u) == 0) {
            if (aborted(wctl)) break;
            const long long now = clock64();
            if (now - idle_since > wctl->limit) {
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
  } else if (warp >= 4) {
    // ------------------------------------------------------------ Q to TMEM, exchange, softmax, correction, epilogue
    // Two warps per TMEM lane quadrant.  Of the block's 64 keys this CTA exponentiates 32c ..
    // 32c+31: warp 4 + q4 the first 16 of its 32 rows, warp 8 + q4 the last 16.  Each warp also
    // sends the peer its partial scores of keys 32p + 16 sub .. (p = the peer's rank).
    const int sm = warp - 4;          // 0..7
    const int q4 = warp & 3;
    const int sub = sm >> 2;          // which 16 of the CTA's 32 keys
    const int row = q4 * 32 + lane;
    const int row_g = mtile * kTileRows + row;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const int own_col = 32 * static_cast<int>(crank) + kOwnN * sub;   // S columns this thread exponentiates
    const int send_col = 32 * static_cast<int>(peer) + kOwnN * sub;   // S columns it sends to the peer
    // its P: tile 2c + sub (keys own_col ..), rows 32 q4 .. 32 q4 + 31 = one contiguous kilobyte
    const uint32_t p_piece = sbase + kOffP + (2 * crank + sub) * kPTile + q4 * 32 * 32;
    float* slots = reinterpret_cast<float*>(smem + kOffRed);  // [parity][source CTA][key quarter][row]
    // a quadrant whose 32 rows are all padding keeps the barrier protocol but skips the math;
    // its peer quadrant skips the same way
    const bool active = mtile * kTileRows + q4 * 32 < R;
    const int active_quadrants = min(4, (R - mtile * kTileRows + 31) / 32);

    // The row's four values of one kind (its block maximum, its row sum), one per thread of the
    // row in either CTA: post puts this thread's into this CTA's slot and (a 4-byte distributed
    // shared memory store completing on the peer's barrier) into the peer's; wait returns all four
    // as v[2 * cta + quarter].  One phase of the quadrant's barrier of parity x & 1 per exchange:
    // the two local warps arrive, the peer's two warps' stores (2 x 32 x 4 bytes) complete it.  A
    // slot of parity x & 1 is written again only in exchange x + 2, which on either side follows
    // this thread's exchange x + 1 and so its reading of exchange x.
    // Abort safety without cost on the normal path (a shared-memory read of the abort flag at each
    // step of this chain measured ~10 % slower): an iteration starts only while the CTA has not
    // aborted, and the two arrivals that could land on a barrier phase still waiting for bytes --
    // re-arming the receive slot, and this warp's arrival on P -- are made only when the wait
    // that precedes them completed.  Stores sent to the peer after a failed wait land in a CTA that
    // is still resident (both pass the closing cluster barrier before exiting).
    uint32_t xc = 0;
    auto xchg_post = [&](float v) {
      const int par = xc & 1;
      const uint32_t xb = bar(kXchg + 2 * q4 + par);
      const int idx = par * 4 * kTileRows + (2 * static_cast<int>(crank) + sub) * kTileRows + row;
      slots[idx] = v;
      st_async_b32(mapa(sbase + kOffRed + 4 * idx, peer), mapa(xb, peer), v);
      __syncwarp();
      if (lane == 0) {
        if (sub == 0)
          mbar_arrive_expect_tx(xb, 2 * 32 * 4);
        else
          mbar_arrive(xb);
      }
    };
    auto xchg_wait = [&](float (&v)[4]) {
      const int par = xc & 1;
      mbar_wait(bar(kXchg + 2 * q4 + par), (xc >> 1) & 1, wctl, err, kDevErrTimeout);
      const float* slot = slots + par * 4 * kTileRows + row;
#pragma unroll
      for (int k = 0; k < 4; ++k) v[k] = slot[k * kTileRows];
      ++xc;
    };

    // Q columns 256c + 128 sub .. +127 of this thread's row of request `req` -> TMEM columns kColQ + 64 sub ..
    auto q_row = [&](int req) {
      return reinterpret_cast<const uint8_t*>(qptr) +
             ((static_cast<int64_t>(req) * R + (row_g < R ? row_g : 0)) * kDK + 256 * crank + 128 * sub) * 2;
    };
    auto prefetch_q = [&](int req) {
      if (row_g >= R) return;
      const uint8_t* q = q_row(req);
      prefetch_l1(q);
      prefetch_l1(q + 128);
    };
    auto store_q = [&](int req) {
      const uint4* qrow = reinterpret_cast<const uint4*>(q_row(req));
#pragma unroll
      for (int c32 = 0; c32 < 2; ++c32) {
        uint32_t w[32];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          uint4 d = make_uint4(0, 0, 0, 0);
          if (row_g < R) d = __ldg(qrow + c32 * 8 + v);
          w[4 * v] = d.x;
          w[4 * v + 1] = d.y;
          w[4 * v + 2] = d.z;
          w[4 * v + 3] = d.w;
        }
        tmem_st32(t_lane + kColQ + 64 * sub + 32 * c32, w);
      }
      tmem_wait_st();
    };

    // Block u's scores are ready: (if u ends its chunk and another chunk follows) put the next
    // chunk's Q into TMEM, then send this warp's part of the partial scores to the peer.
    auto send_partial = [&](uint32_t u, const Walk& wu) {
      const int b = u & 1;
      Walk nx = wu;
      nx.next(p);
      const bool new_q = nx.valid && nx.chunk != wu.chunk;
      if (new_q && active) prefetch_q(nx.req);  // into L1 while the scores finish
      mbar_wait(bar(kSFull + b), (u >> 1) & 1, wctl, err, kDevErrTimeout);
      __syncwarp();  // reconverge before the warp-collective tcgen05 ops
      tc_fence_after();
      if (new_q) {
        // the Q.K^T of block u was the chunk's last: the Q columns are free
        mbar_wait(bar(kQEmpty), wu.chunk & 1, wctl, err, kDevErrTimeout);
        __syncwarp();
        tc_fence_after();
        if (active) store_q(nx.req);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kQtFull));
      }
      if (!active) return;
      uint32_t r[16];
      tmem_ld16(t_lane + kColS + 64 * b + send_col, r);
      tmem_wait_ld();
      {
        uint32_t w[kRowWords];  // 16 scores -> 12 words -> three 16-byte stores into the peer's row
#pragma unroll
        for (int g = 0; g < 4; ++g)
          pack24(r[4 * g], r[4 * g + 1], r[4 * g + 2], r[4 * g + 3], w[3 * g], w[3 * g + 1], w[3 * g + 2]);
        // the peer's receive slot of this warp is free once the peer has combined block u - 1
        if (lane == 0) mbar_wait<true>(bar(kXEmpty + sm), (u & 1) ^ 1, wctl, err, kDevErrTimeout);
        __syncwarp();
        const uint32_t dst = mapa(sbase + kOffRcv + sm * kXWarp + lane * kRowBytes, peer);
        const uint32_t rb = mapa(bar(kXFull + sm), peer);
#pragma unroll
        for (int j = 0; j < 3; ++j)
          st_async_v4(dst + 16 * j, rb, __uint_as_float(w[4 * j]), __uint_as_float(w[4 * j + 1]),
                      __uint_as_float(w[4 * j + 2]), __uint_as_float(w[4 * j + 3]));
      }
    };

    Walk wu, wt;
    wu.init(p, meta);
    wt = wu;
    if (wu.valid) {  // the first chunk's Q, and the first block's partial
      if (active) store_q(wu.req);
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && !(p.withhold_q_ready && sm == 0)) mbar_arrive(bar(kQtFull));
      send_partial(0, wu);
      wu.next(p);
    }
    uint32_t u = 1;
    float m = -INFINITY, l = 0.f;  // m: exponent reference (log2 units), l: this thread's keys' row sum relative to it
    for (uint32_t t = 0; wt.valid; ++t, wt.next(p)) {
      if (aborted(wctl)) break;
      // ---- block t: own partial + the peer's, then release the score buffer.  Only this CTA
      // computes the scores of its keys (the peer gets their P), so its own partial keeps full
      // precision; the peer's arrives rounded to 24 bits.
      const int b = t & 1;
      float x[kOwnN];
      bool got = false;
      if (active) {
        got = mbar_wait<true>(bar(kXFull + sm), t & 1, wctl, err, kDevErrTimeout);
        __syncwarp();
        uint32_t r[16];
        tmem_ld16(t_lane + kColS + 64 * b + own_col, r);
        tmem_wait_ld();
        const uint8_t* rcv_row = smem + kOffRcv + sm * kXWarp + lane * kRowBytes;
        const uint4 c0 = *reinterpret_cast<const uint4*>(rcv_row);
        const uint4 c1 = *reinterpret_cast<const uint4*>(rcv_row + 16);
        const uint4 c2 = *reinterpret_cast<const uint4*>(rcv_row + 32);
        const uint32_t wv[12] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w, c2.x, c2.y, c2.z, c2.w};
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          float a0, a1, a2, a3;
          unpack24(wv[3 * g], wv[3 * g + 1], wv[3 * g + 2], a0, a1, a2, a3);
          const int c = 4 * g;
          x[c] = __uint_as_float(r[c]) + a0;
          x[c + 1] = __uint_as_float(r[c + 1]) + a1;
          x[c + 2] = __uint_as_float(r[c + 2]) + a2;
          x[c + 3] = __uint_as_float(r[c + 3]) + a3;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kSEmpty + b));  // Q.K^T of block t + 2 may overwrite the scores

      if (wt.first()) {
        m = -INFINITY;
        l = 0.f;
      }
      float mx = -INFINITY;  // this thread's maximum of the block's scaled scores
      if (active) {
        // ---- online softmax in log2 units
        int limit = 0;
        if (row_g < R) {
          limit = p.causal ? wt.L - (p.s_q - 1 - row_g / p.h_q) : wt.L;
          limit = limit < 0 ? 0 : limit;
        }
        const int kbase = wt.blk * kBlockN + own_col;
        if (__all_sync(0xffffffffu, kbase + kOwnN <= limit)) {
#pragma unroll
          for (int c = 0; c < kOwnN; ++c) {
            x[c] *= p.scale_log2;
            mx = fmaxf(mx, x[c]);
          }
        } else {
#pragma unroll
          for (int c = 0; c < kOwnN; ++c) {
            x[c] = (kbase + c < limit) ? x[c] * p.scale_log2 : -INFINITY;
            mx = fmaxf(mx, x[c]);
          }
        }
        __syncwarp();
        if (lane == 0) {
          // every lane's mx was computed from every word it read from the receive slot, so those
          // reads are complete: arm the slot's next phase, then let the peer refill it (a relaxed
          // arrive; a release at cluster scope costs ~1000 cycles here)
          if (got) mbar_arrive_expect_tx(bar(kXFull + sm), kXWarp);
          mbar_arrive_cluster_relaxed_after(mapa(bar(kXEmpty + sm), peer), mx);
        }
        xchg_post(mx);
      }
      if (wu.valid) {  // block t + 1's partial travels while block t's maximum does
        send_partial(u, wu);
        wu.next(p);
        ++u;
      }
      if (!active) {
        const bool freed = mbar_wait(bar(kPEmpty), (t & 1) ^ 1, wctl, err, kDevErrTimeout);
        __syncwarp();
        if (lane == 0 && freed) {
          if (sm == 0)
            mbar_arrive_expect_tx(bar(kPFull), active_quadrants * 2 * 1024);
          else
            mbar_arrive(bar(kPFull));
        }
      } else {
        // the row's maximum over all 64 keys, the same in both CTAs
        {
          float v[4];
          xchg_wait(v);
          mx = fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3]));
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
        float s0 = 0.f, s1 = 0.f;
        uint32_t pk[kOwnN / 2];
#pragma unroll
        for (int c2 = 0; c2 < kOwnN / 2; ++c2) {
          const float p0 = ex2(x[2 * c2] - base);
          const float p1 = ex2(x[2 * c2 + 1] - base);
          s0 += p0;
          s1 += p1;
          pk[c2] = pack2<kBF16>(p0, p1);
        }
        l = l * alpha + (s0 + s1);

        // P (this thread's 16 keys of the row), once this CTA's previous P.V has read P (so O also
        // holds every earlier block); then tell the peer it may copy its part of P here
        const bool freed = mbar_wait(bar(kPEmpty), (t & 1) ^ 1, wctl, err, kDevErrTimeout);
        if (lane == 0) {
          mbar_arrive_cluster_relaxed_after(mapa(bar(kPeerFree + sm), peer), 0.f);
          bulk_wait_read_all();  // this piece's copy of the previous block is done
        }
        __syncwarp();
        tc_fence_after();
        {
          uint8_t* prow = smem + kOffP + (2 * crank + sub) * kPTile + row * 32;
          const int sw = (row >> 2) & 1;  // 32-byte swizzle: 16-byte chunk index ^ address bit 7
          *reinterpret_cast<uint4*>(prow + ((0 ^ sw) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4*>(prow + ((1 ^ sw) << 4)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
        fence_proxy_async_smem();  // P is read by the tensor core and the bulk copy (async proxy)
        __syncwarp();
        if (lane == 0) {
          // the peer's P.V of the previous block has read its P too
          mbar_wait<true>(bar(kPeerFree + sm), t & 1, wctl, err, kDevErrTimeout);
          bulk_copy_to_peer(mapa(p_piece, peer), p_piece, 1024, mapa(bar(kPFull), peer));
          bulk_commit_group();
        }
        if (__any_sync(0xffffffffu, resc)) {
          // only blocks after the chunk's first can move an established reference, so O holds
          // the chunk's earlier blocks here; each warp of the quadrant rescales 128 of the 256 columns
#pragma unroll 1
          for (int k = 0; k < 4; ++k) {
            uint32_t o[32];
            const uint32_t ta = t_lane + kColO + 128 * sub + 32 * k;
            tmem_ld32(ta, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(ta, o);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0 && freed) {
          if (sm == 0)
            mbar_arrive_expect_tx(bar(kPFull), active_quadrants * 2 * 1024);
          else
            mbar_arrive(bar(kPFull));
        }
        __syncwarp();
      }

      if (!wt.last()) continue;
      // ---- epilogue of the chunk: normalise this CTA's O half and write it
      float lt = 0.f;
      if (active) {
        float v[4];
        xchg_post(l);
        xchg_wait(v);
        lt = (v[0] + v[1]) + (v[2] + v[3]);  // the same order in both CTAs
      }
      mbar_wait(bar(kOFinal), wt.chunk & 1, wctl, err, kDevErrTimeout);
      __syncwarp();
      tc_fence_after();
      if (active) {
        const bool whole = (wt.lo == 0 && wt.hi == wt.n);
        const int split_idx = (wt.req == wt.br) ? meta[4] : 0;
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
        const int64_t chunk_row =
            whole ? 0 : (static_cast<int64_t>(p.num_splits[wt.req] + split_idx) * R + row_g);
#pragma unroll 1
        for (int k = 0; k < 4; ++k) {
          uint32_t o[32];
          tmem_ld32(t_lane + kColO + 128 * sub + 32 * k, o);
          tmem_wait_ld();
          if (row_g < R) {
            const int col = static_cast<int>(crank) * 256 + 128 * sub + 32 * k;
            if (whole) {
              uint4* dst = reinterpret_cast<uint4*>(
                  reinterpret_cast<uint16_t*>(p.out) + (static_cast<int64_t>(wt.req) * R + row_g) * kDV + col);
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
        if (crank == 0 && sub == 0 && row_g < R) {
          const float lse_v = lt > 0.f ? (m + log2f(lt)) * 0.69314718055994531f : -INFINITY;
          if (whole) {
            const int s = row_g / p.h_q, h = row_g % p.h_q;
            p.lse[static_cast<int64_t>(wt.req) * R + h * p.s_q + s] = lse_v;
          } else {
            p.lse_acc[chunk_row] = lse_v;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kOEmpty));
    }
    if (lane == 0) bulk_wait_read_all();
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
int splitkv_threads() { return splitkv::kThreads; }

const void* splitkv_kernel_ptr(bool bf16) {
  return bf16 ? reinterpret_cast<const void*>(&splitkv::splitkv_pair_kernel<true>)
              : reinterpret_cast<const void*>(&splitkv::splitkv_pair_kernel<false>);
}

cudaError_t launch_splitkv(bool bf16, const void* q, const CUtensorMap& qrmap, const CUtensorMap& kmap,
                           const CUtensorMap& krmap, const DecodeParams& p, cudaStream_t stream) {
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
  if (bf16) return cudaLaunchKernelEx(&cfg, splitkv::splitkv_pair_kernel<true>, q, qrmap, kmap, krmap, p);
  return cudaLaunchKernelEx(&cfg, splitkv::splitkv_pair_kernel<false>, q, qrmap, kmap, krmap, p);
}

}  // namespace mla
