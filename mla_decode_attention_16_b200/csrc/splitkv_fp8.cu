// Split-KV MLA decode kernel over an FP8 (e5m2) latent cache.
//
// What it computes ("云上AI推理新突破：FlashMLA赋能DeepSeek-V2-Lite提速16%", section
// 3. 动态精度缩放; "DeepSeek开源FlashMLA全解析", section 1.2 计算模式创新): the
// decode of the 16-bit kernels with the query cast to e5m2 (round to nearest
// even, saturating) and Q.K^T formed from the 8-bit operands with fp32
// accumulation; the softmax runs in fp32 and the value product at fp16: P is
// rounded to fp16 and V, the first 512 e5m2 values of each cached row, is
// widened to fp16 (exact: e5m2 is the top byte of an fp16).  Output, lse and
// the split-KV partials are those of the 16-bit path, in q's dtype.
//
// A 64-token page is 36 KB instead of 72 KB, so with few query rows the page
// stream is what bounds the kernel (the cost model of "FlashMLA 在 Hopper GPU 上的
// MHA 内核调度优化解析", 计算边界特性与优化方向抉择, at one byte per value).  Per page:
//   S [rows x 64]    = Q8 . K8^T  tcgen05.mma.kind::f8f6f4, M = 128 lanes, A = Q8
//                                 in TMEM (4 values per column), B = the page's
//                                 four 128-column boxes (128-byte swizzle) and its
//                                 64-column box (64-byte swizzle); K = 32 per
//                                 MMA: 18 MMAs
//   V16 [64 x 512]   = widen(page columns 0..511), by two converter warps from
//                      the page stage into a 64 KB shared-memory tile laid out as
//                      the 16-bit kernels' page boxes (128-byte swizzle)
//   O [rows x 512]  += P16 . V16  weight-stationary M = 32, N = 256: 8 MMAs
// S is double-buffered in TMEM (the query in e5m2 takes only 144 columns), so the
// next page's Q.K^T is issued while the softmax still works on this one.
// The page stage is released once its Q.K^T and its conversion are done (not
// after the P.V that follows the next page), so four 36 KB stages keep about
// three pages in flight per SM.  V16 is converted in two halves of 256 values,
// each with its own full/empty barrier pair, so converting page t+1 overlaps
// the second half of page t's P.V.
//
// Query rows come in tiles of up to 32 (rows = s_q * h_q, row = s * h_q + h):
// the CTA for (partition p, tile t) is block p * T + t with T = ceil(rows / 32),
// so the T CTAs of a partition read the same pages at the same time and share
// them through L2.
//
// Roles (384 threads): warp 0 lane 0 TMA producer; warp 1 TMEM owner, lane 0
// issues the Q.K^T MMAs; warps 2-3 widen V; warps 4-7: warp 4 + (chunk & 1)
// runs a chunk's softmax (one thread per query row), all four rescale O when a
// row's exponent reference moves, and warp 6 lane 0 issues the P.V MMAs; warps
// 8-11 write each chunk's epilogue, and warps 8 / 9 cast and load Q for even /
// odd chunks (Q of consecutive chunks in lane quadrants 0 / 1, so the next
// chunk's Q is written while one runs).  Two issuing threads: one thread
// issuing every MMA (~65 cycles per Q.K^T and ~100 per weight-stationary P.V
// instruction, plus its waits and commits) was the bottleneck at ~3,400 cycles
// per page while the tensor pipe was busy for ~900; tcgen05.commit tracks the
// issuing thread's own MMAs, so each issuer commits its own barriers.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <cmath>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace mla {
namespace fp8 {

using namespace ptx;

constexpr int kThreads = 384;
constexpr int kRowTile = 32;                    // query rows per CTA
constexpr int kBox8 = kPage * 128;              // 8 KB: one page x 128 e5m2 columns
constexpr int kBoxR = kPage * 64;               // 4 KB: one page x columns 512..575
constexpr int kStageBytes = 4 * kBox8 + kBoxR;  // 36 KB: one page
constexpr int kStages = 4;
constexpr int kVBox = kPage * 128;              // 8 KB: one page x 64 fp16 values
constexpr int kQCols = kDK / 4;                 // 144 TMEM columns: 4 e5m2 values each
constexpr float kRescaleThreshold = 8.0f;       // see splitkv.cu

enum Bar {
  kKvFull = 0,
  kKvEmpty = kKvFull + kStages,  // count 3: the Q.K^T commit + one arrival per converter warp
  kQFull = kKvEmpty + kStages,   // [2] Q rows of a chunk parity written to TMEM
  kQEmpty = kQFull + 2,          // [2] last Q.K^T of a chunk of that parity completed
  kSFull = kQEmpty + 2,          // [2] S buffer of page parity b written
  kSEmpty = kSFull + 2,          // [2] S buffer read by the softmax
  kPFull = kSEmpty + 2,                        // [2] count 4
  kPEmpty = kPFull + 2,          // [2]
  kVFull = kPEmpty + 2,          // [2] half h of V16 written (count 2: one per converter warp)
  kVEmpty = kVFull + 2,          // [2] the P.V MMAs that read half h completed
  kODone = kVEmpty + 2,          // one phase per P.V
  kOFinal,                       // one phase per chunk
  kOEmpty,                       // count 4: epilogue finished reading O
  kStats = kOEmpty + 1,          // [2] row sums / reference maxima of a chunk parity in smem
  kDrain = kStats + 2,           // Q.K^T issuer's tensor-core work drained
  kDrainPV,                      // P.V issuer's tensor-core work drained
  kNumBars
};

template <int NP>
struct Layout {
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kStages * kStageBytes;  // 1024-aligned
  static constexpr int kOffP = kOffV + 8 * kVBox;
  static constexpr int kPBytes = 32 * 128;  // P: 32 rows (M of the P.V MMA) x 64 keys, fp16
  static constexpr int kOffRed = kOffP + 2 * kPBytes;
  // floats: alpha [2][NP], flag [2], row sums [2][NP], reference max [2][NP]
  static constexpr int kRedFloats = 2 * NP + 2 + 2 * NP + 2 * NP;
  static constexpr int kOffBar = (kOffRed + kRedFloats * 4 + 7) / 8 * 8;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 8 + sizeof(WaitCtl) + 1024;
  static_assert(kOffV % 1024 == 0 && kOffP % 1024 == 0 && kStageBytes % 1024 == 0, "swizzle atom alignment");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColO = 0;  // O: 2 halves of 256 values x 64 columns (see umma_ws_ss)
  static constexpr uint32_t kColS = kColO + 128;  // S: two buffers of 64 columns (page parity)
  static constexpr uint32_t kColQ = kColS + 2 * kPage;
  static_assert(kColQ + kQCols <= kTmemCols, "TMEM budget");
};

template <bool kBF16>
__device__ __forceinline__ uint32_t pack_out(float a, float b) {
  if constexpr (kBF16) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
  } else {
    __half2 v = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
  }
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  __half2 v = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
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
    splitkv_fp8_kernel(const void* __restrict__ qptr, const __grid_constant__ CUtensorMap kmap,
                       const __grid_constant__ CUtensorMap krmap, const DecodeParams p) {
  using Lay = Layout<NP>;
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
  const int tiles = (p.rows + kRowTile - 1) / kRowTile;
  const int part = blockIdx.x / tiles;
  const int r0 = (blockIdx.x % tiles) * kRowTile;  // first query row of this CTA
  const int R = p.rows;
  const int Rt = R - r0 < kRowTile ? R - r0 : kRowTile;  // query rows of this CTA

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      uint32_t count = 1;
      if ((i >= kKvEmpty && i < kKvEmpty + kStages)) count = 3;
      if (i == kPFull || i == kPFull + 1 || i == kOEmpty) count = 4;
      if (i == kVFull || i == kVFull + 1) count = 2;
      mbar_init(bar(i), count);
    }
    wctl->abort = 0;
    wctl->limit = p.wait_cycles;
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
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // launched as a programmatic dependent of the previous kernel in the stream (normally the
  // scheduler): the prologue above overlapped it; nothing it wrote is read before this wait
  pdl_wait_primary();
  if (threadIdx.x == 0) pdl_launch_dependents();

  const int* meta = p.meta + part * kMetaInts;
  const int br = meta[0], bk = meta[1], er = meta[2], ek = meta[3], bs = meta[4];
  int* err = p.err;

  // O[:, 256h ..] += P[:, 16kk ..] . V16[16kk .., 256h ..] for page itp (chunk-relative index jjp of
  // chunk `chunk`), issued by warp 6 lane 0 once the four softmax warps have released P.
  // A = P (32 rows, K-major), B = V16 (MN-major view of value boxes 4h .. 4h+3, 8 KB apart; 16
  // keys = 2 x 1 KB).
  auto issue_pv = [&](uint32_t itp, int jjp, bool last, uint32_t chunk) {
    constexpr uint32_t idesc_pv = idesc_f16(false, 32, 256, false, true);  // fp16 P and V
    const uint32_t vbase = sbase + Lay::kOffV;
    const int b = itp & 1;
    if (jjp == 0) mbar_wait(bar(kOEmpty), (chunk & 1) ^ 1, wctl, err, kDevErrTimeout);
    mbar_wait(bar(kPFull + b), (itp >> 1) & 1, wctl, err, kDevErrTimeout);
    const uint32_t pbuf = sbase + Lay::kOffP + b * Lay::kPBytes;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      mbar_wait(bar(kVFull + h), itp & 1, wctl, err, kDevErrTimeout);
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < kPage / 16; ++kk) {
        const uint64_t adesc = smem_desc_sw128(pbuf + kk * 32, 16, 1024);
        const uint64_t bdesc = smem_desc_sw128(vbase + (4 * h) * kVBox + kk * 2048, kVBox, 1024);
        umma_ws_ss(tmem + Lay::kColO + 64 * h, adesc, bdesc, idesc_pv, (jjp > 0 || kk > 0) ? 1u : 0u);
      }
      umma_commit(bar(kVEmpty + h));
    }
    umma_commit(bar(kPEmpty + b));
    umma_commit(bar(kODone));
    if (last) umma_commit(bar(kOFinal));
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (pages only)
    if (lane == 0) {
      const uint64_t evict_first = policy_evict_first();
      uint32_t it = 0;
      int cur = br;
      Chunk ch;
      while (!aborted(wctl) && next_chunk(p, br, bk, er, ek, bs, cur, ch)) {
        const int32_t* bt = p.block_table + static_cast<int64_t>(ch.req) * p.block_table_stride;
        int page_next = bt[ch.lo];
        for (int blk = ch.lo; blk < ch.hi; ++blk, ++it) {
          if (aborted(wctl)) break;
          const int st = it % kStages;
          int page = page_next;
          if (blk + 1 < ch.hi) page_next = bt[blk + 1];  // read while this stage frees up
          if (!mbar_wait(bar(kKvEmpty + st), ((it / kStages) & 1) ^ 1, wctl, err, kDevErrTimeout)) break;
          if (page < 0 || static_cast<int64_t>(page) >= p.num_pages) {
            atomicOr(err, kDevErrPage);
            atomicCAS(err + 1, 0, page == 0 ? -1 : page);
            page = 0;
          }
          const uint32_t dst = sbase + Lay::kOffK + st * kStageBytes;
          mbar_arrive_expect_tx(bar(kKvFull + st), kStageBytes);
          for (int i = 0; i < 4; ++i)
            tma_load_3d_hint(dst + i * kBox8, &kmap, bar(kKvFull + st), 128 * i, 0, page, evict_first);
          tma_load_3d_hint(dst + 4 * kBox8, &krmap, bar(kKvFull + st), 512, 0, page, evict_first);
        }
      }
      // Before the CTA can exit, every page load issued above must have landed: wait (bounded, abort
      // or not) for the last phase of each stage.  A phase already consumed has completed, so the
      // wait returns at once; only an abort leaves one pending.
      for (uint32_t j = it > kStages ? it - kStages : 0; j < it; ++j)
        mbar_wait_drain(bar(kKvFull + j % kStages), (j / kStages) & 1, wctl->limit);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ Q.K^T issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_e5m2(128, kPage);
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
          mbar_wait(bar(kSEmpty + (itc & 1)), ((itc >> 1) & 1) ^ 1, wctl, err, kDevErrTimeout);
          tc_fence_after();
          const uint32_t kst = sbase + Lay::kOffK + st * kStageBytes;
          // fully unrolled: the descriptors become constants plus the stage base (a rolled loop
          // that picks the box form at run time spent ~95 extra cycles per MMA in this thread,
          // the kernel's bottleneck)
#pragma unroll
          for (int s = 0; s < kDK / 32; ++s) {
            // 32 columns per MMA: columns 0..511 from the four 128-column boxes (4 steps of 32
            // bytes each), 512..575 from the 64-column box (2 steps)
            const uint64_t bdesc = s < 16 ? smem_desc_sw128(kst + (s >> 2) * kBox8 + (s & 3) * 32, 16, 1024)
                                          : smem_desc_sw64(kst + 4 * kBox8 + (s - 16) * 32, 16, 512);
            umma_ts_e5m2(tmem + Lay::kColS + kPage * (itc & 1), tmem + Lay::kColQ + 8 * s, bdesc, idesc_qk,
                         s > 0 ? 1u : 0u);
          }
          umma_commit(bar(kSFull + (itc & 1)));
          umma_commit(bar(kKvEmpty + st));
          if (jj == nb - 1) umma_commit(bar(kQEmpty + qpar));
        }
        it += nb;
        ++chunk;
      }
      umma_commit(bar(kDrain));
      mbar_wait_drain(bar(kDrain), 0, wctl->limit);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ V widening (e5m2 -> fp16)
    const int ct = threadIdx.x - 64;  // 0 .. 63
    uint32_t it = 0;
    int cur = br;
    Chunk ch;
    while (!aborted(wctl) && next_chunk(p, br, bk, er, ek, bs, cur, ch)) {
      for (int blk = ch.lo; blk < ch.hi; ++blk, ++it) {
        if (aborted(wctl)) break;
        const int st = it % kStages;
        mbar_wait(bar(kKvFull + st), (it / kStages) & 1, wctl, err, kDevErrTimeout);
        const uint8_t* kst = smem + Lay::kOffK + st * kStageBytes;
        uint8_t* vdst = smem + Lay::kOffV;
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          mbar_wait(bar(kVEmpty + h), (it & 1) ^ 1, wctl, err, kDevErrTimeout);
          // values 256h .. 256h+255 = e5m2 boxes 2h, 2h+1: thread ct widens key row ct of both boxes
          // (8 16-byte pieces each; piece c holds values 128i + 16c .., stored at piece c ^ (row & 7)
          // by the 128-byte swizzle) into fp16 boxes 4h .. 4h+3 (each e5m2 byte b is the fp16 with
          // bits b << 8).  All 16 loads are issued before the first store, so they overlap instead
          // of each waiting behind the stores before it.  16-byte accesses are served 8 threads
          // at a time, here 8 consecutive rows: the XOR swizzle spreads their loads and each of
          // their two stores over 8 different 16-byte bank groups.
          const int k = ct;
          uint4 xs[16];
#pragma unroll
          for (int n = 0; n < 16; ++n) {
            const int i = 2 * h + (n >> 3), c = n & 7;
            xs[n] = *reinterpret_cast<const uint4*>(kst + i * kBox8 + k * 128 + ((c ^ (k & 7)) << 4));
          }
#pragma unroll
          for (int n = 0; n < 16; ++n) {
            const int i = 2 * h + (n >> 3), c = n & 7;
            const uint4 x = xs[n];
            const uint4 lo = make_uint4(__byte_perm(x.x, 0, 0x1404), __byte_perm(x.x, 0, 0x3424),
                                        __byte_perm(x.y, 0, 0x1404), __byte_perm(x.y, 0, 0x3424));
            const uint4 hi = make_uint4(__byte_perm(x.z, 0, 0x1404), __byte_perm(x.z, 0, 0x3424),
                                        __byte_perm(x.w, 0, 0x1404), __byte_perm(x.w, 0, 0x3424));
            const int j0 = 2 * (c & 3);  // logical fp16 pieces j0, j0 + 1 of the row in box 2i + c / 4
            uint8_t* row = vdst + (2 * i + (c >> 2)) * kVBox + k * 128;
            *reinterpret_cast<uint4*>(row + ((j0 ^ (k & 7)) << 4)) = lo;
            *reinterpret_cast<uint4*>(row + (((j0 + 1) ^ (k & 7)) << 4)) = hi;
          }
          fence_proxy_async_smem();  // V16 is read by the tensor core (async proxy)
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(kVFull + h));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kKvEmpty + st));
      }
    }
  } else if (warp < 8) {
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
      int limit = 0;
      if (smx && row < Rt) {
        limit = p.causal ? ch.L - (p.s_q - 1 - (r0 + row) / p.h_q) : ch.L;
        limit = limit < 0 ? 0 : limit;
      }
      float m = -INFINITY, l = 0.f;
      for (int jj = 0; jj < nb; ++jj) {
        const uint32_t itc = it + jj;
        const int b = itc & 1;
        if (smx) {
          mbar_wait(bar(kSFull + b), (itc >> 1) & 1, wctl, err, kDevErrTimeout);
          __syncwarp();
          tc_fence_after();
          float x[kKeys];
          {
            // tcgen05.ld takes one column address for the whole warp: every lane loads both
            // 32-column halves and keeps its own (all 64 columns when a lane owns a whole row)
            uint32_t v0[32], v1[32];
            tmem_ld32(t_lane + Lay::kColS + kPage * b, v0);
            tmem_ld32(t_lane + Lay::kColS + kPage * b + 32, v1);
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
          if (lane == 0) mbar_arrive(bar(kSEmpty + b));

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
            pk[c2] = pack_half2(p0, p1);
          }
          l = l * alpha + sum;  // this lane's keys of the row
          const bool any_resc = __any_sync(0xffffffffu, resc);
          if (half == 0 && row < NP) s_alpha[b * NP + row] = alpha;
          if (lane == 0) s_flag[b] = any_resc ? 1 : 0;
          mbar_wait(bar(kPEmpty + b), ((itc >> 1) & 1) ^ 1, wctl, err, kDevErrTimeout);
          if (row < NP) {
            // P row: 64 keys = 128 bytes, 16-byte pieces XOR-swizzled by row (128-byte swizzle);
            // this lane's keys are pieces (kKeys / 8) * half ..
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
            const uint32_t col = Lay::kColO + 32 * c32;
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
        if (warp == 6) {  // this page's P.V (after all four warps arrived: P written, O rescaled)
          if (lane == 0 && !aborted(wctl)) issue_pv(itc, jj, jj == nb - 1, chunk);
          __syncwarp();
        }
      }
      if (smx) {
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
    if (warp == 6 && lane == 0) {
      umma_commit(bar(kDrainPV));
      mbar_wait_drain(bar(kDrainPV), 0, wctl->limit);
    }
  } else {
    // ------------------------------------------------------------ Q loads (warps 8 / 9) and epilogue (8-11)
    const int q4 = warp & 3;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const int r = lane;
    auto load_q = [&](const Chunk& c, uint32_t idx) {
      // Q rows of chunk idx, cast to e5m2, into lane quadrant idx & 1 (this warp's quadrant)
      mbar_wait(bar(kQEmpty + (idx & 1)), ((idx >> 1) & 1) ^ 1, wctl, err, kDevErrTimeout);
      __syncwarp();
      tc_fence_after();
      // with 16 rows, lanes r and r + 16 both hold row r (see the softmax)
      const int qr = NP == 16 ? (r & 15) : r;
      const uint4* qrow = reinterpret_cast<const uint4*>(
          reinterpret_cast<const uint16_t*>(qptr) + (static_cast<int64_t>(c.req) * R + r0 + (qr < Rt ? qr : 0)) * kDK);
#pragma unroll 1
      for (int c16 = 0; c16 < kQCols / 16; ++c16) {
        uint32_t w[16];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          uint4 d = make_uint4(0, 0, 0, 0);
          if (qr < Rt) d = __ldg(qrow + c16 * 8 + v);
          w[2 * v] = cast4_e5m2<kBF16>(d.x, d.y);
          w[2 * v + 1] = cast4_e5m2<kBF16>(d.z, d.w);
        }
        tmem_st16(t_lane + Lay::kColQ + 16 * c16, w);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && !(p.withhold_q_ready && idx == 0)) mbar_arrive(bar(kQFull + (idx & 1)));
    };
    auto epilogue = [&](const Chunk& c, uint32_t idx) {
      const int par = idx & 1;
      mbar_wait(bar(kOFinal), idx & 1, wctl, err, kDevErrTimeout);
      mbar_wait(bar(kStats + par), (idx >> 1) & 1, wctl, err, kDevErrTimeout);
      __syncwarp();
      tc_fence_after();
      const bool whole = (c.lo == 0 && c.hi == c.n);
      const int64_t chunk0 = whole ? 0 : static_cast<int64_t>(p.num_splits[c.req] + c.split) * R;
      const float* ls = s_lsum + par * NP;
      // lane r of quadrant q4 holds row r, values 256h + 64 q4 + (0..63) of each half h
      const float lr = r < NP ? ls[r] : 0.f;
      const float inv = lr > 0.f ? 1.f / lr : 0.f;
      const int64_t rg = r0 + r;  // query row within the request
#pragma unroll 1
      for (int c32 = 0; c32 < 4; ++c32) {
        uint32_t o[32];
        tmem_ld32(t_lane + Lay::kColO + 32 * c32, o);
        tmem_wait_ld();
        if (r < Rt) {
          const int d = (c32 >> 1) * 256 + q4 * 64 + (c32 & 1) * 32;
          if (whole) {
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.out) +
                                                  (static_cast<int64_t>(c.req) * R + rg) * kDV + d);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 w;
              w.x = pack_out<kBF16>(__uint_as_float(o[8 * v + 0]) * inv, __uint_as_float(o[8 * v + 1]) * inv);
              w.y = pack_out<kBF16>(__uint_as_float(o[8 * v + 2]) * inv, __uint_as_float(o[8 * v + 3]) * inv);
              w.z = pack_out<kBF16>(__uint_as_float(o[8 * v + 4]) * inv, __uint_as_float(o[8 * v + 5]) * inv);
              w.w = pack_out<kBF16>(__uint_as_float(o[8 * v + 6]) * inv, __uint_as_float(o[8 * v + 7]) * inv);
              dst[v] = w;
            }
          } else {
            float4* dst = reinterpret_cast<float4*>(p.o_acc + (chunk0 + rg) * kDV + d);
#pragma unroll
            for (int v = 0; v < 8; ++v)
              dst[v] = make_float4(__uint_as_float(o[4 * v]) * inv, __uint_as_float(o[4 * v + 1]) * inv,
                                   __uint_as_float(o[4 * v + 2]) * inv, __uint_as_float(o[4 * v + 3]) * inv);
          }
        }
      }
      if (q4 == 0 && r < Rt) {
        const float lr0 = ls[r];
        const float lse_v = lr0 > 0.f ? (s_mref[par * NP + r] + log2f(lr0)) * 0.69314718055994531f : -INFINITY;
        if (whole) {
          const int s = static_cast<int>(rg) / p.h_q, h = static_cast<int>(rg) % p.h_q;
          p.lse[static_cast<int64_t>(c.req) * R + h * p.s_q + s] = lse_v;
        } else {
          p.lse_acc[chunk0 + rg] = lse_v;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kOEmpty));
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
  return bf16 ? reinterpret_cast<const void*>(&splitkv_fp8_kernel<true, NP>)
              : reinterpret_cast<const void*>(&splitkv_fp8_kernel<false, NP>);
}

}  // namespace fp8

int fp8_rows_padded(int rows) { return rows <= 16 ? 16 : 32; }
int fp8_row_tiles(int rows) { return (rows + fp8::kRowTile - 1) / fp8::kRowTile; }

int fp8_smem_bytes(int np) { return np == 16 ? fp8::Layout<16>::kSmemBytes : fp8::Layout<32>::kSmemBytes; }

const void* fp8_kernel_ptr(bool bf16, int np) {
  return np == 16 ? fp8::kernel_ptr<16>(bf16) : fp8::kernel_ptr<32>(bf16);
}

cudaError_t launch_splitkv_fp8(bool bf16, const void* q, const CUtensorMap& kmap, const CUtensorMap& krmap,
                               const DecodeParams& p, cudaStream_t stream) {
  const int np = fp8_rows_padded(p.rows);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.num_parts * fp8_row_tiles(p.rows));
  cfg.blockDim = dim3(fp8::kThreads);
  cfg.dynamicSmemBytes = fp8_smem_bytes(np);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (np == 16) {
    if (bf16) return cudaLaunchKernelEx(&cfg, fp8::splitkv_fp8_kernel<true, 16>, q, kmap, krmap, p);
    return cudaLaunchKernelEx(&cfg, fp8::splitkv_fp8_kernel<false, 16>, q, kmap, krmap, p);
  }
  if (bf16) return cudaLaunchKernelEx(&cfg, fp8::splitkv_fp8_kernel<true, 32>, q, kmap, krmap, p);
  return cudaLaunchKernelEx(&cfg, fp8::splitkv_fp8_kernel<false, 32>, q, kmap, krmap, p);
}

}  // namespace mla
