// Split-KV MLA decode over an FP8 (e5m2) latent cache for many query rows
// (s_q * h_q > 32): 128-row tiles.
//
// Same computation as splitkv_fp8.cu ("云上AI推理新突破：FlashMLA赋能DeepSeek-V2-Lite提速16%",
// section 3. 动态精度缩放): q cast to e5m2, S = scale * Q8 . K8^T with fp32
// accumulation, softmax in fp32, P rounded to fp16, O += P16 . V16 with V the
// page's first 512 e5m2 values widened to fp16.
//
// A 128 x 512 fp32 output tile alone fills an SM's 512 TMEM columns, so a tile
// is split by value between two CTAs (no cluster: they share only the pages,
// through L2).  Because the query in e5m2 is small (128 TMEM columns plus an
// 8 KB tile), each CTA holds all of Q and computes the whole S itself: the two CTAs of a tile do the
// same Q.K^T (18 8-bit MMAs per page, M = 128) and the same softmax, and each
// widens and multiplies only its own 256 values of V.  Nothing is exchanged
// between SMs (the 16-bit row-tile kernel splits the contraction instead and
// trades partial scores, maxima and P through distributed shared memory).
// Per 64-token page and CTA:
//   S [128 x 64]     = Q8 . K8^T     tcgen05.mma.kind::f8f6f4, 18 MMAs: A = Q8 columns
//                                    0..511 in TMEM, 512..575 in shared memory
//   V16 [64 x 256]   = widen(page columns 256c .. 256c+255), two converter warps
//   O [128 x 256]   += P16 . V16     tcgen05.mma.kind::f16, M = 128, N = 256: 4 MMAs
// TMEM: O 256 columns, S 2 x 64, Q 128 (the query's last 64 e5m2 values sit in a
// 64-byte-swizzled shared-memory tile so that S fits twice).  Shared memory:
// three 36 KB page stages, V16 2 x 32 KB, P 2 x 16 KB, Q 8 KB.
//
// CTA (partition p, row tile t, value half c) is block (p * T + t) * 2 + c,
// T = ceil(rows / 128), so the 2T CTAs of a partition are adjacent and read the
// same pages at the same time.
//
// Roles (384 threads): warp 0 lane 0 issues the page loads (TMA) and the P.V
// MMAs, whichever has its inputs first (a load is a few instructions; one
// thread issuing both products had been the bottleneck, ~3,300 cycles per page
// with the M = 128, N = 256 P.V MMAs taking ~300 each, and the converter
// issuing P.V put its ~1,000 cycles on the widening chain); warp 1 TMEM owner,
// lane 0 issues the Q.K^T MMAs (S double-buffered: up to two pages ahead of the
// softmax); warps 2-3 widen V into two alternating buffers; warps 4-7 run the
// softmax of the rows of their lane quadrant (one thread per row) and rescale
// those rows of O; warps 8-11 cast and load the Q rows of their quadrant and
// write its epilogue.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <cmath>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace mla {
namespace fp8rt {

using namespace ptx;

constexpr int kThreads = 384;
constexpr int kTile = 128;                      // query rows per tile (one per TMEM lane)
constexpr int kBox8 = kPage * 128;              // 8 KB: one page x 128 e5m2 columns
constexpr int kBoxR = kPage * 64;               // 4 KB: one page x columns 512..575
constexpr int kStageBytes = 4 * kBox8 + kBoxR;  // 36 KB: one page
constexpr int kStages = 3;
constexpr int kVBox = kPage * 128;              // 8 KB: one page x 64 fp16 values
constexpr int kPBytes = kTile * 128;            // 16 KB: P, 128 rows x 64 keys fp16
constexpr float kRescaleThreshold = 8.0f;       // see splitkv.cu

enum Bar {
  kKvFull = 0,
  kKvEmpty = kKvFull + kStages,  // count 3: the Q.K^T commit + one arrival per converter warp
  kQFull = kKvEmpty + kStages,   // count 4: the Q rows of a chunk written to TMEM
  kQEmpty,                       // the chunk's last Q.K^T completed
  kSFull,                        // [2] S buffer of page parity b written
  kSEmpty = kSFull + 2,          // [2] count 4: every softmax warp read its rows of S
  kPFull = kSEmpty + 2,          // [2] count 4
  kPEmpty = kPFull + 2,          // [2]
  kVFull = kPEmpty + 2,          // [2] count 2: V16 buffer of page parity b written
  kVEmpty = kVFull + 2,          // [2] the P.V MMAs that read that buffer completed
  kODone = kVEmpty + 2,          // one phase per P.V
  kOFinal,                       // one phase per chunk
  kOEmpty,                       // count 4: epilogue finished reading O
  kStats,                        // [2] count 4: row sums / reference maxima of a chunk parity in smem
  kDrain = kStats + 2,           // the Q.K^T issuer's tensor-core work drained
  kDrainPV,                      // the P.V issuer's tensor-core work drained
  kNumBars
};

struct Layout {
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kStages * kStageBytes;
  static constexpr int kOffP = kOffV + 2 * 4 * kVBox;  // V16: two buffers of 256 values x 64 keys
  static constexpr int kOffQR = kOffP + 2 * kPBytes;   // Q columns 512..575: 128 rows x 64 bytes (64-byte swizzle)
  static constexpr int kOffRed = kOffQR + kTile * 64;  // floats: row sums [2][128], reference max [2][128]
  static constexpr int kOffBar = kOffRed + 4 * kTile * 4;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 8 + sizeof(WaitCtl) + 1024;
  static_assert(kOffV % 1024 == 0 && kOffP % 1024 == 0 && kOffQR % 1024 == 0 && kStageBytes % 1024 == 0,
                "swizzle atom alignment");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColO = 0;  // O: 128 rows x this CTA's 256 values
  static constexpr uint32_t kColS = kColO + 256;  // S: two buffers of 64 columns (page parity)
  static constexpr uint32_t kColQ = kColS + 2 * kPage;
  static_assert(kColQ + kDV / 4 <= kTmemCols, "TMEM budget");
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

template <bool kBF16>
__global__ void __launch_bounds__(kThreads, 1)
    splitkv_fp8_rt_kernel(const void* __restrict__ qptr, const __grid_constant__ CUtensorMap kmap,
                          const __grid_constant__ CUtensorMap krmap, const DecodeParams p) {
  using Lay = Layout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + Lay::kOffBar + 8 * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kOffMisc);
  WaitCtl* wctl = reinterpret_cast<WaitCtl*>(smem + Lay::kOffMisc + 8);
  float* s_lsum = reinterpret_cast<float*>(smem + Lay::kOffRed);  // [2][128]
  float* s_mref = s_lsum + 2 * kTile;                              // [2][128]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tiles = (p.rows + kTile - 1) / kTile;
  const int vh = blockIdx.x & 1;                    // value half: values 256 vh .. 256 vh + 255
  const int part = (blockIdx.x >> 1) / tiles;
  const int r0 = ((blockIdx.x >> 1) % tiles) * kTile;  // first query row of this tile
  const int R = p.rows;
  const int Rt = R - r0 < kTile ? R - r0 : kTile;      // query rows of this tile

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      uint32_t count = 1;
      if (i >= kKvEmpty && i < kKvEmpty + kStages) count = 3;
      if (i == kQFull || i == kSEmpty || i == kSEmpty + 1 || i == kPFull || i == kPFull + 1 || i == kOEmpty ||
          i == kStats || i == kStats + 1)
        count = 4;
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
  pdl_wait_primary();
  if (threadIdx.x == 0) pdl_launch_dependents();

  const int* meta = p.meta + part * kMetaInts;
  const int br = meta[0], bk = meta[1], er = meta[2], ek = meta[3], bs = meta[4];
  int* err = p.err;

  if (warp == 0) {
    // ------------------------------------------------------------ page loads and P.V issue
    if (lane == 0) {
      const uint64_t evict_first = policy_evict_first();
      constexpr uint32_t idesc_pv = idesc_f16(false, kTile, 256, false, true);  // fp16 P and V
      Walk wl, wp;
      wl.init(p, meta);
      wp = wl;
      uint32_t tl = 0, tp = 0;
      // The next load needs a free stage; the next P.V needs P, its V16 buffer and, for a chunk's
      // first page, the epilogue having read O.  No phase tested here can run a full phase ahead:
      // its producer waits on this thread's earlier work.
      auto pv_ready = [&]() {
        if (wp.first() && !mbar_test_wait(bar(kOEmpty), (wp.chunk & 1) ^ 1)) return false;
        return mbar_test_wait(bar(kPFull + (tp & 1)), (tp >> 1) & 1) &&
               mbar_test_wait(bar(kVFull + (tp & 1)), (tp >> 1) & 1);
      };
      auto issue_load = [&]() {
        const int st = tl % kStages;
        int page = p.block_table[static_cast<int64_t>(wl.req) * p.block_table_stride + wl.blk];
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
        wl.next(p);
        ++tl;
      };
      auto issue_pv = [&]() {
        // A = P (128 rows, K-major), B = V16 buffer (MN-major view of 4 value boxes, 8 KB apart; 16
        // keys = 2 x 1 KB)
        const int b = tp & 1;
        tc_fence_after();
        const uint32_t pbuf = sbase + Lay::kOffP + b * kPBytes;
        const uint32_t vbase = sbase + Lay::kOffV + b * 4 * kVBox;
#pragma unroll
        for (int kk = 0; kk < kPage / 16; ++kk) {
          const uint64_t adesc = smem_desc_sw128(pbuf + kk * 32, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(vbase + kk * 2048, kVBox, 1024);
          umma_ss(tmem + Lay::kColO, adesc, bdesc, idesc_pv, (!wp.first() || kk > 0) ? 1u : 0u);
        }
        umma_commit(bar(kVEmpty + b));
        umma_commit(bar(kPEmpty + b));
        umma_commit(bar(kODone));
        if (wp.last()) umma_commit(bar(kOFinal));
        wp.next(p);
        ++tp;
      };
      long long idle_since = clock64();
      uint32_t polls = 0;
      while (wp.valid) {
        if (wl.valid && mbar_test_wait(bar(kKvEmpty + tl % kStages), ((tl / kStages) & 1) ^ 1)) {
          issue_load();
        } else if (tp < tl && pv_ready()) {
          issue_pv();
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
      // every page load issued above must land, and every P.V finish, before the CTA exits (bounded,
      // abort or not)
      for (uint32_t j = tl > kStages ? tl - kStages : 0; j < tl; ++j)
        mbar_wait_drain(bar(kKvFull + j % kStages), (j / kStages) & 1, wctl->limit);
      umma_commit(bar(kDrainPV));
      mbar_wait_drain(bar(kDrainPV), 0, wctl->limit);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ Q.K^T issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_e5m2(kTile, kPage);
      const uint32_t qr = sbase + Lay::kOffQR;
      uint32_t it = 0, chunk = 0;
      int cur = br;
      Chunk ch;
      while (!aborted(wctl) && next_chunk(p, br, bk, er, ek, bs, cur, ch)) {
        const int nb = ch.hi - ch.lo;
        mbar_wait(bar(kQFull), chunk & 1, wctl, err, kDevErrTimeout);
        for (int jj = 0; jj < nb; ++jj) {
          const uint32_t itc = it + jj;
          const int st = itc % kStages;
          const int b = itc & 1;
          mbar_wait(bar(kKvFull + st), (itc / kStages) & 1, wctl, err, kDevErrTimeout);
          mbar_wait(bar(kSEmpty + b), ((itc >> 1) & 1) ^ 1, wctl, err, kDevErrTimeout);
          tc_fence_after();
          const uint32_t kst = sbase + Lay::kOffK + st * kStageBytes;
          const uint32_t dS = tmem + Lay::kColS + kPage * b;
#pragma unroll
          for (int s = 0; s < 16; ++s) {  // columns 0..511: Q from TMEM, the page's four 128-column boxes
            const uint64_t bdesc = smem_desc_sw128(kst + (s >> 2) * kBox8 + (s & 3) * 32, 16, 1024);
            umma_ts_e5m2(dS, tmem + Lay::kColQ + 8 * s, bdesc, idesc_qk, s > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int i = 0; i < 2; ++i) {  // columns 512..575: Q and the page's 64-column box from shared memory
            const uint64_t adesc = smem_desc_sw64(qr + i * 32, 16, 512);
            const uint64_t bdesc = smem_desc_sw64(kst + 4 * kBox8 + i * 32, 16, 512);
            umma_ss_e5m2(dS, adesc, bdesc, idesc_qk, 1u);
          }
          umma_commit(bar(kSFull + b));
          umma_commit(bar(kKvEmpty + st));
          if (jj == nb - 1) umma_commit(bar(kQEmpty));
        }
        it += nb;
        ++chunk;
      }
      umma_commit(bar(kDrain));
      mbar_wait_drain(bar(kDrain), 0, wctl->limit);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ V widening (this CTA's 256 values)
    const int k = threadIdx.x - 64;  // key row 0 .. 63 of the page
    uint32_t it = 0;
    int cur = br;
    Chunk ch;
    while (!aborted(wctl) && next_chunk(p, br, bk, er, ek, bs, cur, ch)) {
      for (int blk = ch.lo; blk < ch.hi; ++blk, ++it) {
        if (aborted(wctl)) break;
        const int st = it % kStages;
        mbar_wait(bar(kKvFull + st), (it / kStages) & 1, wctl, err, kDevErrTimeout);
        const uint8_t* kst = smem + Lay::kOffK + st * kStageBytes;
        const int vb = it & 1;  // V16 buffer of this page
        uint8_t* vdst = smem + Lay::kOffV + vb * 4 * kVBox;
        mbar_wait(bar(kVEmpty + vb), ((it >> 1) & 1) ^ 1, wctl, err, kDevErrTimeout);
        // e5m2 boxes 2 vh, 2 vh + 1 (values 256 vh ..): thread k widens key row k (8 16-byte pieces
        // per box; piece c holds values 128i + 16c .., stored at piece c ^ (row & 7) by the 128-byte
        // swizzle) into fp16 boxes 0..3 (each e5m2 byte b is the fp16 with bits b << 8).  The 16
        // loads are issued before the first store; 8 consecutive rows share each 16-byte access,
        // so the swizzle puts their loads and stores on 8 different bank groups.
        uint4 xs[16];
#pragma unroll
        for (int n = 0; n < 16; ++n) {
          const int i = 2 * vh + (n >> 3), c = n & 7;
          xs[n] = *reinterpret_cast<const uint4*>(kst + i * kBox8 + k * 128 + ((c ^ (k & 7)) << 4));
        }
#pragma unroll
        for (int n = 0; n < 16; ++n) {
          const int c = n & 7;
          const uint4 x = xs[n];
          const uint4 lo = make_uint4(__byte_perm(x.x, 0, 0x1404), __byte_perm(x.x, 0, 0x3424),
                                      __byte_perm(x.y, 0, 0x1404), __byte_perm(x.y, 0, 0x3424));
          const uint4 hi = make_uint4(__byte_perm(x.z, 0, 0x1404), __byte_perm(x.z, 0, 0x3424),
                                      __byte_perm(x.w, 0, 0x1404), __byte_perm(x.w, 0, 0x3424));
          const int j0 = 2 * (c & 3);  // logical fp16 pieces j0, j0 + 1 of the row in box 2 (n / 8) + c / 4
          uint8_t* row = vdst + (2 * (n >> 3) + (c >> 2)) * kVBox + k * 128;
          *reinterpret_cast<uint4*>(row + ((j0 ^ (k & 7)) << 4)) = lo;
          *reinterpret_cast<uint4*>(row + (((j0 + 1) ^ (k & 7)) << 4)) = hi;
        }
        fence_proxy_async_smem();  // V16 is read by the tensor core (async proxy)
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(kVFull + vb));
          mbar_arrive(bar(kKvEmpty + st));
        }
      }
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax + O rescale
    const int q4 = warp & 3;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const int row = 32 * q4 + lane;  // tile row of this thread
    uint32_t it = 0, chunk = 0;
    int cur = br;
    Chunk ch;
    while (next_chunk(p, br, bk, er, ek, bs, cur, ch)) {
      const int nb = ch.hi - ch.lo;
      const int par = chunk & 1;
      int limit = 0;
      if (row < Rt) {
        limit = p.causal ? ch.L - (p.s_q - 1 - (r0 + row) / p.h_q) : ch.L;
        limit = limit < 0 ? 0 : limit;
      }
      float m = -INFINITY, l = 0.f;
      for (int jj = 0; jj < nb; ++jj) {
        const uint32_t itc = it + jj;
        const int b = itc & 1;
        mbar_wait(bar(kSFull + b), (itc >> 1) & 1, wctl, err, kDevErrTimeout);
        __syncwarp();
        tc_fence_after();
        float x[64];
        {
          uint32_t v0[32], v1[32];
          tmem_ld32(t_lane + Lay::kColS + kPage * b, v0);
          tmem_ld32(t_lane + Lay::kColS + kPage * b + 32, v1);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            x[c] = __uint_as_float(v0[c]);
            x[32 + c] = __uint_as_float(v1[c]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kSEmpty + b));

        const int kbase = (ch.lo + jj) * kPage;
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float t = (kbase + c < limit) ? x[c] * p.scale_log2 : -INFINITY;
          x[c] = t;
          mx = fmaxf(mx, t);
        }
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
        uint32_t pk[32];
#pragma unroll
        for (int c2 = 0; c2 < 32; ++c2) {
          const float p0 = ex2(x[2 * c2] - base);
          const float p1 = ex2(x[2 * c2 + 1] - base);
          sum += p0 + p1;
          pk[c2] = pack_half2(p0, p1);
        }
        l = l * alpha + sum;
        const bool any_resc = __any_sync(0xffffffffu, resc);
        mbar_wait(bar(kPEmpty + b), ((itc >> 1) & 1) ^ 1, wctl, err, kDevErrTimeout);
        {
          // P row: 64 keys = 128 bytes, 16-byte pieces XOR-swizzled by row (128-byte swizzle)
          uint8_t* prow = smem + Lay::kOffP + b * kPBytes + row * 128;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            *reinterpret_cast<uint4*>(prow + ((k ^ (row & 7)) << 4)) =
                make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
        }
        fence_proxy_async_smem();  // P is read by the tensor core (async proxy)
        if (any_resc) {
          // this warp's rows of O (lane quadrant q4, all 256 columns): wait for the previous P.V
          mbar_wait(bar(kODone), (itc - 1) & 1, wctl, err, kDevErrTimeout);
          __syncwarp();
          tc_fence_after();
#pragma unroll 1
          for (int c32 = 0; c32 < 8; ++c32) {
            uint32_t o[32];
            const uint32_t col = Lay::kColO + 32 * c32;
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
        if (lane == 0) mbar_arrive(bar(kPFull + b));
      }
      // this stats slot was last read by the epilogue of chunk - 2, which finished before the
      // first P.V of chunk - 1 (that P.V waits for it), so before this chunk's pages
      s_lsum[par * kTile + row] = l;
      s_mref[par * kTile + row] = m;
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kStats + par));
      it += nb;
      ++chunk;
    }
  } else {
    // ------------------------------------------------------------ Q loads and epilogue (warps 8-11)
    const int q4 = warp & 3;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const int row = 32 * q4 + lane;  // tile row of this thread
    auto load_q = [&](const Chunk& c, uint32_t idx) {
      // this quadrant's Q rows of chunk idx, cast to e5m2 (Q is single-buffered: wait for the
      // previous chunk's last Q.K^T)
      mbar_wait(bar(kQEmpty), (idx & 1) ^ 1, wctl, err, kDevErrTimeout);
      __syncwarp();
      tc_fence_after();
      const uint4* qrow = reinterpret_cast<const uint4*>(
          reinterpret_cast<const uint16_t*>(qptr) + (static_cast<int64_t>(c.req) * R + r0 + (row < Rt ? row : 0)) * kDK);
#pragma unroll 1
      for (int c16 = 0; c16 < kDV / 64; ++c16) {  // values 0..511: 128 TMEM columns
        uint32_t w[16];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          uint4 d = make_uint4(0, 0, 0, 0);
          if (row < Rt) d = __ldg(qrow + c16 * 8 + v);
          w[2 * v] = cast4_e5m2<kBF16>(d.x, d.y);
          w[2 * v + 1] = cast4_e5m2<kBF16>(d.z, d.w);
        }
        tmem_st16(t_lane + Lay::kColQ + 16 * c16, w);
      }
      // values 512..575: one 64-byte row of the shared-memory tile, its four 16-byte pieces
      // XOR-swizzled by (row / 2) & 3 (64-byte swizzle)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint4 d0 = make_uint4(0, 0, 0, 0), d1 = make_uint4(0, 0, 0, 0);
        if (row < Rt) {
          d0 = __ldg(qrow + 64 + 2 * j);
          d1 = __ldg(qrow + 64 + 2 * j + 1);
        }
        const uint4 e = make_uint4(cast4_e5m2<kBF16>(d0.x, d0.y), cast4_e5m2<kBF16>(d0.z, d0.w),
                                   cast4_e5m2<kBF16>(d1.x, d1.y), cast4_e5m2<kBF16>(d1.z, d1.w));
        *reinterpret_cast<uint4*>(smem + Lay::kOffQR + row * 64 + ((j ^ ((row >> 1) & 3)) << 4)) = e;
      }
      fence_proxy_async_smem();  // the tile is read by the tensor core (async proxy)
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && !(p.withhold_q_ready && idx == 0)) mbar_arrive(bar(kQFull));
    };
    auto epilogue = [&](const Chunk& c, uint32_t idx) {
      const int par = idx & 1;
      mbar_wait(bar(kOFinal), idx & 1, wctl, err, kDevErrTimeout);
      mbar_wait(bar(kStats + par), (idx >> 1) & 1, wctl, err, kDevErrTimeout);
      __syncwarp();
      tc_fence_after();
      const bool whole = (c.lo == 0 && c.hi == c.n);
      const int64_t chunk0 = whole ? 0 : static_cast<int64_t>(p.num_splits[c.req] + c.split) * R;
      const float lr = s_lsum[par * kTile + row];
      const float inv = lr > 0.f ? 1.f / lr : 0.f;
      const int64_t rg = r0 + row;  // query row within the request
#pragma unroll 1
      for (int c32 = 0; c32 < 8; ++c32) {
        uint32_t o[32];
        tmem_ld32(t_lane + Lay::kColO + 32 * c32, o);
        tmem_wait_ld();
        if (row < Rt) {
          const int d = 256 * vh + 32 * c32;  // values d .. d + 31
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
      if (vh == 0 && row < Rt) {  // both CTAs of the tile hold the same row sums and maxima
        const float lse_v = lr > 0.f ? (s_mref[par * kTile + row] + log2f(lr)) * 0.69314718055994531f : -INFINITY;
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
    if (have) load_q(ch, 0);
    uint32_t chunk = 0;
    while (have) {
      const bool more = next_chunk(p, br, bk, er, ek, bs, cur, nx);
      if (more) load_q(nx, chunk + 1);  // after this chunk's last Q.K^T: overlaps its tail
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

}  // namespace fp8rt

int fp8_rt_smem_bytes() { return fp8rt::Layout::kSmemBytes; }

const void* fp8_rt_kernel_ptr(bool bf16) {
  return bf16 ? reinterpret_cast<const void*>(&fp8rt::splitkv_fp8_rt_kernel<true>)
              : reinterpret_cast<const void*>(&fp8rt::splitkv_fp8_rt_kernel<false>);
}

int fp8_rt_tiles(int rows) { return (rows + fp8rt::kTile - 1) / fp8rt::kTile; }

cudaError_t launch_splitkv_fp8_rt(bool bf16, const void* q, const CUtensorMap& kmap, const CUtensorMap& krmap,
                                  const DecodeParams& p, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.num_parts * fp8_rt_tiles(p.rows) * 2);
  cfg.blockDim = dim3(fp8rt::kThreads);
  cfg.dynamicSmemBytes = fp8_rt_smem_bytes();
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (bf16) return cudaLaunchKernelEx(&cfg, fp8rt::splitkv_fp8_rt_kernel<true>, q, kmap, krmap, p);
  return cudaLaunchKernelEx(&cfg, fp8rt::splitkv_fp8_rt_kernel<false>, q, kmap, krmap, p);
}

}  // namespace mla
