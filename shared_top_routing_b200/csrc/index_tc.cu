// Prefill indexer scoring on the 5th-generation tensor cores (sm_100a).
//
// [LC] "长上下文：稀疏注意力 / DSA / IndexShare", section "DSA 与 IndexShare":
// the indexer scores every (query, history token) pair; with causal masking
// the pairs of query t are the tokens j <= q_pos0 + t.  Here the score tile
// S = Q_idx K_idx^T of 128 queries x 256 keys is one tcgen05.mma sequence
// (M=128, N=256, K=16 per instruction; bf16 in, fp32 accumulate in TMEM).
//
// One CTA owns a block of 128 query rows of one sequence and walks a share
// of its causal key tiles.  Warp roles:
//   warp 0      TMA producer: the query block once, then key tiles into a
//               STAGES-deep shared-memory ring (128-byte swizzle, no
//               multicast), completion tracked by mbarriers;
//   warp 1      allocates 512 TMEM columns (two 128x256 fp32 accumulators)
//               and one thread issues the MMAs and tcgen05.commit;
//   warps 2..   epilogue: TMEM lane (= query row) i is read by thread i % 32
//               of the warps with warp % 4 == i / 32, with tcgen05.ld.
// The MMA of tile i+1 overlaps the epilogue of tile i (double-buffered
// accumulator).  Every mbarrier wait is bounded; on a timeout the CTA records
// an error code, stops issuing work and frees its TMEM.
//
// Epilogues (one kernel instance each):
//   kEpiKeys      4 warps; every score's order-preserving key into the row's
//                 slab (rows short enough for one CTA to select from).
//   kEpiGroupMax  8 warps (two per lane quarter, 128 columns each); per row,
//                 the maximum of each group of g consecutive scores as a
//                 16-bit truncated key (the top half of the 32-bit key,
//                 which never exceeds the group's largest key).
//   kEpiCand      as kEpiGroupMax; per row, every score at or above the
//                 row's bound (from the group maxima) is kept as a (score
//                 bits, position) pair.  A CTA's tiles of one row block form
//                 a run; its takes of a row are appended at the run's first
//                 column of the row's pair array (a shared per-row counter
//                 hands out the places, one 8-byte store per take), and the
//                 run's count goes to the run's first tile slot.  A 32-bit mask per 32 columns finds
//                 the takes (the sign of bound' - score, bound' the float
//                 just below the bound, so one add decides "not below"); a
//                 chunk with any is stashed in shared memory so the takes
//                 can be picked by index.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>

#include "sa_common.cuh"
#include "sa_internal.h"
#include "tc_common.cuh"

namespace sa {
namespace {

using namespace tc;

constexpr int kBM = 128;   // query rows per block (TMEM lanes)
constexpr int kBN = 256;   // key columns per MMA tile
constexpr int kTmemCols = 512;
// pipeline waits poll at most this many times, each poll sleeping up to kWaitNs
constexpr uint32_t kWaitPolls = 1u << 20, kWaitNs = 2000;

constexpr int kEpiKeys = 0, kEpiGroupMax = 1, kEpiCand = 2;
constexpr int kStashFloats = 36;   // per thread: one 32-column chunk (rows padded to 36 floats)

template <int D, int EPI>
struct TcShape {
  static constexpr int kAtoms = D / 64;             // 128-byte swizzle atoms along K
  static constexpr int kABytes = kBM * D * 2;
  static constexpr int kBBytes = kBN * D * 2;
  static constexpr int kStages = D == 64 ? 4 : 2;
  // epilogue warps: four per TMEM lane quarter for d = 64 (64 columns of a
  // tile each), two for d = 128 (shared memory), one for the key slab
  static constexpr int kEpiWarps = EPI == kEpiKeys ? 4 : (D == 64 ? 16 : 8);
  static constexpr int kParts = kEpiWarps / 4;
  static constexpr int kPartCols = kBN / kParts;
  static constexpr int kThreads = 64 + 32 * kEpiWarps;
  static constexpr int kBarBytes = 256;
  static constexpr int kStashBytes = EPI == kEpiCand ? kEpiWarps * 32 * kStashFloats * 4 : 0;
  static constexpr int kCntBytes = EPI == kEpiCand ? 4 * kBM * 4 : 0;   // per row: takes, parts done; two runs
  // query-block buffers: with two the next block loads while the last one's
  // MMAs run (the candidate pass needs the room for its stash)
  static constexpr int kABuf = EPI == kEpiCand ? 1 : 2;
  static constexpr int kSmem = 1024 + kABuf * kABytes + kStages * kBBytes + kBarBytes + kCntBytes + kStashBytes;
};
static_assert(TcShape<128, kEpiCand>::kSmem <= 227 * 1024, "shared memory");
static_assert(TcShape<64, kEpiCand>::kSmem <= 227 * 1024, "shared memory");
static_assert(kGroupMax <= TcShape<64, kEpiGroupMax>::kPartCols, "a group must lie in one thread's columns");

struct TcBars {
  uint64_t full[4];
  uint64_t empty[4];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t afull[2], aempty[2];
  uint32_t tmem_base;
  int abort;
};

struct TcParams {
  int Tq, Tk, q_pos0, k;
  const int32_t* kv_len;
  int t0, rows, nblk, B;
  long long tiles_per_seq;   // key tiles of all row blocks of one sequence
  uint32_t* keys;          // kEpiKeys: [rows][ld] slab; kEpiCand: [rows][ld] (score bits, position) pairs
  long long ld;
  uint32_t* tile_cnt;      // kEpiCand: [rows][ld / kBN] takes of the run starting at each tile
  const uint32_t* theta;   // kEpiCand: [rows] 16-bit bound of each row
  uint16_t* gmax;          // kEpiGroupMax: [rows][ld2] group maxima
  long long ld2;
  int* err;
};

// Maximum of three (a NaN operand is ignored, as by fmaxf).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Maximum of N consecutive values, as a chain of three-input maxima
// (ceil((N - 1) / 2) instructions).
template <int N>
__device__ __forceinline__ float chain_max(const float* x) {
  if constexpr (N == 1) {
    return x[0];
  } else {
    float a = N == 2 ? fmaxf(x[0], x[1]) : fmax3(x[0], x[1], x[2]);
    int i = N == 2 ? 2 : 3;
#pragma unroll
    for (; i + 1 < N; i += 2) a = fmax3(a, x[i], x[i + 1]);
    if (i < N) a = fmaxf(a, x[i]);
    return a;
  }
}

// Order-preserving key for the group-maximum bound.  Unlike score_key it
// leaves -0 one below +0: that can only lower a maximum's key, and a lower
// bound stays a bound.
__device__ __forceinline__ uint32_t bound_key(float s) {
  const uint32_t b = __float_as_uint(s);
  return b ^ ((uint32_t)((int32_t)b >> 31) | 0x80000000u);
}

// The 16-bit bound keys of a (low half) and b (high half).
__device__ __forceinline__ uint32_t pack_key16(float a, float b) {
  return __byte_perm(bound_key(a), bound_key(b), 0x7632);
}

__device__ __forceinline__ int tc_row_len(const int32_t* kv_len, int b, int Tk) {
  if (kv_len == nullptr) return Tk;
  int v = kv_len[b];
  return v < 0 ? 0 : (v > Tk ? Tk : v);
}

__device__ __forceinline__ int tc_n_cand(long long q_pos0, int t, int len) {
  long long n = q_pos0 + (long long)t + 1;
  if (n > len) n = len;
  if (n < 0) n = 0;
  return (int)n;
}

// Causal key tiles of row block rb (any sequence: bounded by Tk, a shorter
// cache only masks more of them).
__device__ __forceinline__ int block_tiles(const TcParams& p, int rb) {
  const int t_last = min(p.t0 + min((rb + 1) * kBM, p.rows), p.Tq) - 1;
  long long nc = (long long)p.q_pos0 + t_last + 1;
  if (nc > p.Tk) nc = p.Tk;
  return nc > 0 ? (int)((nc + kBN - 1) / kBN) : 0;
}

// Position in the flat list of (sequence, row block, key tile) work items.
struct TileCursor {
  int b, rb, tile, nt;
  __device__ __forceinline__ void start(const TcParams& p, long long u) {
    b = (int)(u / p.tiles_per_seq);
    long long rem = u % p.tiles_per_seq;
    rb = 0;
    nt = block_tiles(p, 0);
    while (rem >= nt && rb + 1 < p.nblk) {
      rem -= nt;
      ++rb;
      nt = block_tiles(p, rb);
    }
    tile = (int)rem;
  }
  __device__ __forceinline__ void next(const TcParams& p) {
    if (++tile < nt) return;
    tile = 0;
    if (++rb == p.nblk) {
      rb = 0;
      ++b;
    }
    nt = block_tiles(p, rb);
  }
};

// Persistent CTAs (one per SM) each take an equal contiguous share of the
// flat list of (sequence, 128-query row block, causal 256-key tile) items;
// the query block is reloaded whenever the share moves to the next block.
template <int D, int EPI>
__global__ void __launch_bounds__(TcShape<D, EPI>::kThreads, 1)
score_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmap_q,
                        const __grid_constant__ CUtensorMap tmap_k, TcParams p) {
  using S = TcShape<D, EPI>;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  unsigned char* base = smem_raw + ((1024 - (raw & 1023)) & 1023);  // 1024-byte aligned
  unsigned char* sA = base;                       // kABuf query blocks
  unsigned char* sB = base + S::kABuf * S::kABytes;
  TcBars& bars = *reinterpret_cast<TcBars*>(base + S::kABuf * S::kABytes + S::kStages * S::kBBytes);
  // candidate pass: [2][kBM] take counters, [2][kBM] finished-part counters (runs alternate)
  uint32_t* s_cnt = reinterpret_cast<uint32_t*>(base + S::kABuf * S::kABytes + S::kStages * S::kBBytes + S::kBarBytes);
  uint32_t* s_done = s_cnt + 2 * kBM;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long total = p.tiles_per_seq * p.B;
  const long long lo = (long long)blockIdx.x * total / gridDim.x;
  const long long hi = (long long)(blockIdx.x + 1) * total / gridDim.x;
  if (hi <= lo) return;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::kStages; ++s) { mbar_init(&bars.full[s], 1); mbar_init(&bars.empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&bars.tfull[a], 1); mbar_init(&bars.tempty[a], S::kEpiWarps); }
    for (int a = 0; a < 2; ++a) { mbar_init(&bars.afull[a], 1); mbar_init(&bars.aempty[a], 1); }
    bars.abort = 0;
    fence_barrier_init();
  }
  if constexpr (EPI == kEpiCand)
    for (int i = threadIdx.x; i < 4 * kBM; i += blockDim.x) s_cnt[i] = 0u;
  if (warp == 1) {
    tmem_alloc(&bars.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars.tmem_base;
  volatile int* abort_flag = &bars.abort;

  if (warp == 0) {
    if (lane == 0) {
      // producer: the query block at every block change, key tiles into the ring
      TileCursor cur;
      cur.start(p, lo);
      int blk = -1;
      int nA = 0, nB = 0;   // query blocks and key tiles whose loads were issued
      for (long long u = lo; u < hi; ++u, cur.next(p)) {
        if (u == lo || cur.tile == 0) {
          // block blk goes to buffer blk % kABuf, once the MMAs of block blk - kABuf are done
          ++blk;
          const int ab = blk % S::kABuf;
          if (blk >= S::kABuf &&
              !mbar_wait(&bars.aempty[ab], (uint32_t)((blk - S::kABuf) / S::kABuf) & 1u, abort_flag, p.err, 6, kWaitPolls, kWaitNs))
            break;
          mbar_arrive_expect_tx(&bars.afull[ab], S::kABytes);
#pragma unroll
          for (int a = 0; a < S::kAtoms; ++a)
            tma_load_3d(sA + ab * S::kABytes + a * kBM * 128, &tmap_q, &bars.afull[ab], 64 * a,
                        p.t0 + cur.rb * kBM, cur.b);
          nA = blk + 1;
        }
        const int i = (int)(u - lo);
        const int s = i % S::kStages;
        const uint32_t ph = (uint32_t)(i / S::kStages) & 1u;
        if (!mbar_wait(&bars.empty[s], ph ^ 1u, abort_flag, p.err, 1, kWaitPolls, kWaitNs)) break;
        mbar_arrive_expect_tx(&bars.full[s], S::kBBytes);
#pragma unroll
        for (int a = 0; a < S::kAtoms; ++a)
          tma_load_3d(sB + s * S::kBBytes + a * kBN * 128, &tmap_k, &bars.full[s], 64 * a, cur.tile * kBN, cur.b);
        nB = i + 1;
      }
      // every load this CTA issued lands before it exits (also after a wait
      // gave up): bounded waits on the last phase of each buffer
      for (int s = 0; s < S::kStages; ++s)
        if (s < nB && !mbar_wait_drain(&bars.full[s], (uint32_t)((nB - 1 - s) / S::kStages) & 1u) && p.err)
          atomicCAS(p.err, 0, 7);
      for (int a = 0; a < S::kABuf; ++a)
        if (a < nA && !mbar_wait_drain(&bars.afull[a], (uint32_t)((nA - 1 - a) / S::kABuf) & 1u) && p.err)
          atomicCAS(p.err, 0, 7);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // MMA issuer
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN);
      TileCursor cur;
      cur.start(p, lo);
      int blk = -1;
      int last = -1;   // the last tile whose MMAs were committed
      uint32_t a_addr = 0;
      for (long long u = lo; u < hi; ++u, cur.next(p)) {
        if (u == lo || cur.tile == 0) {
          ++blk;
          if (!mbar_wait(&bars.afull[blk % S::kABuf], (uint32_t)(blk / S::kABuf) & 1u, abort_flag, p.err, 2, kWaitPolls, kWaitNs)) break;
          a_addr = smem_u32(sA + (blk % S::kABuf) * S::kABytes);
        }
        const int i = (int)(u - lo);
        const int s = i % S::kStages;
        const uint32_t ph = (uint32_t)(i / S::kStages) & 1u;
        const int acc = i & 1;
        const uint32_t aph = (uint32_t)(i >> 1) & 1u;
        if (!mbar_wait(&bars.tempty[acc], aph ^ 1u, abort_flag, p.err, 3, kWaitPolls, kWaitNs)) break;
        if (!mbar_wait(&bars.full[s], ph, abort_flag, p.err, 4, kWaitPolls, kWaitNs)) break;
        tc_fence_after();
        const uint32_t b_addr = smem_u32(sB + s * S::kBBytes);
        const uint32_t d_tmem = tbase + (uint32_t)(acc * kBN);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (uint32_t)((kk & 3) * 32);  // 16 bf16 = 32 B within the atom
          const uint64_t adesc = sdesc_k_sw128(a_addr + (kk >> 2) * kBM * 128 + koff);
          const uint64_t bdesc = sdesc_k_sw128(b_addr + (kk >> 2) * kBN * 128 + koff);
          umma_bf16(d_tmem, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars.empty[s]);
        umma_commit(&bars.tfull[acc]);
        if (cur.tile == cur.nt - 1 || u == hi - 1) umma_commit(&bars.aempty[blk % S::kABuf]);   // its query block is free
        last = i;
      }
      // every MMA issued completes before the accumulator is freed (a commit
      // covers all earlier MMAs of this thread)
      if (last >= 0 && !mbar_wait_drain(&bars.tfull[last & 1], (uint32_t)(last >> 1) & 1u) && p.err)
        atomicCAS(p.err, 0, 8);
    }
  } else {
    // epilogue: warp w reads TMEM lanes of quarter w % 4, columns part *
    // kPartCols .. +kPartCols of each tile (part = (w - 2) / 4)
    const int quarter = warp & 3;
    const int part = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;
    const uint32_t tlane = (uint32_t)(quarter * 32) << 16;
    TileCursor cur;
    cur.start(p, lo);
    int n = 0, nw = 0, g = 0, run_tile = 0, run_idx = -1;
    bool row_ok = false;
    long long rloc = 0;
    float xth = 0.f;
    for (long long u = lo; u < hi; ++u, cur.next(p)) {
      if (u == lo || cur.tile == 0) {   // a new row block: this thread's row
        const int tq = p.t0 + cur.rb * kBM + r;
        row_ok = tq < p.t0 + p.rows && tq < p.Tq;
        n = row_ok ? tc_n_cand(p.q_pos0, tq, tc_row_len(p.kv_len, cur.b, p.Tk)) : 0;
        // tcgen05.ld is warp-wide: chunks are visited up to the warp's longest row
        nw = (int)__reduce_max_sync(0xffffffffu, (uint32_t)n);
        rloc = (long long)cur.b * p.rows + (tq - p.t0);
        g = prefill_group_size(n, p.k);
        run_tile = cur.tile;   // the candidate run of this block starts at this tile
        ++run_idx;
        // xth: the float just below the bound, so a score s is kept when
        // xth - s < 0 (sign bit set); bound 0 (rows of at most k candidates)
        // keeps every finite score
        if constexpr (EPI == kEpiCand) {
          const uint32_t th = n > 0 ? p.theta[rloc] : 0u;
          xth = th == 0u ? -INFINITY : nextafterf(key_score(th << 16), -INFINITY);
        }
      }
      const int i = (int)(u - lo);
      const int acc = i & 1;
      const uint32_t aph = (uint32_t)(i >> 1) & 1u;
      if (!mbar_wait(&bars.tfull[acc], aph, abort_flag, p.err, 5, kWaitPolls, kWaitNs)) break;
      tc_fence_after();
      const int cb = cur.tile * kBN + part * S::kPartCols;   // first column of this thread's part
      const uint32_t tcol = tbase + tlane + (uint32_t)(acc * kBN + part * S::kPartCols);
      if constexpr (EPI == kEpiKeys) {
        uint32_t* krow = p.keys + rloc * p.ld;
#pragma unroll 1
        for (int ch = 0; ch < S::kPartCols / 32; ++ch) {
          const int c = cb + ch * 32;
          if (c >= nw) break;
          uint32_t v[32];
          tmem_ld32(tcol + (uint32_t)(ch * 32), v);
          tmem_ld_wait();
          if (c < n) {
            uint4* dst = reinterpret_cast<uint4*>(krow + c);
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              dst[q4] = make_uint4(score_key(__uint_as_float(v[4 * q4 + 0])), score_key(__uint_as_float(v[4 * q4 + 1])),
                                   score_key(__uint_as_float(v[4 * q4 + 2])), score_key(__uint_as_float(v[4 * q4 + 3])));
          }
        }
      } else if constexpr (EPI == kEpiGroupMax) {
        // 64 columns per load pair: one wait, then a max tree whose level
        // log2(g) holds this row's group maxima
        uint16_t* gm = p.gmax + rloc * p.ld2;
#pragma unroll 1
        for (int cc = 0; cc < S::kPartCols; cc += 64) {
          const int c = cb + cc;
          if (c >= nw) break;
          uint32_t v[64];
          tmem_ld32(tcol + (uint32_t)cc, v);
          tmem_ld32(tcol + (uint32_t)(cc + 32), v + 32);
          tmem_ld_wait();
          if (g == 0 || c >= n) continue;
          float x[64];
#pragma unroll
          for (int j = 0; j < 64; ++j) x[j] = __uint_as_float(v[j]);
          if (c + 64 > n) {
#pragma unroll
            for (int j = 0; j < 64; ++j) x[j] = c + j < n ? x[j] : -INFINITY;
          }
          if (g == 1) {
            uint4* dst = reinterpret_cast<uint4*>(gm + c);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              dst[q] = make_uint4(pack_key16(x[8 * q + 0], x[8 * q + 1]), pack_key16(x[8 * q + 2], x[8 * q + 3]),
                                  pack_key16(x[8 * q + 4], x[8 * q + 5]), pack_key16(x[8 * q + 6], x[8 * q + 7]));
            continue;
          }
          if (g == 2) {
            float y[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) y[j] = fmaxf(x[2 * j], x[2 * j + 1]);
            uint4* dst = reinterpret_cast<uint4*>(gm + c / 2);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst[q] = make_uint4(pack_key16(y[8 * q + 0], y[8 * q + 1]), pack_key16(y[8 * q + 2], y[8 * q + 3]),
                                  pack_key16(y[8 * q + 4], y[8 * q + 5]), pack_key16(y[8 * q + 6], y[8 * q + 7]));
          } else if (g == 4) {
            float y[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) y[j] = chain_max<4>(x + 4 * j);
            uint4* dst = reinterpret_cast<uint4*>(gm + c / 4);
#pragma unroll
            for (int q = 0; q < 2; ++q)
              dst[q] = make_uint4(pack_key16(y[8 * q + 0], y[8 * q + 1]), pack_key16(y[8 * q + 2], y[8 * q + 3]),
                                  pack_key16(y[8 * q + 4], y[8 * q + 5]), pack_key16(y[8 * q + 6], y[8 * q + 7]));
          } else if (g == 8) {
            float y[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) y[j] = chain_max<8>(x + 8 * j);
            *reinterpret_cast<uint4*>(gm + c / 8) =
                make_uint4(pack_key16(y[0], y[1]), pack_key16(y[2], y[3]), pack_key16(y[4], y[5]), pack_key16(y[6], y[7]));
          } else {
            float y[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) y[j] = chain_max<16>(x + 16 * j);
            if (g == 16) {
              *reinterpret_cast<uint2*>(gm + c / 16) = make_uint2(pack_key16(y[0], y[1]), pack_key16(y[2], y[3]));
            } else if (g == 32) {
              *reinterpret_cast<uint32_t*>(gm + c / 32) = pack_key16(fmaxf(y[0], y[1]), fmaxf(y[2], y[3]));
            } else {   // 64
              gm[c / 64] = (uint16_t)(bound_key(fmax3(y[0], y[1], fmaxf(y[2], y[3]))) >> 16);
            }
          }
        }
      } else {
        uint2* run = reinterpret_cast<uint2*>(p.keys) + rloc * p.ld + (long long)run_tile * kBN;
        uint32_t* cnt = s_cnt + (run_idx & 1) * kBM + r;
        float* stash = reinterpret_cast<float*>(base + S::kABuf * S::kABytes + S::kStages * S::kBBytes +
                                                S::kBarBytes + S::kCntBytes) +
                       ((warp - 2) * 32 + lane) * kStashFloats;
#pragma unroll 1
        for (int cc = 0; cc < S::kPartCols; cc += 64) {
          const int c0 = cb + cc;
          if (c0 >= nw) break;
          uint32_t v[64];
          tmem_ld32(tcol + (uint32_t)cc, v);
          tmem_ld32(tcol + (uint32_t)(cc + 32), v + 32);
          tmem_ld_wait();
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int c = c0 + 32 * h;
            // bit (31 - j) of m marks column c + j as a take: the sign bit of
            // xth - score (four independent 8-column chains, joined)
            uint32_t mq[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int j = 0; j < 8; ++j)
#pragma unroll
              for (int q = 0; q < 4; ++q)
                mq[q] = __funnelshift_l(__float_as_uint(xth - __uint_as_float(v[32 * h + 8 * q + j])), mq[q], 1);
            uint32_t m = mq[0] << 24 | mq[1] << 16 | mq[2] << 8 | mq[3];
            const int valid = n - c;
            m = valid >= 32 ? m : (valid > 0 ? m & (~0u << (32 - valid)) : 0u);
            if (m) {
#pragma unroll
              for (int q4 = 0; q4 < 8; ++q4)
                *reinterpret_cast<uint4*>(stash + 4 * q4) =
                    make_uint4(v[32 * h + 4 * q4], v[32 * h + 4 * q4 + 1], v[32 * h + 4 * q4 + 2], v[32 * h + 4 * q4 + 3]);
              uint2* dst = run + atomicAdd(cnt, (uint32_t)__popc(m));
              while (m) {
                const int j = __clz(m);
                m &= ~(0x80000000u >> j);
                *dst++ = make_uint2(__float_as_uint(stash[j]), (uint32_t)(c + j));
              }
            }
          }
        }
      }
      if constexpr (EPI == kEpiCand) {
        // Tile slots of a run: the first holds the run's count, the others
        // 0.  The last part to finish the run writes the count (no CTA-wide
        // barrier: parts pass each other freely, and runs alternate counters
        // because a part can be one run ahead).  This happens before the
        // accumulator is released, so no part gets two runs ahead.
        const bool run_end = cur.tile == cur.nt - 1 || u == hi - 1;
        uint32_t* tcnt = p.tile_cnt + rloc * (p.ld / kBN);
        if (part == 0 && row_ok && cur.tile != run_tile) tcnt[cur.tile] = 0u;
        if (run_end) {
          const int sel = (run_idx & 1) * kBM + r;
          __threadfence_block();
          if (atomicAdd(s_done + sel, 1u) == (uint32_t)(S::kParts - 1)) {
            const uint32_t takes = atomicExch(s_cnt + sel, 0u);
            s_done[sel] = 0u;
            if (row_ok) tcnt[run_tile] = takes;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.tempty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, kTmemCols);
}

// ------------------------------------------------------------ tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// [batches][rows][d] bf16, box = 64 elements (128 B) x box_rows, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* ptr, int d, long long rows, int batches, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)batches};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)rows * d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

template <int D, int EPI>
static cudaError_t launch_tc(dim3 grid, const CUtensorMap& mq, const CUtensorMap& mk, const TcParams& p,
                             cudaStream_t st) {
  using S = TcShape<D, EPI>;
  auto kern = score_prefill_tc_kernel<D, EPI>;
  cudaError_t e = ensure_dynamic_smem((const void*)kern, S::kSmem);
  if (e != cudaSuccess) return e;
  kern<<<grid, S::kThreads, S::kSmem, st>>>(mq, mk, p);
  return cudaGetLastError();
}

cudaError_t launch_score_prefill(const uint16_t* q, const uint16_t* kmat, int B, int Tq, int d,
                                 int Tk_max, int Tk, int q_pos0, const int32_t* kv_len, int t0,
                                 int rows, int k, int epi, const RowWorkspace& w, cudaStream_t st) {
  if (rows <= 0 || Tk <= 0 || B <= 0) return cudaSuccess;
  CUtensorMap mq, mk;
  if (!make_map(&mq, q, d, Tq, B, kBM) || !make_map(&mk, kmat, d, Tk_max, B, kBN))
    return cudaErrorInvalidValue;
  TcParams p;
  p.Tq = Tq;
  p.Tk = Tk;
  p.q_pos0 = q_pos0;
  p.k = k;
  p.kv_len = kv_len;
  p.t0 = t0;
  p.rows = rows;
  p.nblk = (rows + kBM - 1) / kBM;
  p.B = B;
  p.keys = w.keys;
  p.ld = w.ld;
  p.tile_cnt = w.tile_cnt;
  p.theta = w.theta;
  p.gmax = w.gmax;
  p.ld2 = w.ld2;
  p.err = w.err;
  // causal key tiles of one sequence's row blocks (bounded by Tk)
  long long per_seq = 0;
  for (int rb = 0; rb < p.nblk; ++rb) {
    const int t_last = std::min(t0 + std::min((rb + 1) * kBM, rows), Tq) - 1;
    long long nc = (long long)q_pos0 + t_last + 1;
    if (nc > Tk) nc = Tk;
    per_seq += nc > 0 ? (nc + kBN - 1) / kBN : 0;
  }
  if (per_seq <= 0) return cudaSuccess;
  p.tiles_per_seq = per_seq;
  // one persistent CTA per SM (512 TMEM columns and most of shared memory each)
  const int sms = device_sm_count();
  const long long total = per_seq * B;
  dim3 grid((unsigned)(total < sms ? total : sms));
  if (d == 128) {
    if (epi == kScoreGroupMax) return launch_tc<128, kEpiGroupMax>(grid, mq, mk, p, st);
    if (epi == kScoreCand) return launch_tc<128, kEpiCand>(grid, mq, mk, p, st);
    return launch_tc<128, kEpiKeys>(grid, mq, mk, p, st);
  }
  if (epi == kScoreGroupMax) return launch_tc<64, kEpiGroupMax>(grid, mq, mk, p, st);
  if (epi == kScoreCand) return launch_tc<64, kEpiCand>(grid, mq, mk, p, st);
  return launch_tc<64, kEpiKeys>(grid, mq, mk, p, st);
}

}  // namespace sa
