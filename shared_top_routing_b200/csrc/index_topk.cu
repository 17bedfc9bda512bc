// Indexer scoring and exact per-query top-k (sm_100a).
//
// Method: [LC] "长上下文：稀疏注意力 / DSA / IndexShare", section "DSA 与
// IndexShare" -- a light indexer scores every history token and each query
// keeps its top-k; [YOIO] §2.3 -- the indexer outputs each query's top-k
// token indices.  Selection rule: largest scores, equal scores by lower
// position, emitted in ascending position order.
//
// Kernels
//   score_decode_kernel  one query per sequence.  The indexer-key cache is
//       streamed with 16-byte loads straight into mma.sync B fragments: a dot
//       product is invariant to the order of its terms, so lane (g, t) of a
//       warp loads whole 16-byte chunks 4j+t of key row g and the query
//       fragment is permuted to match.  One m16n8k16 per 16 dims scores 8
//       keys (the query is row 0 of the 16-row A side).  Each warp loads one
//       register buffer of key tiles and scores it; four CTAs per SM keep 32
//       warps of loads in flight.  Writes the order-preserving 32-bit score
//       key of every candidate and a 4096-bin histogram of the keys' top 12
//       bits.  The B x Tk key rows are flattened and split evenly (at
//       multiples of 8 rows) over a grid sized to the resident CTAs.  (Two
//       other designs measured no faster: TMA + tcgen05, where with 128x16
//       tiles the per-tile TMEM hand-off dominates, and a TMA bulk-copy ring
//       into shared memory feeding mma.sync warps.)
//   prefill_threshold_kernel  (long prefill rows) the k-th largest of the
//       row's 16-bit group maxima -- a counting pass over a window below
//       their maximum, or a two-digit radix select -- the bound the second
//       scoring pass keeps keys against.
//   finish_kernel        one CTA per row, one instance per candidate source
//       (the whole row of a short prefill or decode row, or the bounded
//       prefill pass's runs): gathers the row's candidates into shared
//       memory, runs an exact radix select (8-bit digits, warp-aggregated
//       shared histograms) of the k-th key, resolves ties at that key by
//       position (counting within a small tie group, radix passes
//       otherwise), then emits in ascending position order through a
//       position bitmap and popcount prefix sums (rows beyond the bitmap's
//       reach: counts per position range, ranked inside each range).  Also
//       expands chosen gist chunks into cache rows.
//   split_topk_kernel    one-query rows longer than a CTA's share: many CTAs
//       per row filter slices against the scorer histogram's threshold bin
//       and build a second-level histogram; the row's last CTA (ticket, no
//       waiting) finds the exact threshold and writes the chosen positions
//       in order with one packed block scan (see the section below).
#include <cuda_runtime.h>

#include <algorithm>
#include <type_traits>
#include <stddef.h>
#include <stdint.h>

#include "sa_common.cuh"
#include "sa_internal.h"
#include "tc_common.cuh"

namespace sa {
namespace {

constexpr int kScoreThreads = 256;
constexpr int kFinThreads = 1024;
constexpr int kSmemCand = 8192;          // candidates held in shared memory
constexpr int kBitmapMax = 1 << 18;      // rows up to this length emit through a bitmap
constexpr int kBitmapWords = kBitmapMax / 32;

__device__ __forceinline__ int row_len(const int32_t* kv_len, int b, int Tk) {
  if (kv_len == nullptr) return Tk;
  int v = kv_len[b];
  return v < 0 ? 0 : (v > Tk ? Tk : v);
}

// Number of candidates of query t: j <= q_pos0 + t and j < len.
__device__ __forceinline__ int n_cand(long long q_pos0, int t, int len) {
  long long n = q_pos0 + (long long)t + 1;
  if (n > len) n = len;
  if (n < 0) n = 0;
  return (int)n;
}

// ------------------------------------------------------------------ scoring

template <int D>
__global__ void __launch_bounds__(kScoreThreads, 4)
score_decode_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ kmat, int B, int Tk_max,
                    int Tk, int q_pos0, const int32_t* __restrict__ kv_len,
                    uint32_t* __restrict__ keys, long long ld, uint32_t* __restrict__ hist) {
  pdl_wait();
  pdl_launch_dependents();
  constexpr int J = D / 32;          // 16-byte chunks per lane per key row
  constexpr int U = 2;               // 8-row tiles per warp and load
  constexpr int WARPS = kScoreThreads / 32;
  __shared__ uint32_t sh[kHistBins];

  // The B x Tk row space (each batch padded to a multiple of 8 rows) is
  // flattened and split evenly over the grid at multiples of 8 rows, so every
  // CTA streams the same number of key rows and 8-row tiles stay aligned.
  const long long Tp = ((long long)Tk + 7) & ~7ll;
  const long long F = (long long)B * Tp;
  const long long lo = (F * blockIdx.x / gridDim.x) & ~7ll;
  const long long hi = blockIdx.x + 1 == gridDim.x ? F : ((F * (blockIdx.x + 1) / gridDim.x) & ~7ll);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tg = lane & 3;

  for (int b = (int)(lo / Tp); b < B && (long long)b * Tp < hi; ++b) {
    const long long base_f = (long long)b * Tp;
    const int n = n_cand(q_pos0, 0, row_len(kv_len, b, Tk));
    const int r0 = (int)((lo > base_f ? lo : base_f) - base_f);
    const int r1 = (int)min((long long)n, (hi < base_f + Tp ? hi : base_f + Tp) - base_f);
    if (r0 >= r1) continue;
    if (hist != nullptr) {
      for (int i = tid; i < kHistBins; i += kScoreThreads) sh[i] = 0;
      __syncthreads();
    }
    // A fragments: the query is row 0 of the 16-row A side, so only lanes
    // with g == 0 hold data.  Chunk 4j+t (dims 8(4j+t) .. +7) feeds two
    // k-steps: words x, y as (a0, a2) of one and z, w as (a0, a2) of the next.
    uint32_t qe[J][2], qo[J][2];
#pragma unroll
    for (int j = 0; j < J; ++j) {
      uint4 v = make_uint4(0, 0, 0, 0);
      if (g == 0) v = *reinterpret_cast<const uint4*>(q + (long long)b * D + (4 * j + tg) * 8);
      qe[j][0] = v.x; qe[j][1] = v.y;
      qo[j][0] = v.z; qo[j][1] = v.w;
    }
    const uint4* kb = reinterpret_cast<const uint4*>(kmat + (long long)b * Tk_max * D);
    uint32_t* kout = keys + (long long)b * ld;
    // One register buffer of U 8-row tiles per warp, loaded then scored: at
    // 64 registers four CTAs (32 warps) fit on an SM, and it is that many
    // warps with loads in flight, not a second buffer per warp, that keeps
    // HBM streaming (with two buffers, two CTAs fit and the read rate drops
    // by a third).
    auto load = [&](uint4 (&v)[U][J], int base) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int row = base + u * 8 + g;
#pragma unroll
        for (int j = 0; j < J; ++j)
          v[u][j] = row < r1 ? __ldg(kb + (long long)row * (D / 8) + 4 * j + tg) : make_uint4(0, 0, 0, 0);
      }
    };
    auto score = [&](const uint4 (&v)[U][J], int base) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < J; ++j) {
          const uint32_t a_even[4] = {qe[j][0], 0u, qe[j][1], 0u};
          const uint32_t a_odd[4] = {qo[j][0], 0u, qo[j][1], 0u};
          mma_bf16_16816(c, a_even, v[u][j].x, v[u][j].y);
          mma_bf16_16816(c, a_odd, v[u][j].z, v[u][j].w);
        }
        // row 0 of C: lanes 0..3 hold the scores of tile rows 2t and 2t+1
        if (g == 0) {
          const int row = base + u * 8 + 2 * tg;
          const uint32_t k0 = score_key(c[0]), k1 = score_key(c[1]);
          if (row < r1) kout[row] = k0;
          if (row + 1 < r1) kout[row + 1] = k1;
          if (hist != nullptr) {
            if (row < r1) atomicAdd(&sh[k0 >> (32 - kHistBits)], 1u);
            if (row + 1 < r1) atomicAdd(&sh[k1 >> (32 - kHistBits)], 1u);
          }
        }
      }
    };
    constexpr int kStep = WARPS * 8 * U;
    for (int base = r0 + warp * 8 * U; base < r1; base += kStep) {
      uint4 va[U][J];
      load(va, base);
      score(va, base);
    }
    if (hist != nullptr) {
      __syncthreads();
      uint32_t* hg = hist + (long long)b * kHistStride;
      for (int i = tid; i < kHistBins; i += kScoreThreads) {
        const uint32_t cnt = sh[i];
        if (cnt) atomicAdd(hg + i, cnt);
      }
      __syncthreads();
    }
  }
}

// -------------------------------------------------------- multi-head scoring
//
// score_mh_kernel: the multi-head weighted indexer, s = sum_h w_h *
// ReLU(q_h . k), for rows that each carry their own H query vectors and
// weights (one row per decode sequence, or per prefill query) against the
// key cache of their sequence.  The key cache is streamed as in
// score_decode_kernel (16-byte loads straight into mma.sync B fragments;
// here two register buffers of 8-row tiles per warp); the 16-row A side
// holds 16 indexer heads (rows g and g+8 of a lane's fragment are heads
// 16 hg + g and 16 hg + g + 8 of head group hg), so one m16n8k16 per 16
// dimensions scores every head of a group at once.  The epilogue takes
// weight x ReLU per head and sums over heads with three shuffles;
// integer-valued inputs keep every partial sum an exact fp32 integer.
// Grid: (key chunks, rows); each CTA scores one chunk of one row, writes the
// keys and adds its 4096-bin histogram of their top 12 bits to the row's.

template <int D, int HG>
__global__ void __launch_bounds__(kScoreThreads)
score_mh_kernel(const uint16_t* __restrict__ q, const float* __restrict__ wts, const uint16_t* __restrict__ kmat,
                int H, int rows_per_batch, int t0, int Tq, int Tk_max, int Tk, int q_pos0,
                const int32_t* __restrict__ kv_len, int chunk, uint32_t* __restrict__ keys, long long ld,
                uint32_t* __restrict__ hist) {
  pdl_wait();
  pdl_launch_dependents();
  constexpr int J = D / 32;          // 16-byte chunks per lane per key row
  constexpr int U = 2;               // 8-row tiles per register buffer (two buffers)
  constexpr int WARPS = kScoreThreads / 32;
  __shared__ uint32_t sh[kHistBins];
  const int r = blockIdx.y;
  const int b = r / rows_per_batch, t = t0 + r % rows_per_batch;
  const int n = n_cand(q_pos0, t, row_len(kv_len, b, Tk));
  const int r0 = blockIdx.x * chunk;
  if (r0 >= n) return;
  const int r1 = min(n, r0 + chunk);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tg = lane & 3;
  if (hist != nullptr) {
    for (int i = tid; i < kHistBins; i += kScoreThreads) sh[i] = 0;
    __syncthreads();
  }

  // query fragments: for k-step pair j, lane (g, tg) holds dims of chunk
  // 4j + tg of heads 16hg + g (A rows g) and 16hg + g + 8 (A rows g + 8)
  const long long qrow = (long long)b * Tq + t;
  const uint16_t* qr = q + qrow * H * D;
  uint32_t qe[HG][J][4], qo[HG][J][4];
  float w0[HG], w1[HG];
#pragma unroll
  for (int hg = 0; hg < HG; ++hg) {
    const int h0 = 16 * hg + g, h1 = h0 + 8;
    w0[hg] = h0 < H ? wts[qrow * H + h0] : 0.f;
    w1[hg] = h1 < H ? wts[qrow * H + h1] : 0.f;
#pragma unroll
    for (int j = 0; j < J; ++j) {
      uint4 v0 = make_uint4(0, 0, 0, 0), v1 = make_uint4(0, 0, 0, 0);
      if (h0 < H) v0 = *reinterpret_cast<const uint4*>(qr + (long long)h0 * D + (4 * j + tg) * 8);
      if (h1 < H) v1 = *reinterpret_cast<const uint4*>(qr + (long long)h1 * D + (4 * j + tg) * 8);
      qe[hg][j][0] = v0.x; qe[hg][j][1] = v1.x; qe[hg][j][2] = v0.y; qe[hg][j][3] = v1.y;
      qo[hg][j][0] = v0.z; qo[hg][j][1] = v1.z; qo[hg][j][2] = v0.w; qo[hg][j][3] = v1.w;
    }
  }
  const uint4* kb = reinterpret_cast<const uint4*>(kmat + (long long)b * Tk_max * D);
  uint32_t* kout = keys + (long long)r * ld;
  auto load = [&](uint4 (&v)[U][J], int base) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int row = base + u * 8 + g;
#pragma unroll
      for (int j = 0; j < J; ++j)
        v[u][j] = row < r1 ? __ldg(kb + (long long)row * (D / 8) + 4 * j + tg) : make_uint4(0, 0, 0, 0);
    }
  };
  auto score = [&](const uint4 (&v)[U][J], int base) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float s0 = 0.f, s1 = 0.f;   // keys 2tg and 2tg+1 of the tile: this lane's heads
#pragma unroll
      for (int hg = 0; hg < HG; ++hg) {
        float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < J; ++j) {
          mma_bf16_16816(c, qe[hg][j], v[u][j].x, v[u][j].y);
          mma_bf16_16816(c, qo[hg][j], v[u][j].z, v[u][j].w);
        }
        s0 = fmaf(w0[hg], fmaxf(c[0], 0.f), s0);
        s0 = fmaf(w1[hg], fmaxf(c[2], 0.f), s0);
        s1 = fmaf(w0[hg], fmaxf(c[1], 0.f), s1);
        s1 = fmaf(w1[hg], fmaxf(c[3], 0.f), s1);
      }
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {   // sum over g: the lanes sharing tg
        s0 += __shfl_xor_sync(0xffffffffu, s0, o);
        s1 += __shfl_xor_sync(0xffffffffu, s1, o);
      }
      if (g == 0) {
        const int row = base + u * 8 + 2 * tg;
        const uint32_t k0 = score_key(s0), k1 = score_key(s1);
        if (row < r1) {
          kout[row] = k0;
          if (hist != nullptr) atomicAdd(&sh[k0 >> (32 - kHistBits)], 1u);
        }
        if (row + 1 < r1) {
          kout[row + 1] = k1;
          if (hist != nullptr) atomicAdd(&sh[k1 >> (32 - kHistBits)], 1u);
        }
      }
    }
  };
  constexpr int kStep = WARPS * 8 * U;
  uint4 va[U][J], vb[U][J];
  int base = r0 + warp * 8 * U;
  if (base < r1) load(va, base);
  for (; base < r1; base += 2 * kStep) {
    if (base + kStep < r1) load(vb, base + kStep);
    score(va, base);
    if (base + kStep >= r1) break;
    if (base + 2 * kStep < r1) load(va, base + 2 * kStep);
    score(vb, base + kStep);
  }
  if (hist == nullptr) return;
  __syncthreads();
  uint32_t* hg_row = hist + (long long)r * kHistStride;
  for (int i = tid; i < kHistBins; i += kScoreThreads) {
    const uint32_t cnt = sh[i];
    if (cnt) atomicAdd(hg_row + i, cnt);
  }
}

// ------------------------------------------------------------ block scans

// Exclusive prefix sum over the block (blockDim.x a multiple of 32, <= 1024).
// s_warp needs 33 words.  Returns this thread's prefix; `total` the sum.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* s_warp, uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const uint32_t wv = lane < nw ? s_warp[lane] : 0u;
    uint32_t y = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t z = __shfl_up_sync(0xffffffffu, y, o);
      if (lane >= o) y += z;
    }
    if (lane < nw) s_warp[lane] = y - wv;
    if (lane == 31) s_warp[32] = y;
  }
  __syncthreads();
  const uint32_t r = s_warp[warp] + x - v;
  total = s_warp[32];
  __syncthreads();
  return r;
}

// ------------------------------------------------------------------- finish

// Shared memory of the finish kernel for rows of up to CAND candidates held
// in shared memory, a position bitmap of BMW words and MAXK staged outputs.
template <int CAND, int BMW, int MAXK>
struct FinishSmemT {
  static constexpr int kCand = CAND, kBmw = BMW, kOut = MAXK;
  uint32_t hist[256];
  uint32_t swarp[33];
  uint32_t thr[3];
  uint32_t digit, above, bnd_count, ncand;
  uint32_t kor, kand, por, pand;   // OR / AND of every item's key and position
  alignas(16) uint32_t ckey[CAND];
  alignas(16) uint32_t cpos[CAND];
  alignas(16) uint32_t bits[BMW];   // position bitmap; bucket counts for long rows
  uint32_t wpre[BMW];               // word prefix sums; bucket starts for long rows
  uint32_t opos[MAXK];              // long rows: chosen items grouped by bucket
  uint32_t okey[MAXK];
};
// direct rows of more than 2048 candidates and candidate lists of rows over
// 65536 positions (bucketed emission for long rows), 1024 threads
using FinishSmem = FinishSmemT<kSmemCand, kBitmapWords, kMaxK>;
// rows of at most 2048 candidates, 256 threads: several rows per SM
using FinishSmemSmall = FinishSmemT<2048, 64, 1>;
constexpr int kFinThreadsSmall = 256;
// candidate lists of rows up to 65536 positions (4096 held in shared
// memory, more read in place), 256 threads: several rows per SM
using FinishSmemMed = FinishSmemT<4096, 2048, 1>;

__device__ __forceinline__ void hist_add(uint32_t* h, uint32_t digit, bool active) {
  const unsigned act = __ballot_sync(0xffffffffu, active);
  if (!active) return;
  const unsigned peers = __match_any_sync(act, digit);
  if ((int)(threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(h + digit, (uint32_t)__popc(peers));
}

// Warp 0 locates the digit holding the kk-th element, searching from the
// top bin down (desc) or the bottom bin up (asc).
template <class Sm>
__device__ __forceinline__ void find_digit(Sm& s, uint32_t kk, bool desc) {
  if (threadIdx.x >= 32) return;
  const int lane = threadIdx.x;
  uint32_t c[8], loc = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int bin = desc ? 255 - (lane * 8 + j) : lane * 8 + j;
    c[j] = s.hist[bin];
    loc += c[j];
  }
  uint32_t x = loc;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  const uint32_t excl = x - loc;
  if (excl < kk && kk <= excl + loc) {
    uint32_t cum = excl;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (cum + c[j] >= kk) {
        s.digit = desc ? 255 - (lane * 8 + j) : lane * 8 + j;
        s.above = cum;
        s.bnd_count = c[j];
        break;
      }
      cum += c[j];
    }
  }
}

// Items: keys with explicit positions, or a row of keys (position = index).
struct Items {
  const uint32_t* key;
  const uint32_t* pos;
  int n;
  __device__ __forceinline__ uint32_t k(int i) const { return key[i]; }
  __device__ __forceinline__ uint32_t p(int i) const { return pos ? pos[i] : (uint32_t)i; }
};

// The same, for sources that may also hand over (key, position) pairs in
// global memory (shift 1: element i at word 2 i).
struct PairItems {
  const uint32_t* key;
  const uint32_t* pos;
  int n;
  int shift = 0;
  __device__ __forceinline__ uint32_t k(int i) const { return key[i << shift]; }
  __device__ __forceinline__ uint32_t p(int i) const { return pos ? pos[i << shift] : (uint32_t)i; }
};

// Where the search for the K-th key starts: the bits of its key already
// known (prefix under pmask), how many items still to choose inside that
// prefix (kk), how many items share it (bnd), and the first digit's shift.
struct SelStart {
  uint32_t prefix, pmask, kk, bnd;
  int shift;
  bool bits_known;   // s.kor / kand / por / pand already hold the items' OR / AND
};

// Exact selection of the K largest keys (ties: lower position) among `it`:
// on return an item is chosen iff (key & pmask) > prefix, or it equals
// prefix under pmask and its position is <= pmax.  Radix select with 8-bit
// digits from st.shift down; a digit window on which every item agrees
// (from the OR / AND of all keys, or of all positions) is settled without
// a pass -- integer-valued scores leave most low mantissa bits zero, and
// positions below 2^16 leave the high bits zero.
template <class Sm, int THREADS, class It>
__device__ void select_threshold(Sm& s, const It& it, SelStart st, uint32_t& prefix, uint32_t& pmask,
                                 uint32_t& pmax) {
  const int tid = threadIdx.x;
  if (!st.bits_known) {
    if (tid == 0) {
      s.kor = 0u;
      s.kand = ~0u;
      s.por = 0u;
      s.pand = ~0u;
    }
    __syncthreads();
    uint32_t ko = 0u, ka = ~0u, po = 0u, pa = ~0u;
    for (int i = tid; i < it.n; i += THREADS) {
      const uint32_t key = it.k(i), pos = it.p(i);
      ko |= key;
      ka &= key;
      po |= pos;
      pa &= pos;
    }
    ko = __reduce_or_sync(0xffffffffu, ko);
    ka = __reduce_and_sync(0xffffffffu, ka);
    po = __reduce_or_sync(0xffffffffu, po);
    pa = __reduce_and_sync(0xffffffffu, pa);
    if ((tid & 31) == 0) {
      atomicOr(&s.kor, ko);
      atomicAnd(&s.kand, ka);
      atomicOr(&s.por, po);
      atomicAnd(&s.pand, pa);
    }
    __syncthreads();
  }
  const uint32_t kvar = s.kor ^ s.kand, kfix = s.kand;
  const uint32_t pvar = s.por ^ s.pand, pfix = s.pand;

  prefix = st.prefix;
  pmask = st.pmask;
  uint32_t kk = st.kk, bnd = st.bnd;
  for (int shift = st.shift; bnd != kk;) {
    const uint32_t wmask = (255u << shift) & ~pmask;   // undecided bits of this digit
    if ((kvar & wmask) == 0u) {
      prefix |= kfix & wmask;   // every item has these bits: nothing is above
    } else {
      for (int i = tid; i < 256; i += THREADS) s.hist[i] = 0;
      __syncthreads();
      for (int i0 = 0; i0 < it.n; i0 += THREADS) {
        const int i = i0 + tid;
        const uint32_t key = i < it.n ? it.k(i) : 0u;
        const bool act = i < it.n && (key & pmask) == prefix;
        hist_add(s.hist, (key >> shift) & 255u, act);
      }
      __syncthreads();
      find_digit(s, kk, true);
      __syncthreads();
      kk -= s.above;
      prefix |= s.digit << shift;
      bnd = s.bnd_count;
      __syncthreads();
    }
    pmask |= wmask;
    if (shift == 0) break;
    shift = shift >= 8 ? shift - 8 : 0;
  }
  pmax = 0xFFFFFFFFu;
  if (bnd == kk) return;
  // exact key ties: keep the kk lowest positions among the bnd items with
  // key == prefix.  A small tie group is gathered once and the kk-th lowest
  // position found by counting, for each, the tied positions below it
  // (positions are distinct); larger groups take radix passes over positions.
  constexpr uint32_t kTieList = Sm::kBmw < 256 ? Sm::kBmw : 256;
  if (bnd <= kTieList) {
    uint32_t* list = s.bits;   // free until the emission
    if (tid == 0) s.hist[0] = 0u;
    __syncthreads();
    for (int i = tid; i < it.n; i += THREADS) {
      if (it.k(i) == prefix) {
        const uint32_t slot = atomicAdd(&s.hist[0], 1u);
        if (slot < kTieList) list[slot] = it.p(i);
      }
    }
    __syncthreads();
    const uint32_t m = min(s.hist[0], kTieList);   // == bnd
    for (uint32_t i = tid; i < m; i += THREADS) {
      const uint32_t p = list[i];
      uint32_t below = 0;
      for (uint32_t j = 0; j < m; ++j) below += list[j] < p ? 1u : 0u;
      if (below == kk - 1) s.hist[1] = p;
    }
    __syncthreads();
    pmax = s.hist[1];
    __syncthreads();
    return;
  }
  uint32_t pp = 0, pm = 0;
  for (int shift = 24; shift >= 0; shift -= 8) {
    const uint32_t wmask = 255u << shift;
    uint32_t c = bnd;
    if ((pvar & wmask) == 0u) {
      pp |= pfix & wmask;
    } else {
      for (int i = tid; i < 256; i += THREADS) s.hist[i] = 0;
      __syncthreads();
      for (int i0 = 0; i0 < it.n; i0 += THREADS) {
        const int i = i0 + tid;
        bool act = false;
        uint32_t p = 0;
        if (i < it.n && it.k(i) == prefix) {
          p = it.p(i);
          act = (p & pm) == pp;
        }
        hist_add(s.hist, (p >> shift) & 255u, act);
      }
      __syncthreads();
      find_digit(s, kk, false);
      __syncthreads();
      kk -= s.above;
      pp |= s.digit << shift;
      c = s.bnd_count;
      __syncthreads();
    }
    pm |= wmask;
    bnd = c;
    if (c == kk) {
      pmax = pp | ~pm;
      return;
    }
  }
  pmax = pp;
}

__device__ __forceinline__ bool is_selected(uint32_t key, uint32_t pos, uint32_t prefix, uint32_t pmask,
                                            uint32_t pmax) {
  const uint32_t m = key & pmask;
  return m > prefix || (m == prefix && pos <= pmax);
}

// Writes the chosen item with rank `slot` (0-based, ascending position).
__device__ __forceinline__ void emit(const FinishOut& out, long long o_idx, int b, uint32_t slot,
                                     uint32_t pos, uint32_t key) {
  if (out.rows == nullptr) {
    out.idx[o_idx + slot] = (int32_t)pos;
    if (out.score) out.score[o_idx + slot] = key_score(key);
  } else {
    const int stride = out.chunk_len + 1;
    int32_t* rows = out.rows + (long long)b * out.rows_stride + (long long)slot * stride;
    for (int r = 0; r < stride; ++r) rows[r] = (int32_t)pos * stride + r;
    if (out.chunks) out.chunks[o_idx + slot] = (int32_t)pos;
  }
}

// Writes the K chosen items staged in shared memory (spos / skey indexed by
// output slot) like emit, with consecutive threads on consecutive slots (or
// unfolded rows), so the stores coalesce.
__device__ __forceinline__ void emit_staged(const FinishOut& out, long long o_idx, int b, const uint32_t* spos,
                                            const uint32_t* skey, uint32_t K, int tid, int nthreads) {
  if (out.rows == nullptr) {
    for (uint32_t i = (uint32_t)tid; i < K; i += (uint32_t)nthreads) {
      out.idx[o_idx + i] = (int32_t)spos[i];
      if (out.score) out.score[o_idx + i] = key_score(skey[i]);
    }
  } else {
    const uint32_t stride = (uint32_t)out.chunk_len + 1u;
    int32_t* rows = out.rows + (long long)b * out.rows_stride;
    for (uint32_t e = (uint32_t)tid; e < K * stride; e += (uint32_t)nthreads)
      rows[e] = (int32_t)(spos[e / stride] * stride + e % stride);
    if (out.chunks)
      for (uint32_t i = (uint32_t)tid; i < K; i += (uint32_t)nthreads) out.chunks[o_idx + i] = (int32_t)spos[i];
  }
}

// Writes a row's padding (slots K..k-1 = -1, scores -inf) and count, or, for
// gist routing, the partial chunk's rows after the unfolded ones, the row
// padding and the row count.  A failed row (an upstream wait gave up) gets
// count 0 and no rows at all.
__device__ __forceinline__ void finish_tail(const FinishOut& out, int b, int t, int Tq, int k, uint32_t K,
                                            bool failed, int tid, int nthreads) {
  const long long o_idx = ((long long)b * Tq + t) * (long long)k;
  if (out.rows == nullptr) {
    for (int i = (int)K + tid; i < k; i += nthreads) {
      out.idx[o_idx + i] = -1;
      if (out.score) out.score[o_idx + i] = __int_as_float(0xff800000);
    }
    if (tid == 0) out.count[(long long)b * Tq + t] = (int32_t)K;
  } else {
    const int stride = out.chunk_len + 1;
    int p = out.partial_len ? out.partial_len[b] : 0;
    p = p < 0 ? 0 : (p > out.chunk_len ? out.chunk_len : p);
    if (failed) p = 0;
    const int unfolded = (int)K * stride;
    const int total = unfolded + p;
    int32_t* rows = out.rows + (long long)b * out.rows_stride;
    for (int i = unfolded + tid; i < out.rows_stride; i += nthreads)
      rows[i] = i < total ? out.n_chunks * stride + (i - unfolded) : -1;
    if (out.chunks)
      for (int i = (int)K + tid; i < k; i += nthreads) out.chunks[o_idx + i] = -1;
    if (tid == 0) out.count[b] = total;
  }
}

// ---------------------------------------------------------------- threshold

constexpr int kThrBins = 4096;     // window of the counting select
constexpr int kThrThreads = 512;
constexpr int kThrVec = 4;         // 16-byte loads (8 maxima each) per thread
constexpr int kThrRegMax = kThrThreads * kThrVec * 8;   // maxima held in registers

struct ThrSmem {
  uint32_t hist[kThrBins];
  uint32_t swarp[33];
  uint32_t lo, hi;
  uint32_t digit, above, bnd_count;
};

// One CTA per row: the k-th largest of the row's m group maxima (16-bit
// keys).  Up to kThrRegMax maxima are loaded once, 16 bytes at a time, and
// kept in registers.  One counting pass over the kThrBins values ending at
// their maximum finds the k-th when at least k maxima fall in that window
// (the usual case: the upper maxima of large groups sit in a narrow band);
// otherwise a two-digit radix select (high byte, then low byte) does,
// reading the row again.
__global__ void __launch_bounds__(kThrThreads)
prefill_threshold_kernel(const uint16_t* __restrict__ gmax, long long ld2, int rows_per_batch, int t0, int Tk,
                         int q_pos0, const int32_t* __restrict__ kv_len, int k, uint32_t* __restrict__ theta) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ ThrSmem s;
  const int r = blockIdx.x;
  const int b = r / rows_per_batch;
  const int t = t0 + r % rows_per_batch;
  const int tid = threadIdx.x;
  const int n = n_cand(q_pos0, t, row_len(kv_len, b, Tk));
  const int g = prefill_group_size(n, k);
  if (g == 0) {   // every candidate is chosen
    if (tid == 0) theta[r] = 0u;
    return;
  }
  const int m = (n + g - 1) / g;   // > k
  const uint16_t* row = gmax + (long long)r * ld2;
  const bool in_regs = m <= kThrRegMax;
  uint4 v[kThrVec];
  uint32_t vmax = 0u;
  if (in_regs) {
#pragma unroll
    for (int q = 0; q < kThrVec; ++q) {
      const int i = (q * kThrThreads + tid) * 8;
      v[q] = i < m ? *reinterpret_cast<const uint4*>(row + i) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int q = 0; q < kThrVec; ++q) {
      const int i = (q * kThrThreads + tid) * 8;
      const uint32_t w[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if (i + e < m) vmax = max(vmax, (w[e >> 1] >> (16 * (e & 1))) & 0xFFFFu);
      }
    }
  } else {
    for (int i = tid; i < m; i += kThrThreads) vmax = max(vmax, (uint32_t)row[i]);
  }
  vmax = __reduce_max_sync(0xffffffffu, vmax);
  if (tid == 0) s.hi = 0u;
  for (int i = tid; i < kThrBins; i += kThrThreads) s.hist[i] = 0u;
  __syncthreads();
  if ((tid & 31) == 0) atomicMax(&s.hi, vmax);
  __syncthreads();
  const uint32_t lo = s.hi >= (uint32_t)(kThrBins - 1) ? s.hi - (uint32_t)(kThrBins - 1) : 0u;
  {
    uint32_t below = 0;   // maxima under the window
    if (in_regs) {
#pragma unroll
      for (int q = 0; q < kThrVec; ++q) {
        const int i = (q * kThrThreads + tid) * 8;
        const uint32_t w[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint32_t x = (w[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
          if (i + e < m) {
            if (x >= lo) atomicAdd(&s.hist[x - lo], 1u);
            else ++below;
          }
        }
      }
    } else {
      for (int i = tid; i < m; i += kThrThreads) {
        const uint32_t x = row[i];
        if (x >= lo) atomicAdd(&s.hist[x - lo], 1u);
        else ++below;
      }
    }
    below = __reduce_add_sync(0xffffffffu, below);
    if (tid == 0) s.lo = 0u;
    __syncthreads();
    if ((tid & 31) == 0) atomicAdd(&s.lo, below);
    __syncthreads();
  }
  if ((uint32_t)m - s.lo >= (uint32_t)k) {   // the k-th largest lies in the window
    // thread tid holds bins [kThrBins - per (tid + 1), kThrBins - per tid), counted from the top
    constexpr int per = kThrBins / kThrThreads;
    uint32_t c[per], loc = 0;
#pragma unroll
    for (int j = 0; j < per; ++j) {
      c[j] = s.hist[kThrBins - 1 - (tid * per + j)];
      loc += c[j];
    }
    uint32_t total;
    const uint32_t above = block_excl_scan(loc, s.swarp, total);
    if (above < (uint32_t)k && (uint32_t)k <= above + loc) {
      uint32_t cum = above;
#pragma unroll
      for (int j = 0; j < per; ++j) {
        cum += c[j];
        if (cum >= (uint32_t)k) {
          theta[r] = lo + (uint32_t)(kThrBins - 1 - (tid * per + j));
          break;
        }
      }
    }
    return;
  }
  // wide span: high byte, then low byte among the values sharing it
  if (tid < 256) s.hist[tid] = 0u;
  __syncthreads();
  for (int i0 = 0; i0 < m; i0 += kThrThreads) {
    const int i = i0 + tid;
    const uint32_t x = i < m ? row[i] : 0u;
    hist_add(s.hist, x >> 8, i < m);
  }
  __syncthreads();
  find_digit(s, (uint32_t)k, true);
  __syncthreads();
  const uint32_t hi = s.digit;
  const uint32_t kk = (uint32_t)k - s.above;
  __syncthreads();
  if (tid < 256) s.hist[tid] = 0u;
  __syncthreads();
  for (int i0 = 0; i0 < m; i0 += kThrThreads) {
    const int i = i0 + tid;
    const uint32_t x = i < m ? row[i] : 0u;
    hist_add(s.hist, x & 255u, i < m && (x >> 8) == hi);
  }
  __syncthreads();
  find_digit(s, kk, true);
  __syncthreads();
  if (tid == 0) theta[r] = hi << 8 | s.digit;
}

// One instance per (layout, candidate source): each holds only its own
// path, which keeps the instruction footprint of the hot instances small.
template <class Sm, int THREADS, int MODE>
__global__ void __launch_bounds__(THREADS, THREADS >= 1024 ? 1 : 4)
finish_kernel(RowWorkspace w, int rows_per_batch, int t0, int Tq, int Tk, int q_pos0,
              const int32_t* __restrict__ kv_len, int k, FinishOut out) {
  pdl_wait();
  pdl_launch_dependents();
  constexpr int mode = MODE;
  constexpr int kFinThreads = THREADS;
  constexpr int kSmemCand = Sm::kCand;
  constexpr int kBitmapWords = Sm::kBmw;
  constexpr int kMaxK = Sm::kOut;
  constexpr bool kLong = Sm::kCand == ::sa::kSmemCand;   // the layout that serves rows of any length
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Sm& s = *reinterpret_cast<Sm*>(smem_raw);
  const int r = blockIdx.x;
  const int b = r / rows_per_batch;
  const int t = t0 + r % rows_per_batch;
  const int tid = threadIdx.x;
  const int n = n_cand(q_pos0, t, row_len(kv_len, b, Tk));
  // A wait in an earlier kernel of this call (the tensor-core scorer) that
  // gave up left a nonzero error word: the scores are incomplete, so the row
  // gets the failure sentinel (count 0, every slot -1) instead of a
  // plausible but wrong selection.
  bool failed = w.err != nullptr && *reinterpret_cast<volatile const int*>(w.err) != 0;
  uint32_t K = failed ? 0u : (uint32_t)min(k, n);
  const uint32_t* row = w.keys + (long long)r * w.ld;
  if (tid == 0) s.ncand = 0;
  __syncthreads();

  // ---- gather candidates into shared memory
  std::conditional_t<MODE == kFinishCandRows, PairItems, Items> it;
  it.key = row;
  it.pos = nullptr;
  it.n = n;
  bool in_smem = false;
  bool bits_known = false;                   // the candidates' OR / AND is already in s
  if (K > 0) {
    if (mode == kFinishCandRows) {
      // the bounded pass's takes, (score bits, position) pairs: each scoring
      // CTA left its run of this row at the run's first column, the run's
      // count in that tile's slot (0 in the run's other slots).  Counts are
      // clamped to the columns left, so every read stays in the row.  Slots
      // are taken kFinThreads at a time; each warp copies its lanes' runs
      // with all 32 lanes.
      uint2* cr = reinterpret_cast<uint2*>(w.keys) + (long long)r * w.ld;
      const uint32_t* tcnt = w.tile_cnt + (long long)r * (w.ld / 256);
      const int nslot = (n + 255) / 256;
      auto slot_count = [&](int sl) { return sl < nslot ? min(tcnt[sl], (uint32_t)(n - sl * 256)) : 0u; };
      uint32_t total = 0;
      for (int s0 = 0; s0 < nslot; s0 += kFinThreads) {
        uint32_t part;
        block_excl_scan(slot_count(s0 + tid), s.swarp, part);
        total += part;
      }
      if (total <= (uint32_t)kSmemCand) {
        uint32_t ko = 0u, ka = ~0u, po = 0u, pa = ~0u;
        uint32_t base = 0;
        for (int s0 = 0; s0 < nslot; s0 += kFinThreads) {
          const int sl = s0 + tid;
          const uint32_t c = slot_count(sl);
          uint32_t part;
          const uint32_t o = base + block_excl_scan(c, s.swarp, part);
          base += part;
          unsigned todo = __ballot_sync(0xffffffffu, c != 0u);
          while (todo) {
            const int L = __ffs(todo) - 1;
            todo &= todo - 1;
            const uint32_t cL = __shfl_sync(0xffffffffu, c, L);
            const uint32_t oL = __shfl_sync(0xffffffffu, o, L);
            const long long from = (long long)__shfl_sync(0xffffffffu, sl, L) * 256;
            for (uint32_t j = (uint32_t)(tid & 31); j < cL; j += 32) {
              const uint2 e = cr[from + j];
              const uint32_t key = score_key(__uint_as_float(e.x));
              s.ckey[oL + j] = key;
              s.cpos[oL + j] = e.y;
              ko |= key;
              ka &= key;
              po |= e.y;
              pa &= e.y;
            }
          }
        }
        if (tid == 0) {
          s.kor = 0u;
          s.kand = ~0u;
          s.por = 0u;
          s.pand = ~0u;
          s.ncand = total;
        }
        __syncthreads();
        ko = __reduce_or_sync(0xffffffffu, ko);
        ka = __reduce_and_sync(0xffffffffu, ka);
        po = __reduce_or_sync(0xffffffffu, po);
        pa = __reduce_and_sync(0xffffffffu, pa);
        if ((tid & 31) == 0) {
          atomicOr(&s.kor, ko);
          atomicAnd(&s.kand, ka);
          atomicOr(&s.por, po);
          atomicAnd(&s.pand, pa);
        }
        in_smem = true;
        bits_known = true;
      } else {
        // more takes than shared memory holds (heavy ties): close the gaps
        // between runs in place, kFinThreads pairs per round (a round's
        // writes land at or before its reads, which are all done), turning
        // scores into keys on the way
        uint32_t dst = 0;
        for (int sl = 0; sl < nslot; ++sl) {
          const uint32_t c = slot_count(sl);
          for (uint32_t j0 = 0; j0 < c; j0 += kFinThreads) {
            const uint32_t j = j0 + tid;
            uint2 e = make_uint2(0u, 0u);
            if (j < c) e = cr[(long long)sl * 256 + j];
            __syncthreads();
            if (j < c) cr[dst + j] = make_uint2(score_key(__uint_as_float(e.x)), e.y);
            __syncthreads();
          }
          dst += c;
        }
        if constexpr (MODE == kFinishCandRows) {
          it.key = reinterpret_cast<const uint32_t*>(cr);
          it.pos = reinterpret_cast<const uint32_t*>(cr) + 1;
          it.shift = 1;
        }
        it.n = (int)total;
      }
      __syncthreads();
    } else {
      // kFinishDirect: every candidate of the row (direct launches hold rows
      // of at most kSmemCand candidates)
      for (int i = tid; i < n; i += kFinThreads) { s.ckey[i] = row[i]; s.cpos[i] = (uint32_t)i; }
      if (tid == 0) s.ncand = (uint32_t)n;
      in_smem = true;
      __syncthreads();
    }
    if (in_smem) {
      it.key = s.ckey;
      it.pos = s.cpos;
      it.n = (int)s.ncand;
    }
  }

  uint32_t prefix = 0, pmask = 0, pmax = 0;
  if (K > 0) {
    const SelStart st{0u, 0u, K, (uint32_t)it.n, 24, bits_known};
    select_threshold<Sm, THREADS>(s, it, st, prefix, pmask, pmax);
  }

  const long long o_idx = ((long long)b * Tq + t) * (long long)k;
  if (K > 0) {
    if (n <= kBitmapWords * 32) {
      // ---- emission through a position bitmap
      const int W = (n + 31) >> 5;
      for (int i = tid; i < W; i += kFinThreads) s.bits[i] = 0;
      __syncthreads();
      for (int i = tid; i < it.n; i += kFinThreads) {
        const uint32_t key = it.k(i), pos = it.p(i);
        if (is_selected(key, pos, prefix, pmask, pmax)) atomicOr(&s.bits[pos >> 5], 1u << (pos & 31));
      }
      __syncthreads();
      const int per = (W + kFinThreads - 1) / kFinThreads;
      const int w0 = tid * per;
      uint32_t mine = 0;
      for (int j = 0; j < per; ++j)
        if (w0 + j < W) mine += __popc(s.bits[w0 + j]);
      uint32_t total;
      uint32_t run = block_excl_scan(mine, s.swarp, total);
      for (int j = 0; j < per; ++j)
        if (w0 + j < W) {
          s.wpre[w0 + j] = run;
          run += __popc(s.bits[w0 + j]);
        }
      __syncthreads();
      for (int i = tid; i < it.n; i += kFinThreads) {
        const uint32_t key = it.k(i), pos = it.p(i);
        if (is_selected(key, pos, prefix, pmask, pmax)) {
          const uint32_t slot = s.wpre[pos >> 5] + __popc(s.bits[pos >> 5] & ((1u << (pos & 31)) - 1u));
          if (slot < K) emit(out, o_idx, b, slot, pos, key);   // exactly K are chosen
        }
      }
    } else if constexpr (kLong) {
      // ---- long rows: the chosen items are counted into kBitmapWords
      // equal position ranges, placed range by range, and ranked inside
      // their range (ranges hold about K / kBitmapWords items each)
      int bsh = 0;
      while (((n - 1) >> bsh) >= kBitmapWords) ++bsh;
      uint32_t* cnt = s.bits;
      uint32_t* start = s.wpre;
      for (int i = tid; i < kBitmapWords; i += kFinThreads) cnt[i] = 0;
      __syncthreads();
      for (int i = tid; i < it.n; i += kFinThreads) {
        const uint32_t key = it.k(i), pos = it.p(i);
        if (is_selected(key, pos, prefix, pmask, pmax)) atomicAdd(&cnt[pos >> bsh], 1u);
      }
      __syncthreads();
      constexpr int per = kBitmapWords / kFinThreads;
      uint32_t c[per], mine = 0;
#pragma unroll
      for (int j = 0; j < per; ++j) {
        c[j] = cnt[tid * per + j];
        mine += c[j];
      }
      uint32_t total;
      uint32_t run = block_excl_scan(mine, s.swarp, total);
#pragma unroll
      for (int j = 0; j < per; ++j) {
        start[tid * per + j] = run;
        run += c[j];
        cnt[tid * per + j] = 0;   // becomes the fill counter
      }
      __syncthreads();
      for (int i = tid; i < it.n; i += kFinThreads) {
        const uint32_t key = it.k(i), pos = it.p(i);
        if (is_selected(key, pos, prefix, pmask, pmax)) {
          const uint32_t bk = pos >> bsh;
          const uint32_t o = start[bk] + atomicAdd(&cnt[bk], 1u);
          if (o < (uint32_t)kMaxK) {
            s.opos[o] = pos;
            s.okey[o] = key;
          }
        }
      }
      __syncthreads();
      // exactly K items are chosen; the bounds below only keep a broken
      // input (e.g. a histogram that does not match the keys) from reading
      // or writing out of range
      const uint32_t placed = min(min(total, K), (uint32_t)kMaxK);
      for (int i = tid; i < (int)placed; i += kFinThreads) {
        const uint32_t pos = s.opos[i], bk = pos >> bsh;
        if (bk >= (uint32_t)kBitmapWords) continue;
        const uint32_t b0 = start[bk], b1 = min(b0 + cnt[bk], placed);
        uint32_t rank = b0;
        for (uint32_t j = b0; j < b1; ++j) rank += s.opos[j] < pos ? 1u : 0u;
        if (rank < K) emit(out, o_idx, b, rank, pos, s.okey[i]);
      }
    }
  }

  // ---- padding and counts
  finish_tail(out, b, t, Tq, k, K, failed, tid, kFinThreads);
}

// ------------------------------------------------------------- split rows
//
// Rows that carry the scorer's histogram (one query per sequence: decode
// scoring and gist routing over more than kDirectMaxCand candidates) are
// selected by many CTAs per row, with no CTA waiting for another.
//   1. Every CTA finds, from the scorer's histogram of the keys' top 12 bits,
//      the bin of the row's K-th largest key.  CTA c then filters positions
//      [c * chunk, (c + 1) * chunk): each key in or above that bin goes, with
//      its position and in position order (one block scan), into the slice's
//      part of the row's candidate array; keys inside the bin also count in a
//      second histogram of their next 12 bits.  The slice's candidate count
//      goes to its slot, and the CTA takes a ticket on the row's counter
//      (threadfence, then atomicAdd).
//   2. The row's last CTA gathers every slice's candidates (already in
//      ascending position order) and finds, from the second histogram, the
//      24-bit prefix T of the K-th key and how many of the keys with prefix T
//      are still to take (kk).  When those keys are all equal (integer-valued
//      scores make every key a multiple of 256), the first kk of them in
//      position order are the chosen ones, so one block scan of packed
//      (above-T, equal-to-T) counts gives every item both its choice and its
//      output slot.  Otherwise an exact radix select over the low 8 bits and
//      the positions decides, followed by an ordered compaction.
//   3. The last CTA returns the row's histograms and counter to zero.

constexpr int kSplitThreads = 512;
constexpr int kSplitCand = 8192;         // candidates the finishing CTA holds in shared memory
constexpr int kSplitSlice = kSplitThreads * 4;   // positions per slice unit (one uint4 per thread)
constexpr int kSplitPer = 8;             // candidates per thread and pass of the finishing CTA

struct SplitSmem {
  static constexpr int kBmw = 256;       // bounds the select's tie list
  uint32_t hist[256];
  uint32_t swarp[33];
  uint32_t thr[3];                       // first-level bin of the K-th key, keys above it, keys in it
  uint32_t thr2[3];                      // the same for the next 12 bits inside that bin
  uint32_t digit, above, bnd_count, ncand;
  uint32_t kor, kand, por, pand;
  int last;
  uint32_t bits[256];                    // tie list of the general select
  uint32_t pre[kSplitMaxSlices];         // first gathered index of each slice
  alignas(16) uint32_t ckey[kSplitCand];
  alignas(16) uint32_t cpos[kSplitCand];
};
static_assert(offsetof(SplitSmem, ckey) % 16 == 0 && offsetof(SplitSmem, cpos) % 16 == 0,
              "candidate arrays are read as 16-byte vectors");

// A 4096-bin histogram (bins in key order) read with 16-byte loads through
// L2 into registers, thread 0 holding the top bins.  The loads are issued
// here and consumed by hist_pick, so other loads can share their round trip.
template <int THREADS>
struct HistRegs {
  static constexpr int per = kHistBins / THREADS;
  static_assert(per % 4 == 0, "16-byte loads of whole bins");
  uint32_t c[per];
};

template <int THREADS>
__device__ __forceinline__ void hist_load(const uint32_t* __restrict__ h, HistRegs<THREADS>& r) {
  constexpr int per = HistRegs<THREADS>::per;
  const int base = kHistBins - per * ((int)threadIdx.x + 1);
#pragma unroll
  for (int v = 0; v < per / 4; ++v) {
    const uint4 x = __ldcg(reinterpret_cast<const uint4*>(h + base) + v);
    r.c[4 * v] = x.x;
    r.c[4 * v + 1] = x.y;
    r.c[4 * v + 2] = x.z;
    r.c[4 * v + 3] = x.w;
  }
}

// Bin of the K-th largest key of the histogram in r: s_out[0] = bin,
// s_out[1] = keys in the bins above it, s_out[2] = keys in it (0, 0, 0 when
// the histogram holds fewer than K keys).  Every thread of the block calls it.
template <int THREADS>
__device__ __forceinline__ void hist_pick(const HistRegs<THREADS> r, uint32_t K, uint32_t* s_warp,
                                          uint32_t* s_out) {
  constexpr int per = HistRegs<THREADS>::per;
  const int base = kHistBins - per * ((int)threadIdx.x + 1);
  const uint32_t* c = r.c;
  if (threadIdx.x == 0) {
    s_out[0] = 0u;
    s_out[1] = 0u;
    s_out[2] = 0u;
  }
  uint32_t loc = 0;
#pragma unroll
  for (int j = 0; j < per; ++j) loc += c[j];
  uint32_t total;
  const uint32_t excl = block_excl_scan(loc, s_warp, total);   // keys in the bins above this thread's
  if (excl < K && K <= excl + loc) {
    uint32_t cum = excl;
#pragma unroll
    for (int j = per - 1; j >= 0; --j) {
      if (cum < K && cum + c[j] >= K) {
        s_out[0] = (uint32_t)(base + j);
        s_out[1] = cum;
        s_out[2] = c[j];
      }
      cum += c[j];
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kSplitThreads, 2)
split_topk_kernel(RowWorkspace w, int rows_per_batch, int t0, int Tq, int Tk, int q_pos0,
                  const int32_t* __restrict__ kv_len, int k, int chunk, FinishOut out) {
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SplitSmem& s = *reinterpret_cast<SplitSmem*>(smem_raw);
  const int c = blockIdx.x, F = gridDim.x, r = blockIdx.y;
  const int b = r / rows_per_batch;
  const int t = t0 + r % rows_per_batch;
  const int tid = threadIdx.x;
  const int n = n_cand(q_pos0, t, row_len(kv_len, b, Tk));
  uint32_t* hist1 = w.hist + (long long)r * kHistStride;
  uint32_t* hist2 = hist1 + kHistBins;
  // the first histogram's loads share their round trip with the error word's
  HistRegs<kSplitThreads> h1;
  hist_load(hist1, h1);
  // a wait in an earlier kernel of this call that gave up: failure sentinel
  const bool failed = w.err != nullptr && *reinterpret_cast<volatile const int*>(w.err) != 0;
  const uint32_t K = failed ? 0u : (uint32_t)min(k, n);
  const uint32_t* row = w.keys + (long long)r * w.ld;
  uint2* cand = w.cand + (long long)r * w.ld;
  uint32_t* slot = w.slot_cnt + (long long)r * kSplitMaxSlices;
  const int c0 = c * chunk;
  constexpr int kLo = 32 - kHistBits;        // shift of the first-level bin
  constexpr int kLo2 = 32 - 2 * kHistBits;   // shift of the second-level bin

  // ---- 1. filter this slice (in position order)
  uint32_t taken = 0;
  if (K > 0) {
    hist_pick(h1, K, s.swarp, s.thr);
    const uint32_t bin = s.thr[0];
    for (int u0 = 0; u0 < chunk; u0 += kSplitSlice) {
      const int i = c0 + u0 + tid * 4;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (i < n) v = *reinterpret_cast<const uint4*>(row + i);   // rows are padded to 256 keys
      const uint32_t kv[4] = {v.x, v.y, v.z, v.w};
      uint32_t mine = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) mine += (i + e < n && (kv[e] >> kLo) >= bin) ? 1u : 0u;
      uint32_t tot;
      uint32_t o = (uint32_t)c0 + taken + block_excl_scan(mine, s.swarp, tot);
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (i + e < n && (kv[e] >> kLo) >= bin) {
          cand[o++] = make_uint2(kv[e], (uint32_t)(i + e));
          if ((kv[e] >> kLo) == bin) atomicAdd(hist2 + ((kv[e] >> kLo2) & (kHistBins - 1)), 1u);
        }
      taken += tot;
      if (c0 + u0 + kSplitSlice >= n) break;
    }
  }
  if (tid == 0) slot[c] = taken;

  // ---- ticket: the row's last CTA finishes the row
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    s.last = atomicAdd(&w.cand_cnt[r], 1u) == (uint32_t)F - 1u;
  }
  __syncthreads();
  if (!s.last) return;
  __threadfence();

  // ---- 2. the finishing CTA (the second histogram's loads share their
  // round trip with the slice counts')
  HistRegs<kSplitThreads> h2;
  hist_load(hist2, h2);
  uint32_t total = 0;
  for (int s0 = 0; s0 < F; s0 += kSplitThreads) {
    const int sl = s0 + tid;
    const uint32_t v = sl < F ? __ldcg(slot + sl) : 0u;
    uint32_t part;
    const uint32_t o = total + block_excl_scan(v, s.swarp, part);
    if (sl < F) s.pre[sl] = o;
    total += part;
  }
  __syncthreads();
  const bool in_smem = total <= (uint32_t)kSplitCand;
  const long long o_idx = ((long long)b * Tq + t) * (long long)k;
  if (K > 0) {
    // Gathered candidate i belongs to the last slice whose first index is
    // <= i.  A thread's kSplitPer candidates of a pass are consecutive, so one
    // binary search places the first and the slice only moves forward.
    auto fetch = [&](uint32_t i0, uint2 (&e)[kSplitPer]) {
      const uint32_t ib = i0 + (uint32_t)tid * kSplitPer;
      int lo = 0, hi = F - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s.pre[mid] <= ib) lo = mid;
        else hi = mid - 1;
      }
#pragma unroll
      for (int u = 0; u < kSplitPer; ++u) {
        const uint32_t i = ib + u;
        while (lo + 1 < F && s.pre[lo + 1] <= i) ++lo;
        e[u] = i < total ? __ldcg(cand + (long long)lo * chunk + (i - s.pre[lo])) : make_uint2(0u, 0u);
      }
    };
    // the first pass's loads are issued before the second histogram is read,
    // so both are in flight together
    uint2 e[kSplitPer];
    uint32_t i0 = 0;
    if (in_smem) fetch(0u, e);
    hist_pick(h2, K - s.thr[1], s.swarp, s.thr2);
    const uint32_t T = s.thr[0] << kHistBits | s.thr2[0];   // 24-bit prefix of the K-th key
    const uint32_t kk = K - s.thr[1] - s.thr2[1];           // keys with prefix T still to take
    PairItems it;
    it.n = (int)total;
    bool uniform = false;   // every key with prefix T is the same key
    if (in_smem) {
      if (tid == 0) {
        s.kor = 0u;
        s.kand = ~0u;
      }
      uint32_t ko = 0u, ka = ~0u;
      static_assert(kSplitPer == 8, "two 16-byte stores per array and thread");
      for (i0 = 0; i0 < total; i0 += kSplitThreads * kSplitPer) {
        if (i0 > 0) fetch(i0, e);
        const uint32_t ib = i0 + (uint32_t)tid * kSplitPer;
        if (ib + kSplitPer <= total) {   // 16-byte stores: two-way bank conflicts at most
          uint4* dk = reinterpret_cast<uint4*>(s.ckey + ib);
          uint4* dp = reinterpret_cast<uint4*>(s.cpos + ib);
          dk[0] = make_uint4(e[0].x, e[1].x, e[2].x, e[3].x);
          dk[1] = make_uint4(e[4].x, e[5].x, e[6].x, e[7].x);
          dp[0] = make_uint4(e[0].y, e[1].y, e[2].y, e[3].y);
          dp[1] = make_uint4(e[4].y, e[5].y, e[6].y, e[7].y);
        } else {
#pragma unroll
          for (int u = 0; u < kSplitPer; ++u)
            if (ib + u < total) {
              s.ckey[ib + u] = e[u].x;
              s.cpos[ib + u] = e[u].y;
            }
        }
#pragma unroll
        for (int u = 0; u < kSplitPer; ++u)
          if (ib + u < total && (e[u].x >> 8) == T) {
            ko |= e[u].x;
            ka &= e[u].x;
          }
      }
      __syncthreads();
      ko = __reduce_or_sync(0xffffffffu, ko);
      ka = __reduce_and_sync(0xffffffffu, ka);
      if ((tid & 31) == 0) {
        atomicOr(&s.kor, ko);
        atomicAnd(&s.kand, ka);
      }
      __syncthreads();
      uniform = s.kor == s.kand;   // (no key with prefix T at all cannot happen: kk >= 1)
      it.key = s.ckey;
      it.pos = s.cpos;
      it.shift = 0;
    } else {
      // more candidates than shared memory holds (heavy ties): close the gaps
      // between slices in place, kSplitThreads pairs per round (a round's
      // writes land at or before its reads, which are all done)
      for (int sl = 0; sl < F; ++sl) {
        const uint32_t cnt = __ldcg(slot + sl);
        const uint32_t dst = s.pre[sl];
        for (uint32_t j0 = 0; j0 < cnt; j0 += kSplitThreads) {
          const uint32_t j = j0 + tid;
          uint2 v = make_uint2(0u, 0u);
          if (j < cnt) v = __ldcg(cand + (long long)sl * chunk + j);
          __syncthreads();
          if (j < cnt) cand[dst + j] = v;
          __syncthreads();
        }
      }
      it.key = reinterpret_cast<const uint32_t*>(cand);
      it.pos = reinterpret_cast<const uint32_t*>(cand) + 1;
      it.shift = 1;
    }

    if (uniform) {
      // ---- 2a. the first kk keys equal to the K-th key, in position order,
      // are chosen: slot = (chosen keys above T before it) + min(keys equal
      // to T before it, kk); counts packed as (equal << 16 | above)
      uint32_t base = 0;
      for (i0 = 0; i0 < total; i0 += kSplitThreads * kSplitPer) {
        const uint32_t i = i0 + (uint32_t)tid * kSplitPer;
        uint32_t kk8[kSplitPer], pp8[kSplitPer], mine = 0;
#pragma unroll
        for (int u = 0; u < kSplitPer; u += 4) {
          uint4 kv = make_uint4(0u, 0u, 0u, 0u), pv = make_uint4(0u, 0u, 0u, 0u);
          if (i + u + 3 < total) {
            kv = *reinterpret_cast<const uint4*>(s.ckey + i + u);
            pv = *reinterpret_cast<const uint4*>(s.cpos + i + u);
          } else {
            if (i + u < total) { kv.x = s.ckey[i + u]; pv.x = s.cpos[i + u]; }
            if (i + u + 1 < total) { kv.y = s.ckey[i + u + 1]; pv.y = s.cpos[i + u + 1]; }
            if (i + u + 2 < total) { kv.z = s.ckey[i + u + 2]; pv.z = s.cpos[i + u + 2]; }
          }
          kk8[u] = kv.x; kk8[u + 1] = kv.y; kk8[u + 2] = kv.z; kk8[u + 3] = kv.w;
          pp8[u] = pv.x; pp8[u + 1] = pv.y; pp8[u + 2] = pv.z; pp8[u + 3] = pv.w;
        }
#pragma unroll
        for (int u = 0; u < kSplitPer; ++u) {
          const bool v = i + u < total;
          const uint32_t p24 = kk8[u] >> 8;
          mine += v && p24 > T ? 1u : (v && p24 == T ? 0x10000u : 0u);
        }
        uint32_t tot;
        uint32_t run = base + block_excl_scan(mine, s.swarp, tot);
#pragma unroll
        for (int u = 0; u < kSplitPer; ++u) {
          if (i + u < total) {
            const uint32_t p24 = kk8[u] >> 8;
            const uint32_t above = run & 0xFFFFu, equal = run >> 16;
            // staged by output slot (a slot never exceeds its item's index, and
            // this pass's reads are done), written out coalesced below
            if (p24 > T) {
              const uint32_t sl = above + min(equal, kk);
              if (sl < K) {
                s.cpos[sl] = pp8[u];
                s.ckey[sl] = kk8[u];
              }
              run += 1u;
            } else if (p24 == T) {
              if (equal < kk && above + equal < K) {
                s.cpos[above + equal] = pp8[u];
                s.ckey[above + equal] = kk8[u];
              }
              run += 0x10000u;
            }
          }
        }
        base += tot;
      }
    } else {
      // ---- 2b. exact select below the 24-bit prefix (low 8 bits, then
      // positions), then an ordered compaction of the chosen items
      uint32_t prefix = 0u, pmask = 0u, pmax = 0xFFFFFFFFu;
      const SelStart st{T << 8, 0xFFFFFF00u, kk, s.thr2[2], 0, false};
      select_threshold<SplitSmem, kSplitThreads>(s, it, st, prefix, pmask, pmax);
      uint32_t base = 0;
      for (i0 = 0; i0 < total; i0 += kSplitThreads * 4) {
        const uint32_t i = i0 + (uint32_t)tid * 4;
        uint32_t kk4[4], pp4[4];
        bool sel[4];
        uint32_t mine = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          kk4[u] = i + u < total ? it.k((int)(i + u)) : 0u;
          pp4[u] = i + u < total ? it.p((int)(i + u)) : 0u;
          sel[u] = i + u < total && is_selected(kk4[u], pp4[u], prefix, pmask, pmax);
          mine += sel[u] ? 1u : 0u;
        }
        uint32_t tot;
        uint32_t o = base + block_excl_scan(mine, s.swarp, tot);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (sel[u]) {
            if (o < K) {   // exactly K are chosen; staged by slot as in 2a
              s.cpos[o] = pp4[u];
              s.ckey[o] = kk4[u];
            }
            ++o;
          }
        base += tot;
      }
    }
    __syncthreads();
    emit_staged(out, o_idx, b, s.cpos, s.ckey, K, tid, kSplitThreads);
  }
  finish_tail(out, b, t, Tq, k, K, failed, tid, kSplitThreads);

  // ---- 3. every CTA of the row has used the histograms: return them and
  // the ticket to zero for the next call
  for (int i = tid * 4; i < kHistStride; i += kSplitThreads * 4)
    *reinterpret_cast<uint4*>(hist1 + i) = make_uint4(0u, 0u, 0u, 0u);
  if (tid == 0) w.cand_cnt[r] = 0u;
}

// ------------------------------------------------------ two-level gist routing
//
// hier_gist_kernel: one CTA per sequence routes one decode query coarse to
// fine ([SSA] §五 H-SSA, [GSA] 2.4): (1) the query is scored against the
// meta-gist key of every complete group of group_size chunks and the top
// k_groups groups are kept; (2) the candidate chunks -- those of the kept
// groups, in ascending order, then the chunks after the last complete group
// (no meta-gist yet) -- are scored against their gist keys and the top
// k_chunks are kept; (3) they are unfolded like single-level routing.  Both
// selections are the exact radix select of the other paths (equal scores:
// lower group / chunk first); the chosen items are placed in ascending
// order by block scans.  Scores are fp32 sums of bf16 products (exact for
// integer-valued inputs).

constexpr int kHgThreads = 256;
constexpr int kHgMax = 8192;   // meta keys, and candidate chunks, held in shared memory

struct HGistSmem {
  static constexpr int kBmw = 256;   // bounds the select's tie list
  uint32_t hist[256];
  uint32_t swarp[33];
  uint32_t digit, above, bnd_count;
  uint32_t kor, kand, por, pand;
  uint32_t bits[256];
  alignas(16) float q[128];
  alignas(16) uint32_t key[kHgMax];
  uint32_t list[kHgMax];           // kept groups in ascending order
};

template <int D>
__device__ __forceinline__ float hg_dot(const uint16_t* __restrict__ krow, const float* qs) {
  const uint4* kv = reinterpret_cast<const uint4*>(krow);
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < D / 8; ++c) s += dot8(__ldg(kv + c), qs + 8 * c);
  return s;
}

// Ascending list of the chosen items among n (one block scan per pass of
// kHgThreads items): out[slot] = index.  Returns the number placed.
__device__ __forceinline__ uint32_t hg_place(HGistSmem& s, const uint32_t* key, int n, uint32_t prefix,
                                             uint32_t pmask, uint32_t pmax, uint32_t* out, uint32_t cap) {
  uint32_t base = 0;
  for (int i0 = 0; i0 < n; i0 += kHgThreads) {
    const int i = i0 + threadIdx.x;
    const bool sel = i < n && is_selected(key[i], (uint32_t)i, prefix, pmask, pmax);
    uint32_t tot;
    const uint32_t o = base + block_excl_scan(sel ? 1u : 0u, s.swarp, tot);
    if (sel && o < cap) out[o] = (uint32_t)i;
    base += tot;
  }
  __syncthreads();
  return base < cap ? base : cap;
}

template <int D>
__global__ void __launch_bounds__(kHgThreads)
hier_gist_kernel(const uint16_t* __restrict__ q_route, const uint16_t* __restrict__ meta_key,
                 const uint16_t* __restrict__ gist_key, int n_chunks, int group_size, int k_groups, int k,
                 FinishOut out, int32_t* __restrict__ groups_out) {
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ __align__(16) unsigned char smem_raw[];
  HGistSmem& s = *reinterpret_cast<HGistSmem*>(smem_raw);
  const int b = blockIdx.x, tid = threadIdx.x;
  const int n_groups = n_chunks / group_size;
  for (int i = tid; i < D; i += kHgThreads) {
    const uint16_t v = q_route[(long long)b * D + i];
    s.q[i] = __uint_as_float((uint32_t)v << 16);
  }
  __syncthreads();

  // ---- 1. coarse: meta keys of the complete groups
  const uint16_t* mk = meta_key + (long long)b * n_groups * D;
  for (int g = tid; g < n_groups; g += kHgThreads) s.key[g] = score_key(hg_dot<D>(mk + (long long)g * D, s.q));
  __syncthreads();
  const uint32_t KG = (uint32_t)min(k_groups, n_groups);
  uint32_t prefix = 0u, pmask = 0u, pmax = 0xFFFFFFFFu;   // every item chosen
  if (KG > 0 && KG < (uint32_t)n_groups) {
    const Items it{s.key, nullptr, n_groups};
    select_threshold<HGistSmem, kHgThreads>(s, it, SelStart{0u, 0u, KG, (uint32_t)n_groups, 24, false}, prefix,
                                            pmask, pmax);
  }
  const uint32_t n_sel = KG > 0 ? hg_place(s, s.key, n_groups, prefix, pmask, pmax, s.list, KG) : 0u;
  if (groups_out != nullptr)
    for (int i = tid; i < k_groups; i += kHgThreads)
      groups_out[(long long)b * k_groups + i] = i < (int)n_sel ? (int32_t)s.list[i] : -1;

  // ---- 2. fine: gist keys of the candidate chunks (ascending chunk order)
  const int trail0 = n_groups * group_size;
  const int n_cand = (int)n_sel * group_size + (n_chunks - trail0);
  auto cand_chunk = [&](int j) {
    return j < (int)n_sel * group_size ? (int)s.list[j / group_size] * group_size + j % group_size
                                       : trail0 + (j - (int)n_sel * group_size);
  };
  const uint16_t* gk = gist_key + (long long)b * n_chunks * D;
  for (int j = tid; j < n_cand; j += kHgThreads)
    s.key[j] = score_key(hg_dot<D>(gk + (long long)cand_chunk(j) * D, s.q));
  __syncthreads();
  const uint32_t K = (uint32_t)min(k, n_cand);
  prefix = 0u;
  pmask = 0u;
  pmax = 0xFFFFFFFFu;
  if (K > 0 && K < (uint32_t)n_cand) {
    const Items it{s.key, nullptr, n_cand};
    select_threshold<HGistSmem, kHgThreads>(s, it, SelStart{0u, 0u, K, (uint32_t)n_cand, 24, false}, prefix, pmask,
                                            pmax);
  }

  // ---- 3. unfold the chosen chunks in ascending order
  const long long o_idx = (long long)b * k;
  uint32_t base = 0;
  for (int i0 = 0; i0 < n_cand; i0 += kHgThreads) {
    const int j = i0 + tid;
    const bool sel = K > 0 && j < n_cand && is_selected(s.key[j], (uint32_t)j, prefix, pmask, pmax);
    uint32_t tot;
    const uint32_t o = base + block_excl_scan(sel ? 1u : 0u, s.swarp, tot);
    if (sel && o < K) emit(out, o_idx, b, o, (uint32_t)cand_chunk(j), 0u);
    base += tot;
  }
  finish_tail(out, b, 0, 1, k, K, false, tid, kHgThreads);
}

// ------------------------------------------------------------ index overlap
//
// index_overlap_kernel: per row, the number of positions two ascending
// selections share ([IC] §一 measures 70-100% between adjacent layers).  One
// warp per row: each lane binary-searches its share of A's positions in B.

__global__ void __launch_bounds__(256)
index_overlap_kernel(const int32_t* __restrict__ a, const int32_t* __restrict__ ca, const int32_t* __restrict__ b,
                     const int32_t* __restrict__ cb, int rows, int k, int32_t* __restrict__ out) {
  pdl_wait();
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * 8 + warp;
  if (r >= rows) return;
  const int na = min(max(ca[r], 0), k), nb = min(max(cb[r], 0), k);
  const int32_t* A = a + (long long)r * k;
  const int32_t* Bv = b + (long long)r * k;
  int hits = 0;
  for (int i = lane; i < na; i += 32) {
    const int32_t x = A[i];
    int lo = 0, hi = nb;   // first position in B not below x
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (Bv[mid] < x) lo = mid + 1;
      else hi = mid;
    }
    hits += (lo < nb && Bv[lo] == x) ? 1 : 0;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) hits += __shfl_xor_sync(0xffffffffu, hits, o);
  if (lane == 0) out[r] = hits;
}

}  // namespace

// ------------------------------------------------------------------ host side

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
static long long row_ld(int Tk_max) { return ((long long)Tk_max + 255) / 256 * 256; }

// Layout: [error word][fixed histograms + counters for kHistRowsFixed rows]
// [histograms + counters for larger row counts][keys][split rows: candidate
// pairs, slice counts].  The fixed region holds nothing else, so once
// zero-filled it stays valid across calls of any shape (the selection
// returns each row it used to zero).
size_t row_workspace_bytes(int rows, int Tk_max, bool split, bool with_hist) {
  const long long ld = row_ld(Tk_max);
  size_t bytes = 256;
  bytes += align256((size_t)kHistRowsFixed * kHistStride * 4) + align256((size_t)kHistRowsFixed * 4);
  if (with_hist && rows > kHistRowsFixed)
    bytes += align256((size_t)rows * kHistStride * 4) + align256((size_t)rows * 4);
  bytes += align256((size_t)rows * ld * 4);
  if (split) bytes += align256((size_t)rows * ld * 8) + align256((size_t)rows * kSplitMaxSlices * 4);
  return bytes;
}

void carve_row_workspace(void* ws, int rows, int Tk_max, bool split, bool with_hist, RowWorkspace* o) {
  char* p = static_cast<char*>(ws);
  o->ld = row_ld(Tk_max);
  o->err = reinterpret_cast<int*>(p);
  p += 256;
  o->hist = reinterpret_cast<uint32_t*>(p);
  p += align256((size_t)kHistRowsFixed * kHistStride * 4);
  o->cand_cnt = reinterpret_cast<uint32_t*>(p);
  p += align256((size_t)kHistRowsFixed * 4);
  o->hist_zero_bytes = 0;
  if (with_hist && rows > kHistRowsFixed) {
    o->hist = reinterpret_cast<uint32_t*>(p);
    p += align256((size_t)rows * kHistStride * 4);
    o->cand_cnt = reinterpret_cast<uint32_t*>(p);
    p += align256((size_t)rows * 4);
    o->hist_zero_bytes = (size_t)(p - reinterpret_cast<char*>(o->hist));
  }
  o->keys = reinterpret_cast<uint32_t*>(p);
  p += align256((size_t)rows * o->ld * 4);
  if (split) {
    o->cand = reinterpret_cast<uint2*>(p);
    p += align256((size_t)rows * o->ld * 8);
    o->slot_cnt = reinterpret_cast<uint32_t*>(p);
  }
}

template <int D>
int score_grid(long long rows) {
  const int sms = device_sm_count();
  const int occ = device_occupancy((const void*)score_decode_kernel<D>, kScoreThreads, 0);
  long long want = (long long)sms * occ;
  const long long by_rows = (rows + 255) / 256;
  if (want > by_rows) want = by_rows;
  return (int)(want < 1 ? 1 : want);
}

cudaError_t launch_score_decode(const uint16_t* q, const uint16_t* kmat, int B, int d, int Tk_max,
                                int Tk, int q_pos0, const int32_t* kv_len, const RowWorkspace& w,
                                bool with_hist, cudaStream_t st) {
  if (Tk <= 0 || B <= 0) return cudaSuccess;
  uint32_t* hist = with_hist ? w.hist : nullptr;
  const long long rows = (long long)B * (((long long)Tk + 7) & ~7ll);
  cudaError_t e;
  if (d == 128)
    e = launch_pdl(score_decode_kernel<128>, dim3(score_grid<128>(rows)), dim3(kScoreThreads), 0, st, q, kmat, B,
                   Tk_max, Tk, q_pos0, kv_len, w.keys, w.ld, hist);
  else
    e = launch_pdl(score_decode_kernel<64>, dim3(score_grid<64>(rows)), dim3(kScoreThreads), 0, st, q, kmat, B,
                   Tk_max, Tk, q_pos0, kv_len, w.keys, w.ld, hist);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_finish(int B, int rows_per_batch, int t0, int Tq, int Tk, int q_pos0,
                          const int32_t* kv_len, int k, const RowWorkspace& w, int mode,
                          const FinishOut& out, cudaStream_t st) {
  const int rows = B * rows_per_batch;
  if (rows <= 0) return cudaSuccess;
  // the longest row of the launch decides the layout: direct rows of at most
  // 2048 candidates take the small one (256 threads, several rows per SM)
  const long long n_max = std::min<long long>(Tk, (long long)q_pos0 + t0 + rows_per_batch);
  auto go = [&](auto kern, size_t smem, int threads) {
    cudaError_t e = ensure_dynamic_smem((const void*)kern, smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3(rows), dim3(threads), smem, st, w, rows_per_batch, t0, Tq, Tk, q_pos0, kv_len, k,
                      out);
  };
  cudaError_t e;
  if (mode == kFinishDirect && n_max <= FinishSmemSmall::kCand)
    e = go(finish_kernel<FinishSmemSmall, kFinThreadsSmall, kFinishDirect>, sizeof(FinishSmemSmall), kFinThreadsSmall);
  else if (mode == kFinishCandRows && n_max <= FinishSmemMed::kBmw * 32)
    e = go(finish_kernel<FinishSmemMed, kFinThreadsSmall, kFinishCandRows>, sizeof(FinishSmemMed), kFinThreadsSmall);
  else if (mode == kFinishDirect)
    e = go(finish_kernel<FinishSmem, kFinThreads, kFinishDirect>, sizeof(FinishSmem), kFinThreads);
  else
    e = go(finish_kernel<FinishSmem, kFinThreads, kFinishCandRows>, sizeof(FinishSmem), kFinThreads);
  return e != cudaSuccess ? e : cudaGetLastError();
}

int finish_mode_for(int Tk_max) {
  // short rows: one CTA holds the whole row; longer rows: slices over many
  // CTAs, the row's last CTA selects
  return Tk_max <= kDirectMaxCand ? kFinishDirect : kFinishSplit;
}

cudaError_t launch_split_topk(int B, int rows_per_batch, int t0, int Tq, int Tk, int q_pos0,
                              const int32_t* kv_len, int k, const RowWorkspace& w, const FinishOut& out,
                              cudaStream_t st) {
  const int rows = B * rows_per_batch;
  if (rows <= 0) return cudaSuccess;
  // slices of a multiple of kSplitSlice positions: about two CTAs per SM over
  // all rows, at most kSplitMaxSlices per row
  const long long n_max =
      std::max<long long>(1, std::min<long long>(Tk, (long long)q_pos0 + t0 + rows_per_batch));
  const long long target = std::max<long long>(1, 2LL * device_sm_count() / rows);
  long long chunk = (n_max + target - 1) / target;
  const long long floor_chunk = (n_max + kSplitMaxSlices - 1) / kSplitMaxSlices;
  chunk = std::max(chunk, floor_chunk);
  chunk = (chunk + kSplitSlice - 1) / kSplitSlice * kSplitSlice;
  const int F = (int)((n_max + chunk - 1) / chunk);
  const size_t smem = sizeof(SplitSmem);
  cudaError_t e = ensure_dynamic_smem((const void*)split_topk_kernel, smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(split_topk_kernel, dim3((unsigned)F, (unsigned)rows), dim3(kSplitThreads), smem, st, w,
                 rows_per_batch, t0, Tq, Tk, q_pos0, kv_len, k, (int)chunk, out);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_hier_gist(const uint16_t* q_route, const uint16_t* meta_key, const uint16_t* gist_key, int B,
                             int d, int n_chunks, int group_size, int k_groups, int k, const FinishOut& out,
                             int32_t* groups_out, cudaStream_t st) {
  if (B <= 0) return cudaSuccess;
  const size_t smem = sizeof(HGistSmem);
  cudaError_t e;
  if (d == 128) {
    if ((e = ensure_dynamic_smem((const void*)hier_gist_kernel<128>, smem)) != cudaSuccess) return e;
    e = launch_pdl(hier_gist_kernel<128>, dim3((unsigned)B), dim3(kHgThreads), smem, st, q_route, meta_key,
                   gist_key, n_chunks, group_size, k_groups, k, out, groups_out);
  } else {
    if ((e = ensure_dynamic_smem((const void*)hier_gist_kernel<64>, smem)) != cudaSuccess) return e;
    e = launch_pdl(hier_gist_kernel<64>, dim3((unsigned)B), dim3(kHgThreads), smem, st, q_route, meta_key,
                   gist_key, n_chunks, group_size, k_groups, k, out, groups_out);
  }
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_index_overlap(const int32_t* a, const int32_t* ca, const int32_t* b, const int32_t* cb, int rows,
                                 int k, int32_t* out, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  const cudaError_t e =
      launch_pdl(index_overlap_kernel, dim3((unsigned)((rows + 7) / 8)), dim3(256), 0, st, a, ca, b, cb, rows, k, out);
  return e != cudaSuccess ? e : cudaGetLastError();
}

int mh_rows_per_launch(int B, int Tq, int Tk_max) {
  // keys (4 B) and candidate pairs (8 B) per position of every row: at most
  // about 1 GiB per launch
  long long cap = (1ll << 30) / (12ll * row_ld(Tk_max) * (B > 0 ? B : 1));
  if (cap > 64) cap = cap / 64 * 64;
  if (cap < 1) cap = 1;
  if (cap > Tq) cap = Tq;
  return (int)cap;
}

cudaError_t launch_score_mh(const uint16_t* q, const float* wts, const uint16_t* kmat, int B, int H, int d,
                            int rows_per_batch, int t0, int Tq, int Tk_max, int Tk, int q_pos0,
                            const int32_t* kv_len, const RowWorkspace& w, bool with_hist, cudaStream_t st) {
  uint32_t* hist = with_hist ? w.hist : nullptr;
  const int rows = B * rows_per_batch;
  if (rows <= 0 || Tk <= 0) return cudaSuccess;
  const long long n_max = std::min<long long>(Tk, (long long)q_pos0 + t0 + rows_per_batch);
  if (n_max <= 0) return cudaSuccess;
  // chunks of a multiple of 256 keys: about two CTAs per SM over all rows
  const long long target = std::max<long long>(1, 2LL * device_sm_count() / rows);
  long long chunk = (n_max + target - 1) / target;
  chunk = std::max<long long>(256, (chunk + 255) / 256 * 256);
  const unsigned gx = (unsigned)((n_max + chunk - 1) / chunk);
  const dim3 grid(gx, (unsigned)rows);
  const int hg = (H + 15) / 16;
  cudaError_t e;
#define SA_MH_LAUNCH(DD, GG)                                                                                  \
  e = launch_pdl(score_mh_kernel<DD, GG>, grid, dim3(kScoreThreads), 0, st, q, wts, kmat, H, rows_per_batch, t0, \
                 Tq, Tk_max, Tk, q_pos0, kv_len, (int)chunk, w.keys, w.ld, hist)
  if (d == 128) {
    if (hg == 1) SA_MH_LAUNCH(128, 1);
    else SA_MH_LAUNCH(128, 2);
  } else {
    if (hg == 1) SA_MH_LAUNCH(64, 1);
    else if (hg == 2) SA_MH_LAUNCH(64, 2);
    else if (hg == 3) SA_MH_LAUNCH(64, 3);
    else SA_MH_LAUNCH(64, 4);
  }
#undef SA_MH_LAUNCH
  return e != cudaSuccess ? e : cudaGetLastError();
}

// Bytes of the fixed, self-cleaning region of one-query workspaces (the
// histograms and tickets of kHistRowsFixed rows) after the error word.
static size_t fixed_region_bytes() {
  return align256((size_t)kHistRowsFixed * kHistStride * 4) + align256((size_t)kHistRowsFixed * 4);
}

// Prefill layout: [error word][the one-query fixed region, left untouched so
// that a workspace can alternate between prefill and decode calls][keys:
// rows x ld][second slab: rows x ld][group maxima: rows x ld2 (16-bit)]
// [bound: rows][run counts: rows x ld/256].  Short batches use only the key
// slab; long ones use both slabs as one [rows][ld] array of (score bits,
// position) pairs for the bounded pass's takes (each scoring CTA's run of a
// row at the run's first column).
size_t prefill_workspace_bytes(int rows, int Tk_max, int k) {
  const long long ld = row_ld(Tk_max);
  const long long ld2 = prefill_groups_ld(Tk_max, k);
  return 256 + fixed_region_bytes() + 2 * align256((size_t)rows * ld * 4) + align256((size_t)rows * ld2 * 2) +
         align256((size_t)rows * 4) + align256((size_t)rows * (ld / 256) * 4);
}

void carve_prefill_workspace(void* ws, int rows, int Tk_max, int k, RowWorkspace* o) {
  char* p = static_cast<char*>(ws);
  o->ld = row_ld(Tk_max);
  o->ld2 = prefill_groups_ld(Tk_max, k);
  o->err = reinterpret_cast<int*>(p);
  p += 256 + fixed_region_bytes();
  o->keys = reinterpret_cast<uint32_t*>(p);
  p += align256((size_t)rows * o->ld * 4);
  o->cand_pos = reinterpret_cast<uint32_t*>(p);
  p += align256((size_t)rows * o->ld * 4);
  o->gmax = reinterpret_cast<uint16_t*>(p);
  p += align256((size_t)rows * o->ld2 * 2);
  o->theta = reinterpret_cast<uint32_t*>(p);
  p += align256((size_t)rows * 4);
  o->tile_cnt = reinterpret_cast<uint32_t*>(p);
}

int prefill_rows_per_launch(int B, int Tq, int Tk_max, int k) {
  // the two [rows][ld] slabs (keys, candidate positions) take at most 1 GiB;
  // the group maxima and per-row words come on top
  (void)k;
  long long cap = (1ll << 30) / (8ll * row_ld(Tk_max) * (B > 0 ? B : 1));
  cap = cap / 128 * 128;
  if (cap < 128) cap = 128;
  if (cap > Tq) cap = Tq;
  return (int)cap;
}

cudaError_t launch_prefill_threshold(int B, int rows_per_batch, int t0, int Tk, int q_pos0,
                                     const int32_t* kv_len, int k, const RowWorkspace& w, cudaStream_t st) {
  const int rows = B * rows_per_batch;
  if (rows <= 0) return cudaSuccess;
  const cudaError_t e = launch_pdl(prefill_threshold_kernel, dim3(rows), dim3(kThrThreads), 0, st, w.gmax, w.ld2,
                                   rows_per_batch, t0, Tk, q_pos0, kv_len, k, w.theta);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace sa
