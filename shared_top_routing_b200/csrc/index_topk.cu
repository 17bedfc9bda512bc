// Indexer scoring and exact per-query top-k (sm_100a).
//
// Method: [LC] "长上下文：稀疏注意力 / DSA / IndexShare", section "DSA 与
// IndexShare" -- a light indexer scores every history token and each query
// keeps its top-k; [YOIO] §2.3 -- the indexer outputs each query's top-k
// token indices.  Selection rule: largest scores, equal scores by lower
// position, emitted in ascending position order.
//
// Kernels
//   score_decode_kernel   one query per sequence; streams the indexer-key
//                         cache with coalesced 16-byte loads (d/8 lanes per
//                         row), writes order-preserving 32-bit score keys and
//                         a 4096-bin histogram of each key's top 12 bits.
//   collect_kernel        finds, from the histogram, the bin holding the
//                         k-th largest key and appends every key in that bin
//                         or above to a per-row candidate list (warp-
//                         aggregated atomics; order of appends is irrelevant).
//   finish_kernel         one CTA per row: exact radix select (8-bit digits,
//                         warp-aggregated shared-memory histograms) of the
//                         k-th key, then of the tie positions, then emission
//                         in ascending position order (ordered block
//                         compaction in direct mode, bitonic sort of the <=k
//                         chosen candidates in candidate mode).  Also expands
//                         chosen gist chunks into their cache rows.
//   score_prefill_kernel  causal Q_idx K_idx^T tile product (tensor cores,
//                         bf16 in, fp32 accumulate) writing score keys of one
//                         block of query rows into a slab for finish_kernel.
#include <cuda_runtime.h>
#include <stdint.h>

#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

constexpr int kScoreThreads = 256;
constexpr int kFinThreads = 1024;

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

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// ------------------------------------------------------------------ scoring

template <int D>
__global__ void __launch_bounds__(kScoreThreads)
score_decode_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ kmat, int Tk_max,
                    int Tk, int q_pos0, const int32_t* __restrict__ kv_len,
                    uint32_t* __restrict__ keys, long long ld, uint32_t* __restrict__ hist,
                    int chunk) {
  constexpr int LPR = D / 8;        // lanes per row, 16 bytes each
  constexpr int RPW = 32 / LPR;     // rows per warp load
  constexpr int UNROLL = 8;
  constexpr int WARPS = kScoreThreads / 32;
  __shared__ uint32_t sh[kHistBins];

  const int b = blockIdx.y;
  const int n = n_cand(q_pos0, 0, row_len(kv_len, b, Tk));
  const int r0 = blockIdx.x * chunk;
  if (r0 >= n) return;
  const int r1 = min(r0 + chunk, n);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int sub = lane / LPR, slot = lane % LPR;

  if (hist != nullptr) {
    for (int i = tid; i < kHistBins; i += kScoreThreads) sh[i] = 0;
    __syncthreads();
  }
  float qf[8];
  {
    uint4 qv = *reinterpret_cast<const uint4*>(q + (long long)b * D + slot * 8);
    qf[0] = bf_lo(qv.x); qf[1] = bf_hi(qv.x); qf[2] = bf_lo(qv.y); qf[3] = bf_hi(qv.y);
    qf[4] = bf_lo(qv.z); qf[5] = bf_hi(qv.z); qf[6] = bf_lo(qv.w); qf[7] = bf_hi(qv.w);
  }
  const uint4* kb = reinterpret_cast<const uint4*>(kmat + (long long)b * Tk_max * D);
  uint32_t* kout = keys + (long long)b * ld;

  for (int base = r0 + warp * RPW * UNROLL; base < r1; base += WARPS * RPW * UNROLL) {
    uint4 v[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      int row = base + u * RPW + sub;
      v[u] = row < r1 ? __ldg(kb + (long long)row * LPR + slot) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      float s = dot8(v[u], qf);
#pragma unroll
      for (int o = LPR / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      int row = base + u * RPW + sub;
      if (slot == 0 && row < r1) {
        uint32_t key = score_key(s);
        kout[row] = key;
        if (hist != nullptr) atomicAdd(&sh[key >> (32 - kHistBits)], 1u);
      }
    }
  }
  if (hist != nullptr) {
    __syncthreads();
    uint32_t* hg = hist + (long long)b * kHistBins;
    for (int i = tid; i < kHistBins; i += kScoreThreads) {
      uint32_t c = sh[i];
      if (c) atomicAdd(hg + i, c);
    }
  }
}

// ------------------------------------------------------------------ collect

// Exclusive prefix sum over the 256 threads of a block; returns the total.
__device__ __forceinline__ uint32_t block_scan_256(uint32_t v, uint32_t* s_warp, uint32_t& excl) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  uint32_t wsum = 0, total = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    uint32_t c = s_warp[w];
    if (w < warp) wsum += c;
    total += c;
  }
  excl = wsum + x - v;
  return total;
}

__global__ void __launch_bounds__(256)
collect_kernel(const uint32_t* __restrict__ keys, long long ld, const uint32_t* __restrict__ hist,
               int Tk, int q_pos0, const int32_t* __restrict__ kv_len, int k, int chunk,
               uint32_t* __restrict__ cand_cnt, uint32_t* __restrict__ cand_key,
               uint32_t* __restrict__ cand_pos) {
  __shared__ uint32_t s_warp[8];
  __shared__ uint32_t s_bin;
  const int b = blockIdx.y;
  const int n = n_cand(q_pos0, 0, row_len(kv_len, b, Tk));
  const int r0 = blockIdx.x * chunk;
  if (r0 >= n) return;
  const int r1 = min(r0 + chunk, n);
  const uint32_t K = (uint32_t)min(k, n);
  const int tid = threadIdx.x, lane = tid & 31;

  // Bin of the K-th largest key: thread i owns the 16 bins counted from the top.
  const uint32_t* h = hist + (long long)b * kHistBins;
  constexpr int PER = kHistBins / 256;
  uint32_t hv[PER];
  uint32_t loc = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    hv[j] = h[kHistBins - 1 - (tid * PER + j)];
    loc += hv[j];
  }
  uint32_t excl;
  block_scan_256(loc, s_warp, excl);
  if (excl < K && K <= excl + loc) {
    uint32_t cum = excl;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      if (cum + hv[j] >= K) { s_bin = kHistBins - 1 - (tid * PER + j); break; }
      cum += hv[j];
    }
  }
  __syncthreads();
  const uint32_t bin = s_bin;

  const uint32_t* row = keys + (long long)b * ld;
  uint32_t* ck = cand_key + (long long)b * kCandCap;
  uint32_t* cp = cand_pos + (long long)b * kCandCap;
  for (int i0 = r0; i0 < r1; i0 += 256) {
    int i = i0 + tid;
    uint32_t key = i < r1 ? row[i] : 0u;
    bool take = i < r1 && (key >> (32 - kHistBits)) >= bin;
    unsigned m = __ballot_sync(0xffffffffu, take);
    if (m) {
      int leader = __ffs(m) - 1;
      uint32_t base = 0;
      if (lane == leader) base = atomicAdd(cand_cnt + b, (uint32_t)__popc(m));
      base = __shfl_sync(0xffffffffu, base, leader);
      if (take) {
        uint32_t s = base + __popc(m & lanemask_lt());
        if (s < (uint32_t)kCandCap) { ck[s] = key; cp[s] = (uint32_t)i; }
      }
    }
  }
}

// ------------------------------------------------------------------- finish

struct FinishSmem {
  uint32_t hist[256];
  uint32_t wcnt[32];
  uint32_t sel_pos[kMaxK];
  uint32_t sel_key[kMaxK];
  uint32_t digit, above, bnd_count, total, nsel;
};

// Adds 1 to hist[digit] for every active lane, aggregated over equal digits.
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t digit, bool active) {
  unsigned act = __ballot_sync(0xffffffffu, active);
  if (!active) return;
  unsigned peers = __match_any_sync(act, digit);
  if ((int)(threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(hist + digit, (uint32_t)__popc(peers));
}

// Warp 0 locates the digit holding the kk-th element, searching from the
// top bin down (desc) or the bottom bin up (asc).  Writes digit and the
// count strictly before it in search order.
__device__ __forceinline__ void find_digit(FinishSmem& s, uint32_t kk, bool desc) {
  if (threadIdx.x >= 32) return;
  const int lane = threadIdx.x;
  uint32_t c[8], loc = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    int bin = desc ? 255 - (lane * 8 + j) : lane * 8 + j;
    c[j] = s.hist[bin];
    loc += c[j];
  }
  uint32_t x = loc;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  uint32_t excl = x - loc;
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

// Item accessor: candidate lists (explicit positions) or a whole row of keys.
struct Items {
  const uint32_t* key;
  const uint32_t* pos;  // null: position = index
  int n;
  __device__ __forceinline__ uint32_t k(int i) const { return key[i]; }
  __device__ __forceinline__ uint32_t p(int i) const { return pos ? pos[i] : (uint32_t)i; }
};

// Exact selection of the K largest keys (ties by lower position) among `it`.
// Leaves in smem: masked-key threshold (prefix under pmask) and, for the
// boundary set, the largest selected position (pmax).
__device__ void select_threshold(FinishSmem& s, const Items& it, uint32_t K, uint32_t& prefix,
                                 uint32_t& pmask, uint32_t& pmax) {
  const int tid = threadIdx.x;
  prefix = 0;
  pmask = 0;
  uint32_t kk = K;
  uint32_t bnd = (uint32_t)it.n;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kFinThreads) s.hist[i] = 0;
    __syncthreads();
    for (int i0 = 0; i0 < it.n; i0 += kFinThreads) {
      int i = i0 + tid;
      uint32_t key = i < it.n ? it.k(i) : 0u;
      bool act = i < it.n && (key & pmask) == prefix;
      hist_add(s.hist, (key >> shift) & 255u, act);
    }
    __syncthreads();
    find_digit(s, kk, true);
    __syncthreads();
    kk -= s.above;
    prefix |= s.digit << shift;
    pmask |= 255u << shift;
    bnd = s.bnd_count;
    __syncthreads();
    if (bnd == kk) break;  // every item of the boundary prefix is selected
  }
  pmax = 0xFFFFFFFFu;
  if (bnd == kk) return;
  // Exact key ties: keep the kk lowest positions among key == prefix.
  uint32_t pp = 0, pm = 0;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kFinThreads) s.hist[i] = 0;
    __syncthreads();
    for (int i0 = 0; i0 < it.n; i0 += kFinThreads) {
      int i = i0 + tid;
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
    pm |= 255u << shift;
    uint32_t c = s.bnd_count;
    __syncthreads();
    if (c == kk) {  // take every tie whose position prefix is <= pp
      pmax = pp | ~pm;
      return;
    }
  }
  pmax = pp;
}

__device__ __forceinline__ bool is_selected(uint32_t key, uint32_t pos, uint32_t prefix,
                                            uint32_t pmask, uint32_t pmax) {
  uint32_t m = key & pmask;
  return m > prefix || (m == prefix && pos <= pmax);
}

__global__ void __launch_bounds__(kFinThreads)
finish_kernel(RowWorkspace w, bool candidates, int rows_per_batch, int t0, int Tq, int Tk,
              int q_pos0, const int32_t* __restrict__ kv_len, int k, FinishOut out) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  FinishSmem& s = *reinterpret_cast<FinishSmem*>(smem_raw);
  const int r = blockIdx.x;
  const int b = r / rows_per_batch;
  const int t = t0 + r % rows_per_batch;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = n_cand(q_pos0, t, row_len(kv_len, b, Tk));
  const uint32_t K = (uint32_t)min(k, n);

  Items it;
  bool direct = true;
  if (candidates) {
    uint32_t m = w.cand_cnt[r];
    if (m <= (uint32_t)kCandCap) {
      it.key = w.cand_key + (long long)r * kCandCap;
      it.pos = w.cand_pos + (long long)r * kCandCap;
      it.n = (int)m;
      direct = false;
    }
  }
  if (direct) {
    it.key = w.keys + (long long)r * w.ld;
    it.pos = nullptr;
    it.n = n;
  }

  uint32_t prefix = 0, pmask = 0, pmax = 0;
  if (K > 0) select_threshold(s, it, K, prefix, pmask, pmax);

  // Emit the chosen (position, key) pairs into shared memory.
  if (tid == 0) { s.total = 0; s.nsel = 0; }
  __syncthreads();
  if (K > 0) {
    if (direct) {
      // Items are in position order: ordered block compaction.
      for (int i0 = 0; i0 < it.n; i0 += kFinThreads) {
        int i = i0 + tid;
        uint32_t key = i < it.n ? it.k(i) : 0u;
        bool sel = i < it.n && is_selected(key, (uint32_t)i, prefix, pmask, pmax);
        unsigned m = __ballot_sync(0xffffffffu, sel);
        if (lane == 0) s.wcnt[warp] = __popc(m);
        __syncthreads();
        if (warp == 0) {
          uint32_t c = s.wcnt[lane], x = c;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
          }
          s.wcnt[lane] = x - c;
          if (lane == 31) s.nsel = x;
        }
        __syncthreads();
        if (sel) {
          uint32_t o = s.total + s.wcnt[warp] + __popc(m & lanemask_lt());
          if (o < (uint32_t)kMaxK) { s.sel_pos[o] = (uint32_t)i; s.sel_key[o] = key; }
        }
        __syncthreads();
        if (tid == 0) s.total += s.nsel;
        __syncthreads();
        if (s.total >= K) break;
      }
    } else {
      for (int i0 = 0; i0 < it.n; i0 += kFinThreads) {
        int i = i0 + tid;
        bool sel = false;
        uint32_t key = 0, pos = 0;
        if (i < it.n) {
          key = it.k(i);
          pos = it.p(i);
          sel = is_selected(key, pos, prefix, pmask, pmax);
        }
        if (sel) {
          uint32_t o = atomicAdd(&s.total, 1u);
          if (o < (uint32_t)kMaxK) { s.sel_pos[o] = pos; s.sel_key[o] = key; }
        }
      }
      __syncthreads();
      // Bitonic sort of the K chosen pairs by position.
      int P = 1;
      while (P < (int)K) P <<= 1;
      for (int i = (int)K + tid; i < P; i += kFinThreads) { s.sel_pos[i] = 0xFFFFFFFFu; s.sel_key[i] = 0; }
      __syncthreads();
      for (int size = 2; size <= P; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
          for (int i = tid; i < (P >> 1); i += kFinThreads) {
            int lo = 2 * i - (i & (stride - 1));
            int hi = lo + stride;
            bool asc = (lo & size) == 0;
            uint32_t a = s.sel_pos[lo], c = s.sel_pos[hi];
            if ((a > c) == asc) {
              s.sel_pos[lo] = c; s.sel_pos[hi] = a;
              uint32_t ka = s.sel_key[lo]; s.sel_key[lo] = s.sel_key[hi]; s.sel_key[hi] = ka;
            }
          }
          __syncthreads();
        }
      }
    }
  }
  __syncthreads();

  if (out.rows == nullptr) {
    const long long o = ((long long)b * Tq + t) * k;
    for (int i = tid; i < k; i += kFinThreads) {
      bool v = i < (int)K;
      out.idx[o + i] = v ? (int32_t)s.sel_pos[i] : -1;
      if (out.score) out.score[o + i] = v ? key_score(s.sel_key[i]) : __int_as_float(0xff800000);
    }
    if (tid == 0) out.count[(long long)b * Tq + t] = (int32_t)K;
  } else {
    const int stride = out.chunk_len + 1;
    int p = out.partial_len ? out.partial_len[b] : 0;
    p = p < 0 ? 0 : (p > out.chunk_len ? out.chunk_len : p);
    const int unfolded = (int)K * stride;
    const int total = unfolded + p;
    int32_t* rows = out.rows + (long long)b * out.rows_stride;
    for (int i = tid; i < out.rows_stride; i += kFinThreads) {
      int32_t v = -1;
      if (i < unfolded) v = (int32_t)s.sel_pos[i / stride] * stride + i % stride;
      else if (i < total) v = out.n_chunks * stride + (i - unfolded);
      rows[i] = v;
    }
    if (out.chunks) {
      for (int i = tid; i < k; i += kFinThreads)
        out.chunks[(long long)b * k + i] = i < (int)K ? (int32_t)s.sel_pos[i] : -1;
    }
    if (tid == 0) out.count[b] = total;
  }
}

// ------------------------------------------------------------ prefill GEMM

// Causal score tile: 128 query rows x 128 key columns, 8 warps (4 x 2), each
// warp 32 x 64, mma.sync m16n8k16 bf16 -> fp32.
template <int D>
__global__ void __launch_bounds__(256)
score_prefill_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ kmat, int Tq,
                     int Tk_max, int Tk, int q_pos0, const int32_t* __restrict__ kv_len, int t0,
                     int rows, uint32_t* __restrict__ keys, long long ld) {
  constexpr int LDS = D + 8;  // padded row (elements): 16-byte skew per row
  extern __shared__ __align__(16) uint16_t sm[];
  uint16_t* sq = sm;
  uint16_t* sk = sm + 128 * LDS;
  const int b = blockIdx.z;
  const int len = row_len(kv_len, b, Tk);
  const int tr0 = t0 + blockIdx.y * 128;          // first query row of the tile
  const int c0 = blockIdx.x * 128;                // first key column
  const int t_last = min(tr0 + 127, t0 + rows - 1);
  if (tr0 >= t0 + rows) return;
  if ((long long)c0 > (long long)q_pos0 + t_last || c0 >= len) return;  // above the diagonal
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  constexpr int CPR = D / 8;  // 16-byte chunks per row
  for (int i = tid; i < 128 * CPR; i += 256) {
    int rr = i / CPR, cc = i % CPR;
    int tq = tr0 + rr;
    bool vq = tq < t0 + rows && tq < Tq;
    cp_async16(sq + rr * LDS + cc * 8, q + (((long long)b * Tq + (vq ? tq : 0)) * D + cc * 8), vq);
    int j = c0 + rr;
    bool vk = j < len;
    cp_async16(sk + rr * LDS + cc * 8, kmat + (((long long)b * Tk_max + (vk ? j : 0)) * D + cc * 8),
               vk);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();

  const int wm = warp >> 1, wn = warp & 1;  // warp tile: rows wm*32, cols wn*64
  float acc[2][8][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;

#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    uint32_t a[2][4];
#pragma unroll
    for (int mi = 0; mi < 2; ++mi) {
      int mrow = wm * 32 + mi * 16 + (lane & 15);
      int kcol = kk * 16 + (lane >> 4) * 8;
      ldmatrix_x4(a[mi][0], a[mi][1], a[mi][2], a[mi][3], sq + mrow * LDS + kcol);
    }
#pragma unroll
    for (int nj = 0; nj < 8; nj += 2) {
      // four 8x8 matrices: (n-tile nj, k lo), (nj, k hi), (nj+1, k lo), (nj+1, k hi)
      int mtx = lane >> 3;
      int nrow = wn * 64 + (nj + (mtx >> 1)) * 8 + (lane & 7);
      int kcol = kk * 16 + (mtx & 1) * 8;
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4(b0, b1, b2, b3, sk + nrow * LDS + kcol);
#pragma unroll
      for (int mi = 0; mi < 2; ++mi) {
        mma_bf16_16816(acc[mi][nj], a[mi], b0, b1);
        mma_bf16_16816(acc[mi][nj + 1], a[mi], b2, b3);
      }
    }
  }

  // Epilogue: keys of causal, in-range entries.
  const int g = lane >> 2, tg = lane & 3;
#pragma unroll
  for (int mi = 0; mi < 2; ++mi) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      int tq = tr0 + wm * 32 + mi * 16 + g + half * 8;
      if (tq >= t0 + rows || tq >= Tq) continue;
      int lim = n_cand(q_pos0, tq, len);  // columns < lim are candidates
      uint32_t* krow = keys + ((long long)b * rows + (tq - t0)) * ld;
#pragma unroll
      for (int nj = 0; nj < 8; ++nj) {
        int c = c0 + wn * 64 + nj * 8 + tg * 2;
        float s0 = acc[mi][nj][half * 2 + 0], s1 = acc[mi][nj][half * 2 + 1];
        if (c + 1 < lim) {
          *reinterpret_cast<uint2*>(krow + c) = make_uint2(score_key(s0), score_key(s1));
        } else if (c < lim) {
          krow[c] = score_key(s0);
        }
      }
    }
  }
}

}  // namespace

// ------------------------------------------------------------------ host side

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

size_t row_workspace_bytes(int rows, int Tk_max, bool with_candidates) {
  long long ld = ((long long)Tk_max + 63) / 64 * 64;
  size_t bytes = 0;
  if (with_candidates) {
    bytes += align256((size_t)rows * kHistBins * 4);
    bytes += align256((size_t)rows * 4);
  }
  bytes += align256((size_t)rows * ld * 4);
  if (with_candidates) bytes += 2 * align256((size_t)rows * kCandCap * 4);
  return bytes;
}

void carve_row_workspace(void* ws, int rows, int Tk_max, bool with_candidates, RowWorkspace* o) {
  char* p = static_cast<char*>(ws);
  o->ld = ((long long)Tk_max + 63) / 64 * 64;
  if (with_candidates) {
    o->hist = reinterpret_cast<uint32_t*>(p);
    p += align256((size_t)rows * kHistBins * 4);
    o->cand_cnt = reinterpret_cast<uint32_t*>(p);
    p += align256((size_t)rows * 4);
  }
  o->keys = reinterpret_cast<uint32_t*>(p);
  p += align256((size_t)rows * o->ld * 4);
  if (with_candidates) {
    o->cand_key = reinterpret_cast<uint32_t*>(p);
    p += align256((size_t)rows * kCandCap * 4);
    o->cand_pos = reinterpret_cast<uint32_t*>(p);
  }
}

cudaError_t launch_score_decode(const uint16_t* q, const uint16_t* kmat, int B, int d, int Tk_max,
                                int Tk, int q_pos0, const int32_t* kv_len, const RowWorkspace& w,
                                bool with_hist, cudaStream_t st) {
  if (Tk <= 0 || B <= 0) return cudaSuccess;
  const int chunk = (256 * 1024) / (d * 2);  // about 256 KB of keys per CTA
  dim3 grid((Tk + chunk - 1) / chunk, B);
  uint32_t* hist = with_hist ? w.hist : nullptr;
  if (d == 128)
    score_decode_kernel<128><<<grid, kScoreThreads, 0, st>>>(q, kmat, Tk_max, Tk, q_pos0, kv_len,
                                                             w.keys, w.ld, hist, chunk);
  else
    score_decode_kernel<64><<<grid, kScoreThreads, 0, st>>>(q, kmat, Tk_max, Tk, q_pos0, kv_len,
                                                            w.keys, w.ld, hist, chunk);
  return cudaGetLastError();
}

cudaError_t launch_collect(int B, int Tk, int q_pos0, const int32_t* kv_len, int k,
                           const RowWorkspace& w, cudaStream_t st) {
  if (Tk <= 0 || B <= 0) return cudaSuccess;
  const int chunk = 8192;
  dim3 grid((Tk + chunk - 1) / chunk, B);
  collect_kernel<<<grid, 256, 0, st>>>(w.keys, w.ld, w.hist, Tk, q_pos0, kv_len, k, chunk,
                                       w.cand_cnt, w.cand_key, w.cand_pos);
  return cudaGetLastError();
}

cudaError_t launch_finish(int B, int rows_per_batch, int t0, int Tq, int Tk, int q_pos0,
                          const int32_t* kv_len, int k, const RowWorkspace& w, bool candidates,
                          const FinishOut& out, cudaStream_t st) {
  const int rows = B * rows_per_batch;
  if (rows <= 0) return cudaSuccess;
  const size_t smem = sizeof(FinishSmem);
  cudaError_t e = ensure_dynamic_smem((const void*)finish_kernel, smem);
  if (e != cudaSuccess) return e;
  finish_kernel<<<rows, kFinThreads, smem, st>>>(w, candidates, rows_per_batch, t0, Tq, Tk, q_pos0,
                                                 kv_len, k, out);
  return cudaGetLastError();
}

int prefill_rows_per_launch(int B, int Tq, int Tk_max) {
  // Key slab of at most 512 MiB: rows * B * ld * 4 bytes.
  long long ld = ((long long)Tk_max + 63) / 64 * 64;
  long long cap = (512ll << 20) / (4ll * ld * (B > 0 ? B : 1));
  cap = cap / 128 * 128;
  if (cap < 128) cap = 128;
  if (cap > Tq) cap = Tq;
  return (int)cap;
}

cudaError_t launch_score_prefill(const uint16_t* q, const uint16_t* kmat, int B, int Tq, int d,
                                 int Tk_max, int Tk, int q_pos0, const int32_t* kv_len, int t0,
                                 int rows, const RowWorkspace& w, cudaStream_t st) {
  if (rows <= 0 || Tk <= 0) return cudaSuccess;
  long long last = (long long)q_pos0 + t0 + rows;  // columns needed: < min(Tk, last)
  int ncols = (int)(last < Tk ? (last > 0 ? last : 0) : Tk);
  if (ncols <= 0) return cudaSuccess;
  dim3 grid((ncols + 127) / 128, (rows + 127) / 128, B);
  if (d == 128) {
    size_t smem = 2 * 128 * (128 + 8) * 2;
    cudaError_t e = ensure_dynamic_smem((const void*)score_prefill_kernel<128>, smem);
    if (e != cudaSuccess) return e;
    score_prefill_kernel<128><<<grid, 256, smem, st>>>(q, kmat, Tq, Tk_max, Tk, q_pos0, kv_len, t0,
                                                       rows, w.keys, w.ld);
  } else {
    size_t smem = 2 * 128 * (64 + 8) * 2;
    score_prefill_kernel<64><<<grid, 256, smem, st>>>(q, kmat, Tq, Tk_max, Tk, q_pos0, kv_len, t0,
                                                      rows, w.keys, w.ld);
  }
  return cudaGetLastError();
}

}  // namespace sa
