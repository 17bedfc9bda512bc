// Gathered sparse attention over index-selected K/V rows (sm_100a).
//
// Method: [YOIO] §1.1 Attention(Q,K,V) = softmax(QK^T/sqrt(d_k))V, evaluated
// only over the rows named by the shared index ([YOIO] §2.3 selector;
// [LC] "DSA 与 IndexShare", O(L^2) -> O(Lk)).  Decode follows the split-K
// shape of [SSA] §六: CTAs take slices of the compact index list, the rows of
// one kv head are loaded once for all query heads of its GQA group, and the
// partial (max, sum, output) triples are merged by the log-sum-exp rule.
//
// Both kernels share one tile loop (attn_tiles): 64 gathered rows per tile,
// K and V rows of one kv head (256 contiguous bytes each) gathered with
// 16-byte cp.async into padded shared tiles, two stages so the gather of tile
// i+1 overlaps the math of tile i.  Each of the 4 warps owns 16 rows of a
// tile and runs online softmax on mma.sync m16n8k16 (bf16 in, fp32
// accumulate) with the G query heads of the group as the 16-row M side
// (zero padded), S = Q K^T then O += P V (V through ldmatrix.trans).
//
// attn_prefill_kernel  grid (T, Hkv, B), kv-head-major: one query token x one
//                      kv head per CTA, all of its selected rows.
// attn_decode_kernel   the 16-row tiles of all (sequence, kv head) pairs are
//                      split evenly over the warps of a resident-sized grid;
//                      each warp streams its tiles through a private 3-stage
//                      cp.async ring, writes a partial (m, l, o) where its
//                      range leaves a pair, and the warp whose atomic ticket
//                      completes a pair (never a wait) merges its partials.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

constexpr int kD = 128;        // head_dim
constexpr int kLds = kD + 8;   // padded smem row (elements): 272 bytes
constexpr int kTile = 64;      // gathered rows per tile (16 per warp)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ int clamp_row(int j, int Tk_max) {
  return j < 0 ? 0 : (j >= Tk_max ? Tk_max - 1 : j);
}

// Shared memory of one CTA: Q (16 rows), 2 stages of K and V tiles; the
// stage area is reused for the cross-warp merge.
constexpr size_t kSmemQ = 16 * kLds * 2;
constexpr size_t kSmemStage = (size_t)kTile * kLds * 2;
constexpr size_t kSmemTotal = kSmemQ + 4 * kSmemStage;

struct TileAcc {
  float o[16][4];
  float m[2], l[2];
};

// Gathers tile rows [i0, i0+64) (clipped to `end`) of one kv head into a
// stage: 16 consecutive threads copy the 16 chunks of one 256-byte row, so
// every request covers whole 32-byte sectors.
__device__ __forceinline__ void gather_tile(uint16_t* sK, uint16_t* sV, const uint16_t* __restrict__ kc,
                                            const uint16_t* __restrict__ vc, const int32_t* __restrict__ irow,
                                            int i0, int end, long long head_base, long long row_elems,
                                            int Tk_max) {
  const int c = threadIdx.x & 15;
#pragma unroll
  for (int pass = 0; pass < kTile / 8; ++pass) {
    const int r = (threadIdx.x >> 4) + 8 * pass;
    const int i = i0 + r;
    const bool v = i < end;
    const int j = v ? clamp_row(irow[i], Tk_max) : 0;
    const long long off = head_base + (long long)j * row_elems + c * 8;
    cp_async16(sK + r * kLds + c * 8, kc + off, v);
    cp_async16(sV + r * kLds + c * 8, vc + off, v);
  }
}

// Online-softmax attention of the 16 (padded) query rows in sQ over the
// gathered rows [begin, end) of irow.  Leaves per-warp partials in acc
// (rows gq and gq+8 of the M side for this lane).
__device__ __forceinline__ void attn_tiles(unsigned char* smem, const uint16_t* __restrict__ kc,
                                           const uint16_t* __restrict__ vc,
                                           const int32_t* __restrict__ irow, int begin, int end,
                                           long long head_base, long long row_elems, int Tk_max,
                                           float qscale, TileAcc& acc) {
  uint16_t* sQ = reinterpret_cast<uint16_t*>(smem);
  uint16_t* sK = reinterpret_cast<uint16_t*>(smem + kSmemQ);
  uint16_t* sV = sK + 2 * kTile * kLds;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int tg = lane & 3;
#pragma unroll
  for (int i = 0; i < 16; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc.o[i][e] = 0.f;
  acc.m[0] = acc.m[1] = -INFINITY;
  acc.l[0] = acc.l[1] = 0.f;
  const int ntiles = end > begin ? (end - begin + kTile - 1) / kTile : 0;
  if (ntiles > 0) gather_tile(sK, sV, kc, vc, irow, begin, end, head_base, row_elems, Tk_max);
  cp_async_commit();
  uint32_t qa[8][4];
  for (int it = 0; it < ntiles; ++it) {
    const int stage = it & 1;
    if (it + 1 < ntiles)
      gather_tile(sK + (stage ^ 1) * kTile * kLds, sV + (stage ^ 1) * kTile * kLds, kc, vc, irow,
                  begin + (it + 1) * kTile, end, head_base, row_elems, Tk_max);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (it == 0) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        ldmatrix_x4(qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3],
                    sQ + (lane & 15) * kLds + kk * 16 + (lane >> 4) * 8);
    }
    const uint16_t* tK = sK + (stage * kTile + warp * 16) * kLds;
    const uint16_t* tV = sV + (stage * kTile + warp * 16) * kLds;
    float sc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[nt][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int mtx = lane >> 3;
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4(b0, b1, b2, b3, tK + ((mtx >> 1) * 8 + (lane & 7)) * kLds + kk * 16 + (mtx & 1) * 8);
      mma_bf16_16816(sc[0], qa[kk], b0, b1);
      mma_bf16_16816(sc[1], qa[kk], b2, b3);
    }
    const int rbase = begin + it * kTile + warp * 16;
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int row = rbase + nt * 8 + tg * 2 + (e & 1);
        const float z = row < end ? sc[nt][e] * qscale : -INFINITY;
        sc[nt][e] = z;
        mx[e >> 1] = fmaxf(mx[e >> 1], z);
      }
    float alpha[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float v = mx[hh];
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
      const float mnew = fmaxf(acc.m[hh], v);
      const float muse = mnew == -INFINITY ? 0.f : mnew;
      alpha[hh] = exp2f(acc.m[hh] - muse);
      acc.m[hh] = mnew;
      mx[hh] = muse;
    }
    float rs[2] = {0.f, 0.f};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float pv = exp2f(sc[nt][e] - mx[e >> 1]);
        sc[nt][e] = pv;
        rs[e >> 1] += pv;
      }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float v = rs[hh];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      acc.l[hh] = acc.l[hh] * alpha[hh] + v;
    }
#pragma unroll
    for (int dt = 0; dt < 16; ++dt) {
      acc.o[dt][0] *= alpha[0];
      acc.o[dt][1] *= alpha[0];
      acc.o[dt][2] *= alpha[1];
      acc.o[dt][3] *= alpha[1];
    }
    uint32_t pa[4];
    pa[0] = pack_bf2(sc[0][0], sc[0][1]);
    pa[1] = pack_bf2(sc[0][2], sc[0][3]);
    pa[2] = pack_bf2(sc[1][0], sc[1][1]);
    pa[3] = pack_bf2(sc[1][2], sc[1][3]);
#pragma unroll
    for (int dt = 0; dt < 16; dt += 2) {
      const int mtx = lane >> 3;
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4_trans(b0, b1, b2, b3, tV + ((mtx & 1) * 8 + (lane & 7)) * kLds + (dt + (mtx >> 1)) * 8);
      mma_bf16_16816(acc.o[dt], pa, b0, b1);
      mma_bf16_16816(acc.o[dt + 1], pa, b2, b3);
    }
    __syncthreads();
  }
  cp_async_wait<0>();
  __syncthreads();
}

// Loads the G query heads of one token into sQ (rows >= G zero).
__device__ __forceinline__ void load_q(unsigned char* smem, const uint16_t* __restrict__ qh, int G) {
  uint16_t* sQ = reinterpret_cast<uint16_t*>(smem);
  for (int e = threadIdx.x; e < 16 * 16; e += 128) {
    const int h = e >> 4, c = e & 15;
    const bool v = h < G;
    cp_async16(sQ + h * kLds + c * 8, qh + (v ? h : 0) * kD + c * 8, v);
  }
}

// Writes the 4 warps' partials to smem: mo[4][16][kD], mm[4][16][2].
__device__ __forceinline__ void stash_warps(unsigned char* smem, const TileAcc& acc) {
  float* mo = reinterpret_cast<float*>(smem + kSmemQ);
  float* mm = mo + 4 * 16 * kD;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gq = lane >> 2, tg = lane & 3;
#pragma unroll
  for (int dt = 0; dt < 16; ++dt) {
    const int d0 = dt * 8 + tg * 2;
    *reinterpret_cast<float2*>(mo + (warp * 16 + gq) * kD + d0) = make_float2(acc.o[dt][0], acc.o[dt][1]);
    *reinterpret_cast<float2*>(mo + (warp * 16 + gq + 8) * kD + d0) = make_float2(acc.o[dt][2], acc.o[dt][3]);
  }
  if (tg == 0) {
    mm[(warp * 16 + gq) * 2] = acc.m[0];
    mm[(warp * 16 + gq) * 2 + 1] = acc.l[0];
    mm[(warp * 16 + gq + 8) * 2] = acc.m[1];
    mm[(warp * 16 + gq + 8) * 2 + 1] = acc.l[1];
  }
  __syncthreads();
}

// Merge of the 4 warps for head h and dim d (thread = dim): returns the
// unnormalised sum o, and M, L of the CTA's rows.
__device__ __forceinline__ void merge_warps(const unsigned char* smem, int h, int d, float& M, float& L,
                                            float& o) {
  const float* mo = reinterpret_cast<const float*>(smem + kSmemQ);
  const float* mm = mo + 4 * 16 * kD;
  M = -INFINITY;
#pragma unroll
  for (int w = 0; w < 4; ++w) M = fmaxf(M, mm[(w * 16 + h) * 2]);
  L = 0.f;
  o = 0.f;
  if (M == -INFINITY) return;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const float lw = mm[(w * 16 + h) * 2 + 1];
    if (lw == 0.f) continue;
    const float wt = exp2f(mm[(w * 16 + h) * 2] - M);
    L = fmaf(lw, wt, L);
    o = fmaf(mo[(w * 16 + h) * kD + d], wt, o);
  }
}

// ----------------------------------------------------------------- prefill

__global__ void __launch_bounds__(128)
attn_prefill_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ kc,
                    const uint16_t* __restrict__ vc, const int32_t* __restrict__ idx,
                    const int32_t* __restrict__ count, int T, int Tk_max, int Hq, int Hkv, int k,
                    float qscale, uint16_t* __restrict__ out, float* __restrict__ lse) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int t = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int G = Hq / Hkv;
  const long long tok = (long long)b * T + t;
  int cnt = count[tok];
  cnt = cnt < 0 ? 0 : (cnt > k ? k : cnt);
  load_q(smem, q + (tok * Hq + (long long)g * G) * kD, G);
  TileAcc acc;
  attn_tiles(smem, kc, vc, idx + tok * k, 0, cnt, ((long long)b * Tk_max * Hkv + g) * kD,
             (long long)Hkv * kD, Tk_max, qscale, acc);
  stash_warps(smem, acc);
  const int d = threadIdx.x;
  for (int h = 0; h < G; ++h) {
    float M, L, o;
    merge_warps(smem, h, d, M, L, o);
    out[(tok * Hq + g * G + h) * kD + d] = f2bf(L > 0.f ? o / L : 0.f);
    if (d == 0 && lse != nullptr) lse[tok * Hq + g * G + h] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
  }
}

// ------------------------------------------------------------------ decode
//
// Balanced split of the decode work: the 16-row tiles of every (sequence, kv
// head) pair form one list of T tiles, cut into equal contiguous ranges, one
// per warp of a grid sized to the resident warps.  A warp streams its tiles
// through its own STAGES-deep cp.async ring (no block barrier in the loop)
// and writes a partial (m, l, o) whenever its range leaves a pair; the warp
// whose ticket completes a pair merges that pair's partials.

constexpr int kDecWarps = 4;                 // warps per CTA
constexpr int kDecStages = 3;                // per-warp ring depth
constexpr int kDecTile = 16;                 // rows per warp tile
constexpr size_t kDecStageBytes = (size_t)kDecTile * kLds * 2 * 2;   // K + V
constexpr size_t kDecSmem = (size_t)kDecWarps * kDecStages * kDecStageBytes;

struct DecPlan {
  int pairs, tpp, cmax;
  long long T, W;   // tiles, warps
};

// Warp owning tile t: the largest w with floor(w*T/W) <= t.
__device__ __forceinline__ long long tile_owner(long long t, long long T, long long W) {
  return ((t + 1) * W - 1) / T;
}

__device__ __forceinline__ void dec_gather(uint16_t* st, const uint16_t* __restrict__ kc,
                                           const uint16_t* __restrict__ vc, int jlane, int i0, int end,
                                           long long head_base, long long row_elems, int Tk_max, int lane) {
  const int c = lane & 15;
  uint16_t* sK = st;
  uint16_t* sV = st + kDecTile * kLds;
#pragma unroll
  for (int pass = 0; pass < kDecTile / 2; ++pass) {
    const int r = (lane >> 4) + 2 * pass;
    const int j = __shfl_sync(0xffffffffu, jlane, r);
    const bool v = i0 + r < end;
    const long long off = head_base + (long long)(v ? j : 0) * row_elems + c * 8;
    cp_async16(sK + r * kLds + c * 8, kc + off, v);
    cp_async16(sV + r * kLds + c * 8, vc + off, v);
  }
}

__global__ void __launch_bounds__(kDecWarps * 32)
attn_decode_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ kc,
                   const uint16_t* __restrict__ vc, const int32_t* __restrict__ idx,
                   const int32_t* __restrict__ count, int Tk_max, int Hq, int Hkv, int k, DecPlan pl,
                   float qscale, float* __restrict__ part_o, float* __restrict__ part_ml,
                   unsigned* __restrict__ ticket, uint16_t* __restrict__ out, float* __restrict__ lse) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gq = lane >> 2, tg = lane & 3;
  const int G = Hq / Hkv;
  const long long w = (long long)blockIdx.x * kDecWarps + warp;
  if (w >= pl.W) return;
  uint16_t* ring = reinterpret_cast<uint16_t*>(smem + (size_t)warp * kDecStages * kDecStageBytes);
  const long long lo = w * pl.T / pl.W, hi = (w + 1) * pl.T / pl.W;

  for (long long t = lo; t < hi;) {
    const int p = (int)(t / pl.tpp);
    const long long seg_end = min(hi, (long long)(p + 1) * pl.tpp);
    const int b = p / Hkv, g = p % Hkv;
    int cnt = count[b];
    cnt = cnt < 0 ? 0 : (cnt > k ? k : cnt);
    const int first_tile = (int)(t - (long long)p * pl.tpp);
    const int ntiles = (int)(seg_end - t);
    const int32_t* irow = idx + (long long)b * k;
    const long long head_base = ((long long)b * Tk_max * Hkv + g) * kD;
    const long long row_elems = (long long)Hkv * kD;
    const long long head0 = (long long)b * Hq + (long long)g * G;

    // query fragments of the group's heads (rows >= G are zero)
    uint32_t qa[8][4];
    {
      const uint32_t* qr0 = reinterpret_cast<const uint32_t*>(q + (head0 + gq) * kD);
      const uint32_t* qr1 = reinterpret_cast<const uint32_t*>(q + (head0 + gq + 8) * kD);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int c0 = (kk * 16 + 2 * tg) >> 1, c1 = (kk * 16 + 8 + 2 * tg) >> 1;
        qa[kk][0] = gq < G ? __ldg(qr0 + c0) : 0u;
        qa[kk][1] = gq + 8 < G ? __ldg(qr1 + c0) : 0u;
        qa[kk][2] = gq < G ? __ldg(qr0 + c1) : 0u;
        qa[kk][3] = gq + 8 < G ? __ldg(qr1 + c1) : 0u;
      }
    }
    float o[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[i][e] = 0.f;
    float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};

    // pipeline prologue; the row indices of the tile gathered next are
    // loaded one iteration ahead so no gather waits on an index load
    auto idx_of = [&](int tile) -> int {
      const int i = (first_tile + tile) * kDecTile + (lane & 15);
      return (tile < ntiles && i < cnt) ? clamp_row(irow[i], Tk_max) : 0;
    };
    int jl_next = idx_of(kDecStages - 1);
#pragma unroll
    for (int sIdx = 0; sIdx < kDecStages - 1; ++sIdx) {
      if (sIdx < ntiles) {
        const int i0 = (first_tile + sIdx) * kDecTile;
        dec_gather(ring + sIdx * (kDecStageBytes / 2), kc, vc, idx_of(sIdx), i0, cnt, head_base, row_elems,
                   Tk_max, lane);
      }
      cp_async_commit();
    }
    for (int it = 0; it < ntiles; ++it) {
      const int nxt = it + kDecStages - 1;
      if (nxt < ntiles) {
        const int i0 = (first_tile + nxt) * kDecTile;
        dec_gather(ring + (nxt % kDecStages) * (kDecStageBytes / 2), kc, vc, jl_next, i0, cnt, head_base,
                   row_elems, Tk_max, lane);
      }
      jl_next = idx_of(nxt + 1);
      cp_async_commit();
      cp_async_wait<kDecStages - 1>();
      __syncwarp();
      const uint16_t* tK = ring + (it % kDecStages) * (kDecStageBytes / 2);
      const uint16_t* tV = tK + kDecTile * kLds;
      const int rbase = (first_tile + it) * kDecTile;
      if (rbase < cnt) {
        // S = Q K^T over 8 k-steps, in two independent accumulator chains
        float sc[2][4], sd[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) sc[nt][e] = sd[nt][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 8; kk += 2) {
          const int mtx = lane >> 3;
          uint32_t b0, b1, b2, b3, c0, c1, c2, c3;
          ldmatrix_x4(b0, b1, b2, b3, tK + ((mtx >> 1) * 8 + (lane & 7)) * kLds + kk * 16 + (mtx & 1) * 8);
          ldmatrix_x4(c0, c1, c2, c3, tK + ((mtx >> 1) * 8 + (lane & 7)) * kLds + (kk + 1) * 16 + (mtx & 1) * 8);
          mma_bf16_16816(sc[0], qa[kk], b0, b1);
          mma_bf16_16816(sc[1], qa[kk], b2, b3);
          mma_bf16_16816(sd[0], qa[kk + 1], c0, c1);
          mma_bf16_16816(sd[1], qa[kk + 1], c2, c3);
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) sc[nt][e] += sd[nt][e];
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int row = rbase + nt * 8 + tg * 2 + (e & 1);
            const float z = row < cnt ? sc[nt][e] * qscale : -INFINITY;
            sc[nt][e] = z;
            mx[e >> 1] = fmaxf(mx[e >> 1], z);
          }
        float alpha[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float v = mx[hh];
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
          const float mnew = fmaxf(m_r[hh], v);
          const float muse = mnew == -INFINITY ? 0.f : mnew;
          alpha[hh] = exp2f(m_r[hh] - muse);
          m_r[hh] = mnew;
          mx[hh] = muse;
        }
        float rs[2] = {0.f, 0.f};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float pv = exp2f(sc[nt][e] - mx[e >> 1]);
            sc[nt][e] = pv;
            rs[e >> 1] += pv;
          }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float v = rs[hh];
          v += __shfl_xor_sync(0xffffffffu, v, 1);
          v += __shfl_xor_sync(0xffffffffu, v, 2);
          l_r[hh] = l_r[hh] * alpha[hh] + v;
        }
        if (__any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f)) {  // a row max moved
#pragma unroll
          for (int dt = 0; dt < 16; ++dt) {
            o[dt][0] *= alpha[0];
            o[dt][1] *= alpha[0];
            o[dt][2] *= alpha[1];
            o[dt][3] *= alpha[1];
          }
        }
        uint32_t pa[4];
        pa[0] = pack_bf2(sc[0][0], sc[0][1]);
        pa[1] = pack_bf2(sc[0][2], sc[0][3]);
        pa[2] = pack_bf2(sc[1][0], sc[1][1]);
        pa[3] = pack_bf2(sc[1][2], sc[1][3]);
#pragma unroll
        for (int dt = 0; dt < 16; dt += 2) {
          const int mtx = lane >> 3;
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4_trans(b0, b1, b2, b3, tV + ((mtx & 1) * 8 + (lane & 7)) * kLds + (dt + (mtx >> 1)) * 8);
          mma_bf16_16816(o[dt], pa, b0, b1);
          mma_bf16_16816(o[dt + 1], pa, b2, b3);
        }
      }
      __syncwarp();
    }
    cp_async_wait<0>();
    __syncwarp();

    // ---- hand the segment's result on
    const long long w_first = tile_owner((long long)p * pl.tpp, pl.T, pl.W);
    const long long w_last = tile_owner((long long)(p + 1) * pl.tpp - 1, pl.T, pl.W);
    const int ncontrib = (int)(w_last - w_first + 1);
    if (ncontrib == 1) {
      // this warp owns the whole pair: normalise and write
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int h = gq + 8 * hh;
        if (h < G) {
          const float inv = l_r[hh] > 0.f ? 1.f / l_r[hh] : 0.f;
#pragma unroll
          for (int dt = 0; dt < 16; ++dt)
            *reinterpret_cast<uint32_t*>(out + (head0 + h) * kD + dt * 8 + 2 * tg) =
                pack_bf2(o[dt][2 * hh] * inv, o[dt][2 * hh + 1] * inv);
          if (tg == 0 && lse != nullptr)
            lse[head0 + h] = l_r[hh] > 0.f ? (m_r[hh] + log2f(l_r[hh])) * kLn2 : -INFINITY;
        }
      }
    } else {
      const int j = (int)(w - w_first);
      const long long slot = ((long long)p * pl.cmax + j) * G;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int h = gq + 8 * hh;
        if (h < G) {
#pragma unroll
          for (int dt = 0; dt < 16; ++dt)
            *reinterpret_cast<float2*>(part_o + (slot + h) * kD + dt * 8 + 2 * tg) =
                make_float2(o[dt][2 * hh], o[dt][2 * hh + 1]);
          if (tg == 0) {
            part_ml[(slot + h) * 2] = m_r[hh];
            part_ml[(slot + h) * 2 + 1] = l_r[hh];
          }
        }
      }
      __syncwarp();
      unsigned last = 0;
      if (lane == 0) {
        __threadfence();
        last = atomicAdd(ticket + p, 1u) == (unsigned)(ncontrib - 1);
      }
      last = __shfl_sync(0xffffffffu, last, 0);
      if (last) {
        // warp-parallel merge: lane x holds contributor x's (m, l) per head
        // (at most 32 contributors per pair, see decode_plan)
        __threadfence();
        const long long base = (long long)p * pl.cmax * G;
        float wgt[16], Lh[16], Mh[16];
#pragma unroll
        for (int h = 0; h < 16; ++h) {
          wgt[h] = 0.f;
          Lh[h] = 0.f;
          Mh[h] = -INFINITY;
          if (h < G) {
            const long long sl = base + (long long)lane * G + h;
            const float mx = lane < ncontrib ? __ldcg(part_ml + sl * 2) : -INFINITY;
            const float lx = lane < ncontrib ? __ldcg(part_ml + sl * 2 + 1) : 0.f;
            const float M = warp_max(mx);
            const float wv = (lx > 0.f && M != -INFINITY) ? exp2f(mx - M) : 0.f;
            wgt[h] = wv;
            Lh[h] = warp_sum(lx * wv);
            Mh[h] = M;
          }
        }
        // o: every contributor's partial (zero where it saw no rows) scaled by
        // its weight; no branch in the loop, so the loads overlap
        float acc[16][4];
#pragma unroll
        for (int h = 0; h < 16; ++h) acc[h][0] = acc[h][1] = acc[h][2] = acc[h][3] = 0.f;
        const float* po_base = part_o + base * kD + lane * 4;
#pragma unroll 4
        for (int x = 0; x < ncontrib; ++x) {
#pragma unroll
          for (int h = 0; h < 16; ++h) {
            if (h < G) {
              const float wt = __shfl_sync(0xffffffffu, wgt[h], x);
              const float4 ov = __ldcg(reinterpret_cast<const float4*>(po_base + ((long long)x * G + h) * kD));
              acc[h][0] = fmaf(ov.x, wt, acc[h][0]);
              acc[h][1] = fmaf(ov.y, wt, acc[h][1]);
              acc[h][2] = fmaf(ov.z, wt, acc[h][2]);
              acc[h][3] = fmaf(ov.w, wt, acc[h][3]);
            }
          }
        }
#pragma unroll
        for (int h = 0; h < 16; ++h) {
          if (h < G) {
            const float inv = Lh[h] > 0.f ? 1.f / Lh[h] : 0.f;
            *reinterpret_cast<uint2*>(out + (head0 + h) * kD + lane * 4) =
                make_uint2(pack_bf2(acc[h][0] * inv, acc[h][1] * inv), pack_bf2(acc[h][2] * inv, acc[h][3] * inv));
            if (lane == 0 && lse != nullptr)
              lse[head0 + h] = Lh[h] > 0.f ? (Mh[h] + log2f(Lh[h])) * kLn2 : -INFINITY;
          }
        }
        if (lane == 0) ticket[p] = 0u;  // ready for the next call
      }
    }
    t = seg_end;
  }
}

DecPlan decode_plan(int B, int Hkv, int k) {
  static int sms = 0;
  if (sms == 0) {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    sms = n > 0 ? n : 148;
  }
  DecPlan pl;
  pl.pairs = B * Hkv;
  pl.tpp = (k + kDecTile - 1) / kDecTile;
  pl.T = (long long)pl.pairs * pl.tpp;
  // resident warps (2 CTAs of kDecWarps per SM), but at least 2 tiles per
  // warp and at most 30 warps per pair (the merge keeps one contributor per lane)
  long long W = (long long)sms * 2 * kDecWarps;
  const long long by_tiles = (pl.T + 1) / 2;
  if (W > by_tiles) W = by_tiles;
  if (W > 30ll * pl.pairs) W = 30ll * pl.pairs;
  if (W < 1) W = 1;
  pl.W = W;
  // warps meeting one pair's tile range: at most (tpp-1)*W/T + 2
  pl.cmax = (int)((W + pl.pairs - 1) / pl.pairs) + 2;
  return pl;
}

}  // namespace

static size_t align256a(size_t x) { return (x + 255) & ~size_t(255); }

// The merge tickets sit in a fixed region at the start of the workspace
// (room for kTicketSlots (sequence, kv head) pairs) that holds nothing else,
// so a zero-filled workspace stays valid across calls of any shape: the warp
// that merges a pair returns its ticket to zero.
constexpr int kTicketSlots = 16384;

size_t decode_attn_workspace_bytes(int B, int Hq, int Hkv, int D, int k) {
  (void)D;
  const DecPlan pl = decode_plan(B, Hkv, k);
  const int G = Hq / Hkv;
  const size_t tk = (size_t)kTicketSlots * 4;
  const size_t po = align256a((size_t)pl.pairs * pl.cmax * G * kD * 4);
  const size_t pml = align256a((size_t)pl.pairs * pl.cmax * G * 2 * 4);
  return tk + po + pml;
}

cudaError_t launch_attn_decode(const uint16_t* q, const uint16_t* kc, const uint16_t* vc,
                               const int32_t* idx, const int32_t* count, int B, int Tk_max, int Hq,
                               int Hkv, int k, float scale, uint16_t* out, float* lse, void* ws,
                               cudaStream_t st) {
  if (B <= 0) return cudaSuccess;
  const DecPlan pl = decode_plan(B, Hkv, k);
  const int G = Hq / Hkv;
  char* p = static_cast<char*>(ws);
  unsigned* ticket = reinterpret_cast<unsigned*>(p);
  p += (size_t)kTicketSlots * 4;
  float* po = reinterpret_cast<float*>(p);
  p += align256a((size_t)pl.pairs * pl.cmax * G * kD * 4);
  float* pml = reinterpret_cast<float*>(p);
  cudaError_t e = ensure_dynamic_smem((const void*)attn_decode_kernel, kDecSmem);
  if (e != cudaSuccess) return e;
  const int grid = (int)((pl.W + kDecWarps - 1) / kDecWarps);
  attn_decode_kernel<<<grid, kDecWarps * 32, kDecSmem, st>>>(q, kc, vc, idx, count, Tk_max, Hq, Hkv, k, pl,
                                                            scale * kLog2e, po, pml, ticket, out, lse);
  return cudaGetLastError();
}

cudaError_t launch_attn_prefill(const uint16_t* q, const uint16_t* kc, const uint16_t* vc,
                                const int32_t* idx, const int32_t* count, int B, int T, int Tk_max,
                                int Hq, int Hkv, int k, float scale, uint16_t* out, float* lse,
                                cudaStream_t st) {
  if (B <= 0 || T <= 0) return cudaSuccess;
  cudaError_t e = ensure_dynamic_smem((const void*)attn_prefill_kernel, kSmemTotal);
  if (e != cudaSuccess) return e;
  dim3 grid(T, Hkv, B);
  attn_prefill_kernel<<<grid, 128, kSmemTotal, st>>>(q, kc, vc, idx, count, T, Tk_max, Hq, Hkv, k,
                                                     scale * kLog2e, out, lse);
  return cudaGetLastError();
}

}  // namespace sa
