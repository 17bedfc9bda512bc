// Gathered sparse attention over index-selected K/V rows (sm_100a).
//
// Method: [YOIO] §1.1 Attention(Q,K,V) = softmax(QK^T/sqrt(d_k))V, evaluated
// only over the rows named by the shared index ([YOIO] §2.3 selector;
// [LC] "DSA 与 IndexShare", O(L^2) -> O(Lk)).  Decode follows the split-K
// shape of [SSA] §六: CTAs take slices of the compact index list, the rows of
// one kv head are loaded once for all query heads of its GQA group, and the
// partial (max, sum, output) triples are merged by the log-sum-exp rule.
//
// Both paths run online softmax on mma.sync m16n8k16 (bf16 in, fp32
// accumulate) with the G query heads of a kv head as the 16-row M side (zero
// padded): S = Q K^T, then O += P V with V through ldmatrix.trans.
//
// attn_decode_split_kernel / attn_decode_merge_kernel  one query per
//     sequence: the tiles of all (sequence, head block) pairs are cut evenly
//     over one CTA per SM (bulk copies per row run), partials are folded by
//     the merge kernel.
// attn_prefill_kernel  one query token x one kv head per CTA, grid (T, Hkv,
//     B): the token's selected rows of that head (256 bytes each) in 64-row
//     tiles gathered with 16-byte cp.async by all four warps, two stages, the
//     four warps' partials merged in shared memory at the end.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "../../include/sa.h"
#include "sa_common.cuh"
#include "sa_internal.h"
#include "tc_common.cuh"

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

#ifdef SA_DEBUG
// Debug builds record the first violation (code, two details) and count
// them all; nothing traps, and the access is clamped as in release builds.
__device__ int g_dbg[4];
__device__ __noinline__ void dbg_note(int code, int a, int b) {
  if (atomicCAS(&g_dbg[0], 0, code) == 0) {
    g_dbg[1] = a;
    g_dbg[2] = b;
  }
  atomicAdd(&g_dbg[3], 1);
}
#endif

// A gathered row index: checked against [0, Tk_max) in debug builds (site =
// the debug record code), clamped into range in every build.
__device__ __forceinline__ int checked_row(int j, int Tk_max, int site) {
#ifdef SA_DEBUG
  if (j < 0 || j >= Tk_max) dbg_note(site, j, Tk_max);
#else
  (void)site;
#endif
  return clamp_row(j, Tk_max);
}

// Shared memory of one CTA: Q (16 rows), kPfStages stages of K and V tiles;
// the stage area is reused for the cross-warp merge.
constexpr int kPfStages = 2;
constexpr int kRowsPerThread = kTile / 8;   // gathered rows per thread and tile
constexpr size_t kSmemQ = 16 * kLds * 2;
constexpr size_t kSmemStage = (size_t)kTile * kLds * 2;
constexpr size_t kSmemTotal = kSmemQ + 2 * kPfStages * kSmemStage;

struct TileAcc {
  float o[16][4];
  float m[2], l[2];
};

// Thread t gathers rows (t >> 4) + 8 p, p < kRowsPerThread, of a tile: the
// row indices of tile rows [i0, i0+64) (clipped to `end`) it copies.  They
// are loaded one tile ahead of the copies, so the copies never wait on an
// index load.
__device__ __forceinline__ void load_tile_rows(int (&j)[kRowsPerThread], const int32_t* __restrict__ irow, int i0,
                                               int end) {
#pragma unroll
  for (int p = 0; p < kRowsPerThread; ++p) {
    const int i = i0 + (threadIdx.x >> 4) + 8 * p;
    j[p] = i < end ? __ldg(irow + i) : 0;
  }
}

// Gathers tile rows [i0, i0+64) (clipped to `end`) of one kv head into a
// stage: 16 consecutive threads copy the 16 chunks of one 256-byte row, so
// every request covers whole 32-byte sectors.
__device__ __forceinline__ void gather_tile(uint16_t* sK, uint16_t* sV, const uint16_t* __restrict__ kc,
                                            const uint16_t* __restrict__ vc, const int (&j)[kRowsPerThread],
                                            int i0, int end, long long head_base, long long row_elems,
                                            int Tk_max) {
  const int c = threadIdx.x & 15;
#pragma unroll
  for (int p = 0; p < kRowsPerThread; ++p) {
    const int r = (threadIdx.x >> 4) + 8 * p;
    const bool v = i0 + r < end;
    const int row = v ? checked_row(j[p], Tk_max, kDbgPrefillIndex) : 0;
    const long long off = head_base + (long long)row * row_elems + c * 8;
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
  uint16_t* sV = sK + kPfStages * kTile * kLds;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int tg = lane & 3;
#pragma unroll
  for (int i = 0; i < 16; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc.o[i][e] = 0.f;
  acc.m[0] = acc.m[1] = -INFINITY;
  acc.l[0] = acc.l[1] = 0.f;
  const int ntiles = end > begin ? (end - begin + kTile - 1) / kTile : 0;
  // ring of kPfStages stages: tiles it+1 .. it+kPfStages-1 are in flight
  // while tile it is consumed, and the indices of the tile after them sit in
  // registers
  int jn[kRowsPerThread];
#pragma unroll
  for (int s = 0; s < kPfStages - 1; ++s) {
    if (s < ntiles) {
      load_tile_rows(jn, irow, begin + s * kTile, end);
      gather_tile(sK + s * kTile * kLds, sV + s * kTile * kLds, kc, vc, jn, begin + s * kTile, end, head_base,
                  row_elems, Tk_max);
    }
    cp_async_commit();
  }
  if (kPfStages - 1 < ntiles) load_tile_rows(jn, irow, begin + (kPfStages - 1) * kTile, end);
  uint32_t qa[8][4];
  for (int it = 0; it < ntiles; ++it) {
    const int stage = it % kPfStages;
    const int nxt = it + kPfStages - 1;
    if (nxt < ntiles) {
      const int ns = nxt % kPfStages;
      gather_tile(sK + ns * kTile * kLds, sV + ns * kTile * kLds, kc, vc, jn, begin + nxt * kTile, end, head_base,
                  row_elems, Tk_max);
    }
    cp_async_commit();
    if (nxt + 1 < ntiles) load_tile_rows(jn, irow, begin + (nxt + 1) * kTile, end);
    cp_async_wait<kPfStages - 1>();
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
// K/V caches are [B, Tk_max, Hkv, D], so the rows of all kv heads at one
// cache position are one contiguous run of Hkv * 256 bytes.  A work unit is
// a tile of R selected positions of one sequence for a block of up to 8 kv
// heads: one bulk copy per position and cache brings the whole run into
// shared memory (no per-head 256-byte pieces).  The units of all sequences
// form one list, cut into equal contiguous ranges, one per CTA of a grid of
// one CTA per SM.
//
// CTA: warp 8 is the producer (the range's row indices staged in shared
// memory, bulk copies into a 3-stage ring, completion by mbarrier
// transaction counts); warps 0..7 are consumers, warp c taking kv head
// c / wph of the block and rows (c % wph) * 16 .. +16 of the tile (wph = 8 /
// heads per block, so R = 16 * wph).  Each consumer runs online softmax on
// mma.sync m16n8k16 with the G query heads of its kv head as the (zero
// padded) M side and writes a partial (m, l, o) for every (sequence, head
// block) pair its range meets.  attn_decode_merge_kernel, launched with
// programmatic stream serialization, then folds the partials of each query
// head with the log-sum-exp rule, one CTA per (sequence, query head).

constexpr int kDxConsumers = 8;
constexpr int kDxThreads = (kDxConsumers + 1) * 32;
constexpr int kDxStages = 3;
constexpr int kIdxChunk = 2048;   // staged row indices per chunk (two chunks)
constexpr int kCntChunk = kIdxChunk / 16;   // staged counts per chunk (units of >= 16 rows)
constexpr int kDxBarBytes = 64;   // mbarriers + abort word
constexpr int kMergeThreads = 256;
constexpr int kMergeMaxC = 1280;   // contributors of one (sequence, head block)

struct DecPlan {
  int nh, wph, R, HB;     // heads per block, warps per head, rows per tile, blocks per sequence
  int pairs, tpp;         // (sequence, block) pairs, tiles per pair
  int dense;              // rows are the first count[b] rows of compact buffers (one copy per tile)
  int row_bytes;          // shared row: nh * 256, padded by 16 when rows are gathered one by one
  int stage_bytes;        // K and V tiles of one stage
  int U, W;               // units (< 2^31: pairs <= 2^14, tiles per pair <= 2^16), CTAs
};

// CTA owning unit u: the largest c with floor(c*U/W) <= u.
__device__ __forceinline__ long long unit_owner(long long u, long long U, long long W) {
  return ((u + 1) * W - 1) / U;
}

__device__ __forceinline__ int clamp_count(const int32_t* __restrict__ count, int b, int k) {
  const int c = count[b];
  return c < 0 ? 0 : (c > k ? k : c);
}

// One online-softmax step over a 16-row slice of a gathered tile ([YOIO]
// §1.1 softmax(QK^T/sqrt(d))V, evaluated incrementally): S = Q K^T with the
// query fragments qa as the M side (G heads, zero padded to 16 rows), rows at
// or past cnt masked, running max / sum / output rescaled, O += P V.  tK and
// tV point at the slice's first row for this kv head; rs_el is the shared
// row stride in elements; rbase is the slice's first row index.
struct Online {
  float o[16][4];
  float m[2], l[2];
};

__device__ __forceinline__ void online_init(Online& st) {
#pragma unroll
  for (int i = 0; i < 16; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) st.o[i][e] = 0.f;
  st.m[0] = st.m[1] = -INFINITY;
  st.l[0] = st.l[1] = 0.f;
}

__device__ __forceinline__ void online_tile(Online& st, const uint32_t (&qa)[8][4], const uint16_t* tK,
                                            const uint16_t* tV, int rs_el, int rbase, int cnt, float qscale) {
  const int lane = threadIdx.x & 31, tg = lane & 3;
  // S = Q K^T over 8 k-steps, in two independent accumulator chains
  float sc[2][4], sd[2][4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) sc[nt][e] = sd[nt][e] = 0.f;
#pragma unroll
  for (int kk = 0; kk < 8; kk += 2) {
    const int mtx = lane >> 3;
    const uint16_t* kr = tK + ((mtx >> 1) * 8 + (lane & 7)) * rs_el + (mtx & 1) * 8;
    uint32_t b0, b1, b2, b3, c0, c1, c2, c3;
    ldmatrix_x4(b0, b1, b2, b3, kr + kk * 16);
    ldmatrix_x4(c0, c1, c2, c3, kr + (kk + 1) * 16);
    mma_bf16_16816(sc[0], qa[kk], b0, b1);
    mma_bf16_16816(sc[1], qa[kk], b2, b3);
    mma_bf16_16816(sd[0], qa[kk + 1], c0, c1);
    mma_bf16_16816(sd[1], qa[kk + 1], c2, c3);
  }
  float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int row = rbase + nt * 8 + tg * 2 + (e & 1);
      const float z = row < cnt ? (sc[nt][e] + sd[nt][e]) * qscale : -INFINITY;
      sc[nt][e] = z;
      mx[e >> 1] = fmaxf(mx[e >> 1], z);
    }
  float alpha[2];
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    float v = mx[hh];
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
    const float mnew = fmaxf(st.m[hh], v);
    const float muse = mnew == -INFINITY ? 0.f : mnew;
    alpha[hh] = exp2f(st.m[hh] - muse);
    st.m[hh] = mnew;
    mx[hh] = muse;
  }
  float rsum[2] = {0.f, 0.f};
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float pv = exp2f(sc[nt][e] - mx[e >> 1]);
      sc[nt][e] = pv;
      rsum[e >> 1] += pv;
    }
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    float v = rsum[hh];
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    st.l[hh] = st.l[hh] * alpha[hh] + v;
  }
  if (__any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f)) {   // a row max moved
#pragma unroll
    for (int dt = 0; dt < 16; ++dt) {
      st.o[dt][0] *= alpha[0];
      st.o[dt][1] *= alpha[0];
      st.o[dt][2] *= alpha[1];
      st.o[dt][3] *= alpha[1];
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
    ldmatrix_x4_trans(b0, b1, b2, b3, tV + ((mtx & 1) * 8 + (lane & 7)) * rs_el + (dt + (mtx >> 1)) * 8);
    mma_bf16_16816(st.o[dt], pa, b0, b1);
    mma_bf16_16816(st.o[dt + 1], pa, b2, b3);
  }
}

// Query fragments of the G heads starting at row head0 of q (rows >= G, or
// all rows when !active, are zero).
__device__ __forceinline__ void load_q_frags(uint32_t (&qa)[8][4], const uint16_t* __restrict__ q, long long head0,
                                             int G, bool active) {
  const int lane = threadIdx.x & 31, gq = lane >> 2, tg = lane & 3;
  const uint32_t* qr0 = reinterpret_cast<const uint32_t*>(q + (head0 + gq) * kD);
  const uint32_t* qr1 = reinterpret_cast<const uint32_t*>(q + (head0 + gq + 8) * kD);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const int c0 = (kk * 16 + 2 * tg) >> 1, c1 = (kk * 16 + 8 + 2 * tg) >> 1;
    qa[kk][0] = active && gq < G ? __ldg(qr0 + c0) : 0u;
    qa[kk][1] = active && gq + 8 < G ? __ldg(qr1 + c0) : 0u;
    qa[kk][2] = active && gq < G ? __ldg(qr0 + c1) : 0u;
    qa[kk][3] = active && gq + 8 < G ? __ldg(qr1 + c1) : 0u;
  }
}

__global__ void __launch_bounds__(kDxThreads, 1)
attn_decode_split_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ kc,
                         const uint16_t* __restrict__ vc, const int32_t* __restrict__ idx,
                         const int32_t* __restrict__ count, int Tk_max, int Hq, int Hkv, int k, DecPlan pl,
                         float qscale, float* __restrict__ part_o, float* __restrict__ part_ml,
                         int* __restrict__ err) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)kDxStages * pl.stage_bytes);
  uint64_t* empty = full + kDxStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kDxStages);
  int32_t* sidx = reinterpret_cast<int32_t*>(smem + (size_t)kDxStages * pl.stage_bytes + kDxBarBytes);
  int32_t* scnt = sidx + 2 * kIdxChunk;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kDxStages; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], kDxConsumers);
    }
    *abort_flag = 0;
    tc::fence_barrier_init();
  }
  __syncthreads();
  pdl_wait();                 // inputs may come from the kernel before
  pdl_launch_dependents();    // the merge may start launching
  const int lo = (int)((long long)blockIdx.x * pl.U / pl.W);
  const int hi = (int)((long long)(blockIdx.x + 1) * pl.U / pl.W);
  const int G = Hq / Hkv;
  const int R = pl.R, rb = pl.row_bytes;

  if (warp == kDxConsumers) {
    // ------------------------------------------------------------ producer
    // The row indices and counts of the CTA's units are staged in shared
    // memory with cp.async, kIdxChunk rows at a time and one chunk ahead, so
    // issuing a tile never waits on an index load (under full DRAM load a
    // dependent load per tile would pace the ring).  Rows past the count
    // repeat the tile's first row so every byte of the tile is finite (their
    // scores are masked).
    const int CU = kIdxChunk / R;   // units per chunk
    auto stage_chunk = [&](int c0, int buf) {
      const int c1 = min(c0 + CU, hi);
      int32_t* si = sidx + buf * kIdxChunk;
      for (int e = lane; e < (pl.dense ? 0 : (c1 - c0) * R); e += 32) {
        const int u = c0 + e / R;
        const int r = e % R;
        const int b = u / pl.tpp / pl.HB;
        const int row = u % pl.tpp * R + r;
        const bool v = row < k;
        cp_async4(si + e, idx + (long long)b * k + (v ? row : 0), v);
      }
      for (int e = lane; e < c1 - c0; e += 32)
        cp_async4(scnt + buf * kCntChunk + e, count + (c0 + e) / pl.tpp / pl.HB, true);
      cp_async_commit();
    };
    int chunk_lo = lo;
    int buf = 0;
    stage_chunk(lo, 0);
    if (lo + CU < hi) stage_chunk(lo + CU, 1);
    else cp_async_commit();
    cp_async_wait<1>();
    __syncwarp();
    uint32_t fill = 0;
    for (int u = lo; u < hi; ++u) {
      if (u == chunk_lo + CU) {   // next chunk (staged one chunk ago)
        chunk_lo += CU;
        buf ^= 1;
        cp_async_wait<0>();
        __syncwarp();
        if (chunk_lo + CU < hi) stage_chunk(chunk_lo + CU, buf ^ 1);
      }
      const int ul = u - chunk_lo;
      const int p = u / pl.tpp, b = p / pl.HB, hb = p % pl.HB;
      const int cr = scnt[buf * kCntChunk + ul];
      const int cnt = cr < 0 ? 0 : (cr > k ? k : cr);
      const int r0 = u % pl.tpp * R;
      if (r0 >= cnt) continue;   // the consumers skip the same units
      const int32_t* si = sidx + buf * kIdxChunk + ul * R;
      const int h0 = hb * pl.nh;
      const int nh_here = min(pl.nh, Hkv - h0);
      const uint32_t bytes = (uint32_t)nh_here * 256u;
      const int s = (int)(fill % kDxStages);
      const uint32_t use = fill / kDxStages;
      if (use > 0 && !tc::mbar_wait(&empty[s], (use - 1) & 1u, abort_flag, err, 11)) break;
      unsigned char* stK = smem + (size_t)s * pl.stage_bytes;
      unsigned char* stV = stK + (size_t)R * rb;
      // bytes this tile's copies bring (compact rows copy their pads too)
      const int rows_in = pl.dense ? min(R, k - r0) : 0;
      const uint32_t tile_bytes = pl.dense ? (uint32_t)(rows_in * rb) + (uint32_t)(R - rows_in) * bytes
                                           : (uint32_t)R * bytes;
      if (lane == 0) tc::mbar_arrive_expect_tx(&full[s], 2u * tile_bytes);
      __syncwarp();
      if (pl.dense) {
        // compact rows (one head block), each Hkv * 256 bytes plus the same
        // 16-byte pad as a shared row: the tile's rows are contiguous, so one
        // bulk copy per cache brings them all in the padded layout; rows past
        // the buffer's end repeat the tile's first row (finite, masked)
        const long long off = ((long long)b * k + r0) * (rb / 2);
        if (lane == 0) {
          tc::bulk_load(stK, kc + off, (uint32_t)(rows_in * rb), &full[s]);
          tc::bulk_load(stV, vc + off, (uint32_t)(rows_in * rb), &full[s]);
        }
        for (int r = rows_in + lane; r < R; r += 32) {
          tc::bulk_load(stK + (size_t)r * rb, kc + off, bytes, &full[s]);
          tc::bulk_load(stV + (size_t)r * rb, vc + off, bytes, &full[s]);
        }
      } else {
        const int j0 = si[0];   // row r0 < cnt
        for (int r = lane; r < R; r += 32) {
          const int j = checked_row(r0 + r < cnt ? si[r] : j0, Tk_max, kDbgDecodeIndex);
          const long long off = (((long long)b * Tk_max + j) * Hkv + h0) * kD;
          tc::bulk_load(stK + (size_t)r * rb, kc + off, bytes, &full[s]);
          tc::bulk_load(stV + (size_t)r * rb, vc + off, bytes, &full[s]);
        }
      }
      ++fill;
    }
    cp_async_wait<0>();
    // every copy this CTA issued lands before it exits
    for (int s = 0; s < kDxStages; ++s) {
      if ((uint32_t)s < fill) {
        const uint32_t last_use = (fill - 1 - (uint32_t)s) / kDxStages;
        if (!tc::mbar_wait_drain(&full[s], last_use & 1u) && err) atomicCAS(err, 0, 12);
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int gq = lane >> 2, tg = lane & 3;
  const int hs = warp / pl.wph, rs = warp % pl.wph;
  const int rs_el = rb / 2;   // shared row stride in elements
  Online st;
  uint32_t qa[8][4];
  int cur_p = -1, cnt = 0;
  bool active = false;        // this warp's head exists in the current block
  long long head0 = 0;
  uint32_t fill = 0;

  auto flush = [&](int p) {
    if (!active) return;
    // CTA c's partial of pair p sits in slot p + c: the CTAs meeting pair
    // p+1 start at or after the last one meeting p, so slots never collide
    const long long slot = ((long long)p + blockIdx.x) * pl.wph + rs;
    const long long base = (slot * pl.nh + hs) * G;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int h = gq + 8 * hh;
      if (h < G) {
#pragma unroll
        for (int dt = 0; dt < 16; ++dt)
          *reinterpret_cast<float2*>(part_o + (base + h) * kD + dt * 8 + 2 * tg) =
              make_float2(st.o[dt][2 * hh], st.o[dt][2 * hh + 1]);
        if (tg == 0) *reinterpret_cast<float2*>(part_ml + (base + h) * 2) = make_float2(st.m[hh], st.l[hh]);
      }
    }
  };

  for (int u = lo; u < hi; ++u) {
    const int p = u / pl.tpp, b = p / pl.HB, hb = p % pl.HB;
    if (p != cur_p) {
      if (cur_p >= 0) flush(cur_p);
      cur_p = p;
      cnt = clamp_count(count, b, k);
      const int g = hb * pl.nh + hs;
      active = hs < min(pl.nh, Hkv - hb * pl.nh);
      head0 = (long long)b * Hq + (long long)(active ? g : 0) * G;
      online_init(st);
      load_q_frags(qa, q, head0, G, active);
    }
    const int r0 = u % pl.tpp * R;
    if (r0 >= cnt) continue;   // the producer skips this unit too
    const int s = (int)(fill % kDxStages);
    if (!tc::mbar_wait(&full[s], (fill / kDxStages) & 1u, abort_flag, err, 13)) break;
    const int rbase = r0 + rs * 16;
    if (active && rbase < cnt) {
      const uint16_t* tK = reinterpret_cast<const uint16_t*>(smem + (size_t)s * pl.stage_bytes) +
                           (size_t)(rs * 16) * rs_el + hs * kD;
      const uint16_t* tV = tK + (size_t)R * rs_el;
      online_tile(st, qa, tK, tV, rs_el, rbase, cnt, qscale);
    }
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(&empty[s]);
    ++fill;
  }
  if (cur_p >= 0 && !*abort_flag) flush(cur_p);
}

// Folds the partials of one (sequence, query head): out = sum_x w_x o_x / L,
// w_x = 2^(m_x - M), L = sum_x w_x l_x, M = max_x m_x (base-2 logits).  The
// first loads of every kind are issued together, so the usual case (at most
// 128 contributors, 16 per warp) costs one memory round trip.  All index
// arithmetic happens before the wait for the split kernel.
__global__ void __launch_bounds__(kMergeThreads)
attn_decode_merge_kernel(const float* __restrict__ part_o, const float* __restrict__ part_ml, DecPlan pl,
                         int Hq, int Hkv, const int* __restrict__ err, uint16_t* __restrict__ out,
                         float* __restrict__ lse) {
  constexpr int kWarps = kMergeThreads / 32;
  constexpr int kPre = 16;  // o rows prefetched per warp: up to 128 contributors in one round
  __shared__ float wts[kMergeMaxC];
  __shared__ float red[kWarps][kD];
  __shared__ float rmax[kWarps], rsum[kWarps];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = Hq / Hkv;
  const int bh = blockIdx.x;
  const int b = bh / Hq, h = bh % Hq;
  const int g = h / G, gq = h % G;
  const int hb = g / pl.nh, hs = g % pl.nh;
  const int p = b * pl.HB + hb;
  const long long first = unit_owner((long long)p * pl.tpp, pl.U, pl.W);
  const long long last = unit_owner((long long)(p + 1) * pl.tpp - 1, pl.U, pl.W);
  const int C = (int)(last - first + 1) * pl.wph;
  const float* pml = part_ml + ((((long long)p + first) * pl.wph * pl.nh + hs) * G + gq) * 2;
  const float* po = part_o + ((((long long)p + first) * pl.wph * pl.nh + hs) * G + gq) * kD;
  const int xstride = pl.nh * G;   // entries between consecutive contributors
  pdl_wait();   // the partials come from the split kernel
  pdl_launch_dependents();

  const float2 ml0 = tid < C ? __ldcg(reinterpret_cast<const float2*>(pml + (long long)tid * xstride * 2))
                             : make_float2(-INFINITY, 0.f);
  float4 pre[kPre];
#pragma unroll
  for (int i = 0; i < kPre; ++i) {
    const int x = warp + kWarps * i;
    pre[i] = x < C ? __ldcg(reinterpret_cast<const float4*>(po + (long long)x * xstride * kD) + lane)
                   : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const int failed = *err;

  float mloc = ml0.x;
  for (int x = tid + kMergeThreads; x < C; x += kMergeThreads)
    mloc = fmaxf(mloc, __ldcg(pml + (long long)x * xstride * 2));
  mloc = warp_max(mloc);
  if (lane == 0) rmax[warp] = mloc;
  __syncthreads();
  float M = rmax[0];
#pragma unroll
  for (int w = 1; w < kWarps; ++w) M = fmaxf(M, rmax[w]);
  auto weight = [&](float2 ml) { return (ml.y > 0.f && M != -INFINITY) ? exp2f(ml.x - M) : 0.f; };
  float lloc = 0.f;
  if (tid < C) {
    const float wv = weight(ml0);
    wts[tid] = wv;
    lloc = ml0.y * wv;
  }
  for (int x = tid + kMergeThreads; x < C; x += kMergeThreads) {
    const float2 ml = __ldcg(reinterpret_cast<const float2*>(pml + (long long)x * xstride * 2));
    const float wv = weight(ml);
    wts[x] = wv;
    lloc += ml.y * wv;
  }
  lloc = warp_sum(lloc);
  if (lane == 0) rsum[warp] = lloc;
  __syncthreads();
  float L = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) L += rsum[w];

  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  auto fold = [&](float4 ov, float wt) {
    acc.x = fmaf(ov.x, wt, acc.x);
    acc.y = fmaf(ov.y, wt, acc.y);
    acc.z = fmaf(ov.z, wt, acc.z);
    acc.w = fmaf(ov.w, wt, acc.w);
  };
#pragma unroll
  for (int i = 0; i < kPre; ++i) {
    const int x = warp + kWarps * i;
    if (x < C) fold(pre[i], wts[x]);
  }
#pragma unroll 4
  for (int x = warp + kWarps * kPre; x < C; x += kWarps)
    fold(__ldcg(reinterpret_cast<const float4*>(po + (long long)x * xstride * kD) + lane), wts[x]);
  *reinterpret_cast<float4*>(&red[warp][lane * 4]) = acc;
  __syncthreads();
  if (tid < kD) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) v += red[w][tid];
    const float inv = L > 0.f ? 1.f / L : 0.f;
    // a split kernel that gave up leaves NaN, so the failure is visible
    out[(long long)bh * kD + tid] = failed ? (uint16_t)0x7fc0 : f2bf(v * inv);
    if (tid == 0 && lse != nullptr)
      lse[bh] = failed ? __int_as_float(0x7fc00000) : (L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY);
  }
}

// Gathers the selected rows of each sequence (all kv heads of a position,
// Hkv * 256 contiguous bytes per cache) into compact buffers of rows of
// Hkv * 256 bytes plus a 16-byte zero pad ([B][k][Hkv * D + 8] elements),
// the layout of a shared-memory row of the decode split kernel, so that a
// tile of rows is one contiguous copy; rows from count[b] to k are written
// as zeros.  One warp per row, 16-byte loads and stores.
__global__ void __launch_bounds__(256)
gather_rows_kernel(const uint16_t* __restrict__ kc, const uint16_t* __restrict__ vc,
                   const int32_t* __restrict__ idx, const int32_t* __restrict__ count, int Tk_max, int Hkv,
                   int k, uint16_t* __restrict__ ko, uint16_t* __restrict__ vo) {
  pdl_wait();
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int r = blockIdx.x * 8 + warp;
  if (r >= k) return;
  const int cnt = clamp_count(count, b, k);
  const int chunks = Hkv * kD / 8;   // 16-byte chunks per row (then one chunk of pad)
  uint4* dk = reinterpret_cast<uint4*>(ko + ((long long)b * k + r) * (Hkv * kD + 8));
  uint4* dv = reinterpret_cast<uint4*>(vo + ((long long)b * k + r) * (Hkv * kD + 8));
  if (lane == 0) {
    dk[chunks] = make_uint4(0u, 0u, 0u, 0u);
    dv[chunks] = make_uint4(0u, 0u, 0u, 0u);
  }
  if (r < cnt) {
    const int j = checked_row(idx[(long long)b * k + r], Tk_max, kDbgGatherIndex);
    const uint4* sk = reinterpret_cast<const uint4*>(kc + ((long long)b * Tk_max + j) * Hkv * kD);
    const uint4* sv = reinterpret_cast<const uint4*>(vc + ((long long)b * Tk_max + j) * Hkv * kD);
    for (int c = lane; c < chunks; c += 32) {
      const uint4 a = __ldg(sk + c), v = __ldg(sv + c);
      dk[c] = a;
      dv[c] = v;
    }
  } else {
    for (int c = lane; c < chunks; c += 32) {
      dk[c] = make_uint4(0u, 0u, 0u, 0u);
      dv[c] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
}

DecPlan decode_plan(int B, int Hkv, int k, bool dense = false) {
  const int sms = device_sm_count();
  DecPlan pl;
  pl.nh = Hkv < kDxConsumers ? Hkv : kDxConsumers;
  pl.wph = kDxConsumers / pl.nh;
  pl.R = 16 * pl.wph;
  pl.HB = (Hkv + pl.nh - 1) / pl.nh;
  pl.pairs = B * pl.HB;
  pl.tpp = (k + pl.R - 1) / pl.R;
  pl.dense = dense ? 1 : 0;
  pl.row_bytes = pl.nh * kD * 2 + 16;   // the pad keeps the consumers' ldmatrix free of bank conflicts
  pl.stage_bytes = 2 * pl.R * pl.row_bytes;
  pl.U = pl.pairs * pl.tpp;
  int W = sms;   // one CTA per SM
  if (W > kMergeMaxC / pl.wph) W = kMergeMaxC / pl.wph;   // contributors of one pair <= W * wph
  if (W > pl.U) W = pl.U;
  if (W < 1) W = 1;
  pl.W = W;
  return pl;
}

size_t dec_smem_bytes(const DecPlan& pl) {
  return (size_t)kDxStages * pl.stage_bytes + kDxBarBytes + (2 * kIdxChunk + 2 * kCntChunk) * sizeof(int32_t);
}

}  // namespace

static size_t align256a(size_t x) { return (x + 255) & ~size_t(255); }

// Decode workspace: a 256-byte head whose first word is the kernel error
// code (zero when all is well; set if a pipeline wait gave up), then the
// split partials.  Nothing but the error word needs to start at zero.
constexpr size_t kDecHead = 256;

size_t decode_attn_zero_bytes(int B, int Hkv, int k) {
  (void)B, (void)Hkv, (void)k;
  return kDecHead;
}

size_t decode_attn_workspace_bytes(int B, int Hq, int Hkv, int D, int k) {
  (void)D;
  const DecPlan pl = decode_plan(B, Hkv, k);
  const int G = Hq / Hkv;
  const size_t slots = (size_t)(pl.pairs + pl.W) * pl.wph * pl.nh * G;
  return kDecHead + align256a(slots * kD * 4) + align256a(slots * 2 * 4);
}

cudaError_t launch_attn_decode(const uint16_t* q, const uint16_t* kc, const uint16_t* vc,
                               const int32_t* idx, const int32_t* count, int B, int Tk_max, int Hq,
                               int Hkv, int k, float scale, uint16_t* out, float* lse, void* ws,
                               cudaStream_t st) {
  if (B <= 0) return cudaSuccess;
  const bool dense = idx == nullptr;   // compact rows [B][k][Hkv][D] (Hkv <= 8, Tk_max == k)
  const DecPlan pl = decode_plan(B, Hkv, k, dense);
  const int G = Hq / Hkv;
  const size_t slots = (size_t)(pl.pairs + pl.W) * pl.wph * pl.nh * G;
  char* p = static_cast<char*>(ws);
  int* err = reinterpret_cast<int*>(p);
  p += kDecHead;
  float* po = reinterpret_cast<float*>(p);
  p += align256a(slots * kD * 4);
  float* pml = reinterpret_cast<float*>(p);
  const size_t smem = dec_smem_bytes(pl);
  cudaError_t e = ensure_dynamic_smem((const void*)attn_decode_split_kernel, smem);
  if (e != cudaSuccess) return e;
  // both kernels are launched with programmatic stream serialization: each
  // may be scheduled while the kernel before it drains and waits in pdl_wait()
  e = launch_pdl(attn_decode_split_kernel, dim3((unsigned)pl.W), dim3(kDxThreads), smem, st, q, kc, vc, idx, count,
                 Tk_max, Hq, Hkv, k, pl, scale * kLog2e, po, pml, err);
  if (e != cudaSuccess) return e;
  e = launch_pdl(attn_decode_merge_kernel, dim3((unsigned)((long long)B * Hq)), dim3(kMergeThreads), 0, st, po, pml,
                 pl, Hq, Hkv, err, out, lse);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const uint16_t* kc, const uint16_t* vc, const int32_t* idx, const int32_t* count,
                               int B, int Tk_max, int Hkv, int k, uint16_t* ko, uint16_t* vo, cudaStream_t st) {
  if (B <= 0) return cudaSuccess;
  const cudaError_t e = launch_pdl(gather_rows_kernel, dim3((unsigned)((k + 7) / 8), (unsigned)B), dim3(256), 0, st,
                                   kc, vc, idx, count, Tk_max, Hkv, k, ko, vo);
  return e != cudaSuccess ? e : cudaGetLastError();
}

#ifdef SA_DEBUG
namespace {
__global__ void dbg_canary_kernel(const unsigned char* __restrict__ c, int site) {
  if (c[threadIdx.x] != kDbgCanaryByte) dbg_note(kDbgCanary, site, (int)threadIdx.x);
}
}  // namespace
#endif

cudaError_t dbg_arm(void* ws, size_t off, cudaStream_t st) {
#ifdef SA_DEBUG
  if (ws == nullptr) return cudaSuccess;
  return cudaMemsetAsync(static_cast<unsigned char*>(ws) + off, kDbgCanaryByte, kDbgCanaryBytes, st);
#else
  (void)ws, (void)off, (void)st;
  return cudaSuccess;
#endif
}

cudaError_t dbg_check(const void* ws, size_t off, int site, cudaStream_t st) {
#ifdef SA_DEBUG
  if (ws == nullptr) return cudaSuccess;
  dbg_canary_kernel<<<1, kDbgCanaryBytes, 0, st>>>(static_cast<const unsigned char*>(ws) + off, site);
  return cudaGetLastError();
#else
  (void)ws, (void)off, (void)site, (void)st;
  return cudaSuccess;
#endif
}

cudaError_t dbg_read(int* host4, bool reset) {
#ifdef SA_DEBUG
  cudaError_t e = cudaMemcpyFromSymbol(host4, g_dbg, 4 * sizeof(int));
  if (e == cudaSuccess && reset) {
    const int zero[4] = {0, 0, 0, 0};
    e = cudaMemcpyToSymbol(g_dbg, zero, sizeof(zero));
  }
  return e;
#else
  (void)reset;
  for (int i = 0; i < 4; ++i) host4[i] = 0;
  return cudaSuccess;
#endif
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
