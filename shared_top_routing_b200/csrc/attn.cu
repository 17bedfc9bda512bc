// Gathered sparse attention over index-selected K/V rows (sm_100a).
//
// Method: [YOIO] §1.1 Attention(Q,K,V) = softmax(QK^T/sqrt(d_k))V, evaluated
// only over the rows named by the shared index ([YOIO] §2.3 selector;
// [LC] "DSA 与 IndexShare", O(L^2) -> O(Lk)).  Decode follows the split-K
// shape of [SSA] §六: CTAs take slices of the compact index list, the rows of
// one kv head are loaded once for all query heads of its GQA group, and the
// partial (max, sum, output) triples are merged by the log-sum-exp rule.
//
// attn_decode_kernel   grid (splits, Hkv, B), 128 threads.  cp.async gathers
//                      the split's K rows and V rows into padded shared tiles
//                      (two commit groups so scores overlap the V transfer),
//                      CUDA-core fp32 dot products and softmax, and the last
//                      CTA of each (sequence, kv head) -- found with an atomic
//                      ticket, never a wait -- merges the partials.
// attn_prefill_kernel  grid (T, Hkv, B) kv-head-major, 128 threads.  For one
//                      query token and one kv head, 64-row tiles of gathered
//                      K/V are double-buffered through shared memory with
//                      cp.async; each warp owns 16 rows of a tile and runs
//                      FlashAttention-style online softmax on mma.sync
//                      m16n8k16 (the G query heads padded to 16 rows); the 4
//                      warps' partials are merged at the end.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

constexpr int kD = 128;        // head_dim
constexpr int kLds = kD + 8;   // padded smem row (elements)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ int clamp_row(int j, int Tk_max) {
  return j < 0 ? 0 : (j >= Tk_max ? Tk_max - 1 : j);
}

// ------------------------------------------------------------------ decode

template <int G>
__global__ void __launch_bounds__(128)
attn_decode_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ kc,
                   const uint16_t* __restrict__ vc, const int32_t* __restrict__ idx,
                   const int32_t* __restrict__ count, int Tk_max, int Hq, int Hkv, int k, int R,
                   int S, float qscale, float* __restrict__ part_o, float* __restrict__ part_ml,
                   unsigned* __restrict__ ticket, uint16_t* __restrict__ out,
                   float* __restrict__ lse) {
  extern __shared__ __align__(16) unsigned char smem[];
  // layout: qs[G][kD] f32 | sc[DS][G][R] f32 | ml[32] f32 | Ks[R][kLds] | Vs[R][kLds]
  // (every region a multiple of 16 bytes, so the cp.async targets stay aligned)
  const int DS = 128 / R;  // dim slices for the score phase (R in {32, 64, 128})
  float* qs = reinterpret_cast<float*>(smem);
  float* sc = qs + G * kD;
  float* mls = sc + DS * G * R;
  uint16_t* Ks = reinterpret_cast<uint16_t*>(mls + 32);
  uint16_t* Vs = Ks + R * kLds;
  __shared__ int s_last;

  const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int cnt = count[b];
  cnt = cnt < 0 ? 0 : (cnt > k ? k : cnt);
  const int i0 = s * R;
  const int nrow = max(0, min(R, cnt - i0));
  const long long part = ((long long)b * Hq + g * G);  // first head of the group

  if (nrow > 0) {
    // gather: thread -> (row, 16-byte chunk); K group first, then V group
    const int32_t* irow = idx + (long long)b * k + i0;
    for (int e = tid; e < R * 16; e += 128) {
      int r = e >> 4, c = e & 15;
      bool v = r < nrow;
      int j = v ? clamp_row(irow[r], Tk_max) : 0;
      long long off = (((long long)b * Tk_max + j) * Hkv + g) * kD + c * 8;
      cp_async16(Ks + r * kLds + c * 8, kc + off, v);
    }
    cp_async_commit();
    for (int e = tid; e < R * 16; e += 128) {
      int r = e >> 4, c = e & 15;
      bool v = r < nrow;
      int j = v ? clamp_row(irow[r], Tk_max) : 0;
      long long off = (((long long)b * Tk_max + j) * Hkv + g) * kD + c * 8;
      cp_async16(Vs + r * kLds + c * 8, vc + off, v);
    }
    cp_async_commit();
    // q of the group's heads, pre-scaled into the log2 domain
    for (int e = tid; e < G * kD / 2; e += 128) {
      int h = e / (kD / 2), c2 = e % (kD / 2);
      uint32_t v = *reinterpret_cast<const uint32_t*>(q + (part + h) * kD + 2 * c2);
      qs[h * kD + 2 * c2] = bf_lo(v) * qscale;
      qs[h * kD + 2 * c2 + 1] = bf_hi(v) * qscale;
    }
    cp_async_wait<1>();
    __syncthreads();

    // scores: thread -> (row within a 32-row band, dim slice)
    {
      const int bands = 4 / DS;
      const int r = (warp % bands) * 32 + lane;
      const int slice = warp / bands;
      const int dlen = kD / DS;
      float acc[G];
#pragma unroll
      for (int h = 0; h < G; ++h) acc[h] = 0.f;
      const uint16_t* krow = Ks + r * kLds + slice * dlen;
      for (int c = 0; c < dlen; c += 8) {
        uint4 kv = *reinterpret_cast<const uint4*>(krow + c);
        float kf[8] = {bf_lo(kv.x), bf_hi(kv.x), bf_lo(kv.y), bf_hi(kv.y),
                       bf_lo(kv.z), bf_hi(kv.z), bf_lo(kv.w), bf_hi(kv.w)};
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float4* qp = reinterpret_cast<const float4*>(qs + h * kD + slice * dlen + c);
          float4 qa = qp[0], qb = qp[1];
          float a = acc[h];
          a = fmaf(kf[0], qa.x, a); a = fmaf(kf[1], qa.y, a);
          a = fmaf(kf[2], qa.z, a); a = fmaf(kf[3], qa.w, a);
          a = fmaf(kf[4], qb.x, a); a = fmaf(kf[5], qb.y, a);
          a = fmaf(kf[6], qb.z, a); a = fmaf(kf[7], qb.w, a);
          acc[h] = a;
        }
      }
#pragma unroll
      for (int h = 0; h < G; ++h) sc[(slice * G + h) * R + r] = acc[h];
    }
    __syncthreads();
    // softmax per head (warp per head), p overwrites slice 0
    for (int h = warp; h < G; h += 4) {
      float m = -INFINITY;
      for (int r = lane; r < R; r += 32) {
        float z = 0.f;
        for (int sl = 0; sl < DS; ++sl) z += sc[(sl * G + h) * R + r];
        z = r < nrow ? z : -INFINITY;
        sc[h * R + r] = z;
        m = fmaxf(m, z);
      }
      m = warp_max(m);
      float l = 0.f;
      for (int r = lane; r < R; r += 32) {
        float p = r < nrow ? exp2f(sc[h * R + r] - m) : 0.f;
        sc[h * R + r] = p;
        l += p;
      }
      l = warp_sum(l);
      if (lane == 0) { mls[2 * h] = m; mls[2 * h + 1] = l; }
    }
    cp_async_wait<0>();
    __syncthreads();
    // P V: thread -> dims (2c2, 2c2+1), heads of one parity
    {
      const int c2 = tid & 63, hp = tid >> 6;
      float o0[(G + 1) / 2], o1[(G + 1) / 2];
#pragma unroll
      for (int u = 0; u < (G + 1) / 2; ++u) { o0[u] = 0.f; o1[u] = 0.f; }
      for (int r = 0; r < nrow; ++r) {
        uint32_t v = *reinterpret_cast<const uint32_t*>(Vs + r * kLds + 2 * c2);
        float v0 = bf_lo(v), v1 = bf_hi(v);
#pragma unroll
        for (int u = 0; u < (G + 1) / 2; ++u) {
          int h = hp + 2 * u;
          if (h < G) {
            float p = sc[h * R + r];
            o0[u] = fmaf(p, v0, o0[u]);
            o1[u] = fmaf(p, v1, o1[u]);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < (G + 1) / 2; ++u) {
        int h = hp + 2 * u;
        if (h < G) {
          float2* dst = reinterpret_cast<float2*>(part_o + ((part + h) * S + s) * kD + 2 * c2);
          *dst = make_float2(o0[u], o1[u]);
        }
      }
    }
    if (tid < G) {
      part_ml[((part + tid) * S + s) * 2] = mls[2 * tid];
      part_ml[((part + tid) * S + s) * 2 + 1] = mls[2 * tid + 1];
    }
  } else if (tid < G) {
    part_ml[((part + tid) * S + s) * 2] = -INFINITY;
    part_ml[((part + tid) * S + s) * 2 + 1] = 0.f;
  }

  // Last CTA of this (sequence, kv head) merges the S partials.
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    unsigned prev = atomicAdd(ticket + (long long)b * Hkv + g, 1u);
    s_last = (prev == (unsigned)(S - 1));
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  {
    const int c2 = tid & 63, hp = tid >> 6;
    for (int h = hp; h < G; h += 2) {
      const float* ml = part_ml + (part + h) * S * 2;
      float M = -INFINITY;
      for (int x = 0; x < S; ++x) M = fmaxf(M, __ldcg(ml + 2 * x));
      float L = 0.f, a0 = 0.f, a1 = 0.f;
      if (M != -INFINITY) {
        for (int x = 0; x < S; ++x) {
          float mx = __ldcg(ml + 2 * x), lx = __ldcg(ml + 2 * x + 1);
          if (lx == 0.f) continue;
          float w = exp2f(mx - M);
          L = fmaf(lx, w, L);
          float2 o = __ldcg(reinterpret_cast<const float2*>(part_o + ((part + h) * S + x) * kD + 2 * c2));
          a0 = fmaf(o.x, w, a0);
          a1 = fmaf(o.y, w, a1);
        }
      }
      float inv = L > 0.f ? 1.f / L : 0.f;
      *reinterpret_cast<uint32_t*>(out + (part + h) * kD + 2 * c2) = pack_bf2(a0 * inv, a1 * inv);
      if (c2 == 0 && lse != nullptr)
        lse[part + h] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
    }
  }
  if (tid == 0) ticket[(long long)b * Hkv + g] = 0u;  // ready for the next call
}

// ----------------------------------------------------------------- prefill

constexpr int kPTile = 64;  // gathered rows per tile (16 per warp)

template <int G>
__global__ void __launch_bounds__(128)
attn_prefill_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ kc,
                    const uint16_t* __restrict__ vc, const int32_t* __restrict__ idx,
                    const int32_t* __restrict__ count, int T, int Tk_max, int Hq, int Hkv, int k,
                    float qscale, uint16_t* __restrict__ out, float* __restrict__ lse) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint16_t* sQ = reinterpret_cast<uint16_t*>(smem);          // [16][kLds]
  uint16_t* sK = sQ + 16 * kLds;                              // [2][kPTile][kLds]
  uint16_t* sV = sK + 2 * kPTile * kLds;                      // [2][kPTile][kLds]

  const int t = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long tok = (long long)b * T + t;
  int cnt = count[tok];
  cnt = cnt < 0 ? 0 : (cnt > k ? k : cnt);
  const int32_t* irow = idx + tok * k;
  const int ntiles = (cnt + kPTile - 1) / kPTile;

  auto load_tile = [&](int it, int stage) {
    const int r = tid >> 1, h = tid & 1;
    const int i = it * kPTile + r;
    const bool v = i < cnt;
    const int j = v ? clamp_row(irow[i], Tk_max) : 0;
    const long long off = (((long long)b * Tk_max + j) * Hkv + g) * kD;
    uint16_t* dk = sK + (stage * kPTile + r) * kLds;
    uint16_t* dv = sV + (stage * kPTile + r) * kLds;
#pragma unroll
    for (int c = h * 8; c < h * 8 + 8; ++c) {
      cp_async16(dk + c * 8, kc + off + c * 8, v);
      cp_async16(dv + c * 8, vc + off + c * 8, v);
    }
  };

  // Q (G heads, zero padded to 16 rows)
  for (int e = tid; e < 16 * 16; e += 128) {
    int h = e >> 4, c = e & 15;
    bool v = h < G;
    cp_async16(sQ + h * kLds + c * 8, q + ((tok * Hq) + g * G + (v ? h : 0)) * kD + c * 8, v);
  }
  if (ntiles > 0) load_tile(0, 0);
  cp_async_commit();

  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[i][e] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
  uint32_t qa[8][4];
  const int gq = lane >> 2, tg = lane & 3;

  for (int it = 0; it < ntiles; ++it) {
    const int stage = it & 1;
    if (it + 1 < ntiles) load_tile(it + 1, stage ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (it == 0) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        ldmatrix_x4(qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3],
                    sQ + (lane & 15) * kLds + kk * 16 + (lane >> 4) * 8);
    }
    const uint16_t* tK = sK + (stage * kPTile + warp * 16) * kLds;
    const uint16_t* tV = sV + (stage * kPTile + warp * 16) * kLds;
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
    // mask rows past the count, scale into the log2 domain
    const int rbase = it * kPTile + warp * 16;
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        int row = rbase + nt * 8 + tg * 2 + (e & 1);
        float z = row < cnt ? sc[nt][e] * qscale : -INFINITY;
        sc[nt][e] = z;
        mx[e >> 1] = fmaxf(mx[e >> 1], z);
      }
    float alpha[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float v = mx[hh];
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
      float mnew = fmaxf(m_r[hh], v);
      float muse = mnew == -INFINITY ? 0.f : mnew;
      alpha[hh] = exp2f(m_r[hh] - muse);
      m_r[hh] = mnew;
      mx[hh] = muse;
    }
    float rs[2] = {0.f, 0.f};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float p = exp2f(sc[nt][e] - mx[e >> 1]);
        sc[nt][e] = p;
        rs[e >> 1] += p;
      }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float v = rs[hh];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      l_r[hh] = l_r[hh] * alpha[hh] + v;
    }
#pragma unroll
    for (int dt = 0; dt < 16; ++dt) {
      o[dt][0] *= alpha[0]; o[dt][1] *= alpha[0];
      o[dt][2] *= alpha[1]; o[dt][3] *= alpha[1];
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
    __syncthreads();
  }
  cp_async_wait<0>();
  __syncthreads();

  // Merge the 4 warps: smem reuse of the K/V stages.
  float* mo = reinterpret_cast<float*>(sK);       // [4][16][kD]
  float* mm = mo + 4 * 16 * kD;                   // [4][16][2]
#pragma unroll
  for (int dt = 0; dt < 16; ++dt) {
    int d0 = dt * 8 + tg * 2;
    *reinterpret_cast<float2*>(mo + ((warp * 16) + gq) * kD + d0) = make_float2(o[dt][0], o[dt][1]);
    *reinterpret_cast<float2*>(mo + ((warp * 16) + gq + 8) * kD + d0) = make_float2(o[dt][2], o[dt][3]);
  }
  if (tg == 0) {
    mm[((warp * 16) + gq) * 2] = m_r[0];
    mm[((warp * 16) + gq) * 2 + 1] = l_r[0];
    mm[((warp * 16) + gq + 8) * 2] = m_r[1];
    mm[((warp * 16) + gq + 8) * 2 + 1] = l_r[1];
  }
  __syncthreads();
  const int d = tid;  // 128 threads <-> 128 dims
  for (int h = 0; h < G; ++h) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, mm[(w * 16 + h) * 2]);
    float L = 0.f, a = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        float lw = mm[(w * 16 + h) * 2 + 1];
        if (lw == 0.f) continue;
        float wt = exp2f(mm[(w * 16 + h) * 2] - M);
        L = fmaf(lw, wt, L);
        a = fmaf(mo[(w * 16 + h) * kD + d], wt, a);
      }
    }
    float v = L > 0.f ? a / L : 0.f;
    out[(tok * Hq + g * G + h) * kD + d] = f2bf(v);
    if (d == 0 && lse != nullptr) lse[tok * Hq + g * G + h] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
  }
}

// -------------------------------------------------------------- dispatch

int decode_rows_per_split(int B, int Hkv, int k) {
  // Enough CTAs to cover 148 SMs about twice, rows a multiple of 32.
  for (int R : {128, 64}) {
    long long ctas = (long long)B * Hkv * ((k + R - 1) / R);
    if (ctas >= 296) return R;
  }
  return 32;
}

size_t decode_smem(int G, int R) {
  int DS = 128 / R;
  size_t f = (size_t)G * kD + (size_t)DS * G * R + 32;
  return f * 4 + 2 * (size_t)R * kLds * 2;
}

template <int G>
cudaError_t launch_decode_g(const uint16_t* q, const uint16_t* kc, const uint16_t* vc,
                            const int32_t* idx, const int32_t* count, int B, int Tk_max, int Hq,
                            int Hkv, int k, float qscale, uint16_t* out, float* lse, float* po,
                            float* pml, unsigned* ticket, int R, int S, cudaStream_t st) {
  size_t smem = decode_smem(G, R);
  cudaError_t e = ensure_dynamic_smem((const void*)attn_decode_kernel<G>, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(S, Hkv, B);
  attn_decode_kernel<G><<<grid, 128, smem, st>>>(q, kc, vc, idx, count, Tk_max, Hq, Hkv, k, R, S,
                                                 qscale, po, pml, ticket, out, lse);
  return cudaGetLastError();
}

size_t prefill_smem() { return (size_t)(16 + 4 * kPTile) * kLds * 2; }

template <int G>
cudaError_t launch_prefill_g(const uint16_t* q, const uint16_t* kc, const uint16_t* vc,
                             const int32_t* idx, const int32_t* count, int B, int T, int Tk_max,
                             int Hq, int Hkv, int k, float qscale, uint16_t* out, float* lse,
                             cudaStream_t st) {
  size_t smem = prefill_smem();
  cudaError_t e = ensure_dynamic_smem((const void*)attn_prefill_kernel<G>, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(T, Hkv, B);
  attn_prefill_kernel<G><<<grid, 128, smem, st>>>(q, kc, vc, idx, count, T, Tk_max, Hq, Hkv, k,
                                                  qscale, out, lse);
  return cudaGetLastError();
}

}  // namespace

static size_t align256a(size_t x) { return (x + 255) & ~size_t(255); }

size_t decode_attn_workspace_bytes(int B, int Hq, int Hkv, int D, int k) {
  (void)D;
  int R = decode_rows_per_split(B, Hkv, k);
  int S = (k + R - 1) / R;
  size_t po = align256a((size_t)B * Hq * S * kD * 4);
  size_t pml = align256a((size_t)B * Hq * S * 2 * 4);
  size_t tk = align256a((size_t)B * Hkv * 4);
  return tk + po + pml;
}

cudaError_t launch_attn_decode(const uint16_t* q, const uint16_t* kc, const uint16_t* vc,
                               const int32_t* idx, const int32_t* count, int B, int Tk_max, int Hq,
                               int Hkv, int k, float scale, uint16_t* out, float* lse, void* ws,
                               cudaStream_t st) {
  if (B <= 0) return cudaSuccess;
  const int R = decode_rows_per_split(B, Hkv, k);
  const int S = (k + R - 1) / R;
  char* p = static_cast<char*>(ws);
  unsigned* ticket = reinterpret_cast<unsigned*>(p);
  p += align256a((size_t)B * Hkv * 4);
  float* po = reinterpret_cast<float*>(p);
  p += align256a((size_t)B * Hq * S * kD * 4);
  float* pml = reinterpret_cast<float*>(p);
  cudaError_t e = cudaMemsetAsync(ticket, 0, (size_t)B * Hkv * 4, st);
  if (e != cudaSuccess) return e;
  const float qscale = scale * kLog2e;
  const int G = Hq / Hkv;
  switch (G) {
#define SA_DEC_CASE(n) \
  case n: return launch_decode_g<n>(q, kc, vc, idx, count, B, Tk_max, Hq, Hkv, k, qscale, out, lse, po, pml, ticket, R, S, st);
    SA_DEC_CASE(1) SA_DEC_CASE(2) SA_DEC_CASE(3) SA_DEC_CASE(4) SA_DEC_CASE(5) SA_DEC_CASE(6)
    SA_DEC_CASE(7) SA_DEC_CASE(8) SA_DEC_CASE(9) SA_DEC_CASE(10) SA_DEC_CASE(11) SA_DEC_CASE(12)
    SA_DEC_CASE(13) SA_DEC_CASE(14) SA_DEC_CASE(15) SA_DEC_CASE(16)
#undef SA_DEC_CASE
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_attn_prefill(const uint16_t* q, const uint16_t* kc, const uint16_t* vc,
                                const int32_t* idx, const int32_t* count, int B, int T, int Tk_max,
                                int Hq, int Hkv, int k, float scale, uint16_t* out, float* lse,
                                cudaStream_t st) {
  if (B <= 0 || T <= 0) return cudaSuccess;
  const float qscale = scale * kLog2e;
  const int G = Hq / Hkv;
  switch (G) {
#define SA_PRE_CASE(n) \
  case n: return launch_prefill_g<n>(q, kc, vc, idx, count, B, T, Tk_max, Hq, Hkv, k, qscale, out, lse, st);
    SA_PRE_CASE(1) SA_PRE_CASE(2) SA_PRE_CASE(3) SA_PRE_CASE(4) SA_PRE_CASE(5) SA_PRE_CASE(6)
    SA_PRE_CASE(7) SA_PRE_CASE(8) SA_PRE_CASE(9) SA_PRE_CASE(10) SA_PRE_CASE(11) SA_PRE_CASE(12)
    SA_PRE_CASE(13) SA_PRE_CASE(14) SA_PRE_CASE(15) SA_PRE_CASE(16)
#undef SA_PRE_CASE
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace sa
