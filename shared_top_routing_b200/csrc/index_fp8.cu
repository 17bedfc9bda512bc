// fp8 (OCP FP8 E4M3) indexer scoring of one-query rows (decode): queries and
// keys stored as e4m3 bytes, half the bytes of the bf16 indexer cache.
//
//   score_fp8_kernel<D, HG, WEIGHTED>  streams the key cache with 16-byte
//       loads straight into mma.sync m16n8k32 e4m3 B fragments.  A dot
//       product is invariant to the order of its terms, so lane (g, t) of a
//       warp loads whole 16-byte chunks 4j+t of key row g (16 keys' elements
//       each) and the query fragments are permuted to match: words x, y of a
//       chunk are (b0, b1) of one MMA and z, w of the next.  One m16n8k32 per
//       32 dims scores 8 keys.
//       - WEIGHTED = false: one indexer head, s = q . k ([LC] "DSA 与
//         IndexShare"), the query as row 0 of the 16-row A side.
//       - WEIGHTED = true: the multi-head form s = sum_h w_h * ReLU(q_h . k),
//         16 heads per A side (rows g and g+8 of a lane's fragment are heads
//         16 hg + g and 16 hg + g + 8); the epilogue takes weight x ReLU per
//         head and sums over heads with three shuffles.
//       Products of e4m3 values are exact in the fp32 accumulator, and for
//       integer-valued inputs every partial sum is an exact fp32 integer.
//       Each CTA scores one chunk of one sequence's candidates, writes the
//       order-preserving 32-bit key of every score and adds a 4096-bin
//       histogram of their top 12 bits to the sequence's, the input of the
//       exact split top-k.  One register buffer of key tiles per warp; three
//       or four CTAs per SM (by register count) keep the loads in flight.

#include <cuda_runtime.h>

#include <algorithm>
#include <stddef.h>
#include <stdint.h>

#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

constexpr int kF8Threads = 256;

__device__ __forceinline__ int f8_row_len(const int32_t* kv_len, int b, int Tk) {
  if (kv_len == nullptr) return Tk;
  const int v = kv_len[b];
  return v < 0 ? 0 : (v > Tk ? Tk : v);
}

// Candidates of the decode query of a sequence of length len: j <= q_pos0, j < len.
__device__ __forceinline__ int f8_n_cand(long long q_pos0, int len) {
  long long n = q_pos0 + 1;
  if (n > len) n = len;
  if (n < 0) n = 0;
  return (int)n;
}

// d += A (16 x 32, row) * B (32 x 8, col), e4m3 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_e4m3_16832(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int D, int HG, bool WEIGHTED>
__global__ void __launch_bounds__(kF8Threads, WEIGHTED ? (HG == 1 ? 3 : 2) : (D == 128 ? 3 : 4))
score_fp8_kernel(const uint8_t* __restrict__ q, const float* __restrict__ wts, const uint8_t* __restrict__ kmat,
                 int H, int Tk_max, int Tk, int q_pos0, const int32_t* __restrict__ kv_len, int chunk,
                 uint32_t* __restrict__ keys, long long ld, uint32_t* __restrict__ hist) {
  pdl_wait();
  pdl_launch_dependents();
  constexpr int J = D / 64;          // 16-byte chunks per lane per key row
  constexpr int U = 2;               // 8-row tiles per warp and load
  constexpr int WARPS = kF8Threads / 32;
  static_assert(D % 64 == 0, "whole 64-byte chunk groups per key row");
  __shared__ uint32_t sh[kHistBins];
  const int b = blockIdx.y;
  const int n = f8_n_cand(q_pos0, f8_row_len(kv_len, b, Tk));
  const int r0 = blockIdx.x * chunk;
  if (r0 >= n) return;
  const int r1 = min(n, r0 + chunk);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tg = lane & 3;
  if (hist != nullptr) {
    for (int i = tid; i < kHistBins; i += kF8Threads) sh[i] = 0;
    __syncthreads();
  }

  // A fragments: for chunk group j, lane (g, tg) holds chunk 4j + tg of the
  // heads of rows g and g + 8 (one head: row 0 only, so lanes with g == 0)
  const uint8_t* qr = q + (long long)b * H * D;
  uint32_t qe[HG][J][4], qo[HG][J][4];
  float w0[HG], w1[HG];
#pragma unroll
  for (int hg = 0; hg < HG; ++hg) {
    const int h0 = WEIGHTED ? 16 * hg + g : 0;
    const int h1 = h0 + 8;
    const bool v0ok = WEIGHTED ? h0 < H : g == 0;
    const bool v1ok = WEIGHTED && h1 < H;
    w0[hg] = WEIGHTED && v0ok ? wts[(long long)b * H + h0] : 0.f;
    w1[hg] = v1ok ? wts[(long long)b * H + h1] : 0.f;
#pragma unroll
    for (int j = 0; j < J; ++j) {
      uint4 v0 = make_uint4(0, 0, 0, 0), v1 = make_uint4(0, 0, 0, 0);
      if (v0ok) v0 = *reinterpret_cast<const uint4*>(qr + (long long)h0 * D + (4 * j + tg) * 16);
      if (v1ok) v1 = *reinterpret_cast<const uint4*>(qr + (long long)h1 * D + (4 * j + tg) * 16);
      qe[hg][j][0] = v0.x; qe[hg][j][1] = v1.x; qe[hg][j][2] = v0.y; qe[hg][j][3] = v1.y;
      qo[hg][j][0] = v0.z; qo[hg][j][1] = v1.z; qo[hg][j][2] = v0.w; qo[hg][j][3] = v1.w;
    }
  }
  const uint4* kb = reinterpret_cast<const uint4*>(kmat + (long long)b * Tk_max * D);
  uint32_t* kout = keys + (long long)b * ld;
  constexpr int kStep = WARPS * 8 * U;
#pragma unroll 1
  for (int base = r0 + warp * 8 * U; base < r1; base += kStep) {
    uint4 v[U][J];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int row = base + u * 8 + g;
#pragma unroll
      for (int j = 0; j < J; ++j)
        v[u][j] = row < r1 ? __ldg(kb + (long long)row * (D / 16) + 4 * j + tg) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float s0 = 0.f, s1 = 0.f;   // keys 2tg and 2tg+1 of the tile
#pragma unroll
      for (int hg = 0; hg < HG; ++hg) {
        float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < J; ++j) {
          if (WEIGHTED) {
            mma_e4m3_16832(c, qe[hg][j], v[u][j].x, v[u][j].y);
            mma_e4m3_16832(c, qo[hg][j], v[u][j].z, v[u][j].w);
          } else {   // rows 8..15 of the A side are zero
            const uint32_t ae[4] = {qe[0][j][0], 0u, qe[0][j][2], 0u};
            const uint32_t ao[4] = {qo[0][j][0], 0u, qo[0][j][2], 0u};
            mma_e4m3_16832(c, ae, v[u][j].x, v[u][j].y);
            mma_e4m3_16832(c, ao, v[u][j].z, v[u][j].w);
          }
        }
        if (WEIGHTED) {
          s0 = fmaf(w0[hg], fmaxf(c[0], 0.f), s0);
          s0 = fmaf(w1[hg], fmaxf(c[2], 0.f), s0);
          s1 = fmaf(w0[hg], fmaxf(c[1], 0.f), s1);
          s1 = fmaf(w1[hg], fmaxf(c[3], 0.f), s1);
        } else {
          s0 = c[0];   // row 0 of C: lanes 0..3
          s1 = c[1];
        }
      }
      if (WEIGHTED) {
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {   // sum over g: the lanes sharing tg
          s0 += __shfl_xor_sync(0xffffffffu, s0, o);
          s1 += __shfl_xor_sync(0xffffffffu, s1, o);
        }
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
  }
  if (hist == nullptr) return;
  __syncthreads();
  uint32_t* hg_row = hist + (long long)b * kHistStride;
  for (int i = tid; i < kHistBins; i += kF8Threads) {
    const uint32_t cnt = sh[i];
    if (cnt) atomicAdd(hg_row + i, cnt);
  }
}

}  // namespace

cudaError_t launch_score_fp8(const uint8_t* q, const float* wts, const uint8_t* kmat, int B, int H, int d, int Tk_max,
                             int Tk, int q_pos0, const int32_t* kv_len, const RowWorkspace& w, bool with_hist,
                             cudaStream_t st) {
  uint32_t* hist = with_hist ? w.hist : nullptr;
  if (B <= 0 || Tk <= 0) return cudaSuccess;
  const long long n_max = std::min<long long>(Tk, (long long)q_pos0 + 1);
  if (n_max <= 0) return cudaSuccess;
  using Kern = void (*)(const uint8_t*, const float*, const uint8_t*, int, int, int, int, const int32_t*, int,
                        uint32_t*, long long, uint32_t*);
  const bool weighted = wts != nullptr;
  const int hg = (H + 15) / 16;
  Kern kern;
  if (d == 128)
    kern = !weighted ? score_fp8_kernel<128, 1, false>
                     : (hg == 1 ? score_fp8_kernel<128, 1, true> : score_fp8_kernel<128, 2, true>);
  else
    kern = !weighted ? score_fp8_kernel<64, 1, false>
                     : (hg == 1 ? score_fp8_kernel<64, 1, true> : score_fp8_kernel<64, 2, true>);
  // one wave of resident CTAs over all rows, each CTA's chunk a whole number
  // of 128-row steps of its eight warps
  const long long slots = (long long)device_sm_count() * std::max(1, device_occupancy((const void*)kern, kF8Threads, 0));
  long long chunk = (n_max * B + slots - 1) / slots;
  chunk = std::max<long long>(128, (chunk + 127) / 128 * 128);
  const dim3 grid((unsigned)((n_max + chunk - 1) / chunk), (unsigned)B);
  const cudaError_t e = launch_pdl(kern, grid, dim3(kF8Threads), 0, st, q, wts, kmat, H, Tk_max, Tk, q_pos0, kv_len,
                                   (int)chunk, w.keys, w.ld, hist);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace sa
