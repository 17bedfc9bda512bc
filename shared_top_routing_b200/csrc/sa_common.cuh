// Shared device helpers for libsa.so (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace sa {

constexpr int kMaxK = 4096;          // SA_MAX_K
constexpr int kHistBits = 12;        // first radix digit of a score key
constexpr int kHistBins = 1 << kHistBits;
// Words per row of the one-query histograms: the scorer's histogram of the
// keys' top 12 bits, then the split selection's histogram of the next 12
// bits of the keys in the K-th key's first bin.
constexpr int kHistStride = 2 * kHistBins;

// Long prefill rows are selected in two scoring passes.  The first keeps,
// per row, only the maximum score of each group of g consecutive positions
// (g a power of two <= kGroupMax, the largest with n >= 2 k g, so a row has
// between k+1 and 4k groups while g < kGroupMax).  At least k keys are >= the
// k-th largest group maximum, so it bounds the k-th largest key from below;
// the second pass keeps only the keys at or above that bound.
constexpr int kGroupMax = 64;

// Group size of a row of n candidates for top-k (0: n <= k, every candidate
// is chosen and no bound is needed).
__host__ __device__ __forceinline__ int prefill_group_size(int n, int k) {
  if (n <= k) return 0;
  int g = 1;
  while (g * 2 <= kGroupMax && (long long)n >= 4LL * k * g) g *= 2;
  return g;
}

// Group maxima kept per row for rows of at most n_max candidates (plus one
// 32-column chunk of slack: a chunk past the row end is written whole),
// rounded to 8 entries so rows stay 16-byte aligned.
__host__ __device__ __forceinline__ long long prefill_groups_ld(long long n_max, int k) {
  long long m = 4LL * k;
  const long long m_cap = (n_max + kGroupMax - 1) / kGroupMax;
  if (m_cap > m) m = m_cap;
  return (m + 32 + 7) / 8 * 8;
}

// Order-preserving 32-bit key of an fp32 score: a larger key is a larger
// score.  -0.0 is mapped to +0.0 first so that the two compare equal.
__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t b = __float_as_uint(s);
  b = (b == 0x80000000u) ? 0u : b;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float key_score(uint32_t k) {
  uint32_t b = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(b);
}

// Two packed bfloat16 values (element 0 in the low half) -> two floats.
__device__ __forceinline__ float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ float dot8(uint4 k, const float* q) {
  float s = bf_lo(k.x) * q[0];
  s = fmaf(bf_hi(k.x), q[1], s);
  s = fmaf(bf_lo(k.y), q[2], s);
  s = fmaf(bf_hi(k.y), q[3], s);
  s = fmaf(bf_lo(k.z), q[4], s);
  s = fmaf(bf_hi(k.z), q[5], s);
  s = fmaf(bf_lo(k.w), q[6], s);
  s = fmaf(bf_hi(k.w), q[7], s);
  return s;
}

// fp32 -> bf16 bits, round to nearest even (finite values).
__device__ __forceinline__ uint16_t f2bf(float x) {
  uint32_t b = __float_as_uint(x);
  b += 0x7FFFu + ((b >> 16) & 1u);
  return (uint16_t)(b >> 16);
}

__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
  return (uint32_t)f2bf(lo) | ((uint32_t)f2bf(hi) << 16);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---- cp.async (16-byte, global -> shared) ------------------------------
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
  uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  int n = valid ? 16 : 0;  // src-size 0 zero-fills the destination
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(n));
}
// 4-byte variant (cp.async.ca; .cg takes 16 bytes only).
// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start while the kernel before it drains; it waits in
// pdl_wait() (a no-op for an ordinary launch) until that kernel has completed
// and its writes are visible, so pdl_wait() comes before any global memory
// access.  pdl_launch_dependents() lets the next such kernel start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void cp_async4(void* smem, const void* gmem, bool valid) {
  uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  int n = valid ? 4 : 0;
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(s), "l"(gmem), "r"(n));
}
__device__ __forceinline__ void cp_async8(void* smem, const void* gmem, bool valid) {
  uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  int n = valid ? 8 : 0;
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;\n" ::"r"(s), "l"(gmem), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

// ---- ldmatrix / mma.sync (bf16, fp32 accumulate) -------------------------
__device__ __forceinline__ void ldmatrix_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                            const void* smem) {
  uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(s));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                                  uint32_t& r3, const void* smem) {
  uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(s));
}
// D = A(16x16, row) * B(16x8, col) + D
__device__ __forceinline__ void mma_bf16_16816(float* d, const uint32_t* a, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

}  // namespace sa
