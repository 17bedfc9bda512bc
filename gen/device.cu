// Device-side counter-based input generator (libsagen.so).
//
// Implements, independently of the host numpy code, the generator defined in
// gen/counter_hash.py: SplitMix64 (Steele, Lea and Flood, OOPSLA 2014; the
// output finaliser of the public-domain splitmix64.c) evaluated at counter
// i + 1 of the stream whose state is (seed << 32) | tid.
//   * integers in [lo, hi]: lo + ((out(i) >> 32) * (hi - lo + 1)) >> 32
//   * normal-like reals: Irwin-Hall(12) of 16-bit uniforms taken from
//     out(3i), out(3i+1), out(3i+2), x = (S - 6*65536) / 65536,
//     rounded to bfloat16 with round-to-nearest-even.
// Input generation only: none of the sparse-attention arithmetic lives here.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace {

constexpr unsigned long long kGamma = 0x9E3779B97F4A7C15ull;

__device__ __forceinline__ unsigned long long mix64(unsigned long long z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ unsigned long long stream_out(unsigned long long s0,
                                                         unsigned long long i) {
  return mix64(s0 + (i + 1ull) * kGamma);
}

__global__ void fill_int_kernel(uint16_t* __restrict__ out, long long n,
                                unsigned long long s0, long long start, int lo,
                                unsigned long long span) {
  long long stride = (long long)gridDim.x * blockDim.x;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += stride) {
    unsigned long long u = stream_out(s0, (unsigned long long)(start + e));
    long long v = (long long)(((u >> 32) * span) >> 32) + lo;
    __nv_bfloat16 b = __float2bfloat16_rn((float)v);
    out[e] = *reinterpret_cast<uint16_t*>(&b);
  }
}

__global__ void fill_normal_kernel(uint16_t* __restrict__ out, long long n,
                                   unsigned long long s0, long long start) {
  long long stride = (long long)gridDim.x * blockDim.x;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += stride) {
    unsigned long long i = (unsigned long long)(start + e);
    int s = 0;
#pragma unroll
    for (int r = 0; r < 3; ++r) {
      unsigned long long u = stream_out(s0, 3ull * i + (unsigned long long)r);
#pragma unroll
      for (int c = 0; c < 4; ++c) s += (int)((u >> (16 * c)) & 0xFFFFull);
    }
    float x = (float)(s - 6 * 65536) * (1.0f / 65536.0f);  // exact
    __nv_bfloat16 b = __float2bfloat16_rn(x);
    out[e] = *reinterpret_cast<uint16_t*>(&b);
  }
}

int grid_for(long long n) {
  long long blocks = (n + 255) / 256;
  if (blocks > 148 * 32) blocks = 148 * 32;
  if (blocks < 1) blocks = 1;
  return (int)blocks;
}

}  // namespace

extern "C" {

// Fills out[0..n) with integers in [lo, hi] as bf16 bits; element e uses
// counter start + e of stream (seed, tid).  Returns a cudaError_t value.
int sagen_fill_int_bf16(uint16_t* out, long long n, unsigned int seed, unsigned int tid,
                        long long start, int lo, int hi, cudaStream_t stream) {
  if (n <= 0) return 0;
  if (hi < lo || out == nullptr) return (int)cudaErrorInvalidValue;
  unsigned long long s0 = ((unsigned long long)seed << 32) | (unsigned long long)tid;
  fill_int_kernel<<<grid_for(n), 256, 0, stream>>>(out, n, s0, start, lo,
                                                   (unsigned long long)(hi - lo + 1));
  return (int)cudaGetLastError();
}

// Fills out[0..n) with the Irwin-Hall(12) normal as bf16 bits.
int sagen_fill_normal_bf16(uint16_t* out, long long n, unsigned int seed, unsigned int tid,
                           long long start, cudaStream_t stream) {
  if (n <= 0) return 0;
  if (out == nullptr) return (int)cudaErrorInvalidValue;
  unsigned long long s0 = ((unsigned long long)seed << 32) | (unsigned long long)tid;
  fill_normal_kernel<<<grid_for(n), 256, 0, stream>>>(out, n, s0, start);
  return (int)cudaGetLastError();
}

}  // extern "C"
