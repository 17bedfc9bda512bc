// Decode attention for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc: a host process that may only pass on
// buffers it was handed (for example across a plugin boundary), or code on a
// path where allocation is not allowed.  They cannot supply the workspace that
// sa_sparse_attn_decode needs.  sa_sparse_attn_decode_noalloc takes the same
// inputs and outputs and uses a scratch array that lives in this library
// instead: a file-scope __device__ array of SA_NOALLOC_SCRATCH_BYTES, present
// on every GPU that loads the library until the process exits.
//
// Host code cannot use the array's name as a device address, so on the first
// call on each device (with that device current) the address is looked up
// once with cudaGetSymbolAddress and cached.  Every call shares the one array:
// calls that overlap on the GPU (for example on two streams) race on it.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/sa.h"
#include "sa_internal.h"

namespace {

constexpr size_t kScratchBytes = SA_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// The scratch: the kernel error word (which must start at zero) and the
// split partials.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_scratch on the current device (looked up once per device).
sa_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    sa::set_last_error("cudaGetDevice failed: %s", cudaGetErrorString(e));
    return SA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    sa::set_last_error("device %d beyond the %d devices the no-allocation scratch supports", dev, kMaxDevices);
    return SA_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || p == nullptr) {
      sa::set_last_error("cudaGetSymbolAddress of the no-allocation scratch failed: %s",
                         cudaGetErrorString(e));
      return SA_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return SA_OK;
}

}  // namespace

extern "C" sa_status sa_sparse_attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                                   const int32_t* idx, const int32_t* count, int B,
                                                   int Tk_max, int Hq, int Hkv, int D, int k, float scale,
                                                   void* out, float* lse, sa_stream_t stream) {
  // every argument is checked before anything runs on the GPU
  sa_status st = sa::check_decode_args(q, k_cache, v_cache, idx, count, B, Tk_max, Hq, Hkv, D, k, out);
  if (st != SA_OK) return st;
  if (B > 0) {
    const size_t need = sa_sparse_attn_decode_workspace(B, Hq, Hkv, D, k);
    if (need > kScratchBytes) {
      sa::set_last_error(
          "this shape needs %zu bytes of scratch; the no-allocation entry point holds %zu "
          "(use sa_sparse_attn_decode with a caller workspace)",
          need, kScratchBytes);
      return SA_ERR_UNSUPPORTED;
    }
  }
  void* scratch = nullptr;
  if (B > 0) {
    st = scratch_address(&scratch);
    if (st != SA_OK) return st;
    // The error word must start at zero; clear it on the call's stream (no
    // allocation involved).
    cudaError_t e = cudaMemsetAsync(scratch, 0, sa::decode_attn_zero_bytes(B, Hkv, k),
                                    reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
      sa::set_last_error("clearing the no-allocation scratch failed: %s", cudaGetErrorString(e));
      return SA_ERR_CUDA;
    }
  }
  return sa_sparse_attn_decode(q, k_cache, v_cache, idx, count, B, Tk_max, Hq, Hkv, D, k, scale, out, lse,
                               scratch, kScratchBytes, stream);
}
