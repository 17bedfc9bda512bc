// C ABI of libsa.so: host-side validation, workspace sizing, dispatch and
// the shared index cache.  Declarations and contracts are in include/sa.h.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <map>
#include <mutex>
#include <set>
#include <string>
#include <utility>
#include <vector>

#include "../../include/sa.h"
#include "sa_common.cuh"
#include "sa_internal.h"

namespace {

thread_local std::string g_last_error;

sa_status fail(sa_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

sa_status ok() {
  g_last_error.clear();
  return SA_OK;
}

sa_status cuda_fail(cudaError_t e, const char* where) {
  return fail(SA_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

sa_status check_ws(const void* ws, size_t ws_bytes, size_t need) {
  if (need == 0) return SA_OK;
  if (ws == nullptr) return fail(SA_ERR_WORKSPACE, "workspace is NULL but %zu bytes are needed", need);
  if (!aligned(ws, SA_WS_ALIGN)) return fail(SA_ERR_WORKSPACE, "workspace is not %d-byte aligned", SA_WS_ALIGN);
  if (ws_bytes < need)
    return fail(SA_ERR_WORKSPACE, "workspace has %zu bytes, %zu are needed", ws_bytes, need);
  return SA_OK;
}

cudaStream_t as_cuda(sa_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

sa_status validate_index(const void* q_idx, const void* k_idx, int B, int Tq, int Tk, int Tk_max,
                         int d, int k, const int32_t* idx_out, const int32_t* count_out) {
  if (B < 0 || Tq < 1 || Tk < 0 || Tk_max < 0 || Tk > Tk_max)
    return fail(SA_ERR_INVALID_ARG, "bad sizes: B=%d Tq=%d Tk=%d Tk_max=%d (need B>=0, Tq>=1, 0<=Tk<=Tk_max)",
                B, Tq, Tk, Tk_max);
  if (k < 1) return fail(SA_ERR_INVALID_ARG, "k=%d must be >= 1", k);
  if (k > SA_MAX_K) return fail(SA_ERR_UNSUPPORTED, "k=%d exceeds SA_MAX_K=%d", k, SA_MAX_K);
  if (d != 64 && d != 128) return fail(SA_ERR_UNSUPPORTED, "d=%d unsupported (64 or 128)", d);
  if ((long long)Tk_max * d > (1ll << 40))
    return fail(SA_ERR_UNSUPPORTED, "Tk_max=%d too large", Tk_max);
  if (B == 0) return SA_OK;
  if (!q_idx || !k_idx || !idx_out || !count_out)
    return fail(SA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned(q_idx, 16) || !aligned(k_idx, 16))
    return fail(SA_ERR_INVALID_ARG, "q_idx and k_idx must be 16-byte aligned");
  if (!aligned(idx_out, 4) || !aligned(count_out, 4))
    return fail(SA_ERR_INVALID_ARG, "idx_out and count_out must be 4-byte aligned");
  return SA_OK;
}

sa_status validate_attn(const void* q, const void* kc, const void* vc, const int32_t* idx,
                        const int32_t* count, int B, int T, int Tk_max, int Hq, int Hkv, int D,
                        int k, const void* out) {
  if (B < 0 || T < 0 || Tk_max < 1 || Hq < 1 || Hkv < 1 || k < 1)
    return fail(SA_ERR_INVALID_ARG, "bad sizes: B=%d T=%d Tk_max=%d Hq=%d Hkv=%d k=%d", B, T,
                Tk_max, Hq, Hkv, k);
  if (D != SA_HEAD_DIM) return fail(SA_ERR_UNSUPPORTED, "D=%d unsupported (only %d)", D, SA_HEAD_DIM);
  if (Hq % Hkv != 0) return fail(SA_ERR_INVALID_ARG, "Hq=%d is not a multiple of Hkv=%d", Hq, Hkv);
  if (Hq / Hkv > 16) return fail(SA_ERR_UNSUPPORTED, "Hq/Hkv=%d > 16 unsupported", Hq / Hkv);
  if (k > (1 << 20)) return fail(SA_ERR_UNSUPPORTED, "k=%d too large", k);
  if (B == 0 || T == 0) return SA_OK;
  if (!q || !kc || !vc || !idx || !count || !out) return fail(SA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned(q, 16) || !aligned(kc, 16) || !aligned(vc, 16) || !aligned(out, 16))
    return fail(SA_ERR_INVALID_ARG, "q, k_cache, v_cache and out must be 16-byte aligned");
  if (!aligned(idx, 4) || !aligned(count, 4)) return fail(SA_ERR_INVALID_ARG, "idx/count misaligned");
  return SA_OK;
}

}  // namespace

namespace sa {

sa_status check_decode_args(const void* q, const void* kc, const void* vc, const int32_t* idx,
                            const int32_t* count, int B, int Tk_max, int Hq, int Hkv, int D, int k,
                            const void* out) {
  sa_status st = validate_attn(q, kc, vc, idx, count, B, 1, Tk_max, Hq, Hkv, D, k, out);
  if (st != SA_OK) return st;
  if ((long long)B * Hkv > SA_DECODE_MAX_PAIRS)
    return fail(SA_ERR_UNSUPPORTED, "B*Hkv=%lld exceeds %d", (long long)B * Hkv, SA_DECODE_MAX_PAIRS);
  return SA_OK;
}

void set_last_error(const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
}

cudaError_t ensure_dynamic_smem(const void* func, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, size_t> done;   // largest size set so far
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  auto key = std::make_pair(func, dev);
  auto it = done.find(key);
  if (it != done.end() && it->second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) done[key] = bytes;
  return e;
}

namespace {
constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];
}  // namespace

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
  const bool cached = dev >= 0 && dev < kMaxDevices;
  if (cached) {
    const int v = g_sm_count[dev].load(std::memory_order_relaxed);
    if (v > 0) return v;
  }
  int n = 0;
  if (dev >= 0) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  n = n > 0 ? n : 148;
  if (cached) g_sm_count[dev].store(n, std::memory_order_relaxed);
  return n;
}

int device_occupancy(const void* func, int threads, size_t smem) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
  std::lock_guard<std::mutex> lock(mu);
  auto key = std::make_pair(func, dev);
  auto it = done.find(key);
  if (it != done.end()) return it->second;
  int o = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, func, threads, smem) != cudaSuccess) o = 0;
  o = o > 0 ? o : 1;
  done[key] = o;
  return o;
}

}  // namespace sa

// =============================================================== C ABI

extern "C" {

const char* sa_status_string(sa_status s) {
  switch (s) {
    case SA_OK: return "SA_OK";
    case SA_ERR_INVALID_ARG: return "SA_ERR_INVALID_ARG: invalid argument";
    case SA_ERR_UNSUPPORTED: return "SA_ERR_UNSUPPORTED: shape not supported by this build";
    case SA_ERR_WORKSPACE: return "SA_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case SA_ERR_CUDA: return "SA_ERR_CUDA: CUDA runtime or launch failure";
    case SA_ERR_TIMEOUT: return "SA_ERR_TIMEOUT: a kernel wait gave up";
    case SA_ERR_STALE_INDEX: return "SA_ERR_STALE_INDEX: shared layer read before its full layer wrote";
  }
  return "unknown sa_status";
}

const char* sa_last_error(void) { return g_last_error.c_str(); }

int sa_version(void) { return 100; }

// ------------------------------------------------------------- indexer

size_t sa_index_score_topk_workspace(int B, int Tq, int Tk_max, int d, int k) {
  (void)d;
  (void)k;
  if (B <= 0 || Tq <= 0 || Tk_max < 0) return 0;
  if (Tq == 1) {
    const int mode = sa::finish_mode_for(Tk_max);
    return sa::row_workspace_bytes(B, Tk_max, mode == sa::kFinishSplit, mode != sa::kFinishDirect) + sa::kWsCanary;
  }
  const int rows = sa::prefill_rows_per_launch(B, Tq, Tk_max, k);
  return sa::prefill_workspace_bytes(B * rows, Tk_max, k) + sa::kWsCanary;
}

sa_status sa_index_score_topk(const void* q_idx, const void* k_idx, int B, int Tq, int Tk,
                              int Tk_max, int d, int k, int q_pos0, const int32_t* kv_len,
                              int32_t* idx_out, int32_t* count_out, float* score_out, void* ws,
                              size_t ws_bytes, sa_stream_t stream) {
  sa_status st = validate_index(q_idx, k_idx, B, Tq, Tk, Tk_max, d, k, idx_out, count_out);
  if (st != SA_OK) return st;
  if (B == 0) return ok();
  const size_t need = sa_index_score_topk_workspace(B, Tq, Tk_max, d, k);
  if ((st = check_ws(ws, ws_bytes, need)) != SA_OK) return st;
  cudaStream_t cs = as_cuda(stream);
  cudaError_t e;
  if ((e = sa::dbg_arm(ws, need - sa::kWsCanary, cs)) != cudaSuccess) return cuda_fail(e, "debug canary");
  const uint16_t* q = static_cast<const uint16_t*>(q_idx);
  const uint16_t* km = static_cast<const uint16_t*>(k_idx);
  sa::FinishOut out;
  out.idx = idx_out;
  out.count = count_out;
  out.score = score_out;
  if (Tq == 1) {
    const int mode = sa::finish_mode_for(Tk_max);
    sa::RowWorkspace w;
    sa::carve_row_workspace(ws, B, Tk_max, mode == sa::kFinishSplit, mode != sa::kFinishDirect, &w);
    const bool hist = mode != sa::kFinishDirect;
    if (hist && w.hist_zero_bytes &&
        (e = cudaMemsetAsync(w.hist, 0, w.hist_zero_bytes, cs)) != cudaSuccess)
      return cuda_fail(e, "memset");
    if ((e = sa::launch_score_decode(q, km, B, d, Tk_max, Tk, q_pos0, kv_len, w, hist, cs)) != cudaSuccess)
      return cuda_fail(e, "score_decode launch");
    if (mode == sa::kFinishSplit) {
      if ((e = sa::launch_split_topk(B, 1, 0, 1, Tk, q_pos0, kv_len, k, w, out, cs)) != cudaSuccess)
        return cuda_fail(e, "split top-k launch");
    } else if ((e = sa::launch_finish(B, 1, 0, 1, Tk, q_pos0, kv_len, k, w, mode, out, cs)) != cudaSuccess) {
      return cuda_fail(e, "finish launch");
    }
    if ((e = sa::dbg_check(ws, need - sa::kWsCanary, 1, cs)) != cudaSuccess) return cuda_fail(e, "debug canary");
    return ok();
  }
  const int rows = sa::prefill_rows_per_launch(B, Tq, Tk_max, k);
  sa::RowWorkspace w;
  sa::carve_prefill_workspace(ws, B * rows, Tk_max, k, &w);
  for (int t0 = 0; t0 < Tq; t0 += rows) {
    const int nr = (Tq - t0 < rows) ? Tq - t0 : rows;
    const long long n_max = std::min<long long>(Tk, (long long)q_pos0 + t0 + nr);
    if (n_max <= sa::kBoundedMinCand) {
      // short rows: every score's key, then one CTA per row selects
      if ((e = sa::launch_score_prefill(q, km, B, Tq, d, Tk_max, Tk, q_pos0, kv_len, t0, nr, k, sa::kScoreKeys, w,
                                        cs)) != cudaSuccess)
        return cuda_fail(e, "score_prefill launch");
      if ((e = sa::launch_finish(B, nr, t0, Tq, Tk, q_pos0, kv_len, k, w, sa::kFinishDirect, out, cs)) != cudaSuccess)
        return cuda_fail(e, "finish launch");
    } else {
      // long rows: group maxima, the per-row bound, the keys at or above it,
      // then the exact selection among those
      if ((e = sa::launch_score_prefill(q, km, B, Tq, d, Tk_max, Tk, q_pos0, kv_len, t0, nr, k, sa::kScoreGroupMax,
                                        w, cs)) != cudaSuccess)
        return cuda_fail(e, "score_prefill launch");
      if ((e = sa::launch_prefill_threshold(B, nr, t0, Tk, q_pos0, kv_len, k, w, cs)) != cudaSuccess)
        return cuda_fail(e, "threshold launch");
      if ((e = sa::launch_score_prefill(q, km, B, Tq, d, Tk_max, Tk, q_pos0, kv_len, t0, nr, k, sa::kScoreCand, w,
                                        cs)) != cudaSuccess)
        return cuda_fail(e, "score_prefill launch");
      if ((e = sa::launch_finish(B, nr, t0, Tq, Tk, q_pos0, kv_len, k, w, sa::kFinishCandRows, out, cs)) !=
          cudaSuccess)
        return cuda_fail(e, "finish launch");
    }
  }
  if ((e = sa::dbg_check(ws, need - sa::kWsCanary, 1, cs)) != cudaSuccess) return cuda_fail(e, "debug canary");
  return ok();
}

// --------------------------------------------------- multi-head indexer

size_t sa_index_score_topk_mh_workspace(int B, int Tq, int Tk_max, int H, int d, int k) {
  (void)d;
  (void)k;
  if (B <= 0 || Tq <= 0 || Tk_max < 0 || H < 1) return 0;
  const int rows = sa::mh_rows_per_launch(B, Tq, Tk_max);
  return sa::row_workspace_bytes(B * rows, Tk_max, true, true) + sa::kWsCanary;
}

sa_status sa_index_score_topk_mh(const void* q_idx, const float* w, const void* k_idx, int B, int Tq, int H,
                                 int Tk, int Tk_max, int d, int k, int q_pos0, const int32_t* kv_len,
                                 int32_t* idx_out, int32_t* count_out, float* score_out, void* ws,
                                 size_t ws_bytes, sa_stream_t stream) {
  sa_status st = validate_index(q_idx, k_idx, B, Tq, Tk, Tk_max, d, k, idx_out, count_out);
  if (st != SA_OK) return st;
  if (H < 1) return fail(SA_ERR_INVALID_ARG, "H=%d must be >= 1", H);
  if (H > sa::mh_max_heads(d))
    return fail(SA_ERR_UNSUPPORTED, "H=%d indexer heads exceed %d for d=%d", H, sa::mh_max_heads(d), d);
  if (B == 0) return ok();
  if (w == nullptr) return fail(SA_ERR_INVALID_ARG, "NULL weight pointer");
  if (!aligned(w, 4)) return fail(SA_ERR_INVALID_ARG, "w must be 4-byte aligned");
  const size_t need = sa_index_score_topk_mh_workspace(B, Tq, Tk_max, H, d, k);
  if ((st = check_ws(ws, ws_bytes, need)) != SA_OK) return st;
  cudaStream_t cs = as_cuda(stream);
  const int rows = sa::mh_rows_per_launch(B, Tq, Tk_max);
  sa::RowWorkspace wsp;
  sa::carve_row_workspace(ws, B * rows, Tk_max, true, true, &wsp);
  cudaError_t e;
  if ((e = sa::dbg_arm(ws, need - sa::kWsCanary, cs)) != cudaSuccess) return cuda_fail(e, "debug canary");
  if (wsp.hist_zero_bytes && (e = cudaMemsetAsync(wsp.hist, 0, wsp.hist_zero_bytes, cs)) != cudaSuccess)
    return cuda_fail(e, "memset");
  sa::FinishOut out;
  out.idx = idx_out;
  out.count = count_out;
  out.score = score_out;
  const uint16_t* q = static_cast<const uint16_t*>(q_idx);
  const uint16_t* km = static_cast<const uint16_t*>(k_idx);
  for (int t0 = 0; t0 < Tq; t0 += rows) {
    const int nr = (Tq - t0 < rows) ? Tq - t0 : rows;
    const long long n_max = std::min<long long>(Tk, (long long)q_pos0 + t0 + nr);
    const bool split = n_max > sa::kDirectMaxCand;   // short rows: one CTA holds the whole row
    if ((e = sa::launch_score_mh(q, w, km, B, H, d, nr, t0, Tq, Tk_max, Tk, q_pos0, kv_len, wsp, split, cs)) !=
        cudaSuccess)
      return cuda_fail(e, "multi-head score launch");
    if (split) {
      if ((e = sa::launch_split_topk(B, nr, t0, Tq, Tk, q_pos0, kv_len, k, wsp, out, cs)) != cudaSuccess)
        return cuda_fail(e, "split top-k launch");
    } else if ((e = sa::launch_finish(B, nr, t0, Tq, Tk, q_pos0, kv_len, k, wsp, sa::kFinishDirect, out, cs)) !=
               cudaSuccess) {
      return cuda_fail(e, "finish launch");
    }
  }
  if ((e = sa::dbg_check(ws, need - sa::kWsCanary, 2, cs)) != cudaSuccess) return cuda_fail(e, "debug canary");
  return ok();
}

size_t sa_index_score_topk_fp8_workspace(int B, int Tk_max, int H, int d, int k) {
  (void)H;
  return sa_index_score_topk_workspace(B, 1, Tk_max, d, k);
}

sa_status sa_index_score_topk_fp8(const void* q_idx, const float* w, const void* k_idx, int B, int H, int Tk,
                                  int Tk_max, int d, int k, int q_pos0, const int32_t* kv_len, int32_t* idx_out,
                                  int32_t* count_out, float* score_out, void* ws, size_t ws_bytes,
                                  sa_stream_t stream) {
  sa_status st = validate_index(q_idx, k_idx, B, 1, Tk, Tk_max, d, k, idx_out, count_out);
  if (st != SA_OK) return st;
  if (H < 1) return fail(SA_ERR_INVALID_ARG, "H=%d must be >= 1", H);
  if (w == nullptr && H != 1) return fail(SA_ERR_INVALID_ARG, "H=%d heads need weights (w is NULL)", H);
  if (H > sa::kFp8MaxHeads) return fail(SA_ERR_UNSUPPORTED, "H=%d indexer heads exceed %d", H, sa::kFp8MaxHeads);
  if (B == 0) return ok();
  if (w != nullptr && !aligned(w, 4)) return fail(SA_ERR_INVALID_ARG, "w must be 4-byte aligned");
  const size_t need = sa_index_score_topk_fp8_workspace(B, Tk_max, H, d, k);
  if ((st = check_ws(ws, ws_bytes, need)) != SA_OK) return st;
  cudaStream_t cs = as_cuda(stream);
  cudaError_t e;
  if ((e = sa::dbg_arm(ws, need - sa::kWsCanary, cs)) != cudaSuccess) return cuda_fail(e, "debug canary");
  const int mode = sa::finish_mode_for(Tk_max);
  sa::RowWorkspace wsp;
  sa::carve_row_workspace(ws, B, Tk_max, mode == sa::kFinishSplit, mode != sa::kFinishDirect, &wsp);
  const bool hist = mode != sa::kFinishDirect;
  if (hist && wsp.hist_zero_bytes && (e = cudaMemsetAsync(wsp.hist, 0, wsp.hist_zero_bytes, cs)) != cudaSuccess)
    return cuda_fail(e, "memset");
  if ((e = sa::launch_score_fp8(static_cast<const uint8_t*>(q_idx), w, static_cast<const uint8_t*>(k_idx), B, H, d,
                                Tk_max, Tk, q_pos0, kv_len, wsp, hist, cs)) != cudaSuccess)
    return cuda_fail(e, "fp8 score launch");
  sa::FinishOut out;
  out.idx = idx_out;
  out.count = count_out;
  out.score = score_out;
  if (mode == sa::kFinishSplit) {
    if ((e = sa::launch_split_topk(B, 1, 0, 1, Tk, q_pos0, kv_len, k, wsp, out, cs)) != cudaSuccess)
      return cuda_fail(e, "split top-k launch");
  } else if ((e = sa::launch_finish(B, 1, 0, 1, Tk, q_pos0, kv_len, k, wsp, mode, out, cs)) != cudaSuccess) {
    return cuda_fail(e, "finish launch");
  }
  if ((e = sa::dbg_check(ws, need - sa::kWsCanary, 5, cs)) != cudaSuccess) return cuda_fail(e, "debug canary");
  return ok();
}

sa_status sa_workspace_status(const void* ws, sa_stream_t stream) {
  if (ws == nullptr) return fail(SA_ERR_INVALID_ARG, "NULL workspace");
  cudaStream_t cs = as_cuda(stream);
  int word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, cs);
  if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
  if (e != cudaSuccess) return cuda_fail(e, "reading the error word");
  if (word != 0) return fail(SA_ERR_TIMEOUT, "a pipeline wait gave up (wait code %d)", word);
  return ok();
}

// ----------------------------------------------------------- attention

sa_status sa_sparse_attn_prefill(const void* q, const void* k_cache, const void* v_cache,
                                 const int32_t* idx, const int32_t* count, int B, int T, int Tk_max,
                                 int Hq, int Hkv, int D, int k, float scale, void* out, float* lse,
                                 sa_stream_t stream) {
  sa_status st = validate_attn(q, k_cache, v_cache, idx, count, B, T, Tk_max, Hq, Hkv, D, k, out);
  if (st != SA_OK) return st;
  if (B == 0 || T == 0) return ok();
  const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)D);
  cudaError_t e = sa::launch_attn_prefill(
      static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k_cache),
      static_cast<const uint16_t*>(v_cache), idx, count, B, T, Tk_max, Hq, Hkv, k, sc,
      static_cast<uint16_t*>(out), lse, as_cuda(stream));
  if (e != cudaSuccess) return cuda_fail(e, "attn_prefill launch");
  return ok();
}

size_t sa_sparse_attn_decode_workspace(int B, int Hq, int Hkv, int D, int k) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || k <= 0) return 0;
  return sa::decode_attn_workspace_bytes(B, Hq, Hkv, D, k) + sa::kWsCanary;
}

sa_status sa_sparse_attn_decode(const void* q, const void* k_cache, const void* v_cache,
                                const int32_t* idx, const int32_t* count, int B, int Tk_max, int Hq,
                                int Hkv, int D, int k, float scale, void* out, float* lse, void* ws,
                                size_t ws_bytes, sa_stream_t stream) {
  sa_status st = validate_attn(q, k_cache, v_cache, idx, count, B, 1, Tk_max, Hq, Hkv, D, k, out);
  if (st != SA_OK) return st;
  if (B == 0) return ok();
  if ((long long)B * Hkv > SA_DECODE_MAX_PAIRS)
    return fail(SA_ERR_UNSUPPORTED, "B*Hkv=%lld exceeds %d", (long long)B * Hkv, SA_DECODE_MAX_PAIRS);
  const size_t need = sa_sparse_attn_decode_workspace(B, Hq, Hkv, D, k);
  if ((st = check_ws(ws, ws_bytes, need)) != SA_OK) return st;
  const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)D);
  cudaError_t e = sa::dbg_arm(ws, need - sa::kWsCanary, as_cuda(stream));
  if (e != cudaSuccess) return cuda_fail(e, "debug canary");
  e = sa::launch_attn_decode(
      static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k_cache),
      static_cast<const uint16_t*>(v_cache), idx, count, B, Tk_max, Hq, Hkv, k, sc,
      static_cast<uint16_t*>(out), lse, ws, as_cuda(stream));
  if (e != cudaSuccess) return cuda_fail(e, "attn_decode launch");
  if ((e = sa::dbg_check(ws, need - sa::kWsCanary, 3, as_cuda(stream))) != cudaSuccess)
    return cuda_fail(e, "debug canary");
  return ok();
}

// ------------------------------------------------------- gather once

sa_status sa_gather_rows(const void* k_cache, const void* v_cache, const int32_t* idx, const int32_t* count,
                         int B, int Tk_max, int Hkv, int D, int k, void* k_rows, void* v_rows,
                         sa_stream_t stream) {
  if (B < 0 || Tk_max < 1 || Hkv < 1 || k < 1)
    return fail(SA_ERR_INVALID_ARG, "bad sizes: B=%d Tk_max=%d Hkv=%d k=%d", B, Tk_max, Hkv, k);
  if (D != SA_HEAD_DIM) return fail(SA_ERR_UNSUPPORTED, "D=%d unsupported (only %d)", D, SA_HEAD_DIM);
  if (k > (1 << 20)) return fail(SA_ERR_UNSUPPORTED, "k=%d too large", k);
  if (B == 0) return ok();
  if (!k_cache || !v_cache || !idx || !count || !k_rows || !v_rows) return fail(SA_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(k_rows, 16) || !aligned(v_rows, 16))
    return fail(SA_ERR_INVALID_ARG, "caches and row buffers must be 16-byte aligned");
  if (!aligned(idx, 4) || !aligned(count, 4)) return fail(SA_ERR_INVALID_ARG, "idx/count misaligned");
  const cudaError_t e = sa::launch_gather_rows(
      static_cast<const uint16_t*>(k_cache), static_cast<const uint16_t*>(v_cache), idx, count, B, Tk_max, Hkv, k,
      static_cast<uint16_t*>(k_rows), static_cast<uint16_t*>(v_rows), as_cuda(stream));
  if (e != cudaSuccess) return cuda_fail(e, "gather_rows launch");
  return ok();
}

sa_status sa_sparse_attn_decode_rows(const void* q, const void* k_rows, const void* v_rows, const int32_t* count,
                                     int B, int Hq, int Hkv, int D, int k, float scale, void* out, float* lse,
                                     void* ws, size_t ws_bytes, sa_stream_t stream) {
  if (B < 0 || Hq < 1 || Hkv < 1 || k < 1)
    return fail(SA_ERR_INVALID_ARG, "bad sizes: B=%d Hq=%d Hkv=%d k=%d", B, Hq, Hkv, k);
  if (Hkv > 8) return fail(SA_ERR_UNSUPPORTED, "Hkv=%d > 8 unsupported for compact rows", Hkv);
  // idx is not read for compact rows; any aligned non-null pointer passes validation
  sa_status st = validate_attn(q, k_rows, v_rows, count, count, B, 1, k, Hq, Hkv, D, k, out);
  if (st != SA_OK) return st;
  if (B == 0) return ok();
  if ((long long)B * Hkv > SA_DECODE_MAX_PAIRS)
    return fail(SA_ERR_UNSUPPORTED, "B*Hkv=%lld exceeds %d", (long long)B * Hkv, SA_DECODE_MAX_PAIRS);
  const size_t need = sa_sparse_attn_decode_workspace(B, Hq, Hkv, D, k);
  if ((st = check_ws(ws, ws_bytes, need)) != SA_OK) return st;
  const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)D);
  cudaError_t e = sa::dbg_arm(ws, need - sa::kWsCanary, as_cuda(stream));
  if (e != cudaSuccess) return cuda_fail(e, "debug canary");
  e = sa::launch_attn_decode(
      static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k_rows), static_cast<const uint16_t*>(v_rows),
      nullptr, count, B, k, Hq, Hkv, k, sc, static_cast<uint16_t*>(out), lse, ws, as_cuda(stream));
  if (e != cudaSuccess) return cuda_fail(e, "attn_decode_rows launch");
  if ((e = sa::dbg_check(ws, need - sa::kWsCanary, 3, as_cuda(stream))) != cudaSuccess)
    return cuda_fail(e, "debug canary");
  return ok();
}

// ---------------------------------------------------------------- gist

size_t sa_gist_route_unfold_workspace(int B, int n_chunks, int d, int k_chunks) {
  (void)d;
  (void)k_chunks;
  if (B <= 0 || n_chunks < 0) return 0;
  const int mode = sa::finish_mode_for(n_chunks);
  return sa::row_workspace_bytes(B, n_chunks, mode == sa::kFinishSplit, mode != sa::kFinishDirect) + sa::kWsCanary;
}

sa_status sa_gist_route_unfold(const void* q_route, const void* gist_key, int B, int n_chunks,
                               int chunk_len, int d, int k_chunks, const int32_t* partial_len,
                               int32_t* rows_out, int32_t* count_out, int32_t* chunks_out, void* ws,
                               size_t ws_bytes, sa_stream_t stream) {
  if (B < 0 || n_chunks < 0) return fail(SA_ERR_INVALID_ARG, "bad sizes: B=%d n_chunks=%d", B, n_chunks);
  if (chunk_len < 1 || chunk_len > 256)
    return fail(SA_ERR_UNSUPPORTED, "chunk_len=%d unsupported (1..256)", chunk_len);
  if (k_chunks < 1) return fail(SA_ERR_INVALID_ARG, "k_chunks=%d must be >= 1", k_chunks);
  if (k_chunks > SA_MAX_K) return fail(SA_ERR_UNSUPPORTED, "k_chunks=%d exceeds SA_MAX_K", k_chunks);
  if (d != 64 && d != 128) return fail(SA_ERR_UNSUPPORTED, "d=%d unsupported (64 or 128)", d);
  if ((long long)(n_chunks + 1) * (chunk_len + 1) > 0x7FFFFFFFll)
    return fail(SA_ERR_UNSUPPORTED, "row ids overflow int32");
  if (B == 0) return ok();
  if (!q_route || !gist_key || !rows_out || !count_out) return fail(SA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned(q_route, 16) || !aligned(gist_key, 16))
    return fail(SA_ERR_INVALID_ARG, "q_route and gist_key must be 16-byte aligned");
  const size_t need = sa_gist_route_unfold_workspace(B, n_chunks, d, k_chunks);
  sa_status st = check_ws(ws, ws_bytes, need);
  if (st != SA_OK) return st;
  cudaStream_t cs = as_cuda(stream);
  const int mode = sa::finish_mode_for(n_chunks);
  sa::RowWorkspace w;
  sa::carve_row_workspace(ws, B, n_chunks, mode == sa::kFinishSplit, mode != sa::kFinishDirect, &w);
  cudaError_t e;
  if ((e = sa::dbg_arm(ws, need - sa::kWsCanary, cs)) != cudaSuccess) return cuda_fail(e, "debug canary");
  const bool hist = mode != sa::kFinishDirect;
  if (hist && w.hist_zero_bytes && (e = cudaMemsetAsync(w.hist, 0, w.hist_zero_bytes, cs)) != cudaSuccess)
    return cuda_fail(e, "memset");
  const int q_pos0 = n_chunks - 1;  // every complete chunk is a candidate
  if ((e = sa::launch_score_decode(static_cast<const uint16_t*>(q_route),
                                   static_cast<const uint16_t*>(gist_key), B, d, n_chunks, n_chunks,
                                   q_pos0, nullptr, w, hist, cs)) != cudaSuccess)
    return cuda_fail(e, "gist score launch");
  sa::FinishOut out;
  out.count = count_out;
  out.rows = rows_out;
  out.rows_stride = k_chunks * (chunk_len + 1) + chunk_len;
  out.chunk_len = chunk_len;
  out.n_chunks = n_chunks;
  out.partial_len = partial_len;
  out.chunks = chunks_out;
  if (mode == sa::kFinishSplit) {
    if ((e = sa::launch_split_topk(B, 1, 0, 1, n_chunks, q_pos0, nullptr, k_chunks, w, out, cs)) != cudaSuccess)
      return cuda_fail(e, "gist split top-k launch");
  } else if ((e = sa::launch_finish(B, 1, 0, 1, n_chunks, q_pos0, nullptr, k_chunks, w, mode, out, cs)) !=
             cudaSuccess) {
    return cuda_fail(e, "gist finish launch");
  }
  if ((e = sa::dbg_check(ws, need - sa::kWsCanary, 4, cs)) != cudaSuccess) return cuda_fail(e, "debug canary");
  return ok();
}

sa_status sa_hier_gist_route_unfold(const void* q_route, const void* meta_key, const void* gist_key, int B,
                                    int n_chunks, int chunk_len, int group_size, int d, int k_groups, int k_chunks,
                                    const int32_t* partial_len, int32_t* rows_out, int32_t* count_out,
                                    int32_t* chunks_out, int32_t* groups_out, sa_stream_t stream) {
  if (B < 0 || n_chunks < 0) return fail(SA_ERR_INVALID_ARG, "bad sizes: B=%d n_chunks=%d", B, n_chunks);
  if (group_size < 1) return fail(SA_ERR_INVALID_ARG, "group_size=%d must be >= 1", group_size);
  if (chunk_len < 1 || chunk_len > 256)
    return fail(SA_ERR_UNSUPPORTED, "chunk_len=%d unsupported (1..256)", chunk_len);
  if (k_groups < 1 || k_chunks < 1) return fail(SA_ERR_INVALID_ARG, "k_groups and k_chunks must be >= 1");
  if (k_chunks > SA_MAX_K) return fail(SA_ERR_UNSUPPORTED, "k_chunks=%d exceeds SA_MAX_K", k_chunks);
  if (d != 64 && d != 128) return fail(SA_ERR_UNSUPPORTED, "d=%d unsupported (64 or 128)", d);
  const long long n_groups = n_chunks / group_size;
  const long long cand = std::min<long long>(k_groups, n_groups) * group_size + (n_chunks - n_groups * group_size);
  if (n_groups > sa::kHierMax || cand > sa::kHierMax)
    return fail(SA_ERR_UNSUPPORTED, "%lld groups / %lld candidate chunks exceed %d", n_groups, cand, sa::kHierMax);
  if ((long long)(n_chunks + 1) * (chunk_len + 1) > 0x7FFFFFFFll) return fail(SA_ERR_UNSUPPORTED, "row ids overflow int32");
  if (B == 0) return ok();
  if (!q_route || !gist_key || !rows_out || !count_out || (n_groups > 0 && !meta_key))
    return fail(SA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned(q_route, 16) || !aligned(gist_key, 16) || (meta_key && !aligned(meta_key, 16)))
    return fail(SA_ERR_INVALID_ARG, "q_route, meta_key and gist_key must be 16-byte aligned");
  sa::FinishOut out;
  out.count = count_out;
  out.rows = rows_out;
  out.rows_stride = k_chunks * (chunk_len + 1) + chunk_len;
  out.chunk_len = chunk_len;
  out.n_chunks = n_chunks;
  out.partial_len = partial_len;
  out.chunks = chunks_out;
  const cudaError_t e = sa::launch_hier_gist(
      static_cast<const uint16_t*>(q_route), static_cast<const uint16_t*>(meta_key),
      static_cast<const uint16_t*>(gist_key), B, d, n_chunks, group_size, k_groups, k_chunks, out, groups_out,
      as_cuda(stream));
  if (e != cudaSuccess) return cuda_fail(e, "hier gist launch");
  return ok();
}

sa_status sa_index_overlap(const int32_t* idx_a, const int32_t* count_a, const int32_t* idx_b,
                           const int32_t* count_b, int rows, int k, int32_t* inter_out, sa_stream_t stream) {
  if (rows < 0 || k < 1) return fail(SA_ERR_INVALID_ARG, "bad sizes: rows=%d k=%d", rows, k);
  if (rows == 0) return ok();
  if (!idx_a || !count_a || !idx_b || !count_b || !inter_out) return fail(SA_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(idx_a, 4) || !aligned(idx_b, 4) || !aligned(count_a, 4) || !aligned(count_b, 4) ||
      !aligned(inter_out, 4))
    return fail(SA_ERR_INVALID_ARG, "pointers must be 4-byte aligned");
  const cudaError_t e = sa::launch_index_overlap(idx_a, count_a, idx_b, count_b, rows, k, inter_out,
                                                 as_cuda(stream));
  if (e != cudaSuccess) return cuda_fail(e, "index_overlap launch");
  return ok();
}

sa_status sa_index_pattern_greedy(const double* overlap, int n_layers, int n_full, char* pattern_out) {
  if (!overlap || !pattern_out) return fail(SA_ERR_INVALID_ARG, "NULL pointer");
  if (n_layers < 1 || n_full < 1) return fail(SA_ERR_INVALID_ARG, "n_layers=%d and n_full=%d must be >= 1",
                                              n_layers, n_full);
  std::vector<char> full(n_layers, 1);
  auto total = [&](const std::vector<char>& f) {
    int owner = 0;
    double t = 0.0;
    for (int l = 0; l < n_layers; ++l) {
      if (f[l]) owner = l;
      t += overlap[(size_t)l * n_layers + owner];
    }
    return t;
  };
  int n = n_layers;
  while (n > n_full) {
    int best = -1;
    double best_t = 0.0;
    for (int l = 1; l < n_layers; ++l) {
      if (!full[l]) continue;
      full[l] = 0;
      const double t = total(full);
      full[l] = 1;
      if (best < 0 || t > best_t) {
        best = l;
        best_t = t;
      }
    }
    if (best < 0) break;   // only layer 0 is left
    full[best] = 0;
    --n;
  }
  for (int l = 0; l < n_layers; ++l) pattern_out[l] = full[l] ? 'F' : 'S';
  pattern_out[n_layers] = '\0';
  return ok();
}

int sa_debug_enabled(void) {
#ifdef SA_DEBUG
  return 1;
#else
  return 0;
#endif
}

sa_status sa_debug_check_canary(const void* ws, size_t offset, int site, sa_stream_t stream) {
  if (ws == nullptr) return fail(SA_ERR_INVALID_ARG, "ws is NULL");
  const cudaError_t e = sa::dbg_check(ws, offset, site, as_cuda(stream));
  if (e != cudaSuccess) return cuda_fail(e, "debug canary check");
  return ok();
}

sa_status sa_debug_read(int32_t* record, int reset) {
  if (record == nullptr) return fail(SA_ERR_INVALID_ARG, "record is NULL");
  const cudaError_t e = sa::dbg_read(record, reset != 0);
  if (e != cudaSuccess) return cuda_fail(e, "debug record read");
  return ok();
}

}  // extern "C"

// ========================================================= index cache

struct sa_index_cache {
  int n_layers = 0;
  std::vector<int> owner;
  int B = 0, Tq = 0, k = 0;
  int32_t* idx_buf = nullptr;
  int32_t* count_buf = nullptr;
  uint64_t version = 0;      // bumped at every write
  int last_writer = -1;      // full layer whose index the buffer holds in this step
  uint64_t last_version = 0;
};

extern "C" {

sa_status sa_index_cache_create(int n_layers, const char* pattern, int share_every, int B, int Tq,
                                int k, int32_t* idx_buf, int32_t* count_buf, sa_index_cache** out) {
  if (out == nullptr) return fail(SA_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (n_layers < 1) return fail(SA_ERR_INVALID_ARG, "n_layers=%d must be >= 1", n_layers);
  if (B < 0 || Tq < 1 || k < 1) return fail(SA_ERR_INVALID_ARG, "bad sizes B=%d Tq=%d k=%d", B, Tq, k);
  if (k > SA_MAX_K) return fail(SA_ERR_UNSUPPORTED, "k=%d exceeds SA_MAX_K", k);
  if (B > 0 && (!idx_buf || !count_buf)) return fail(SA_ERR_INVALID_ARG, "NULL index buffer");
  std::string pat;
  if (pattern != nullptr) {
    pat = pattern;
    if ((int)pat.size() != n_layers)
      return fail(SA_ERR_INVALID_ARG, "pattern length %zu != n_layers %d", pat.size(), n_layers);
  } else {
    if (share_every < 1) return fail(SA_ERR_INVALID_ARG, "share_every=%d must be >= 1", share_every);
    for (int l = 0; l < n_layers; ++l) pat.push_back(l % share_every == 0 ? 'F' : 'S');
  }
  if (pat[0] != 'F') return fail(SA_ERR_INVALID_ARG, "layer 0 must be a full layer ('F')");
  auto* c = new sa_index_cache();
  c->n_layers = n_layers;
  int cur = 0;
  for (int l = 0; l < n_layers; ++l) {
    if (pat[l] == 'F') cur = l;
    else if (pat[l] != 'S') {
      delete c;
      return fail(SA_ERR_INVALID_ARG, "pattern character %d is '%c' (need 'F' or 'S')", l, pat[l]);
    }
    c->owner.push_back(cur);
  }
  c->B = B;
  c->Tq = Tq;
  c->k = k;
  c->idx_buf = idx_buf;
  c->count_buf = count_buf;
  *out = c;
  return ok();
}

void sa_index_cache_destroy(sa_index_cache* cache) { delete cache; }

int sa_index_cache_is_full(const sa_index_cache* c, int layer) {
  if (!c || layer < 0 || layer >= c->n_layers) return -1;
  return c->owner[layer] == layer ? 1 : 0;
}

int sa_index_cache_owner(const sa_index_cache* c, int layer) {
  if (!c || layer < 0 || layer >= c->n_layers) return -1;
  return c->owner[layer];
}

sa_status sa_index_cache_begin_step(sa_index_cache* c) {
  if (!c) return fail(SA_ERR_INVALID_ARG, "cache is NULL");
  c->last_writer = -1;
  return ok();
}

sa_status sa_index_cache_mark_written(sa_index_cache* c, int layer) {
  if (!c) return fail(SA_ERR_INVALID_ARG, "cache is NULL");
  if (layer < 0 || layer >= c->n_layers) return fail(SA_ERR_INVALID_ARG, "layer %d out of range", layer);
  if (c->owner[layer] != layer) return fail(SA_ERR_INVALID_ARG, "layer %d is a shared layer", layer);
  c->version += 1;
  c->last_writer = layer;
  c->last_version = c->version;
  return ok();
}

sa_status sa_index_cache_update(sa_index_cache* c, int layer, const void* q_idx, const void* k_idx,
                                int Tk, int Tk_max, int d, int q_pos0, const int32_t* kv_len,
                                void* ws, size_t ws_bytes, sa_stream_t stream) {
  if (!c) return fail(SA_ERR_INVALID_ARG, "cache is NULL");
  if (layer < 0 || layer >= c->n_layers) return fail(SA_ERR_INVALID_ARG, "layer %d out of range", layer);
  if (c->owner[layer] != layer)
    return fail(SA_ERR_INVALID_ARG, "layer %d is a shared layer; it reuses layer %d's index", layer,
                c->owner[layer]);
  sa_status st = sa_index_score_topk(q_idx, k_idx, c->B, c->Tq, Tk, Tk_max, d, c->k, q_pos0, kv_len,
                                     c->idx_buf, c->count_buf, nullptr, ws, ws_bytes, stream);
  if (st != SA_OK) return st;
  return sa_index_cache_mark_written(c, layer);
}

sa_status sa_index_cache_get(sa_index_cache* c, int layer, const int32_t** idx,
                             const int32_t** count, uint64_t* version) {
  if (!c) return fail(SA_ERR_INVALID_ARG, "cache is NULL");
  if (layer < 0 || layer >= c->n_layers) return fail(SA_ERR_INVALID_ARG, "layer %d out of range", layer);
  const int o = c->owner[layer];
  if (c->last_writer != o)
    return fail(SA_ERR_STALE_INDEX, "layer %d reads full layer %d's index, but the buffer holds %s", layer,
                o, c->last_writer < 0 ? "no index of this step" : "a later full layer's index");
  if (idx) *idx = c->idx_buf;
  if (count) *count = c->count_buf;
  if (version) *version = c->last_version;
  return ok();
}

}  // extern "C"
