// Internal launchers of libsa.so (host side).  Not part of the C ABI.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/sa.h"

namespace sa {

// One-query rows (decode, gist routing) of at most this many candidates are
// selected by one CTA holding the whole row in shared memory ("direct"
// mode); longer rows carry the scorer's key histogram and are selected by
// slices over many CTAs (kFinishSplit).
constexpr int kDirectMaxCand = 4096;

// finish_kernel candidate sources
constexpr int kFinishDirect = 0;    // the whole row (no histogram)
constexpr int kFinishCandRows = 3;  // prefill: candidates appended by the bounded scoring pass
constexpr int kFinishSplit = 4;     // many CTAs per row filter slices, the row's last CTA selects

// Slices (CTAs) per row of the split selection, at most.
constexpr int kSplitMaxSlices = 1024;

// Prefill scoring passes (launch_score_prefill `epi`)
constexpr int kScoreKeys = 0;       // every score's key into the row slab
constexpr int kScoreGroupMax = 1;   // per-row group maxima (16-bit keys)
constexpr int kScoreCand = 2;       // keys at or above the row's bound, appended with positions

// Debug builds (SA_DEBUG): codes of the device debug record, and the canary
// after every workspace's used bytes.
constexpr int kDbgPrefillIndex = 1;
constexpr int kDbgDecodeIndex = 2;
constexpr int kDbgGatherIndex = 3;
constexpr int kDbgCanary = 4;
constexpr int kDbgCanaryBytes = 256;
constexpr unsigned char kDbgCanaryByte = 0xA5;
#ifdef SA_DEBUG
constexpr size_t kWsCanary = kDbgCanaryBytes;
#else
constexpr size_t kWsCanary = 0;
#endif
// Writes the canary at ws + off / checks it after a call's kernels (site:
// which call) / copies (and optionally clears) the record.  No-ops (zeros)
// in release builds.
cudaError_t dbg_arm(void* ws, size_t off, cudaStream_t st);
cudaError_t dbg_check(const void* ws, size_t off, int site, cudaStream_t st);
cudaError_t dbg_read(int* host4, bool reset);

// Rows whose histograms live in the fixed, self-cleaning workspace region.
constexpr int kHistRowsFixed = 64;

struct RowWorkspace {
  int* err = nullptr;            // first word: kernel error code (0 = none)
  size_t hist_zero_bytes = 0;    // > 0: histograms + counters must be zeroed per call
  uint32_t* keys = nullptr;      // [rows][ld] order-preserving score keys (prefill candidate rows: their keys)
  long long ld = 0;
  uint32_t* hist = nullptr;      // [rows][kHistBins]
  uint32_t* cand_cnt = nullptr;  // [rows] split rows: the row's ticket counter
  uint32_t* cand_pos = nullptr;  // prefill: [rows][ld] second slab
  uint16_t* gmax = nullptr;      // prefill: [rows][ld2] group maxima
  long long ld2 = 0;
  uint32_t* theta = nullptr;     // prefill: [rows] 16-bit bound per row
  uint32_t* tile_cnt = nullptr;  // prefill: [rows][ld / 256] takes of the run starting at each key tile
  uint2* cand = nullptr;         // split rows: [rows][ld] (key, position) candidates, slice c at c * chunk
  uint32_t* slot_cnt = nullptr;  // split rows: [rows][kSplitMaxSlices] candidates of each slice
};

// Finish-kernel output description.
struct FinishOut {
  int32_t* idx = nullptr;        // [B, Tq, k]
  int32_t* count = nullptr;      // [B, Tq]
  float* score = nullptr;        // [B, Tq, k] or null
  // gist unfolding (when rows != null)
  int32_t* rows = nullptr;       // [B, rows_stride]
  int rows_stride = 0;
  int chunk_len = 0;
  int n_chunks = 0;
  const int32_t* partial_len = nullptr;
  int32_t* chunks = nullptr;     // [B, k] or null
};

// Host-side argument check of sa_sparse_attn_decode (sets the error detail).
sa_status check_decode_args(const void* q, const void* kc, const void* vc, const int32_t* idx,
                            const int32_t* count, int B, int Tk_max, int Hq, int Hkv, int D, int k,
                            const void* out);

// Launches `kernel` with programmatic stream serialization, so it may start
// while the kernel before it on `st` drains (the kernel calls pdl_wait()
// before touching global memory).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Sets the detail string sa_last_error() returns for this host thread.
void set_last_error(const char* fmt, ...);

// Raises a kernel's dynamic shared-memory limit once per (kernel, device).
cudaError_t ensure_dynamic_smem(const void* func, size_t bytes);

// Number of SMs of the current device, looked up once per device (safe to
// call from several host threads).
int device_sm_count();
// Resident CTAs per SM of `func` at `threads` threads and `smem` dynamic
// shared bytes on the current device, looked up once per (func, device).
int device_occupancy(const void* func, int threads, size_t smem);

// Workspace of one-query rows: error word, histograms and counters, the key
// rows, and for split rows the candidate pairs and slice counts.
size_t row_workspace_bytes(int rows, int Tk_max, bool split, bool with_hist);
void carve_row_workspace(void* ws, int rows, int Tk_max, bool split, bool with_hist, RowWorkspace* out);

// One query per batch row (decode / gist): keys[b][j] = key(q[b].k[b][j]) for
// j < n_b = clamp(min(q_pos0+1, len_b), 0), plus the first-digit histogram.
cudaError_t launch_score_decode(const uint16_t* q, const uint16_t* kmat, int B, int d, int Tk_max,
                                int Tk, int q_pos0, const int32_t* kv_len, const RowWorkspace& w,
                                bool with_hist, cudaStream_t st);
// Exact selection per row.  rows = B * rows_per_batch; row r is query
// t0 + r % rows_per_batch of batch r / rows_per_batch.
cudaError_t launch_finish(int B, int rows_per_batch, int t0, int Tq, int Tk, int q_pos0,
                          const int32_t* kv_len, int k, const RowWorkspace& w, int mode,
                          const FinishOut& out, cudaStream_t st);
// Selection of one-query rows of Tk_max positions: kFinishDirect or kFinishSplit.
int finish_mode_for(int Tk_max);
// Exact selection of one-query rows by slices: many CTAs per row filter, the
// row's last CTA selects (the rows' histograms must come from the scorer).
cudaError_t launch_split_topk(int B, int rows_per_batch, int t0, int Tq, int Tk, int q_pos0,
                              const int32_t* kv_len, int k, const RowWorkspace& w, const FinishOut& out,
                              cudaStream_t st);
// Multi-head weighted indexer: rows per launch (B * rows rows at once) and
// the scoring of queries [t0, t0 + rows_per_batch) of every sequence into
// the keys and histograms of a split-row workspace.
int mh_rows_per_launch(int B, int Tq, int Tk_max);
cudaError_t launch_score_mh(const uint16_t* q, const float* wts, const uint16_t* kmat, int B, int H, int d,
                            int rows_per_batch, int t0, int Tq, int Tk_max, int Tk, int q_pos0,
                            const int32_t* kv_len, const RowWorkspace& w, bool with_hist, cudaStream_t st);
// Two-level gist routing, one CTA per sequence (shared memory holds up to
// kHierMax meta keys and kHierMax candidate chunks).
constexpr int kHierMax = 8192;
cudaError_t launch_hier_gist(const uint16_t* q_route, const uint16_t* meta_key, const uint16_t* gist_key, int B,
                             int d, int n_chunks, int group_size, int k_groups, int k, const FinishOut& out,
                             int32_t* groups_out, cudaStream_t st);
// Per-row shared positions of two ascending selections.
cudaError_t launch_index_overlap(const int32_t* a, const int32_t* ca, const int32_t* b, const int32_t* cb, int rows,
                                 int k, int32_t* out, cudaStream_t st);
// fp8 (e4m3) indexer scoring of one-query rows (index_fp8.cu): wts == null
// is the one-head dot product (H == 1), otherwise sum_h w_h * ReLU(q_h . k)
// over H <= kFp8MaxHeads heads.  Keys and the first-digit histogram go to the
// row workspace as for launch_score_decode.
constexpr int kFp8MaxHeads = 32;
cudaError_t launch_score_fp8(const uint8_t* q, const float* wts, const uint8_t* kmat, int B, int H, int d, int Tk_max,
                             int Tk, int q_pos0, const int32_t* kv_len, const RowWorkspace& w, bool with_hist,
                             cudaStream_t st);
// Largest number of indexer heads of the multi-head indexer for key width d.
constexpr int mh_max_heads(int d) { return d == 64 ? 64 : 32; }
// Prefill scoring of queries [t0, t0+rows) (tcgen05, index_tc.cu); `epi`
// picks what is kept per score (kScoreKeys / kScoreGroupMax / kScoreCand).
cudaError_t launch_score_prefill(const uint16_t* q, const uint16_t* kmat, int B, int Tq, int d,
                                 int Tk_max, int Tk, int q_pos0, const int32_t* kv_len, int t0,
                                 int rows, int k, int epi, const RowWorkspace& w, cudaStream_t st);
// Per-row bound of the bounded pass: the k-th largest group maximum (rows of
// at most k candidates: 0).
cudaError_t launch_prefill_threshold(int B, int rows_per_batch, int t0, int Tk, int q_pos0,
                                     const int32_t* kv_len, int k, const RowWorkspace& w, cudaStream_t st);
// Prefill rows per launch and workspace: the key slab, candidate positions,
// group maxima and per-row bound and counter for B * rows rows.
int prefill_rows_per_launch(int B, int Tq, int Tk_max, int k);
size_t prefill_workspace_bytes(int rows, int Tk_max, int k);
void carve_prefill_workspace(void* ws, int rows, int Tk_max, int k, RowWorkspace* out);
// Rows whose candidates exceed this many use the two bounded passes.
constexpr int kBoundedMinCand = 8192;

// Attention.
size_t decode_attn_workspace_bytes(int B, int Hq, int Hkv, int D, int k);
// Leading bytes of the decode workspace that must be zero when a call starts
// (the kernel error word).
size_t decode_attn_zero_bytes(int B, int Hkv, int k);
// idx == nullptr: kc / vc are compact rows [B][k][Hkv][D] (Hkv <= 8, Tk_max ==
// k) and each sequence attends over its first count[b] rows.
cudaError_t launch_attn_decode(const uint16_t* q, const uint16_t* kc, const uint16_t* vc,
                               const int32_t* idx, const int32_t* count, int B, int Tk_max, int Hq,
                               int Hkv, int k, float scale, uint16_t* out, float* lse, void* ws,
                               cudaStream_t st);
// Compact copies of the selected rows (rows past count zero-filled).
cudaError_t launch_gather_rows(const uint16_t* kc, const uint16_t* vc, const int32_t* idx, const int32_t* count,
                               int B, int Tk_max, int Hkv, int k, uint16_t* ko, uint16_t* vo, cudaStream_t st);
cudaError_t launch_attn_prefill(const uint16_t* q, const uint16_t* kc, const uint16_t* vc,
                                const int32_t* idx, const int32_t* count, int B, int T, int Tk_max,
                                int Hq, int Hkv, int k, float scale, uint16_t* out, float* lse,
                                cudaStream_t st);

}  // namespace sa
