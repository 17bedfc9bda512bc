/*
 * sa.h -- C ABI of libsa.so: indexer-routed token-sparse attention with one
 * routing index shared by a group of layers, plus gist-chunk routing.
 *
 * Sources (page title, section):
 *   [YOIO] "你只索引一次：当AI学会'过目不忘'的遗忘艺术", a write-up of
 *          "You Only Index Once: Cross-Layer Sparse Attention with Shared Routing".
 *   [LC]   "长上下文：稀疏注意力 / DSA / IndexShare".
 *   [SSA]  "斯坦福大学研究团队如何让AI'聪明地遗忘'" (Simplified Sparse Attention).
 *   [IC]   "清华提出IndexCache技术：让AI大模型处理长文本时速度提升80%".
 *   [GSA]  "Forget, Then Recall: Learnable Compression and Selective Unfolding
 *          via Gist Sparse Attention".
 *
 * Conventions shared by every call
 *   - Tensors are caller-owned DEVICE pointers, contiguous, row-major.
 *     bf16 tensors are passed as void* and hold bfloat16 bit patterns.
 *   - Every call validates its arguments on the host first and returns an
 *     error WITHOUT launching anything if they are bad.  Valid calls enqueue
 *     their kernels on `stream` and return at once: no host synchronisation,
 *     no device allocation, no host allocation on the hot path.
 *   - Kernel launch failures return SA_ERR_CUDA; sa_last_error() gives the
 *     detail.  Faults inside a kernel surface later, on the stream, as for
 *     any CUDA kernel.
 *   - Selected positions are int32 absolute cache rows; unused slots hold -1.
 *   - No kernel of this library waits on another CTA, kernel or device.
 *     Waits inside a kernel (its own pipeline barriers) are bounded.  A wait
 *     that gave up is recorded as a nonzero error word at the start of the
 *     call's workspace, and the outputs show it: decode attention writes
 *     NaN, indexer top-k and gist routing write the failure sentinel
 *     (count 0, every index -1).
 *   - Workspaces are caller-owned device memory, SA_WS_ALIGN-aligned, and
 *     must be ZERO-FILLED before their first use.  The counters that must
 *     start at zero (histograms, candidate counts, merge tickets) live in a
 *     fixed region at the start of each workspace that every completed call
 *     returns to zero, so one workspace then serves any number of calls of
 *     any shape made one after another on one stream.  Zero it again after a
 *     failed or interrupted call.  Calls that overlap on the GPU (different
 *     streams) need different workspaces.
 */
#ifndef SA_H_
#define SA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; 0 is the legacy default stream. */
typedef struct CUstream_st* sa_stream_t;

typedef enum {
  SA_OK = 0,
  SA_ERR_INVALID_ARG = 1,   /* null pointer, negative or inconsistent size   */
  SA_ERR_UNSUPPORTED = 2,   /* valid but outside this build's shape support  */
  SA_ERR_WORKSPACE = 3,     /* workspace missing, too small or misaligned    */
  SA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed          */
  SA_ERR_TIMEOUT = 5,       /* a kernel wait gave up (read by sa_workspace_status) */
  SA_ERR_STALE_INDEX = 6    /* shared layer read before its full layer ran   */
} sa_status;

/* Limits of this build. */
#define SA_MAX_K 4096           /* largest top-k                                */
#define SA_HEAD_DIM 128         /* attention head_dim supported                 */
#define SA_WS_ALIGN 256         /* workspace pointers must be 256-byte aligned  */
#define SA_DECODE_MAX_PAIRS 16384 /* largest B * Hkv of one decode attention call */

/* Static, never-null description of a status code. */
const char* sa_status_string(sa_status s);
/* Detail of the last failing call made by this host thread ("" if none). */
const char* sa_last_error(void);
/* Library ABI version (major * 100 + minor). */
int sa_version(void);

/* ------------------------------------------------------------------------
 * Indexer scoring + per-query top-k.
 *
 * [LC] "DSA 与 IndexShare": a light indexer scores every history token and
 * each query keeps only its top-k tokens; [YOIO] §1.3 (token-level top-k)
 * and §2.3 (the indexer's output is each query's top-k token indices).
 *
 * Score of query t against cached token j: s = q_idx[b,t,:] . k_idx[b,j,:],
 * one indexer head, accumulated in fp32 (exact for integer-valued bf16
 * inputs with |s| < 2^24).  Candidates of query t are the positions
 *     0 <= j <= q_pos0 + t   and   j < len_b,
 * where len_b = kv_len[b] if kv_len is given, else Tk.  (Causality is
 * inclusive: a token may select itself.  For decode pass Tq = 1 and
 * q_pos0 = len - 1, or any q_pos0 >= len - 1.)
 *
 * Selection keeps k_eff = min(k, n_candidates) positions: the largest
 * scores, equal scores ordered by LOWER position first.  Row (b,t) of
 * idx_out holds them in ASCENDING position order followed by -1 padding;
 * count_out[b,t] = k_eff.  score_out, if given, holds each kept position's
 * fp32 score in the same slots (NaN-free padding value: -inf).
 *
 *   q_idx      [B, Tq, d]      bf16
 *   k_idx      [B, Tk_max, d]  bf16   (rows >= len_b never affect the result;
 *                                      prefill may read them, within Tk_max,
 *                                      as parts of whole 256-row tiles)
 *   kv_len     [B] int32 or NULL      (each 0 <= kv_len[b] <= Tk; values
 *                                      outside are clamped on the device)
 *   idx_out    [B, Tq, k] int32;  count_out [B, Tq] int32
 *   score_out  [B, Tq, k] fp32 or NULL
 *   ws         device workspace of >= sa_index_score_topk_workspace(...) bytes
 *              (zero-filled before first use; see the conventions above).
 *              Its first int32 is the kernel error word: 0 after a good call.
 *              If a pipeline wait of the call's kernels gave up, the word is
 *              nonzero and every row gets count 0 and idx -1 (score -inf);
 *              a workspace whose word is nonzero keeps giving that sentinel
 *              until the caller zero-fills it again.
 * Supported: d in {64, 128}; 1 <= k <= SA_MAX_K; Tq >= 1; 0 <= Tk <= Tk_max.
 * Scores must be free of NaN (NaN inputs give an unspecified selection).
 * ---------------------------------------------------------------------- */
size_t sa_index_score_topk_workspace(int B, int Tq, int Tk_max, int d, int k);
sa_status sa_index_score_topk(const void* q_idx, const void* k_idx,
                              int B, int Tq, int Tk, int Tk_max, int d, int k,
                              int q_pos0, const int32_t* kv_len,
                              int32_t* idx_out, int32_t* count_out, float* score_out,
                              void* ws, size_t ws_bytes, sa_stream_t stream);

/* ------------------------------------------------------------------------
 * Multi-head weighted indexer scoring + per-query top-k.
 *
 * A wider score function for the same selection ([LC] "DSA 与 IndexShare"
 * names only a light indexer; this is the multi-head form of DeepSeek's
 * published lightning indexer): H indexer heads, each with its own query
 * vector and weight, score one shared key per cached token as
 *     s = sum_h w[b,t,h] * max(0, q_idx[b,t,h,:] . k_idx[b,j,:]),
 * accumulated in fp32 (exact for integer-valued inputs with every partial
 * sum below 2^24).  Candidates, tie rule, output order, kv_len, q_pos0,
 * score_out and the error word are exactly as for sa_index_score_topk.
 *
 *   q_idx  [B, Tq, H, d] bf16;   w [B, Tq, H] fp32;   k_idx [B, Tk_max, d] bf16
 *   ws     >= sa_index_score_topk_mh_workspace(...) bytes (zero-filled
 *          before first use; see the conventions above)
 * Supported: d in {64, 128}; 1 <= H <= 64 (d = 64) or 32 (d = 128);
 * 1 <= k <= SA_MAX_K.
 * ---------------------------------------------------------------------- */
size_t sa_index_score_topk_mh_workspace(int B, int Tq, int Tk_max, int H, int d, int k);
sa_status sa_index_score_topk_mh(const void* q_idx, const float* w, const void* k_idx,
                                 int B, int Tq, int H, int Tk, int Tk_max, int d, int k,
                                 int q_pos0, const int32_t* kv_len,
                                 int32_t* idx_out, int32_t* count_out, float* score_out,
                                 void* ws, size_t ws_bytes, sa_stream_t stream);

/* ------------------------------------------------------------------------
 * fp8 indexer, decode (one query per sequence; no counterpart in the pages,
 * which name only a light indexer: an extension for an indexer cache stored
 * in 8 bits, half the bytes the decode scorer streams).
 *
 * q_idx and k_idx hold OCP FP8 E4M3 bytes (1 sign, 4 exponent bits with bias
 * 7, 3 mantissa bits; no infinities; S.1111.111 is NaN).  Products are exact
 * and accumulate in fp32, so integer-valued inputs give exact scores.
 *   w == NULL (then H must be 1): s = q_idx[b,0,:] . k_idx[b,j,:], the
 *     one-head score of sa_index_score_topk;
 *   w != NULL: s = sum_h w[b,h] * max(0, q_idx[b,h,:] . k_idx[b,j,:]), the
 *     multi-head score of sa_index_score_topk_mh.
 * The query of sequence b sits at position q_pos0; its candidates are
 * j <= q_pos0, j < kv_len[b].  Selection, tie rule, output order, score_out
 * and the error word are exactly as for sa_index_score_topk with Tq = 1.
 *
 *   q_idx  [B, H, d] e4m3 bytes (16-byte aligned);  w [B, H] fp32 or NULL
 *   k_idx  [B, Tk_max, d] e4m3 bytes (16-byte aligned)
 *   kv_len [B] int32 or NULL;  idx_out [B, k] int32;  count_out [B] int32
 *   score_out [B, k] fp32 or NULL
 *   ws     >= sa_index_score_topk_fp8_workspace(...) bytes (zero-filled
 *          before first use; see the conventions above)
 * Supported: d in {64, 128}; 1 <= H <= 32; 1 <= k <= SA_MAX_K.
 * ---------------------------------------------------------------------- */
size_t sa_index_score_topk_fp8_workspace(int B, int Tk_max, int H, int d, int k);
sa_status sa_index_score_topk_fp8(const void* q_idx, const float* w, const void* k_idx,
                                  int B, int H, int Tk, int Tk_max, int d, int k,
                                  int q_pos0, const int32_t* kv_len,
                                  int32_t* idx_out, int32_t* count_out, float* score_out,
                                  void* ws, size_t ws_bytes, sa_stream_t stream);

/* ------------------------------------------------------------------------
 * Gathered sparse attention, prefill (one call per layer).
 *
 * [YOIO] §1.1: Attention(Q,K,V) = softmax(QK^T/sqrt(d_k))V; §2.3: each
 * layer's selector fetches from its KV cache only the rows named by the
 * shared index and attends over them.  [LC] "DSA 与 IndexShare": core
 * attention drops from O(L^2) to O(Lk).
 *
 * For token t of sequence b and query head h (kv head g = h / (Hq/Hkv)):
 *   z_i = scale * q[b,t,h,:] . k_cache[b, j_i, g, :],  j_i = idx[b,t,i], i < count[b,t]
 *   out[b,t,h,:] = sum_i softmax(z)_i v_cache[b, j_i, g, :]
 *   lse[b,t,h]   = ln sum_i exp(z_i)          (natural log; -inf if count = 0)
 * An empty row (count = 0) gives out = 0.  scale <= 0 selects 1/sqrt(D).
 * bf16 inputs, fp32 accumulation and softmax, bf16 output.
 *
 *   q        [B, T, Hq, D] bf16
 *   k_cache  [B, Tk_max, Hkv, D] bf16;  v_cache same shape
 *   idx      [B, T, k] int32 (each used entry in [0, Tk_max); entries past
 *            count are ignored); count [B, T] int32 (clamped to [0, k])
 *   out      [B, T, Hq, D] bf16;  lse [B, T, Hq] fp32 or NULL
 * Supported: D = 128; Hq % Hkv == 0; 1 <= Hq/Hkv <= 16.
 * Used indices outside [0, Tk_max) are a caller error; the kernels clamp
 * them into range (reading a wrong row) rather than fault.
 * ---------------------------------------------------------------------- */
sa_status sa_sparse_attn_prefill(const void* q, const void* k_cache, const void* v_cache,
                                 const int32_t* idx, const int32_t* count,
                                 int B, int T, int Tk_max, int Hq, int Hkv, int D, int k,
                                 float scale, void* out, float* lse, sa_stream_t stream);

/* ------------------------------------------------------------------------
 * Gathered sparse attention, decode (one query token per sequence).
 *
 * Same arithmetic as the prefill call.  The selected rows are split across
 * CTAs; each CTA loads every selected K/V row once for all Hq/Hkv query
 * heads of each kv head, and the partial results are merged with the
 * log-sum-exp rule ([SSA] §六: split-K partial attention over a compact
 * index list, KV shared by a GQA group loaded once, then a log-sum-exp
 * merge).
 *
 *   q        [B, Hq, D] bf16
 *   idx      [B, k] int32 (row stride k); count [B] int32 (clamped to [0, k])
 *   out      [B, Hq, D] bf16;  lse [B, Hq] fp32 or NULL
 *   ws       >= sa_sparse_attn_decode_workspace(...) bytes (zero-filled before
 *            first use; see the conventions above).  Its first int32 is the
 *            kernel error word: 0 after a good call.
 * Supported: as for prefill; B * Hkv <= SA_DECODE_MAX_PAIRS.
 * ---------------------------------------------------------------------- */
size_t sa_sparse_attn_decode_workspace(int B, int Hq, int Hkv, int D, int k);
sa_status sa_sparse_attn_decode(const void* q, const void* k_cache, const void* v_cache,
                                const int32_t* idx, const int32_t* count,
                                int B, int Tk_max, int Hq, int Hkv, int D, int k,
                                float scale, void* out, float* lse,
                                void* ws, size_t ws_bytes, sa_stream_t stream);

/* ------------------------------------------------------------------------
 * Gather once, attend many (one KV cache shared by every layer).
 *
 * [YOIO] §2.1-§2.2: YOCO keeps one KV cache for all layers, and the shared
 * routing adds one index for all layers, so each decode step needs the
 * selected K/V rows only once.  sa_gather_rows copies them into compact
 * buffers; each layer then runs sa_sparse_attn_decode_rows over those rows
 * with its own queries.
 *
 * sa_gather_rows:
 *   k_cache, v_cache  [B, Tk_max, Hkv, D] bf16;  idx [B, k] int32 (entries
 *                     below count[b] in [0, Tk_max); others are not read);
 *                     count [B] int32 (clamped to [0, k])
 *   k_rows, v_rows    [B, k, Hkv * D + 8] bf16: row i of sequence b holds the
 *                     Hkv * D values of cache row idx[b, i] for i < count[b],
 *                     zeros after it; the last 8 values (16 bytes) of every
 *                     row are a zero pad (the layout the attention stages a
 *                     tile in, so one copy moves a whole tile).
 * sa_sparse_attn_decode_rows: the attention of sa_sparse_attn_decode over
 *   the first count[b] rows of k_rows / v_rows (laid out as above, pad
 *   included; rows from count[b] to k must hold finite values, as the
 *   gather's zeros do).
 *   q [B, Hq, D]; out [B, Hq, D]; lse [B, Hq] or NULL;
 *   ws >= sa_sparse_attn_decode_workspace(B, Hq, Hkv, D, k) bytes (same
 *   conventions).  Supported: D = 128, Hkv <= 8, Hq % Hkv == 0, Hq/Hkv <= 16.
 * ---------------------------------------------------------------------- */
sa_status sa_gather_rows(const void* k_cache, const void* v_cache, const int32_t* idx,
                         const int32_t* count, int B, int Tk_max, int Hkv, int D, int k,
                         void* k_rows, void* v_rows, sa_stream_t stream);
sa_status sa_sparse_attn_decode_rows(const void* q, const void* k_rows, const void* v_rows,
                                     const int32_t* count, int B, int Hq, int Hkv, int D, int k,
                                     float scale, void* out, float* lse,
                                     void* ws, size_t ws_bytes, sa_stream_t stream);

/* ------------------------------------------------------------------------
 * Decode attention without a caller workspace.
 *
 * No counterpart in the paper: this is an interface for callers that cannot
 * call cudaMalloc -- for example a host process that may only pass on the
 * buffers it was handed, or code on a path where allocation is not allowed
 * -- and so cannot supply the workspace sa_sparse_attn_decode needs.
 * Arguments, results and limits are those of sa_sparse_attn_decode.  The
 * scratch is a fixed array of SA_NOALLOC_SCRATCH_BYTES inside the library,
 * held on every GPU that loads it until the process exits; shapes that need
 * more scratch (sa_sparse_attn_decode_workspace(...) > SA_NOALLOC_SCRATCH_BYTES)
 * are rejected with SA_ERR_UNSUPPORTED.  The call allocates nothing.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - Every call clears, on `stream`, the part of the array that must start
 *     at zero, then leaves its results in the array until the next call.
 *   - All calls share the one array: calls that overlap on the GPU (e.g. on
 *     different streams) race and give undefined results.
 * ---------------------------------------------------------------------- */
#define SA_NOALLOC_SCRATCH_BYTES (8u << 20)
sa_status sa_sparse_attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                        const int32_t* idx, const int32_t* count,
                                        int B, int Tk_max, int Hq, int Hkv, int D, int k,
                                        float scale, void* out, float* lse, sa_stream_t stream);

/* ------------------------------------------------------------------------
 * Self-test of the bounded waits (no counterpart in the pages).
 *
 * Every pipeline kernel of the library waits on mbarrier phases with a poll
 * limit: a wait that runs out sets the kernel's abort flag and records its
 * code in an error word instead of hanging the GPU.  This call launches a
 * one-thread probe that (1) waits on a phase nothing completes, with
 * `poll_limit` polls, and (2) waits on a phase that does complete.
 *   err  device int32[5], zero-filled by the caller.  After the stream
 *        reaches the call: err[0] = 77 (the timed-out wait's code),
 *        err[1] = 0, err[2] = 0 (the first wait returned false),
 *        err[3] = 1 (its abort flag was set), err[4] = 1 (the second wait
 *        returned true).
 * Faults nothing; returns SA_ERR_INVALID_ARG for a null err or a zero limit.
 * ---------------------------------------------------------------------- */
sa_status sa_self_test_bounded_wait(int32_t* err, uint32_t poll_limit, sa_stream_t stream);

/* ------------------------------------------------------------------------
 * Gist-chunk routing with selective unfolding (decode).
 *
 * [SSA] §二/§三 and [GSA] 2.1-2.2: the sequence is cut into chunks of
 * chunk_len raw tokens, each followed by one gist token; the query is
 * scored by dot product against every chunk's gist key, the top k_chunks
 * chunks are kept, and each kept chunk is unfolded into its raw tokens plus
 * its own gist.  Unkept gists are left out ([SSA] §八 and [GSA] 4 find this
 * "selected gists + selected raw" context best).  The current, incomplete
 * chunk (partial_len[b] tokens) is always appended.
 *
 * Cache layout assumed for the row ids: chunk c occupies rows
 * (chunk_len+1)*c .. (chunk_len+1)*c + chunk_len - 1 (raw) and
 * (chunk_len+1)*c + chunk_len (gist); the partial chunk starts at
 * (chunk_len+1)*n_chunks.
 *
 * Chunk selection follows the top-k rule above (equal scores: lower chunk).
 * rows_out row b: for each kept chunk in ascending order its chunk_len+1
 * rows, then the partial rows, then -1 padding; count_out[b] = number of
 * rows.  chunks_out (optional) holds the kept chunk ids, ascending, -1 padded.
 *
 *   q_route     [B, d] bf16;   gist_key [B, n_chunks, d] bf16
 *   partial_len [B] int32 (clamped on the device to [0, chunk_len])
 *   ws          >= sa_gist_route_unfold_workspace(...) bytes (zero-filled
 *               before first use; see the conventions above).  Its first
 *               int32 is the kernel error word, as for sa_index_score_topk;
 *               when it is nonzero every row gets count 0 and rows -1.
 *   rows_out    [B, k_chunks*(chunk_len+1) + chunk_len] int32
 *   count_out   [B] int32;    chunks_out [B, k_chunks] int32 or NULL
 * Supported: d in {64, 128}; 1 <= k_chunks <= SA_MAX_K; 1 <= chunk_len <= 256.
 * ---------------------------------------------------------------------- */
size_t sa_gist_route_unfold_workspace(int B, int n_chunks, int d, int k_chunks);
sa_status sa_gist_route_unfold(const void* q_route, const void* gist_key,
                               int B, int n_chunks, int chunk_len, int d, int k_chunks,
                               const int32_t* partial_len,
                               int32_t* rows_out, int32_t* count_out, int32_t* chunks_out,
                               void* ws, size_t ws_bytes, sa_stream_t stream);

/* ------------------------------------------------------------------------
 * Two-level (coarse-to-fine) gist routing with selective unfolding.
 *
 * [SSA] §五 (H-SSA) and [GSA] 2.4 (H-GSA): gists of gists.  Every complete
 * group of group_size consecutive chunks has one meta-gist routing key.  The
 * query is scored against every meta key and the top k_groups groups are
 * kept (equal scores: lower group first); the candidate chunks are those of
 * the kept groups plus the chunks after the last complete group (which has
 * no meta-gist yet); the query is scored against their gist keys and the top
 * k_chunks candidates are kept (equal scores: lower chunk first) and
 * unfolded exactly as by sa_gist_route_unfold.  Meta-gists are routing keys
 * only: their rows are not part of the attended context.
 *
 *   q_route   [B, d] bf16;  meta_key [B, n_chunks / group_size, d] bf16;
 *   gist_key  [B, n_chunks, d] bf16;  partial_len [B] int32 or NULL
 *   rows_out  [B, k_chunks*(chunk_len+1) + chunk_len] int32;  count_out [B]
 *   chunks_out [B, k_chunks] int32 or NULL;  groups_out [B, k_groups] int32
 *   or NULL (kept groups ascending, -1 padded)
 * No workspace.  Supported: d in {64, 128}; 1 <= chunk_len <= 256;
 * n_chunks / group_size <= 8192 and min(k_groups, n_chunks / group_size) *
 * group_size + (n_chunks % group_size) <= 8192; 1 <= k_chunks <= SA_MAX_K.
 * ---------------------------------------------------------------------- */
sa_status sa_hier_gist_route_unfold(const void* q_route, const void* meta_key, const void* gist_key,
                                    int B, int n_chunks, int chunk_len, int group_size, int d,
                                    int k_groups, int k_chunks, const int32_t* partial_len,
                                    int32_t* rows_out, int32_t* count_out, int32_t* chunks_out,
                                    int32_t* groups_out, sa_stream_t stream);

/* ------------------------------------------------------------------------
 * Index overlap between layers, and a training-free layer-role search.
 *
 * [IC] §一: the top-k sets of adjacent layers' indexers overlap by 70-100%,
 * which is why a shared layer can reuse a full layer's index.
 * sa_index_overlap counts, per row, the positions two selections share:
 *   idx_a, idx_b   [rows, k] int32, each row ascending (as every selection
 *                  of this library is) within its count; count_a, count_b
 *                  [rows] int32 (clamped to [0, k]); inter_out [rows] int32.
 *
 * [IC] §三: starting with every layer full, the indexer whose removal hurts
 * least is removed, repeatedly.  sa_index_pattern_greedy runs that search on
 * the host with the retained overlap as the measure (the pages measure a
 * model's loss on calibration data, which needs a trained model):
 *   overlap        [n_layers, n_layers] row-major: overlap[l, j] = mean
 *                  fraction of layer l's own selection contained in layer
 *                  j's (j <= l is what a shared layer reads)
 *   pattern_out    n_layers + 1 chars: 'F'/'S' per layer and a NUL.  Layer 0
 *                  stays full; n_full layers stay full; ties remove the
 *                  lower layer first.  The pattern feeds sa_index_cache_create.
 * ---------------------------------------------------------------------- */
sa_status sa_index_overlap(const int32_t* idx_a, const int32_t* count_a, const int32_t* idx_b,
                           const int32_t* count_b, int rows, int k, int32_t* inter_out,
                           sa_stream_t stream);
sa_status sa_index_pattern_greedy(const double* overlap, int n_layers, int n_full, char* pattern_out);

/* ------------------------------------------------------------------------
 * The error word of a workspace, read on the host.
 *
 * Waits for the work queued on `stream` so far (synchronizes it), then reads
 * the kernel error word at the start of `ws`, the workspace of any call above
 * that takes one (indexer top-k of every form, gist routing, decode
 * attention).  Returns SA_OK when the word is zero and SA_ERR_TIMEOUT when a
 * pipeline wait of a call that used the workspace gave up; sa_last_error()
 * then names the wait's code.  The word is left as it is (zero-fill the
 * workspace to use it again).  SA_ERR_INVALID_ARG for a NULL ws,
 * SA_ERR_CUDA if the copy fails.
 * ---------------------------------------------------------------------- */
sa_status sa_workspace_status(const void* ws, sa_stream_t stream);

/* ------------------------------------------------------------------------
 * Debug builds (libsa_debug.so, compiled with SA_DEBUG; no counterpart in the
 * pages).
 *
 * The debug build checks, on the device, every gathered row index a call
 * uses (those below its count) against [0, Tk_max), and puts a 256-byte
 * canary after the bytes each workspace call may use (the *_workspace
 * functions count it; every call writes it and checks it after its
 * kernels).  A violation is recorded -- never trapped -- and the access is
 * clamped exactly as in the release build, so results match it.
 *   sa_debug_enabled(): 1 in a debug build, 0 otherwise.
 *   sa_debug_read(record, reset): host int32[4] = {code of the first
 *     violation (0 none, 1 prefill attention index, 2 decode attention index,
 *     3 gathered-rows index, 4 workspace canary), its first detail (the index;
 *     for a canary the call: 1 index top-k, 2 multi-head top-k, 3 decode
 *     attention, 4 gist routing, 5 fp8 top-k), its second detail (Tk_max; for a canary the
 *     first changed byte), number of violations}; reset != 0 clears it.
 *     Synchronous; the release build reports zeros.
 * ---------------------------------------------------------------------- */
int sa_debug_enabled(void);
sa_status sa_debug_read(int32_t* record, int reset);
/* The canary check every workspace call runs after its kernels, on its own:
 * the 256 bytes at ws + offset must all be 0xA5, else code 4 is recorded with
 * `site` and the first changed byte.  Asynchronous on `stream`; a no-op in
 * the release build. */
sa_status sa_debug_check_canary(const void* ws, size_t offset, int site, sa_stream_t stream);

/* ------------------------------------------------------------------------
 * Shared index cache (host object; its device buffers are caller-owned).
 *
 * [IC] §二 and §六: layers are "full" (run their own indexer and store the
 * result) or "shared" (reuse the index of the nearest full layer before
 * them); one temporary buffer holds the current index and is overwritten at
 * the next full layer, so sharing adds no memory.  [LC] "DSA 与 IndexShare"
 * and [YOIO] §2.2: the expensive top-k is done once and reused by every layer
 * of the group.
 *
 * create: pattern is a string of 'F'/'S' of length n_layers starting with
 *   'F', or NULL to use share_every (layer l is full iff l % share_every == 0).
 *   idx_buf [B, Tq, k] int32 and count_buf [B, Tq] int32 are device buffers
 *   that must outlive the cache.
 * begin_step: starts a new forward step; every shared layer becomes stale
 *   until its full layer writes again.
 * update: full layers only; runs sa_index_score_topk into the buffers.
 * mark_written: records that the caller itself filled the buffers for full
 *   layer `layer` (e.g. with sa_index_score_topk on its own stream).
 * get: returns the buffers for `layer` and the version of the write it reads.
 *   SA_ERR_STALE_INDEX if, in this step, the layer's full layer has not
 *   written or a later full layer has overwritten the buffer.
 * The object is not thread-safe.
 * ---------------------------------------------------------------------- */
typedef struct sa_index_cache sa_index_cache;
sa_status sa_index_cache_create(int n_layers, const char* pattern, int share_every,
                                int B, int Tq, int k, int32_t* idx_buf, int32_t* count_buf,
                                sa_index_cache** out);
void sa_index_cache_destroy(sa_index_cache* cache);
/* 1 if `layer` is a full layer, 0 if shared, -1 if out of range or cache NULL. */
int sa_index_cache_is_full(const sa_index_cache* cache, int layer);
/* The full layer whose index `layer` reads, or -1 if out of range. */
int sa_index_cache_owner(const sa_index_cache* cache, int layer);
sa_status sa_index_cache_begin_step(sa_index_cache* cache);
sa_status sa_index_cache_update(sa_index_cache* cache, int layer, const void* q_idx,
                                const void* k_idx, int Tk, int Tk_max, int d, int q_pos0,
                                const int32_t* kv_len, void* ws, size_t ws_bytes,
                                sa_stream_t stream);
sa_status sa_index_cache_mark_written(sa_index_cache* cache, int layer);
sa_status sa_index_cache_get(sa_index_cache* cache, int layer, const int32_t** idx,
                             const int32_t** count, uint64_t* version);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* SA_H_ */
