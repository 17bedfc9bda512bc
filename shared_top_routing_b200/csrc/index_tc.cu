// Prefill indexer scoring on the 5th-generation tensor cores (sm_100a).
//
// [LC] "长上下文：稀疏注意力 / DSA / IndexShare", section "DSA 与 IndexShare":
// the indexer scores every (query, history token) pair; with causal masking
// the pairs of query t are the tokens j <= q_pos0 + t.  Here the score tile
// S = Q_idx K_idx^T of 128 queries x 256 keys is one tcgen05.mma sequence
// (M=128, N=256, K=16 per instruction; bf16 in, fp32 accumulate in TMEM).
//
// One CTA owns a block of 128 query rows of one sequence and walks its
// causal key tiles.  Warp roles (192 threads):
//   warp 0      TMA producer: the query block once, then key tiles into a
//               STAGES-deep shared-memory ring (128-byte swizzle, no
//               multicast), completion tracked by mbarriers;
//   warp 1      allocates 512 TMEM columns (two 128x256 fp32 accumulators)
//               and one thread issues the MMAs and tcgen05.commit;
//   warps 2-5   epilogue: thread i of the warpgroup owns TMEM lane (= query
//               row) i and reads its 256 scores per tile with tcgen05.ld.
// The MMA of tile i+1 overlaps the epilogue of tile i (double-buffered
// accumulator).  Every mbarrier wait is bounded; on a timeout the CTA records
// an error code, stops issuing work and frees its TMEM.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "sa_common.cuh"
#include "sa_internal.h"
#include "tc_common.cuh"

namespace sa {
namespace {

using namespace tc;

constexpr int kBM = 128;   // query rows per CTA (TMEM lanes)
constexpr int kBN = 256;   // key columns per MMA tile
constexpr int kTmemCols = 512;

template <int D>
struct TcShape {
  static constexpr int kAtoms = D / 64;             // 128-byte swizzle atoms along K
  static constexpr int kABytes = kBM * D * 2;
  static constexpr int kBBytes = kBN * D * 2;
  static constexpr int kStages = D == 64 ? 4 : 2;
  static constexpr int kSmem = 1024 + kABytes + kStages * kBBytes + 256;
};

struct TcBars {
  uint64_t full[4];
  uint64_t empty[4];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t afull;
  uint32_t tmem_base;
  int abort;
};

struct TcParams {
  int Tq, Tk, q_pos0;
  const int32_t* kv_len;
  int t0, rows, nblk;
  uint32_t* keys;
  long long ld;
  int* err;
};

__device__ __forceinline__ int tc_row_len(const int32_t* kv_len, int b, int Tk) {
  if (kv_len == nullptr) return Tk;
  int v = kv_len[b];
  return v < 0 ? 0 : (v > Tk ? Tk : v);
}

__device__ __forceinline__ int tc_n_cand(long long q_pos0, int t, int len) {
  long long n = q_pos0 + (long long)t + 1;
  if (n > len) n = len;
  if (n < 0) n = 0;
  return (int)n;
}

template <int D>
__global__ void __launch_bounds__(192, 1)
score_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmap_q,
                        const __grid_constant__ CUtensorMap tmap_k, TcParams p) {
  using S = TcShape<D>;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  unsigned char* base = smem_raw + ((1024 - (raw & 1023)) & 1023);  // 1024-byte aligned
  unsigned char* sA = base;
  unsigned char* sB = base + S::kABytes;
  TcBars& bars = *reinterpret_cast<TcBars*>(base + S::kABytes + S::kStages * S::kBBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int rb = p.nblk - 1 - blockIdx.x;  // long (late) row blocks first
  const int tr0 = p.t0 + rb * kBM;
  const int len = tc_row_len(p.kv_len, b, p.Tk);
  const int t_last = min(tr0 + kBM - 1, min(p.t0 + p.rows, p.Tq) - 1);
  long long nc = (long long)p.q_pos0 + t_last + 1;
  if (nc > len) nc = len;
  const int ntiles_all = nc > 0 ? (int)((nc + kBN - 1) / kBN) : 0;
  // key tiles [i_lo, i_lo + ntiles) of the row block: the block's causal
  // tiles are split evenly over gridDim.z CTAs (each score is written once)
  const int i_lo = (int)((long long)blockIdx.z * ntiles_all / gridDim.z);
  const int ntiles = (int)((long long)(blockIdx.z + 1) * ntiles_all / gridDim.z) - i_lo;
  if (ntiles <= 0 || t_last < tr0) return;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::kStages; ++s) { mbar_init(&bars.full[s], 1); mbar_init(&bars.empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&bars.tfull[a], 1); mbar_init(&bars.tempty[a], 4); }
    mbar_init(&bars.afull, 1);
    bars.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars.tmem_base;
  volatile int* abort_flag = &bars.abort;

  if (warp == 0) {
    if (lane == 0) {
      // producer
      mbar_arrive_expect_tx(&bars.afull, S::kABytes);
#pragma unroll
      for (int a = 0; a < S::kAtoms; ++a) tma_load_3d(sA + a * kBM * 128, &tmap_q, &bars.afull, 64 * a, tr0, b);
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % S::kStages;
        const uint32_t ph = (uint32_t)(i / S::kStages) & 1u;
        if (!mbar_wait(&bars.empty[s], ph ^ 1u, abort_flag, p.err, 1)) break;
        mbar_arrive_expect_tx(&bars.full[s], S::kBBytes);
#pragma unroll
        for (int a = 0; a < S::kAtoms; ++a)
          tma_load_3d(sB + s * S::kBBytes + a * kBN * 128, &tmap_k, &bars.full[s], 64 * a, (i_lo + i) * kBN, b);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // MMA issuer
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN);
      bool ok = mbar_wait(&bars.afull, 0, abort_flag, p.err, 2);
      const uint32_t a_addr = smem_u32(sA);
      for (int i = 0; ok && i < ntiles; ++i) {
        const int s = i % S::kStages;
        const uint32_t ph = (uint32_t)(i / S::kStages) & 1u;
        const int acc = i & 1;
        const uint32_t aph = (uint32_t)(i >> 1) & 1u;
        if (!mbar_wait(&bars.tempty[acc], aph ^ 1u, abort_flag, p.err, 3)) break;
        if (!mbar_wait(&bars.full[s], ph, abort_flag, p.err, 4)) break;
        tc_fence_after();
        const uint32_t b_addr = smem_u32(sB + s * S::kBBytes);
        const uint32_t d_tmem = tbase + (uint32_t)(acc * kBN);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (uint32_t)((kk & 3) * 32);  // 16 bf16 = 32 B within the atom
          const uint64_t adesc = sdesc_k_sw128(a_addr + (kk >> 2) * kBM * 128 + koff);
          const uint64_t bdesc = sdesc_k_sw128(b_addr + (kk >> 2) * kBN * 128 + koff);
          umma_bf16(d_tmem, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars.empty[s]);
        umma_commit(&bars.tfull[acc]);
      }
    }
  } else {
    // epilogue: warps 2..5; TMEM lane quarter = warp % 4
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int tq = tr0 + r;
    const bool row_ok = tq < p.t0 + p.rows && tq < p.Tq;
    const int lim = row_ok ? tc_n_cand(p.q_pos0, tq, len) : 0;
    uint32_t* krow = p.keys + ((long long)b * p.rows + (tq - p.t0)) * p.ld;
    for (int i = 0; i < ntiles; ++i) {
      const int acc = i & 1;
      const uint32_t aph = (uint32_t)(i >> 1) & 1u;
      if (!mbar_wait(&bars.tfull[acc], aph, abort_flag, p.err, 5)) break;
      tc_fence_after();
#pragma unroll 1
      for (int ch = 0; ch < kBN / 32; ++ch) {
        uint32_t v[32];
        tmem_ld32(tbase + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * kBN + ch * 32), v);
        tmem_ld_wait();
        const int c = (i_lo + i) * kBN + ch * 32;
        if (c < lim) {
          uint4* dst = reinterpret_cast<uint4*>(krow + c);
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            dst[q4] = make_uint4(score_key(__uint_as_float(v[4 * q4 + 0])), score_key(__uint_as_float(v[4 * q4 + 1])),
                                 score_key(__uint_as_float(v[4 * q4 + 2])), score_key(__uint_as_float(v[4 * q4 + 3])));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.tempty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, kTmemCols);
}

// ------------------------------------------------------------ tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// [batches][rows][d] bf16, box = 64 elements (128 B) x box_rows, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* ptr, int d, long long rows, int batches, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)batches};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)rows * d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_score_prefill(const uint16_t* q, const uint16_t* kmat, int B, int Tq, int d,
                                 int Tk_max, int Tk, int q_pos0, const int32_t* kv_len, int t0,
                                 int rows, const RowWorkspace& w, cudaStream_t st) {
  if (rows <= 0 || Tk <= 0 || B <= 0) return cudaSuccess;
  CUtensorMap mq, mk;
  if (!make_map(&mq, q, d, Tq, B, kBM) || !make_map(&mk, kmat, d, Tk_max, B, kBN))
    return cudaErrorInvalidValue;
  TcParams p;
  p.Tq = Tq;
  p.Tk = Tk;
  p.q_pos0 = q_pos0;
  p.kv_len = kv_len;
  p.t0 = t0;
  p.rows = rows;
  p.nblk = (rows + kBM - 1) / kBM;
  p.keys = w.keys;
  p.ld = w.ld;
  p.err = w.err;
  // key tiles of a row block are split over enough CTAs to fill the GPU
  // (one CTA per SM: 512 TMEM columns and ~150 KB of shared memory each)
  static int sms = 0;
  if (sms == 0) {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    sms = n > 0 ? n : 148;
  }
  const long long max_tiles = ((long long)q_pos0 + t0 + rows + kBN - 1) / kBN;   // of the last row block
  long long ks = (2LL * sms + (long long)p.nblk * B - 1) / ((long long)p.nblk * B);
  if (ks > max_tiles) ks = max_tiles;
  if (ks > 64) ks = 64;
  if (ks < 1) ks = 1;
  dim3 grid(p.nblk, B, (unsigned)ks);
  if (d == 128) {
    constexpr int smem = TcShape<128>::kSmem;
    cudaError_t e = ensure_dynamic_smem((const void*)score_prefill_tc_kernel<128>, smem);
    if (e != cudaSuccess) return e;
    score_prefill_tc_kernel<128><<<grid, 192, smem, st>>>(mq, mk, p);
  } else {
    constexpr int smem = TcShape<64>::kSmem;
    cudaError_t e = ensure_dynamic_smem((const void*)score_prefill_tc_kernel<64>, smem);
    if (e != cudaSuccess) return e;
    score_prefill_tc_kernel<64><<<grid, 192, smem, st>>>(mq, mk, p);
  }
  return cudaGetLastError();
}

}  // namespace sa
