// libpisa C ABI: argument checking, scratch layout and kernel launches.
// One translation unit: every kernel header is included here.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <cmath>
#include <mutex>
#include <string>

#include "pisa.h"
#include "pisa_common.cuh"
#include "k1_block_stats.cuh"
#include "k2_select.cuh"
#include "k2_scores_tc.cuh"
#include "k3_pack.cuh"
#include "k3_attention_tc.cuh"
#include "k5_tail_histogram.cuh"
#include "k6_backward.cuh"
#include "k7_bwd_dq_tc.cuh"
#include "k8_bwd_kv_tc.cuh"

namespace pisa {

static thread_local std::string t_last_error;

void set_last_error(cudaError_t e) {
  t_last_error = std::string(cudaGetErrorName(e)) + ": " + cudaGetErrorString(e);
}

pisa_status check_launch() {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_last_error(e);
    return PISA_ERR_CUDA;
  }
  return PISA_OK;
}

#define PISA_TRY(expr)                         \
  do {                                         \
    pisa_status _s = (expr);                   \
    if (_s != PISA_OK) return _s;              \
  } while (0)

#define PISA_CUDA(expr)                        \
  do {                                         \
    cudaError_t _e = (expr);                   \
    if (_e != cudaSuccess) {                   \
      set_last_error(_e);                      \
      return PISA_ERR_CUDA;                    \
    }                                          \
  } while (0)

static bool aligned16(const void *p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static pisa_status check_shape(int B, int H, int L, int d, int block_size) {
  if (B < 1 || H < 1 || L < 1 || d < 1 || block_size < 1) return PISA_ERR_INVALID_ARG;
  if ((long long)B * H > 65535) return PISA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return PISA_ERR_UNSUPPORTED;
  if (block_size != 64 && block_size != 128) return PISA_ERR_UNSUPPORTED;
  if ((long long)L > (1LL << 24)) return PISA_ERR_UNSUPPORTED;
  return PISA_OK;
}

// Shared memory of the fused kernel grows with the number of blocks (selection
// bitmaps and the tile list); shapes beyond the 227 KB a CTA can hold are
// refused before anything is launched.
static bool fused_fits(int d, int L, int block_size) {
  const int N = ceil_div(L, 64), Nc = ceil_div(L, block_size);
  const int smem = d == 128 ? TcCfg<128>::smem_bytes(N, Nc) : TcCfg<64>::smem_bytes(N, Nc);
  return smem <= 227 * 1024;
}
static bool bwd_fits(int d, int L, int block_size) {
  const int N = ceil_div(L, 64), Nc = ceil_div(L, block_size);
  const int smem = d == 128 ? DqTcCfg<128>::smem_bytes(N, Nc) : DqTcCfg<64>::smem_bytes(N, Nc);
  return smem <= 227 * 1024;
}

static int sink_block(int sink_idx, int N) {
  if (sink_idx == PISA_SINK_NONE) return -1;
  return sink_idx == 0 ? 0 : N - 1;
}

static bool sink_valid(int sink_idx) {
  return sink_idx == PISA_SINK_NONE || sink_idx == 0 || sink_idx == -1;
}

// ---- scratch sizes --------------------------------------------------------
// chunk partials of the f32 pass, or head-segment partials of the streamed bf16 pass
static size_t stats_ws(int B, int H, int L, int d, int block_size) {
  const int N = ceil_div(L, block_size), BH = B * H;
  const int parts = std::max(stats_num_chunks(BH, N), stats_max_segments(BH, N));
  return align_up((size_t)BH * parts * d * d * sizeof(float), 256);
}
// two-pass selection: the score matrix (rows padded to a multiple of 32 floats),
// then the three-part bf16 splits of qbar and kbar (sized for d = 128)
static int score_ld(int N) { return ceil_div(N, 32) * 32; }
struct SelectLayout {
  size_t qs, ks, total;
};
static SelectLayout select_layout(int B, int H, int N) {
  const size_t BH = (size_t)B * H;
  SelectLayout p;
  p.qs = align_up(BH * N * score_ld(N) * sizeof(float), 256);
  const size_t planes = align_up(BH * 3 * N * 128 * 2, 256);
  p.ks = p.qs + planes;
  p.total = p.ks + planes;
  return p;
}
static size_t select_ws(int B, int H, int N) { return select_layout(B, H, N).total; }
// scratch of the fused-attention step: bf16 kbar/vsum/hbar, query-block
// pairing (selection bitmaps, overlaps, pairs), bf16 copies of f32 inputs
struct SparseLayout {
  size_t kbar16, vsum16, hbar16, bm, ov, pairs, qkv16, total;
};
static SparseLayout sparse_layout(int B, int H, int L, int d, pisa_dtype dt) {
  const int N = ceil_div(L, 64), Npad = ceil_div(N, 64) * 64, nwords = ceil_div(N, 32);
  const size_t BH = (size_t)B * H;
  SparseLayout p;
  size_t o = 0;
  p.kbar16 = o; o += align_up(BH * Npad * d * 2, 256);
  p.vsum16 = o; o += align_up(BH * Npad * d * 2, 256);
  p.hbar16 = o; o += align_up(BH * d * d * 2, 256);
  p.bm = o; o += align_up(BH * N * nwords * 4, 256);
  p.ov = o; o += align_up(BH * N * kPairWindow * 2, 256);
  p.pairs = o; o += align_up(BH * ((N + 1) / 2) * 8, 256);
  p.qkv16 = o; o += dt == PISA_F32 ? 3 * align_up(BH * L * d * 2, 256) : 0;
  p.total = o;
  return p;
}
static size_t sparse_ws(int B, int H, int L, int d, pisa_dtype dt) {
  return sparse_layout(B, H, L, d, dt).total;
}

struct PathLayout {
  size_t qbar, kbar, vsum, hbar, cov, idx, scratch, total;
};

static PathLayout path_layout(int B, int H, int L, int d, int block_size, double density,
                              pisa_dtype dt, int want_cov) {
  const int N = ceil_div(L, block_size);
  const size_t BH = (size_t)B * H;
  const int k_sel = pisa_num_selected(N, density);
  PathLayout p;
  size_t o = 0;
  const size_t st = align_up(BH * N * d * sizeof(float), 256);
  p.qbar = o; o += st;
  p.kbar = o; o += st;
  p.vsum = o; o += st;
  p.hbar = o; o += align_up(BH * d * d * sizeof(float), 256);
  p.cov = o; o += want_cov ? align_up(BH * N * sizeof(float), 256) : 0;
  p.idx = o; o += align_up(BH * N * (size_t)(k_sel > 0 ? k_sel : 1) * sizeof(int32_t), 256);
  p.scratch = o;
  size_t s = stats_ws(B, H, L, d, block_size);
  s = s > select_ws(B, H, N) ? s : select_ws(B, H, N);
  const size_t a = sparse_ws(B, H, L, d, dt);
  s = s > a ? s : a;
  o += s;
  p.total = o;
  return p;
}

static unsigned grid_1d(size_t n, int threads) {
  size_t b = (n + threads - 1) / threads;
  if (b > 148 * 32) b = 148 * 32;
  return (unsigned)(b ? b : 1);
}

static pisa_status make_map(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows,
                            uint64_t planes, uint32_t box_rows);

// ---- launches ---------------------------------------------------------------
template <int D>
static pisa_status launch_stats(const void *q, const void *k, const void *v, pisa_dtype dt,
                                int BH, int L, int sub, int want_cov, float *qbar, float *kbar,
                                float *vsum, float *hbar, float *cov, float *partial,
                                cudaStream_t st) {
  const int N = ceil_div(L, 64 * sub);   // blocks of sub x 64 tokens
  const int nchunk = stats_num_chunks(BH, N);
  dim3 grid(nchunk, BH);
  bool streamed = false;
  if constexpr (D == 128) {
    if (dt == PISA_BF16) {
      // one CTA per SM streams a contiguous range of blocks through a TMA ring
      streamed = true;
      const long long total = (long long)BH * N;
      const int nc = stats_stream_ctas(total);
      const int maxseg = stats_max_segments(BH, N);
      CUtensorMap mq, mk, mv;
      PISA_TRY(make_map(&mq, q, D, L, BH, kBlk));
      PISA_TRY(make_map(&mk, k, D, L, BH, kBlk));
      PISA_TRY(make_map(&mv, v, D, L, BH, kBlk));
      PISA_CUDA(cudaFuncSetAttribute(stats_pass_tma_kernel<D>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     StatsTmaCfg<D>::kSmem));
      stats_pass_tma_kernel<D><<<nc, StatsTmaCfg<D>::kThreads, StatsTmaCfg<D>::kSmem, st>>>(
          mq, mk, mv, L, N, sub, BH, maxseg, qbar, kbar, vsum, partial);
      PISA_TRY(check_launch());
      hbar_reduce_seg_kernel<<<dim3(ceil_div(D * D, 256), BH), 256, 0, st>>>(
          partial, maxseg, D * D, N, BH, nc, hbar);
      PISA_TRY(check_launch());
      if (want_cov) {
        // pass 3 on the same ranges: K and V again, G_j on tcgen05
        PISA_CUDA(cudaFuncSetAttribute(cov_pass_tma_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       CovTmaCfg<D>::kSmem));
        cov_pass_tma_kernel<D><<<nc, CovTmaCfg<D>::kThreads, CovTmaCfg<D>::kSmem, st>>>(
            mk, mv, L, N, sub, BH, kbar, vsum, hbar, cov);
        PISA_TRY(check_launch());
      }
    }
  }
  if (streamed) {
    // done above
  } else if (dt == PISA_BF16) {
    // head dimension 64: chunked pass (cp.async double buffer, mma.sync)
    const int smem = 2 * 3 * StatsMmaCfg<D>::kTileBytes + 3 * D * (int)sizeof(float);
    PISA_CUDA(cudaFuncSetAttribute(stats_pass_bf16_kernel<D>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    stats_pass_bf16_kernel<D><<<grid, kStatsThreads, smem, st>>>(
        (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, L, N, sub,
        nchunk, qbar, kbar, vsum, partial);
    PISA_TRY(check_launch());
    hbar_reduce_kernel<<<dim3(ceil_div(D * D, 256), BH), 256, 0, st>>>(partial, nchunk, D * D,
                                                                        N, hbar);
    PISA_TRY(check_launch());
  } else {
    const int smem = 3 * kBlk * D * (int)sizeof(float) + 3 * D * (int)sizeof(float);
    PISA_CUDA(cudaFuncSetAttribute(stats_pass_f32_kernel<D>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    stats_pass_f32_kernel<D><<<grid, kStatsThreads, smem, st>>>(
        (const float *)q, (const float *)k, (const float *)v, L, N, sub, nchunk, qbar, kbar,
        vsum, partial);
    PISA_TRY(check_launch());
    hbar_reduce_kernel<<<dim3(ceil_div(D * D, 256), BH), 256, 0, st>>>(partial, nchunk, D * D,
                                                                        N, hbar);
    PISA_TRY(check_launch());
  }
  if (want_cov && !streamed) {
    if (dt == PISA_BF16) {
      const int smem = 2 * 2 * StatsMmaCfg<D>::kTileBytes + 32 * (int)sizeof(float);
      PISA_CUDA(cudaFuncSetAttribute(cov_pass_bf16_kernel<D>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
      cov_pass_bf16_kernel<D><<<grid, kStatsThreads, smem, st>>>(
          (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, L, N, sub, nchunk, kbar, vsum,
          hbar, cov);
    } else {
      const int smem = 2 * kBlk * D * (int)sizeof(float) + 32 * (int)sizeof(float);
      PISA_CUDA(cudaFuncSetAttribute(cov_pass_f32_kernel<D>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
      cov_pass_f32_kernel<D><<<dim3(N, BH), kStatsThreads, smem, st>>>(
          (const float *)k, (const float *)v, L, N, sub, kbar, vsum, hbar, cov);
    }
    PISA_TRY(check_launch());
  }
  return PISA_OK;
}

static pisa_status launch_select(const float *qbar, const float *kbar, const float *cov,
                                 float cov_weight, float scale, int BH, int N, int d, int k_sel,
                                 int sink, int32_t *idx, unsigned char *ws, cudaStream_t st) {
  float *scores = (float *)ws;   // [BH, N, N] for the two-pass path
  const int fsmem = select_fused_smem(N, d);
  if (N <= kSelFusedMaxN && fsmem <= 227 * 1024) {
    // short sequences: the score rows of a query-block group stay in shared
    // memory (for long ones the tiled two-pass path is faster: it streams each
    // k-bar tile once per 128 x 128 score tile instead of once per 24 rows)
    PISA_CUDA(cudaFuncSetAttribute(select_fused_kernel,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, fsmem));
    select_fused_kernel<<<dim3(ceil_div(N, kSelRows), BH), kSelThreads, fsmem, st>>>(
        qbar, kbar, cov, cov_weight, scale, N, d, k_sel, sink, idx);
    return check_launch();
  }
  // pass 1: three-part bf16 splits of the centroids, then the score tiles on
  // the tensor cores
  const SelectLayout lay = select_layout(1, BH, N);
  __nv_bfloat16 *qs = (__nv_bfloat16 *)(ws + lay.qs), *ks = (__nv_bfloat16 *)(ws + lay.ks);
  const long long rows = (long long)BH * N;
  centroid_split_kernel<<<grid_1d((size_t)rows * d / 4, 256), 256, 0, st>>>(qbar, kbar, rows, N,
                                                                             d, qs, ks);
  PISA_TRY(check_launch());
  CUtensorMap mqs, mks;
  PISA_TRY(make_map(&mqs, qs, d, N, (uint64_t)BH * 3, ScoreTcCfg<128>::kRows));
  PISA_TRY(make_map(&mks, ks, d, N, (uint64_t)BH * 3, ScoreTcCfg<128>::kCols));
  const int ld = score_ld(N);
  const dim3 g1(ceil_div(N, ScoreTcCfg<128>::kRows), BH);
  if (d == 128) {
    PISA_CUDA(cudaFuncSetAttribute(scores_tc_kernel<128>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   ScoreTcCfg<128>::kSmem));
    scores_tc_kernel<128><<<g1, ScoreTcCfg<128>::kThreads, ScoreTcCfg<128>::kSmem, st>>>(
        mqs, mks, cov, cov_weight, scale, N, ld, scores);
  } else {
    PISA_CUDA(cudaFuncSetAttribute(scores_tc_kernel<64>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   ScoreTcCfg<64>::kSmem));
    scores_tc_kernel<64><<<g1, ScoreTcCfg<64>::kThreads, ScoreTcCfg<64>::kSmem, st>>>(
        mqs, mks, cov, cov_weight, scale, N, ld, scores);
  }
  PISA_TRY(check_launch());
  // pass 2: one warp per query block, its row staged in shared memory (rows
  // too long for eight of them in shared memory: the radix select from L2)
  const int per_cta = kTopkThreads / 32;
  const unsigned g2 = (unsigned)((rows + per_cta - 1) / per_cta);
  const int tsmem = topk_bins_smem(ld);
  if (tsmem <= 227 * 1024) {
    PISA_CUDA(cudaFuncSetAttribute(topk_bins_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   tsmem));
    topk_bins_kernel<<<g2, kTopkThreads, tsmem, st>>>(scores, N, ld, k_sel, sink, rows, idx);
  } else
    topk_kernel<<<g2, kTopkThreads, 0, st>>>(scores, N, ld, k_sel, sink, rows, idx);
  return check_launch();
}

// ---- tensor maps for the tensor-memory-accelerator loads ------------------------
using EncodeTiledFn = PFN_cuTensorMapEncodeTiled_v12000;

static EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 tensor [planes][rows][cols] (cols contiguous, cols multiple of 64), read
// in boxes of 64 columns x box_rows rows with the 128-byte swizzle; rows past
// `rows` read as zero.
static pisa_status make_map(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows,
                            uint64_t planes, uint32_t box_rows) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc) {
    t_last_error = "cuTensorMapEncodeTiled is not available from the driver";
    return PISA_ERR_CUDA;
  }
  cuuint64_t dims[3] = {cols, rows, planes};
  cuuint64_t strides[2] = {cols * 2, rows * cols * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    t_last_error = "cuTensorMapEncodeTiled failed with CUresult " + std::to_string((int)r);
    return PISA_ERR_CUDA;
  }
  return PISA_OK;
}

template <int D>
static pisa_status launch_attention_kernel(const __nv_bfloat16 *q, const __nv_bfloat16 *k,
                                           const __nv_bfloat16 *v, const __nv_bfloat16 *kbar16,
                                           const __nv_bfloat16 *vsum16,
                                           const __nv_bfloat16 *hbar16, const int32_t *idx,
                                           const int2 *pairs, int k_sel, int BH, int L, int bsub,
                                           float scale, int hyd, int dense, int blockwise,
                                           void *out, int out_f32, float *lse,
                                           float *o_keep, cudaStream_t st,
                                           const FusedSelect &fsel = FusedSelect{}) {
  const int N = ceil_div(L, 64);
  const int Nc = ceil_div(L, 64 * bsub), Ncpad = ceil_div(Nc, 64) * 64;
  const int smem = TcCfg<D>::smem_bytes(N, Nc);
  if (smem > 227 * 1024) return PISA_ERR_UNSUPPORTED;
  CUtensorMap mq, mk, mv, mkb, mvs, mh;
  PISA_TRY(make_map(&mq, q, D, L, BH, 64));
  PISA_TRY(make_map(&mk, k, D, L, BH, 64));
  PISA_TRY(make_map(&mv, v, D, L, BH, 64));
  if (dense) {
    mkb = mk;
    mvs = mv;
    mh = mk;
  } else {
    PISA_TRY(make_map(&mkb, kbar16, D, Ncpad, BH, 64));
    PISA_TRY(make_map(&mvs, vsum16, D, Ncpad, BH, 64));
    PISA_TRY(make_map(&mh, hbar16, D, D, BH, D));
  }
  PISA_CUDA(cudaFuncSetAttribute(piecewise_attention_tc_kernel<D>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  piecewise_attention_tc_kernel<D><<<dim3(ceil_div(N, 2), BH), TcCfg<D>::kThreads, smem, st>>>(
      mq, mk, mv, mkb, mvs, mh, idx, pairs, k_sel, L, N, bsub, Nc, scale, hyd, dense, blockwise,
      out, out_f32, lse, o_keep, fsel);
  return check_launch();
}

static pisa_status to_bf16(const void *src, __nv_bfloat16 *dst, size_t n, cudaStream_t st) {
  f32_to_bf16_kernel<<<grid_1d(n, 256), 256, 0, st>>>((const float *)src, dst, n);
  return check_launch();
}

static pisa_status run_sparse_attention(const void *q, const void *k, const void *v,
                                        pisa_dtype dt, const float *kbar, const float *vsum,
                                        const float *hbar, const int32_t *idx, int k_sel, int BH,
                                        int L, int d, int bsub, float scale, pisa_mode mode,
                                        void *out, float *lse, float *o_keep,
                                        unsigned char *ws, cudaStream_t st,
                                        const FusedSelect &fsel = FusedSelect{}) {
  // N 64-token tiles; Nc blocks of bsub tiles (the selection's and the
  // centroids' index space); with bsub = 1 they coincide
  const int N = ceil_div(L, 64), nwords = ceil_div(N, 32);
  const int Nc = ceil_div(L, 64 * bsub), Ncpad = ceil_div(Nc, 64) * 64;
  const SparseLayout lay = sparse_layout(1, BH, L, d, dt);
  __nv_bfloat16 *kbar16 = (__nv_bfloat16 *)(ws + lay.kbar16);
  __nv_bfloat16 *vsum16 = (__nv_bfloat16 *)(ws + lay.vsum16);
  __nv_bfloat16 *hbar16 = (__nv_bfloat16 *)(ws + lay.hbar16);
  uint32_t *bm = (uint32_t *)(ws + lay.bm);
  uint16_t *ov = (uint16_t *)(ws + lay.ov);
  int2 *pairs = (int2 *)(ws + lay.pairs);
  if (bsub == 1) {
    // statistics packing and the selection bitmap in one launch; then the
    // schedule: pair query blocks whose exact sets overlap most
    const unsigned npack = grid_1d((size_t)BH * (Ncpad * d + d * d), kPackThreads);
    pack_and_bitmap_kernel<<<(unsigned)((size_t)N * BH) + npack, kPackThreads,
                             nwords * sizeof(uint32_t), st>>>(
        kbar, vsum, hbar, Nc, Ncpad, d, BH, kbar16, vsum16, hbar16, idx, k_sel, nwords, bm);
    PISA_TRY(check_launch());
    pair_overlap_kernel<<<dim3(ceil_div(N, 8), BH), 256, 0, st>>>(bm, N, nwords, ov);
    PISA_TRY(check_launch());
    const int staged = N * (kPairWindow * 2 + 1) <= 200 * 1024;
    const int pair_smem = staged ? N * (kPairWindow * 2 + 1) : N;
    if (pair_smem > 48 * 1024)
      PISA_CUDA(cudaFuncSetAttribute(pairing_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     pair_smem));
    pairing_kernel<<<BH, kPairThreads, pair_smem, st>>>(ov, N, staged, pairs);
    PISA_TRY(check_launch());
  } else {
    pack_stats_kernel<<<grid_1d((size_t)BH * (Ncpad * d + d * d), 256), 256, 0, st>>>(
        kbar, vsum, hbar, Nc, Ncpad, d, BH, kbar16, vsum16, hbar16);
    PISA_TRY(check_launch());
    pairs = nullptr;   // the two 64-row halves of one 128-token query block share S_i
  }
  const __nv_bfloat16 *q16 = (const __nv_bfloat16 *)q, *k16 = (const __nv_bfloat16 *)k,
                      *v16 = (const __nv_bfloat16 *)v;
  if (dt == PISA_F32) {
    const size_t n = (size_t)BH * L * d, sz = align_up(n * 2, 256);
    unsigned char *next = ws + lay.qkv16;
    __nv_bfloat16 *a = (__nv_bfloat16 *)next, *b = (__nv_bfloat16 *)(next + sz),
                  *c = (__nv_bfloat16 *)(next + 2 * sz);
    PISA_TRY(to_bf16(q, a, n, st));
    PISA_TRY(to_bf16(k, b, n, st));
    PISA_TRY(to_bf16(v, c, n, st));
    q16 = a;
    k16 = b;
    v16 = c;
  }
  const int hyd = mode == PISA_MODE_HYD;
  const int blockwise = mode == PISA_MODE_1ST;
  const int of32 = dt == PISA_F32;
  if (d == 128)
    return launch_attention_kernel<128>(q16, k16, v16, kbar16, vsum16, hbar16, idx, pairs, k_sel,
                                        BH, L, bsub, scale, hyd, 0, blockwise, out, of32, lse,
                                        o_keep, st, fsel);
  return launch_attention_kernel<64>(q16, k16, v16, kbar16, vsum16, hbar16, idx, pairs, k_sel, BH,
                                     L, bsub, scale, hyd, 0, blockwise, out, of32, lse, o_keep,
                                     st, fsel);
}

// ---- backward of the zeroth-order variant ------------------------------------
struct BwdLayout {
  size_t lse_pad, delta, kbar16, vbar16, bm, ov, pairs, bmT, kpairs, dkbar, dvbar, counts,
      offsets, entries, total;
  long long cap;   // list entries per head
};
static BwdLayout bwd_layout(int B, int H, int L, int d, int k_sel, int block_size) {
  // N 64-token tiles; Nc blocks (= N with 64-token blocks)
  const int N = ceil_div(L, 64), Nc = ceil_div(L, block_size);
  const int Npad = ceil_div(Nc, 64) * 64, nwords = ceil_div(Nc, 32);
  const int Lpad = N * 64, P = (N + 1) / 2;
  const size_t BH = (size_t)B * H;
  BwdLayout p;
  size_t o = 0;
  p.lse_pad = o; o += align_up(BH * Lpad * 4, 256);
  p.delta = o; o += align_up(BH * Lpad * 4, 256);
  p.kbar16 = o; o += align_up(BH * Npad * d * 2, 256);
  p.vbar16 = o; o += align_up(BH * Npad * d * 2, 256);
  p.bm = o; o += align_up(BH * N * nwords * 4, 256);
  p.ov = o; o += align_up(BH * N * kPairWindow * 2, 256);
  p.pairs = o; o += align_up(BH * P * 8, 256);
  // key-block pairs of the dk / dv pass (64-token blocks): the transposed
  // bitmap, then pairs chosen like the query pairs (ov is reused)
  p.bmT = o; o += block_size == 64 ? align_up(BH * N * nwords * 4, 256) : 0;
  p.kpairs = o; o += block_size == 64 ? align_up(BH * P * 8, 256) : 0;
  p.dkbar = o; o += align_up(BH * Npad * d * 4, 256);
  p.dvbar = o; o += align_up(BH * Npad * d * 4, 256);
  p.counts = o; o += align_up(BH * P * 4, 256);
  p.offsets = o; o += align_up(BH * P * 8, 256);
  // the lists of a head hold each selected (query block, key block) pair at most
  // once, as one (64-token blocks) or two (128-token blocks) query tiles
  p.cap = (long long)(block_size == 64 ? N : 2 * Nc) * k_sel;
  p.entries = o; o += align_up(BH * (size_t)p.cap * 4, 256);
  p.total = o;
  return p;
}

// f32 [rows, cols] map with 64-element boxes of one row (per-row vectors)
static pisa_status make_map_f32_rows(CUtensorMap *m, const void *base, uint64_t cols,
                                     uint64_t rows) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc) {
    t_last_error = "cuTensorMapEncodeTiled is not available from the driver";
    return PISA_ERR_CUDA;
  }
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 4};
  cuuint32_t box[2] = {64, 1};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    t_last_error = "cuTensorMapEncodeTiled failed with CUresult " + std::to_string((int)r);
    return PISA_ERR_CUDA;
  }
  return PISA_OK;
}

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

// Unique id of the calling thread's current context (cuCtxGetId: ids are never
// reused within a process), or 0 when there is none or the driver lacks the call.
static unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// A second stream of this thread on the current device, with two events, for
// work of one call that may run beside the work on the caller's stream: it
// starts after an event recorded on that stream and the caller's stream waits
// for it before going on, so to the caller everything stays ordered on its
// stream (graph capture included).  Created once, kept for the process.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  unsigned long long ctx = 0;   // context the handles belong to
};

static pisa_status side_stream(SideStream **out) {
  int dev = 0;
  PISA_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) {
    t_last_error = "side stream: device ordinal " + std::to_string(dev) + " out of range";
    return PISA_ERR_UNSUPPORTED;
  }
  static thread_local SideStream cache[64];
  SideStream &ss = cache[dev];
  // after cudaDeviceReset the old handles died with their context: make new ones
  const unsigned long long ctx = current_context_id();
  if (ss.s == nullptr || ctx == 0 || ctx != ss.ctx) {
    int lo = 0, hi = 0;
    PISA_CUDA(cudaDeviceGetStreamPriorityRange(&lo, &hi));
    cudaStream_t s = nullptr;
    PISA_CUDA(cudaStreamCreateWithPriority(&s, cudaStreamNonBlocking, hi));
    cudaEvent_t f = nullptr, j = nullptr;
    PISA_CUDA(cudaEventCreateWithFlags(&f, cudaEventDisableTiming));
    PISA_CUDA(cudaEventCreateWithFlags(&j, cudaEventDisableTiming));
    ss.s = s;
    ss.fork = f;
    ss.join = j;
    ss.ctx = ctx;
  }
  *out = &ss;
  return PISA_OK;
}

template <int D>
static pisa_status launch_bwd(const __nv_bfloat16 *q, const __nv_bfloat16 *k,
                              const __nv_bfloat16 *v, const __nv_bfloat16 *dout, const float *lse,
                              const float *o32, const int32_t *idx, int k_sel, int BH, int L,
                              int bsub, float scale, const BwdLayout &lay, unsigned char *ws,
                              __nv_bfloat16 *dq,
                              __nv_bfloat16 *dk, __nv_bfloat16 *dv, cudaStream_t st) {
  // N 64-token tiles, Nc blocks of bsub tiles (the selection's and the
  // centroids' index space)
  const int N = ceil_div(L, 64), Nc = ceil_div(L, 64 * bsub);
  const int Ncpad = ceil_div(Nc, 64) * 64, cwords = ceil_div(Nc, 32);
  const int Lpad = N * 64, P = (N + 1) / 2;
  float *lse_pad = (float *)(ws + lay.lse_pad);
  float *delta = (float *)(ws + lay.delta);
  const __nv_bfloat16 *kb = (const __nv_bfloat16 *)(ws + lay.kbar16);
  const __nv_bfloat16 *vb = (const __nv_bfloat16 *)(ws + lay.vbar16);
  uint32_t *bm = (uint32_t *)(ws + lay.bm);
  float *dkbar = (float *)(ws + lay.dkbar), *dvbar = (float *)(ws + lay.dvbar);
  int *counts = (int *)(ws + lay.counts);
  long long *offsets = (long long *)(ws + lay.offsets);
  int *entries = (int *)(ws + lay.entries);
  pad_lse_kernel<<<grid_1d((size_t)BH * Lpad, 256), 256, 0, st>>>(lse, L, Lpad, BH, lse_pad);
  PISA_TRY(check_launch());
  // dq on the tensor cores: with 64-token blocks the query blocks are paired
  // like the forward's; with 128-token blocks a CTA is one query block
  int2 *pairs = nullptr;
  if (bsub == 1) {
    uint16_t *ov = (uint16_t *)(ws + lay.ov);
    pairs = (int2 *)(ws + lay.pairs);
    pair_overlap_kernel<<<dim3(ceil_div(N, 8), BH), 256, 0, st>>>(bm, N, cwords, ov);
    PISA_TRY(check_launch());
    const int staged = N * (kPairWindow * 2 + 1) <= 200 * 1024;
    const int pair_smem = staged ? N * (kPairWindow * 2 + 1) : N;
    if (pair_smem > 48 * 1024)
      PISA_CUDA(cudaFuncSetAttribute(pairing_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     pair_smem));
    pairing_kernel<<<BH, kPairThreads, pair_smem, st>>>(ov, N, staged, pairs);
    PISA_TRY(check_launch());
  }
  const int dq_smem = DqTcCfg<D>::smem_bytes(N, Nc);
  if (dq_smem > 227 * 1024) return PISA_ERR_UNSUPPORTED;
  CUtensorMap mq, mdo, mk, mv, mkb, mvb, mlse, mdel;
  PISA_TRY(make_map(&mq, q, D, L, BH, 64));
  PISA_TRY(make_map(&mdo, dout, D, L, BH, 64));
  PISA_TRY(make_map(&mk, k, D, L, BH, 64));
  PISA_TRY(make_map(&mv, v, D, L, BH, 64));
  PISA_TRY(make_map(&mkb, kb, D, Ncpad, BH, 64));
  PISA_TRY(make_map(&mvb, vb, D, Ncpad, BH, 64));
  PISA_TRY(make_map_f32_rows(&mlse, lse_pad, Lpad, BH));
  PISA_TRY(make_map_f32_rows(&mdel, delta, Lpad, BH));
  PISA_CUDA(cudaFuncSetAttribute(bwd_dq_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 dq_smem));
  if (o32) {
    // Delta from the forward's float32 output: the dq kernel then makes one sweep
    bwd_delta_kernel<<<grid_1d((size_t)BH * Lpad * 32, 256), 256, 0, st>>>(dout, o32, L, Lpad, D,
                                                                          BH, delta);
    PISA_TRY(check_launch());
  }
  // With Delta given, the centroid gradients, the key-block pairing and the
  // query-tile lists need nothing from dq: they run on a side stream beside it
  // (high priority, so their few CTAs are placed as dq's CTAs retire), and the
  // exact keys' dk, dv wait for both.  With the Delta sweep, dq writes Delta
  // and everything runs in order on the caller's stream.
  cudaStream_t ss = st;
  SideStream *side = nullptr;
  if (o32) {
    PISA_TRY(side_stream(&side));
    PISA_CUDA(cudaEventRecord(side->fork, st));
    PISA_CUDA(cudaStreamWaitEvent(side->s, side->fork, 0));
    ss = side->s;
  }
  // on every return from here on, the caller's stream waits for the side
  // stream's work (so an early error never leaves kernels running on a
  // workspace the caller may free)
  struct JoinGuard {
    SideStream *side;
    cudaStream_t ss, st;
    cudaError_t join() {
      if (!side) return cudaSuccess;
      cudaError_t e = cudaEventRecord(side->join, ss);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(st, side->join, 0);
      side = nullptr;
      return e;
    }
    ~JoinGuard() { join(); }
  } guard{side, ss, st};
  bwd_dq_tc_kernel<D><<<dim3(P, BH), DqTcCfg<D>::kThreads, dq_smem, st>>>(
      mq, mdo, mk, mv, mkb, mvb, idx, pairs, k_sel, L, N, bsub, Nc, scale, lse, delta,
      o32 != nullptr, Lpad, dq);
  PISA_TRY(check_launch());
  // centroid gradients, then the exact keys' dk, dv, both on the tensor cores
  // (the exact pass over the query-tile lists of each key-block pair)
  const int kvtc_smem = KvTcCfg<D>::kSmem;
  PISA_CUDA(cudaFuncSetAttribute(bwd_kv_tc_kernel<D, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, kvtc_smem));
  PISA_CUDA(cudaFuncSetAttribute(bwd_kv_tc_kernel<D, false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, kvtc_smem));
  bwd_kv_tc_kernel<D, true><<<dim3(ceil_div(Ncpad, 128), BH), KvTcCfg<D>::kThreads, kvtc_smem,
                              ss>>>(
      mq, mdo, mkb, mvb, mlse, mdel, nullptr, nullptr, 0, nullptr, nullptr, bm, cwords, bsub, Nc,
      L, N, scale, dkbar, dvbar, Ncpad, nullptr, nullptr);
  PISA_TRY(check_launch());
  // 64-token blocks: key blocks paired by how many query blocks select both
  // (the dk / dv tiles of a query block that selected only one of the two are
  // half wasted), with the query pairing's greedy over the transposed bitmap
  int2 *kpairs = nullptr;
  if (bsub == 1) {
    uint32_t *bmT = (uint32_t *)(ws + lay.bmT);
    uint16_t *ov = (uint16_t *)(ws + lay.ov);
    kpairs = (int2 *)(ws + lay.kpairs);
    bitmap_transpose_kernel<<<dim3(cwords, cwords, BH), 32, 0, ss>>>(bm, N, cwords, bmT);
    PISA_TRY(check_launch());
    pair_overlap_kernel<<<dim3(ceil_div(N, 8), BH), 256, 0, ss>>>(bmT, N, cwords, ov);
    PISA_TRY(check_launch());
    const int staged = N * (kPairWindow * 2 + 1) <= 200 * 1024;
    const int pair_smem = staged ? N * (kPairWindow * 2 + 1) : N;
    if (pair_smem > 48 * 1024)
      PISA_CUDA(cudaFuncSetAttribute(pairing_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     pair_smem));
    pairing_kernel<<<BH, kPairThreads, pair_smem, ss>>>(ov, N, staged, kpairs);
    PISA_TRY(check_launch());
  }
  kvlist_kernel<<<dim3(P, BH), 32, 0, ss>>>(bm, N, Nc, cwords, bsub, P, kpairs, 0, counts,
                                            offsets, lay.cap, entries);
  PISA_TRY(check_launch());
  kvlist_scan_kernel<<<BH, 1024, 0, ss>>>(counts, P, offsets);
  PISA_TRY(check_launch());
  kvlist_kernel<<<dim3(P, BH), 32, 0, ss>>>(bm, N, Nc, cwords, bsub, P, kpairs, 1, counts,
                                            offsets, lay.cap, entries);
  PISA_TRY(check_launch());
  PISA_CUDA(guard.join());
  bwd_kv_tc_kernel<D, false><<<dim3(P, BH), KvTcCfg<D>::kThreads, kvtc_smem, st>>>(
      mq, mdo, mk, mv, mlse, mdel, counts, offsets, lay.cap, entries, kpairs, bm, cwords, bsub,
      Nc, L, N, scale, dkbar, dvbar, Ncpad, dk, dv);
  return check_launch();
}

}  // namespace pisa

using namespace pisa;

// ---------------------------------------------------------------------------
// pisa_block_stats_noalloc: scratch in a static device array
// ---------------------------------------------------------------------------
// Chunk partial sums of the statistics pass live here instead of in a caller
// workspace.  The host-side symbol is only a stand-in: kernels must be given
// the device address that cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[PISA_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
// per device: the array's device address and the unique id of the context it
// was looked up in (0 = not looked up yet)
void *g_noalloc_ptr[kMaxDevices] = {nullptr};
unsigned long long g_noalloc_ctx[kMaxDevices] = {0};

// Device address of g_noalloc_scratch on the current device.  Looked up with
// the device current on the first call on each device, and again whenever the
// device's context has changed since (cudaDeviceReset destroys the context and
// the array with it; the next context holds a fresh copy at a new address).
pisa_status noalloc_scratch(void **out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    set_last_error(e);
    return PISA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    t_last_error = "pisa_block_stats_noalloc: device ordinal " + std::to_string(dev) +
                   " is beyond the " + std::to_string(kMaxDevices) + " devices it supports";
    return PISA_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  const unsigned long long ctx = current_context_id();
  if (!g_noalloc_ptr[dev] || ctx == 0 || ctx != g_noalloc_ctx[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      set_last_error(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
      return PISA_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = p;
    // the lookup makes the device's primary context current if none was
    g_noalloc_ctx[dev] = current_context_id();
  }
  *out = g_noalloc_ptr[dev];
  return PISA_OK;
}
}  // namespace


// =============================================================================
// C ABI
// =============================================================================
extern "C" {

int pisa_num_blocks(int L, int block_size) {
  if (L < 1 || block_size < 1) return -1;
  return ceil_div(L, block_size);
}

int pisa_num_selected(int N, double density) {
  if (N < 1 || !(density > 0.0) || density > 1.0) return -1;
  double k = std::floor(density * (double)N + 1e-6);
  if (k < 1.0) k = 1.0;
  if (k > (double)N) k = (double)N;
  return (int)k;
}

size_t pisa_block_stats_workspace_bytes(int B, int H, int L, int d, int block_size) {
  if (check_shape(B, H, L, d, block_size) != PISA_OK) return 0;
  return stats_ws(B, H, L, d, block_size);
}

size_t pisa_select_workspace_bytes(int B, int H, int N) {
  if (B < 1 || H < 1 || N < 1) return 0;
  return select_ws(B, H, N);
}

size_t pisa_sparse_attention_workspace_bytes(int B, int H, int L, int d, int block_size,
                                             pisa_dtype dtype) {
  if (check_shape(B, H, L, d, block_size) != PISA_OK) return 0;
  return sparse_ws(B, H, L, d, dtype);
}

size_t pisa_workspace_bytes(int B, int H, int L, int d, int block_size, double density,
                            pisa_dtype dtype, int want_cov) {
  if (check_shape(B, H, L, d, block_size) != PISA_OK) return 0;
  if (pisa_num_selected(ceil_div(L, block_size), density) < 1) return 0;
  return path_layout(B, H, L, d, block_size, density, dtype, want_cov).total;
}

pisa_status pisa_block_stats(const void *q, const void *k, const void *v, pisa_dtype dtype,
                             int B, int H, int L, int d, int block_size, int want_cov,
                             float *qbar, float *kbar, float *vsum, float *hbar, float *cov,
                             void *workspace, size_t ws_bytes, pisa_stream_t stream) {
  PISA_TRY(check_shape(B, H, L, d, block_size));
  if (dtype != PISA_BF16 && dtype != PISA_F32) return PISA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(qbar) || !aligned16(kbar) ||
      !aligned16(vsum) || !aligned16(hbar) || !aligned16(workspace))
    return PISA_ERR_INVALID_ARG;
  if (want_cov && !aligned16(cov)) return PISA_ERR_INVALID_ARG;
  if (ws_bytes < stats_ws(B, H, L, d, block_size)) return PISA_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  float *partial = (float *)workspace;
  const int sub = block_size / 64;
  if (d == 128)
    return launch_stats<128>(q, k, v, dtype, B * H, L, sub, want_cov, qbar, kbar, vsum, hbar,
                             cov, partial, st);
  return launch_stats<64>(q, k, v, dtype, B * H, L, sub, want_cov, qbar, kbar, vsum, hbar, cov,
                          partial, st);
}

pisa_status pisa_select(const float *qbar, const float *kbar, const float *cov, float cov_weight,
                        float scale, int B, int H, int N, int d, double density, int sink_idx,
                        int32_t *idx, void *workspace, size_t ws_bytes, pisa_stream_t stream) {
  if (B < 1 || H < 1 || N < 1 || (d != 64 && d != 128)) return PISA_ERR_INVALID_ARG;
  if ((long long)B * H > 65535) return PISA_ERR_UNSUPPORTED;
  if ((long long)N * 4 > 200 * 1024) return PISA_ERR_UNSUPPORTED;
  if (!sink_valid(sink_idx) || !std::isfinite(scale) || !std::isfinite(cov_weight))
    return PISA_ERR_INVALID_ARG;
  const int k_sel = pisa_num_selected(N, density);
  if (k_sel < 1) return PISA_ERR_INVALID_ARG;
  if (!aligned16(qbar) || !aligned16(kbar) || !idx || !aligned16(workspace))
    return PISA_ERR_INVALID_ARG;
  if (cov_weight != 0.f && !cov) return PISA_ERR_INVALID_ARG;
  if (ws_bytes < select_ws(B, H, N)) return PISA_ERR_WORKSPACE;
  return launch_select(qbar, kbar, cov, cov_weight, scale, B * H, N, d, k_sel,
                       sink_block(sink_idx, N), idx, (unsigned char *)workspace,
                       (cudaStream_t)stream);
}

static pisa_status sparse_attention_checked(const void *q, const void *k, const void *v,
                                            pisa_dtype dtype, const float *kbar,
                                            const float *vsum, const float *hbar,
                                            const int32_t *idx, int k_sel, int B, int H, int L,
                                            int d, int block_size, float scale, pisa_mode mode,
                                            void *out, float *lse, float *o_keep,
                                            void *workspace, size_t ws_bytes,
                                            pisa_stream_t stream) {
  PISA_TRY(check_shape(B, H, L, d, block_size));
  if (dtype != PISA_BF16 && dtype != PISA_F32) return PISA_ERR_INVALID_ARG;
  if (mode != PISA_MODE_HYD && mode != PISA_MODE_0TH && mode != PISA_MODE_1ST) return PISA_ERR_INVALID_ARG;
  if (mode == PISA_MODE_1ST && block_size != 64) return PISA_ERR_UNSUPPORTED;
  if (!fused_fits(d, L, block_size)) return PISA_ERR_UNSUPPORTED;
  const int N = ceil_div(L, block_size);
  if (k_sel < 1 || k_sel > N) return PISA_ERR_INVALID_ARG;
  if (!(scale >= 0.f) || !std::isfinite(scale)) return PISA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(kbar) ||
      !aligned16(vsum) || !aligned16(hbar) || !idx || !aligned16(workspace))
    return PISA_ERR_INVALID_ARG;
  if (out == q || out == k || out == v) return PISA_ERR_INVALID_ARG;
  if (o_keep && (!aligned16(o_keep) || (void *)o_keep == out || (const void *)o_keep == q ||
                 (const void *)o_keep == k || (const void *)o_keep == v))
    return PISA_ERR_INVALID_ARG;
  if (ws_bytes < sparse_ws(B, H, L, d, dtype)) return PISA_ERR_WORKSPACE;
  const float s = scale == 0.f ? 1.f / std::sqrt((float)d) : scale;
  return run_sparse_attention(q, k, v, dtype, kbar, vsum, hbar, idx, k_sel, B * H, L, d,
                              block_size / 64, s, mode, out, lse, o_keep,
                              (unsigned char *)workspace, (cudaStream_t)stream);
}

pisa_status pisa_sparse_attention(const void *q, const void *k, const void *v, pisa_dtype dtype,
                                  const float *kbar, const float *vsum, const float *hbar,
                                  const int32_t *idx, int k_sel, int B, int H, int L, int d,
                                  int block_size, float scale, pisa_mode mode, void *out,
                                  void *workspace, size_t ws_bytes, pisa_stream_t stream) {
  return sparse_attention_checked(q, k, v, dtype, kbar, vsum, hbar, idx, k_sel, B, H, L, d,
                                  block_size, scale, mode, out, nullptr, nullptr, workspace,
                                  ws_bytes, stream);
}

pisa_status pisa_sparse_attention_fwd(const void *q, const void *k, const void *v,
                                      pisa_dtype dtype, const float *kbar, const float *vsum,
                                      const float *hbar, const int32_t *idx, int k_sel, int B,
                                      int H, int L, int d, int block_size, float scale,
                                      pisa_mode mode, void *out, float *lse, float *out_f32,
                                      void *workspace, size_t ws_bytes, pisa_stream_t stream) {
  if (!lse || (reinterpret_cast<uintptr_t>(lse) & 3u)) return PISA_ERR_INVALID_ARG;
  return sparse_attention_checked(q, k, v, dtype, kbar, vsum, hbar, idx, k_sel, B, H, L, d,
                                  block_size, scale, mode, out, lse, out_f32, workspace, ws_bytes,
                                  stream);
}

size_t pisa_sparse_attention_bwd_workspace_bytes(int B, int H, int L, int d, int block_size,
                                                 int k_sel) {
  if (check_shape(B, H, L, d, block_size) != PISA_OK) return 0;
  if (k_sel < 1 || k_sel > ceil_div(L, block_size)) return 0;
  return bwd_layout(B, H, L, d, k_sel, block_size).total;
}

pisa_status pisa_sparse_attention_bwd(const void *q, const void *k, const void *v,
                                      const void *dout, const float *lse, const float *out_f32,
                                      const float *kbar, const float *vsum, const int32_t *idx,
                                      int k_sel, int B, int H, int L, int d, int block_size,
                                      float scale, void *dq, void *dk, void *dv, void *workspace,
                                      size_t ws_bytes, pisa_stream_t stream) {
  PISA_TRY(check_shape(B, H, L, d, block_size));
  if (!bwd_fits(d, L, block_size)) return PISA_ERR_UNSUPPORTED;
  // Nc blocks of block_size tokens (the selection's index space)
  const int Nc = ceil_div(L, block_size), Ncpad = ceil_div(Nc, 64) * 64,
            cwords = ceil_div(Nc, 32);
  if (k_sel < 1 || k_sel > Nc) return PISA_ERR_INVALID_ARG;
  if (!(scale >= 0.f) || !std::isfinite(scale)) return PISA_ERR_INVALID_ARG;
  const void *ins[] = {q, k, v, dout};
  void *outs[] = {dq, dk, dv};
  for (const void *p : ins)
    if (!aligned16(p)) return PISA_ERR_INVALID_ARG;
  for (void *p : outs) {
    if (!aligned16(p)) return PISA_ERR_INVALID_ARG;
    for (const void *i : ins)
      if (p == i) return PISA_ERR_INVALID_ARG;
  }
  if (dq == dk || dq == dv || dk == dv) return PISA_ERR_INVALID_ARG;
  if (out_f32 && !aligned16(out_f32)) return PISA_ERR_INVALID_ARG;
  for (void *p : outs)
    if (out_f32 && p == (const void *)out_f32) return PISA_ERR_INVALID_ARG;
  if (!lse || (reinterpret_cast<uintptr_t>(lse) & 3u) || !aligned16(kbar) || !aligned16(vsum) ||
      !idx || !aligned16(workspace))
    return PISA_ERR_INVALID_ARG;
  const BwdLayout lay = bwd_layout(B, H, L, d, k_sel, block_size);
  if (ws_bytes < lay.total) return PISA_ERR_WORKSPACE;
  const float s = scale == 0.f ? 1.f / std::sqrt((float)d) : scale;
  const int BH = B * H;
  cudaStream_t st = (cudaStream_t)stream;
  unsigned char *ws = (unsigned char *)workspace;
  bwd_pack_centroids_kernel<<<grid_1d((size_t)BH * Ncpad * d, 256), 256, 0, st>>>(
      kbar, vsum, Nc, Ncpad, d, BH, L, block_size, (__nv_bfloat16 *)(ws + lay.kbar16),
      (__nv_bfloat16 *)(ws + lay.vbar16));
  PISA_TRY(check_launch());
  selection_bitmap_kernel<<<dim3(Nc, BH), 64, cwords * sizeof(uint32_t), st>>>(
      idx, Nc, k_sel, cwords, (uint32_t *)(ws + lay.bm));
  PISA_TRY(check_launch());
  const __nv_bfloat16 *q16 = (const __nv_bfloat16 *)q, *k16 = (const __nv_bfloat16 *)k,
                      *v16 = (const __nv_bfloat16 *)v, *g16 = (const __nv_bfloat16 *)dout;
  if (d == 128)
    return launch_bwd<128>(q16, k16, v16, g16, lse, out_f32, idx, k_sel, BH, L, block_size / 64,
                           s, lay, ws, (__nv_bfloat16 *)dq, (__nv_bfloat16 *)dk,
                           (__nv_bfloat16 *)dv, st);
  return launch_bwd<64>(q16, k16, v16, g16, lse, out_f32, idx, k_sel, BH, L, block_size / 64, s,
                        lay, ws, (__nv_bfloat16 *)dq, (__nv_bfloat16 *)dk, (__nv_bfloat16 *)dv,
                        st);
}

pisa_status pisa_attention_ex(const void *q, const void *k, const void *v, void *out, int B,
                              int H, int L, int d, int block_size, double density, int sink_idx,
                              pisa_mode mode, const pisa_options *opts, pisa_stream_t stream) {
  pisa_options o;
  memset(&o, 0, sizeof(o));
  if (opts) o = *opts;
  PISA_TRY(check_shape(B, H, L, d, block_size));
  if (o.dtype != PISA_BF16 && o.dtype != PISA_F32) return PISA_ERR_INVALID_ARG;
  if (mode != PISA_MODE_HYD && mode != PISA_MODE_0TH && mode != PISA_MODE_1ST) return PISA_ERR_INVALID_ARG;
  if (!sink_valid(sink_idx)) return PISA_ERR_INVALID_ARG;
  if (!(o.scale >= 0.f) || !std::isfinite(o.scale) || !std::isfinite(o.cov_weight))
    return PISA_ERR_INVALID_ARG;
  if (mode == PISA_MODE_1ST && block_size != 64) return PISA_ERR_UNSUPPORTED;
  if (o.fuse_select && block_size != 128) return PISA_ERR_UNSUPPORTED;
  if (!fused_fits(d, L, block_size)) return PISA_ERR_UNSUPPORTED;
  const int N = ceil_div(L, block_size);
  const int k_sel = pisa_num_selected(N, density);
  if (k_sel < 1) return PISA_ERR_INVALID_ARG;
  if (o.idx_out && ((uintptr_t)o.idx_out & 3u)) return PISA_ERR_INVALID_ARG;
  if ((long long)N * 4 > 200 * 1024) return PISA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return PISA_ERR_INVALID_ARG;
  if (out == q || out == k || out == v) return PISA_ERR_INVALID_ARG;
  const int want_cov = o.cov_weight != 0.f;
  const PathLayout p = path_layout(B, H, L, d, block_size, density, o.dtype, want_cov);
  cudaStream_t st = (cudaStream_t)stream;
  unsigned char *ws = (unsigned char *)o.workspace;
  bool owned = false;
  if (ws) {
    if (!aligned16(ws)) return PISA_ERR_INVALID_ARG;
    if (o.ws_bytes < p.total) return PISA_ERR_WORKSPACE;
  } else {
    void *mem = nullptr;
    PISA_CUDA(cudaMallocAsync(&mem, p.total, st));
    ws = (unsigned char *)mem;
    owned = true;
  }
  const float s = o.scale == 0.f ? 1.f / std::sqrt((float)d) : o.scale;
  const int BH = B * H;
  float *qbar = (float *)(ws + p.qbar), *kbar = (float *)(ws + p.kbar),
        *vsum = (float *)(ws + p.vsum), *hbar = (float *)(ws + p.hbar),
        *cov = want_cov ? (float *)(ws + p.cov) : nullptr;
  int32_t *idx = o.idx_out ? o.idx_out : (int32_t *)(ws + p.idx);
  unsigned char *scratch = ws + p.scratch;
  pisa_status r;
  const int sub = block_size / 64;
  FusedSelect fsel{};
  if (o.fuse_select) {
    fsel.qbar = qbar;
    fsel.kbar = kbar;
    fsel.cov = cov;
    fsel.cov_weight = o.cov_weight;
    fsel.sink = sink_block(sink_idx, N);
    fsel.idx_out = o.idx_out;
  }
  if (d == 128)
    r = launch_stats<128>(q, k, v, o.dtype, BH, L, sub, want_cov, qbar, kbar, vsum, hbar, cov,
                          (float *)scratch, st);
  else
    r = launch_stats<64>(q, k, v, o.dtype, BH, L, sub, want_cov, qbar, kbar, vsum, hbar, cov,
                         (float *)scratch, st);
  if (r == PISA_OK && !o.fuse_select)
    r = launch_select(qbar, kbar, cov, o.cov_weight, s, BH, N, d, k_sel,
                      sink_block(sink_idx, N), idx, (unsigned char *)scratch, st);
  if (r == PISA_OK)
    r = run_sparse_attention(q, k, v, o.dtype, kbar, vsum, hbar, idx, k_sel, BH, L, d, sub, s,
                             mode, out, nullptr, nullptr, scratch, st, fsel);
  if (owned) {
    cudaError_t e = cudaFreeAsync(ws, st);
    if (e != cudaSuccess && r == PISA_OK) {
      set_last_error(e);
      r = PISA_ERR_CUDA;
    }
  }
  return r;
}

pisa_status pisa_attention(const void *q, const void *k, const void *v, void *out, int B, int H,
                           int L, int d, int block_size, double density, int sink_idx,
                           pisa_mode mode, pisa_stream_t stream) {
  return pisa_attention_ex(q, k, v, out, B, H, L, d, block_size, density, sink_idx, mode, nullptr,
                           stream);
}

size_t pisa_dense_attention_workspace_bytes(int B, int H, int L, int d, pisa_dtype dtype) {
  if (check_shape(B, H, L, d, 64) != PISA_OK) return 0;
  return dtype == PISA_F32 ? 3 * align_up((size_t)B * H * L * d * 2, 256) : 0;
}

pisa_status pisa_dense_attention(const void *q, const void *k, const void *v, void *out,
                                 pisa_dtype dtype, int B, int H, int L, int d, float scale,
                                 void *workspace, size_t ws_bytes, pisa_stream_t stream) {
  PISA_TRY(check_shape(B, H, L, d, 64));
  if (dtype != PISA_BF16 && dtype != PISA_F32) return PISA_ERR_INVALID_ARG;
  if (!fused_fits(d, L, 64)) return PISA_ERR_UNSUPPORTED;
  if (!(scale >= 0.f) || !std::isfinite(scale)) return PISA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return PISA_ERR_INVALID_ARG;
  if (out == q || out == k || out == v) return PISA_ERR_INVALID_ARG;
  const size_t need = pisa_dense_attention_workspace_bytes(B, H, L, d, dtype);
  if (ws_bytes < need) return PISA_ERR_WORKSPACE;
  if (need && !aligned16(workspace)) return PISA_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  const int BH = B * H;
  const float s = scale == 0.f ? 1.f / std::sqrt((float)d) : scale;
  const __nv_bfloat16 *q16 = (const __nv_bfloat16 *)q, *k16 = (const __nv_bfloat16 *)k,
                      *v16 = (const __nv_bfloat16 *)v;
  if (dtype == PISA_F32) {
    const size_t n = (size_t)BH * L * d, sz = align_up(n * 2, 256);
    unsigned char *w = (unsigned char *)workspace;
    PISA_TRY(to_bf16(q, (__nv_bfloat16 *)w, n, st));
    PISA_TRY(to_bf16(k, (__nv_bfloat16 *)(w + sz), n, st));
    PISA_TRY(to_bf16(v, (__nv_bfloat16 *)(w + 2 * sz), n, st));
    q16 = (const __nv_bfloat16 *)w;
    k16 = (const __nv_bfloat16 *)(w + sz);
    v16 = (const __nv_bfloat16 *)(w + 2 * sz);
  }
  const int of32 = dtype == PISA_F32;
  if (d == 128)
    return launch_attention_kernel<128>(q16, k16, v16, nullptr, nullptr, nullptr, nullptr,
                                        nullptr, 0, BH, L, 1, s, 0, 1, 0, out, of32, nullptr,
                                        nullptr, st);
  return launch_attention_kernel<64>(q16, k16, v16, nullptr, nullptr, nullptr, nullptr, nullptr,
                                     0, BH, L, 1, s, 0, 1, 0, out, of32, nullptr, nullptr, st);
}

pisa_status pisa_block_stats_noalloc(const void *q, const void *k, const void *v,
                                     pisa_dtype dtype, int B, int H, int L, int d,
                                     int block_size, int want_cov, float *qbar, float *kbar,
                                     float *vsum, float *hbar, float *cov,
                                     pisa_stream_t stream) {
  PISA_TRY(check_shape(B, H, L, d, block_size));
  if (dtype != PISA_BF16 && dtype != PISA_F32) return PISA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(qbar) || !aligned16(kbar) ||
      !aligned16(vsum) || !aligned16(hbar))
    return PISA_ERR_INVALID_ARG;
  if (want_cov && !aligned16(cov)) return PISA_ERR_INVALID_ARG;
  const size_t need = stats_ws(B, H, L, d, block_size);
  if (need > (size_t)PISA_NOALLOC_SCRATCH_BYTES) {
    t_last_error = "pisa_block_stats_noalloc: this shape needs " + std::to_string(need) +
                   " bytes of scratch; the static array holds " +
                   std::to_string((size_t)PISA_NOALLOC_SCRATCH_BYTES);
    return PISA_ERR_WORKSPACE;
  }
  void *scratch = nullptr;
  PISA_TRY(noalloc_scratch(&scratch));
  cudaStream_t st = (cudaStream_t)stream;
  float *partial = (float *)scratch;
  const int sub = block_size / 64;
  if (d == 128)
    return launch_stats<128>(q, k, v, dtype, B * H, L, sub, want_cov, qbar, kbar, vsum, hbar,
                             cov, partial, st);
  return launch_stats<64>(q, k, v, dtype, B * H, L, sub, want_cov, qbar, kbar, vsum, hbar, cov,
                          partial, st);
}

pisa_status pisa_tail_score_histogram(const void *q, const void *k, pisa_dtype dtype,
                                      const int32_t *idx, int k_sel, int B, int H, int L, int d,
                                      int block_size, float scale, float lo, float hi, int nbins,
                                      int query_stride, unsigned long long *hist_x,
                                      unsigned long long *hist_y, double *moments,
                                      pisa_stream_t stream) {
  PISA_TRY(check_shape(B, H, L, d, block_size));
  if (block_size != 64) return PISA_ERR_UNSUPPORTED;
  if (dtype != PISA_BF16) return PISA_ERR_UNSUPPORTED;
  const int N = ceil_div(L, 64);
  if (k_sel < 1 || k_sel > N || nbins < 1 || nbins > 4096 || query_stride < 1)
    return PISA_ERR_INVALID_ARG;
  if (!std::isfinite(lo) || !std::isfinite(hi) || !(lo < hi) || !(scale >= 0.f) ||
      !std::isfinite(scale))
    return PISA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !idx || !hist_x || !hist_y || !moments)
    return PISA_ERR_INVALID_ARG;
  const float s = scale == 0.f ? 1.f / std::sqrt((float)d) : scale;
  cudaStream_t st = (cudaStream_t)stream;
  const int smem = 3 * 64 * d * 2 + 8 * (nbins + 2) * 4 + ceil_div(N, 32) * 4;
  if (smem > 227 * 1024) return PISA_ERR_UNSUPPORTED;
  PISA_CUDA(cudaMemsetAsync(hist_x, 0, sizeof(unsigned long long) * (nbins + 2), st));
  PISA_CUDA(cudaMemsetAsync(hist_y, 0, sizeof(unsigned long long) * (nbins + 2), st));
  PISA_CUDA(cudaMemsetAsync(moments, 0, sizeof(double) * 5, st));
  dim3 grid(ceil_div(N, query_stride), B * H);
  const __nv_bfloat16 *q16 = (const __nv_bfloat16 *)q, *k16 = (const __nv_bfloat16 *)k;
  if (d == 128) {
    PISA_CUDA(cudaFuncSetAttribute(tail_histogram_kernel<128>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    tail_histogram_kernel<128><<<grid, kHistThreads, smem, st>>>(
        q16, k16, idx, k_sel, L, N, s, lo, hi, nbins, query_stride, hist_x, hist_y, moments);
  } else {
    PISA_CUDA(cudaFuncSetAttribute(tail_histogram_kernel<64>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    tail_histogram_kernel<64><<<grid, kHistThreads, smem, st>>>(
        q16, k16, idx, k_sel, L, N, s, lo, hi, nbins, query_stride, hist_x, hist_y, moments);
  }
  return check_launch();
}

pisa_status pisa_selftest_timeout(uint64_t limit_ns, pisa_stream_t stream) {
  if (limit_ns == 0 || limit_ns > 1000000000ull) return PISA_ERR_INVALID_ARG;
  wait_timeout_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(limit_ns);
  return check_launch();
}

pisa_status pisa_device_status(pisa_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) {
    set_last_error(e);
    return PISA_ERR_CUDA;
  }
  unsigned v = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v));
  if (e != cudaSuccess) {
    set_last_error(e);
    return PISA_ERR_CUDA;
  }
  if (v) {
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero));
    if (e != cudaSuccess) {
      set_last_error(e);
      return PISA_ERR_CUDA;
    }
  }
  if (v & kDevErrTimeout) return PISA_ERR_TIMEOUT;
  if (v & kDevErrRange) return PISA_ERR_DEVICE;
  return PISA_OK;
}

const char *pisa_status_string(pisa_status s) {
  switch (s) {
    case PISA_OK: return "ok";
    case PISA_ERR_INVALID_ARG: return "invalid argument";
    case PISA_ERR_UNSUPPORTED: return "unsupported configuration";
    case PISA_ERR_CUDA: return "CUDA error";
    case PISA_ERR_WORKSPACE: return "workspace too small";
    case PISA_ERR_TIMEOUT: return "device-side bounded wait timed out";
    case PISA_ERR_DEVICE: return "device-side range check failed";
  }
  return "unknown status";
}

const char *pisa_last_error(void) { return t_last_error.c_str(); }

}  // extern "C"
