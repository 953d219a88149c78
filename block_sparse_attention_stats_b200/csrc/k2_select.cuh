// K2: covariance-aware top-k routing with attention-sink forcing.
//
// "Technical Summary: PISA" (gist.science), section 2 "Covariance-Aware
// Routing": a block's selection score combines the query-key attention score
// with the norm of its covariance matrix M_j.  The authors' README, "Attention
// sink for MMDiT": sink_idx 0 / -1 forces the first / last K/V block into the
// exact set of every query block.
//
//   score_ij = scale * (qbar_i . kbar_j) + lambda * M_j      (float32)
//
// Fused path (select_fused_kernel, short sequences, N <= 512): a group of query
// blocks computes its score rows into shared memory and selects from there
// (FLUX shape: 0.028 ms against 0.032 ms; at N = 1182 it is 1.9x slower than the
// two-pass path, which streams each k-bar tile once per 128 x 128 score tile).
// Two-pass path otherwise:
// Pass 1 (scores_kernel): a float32 FMA GEMM per head, 128 x 128 output tiles,
// each score summed over the head dimension in ascending order.
// Pass 2 (topk_kernel): one warp per query block.  Scores become 32-bit keys
// whose unsigned order is the float order; an MSB-first radix select (4 x 8
// bits) finds the k-th largest key T; every key > T is kept, and of the keys
// equal to T the lowest block indices are kept (ties go to the lower index).
// The sink block is set aside first and always kept.  Indices come out
// ascending via warp ballots.
#pragma once

#include "pisa_common.cuh"

namespace pisa {

// Scores: C = scale * Qbar Kbar^T + lambda * cov over 128 x 128 tiles, 256
// threads with 8 x 8 outputs each; operands staged in shared memory as
// [dim][row] so every thread reads its 8 rows / 8 columns as two float4.
// Each score is accumulated over the head dimension in ascending order.
constexpr int kScoreTile = 128;
constexpr int kScoreK = 16;
constexpr int kScorePad = 4;

__global__ void __launch_bounds__(256, 2)
    scores_kernel(const float *__restrict__ qbar, const float *__restrict__ kbar,
                  const float *__restrict__ cov, float cov_weight, float scale, int N, int D,
                  float *__restrict__ scores) {
  __shared__ __align__(16) float As[kScoreK][kScoreTile + kScorePad];
  __shared__ __align__(16) float Bs[kScoreK][kScoreTile + kScorePad];
  const int bh = blockIdx.z;
  const int i0 = blockIdx.y * kScoreTile, j0 = blockIdx.x * kScoreTile;
  const float *qb = qbar + (size_t)bh * N * D;
  const float *kb = kbar + (size_t)bh * N * D;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  float acc[8][8];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[r][c] = 0.f;

  // 128 rows x 16 dims of each operand per chunk, two float4 per thread per
  // operand; the next chunk is fetched into registers while this one is used
  float4 pa[2], pb[2];
  auto fetch = [&](int e0) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int t = tid + 256 * h;
      const int row = t >> 2, e4 = (t & 3) * 4;
      const int gi = i0 + row, gj = j0 + row;
      pa[h] = gi < N ? *reinterpret_cast<const float4 *>(qb + (size_t)gi * D + e0 + e4)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
      pb[h] = gj < N ? *reinterpret_cast<const float4 *>(kb + (size_t)gj * D + e0 + e4)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  fetch(0);
  for (int e0 = 0; e0 < D; e0 += kScoreK) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int t = tid + 256 * h;
      const int row = t >> 2, e4 = (t & 3) * 4;
      const float4 a = pa[h], b = pb[h];
      As[e4 + 0][row] = a.x; As[e4 + 1][row] = a.y; As[e4 + 2][row] = a.z; As[e4 + 3][row] = a.w;
      Bs[e4 + 0][row] = b.x; Bs[e4 + 1][row] = b.y; Bs[e4 + 2][row] = b.z; Bs[e4 + 3][row] = b.w;
    }
    __syncthreads();
    if (e0 + kScoreK < D) fetch(e0 + kScoreK);
#pragma unroll
    for (int e = 0; e < kScoreK; ++e) {
      const float4 a0 = *reinterpret_cast<const float4 *>(&As[e][ty * 8]);
      const float4 a1 = *reinterpret_cast<const float4 *>(&As[e][ty * 8 + 4]);
      const float4 b0 = *reinterpret_cast<const float4 *>(&Bs[e][tx * 8]);
      const float4 b1 = *reinterpret_cast<const float4 *>(&Bs[e][tx * 8 + 4]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[r][c] = fmaf(av[r], bv[c], acc[r][c]);
    }
    __syncthreads();
  }
  float cw[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const int gj = j0 + tx * 8 + c;
    cw[c] = (cov_weight != 0.f && gj < N) ? cov_weight * cov[(size_t)bh * N + gj] : 0.f;
  }
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int gi = i0 + ty * 8 + r;
    if (gi >= N) continue;
    float *out = scores + ((size_t)bh * N + gi) * N;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int gj = j0 + tx * 8 + c;
      if (gj < N) out[gj] = fmaf(scale, acc[r][c], cw[c]);
    }
  }
}

// Order-preserving map float32 -> uint32 (-0 is treated as +0).
__device__ __forceinline__ uint32_t float_key(float f) {
  if (f == 0.f) f = 0.f;
  uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

constexpr int kTopkThreads = 256;  // 8 warps, one query block per warp

// One warp selects the exact set of one query block from its scores `sc`
// (global memory, re-read from L2 on every pass, or shared memory); `hist` is
// the warp's 256-entry histogram.
__device__ __forceinline__ void topk_row(const float *sc, int N, int k_sel, int sink,
                                         unsigned *hist, int32_t *__restrict__ out, int lane) {
  const int need = k_sel - (sink >= 0 ? 1 : 0);
  const int candidates = N - (sink >= 0 ? 1 : 0);
  const bool take_all = need >= candidates;

  uint32_t prefix = 0u, mask = 0u;
  int rem = need;
  if (!take_all && need > 0) {
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
#pragma unroll
      for (int q = 0; q < 8; ++q) hist[lane * 8 + q] = 0u;
      __syncwarp();
      for (int j0 = 0; j0 < N; j0 += 128) {
        // four loads in flight per lane, then the four histogram updates
        uint32_t kv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = j0 + 32 * u + lane;
          kv[u] = j < N ? float_key(sc[j]) : 0u;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = j0 + 32 * u + lane;
          const uint32_t key = kv[u];
          const bool part = j < N && j != sink && (key & mask) == prefix;
          const unsigned act = __ballot_sync(0xffffffffu, part);
          if (part) {
            // aggregate lanes that hit the same bin into one shared-memory atomic
            const unsigned digit = (key >> shift) & 255u;
            const unsigned peers = __match_any_sync(act, digit);
            if (lane == __ffs(peers) - 1) atomicAdd(&hist[digit], (unsigned)__popc(peers));
          }
        }
      }
      __syncwarp();
      // lane l owns digits 255-8l .. 248-8l (largest first)
      unsigned own = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) own += hist[255 - 8 * lane - q];
      unsigned incl = own;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const unsigned excl = incl - own;
      const bool here = excl < (unsigned)rem && (unsigned)rem <= incl;
      const unsigned who = __ballot_sync(0xffffffffu, here);
      const int src = __ffs(who) - 1;
      int digit_sel = 0, new_rem = 0;
      if (lane == src) {
        unsigned cum = excl;
        for (int q = 0; q < 8; ++q) {
          const int digit = 255 - 8 * lane - q;
          const unsigned c = hist[digit];
          if ((unsigned)rem <= cum + c) {
            digit_sel = digit;
            new_rem = rem - (int)cum;
            break;
          }
          cum += c;
        }
      }
      digit_sel = __shfl_sync(0xffffffffu, digit_sel, src);
      new_rem = __shfl_sync(0xffffffffu, new_rem, src);
      prefix |= (uint32_t)digit_sel << shift;
      mask |= 255u << shift;
      rem = new_rem;
      __syncwarp();
    }
  }
  // keep: the sink, every key > T, and the lowest-index `rem` keys equal to T
  const uint32_t T = prefix;
  int eq_base = 0, out_base = 0;
  for (int j0 = 0; j0 < N; j0 += 32) {
    const int j = j0 + lane;
    const bool valid = j < N;
    const uint32_t key = valid ? float_key(sc[j]) : 0u;
    const bool cand = valid && j != sink;
    const bool is_eq = cand && !take_all && need > 0 && key == T;
    const unsigned eq_bal = __ballot_sync(0xffffffffu, is_eq);
    const int eq_rank = eq_base + __popc(eq_bal & ((1u << lane) - 1u));
    bool sel;
    if (!valid) sel = false;
    else if (j == sink) sel = true;
    else if (take_all) sel = true;
    else if (need <= 0) sel = false;
    else sel = key > T || (is_eq && eq_rank < rem);
    const unsigned sel_bal = __ballot_sync(0xffffffffu, sel);
    const int pos = out_base + __popc(sel_bal & ((1u << lane) - 1u));
    if (sel) {
      if (pos < k_sel) out[pos] = j;
      else report_device_error(kDevErrRange);
    }
    eq_base += __popc(eq_bal);
    out_base += __popc(sel_bal);
  }
  if (lane == 0 && out_base != k_sel) report_device_error(kDevErrRange);
}

// One warp per query block over the N x N score matrix in global memory.
__global__ void __launch_bounds__(kTopkThreads)
    topk_kernel(const float *__restrict__ scores, int N, int k_sel, int sink, size_t rows,
                int32_t *__restrict__ idx) {
  __shared__ unsigned hist_all[kTopkThreads / 32][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t row = (size_t)blockIdx.x * (kTopkThreads / 32) + warp;
  if (row >= rows) return;
  topk_row(scores + row * N, N, k_sel, sink, hist_all[warp], idx + row * k_sel, lane);
}

// ---------------------------------------------------------------------------
// Fused scores + top-k for a group of kSelRows query blocks: the group's score
// rows live in shared memory only (no N x N matrix in HBM).  Each score is the
// same fp32 computation as in scores_kernel (head dimension summed in ascending
// order, then scale * acc + lambda * M_j), so both paths select the same sets.
// 384 threads compute 4 x 4 score blocks from k-bar chunks of 256 blocks x 32
// dimensions staged transposed in shared memory; then 12 warps take two rows
// each through the radix select.
// ---------------------------------------------------------------------------
constexpr int kSelRows = 24;
constexpr int kSelFusedMaxN = 512;  // longer rows: the two-pass path (measured faster)
constexpr int kSelThreads = 384;
constexpr int kSelCols = 256;      // k-bar blocks per staged chunk
constexpr int kSelDims = 32;       // head dimensions per staged chunk

__host__ __device__ inline int select_fused_smem(int N, int D) {
  const int stage = (kSelDims * kSelCols + D * kSelRows) * 4;      // kbar^T chunk, qbar^T
  const int hist = (kSelThreads / 32) * 256 * 4;
  return kSelRows * N * 4 + (stage > hist ? stage : hist);
}

__global__ void __launch_bounds__(kSelThreads, 1)
    select_fused_kernel(const float *__restrict__ qbar, const float *__restrict__ kbar,
                        const float *__restrict__ cov, float cov_weight, float scale, int N,
                        int D, int k_sel, int sink, int32_t *__restrict__ idx) {
  extern __shared__ __align__(16) float sel_smem[];
  float *S = sel_smem;                              // [kSelRows][N]
  float *kT = S + (size_t)kSelRows * N;             // [kSelDims][kSelCols]
  float *qT = kT + kSelDims * kSelCols;             // [D][kSelRows]
  unsigned *hist = reinterpret_cast<unsigned *>(kT);   // after the scores: per-warp histograms
  const int bh = blockIdx.y, i0 = blockIdx.x * kSelRows;
  const int tid = threadIdx.x;
  const float *qb = qbar + (size_t)bh * N * D;
  const float *kb = kbar + (size_t)bh * N * D;
  const int rg = tid >> 6, cg = tid & 63;           // rows 4 rg .. +3, columns 4 cg .. +3

  for (int e = tid; e < D * kSelRows; e += kSelThreads) {
    const int r = e % kSelRows, dd = e / kSelRows;
    qT[e] = i0 + r < N ? qb[(size_t)(i0 + r) * D + dd] : 0.f;
  }
  for (int c0 = 0; c0 < N; c0 += kSelCols) {
    float acc[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int x = 0; x < 4; ++x) acc[r][x] = 0.f;
    for (int e0 = 0; e0 < D; e0 += kSelDims) {
      __syncthreads();   // qT written / the previous chunk consumed
      for (int f = tid; f < kSelCols * kSelDims / 4; f += kSelThreads) {
        const int c = f % kSelCols, e4 = (f / kSelCols) * 4;
        const int j = c0 + c;
        const float4 v = j < N ? *reinterpret_cast<const float4 *>(kb + (size_t)j * D + e0 + e4)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
        kT[(e4 + 0) * kSelCols + c] = v.x;
        kT[(e4 + 1) * kSelCols + c] = v.y;
        kT[(e4 + 2) * kSelCols + c] = v.z;
        kT[(e4 + 3) * kSelCols + c] = v.w;
      }
      __syncthreads();
#pragma unroll 8
      for (int e = 0; e < kSelDims; ++e) {
        const float4 a = *reinterpret_cast<const float4 *>(qT + (e0 + e) * kSelRows + 4 * rg);
        const float4 b = *reinterpret_cast<const float4 *>(kT + e * kSelCols + 4 * cg);
        const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
          for (int x = 0; x < 4; ++x) acc[r][x] = fmaf(av[r], bv[x], acc[r][x]);
      }
    }
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const int j = c0 + 4 * cg + x;
      if (j >= N) continue;
      const float cw = cov_weight != 0.f ? cov_weight * cov[(size_t)bh * N + j] : 0.f;
#pragma unroll
      for (int r = 0; r < 4; ++r) S[(size_t)(4 * rg + r) * N + j] = fmaf(scale, acc[r][x], cw);
    }
  }
  __syncthreads();
  const int warp = tid >> 5, lane = tid & 31;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int r = 2 * warp + h;
    if (i0 + r < N)
      topk_row(S + (size_t)r * N, N, k_sel, sink, hist + warp * 256,
               idx + ((size_t)bh * N + i0 + r) * k_sel, lane);
  }
}

}  // namespace pisa
