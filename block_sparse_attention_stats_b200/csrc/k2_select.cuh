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
// Pass 1 (scores_kernel): a float32 FMA GEMM per head, 64 x 64 output tiles,
// each score summed over the head dimension in ascending order.
// Pass 2 (topk_kernel): one CTA per query block.  Scores become 32-bit keys
// whose unsigned order is the float order; an MSB-first radix select (4 x 8
// bits) finds the k-th largest key T; every key > T is kept, and of the keys
// equal to T the lowest block indices are kept (ties go to the lower index).
// The sink block is set aside first and always kept.  Indices come out
// ascending via a block-wide prefix sum.
#pragma once

#include "pisa_common.cuh"

namespace pisa {

constexpr int kScoreTile = 64;
constexpr int kScoreK = 32;

__global__ void __launch_bounds__(256)
    scores_kernel(const float *__restrict__ qbar, const float *__restrict__ kbar,
                  const float *__restrict__ cov, float cov_weight, float scale, int N, int D,
                  float *__restrict__ scores) {
  __shared__ __align__(16) float As[kScoreK][kScoreTile];
  __shared__ __align__(16) float Bs[kScoreK][kScoreTile];
  const int bh = blockIdx.z;
  const int i0 = blockIdx.y * kScoreTile, j0 = blockIdx.x * kScoreTile;
  const float *qb = qbar + (size_t)bh * N * D;
  const float *kb = kbar + (size_t)bh * N * D;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  float acc[4][4];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;

  for (int e0 = 0; e0 < D; e0 += kScoreK) {
    // load 64 rows x 32 dims of qbar and kbar, transposed into [dim][row]
    for (int t = tid; t < kScoreTile * kScoreK; t += 256) {
      const int row = t / kScoreK, e = t % kScoreK;
      const int gi = i0 + row, gj = j0 + row;
      As[e][row] = gi < N ? qb[(size_t)gi * D + e0 + e] : 0.f;
      Bs[e][row] = gj < N ? kb[(size_t)gj * D + e0 + e] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int e = 0; e < kScoreK; ++e) {
      const float4 a = *reinterpret_cast<const float4 *>(&As[e][ty * 4]);
      const float4 b = *reinterpret_cast<const float4 *>(&Bs[e][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(av[r], bv[c], acc[r][c]);
    }
    __syncthreads();
  }
  float cw[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int gj = j0 + tx * 4 + c;
    cw[c] = (cov_weight != 0.f && gj < N) ? cov_weight * cov[(size_t)bh * N + gj] : 0.f;
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int gi = i0 + ty * 4 + r;
    if (gi >= N) continue;
    float *out = scores + ((size_t)bh * N + gi) * N;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int gj = j0 + tx * 4 + c;
      if (gj < N) out[gj] = scale * acc[r][c] + cw[c];
    }
  }
}

// Order-preserving map float32 -> uint32 (-0 is treated as +0).
__device__ __forceinline__ uint32_t float_key(float f) {
  if (f == 0.f) f = 0.f;
  uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

constexpr int kTopkThreads = 256;

// Block-wide exclusive prefix sum of 0/1 flags in thread order; returns this
// thread's prefix and writes the block total to *total.
__device__ __forceinline__ int block_exclusive_scan(int flag, int *warp_tot, int *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, flag);
  const int in_warp = __popc(bal & ((1u << lane) - 1u));
  if (lane == 0) warp_tot[warp] = __popc(bal);
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kTopkThreads / 32; ++w) {
    const int c = warp_tot[w];
    before += (w < warp) ? c : 0;
    all += c;
  }
  __syncthreads();
  *total = all;
  return before + in_warp;
}

__global__ void __launch_bounds__(kTopkThreads)
    topk_kernel(const float *__restrict__ scores, int N, int k_sel, int sink,
                int32_t *__restrict__ idx) {
  extern __shared__ uint32_t keys[];  // N
  __shared__ unsigned hist[256];
  __shared__ int warp_tot[kTopkThreads / 32];
  __shared__ uint32_t s_prefix, s_mask;
  __shared__ int s_remaining;

  const size_t row = blockIdx.x;
  const float *sc = scores + row * N;
  int32_t *out = idx + row * k_sel;
  const int tid = threadIdx.x;

  for (int j = tid; j < N; j += kTopkThreads) keys[j] = float_key(sc[j]);
  if (tid == 0) {
    s_prefix = 0u;
    s_mask = 0u;
    s_remaining = k_sel - (sink >= 0 ? 1 : 0);
  }
  __syncthreads();

  const int candidates = N - (sink >= 0 ? 1 : 0);
  const bool take_all = s_remaining >= candidates;
  if (!take_all && s_remaining > 0) {
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      hist[tid] = 0u;  // kTopkThreads == 256 bins
      __syncthreads();
      const uint32_t prefix = s_prefix, mask = s_mask;
      for (int j = tid; j < N; j += kTopkThreads) {
        const uint32_t key = keys[j];
        if (j != sink && (key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (tid < 32) {
        // lane l owns digits 255-8l down to 248-8l (largest digits first)
        const int lane = tid;
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
        const int rem = s_remaining;
        const bool here = excl < (unsigned)rem && (unsigned)rem <= incl;
        const unsigned who = __ballot_sync(0xffffffffu, here);
        if (here && lane == __ffs(who) - 1) {
          unsigned cum = excl;
          for (int q = 0; q < 8; ++q) {
            const int digit = 255 - 8 * lane - q;
            const unsigned c = hist[digit];
            if ((unsigned)rem <= cum + c) {
              s_remaining = rem - (int)cum;
              s_prefix = prefix | ((uint32_t)digit << shift);
              s_mask = mask | (255u << shift);
              break;
            }
            cum += c;
          }
        }
      }
      __syncthreads();
    }
  }
  const uint32_t T = s_prefix;
  const int take_eq = s_remaining;

  // selection flags in index order, then ascending compaction
  int eq_base = 0, out_base = 0;
  for (int j0 = 0; j0 < N; j0 += kTopkThreads) {
    const int j = j0 + tid;
    const bool valid = j < N;
    const uint32_t key = valid ? keys[j] : 0u;
    const bool cand = valid && j != sink;
    const int is_eq = (cand && !take_all && key == T) ? 1 : 0;
    int eq_tot;
    const int eq_rank = eq_base + block_exclusive_scan(is_eq, warp_tot, &eq_tot);
    bool sel;
    if (!valid) sel = false;
    else if (j == sink) sel = true;
    else if (take_all) sel = true;
    else if (k_sel - (sink >= 0 ? 1 : 0) <= 0) sel = false;
    else sel = key > T || (is_eq && eq_rank < take_eq);
    int sel_tot;
    const int pos = out_base + block_exclusive_scan(sel ? 1 : 0, warp_tot, &sel_tot);
    if (sel) {
      if (pos < k_sel) out[pos] = j;
      else report_device_error(kDevErrRange);
    }
    eq_base += eq_tot;
    out_base += sel_tot;
  }
  if (tid == 0 && out_base != k_sel) report_device_error(kDevErrRange);
}

}  // namespace pisa
