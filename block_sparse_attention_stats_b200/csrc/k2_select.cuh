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
// blocks computes its score rows into shared memory (float32 FMAs, the head
// dimension summed in ascending order) and selects from there (FLUX shape:
// 0.028 ms against 0.032 ms two-pass).
// Two-pass path otherwise:
// Pass 1 (k2_scores_tc.cuh): the score matrix on the tensor cores from
// three-part bf16 splits of qbar and kbar, to float32 accuracy.
// Pass 2 (topk_bins_kernel; topk_kernel for rows too long to stage in shared
// memory): one warp per query block.  Scores map to 32-bit keys whose
// unsigned order is the float order; the k-th largest key T is found, every
// key > T is kept, and of the keys equal to T the lowest block indices are
// kept (ties go to the lower index).  The sink block is set aside first and
// always kept.  Indices come out ascending via warp ballots.
#pragma once

#include "pisa_common.cuh"

namespace pisa {

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

// One warp per query block over the score matrix in global memory (row
// stride ld >= N).
__global__ void __launch_bounds__(kTopkThreads)
    topk_kernel(const float *__restrict__ scores, int N, int ld, int k_sel, int sink,
                size_t rows, int32_t *__restrict__ idx) {
  __shared__ unsigned hist_all[kTopkThreads / 32][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t row = (size_t)blockIdx.x * (kTopkThreads / 32) + warp;
  if (row >= rows) return;
  topk_row(scores + row * ld, N, k_sel, sink, hist_all[warp], idx + row * k_sel, lane);
}

// ---------------------------------------------------------------------------
// The same selection with one histogram pass instead of four radix passes.
// Each warp copies its row into shared memory, then finds the k-th largest key
// T and the number of keys equal to T to keep:
//  1. lo / hi = the smallest / largest candidate score; bin(x) =
//     min(255, int((x - lo) * (256 / (hi - lo)))).  Every step of bin() is a
//     monotone float32 operation, so x >= y implies bin(x) >= bin(y): the bins
//     order the keys.
//  2. One histogram of the candidates' bins; scanning from the top bin gives
//     the bin b* that holds the `need`-th largest key and how many keys of b*
//     are still to be taken.
//  3. The (at most kBinCand) scores of b* are gathered (in any order: only
//     their multiset matters) and T is the one whose count of larger scores is
//     below, and whose count of larger or equal scores reaches, the number
//     still to be taken.
// Comparing floats gives the key order (only -0 and +0 share a key, and they
// compare equal).  Then the same compaction as topk_row keeps the sink, every
// score > T and the lowest-index scores equal to T.  Rows where the bins do
// not apply (all scores equal, a non-finite score, more than kBinCand scores
// in b*) go through topk_row on the staged row, so the result is the same set
// in every case.
// ---------------------------------------------------------------------------
constexpr int kBinCand = 64;

// shared memory per warp: the row (ld floats), the histogram, the gathered bin
__host__ __device__ inline int topk_bins_smem(int ld) {
  return (kTopkThreads / 32) * (ld + 256 + kBinCand) * 4;
}

__global__ void __launch_bounds__(kTopkThreads)
    topk_bins_kernel(const float *__restrict__ scores, int N, int ld, int k_sel, int sink,
                     size_t rows, int32_t *__restrict__ idx) {
  extern __shared__ __align__(16) float tk_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t row = (size_t)blockIdx.x * (kTopkThreads / 32) + warp;
  if (row >= rows) return;
  float *srow = tk_smem + (size_t)warp * (ld + 256 + kBinCand);
  unsigned *hist = reinterpret_cast<unsigned *>(srow + ld);
  float *cand = reinterpret_cast<float *>(hist + 256);
  const float *sc = scores + row * ld;
  int32_t *out = idx + row * k_sel;
  const int need = k_sel - (sink >= 0 ? 1 : 0);
  const int candidates = N - (sink >= 0 ? 1 : 0);
  // stage the row (16-byte loads), and 1. the range of the candidates on the
  // way; a NaN or infinite score sends the row to topk_row
  const float inf = __int_as_float(0x7f800000);
  float lo = inf, hi = -inf;
  bool bad = false;
#pragma unroll 2
  for (int c = lane; c < ld / 4; c += 32) {
    const float4 x4 = __ldcs(reinterpret_cast<const float4 *>(sc) + c);
    *reinterpret_cast<float4 *>(srow + 4 * c) = x4;
    const float xs[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = 4 * c + e;
      if (j < N && j != sink) {
        bad |= !(fabsf(xs[e]) < inf);
        lo = fminf(lo, xs[e]);
        hi = fmaxf(hi, xs[e]);
      }
    }
  }
  __syncwarp();
  if (need <= 0 || need >= candidates) {
    topk_row(srow, N, k_sel, sink, hist, out, lane);
    return;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  const float span = hi - lo, w = 256.f / span;
  if (__any_sync(0xffffffffu, bad) || !(span > 0.f && span < inf && w < inf)) {
    topk_row(srow, N, k_sel, sink, hist, out, lane);
    return;
  }
  auto bin_of = [&](float x) { return min((int)((x - lo) * w), 255); };
  // 2. histogram and the boundary bin
#pragma unroll
  for (int q = 0; q < 8; ++q) hist[lane * 8 + q] = 0u;
  __syncwarp();
#pragma unroll 2
  for (int c = lane; c < ld / 4; c += 32) {
    const float4 x4 = *reinterpret_cast<const float4 *>(srow + 4 * c);
    const float xs[4] = {x4.x, x4.y, x4.z, x4.w};
    if (4 * c + 3 < N && (unsigned)(sink - 4 * c) > 3u) {
#pragma unroll
      for (int e = 0; e < 4; ++e) atomicAdd(&hist[bin_of(xs[e])], 1u);
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = 4 * c + e;
        if (j < N && j != sink) atomicAdd(&hist[bin_of(xs[e])], 1u);
      }
    }
  }
  __syncwarp();
  unsigned own = 0;                      // lane l owns bins 255-8l .. 248-8l
#pragma unroll
  for (int q = 0; q < 8; ++q) own += hist[255 - 8 * lane - q];
  unsigned incl = own;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  const unsigned excl = incl - own;
  const unsigned who = __ballot_sync(0xffffffffu, excl < (unsigned)need && (unsigned)need <= incl);
  const int src = __ffs(who) - 1;
  int bstar = 0, take = 0, cnt = 0;
  if (lane == src) {
    unsigned cum = excl;
    for (int q = 0; q < 8; ++q) {
      const int b = 255 - 8 * lane - q;
      const unsigned c = hist[b];
      if ((unsigned)need <= cum + c) {
        bstar = b;
        take = need - (int)cum;
        cnt = (int)c;
        break;
      }
      cum += c;
    }
  }
  bstar = __shfl_sync(0xffffffffu, bstar, src);
  take = __shfl_sync(0xffffffffu, take, src);
  cnt = __shfl_sync(0xffffffffu, cnt, src);
  if (cnt > kBinCand) {
    topk_row(srow, N, k_sel, sink, hist, out, lane);
    return;
  }
  // 3. the scores of b*, and T among them: the `take`-th largest; eq = how
  //    many candidates equal T, rem = how many of those are kept
  // (the order of the gathered scores does not matter: T and the counts
  // depend only on their multiset)
  unsigned *ncand = hist;                // the histogram is no longer needed
  __syncwarp();
  if (lane == 0) *ncand = 0u;
  __syncwarp();
#pragma unroll 2
  for (int c = lane; c < ld / 4; c += 32) {
    const float4 x4 = *reinterpret_cast<const float4 *>(srow + 4 * c);
    const float xs[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = 4 * c + e;
      if (j < N && j != sink && bin_of(xs[e]) == bstar) cand[atomicAdd(ncand, 1u)] = xs[e];
    }
  }
  __syncwarp();
  float T = 0.f;
  int rem = 0, eq = 0;
  bool found = false;
  for (int m = lane; m < cnt; m += 32) {
    const float xm = cand[m];
    int gt = 0, ge = 0;
    for (int n = 0; n < cnt; ++n) {
      const float xn = cand[n];
      gt += xn > xm;
      ge += xn >= xm;
    }
    if (gt < take && take <= ge) {
      found = true;
      T = xm;
      rem = take - gt;
      eq = ge - gt;
    }
  }
  const unsigned fb = __ballot_sync(0xffffffffu, found);
  if (fb == 0u) {                        // cannot happen; keep the result exact anyway
    topk_row(srow, N, k_sel, sink, hist, out, lane);
    return;
  }
  const int fl = __ffs(fb) - 1;
  T = __shfl_sync(0xffffffffu, T, fl);
  rem = __shfl_sync(0xffffffffu, rem, fl);
  eq = __shfl_sync(0xffffffffu, eq, fl);
  // keep: the sink, every score > T, and the lowest-index `rem` scores equal
  // to T (all of them when rem == eq, the usual case)
  const bool ties = rem != eq;
  int out_base = 0, eq_base = 0;
  if (!ties) {
    // lane l holds blocks 4 (32 it + l) .. +3; its kept count goes into the
    // warp's exclusive prefix as three bit-plane ballots
    const unsigned lt = (1u << lane) - 1u;
#pragma unroll 2
    for (int c0 = 0; c0 < ld / 4; c0 += 32) {
      const int c = c0 + lane;
      const float4 x4 = c < ld / 4 ? *reinterpret_cast<const float4 *>(srow + 4 * c)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
      const float xs[4] = {x4.x, x4.y, x4.z, x4.w};
      unsigned keep = 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = 4 * c + e;
        if (j < N && (j == sink || xs[e] >= T)) keep |= 1u << e;
      }
      const unsigned n = __popc(keep);
      const unsigned b0 = __ballot_sync(0xffffffffu, n & 1u);
      const unsigned b1 = __ballot_sync(0xffffffffu, n & 2u);
      const unsigned b2 = __ballot_sync(0xffffffffu, n & 4u);
      int pos = out_base + __popc(b0 & lt) + 2 * __popc(b1 & lt) + 4 * __popc(b2 & lt);
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if ((keep >> e) & 1u) {
          if (pos < k_sel) out[pos] = 4 * c + e;
          else report_device_error(kDevErrRange);
          ++pos;
        }
      out_base += __popc(b0) + 2 * __popc(b1) + 4 * __popc(b2);
    }
    if (lane == 0 && out_base != k_sel) report_device_error(kDevErrRange);
    return;
  }
  for (int j0 = 0; j0 < N; j0 += 32) {
    const int j = j0 + lane;
    const bool valid = j < N;
    const float x = valid ? srow[j] : 0.f;
    const bool cnd = valid && j != sink;
    bool sel;
    if (ties) {
      const bool is_eq = cnd && x == T;
      const unsigned eq_bal = __ballot_sync(0xffffffffu, is_eq);
      sel = (cnd && x > T) || (is_eq && eq_base + __popc(eq_bal & ((1u << lane) - 1u)) < rem);
      eq_base += __popc(eq_bal);
    } else {
      sel = cnd && x >= T;
    }
    sel = sel || (valid && j == sink);
    const unsigned bal = __ballot_sync(0xffffffffu, sel);
    if (sel) out[out_base + __popc(bal & ((1u << lane) - 1u))] = j;
    out_base += __popc(bal);
  }
  if (lane == 0 && out_base != k_sel) report_device_error(kDevErrRange);
}

// ---------------------------------------------------------------------------
// Fused scores + top-k for a group of kSelRows query blocks: the group's score
// rows live in shared memory only (no N x N matrix in HBM).  Each score is a
// float32 FMA chain over the head dimension in ascending order, then
// scale * acc + lambda * M_j.
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

__global__ void __launch_bounds__(kSelThreads, 2)
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
  // the k-bar chunk of the next head-dimension step is fetched into registers
  // while the current one is used
  constexpr int kPf = (kSelCols * kSelDims / 4 + kSelThreads - 1) / kSelThreads;
  float4 pf[kPf];
  auto fetch = [&](int c0, int e0) {
#pragma unroll
    for (int h = 0; h < kPf; ++h) {
      const int f = tid + kSelThreads * h;
      const int c = f % kSelCols, e4 = (f / kSelCols) * 4, j = c0 + c;
      pf[h] = (f < kSelCols * kSelDims / 4 && j < N)
                  ? *reinterpret_cast<const float4 *>(kb + (size_t)j * D + e0 + e4)
                  : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  // warp w computes columns 128 (w & 1) .. +127 of a chunk: none of them may
  // exist on short rows
  const int wcol = 128 * ((tid >> 5) & 1);
  for (int c0 = 0; c0 < N; c0 += kSelCols) {
    float acc[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int x = 0; x < 4; ++x) acc[r][x] = 0.f;
    fetch(c0, 0);
    for (int e0 = 0; e0 < D; e0 += kSelDims) {
      __syncthreads();   // qT written / the previous chunk consumed
#pragma unroll
      for (int h = 0; h < kPf; ++h) {
        const int f = tid + kSelThreads * h;
        if (f < kSelCols * kSelDims / 4) {
          const int c = f % kSelCols, e4 = (f / kSelCols) * 4;
          kT[(e4 + 0) * kSelCols + c] = pf[h].x;
          kT[(e4 + 1) * kSelCols + c] = pf[h].y;
          kT[(e4 + 2) * kSelCols + c] = pf[h].z;
          kT[(e4 + 3) * kSelCols + c] = pf[h].w;
        }
      }
      __syncthreads();
      if (e0 + kSelDims < D) fetch(c0, e0 + kSelDims);
      if (c0 + wcol < N) {
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
