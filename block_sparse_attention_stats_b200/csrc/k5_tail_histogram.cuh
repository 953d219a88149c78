// Distributional-stability diagnostic of the unselected (non-critical) blocks.
//
// "Technical Summary: PISA" (gist.science), section 2 "Key Insights" 1: the
// pre-softmax scores of non-critical blocks are bell-shaped and centred at or
// below zero, which is what makes their block-wise Taylor approximation
// accurate.  This kernel measures that distribution: for every token t of the
// sampled query blocks i, every unselected block j in U_i and every key n of j
//   x = s q_t k_n                 (pre-softmax score)
//   y = s q_t (k_n - kbar_j)      (the Taylor variable about the block centroid)
// and histograms both over nbins equal bins of [lo, hi) plus an underflow and
// an overflow bin, with the count and the sums of x, x^2, y, y^2.
//
// One CTA (4 warps, 16 rows each) per sampled query block; 64 x 64 score tiles
// with mma.sync (bf16 in, f32 out).  s q_t kbar_j is the mean of the tile's
// exact scores over the block's keys (the centroid is the mean key).  Each
// warp counts into its own shared-memory histogram; the CTA adds its counts to
// the global ones at the end.
#pragma once

#include "pisa_common.cuh"

namespace pisa {

constexpr int kHistThreads = 128;

template <int D>
__global__ void __launch_bounds__(kHistThreads)
    tail_histogram_kernel(const __nv_bfloat16 *__restrict__ Q, const __nv_bfloat16 *__restrict__ K,
                          const int32_t *__restrict__ idx, int k_sel, int L, int N, float scale,
                          float lo, float hi, int nbins, int query_stride,
                          unsigned long long *__restrict__ hist_x,
                          unsigned long long *__restrict__ hist_y,
                          double *__restrict__ moments) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int kTileBytes = 64 * D * 2;
  const uint32_t sbase = smem_u32(smem);
  const int nb2 = nbins + 2;
  const int nwords = (N + 31) / 32;
  // [Q tile][K tile x 2 stages][per-warp hist x, hist y][membership words]
  unsigned *hist = reinterpret_cast<unsigned *>(smem + 3 * kTileBytes);
  uint32_t *mask = reinterpret_cast<uint32_t *>(hist + 2 * 4 * nb2);

  const int qb = blockIdx.x * query_stride, bh = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tq = lane & 3, mi = lane >> 3, r8 = lane & 7;
  const size_t head = (size_t)bh * L * D;

  for (int i = tid; i < 2 * 4 * nb2; i += kHistThreads) hist[i] = 0u;
  for (int w = tid; w < nwords; w += kHistThreads) mask[w] = 0u;
  __syncthreads();
  const int32_t *row = idx + ((size_t)bh * N + qb) * k_sel;
  for (int t = tid; t < k_sel; t += kHistThreads) {
    const int j = row[t];
    if (j >= 0 && j < N) atomicOr(&mask[j >> 5], 1u << (j & 31));
    else report_device_error(kDevErrRange);
  }

  auto load_rows = [&](uint32_t dst, const __nv_bfloat16 *src, int valid) {
    constexpr int kChunksPerRow = D / 8;
    for (int c = tid; c < 64 * kChunksPerRow; c += kHistThreads) {
      const int r = c / kChunksPerRow, col = (c % kChunksPerRow) * 8;
      const bool ok = r < valid;
      cp_async_16(dst + SwizzledTile<D>::offset(r, col), src + (size_t)(ok ? r : 0) * D + col,
                  ok ? 16 : 0);
    }
  };
  load_rows(sbase, Q + head + (size_t)qb * 64 * D, min(64, L - qb * 64));
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
  uint32_t qf[D / 16][4];
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    const int rr = warp * 16 + r8 + 8 * (mi & 1), col = ks * 16 + 8 * (mi >> 1);
    ldmatrix_x4(sbase + SwizzledTile<D>::offset(rr, col), qf[ks][0], qf[ks][1], qf[ks][2],
                qf[ks][3]);
  }
  const int row0 = qb * 64 + warp * 16 + g;   // this thread's rows: row0, row0 + 8
  const bool rv0 = row0 < L, rv1 = row0 + 8 < L;
  unsigned *hx = hist + warp * nb2;
  unsigned *hy = hist + (4 + warp) * nb2;
  const float inv_w = (float)nbins / (hi - lo);
  double m_n = 0, m_x = 0, m_x2 = 0, m_y = 0, m_y2 = 0;
  auto bin = [&](float v) -> int {
    if (!(v >= lo)) return 0;
    if (v >= hi) return nbins + 1;
    return 1 + min(nbins - 1, max(0, __float2int_rd((v - lo) * inv_w)));
  };

  // unselected blocks, in order, double-buffered
  auto next_u = [&](int from) -> int {
    for (int j = from; j < N; ++j)
      if (!((mask[j >> 5] >> (j & 31)) & 1u)) return j;
    return N;
  };
  int j = next_u(0);
  int stage = 0;
  if (j < N) load_rows(sbase + kTileBytes, K + head + (size_t)j * 64 * D, min(64, L - j * 64));
  cp_async_commit();
  while (j < N) {
    const int jn = next_u(j + 1);
    if (jn < N)
      load_rows(sbase + (2 - stage) * kTileBytes, K + head + (size_t)jn * 64 * D,
                min(64, L - jn * 64));
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint32_t sK = sbase + (1 + stage) * kTileBytes;
    float s[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int x = 0; x < 4; ++x) s[n][x] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
      for (int n = 0; n < 8; n += 2) {
        const int key = n * 8 + r8 + 8 * (mi >> 1), dim = ks * 16 + 8 * (mi & 1);
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4(sK + SwizzledTile<D>::offset(key, dim), b0, b1, b2, b3);
        mma_bf16_16816(s[n], qf[ks], b0, b1);
        mma_bf16_16816(s[n + 1], qf[ks], b2, b3);
      }
    }
    const int nj = min(64, L - j * 64);
    // row sums over the block's keys -> centroid score (quad reduction)
    float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int x = 0; x < 2; ++x)
        if (n * 8 + 2 * tq + x < nj) {
          rs0 += s[n][x];
          rs1 += s[n][2 + x];
        }
    rs0 += __shfl_xor_sync(0xffffffffu, rs0, 1);
    rs0 += __shfl_xor_sync(0xffffffffu, rs0, 2);
    rs1 += __shfl_xor_sync(0xffffffffu, rs1, 1);
    rs1 += __shfl_xor_sync(0xffffffffu, rs1, 2);
    const float c0 = scale * rs0 / (float)nj, c1 = scale * rs1 / (float)nj;
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        const bool kv = n * 8 + 2 * tq + x < nj;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (!kv || !(h ? rv1 : rv0)) continue;
          const float xv = scale * s[n][2 * h + x];
          const float yv = xv - (h ? c1 : c0);
          atomicAdd(&hx[bin(xv)], 1u);
          atomicAdd(&hy[bin(yv)], 1u);
          m_n += 1.0;
          m_x += xv;
          m_x2 += (double)xv * xv;
          m_y += yv;
          m_y2 += (double)yv * yv;
        }
      }
    __syncthreads();
    j = jn;
    stage ^= 1;
  }
  cp_async_wait<0>();
  __syncthreads();
  for (int i = tid; i < nb2; i += kHistThreads) {
    unsigned long long sx = 0, sy = 0;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      sx += hist[w * nb2 + i];
      sy += hist[(4 + w) * nb2 + i];
    }
    if (sx) atomicAdd(&hist_x[i], sx);
    if (sy) atomicAdd(&hist_y[i], sy);
  }
  // moments: warp reduction, then one fp64 atomic per warp
  double mv[5] = {m_n, m_x, m_x2, m_y, m_y2};
#pragma unroll
  for (int c = 0; c < 5; ++c) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mv[c] += __shfl_xor_sync(0xffffffffu, mv[c], o);
    if (lane == 0) atomicAdd(&moments[c], mv[c]);
  }
}

}  // namespace pisa
