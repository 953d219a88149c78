// K3 (warp-MMA version): fused exact-or-approximate attention.
//
// "Technical Summary: PISA" (gist.science), section 2: "Core Algorithm" (the
// numerator N_t equation with alpha_{t,j} = exp(q_t kbar_j^T), o_t = N_t/D_t),
// "Key Insights" 2 (normalization consistency: the approximations enter the
// same numerator and denominator), "Hardware Implementation" phases 1-3
// (exact phase over the selected blocks, zeroth-order scan of the aggregated
// block vectors of the unselected blocks, global first-order correction).
//
// One CTA = one 64-row query block of one head, 4 warps x 16 rows, bf16
// mma.sync m16n8k16 with float32 accumulators, one online softmax (running
// row max m, denominator l, output accumulator o) shared by
//   * exact tiles: the 64 keys/values of each selected block j in S_i;
//   * centroid tiles: 64 consecutive block centroids kbar_j as keys and the
//     block value sums vsum_j as values, weight n_j in the denominator,
//     masked to the unselected blocks U_i; their softmax weights are also
//     summed into a_t = sum_{U_i} alpha_tj;
//   * hyd: o += (s a_t q_t) Hbar as one more MMA (rows of Q scaled by s a_t).
// Logits live in the log2 domain (scaled by s log2 e) for exp2.
// K/V tiles are double-buffered with cp.async into XOR-swizzled smem.
#pragma once

#include "pisa_common.cuh"

namespace pisa {

constexpr int kAttnWarps = 4;
constexpr int kAttnThreads = kAttnWarps * 32;
constexpr int kAttnRows = 64;

template <int D> struct AttnSmem {
  static constexpr int kTileBytes = kAttnRows * D * 2;
  // Q, then stages [K0 V0 K1 V1] (K0+V0 also hold Hbar, D x D, in the epilogue)
  static constexpr int kQ = 0;
  static constexpr int kStage0 = kTileBytes;
  static constexpr int kFixed = 5 * kTileBytes;
};

template <int D>
__device__ __forceinline__ void attn_load_rows(uint32_t dst, const __nv_bfloat16 *src, int rows,
                                               int valid_rows) {
  constexpr int kChunksPerRow = D / 8;
  const int total = rows * kChunksPerRow;
  for (int c = threadIdx.x; c < total; c += kAttnThreads) {
    const int row = c / kChunksPerRow, col = (c % kChunksPerRow) * 8;
    const bool ok = row < valid_rows;
    cp_async_16(dst + SwizzledTile<D>::offset(row, col), src + (size_t)(ok ? row : 0) * D + col,
                ok ? 16 : 0);
  }
}

// Tile list entry: >= 0 exact block j; < 0 centroid chunk -(c + 1).
// DENSE: every block is an exact tile, no centroids, no first-order term.
template <int D, bool DENSE>
__global__ void __launch_bounds__(kAttnThreads)
    piecewise_attention_mma_kernel(const __nv_bfloat16 *__restrict__ Q,
                                   const __nv_bfloat16 *__restrict__ K,
                                   const __nv_bfloat16 *__restrict__ V,
                                   const __nv_bfloat16 *__restrict__ kbar16,  // [BH, Npad, D]
                                   const __nv_bfloat16 *__restrict__ vsum16,  // [BH, Npad, D]
                                   const __nv_bfloat16 *__restrict__ hbar16,  // [BH, D, D]
                                   const int32_t *__restrict__ idx,           // [BH, N, k_sel]
                                   int k_sel, int L, int N, int Npad, float scale, int hyd,
                                   void *__restrict__ out, int out_f32) {
  using S = AttnSmem<D>;
  extern __shared__ __align__(128) unsigned char smem[];
  const uint32_t sbase = smem_u32(smem);
  const int nwords = (N + 31) / 32;
  uint32_t *mask = reinterpret_cast<uint32_t *>(smem + S::kFixed);
  int *tiles = reinterpret_cast<int *>(mask + nwords);
  __shared__ int s_ntiles;

  const int qb = blockIdx.x, bh = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tq = lane & 3, mi = lane >> 3, r8 = lane & 7;
  const size_t head = (size_t)bh * L * D;
  const int nchunks = (N + 63) / 64;

  // ---- membership mask of S_i and the tile list -------------------------
  if (!DENSE) {
    for (int w = tid; w < nwords; w += kAttnThreads) mask[w] = 0u;
    __syncthreads();
    const int32_t *row = idx + ((size_t)bh * N + qb) * k_sel;
    for (int t = tid; t < k_sel; t += kAttnThreads) {
      const int j = row[t];
      if (j >= 0 && j < N) {
        atomicOr(&mask[j >> 5], 1u << (j & 31));
        tiles[t] = j;
      } else {
        report_device_error(kDevErrRange);
        tiles[t] = 0;  // keeps the loads in bounds; result is flagged invalid
      }
    }
    __syncthreads();
    if (tid == 0) {
      int n = k_sel;
      for (int c = 0; c < nchunks; ++c) {
        const int lo = c * 64, cnt = min(64, N - lo);
        // skip chunks whose blocks are all selected
        int sel = __popc(mask[lo >> 5] & (cnt >= 32 ? 0xffffffffu : ((1u << cnt) - 1u)));
        if (cnt > 32) sel += __popc(mask[(lo >> 5) + 1] & (cnt == 64 ? 0xffffffffu : ((1u << (cnt - 32)) - 1u)));
        if (sel < cnt) tiles[n++] = -(c + 1);
      }
      s_ntiles = n;
    }
    __syncthreads();
  } else {
    if (tid == 0) s_ntiles = N;
    __syncthreads();
  }
  const int ntiles = s_ntiles;

  auto tile_block = [&](int t) -> int { return DENSE ? t : tiles[t]; };
  auto issue = [&](int t) {
    const int e = tile_block(t);
    const uint32_t st = sbase + S::kStage0 + (t & 1) * 2 * S::kTileBytes;
    if (e >= 0) {
      const size_t off = head + (size_t)e * 64 * D;
      const int valid = min(64, L - e * 64);
      attn_load_rows<D>(st, K + off, 64, valid);
      attn_load_rows<D>(st + S::kTileBytes, V + off, 64, valid);
    } else {
      const int c = -e - 1;
      const size_t off = ((size_t)bh * Npad + (size_t)c * 64) * D;
      attn_load_rows<D>(st, kbar16 + off, 64, 64);
      attn_load_rows<D>(st + S::kTileBytes, vsum16 + off, 64, 64);
    }
  };

  // ---- Q tile + first K/V tile ------------------------------------------
  attn_load_rows<D>(sbase + S::kQ, Q + head + (size_t)qb * 64 * D, 64, min(64, L - qb * 64));
  issue(0);
  cp_async_commit();

  float o[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[n][e] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f}, a_run[2] = {0.f, 0.f};
  uint32_t qf[D / 16][4];
  const float sl2 = scale * kLog2e;

  for (int t = 0; t < ntiles; ++t) {
    if (t + 1 < ntiles) issue(t + 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (t == 0) {
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const int row = warp * 16 + r8 + 8 * (mi & 1), col = ks * 16 + 8 * (mi >> 1);
        ldmatrix_x4(sbase + S::kQ + SwizzledTile<D>::offset(row, col), qf[ks][0], qf[ks][1],
                    qf[ks][2], qf[ks][3]);
      }
    }
    const int e = tile_block(t);
    const bool centroid = e < 0;
    const uint32_t sK = sbase + S::kStage0 + (t & 1) * 2 * S::kTileBytes;
    const uint32_t sV = sK + S::kTileBytes;

    // S = Q K^T for 16 rows x 64 keys
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
    // mask, key weights
    float w[8][2];
    float tile_max[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int n = 0; n < 8; ++n) {
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        const int col = n * 8 + 2 * tq + x;
        bool ok;
        float wt;
        if (!centroid) {
          ok = e * 64 + col < L;
          wt = 1.f;
        } else {
          const int jj = (-e - 1) * 64 + col;
          ok = jj < N && !((mask[jj >> 5] >> (jj & 31)) & 1u);
          wt = (float)min(64, L - jj * 64);
        }
        w[n][x] = ok ? wt : 0.f;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float v = ok ? s[n][2 * h + x] * sl2 : -INFINITY;
          s[n][2 * h + x] = v;
          tile_max[h] = fmaxf(tile_max[h], v);
        }
      }
    }
    float corr[2], shift[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      tile_max[h] = fmaxf(tile_max[h], __shfl_xor_sync(0xffffffffu, tile_max[h], 1));
      tile_max[h] = fmaxf(tile_max[h], __shfl_xor_sync(0xffffffffu, tile_max[h], 2));
      const float m_new = fmaxf(m_run[h], tile_max[h]);
      shift[h] = (m_new == -INFINITY) ? 0.f : m_new;
      corr[h] = exp2f(m_run[h] - shift[h]);  // 0 when m_run = -inf
      m_run[h] = m_new;
    }
    float psum[2] = {0.f, 0.f}, wsum[2] = {0.f, 0.f};
    uint32_t pf[4][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float p0 = exp2f(s[n][2 * h] - shift[h]);
        const float p1 = exp2f(s[n][2 * h + 1] - shift[h]);
        psum[h] += p0 + p1;
        wsum[h] += p0 * w[n][0] + p1 * w[n][1];
        s[n][2 * h] = p0;
        s[n][2 * h + 1] = p1;
      }
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      pf[kk][0] = pack_bf16x2(s[2 * kk][0], s[2 * kk][1]);
      pf[kk][1] = pack_bf16x2(s[2 * kk][2], s[2 * kk][3]);
      pf[kk][2] = pack_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pf[kk][3] = pack_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      l_run[h] = l_run[h] * corr[h] + wsum[h];
      a_run[h] = a_run[h] * corr[h] + (centroid ? psum[h] : 0.f);
    }
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      o[n][0] *= corr[0];
      o[n][1] *= corr[0];
      o[n][2] *= corr[1];
      o[n][3] *= corr[1];
    }
    // o += P V
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
      for (int n = 0; n < D / 8; n += 2) {
        const int key = kk * 16 + r8 + 8 * (mi & 1), dim = n * 8 + 8 * (mi >> 1);
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4_trans(sV + SwizzledTile<D>::offset(key, dim), b0, b1, b2, b3);
        mma_bf16_16816(o[n], pf[kk], b0, b1);
        mma_bf16_16816(o[n + 1], pf[kk], b2, b3);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  // a_t and l_t are partial per thread: reduce across the quad
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 1);
    l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 2);
    a_run[h] += __shfl_xor_sync(0xffffffffu, a_run[h], 1);
    a_run[h] += __shfl_xor_sync(0xffffffffu, a_run[h], 2);
  }

  // ---- hyd: o += (s a_t q_t) Hbar ----------------------------------------
  if (!DENSE && hyd) {
    __syncthreads();
    const uint32_t sH = sbase + S::kStage0;  // D rows x D cols, swizzled
    attn_load_rows<D>(sH, hbar16 + (size_t)bh * D * D, D, D);
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    const float f0 = scale * a_run[0], f1 = scale * a_run[1];
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t a[4];
      // A fragment registers: a0 row g, a1 row g+8, a2 row g, a3 row g+8
      const float fr[4] = {f0, f1, f0, f1};
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162 *>(&qf[ks][x]);
        float2 f = __bfloat1622float2(v);
        a[x] = pack_bf16x2(f.x * fr[x], f.y * fr[x]);
      }
#pragma unroll
      for (int n = 0; n < D / 8; n += 2) {
        const int krow = ks * 16 + r8 + 8 * (mi & 1), dim = n * 8 + 8 * (mi >> 1);
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4_trans(sH + SwizzledTile<D>::offset(krow, dim), b0, b1, b2, b3);
        mma_bf16_16816(o[n], a, b0, b1);
        mma_bf16_16816(o[n + 1], a, b2, b3);
      }
    }
  }

  // ---- epilogue: out = o / l ---------------------------------------------
  const float inv0 = 1.f / l_run[0], inv1 = 1.f / l_run[1];
  const int row0 = qb * 64 + warp * 16 + g, row1 = row0 + 8;
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    const int col = n * 8 + 2 * tq;
    if (out_f32) {
      float *O = reinterpret_cast<float *>(out) + head;
      if (row0 < L)
        *reinterpret_cast<float2 *>(O + (size_t)row0 * D + col) =
            make_float2(o[n][0] * inv0, o[n][1] * inv0);
      if (row1 < L)
        *reinterpret_cast<float2 *>(O + (size_t)row1 * D + col) =
            make_float2(o[n][2] * inv1, o[n][3] * inv1);
    } else {
      __nv_bfloat16 *O = reinterpret_cast<__nv_bfloat16 *>(out) + head;
      if (row0 < L)
        *reinterpret_cast<uint32_t *>(O + (size_t)row0 * D + col) =
            pack_bf16x2(o[n][0] * inv0, o[n][1] * inv0);
      if (row1 < L)
        *reinterpret_cast<uint32_t *>(O + (size_t)row1 * D + col) =
            pack_bf16x2(o[n][2] * inv1, o[n][3] * inv1);
    }
  }
}

// ---------------------------------------------------------------------------
// packing helpers for K3
// ---------------------------------------------------------------------------
// kbar16/vsum16 [BH, Npad, D] (rows >= N zero), hbar16 [BH, D, D]
__global__ void pack_stats_kernel(const float *__restrict__ kbar, const float *__restrict__ vsum,
                                  const float *__restrict__ hbar, int N, int Npad, int D, int BH,
                                  __nv_bfloat16 *__restrict__ kbar16,
                                  __nv_bfloat16 *__restrict__ vsum16,
                                  __nv_bfloat16 *__restrict__ hbar16) {
  const size_t nrow = (size_t)BH * Npad * D;
  const size_t nh = (size_t)BH * D * D;
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < nrow + nh;
       e += (size_t)gridDim.x * blockDim.x) {
    if (e < nrow) {
      const size_t bh = e / ((size_t)Npad * D), rem = e % ((size_t)Npad * D);
      const int j = (int)(rem / D), c = (int)(rem % D);
      const bool ok = j < N;
      const size_t src = (bh * N + j) * D + c;
      kbar16[e] = __float2bfloat16_rn(ok ? kbar[src] : 0.f);
      vsum16[e] = __float2bfloat16_rn(ok ? vsum[src] : 0.f);
    } else {
      const size_t h = e - nrow;
      hbar16[h] = __float2bfloat16_rn(hbar[h]);
    }
  }
}

__global__ void f32_to_bf16_kernel(const float *__restrict__ src, __nv_bfloat16 *__restrict__ dst,
                                   size_t n) {
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n;
       e += (size_t)gridDim.x * blockDim.x)
    dst[e] = __float2bfloat16_rn(src[e]);
}

}  // namespace pisa
