// K1: block statistics of PISA (pre-computation phase).
//
// "Technical Summary: PISA" (gist.science), section 2: "Hardware
// Implementation" step 1 (block centroids, value sums and the global statistic
// Hbar), "Core Algorithm" (kbar_j, sum of values), "Global First-Order
// Correction" (Hbar = mean of the block-wise first-order matrices) and
// "Covariance-Aware Routing" (M_j = ||H_j - Hbar||).
//
// Per (b, h) and block j of n_j tokens:
//   qbar_j = (1/n_j) sum_n q_n          kbar_j = (1/n_j) sum_n k_n
//   vsum_j = sum_n v_n                   H_j = sum_n k_n^T v_n - kbar_j^T vsum_j
//   hbar = (1/N) sum_j H_j               cov_j = ||H_j - hbar||_F
// (sum_n (k_n - kbar_j)^T v_n = sum_n k_n^T v_n - n_j kbar_j^T vbar_j.)
//
// Pass 1 (stats_pass_*): one CTA per (chunk of consecutive blocks, head).  It
// streams the Q/K/V tiles of its blocks once, writes qbar/kbar/vsum, and keeps
// sum_j H_j of its chunk in registers; the chunk partial goes to scratch.
// Pass 2 (hbar_reduce): sums the chunk partials in chunk order -> hbar.
// Pass 3 (cov_pass_*, only with covariance-aware scoring): re-streams K/V,
// rebuilds each H_j and reduces ||H_j - hbar||_F.
// Reduction orders are fixed, so the results are bitwise reproducible.
#pragma once

#include "pisa_common.cuh"
#include "sm100_primitives.cuh"

namespace pisa {

constexpr int kStatsThreads = 256;
constexpr int kBlk = 64;  // tokens per streamed tile; a block is 1 or 2 tiles (block_size 64 / 128)

// Chunking of pass 1: at most two CTAs per SM over the whole problem (one wave).
__host__ __device__ inline int stats_num_chunks(int BH, int N) {
  int want = (2 * 148) / BH;
  if (want < 1) want = 1;
  return want < N ? want : N;
}

// ---------------------------------------------------------------------------
// bf16 pass 1: tensor-core K_j^T V_j with mma.sync, cp.async double buffering.
// ---------------------------------------------------------------------------
template <int D> struct StatsMmaCfg {
  static constexpr int kWarpsM = (D == 128) ? 4 : 2;
  static constexpr int kWarpsN = 8 / kWarpsM;
  static constexpr int kWarpRows = D / kWarpsM;  // 32
  static constexpr int kWarpCols = D / kWarpsN;  // 64 (D=128) or 16 (D=64)
  static constexpr int kMT = kWarpRows / 16;     // 2
  static constexpr int kNT = kWarpCols / 8;      // 8 or 2
  static constexpr int kTileBytes = kBlk * D * 2;
};

template <int D>
__device__ __forceinline__ void stats_load_tile_bf16(uint32_t dst, const __nv_bfloat16 *src,
                                                     int valid_rows) {
  constexpr int kChunksPerRow = D / 8;
  constexpr int kChunks = kBlk * kChunksPerRow;
  for (int c = threadIdx.x; c < kChunks; c += kStatsThreads) {
    int row = c / kChunksPerRow, col = (c % kChunksPerRow) * 8;
    bool ok = row < valid_rows;
    const __nv_bfloat16 *g = src + (size_t)(ok ? row : 0) * D + col;
    cp_async_16(dst + SwizzledTile<D>::offset(row, col), g, ok ? 16 : 0);
  }
}

// Accumulates acc += K^T V for one 64-token tile pair (swizzled smem tiles).
template <int D>
__device__ __forceinline__ void ktv_mma(float (&acc)[StatsMmaCfg<D>::kMT][StatsMmaCfg<D>::kNT][4],
                                        uint32_t sK, uint32_t sV, int warp_m0, int warp_n0,
                                        int lane) {
  using C = StatsMmaCfg<D>;
  const int mi = lane >> 3, r = lane & 7;
#pragma unroll
  for (int k0 = 0; k0 < kBlk; k0 += 16) {
    uint32_t a[C::kMT][4];
#pragma unroll
    for (int mt = 0; mt < C::kMT; ++mt) {
      int tok = k0 + r + 8 * (mi >> 1);
      int dim = warp_m0 + mt * 16 + 8 * (mi & 1);
      ldmatrix_x4_trans(sK + SwizzledTile<D>::offset(tok, dim), a[mt][0], a[mt][1], a[mt][2],
                        a[mt][3]);
    }
#pragma unroll
    for (int nt = 0; nt < C::kNT; nt += 2) {
      int tok = k0 + r + 8 * (mi & 1);
      int dim = warp_n0 + nt * 8 + 8 * (mi >> 1);
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4_trans(sV + SwizzledTile<D>::offset(tok, dim), b0, b1, b2, b3);
#pragma unroll
      for (int mt = 0; mt < C::kMT; ++mt) {
        mma_bf16_16816(acc[mt][nt], a[mt], b0, b1);
        mma_bf16_16816(acc[mt][nt + 1], a[mt], b2, b3);
      }
    }
  }
}

// Column sums of the Q, K and V tiles (3 x D columns, 64 rows each) on the
// tensor cores: C = 1^T X with an all-ones A operand; every row of C holds the
// column sums.  Warp w handles n-tiles 6w .. 6w+5 of the 3D/8 tiles.
template <int D>
__device__ __forceinline__ void colsum_mma(uint32_t tiles, float *colsum, int warp, int lane,
                                           bool accumulate) {
  using C = StatsMmaCfg<D>;
  constexpr int kNT = 3 * D / 8;           // 8-column tiles over Q, K, V
  constexpr int kPerWarp = kNT / 8;        // 6 (D=128) or 3 (D=64)
  const uint32_t one2 = 0x3F803F80u;       // two bf16 1.0
  const uint32_t ones[4] = {one2, one2, one2, one2};
  float acc[kPerWarp][4];
#pragma unroll
  for (int i = 0; i < kPerWarp; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[i][e] = 0.f;
  const int mi = lane >> 3, r = lane & 7;
#pragma unroll
  for (int k0 = 0; k0 < kBlk; k0 += 16) {
#pragma unroll
    for (int i = 0; i < kPerWarp; ++i) {
      const int nt = warp * kPerWarp + i;
      const int which = nt / (D / 8), col = (nt % (D / 8)) * 8;
      // B fragment (16 tokens x 8 columns) of tile `which`, via ldmatrix.trans
      const int tok = k0 + r + 8 * (mi & 1);
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4_trans(tiles + which * C::kTileBytes + SwizzledTile<D>::offset(tok, col), b0, b1,
                        b2, b3);
      (void)b2;
      (void)b3;
      mma_bf16_16816(acc[i], ones, b0, b1);
    }
  }
  if (lane < 4) {
#pragma unroll
    for (int i = 0; i < kPerWarp; ++i) {
      const int nt = warp * kPerWarp + i;
      const int which = nt / (D / 8), col = (nt % (D / 8)) * 8 + 2 * lane;
      colsum[which * D + col] = accumulate ? colsum[which * D + col] + acc[i][0] : acc[i][0];
      colsum[which * D + col + 1] =
          accumulate ? colsum[which * D + col + 1] + acc[i][1] : acc[i][1];
    }
  }
}

// Two CTAs per SM (registers capped at 128): one CTA's loads stay in flight
// while the other computes, which the HBM-bound pass needs.
template <int D>
__global__ void __launch_bounds__(kStatsThreads, 2)
    stats_pass_bf16_kernel(const __nv_bfloat16 *__restrict__ Q, const __nv_bfloat16 *__restrict__ K,
                           const __nv_bfloat16 *__restrict__ V, int L, int N, int sub, int nchunk,
                           float *__restrict__ qbar, float *__restrict__ kbar,
                           float *__restrict__ vsum, float *__restrict__ partial) {
  // N blocks of sub x 64 tokens; the kernel streams 64-token tiles
  using C = StatsMmaCfg<D>;
  extern __shared__ __align__(128) unsigned char smem[];
  // [stage][Q,K,V] tiles, then column sums (3 x D floats)
  float *colsum = reinterpret_cast<float *>(smem + 2 * 3 * C::kTileBytes);
  const uint32_t sbase = smem_u32(smem);

  const int chunk = blockIdx.x, bh = blockIdx.y;
  const int per = ceil_div(N, nchunk);
  const int j0 = chunk * per, j1 = min(N, j0 + per);
  const int ntile = ceil_div(L, kBlk);
  const int u0 = j0 * sub, u1 = min(ntile, j1 * sub);   // 64-token tiles of this chunk
  const size_t head = (size_t)bh * L * D;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int warp_m0 = (warp / C::kWarpsN) * C::kWarpRows;
  const int warp_n0 = (warp % C::kWarpsN) * C::kWarpCols;

  float acc[C::kMT][C::kNT][4];
#pragma unroll
  for (int mt = 0; mt < C::kMT; ++mt)
#pragma unroll
    for (int nt = 0; nt < C::kNT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;

  auto issue = [&](int u, int stage) {
    int valid = min(kBlk, L - u * kBlk);
    size_t off = head + (size_t)u * kBlk * D;
    uint32_t st = sbase + stage * 3 * C::kTileBytes;
    stats_load_tile_bf16<D>(st, Q + off, valid);
    stats_load_tile_bf16<D>(st + C::kTileBytes, K + off, valid);
    stats_load_tile_bf16<D>(st + 2 * C::kTileBytes, V + off, valid);
  };

  if (u0 < u1) issue(u0, 0);
  cp_async_commit();
  for (int u = u0; u < u1; ++u) {
    const int stage = (u - u0) & 1;
    if (u + 1 < u1) issue(u + 1, stage ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();

    const int j = u / sub, s = u - j * sub;
    const bool last = s == sub - 1 || u == ntile - 1;   // block j ends with this tile
    // column sums of Q, K, V (zero-filled rows past L add nothing), summed
    // over the tiles of block j
    colsum_mma<D>(sbase + stage * 3 * C::kTileBytes, colsum, warp, lane, s > 0);
    const uint32_t sK = sbase + stage * 3 * C::kTileBytes + C::kTileBytes;
    ktv_mma<D>(acc, sK, sK + C::kTileBytes, warp_m0, warp_n0, lane);
    __syncthreads();  // colsum visible
    if (last) {
      const int n_j = min(sub * kBlk, L - j * sub * kBlk);
      const float inv_n = 1.f / (float)n_j;
      const size_t so = ((size_t)bh * N + j) * D;
      for (int t = tid; t < 3 * D; t += kStatsThreads) {
        const int which = t / D, col = t % D;
        if (which == 0) qbar[so + col] = colsum[t] * inv_n;
        else if (which == 1) kbar[so + col] = colsum[t] * inv_n;
        else vsum[so + col] = colsum[t];
      }
      // acc -= kbar_j^T vsum_j
      const int g = lane >> 2, tq = lane & 3;
#pragma unroll
      for (int mt = 0; mt < C::kMT; ++mt)
#pragma unroll
        for (int nt = 0; nt < C::kNT; ++nt) {
          const int a0 = warp_m0 + mt * 16 + g, c0 = warp_n0 + nt * 8 + 2 * tq;
          const float ka = colsum[D + a0] * inv_n, kb = colsum[D + a0 + 8] * inv_n;
          const float v0 = colsum[2 * D + c0], v1 = colsum[2 * D + c0 + 1];
          acc[mt][nt][0] -= ka * v0;
          acc[mt][nt][1] -= ka * v1;
          acc[mt][nt][2] -= kb * v0;
          acc[mt][nt][3] -= kb * v1;
        }
    }
    __syncthreads();  // stage and colsum free for reuse
  }
  cp_async_wait<0>();

  float *P = partial + ((size_t)bh * nchunk + chunk) * D * D;
  const int g = lane >> 2, tq = lane & 3;
#pragma unroll
  for (int mt = 0; mt < C::kMT; ++mt)
#pragma unroll
    for (int nt = 0; nt < C::kNT; ++nt) {
      const int a0 = warp_m0 + mt * 16 + g, c0 = warp_n0 + nt * 8 + 2 * tq;
      *reinterpret_cast<float2 *>(P + (size_t)a0 * D + c0) =
          make_float2(acc[mt][nt][0], acc[mt][nt][1]);
      *reinterpret_cast<float2 *>(P + (size_t)(a0 + 8) * D + c0) =
          make_float2(acc[mt][nt][2], acc[mt][nt][3]);
    }
}

// ---------------------------------------------------------------------------
// bf16 pass 1, streamed: one CTA per SM walks a contiguous range of the
// B*H*N blocks (its range may end inside a head and the next CTA's begin
// there).  Q, K and V tiles arrive by TMA (cp.async.bulk.tensor, no multicast)
// into a four-stage mbarrier ring.
//   warp 0      issues the copies;
//   warp 1      allocates TMEM and issues G_j = K_j^T V_j of each block as
//               tcgen05 MMAs (M = N = D, both operands MN-major straight from
//               the tiles, 16 tokens per MMA) into one of two TMEM buffers;
//   warps 2-9   sum the columns of Q, K and V on the CUDA cores (float32, in
//               token order), write qbar, kbar, vsum at the end of each block,
//               then read G_j back and add G_j - kbar_j^T vsum_j to a float32
//               register accumulator of sum_j H_j (warps w and w + 4 take the
//               rows of TMEM sub-partition w % 4 and half of the columns each).
// The accumulator goes to the partial of the head segment (segment s of head
// bh is the s-th CTA whose range meets that head) when the head changes;
// hbar_reduce_seg_kernel adds a head's segments in order, so the result is
// bitwise reproducible.
// ---------------------------------------------------------------------------
constexpr int kStatsCtas = 148;       // one per SM of a B200
constexpr int kStatsStages = 4;

__host__ __device__ inline int stats_stream_ctas(long long total_blocks) {
  return total_blocks < kStatsCtas ? (int)total_blocks : kStatsCtas;
}
// first global block (bh * N + j) of CTA c's range
__host__ __device__ inline long long stats_first_block(int c, long long total, int nc) {
  return (long long)c * total / nc;
}
// the CTA whose range holds global block G
__host__ __device__ inline int stats_cta_of(long long G, long long total, int nc) {
  return (int)(((G + 1) * nc + total - 1) / total) - 1;
}
// an upper bound on the CTAs whose range meets one head of N blocks
__host__ __device__ inline int stats_max_segments(int BH, int N) {
  const long long total = (long long)BH * N;
  const int nc = stats_stream_ctas(total);
  long long per = total / nc;
  if (per < 1) per = 1;
  return (int)(N / per) + 2;
}

template <int D> struct StatsTmaCfg {
  static constexpr int kThreads = 32 * 10;
  static constexpr int kTileBytes = kBlk * D * 2;           // one 64-token tile of one tensor
  static constexpr int kStageBytes = 3 * kTileBytes;        // Q, K, V
  static constexpr int kBoxBytes = kBlk * 128;              // 64 tokens x 64 columns
  // kbar_j and vsum_j of the block being finished, double-buffered by block parity
  static constexpr int kOffKV = kStatsStages * kStageBytes;
  static constexpr int kOffBar = kOffKV + 2 * 2 * D * 4;
  // bars: full[4], empty[4], gfull[2], gempty[2], teardown
  static constexpr int kNumBars = 2 * kStatsStages + 5;
  static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
  static constexpr int kOffMisc = kOffTmemSlot + 16;
  static constexpr int kSmem = kOffMisc + 16 + 1024;        // + alignment slack
  static constexpr uint32_t kTmemCols = 2 * D < 32 ? 32 : 2 * D;   // two G buffers
};

// named barrier 1 over the consumer warps of one kernel (every warp from
// index 2 up): kCount = 32 x that kernel's consumer warps
template <int kCount> __device__ __forceinline__ void stats_consumer_barrier() {
  static_assert(kCount % 32 == 0, "whole warps");
  asm volatile("bar.sync 1, %0;" ::"n"(kCount) : "memory");
}

template <int D>
__global__ void __launch_bounds__(32 * 10, 1)
    stats_pass_tma_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, int L, int N, int sub,
                          int BH, int maxseg, float *__restrict__ qbar,
                          float *__restrict__ kbar, float *__restrict__ vsum,
                          float *__restrict__ partial) {
  using T = StatsTmaCfg<D>;
  using namespace sm100;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  unsigned char *smem = smem_raw + (sbase - raw);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + T::kOffMisc);
  volatile int *cflag = abort_flag + 1;   // [2]: consumers' abort, by block parity
  auto bar = [&](int i) -> uint32_t { return sbase + T::kOffBar + 8 * i; };
  auto full = [&](int s) { return bar(s); };
  auto empty = [&](int s) { return bar(kStatsStages + s); };
  auto gfull = [&](int g) { return bar(2 * kStatsStages + g); };
  auto gempty = [&](int g) { return bar(2 * kStatsStages + 2 + g); };
  const uint32_t teardown = bar(2 * kStatsStages + 4);

  const long long total = (long long)BH * N;
  const int nc = gridDim.x, c = blockIdx.x;
  const long long g0 = stats_first_block(c, total, nc), g1 = stats_first_block(c + 1, total, nc);
  const int ntile = ceil_div(L, kBlk);
  const int tid = threadIdx.x, lane = tid & 31;
  const int warp = __shfl_sync(0xffffffffu, tid >> 5, 0);
  auto tiles_of = [&](long long G) -> int {
    const int j = (int)(G % N);
    return min(sub, ntile - j * sub);
  };

  if (warp == 1) {
    tmem_alloc(sbase + T::kOffTmemSlot, T::kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < kStatsStages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1 + 8);     // the MMA commit and the eight consumer warps
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(gfull(g), 1);
      mbar_init(gempty(g), 8);
    }
    mbar_init(teardown, 1);
    fence_mbar_init();
    abort_flag[0] = 0;
    abort_flag[1] = 0;
    abort_flag[2] = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + T::kOffTmemSlot);

  if (warp == 0) {
    // ======================= TMA producer =====================================
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      int t = 0;
      bool ok = true;
      for (long long G = g0; ok && G < g1; ++G) {
        const int bh = (int)(G / N), j = (int)(G % N);
        const int nt = tiles_of(G);
        for (int s = 0; s < nt; ++s, ++t) {
          const int slot = t % kStatsStages;
          if (t >= kStatsStages && !mbar_wait(empty(slot), ((t / kStatsStages) - 1) & 1)) {
            ok = false;
            break;
          }
          if (*abort_flag) { ok = false; break; }
          const uint32_t dst = sbase + slot * T::kStageBytes;
          const int row = (j * sub + s) * kBlk;
          mbar_expect_tx(full(slot), T::kStageBytes);
#pragma unroll
          for (int b = 0; b < D / 64; ++b) {
            tma_load_3d(dst + b * T::kBoxBytes, &tm_q, full(slot), 64 * b, row, bh);
            tma_load_3d(dst + T::kTileBytes + b * T::kBoxBytes, &tm_k, full(slot), 64 * b, row, bh);
            tma_load_3d(dst + 2 * T::kTileBytes + b * T::kBoxBytes, &tm_v, full(slot), 64 * b, row,
                        bh);
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        // copies in flight land before the CTA exits (at most one per stage)
        for (int u = (t >= kStatsStages ? t - kStatsStages : 0); u < t; ++u)
          mbar_wait(full(u % kStatsStages), (u / kStatsStages) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ======================= MMA issuer =======================================
    if (lane == 0) {
      // G = K^T V: A = K^T (M = D dimensions, MN-major), B = V (N = D, MN-major);
      // 16 tokens (2048 bytes of a 128-byte-row tile) per instruction
      constexpr uint32_t kId = idesc_bf16_f32(128, D, 1, 1);
      int t = 0, blk = 0;
      bool ok = true;
      for (long long G = g0; ok && G < g1; ++G, ++blk) {
        const int g = blk & 1;
        // the consumers have read G of block blk - 2 out of this buffer
        if (blk >= 2 && !mbar_wait(gempty(g), ((blk >> 1) - 1) & 1)) { ok = false; break; }
        const int nt = tiles_of(G);
        for (int s = 0; s < nt; ++s, ++t) {
          const int slot = t % kStatsStages;
          if (!mbar_wait(full(slot), (t / kStatsStages) & 1)) { ok = false; break; }
          if (*abort_flag) { ok = false; break; }
          tc_fence_after();
          const uint32_t kst = sbase + slot * T::kStageBytes + T::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < kBlk / 16; ++kk)
            mma_ss(tmem + D * g, smem_desc_sw128(kst + kk * 2048, T::kBoxBytes, 1024),
                   smem_desc_sw128(kst + T::kTileBytes + kk * 2048, T::kBoxBytes, 1024), kId,
                   (s > 0 || kk > 0) ? 1u : 0u);
          tc_commit(empty(slot));
        }
        if (ok) tc_commit(gfull(g));
      }
      if (!ok) *abort_flag = 1;
      // every MMA issued must finish before TMEM is released
      tc_commit(teardown);
      mbar_wait(teardown, 0);
    }
    __syncwarp();
  } else {
    // ======================= consumers ========================================
    const int cw = warp - 2, ctid = tid - 64;
    const int sp = warp & 3, ch = cw >> 2;      // TMEM sub-partition, column half of G
    const int arow = sp * 32 + lane;            // row of G (a key dimension)
    constexpr int kH = D / 2;                   // columns of G per thread
    float hacc[kH];
#pragma unroll
    for (int i = 0; i < kH; ++i) hacc[i] = 0.f;
    // column sums: thread p < 3 D / 2 owns the column pair (2 lp, 2 lp + 1) of
    // tensor p / (D / 2) (Q, K or V)
    const int p = ctid, tns = p / (D / 2), lp = p % (D / 2);
    const bool sums = p < 3 * (D / 2);
    const uint32_t col_off = (uint32_t)(tns * T::kTileBytes + (lp / 32) * T::kBoxBytes);
    const int chunk = (lp % 32) / 4, inword = (lp % 4) * 4;
    float ps0[4] = {0.f, 0.f, 0.f, 0.f}, ps1[4] = {0.f, 0.f, 0.f, 0.f};
    auto flush = [&](int bh) {
      const int seg = c - stats_cta_of((long long)bh * N, total, nc);
      float *P = partial + ((size_t)bh * maxseg + seg) * D * D + (size_t)arow * D + ch * kH;
#pragma unroll
      for (int i = 0; i < kH; i += 4)
        *reinterpret_cast<float4 *>(P + i) = make_float4(hacc[i], hacc[i + 1], hacc[i + 2], hacc[i + 3]);
#pragma unroll
      for (int i = 0; i < kH; ++i) hacc[i] = 0.f;
    };
    int cur_bh = (int)(g0 / N);
    int t = 0, blk = 0;
    bool ok = true;
    for (long long G = g0; ok && G < g1; ++G, ++blk) {
      const int bh = (int)(G / N), j = (int)(G % N), g = blk & 1;
      if (bh != cur_bh) {
        flush(cur_bh);
        cur_bh = bh;
      }
      const int nt = tiles_of(G);
      bool bad = false;
      for (int s = 0; s < nt; ++s, ++t) {
        const int slot = t % kStatsStages;
        if (!__all_sync(0xffffffffu, mbar_wait(full(slot), (t / kStatsStages) & 1))) {
          bad = true;
          break;
        }
        if (sums) {
          // four interleaved partial sums (rows r % 4) keep four load-add
          // chains in flight; they are combined in a fixed order at block end
          const unsigned char *tile = smem + slot * T::kStageBytes + col_off + inword;
#pragma unroll 16
          for (int r = 0; r < kBlk; ++r) {
            const uint32_t w =
                *reinterpret_cast<const uint32_t *>(tile + r * 128 + ((chunk ^ (r & 7)) << 4));
            ps0[r & 3] += __uint_as_float(w << 16);
            ps1[r & 3] += __uint_as_float(w & 0xffff0000u);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty(slot));
      }
      // block end: statistics, then G_j - kbar_j^T vsum_j into the accumulator
      const int n_j = min(sub * kBlk, L - j * sub * kBlk);
      const float inv_n = 1.f / (float)n_j;
      float *kv = reinterpret_cast<float *>(smem + T::kOffKV) + g * 2 * D;   // kbar, vsum
      const float cs0 = (ps0[0] + ps0[1]) + (ps0[2] + ps0[3]);
      const float cs1 = (ps1[0] + ps1[1]) + (ps1[2] + ps1[3]);
      if (sums && !bad) {
        const size_t so = ((size_t)bh * N + j) * D + 2 * lp;
        if (tns == 0) {
          *reinterpret_cast<float2 *>(qbar + so) = make_float2(cs0 * inv_n, cs1 * inv_n);
        } else if (tns == 1) {
          *reinterpret_cast<float2 *>(kbar + so) = make_float2(cs0 * inv_n, cs1 * inv_n);
          kv[2 * lp] = cs0 * inv_n;
          kv[2 * lp + 1] = cs1 * inv_n;
        } else {
          *reinterpret_cast<float2 *>(vsum + so) = make_float2(cs0, cs1);
          kv[D + 2 * lp] = cs0;
          kv[D + 2 * lp + 1] = cs1;
        }
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) ps0[k] = ps1[k] = 0.f;
      if (!__all_sync(0xffffffffu, mbar_wait(gfull(g), (blk >> 1) & 1))) bad = true;
      // every consumer warp takes the same decision: the flag of this block's
      // parity is written only before this barrier and read only after it
      if (bad) {
        cflag[blk & 1] = 1;
        *abort_flag = 1;
      }
      stats_consumer_barrier<T::kThreads - 64>();
      if (cflag[blk & 1]) { ok = false; break; }
      tc_fence_after();
      const float ka = kv[arow];
      const uint32_t taddr = tmem + ((uint32_t)(sp * 32) << 16) + D * g + ch * kH;
#pragma unroll
      for (int q = 0; q < kH / 32; ++q) {
        uint32_t r[32];
        tmem_ld_x32(taddr + 32 * q, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i)
          hacc[32 * q + i] += __uint_as_float(r[i]) - ka * kv[D + ch * kH + 32 * q + i];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(gempty(g));
    }
    if (ok && g0 < g1) flush(cur_bh);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, T::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Streamed pass 3 (bf16, d = 128): cov_j = ||G_j - kbar_j^T vsum_j - hbar||_F
// with G_j = K_j^T V_j formed again on tcgen05.  Same CTA ranges as pass 1.
// Warp 0 streams K and V tiles through a four-stage TMA ring, warp 1 issues
// the K^T V products into two TMEM buffers, warps 2-9 read each block's G
// back (thread = row arow of G, half ch of its columns), subtract
// kbar_j[arow] vsum_j and the thread's 64 entries of hbar (kept in registers
// per head), and sum the squares; the 256 partial sums meet in a fixed order
// (warp shuffles, then the eight warps in index order), so cov is bitwise
// reproducible.
// ---------------------------------------------------------------------------
template <int D> struct CovTmaCfg {
  static constexpr int kThreads = 32 * 10;
  static constexpr int kTileBytes = kBlk * D * 2;           // one 64-token tile of K or V
  static constexpr int kStageBytes = 2 * kTileBytes;        // K, V
  static constexpr int kBoxBytes = kBlk * 128;              // 64 tokens x 64 columns
  static constexpr int kOffRed = kStatsStages * kStageBytes;   // [2][8] warp sums
  static constexpr int kOffBar = kOffRed + 2 * 8 * 4;
  // bars: full[4], empty[4], gfull[2], gempty[2], teardown
  static constexpr int kNumBars = 2 * kStatsStages + 5;
  static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
  static constexpr int kOffMisc = kOffTmemSlot + 16;
  static constexpr int kSmem = kOffMisc + 16 + 1024;        // + alignment slack
  static constexpr uint32_t kTmemCols = 2 * D;              // two G buffers
};

template <int D>
__global__ void __launch_bounds__(32 * 10, 1)
    cov_pass_tma_kernel(const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, int L, int N, int sub, int BH,
                        const float *__restrict__ kbar, const float *__restrict__ vsum,
                        const float *__restrict__ hbar, float *__restrict__ cov) {
  using T = CovTmaCfg<D>;
  using namespace sm100;
  static_assert(D == 128, "the consumer layout assumes 128 rows of G");
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  unsigned char *smem = smem_raw + (sbase - raw);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + T::kOffMisc);
  volatile int *cflag = abort_flag + 1;   // [2]: consumers' abort, by block parity
  float *red = reinterpret_cast<float *>(smem + T::kOffRed);
  auto bar = [&](int i) -> uint32_t { return sbase + T::kOffBar + 8 * i; };
  auto full = [&](int s) { return bar(s); };
  auto empty = [&](int s) { return bar(kStatsStages + s); };
  auto gfull = [&](int g) { return bar(2 * kStatsStages + g); };
  auto gempty = [&](int g) { return bar(2 * kStatsStages + 2 + g); };
  const uint32_t teardown = bar(2 * kStatsStages + 4);

  const long long total = (long long)BH * N;
  const int nc = gridDim.x, c = blockIdx.x;
  const long long g0 = stats_first_block(c, total, nc), g1 = stats_first_block(c + 1, total, nc);
  const int ntile = ceil_div(L, kBlk);
  const int tid = threadIdx.x, lane = tid & 31;
  const int warp = __shfl_sync(0xffffffffu, tid >> 5, 0);
  auto tiles_of = [&](long long G) -> int {
    const int j = (int)(G % N);
    return min(sub, ntile - j * sub);
  };

  if (warp == 1) {
    tmem_alloc(sbase + T::kOffTmemSlot, T::kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < kStatsStages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);         // the MMA commit
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(gfull(g), 1);
      mbar_init(gempty(g), 8);
    }
    mbar_init(teardown, 1);
    fence_mbar_init();
    abort_flag[0] = 0;
    abort_flag[1] = 0;
    abort_flag[2] = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + T::kOffTmemSlot);

  if (warp == 0) {
    // ======================= TMA producer =====================================
    if (lane == 0) {
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      int t = 0;
      bool ok = true;
      for (long long G = g0; ok && G < g1; ++G) {
        const int bh = (int)(G / N), j = (int)(G % N);
        const int nt = tiles_of(G);
        for (int s = 0; s < nt; ++s, ++t) {
          const int slot = t % kStatsStages;
          if (t >= kStatsStages && !mbar_wait(empty(slot), ((t / kStatsStages) - 1) & 1)) {
            ok = false;
            break;
          }
          if (*abort_flag) { ok = false; break; }
          const uint32_t dst = sbase + slot * T::kStageBytes;
          const int row = (j * sub + s) * kBlk;
          mbar_expect_tx(full(slot), T::kStageBytes);
#pragma unroll
          for (int b = 0; b < D / 64; ++b) {
            tma_load_3d(dst + b * T::kBoxBytes, &tm_k, full(slot), 64 * b, row, bh);
            tma_load_3d(dst + T::kTileBytes + b * T::kBoxBytes, &tm_v, full(slot), 64 * b, row,
                        bh);
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        for (int u = (t >= kStatsStages ? t - kStatsStages : 0); u < t; ++u)
          mbar_wait(full(u % kStatsStages), (u / kStatsStages) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ======================= MMA issuer =======================================
    if (lane == 0) {
      constexpr uint32_t kId = idesc_bf16_f32(128, D, 1, 1);
      int t = 0, blk = 0;
      bool ok = true;
      for (long long G = g0; ok && G < g1; ++G, ++blk) {
        const int g = blk & 1;
        if (blk >= 2 && !mbar_wait(gempty(g), ((blk >> 1) - 1) & 1)) { ok = false; break; }
        const int nt = tiles_of(G);
        for (int s = 0; s < nt; ++s, ++t) {
          const int slot = t % kStatsStages;
          if (!mbar_wait(full(slot), (t / kStatsStages) & 1)) { ok = false; break; }
          if (*abort_flag) { ok = false; break; }
          tc_fence_after();
          const uint32_t kst = sbase + slot * T::kStageBytes;
#pragma unroll
          for (int kk = 0; kk < kBlk / 16; ++kk)
            mma_ss(tmem + D * g, smem_desc_sw128(kst + kk * 2048, T::kBoxBytes, 1024),
                   smem_desc_sw128(kst + T::kTileBytes + kk * 2048, T::kBoxBytes, 1024), kId,
                   (s > 0 || kk > 0) ? 1u : 0u);
          tc_commit(empty(slot));
        }
        if (ok) tc_commit(gfull(g));
      }
      if (!ok) *abort_flag = 1;
      tc_commit(teardown);
      mbar_wait(teardown, 0);
    }
    __syncwarp();
  } else {
    // ======================= consumers ========================================
    const int cw = warp - 2, ctid = tid - 64;
    const int sp = warp & 3, ch = cw >> 2;      // TMEM sub-partition, column half of G
    const int arow = sp * 32 + lane;            // row of G (a key dimension)
    constexpr int kH = D / 2;                   // columns of G per thread
    float hb[kH];
    int cur_bh = -1;
    int blk = 0;
    bool ok = true;
    for (long long G = g0; ok && G < g1; ++G, ++blk) {
      const int bh = (int)(G / N), g = blk & 1;
      if (bh != cur_bh) {
        const float4 *h4 =
            reinterpret_cast<const float4 *>(hbar + ((size_t)bh * D + arow) * D + ch * kH);
#pragma unroll
        for (int i = 0; i < kH / 4; ++i) {
          const float4 x = h4[i];
          hb[4 * i] = x.x;
          hb[4 * i + 1] = x.y;
          hb[4 * i + 2] = x.z;
          hb[4 * i + 3] = x.w;
        }
        cur_bh = bh;
      }
      const float ka = kbar[(size_t)G * D + arow];
      const float *vs = vsum + (size_t)G * D + ch * kH;
      bool bad = !__all_sync(0xffffffffu, mbar_wait(gfull(g), (blk >> 1) & 1));
      float ss = 0.f;
      if (!bad) {
        tc_fence_after();
        const uint32_t taddr = tmem + ((uint32_t)(sp * 32) << 16) + D * g + ch * kH;
#pragma unroll
        for (int q = 0; q < kH / 32; ++q) {
          uint32_t r[32];
          tmem_ld_x32(taddr + 32 * q, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float e = __uint_as_float(r[i]) - ka * vs[32 * q + i] - hb[32 * q + i];
            ss = fmaf(e, e, ss);
          }
        }
        tc_fence_before();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(gempty(g));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (lane == 0) red[g * 8 + cw] = ss;
      // every consumer warp takes the same decision: the flag of this block's
      // parity is written only before this barrier and read only after it
      if (bad) {
        cflag[blk & 1] = 1;
        *abort_flag = 1;
      }
      stats_consumer_barrier<T::kThreads - 64>();
      if (cflag[blk & 1]) { ok = false; break; }
      if (ctid == 0) {
        const float *rg = red + g * 8;
        const float tot = ((rg[0] + rg[1]) + (rg[2] + rg[3])) + ((rg[4] + rg[5]) + (rg[6] + rg[7]));
        cov[G] = sqrtf(tot);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, T::kTmemCols);
  }
}

// pass 2 of the streamed pass: hbar = (1/N) sum of the head's segment partials,
// in segment order.
__global__ void hbar_reduce_seg_kernel(const float *__restrict__ partial, int maxseg, int DD,
                                       int N, int BH, int nc, float *__restrict__ hbar) {
  const int bh = blockIdx.y;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= DD) return;
  const long long total = (long long)BH * N;
  const int c0 = stats_cta_of((long long)bh * N, total, nc);
  const int c1 = stats_cta_of((long long)(bh + 1) * N - 1, total, nc);
  const float *p = partial + (size_t)bh * maxseg * DD + e;
  float s = 0.f;
  // the loads of four segments go out together; the sum stays in segment order
#pragma unroll 4
  for (int seg = 0; seg <= c1 - c0; ++seg) s += p[(size_t)seg * DD];
  hbar[(size_t)bh * DD + e] = s / (float)N;
}

// ---------------------------------------------------------------------------
// f32 pass 1: plain FMA version (small f32 workloads).
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kStatsThreads)
    stats_pass_f32_kernel(const float *__restrict__ Q, const float *__restrict__ K,
                          const float *__restrict__ V, int L, int N, int sub, int nchunk,
                          float *__restrict__ qbar, float *__restrict__ kbar,
                          float *__restrict__ vsum, float *__restrict__ partial) {
  constexpr int kPer = D * D / kStatsThreads;
  extern __shared__ __align__(128) unsigned char smem[];
  float *sQ = reinterpret_cast<float *>(smem);
  float *sK = sQ + kBlk * D;
  float *sV = sK + kBlk * D;
  float *colsum = sV + kBlk * D;  // 3 x D

  const int chunk = blockIdx.x, bh = blockIdx.y;
  const int per = ceil_div(N, nchunk);
  const int j0 = chunk * per, j1 = min(N, j0 + per);
  const size_t head = (size_t)bh * L * D;
  const int tid = threadIdx.x;
  float acc[kPer];
#pragma unroll
  for (int r = 0; r < kPer; ++r) acc[r] = 0.f;

  for (int j = j0; j < j1; ++j) {
    const int n_j = min(sub * kBlk, L - j * sub * kBlk);
    for (int t = tid; t < 3 * D; t += kStatsThreads) colsum[t] = 0.f;
    // the block's 64-token tiles: column sums and sum_n k_n^T v_n
    for (int s0 = 0; s0 < n_j; s0 += kBlk) {
      const int rows = min(kBlk, n_j - s0);
      const size_t off = head + ((size_t)j * sub * kBlk + s0) * D;
      __syncthreads();
      for (int e = tid; e < kBlk * D; e += kStatsThreads) {
        const bool ok = e < rows * D;
        sQ[e] = ok ? Q[off + e] : 0.f;
        sK[e] = ok ? K[off + e] : 0.f;
        sV[e] = ok ? V[off + e] : 0.f;
      }
      __syncthreads();
      for (int t = tid; t < 3 * D; t += kStatsThreads) {
        const float *tile = (t < D) ? sQ : (t < 2 * D ? sK : sV);
        const int col = t % D;
        float sum = 0.f;
        for (int row = 0; row < kBlk; ++row) sum += tile[row * D + col];
        colsum[t] += sum;
      }
#pragma unroll
      for (int r = 0; r < kPer; ++r) {
        const int e = tid + r * kStatsThreads, a = e / D, c = e % D;
        float sum = 0.f;
        for (int row = 0; row < kBlk; ++row) sum += sK[row * D + a] * sV[row * D + c];
        acc[r] += sum;
      }
    }
    __syncthreads();
    const float inv_n = 1.f / (float)n_j;
#pragma unroll
    for (int r = 0; r < kPer; ++r) {
      const int e = tid + r * kStatsThreads, a = e / D, c = e % D;
      acc[r] -= (colsum[D + a] * inv_n) * colsum[2 * D + c];
    }
    const size_t so = ((size_t)bh * N + j) * D;
    for (int t = tid; t < 3 * D; t += kStatsThreads) {
      const int col = t % D;
      if (t < D) qbar[so + col] = colsum[t] * inv_n;
      else if (t < 2 * D) kbar[so + col] = colsum[t] * inv_n;
      else vsum[so + col] = colsum[t];
    }
    __syncthreads();
  }
  float *P = partial + ((size_t)bh * nchunk + chunk) * D * D;
#pragma unroll
  for (int r = 0; r < kPer; ++r) P[tid + r * kStatsThreads] = acc[r];
}

// ---------------------------------------------------------------------------
// pass 2: hbar = (1/N) sum over chunk partials, in chunk order.
// ---------------------------------------------------------------------------
__global__ void hbar_reduce_kernel(const float *__restrict__ partial, int nchunk, int DD, int N,
                                   float *__restrict__ hbar) {
  const int bh = blockIdx.y;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= DD) return;
  const float *p = partial + (size_t)bh * nchunk * DD + e;
  float s = 0.f;
  for (int c = 0; c < nchunk; ++c) s += p[(size_t)c * DD];
  hbar[(size_t)bh * DD + e] = s / (float)N;
}

// ---------------------------------------------------------------------------
// pass 3: cov_j = ||H_j - hbar||_F
// ---------------------------------------------------------------------------
__device__ __forceinline__ float block_reduce_sum(float v, float *red) {
  // fixed-order reduction: butterfly inside each warp, then warp 0 over warps
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
  if (warp == 0) {
    t = lane < (int)(blockDim.x >> 5) ? red[lane] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  }
  __syncthreads();
  return t;  // valid in warp 0
}

template <int D>
__global__ void __launch_bounds__(kStatsThreads)
    cov_pass_bf16_kernel(const __nv_bfloat16 *__restrict__ K, const __nv_bfloat16 *__restrict__ V,
                         int L, int N, int sub, int nchunk, const float *__restrict__ kbar,
                         const float *__restrict__ vsum, const float *__restrict__ hbar,
                         float *__restrict__ cov) {
  using C = StatsMmaCfg<D>;
  extern __shared__ __align__(128) unsigned char smem[];
  float *red = reinterpret_cast<float *>(smem + 2 * 2 * C::kTileBytes);
  const uint32_t sbase = smem_u32(smem);
  const int chunk = blockIdx.x, bh = blockIdx.y;
  const int per = ceil_div(N, nchunk);
  const int j0 = chunk * per, j1 = min(N, j0 + per);
  const int ntile = ceil_div(L, kBlk);
  const int u0 = j0 * sub, u1 = min(ntile, j1 * sub);
  const size_t head = (size_t)bh * L * D;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int warp_m0 = (warp / C::kWarpsN) * C::kWarpRows;
  const int warp_n0 = (warp % C::kWarpsN) * C::kWarpCols;
  const int g = lane >> 2, tq = lane & 3;

  // hbar entries matching this thread's accumulator fragment
  float hb[C::kMT][C::kNT][4];
  const float *Hb = hbar + (size_t)bh * D * D;
#pragma unroll
  for (int mt = 0; mt < C::kMT; ++mt)
#pragma unroll
    for (int nt = 0; nt < C::kNT; ++nt) {
      const int a0 = warp_m0 + mt * 16 + g, c0 = warp_n0 + nt * 8 + 2 * tq;
      hb[mt][nt][0] = Hb[a0 * D + c0];
      hb[mt][nt][1] = Hb[a0 * D + c0 + 1];
      hb[mt][nt][2] = Hb[(a0 + 8) * D + c0];
      hb[mt][nt][3] = Hb[(a0 + 8) * D + c0 + 1];
    }

  auto issue = [&](int u, int stage) {
    int valid = min(kBlk, L - u * kBlk);
    size_t off = head + (size_t)u * kBlk * D;
    uint32_t st = sbase + stage * 2 * C::kTileBytes;
    stats_load_tile_bf16<D>(st, K + off, valid);
    stats_load_tile_bf16<D>(st + C::kTileBytes, V + off, valid);
  };
  float acc[C::kMT][C::kNT][4];
  if (u0 < u1) issue(u0, 0);
  cp_async_commit();
  for (int u = u0; u < u1; ++u) {
    const int stage = (u - u0) & 1;
    if (u + 1 < u1) issue(u + 1, stage ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const int j = u / sub, s = u - j * sub;
    const bool last = s == sub - 1 || u == ntile - 1;
    if (s == 0) {
#pragma unroll
      for (int mt = 0; mt < C::kMT; ++mt)
#pragma unroll
        for (int nt = 0; nt < C::kNT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
    }
    const uint32_t sK = sbase + stage * 2 * C::kTileBytes;
    ktv_mma<D>(acc, sK, sK + C::kTileBytes, warp_m0, warp_n0, lane);
    __syncthreads();  // tiles of this stage consumed
    if (last) {
      const float *kb = kbar + ((size_t)bh * N + j) * D;
      const float *vs = vsum + ((size_t)bh * N + j) * D;
      float ss = 0.f;
#pragma unroll
      for (int mt = 0; mt < C::kMT; ++mt)
#pragma unroll
        for (int nt = 0; nt < C::kNT; ++nt) {
          const int a0 = warp_m0 + mt * 16 + g, c0 = warp_n0 + nt * 8 + 2 * tq;
          const float ka = kb[a0], kc = kb[a0 + 8], v0 = vs[c0], v1 = vs[c0 + 1];
          float e0 = acc[mt][nt][0] - ka * v0 - hb[mt][nt][0];
          float e1 = acc[mt][nt][1] - ka * v1 - hb[mt][nt][1];
          float e2 = acc[mt][nt][2] - kc * v0 - hb[mt][nt][2];
          float e3 = acc[mt][nt][3] - kc * v1 - hb[mt][nt][3];
          ss += e0 * e0 + e1 * e1 + e2 * e2 + e3 * e3;
        }
      float tot = block_reduce_sum(ss, red);
      if (tid == 0) cov[(size_t)bh * N + j] = sqrtf(tot);
    }
  }
  cp_async_wait<0>();
}

template <int D>
__global__ void __launch_bounds__(kStatsThreads)
    cov_pass_f32_kernel(const float *__restrict__ K, const float *__restrict__ V, int L, int N,
                        int sub, const float *__restrict__ kbar, const float *__restrict__ vsum,
                        const float *__restrict__ hbar, float *__restrict__ cov) {
  constexpr int kPer = D * D / kStatsThreads;
  extern __shared__ __align__(128) unsigned char smem[];
  float *sK = reinterpret_cast<float *>(smem);
  float *sV = sK + kBlk * D;
  float *red = sV + kBlk * D;
  const int j = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
  const int n_j = min(sub * kBlk, L - j * sub * kBlk);
  float acc[kPer];
#pragma unroll
  for (int r = 0; r < kPer; ++r) acc[r] = 0.f;
  for (int s0 = 0; s0 < n_j; s0 += kBlk) {
    const int rows = min(kBlk, n_j - s0);
    const size_t off = (size_t)bh * L * D + ((size_t)j * sub * kBlk + s0) * D;
    __syncthreads();
    for (int e = tid; e < kBlk * D; e += kStatsThreads) {
      const bool ok = e < rows * D;
      sK[e] = ok ? K[off + e] : 0.f;
      sV[e] = ok ? V[off + e] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kPer; ++r) {
      const int e = tid + r * kStatsThreads, a = e / D, c = e % D;
      float sum = 0.f;
      for (int row = 0; row < kBlk; ++row) sum += sK[row * D + a] * sV[row * D + c];
      acc[r] += sum;
    }
  }
  const float *kb = kbar + ((size_t)bh * N + j) * D;
  const float *vs = vsum + ((size_t)bh * N + j) * D;
  const float *Hb = hbar + (size_t)bh * D * D;
  float ss = 0.f;
#pragma unroll
  for (int r = 0; r < kPer; ++r) {
    const int e = tid + r * kStatsThreads, a = e / D, c = e % D;
    const float h = acc[r] - kb[a] * vs[c] - Hb[e];
    ss += h * h;
  }
  float tot = block_reduce_sum(ss, red);
  if (tid == 0) cov[(size_t)bh * N + j] = sqrtf(tot);
}

}  // namespace pisa
