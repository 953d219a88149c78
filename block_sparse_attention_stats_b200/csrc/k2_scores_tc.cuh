// K2 pass 1 on the tensor cores: the block score matrix of long rows.
//
// "Technical Summary: PISA" (gist.science), section 2 "Covariance-Aware
// Routing": score_ij = scale * (qbar_i . kbar_j) + lambda * M_j.  The
// selection must be exact to float32 rounding, so bf16 operands alone (8
// significant bits) are not enough.  Each centroid coordinate is split into
// three bf16 parts,
//
//   x = x0 + x1 + x2 + r,   x0 = bf16(x), x1 = bf16(x - x0), x2 = bf16(x - x0 - x1),
//
// with |r| <= 2^-27 |x| (every subtraction is exact in float32: it keeps the
// low bits of a float32 value).  The dot product keeps the six cross terms of
// order up to 2^-16,
//
//   q . k ~ q0.k0 + (q0.k1 + q1.k0) + (q0.k2 + q1.k1 + q2.k0),
//
// dropping q1.k2, q2.k1, q2.k2 (order 2^-27 and below), so the float32
// accumulator in tensor memory sees an error of the same order as a
// float32 FMA loop over the head dimension.  The small terms are issued first
// and q0.k0 last, so the large partial sums are formed once.
//
// centroid_split_kernel writes the parts as [B*H][3][N][d] bf16 planes.
// scores_tc_kernel: one CTA per 128 query blocks of one head.  Its three A
// planes (128 x d each) stay in shared memory; a TMA producer warp streams the
// k-bar planes in 256-block x 64-column boxes through a 3-stage ring, one
// elected thread issues tcgen05.mma (M = 128, N = 256, K = 16) into one of two
// 256-column float32 accumulators in tensor memory, and eight epilogue warps
// read the other accumulator, transpose 32 x 32 pieces through shared memory,
// add lambda * M_j and store the score rows with row-contiguous 128-byte
// writes (row stride `ld`, a multiple of 32 floats).
#pragma once

#include "pisa_common.cuh"
#include "sm100_primitives.cuh"

namespace pisa {

// a, b: [rows][D] float32 (rows = B*H*N); a_out, b_out: [B*H][3][N][D] bf16.
__global__ void centroid_split_kernel(const float *__restrict__ a, const float *__restrict__ b,
                                      long long rows, int N, int D,
                                      __nv_bfloat16 *__restrict__ a_out,
                                      __nv_bfloat16 *__restrict__ b_out) {
  const long long n4 = rows * D / 4;
  for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < 2 * n4;
       t += (long long)gridDim.x * blockDim.x) {
    const bool second = t >= n4;
    const float *x = second ? b : a;
    __nv_bfloat16 *out = second ? b_out : a_out;
    const long long e = 4 * (second ? t - n4 : t);
    const long long row = e / D;
    const int col = (int)(e - row * D);
    const long long bh = row / N;
    const int i = (int)(row - bh * N);
    const float4 v = *reinterpret_cast<const float4 *>(x + e);
    float r[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int p = 0; p < 3; ++p) {
      __nv_bfloat16 h[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        h[c] = __float2bfloat16_rn(r[c]);
        r[c] -= __bfloat162float(h[c]);
      }
      uint2 w;
      w.x = (uint32_t)__bfloat16_as_ushort(h[0]) | ((uint32_t)__bfloat16_as_ushort(h[1]) << 16);
      w.y = (uint32_t)__bfloat16_as_ushort(h[2]) | ((uint32_t)__bfloat16_as_ushort(h[3]) << 16);
      *reinterpret_cast<uint2 *>(out + ((bh * 3 + p) * N + i) * (long long)D + col) = w;
    }
  }
}

template <int D> struct ScoreTcCfg {
  static constexpr int kThreads = 320;            // producer, MMA, 8 epilogue warps
  static constexpr int kRows = 128;               // query blocks per CTA (MMA M)
  static constexpr int kCols = 256;               // key blocks per tile (MMA N)
  static constexpr int kBoxes = D / 64;           // 64-column boxes per plane
  static constexpr int kABox = kRows * 128;       // 128 rows x 64 bf16
  static constexpr int kBBox = kCols * 128;       // 256 rows x 64 bf16
  static constexpr int kStages = 3;
  static constexpr int kOffA = 0;
  static constexpr int kOffB = 3 * kBoxes * kABox;
  // per epilogue warp: 32 rows x 32 scores for the transpose that turns
  // one-row-per-thread data into row-contiguous stores; float4 k of row r sits
  // in slot k ^ (r & 7), so both sides of the transpose are conflict-free
  static constexpr int kOffStage = kOffB + kStages * kBBox;
  static constexpr int kStageFloats = 32 * 32;
  static constexpr int kOffBar = kOffStage + 8 * kStageFloats * 4;
  // bars: afull, full[kStages], empty[kStages], accfull[2], accempty[2], teardown
  static constexpr int kNumBars = 1 + 2 * kStages + 4 + 1;
  static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
  static constexpr int kOffMisc = kOffTmemSlot + 16;
  static constexpr int kSmem = kOffMisc + 16 + 1024;   // + alignment slack
  static constexpr uint32_t kTmemCols = 2 * kCols;
  static constexpr int kBoxesPerTile = 3 * kBoxes;     // k-bar boxes per 256-block tile
};
static_assert(ScoreTcCfg<128>::kSmem <= 227 * 1024, "score tile does not fit");

// scores[(bh * N + i) * ld + j] for i, j < N; columns N .. ld-1 of a row may be
// written with values that mean nothing.
template <int D>
__global__ void __launch_bounds__(320, 1)
    scores_tc_kernel(const __grid_constant__ CUtensorMap tm_qs,
                     const __grid_constant__ CUtensorMap tm_ks, const float *__restrict__ cov,
                     float cov_weight, float scale, int N, int ld, float *__restrict__ scores) {
  using C = ScoreTcCfg<D>;
  using namespace sm100;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  unsigned char *smem = smem_raw + (sbase - raw);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kOffMisc);
  auto bar = [&](int i) -> uint32_t { return sbase + C::kOffBar + 8 * i; };
  const uint32_t afull = bar(0);
  auto full = [&](int s) { return bar(1 + s); };
  auto empty = [&](int s) { return bar(1 + C::kStages + s); };
  auto accfull = [&](int g) { return bar(1 + 2 * C::kStages + g); };
  auto accempty = [&](int g) { return bar(3 + 2 * C::kStages + g); };
  const uint32_t teardown = bar(5 + 2 * C::kStages);

  const int i0 = blockIdx.x * C::kRows, bh = blockIdx.y;
  const int ntile = ceil_div(N, C::kCols);
  const int tid = threadIdx.x, lane = tid & 31;
  const int warp = __shfl_sync(0xffffffffu, tid >> 5, 0);

  if (warp == 1) {
    tmem_alloc(sbase + C::kOffTmemSlot, C::kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(afull, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(accfull(g), 1);
      mbar_init(accempty(g), 8);
    }
    mbar_init(teardown, 1);
    fence_mbar_init();
    *abort_flag = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + C::kOffTmemSlot);

  if (warp == 0) {
    // ======================= TMA producer =====================================
    if (lane == 0) {
      prefetch_tmap(&tm_qs);
      prefetch_tmap(&tm_ks);
      mbar_expect_tx(afull, 3 * C::kBoxes * C::kABox);
#pragma unroll
      for (int p = 0; p < 3; ++p)
#pragma unroll
        for (int b = 0; b < C::kBoxes; ++b)
          tma_load_3d(sbase + C::kOffA + (p * C::kBoxes + b) * C::kABox, &tm_qs, afull, 64 * b,
                      i0, bh * 3 + p);
      int t = 0;
      bool ok = true;
      for (int c = 0; ok && c < ntile; ++c) {
        for (int u = 0; u < C::kBoxesPerTile; ++u, ++t) {
          const int q = 2 - u / C::kBoxes, b = u % C::kBoxes;   // planes 2, 1, 0
          const int slot = t % C::kStages;
          if (t >= C::kStages && !mbar_wait(empty(slot), ((t / C::kStages) - 1) & 1)) {
            ok = false;
            break;
          }
          if (*abort_flag) { ok = false; break; }
          mbar_expect_tx(full(slot), C::kBBox);
          tma_load_3d(sbase + C::kOffB + slot * C::kBBox, &tm_ks, full(slot), 64 * b,
                      c * C::kCols, bh * 3 + q);
        }
      }
      if (!ok) {
        *abort_flag = 1;
        // copies in flight land before the CTA exits
        mbar_wait(afull, 0);
        for (int u = (t >= C::kStages ? t - C::kStages : 0); u < t; ++u)
          mbar_wait(full(u % C::kStages), (u / C::kStages) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ======================= MMA issuer =======================================
    if (lane == 0) {
      constexpr uint32_t kId = idesc_bf16_f32(C::kRows, C::kCols, 0, 0);
      bool ok = mbar_wait(afull, 0);
      int t = 0;
      for (int c = 0; ok && c < ntile; ++c) {
        const int g = c & 1;
        if (c >= 2 && !mbar_wait(accempty(g), ((c >> 1) - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        bool first = true;
        for (int u = 0; u < C::kBoxesPerTile; ++u, ++t) {
          const int q = 2 - u / C::kBoxes, b = u % C::kBoxes;
          const int slot = t % C::kStages;
          if (!mbar_wait(full(slot), (t / C::kStages) & 1)) { ok = false; break; }
          if (*abort_flag) { ok = false; break; }
          tc_fence_after();
          const uint32_t bst = sbase + C::kOffB + slot * C::kBBox;
          // A planes p with p + q <= 2, the smaller terms first
          for (int p = 2 - q; p >= 0; --p) {
            const uint32_t ast = sbase + C::kOffA + (p * C::kBoxes + b) * C::kABox;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              mma_ss(tmem + C::kCols * g, smem_desc_sw128(ast + kk * 32, 16, 1024),
                     smem_desc_sw128(bst + kk * 32, 16, 1024), kId, first ? 0u : 1u);
              first = false;
            }
          }
          tc_commit(empty(slot));
        }
        if (ok) tc_commit(accfull(g));
      }
      if (!ok) *abort_flag = 1;
      // every MMA issued must finish before tensor memory is released
      tc_commit(teardown);
      mbar_wait(teardown, 0);
    }
    __syncwarp();
  } else {
    // ======================= epilogue =========================================
    // Warps 2-5 take the even 32-column chunks of a tile, warps 6-9 the odd
    // ones; warp w reads tensor-memory lanes 32 (w % 4) .. +31.  Thread = one
    // row for the load; after the transpose through shared memory lane l
    // stores floats 4 (l % 8) .. +3 of rows 4 rr + l / 8, so each store
    // instruction writes 4 rows x 128 bytes.
    const int sp = warp & 3;                 // tensor-memory lane quarter
    const int half = (warp - 2) >> 2;        // chunk parity
    float *stg = reinterpret_cast<float *>(smem + C::kOffStage) + (warp - 2) * C::kStageFloats;
    const int cq = lane & 7, rq = lane >> 3;
    const float *covh = cov + (size_t)bh * N;
    const int rbase = i0 + sp * 32;          // query block of stage row 0
    float *dst = scores + ((size_t)bh * N + rbase + rq) * (size_t)ld + 4 * cq;
    for (int c = 0; c < ntile; ++c) {
      const int g = c & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(accfull(g), (c >> 1) & 1))) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(sp * 32) << 16) + C::kCols * g;
#pragma unroll 1
      for (int q8 = half; q8 < C::kCols / 32; q8 += 2) {
        const int j = c * C::kCols + 32 * q8;
        if (j >= N) break;                   // the same for every lane
        uint32_t v[32];
        tmem_ld_x32(taddr + 32 * q8, v);
        // lambda * M_j of this lane's four columns (0 past N)
        float cw[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int jj = j + 4 * cq + x;
          cw[x] = (cov_weight != 0.f && jj < N) ? cov_weight * covh[jj] : 0.f;
        }
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 8; ++k)
          *reinterpret_cast<float4 *>(stg + lane * 32 + 4 * (k ^ (lane & 7))) =
              make_float4(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]),
                          __uint_as_float(v[4 * k + 2]), __uint_as_float(v[4 * k + 3]));
        __syncwarp();
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) {
          const int r = 4 * rr + rq;
          const float4 a = *reinterpret_cast<const float4 *>(stg + r * 32 + 4 * (cq ^ (r & 7)));
          float4 o;
          o.x = fmaf(scale, a.x, cw[0]);
          o.y = fmaf(scale, a.y, cw[1]);
          o.z = fmaf(scale, a.z, cw[2]);
          o.w = fmaf(scale, a.w, cw[3]);
          if (rbase + r < N) *reinterpret_cast<float4 *>(dst + (size_t)(4 * rr) * ld + j) = o;
        }
        __syncwarp();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(accempty(g));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace pisa
