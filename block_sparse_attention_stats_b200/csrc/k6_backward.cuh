// Backward of the zeroth-order ("_0th") piecewise attention.
//
// The authors' README ("Kernel variants") ships the zeroth-order variant as
// the one that trains.  Its forward ("Technical Summary: PISA", gist.science,
// section 2 "Core Algorithm", without the first-order term) is a softmax over
// an augmented key set per query block i:
//   exact keys    k_n of the blocks in S_i, logit z = s q.k_n,             value v_n
//   centroid keys kbar_j of the blocks in U_i, logit z = s q.kbar_j + ln n_j,
//                                                        value vbar_j = SigmaV_j / n_j
// so o_t = sum_m P_tm value_m with P_t = softmax(z_t), lse_t = ln D_t.  With
// dP_tm = dout_t . value_m, Delta_t = sum_m P_tm dP_tm (= dout_t . o_t) and
// dz_tm = P_tm (dP_tm - Delta_t):
//   dq_t      = s sum_m dz_tm key_m
//   dk_n      = s sum_t dz_tn q_t     + dkbar_j / n_j    (n in block j)
//   dv_n      =   sum_t P_tn dout_t   + dvbar_j / n_j
//   dkbar_j   = s sum_t dz_tj q_t,  dvbar_j = sum_t P_tj dout_t   (t with j in U_i)
// The selection is a discrete step and is held fixed.
//
// Kernels of this file: bf16 operands, f32 accumulation, mma.sync m16n8k16,
// 4 warps of 16 rows; tiles of 64 rows x D in XOR-swizzled shared memory,
// cp.async double buffering.
//   bwd_pack_centroids_kernel bf16 kbar_j and vbar_j (rows >= N zero)
//   bwd_dq_tc_kernel          (k7_bwd_dq_tc.cuh, tcgen05) one CTA per pair of
//                             query blocks, two sweeps over their exact tiles and
//                             the centroid chunks: Delta_t = sum_m P_tm dP_tm,
//                             then dq
//   bwd_centroid_kernel       one CTA per 64-centroid chunk, over every query
//                             block that leaves one of them unselected
//                             -> dkbar_j / n_j, dvbar_j / n_j (float32)
//   bwd_kv_tc_kernel          (k8_bwd_kv_tc.cuh, tcgen05) one CTA per pair of key
//                             blocks, over the query blocks that selected either
//                             -> dk, dv, plus the centroid terms
// No atomics: every output element is written by one CTA, so the results are
// reproducible bit for bit.
#pragma once

#include "pisa_common.cuh"
#include "sm100_primitives.cuh"

namespace pisa {

constexpr int kBwdThreads = 128;
constexpr int kBwdListChunk = 8 * kBwdThreads;   // query blocks examined per list build

// ---------------------------------------------------------------------------
// preprocessing
// ---------------------------------------------------------------------------
// kbar16[bh, j] = bf16(kbar_j), vbar16[bh, j] = bf16(vsum_j / n_j); rows N..Npad-1 zero
__global__ void bwd_pack_centroids_kernel(const float *__restrict__ kbar,
                                          const float *__restrict__ vsum, int N, int Npad, int D,
                                          int BH, int L, __nv_bfloat16 *__restrict__ kbar16,
                                          __nv_bfloat16 *__restrict__ vbar16) {
  const size_t n = (size_t)BH * Npad * D;
  const float inv_last = 1.f / (float)(L - 64 * (N - 1));
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n;
       e += (size_t)gridDim.x * blockDim.x) {
    const size_t bh = e / ((size_t)Npad * D), rem = e % ((size_t)Npad * D);
    const int j = (int)(rem / D), c = (int)(rem % D);
    const bool ok = j < N;
    const size_t src = (bh * N + (ok ? j : 0)) * D + c;
    const float inv_n = j == N - 1 ? inv_last : (1.f / 64.f);
    kbar16[e] = __float2bfloat16_rn(ok ? kbar[src] : 0.f);
    vbar16[e] = __float2bfloat16_rn(ok ? vsum[src] * inv_n : 0.f);
  }
}

// ---------------------------------------------------------------------------
// warp-level tile products
// ---------------------------------------------------------------------------
// 64 x D tile rows [0, valid) from global rows of D elements; the rest zero.
template <int D>
__device__ __forceinline__ void bwd_load_tile(uint32_t dst, const __nv_bfloat16 *src, int valid,
                                              int tid) {
  constexpr int kChunksPerRow = D / 8;
  for (int c = tid; c < 64 * kChunksPerRow; c += kBwdThreads) {
    const int r = c / kChunksPerRow, col = (c % kChunksPerRow) * 8;
    const bool ok = r < valid;
    cp_async_16(dst + SwizzledTile<D>::offset(r, col), src + (size_t)(ok ? r : 0) * D + col,
                ok ? 16 : 0);
  }
}

__device__ __forceinline__ void cp_async_4(uint32_t dst, const void *src, int src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(dst), "l"(src),
               "r"(src_bytes));
}

// acc[n] (16 x 8 each, n < NT) = A[a_row0 + 0..15, 0..D) . B[b_row0 + 8n + 0..7, 0..D)^T
// for swizzled row-major tiles A and B (the contraction runs over the D columns).
template <int D, int NT>
__device__ __forceinline__ void bwd_gemm_abt(float (&acc)[NT][4], uint32_t sA, int a_row0,
                                             uint32_t sB, int b_row0, int lane) {
  const int mi = lane >> 3, r8 = lane & 7;
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int x = 0; x < 4; ++x) acc[n][x] = 0.f;
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    uint32_t a[4];
    ldmatrix_x4(sA + SwizzledTile<D>::offset(a_row0 + r8 + 8 * (mi & 1), ks * 16 + 8 * (mi >> 1)),
                a[0], a[1], a[2], a[3]);
#pragma unroll
    for (int n = 0; n < NT; n += 2) {
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4(sB + SwizzledTile<D>::offset(b_row0 + n * 8 + r8 + 8 * (mi >> 1),
                                               ks * 16 + 8 * (mi & 1)),
                  b0, b1, b2, b3);
      mma_bf16_16816(acc[n], a, b0, b1);
      mma_bf16_16816(acc[n + 1], a, b2, b3);
    }
  }
}

// acc (16 x D) += A (16 x 16 KT, bf16 fragments) . B[b_row0 + 0 .. 16 KT, 0..D)
// where B is a swizzled row-major tile whose rows run along the contraction.
template <int D, int KT>
__device__ __forceinline__ void bwd_gemm_ab(float (&acc)[D / 8][4], const uint32_t (&a)[KT][4],
                                            uint32_t sB, int b_row0, int lane) {
  const int mi = lane >> 3, r8 = lane & 7;
#pragma unroll
  for (int kk = 0; kk < KT; ++kk) {
#pragma unroll
    for (int n0 = 0; n0 < D; n0 += 16) {
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4_trans(sB + SwizzledTile<D>::offset(b_row0 + kk * 16 + r8 + 8 * (mi & 1),
                                                     n0 + 8 * (mi >> 1)),
                        b0, b1, b2, b3);
      mma_bf16_16816(acc[n0 / 8], a[kk], b0, b1);
      mma_bf16_16816(acc[n0 / 8 + 1], a[kk], b2, b3);
    }
  }
}

// C fragments of a 16 x 16 KT product -> bf16 A fragments over the same columns
template <int KT>
__device__ __forceinline__ void bwd_c_to_a(const float (&c)[2 * KT][4], uint32_t (&a)[KT][4]) {
#pragma unroll
  for (int kk = 0; kk < KT; ++kk) {
    a[kk][0] = pack_bf16x2(c[2 * kk][0], c[2 * kk][1]);
    a[kk][1] = pack_bf16x2(c[2 * kk][2], c[2 * kk][3]);
    a[kk][2] = pack_bf16x2(c[2 * kk + 1][0], c[2 * kk + 1][1]);
    a[kk][3] = pack_bf16x2(c[2 * kk + 1][2], c[2 * kk + 1][3]);
  }
}

__device__ __forceinline__ uint64_t bwd_valid_bits64(int c, int N) {   // centroids 64c.. < N
  const int n = N - 64 * c;
  return n >= 64 ? ~0ull : ((1ull << n) - 1ull);
}

// ---------------------------------------------------------------------------
// centroid gradients: one CTA per chunk of 64 centroids
// ---------------------------------------------------------------------------
template <int D> struct BwdCentCfg {
  static constexpr int kTile = 64 * D * 2;
  static constexpr int kOffVec = 6 * kTile;                 // lse, delta: 2 stages x 2 x 64 f32
  static constexpr int kOffList = kOffVec + 2 * 2 * 64 * 4;  // query-block list
  static constexpr int kOffWarp = kOffList + kBwdListChunk * 4;
  static constexpr int kSmem = kOffWarp + 4 * 4;
};

// The chunk's kbar_j / vbar_j tiles stay in shared memory; the CTA visits
// every query block that leaves one of the chunk's centroids unselected
// (lists built 1024 query blocks at a time).  lse and delta are the padded
// [BH, Lpad] arrays (rows past L: lse +inf, delta 0).
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 2)
    bwd_centroid_kernel(const __nv_bfloat16 *__restrict__ Q,
                        const __nv_bfloat16 *__restrict__ dO, const float *__restrict__ lse,
                        const float *__restrict__ delta, const __nv_bfloat16 *__restrict__ kbar16,
                        const __nv_bfloat16 *__restrict__ vbar16,
                        const uint32_t *__restrict__ bm, int L, int Lpad, int N, int Npad,
                        int nwords, float scale, float *__restrict__ dkbar,
                        float *__restrict__ dvbar) {
  using Cfg = BwdCentCfg<D>;
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int kT = Cfg::kTile;
  const uint32_t sb = smem_u32(smem);
  const uint32_t sK = sb, sV = sb + kT;
  float *vec = reinterpret_cast<float *>(smem + Cfg::kOffVec);   // [stage][lse | delta][64]
  int *list = reinterpret_cast<int *>(smem + Cfg::kOffList);
  int *wsum = reinterpret_cast<int *>(smem + Cfg::kOffWarp);
  const int jb = blockIdx.x, bh = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tq = lane & 3;
  const size_t head = (size_t)bh * L * D;
  const int n_last = L - 64 * (N - 1);
  const float sl2 = scale * kLog2e;

  const size_t cb = ((size_t)bh * Npad + 64 * jb) * D;
  bwd_load_tile<D>(sK, kbar16 + cb, 64, tid);
  bwd_load_tile<D>(sV, vbar16 + cb, 64, tid);
  const int kA = warp * 16 + g, kB = kA + 8;       // this thread's centroid rows
  const float fixA = 64 * jb + kA == N - 1 ? (float)n_last : 64.f;   // n_j
  const float fixB = 64 * jb + kB == N - 1 ? (float)n_last : 64.f;
  const uint64_t cvalid = bwd_valid_bits64(jb, N);

  auto selected_word = [&](int i, int w) -> uint32_t {
    return w < nwords ? bm[((size_t)bh * N + i) * nwords + w] : 0u;
  };
  auto unselected = [&](int i) -> uint64_t {
    const uint64_t sel = (uint64_t)selected_word(i, 2 * jb) |
                         ((uint64_t)selected_word(i, 2 * jb + 1) << 32);
    return ~sel & cvalid;
  };
  auto issue = [&](int i, int stage) {
    const uint32_t dq = sb + (2 + 2 * stage) * kT, ddo = dq + kT;
    const int nq = min(64, L - 64 * i);
    bwd_load_tile<D>(dq, Q + head + (size_t)i * 64 * D, nq, tid);
    bwd_load_tile<D>(ddo, dO + head + (size_t)i * 64 * D, nq, tid);
    const int r = tid & 63;
    const float *src = (tid < 64 ? lse : delta) + (size_t)bh * Lpad + 64 * i;
    cp_async_4(smem_u32(vec + (stage * 2 + (tid >> 6)) * 64 + r), src + r, 4);
  };

  float accK[D / 8][4], accV[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      accK[n][x] = 0.f;
      accV[n][x] = 0.f;
    }

  for (int base = 0; base < N; base += kBwdListChunk) {
    // ---- ordered list of the query blocks of this chunk that use the tile ----
    unsigned m = 0;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int i = base + tid * 8 + r;
      if (i < N && unselected(i) != 0ull) m |= 1u << r;
    }
    const int c = __popc(m);
    int x = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    int off = x - c;
    for (int w = 0; w < warp; ++w) off += wsum[w];
    const int cnt = wsum[0] + wsum[1] + wsum[2] + wsum[3];
#pragma unroll
    for (int r = 0; r < 8; ++r)
      if ((m >> r) & 1u) list[off++] = base + tid * 8 + r;
    __syncthreads();
    if (cnt == 0) continue;

    issue(list[0], 0);
    cp_async_commit();
    for (int e = 0; e < cnt; ++e) {
      const int st = e & 1;
      if (e + 1 < cnt) issue(list[e + 1], st ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
      __syncthreads();
      const int i = list[e];
      const uint32_t sQ = sb + (2 + 2 * st) * kT, sdO = sQ + kT;
      const float *ls = vec + (st * 2) * 64, *dl = vec + (st * 2 + 1) * 64;
      const uint64_t use = unselected(i);
      const float wA = ((use >> kA) & 1ull) ? fixA : 0.f;
      const float wB = ((use >> kB) & 1ull) ? fixB : 0.f;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float s[4][4], dp[4][4];
        bwd_gemm_abt<D, 4>(s, sK, warp * 16, sQ, 32 * h, lane);
        bwd_gemm_abt<D, 4>(dp, sV, warp * 16, sdO, 32 * h, lane);
#pragma unroll
        for (int n = 0; n < 4; ++n)
#pragma unroll
          for (int xx = 0; xx < 4; ++xx) {
            const int col = 32 * h + n * 8 + 2 * tq + (xx & 1);   // query row in block i
            const float w = xx >= 2 ? wB : wA;
            // padded query rows carry lse = +inf, so their probability is 0
            const float p =
                w != 0.f ? w * sm100::ex2_approx(fmaf(s[n][xx], sl2, -ls[col] * kLog2e)) : 0.f;
            s[n][xx] = p * (dp[n][xx] - dl[col]);   // dz
            dp[n][xx] = p;
          }
        uint32_t ap[2][4], az[2][4];
        bwd_c_to_a<2>(dp, ap);
        bwd_c_to_a<2>(s, az);
        bwd_gemm_ab<D, 2>(accV, ap, sdO, 32 * h, lane);
        bwd_gemm_ab<D, 2>(accK, az, sQ, 32 * h, lane);
      }
      __syncthreads();
    }
  }
  cp_async_commit();
  cp_async_wait<0>();

  // ---- epilogue: dkbar_j / n_j and dvbar_j / n_j (float32) -------------------
#pragma unroll
  for (int hrow = 0; hrow < 2; ++hrow) {
    const int j = 64 * jb + (hrow ? kB : kA);
    if (j >= N) continue;
    const float inv_n = 1.f / (j == N - 1 ? (float)n_last : 64.f);
    float *pk = dkbar + ((size_t)bh * Npad + j) * D;
    float *pv = dvbar + ((size_t)bh * Npad + j) * D;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      const int col = n * 8 + 2 * tq;
      *reinterpret_cast<float2 *>(pk + col) =
          make_float2(scale * accK[n][2 * hrow] * inv_n, scale * accK[n][2 * hrow + 1] * inv_n);
      *reinterpret_cast<float2 *>(pv + col) =
          make_float2(accV[n][2 * hrow] * inv_n, accV[n][2 * hrow + 1] * inv_n);
    }
  }
}

}  // namespace pisa
