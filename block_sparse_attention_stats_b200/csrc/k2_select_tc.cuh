// K2, certified path for long rows (512 < N <= 2048 blocks).
//
// "Technical Summary: PISA" (gist.science), section 2 "Covariance-Aware
// Routing" defines the score s qbar_i . kbar_j + lambda M_j and the per-query-
// block top-k; the authors' README, "Attention sink for MMDiT", the forced sink.
// The selected set is, exactly, the top k_sel of the float32 scores that
// scores_kernel computes (head dimension summed in ascending order with fmaf,
// then fmaf(scale, acc, lambda M_j)), ties to the lower block index -- the same
// set as the two-pass path -- but most of those float32 dot products are never
// formed:
//
//  1. select_pack_kernel: every float32 value x of qbar and kbar split into
//     two bf16 terms x_hi = bf16(x), x_lo = bf16(x - x_hi), laid out for the
//     tensor memory accelerator, and the Euclidean norm of every row.
//  2. select_approx_tc_kernel: approximate scores A_ij = fmaf(s, acc, lambda
//     M_j), acc = q_hi.k_hi + q_hi.k_lo + q_lo.k_hi summed over the head
//     dimension by tcgen05 (M = 128, N = 128 tiles; every bf16 product is
//     exact in float32, the sums accumulate in tensor memory).
//  3. select_certified_kernel (one warp per query block): with the float32
//     score F_ij, |F_ij - A_ij| <= E_ij where
//       E_ij = s |qbar_i| |kbar_j| c + 2^-21 |A_ij|
//     (c: see kCertBound; the last term covers the final fmaf roundings).
//     Let T_A be the need-th largest A_ij of the row (need = k_sel, minus one
//     with a sink) and E_max the largest E_ij: the need-th largest F, T_F,
//     lies within E_max of T_A.  A block with A - E > T_A + E_max is certainly
//     selected, one with A + E < T_A - E_max certainly not; only the blocks in
//     between get their float32 score, and the best of them (ties to the
//     lower index) fill the remaining places.  T_A itself is only needed to
//     within a known width, so its radix select stops after the leading 24
//     bits of the order-preserving key and the band is widened by that width.
// Every step is deterministic; the result does not depend on the data beyond
// the float32 scores (a row whose scores are all close only costs more
// exact dot products).
#pragma once

#include "k2_select.cuh"
#include "pisa_common.cuh"
#include "sm100_primitives.cuh"

namespace pisa {

constexpr int kCertMaxN = 2048;     // 64 scores per lane
constexpr int kCertTile = 128;      // approximate-score tile (rows and columns)

// Two-term bf16 split of qbar and kbar, [2][BH][Npad][D] each (the high terms,
// then the low terms; rows >= N zero), and float32 norms [BH, N]; one warp per
// row of either tensor.
template <int D>
__global__ void __launch_bounds__(256)
    select_pack_kernel(const float *__restrict__ qbar, const float *__restrict__ kbar, int N,
                       int Npad, int BH, __nv_bfloat16 *__restrict__ qbar16,
                       __nv_bfloat16 *__restrict__ kbar16, float *__restrict__ qn,
                       float *__restrict__ kn) {
  constexpr int kPer = D / 32;   // elements per lane (4 or 2)
  const int lane = threadIdx.x & 31;
  const size_t rows = (size_t)2 * BH * Npad;
  for (size_t w = (blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5; w < rows;
       w += ((size_t)gridDim.x * blockDim.x) >> 5) {
    const int which = (int)(w / ((size_t)BH * Npad));           // 0: qbar, 1: kbar
    const size_t r = w % ((size_t)BH * Npad);
    const int bh = (int)(r / Npad), j = (int)(r % Npad);
    const float *src = (which ? kbar : qbar) + ((size_t)bh * N + j) * D + lane * kPer;
    float x[kPer];
#pragma unroll
    for (int e = 0; e < kPer; ++e) x[e] = 0.f;
    if (j < N) {
      if (kPer == 4) {
        const float4 v = *reinterpret_cast<const float4 *>(src);
        x[0] = v.x; x[1] = v.y; x[2 % kPer] = v.z; x[3 % kPer] = v.w;
      } else {
        const float2 v = *reinterpret_cast<const float2 *>(src);
        x[0] = v.x; x[1 % kPer] = v.y;
      }
    }
    __nv_bfloat16 *dst = (which ? kbar16 : qbar16) + r * D + lane * kPer;
    const size_t lo_off = (size_t)BH * Npad * D;
    float hi[kPer], lo[kPer];
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      hi[e] = __bfloat162float(__float2bfloat16_rn(x[e]));
      lo[e] = x[e] - hi[e];   // exact in float32
    }
    if (kPer == 4) {
      *reinterpret_cast<uint2 *>(dst) =
          make_uint2(pack_bf16x2(hi[0], hi[1 % kPer]), pack_bf16x2(hi[2 % kPer], hi[3 % kPer]));
      *reinterpret_cast<uint2 *>(dst + lo_off) =
          make_uint2(pack_bf16x2(lo[0], lo[1 % kPer]), pack_bf16x2(lo[2 % kPer], lo[3 % kPer]));
    } else {
      *reinterpret_cast<uint32_t *>(dst) = pack_bf16x2(hi[0], hi[1 % kPer]);
      *reinterpret_cast<uint32_t *>(dst + lo_off) = pack_bf16x2(lo[0], lo[1 % kPer]);
    }
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < kPer; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (j < N && lane == 0) (which ? kn : qn)[(size_t)bh * N + j] = sqrtf(ss);
  }
}

// Approximate scores of one 128-row tile of query blocks against every key
// block of its head: tcgen05 M = 128, N = 128 tiles over K = D, two TMEM
// accumulators so that the epilogue of one key tile overlaps the products of
// the next.  Output rows [BH][N][ldS] (ldS = Npad), columns >= N not written.
// Roles (160 threads): warps 0-3 epilogue (thread = TMEM lane = row), warp 4
// TMEM allocation and one lane issuing every copy and MMA.
template <int D> struct SelTcCfg {
  static constexpr int kThreads = 160;
  static constexpr int kBoxBytes = kCertTile * 128;        // 128 rows x 64 bf16
  static constexpr int kTileBytes = 2 * kCertTile * D * 2; // high and low terms
  static constexpr int kTermBytes = kCertTile * D * 2;
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kTileBytes;                  // two slots
  // per epilogue warp a 32 x 32 block of scores, rows padded to 33 floats, so
  // that the warp stores whole 128-byte row segments
  static constexpr int kOffT = kOffB + 2 * kTileBytes;
  static constexpr int kOffBar = kOffT + 4 * 32 * 33 * 4;
  static constexpr int kOffTmemSlot = kOffBar + 16 * 8;
  static constexpr int kOffMisc = kOffTmemSlot + 16;
  static constexpr int kSmem = kOffMisc + 16 + 1024;         // + alignment slack
  static constexpr uint32_t kTmemCols = 256;
  static constexpr int kBarA = 0, kBarBFull = 1, kBarBEmpty = 3, kBarSFull = 5, kBarSEmpty = 7,
                       kBarTeardown = 9;
};

template <int D>
__global__ void __launch_bounds__(160, 1)
    select_approx_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                            const __grid_constant__ CUtensorMap tm_k,
                            const float *__restrict__ cov, float cov_weight, float scale, int N,
                            int Npad, int BH, float *__restrict__ approx) {
  using C = SelTcCfg<D>;
  using namespace sm100;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  unsigned char *smem = smem_raw + (sbase - raw);
  auto bar = [&](int i) -> uint32_t { return sbase + C::kOffBar + 8 * i; };
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kOffMisc);
  const int tid = threadIdx.x, lane = tid & 31;
  const int warp = __shfl_sync(0xffffffffu, tid >> 5, 0);
  const int i0 = blockIdx.x * kCertTile, bh = blockIdx.y;
  const int nt = Npad / kCertTile;

  if (warp == 4) {
    tmem_alloc(sbase + C::kOffTmemSlot, C::kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int b = 0; b < 10; ++b) mbar_init(bar(b), (b == C::kBarSEmpty || b == C::kBarSEmpty + 1) ? 128 : 1);
    fence_mbar_init();
    *abort_flag = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + C::kOffTmemSlot);

  if (warp == 4) {
    if (lane == 0) {
      constexpr uint32_t kId = idesc_bf16_f32(128, 128, 0, 0);
      auto load_b = [&](int c) {
        const int sl = c & 1;
        mbar_expect_tx(bar(C::kBarBFull + sl), C::kTileBytes);
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int b = 0; b < D / 64; ++b)
            tma_load_3d(sbase + C::kOffB + sl * C::kTileBytes + h * C::kTermBytes + b * C::kBoxBytes,
                        &tm_k, bar(C::kBarBFull + sl), 64 * b, c * kCertTile, bh + h * BH);
      };
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      mbar_expect_tx(bar(C::kBarA), C::kTileBytes);
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int b = 0; b < D / 64; ++b)
          tma_load_3d(sbase + C::kOffA + h * C::kTermBytes + b * C::kBoxBytes, &tm_q, bar(C::kBarA),
                      64 * b, i0, bh + h * BH);
      int issued = 0;      // key tiles whose copy was issued
      int mma_done = 0;    // key tiles whose MMAs were issued
      load_b(0);
      issued = 1;
      if (nt > 1) { load_b(1); issued = 2; }
      bool ok = mbar_wait(bar(C::kBarA), 0);
      for (int c = 0; ok && c < nt; ++c) {
        const int sl = c & 1;
        if (!mbar_wait(bar(C::kBarBFull + sl), (c >> 1) & 1)) { ok = false; break; }
        if (c >= 2 && !mbar_wait(bar(C::kBarSEmpty + sl), ((c >> 1) - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        // q_hi.k_hi, q_hi.k_lo, q_lo.k_hi (q_lo.k_lo is below the bound's terms)
#pragma unroll
        for (int p = 0; p < 3; ++p) {
          const uint32_t ta = (p == 2 ? C::kTermBytes : 0), tb = (p == 1 ? C::kTermBytes : 0);
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off = (k >> 2) * C::kBoxBytes + (k & 3) * 32;
            mma_ss(tmem + 128 * sl, smem_desc_sw128(sbase + C::kOffA + ta + off, 16, 1024),
                   smem_desc_sw128(sbase + C::kOffB + sl * C::kTileBytes + tb + off, 16, 1024),
                   kId, (p > 0 || k > 0) ? 1u : 0u);
          }
        }
        tc_commit(bar(C::kBarSFull + sl));
        tc_commit(bar(C::kBarBEmpty + sl));
        mma_done = c + 1;
        if (c + 2 < nt) {
          if (!mbar_wait(bar(C::kBarBEmpty + sl), (c >> 1) & 1)) { ok = false; break; }
          load_b(c + 2);
          issued = c + 3;
        }
      }
      if (!ok) {
        *abort_flag = 1;
        // copies in flight land before the CTA exits; issued MMAs finish before
        // TMEM is released
        mbar_wait(bar(C::kBarA), 0);
        for (int c = mma_done; c < issued; ++c) mbar_wait(bar(C::kBarBFull + (c & 1)), (c >> 1) & 1);
        tc_commit(bar(C::kBarTeardown));
        mbar_wait(bar(C::kBarTeardown), 0);
      }
    }
    __syncwarp();
  } else {
    // epilogue: thread = row of the tile = TMEM lane.  Each 32-column chunk
    // goes through shared memory so that the warp writes 128-byte row segments.
    const int gi0 = i0 + warp * 32;
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    float *tb = reinterpret_cast<float *>(smem + C::kOffT) + warp * 32 * 33;
    for (int c = 0; c < nt; ++c) {
      const int sl = c & 1;
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(C::kBarSFull + sl), (c >> 1) & 1))) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        uint32_t r[32];
        tmem_ld_x32(lane_addr + 128 * sl + 32 * q, r);
        tmem_wait_ld();
        if (q == 3) {
          // the accumulator may take the next key tile
          tc_fence_before();
          mbar_arrive(bar(C::kBarSEmpty + sl));
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) tb[lane * 33 + e] = __uint_as_float(r[e]);
        __syncwarp();
        const int j = c * kCertTile + 32 * q + lane;
        const float cw = (cov_weight != 0.f && j < N) ? cov_weight * __ldg(cov + (size_t)bh * N + j) : 0.f;
#pragma unroll 4
        for (int rr = 0; rr < 32; ++rr) {
          if (gi0 + rr < N)
            approx[((size_t)bh * N + gi0 + rr) * Npad + j] = fmaf(scale, tb[rr * 33 + lane], cw);
        }
        __syncwarp();
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// Inverse of float_key.
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Radix select over a warp's keys in shared memory (key of column j at
// keys[j]; lane l examines the columns 32 u + l).  Finds the need-th largest
// key among the columns whose bit u is set in the lane's mask `cand`,
// examining the leading `bits` bits (multiple of 8) of the key.  Returns the
// selected key prefix (remaining bits zero) and, in rem_out, how many of the
// keys with that prefix rank within the first `need`.  Requires
// 1 <= need <= number of candidates.
__device__ __forceinline__ uint32_t warp_radix_select(const uint32_t *keys, uint64_t cand, int nv,
                                                      int need, int bits, unsigned *hist,
                                                      int lane, int &rem_out) {
  uint32_t prefix = 0u, mask = 0u;
  int rem = need;
  for (int pass = 0; pass < bits / 8; ++pass) {
    const int shift = 24 - 8 * pass;
#pragma unroll
    for (int q = 0; q < 8; ++q) hist[lane * 8 + q] = 0u;
    __syncwarp();
    for (int u = 0; u < nv; ++u) {
      const uint32_t key = keys[32 * u + lane];
      const bool part = ((cand >> u) & 1ull) && (key & mask) == prefix;
      const unsigned act = __ballot_sync(0xffffffffu, part);
      if (part) {
        const unsigned digit = (key >> shift) & 255u;
        const unsigned peers = __match_any_sync(act, digit);
        if (lane == __ffs(peers) - 1) atomicAdd(&hist[digit], (unsigned)__popc(peers));
      }
    }
    __syncwarp();
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
    const int src = who ? __ffs(who) - 1 : 0;
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
  rem_out = rem;
  return prefix;
}

// Bound constant c of E_ij.  Per product term, with x = x_hi + x_lo + e_x and
// |e_x| <= 2^-18 |x| (two bf16 terms of 8 bits each),
//   |q k - (q_hi k_hi + q_hi k_lo + q_lo k_hi)| <= 3.01 2^-18 |q k| < 1.2e-5 |q k|;
// the tensor-core sum of the 3 D exact products into float32, allowing every
// addition an error of 2^-22 of the running magnitude (four times the unit of
// a truncating accumulator): (3 D) 2^-22 1.004 sum|q k| <= 9.2e-5 sum|q k| at
// D = 128; the fixed-order fmaf sum of the float32 score: D 2^-24 = 7.6e-6 of
// sum|q k|; sum_e |q_e k_e| <= |qbar_i| |kbar_j| (Cauchy-Schwarz), the norms
// rounded to within 1e-6: 1.12e-4 in all, rounded up.
constexpr float kCertBound = 1.5e-4f;
constexpr float kCertRel = 4.76837158e-7f;   // 2^-21

constexpr int kCertWarps = 4;

// shared memory of select_certified_kernel: per warp the N keys of its row
// (rounded up to 32), a 256-bin histogram and its qbar row
__host__ __device__ inline int certified_smem(int N, int D) {
  return kCertWarps * (((N + 31) / 32) * 32 * 4 + 256 * 4 + D * 4);
}

template <int D>
__global__ void __launch_bounds__(kCertWarps * 32)
    select_certified_kernel(const float *__restrict__ approx, int ldS,
                            const float *__restrict__ qbar, const float *__restrict__ kbar,
                            const float *__restrict__ qn, const float *__restrict__ kn,
                            const float *__restrict__ cov, float cov_weight, float scale, int N,
                            int k_sel, int sink, size_t rows, int32_t *__restrict__ idx) {
  extern __shared__ __align__(16) unsigned char cert_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nv = (N + 31) / 32;
  unsigned char *mine = cert_smem + (size_t)warp * (nv * 32 * 4 + 256 * 4 + D * 4);
  uint32_t *keys = reinterpret_cast<uint32_t *>(mine);
  unsigned *hist = reinterpret_cast<unsigned *>(mine + nv * 32 * 4);
  float *qrow = reinterpret_cast<float *>(mine + nv * 32 * 4 + 256 * 4);
  const size_t row = (size_t)blockIdx.x * kCertWarps + warp;
  if (row >= rows) return;
  const int bh = (int)(row / N);
  int32_t *out = idx + row * k_sel;
  const int need = k_sel - (sink >= 0 ? 1 : 0);
  const int candidates = N - (sink >= 0 ? 1 : 0);

  // candidates of this lane: columns 32 u + lane < N, the sink excluded (at
  // most 64 per lane: N <= 2048)
  uint64_t cand = 0ull;
  for (int u = 0; u < nv; ++u) {
    const int j = 32 * u + lane;
    if (j < N && j != sink) cand |= 1ull << u;
  }
  uint64_t chosen = 0ull;   // bit u: column 32 u + lane is selected (sink aside)
  if (need >= candidates) {
    chosen = cand;
  } else if (need > 0) {
    for (int e = lane; e < D; e += 32) qrow[e] = qbar[row * D + e];
    const float s_abs = fabsf(scale);
    const float qnorm = qn[row];
    const float *knr = kn + (size_t)bh * N;
    // keys of the approximate scores (key_float recovers each score exactly)
    float emax = 0.f;
    for (int u = 0; u < nv; ++u) {
      const int j = 32 * u + lane;
      uint32_t key = 0u;
      if ((cand >> u) & 1ull) {
        const float a = approx[row * (size_t)ldS + j];
        key = float_key(a);
        emax = fmaxf(emax, s_abs * kCertBound * qnorm * knr[j] + kCertRel * fabsf(a));
      }
      keys[j] = key;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) emax = fmaxf(emax, __shfl_xor_sync(0xffffffffu, emax, o));
    __syncwarp();
    // T_A to its leading 24 key bits: T_A lies in [t_lo, t_hi]
    int rem24;
    const uint32_t p24 = warp_radix_select(keys, cand, nv, need, 24, hist, lane, rem24);
    const float t_lo = key_float(p24), t_hi = key_float(p24 | 0xffu);
    const float band_hi = t_hi + emax, band_lo = t_lo - emax;
    // classify; the float32 score of every undecided column, in the same fixed
    // order as scores_kernel
    uint64_t in = 0ull, und = 0ull;
    for (int u = 0; u < nv; ++u) {
      if (!((cand >> u) & 1ull)) continue;
      const int j = 32 * u + lane;
      const float a = key_float(keys[j]);
      const float e = s_abs * kCertBound * qnorm * knr[j] + kCertRel * fabsf(a);
      if (a - e > band_hi) {
        in |= 1ull << u;
      } else if (!(a + e < band_lo)) {
        const float4 *kr = reinterpret_cast<const float4 *>(kbar + ((size_t)bh * N + j) * D);
        float acc = 0.f;
#pragma unroll 8
        for (int e4 = 0; e4 < D / 4; ++e4) {
          const float4 kv = __ldg(kr + e4);
          acc = fmaf(qrow[4 * e4 + 0], kv.x, acc);
          acc = fmaf(qrow[4 * e4 + 1], kv.y, acc);
          acc = fmaf(qrow[4 * e4 + 2], kv.z, acc);
          acc = fmaf(qrow[4 * e4 + 3], kv.w, acc);
        }
        const float cw = cov_weight != 0.f ? cov_weight * cov[(size_t)bh * N + j] : 0.f;
        keys[j] = float_key(fmaf(scale, acc, cw));
        und |= 1ull << u;
      }
    }
    int n_in = __popcll(in), n_und = __popcll(und);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      n_in += __shfl_xor_sync(0xffffffffu, n_in, o);
      n_und += __shfl_xor_sync(0xffffffffu, n_und, o);
    }
    const int r = need - n_in;   // places left for the undecided columns
    __syncwarp();
    if (r <= 0 || n_und == 0) {
      // the bound decided every place (r == 0 is guaranteed by it)
      if (r != 0 && lane == 0) report_device_error(kDevErrRange);
      chosen = in;
    } else if (n_und <= 32) {
      // few undecided columns: gather them (ascending column) into lanes and
      // rank each against the others: higher score first, then lower column
      uint32_t *ukey = hist, *ucol = hist + 32;
      int base = 0;
      for (int u = 0; u < nv; ++u) {
        const bool x = (und >> u) & 1ull;
        const unsigned bal = __ballot_sync(0xffffffffu, x);
        if (x) {
          const int pos = base + __popc(bal & ((1u << lane) - 1u));
          ukey[pos] = keys[32 * u + lane];
          ucol[pos] = 32 * u + lane;
        }
        base += __popc(bal);
      }
      __syncwarp();
      const uint32_t mk = lane < n_und ? ukey[lane] : 0u;
      const int mj = lane < n_und ? (int)ucol[lane] : 0x7fffffff;
      int rank = 0;
      for (int m = 0; m < n_und; ++m) {
        const uint32_t ok = __shfl_sync(0xffffffffu, mk, m);
        const int oj = __shfl_sync(0xffffffffu, mj, m);
        rank += (ok > mk || (ok == mk && oj < mj)) ? 1 : 0;
      }
      __syncwarp();
      if (lane < n_und) keys[mj] = rank < r ? 0xffffffffu : 0u;
      __syncwarp();
      chosen = in;
      for (int u = 0; u < nv; ++u)
        if (((und >> u) & 1ull) && keys[32 * u + lane] == 0xffffffffu) chosen |= 1ull << u;
    } else {
      // many undecided columns: radix select over the final keys, the
      // certainly selected ones above every finite score
      for (int u = 0; u < nv; ++u)
        if ((in >> u) & 1ull) keys[32 * u + lane] = 0xffffffffu;
      __syncwarp();
      const uint64_t live = in | und;
      int rem;
      const uint32_t T = warp_radix_select(keys, live, nv, need, 32, hist, lane, rem);
      int eq_base = 0;
      for (int u = 0; u < nv; ++u) {
        const bool lv = (live >> u) & 1ull;
        const uint32_t key = keys[32 * u + lane];
        const bool is_eq = lv && key == T;
        const unsigned eq_bal = __ballot_sync(0xffffffffu, is_eq);
        const int eq_rank = eq_base + __popc(eq_bal & ((1u << lane) - 1u));
        if (lv && (key > T || (is_eq && eq_rank < rem))) chosen |= 1ull << u;
        eq_base += __popc(eq_bal);
      }
    }
  }
  // ascending output: the sink and the chosen columns
  int base = 0;
  for (int u = 0; u < nv; ++u) {
    const int j = 32 * u + lane;
    const bool sel = (j == sink && j < N) || ((chosen >> u) & 1ull);
    const unsigned bal = __ballot_sync(0xffffffffu, sel);
    const int pos = base + __popc(bal & ((1u << lane) - 1u));
    if (sel) {
      if (pos < k_sel) out[pos] = j;
      else report_device_error(kDevErrRange);
    }
    base += __popc(bal);
  }
  if (lane == 0 && base != k_sel) report_device_error(kDevErrRange);
}

}  // namespace pisa
