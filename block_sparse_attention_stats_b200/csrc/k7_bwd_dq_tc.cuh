// dq of the zeroth-order backward on the sm_100a tensor cores (tcgen05).
//
// Same work unit as the fused forward: one CTA = two paired query blocks
// (128 query rows, M = 128 MMAs) over the union of their exact tiles, then the
// 64-centroid chunks masked per half to the half's unselected blocks.  With
// P_tm = w_m exp(s q_t.key_m - lse_t) (w = 1 for exact keys, n_j for
// centroids), dP_tm = dout_t . value_m and Delta_t = sum_m P_tm dP_tm:
//   dq_t = s sum_m P_tm (dP_tm - Delta_t) key_m
// Delta_t is either given (formed from the forward's float32 output, see
// bwd_delta_kernel) and the kernel makes one sweep over the tile list, or the
// kernel makes two sweeps: the first forms Delta_t from its own P and dP (so
// that sum_m dz_tm vanishes to f32 rounding), the second accumulates dq in
// tensor memory.
//
// Roles (352 threads):
//   warp 0      TMA producer: Q and dout once, then K and V (or kbar and vbar)
//               of every tile of every sweep into 3-stage rings;
//   warp 1      TMEM allocation; issues S_u = Q K^T into TMEM buffer u & 1;
//   warp 10     issues dP_u = dout V^T into the same buffer and, in the dq
//               sweep (the only one when Delta is given), dQ += dS_u K_u with
//               dS read from TMEM (one warp's issue rate would otherwise bound
//               the kernel);
//   warps 2-9   two warpgroups of 4 warps; warpgroup g takes the tiles with
//               u & 1 == g (buffer g), one thread per query row (TMEM lane):
//               P and dP from TMEM, Delta partial sums (Delta sweep) or dS
//               written as bf16 over the dP columns it was formed from (dq
//               sweep); the two Delta partials are combined through shared
//               memory between sweeps (with Delta given, each thread reads its
//               row's value); the epilogue scales dQ by s and stores it (half
//               the columns each).  Before the loop warpgroup 0 copies Q and
//               warpgroup 1 copies dout into tensor memory.
// TMEM columns: dQ [0, D); buffer b: S [D + 128 b, D + 128 b + 64), dP the next
// 64 (dS, packed bf16, over its first 32); dout [D + 256, D + 256 + D / 2) and
// Q [D + 320, D + 320 + D / 2) as packed bf16 pairs, the A operands of the dP
// and S products.  dP_u + 2 rewrites the dS of tile u only after dQ_u has read
// it: warp 10 issues both, in that order, and one thread's tcgen05 products
// run in issue order; the commit that signals dP_u also covers dQ_u - 2.
// Every mbarrier wait is bounded; on a timeout the CTA records the error,
// stops issuing, drains its copies and MMAs, frees TMEM and exits.
#pragma once

#include "pisa_common.cuh"
#include "sm100_primitives.cuh"

namespace pisa {

template <int D> struct DqTcCfg {
  static constexpr int kThreads = 352;
  static constexpr int kStages = 3;
  static constexpr int kQBytes = 128 * D * 2;
  static constexpr int kBoxQBytes = 128 * 128;     // one 64-column box of 128 rows
  static constexpr int kBoxKBytes = 64 * 128;      // one 64-column box of 64 rows
  static constexpr int kTileBytes = 64 * D * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffDO = kQBytes;
  static constexpr int kOffK = 2 * kQBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kStages * kTileBytes;
  static constexpr int kNumBars = 24;
  static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
  static constexpr int kOffMisc = kOffTmemSlot + 16;
  static constexpr int kOffDelta = kOffMisc + 16;               // [2][128] f32
  static constexpr int kOffDyn = kOffDelta + 2 * 128 * 4;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColDQ = 0;
  static constexpr uint32_t kColBuf = D;                        // + 128 b
  // dout and Q as packed bf16 pairs (D / 2 columns each), the A operands of
  // the dP and S products: read from tensor memory, an N = 64 product needs
  // only its 2 KB of V or K tile from shared memory instead of 6 KB, which
  // bounds it at ~52 pipe cycles
  static constexpr uint32_t kColDO = D + 256;
  static constexpr uint32_t kColQ = D + 320;
  static constexpr int kBarQ = 0;
  static constexpr int kBarKFull = 1;                           // + slot
  static constexpr int kBarKEmpty = kBarKFull + kStages;
  static constexpr int kBarVFull = kBarKEmpty + kStages;
  static constexpr int kBarVEmpty = kBarVFull + kStages;
  static constexpr int kBarSFull = kBarVEmpty + kStages;        // + buffer
  static constexpr int kBarPFull = kBarSFull + 2;               // + buffer
  static constexpr int kBarDelta = kBarPFull + 2;
  static constexpr int kBarFinal = kBarDelta + 1;
  static constexpr int kBarTeardown = kBarFinal + 1;
  static constexpr int kBarQT = kBarTeardown + 1;                // Q copied into TMEM
  static constexpr int kBarDOT = kBarQT + 1;                     // dout copied into TMEM
  static_assert(kBarDOT < kNumBars, "barrier slots");
  static_assert(kColDO + D / 2 <= kColQ, "tensor memory columns");
  static_assert(kColQ + D / 2 <= kTmemCols, "tensor memory columns");

  // N 64-token tiles, Nc blocks (= centroids)
  __host__ __device__ static int smem_bytes(int N, int Nc) {
    const int nwords = (N + 31) / 32, cwords = (Nc + 31) / 32;
    return kOffDyn + (2 * nwords + 2 * cwords + N + (Nc + 63) / 64) * 4 + 1024;   // + slack
  }
};

__device__ __forceinline__ uint32_t dq_valid_bits(int w, int N) {
  const int lo = w * 32;
  if (lo + 32 <= N) return 0xffffffffu;
  if (lo >= N) return 0u;
  return (1u << (N - lo)) - 1u;
}

template <int D>
__global__ void __launch_bounds__(352, 1)
    bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_do,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_kbar,
                     const __grid_constant__ CUtensorMap tm_vbar,
                     const int32_t *__restrict__ idx, const int2 *__restrict__ pairs, int k_sel,
                     int L, int N, int bsub, int Nc, float scale, const float *__restrict__ lse,
                     float *__restrict__ delta, int delta_given, int Lpad,
                     __nv_bfloat16 *__restrict__ dq) {
  using C = DqTcCfg<D>;
  using namespace sm100;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  unsigned char *smem = smem_raw + (sbase - raw);
  auto bar = [&](int i) -> uint32_t { return sbase + C::kOffBar + 8 * i; };
  volatile int *misc = reinterpret_cast<volatile int *>(smem + C::kOffMisc);  // [0] tiles, [1] abort
  float *delta_sm = reinterpret_cast<float *>(smem + C::kOffDelta);
  // bm_*: selected 64-token tiles per half; cbm_*: selected blocks (the
  // centroid index space) per half.  With 64-token blocks the two coincide;
  // with 128-token blocks both halves are one query block and share them.
  const int nwords = (N + 31) / 32, cwords = (Nc + 31) / 32;
  uint32_t *bm_lo = reinterpret_cast<uint32_t *>(smem + C::kOffDyn);
  uint32_t *bm_hi = bsub == 1 ? bm_lo + nwords : bm_lo;
  uint32_t *cbm_lo = bsub == 1 ? bm_lo : bm_lo + 2 * nwords;
  uint32_t *cbm_hi = bsub == 1 ? bm_hi : cbm_lo;
  int *tiles = reinterpret_cast<int *>(bm_lo + 2 * nwords + 2 * cwords);

  const int pair = blockIdx.x, bh = blockIdx.y;
  int qb0 = 2 * pair, qb1 = 2 * pair + 1 < N ? 2 * pair + 1 : -1;
  int sr0 = qb0, sr1 = qb1;                     // selection rows of the halves
  if (bsub == 2) {
    sr0 = pair;
    sr1 = pair;
  } else if (pairs) {
    const int2 pr = pairs[(size_t)bh * ((N + 1) / 2) + pair];
    qb0 = pr.x;
    qb1 = pr.y;
    sr0 = qb0;
    sr1 = qb1;
  }
  const bool has_hi = qb1 >= 0;
  const int tid = threadIdx.x, lane = tid & 31;
  const int warp = __shfl_sync(0xffffffffu, tid >> 5, 0);

  // ---- set-up ---------------------------------------------------------------
  if (warp == 1) {
    tmem_alloc(sbase + C::kOffTmemSlot, C::kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar(C::kBarQ), 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar(C::kBarKFull + s), 1);
      mbar_init(bar(C::kBarKEmpty + s), 1);
      mbar_init(bar(C::kBarVFull + s), 1);
      mbar_init(bar(C::kBarVEmpty + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(C::kBarSFull + b), 2);       // S from warp 1, dP from warp 10
      mbar_init(bar(C::kBarPFull + b), 128);
    }
    mbar_init(bar(C::kBarDelta), 256);
    mbar_init(bar(C::kBarFinal), 1);
    mbar_init(bar(C::kBarTeardown), 2);
    mbar_init(bar(C::kBarQT), 4);
    mbar_init(bar(C::kBarDOT), 4);
    fence_mbar_init();
    misc[1] = 0;
  }
  if (tid == 32) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_do);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_kbar);
    prefetch_tmap(&tm_vbar);
  }
  for (int w = tid; w < 2 * nwords + 2 * cwords; w += C::kThreads) bm_lo[w] = 0u;
  __syncthreads();
  if (bsub == 1) {
    const int32_t *r0 = idx + ((size_t)bh * Nc + sr0) * k_sel;
    const int32_t *r1 = idx + ((size_t)bh * Nc + (has_hi ? sr1 : sr0)) * k_sel;
    for (int t = tid; t < (has_hi ? 2 : 1) * k_sel; t += C::kThreads) {
      const int j = t < k_sel ? r0[t] : r1[t - k_sel];
      uint32_t *bm = t < k_sel ? bm_lo : bm_hi;
      if (j >= 0 && j < N) atomicOr(&bm[j >> 5], 1u << (j & 31));
      else report_device_error(kDevErrRange);
    }
  } else {
    // one selection row: block j covers the 64-token tiles 2j and 2j + 1
    const int32_t *r0 = idx + ((size_t)bh * Nc + sr0) * k_sel;
    for (int t = tid; t < k_sel; t += C::kThreads) {
      const int j = r0[t];
      if (j >= 0 && j < Nc) {
        atomicOr(&cbm_lo[j >> 5], 1u << (j & 31));
        for (int u = bsub * j; u < bsub * j + bsub && u < N; ++u)
          atomicOr(&bm_lo[u >> 5], 1u << (u & 31));
      } else {
        report_device_error(kDevErrRange);
      }
    }
  }
  __syncthreads();
  if (warp == 0) {
    // exact tiles: ascending union of both halves' sets, with per-half flags
    int base = 0;
    for (int w0 = 0; w0 < nwords; w0 += 32) {
      const int w = w0 + lane;
      const uint32_t lo = w < nwords ? bm_lo[w] : 0u, hi = w < nwords ? bm_hi[w] : 0u;
      uint32_t u = lo | hi;
      const int cnt = __popc(u);
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      int pos = base + incl - cnt;
      while (u) {
        const int bit = __ffs(u) - 1;
        u &= u - 1u;
        tiles[pos++] = ((w * 32 + bit) << 2) | ((lo >> bit) & 1u) | (((hi >> bit) & 1u) << 1);
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    // centroid chunks that hold an unselected block for either half
    const int nch = (Nc + 63) / 64;
    for (int c0 = 0; c0 < nch; c0 += 32) {
      const int c = c0 + lane;
      bool need = false;
      if (c < nch) {
        for (int h = 0; h < (has_hi ? 2 : 1); ++h) {
          const uint32_t *cb = h ? cbm_hi : cbm_lo;
          const uint32_t m0 = ~cb[2 * c] & dq_valid_bits(2 * c, Nc);
          const uint32_t m1 = (2 * c + 1 < cwords) ? (~cb[2 * c + 1] & dq_valid_bits(2 * c + 1, Nc)) : 0u;
          need = need || ((m0 | m1) != 0u);
        }
      }
      const unsigned bal = __ballot_sync(0xffffffffu, need);
      if (need) tiles[base + __popc(bal & ((1u << lane) - 1u))] = -(c + 1);
      base += __popc(bal);
    }
    if (lane == 0) misc[0] = base;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + C::kOffTmemSlot);
  const int T = misc[0];
  const int T1 = delta_given ? 0 : T;  // tiles of the Delta sweep
  const int U = T1 + T;

  auto uwait = [&](uint32_t b_addr, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, mbar_wait(b_addr, parity));
  };
  auto aborted = [&]() -> bool { return __any_sync(0xffffffffu, misc[1] != 0); };

  if (warp == 0) {
    // ======================= TMA producer =====================================
    if (elect_one()) {
      mbar_expect_tx(bar(C::kBarQ), 2 * C::kQBytes);
#pragma unroll
      for (int b = 0; b < D / 64; ++b) {
        const uint32_t dq_ = sbase + C::kOffQ + b * C::kBoxQBytes;
        const uint32_t dd_ = sbase + C::kOffDO + b * C::kBoxQBytes;
        tma_load_3d(dq_, &tm_q, bar(C::kBarQ), 64 * b, qb0 * 64, bh);
        tma_load_3d(dq_ + 64 * 128, &tm_q, bar(C::kBarQ), 64 * b, has_hi ? qb1 * 64 : L, bh);
        tma_load_3d(dd_, &tm_do, bar(C::kBarQ), 64 * b, qb0 * 64, bh);
        tma_load_3d(dd_ + 64 * 128, &tm_do, bar(C::kBarQ), 64 * b, has_hi ? qb1 * 64 : L, bh);
      }
    }
    __syncwarp();
    int issued = 0;
    bool ok = true;
    for (int u = 0; u < U; ++u) {
      if (aborted()) { ok = false; break; }
      const int sl = u % C::kStages;
      if (u >= C::kStages) {
        if (!uwait(bar(C::kBarKEmpty + sl), ((u / C::kStages) - 1) & 1)) { ok = false; break; }
        if (!uwait(bar(C::kBarVEmpty + sl), ((u / C::kStages) - 1) & 1)) { ok = false; break; }
      }
      const int e = tiles[u < T1 ? u : u - T1];
      const CUtensorMap *mk = e >= 0 ? &tm_k : &tm_kbar;
      const CUtensorMap *mv = e >= 0 ? &tm_v : &tm_vbar;
      const int row = e >= 0 ? (e >> 2) * 64 : (-e - 1) * 64;
      const uint32_t dk = sbase + C::kOffK + sl * C::kTileBytes;
      const uint32_t dv = sbase + C::kOffV + sl * C::kTileBytes;
      if (elect_one()) {
        mbar_expect_tx(bar(C::kBarKFull + sl), C::kTileBytes);
        mbar_expect_tx(bar(C::kBarVFull + sl), C::kTileBytes);
#pragma unroll
        for (int b = 0; b < D / 64; ++b) {
          tma_load_3d(dk + b * C::kBoxKBytes, mk, bar(C::kBarKFull + sl), 64 * b, row, bh);
          tma_load_3d(dv + b * C::kBoxKBytes, mv, bar(C::kBarVFull + sl), 64 * b, row, bh);
        }
      }
      __syncwarp();
      issued = u + 1;
    }
    if (!ok) {
      misc[1] = 1;
      // let the copies already in flight land before the CTA exits
      uwait(bar(C::kBarQ), 0);
      for (int u = issued - C::kStages; u < issued; ++u)
        if (u >= 0) {
          uwait(bar(C::kBarKFull + u % C::kStages), (u / C::kStages) & 1);
          uwait(bar(C::kBarVFull + u % C::kStages), (u / C::kStages) & 1);
        }
    }
  } else if (warp == 1 || warp == 10) {
    // ======================= MMA issuers ======================================
    // One warp issues tcgen05.mma at a bounded rate, so the products are
    // split: warp 1 issues S_u = Q K_u^T; warp 10 issues dP_u = dout V_u^T and,
    // in the second sweep, dQ += dS_u K_u.  Buffer u & 1 is rewritten by S_u
    // once the dS warpgroup has read tile u - 2 from it (PFull); its dP half,
    // which then holds dS_u - 2, by dP_u after dQ_u - 2 (warp 10's order).
    constexpr uint32_t kIdQK = idesc_bf16_f32(128, 64, 0, 0);
    constexpr uint32_t kIdDQ = idesc_bf16_f32(128, D, 0, 1);
    const bool s_warp = warp == 1;
    bool ok = uwait(bar(C::kBarQ), 0);
    tc_fence_after();
    // descriptors are built once per buffer; a K step adds its byte offset / 16
    // to the start-address field (which cannot carry below 256 KB)
    if (ok) ok = uwait(bar(s_warp ? C::kBarQT : C::kBarDOT), 0);   // Q / dout in tensor memory
    tc_fence_after();
    auto b_step = [](int k) -> uint64_t {
      return (uint64_t)(((k >> 2) * C::kBoxKBytes + (k & 3) * 32) >> 4);
    };
    // warp 10: the second-sweep product for tile w once its dS is in TMEM (in
    // the first sweep only the wait for the dS warpgroup)
    auto finish = [&](int w) -> bool {
      const int b = w & 1, sl = w % C::kStages;
      if (!uwait(bar(C::kBarPFull + b), (w >> 1) & 1)) return false;
      if (w >= T1) {
        tc_fence_after();
        const uint64_t kd = smem_desc_sw128(sbase + C::kOffK + sl * C::kTileBytes, C::kBoxKBytes, 1024);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ts(tmem + C::kColDQ, tmem + C::kColBuf + 128 * b + 64 + kk * 8,
                   kd + (uint64_t)((kk * 2048) >> 4), kIdDQ, (w > T1 || kk > 0) ? 1u : 0u);
          tc_commit(bar(C::kBarKEmpty + sl));
        }
        __syncwarp();
      }
      return true;
    };
    for (int u = 0; ok && u < U; ++u) {
      if (aborted()) { ok = false; break; }
      const int sl = u % C::kStages, b = u & 1;
      if (s_warp) {
        if (u >= 2 && !uwait(bar(C::kBarPFull + b), ((u - 2) >> 1) & 1)) { ok = false; break; }
        if (!uwait(bar(C::kBarKFull + sl), (u / C::kStages) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint64_t kd = smem_desc_sw128(sbase + C::kOffK + sl * C::kTileBytes, 16, 1024);
        if (elect_one()) {
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            mma_ts(tmem + C::kColBuf + 128 * b, tmem + C::kColQ + 8 * k, kd + b_step(k), kIdQK,
                   k > 0 ? 1u : 0u);
          tc_commit(bar(C::kBarSFull + b));
          if (u < T1) tc_commit(bar(C::kBarKEmpty + sl));
        }
        __syncwarp();
      } else {
        if (!uwait(bar(C::kBarVFull + sl), (u / C::kStages) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint64_t vd = smem_desc_sw128(sbase + C::kOffV + sl * C::kTileBytes, 16, 1024);
        if (elect_one()) {
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            mma_ts(tmem + C::kColBuf + 128 * b + 64, tmem + C::kColDO + 8 * k, vd + b_step(k), kIdQK,
                   k > 0 ? 1u : 0u);
          tc_commit(bar(C::kBarSFull + b));
          tc_commit(bar(C::kBarVEmpty + sl));
        }
        __syncwarp();
        if (u >= 1 && !finish(u - 1)) { ok = false; break; }
      }
    }
    if (!s_warp && ok && U >= 1) ok = finish(U - 1);
    if (!s_warp && ok) {
      // dQ is complete once warp 10's last product is (every dS waited on S)
      if (elect_one()) tc_commit(bar(C::kBarFinal));
      __syncwarp();
    }
    if (!ok) misc[1] = 1;
    // before TMEM is released, every product either warp issued must finish
    if (elect_one()) tc_commit(bar(C::kBarTeardown));
    __syncwarp();
    uwait(bar(C::kBarTeardown), 0);
  } else {
    // ======================= dS warpgroups =====================================
    const int g = (warp - 2) >> 2;               // warpgroup: tiles with u & 1 == g
    const int sp = warp & 3;                     // TMEM sub-partition of this warp
    const int row = sp * 32 + lane;              // query row in the tile = TMEM lane
    const int half = row >> 6;
    const bool exists = half == 0 || has_hi;
    const int grow = (half ? qb1 : qb0) * 64 + (row & 63);
    const bool valid = exists && grow < L;
    const uint32_t *cbm = half ? cbm_hi : cbm_lo;
    const uint32_t lane_addr = tmem + ((uint32_t)(sp * 32) << 16);
    const uint32_t s_addr = lane_addr + C::kColBuf + 128 * g, dp_addr = s_addr + 64;
    const float sl2 = scale * kLog2e;
    const float lse2 = valid ? lse[(size_t)bh * L + grow] * kLog2e : INFINITY;
    const int n_last = L - (N - 1) * 64;                 // tokens in the last 64-token tile
    const float wblk = 64.f * (float)bsub;               // n_j of a full block
    const int nc_last = L - (Nc - 1) * 64 * bsub;        // n_j of the last block
    float dpart = 0.f, dfull = 0.f;
    bool exchanged = false, ok = true;
    auto warp_wait = [&](uint32_t b_addr, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(b_addr, parity));
    };
    {
      // this thread's query row of Q (warpgroup 0) or dout (warpgroup 1), from
      // the 128-byte-swizzled TMA boxes (16-byte chunk c of row r sits at
      // chunk c ^ (r & 7)) into tensor memory as packed bf16 pairs; every warp
      // arrives, even after a timeout
      const int src = g == 0 ? C::kOffQ : C::kOffDO;
      const uint32_t dst = lane_addr + (g == 0 ? C::kColQ : C::kColDO);
      if (warp_wait(bar(C::kBarQ), 0)) {
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
          uint32_t w[32];
          const unsigned char *box = smem + src + h * C::kBoxQBytes + row * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 v = *reinterpret_cast<const uint4 *>(box + ((c ^ (row & 7)) << 4));
            w[4 * c] = v.x;
            w[4 * c + 1] = v.y;
            w[4 * c + 2] = v.z;
            w[4 * c + 3] = v.w;
          }
          tmem_st_x32(dst + 32 * h, w);
        }
        tmem_wait_st();
      } else {
        ok = false;
        misc[1] = 1;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(g == 0 ? C::kBarQT : C::kBarDOT));
    }
    // combine the two warpgroups' Delta partial sums (once, before the first
    // second-sweep tile of this warpgroup, or after its loop)
    auto exchange = [&]() -> bool {
      if (delta_given) {
        dfull = valid ? delta[(size_t)bh * Lpad + grow] : 0.f;
        exchanged = true;
        return true;
      }
      delta_sm[g * 128 + row] = dpart;
      mbar_arrive(bar(C::kBarDelta));
      if (!warp_wait(bar(C::kBarDelta), 0)) return false;
      dfull = delta_sm[row] + delta_sm[128 + row];
      // Delta into the padded [BH, Lpad] array (0 for rows past L)
      if (g == 0 && exists) delta[(size_t)bh * Lpad + grow] = valid ? dfull : 0.f;
      exchanged = true;
      return true;
    };
    for (int u = g; u < U; u += 2) {
      if (__any_sync(0xffffffffu, misc[1] != 0)) { ok = false; break; }
      const bool second = u >= T1;
      if (second && !exchanged && !exchange()) { ok = false; break; }
      if (!warp_wait(bar(C::kBarSFull + g), (u >> 1) & 1)) { ok = false; break; }
      tc_fence_after();
      const int e = tiles[second ? u - T1 : u];
      const bool centroid = e < 0;
      // dS of second-sweep tile u goes over the first 32 dP columns of its
      // buffer (read above into registers); dQ_u - 2 has read the dS there
      // before dP_u completed (SFull covers it)
      const uint32_t ds_addr = dp_addr;
      uint64_t keep = 0ull;
      float w_full = 1.f, w_last = 0.f;
      int last_col = -1;
      if (!exists) {
        keep = 0ull;
      } else if (!centroid) {
        if ((e >> half) & 1) {
          keep = ((e >> 2) == N - 1 && n_last < 64) ? ((1ull << n_last) - 1ull) : ~0ull;
        }
      } else {
        const int c = -e - 1;
        const uint32_t m0 = ~cbm[2 * c] & dq_valid_bits(2 * c, Nc);
        const uint32_t m1 = (2 * c + 1 < cwords) ? (~cbm[2 * c + 1] & dq_valid_bits(2 * c + 1, Nc)) : 0u;
        keep = (uint64_t)m0 | ((uint64_t)m1 << 32);
        w_full = wblk;
        if (c == (Nc - 1) / 64 && nc_last < 64 * bsub) {
          last_col = (Nc - 1) % 64;
          w_last = (float)nc_last;
        }
      }
      const bool active = __any_sync(0xffffffffu, keep != 0ull);
      if (active) {
        // all 64 S and 64 dP columns in one TMEM round trip; dS of columns
        // 32h .. 32h+31 goes, packed, into dS-buffer columns 16h .. 16h+15
        uint32_t r[4][32];   // S columns 0-31, 32-63, dP columns 0-31, 32-63
        tmem_ld_x32(s_addr, r[0]);
        tmem_ld_x32(s_addr + 32, r[1]);
        tmem_ld_x32(dp_addr, r[2]);
        tmem_ld_x32(dp_addr + 32, r[3]);
        tmem_wait_ld();
        if (second && !centroid && __all_sync(0xffffffffu, keep == ~0ull)) {
          // an exact tile every row of the warp keeps whole: weight 1, no mask
          // (the same arithmetic as below with on = true, w = 1)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              const float p0 = ex2_approx(fmaf(__uint_as_float(r[h][i]), sl2, -lse2));
              const float p1 = ex2_approx(fmaf(__uint_as_float(r[h][i + 1]), sl2, -lse2));
              pk[i / 2] = pack_bf16x2(p0 * (__uint_as_float(r[2 + h][i]) - dfull),
                                      p1 * (__uint_as_float(r[2 + h][i + 1]) - dfull));
            }
            tmem_st_x16(ds_addr + 16 * h, pk);
          }
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(bar(C::kBarPFull + g));
          continue;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            float pz[2] = {0.f, 0.f};
#pragma unroll
            for (int x = 0; x < 2; ++x) {
              const int col = 32 * h + i + x;
              const bool on = (keep >> col) & 1ull;
              const float w = col == last_col ? w_last : w_full;
              const float p = on ? w * ex2_approx(fmaf(__uint_as_float(r[h][i + x]), sl2, -lse2))
                                 : 0.f;
              const float dp = __uint_as_float(r[2 + h][i + x]);
              if (second) pz[x] = p * (dp - dfull);
              else dpart = fmaf(p, dp, dpart);
            }
            pk[i / 2] = pack_bf16x2(pz[0], pz[1]);
          }
          if (second) tmem_st_x16(ds_addr + 16 * h, pk);
        }
        if (second) tmem_wait_st();
      } else if (second) {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = 0u;
        tmem_st_x32(ds_addr, pk);
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(bar(C::kBarPFull + g));
    }
    if (ok && !exchanged) ok = exchange();
    // ---- epilogue: dq = s dQ, this warpgroup's half of the columns ----------
    if (ok && !__any_sync(0xffffffffu, misc[1] != 0)) {
      if (!warp_wait(bar(C::kBarFinal), 0)) {
        ok = false;
      } else {
        tc_fence_after();
        const size_t obase = ((size_t)bh * L + (size_t)(valid ? grow : 0)) * D;
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          const int col0 = g * (D / 2) + 32 * c;
          uint32_t r[32];
          tmem_ld_x32(lane_addr + C::kColDQ + col0, r);
          tmem_wait_ld();
          if (valid) {
            uint4 *dst = reinterpret_cast<uint4 *>(dq + obase + col0);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(
                  pack_bf16x2(scale * __uint_as_float(r[8 * i]), scale * __uint_as_float(r[8 * i + 1])),
                  pack_bf16x2(scale * __uint_as_float(r[8 * i + 2]), scale * __uint_as_float(r[8 * i + 3])),
                  pack_bf16x2(scale * __uint_as_float(r[8 * i + 4]), scale * __uint_as_float(r[8 * i + 5])),
                  pack_bf16x2(scale * __uint_as_float(r[8 * i + 6]), scale * __uint_as_float(r[8 * i + 7])));
          }
        }
      }
    }
    if (!ok) misc[1] = 1;
  }

  // ---- teardown -----------------------------------------------------------------
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace pisa
