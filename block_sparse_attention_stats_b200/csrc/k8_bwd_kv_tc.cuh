// dk, dv of the exact keys in the zeroth-order backward, on the sm_100a tensor
// cores (tcgen05).
//
// Work unit: one CTA = two adjacent key blocks (2p, 2p+1): 128 key rows, so
// every product is an M = 128 MMA with the keys as rows.  The CTA visits, in
// ascending order, every query block i whose exact set S_i holds either key
// block (a list built beforehand, each entry flagged with which of the two
// i selected); for a key row whose block i did not select, the probabilities
// are zero.  With P_tn = exp(s q_t.k_n - lse_t), dP_tn = dout_t . v_n and the
// row terms Delta_t (from bwd_delta_kernel or the dq kernel's first sweep):
//   dV_n += sum_t P_tn dout_t          dK_n += s sum_t P_tn (dP_tn - Delta_t) q_t
// The epilogue adds the centroid chain terms dkbar_j / n_j, dvbar_j / n_j of
// the key's block and stores bf16.
//
// Roles (352 threads):
//   warp 0      TMA producer: K and V of the two key blocks once, then Q_i,
//               dout_i, lse_i and Delta_i of every listed query block into a
//               3-stage ring;
//   warp 1      TMEM allocation; issues S^T_u = K Q_i^T into TMEM buffer u & 1
//               and, once P^T_u is back in it, dV += P^T_u dout_i;
//   warp 10     issues dP^T_u = V dout_i^T into the same buffer and dK +=
//               dS^T_u Q_i (one warp's issue rate, about 70 cycles per
//               tcgen05.mma, would otherwise bound the kernel at 24 products
//               per tile).  Each half of a buffer is rewritten only by the warp
//               that also reads its bf16 overwrite, in that warp's issue order;
//   warps 2-9   two warpgroups of 4 warps; warpgroup g takes the tiles with
//               u & 1 == g, one thread per key row (TMEM lane): P^T and dS^T
//               written back as bf16 over S^T and dP^T; the epilogue (half of
//               the columns each).
// TMEM columns: dK [0, D), dV [D, 2D), buffer b: S^T [2D + 128 b, +64), dP^T
// the next 64.  Every mbarrier wait is bounded; on a timeout the CTA records
// the error, stops issuing, drains its copies and MMAs, frees TMEM and exits.
#pragma once

#include "pisa_common.cuh"
#include "sm100_primitives.cuh"

namespace pisa {

// ---------------------------------------------------------------------------
// query-block lists of key-block pairs (CSR per head)
// ---------------------------------------------------------------------------
// entry = (t << 2) | (flag: key tile j0 selected) | (flag: key tile j1) << 1,
// ascending query tile t (64 tokens).  bm: the selection bitmap at block level
// [BH, Nc, cwords].  With 64-token blocks (bsub = 1) query and key tiles are
// blocks and pair p is (j0, j1) = kpairs[bh][p] (j1 = -1: a single block), each
// flagged on its own.  With 128-token blocks (bsub = 2) pair p is block p and a
// selecting query block i contributes its two query tiles 2i, 2i+1, with both
// key halves flagged.
// fill == 0: counts[bh * P + p] = list length; fill == 1: write the entries at
// entries + bh * cap + offsets[bh * P + p].  One warp per (p, bh).
__global__ void kvlist_kernel(const uint32_t *__restrict__ bm, int N, int Nc, int cwords,
                              int bsub, int P, const int2 *__restrict__ kpairs, int fill,
                              int *__restrict__ counts, const long long *__restrict__ offsets,
                              long long cap, int *__restrict__ entries) {
  const int p = blockIdx.x, bh = blockIdx.y, lane = threadIdx.x;
  const int2 pr = bsub == 1 ? kpairs[(size_t)bh * P + p] : make_int2(p, -1);
  const uint32_t fmask = (2 * p + 1 < N) ? 3u : 1u;     // key tiles of a 128-token block
  int total = 0;
  int *out = fill ? entries + bh * cap + offsets[(size_t)bh * P + p] : nullptr;
  for (int i0 = 0; i0 < Nc; i0 += 32) {
    const int i = i0 + lane;
    uint32_t bits = 0u;
    if (i < Nc) {
      const uint32_t *row = bm + ((size_t)bh * Nc + i) * cwords;
      bits = (row[pr.x >> 5] >> (pr.x & 31)) & 1u;
      if (pr.y >= 0) bits |= ((row[pr.y >> 5] >> (pr.y & 31)) & 1u) << 1;
    }
    // query tiles this lane contributes, in order
    int n = 0;
    if (bits) n = bsub == 1 ? 1 : (2 * i + 1 < N ? 2 : 1);
    int incl = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (fill && n) {
      const int pos = total + incl - n;
      if (bsub == 1) {
        out[pos] = (i << 2) | (int)bits;
      } else {
        out[pos] = ((2 * i) << 2) | (int)fmask;
        if (n == 2) out[pos + 1] = ((2 * i + 1) << 2) | (int)fmask;
      }
    }
    total += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (!fill && lane == 0) counts[(size_t)bh * P + p] = total;
}

// bmT[bh][j][w]: bit l of word w set iff key block j is in S_(32w + l), the
// transpose of bm (one warp per 32 x 32 bit square).
__global__ void bitmap_transpose_kernel(const uint32_t *__restrict__ bm, int N, int nwords,
                                        uint32_t *__restrict__ bmT) {
  const int wi = blockIdx.x, wj = blockIdx.y, bh = blockIdx.z, lane = threadIdx.x;
  const int i = 32 * wi + lane;
  const uint32_t word = i < N ? bm[((size_t)bh * N + i) * nwords + wj] : 0u;
#pragma unroll 4
  for (int b = 0; b < 32; ++b) {
    const uint32_t col = __ballot_sync(0xffffffffu, (word >> b) & 1u);
    const int j = 32 * wj + b;
    if (lane == b && j < N) bmT[((size_t)bh * N + j) * nwords + wi] = col;
  }
}

// offsets[bh * P + p] = exclusive prefix sum of counts over p (one CTA per head)
__global__ void kvlist_scan_kernel(const int *__restrict__ counts, int P,
                                   long long *__restrict__ offsets) {
  __shared__ long long warp_tot[32];
  __shared__ long long carry;
  const int bh = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int p0 = 0; p0 < P; p0 += blockDim.x) {
    const int p = p0 + tid;
    const long long c = p < P ? counts[(size_t)bh * P + p] : 0;
    long long x = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    long long before = carry;
    for (int k = 0; k < warp; ++k) before += warp_tot[k];
    if (p < P) offsets[(size_t)bh * P + p] = before + x - c;
    __syncthreads();
    if (tid == blockDim.x - 1) carry = before + x;
    __syncthreads();
  }
}

// lse_pad[bh, t] = lse[bh, t] * log2(e) for t < L, +inf up to the padded length
// (the kernels exponentiate with ex2)
__global__ void pad_lse_kernel(const float *__restrict__ lse, int L, int Lpad, int BH,
                               float *__restrict__ lse_pad) {
  const size_t n = (size_t)BH * Lpad;
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n;
       e += (size_t)gridDim.x * blockDim.x) {
    const size_t bh = e / Lpad;
    const int t = (int)(e % Lpad);
    lse_pad[e] = t < L ? lse[bh * L + t] * kLog2e : INFINITY;
  }
}

// ---------------------------------------------------------------------------
// the tensor-core dk / dv kernel
// ---------------------------------------------------------------------------
template <int D> struct KvTcCfg {
  static constexpr int kThreads = 352;
  static constexpr int kStages = 3;
  static constexpr int kPairBytes = 128 * D * 2;   // K or V of the two key blocks
  static constexpr int kBoxPairBytes = 128 * 128;  // one 64-column box of 128 rows
  static constexpr int kBoxRowBytes = 64 * 128;    // one 64-column box of 64 rows
  static constexpr int kTileBytes = 64 * D * 2;    // Q_i or dout_i
  static constexpr int kVecBytes = 2 * 64 * 4;     // lse_i, Delta_i
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kPairBytes;
  static constexpr int kOffQ = 2 * kPairBytes;
  static constexpr int kOffDO = kOffQ + kStages * kTileBytes;
  static constexpr int kOffVec = kOffDO + kStages * kTileBytes;
  static constexpr int kOffBar = kOffVec + kStages * kVecBytes;
  static constexpr int kNumBars = 16;
  static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
  static constexpr int kOffMisc = kOffTmemSlot + 16;
  static constexpr int kSmem = kOffMisc + 16 + 1024;   // + alignment slack
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColDK = 0;
  static constexpr uint32_t kColDV = D;
  static constexpr uint32_t kColBuf = 2 * D;       // + 128 b
  static constexpr int kBarKV = 0;
  static constexpr int kBarQFull = 1;              // + slot
  static constexpr int kBarQEmpty = kBarQFull + kStages;
  static constexpr int kBarSFull = kBarQEmpty + kStages;   // + buffer
  static constexpr int kBarPFull = kBarSFull + 2;          // + buffer
  static constexpr int kBarFinal = kBarPFull + 2;
  static constexpr int kBarTeardown = kBarFinal + 1;
  static_assert(kBarTeardown < kNumBars, "barrier slots");
};

// CENT = false: exact keys, as above.  CENT = true: the rows are 128
// consecutive block centroids (kbar_j, vbar_j = vsum_j / n_j from the packed
// centroid arrays) instead of keys; every query block is visited, a centroid
// row takes weight n_j where the query block left block j unselected (0
// elsewhere), and the epilogue writes dkbar_j / n_j and dvbar_j / n_j (float32)
// for the exact pass's chain terms.
template <int D, bool CENT>
__global__ void __launch_bounds__(352, 1)
    bwd_kv_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_do,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_lse,
                     const __grid_constant__ CUtensorMap tm_delta,
                     const int *__restrict__ counts, const long long *__restrict__ offsets,
                     long long cap, const int *__restrict__ entries,
                     const int2 *__restrict__ kpairs,
                     const uint32_t *__restrict__ bm, int cwords, int bsub, int Nc, int L,
                     int N, float scale,
                     float *__restrict__ dkbar, float *__restrict__ dvbar, int Npad,
                     __nv_bfloat16 *__restrict__ dK, __nv_bfloat16 *__restrict__ dV) {
  using C = KvTcCfg<D>;
  using namespace sm100;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  unsigned char *smem = smem_raw + (sbase - raw);
  auto bar = [&](int i) -> uint32_t { return sbase + C::kOffBar + 8 * i; };
  volatile int *misc = reinterpret_cast<volatile int *>(smem + C::kOffMisc);  // [1] abort
  const float *vec = reinterpret_cast<const float *>(smem + C::kOffVec);

  const int p = blockIdx.x, bh = blockIdx.y;
  const int P = (N + 1) / 2;
  // row chunks (64 rows each) of this CTA: key blocks, or 64-centroid chunks
  const int nchunk = CENT ? Npad / 64 : N;
  // 64-row chunks of this CTA: a key-block pair (64-token blocks), the two
  // tiles of one 128-token block, or 128 consecutive centroids
  const int2 kp = kpairs ? kpairs[(size_t)bh * P + p] : make_int2(-1, -1);
  const int j0 = kpairs ? kp.x : 2 * p;
  const int j1 = kpairs ? kp.y : (2 * p + 1 < nchunk ? 2 * p + 1 : -1);
  const int T = CENT ? N : counts[(size_t)bh * P + p];
  const int *list = CENT ? nullptr : entries + bh * cap + offsets[(size_t)bh * P + p];
  const int row_end = CENT ? Npad : L;   // first row past the K / V (or centroid) rows
  const int tid = threadIdx.x, lane = tid & 31;
  const int warp = __shfl_sync(0xffffffffu, tid >> 5, 0);

  if (warp == 1) {
    tmem_alloc(sbase + C::kOffTmemSlot, C::kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar(C::kBarKV), 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar(C::kBarQFull + s), 1);
      mbar_init(bar(C::kBarQEmpty + s), 2);      // dV from warp 1, dK from warp 10
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(C::kBarSFull + b), 2);       // S^T from warp 1, dP^T from warp 10
      mbar_init(bar(C::kBarPFull + b), 128);
    }
    mbar_init(bar(C::kBarFinal), 2);
    mbar_init(bar(C::kBarTeardown), 2);
    fence_mbar_init();
    misc[1] = 0;
  }
  if (tid == 32) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_do);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_lse);
    prefetch_tmap(&tm_delta);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + C::kOffTmemSlot);

  auto uwait = [&](uint32_t b_addr, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, mbar_wait(b_addr, parity));
  };
  auto aborted = [&]() -> bool { return __any_sync(0xffffffffu, misc[1] != 0); };

  if (warp == 0) {
    // ======================= TMA producer =====================================
    bool ok = true;
    int issued = 0;
    if (T > 0) {
      if (elect_one()) {
        mbar_expect_tx(bar(C::kBarKV), 2 * C::kPairBytes);
#pragma unroll
        for (int b = 0; b < D / 64; ++b) {
          const uint32_t dk = sbase + C::kOffK + b * C::kBoxPairBytes;
          const uint32_t dv = sbase + C::kOffV + b * C::kBoxPairBytes;
          tma_load_3d(dk, &tm_k, bar(C::kBarKV), 64 * b, j0 * 64, bh);
          tma_load_3d(dk + 64 * 128, &tm_k, bar(C::kBarKV), 64 * b, j1 >= 0 ? j1 * 64 : row_end, bh);
          tma_load_3d(dv, &tm_v, bar(C::kBarKV), 64 * b, j0 * 64, bh);
          tma_load_3d(dv + 64 * 128, &tm_v, bar(C::kBarKV), 64 * b, j1 >= 0 ? j1 * 64 : row_end, bh);
        }
      }
      __syncwarp();
      for (int u = 0; u < T; ++u) {
        if (aborted()) { ok = false; break; }
        const int sl = u % C::kStages;
        if (u >= C::kStages && !uwait(bar(C::kBarQEmpty + sl), ((u / C::kStages) - 1) & 1)) {
          ok = false;
          break;
        }
        const int i = CENT ? u : list[u] >> 2;
        if (elect_one()) {
          const uint32_t full = bar(C::kBarQFull + sl);
          mbar_expect_tx(full, 2 * C::kTileBytes + C::kVecBytes);
          const uint32_t dq_ = sbase + C::kOffQ + sl * C::kTileBytes;
          const uint32_t dd_ = sbase + C::kOffDO + sl * C::kTileBytes;
#pragma unroll
          for (int b = 0; b < D / 64; ++b) {
            tma_load_3d(dq_ + b * C::kBoxRowBytes, &tm_q, full, 64 * b, i * 64, bh);
            tma_load_3d(dd_ + b * C::kBoxRowBytes, &tm_do, full, 64 * b, i * 64, bh);
          }
          const uint32_t dvec = sbase + C::kOffVec + sl * C::kVecBytes;
          tma_load_2d(dvec, &tm_lse, full, i * 64, bh);
          tma_load_2d(dvec + 256, &tm_delta, full, i * 64, bh);
        }
        __syncwarp();
        issued = u + 1;
      }
    }
    if (!ok) {
      misc[1] = 1;
      uwait(bar(C::kBarKV), 0);
      for (int u = issued - C::kStages; u < issued; ++u)
        if (u >= 0) uwait(bar(C::kBarQFull + u % C::kStages), (u / C::kStages) & 1);
    }
  } else if (warp == 1 || warp == 10) {
    // ======================= MMA issuers ======================================
    // warp 1: S^T_u into the S half of buffer u & 1, dV += P^T_w dout_w from
    // it; warp 10: dP^T_u into the dP half, dK += dS^T_w Q_w from it.  A half
    // is rewritten (by the product of tile w + 2) only after the same warp
    // has issued the product that reads tile w's overwrite, and one thread's
    // tcgen05 products run in issue order.
    constexpr uint32_t kIdS = idesc_bf16_f32(128, 64, 0, 0);
    constexpr uint32_t kIdAcc = idesc_bf16_f32(128, D, 0, 1);
    const bool s_warp = warp == 1;
    const uint32_t half_col = s_warp ? 0u : 64u;     // S^T or dP^T half of a buffer
    const uint32_t acc_col = s_warp ? C::kColDV : C::kColDK;
    bool ok = true;
    if (T > 0) {
      ok = uwait(bar(C::kBarKV), 0);
      tc_fence_after();
      // descriptors are built once per buffer; a K step adds its byte offset /
      // 16 to the start-address field (which cannot carry below 256 KB)
      const uint64_t ad0 = smem_desc_sw128(sbase + (s_warp ? C::kOffK : C::kOffV), 16, 1024);
      const int b_off = s_warp ? C::kOffQ : C::kOffDO;    // B of S^T / dP^T
      const int acc_b_off = s_warp ? C::kOffDO : C::kOffQ;  // B of dV / dK
      auto a_step = [](int k) -> uint64_t {
        return (uint64_t)(((k >> 2) * C::kBoxPairBytes + (k & 3) * 32) >> 4);
      };
      auto b_step = [](int k) -> uint64_t {
        return (uint64_t)(((k >> 2) * C::kBoxRowBytes + (k & 3) * 32) >> 4);
      };
      // the accumulating product of tile w once its bf16 overwrite is in TMEM
      auto finish = [&](int w) -> bool {
        const int b = w & 1, sl = w % C::kStages;
        if (!uwait(bar(C::kBarPFull + b), (w >> 1) & 1)) return false;
        tc_fence_after();
        const uint64_t bd = smem_desc_sw128(sbase + acc_b_off + sl * C::kTileBytes,
                                            C::kBoxRowBytes, 1024);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ts(tmem + acc_col, tmem + C::kColBuf + 128 * b + half_col + kk * 8,
                   bd + (uint64_t)((kk * 2048) >> 4), kIdAcc, (w > 0 || kk > 0) ? 1u : 0u);
          tc_commit(bar(C::kBarQEmpty + sl));
        }
        __syncwarp();
        return true;
      };
      for (int u = 0; ok && u < T; ++u) {
        if (aborted()) { ok = false; break; }
        const int sl = u % C::kStages, b = u & 1;
        if (!uwait(bar(C::kBarQFull + sl), (u / C::kStages) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint64_t bd = smem_desc_sw128(sbase + b_off + sl * C::kTileBytes, 16, 1024);
        if (elect_one()) {
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            mma_ss(tmem + C::kColBuf + 128 * b + half_col, ad0 + a_step(k), bd + b_step(k), kIdS,
                   k > 0 ? 1u : 0u);
          tc_commit(bar(C::kBarSFull + b));
        }
        __syncwarp();
        if (u >= 1 && !finish(u - 1)) { ok = false; break; }
      }
      if (ok) ok = finish(T - 1);
      if (ok) {
        if (elect_one()) tc_commit(bar(C::kBarFinal));
        __syncwarp();
      }
    }
    if (!ok) misc[1] = 1;
    // every MMA this warp issued must finish before TMEM is released
    if (elect_one()) tc_commit(bar(C::kBarTeardown));
    __syncwarp();
    uwait(bar(C::kBarTeardown), 0);
  } else {
    // ======================= P / dS warpgroups ================================
    const int g = (warp - 2) >> 2;
    const int sp = warp & 3;
    const int row = sp * 32 + lane;              // key row in the tile = TMEM lane
    const int half = row >> 6;
    const int jb = half ? j1 : j0;
    const int key = jb * 64 + (row & 63);          // key token, or centroid index
    const bool kvalid = jb >= 0 && key < (CENT ? Nc : L);
    // centroid rows: n_j (64 bsub, or the last block's size)
    const float wn = (CENT && key == Nc - 1) ? (float)(L - 64 * bsub * (Nc - 1)) : 64.f * bsub;
    const uint32_t lane_addr = tmem + ((uint32_t)(sp * 32) << 16);
    const uint32_t s_addr = lane_addr + C::kColBuf + 128 * g, dp_addr = s_addr + 64;
    const float sl2 = scale * kLog2e;
    bool ok = true;
    auto warp_wait = [&](uint32_t b_addr, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(b_addr, parity));
    };
    for (int u = g; u < T; u += 2) {
      if (__any_sync(0xffffffffu, misc[1] != 0)) { ok = false; break; }
      // centroid rows: was block `key` left unselected by query block u?
      const uint32_t selw =
          (CENT && kvalid) ? bm[((size_t)bh * Nc + u / bsub) * cwords + (key >> 5)] : 0u;
      if (!warp_wait(bar(C::kBarSFull + g), (u >> 1) & 1)) { ok = false; break; }
      tc_fence_after();
      const int sl = u % C::kStages;
      const bool on = CENT ? (kvalid && !((selw >> (key & 31)) & 1u))
                           : (kvalid && (((list[u] & 3) >> half) & 1));
      const float wrow = CENT ? wn : 1.f;
      const float *ls = vec + sl * (C::kVecBytes / 4);     // lse * log2 e of the 64 query rows
      const float *dl = ls + 64;                            // Delta of the 64 query rows
      uint32_t pp[32], pd[32];
      if (__any_sync(0xffffffffu, on)) {
        uint32_t r[4][32];   // S^T columns 0-31, 32-63, dP^T columns 0-31, 32-63
        tmem_ld_x32(s_addr, r[0]);
        tmem_ld_x32(s_addr + 32, r[1]);
        tmem_ld_x32(dp_addr, r[2]);
        tmem_ld_x32(dp_addr + 32, r[3]);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            const float4 l4 = *reinterpret_cast<const float4 *>(ls + 32 * h + i);
            const float4 d4 = *reinterpret_cast<const float4 *>(dl + 32 * h + i);
            const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dv4[4] = {d4.x, d4.y, d4.z, d4.w};
            float pv[4], zv[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              const float pr = on ? wrow * ex2_approx(fmaf(__uint_as_float(r[h][i + x]), sl2,
                                                           -lv[x]))
                                  : 0.f;
              pv[x] = pr;
              zv[x] = pr * (__uint_as_float(r[2 + h][i + x]) - dv4[x]);
            }
            pp[16 * h + i / 2] = pack_bf16x2(pv[0], pv[1]);
            pp[16 * h + i / 2 + 1] = pack_bf16x2(pv[2], pv[3]);
            pd[16 * h + i / 2] = pack_bf16x2(zv[0], zv[1]);
            pd[16 * h + i / 2 + 1] = pack_bf16x2(zv[2], zv[3]);
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          pp[i] = 0u;
          pd[i] = 0u;
        }
      }
      tmem_st_x32(s_addr, pp);
      tmem_st_x32(dp_addr, pd);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(C::kBarPFull + g));
    }
    // ---- epilogue: dk = s dK + dkbar_j / n_j, dv = dV + dvbar_j / n_j ---------
    if (ok && T > 0 && !__any_sync(0xffffffffu, misc[1] != 0)) {
      if (!warp_wait(bar(C::kBarFinal), 0)) ok = false;
      else tc_fence_after();
    }
    if (CENT && ok && !__any_sync(0xffffffffu, misc[1] != 0)) {
      // dkbar_j / n_j = s dK / n_j, dvbar_j / n_j = dV / n_j
      const float inv_n = 1.f / wn;
      float *pk = dkbar + ((size_t)bh * Npad + (kvalid ? key : 0)) * D;
      float *pv = dvbar + ((size_t)bh * Npad + (kvalid ? key : 0)) * D;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        const int col0 = g * (D / 2) + 32 * c;
        uint32_t rk[32], rv[32];
        tmem_ld_x32(lane_addr + C::kColDK + col0, rk);
        tmem_ld_x32(lane_addr + C::kColDV + col0, rv);
        tmem_wait_ld();
        if (kvalid) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            reinterpret_cast<float4 *>(pk + col0)[i] =
                make_float4(scale * inv_n * __uint_as_float(rk[4 * i]),
                            scale * inv_n * __uint_as_float(rk[4 * i + 1]),
                            scale * inv_n * __uint_as_float(rk[4 * i + 2]),
                            scale * inv_n * __uint_as_float(rk[4 * i + 3]));
            reinterpret_cast<float4 *>(pv + col0)[i] =
                make_float4(inv_n * __uint_as_float(rv[4 * i]), inv_n * __uint_as_float(rv[4 * i + 1]),
                            inv_n * __uint_as_float(rv[4 * i + 2]),
                            inv_n * __uint_as_float(rv[4 * i + 3]));
          }
        }
      }
    }
    if (!CENT && ok && !__any_sync(0xffffffffu, misc[1] != 0)) {
      const int blk = jb >= 0 ? jb / bsub : 0;          // the key's block
      const float *ck = dkbar + ((size_t)bh * Npad + blk) * D;
      const float *cv = dvbar + ((size_t)bh * Npad + blk) * D;
      const size_t obase = ((size_t)bh * L + (size_t)(kvalid ? key : 0)) * D;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        const int col0 = g * (D / 2) + 32 * c;
        uint32_t rk[32], rv[32];
        if (T > 0) {
          tmem_ld_x32(lane_addr + C::kColDK + col0, rk);
          tmem_ld_x32(lane_addr + C::kColDV + col0, rv);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            rk[i] = 0u;
            rv[i] = 0u;
          }
        }
        if (kvalid) {
          uint4 *pk = reinterpret_cast<uint4 *>(dK + obase + col0);
          uint4 *pv = reinterpret_cast<uint4 *>(dV + obase + col0);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t wk[4], wv[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              const int cc = col0 + 8 * i + 2 * x;
              wk[x] = pack_bf16x2(fmaf(scale, __uint_as_float(rk[8 * i + 2 * x]), ck[cc]),
                                  fmaf(scale, __uint_as_float(rk[8 * i + 2 * x + 1]), ck[cc + 1]));
              wv[x] = pack_bf16x2(__uint_as_float(rv[8 * i + 2 * x]) + cv[cc],
                                  __uint_as_float(rv[8 * i + 2 * x + 1]) + cv[cc + 1]);
            }
            pk[i] = make_uint4(wk[0], wk[1], wk[2], wk[3]);
            pv[i] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
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
