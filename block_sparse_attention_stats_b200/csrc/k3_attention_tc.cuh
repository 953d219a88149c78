// K3 (tcgen05 version): fused exact-or-approximate attention on sm_100a.
//
// "Technical Summary: PISA" (gist.science), section 2: "Core Algorithm" (the
// numerator N_t equation, alpha_{t,j} = exp(q_t kbar_j^T), o_t = N_t / D_t),
// "Key Insights" 2 (both approximations enter the same softmax numerator and
// denominator) and "Hardware Implementation" (one fused kernel running the
// exact phase over selected blocks, the zeroth-order scan over aggregated
// block vectors of unselected blocks and the global first-order correction
// inside one online softmax).
//
// Work unit: one CTA = two adjacent query blocks (2p, 2p+1) of one head, i.e.
// 128 query rows, so every tensor-core product is an M = 128 tcgen05 MMA.
// The exact tiles are the union S_2p u S_2p+1 (ascending); each carries two
// flags saying which half selected it.  A half that did not select a tile
// gives it zero probability (and spends no exp on it); that block then reaches
// that half through its centroid, as in the method.  After the exact tiles
// come the centroid chunks: 64 consecutive block centroids kbar_j as keys and
// value sums vsum_j as values, masked per half to that half's unselected
// blocks U_i, with weight n_j in the denominator; their probabilities are also
// summed into a_t = sum_{U_i} alpha_tj.  In the paper ("hyd") mode a last MMA
// forms Q Hbar and the epilogue adds s a_t (q_t Hbar) to the numerator.
//
// With 128-token blocks (block_size 128) a CTA is one query block: both
// halves share S_i, every selected block contributes its two 64-token tiles,
// and the centroids (one per 128-token block, n_j = 128) are masked by the
// block-level selection.
//
// Roles (192 threads):
//   warp 0      TMA producer: Q once, then the K/V (or kbar/vsum) tile of every
//               list entry into a 2-stage ring, then Hbar;
//   warp 1      TMEM allocation; one thread issues every tcgen05.mma:
//               S_b = Q K^T (two S buffers), O += P V with P read from TMEM,
//               and Q Hbar at the end;
//   warps 2-5   softmax: one thread per query row (= TMEM lane); reads S, keeps
//               the running max m (log2 domain), denominator l and tail weight
//               a in registers, writes P (bf16) into the S columns, rescales
//               the O row in TMEM only when the max grows by more than 2^8,
//               and runs the epilogue o = (O + s a QHbar) / l.
// TMEM columns: O [0, D), S buffers [D, D+64) and [D+64, D+128); Q Hbar
// reuses [D, 2D) after the last P V.
// Every mbarrier wait is bounded (sm100::mbar_wait); on a timeout the CTA
// records the error, stops issuing work, waits for its own copies and MMAs,
// frees TMEM and exits.
#pragma once

#include "k2_select.cuh"
#include "pisa_common.cuh"
#include "sm100_primitives.cuh"

namespace pisa {

// Selection inside the fused kernel (128-token blocks only, where a CTA is one
// query block and needs no partner): the CTA scores its own pooled query
// against every block centroid (a float32 FMA chain over the head dimension,
// as select_fused_kernel does) and takes the top k_sel with the sink forced
// in, by the same rule as pisa_select.  Up to 512 blocks the sets are the
// separate step's bit for bit; on longer rows the separate step's scores come
// from the tensor cores and may order two blocks whose scores agree to float32
// rounding the other way.
struct FusedSelect {
  const float *qbar;   // [BH, Nc, D] (NULL: the selection comes from idx)
  const float *kbar;   // [BH, Nc, D]
  const float *cov;    // [BH, Nc] or NULL
  float cov_weight;
  int sink;            // forced block, or -1
  int32_t *idx_out;    // optional [BH, Nc, k_sel] copy of the selection
};

template <int D> struct TcCfg {
  static constexpr int kThreads = 192;
  static constexpr int kRows = 128;
  static constexpr int kKeys = 64;
  static constexpr int kKStages = 2;                // K ring: a slot frees when its S MMA is done
  static constexpr int kVStages = 2;                // V ring: a slot frees when its P V MMA is done
  static constexpr int kQBytes = kRows * D * 2;
  static constexpr int kBoxQBytes = kRows * 128;   // one 64-column box of Q
  static constexpr int kBoxKBytes = kKeys * 128;   // one 64-column box of a K/V tile
  static constexpr int kTileBytes = kKeys * D * 2;
  static constexpr int kHbarBytes = D * D * 2;
  static_assert(kHbarBytes <= kKStages * kTileBytes, "Hbar must fit in the K ring");
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kQBytes;
  static constexpr int kOffV = kOffK + kKStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kVStages * kTileBytes;
  static constexpr int kNumBars = 24;
  static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
  static constexpr int kOffMisc = kOffTmemSlot + 16;
  static constexpr int kOffDyn = kOffMisc + 16;
  static constexpr uint32_t kTmemCols = 256;
  static constexpr uint32_t kColO = 0;
  static constexpr uint32_t kColS = D;
  static constexpr uint32_t kColQH = D;
  // barrier indices
  static constexpr int kBarQ = 0;
  static constexpr int kBarKFull = 1;                   // + slot
  static constexpr int kBarKEmpty = kBarKFull + kKStages;
  static constexpr int kBarVFull = kBarKEmpty + kKStages;
  static constexpr int kBarVEmpty = kBarVFull + kVStages;
  static constexpr int kBarSFull = kBarVEmpty + kVStages;  // + S buffer
  static constexpr int kBarPFull = kBarSFull + 2;          // + S buffer
  static constexpr int kBarODone = kBarPFull + 2;
  static constexpr int kBarFinal = kBarODone + 1;          // after the last MMA
  static constexpr int kBarTeardown = kBarFinal + 1;
  static constexpr int kBarHFull = kBarTeardown + 1;
  static_assert(kBarHFull < kNumBars, "barrier slots");

  // N 64-token tiles, Nc blocks (= centroids)
  __host__ __device__ static int smem_bytes(int N, int Nc) {
    const int nwords = (N + 31) / 32, cwords = (Nc + 31) / 32;
    return kOffDyn + (2 * nwords + 2 * cwords + N + (Nc + 63) / 64) * 4 + 1024;  // + slack
  }
};

__device__ __forceinline__ uint32_t valid_bits(int w, int N) {
  const int lo = w * 32;
  if (lo + 32 <= N) return 0xffffffffu;
  if (lo >= N) return 0u;
  return (1u << (N - lo)) - 1u;
}

template <int D>
__global__ void __launch_bounds__(192, 2)
    piecewise_attention_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                                  const __grid_constant__ CUtensorMap tm_k,
                                  const __grid_constant__ CUtensorMap tm_v,
                                  const __grid_constant__ CUtensorMap tm_kbar,
                                  const __grid_constant__ CUtensorMap tm_vsum,
                                  const __grid_constant__ CUtensorMap tm_hbar,
                                  const int32_t *__restrict__ idx,
                                  const int2 *__restrict__ pairs, int k_sel, int L, int N,
                                  int bsub, int Nc, float scale, int hyd, int dense, int blockwise,
                                  void *__restrict__ out, int out_f32,
                                  float *__restrict__ lse, float *__restrict__ o_keep,
                                  const FusedSelect fsel) {
  using C = TcCfg<D>;
  using namespace sm100;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  unsigned char *smem = smem_raw + (sbase - raw);
  auto bar = [&](int i) -> uint32_t { return sbase + C::kOffBar + 8 * i; };
  volatile int *misc = reinterpret_cast<volatile int *>(smem + C::kOffMisc);  // [0] tiles, [1] abort
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
  // query blocks of the two halves (rows 0-63 and 64-127 of the tile), as
  // 64-token tiles; the selection row of each half
  int qb0 = 2 * pair, qb1 = 2 * pair + 1 < N ? 2 * pair + 1 : -1;
  int sr0 = qb0, sr1 = qb1;
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
  // warp index through a shuffle so the compiler knows it is warp-uniform: the
  // producer and MMA warps then run converged and keep their descriptors in
  // uniform registers (one elected lane issues each TMA copy / MMA)
  const int tid = threadIdx.x, lane = tid & 31;
  const int warp = __shfl_sync(0xffffffffu, tid >> 5, 0);

  // ---- set-up ---------------------------------------------------------------
  if (warp == 1) {
    tmem_alloc(sbase + C::kOffTmemSlot, C::kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar(C::kBarQ), 1);
    for (int s = 0; s < C::kKStages; ++s) {
      mbar_init(bar(C::kBarKFull + s), 1);
      mbar_init(bar(C::kBarKEmpty + s), 1);
    }
    for (int s = 0; s < C::kVStages; ++s) {
      mbar_init(bar(C::kBarVFull + s), 1);
      mbar_init(bar(C::kBarVEmpty + s), 1);
    }
    mbar_init(bar(C::kBarHFull), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(C::kBarSFull + b), 1);
      mbar_init(bar(C::kBarPFull + b), 128);
    }
    mbar_init(bar(C::kBarODone), 1);
    mbar_init(bar(C::kBarFinal), 1);
    mbar_init(bar(C::kBarTeardown), 1);
    fence_mbar_init();
    misc[1] = 0;
  }
  if (tid == 32) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_kbar);
    prefetch_tmap(&tm_vsum);
    prefetch_tmap(&tm_hbar);
  }
  for (int w = tid; w < 2 * nwords + 2 * cwords; w += C::kThreads) bm_lo[w] = 0u;
  __syncthreads();
  if (dense) {
    for (int w = tid; w < nwords; w += C::kThreads) {
      bm_lo[w] = valid_bits(w, N);
      bm_hi[w] = has_hi ? valid_bits(w, N) : 0u;
    }
  } else if (bsub == 1) {
    const int32_t *r0 = idx + ((size_t)bh * Nc + sr0) * k_sel;
    const int32_t *r1 = idx + ((size_t)bh * Nc + (has_hi ? sr1 : sr0)) * k_sel;
    for (int t = tid; t < (has_hi ? 2 : 1) * k_sel; t += C::kThreads) {
      const int j = t < k_sel ? r0[t] : r1[t - k_sel];
      uint32_t *bm = t < k_sel ? bm_lo : bm_hi;
      if (j >= 0 && j < N) atomicOr(&bm[j >> 5], 1u << (j & 31));
      else report_device_error(kDevErrRange);
    }
  } else {
    // one selection row for the 128-token query block: block j covers the
    // 64-token tiles 2j and 2j + 1 (the last block may have only the first)
    const int32_t *r0 = idx + ((size_t)bh * Nc + sr0) * k_sel;
    if (fsel.qbar != nullptr) {
      // select here: scores of this query block against every centroid (the
      // tile list's space holds them and, after them, the selected indices;
      // the V ring, not yet in use, holds the pooled query and the radix
      // histogram)
      float *sc = reinterpret_cast<float *>(tiles);
      int32_t *sel = tiles + Nc;
      float *qrow = reinterpret_cast<float *>(smem + C::kOffV);
      unsigned *hist = reinterpret_cast<unsigned *>(smem + C::kOffV + D * 4);
      const float *qb = fsel.qbar + ((size_t)bh * Nc + sr0) * D;
      for (int e = tid; e < D; e += C::kThreads) qrow[e] = qb[e];
      __syncthreads();
      for (int j = tid; j < Nc; j += C::kThreads) {
        const float4 *kr = reinterpret_cast<const float4 *>(fsel.kbar + ((size_t)bh * Nc + j) * D);
        float acc = 0.f;
#pragma unroll 8
        for (int e4 = 0; e4 < D / 4; ++e4) {
          const float4 kv = __ldg(kr + e4);
          acc = fmaf(qrow[4 * e4 + 0], kv.x, acc);
          acc = fmaf(qrow[4 * e4 + 1], kv.y, acc);
          acc = fmaf(qrow[4 * e4 + 2], kv.z, acc);
          acc = fmaf(qrow[4 * e4 + 3], kv.w, acc);
        }
        const float cw = fsel.cov_weight != 0.f ? fsel.cov_weight * fsel.cov[(size_t)bh * Nc + j] : 0.f;
        sc[j] = fmaf(scale, acc, cw);
      }
      __syncthreads();
      if (tid < 32) topk_row(sc, Nc, k_sel, fsel.sink, hist, sel, lane);
      __syncthreads();
      if (fsel.idx_out != nullptr)
        for (int t = tid; t < k_sel; t += C::kThreads)
          fsel.idx_out[((size_t)bh * Nc + sr0) * k_sel + t] = sel[t];
      r0 = sel;
    }
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
      // block-wise first order visits every block (Taylor weights where unselected)
      uint32_t u = blockwise ? (w < nwords ? valid_bits(w, N) : 0u) : (lo | hi);
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
    if (!dense && !blockwise) {
      const int nch = (Nc + 63) / 64;
      for (int c0 = 0; c0 < nch; c0 += 32) {
        const int c = c0 + lane;
        bool need = false;
        if (c < nch) {
          for (int h = 0; h < (has_hi ? 2 : 1); ++h) {
            const uint32_t *cb = h ? cbm_hi : cbm_lo;
            const uint32_t m0 = ~cb[2 * c] & valid_bits(2 * c, Nc);
            const uint32_t m1 = (2 * c + 1 < cwords) ? (~cb[2 * c + 1] & valid_bits(2 * c + 1, Nc)) : 0u;
            need = need || ((m0 | m1) != 0u);
          }
        }
        const unsigned bal = __ballot_sync(0xffffffffu, need);
        if (need) tiles[base + __popc(bal & ((1u << lane) - 1u))] = -(c + 1);
        base += __popc(bal);
      }
    }
    if (lane == 0) misc[0] = base;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + C::kOffTmemSlot);
  const int T = misc[0];

  // warp-uniform bounded wait (every lane polls; all agree on the outcome)
  auto uwait = [&](uint32_t b_addr, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, mbar_wait(b_addr, parity));
  };
  auto aborted = [&]() -> bool { return __any_sync(0xffffffffu, misc[1] != 0); };

  if (warp == 0) {
    // ======================= TMA producer =====================================
    // Q rows of both query blocks (an absent upper block reads as zeros)
    if (elect_one()) {
      mbar_expect_tx(bar(C::kBarQ), C::kQBytes);
#pragma unroll
      for (int b = 0; b < D / 64; ++b) {
        const uint32_t dst = sbase + C::kOffQ + b * C::kBoxQBytes;
        tma_load_3d(dst, &tm_q, bar(C::kBarQ), 64 * b, qb0 * 64, bh);
        tma_load_3d(dst + 64 * 128, &tm_q, bar(C::kBarQ), 64 * b, has_hi ? qb1 * 64 : L, bh);
      }
    }
    __syncwarp();
    int k_issued = 0, v_issued = 0;
    bool h_issued = false, ok = true;
    // tile t of the list: exact block j (K, V rows) or centroid chunk c (kbar, vsum rows)
    auto load = [&](int t, bool is_k) -> bool {
      const int ns = is_k ? C::kKStages : C::kVStages;
      const int sl = t % ns;
      const uint32_t empty = bar((is_k ? C::kBarKEmpty : C::kBarVEmpty) + sl);
      const uint32_t full = bar((is_k ? C::kBarKFull : C::kBarVFull) + sl);
      if (t >= ns && !uwait(empty, ((t / ns) - 1) & 1)) return false;
      const int e = tiles[t];
      const CUtensorMap *m = e >= 0 ? (is_k ? &tm_k : &tm_v) : (is_k ? &tm_kbar : &tm_vsum);
      const int row = e >= 0 ? (e >> 2) * 64 : (-e - 1) * 64;
      const uint32_t dst = sbase + (is_k ? C::kOffK : C::kOffV) + sl * C::kTileBytes;
      if (elect_one()) {
        mbar_expect_tx(full, C::kTileBytes);
#pragma unroll
        for (int b = 0; b < D / 64; ++b) tma_load_3d(dst + b * C::kBoxKBytes, m, full, 64 * b, row, bh);
      }
      __syncwarp();
      return true;
    };
    // K runs one tile ahead of V: K_t is due at S_t, V_t only after softmax_t
    for (int t = 0; ok && t <= T; ++t) {
      if (aborted()) { ok = false; break; }
      if (t < T) {
        if (!load(t, true)) { ok = false; break; }
        k_issued = t + 1;
      }
      if (t >= 1) {
        if (!load(t - 1, false)) { ok = false; break; }
        v_issued = t;
      }
    }
    if (ok && hyd) {
      // Hbar goes into the K ring once every S = Q K^T has completed
      for (int u = (T >= C::kKStages ? T - C::kKStages : 0); ok && u < T; ++u)
        ok = uwait(bar(C::kBarKEmpty + u % C::kKStages), (u / C::kKStages) & 1);
      if (ok) {
        if (elect_one()) {
          mbar_expect_tx(bar(C::kBarHFull), C::kHbarBytes);
#pragma unroll
          for (int b = 0; b < D / 64; ++b)
            tma_load_3d(sbase + C::kOffK + b * (D * 128), &tm_hbar, bar(C::kBarHFull), 64 * b, 0, bh);
        }
        __syncwarp();
        h_issued = true;
      }
    }
    if (!ok) {
      misc[1] = 1;
      // let the copies already in flight land before the CTA exits
      uwait(bar(C::kBarQ), 0);
      for (int t = k_issued - C::kKStages; t < k_issued; ++t)
        if (t >= 0) uwait(bar(C::kBarKFull + t % C::kKStages), (t / C::kKStages) & 1);
      for (int t = v_issued - C::kVStages; t < v_issued; ++t)
        if (t >= 0) uwait(bar(C::kBarVFull + t % C::kVStages), (t / C::kVStages) & 1);
      if (h_issued) uwait(bar(C::kBarHFull), 0);
    }
  } else if (warp == 1) {
    // ======================= MMA issuer =======================================
    constexpr uint32_t kIdQK = idesc_bf16_f32(128, 64, 0, 0);
    constexpr uint32_t kIdPV = idesc_bf16_f32(128, D, 0, 1);
    bool ok = uwait(bar(C::kBarQ), 0);
    tc_fence_after();
    // descriptors are built once per buffer; a K step adds its byte offset / 16
    // to the start-address field (the field cannot carry: shared memory is
    // below 256 KB)
    const uint64_t qd0 = smem_desc_sw128(sbase + C::kOffQ, 16, 1024);
    auto q_desc = [&](int k) -> uint64_t {
      return qd0 + (uint64_t)(((k >> 2) * C::kBoxQBytes + (k & 3) * 32) >> 4);
    };
    auto issue_pv = [&](int u) -> bool {
      const int bu = u & 1, sv = u % C::kVStages;
      if (!uwait(bar(C::kBarPFull + bu), (u >> 1) & 1)) return false;
      if (!uwait(bar(C::kBarVFull + sv), (u / C::kVStages) & 1)) return false;
      tc_fence_after();
      const uint64_t vd0 = smem_desc_sw128(sbase + C::kOffV + sv * C::kTileBytes, C::kBoxKBytes, 1024);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ts(tmem + C::kColO, tmem + C::kColS + 64 * bu + kk * 8,
                 vd0 + (uint64_t)((kk * 2048) >> 4), kIdPV, (u > 0 || kk > 0) ? 1u : 0u);
        tc_commit(bar(C::kBarVEmpty + sv));
        tc_commit(bar(C::kBarODone));
      }
      __syncwarp();
      return true;
    };
    for (int t = 0; ok && t < T; ++t) {
      if (aborted()) { ok = false; break; }
      const int sk = t % C::kKStages, b = t & 1;
      if (!uwait(bar(C::kBarKFull + sk), (t / C::kKStages) & 1)) { ok = false; break; }
      tc_fence_after();
      const uint64_t kd0 = smem_desc_sw128(sbase + C::kOffK + sk * C::kTileBytes, 16, 1024);
      if (elect_one()) {
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          mma_ss(tmem + C::kColS + 64 * b, q_desc(k),
                 kd0 + (uint64_t)(((k >> 2) * C::kBoxKBytes + (k & 3) * 32) >> 4), kIdQK,
                 k > 0 ? 1u : 0u);
        tc_commit(bar(C::kBarSFull + b));
        tc_commit(bar(C::kBarKEmpty + sk));
      }
      __syncwarp();
      if (t >= 1 && !issue_pv(t - 1)) { ok = false; break; }
    }
    if (ok && T >= 1) ok = issue_pv(T - 1);
    if (ok && !hyd) {
      if (elect_one()) tc_commit(bar(C::kBarFinal));
      __syncwarp();
    }
    if (ok && hyd) {
      if (uwait(bar(C::kBarHFull), 0)) {
        tc_fence_after();
        const uint32_t hst = sbase + C::kOffK;
        if (elect_one()) {
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            mma_ss(tmem + C::kColQH, q_desc(k), smem_desc_sw128(hst + k * 2048, D * 128, 1024),
                   kIdPV, k > 0 ? 1u : 0u);
          tc_commit(bar(C::kBarFinal));
        }
        __syncwarp();
      } else {
        ok = false;
      }
    }
    if (!ok) {
      misc[1] = 1;
      // every MMA issued so far must finish before TMEM is released
      if (elect_one()) tc_commit(bar(C::kBarTeardown));
      __syncwarp();
      uwait(bar(C::kBarTeardown), 0);
    }
  } else {
    // ======================= softmax warps ====================================
    const int sp = warp & 3;                 // TMEM sub-partition of this warp
    const int row = sp * 32 + lane;          // query row in the tile = TMEM lane
    const int half = row >> 6;               // warp-uniform
    const bool exists = half == 0 || has_hi;
    const uint32_t *cbm = half ? cbm_hi : cbm_lo;
    const uint32_t lane_addr = tmem + ((uint32_t)(sp * 32) << 16);
    const float sl2 = scale * kLog2e;
    const int n_last = L - (N - 1) * 64;                 // tokens in the last 64-token tile
    const float wblk = 64.f * (float)bsub;               // n_j of a full block
    const int nc_last = L - (Nc - 1) * 64 * bsub;        // n_j of the last block
    float m_run = -INFINITY, l_run = 0.f, a_run = 0.f;
    bool ok = true;
    // waits and abort checks are made warp-uniform: TMEM access is warp-collective
    auto warp_wait = [&](uint32_t b_addr, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(b_addr, parity));
    };
    for (int t = 0; t < T; ++t) {
      if (__any_sync(0xffffffffu, misc[1] != 0)) { ok = false; break; }
      const int b = t & 1;
      if (!warp_wait(bar(C::kBarSFull + b), (t >> 1) & 1)) { ok = false; break; }
      tc_fence_after();
      const int e = tiles[t];
      const bool centroid = e < 0;
      uint64_t cmask = 0;
      bool active;
      // block-wise first order: an unselected block enters through its own
      // first-order Taylor expansion about its centroid
      const bool taylor = blockwise && exists && !centroid && ((e >> half) & 1) == 0;
      if (!exists) {
        active = false;
      } else if (!centroid) {
        active = ((e >> half) & 1) != 0 || taylor;
      } else {
        const int c = -e - 1;
        const uint32_t m0 = ~cbm[2 * c] & valid_bits(2 * c, Nc);
        const uint32_t m1 = (2 * c + 1 < cwords) ? (~cbm[2 * c + 1] & valid_bits(2 * c + 1, Nc)) : 0u;
        cmask = (uint64_t)m0 | ((uint64_t)m1 << 32);
        active = cmask != 0;
      }
      float sv[64];
      float tmax = -INFINITY;
      const uint32_t s_addr = lane_addr + C::kColS + 64 * b;
      uint32_t pk[32];
      float taylor_ell = 0.f;
      int taylor_nj = 0;
      if (active) {
        uint32_t r0[32], r1[32];
        tmem_ld_x32(s_addr, r0);
        tmem_ld_x32(s_addr + 32, r1);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          sv[i] = __uint_as_float(r0[i]);
          sv[i + 32] = __uint_as_float(r1[i]);
        }
        // columns that are not keys of this row: past the sequence end in the
        // partial last block, or centroids of blocks this half selected
        uint64_t keep = ~0ull;
        if (centroid) keep = cmask;
        else if ((e >> 2) == N - 1 && n_last < 64) keep = (1ull << n_last) - 1ull;
        if (taylor) {
          // alpha = exp(s q kbar_j) with s q kbar_j = mean of the exact logits of
          // the block; weights alpha (1 + s q k_n - s q kbar_j); D gains alpha n_j
          const int nj = popcount64(keep);
          float acc8[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) acc8[i] = 0.f;
#pragma unroll
          for (int i = 0; i < 64; ++i) acc8[i & 7] += ((keep >> i) & 1ull) ? sv[i] : 0.f;
          const float sum = ((acc8[0] + acc8[1]) + (acc8[2] + acc8[3])) +
                            ((acc8[4] + acc8[5]) + (acc8[6] + acc8[7]));
          const float mean = sum / (float)nj;
          taylor_ell = mean;
          taylor_nj = nj;
#pragma unroll
          for (int i = 0; i < 64; ++i) sv[i] = ((keep >> i) & 1ull) ? sv[i] : 0.f;
        } else if (keep != ~0ull) {
#pragma unroll
          for (int i = 0; i < 64; ++i) sv[i] = ((keep >> i) & 1ull) ? sv[i] : -INFINITY;
        }
        {
          float mx[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) mx[i] = max3f(sv[i], sv[i + 8], sv[i + 16]);
#pragma unroll
          for (int i = 0; i < 8; ++i) mx[i] = max3f(mx[i], sv[i + 24], sv[i + 32]);
#pragma unroll
          for (int i = 0; i < 8; ++i) mx[i] = max3f(mx[i], sv[i + 40], sv[i + 48]);
#pragma unroll
          for (int i = 0; i < 8; ++i) mx[i] = fmaxf(mx[i], sv[i + 56]);
          tmax = max3f(max3f(mx[0], mx[1], mx[2]), max3f(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
        }
        if (taylor) tmax = taylor_ell;
        const float m_t = tmax * sl2;                  // finite: the row has a key here
        const bool grow = m_t > m_run + 8.0f;          // lazy rescale threshold 2^8
        const bool need_o = grow && m_run != -INFINITY;
        const float f = grow ? ex2_approx(m_run - m_t) : 1.0f;  // 0 when m_run = -inf
        if (__any_sync(0xffffffffu, need_o)) {
          // O is stable once P V of the previous tile is done (P V of the tile
          // before that finished before S of this tile, by commit order)
          if (!warp_wait(bar(C::kBarODone), (t - 1) & 1)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld_x32(lane_addr + C::kColO + 32 * c, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
            tmem_st_x32(lane_addr + C::kColO + 32 * c, o);
          }
        }
        if (grow) {
          m_run = m_t;
          l_run *= f;
          a_run *= f;
        }
        if (taylor) {
          const float alpha = ex2_approx(fmaf(taylor_ell, sl2, -m_run));
          const float c1 = alpha * scale, c0 = alpha * (1.f - scale * taylor_ell);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const bool k0 = (keep >> (2 * i)) & 1ull, k1 = (keep >> (2 * i + 1)) & 1ull;
            pk[i] = pack_bf16x2(k0 ? fmaf(sv[2 * i], c1, c0) : 0.f, k1 ? fmaf(sv[2 * i + 1], c1, c0) : 0.f);
          }
          l_run += alpha * (float)taylor_nj;
        } else {
        const float neg = -m_run;
        const float2 sl2x2 = make_float2(sl2, sl2), neg2 = make_float2(neg, neg);
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                         make_float2(0.f, 0.f)};
        if (o_keep == nullptr) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float2 x = fma2(make_float2(sv[2 * i], sv[2 * i + 1]), sl2x2, neg2);
            const float2 p = make_float2(ex2_approx(x.x), ex2_approx(x.y));
            acc[i & 3] = add2(acc[i & 3], p);
            pk[i] = pack_bf16x2(p.x, p.y);
          }
        } else {
          // the denominator sums the same bf16 weights the P V product uses, so
          // o_t is normalised exactly and dout_t . o_t matches the backward's
          // sum_m P_tm dP_tm to the rounding of each weight's deviation
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float2 x = fma2(make_float2(sv[2 * i], sv[2 * i + 1]), sl2x2, neg2);
            pk[i] = pack_bf16x2(ex2_approx(x.x), ex2_approx(x.y));
            acc[i & 3] = add2(acc[i & 3], make_float2(__uint_as_float(pk[i] << 16),
                                                      __uint_as_float(pk[i] & 0xffff0000u)));
          }
        }
        const float2 s2 = add2(add2(acc[0], acc[1]), add2(acc[2], acc[3]));
        const float ps = s2.x + s2.y;
        if (centroid) {
          // weight n_j = 64 bsub except for the last block, which holds nc_last tokens
          float pl = 0.f;
          if ((-e - 1) == (Nc - 1) / 64 && nc_last < 64 * bsub) {
            const int col = (Nc - 1) % 64;
#pragma unroll
            for (int i = 0; i < 64; ++i)
              if (i == col) pl = ex2_approx(fmaf(sv[i], sl2, neg));
            if (o_keep != nullptr) pl = __bfloat162float(__float2bfloat16_rn(pl));
          }
          a_run += ps;
          l_run += wblk * ps - (wblk - (float)nc_last) * pl;
        } else {
          l_run += ps;
        }
        }  // exponential weights
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = 0u;
      }
      tmem_st_x32(s_addr, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(C::kBarPFull + b));
    }
    // ---- epilogue -----------------------------------------------------------
    if (ok && T >= 1 && !__any_sync(0xffffffffu, misc[1] != 0)) {
      const bool ready = warp_wait(bar(C::kBarFinal), 0);
      if (!ready) {
        misc[1] = 1;
      } else {
        tc_fence_after();
        const int grow_row = (half ? qb1 : qb0) * 64 + (row & 63);
        const bool store = exists && grow_row < L;
        const float inv = 1.f / l_run;
        const float fa = hyd ? scale * a_run : 0.f;
        const size_t obase = ((size_t)bh * L + (size_t)(store ? grow_row : 0)) * D;
        // natural log of D_t: the weights were 2^(s q k log2(e) - m_run), summed in l_run
        if (lse != nullptr && store)
          lse[(size_t)bh * L + grow_row] = (m_run + log2f(l_run)) * 0.6931471805599453f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32], qh[32];
          tmem_ld_x32(lane_addr + C::kColO + 32 * c, o);
          if (hyd) tmem_ld_x32(lane_addr + C::kColQH + 32 * c, qh);
          tmem_wait_ld();
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            float acc = __uint_as_float(o[i]);
            if (hyd) acc = fmaf(fa, __uint_as_float(qh[i]), acc);
            v[i] = acc * inv;
          }
          if (store && o_keep != nullptr) {
            float4 *dst = reinterpret_cast<float4 *>(o_keep + obase + 32 * c);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
          }
          if (store) {
            if (out_f32) {
              float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(out) + obase + 32 * c);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            } else {
              uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(out) + obase + 32 * c);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                dst[i] = make_uint4(pack_bf16x2(v[8 * i], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                                    pack_bf16x2(v[8 * i + 4], v[8 * i + 5]), pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
            }
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
