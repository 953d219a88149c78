// Packing kernels of the fused-attention step: float32 statistics -> bf16
// operands laid out for the tensor-memory-accelerator loads, and f32 -> bf16
// copies of f32 inputs (the tensor-core products run on bf16).
#pragma once

#include "pisa_common.cuh"
#include "sm100_primitives.cuh"

namespace pisa {

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

// ---------------------------------------------------------------------------
// Pairing of query blocks for the 128-row attention tiles.
//
// The fused kernel runs two query blocks per CTA and loads the union of their
// exact sets, so a partner whose selected set overlaps more costs fewer
// tensor-core tiles.  Each query block i is paired greedily (ascending i) with
// the still-unpaired block among i+1 .. i+kPairWindow whose exact set shares
// the most blocks with S_i (ties: the nearer one); when all of those are taken,
// with the next unpaired block.  Only the schedule changes: every row still
// sees exactly its own S_i and U_i.  On the Wan-like inputs the union of a
// pair's exact sets averages 1.45 k_sel with adjacent pairs, 1.25 with a
// window of 16 and 1.20 with 64.
// ---------------------------------------------------------------------------
constexpr int kPairWindow = 64;

// bm[bh][i][w]: bit j of word w set iff block 32w + j is in S_i.
__global__ void selection_bitmap_kernel(const int32_t *__restrict__ idx, int N, int k_sel,
                                        int nwords, uint32_t *__restrict__ bm) {
  extern __shared__ uint32_t words[];
  const size_t row = (size_t)blockIdx.y * N + blockIdx.x;
  for (int w = threadIdx.x; w < nwords; w += blockDim.x) words[w] = 0u;
  __syncthreads();
  for (int t = threadIdx.x; t < k_sel; t += blockDim.x) {
    const int j = idx[row * k_sel + t];
    if (j >= 0 && j < N) atomicOr(&words[j >> 5], 1u << (j & 31));
  }
  __syncthreads();
  for (int w = threadIdx.x; w < nwords; w += blockDim.x) bm[row * nwords + w] = words[w];
}

// The two preparation steps of the 64-token fused step in one launch: CTAs
// 0 .. N*BH-1 build the selection bitmap rows (as selection_bitmap_kernel),
// the rest pack the statistics (as pack_stats_kernel, grid-stride).
constexpr int kPackThreads = 128;
__global__ void __launch_bounds__(kPackThreads)
    pack_and_bitmap_kernel(const float *__restrict__ kbar, const float *__restrict__ vsum,
                           const float *__restrict__ hbar, int N, int Npad, int D, int BH,
                           __nv_bfloat16 *__restrict__ kbar16, __nv_bfloat16 *__restrict__ vsum16,
                           __nv_bfloat16 *__restrict__ hbar16, const int32_t *__restrict__ idx,
                           int k_sel, int nwords, uint32_t *__restrict__ bm) {
  extern __shared__ uint32_t words[];
  const size_t nbm = (size_t)N * BH;
  if (blockIdx.x < nbm) {
    const size_t row = blockIdx.x;     // bh * N + i
    for (int w = threadIdx.x; w < nwords; w += blockDim.x) words[w] = 0u;
    __syncthreads();
    for (int t = threadIdx.x; t < k_sel; t += blockDim.x) {
      const int j = idx[row * k_sel + t];
      if (j >= 0 && j < N) atomicOr(&words[j >> 5], 1u << (j & 31));
    }
    __syncthreads();
    for (int w = threadIdx.x; w < nwords; w += blockDim.x) bm[row * nwords + w] = words[w];
    return;
  }
  const size_t nrow = (size_t)BH * Npad * D;
  const size_t nh = (size_t)BH * D * D;
  const size_t stride = (size_t)(gridDim.x - nbm) * blockDim.x;
  for (size_t e = (blockIdx.x - nbm) * (size_t)blockDim.x + threadIdx.x; e < nrow + nh;
       e += stride) {
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

// ov[bh][i][d-1] = |S_i n S_{i+d}| for d = 1 .. kPairWindow (0 past the end).
// One CTA per 8 consecutive blocks i (a warp each, lane l takes d = l + 1 and
// l + 33).  The 72 bitmap rows they touch are staged in shared memory 32
// words at a time with coalesced loads; the row stride of 33 words keeps the
// lanes' reads of 32 different rows on 32 different banks.
static_assert(kPairWindow == 64, "two window positions per lane");
constexpr int kOvRows = 8 + kPairWindow;

__global__ void __launch_bounds__(256)
    pair_overlap_kernel(const uint32_t *__restrict__ bm, int N, int nwords,
                        uint16_t *__restrict__ ov) {
  __shared__ uint32_t rows[kOvRows][33];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int i0 = blockIdx.x * 8, bh = blockIdx.y;
  const int i = i0 + warp;
  int c0 = 0, c1 = 0;
  for (int w0 = 0; w0 < nwords; w0 += 32) {
    __syncthreads();
    for (int t = tid; t < kOvRows * 32; t += 256) {
      const int r = t >> 5, w = t & 31, row = i0 + r;
      rows[r][w] = (row < N && w0 + w < nwords) ? bm[((size_t)bh * N + row) * nwords + w0 + w] : 0u;
    }
    __syncthreads();
    const int nw = min(32, nwords - w0);
    for (int w = 0; w < nw; ++w) {
      const uint32_t a = rows[warp][w];
      c0 += __popc(a & rows[warp + 1 + lane][w]);
      c1 += __popc(a & rows[warp + 33 + lane][w]);
    }
  }
  if (i < N) {
    uint16_t *o = ov + ((size_t)bh * N + i) * kPairWindow;
    o[lane] = (uint16_t)(i + 1 + lane < N ? c0 : 0);
    o[lane + 32] = (uint16_t)(i + 33 + lane < N ? c1 : 0);
  }
}

// One CTA per head; pairs[bh][p] = (i0, i1), i1 = -1 for an unpaired block.
// Writes exactly ceil(N / 2) entries.  The head's overlap table is staged in
// shared memory first (N * kPairWindow * 2 bytes), then the greedy pass runs
// from shared memory only; with staged == 0 (tables too large for shared
// memory) the table is read from global memory instead.
// Greedy in block order: an unpaired block i takes the unpaired block in
// i + 1 .. i + kPairWindow with the largest overlap (the nearer one on equal
// overlap), else the first unpaired block past the window.  Which blocks of
// the window are paired already is a 64-bit mask in registers (bit d: block
// i + 1 + d), shifted by one per step; only partners found past the window
// go through shared memory (`used`), entering the mask when the window
// reaches them.  Each step is one warp max-reduction (redux.sync).
constexpr int kPairThreads = 256;   // all stage the table; warp 0 pairs

__global__ void __launch_bounds__(kPairThreads)
    pairing_kernel(const uint16_t *__restrict__ ov, int N, int staged,
                   int2 *__restrict__ pairs) {
  extern __shared__ __align__(16) unsigned char pair_smem[];
  const int bh = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
  const uint16_t *head = ov + (size_t)bh * N * kPairWindow;
  const uint16_t *o = head;
  unsigned char *used = pair_smem;
  if (staged) {
    uint16_t *t = reinterpret_cast<uint16_t *>(pair_smem);
    const uint4 *src = reinterpret_cast<const uint4 *>(head);
    uint4 *dst = reinterpret_cast<uint4 *>(t);
#pragma unroll 4
    for (int i = tid; i < N * kPairWindow / 8; i += kPairThreads) dst[i] = src[i];
    o = t;
    used = pair_smem + (size_t)N * kPairWindow * 2;
  }
  for (int i = tid; i < N; i += kPairThreads) used[i] = 0;
  __syncthreads();
  if (tid >= 32) return;
  int2 *out = pairs + (size_t)bh * ((N + 1) / 2);
  int np = 0;
  uint64_t ahead = 0ull;       // bit d: block i + 1 + d is paired already
  bool self = false;           // block i is paired already
  const uint64_t bit_lo = 1ull << lane, bit_hi = 1ull << (32 + lane);
  // the overlaps of the current block's window positions lane and lane + 32
  unsigned o0 = o[lane], o1 = o[32 + lane];
  for (int i = 0; i < N; ++i) {
    const unsigned n0 = i + 1 < N ? o[(size_t)(i + 1) * kPairWindow + lane] : 0u;
    const unsigned n1 = i + 1 < N ? o[(size_t)(i + 1) * kPairWindow + 32 + lane] : 0u;
    // the block entering the window next; re-read below if this step pairs
    // past the window (the only writes to `used`)
    const bool in_next = i + 1 + kPairWindow < N;
    bool next_used = in_next && used[i + 1 + kPairWindow];
    if (!self) {
      // key + 1: overlap high, then nearer partner first; 0 = no candidate
      unsigned key = 0u;
      if (i + 1 + lane < N && !(ahead & bit_lo)) key = ((o0 << 8) | (255u - lane)) + 1u;
      if (i + 33 + lane < N && !(ahead & bit_hi))
        key = max(key, ((o1 << 8) | (223u - lane)) + 1u);
      const unsigned best = __reduce_max_sync(0xffffffffu, key);
      int partner = -1;
      if (best > 0u) {
        const int dd = 255 - (int)((best - 1u) & 255u);
        partner = i + 1 + dd;
        ahead |= 1ull << dd;
      } else {
        for (int jj = i + 1 + kPairWindow; jj < N; ++jj)
          if (!used[jj]) { partner = jj; break; }
        __syncwarp();
        if (lane == 0 && partner >= 0) used[partner] = 1;
        __syncwarp();
        next_used = in_next && used[i + 1 + kPairWindow];
      }
      if (lane == 0) out[np] = make_int2(i, partner);
      ++np;
    }
    // slide the window by one block
    self = ahead & 1ull;
    ahead >>= 1;
    if (next_used) ahead |= 1ull << (kPairWindow - 1);
    o0 = n0;
    o1 = n1;
  }
}

// Self-test of the error path of the bounded waits: one warp waits on an
// mbarrier that nothing ever completes, with a short limit.  The wait gives up,
// records the timeout in the device status word and the kernel returns.
__global__ void wait_timeout_selftest_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t barrier;
  const uint32_t b = smem_u32(&barrier);
  if (threadIdx.x == 0) {
    sm100::mbar_init(b, 1);
    sm100::fence_mbar_init();
  }
  __syncwarp();
  sm100::mbar_wait(b, 0, limit_ns);
}

}  // namespace pisa
