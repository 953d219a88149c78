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

// ov[bh][i][d-1] = |S_i n S_{i+d}| for d = 1 .. kPairWindow (0 past the end).
__global__ void pair_overlap_kernel(const uint32_t *__restrict__ bm, int N, int nwords,
                                    uint16_t *__restrict__ ov) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * (blockDim.x >> 5) + warp;
  const int bh = blockIdx.y;
  if (i >= N) return;
  const uint32_t *a = bm + ((size_t)bh * N + i) * nwords;
  for (int dd = lane; dd < kPairWindow; dd += 32) {
    const int j = i + 1 + dd;
    int cnt = 0;
    if (j < N) {
      const uint32_t *b = bm + ((size_t)bh * N + j) * nwords;
      for (int w = 0; w < nwords; ++w) cnt += __popc(a[w] & b[w]);
    }
    ov[((size_t)bh * N + i) * kPairWindow + dd] = (uint16_t)cnt;
  }
}

// One warp per head; pairs[bh][p] = (i0, i1), i1 = -1 for an unpaired block.
// Writes exactly ceil(N / 2) entries.  The head's overlap table is staged in
// shared memory first (N * kPairWindow * 2 bytes), then the greedy pass runs
// from shared memory only.
// With staged == 0 (tables too large for shared memory) the table is read
// from global memory instead.
__global__ void pairing_kernel(const uint16_t *__restrict__ ov, int N, int staged,
                               int2 *__restrict__ pairs) {
  extern __shared__ __align__(16) unsigned char pair_smem[];
  const int bh = blockIdx.x, lane = threadIdx.x;
  const uint16_t *head = ov + (size_t)bh * N * kPairWindow;
  const uint16_t *o = head;
  unsigned char *used = pair_smem;
  if (staged) {
    uint16_t *t = reinterpret_cast<uint16_t *>(pair_smem);
    const uint4 *src = reinterpret_cast<const uint4 *>(head);
    uint4 *dst = reinterpret_cast<uint4 *>(t);
    for (int i = lane; i < N * kPairWindow / 8; i += 32) dst[i] = src[i];
    o = t;
    used = pair_smem + (size_t)N * kPairWindow * 2;
  }
  for (int i = lane; i < N; i += 32) used[i] = 0;
  __syncwarp();
  int2 *out = pairs + (size_t)bh * ((N + 1) / 2);
  int np = 0;
  for (int i = 0; i < N; ++i) {
    if (used[i]) continue;  // uniform: every lane reads the same byte
    // key: overlap high, then nearer partner first; lane l looks at distances
    // l + 1 and l + 33
    int best = -1;
    for (int dd = lane; dd < kPairWindow; dd += 32) {
      const int j = i + 1 + dd;
      if (j < N && !used[j])
        best = max(best, ((int)o[(size_t)i * kPairWindow + dd] << 8) | (255 - dd));
    }
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) best = max(best, __shfl_xor_sync(0xffffffffu, best, s));
    int partner = -1;
    if (best >= 0) {
      partner = i + 1 + (255 - (best & 255));
    } else {
      for (int jj = i + 1 + kPairWindow; jj < N; ++jj)
        if (!used[jj]) { partner = jj; break; }
    }
    __syncwarp();
    if (lane == 0) {
      used[i] = 1;
      if (partner >= 0) used[partner] = 1;
      out[np] = make_int2(i, partner);
    }
    __syncwarp();
    ++np;
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
