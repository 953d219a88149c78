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
// Kernels (11 launches per call; 12 when the forward's float32 output is
// given, which replaces the dq kernel's first sweep by bwd_delta_kernel):
//   bwd_pack_centroids_kernel (this file) bf16 kbar_j and vbar_j = vsum_j / n_j,
//                             rows >= N zero
//   selection_bitmap_kernel, pair_overlap_kernel, pairing_kernel (k3_pack.cuh)
//                             the forward's query-block pairing
//   pad_lse_kernel, kvlist_kernel (x2), kvlist_scan_kernel (k8_bwd_kv_tc.cuh)
//                             padded lse; per key-block pair, the ascending list
//                             of query blocks that selected either block
//   bwd_delta_kernel          (this file, when the forward's float32 output
//                             o is given) Delta_t = dout_t . o_t
//   bwd_dq_tc_kernel          (k7_bwd_dq_tc.cuh, tcgen05) one CTA per pair of
//                             query blocks over their exact tiles and the
//                             centroid chunks: without a given Delta, a first
//                             sweep forms Delta_t = sum_m P_tm dP_tm; then dq
//   bwd_kv_tc_kernel<true>    (tcgen05) one CTA per 128 centroids, over every
//                             query block -> dkbar_j / n_j, dvbar_j / n_j (float32)
//   bwd_kv_tc_kernel<false>   (tcgen05) one CTA per pair of key blocks, over the
//                             query blocks that selected either -> dk, dv, plus
//                             the centroid terms
// No atomics: every output element is written by one CTA, so the results are
// reproducible bit for bit.
#pragma once

#include "pisa_common.cuh"
#include "sm100_primitives.cuh"

namespace pisa {

// ---------------------------------------------------------------------------
// preprocessing
// ---------------------------------------------------------------------------
// kbar16[bh, j] = bf16(kbar_j), vbar16[bh, j] = bf16(vsum_j / n_j); rows N..Npad-1
// zero.  N blocks of block_size tokens (the last may be partial).
__global__ void bwd_pack_centroids_kernel(const float *__restrict__ kbar,
                                          const float *__restrict__ vsum, int N, int Npad, int D,
                                          int BH, int L, int block_size,
                                          __nv_bfloat16 *__restrict__ kbar16,
                                          __nv_bfloat16 *__restrict__ vbar16) {
  const size_t n = (size_t)BH * Npad * D;
  const float inv_full = 1.f / (float)block_size;
  const float inv_last = 1.f / (float)(L - block_size * (N - 1));
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n;
       e += (size_t)gridDim.x * blockDim.x) {
    const size_t bh = e / ((size_t)Npad * D), rem = e % ((size_t)Npad * D);
    const int j = (int)(rem / D), c = (int)(rem % D);
    const bool ok = j < N;
    const size_t src = (bh * N + (ok ? j : 0)) * D + c;
    const float inv_n = j == N - 1 ? inv_last : inv_full;
    kbar16[e] = __float2bfloat16_rn(ok ? kbar[src] : 0.f);
    vbar16[e] = __float2bfloat16_rn(ok ? vsum[src] * inv_n : 0.f);
  }
}

// Delta_t = dout_t . o_t for t < L from the forward's float32 output o (the
// same quantity as sum_m P_tm dP_tm, since o_t = sum_m P_tm value_m), 0 for
// the padding rows L .. Lpad-1 of each head.  One warp per row; D a multiple
// of 64; dout 8-byte and o 16-byte aligned.
__global__ void bwd_delta_kernel(const __nv_bfloat16 *__restrict__ dout,
                                 const float *__restrict__ o, int L, int Lpad, int D, int BH,
                                 float *__restrict__ delta) {
  const size_t rows = (size_t)BH * Lpad;
  const int lane = threadIdx.x & 31;
  const size_t warps = ((size_t)gridDim.x * blockDim.x) >> 5;
  for (size_t r = (blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5; r < rows; r += warps) {
    const size_t bh = r / Lpad;
    const int t = (int)(r % Lpad);
    float acc = 0.f;
    if (t < L) {
      const size_t base = (bh * L + t) * D;
      for (int c = 4 * lane; c < D; c += 128) {
        const uint2 g = *reinterpret_cast<const uint2 *>(dout + base + c);
        const float4 x = *reinterpret_cast<const float4 *>(o + base + c);
        acc = fmaf(__uint_as_float(g.x << 16), x.x, acc);
        acc = fmaf(__uint_as_float(g.x & 0xffff0000u), x.y, acc);
        acc = fmaf(__uint_as_float(g.y << 16), x.z, acc);
        acc = fmaf(__uint_as_float(g.y & 0xffff0000u), x.w, acc);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) delta[r] = acc;
  }
}

}  // namespace pisa
