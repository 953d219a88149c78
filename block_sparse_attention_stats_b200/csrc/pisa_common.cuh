// Shared device helpers of libpisa (sm_100a).  libpisa is one translation
// unit: pisa_api.cu includes every kernel header, so no relocatable device
// code is needed.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pisa.h"

namespace pisa {

// ---------------------------------------------------------------------------
// device status word: bit 0 = range check failed, bit 1 = bounded wait ran out
// ---------------------------------------------------------------------------
enum : unsigned { kDevErrRange = 1u, kDevErrTimeout = 2u };
__device__ unsigned g_device_status;

__device__ __forceinline__ void report_device_error(unsigned bits) {
  atomicOr(&g_device_status, bits);
}

// ---------------------------------------------------------------------------
// small math
// ---------------------------------------------------------------------------
constexpr float kLog2e = 1.4426950408889634f;

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ __forceinline__ size_t align_up(size_t x, size_t a) {
  return (x + a - 1) / a * a;
}

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

__device__ __forceinline__ int popcount64(uint64_t x) { return __popcll(x); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// ---------------------------------------------------------------------------
// shared-memory addressing and asynchronous copies
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte global->shared copy; src_bytes < 16 zero-fills the rest.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void *src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n"); }
template <int N> __device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

// Row-major tile of ROWS x COLS 16-bit elements in shared memory with the
// 16-byte chunks of each row XOR-swizzled by (row & 7): conflict-free for
// ldmatrix reads of 8 consecutive rows at one column offset.
template <int COLS> struct SwizzledTile {
  static constexpr int kChunks = COLS / 8;  // 16-byte chunks per row
  static_assert(kChunks >= 8, "rows must be at least 128 bytes");
  __device__ __forceinline__ static uint32_t offset(int row, int col) {  // bytes
    int chunk = (col >> 3) ^ (row & 7);
    return static_cast<uint32_t>((row * kChunks + chunk) * 16 + (col & 7) * 2);
  }
};

// ---------------------------------------------------------------------------
// warp-level tensor-core primitives (mma.sync m16n8k16, bf16 -> f32)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t &r0, uint32_t &r1,
                                            uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t &r0, uint32_t &r1,
                                                  uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------------------
// host-side helpers
// ---------------------------------------------------------------------------
void set_last_error(cudaError_t e);
pisa_status check_launch();

}  // namespace pisa
