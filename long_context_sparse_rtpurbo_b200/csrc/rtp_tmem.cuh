// Tensor memory (sm_100a) as a per-CTA scratch for scores: a CTA allocates all 512 columns of
// its SM's tensor memory (128 lanes x 512 columns x 32 bit = 256 KB) at the start of the
// decode kernel and frees them before it exits. A warp reaches only the 32 lanes of its
// quarter (warp % 4); the four warps of a quarter split the columns (warp / 4 selects 128 of
// them), so every thread owns one lane and 128 columns.
#pragma once

#include <stdint.h>

namespace rtp {

constexpr uint32_t kTmemCols = 512;
constexpr int kTmemColsPerThread = 128;

// warp-collective (one full warp): allocate kTmemCols columns; the base address goes to the
// shared word at smem_dst
__device__ __forceinline__ void tmem_alloc(uint32_t smem_dst) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               ::"r"(smem_dst), "r"(kTmemCols) : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
// warp-collective: free the columns (after every access of the CTA has completed)
__device__ __forceinline__ void tmem_dealloc(uint32_t base) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
               ::"r"(base), "r"(kTmemCols) : "memory");
}
__device__ __forceinline__ void tmem_fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Address of this thread's column `col` (0..127): lane quarter from the warp, column block
// from warp / 4.
__device__ __forceinline__ uint32_t tmem_addr(uint32_t base, int col) {
  const int warp = threadIdx.x >> 5;
  return base + ((uint32_t)(warp & 3) << 21) + (uint32_t)((warp >> 2) * kTmemColsPerThread + col);
}

// warp-collective store / load of N consecutive 32-bit columns of each thread's lane
template <int N> struct Tmem;
template <> struct Tmem<1> {
  static __device__ __forceinline__ void st(uint32_t a, const float (&v)[1]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(a), "r"(__float_as_uint(v[0])) : "memory");
  }
  static __device__ __forceinline__ void ld(uint32_t a, float (&v)[1]) {
    uint32_t r0;
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r0) : "r"(a) : "memory");
    v[0] = __uint_as_float(r0);
  }
};
template <> struct Tmem<2> {
  static __device__ __forceinline__ void st(uint32_t a, const float (&v)[2]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x2.b32 [%0], {%1, %2};"
                 ::"r"(a), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])) : "memory");
  }
  static __device__ __forceinline__ void ld(uint32_t a, float (&v)[2]) {
    uint32_t r0, r1;
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(a) : "memory");
    v[0] = __uint_as_float(r0); v[1] = __uint_as_float(r1);
  }
};
template <> struct Tmem<4> {
  static __device__ __forceinline__ void st(uint32_t a, const float (&v)[4]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};"
                 ::"r"(a), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])),
                 "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])) : "memory");
  }
  static __device__ __forceinline__ void ld(uint32_t a, float (&v)[4]) {
    uint32_t r0, r1, r2, r3;
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(a) : "memory");
    v[0] = __uint_as_float(r0); v[1] = __uint_as_float(r1);
    v[2] = __uint_as_float(r2); v[3] = __uint_as_float(r3);
  }
};
template <> struct Tmem<8> {
  static __device__ __forceinline__ void st(uint32_t a, const float (&v)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
                 ::"r"(a), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])),
                 "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])),
                 "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
                 : "memory");
  }
  static __device__ __forceinline__ void ld(uint32_t a, float (&v)[8]) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(a) : "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
  }
};

}  // namespace rtp
