// Shared device helpers of librtp (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace rtp {

constexpr int kD = 128;        // head dim
constexpr int kR = 16;         // index projection rank
constexpr int kBins = 256;     // histogram bins per query head
constexpr int kMaxHkv = 64;
constexpr int kThreads = 256;  // threads of the decode kernels
constexpr float kLog2e = 1.4426950408889634f;
// Fixed-point scale of the histogram mass: exp(s - max) in (0, 1] is stored as an integer
// multiple of 2^-40, so bin sums are exact and independent of summation order.
constexpr float kMassScale = 1099511627776.0f;  // 2^40

// bf16 bit patterns -> float
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float bf1(uint16_t b) { return __uint_as_float(((uint32_t)b) << 16); }

__device__ __forceinline__ uint16_t f2bf_rn(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

// double -> bf16, round to nearest even: round to float32 with round-to-odd first (24 bits keep
// enough guard bits that the second rounding is exact), then float32 -> bf16 nearest-even.
__device__ __forceinline__ uint16_t d2bf_rn(double x) {
  float f = __double2float_rz(x);
  if ((double)f != x) f = __uint_as_float(__float_as_uint(f) | 1u);
  return f2bf_rn(f);
}

// Order-preserving float <-> uint32 map (for integer atomics on floats).
__device__ __forceinline__ uint32_t f2ord(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float ord2f(uint32_t o) {
  uint32_t u = (o & 0x80000000u) ? (o & 0x7fffffffu) : ~o;
  return __uint_as_float(u);
}

__device__ __forceinline__ void unpack8(const uint4& w, float* x) {
  x[0] = bf_lo(w.x); x[1] = bf_hi(w.x);
  x[2] = bf_lo(w.y); x[3] = bf_hi(w.y);
  x[4] = bf_lo(w.z); x[5] = bf_hi(w.z);
  x[6] = bf_lo(w.w); x[7] = bf_hi(w.w);
}

// Streaming 16-byte load that does not allocate in L1 (data read once).
__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Sticky device status: the first error code wins.
__device__ __forceinline__ void set_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Bounds checks of data-dependent indices (the debug build that stands in for a memory checker,
// compiled with -DRTP_CHECKS): true when `cond` holds; otherwise records RTP_ECHECK (-7) in the
// status word and returns false, and the caller redirects the access to a valid location that
// contributes nothing. Release builds compile every check to `true`.
#ifdef RTP_CHECKS
#define RTP_CHECK(cond, status) ((cond) ? true : (::rtp::set_status((status), -7), false))
#else
#define RTP_CHECK(cond, status) true
#endif

}  // namespace rtp
