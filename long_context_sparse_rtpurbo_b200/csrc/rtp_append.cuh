// Append step: RoPE'd key, value and 16-dim index key of new tokens.
//
// "Full Attention Strikes Back" (paper text) §2.2 eq. (1): k_n = R(n) k; §3.2 eq. (4): the
// index side of the score is W^K k^pre, computed on the pre-RoPE key. Both are evaluated in
// double precision and rounded once to the bf16 cache format.
#pragma once

#include "rtp_common.cuh"

namespace rtp {

struct LayerShape {
  int B, Hq, Hkv, G, n_ret, n_loc, sinks, window, ring;
  int64_t T_total, maxN;
  double rope_base;
  double theta[kD / 2];     // base^(-2i/d), computed on the host
  int16_t slot[kMaxHkv];    // kv head -> slot (>= 0 retrieval, < 0 local: -1 - x)
  int16_t ret_kv[kMaxHkv];  // retrieval slot -> kv head
  int16_t loc_kv[kMaxHkv];  // local slot -> kv head
};

struct CachePtrs {
  uint16_t *k_ret, *v_ret, *idx, *k_loc, *v_loc;
  const int64_t* seq_off;
  const int32_t* seq_cap;
};

// sin and cos of pos * theta in double precision, after an explicit reduction of the angle
// modulo 2 pi (two-constant Cody-Waite split of 2 pi), so the library sincos runs on |r| <= pi.
__device__ __forceinline__ void rope_sincos(double pos, double theta, double* s, double* c) {
  const double x = pos * theta;
  const double k = rint(x * 0.15915494309189535);
  double r = fma(-k, 6.283185307179586, x);
  r = fma(-k, 2.4492935982947064e-16, r);
  sincos(r, s, c);
}

// The same angle reduction in double, then single-precision sin and cos of the reduced angle
// (|r| <= pi): for the query rotation, which is used in single precision anyway.
__device__ __forceinline__ void rope_sincosf(double pos, double theta, float* s, float* c) {
  const double x = pos * theta;
  const double k = rint(x * 0.15915494309189535);
  double r = fma(-k, 6.283185307179586, x);
  r = fma(-k, 2.4492935982947064e-16, r);
  sincosf((float)r, s, c);
}

// One CTA of 128 threads appends kAppendTok consecutive tokens of one (sequence, KV head).
constexpr int kAppendTok = 4;

__global__ void __launch_bounds__(128)
append_kernel(LayerShape L, CachePtrs C, const uint16_t* __restrict__ k_pre,
              const uint16_t* __restrict__ v, const float* __restrict__ w_kidx,
              const int32_t* __restrict__ start_pos, const int32_t* __restrict__ n_new_b,
              int n_new, int* status) {
  const int b = blockIdx.y, g = blockIdx.z;
  const int t = threadIdx.x;
  const int nb = n_new_b ? min(max(n_new_b[b], 0), n_new) : n_new;
  const int j0 = blockIdx.x * kAppendTok;
  if (j0 >= nb) return;
  const int64_t p0 = start_pos[b];
  const int64_t end = p0 + nb;
  const int cap = C.seq_cap[b];
  const int64_t off = C.seq_off[b];
  if (p0 < 0 || (L.n_ret > 0 && (off < 0 || off + (int64_t)cap > L.T_total))) {
    if (t == 0 && blockIdx.x == 0 && g == 0) set_status(status, -6);
    return;
  }
  const int s = L.slot[g];
  __shared__ double part[8][16];
  const int i = t & 63;
  const double th = L.theta[i];
  float wcol[16];                        // W_kidx[g][kq*16 + e][o] for this thread's (o, kq)
  const int o = t & 15, kq = t >> 4;
  if (s >= 0) {
#pragma unroll
    for (int e = 0; e < 16; ++e) wcol[e] = __ldg(w_kidx + ((int64_t)g * kD + kq * 16 + e) * kR + o);
  }
  for (int jj = 0; jj < kAppendTok; ++jj) {
    const int j = j0 + jj;
    if (j >= nb) break;                   // uniform over the CTA
    const int64_t pos = p0 + j;
    const uint16_t* kp = k_pre + (((int64_t)b * n_new + j) * L.Hkv + g) * kD;
    const uint16_t* vp = v + (((int64_t)b * n_new + j) * L.Hkv + g) * kD;
    uint16_t *kdst, *vdst, *idst = nullptr;
    if (s >= 0) {
      if (pos >= cap) {
        if (t == 0) set_status(status, -6);
        continue;
      }
      const int64_t row = (int64_t)s * L.T_total + off + pos;
      kdst = C.k_ret + row * kD;
      vdst = C.v_ret + row * kD;
      idst = C.idx + row * kR;
    } else {
      if (pos >= L.sinks && pos < end - L.window) continue;   // overwritten later in this call
      const int x = -1 - s;
      const int64_t rr = pos < L.sinks ? pos : L.sinks + (pos - L.sinks) % L.window;
      const int64_t row = ((int64_t)x * L.B + b) * L.ring + rr;
      kdst = C.k_loc + row * kD;
      vdst = C.v_loc + row * kD;
    }
    double sn, cs;
    rope_sincos((double)pos, th, &sn, &cs);
    const double xa = bf1(kp[i]), xb = bf1(kp[i + 64]);
    const double r = (t < 64) ? (xa * cs - xb * sn) : (xa * sn + xb * cs);
    kdst[t] = d2bf_rn(r);
    vdst[t] = vp[t];
    if (idst) {                           // uniform over the CTA
      double acc = 0.0;
#pragma unroll
      for (int e = 0; e < 16; ++e) acc = fma((double)bf1(kp[kq * 16 + e]), (double)wcol[e], acc);
      part[kq][o] = acc;
      __syncthreads();
      if (t < 16) {
        double sum = part[0][t];
#pragma unroll
        for (int k2 = 1; k2 < 8; ++k2) sum += part[k2][t];
        idst[t] = d2bf_rn(sum);
      }
      __syncthreads();
    }
  }
}

// The decode token of one (sequence b, KV head g) at position pos, written by a whole CTA of
// nthreads >= 128 threads inside another kernel: the arithmetic of append_kernel for one token
// (threads 0..127 compute; every thread passes the barriers). k_row / v_row: its pre-RoPE key
// and value; part: 8 x 16 doubles of shared memory; idx_patch (shared, nullable) also receives
// the index row. The caller checked pos < seq_cap[b].
__device__ __noinline__ void append_token(const LayerShape& L, const CachePtrs& C,
                                          const uint16_t* k_row, const uint16_t* v_row,
                                          const float* w_kidx, int b, int g, int64_t pos,
                                          double* part, uint16_t* idx_patch) {
  const int t = threadIdx.x;
  const int s = L.slot[g];
  uint16_t *kdst = nullptr, *vdst = nullptr, *idst = nullptr;
  if (s >= 0) {
    const int64_t row = (int64_t)s * L.T_total + C.seq_off[b] + pos;
    kdst = C.k_ret + row * kD;
    vdst = C.v_ret + row * kD;
    idst = C.idx + row * kR;
  } else {
    const int64_t rr = pos < L.sinks ? pos : L.sinks + (pos - L.sinks) % L.window;
    const int64_t row = ((int64_t)(-1 - s) * L.B + b) * L.ring + rr;
    kdst = C.k_loc + row * kD;
    vdst = C.v_loc + row * kD;
  }
  if (t < kD) {
    const int i = t & 63;
    double sn, cs;
    rope_sincos((double)pos, L.theta[i], &sn, &cs);
    const double xa = bf1(k_row[i]), xb = bf1(k_row[i + 64]);
    const double r = (t < 64) ? (xa * cs - xb * sn) : (xa * sn + xb * cs);
    kdst[t] = d2bf_rn(r);
    vdst[t] = v_row[t];
    if (idst) {
      const int o = t & 15, kq = t >> 4;
      double acc = 0.0;
#pragma unroll
      for (int e = 0; e < 16; ++e)
        acc = fma((double)bf1(k_row[kq * 16 + e]),
                  (double)__ldg(w_kidx + ((int64_t)g * kD + kq * 16 + e) * kR + o), acc);
      part[kq * 16 + o] = acc;
    }
  }
  __syncthreads();
  if (idst && t < kR) {
    double sum = part[t];
#pragma unroll
    for (int k2 = 1; k2 < 8; ++k2) sum += part[k2 * 16 + t];
    const uint16_t bits = d2bf_rn(sum);
    idst[t] = bits;
    if (idx_patch) idx_patch[t] = bits;
  }
  __threadfence();                        // visible to this CTA's copies and, after its next
  __syncthreads();                        // arrival, to every other CTA
}

}  // namespace rtp
