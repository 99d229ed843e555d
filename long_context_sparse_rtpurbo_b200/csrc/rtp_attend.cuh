// Exact softmax attention of the G query heads of one KV head over a list of K/V rows
// ("Full Attention Strikes Back" (paper text) §3.2 eq. (5): O = sum_n softmax(q^T k_n / sqrt(d)) v_n).
//
// Layout on the SM: a half-warp (16 lanes) owns one row per step, each lane 8 of the 128
// channels (one 16-byte load of K and one of V). A half-warp keeps kRows rows in flight. The
// kRows x G partial dot products of a lane are reduced over the 16 lanes by recursive halving
// (each step exchanges half of the remaining values), so every lane ends with one complete
// logit; the probabilities are then broadcast for the V update. Softmax state (running max,
// sum, 8-channel accumulator per head) is kept per half-warp in the log2 domain (q carries
// log2(e)/sqrt(d)) and merged across half-warps at the end.
#pragma once

#include "rtp_common.cuh"

namespace rtp {

template <int G> struct AttnCfg {
  static constexpr int kRows = (G >= 8) ? 2 : 4;          // rows in flight per half-warp
  static constexpr int kVals = kRows * G;                 // partial dots per lane
};

// Recursive-halving reduction of n values over the 16 lanes of a half-warp. On exit v[0] of
// lane hl holds the full sum of value index (hl >> (4 - log2 n)) (n <= 16).
template <int N>
__device__ __forceinline__ void halving_reduce(float (&v)[N], int hl) {
  static_assert(N >= 1 && N <= 16 && (N & (N - 1)) == 0, "power of two up to 16");
  int n = N;
#pragma unroll
  for (int m = 8; m >= 1; m >>= 1) {
    if (n > 1) {
      const bool up = (hl & m) != 0;
#pragma unroll
      for (int i = 0; i < N / 2; ++i) {
        if (i < n / 2) {
          const float send = up ? v[i] : v[i + n / 2];
          const float keep = up ? v[i + n / 2] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
      }
      n >>= 1;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], m);
    }
  }
}

// Softmax state of one half-warp.
template <int G> struct AttnState {
  float m[G], l[G], acc[G][8];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m[h] = -INFINITY;
      l[h] = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[h][e] = 0.f;
    }
  }
};

// One step of kRows rows for a half-warp. kp/vp: row pointers (lane-independent within the
// half-warp), mask: heads that attend each row (0 for an invalid row).
template <int G>
__device__ __forceinline__ void attend_step(AttnState<G>& st, const float (&q)[G][8],
                                            const uint16_t* const (&kp)[AttnCfg<G>::kRows],
                                            const uint16_t* const (&vp)[AttnCfg<G>::kRows],
                                            const uint32_t (&mask)[AttnCfg<G>::kRows], int hl) {
  constexpr int R = AttnCfg<G>::kRows;
  constexpr int V = AttnCfg<G>::kVals;
  uint4 kw[R], vw[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    kw[r] = mask[r] ? ld_stream(kp[r] + hl * 8) : make_uint4(0, 0, 0, 0);
    vw[r] = mask[r] ? ld_stream(vp[r] + hl * 8) : make_uint4(0, 0, 0, 0);
  }
  float d[V];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    float k[8];
    unpack8(kw[r], k);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float a = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) a = fmaf(q[h][e], k[e], a);
      d[r * G + h] = a;
    }
  }
  halving_reduce<V>(d, hl);
  // lane hl holds the logit of value index (r, h) = (hl * V / 16) split as r * G + h
  constexpr int kShift = (V == 16) ? 0 : (V == 8 ? 1 : (V == 4 ? 2 : (V == 2 ? 3 : 4)));
  const int vi = hl >> kShift;
  const int my_r = vi / G, my_h = vi % G;
  uint32_t my_mask = 0;
#pragma unroll
  for (int r = 0; r < R; ++r) my_mask = (r == my_r) ? mask[r] : my_mask;
  float logit = ((my_mask >> my_h) & 1u) ? d[0] : -INFINITY;
  // block max per head over the R rows: lanes holding the same head differ in the row bits
  float bm = logit;
#pragma unroll
  for (int o = 1; o < R; o <<= 1) {
    const int lanebit = (o * G) << kShift;
    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, lanebit));
  }
  // new running max and p for my value
  float mnew_my = -INFINITY;
#pragma unroll
  for (int h = 0; h < G; ++h) mnew_my = (h == my_h) ? fmaxf(st.m[h], bm) : mnew_my;
  const float p_my = (logit == -INFINITY) ? 0.f : exp2f(logit - mnew_my);
  // broadcast: every lane gets p of each (r, h) and the block max of each head
  const int base = (threadIdx.x & 31) & 16;
  float scale[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float bmh = __shfl_sync(0xffffffffu, bm, base + ((h) << kShift));
    const float mn = fmaxf(st.m[h], bmh);
    scale[h] = (mn == -INFINITY) ? 1.f : exp2f(st.m[h] - mn);
    st.m[h] = mn;
    st.l[h] *= scale[h];
#pragma unroll
    for (int e = 0; e < 8; ++e) st.acc[h][e] *= scale[h];
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    float v[8];
    unpack8(vw[r], v);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float p = __shfl_sync(0xffffffffu, p_my, base + ((r * G + h) << kShift));
      st.l[h] += p;
#pragma unroll
      for (int e = 0; e < 8; ++e) st.acc[h][e] = fmaf(p, v[e], st.acc[h][e]);
    }
  }
}

// Merges the per-half-warp states of a CTA of nthreads threads into res[G][2 + 128]
// (M, L, A). scratch: >= (nthreads / 32) * G * 128 floats plus 2 * (nthreads / 32) * G.
template <int G>
__device__ __forceinline__ void attend_merge(AttnState<G>& st, float* scratch, float* res,
                                             int nthreads) {
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5, hl = lane & 15;
  const int nw = nthreads >> 5;
  // merge the two half-warps of each warp with shuffles
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float mo = __shfl_xor_sync(0xffffffffu, st.m[h], 16);
    const float lo = __shfl_xor_sync(0xffffffffu, st.l[h], 16);
    const float mn = fmaxf(st.m[h], mo);
    const float fa = (mn == -INFINITY) ? 0.f : exp2f(st.m[h] - mn);
    const float fb = (mn == -INFINITY) ? 0.f : exp2f(mo - mn);
    st.l[h] = st.l[h] * fa + lo * fb;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float ao = __shfl_xor_sync(0xffffffffu, st.acc[h][e], 16);
      st.acc[h][e] = st.acc[h][e] * fa + ao * fb;
    }
    st.m[h] = mn;
  }
  float* sm_m = scratch + nw * G * kD;
  float* sm_l = sm_m + nw * G;
  if (lane < 16) {
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int e = 0; e < 8; ++e) scratch[(warp * G + h) * kD + hl * 8 + e] = st.acc[h][e];
    if (hl == 0) {
#pragma unroll
      for (int h = 0; h < G; ++h) { sm_m[warp * G + h] = st.m[h]; sm_l[warp * G + h] = st.l[h]; }
    }
  }
  __syncthreads();
  for (int o = t; o < G * kD; o += nthreads) {
    const int h = o / kD, dch = o % kD;
    float M = -INFINITY;
    for (int w = 0; w < nw; ++w) M = fmaxf(M, sm_m[w * G + h]);
    float Ls = 0.f, A = 0.f;
    if (M != -INFINITY) {
      for (int w = 0; w < nw; ++w) {
        const float f = exp2f(sm_m[w * G + h] - M);
        Ls += sm_l[w * G + h] * f;
        A += scratch[(w * G + h) * kD + dch] * f;
      }
    }
    res[h * (kD + 2) + 2 + dch] = A;
    if (dch == 0) { res[h * (kD + 2)] = M; res[h * (kD + 2) + 1] = Ls; }
  }
  __syncthreads();
}

// Merges n partial states (stride G*(2+128) floats, in global memory written by other CTAs)
// into one; result into `dst` (global, same format) or, when out_rows is given, the bf16
// output rows of the G heads.
template <int G>
__device__ __forceinline__ void merge_partials(const float* parts, int n, float* dst,
                                               uint16_t* out_rows, int nthreads) {
  for (int o = threadIdx.x; o < G * kD; o += nthreads) {
    const int h = o / kD, dch = o % kD;
    float M = -INFINITY;
    for (int i = 0; i < n; ++i) M = fmaxf(M, __ldcg(parts + ((int64_t)i * G + h) * (kD + 2)));
    float Ls = 0.f, A = 0.f;
    if (M != -INFINITY) {
      for (int i = 0; i < n; ++i) {
        const float* pp = parts + ((int64_t)i * G + h) * (kD + 2);
        const float mi = __ldcg(pp);
        if (mi == -INFINITY) continue;
        const float f = exp2f(mi - M);
        Ls += __ldcg(pp + 1) * f;
        A += __ldcg(pp + 2 + dch) * f;
      }
    }
    if (out_rows) {
      out_rows[(int64_t)h * kD + dch] = f2bf_rn(Ls > 0.f ? A / Ls : 0.f);
    } else {
      dst[h * (kD + 2) + 2 + dch] = A;
      if (dch == 0) { dst[h * (kD + 2)] = M; dst[h * (kD + 2) + 1] = Ls; }
    }
  }
}

}  // namespace rtp
