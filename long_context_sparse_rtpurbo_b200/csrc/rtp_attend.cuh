// Exact softmax attention of the G query heads of one KV head over a list of K/V rows
// ("Full Attention Strikes Back" (paper text) §3.2 eq. (5): O = sum_n softmax(q^T k_n / sqrt(d)) v_n).
//
// Layout on the SM: a half-warp (16 lanes) owns kRows rows per step, each lane 8 of the 128
// channels (16 bytes of K and of V per row). Rows are staged in shared memory with cp.async
// (16 bytes per lane, L2-only), two steps deep, so the loads of step i+1 are in flight while
// step i is computed and no registers are held by loads in flight. A lane only ever reads the
// bytes it copied itself, so no barrier is needed between copy and use. The kRows x G partial
// dot products of a lane are reduced over the 16 lanes by recursive halving (each step
// exchanges half of the remaining values), so every lane ends with one complete logit; the
// probabilities are then broadcast for the V update. Softmax state (running max, sum,
// 8-channel accumulator per head) is kept per half-warp in the log2 domain (q carries
// log2(e)/sqrt(d)) and merged across half-warps at the end.
#pragma once

#include "rtp_common.cuh"

namespace rtp {

template <int G> struct AttnCfg {
  static constexpr int kRows = 2;                         // rows per half-warp per step
  static constexpr int kVals = kRows * G;                 // partial dots per lane
  static constexpr int kStages = 2;
  // staging bytes for a CTA of nthreads threads
  static constexpr int stage_bytes(int nthreads) { return kStages * (nthreads / 16) * kRows * 512; }
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

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

// Softmax state of one half-warp; the accumulator holds channel pairs (2e, 2e + 1), so the
// V update is one packed f32x2 multiply-add per pair.
template <int G> struct AttnState {
  float m[G], l[G];
  float2 a2[G][4];
  __device__ __forceinline__ float& acc(int h, int e) { return (&a2[h][e >> 1].x)[e & 1]; }
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m[h] = -INFINITY;
      l[h] = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) a2[h][e] = make_float2(0.f, 0.f);
    }
  }
};

// 8 bf16 -> 4 packed channel pairs
__device__ __forceinline__ void unpack_pairs(const uint4& w, float2 (&f)[4]) {
  f[0] = make_float2(bf_lo(w.x), bf_hi(w.x));
  f[1] = make_float2(bf_lo(w.y), bf_hi(w.y));
  f[2] = make_float2(bf_lo(w.z), bf_hi(w.z));
  f[3] = make_float2(bf_lo(w.w), bf_hi(w.w));
}

// One step of kRows staged rows for a half-warp; kw/vw: this lane's 16 bytes of each row
// (zero for rows no head attends), mask: heads that attend each row.
template <int G>
__device__ __forceinline__ void attend_step(AttnState<G>& st, const float2 (&q)[G][4],
                                            const uint4 (&kw)[AttnCfg<G>::kRows],
                                            const uint4 (&vw)[AttnCfg<G>::kRows],
                                            const uint32_t (&mask)[AttnCfg<G>::kRows], int hl) {
  constexpr int R = AttnCfg<G>::kRows;
  constexpr int V = AttnCfg<G>::kVals;
  float d[V];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    float2 k[4];
    unpack_pairs(kw[r], k);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float2 a = __fmul2_rn(q[h][0], k[0]);
#pragma unroll
      for (int e = 1; e < 4; ++e) a = __ffma2_rn(q[h][e], k[e], a);
      d[r * G + h] = a.x + a.y;
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
  const float logit = ((my_mask >> my_h) & 1u) ? d[0] : -INFINITY;
  // block max per head over the R rows: lanes holding the same head differ in the row bits
  float bm = logit;
#pragma unroll
  for (int o = 1; o < R; o <<= 1) {
    const int lanebit = (o * G) << kShift;
    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, lanebit));
  }
  float mnew_my = -INFINITY;
#pragma unroll
  for (int h = 0; h < G; ++h) mnew_my = (h == my_h) ? fmaxf(st.m[h], bm) : mnew_my;
  const float p_my = (logit == -INFINITY) ? 0.f : exp2f(logit - mnew_my);
  // broadcast: every lane gets p of each (r, h) and the block max of each head
  const int base = (threadIdx.x & 31) & 16;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float bmh = __shfl_sync(0xffffffffu, bm, base + (h << kShift));
    if (bmh > st.m[h]) {                       // the running max moved: rescale the state
      const float scale = exp2f(st.m[h] - bmh);  // 0 when the state was empty (m = -inf)
      st.m[h] = bmh;
      st.l[h] *= scale;
      const float2 sc2 = make_float2(scale, scale);
#pragma unroll
      for (int e = 0; e < 4; ++e) st.a2[h][e] = __fmul2_rn(st.a2[h][e], sc2);
    }
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    float2 v[4];
    unpack_pairs(vw[r], v);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float p = __shfl_sync(0xffffffffu, p_my, base + ((r * G + h) << kShift));
      st.l[h] += p;
      const float2 p2 = make_float2(p, p);
#pragma unroll
      for (int e = 0; e < 4; ++e) st.a2[h][e] = __ffma2_rn(p2, v[e], st.a2[h][e]);
    }
  }
}

// Attention of the G heads over rows [0, cnt), row i given by rowfn(i, kp, vp, mask).
// stage: AttnCfg<G>::stage_bytes(nthreads) bytes of shared memory. Leaves the half-warp
// states in st (merge with attend_merge).
template <int G, class RowFn>
__device__ __forceinline__ void attend_rows(AttnState<G>& st, const float2 (&q)[G][4], int cnt,
                                            RowFn rowfn, unsigned char* stage, int nthreads) {
  constexpr int R = AttnCfg<G>::kRows;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5, hl = lane & 15, hw = t >> 4;
  const int nhw = nthreads >> 4;
  const int step = (nthreads >> 5) * 2 * R;                  // rows per CTA step
  // this half-warp's slot: stage s, row r -> stage + ((s * nhw + hw) * R + r) * 512
  auto slot = [&](int s, int r) -> unsigned char* {
    return stage + ((size_t)(s * nhw + hw) * R + r) * 512;
  };
  uint32_t mask_cur[R], mask_nxt[R];
  auto issue = [&](int wb, int s, uint32_t (&mk)[R]) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int i = wb + (lane >> 4) * R + r;
      const uint16_t* kp = nullptr;
      const uint16_t* vp = nullptr;
      mk[r] = 0;
      if (i < cnt) rowfn(i, kp, vp, mk[r]);
      if (mk[r]) {
        cp_async16(slot(s, r) + hl * 16, kp + hl * 8);
        cp_async16(slot(s, r) + 256 + hl * 16, vp + hl * 8);
      }
    }
    cp_async_commit();
  };
  int wb = warp * 2 * R;
  int s = 0;
  if (wb < cnt) issue(wb, 0, mask_cur);
#pragma unroll 1
  for (; wb < cnt; wb += step, s ^= 1) {
    if (wb + step < cnt) issue(wb + step, s ^ 1, mask_nxt);
    else cp_async_commit();                                   // keep one group per step
    cp_async_wait<1>();
    uint4 kw[R], vw[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (mask_cur[r]) {
        kw[r] = *reinterpret_cast<const uint4*>(slot(s, r) + hl * 16);
        vw[r] = *reinterpret_cast<const uint4*>(slot(s, r) + 256 + hl * 16);
      } else {
        kw[r] = make_uint4(0, 0, 0, 0);
        vw[r] = make_uint4(0, 0, 0, 0);
      }
    }
    attend_step<G>(st, q, kw, vw, mask_cur, hl);
#pragma unroll
    for (int r = 0; r < R; ++r) mask_cur[r] = mask_nxt[r];
  }
  cp_async_wait<0>();
}

// Merges the per-half-warp states of a CTA of nthreads threads into res[G][2 + 128]
// (M, L, A). scratch: >= (nthreads / 32) * G * 128 + 2 * (nthreads / 32) * G floats.
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
      const float ao = __shfl_xor_sync(0xffffffffu, st.acc(h, e), 16);
      st.acc(h, e) = st.acc(h, e) * fa + ao * fb;
    }
    st.m[h] = mn;
  }
  __syncthreads();                                // scratch may alias the staging buffer
  float* sm_m = scratch + nw * G * kD;
  float* sm_l = sm_m + nw * G;
  if (lane < 16) {
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int e = 0; e < 8; ++e) scratch[(warp * G + h) * kD + hl * 8 + e] = st.acc(h, e);
    if (hl == 0) {
#pragma unroll
      for (int h = 0; h < G; ++h) { sm_m[warp * G + h] = st.m[h]; sm_l[warp * G + h] = st.l[h]; }
    }
  }
  __syncthreads();
#pragma unroll 1
  for (int o = t; o < G * kD; o += nthreads) {
    const int h = o / kD, dch = o % kD;
    float M = -INFINITY;
#pragma unroll 1
    for (int w = 0; w < nw; ++w) M = fmaxf(M, sm_m[w * G + h]);
    float Ls = 0.f, A = 0.f;
    if (M != -INFINITY) {
#pragma unroll 1
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

// Largest number of partial states one merge combines (the host plan sizes splits by it).
constexpr int kMaxMerge = 64;

// Merges n partial states (contiguous in global memory, stride G*(2+128) floats, written by
// other CTAs) into `dst` (same format) or, when out_rows is given, into the bf16 output rows
// of the G heads. The partials are first copied into shared memory (buf, buf_bytes) with
// cp.async, as many per batch as fit, so all loads of a batch are in flight together; each
// thread then folds its output channels over the batch with the online softmax rule. The
// code is kept small on purpose: it runs once per group at the end of a step, when the
// instruction cache does not hold it.
template <int G>
__device__ __forceinline__ void merge_partials(const float* parts, int n, float* dst,
                                               uint16_t* out_rows, float* buf, int buf_bytes,
                                               int nthreads) {
  constexpr int S = G * (kD + 2);                    // floats per partial
  constexpr int kPer = (G * kD + 511) / 512;         // outputs per thread for 512 threads
  const int per = max(1, buf_bytes / (S * 4));       // partials per batch
  const int t = threadIdx.x;
  float M[kPer], Ls[kPer], A[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) { M[u] = -INFINITY; Ls[u] = 0.f; A[u] = 0.f; }
#pragma unroll 1
  for (int b0 = 0; b0 < n; b0 += per) {
    const int nb = min(per, n - b0);
    __syncthreads();                                 // the buffer is free
    const float* src = parts + (int64_t)b0 * S;
    if constexpr (S % 4 == 0) {                      // 16-byte partials (G >= 2): cp.async
      for (int i = t; i < nb * (S / 4); i += nthreads) cp_async16(buf + 4 * i, src + 4 * i);
      cp_async_commit();
      cp_async_wait<0>();
    } else {                                         // G = 1: 520-byte partials, plain loads
      for (int i = t; i < nb * S; i += nthreads) buf[i] = __ldcg(src + i);
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int o = t + u * nthreads;
      if (o >= G * kD) break;
      const int h = o / kD, dch = o % kD;
#pragma unroll 1
      for (int i = 0; i < nb; ++i) {
        const float* pp = buf + i * S + h * (kD + 2);
        const float mi = pp[0];
        if (mi == -INFINITY) continue;               // a split without rows
        const float mn = fmaxf(M[u], mi);
        const float fo = exp2f(M[u] - mn), fi = exp2f(mi - mn);   // exp2(-inf) = 0
        A[u] = A[u] * fo + pp[2 + dch] * fi;
        Ls[u] = Ls[u] * fo + pp[1] * fi;
        M[u] = mn;
      }
    }
  }
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int o = t + u * nthreads;
    if (o >= G * kD) break;
    const int h = o / kD, dch = o % kD;
    if (out_rows) {
      out_rows[(int64_t)h * kD + dch] = f2bf_rn(Ls[u] > 0.f ? A[u] / Ls[u] : 0.f);
    } else {
      dst[h * (kD + 2) + 2 + dch] = A[u];
      if (dch == 0) { dst[h * (kD + 2)] = M[u]; dst[h * (kD + 2) + 1] = Ls[u]; }
    }
  }
  __syncthreads();                                   // the caller may reuse the buffer
}

}  // namespace rtp
