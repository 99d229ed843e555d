// Decode step of one layer: index scoring, 256-bin top-p threshold, selection, and exact
// softmax attention over the selected rows (retrieval heads) or the sinks + window (local
// heads).
//
// "Full Attention Strikes Back" (paper text) §3.2: eq. (4) s(m,n) = (W^Q q^pre)^T (W^K k^pre),
// eq. (5) O = sum over S of softmax(q^T k / sqrt(d)) v with S = Top-P(s, p); local heads use
// attention sinks plus a sliding window. MCISLAB DeepRead notes on RTPurbo, "Method": top-p
// is found sort-free with a 256-bin histogram per head, fused with the scoring.
//
// Phases (one kernel each in this file, all on the caller's stream):
//   score  : per chunk of C tokens of a (sequence, retrieval KV head) group, the G query
//            heads' index scores -> workspace; group min / max through integer atomics.
//   hist   : per chunk, the 256-bin mass histogram exp(s - max) of each head -> group
//            histogram (exact 2^-40 fixed point, order independent).
//   select : per chunk, b* of each head from the group histogram; tokens whose bin >= b* for
//            any head of the group are compacted, in ascending order, into entries
//            (n << 8 | head mask); per-chunk entry counts.
//   attend : split-KV attention. Retrieval items take an equal share of the group's entries
//            (each K/V row is read once for all G heads of the group, heads that did not
//            select the row skip it); local items take a slice of the ring. Each item writes
//            (max, sum, acc[128]) per head; the last item of a group merges them.
#pragma once

#include "rtp_append.cuh"

namespace rtp {

struct DecodeParams {
  LayerShape L;
  int C;           // tokens per score chunk
  int MC;          // chunks per group (upper bound)
  int S;           // attention splits per retrieval group
  int RL;          // ring rows per local item
  int PL;          // local items per (sequence, local head)
  int n_groups;    // B * n_ret
  int n_ret_items; // n_groups * S
  int n_loc_items; // B * n_loc * PL
  int select_all;  // p >= 1
  double p;
  // inputs / outputs
  const uint16_t* q_pre;
  const float* w_qidx;
  const int32_t* seq_lens;
  CachePtrs cache;
  uint16_t* out;
  int32_t* sel_counts;
  // workspace
  int* status;
  uint32_t* lohi;              // [n_groups][2][G]   (~ord(min), ord(max)), zeroed per call
  int32_t* hcnt;               // [n_groups][G]      selected tokens per head, zeroed
  uint32_t* arrive_ret;        // [n_groups]         zeroed
  uint32_t* arrive_loc;        // [B * n_loc]        zeroed
  unsigned long long* hist;    // [n_groups][G][256] zeroed
  float* scores;               // [n_groups][G][MC * C]
  uint32_t* ent;               // [n_groups][MC * C]
  uint32_t* chunk_cnt;         // [n_groups][MC]
  float* part_ret;             // [n_ret_items][G][2 + 128]
  float* part_loc;             // [n_loc_items][G][2 + 128]
};

__device__ __forceinline__ int seq_len_checked(const DecodeParams& P, int b) {
  const int N = P.seq_lens[b];
  if (N < 1 || N > P.cache.seq_cap[b] || (int64_t)N > P.L.maxN) return 0;
  if (P.L.n_ret > 0 && (P.cache.seq_off[b] < 0 || P.cache.seq_off[b] + N > P.L.T_total)) return 0;
  return N;
}

// Index score of one token: fixed order of fused multiply-adds (identical in every phase).
template <int G>
__device__ __forceinline__ void score_row(const float (&qi)[G][kR], const uint4& a,
                                          const uint4& c, float (&s)[G]) {
  float x[16];
  unpack8(a, x);
  unpack8(c, x + 8);
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < kR; ++j) acc = fmaf(qi[h][j], x[j], acc);
    s[h] = acc;
  }
}

// q_idx = W_qidx[h]^T q_pre[b][h] for the G query heads of KV head kvh, into smem.
template <int G>
__device__ __forceinline__ void index_query(const DecodeParams& P, int b, int kvh,
                                            float (*qi)[kR]) {
  const int t = threadIdx.x;
  if (t < G * kR) {
    const int h = kvh * G + t / kR, j = t % kR;
    const uint16_t* q = P.q_pre + ((int64_t)b * P.L.Hq + h) * kD;
    const float* w = P.w_qidx + (int64_t)h * kD * kR + j;
    float acc = 0.f;
    for (int i = 0; i < kD; ++i) acc = fmaf(bf1(q[i]), __ldg(w + i * kR), acc);
    qi[t / kR][j] = acc;
  }
}

// ------------------------------------------------------------------------------ score
template <int G>
__global__ void __launch_bounds__(kThreads) score_kernel(DecodeParams P) {
  const int c = blockIdx.x, gr = blockIdx.y;
  const int b = gr / P.L.n_ret, r = gr % P.L.n_ret;
  const int N = seq_len_checked(P, b);
  const int n0 = c * P.C;
  if (n0 >= N) return;
  const int n1 = min(N, n0 + P.C);
  const int kvh = P.L.ret_kv[r];
  __shared__ float qs[G][kR];
  __shared__ float red[2][G][kThreads / 32];
  index_query<G>(P, b, kvh, qs);
  __syncthreads();
  float qi[G][kR];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int j = 0; j < kR; ++j) qi[h][j] = qs[h][j];
  float mn[G], mx[G];
#pragma unroll
  for (int h = 0; h < G; ++h) { mn[h] = INFINITY; mx[h] = -INFINITY; }
  const uint16_t* idx = P.cache.idx + ((int64_t)r * P.L.T_total + P.cache.seq_off[b]) * kR;
  const int64_t stride = (int64_t)P.MC * P.C;
  float* sc = P.scores + (int64_t)gr * G * stride;
  for (int n = n0 + threadIdx.x; n < n1; n += kThreads) {
    const uint4 a = ld_stream(idx + (int64_t)n * kR);
    const uint4 d = ld_stream(idx + (int64_t)n * kR + 8);
    float s[G];
    score_row<G>(qi, a, d, s);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      sc[h * stride + n] = s[h];
      mn[h] = fminf(mn[h], s[h]);
      mx[h] = fmaxf(mx[h], s[h]);
    }
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int h = 0; h < G; ++h) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mn[h] = fminf(mn[h], __shfl_xor_sync(0xffffffffu, mn[h], o));
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], o));
    }
    if (lane == 0) { red[0][h][warp] = mn[h]; red[1][h][warp] = mx[h]; }
  }
  __syncthreads();
  if (threadIdx.x < G) {
    const int h = threadIdx.x;
    float a = red[0][h][0], z = red[1][h][0];
    for (int w = 1; w < kThreads / 32; ++w) { a = fminf(a, red[0][h][w]); z = fmaxf(z, red[1][h][w]); }
    atomicMax(P.lohi + ((int64_t)gr * 2 + 0) * G + h, ~f2ord(a));
    atomicMax(P.lohi + ((int64_t)gr * 2 + 1) * G + h, f2ord(z));
  }
}

template <int G>
__device__ __forceinline__ void load_range(const DecodeParams& P, int gr, float* lo, float* hi,
                                           float* inv) {
#pragma unroll
  for (int h = 0; h < G; ++h) {
    lo[h] = ord2f(~P.lohi[((int64_t)gr * 2 + 0) * G + h]);
    hi[h] = ord2f(P.lohi[((int64_t)gr * 2 + 1) * G + h]);
    inv[h] = (hi[h] > lo[h] && !P.select_all) ? (float)kBins / (hi[h] - lo[h]) : 0.f;
  }
}

__device__ __forceinline__ int bin_of(float s, float lo, float inv) {
  return min(kBins - 1, (int)((s - lo) * inv));
}

// ------------------------------------------------------------------------------ hist
template <int G>
__global__ void __launch_bounds__(kThreads) hist_kernel(DecodeParams P) {
  const int c = blockIdx.x, gr = blockIdx.y;
  const int b = gr / P.L.n_ret;
  const int N = seq_len_checked(P, b);
  const int n0 = c * P.C;
  if (n0 >= N || P.select_all) return;
  const int n1 = min(N, n0 + P.C);
  __shared__ unsigned long long hs[G][kBins];
  for (int i = threadIdx.x; i < G * kBins; i += kThreads) (&hs[0][0])[i] = 0ull;
  float lo[G], hi[G], inv[G];
  load_range<G>(P, gr, lo, hi, inv);
  __syncthreads();
  const int64_t stride = (int64_t)P.MC * P.C;
  const float* sc = P.scores + (int64_t)gr * G * stride;
  for (int n = n0 + threadIdx.x; n < n1; n += kThreads) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float s = sc[h * stride + n];
      const float m = exp2f((s - hi[h]) * kLog2e);
      const unsigned long long q = __float2ull_rn(m * kMassScale);
      if (q) atomicAdd(&hs[h][bin_of(s, lo[h], inv[h])], q);
    }
  }
  __syncthreads();
  unsigned long long* gh = P.hist + (int64_t)gr * G * kBins;
  for (int i = threadIdx.x; i < G * kBins; i += kThreads) {
    const unsigned long long v = (&hs[0][0])[i];
    if (v) atomicAdd(gh + i, v);
  }
}

// b* of the G heads of a group from its histogram; warp h < G handles head h.
template <int G>
__device__ __forceinline__ void find_bstar(const DecodeParams& P, int gr, int* bstar) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (warp < G) {
    const int h = warp;
    if (P.select_all) {
      if (lane == 0) bstar[h] = 0;
      return;
    }
    const unsigned long long* gh = P.hist + ((int64_t)gr * G + h) * kBins;
    unsigned long long v[8], tot = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) { v[e] = gh[lane * 8 + e]; tot += v[e]; }
    // x = inclusive suffix sum of the lane totals (this lane and every higher lane)
    unsigned long long x = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long y = __shfl_down_sync(0xffffffffu, x, o);
      if (lane + o < 32) x += y;
    }
    const unsigned long long above = x - tot;
    const unsigned long long T = __shfl_sync(0xffffffffu, x, 0);
    const double thr = P.p * (double)T;
    int best = -1;
    unsigned long long cum = above;
#pragma unroll
    for (int e = 7; e >= 0; --e) {
      cum += v[e];
      if (best < 0 && (double)cum >= thr) best = lane * 8 + e;
    }
    // b* = largest bin b with C_b >= p T: the largest candidate over lanes
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) best = max(best, __shfl_xor_sync(0xffffffffu, best, o));
    if (lane == 0) bstar[h] = best < 0 ? 0 : best;
  }
}

// ------------------------------------------------------------------------------ select
template <int G>
__global__ void __launch_bounds__(kThreads) select_kernel(DecodeParams P) {
  const int c = blockIdx.x, gr = blockIdx.y;
  const int b = gr / P.L.n_ret;
  const int N = seq_len_checked(P, b);
  const int n0 = c * P.C;
  if (n0 >= N) return;
  const int n1 = min(N, n0 + P.C);
  __shared__ int bstar[G];
  __shared__ int wsum[kThreads / 32];
  __shared__ int hsum[G];
  __shared__ int base;
  float lo[G], hi[G], inv[G];
  load_range<G>(P, gr, lo, hi, inv);
  find_bstar<G>(P, gr, bstar);
  if (threadIdx.x < G) hsum[threadIdx.x] = 0;
  if (threadIdx.x == 0) base = 0;
  __syncthreads();
  int bs[G];
#pragma unroll
  for (int h = 0; h < G; ++h) bs[h] = bstar[h];
  const int64_t stride = (int64_t)P.MC * P.C;
  const float* sc = P.scores + (int64_t)gr * G * stride;
  uint32_t* ent = P.ent + (int64_t)gr * stride + n0;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int hc[G];
#pragma unroll
  for (int h = 0; h < G; ++h) hc[h] = 0;
  for (int nb = n0; nb < n1; nb += kThreads) {
    const int n = nb + threadIdx.x;
    uint32_t mask = 0;
    if (n < n1) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float s = sc[h * stride + n];
        if (bin_of(s, lo[h], inv[h]) >= bs[h]) { mask |= 1u << h; hc[h]++; }
      }
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, mask != 0);
    if (lane == 0) wsum[warp] = __popc(bal);
    __syncthreads();
    int before = 0, total = 0;
    for (int w = 0; w < kThreads / 32; ++w) {
      const int x = wsum[w];
      before += (w < warp) ? x : 0;
      total += x;
    }
    if (mask) ent[base + before + __popc(bal & ((1u << lane) - 1u))] = ((uint32_t)n << 8) | mask;
    __syncthreads();
    if (threadIdx.x == 0) base += total;
    __syncthreads();
  }
#pragma unroll
  for (int h = 0; h < G; ++h) {
    int v = hc[h];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0 && v) atomicAdd(&hsum[h], v);
  }
  __syncthreads();
  if (threadIdx.x == 0) P.chunk_cnt[(int64_t)gr * P.MC + c] = (uint32_t)base;
  if (threadIdx.x < G && hsum[threadIdx.x])
    atomicAdd(P.hcnt + (int64_t)gr * G + threadIdx.x, hsum[threadIdx.x]);
}

// ------------------------------------------------------------------------------ attend
// RoPE'd, pre-scaled query of the G heads of KV head kvh at position m = N - 1, into smem.
template <int G>
__device__ __forceinline__ void rope_query(const DecodeParams& P, int b, int kvh, int N,
                                           float (*qs)[kD]) {
  const int t = threadIdx.x;
  if (t < kD) {
    const int i = t & 63;
    const double th = pow(P.L.rope_base, -2.0 * (double)i / (double)kD);
    double sn, cs;
    sincos((double)(N - 1) * th, &sn, &cs);
    const float scale = kLog2e * 0.08838834764831845f;   // log2(e) / sqrt(128)
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const uint16_t* q = P.q_pre + ((int64_t)b * P.L.Hq + kvh * G + h) * kD;
      const double qa = bf1(q[i]), qb = bf1(q[i + 64]);
      const double r = (t < 64) ? (qa * cs - qb * sn) : (qa * sn + qb * cs);
      qs[h][t] = (float)r * scale;
    }
  }
}

struct AttnSmem {
  float m[16][8];
  float l[16][8];
};

// Online-softmax attention of G heads over rows given by `row(i, &kp, &vp, &mask)`, i < nrows.
// Half-warp per row, lane owns 8 channels. Result: per-head (M, L, A[128]) in `res`
// ([G][2 + 128], shared memory). Log2 domain: logits carry log2(e) / sqrt(d).
template <int G, class RowFn>
__device__ __forceinline__ void attend_rows(const float (*qs)[kD], int nrows, RowFn row,
                                            float* acc_smem /*[16][G][128]*/, AttnSmem& sm,
                                            float* res /*[G][130]*/) {
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int hl = lane & 15, hw = t >> 4;
  float q[G][8];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < 8; ++e) q[h][e] = qs[h][hl * 8 + e];
  float m[G], l[G], acc[G][8];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[h][e] = 0.f;
  }
  for (int base = warp * 2; base < nrows; base += kThreads / 16) {
    const int i = base + (lane >> 4);
    const bool valid = i < nrows;
    const uint16_t *kp = nullptr, *vp = nullptr;
    uint32_t mask = 0;
    if (valid) row(i, kp, vp, mask);
    uint4 kw = make_uint4(0, 0, 0, 0), vw = make_uint4(0, 0, 0, 0);
    if (valid) {
      kw = ld_stream(kp + hl * 8);
      vw = ld_stream(vp + hl * 8);
    }
    float k[8], v[8];
    unpack8(kw, k);
    unpack8(vw, v);
    float d[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float a = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) a = fmaf(q[h][e], k[e], a);
      d[h] = a;
    }
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) d[h] += __shfl_xor_sync(0xffffffffu, d[h], o);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      if (valid && (mask >> h) & 1u) {
        const float mn = fmaxf(m[h], d[h]);
        const float cf = exp2f(m[h] - mn);
        const float pr = exp2f(d[h] - mn);
        l[h] = l[h] * cf + pr;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[h][e] = fmaf(pr, v[e], acc[h][e] * cf);
        m[h] = mn;
      }
    }
  }
  // merge the 16 half-warps
  if (hl == 0) {
#pragma unroll
    for (int h = 0; h < G; ++h) { sm.m[hw][h] = m[h]; sm.l[hw][h] = l[h]; }
  }
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc_smem[(hw * G + h) * kD + hl * 8 + e] = acc[h][e];
  __syncthreads();
  for (int o = t; o < G * kD; o += kThreads) {
    const int h = o / kD, dch = o % kD;
    float M = -INFINITY;
    for (int w = 0; w < 16; ++w) M = fmaxf(M, sm.m[w][h]);
    float Ls = 0.f, A = 0.f;
    if (M != -INFINITY) {
      for (int w = 0; w < 16; ++w) {
        const float f = exp2f(sm.m[w][h] - M);
        Ls += sm.l[w][h] * f;
        A += acc_smem[(w * G + h) * kD + dch] * f;
      }
    }
    res[h * (kD + 2) + 2 + dch] = A;
    if (dch == 0) { res[h * (kD + 2)] = M; res[h * (kD + 2) + 1] = Ls; }
  }
  __syncthreads();
}

// Merge n partial states (M, L, A) per head and write bf16 output rows of the G heads.
template <int G>
__device__ __forceinline__ void combine_partials(const float* parts, int n, uint16_t* out_rows) {
  for (int o = threadIdx.x; o < G * kD; o += kThreads) {
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
    out_rows[(int64_t)h * kD + dch] = f2bf_rn(Ls > 0.f ? A / Ls : 0.f);
  }
}

template <int G>
__global__ void __launch_bounds__(kThreads) attend_kernel(DecodeParams P) {
  extern __shared__ __align__(16) float dyn[];
  float* acc_smem = dyn;                                  // [16][G][128]
  float* res = dyn + 16 * G * kD;                         // [G][130]
  __shared__ float qs[G][kD];
  __shared__ AttnSmem sm;
  __shared__ uint32_t pref[1025];
  __shared__ int is_last;
  const int item = blockIdx.x;
  const int t = threadIdx.x;
  if (item < P.n_ret_items) {
    const int gr = item / P.S, s = item % P.S;
    const int b = gr / P.L.n_ret, r = gr % P.L.n_ret;
    const int kvh = P.L.ret_kv[r];
    const int N = seq_len_checked(P, b);
    if (N == 0) {
      if (s == 0) {
        if (t == 0) set_status(P.status, -6);
        for (int o = t; o < G * kD; o += kThreads)
          P.out[((int64_t)b * P.L.Hq + kvh * G) * kD + o] = 0;
        if (t < G) P.sel_counts[(int64_t)b * P.L.Hq + kvh * G + t] = 0;
      }
      return;
    }
    const int nch = (N + P.C - 1) / P.C;
    // prefix of entry counts over chunks (nch <= 1024)
    if (t == 0) {
      uint32_t acc = 0;
      for (int c = 0; c < nch; ++c) { pref[c] = acc; acc += __ldcg(P.chunk_cnt + (int64_t)gr * P.MC + c); }
      pref[nch] = acc;
    }
    rope_query<G>(P, b, kvh, N, qs);
    __syncthreads();
    const uint32_t U = pref[nch];
    const uint32_t e0 = (uint32_t)(((uint64_t)U * s) / P.S);
    const uint32_t e1 = (uint32_t)(((uint64_t)U * (s + 1)) / P.S);
    const int64_t stride = (int64_t)P.MC * P.C;
    const uint32_t* ent = P.ent + (int64_t)gr * stride;
    const int64_t rowbase = (int64_t)r * P.L.T_total + P.cache.seq_off[b];
    const uint16_t* kb = P.cache.k_ret;
    const uint16_t* vb = P.cache.v_ret;
    auto rowfn = [&](int i, const uint16_t*& kp, const uint16_t*& vp, uint32_t& mask) {
      const uint32_t e = e0 + (uint32_t)i;
      int lo = 0, hi = nch - 1;                 // last chunk with pref[c] <= e
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pref[mid] <= e) lo = mid; else hi = mid - 1;
      }
      const uint32_t w = __ldcg(ent + (int64_t)lo * P.C + (e - pref[lo]));
      const int64_t n = w >> 8;
      mask = w & 0xffu;
      kp = kb + (rowbase + n) * kD;
      vp = vb + (rowbase + n) * kD;
    };
    attend_rows<G>(qs, (int)(e1 - e0), rowfn, acc_smem, sm, res);
    float* part = P.part_ret + (int64_t)item * G * (kD + 2);
    for (int o = t; o < G * (kD + 2); o += kThreads) part[o] = res[o];
    __threadfence();
    __syncthreads();
    if (t == 0) is_last = (atomicAdd(P.arrive_ret + gr, 1u) == (uint32_t)(P.S - 1));
    __syncthreads();
    if (is_last) {
      __threadfence();
      combine_partials<G>(P.part_ret + (int64_t)gr * P.S * G * (kD + 2), P.S,
                          P.out + ((int64_t)b * P.L.Hq + kvh * G) * kD);
      if (t < G)
        P.sel_counts[(int64_t)b * P.L.Hq + kvh * G + t] = __ldcg(P.hcnt + (int64_t)gr * G + t);
    }
  } else {
    const int li = item - P.n_ret_items;
    const int lg = li / P.PL, piece = li % P.PL;   // lg = b * n_loc + x
    const int b = lg / P.L.n_loc, x = lg % P.L.n_loc;
    const int kvh = P.L.loc_kv[x];
    const int N = seq_len_checked(P, b);
    if (N == 0) {
      if (piece == 0) {
        if (t == 0) set_status(P.status, -6);
        for (int o = t; o < G * kD; o += kThreads)
          P.out[((int64_t)b * P.L.Hq + kvh * G) * kD + o] = 0;
        if (t < G) P.sel_counts[(int64_t)b * P.L.Hq + kvh * G + t] = 0;
      }
      return;
    }
    const int nrows_all = min(N, P.L.ring);
    const int r0 = piece * P.RL;
    const int nrows = max(0, min(nrows_all - r0, P.RL));
    rope_query<G>(P, b, kvh, N, qs);
    __syncthreads();
    const uint16_t* kb = P.cache.k_loc + ((int64_t)x * P.L.B + b) * P.L.ring * kD;
    const uint16_t* vb = P.cache.v_loc + ((int64_t)x * P.L.B + b) * P.L.ring * kD;
    auto rowfn = [&](int i, const uint16_t*& kp, const uint16_t*& vp, uint32_t& mask) {
      kp = kb + (int64_t)(r0 + i) * kD;
      vp = vb + (int64_t)(r0 + i) * kD;
      mask = 0xffu;
    };
    attend_rows<G>(qs, nrows, rowfn, acc_smem, sm, res);
    float* part = P.part_loc + (int64_t)li * G * (kD + 2);
    for (int o = t; o < G * (kD + 2); o += kThreads) part[o] = res[o];
    __threadfence();
    __syncthreads();
    if (t == 0) is_last = (atomicAdd(P.arrive_loc + lg, 1u) == (uint32_t)(P.PL - 1));
    __syncthreads();
    if (is_last) {
      __threadfence();
      combine_partials<G>(P.part_loc + (int64_t)lg * P.PL * G * (kD + 2), P.PL,
                          P.out + ((int64_t)b * P.L.Hq + kvh * G) * kD);
      if (t < G) P.sel_counts[(int64_t)b * P.L.Hq + kvh * G + t] = nrows_all;
    }
  }
}

// ------------------------------------------------------------------------------ sel_idx
// Debug output: ascending positions each query head attended to. One CTA per (b, h).
template <int G>
__global__ void __launch_bounds__(kThreads) emit_sel_kernel(DecodeParams P, int32_t* sel_idx,
                                                            int64_t sel_stride) {
  const int b = blockIdx.x / P.L.Hq, h = blockIdx.x % P.L.Hq;
  const int kvh = h / G, j = h % G;
  const int N = seq_len_checked(P, b);
  int32_t* dst = sel_idx + ((int64_t)b * P.L.Hq + h) * sel_stride;
  if (N == 0) return;
  const int slot = P.L.slot[kvh];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __shared__ int wsum[kThreads / 32];
  if (slot < 0) {
    const int s1 = min(N, P.L.sinks);
    const int w0 = max(P.L.sinks, N - P.L.window);
    const int cnt = s1 + max(0, N - w0);
    for (int k = threadIdx.x; k < cnt; k += kThreads) dst[k] = k < s1 ? k : w0 + (k - s1);
    return;
  }
  const int gr = b * P.L.n_ret + slot;
  const int nch = (N + P.C - 1) / P.C;
  const int64_t stride = (int64_t)P.MC * P.C;
  const uint32_t* ent = P.ent + (int64_t)gr * stride;
  int base = 0;
  for (int c = 0; c < nch; ++c) {
    const int cnt = (int)__ldcg(P.chunk_cnt + (int64_t)gr * P.MC + c);
    for (int k0 = 0; k0 < cnt; k0 += kThreads) {
      const int k = k0 + threadIdx.x;
      uint32_t w = 0;
      bool keep = false;
      if (k < cnt) { w = __ldcg(ent + (int64_t)c * P.C + k); keep = (w >> j) & 1u; }
      const uint32_t bal = __ballot_sync(0xffffffffu, keep);
      if (lane == 0) wsum[warp] = __popc(bal);
      __syncthreads();
      int before = 0, total = 0;
      for (int ww = 0; ww < kThreads / 32; ++ww) { before += ww < warp ? wsum[ww] : 0; total += wsum[ww]; }
      if (keep) dst[base + before + __popc(bal & ((1u << lane) - 1u))] = (int32_t)(w >> 8);
      __syncthreads();
      base += total;
    }
  }
}

}  // namespace rtp
