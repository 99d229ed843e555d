// Causal prefill attention ("Full Attention Strikes Back" (paper text) §3.2: retrieval heads
// use dense attention in prefill, local heads attention sinks plus a sliding window in prefill
// and decode), for a prompt at positions 0..n_b-1 of each sequence.
//
// prefill_rope_keys: the prompt's keys rotated by R(j) with the append's arithmetic (double
// angles and rotation, one rounding to bf16), so they equal the cache rows the append writes;
// local heads need them because their ring keeps only the last window.
// prefill_kernel: one CTA of 8 warps per (128 query rows, query head, sequence), two CTAs per
// SM; thread t owns query row t % 128 (its tensor-memory lane) and half t / 128 of the row's
// keys in the softmax and of its output dims. Over the 64-key tiles the rows can see (causal;
// local heads skip the tiles between the sinks and the window), with K and V tiles staged by
// cp.async in the 128-byte-swizzled operand layout:
//   S = Q K^T on the fifth-generation tensor cores (tcgen05.mma, 128 x 64, fp32 in tensor
//   memory), the query as two bf16 terms (the rounded value and its rounded remainder) so the
//   logits keep fp32-level accuracy;
//   online softmax in the log2 domain (the query carries log2(e) / sqrt(128)), keys checked
//   one by one only where a tile crosses the row's diagonal, window edge or prompt end; the
//   probabilities written back to tensor memory as two bf16 terms;
//   the tile's P V from tensor memory (TS form, 128 x 128) accumulated into the output in
//   tensor memory; a row's softmax reference moves only when a tile's maximum exceeds it by
//   2^8, and only then is the row's accumulated output rescaled in place.
// The next K tile loads while the softmax runs, the next V tile while the next S is computed.
#pragma once

#include "rtp_append.cuh"
#include "rtp_attend.cuh"
#include "rtp_tmem.cuh"
#include "rtp_umma.cuh"

namespace rtp {

constexpr int kPfThreads = 256;      // 8 warps: thread t owns row t % 128 (tensor-memory lane),
                                     // the columns and output dims of half t / 128
constexpr int kPfQ = 128;            // query rows per CTA (the MMA's M)
constexpr int kPfK = 64;             // keys per tile
constexpr uint32_t kPfQBlock = kPfQ * 128;                // one 64-dim block of the query tile
constexpr uint32_t kPfBlock = kPfK * 128;                 // one 64-dim block of a K or V tile
constexpr uint32_t kPfQHi = 0, kPfQLo = 2 * kPfQBlock;    // query terms: 2 blocks each
constexpr uint32_t kPfKt = 4 * kPfQBlock, kPfVt = kPfKt + 2 * kPfBlock;
constexpr uint32_t kPfBar = kPfVt + 2 * kPfBlock;         // two mbarriers, the tensor-memory word
constexpr uint32_t kPfLsum = kPfBar + 64;                 // [2][128] row-sum halves
constexpr int kPfSmem = (int)kPfLsum + 1024 + 1024;       // + slack to align the base to 1024
constexpr uint32_t kPfTmemCols = 256;  // S, then P hi / lo, in [0, 64); the output in [128, 256)
constexpr uint32_t kPfColO = 128;
constexpr float kPfSlack = 8.f;      // log2 units the softmax reference may lag a row's maximum

__global__ void __launch_bounds__(128)
prefill_rope_keys(LayerShape L, const uint16_t* __restrict__ k_pre, const int32_t* __restrict__ n_b,
                  int n_max, uint16_t* __restrict__ k_rope) {
  const int b = blockIdx.y, g = blockIdx.z, t = threadIdx.x;
  const int nb = min(max(n_b[b], 0), n_max);
  const int j0 = blockIdx.x * kAppendTok;
  const int i = t & 63;
  const double th = L.theta[i];
  for (int jj = 0; jj < kAppendTok; ++jj) {
    const int j = j0 + jj;
    if (j >= nb) break;
    const uint16_t* kp = k_pre + (((int64_t)b * n_max + j) * L.Hkv + g) * kD;
    double sn, cs;
    rope_sincos((double)j, th, &sn, &cs);
    const double xa = bf1(kp[i]), xb = bf1(kp[i + 64]);
    const double r = (t < 64) ? (xa * cs - xb * sn) : (xa * sn + xb * cs);
    k_rope[(((int64_t)b * L.Hkv + g) * n_max + j) * kD + t] = d2bf_rn(r);
  }
}

// next key tile at or after kt that a query tile [q0, q1] can see (-1: none); local heads see
// keys [0, sinks) and (q0 - window, q1]
__device__ __forceinline__ int pf_next_tile(int kt, int q0, int q1, bool local, int sinks,
                                            int window) {
  const int last = q1 / kPfK;
  if (kt > last) return -1;
  if (!local || kt * kPfK < sinks) return kt;
  const int first_win = max(q0 - window + 1, 0) / kPfK;   // tile of the lowest window key
  const int n = max(kt, first_win);
  return n <= last ? n : -1;
}

struct PrefillParams {
  LayerShape L;
  const uint16_t* q_pre;     // [B][n_max][Hq][128]
  const uint16_t* k_rope;    // [B][Hkv][n_max][128]
  const uint16_t* v;         // [B][n_max][Hkv][128]
  const int32_t* n_b;
  uint16_t* out;             // [B][n_max][Hq][128]
  int* status;
  long long spin_limit;
  int n_max;
};

__device__ __forceinline__ float pf_ex2(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// Load one 64-row K or V tile into its 128-byte-swizzled blocks (dims 0-63, then 64-127);
// rows past the prompt are zeros (their probabilities are 0 and must meet finite values).
__device__ __forceinline__ void pf_load_tile(uint32_t dst, const uint16_t* src, int64_t stride,
                                             int kt, int nb) {
  const int t = threadIdx.x;
#pragma unroll
  for (int u = 0; u < (kPfK * 16) / kPfThreads; ++u) {
    const int e = t + u * kPfThreads, r = e >> 4, c16 = e & 15;
    const int key = kt * kPfK + r;
    const uint32_t off = dst + (uint32_t)(c16 >> 3) * kPfBlock + sw128_off(r, c16 & 7);
    if (key < nb) cp_async16_s(off, src + key * stride + c16 * 8);
    else st_shared_zero16(off);
  }
}

__global__ void __launch_bounds__(kPfThreads, 2) prefill_kernel(PrefillParams P) {
  extern __shared__ __align__(1024) unsigned char pf_raw[];
  const LayerShape& L = P.L;
  const int qt = gridDim.x - 1 - blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int nb = min(max(P.n_b[b], 0), P.n_max);
  const int q0 = qt * kPfQ;
  if (q0 >= nb) return;
  const int q1 = min(q0 + kPfQ, nb) - 1;                 // last query row of the CTA
  const int g = h / L.G;
  const bool local = L.slot[g] < 0;
  const int t = threadIdx.x, warp = t >> 5;
  const uint32_t raw = smem_u32(pf_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;          // swizzle atoms need 1024-byte alignment
  unsigned char* sm = pf_raw + (base - raw);
  const uint32_t sQh = base + kPfQHi, sQl = base + kPfQLo, sK = base + kPfKt, sV = base + kPfVt;
  const uint32_t barS = base + kPfBar, barO = barS + 8, tword = barS + 16;
  const uint16_t* kbase = P.k_rope + ((int64_t)b * L.Hkv + g) * P.n_max * kD;
  const uint16_t* vbase = P.v + (int64_t)b * P.n_max * L.Hkv * kD + (int64_t)g * kD;
  const int64_t vstride = (int64_t)L.Hkv * kD;

  int kt = pf_next_tile(0, q0, q1, local, L.sinks, L.window);
  pf_load_tile(sK, kbase, kD, kt, nb);
  cp_async_commit();
  pf_load_tile(sV, vbase, vstride, kt, nb);
  cp_async_commit();
  // the rotated, scaled query rows as two bf16 terms (hi, lo), K-major 128-byte-swizzled
  const float scale = kLog2e * 0.08838834764831845f;    // log2(e) / sqrt(128)
#pragma unroll 1
  for (int u = 0; u < (kPfQ * 8) / kPfThreads; ++u) {
    const int e = t + u * kPfThreads, r = e >> 3, c = e & 7;   // row r, dims 8c.. and 64 + 8c..
    const int m = q0 + r;
    uint32_t h0[4] = {0, 0, 0, 0}, l0[4] = {0, 0, 0, 0}, h1[4] = {0, 0, 0, 0}, l1[4] = {0, 0, 0, 0};
    if (m < nb) {
      const uint16_t* q = P.q_pre + (((int64_t)b * P.n_max + m) * L.Hq + h) * kD;
      const uint4 wa = *reinterpret_cast<const uint4*>(q + 8 * c);
      const uint4 wb = *reinterpret_cast<const uint4*>(q + 64 + 8 * c);
      float qa[8], qb[8];
      unpack8(wa, qa);
      unpack8(wb, qb);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float x[2], y[2];
#pragma unroll
        for (int z = 0; z < 2; ++z) {
          const int j = 2 * k + z;
          float sn, cs;
          rope_sincosf((double)m, L.theta[8 * c + j], &sn, &cs);
          x[z] = (qa[j] * cs - qb[j] * sn) * scale;
          y[z] = (qa[j] * sn + qb[j] * cs) * scale;
        }
        split_bf2(x[0], x[1], h0[k], l0[k]);
        split_bf2(y[0], y[1], h1[k], l1[k]);
      }
    }
    const uint32_t o0 = sw128_off(r, c);
    *reinterpret_cast<uint4*>(sm + kPfQHi + o0) = make_uint4(h0[0], h0[1], h0[2], h0[3]);
    *reinterpret_cast<uint4*>(sm + kPfQHi + kPfQBlock + o0) = make_uint4(h1[0], h1[1], h1[2], h1[3]);
    *reinterpret_cast<uint4*>(sm + kPfQLo + o0) = make_uint4(l0[0], l0[1], l0[2], l0[3]);
    *reinterpret_cast<uint4*>(sm + kPfQLo + kPfQBlock + o0) = make_uint4(l1[0], l1[1], l1[2], l1[3]);
  }
  fence_async_smem();
  if (t == 0) {
    mbar_init(barS, 1);
    mbar_init(barO, 1);
    mbar_init_fence();
  }
  if (warp == 0) tmem_alloc_cols(tword, kPfTmemCols);
  tmem_fence_before_sync();
  __syncthreads();
  tmem_fence_after_sync();
  const uint32_t tm = *reinterpret_cast<volatile uint32_t*>(sm + kPfBar + 16);
  const uint32_t tl = tm + ((uint32_t)((warp & 3) * 32) << 16);   // this thread's lane (row)
  constexpr uint32_t idS = umma_idesc_bf16(kPfQ, kPfK, 0);   // S = Q K^T: 128 x 64, K-major B
  constexpr uint32_t idO = umma_idesc_bf16(kPfQ, kD, 1);     // O = P V: 128 x 128, MN-major B

  // The output accumulates in tensor memory across tiles (the PV MMAs add into it). The
  // softmax reference m_ref of a row moves only when a tile's maximum exceeds it by more than
  // kPfSlack (log2 units): then the row's accumulated output and sum are scaled by
  // 2^(m_ref - m_new) in place; otherwise the probabilities 2^(s - m_ref) stay below 2^kPfSlack.
  float m_ref = -INFINITY, l_run = 0.f;
  const int row = q0 + (t & (kPfQ - 1)), hf = t >> 7;
  const uint32_t to = tl + kPfColO + 64 * hf;               // this thread's 64 output columns
  int j = 0, pend = 0;                                      // pend: 1 S, 2 PV in flight at an abort
#pragma unroll 1
  while (kt >= 0) {
    const int kn = pf_next_tile(kt + 1, q0, q1, local, L.sinks, L.window);
    cp_async_wait<1>();                                     // K tile kt landed (V may be pending)
    fence_async_smem();
    tmem_fence_before_sync();
    __syncthreads();
    if (t == 0) {
      tmem_fence_after_sync();
#pragma unroll
      for (int ks = 0; ks < kD / 16; ++ks) {
        const uint32_t ko = (uint32_t)(ks >> 2) * kPfBlock + (uint32_t)(ks & 3) * 32;
        const uint32_t qo = (uint32_t)(ks >> 2) * kPfQBlock + (uint32_t)(ks & 3) * 32;
        const uint64_t bk = umma_desc_sw128(sK + ko, 16, 1024);
        umma_ss(tm, umma_desc_sw128(sQh + qo, 16, 1024), bk, idS, ks > 0);
        umma_ss(tm, umma_desc_sw128(sQl + qo, 16, 1024), bk, idS, 1);
      }
      umma_commit(barS);
    }
    __syncwarp();
    if (__syncthreads_or(!mbar_wait(barS, j & 1, P.spin_limit))) { pend = 1; break; }
    tmem_fence_after_sync();
    if (kn >= 0) pf_load_tile(sK, kbase, kD, kn, nb);       // the K buffer is free again
    cp_async_commit();
    // softmax of row `row`: the maximum over the tile's 64 keys (both halves of the row read it
    // whole), then the probabilities of this thread's 32 keys, each 16-key group's two bf16
    // terms written over its own scores (hi in the first 8 columns, lo in the next 8). Keys are
    // checked one by one only in a tile this row does not see whole (the diagonal, the window's
    // edge, the prompt's end); tensor-memory accesses stay outside per-row branches (they are
    // warp-wide).
    const int k0 = kt * kPfK, k1 = k0 + kPfK - 1;
    const int lo_ok = local ? row - L.window : -1;          // local: keys > lo_ok or < sinks
    const bool whole = k1 <= row && k1 < nb && (k0 > lo_ok || k1 < L.sinks);
    float mx = -INFINITY;
    {
      uint32_t sr[64];
      __syncwarp();
      tmem_ld32(tl, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(tl + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_wait_ld();
      if (whole) {
#pragma unroll
        for (int i = 0; i < 64; ++i) mx = fmaxf(mx, __uint_as_float(sr[i]));
      } else {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const int key = k0 + i;
          const bool ok = key <= row && key < nb && (key > lo_ok || key < L.sinks);
          mx = ok ? fmaxf(mx, __uint_as_float(sr[i])) : mx;
        }
      }
    }
    // the row's other half (warp w ^ 4) reads these columns for its maximum too: both halves
    // finish reading before either writes its probabilities over them
    tmem_fence_before_sync();
    switch (warp & 3) {                                     // named barrier of the warp pair
      case 0: asm volatile("bar.sync 1, 64;" ::: "memory"); break;
      case 1: asm volatile("bar.sync 2, 64;" ::: "memory"); break;
      case 2: asm volatile("bar.sync 3, 64;" ::: "memory"); break;
      default: asm volatile("bar.sync 4, 64;" ::: "memory"); break;
    }
    tmem_fence_after_sync();
    const bool move = mx > m_ref + kPfSlack;                // also the first visible key
    const float m_new = move ? mx : m_ref;
    const float alpha = move ? pf_ex2(m_ref - m_new) : 1.f; // 0 while nothing was seen
    m_ref = m_new;
    l_run *= alpha;
    if (j > 0 && __any_sync(0xffffffffu, move)) {          // scale the accumulated output
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t r[32];
        __syncwarp();
        tmem_ld32(to + 32 * c, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
        __syncwarp();
        tmem_st32(to + 32 * c, r);
      }
    }
    {
      const uint32_t col = 32 * hf;                         // this thread's 32 keys
      uint32_t sr[32], ph[16], pl[16];
      __syncwarp();
      tmem_ld32(tl + col, sr);
      tmem_wait_ld();
      float lsum = 0.f;
      if (whole) {
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float p0 = pf_ex2(__uint_as_float(sr[2 * c]) - m_ref);
          const float p1 = pf_ex2(__uint_as_float(sr[2 * c + 1]) - m_ref);
          lsum += p0 + p1;
          split_bf2(p0, p1, ph[c], pl[c]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int key = k0 + (int)col + 2 * c;
          const bool ok0 = key <= row && key < nb && (key > lo_ok || key < L.sinks);
          const bool ok1 = key + 1 <= row && key + 1 < nb && (key + 1 > lo_ok || key + 1 < L.sinks);
          const float p0 = ok0 ? pf_ex2(__uint_as_float(sr[2 * c]) - m_ref) : 0.f;
          const float p1 = ok1 ? pf_ex2(__uint_as_float(sr[2 * c + 1]) - m_ref) : 0.f;
          lsum += p0 + p1;
          split_bf2(p0, p1, ph[c], pl[c]);
        }
      }
      l_run += lsum;
      // groups g = 0, 1 of 16 keys: hi in columns col + 16 g + [0, 8), lo in + [8, 16)
      uint32_t a[8], b[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) { a[c] = ph[c]; b[c] = pl[c]; }
      __syncwarp();
      tmem_st8(tl + col, a);
      tmem_st8(tl + col + 8, b);
#pragma unroll
      for (int c = 0; c < 8; ++c) { a[c] = ph[8 + c]; b[c] = pl[8 + c]; }
      tmem_st8(tl + col + 16, a);
      tmem_st8(tl + col + 24, b);
    }
    __syncwarp();
    tmem_wait_st();
    cp_async_wait<1>();                                     // V tile kt landed
    fence_async_smem();
    tmem_fence_before_sync();
    __syncthreads();
    if (t == 0) {
      tmem_fence_after_sync();
#pragma unroll
      for (int ks = 0; ks < kPfK / 16; ++ks) {
        const uint64_t bv = umma_desc_sw128(sV + (uint32_t)ks * 2048, kPfBlock, 1024);
        const uint32_t pa = tm + 16 * ks;                   // P hi of keys 16 ks .. 16 ks + 15
        umma_ts(tm + kPfColO, pa, bv, idO, j > 0 || ks > 0);
        umma_ts(tm + kPfColO, pa + 8, bv, idO, 1);          // P lo
      }
      umma_commit(barO);
    }
    __syncwarp();
    if (__syncthreads_or(!mbar_wait(barO, j & 1, P.spin_limit))) { pend = 2; break; }
    tmem_fence_after_sync();
    if (kn >= 0) pf_load_tile(sV, vbase, vstride, kn, nb);  // the V buffer is free again
    cp_async_commit();
    kt = kn;
    ++j;
  }
  if (pend) {
    // a wait ran out: record it, let the MMA in flight finish (bounded) before the columns are
    // freed, and leave this CTA's rows unwritten
    if (t == 0) set_status(P.status, -5);
    mbar_wait(pend == 1 ? barS : barO, j & 1, 2000000000LL);
  }
  // the row sum: this thread's half plus the other half's
  float* lsh = reinterpret_cast<float*>(sm + kPfLsum);
  lsh[t] = l_run;
  __syncthreads();
  if (!pend) {
    uint32_t r[64];
    __syncwarp();
    tmem_ld32(to, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
    tmem_ld32(to + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
    tmem_wait_ld();
    if (row <= q1) {
      const float l_all = lsh[t & (kPfQ - 1)] + lsh[kPfQ + (t & (kPfQ - 1))];
      uint16_t* dst = P.out + (((int64_t)b * P.n_max + row) * L.Hq + h) * kD + 64 * hf;
      const float inv = l_all > 0.f ? 1.f / l_all : 0.f;
#pragma unroll
      for (int c = 0; c < kD / 16; ++c) {
        uint4 w;
        w.x = pack_bf2(__uint_as_float(r[8 * c]) * inv, __uint_as_float(r[8 * c + 1]) * inv);
        w.y = pack_bf2(__uint_as_float(r[8 * c + 2]) * inv, __uint_as_float(r[8 * c + 3]) * inv);
        w.z = pack_bf2(__uint_as_float(r[8 * c + 4]) * inv, __uint_as_float(r[8 * c + 5]) * inv);
        w.w = pack_bf2(__uint_as_float(r[8 * c + 6]) * inv, __uint_as_float(r[8 * c + 7]) * inv);
        *reinterpret_cast<uint4*>(dst + 8 * c) = w;
      }
    }
  }
  cp_async_wait<0>();
  tmem_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tmem_dealloc_cols(tm, kPfTmemCols);
  }
}

}  // namespace rtp
