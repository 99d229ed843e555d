// Causal prefill attention ("Full Attention Strikes Back" (paper text) §3.2: retrieval heads
// use dense attention in prefill, local heads attention sinks plus a sliding window in prefill
// and decode), for a prompt at positions 0..n_b-1 of each sequence.
//
// prefill_rope_keys: the prompt's keys rotated by R(j) with the append's arithmetic (double
// angles and rotation, one rounding to bf16), so they equal the cache rows the append writes;
// local heads need them because their ring keeps only the last window.
// prefill_kernel: one CTA of 4 warps per (64 query rows, query head, sequence); K/V tiles of
// 64 rows, double-buffered with cp.async (16-byte chunks XOR-swizzled by the row), over the
// tiles the head can see (causal; local heads skip the tiles between the sinks and the
// window). Per warp 16 query rows: S = Q K^T and O += P V on the tensor cores (mma.sync
// m16n8k16, bf16 x bf16 -> fp32), the query and the probabilities each as two bf16 terms (the
// rounded value and its rounded remainder) so logits and outputs keep fp32-level accuracy;
// online softmax in the log2 domain (the query carries log2(e) / sqrt(128)).
#pragma once

#include "rtp_append.cuh"
#include "rtp_attend.cuh"

namespace rtp {

constexpr int kPfThreads = 128;      // 4 warps
constexpr int kPfQ = 64;             // query rows per CTA (16 per warp)
constexpr int kPfK = 64;             // key rows per tile
constexpr int kPfQBytes = 2 * kPfQ * 256;            // q hi, q lo: [64 rows][256 B] each
constexpr int kPfTileBytes = 2 * kPfK * 256;         // K then V
constexpr int kPfSmem = kPfQBytes + 2 * kPfTileBytes;   // 96 KB

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

// byte offset of channel c (bf16) of row r in a 256-byte-row tile with swizzled chunks
__device__ __forceinline__ int pf_off(int r, int c) {
  return r * 256 + ((((c >> 3) ^ (r & 7))) << 4) + (c & 7) * 2;
}

// next key tile at or after kt that a query tile [q0, q1] can see (-1: none); local heads see
// keys [0, sinks) and (q0 - window, q1]
__device__ __forceinline__ int pf_next_tile(int kt, int q0, int q1, bool local, int sinks,
                                            int window) {
  const int last = q1 / kPfK;
  for (; kt <= last; ++kt) {
    if (!local) return kt;
    const int k0 = kt * kPfK, k1 = k0 + kPfK - 1;
    if (k0 < sinks || k1 > q0 - window) return kt;
  }
  return -1;
}

__global__ void __launch_bounds__(kPfThreads)
prefill_kernel(LayerShape L, const uint16_t* __restrict__ q_pre, const uint16_t* __restrict__ k_rope,
               const uint16_t* __restrict__ v, const int32_t* __restrict__ n_b, int n_max,
               uint16_t* __restrict__ out) {
  extern __shared__ __align__(16) unsigned char pf_smem[];
  // the longest causal rows first, so the short tiles fill the tail of the grid
  const int qt = gridDim.x - 1 - blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int nb = min(max(n_b[b], 0), n_max);
  const int q0 = qt * kPfQ;
  if (q0 >= nb) return;
  const int q1 = min(q0 + kPfQ, nb) - 1;                 // last query row of the CTA
  const int g = h / L.G;
  const bool local = L.slot[g] < 0;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5, gid = lane >> 2, tig = lane & 3;
  unsigned char* qs = pf_smem;                            // hi, then lo at + kPfQ * 256
  unsigned char* tiles = pf_smem + kPfQBytes;
  const uint16_t* kbase = k_rope + ((int64_t)b * L.Hkv + g) * n_max * kD;

  auto issue = [&](int kt, int stage) {
    unsigned char* kd = tiles + stage * kPfTileBytes;
    unsigned char* vd = kd + kPfK * 256;
#pragma unroll
    for (int u = 0; u < (kPfK * 16) / kPfThreads; ++u) {
      const int e = t + u * kPfThreads, r = e >> 4, c = e & 15;
      const int key = kt * kPfK + r;
      const int off = r * 256 + ((c ^ (r & 7)) << 4);
      if (key < nb) {
        cp_async16(kd + off, kbase + (int64_t)key * kD + c * 8);
        cp_async16(vd + off, v + (((int64_t)b * n_max + key) * L.Hkv + g) * kD + c * 8);
      } else {                                            // zero V: masked keys must add 0
        *reinterpret_cast<uint4*>(vd + off) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    cp_async_commit();
  };

  int kt = pf_next_tile(0, q0, q1, local, L.sinks, L.window);
  issue(kt, 0);
  // the rotated, scaled query rows, split into two bf16 terms
  const float scale = kLog2e * 0.08838834764831845f;    // log2(e) / sqrt(128)
  for (int e = t; e < kPfQ * 64; e += kPfThreads) {
    const int r = e >> 6, i = e & 63, m = q0 + r;
    float x0 = 0.f, x1 = 0.f;
    if (m < nb) {
      const uint16_t* q = q_pre + (((int64_t)b * n_max + m) * L.Hq + h) * kD;
      float sn, cs;
      rope_sincosf((double)m, L.theta[i], &sn, &cs);
      const float qa = bf1(q[i]), qb = bf1(q[i + 64]);
      x0 = (qa * cs - qb * sn) * scale;
      x1 = (qa * sn + qb * cs) * scale;
    }
    uint32_t h0, l0, h1, l1;
    split_bf2(x0, 0.f, h0, l0);
    split_bf2(x1, 0.f, h1, l1);
    *reinterpret_cast<uint16_t*>(qs + pf_off(r, i)) = (uint16_t)h0;
    *reinterpret_cast<uint16_t*>(qs + kPfQ * 256 + pf_off(r, i)) = (uint16_t)l0;
    *reinterpret_cast<uint16_t*>(qs + pf_off(r, i + 64)) = (uint16_t)h1;
    *reinterpret_cast<uint16_t*>(qs + kPfQ * 256 + pf_off(r, i + 64)) = (uint16_t)l1;
  }

  float o[16][4];
#pragma unroll
  for (int d = 0; d < 16; ++d)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[d][e] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  const int row0 = q0 + warp * 16 + gid;                  // this thread's rows: row0, row0 + 8
  const uint32_t qaddr = smem_u32(qs);
  int stage = 0;
#pragma unroll 1
  while (kt >= 0) {
    const int kn = pf_next_tile(kt + 1, q0, q1, local, L.sinks, L.window);
    cp_async_wait<0>();
    __syncthreads();                                      // tile kt landed; the other stage is free
    if (kn >= 0) issue(kn, stage ^ 1);
    const uint32_t kaddr = smem_u32(tiles + stage * kPfTileBytes);
    const uint32_t vaddr = kaddr + kPfK * 256;
    // S = Q K^T: 16 rows x 64 keys (8 key tiles of 8)
    float s[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[n][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t ah[4], al[4];
      {
        const int r = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8, c = 2 * kk + (lane >> 4);
        const uint32_t off = r * 256 + ((c ^ (r & 7)) << 4);
        ldsm_x4(qaddr + off, ah);
        ldsm_x4(qaddr + kPfQ * 256 + off, al);
      }
#pragma unroll
      for (int np = 0; np < 4; ++np) {                     // key tiles 2 np, 2 np + 1
        uint32_t bk[4];
        const int r = (2 * np + (lane >> 4)) * 8 + (lane & 7), c = 2 * kk + ((lane >> 3) & 1);
        ldsm_x4(kaddr + r * 256 + ((c ^ (r & 7)) << 4), bk);
        mma_bf16(s[2 * np], ah, bk[0], bk[1]);
        mma_bf16(s[2 * np], al, bk[0], bk[1]);
        mma_bf16(s[2 * np + 1], ah, bk[2], bk[3]);
        mma_bf16(s[2 * np + 1], al, bk[2], bk[3]);
      }
    }
    // masks and the online softmax (rows row0 and row0 + 8; a quad of lanes shares a row)
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int n = 0; n < 8; ++n) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int row = row0 + (e >> 1) * 8;
        const int key = kt * kPfK + n * 8 + 2 * tig + (e & 1);
        bool ok = key <= row && key < nb;
        if (local) ok = ok && (key < L.sinks || key > row - L.window);
        s[n][e] = ok ? s[n][e] : -INFINITY;
        mx[e >> 1] = fmaxf(mx[e >> 1], s[n][e]);
      }
    }
    float al2[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      mx[u] = fmaxf(mx[u], __shfl_xor_sync(0xffffffffu, mx[u], 1));
      mx[u] = fmaxf(mx[u], __shfl_xor_sync(0xffffffffu, mx[u], 2));
      const float mn = fmaxf(mrow[u], mx[u]);
      al2[u] = mn == -INFINITY ? 1.f : exp2f(mrow[u] - mn);
      mrow[u] = mn;
      lrow[u] *= al2[u];
    }
#pragma unroll
    for (int d = 0; d < 16; ++d) {
      o[d][0] *= al2[0]; o[d][1] *= al2[0];
      o[d][2] *= al2[1]; o[d][3] *= al2[1];
    }
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float m = mrow[e >> 1];
        const float pv = s[n][e] == -INFINITY ? 0.f : exp2f(s[n][e] - m);
        s[n][e] = pv;
        lrow[e >> 1] += pv;
      }
    // O += P V: P (16 x 64) as the A operand, 4 key steps of 16; V^T fragments by ldmatrix.trans
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t ph[4], pl[4];
      split_bf2(s[2 * kk][0], s[2 * kk][1], ph[0], pl[0]);
      split_bf2(s[2 * kk][2], s[2 * kk][3], ph[1], pl[1]);
      split_bf2(s[2 * kk + 1][0], s[2 * kk + 1][1], ph[2], pl[2]);
      split_bf2(s[2 * kk + 1][2], s[2 * kk + 1][3], ph[3], pl[3]);
#pragma unroll
      for (int dp = 0; dp < 8; ++dp) {                     // dim tiles 2 dp, 2 dp + 1
        uint32_t bv[4];
        const int r = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8, c = 2 * dp + (lane >> 4);
        ldsm_x4_t(vaddr + r * 256 + ((c ^ (r & 7)) << 4), bv);
        mma_bf16(o[2 * dp], ph, bv[0], bv[1]);
        mma_bf16(o[2 * dp], pl, bv[0], bv[1]);
        mma_bf16(o[2 * dp + 1], ph, bv[2], bv[3]);
        mma_bf16(o[2 * dp + 1], pl, bv[2], bv[3]);
      }
    }
    kt = kn;
    stage ^= 1;
  }
  cp_async_wait<0>();
  // the row sums over the quad, then O / l in bf16
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    lrow[u] += __shfl_xor_sync(0xffffffffu, lrow[u], 1);
    lrow[u] += __shfl_xor_sync(0xffffffffu, lrow[u], 2);
  }
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int row = row0 + u * 8;
    if (row > q1) continue;
    uint16_t* dst = out + (((int64_t)b * n_max + row) * L.Hq + h) * kD;
    const float inv = lrow[u] > 0.f ? 1.f / lrow[u] : 0.f;
#pragma unroll
    for (int d = 0; d < 16; ++d) {
      const int c = d * 8 + 2 * tig;
      const uint32_t pk = (uint32_t)f2bf_rn(o[d][2 * u] * inv) |
                          ((uint32_t)f2bf_rn(o[d][2 * u + 1] * inv) << 16);
      *reinterpret_cast<uint32_t*>(dst + c) = pk;
    }
  }
}

}  // namespace rtp
