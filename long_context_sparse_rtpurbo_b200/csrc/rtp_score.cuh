// Index scores on the tensor cores ("Full Attention Strikes Back" (paper text) §3.2 eq. (4):
// s(m, n) = (W^Q q^pre)^T (W^K k^pre), a 16-term dot product per token and query head).
//
// A warp scores 32 staged index rows at a time with mma.sync m16n8k16 (bf16 x bf16 -> fp32):
// the rows are M, the 16 index channels K, the query heads N. The fp32 index query is split
// into three bf16 terms (q = hi + mid + lo, each the rounded remainder of the previous), so
// the products keep the full 24-bit query and the score carries fp32-level error; each term
// has its own accumulator and the score is (hi + mid) + lo. With G <= 4 heads the 8 columns
// hold both 16-row halves of the tile: columns [0, G) score rows 0..15 and columns [G, 2G)
// rows 16..31 (K is folded twice, the B operand block-diagonal), so no column is idle for
// G = 4; with G = 8 each half is its own m16n8 tile.
//
// Lane layout of the result (gid = lane / 4, tig = lane % 4): value v of a lane belongs to
// slot e = v % 2 (head head[e], a real column when ok[e]) and to tile row row[v]. Every
// (row, head) pair of the 32 x G scores is held by exactly one (lane, value).
//
// Staged rows are 32 bytes; the two 16-byte halves of rows 4..7 (mod 8) are swapped so the
// eight row addresses of an ldmatrix phase fall in distinct bank groups.
#pragma once

#include "rtp_attend.cuh"

namespace rtp {

constexpr int kWRows = 32;                       // index rows per warp tile

// byte offset of half hh (0, 1) of row r in a staged tile
__device__ __forceinline__ int idx_half_off(int r, int hh) {
  return r * 32 + ((hh ^ ((r >> 2) & 1)) << 4);
}

// x, y -> three bf16x2 terms (x in the low halves); each subtraction is exact
__device__ __forceinline__ void split3_bf2(float x, float y, uint32_t& h, uint32_t& m,
                                           uint32_t& l) {
  h = pack_bf2(x, y);
  const float rx = x - __uint_as_float(h << 16), ry = y - __uint_as_float(h & 0xffff0000u);
  m = pack_bf2(rx, ry);
  const float sx = rx - __uint_as_float(m << 16), sy = ry - __uint_as_float(m & 0xffff0000u);
  l = pack_bf2(sx, sy);
}

template <int G>
struct ScoreTile {
  static constexpr int V = G == 8 ? 8 : 4;       // scores per lane per tile
  static constexpr int KS = G == 8 ? 1 : 2;      // k-steps (row halves folded into K)
  uint32_t b[KS][3][2];                          // B fragments [k-step][hi, mid, lo][reg]
  int row[V];                                    // tile row of value v
  int head[2];                                   // head of slot e
  bool ok[2];                                    // slot e is a real column

  // qidx: [G][16] fp32 index query (shared memory)
  __device__ __forceinline__ void init(const float* qidx) {
    const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int s = 0; s < KS; ++s) {
      int h;
      bool real;
      if (G == 8) { h = gid; real = true; }
      else { h = gid % G; real = gid < 2 * G && gid / G == s; }
      const float* q = qidx + h * kR;
      const float x0 = real ? q[2 * tig] : 0.f, x1 = real ? q[2 * tig + 1] : 0.f;
      const float x2 = real ? q[2 * tig + 8] : 0.f, x3 = real ? q[2 * tig + 9] : 0.f;
      split3_bf2(x0, x1, b[s][0][0], b[s][1][0], b[s][2][0]);
      split3_bf2(x2, x3, b[s][0][1], b[s][1][1], b[s][2][1]);
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int n = 2 * tig + e;
      head[e] = G == 8 ? n : n % G;
      ok[e] = G == 8 ? true : n < 2 * G;
    }
#pragma unroll
    for (int v = 0; v < V; ++v) {
      const int m = gid + 8 * ((v >> 1) & 1);
      if (G == 8) {
        row[v] = 16 * (v >> 2) + m;
      } else {
        const int n = 2 * tig + (v & 1);
        row[v] = n < 2 * G ? 16 * (n / G) + m : m;
      }
    }
  }

  // scores of the 32 rows staged at shared address `slot`
  __device__ __forceinline__ void score(uint32_t slot, float (&c)[V]) const {
    const int lane = threadIdx.x & 31;
    const int r = (lane & 7) + ((lane >> 3) & 1) * 8;
    const uint32_t off = (uint32_t)idx_half_off(r, lane >> 4);
    uint32_t a0[4], a1[4];
    ldsm_x4(slot + off, a0);
    ldsm_x4(slot + 512 + off, a1);             // rows 16..31: the same swap pattern
    // one accumulator per query term (short dependency chains), added hi + mid, then + lo
    if constexpr (G == 8) {
      float d[2][3][4];
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int t = 0; t < 3; ++t) {
#pragma unroll
          for (int i = 0; i < 4; ++i) d[j][t][i] = 0.f;
          mma_bf16(d[j][t], j ? a1 : a0, b[0][t][0], b[0][t][1]);
        }
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int i = 0; i < 4; ++i) c[4 * j + i] = (d[j][0][i] + d[j][1][i]) + d[j][2][i];
    } else {
      float d[3][4];
#pragma unroll
      for (int t = 0; t < 3; ++t) {
#pragma unroll
        for (int i = 0; i < 4; ++i) d[t][i] = 0.f;
        mma_bf16(d[t], a0, b[0][t][0], b[0][t][1]);   // columns of the low half (zero elsewhere)
        mma_bf16(d[t], a1, b[KS - 1][t][0], b[KS - 1][t][1]);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) c[i] = (d[0][i] + d[1][i]) + d[2][i];
    }
  }
};

}  // namespace rtp
