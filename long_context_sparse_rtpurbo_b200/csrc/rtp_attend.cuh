// Exact softmax attention of the G query heads of one KV head over a list of K/V rows, on the
// tensor cores ("Full Attention Strikes Back" (paper text) §3.2 eq. (5):
// O = sum_n softmax(q^T k_n / sqrt(d)) v_n over the rows of S).
//
// A warp takes tiles of 16 rows. Logits come from mma.sync m16n8k16 (bf16 x bf16 -> fp32)
// with the rows as M, the heads as N (G <= 8 real columns) and the channels as K:
// S^T = K Q^T. The query is split into two bf16 terms (q = q_hi + q_lo, with q_lo the rounded
// remainder), so the logits carry ~16 significant bits of q instead of 8. The probabilities
// P of a tile are transposed in registers (movmatrix) into the B operand of O^T += V^T P^T
// (channels as M, heads as N, the 16 rows as K), again as two bf16 terms, so the result keeps
// fp32-level accuracy; the softmax state (running max, sum) is fp32 in the log2 domain
// (the query carries log2(e)/sqrt(d)).
//
// Staging: rows are copied with cp.async (16 bytes per lane, L2 only) into the warp's own
// tile buffer, 16-byte chunks XOR-swizzled by the row index so the ldmatrix reads of eight
// rows hit eight different bank groups. A warp only reads what it copied itself, so the only
// synchronisation inside the loop is __syncwarp.
#pragma once

#include <cuda_fp16.h>

#include "rtp_common.cuh"

namespace rtp {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async16_s(uint32_t saddr, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr), "l"(gmem) : "memory");
}
// L2 policy for data read once per launch (the index rows, gathered K/V rows, local rings):
// evict first, so the stream does not push the kernel's code and the launch's small shared
// arrays (histograms, statistics, partials) out of L2.
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void cp_async16_s_ef(uint32_t saddr, const void* gmem, uint64_t pol) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;"
               ::"r"(saddr), "l"(gmem), "l"(pol) : "memory");
}
__device__ __forceinline__ void st_shared_zero16(uint32_t saddr) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(saddr), "r"(0u) : "memory");
}
__device__ __forceinline__ void st_shared_u32(uint32_t saddr, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(saddr), "r"(v) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ uint32_t movm_t(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}
// d += A B, m16n8k16, bf16 inputs, fp32 accumulators
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// two floats -> bf16x2 (x in the low half), round to nearest even
__device__ __forceinline__ uint32_t pack_bf2(float x, float y) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(y), "f"(x));
  return r;
}
// (x, y) = hi + lo with hi = bf16(x, y) and lo = bf16 of the exact float remainders
__device__ __forceinline__ void split_bf2(float x, float y, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf2(x, y);
  lo = pack_bf2(x - __uint_as_float(hi << 16), y - __uint_as_float(hi & 0xffff0000u));
}

constexpr int kTileRows = 16;
constexpr int kTileBytes = kTileRows * 512;     // K (16 x 256 B) then V (16 x 256 B)
constexpr int kAccStride = 132;                  // floats per head row of the merge scratch

// Online-softmax state of one warp: heads h0 = 2 (lane & 3) and h0 + 1 of the thread,
// O^T fragments of 8 channel tiles. The query's B fragments are read from a shared buffer.
struct WarpAttn {
  float acc[8][4];
  float m[2], l[2];              // running max; this thread's share of the running sum
  uint32_t qb;                   // shared address of the query buffer (kQBytes)
};

// Query buffer: q_hi and q_lo as bf16 [8 heads][128] each (rows of heads >= G are zero),
// 16-byte chunks XOR-swizzled by the head, so one ldmatrix.x4 per 16-channel step gives the
// B fragments of Q^T (hi: matrices 0, 1; lo: matrices 2, 3).
constexpr int kQBytes = 2 * 8 * kD * 2;

// Fills the query buffer from q_s: [G][128] fp32 query rows pre-scaled by log2(e)/sqrt(d).
// Called by every thread of the CTA; ends with a barrier.
template <int G>
__device__ __forceinline__ void fill_qbuf(unsigned char* qbuf, const float* q_s, int nthreads) {
  for (int e = threadIdx.x; e < 8 * kD / 2; e += nthreads) {
    const int h = e / (kD / 2), c = (e % (kD / 2)) * 2;
    const float x = h < G ? q_s[h * kD + c] : 0.f;
    const float y = h < G ? q_s[h * kD + c + 1] : 0.f;
    uint32_t hi, lo;
    split_bf2(x, y, hi, lo);
    const int off = h * 256 + (((c >> 3) ^ h) << 4) + (c & 7) * 2;
    *reinterpret_cast<uint32_t*>(qbuf + off) = hi;
    *reinterpret_cast<uint32_t*>(qbuf + 2048 + off) = lo;
  }
  __syncthreads();
}

__device__ __forceinline__ void warp_attn_init(WarpAttn& W, const unsigned char* qbuf) {
#pragma unroll
  for (int mt = 0; mt < 8; ++mt)
#pragma unroll
    for (int e = 0; e < 4; ++e) W.acc[mt][e] = 0.f;
  W.m[0] = W.m[1] = -INFINITY;
  W.l[0] = W.l[1] = 0.f;
  W.qb = smem_u32(qbuf);
}

// Copies up to 16 rows into a tile. Lane 2 r holds row r's pointers and flag (the caller's
// lane -> row l / 2 mapping); they are broadcast so that each copy instruction moves two
// whole rows (lane l: row 2 u + l / 16, 16-byte chunk l % 16 of its K and of its V), every
// 128-byte line requested once and whole. Chunks are XOR-swizzled by the row. Rows with
// ok = false get zero V (their logits are masked; a zero V keeps stale shared memory out of
// the P V product).
__device__ __forceinline__ void tile_copy(unsigned char* tile, const uint16_t* krow,
                                          const uint16_t* vrow, bool ok) {
  const int lane = threadIdx.x & 31, c = lane & 15;
  const unsigned long long kq = reinterpret_cast<unsigned long long>(krow);
  const unsigned long long vq = reinterpret_cast<unsigned long long>(vrow);
  const uint32_t okb = __ballot_sync(0xffffffffu, ok);
  const uint64_t pol = l2_evict_first();
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int r = 2 * u + (lane >> 4);
    const unsigned long long kr = __shfl_sync(0xffffffffu, kq, 2 * r);
    const unsigned long long vr = __shfl_sync(0xffffffffu, vq, 2 * r);
    unsigned char* kd = tile + r * 256 + ((c ^ (r & 7)) << 4);
    unsigned char* vd = tile + 4096 + r * 256 + ((c ^ (r & 7)) << 4);
    if ((okb >> (2 * r)) & 1u) {
      cp_async16_s_ef(smem_u32(kd), reinterpret_cast<const uint16_t*>(kr) + c * 8, pol);
      cp_async16_s_ef(smem_u32(vd), reinterpret_cast<const uint16_t*>(vr) + c * 8, pol);
    } else {
      *reinterpret_cast<uint4*>(vd) = make_uint4(0, 0, 0, 0);
    }
  }
}

// One staged tile: nrows valid rows; mask_row: this lane's row (lane / 2) head mask.
template <int G>
__device__ __forceinline__ void tile_attend(WarpAttn& W, const unsigned char* tile, int nrows,
                                            uint32_t mask_row) {
  const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
  const uint32_t tk = smem_u32(tile), tv = tk + 4096;
  float s[4] = {0.f, 0.f, 0.f, 0.f};
  {
    const int r = (lane & 7) + ((lane >> 3) & 1) * 8;     // K row for this lane's address
    const int chi = lane >> 4;
    // query matrices: lane l addresses head l & 7 of matrix l >> 3 (hi: chunk 2kk, 2kk+1;
    // lo: the same chunks 2048 bytes on)
    const int qh = lane & 7, qm = lane >> 3;
    const uint32_t qrow = W.qb + (qm >> 1) * 2048 + qh * 256;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t a[4], b[4];
      ldsm_x4(qrow + (((2 * kk + (qm & 1)) ^ qh) << 4), b);
      ldsm_x4(tk + r * 256 + (((2 * kk + chi) ^ (r & 7)) << 4), a);
      mma_bf16(s, a, b[0], b[1]);
      mma_bf16(s, a, b[2], b[3]);
    }
  }
  // masks of rows gid and gid + 8 (held by lanes 2 gid and 2 gid + 16)
  const uint32_t mk0 = __shfl_sync(0xffffffffu, mask_row, 2 * gid);
  const uint32_t mk1 = __shfl_sync(0xffffffffu, mask_row, 2 * gid + 16);
  const int h0 = 2 * tig;
  const bool r0 = gid < nrows, r1 = gid + 8 < nrows;
  float x[4];
  x[0] = (r0 && ((mk0 >> h0) & 1u)) ? s[0] : -INFINITY;
  x[1] = (r0 && ((mk0 >> (h0 + 1)) & 1u)) ? s[1] : -INFINITY;
  x[2] = (r1 && ((mk1 >> h0) & 1u)) ? s[2] : -INFINITY;
  x[3] = (r1 && ((mk1 >> (h0 + 1)) & 1u)) ? s[3] : -INFINITY;
  float mx0 = fmaxf(x[0], x[2]), mx1 = fmaxf(x[1], x[3]);
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
  }
  const float mn0 = fmaxf(W.m[0], mx0), mn1 = fmaxf(W.m[1], mx1);
  const float al0 = mn0 == -INFINITY ? 1.f : exp2f(W.m[0] - mn0);
  const float al1 = mn1 == -INFINITY ? 1.f : exp2f(W.m[1] - mn1);
  float p[4];
  p[0] = x[0] == -INFINITY ? 0.f : exp2f(x[0] - mn0);
  p[1] = x[1] == -INFINITY ? 0.f : exp2f(x[1] - mn1);
  p[2] = x[2] == -INFINITY ? 0.f : exp2f(x[2] - mn0);
  p[3] = x[3] == -INFINITY ? 0.f : exp2f(x[3] - mn1);
  W.l[0] = W.l[0] * al0 + (p[0] + p[2]);
  W.l[1] = W.l[1] * al1 + (p[1] + p[3]);
  W.m[0] = mn0;
  W.m[1] = mn1;
  if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      W.acc[mt][0] *= al0; W.acc[mt][1] *= al1;
      W.acc[mt][2] *= al0; W.acc[mt][3] *= al1;
    }
  }
  uint32_t h01, l01, h23, l23;
  split_bf2(p[0], p[1], h01, l01);
  split_bf2(p[2], p[3], h23, l23);
  const uint32_t bh0 = movm_t(h01), bh1 = movm_t(h23);
  const uint32_t bl0 = movm_t(l01), bl1 = movm_t(l23);
  {
    const int j = lane >> 3;
    const int r = (lane & 7) + (j >> 1) * 8;             // V row for this lane's address
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      uint32_t a[4];
      ldsm_x4_t(tv + r * 256 + (((2 * mt + (j & 1)) ^ (r & 7)) << 4), a);
      mma_bf16(W.acc[mt], a, bh0, bh1);
      mma_bf16(W.acc[mt], a, bl0, bl1);
    }
  }
}

// Attention of the G heads over a row list, in three steps so a caller can feed the rows
// in batches: attn_begin (state from the query), attn_tiles (rows [0, cnt) of one batch,
// rowfn(i, kp, vp, mask) gives row i), attn_end (merge of the warps' states). Warps
// [0, nwa) take tiles w, w + nwa, ... with one tile buffer each at stage + w * kTileBytes.
template <int G>
__device__ __forceinline__ void attn_begin(WarpAttn& W, unsigned char* qbuf, const float* q_s,
                                           int nthreads) {
  fill_qbuf<G>(qbuf, q_s, nthreads);
  warp_attn_init(W, qbuf);
}

// Issues the copy of each warp's first tile (rows warp * 16 ...), so the loads are in flight
// while the caller prepares the query; attn_tiles(..., first_issued = true) then uses them.
template <class RowFn>
__device__ __forceinline__ void attn_first_copy(int cnt, const RowFn& rowfn, unsigned char* stage,
                                                int nwa) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t0 = warp * kTileRows;
  if (warp >= nwa || t0 >= cnt) return;
  const int i = lane >> 1;
  const int nrows = min(kTileRows, cnt - t0);
  const uint16_t* kp = nullptr;
  const uint16_t* vp = nullptr;
  uint32_t mk = 0;
  if (i < nrows) rowfn(t0 + i, kp, vp, mk);
  tile_copy(stage + warp * kTileBytes, kp, vp, i < nrows && mk != 0);
  cp_async_commit();
}

template <int G, class RowFn>
__device__ __forceinline__ void attn_tiles(WarpAttn& W, int cnt, const RowFn& rowfn,
                                           unsigned char* stage, int nwa, bool first_issued) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (warp >= nwa) return;
  unsigned char* tile = stage + warp * kTileBytes;
  const int i = lane >> 1;
#pragma unroll 1
  for (int t0 = warp * kTileRows; t0 < cnt; t0 += nwa * kTileRows) {
    const int nrows = min(kTileRows, cnt - t0);
    const uint16_t* kp = nullptr;
    const uint16_t* vp = nullptr;
    uint32_t mk = 0;
    if (i < nrows) rowfn(t0 + i, kp, vp, mk);
    if (!(first_issued && t0 == warp * kTileRows)) {
      tile_copy(tile, kp, vp, i < nrows && mk != 0);
      cp_async_commit();
    }
    cp_async_wait<0>();
    __syncwarp();
    tile_attend<G>(W, tile, nrows, mk);
    __syncwarp();                         // the tile is rewritten by the next copy
  }
}

// Merges the warps' states into res[G][2 + 128] (M, L, A) through scratch (>= 16 *
// G * (kAccStride + 2) floats; may alias the tile buffers). Every thread of the CTA calls it.
template <int G>
__device__ __forceinline__ void attn_end(WarpAttn& W, int nwa, float* res, float* scratch,
                                         int nthreads) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = nthreads >> 5;
  const bool active = warp < nwa;
  if (active) {
    // a thread's sum covered its own rows: reduce over the 8 row groups
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      W.l[0] += __shfl_xor_sync(0xffffffffu, W.l[0], o);
      W.l[1] += __shfl_xor_sync(0xffffffffu, W.l[1], o);
    }
  }
  __syncthreads();                        // scratch may alias the tile buffers
  float* sm_ml = scratch + nw * G * kAccStride;           // [nw][G][2]
  if (active) {
    const int gid = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int h = 2 * tig + e;
      if (h < G) {
        float* a = scratch + (warp * G + h) * kAccStride;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          a[mt * 16 + gid] = W.acc[mt][e];
          a[mt * 16 + gid + 8] = W.acc[mt][2 + e];
        }
        if (gid == 0) {
          sm_ml[(warp * G + h) * 2 + 0] = W.m[e];
          sm_ml[(warp * G + h) * 2 + 1] = W.l[e];
        }
      }
    }
  }
  __syncthreads();
  for (int o = threadIdx.x; o < G * kD; o += nthreads) {
    const int h = o / kD, c = o % kD;
    float M = -INFINITY;
    for (int w = 0; w < nwa; ++w) M = fmaxf(M, sm_ml[(w * G + h) * 2]);
    float L = 0.f, A = 0.f;
    if (M != -INFINITY) {
      for (int w = 0; w < nwa; ++w) {
        const float f = exp2f(sm_ml[(w * G + h) * 2] - M);   // 0 for a warp without rows
        L += sm_ml[(w * G + h) * 2 + 1] * f;
        A += scratch[(w * G + h) * kAccStride + c] * f;
      }
    }
    res[h * (kD + 2) + 2 + c] = A;
    if (c == 0) { res[h * (kD + 2)] = M; res[h * (kD + 2) + 1] = L; }
  }
  __syncthreads();
}

// Partial softmax state of the G heads in global memory: per head (m, L) as floats (the
// block padded to 16 bytes), then per head the 128 normalised outputs A / L as fp16 (0 for a
// partial without rows).
template <int G>
struct Part {
  static constexpr int kMLBytes = (8 * G + 15) / 16 * 16;
  static constexpr int kBytes = kMLBytes + 2 * G * kD;
};

// res[G][130] (m, L, A) in shared memory -> the partial at dst. Every thread of the CTA
// calls it (NT threads).
template <int G, int NT>
__device__ __forceinline__ void write_partial(const float* res, unsigned char* dst) {
  float* ml = reinterpret_cast<float*>(dst);
  __half* o = reinterpret_cast<__half*>(dst + Part<G>::kMLBytes);
  for (int i = threadIdx.x; i < G * kD; i += NT) {
    const int h = i / kD, c = i % kD;
    const float L = res[h * (kD + 2) + 1];
    o[i] = __float2half_rn(L > 0.f ? res[h * (kD + 2) + 2 + c] / L : 0.f);
    if (c == 0) { ml[2 * h] = res[h * (kD + 2)]; ml[2 * h + 1] = L; }
  }
}

// Merges n partials (contiguous in global memory, Part<G>::kBytes each, written by other
// CTAs) into the bf16 output rows of the G heads: with M = max_i m_i per head and weights
// w_i = 2^(m_i - M) L_i, O = sum_i w_i O_i / sum_i w_i. When the n partials fit in buf they
// are copied into shared memory with cp.async, all copies in flight at once, and everything
// is read from there: warp h finds M, the weights and their sum for head h (lanes over the
// partials, a fixed butterfly for the sum), then every thread sums its output channels (four
// running sums, added in a fixed order). Otherwise the partials are processed in batches,
// M and the sum of the weights first from global memory. A partial without rows has
// m = -inf and weight 0. sml: G floats of shared memory. Every thread of the CTA calls it;
// NT threads.
template <int G, int NT>
__device__ __forceinline__ void merge_all(const unsigned char* parts, int n, uint16_t* out_rows,
                                          unsigned char* buf, int buf_bytes, float* sml) {
  constexpr int PB = Part<G>::kBytes, ML = Part<G>::kMLBytes;
  constexpr int kPer = (G * kD + NT - 1) / NT;       // outputs per thread
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int per = max(1, buf_bytes / (PB + 4 * G));  // partials per batch (data + weights)
  float* wbuf = reinterpret_cast<float*>(buf + per * PB);
  const bool one = n <= per;
  {
    const int nb = min(per, n);
    for (int i = t; i < nb * (PB / 16); i += NT) cp_async16(buf + 16 * i, parts + 16 * i);
    cp_async_commit();
  }
  if (one) {
    cp_async_wait<0>();
    __syncthreads();
    if (warp < G) {
      float m = -INFINITY;
      for (int i = lane; i < n; i += 32)
        m = fmaxf(m, reinterpret_cast<const float*>(buf + i * PB)[2 * warp]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float W = 0.f;
      for (int i = lane; i < n; i += 32) {
        const float* ml = reinterpret_cast<const float*>(buf + i * PB);
        const float w = ml[2 * warp] == -INFINITY ? 0.f : exp2f(ml[2 * warp] - m) * ml[2 * warp + 1];
        wbuf[i * G + warp] = w;
        W += w;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) W += __shfl_xor_sync(0xffffffffu, W, o);
      if (lane == 0) sml[warp] = W;
    }
  } else if (warp < G) {
    float m = -INFINITY;
    for (int i = lane; i < n; i += 32)
      m = fmaxf(m, __ldcg(reinterpret_cast<const float*>(parts + (int64_t)i * PB) + 2 * warp));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float W = 0.f;
    for (int i = lane; i < n; i += 32) {
      const float* ml = reinterpret_cast<const float*>(parts + (int64_t)i * PB);
      const float mi = __ldcg(ml + 2 * warp);
      if (mi != -INFINITY) W += exp2f(mi - m) * __ldcg(ml + 2 * warp + 1);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) W += __shfl_xor_sync(0xffffffffu, W, o);
    if (lane == 0) { sml[warp] = W; sml[G + warp] = m; }
  }
  float acc[kPer][4];
#pragma unroll
  for (int u = 0; u < kPer; ++u)
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[u][k] = 0.f;
#pragma unroll 1
  for (int b0 = 0; b0 < n; b0 += per) {
    const int nb = min(per, n - b0);
    if (!one) {
      if (b0 > 0) {
        for (int i = t; i < nb * (PB / 16); i += NT)
          cp_async16(buf + 16 * i, parts + (int64_t)b0 * PB + 16 * i);
        cp_async_commit();
      }
      __syncthreads();                               // sml (first batch) is ready
      for (int idx = t; idx < nb * G; idx += NT) {
        const int i = idx / G, h = idx % G;
        const float* ml = reinterpret_cast<const float*>(parts + (int64_t)(b0 + i) * PB);
        const float M = sml[G + h], mi = __ldcg(ml + 2 * h);
        wbuf[idx] = (mi == -INFINITY || M == -INFINITY) ? 0.f : exp2f(mi - M) * __ldcg(ml + 2 * h + 1);
      }
      cp_async_wait<0>();
    }
    __syncthreads();
    const __half* ob = reinterpret_cast<const __half*>(buf + ML);
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int o = t + u * NT;
      if (o < G * kD) {
        const int h = o / kD;
        const __half* src = ob + o;
        int i = 0;
#pragma unroll 1
        for (; i + 4 <= nb; i += 4) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            acc[u][k] = fmaf(__half2float(src[(i + k) * (PB / 2)]), wbuf[(i + k) * G + h], acc[u][k]);
        }
        for (; i < nb; ++i) acc[u][0] = fmaf(__half2float(src[i * (PB / 2)]), wbuf[i * G + h], acc[u][0]);
      }
    }
    __syncthreads();                                 // buf is rewritten by the next batch
  }
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int o = t + u * NT;
    if (o < G * kD) {
      const int h = o / kD;
      const float A = (acc[u][0] + acc[u][1]) + (acc[u][2] + acc[u][3]);
      const float W = sml[h];
      out_rows[o] = f2bf_rn(W > 0.f ? A / W : 0.f);
    }
  }
  __syncthreads();                                   // the caller may reuse buf and sml
}

}  // namespace rtp
