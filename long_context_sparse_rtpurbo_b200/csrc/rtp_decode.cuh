// Decode step of one layer in one persistent kernel: index scoring, the 256-bin top-p
// threshold, and exact softmax attention over the selected rows (retrieval heads) or over the
// sinks + window (local heads).
//
// "Full Attention Strikes Back" (paper text) §3.2: eq. (4) s(m,n) = (W^Q q^pre)^T (W^K k^pre),
// eq. (5) O = sum over S of softmax(q^T k / sqrt(d)) v with S = Top-P(s, p); local heads use
// attention sinks plus a sliding window. MCISLAB DeepRead notes on RTPurbo, "Method": top-p
// is found sort-free with a 256-bin histogram per head, fused with the scoring.
//
// Work split. A retrieval group is one (sequence, retrieval KV head) with its G query heads;
// its N tokens are cut into chunks of C tokens; chunk k runs on CTA k mod P_ret (CTAs
// [0, P_ret) hold a few chunks each, in group order; CTAs [P_ret, P) start on the local
// heads at once, P_ret following the byte share of the two sides). Per group the chunks pass
// three phases, separated by arrival counters in global memory (two device-wide
// dependencies):
//   S  the chunk's index rows are streamed once from HBM; G scores per row (in log2 units:
//      the index query carries log2(e)); per-chunk (min, max, sum 2^(y - max)) per head. The
//      CTA's last chunk keeps its scores in shared memory; the scores of earlier chunks are
//      recomputed from the index rows, which are still in L2, when their phase H comes.
//   H  from the group's (min, max, total mass): the 256 linear bins and a cutoff bin under
//      which no token can be selected (their total mass is below (1 - p) of the total); per
//      bin fixed-point masses of the tokens at or above the cutoff go to the group's
//      histogram (exact 64-bit sums), and these tokens are emitted as candidates with their
//      bins, in token order. Phase H of a group runs after phase S of the CTA's next group,
//      which hides the wait for the other chunks.
//   W  b* per head from the group's histogram; the group's candidates are split evenly over
//      at most kTeam of the chunks' CTAs; each keeps the candidates with bin >= b* for some
//      head, gathers their K/V rows once for all G heads (tensor-core tiles, a head that did
//      not select a row masks it) and writes a partial softmax state; the last split merges
//      them into the output rows and the selected counts.
// Local items (a slice of one local head's ring) come from a global queue; the chunk CTAs
// drain it when their chunks are done.
// Every wait is bounded (clock64 limit): on expiry the kernel records RTP_ETIMEOUT, raises
// an abort flag that ends every other wait, and returns.
#pragma once

#include "rtp_append.cuh"
#include "rtp_attend.cuh"
#include "rtp_tmem.cuh"

namespace rtp {

constexpr int kFThreads = 512;          // threads of the decode kernel
constexpr int kTeam = 32;               // partials merged per team (gather splits per group)
constexpr int kHeadPad = 8;             // words between the heads' rows of shared buffers
constexpr int kHistStride = 256 + kHeadPad;
constexpr int kSplitRows = 64;          // fewest candidates per gather split
constexpr int kMaxSteps = 32;           // chunks per CTA, upper bound
constexpr int kListCap = 4096;          // gather entries staged per batch
// Mass bands of phase S (log2 units, relative to the chunk's first-stage maximum R): band
// i < kBandN covers (R - i + 3, R - i + 4]; kBandOver: above R + 4; kBandTail: at or below
// R - kBandN + 4. In shared memory a band i < kBandN holds its masses scaled by 2^(i - 4 + 19)
// (each rounded up to an integer, so the sum bounds the band's mass from above) in one 32-bit
// word per lane position ([G][kBandN][32]: the lanes of a warp never collide; at most 2^19 per
// row and kMaxChunk / 32 = 4096 rows per word); the over and tail bands are kept in registers
// (the tail as a count). A
// published record holds the band masses relative to R as floats, and R in slot kBandR.
constexpr int kBandN = 26, kBandOver = 26, kBandTail = 27, kBandR = 28, kBandRec = 32;
constexpr int kMaxChunk = 131072;      // rows per chunk, upper bound

struct DecodeParams {
  LayerShape L;
  int P;             // CTAs of the launch
  int C_min;         // smallest chunk (tokens), bounds the chunks per group
  int C_cap;         // chunk tokens whose scores fit the CTA's tensor memory
  int max_nch;       // chunks per group upper bound (workspace arrays)
  int NC_max;        // chunks per launch upper bound (workspace arrays)
  int n_groups;      // B * n_ret
  int n_lgroups;     // B * n_loc
  int PL;            // local items per local group
  int RL;            // ring rows per local item
  int n_loc_items;
  int select_all;    // p >= 1
  double p;
  long long spin_limit;
  int64_t cand_stride;   // candidate entries per group (>= max_seq_len)
  // shared-memory layout (byte offsets into the dynamic buffer)
  int sm_stage, sm_q, sm_qbuf, sm_qidx, sm_hist, sm_res, sm_tmp, sm_int, sm_N, sm_cbase,
      sm_tcache, sm_band, free_bytes;
  // inputs / outputs
  const uint16_t* q_pre;
  const float* w_qidx;
  const int32_t* seq_lens;
  // decode token appended in the same launch (null: appended beforehand): pre-RoPE key and
  // value [B][Hkv][128] bf16 of position seq_lens[b] - 1, W_kidx [Hkv][128][16]
  const uint16_t* k_new;
  const uint16_t* v_new;
  const float* w_kidx;
  CachePtrs cache;
  uint16_t* out;
  int32_t* sel_counts;
  // workspace
  int* status;
  uint32_t* bar;               // [n_groups][4]  S arrivals, H arrivals, teams done  (zeroed)
  uint32_t* team_arr;          // [NC_max]       team arrivals                      (zeroed)
  uint32_t* loc_arr;           // [n_lgroups]    local item arrivals                (zeroed)
  uint32_t* misc;              // [0] local queue head, [1] abort, [2] chunk size     (zeroed)
  unsigned long long* hist;    // [n_groups][G][256] fixed-point bin masses          (zeroed)
  int32_t* hcnt;               // [n_groups][G]  selected tokens per head            (zeroed)
  int32_t* bstar;              // [n_groups][G]  threshold bins (debug output)
  float4* cstat;               // [n_groups][max_nch][G]  chunk (min, max, sum 2^(y - max))
  float* bands;                // [n_groups][max_nch][G][kBandRec] chunk mass bands and R
  uint32_t* ccnt;              // [n_groups][max_nch]     candidates per chunk
  uint32_t* cpos;              // [n_groups][cand_stride] candidate positions
  uint2* cbin;                 // [n_groups][cand_stride] candidate bins (byte h: head h)
  float* part;                 // [NC_max][G][130]
  float* tpart;                // [NC_max][G][130]
  float* lpart;                // [n_loc_items][G][130]
  unsigned long long* trace;   // [P][kTraceEvents] %globaltimer stamps (tracing builds only)
};

// Phase-boundary timestamps, recorded only when built with -DRTP_TRACE.
// Each event keeps its last occurrence; kEvNLocWait / kEvNLocDrain count local items.
enum TraceEvent { kEvStart, kEvPlan, kEvS0, kEvS1, kEvH0, kEvHw, kEvH1, kEvW0, kEvW1, kEvW2,
                  kEvW3, kEvLoc0, kEvLoc1, kEvDrain, kEvEnd, kEvNLocWait, kEvNLocDrain,
                  kEvHs, kEvWl, kEvHb, kEvNCand, kEvBch0, kEvBand0, kTraceEvents = 32 };

// ------------------------------------------------------------------------------ helpers
__device__ __forceinline__ int seq_len_checked(const DecodeParams& P, int b) {
  const int N = __ldg(P.seq_lens + b);
  const int cap = __ldg(P.cache.seq_cap + b);
  const int64_t off = __ldg(P.cache.seq_off + b);
  bool ok = N >= 1 && N <= cap && (int64_t)N <= P.L.maxN;
  if (P.L.n_ret > 0) ok = ok && off >= 0 && off + N <= P.L.T_total;
  return ok ? N : 0;
}

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ int block_sum_int(int v, int* scratch /*>= 32 ints*/) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  int s = 0;
  for (int w = 0; w < kFThreads / 32; ++w) s += scratch[w];
  __syncthreads();
  return s;
}

// Exclusive scan of n ints in smem (in place), n <= kFThreads * 8; returns the total.
__device__ __forceinline__ int block_scan_excl(int* a, int n, int* scratch /*>= 32*/) {
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  constexpr int PER = 8;
  int v[PER], local = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int idx = t * PER + i;
    v[i] = idx < n ? a[idx] : 0;
    local += v[i];
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  __syncthreads();
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  int wbase = 0, total = 0;
  for (int w = 0; w < kFThreads / 32; ++w) {
    const int x = scratch[w];
    wbase += (w < warp) ? x : 0;
    total += x;
  }
  int run = wbase + incl - local;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int idx = t * PER + i;
    if (idx < n) a[idx] = run;
    run += v[i];
  }
  __syncthreads();
  return total;
}

// Last index i in [0, n) with a[i] <= key (a non-decreasing, a[0] <= key).
__device__ __forceinline__ int upper_index(const int* a, int n, int key) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a[mid] <= key) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Dynamic shared memory of the decode kernel; its regions sit at the offsets in DecodeParams.
// The staging region (free_bytes) comes first.
extern __shared__ __align__(16) unsigned char rtp_smem[];

// Shared-memory accesses through byte offsets into rtp_smem, so the compiler always emits
// shared-space instructions (a pointer kept in a struct would be generic).
template <class T>
__device__ __forceinline__ T* smem_at(int off) { return reinterpret_cast<T*>(rtp_smem + off); }

__device__ __forceinline__ void block_flag_prefix_impl(bool flag, int* w, int& before,
                                                       int& total);
__device__ __forceinline__ void block_flag_prefix(bool flag, int wc_off, int par, int& before,
                                                  int& total) {
  block_flag_prefix_impl(flag, smem_at<int>(wc_off) + par * 16, before, total);
}

template <int G> struct Smem {
  const DecodeParams& P;
  __device__ explicit Smem(const DecodeParams& p) : P(p) {}
  __device__ unsigned char* stage() const { return rtp_smem + P.sm_stage; }
  __device__ float* q() const { return (float*)(rtp_smem + P.sm_q); }
  __device__ unsigned char* qbuf() const { return rtp_smem + P.sm_qbuf; }
  __device__ float* qidx() const { return (float*)(rtp_smem + P.sm_qidx); }
  __device__ uint32_t* hist() const { return (uint32_t*)(rtp_smem + P.sm_hist); }
  __device__ float* res() const { return (float*)(rtp_smem + P.sm_res); }
  __device__ double* tmp() const { return (double*)(rtp_smem + P.sm_tmp); }
  __device__ int* ints() const { return (int*)(rtp_smem + P.sm_int); }
  __device__ int* N() const { return (int*)(rtp_smem + P.sm_N); }
  __device__ int* cbase() const { return (int*)(rtp_smem + P.sm_cbase); }
  __device__ double* tcache() const { return (double*)(rtp_smem + P.sm_tcache); }
  __device__ float* band() const { return (float*)(rtp_smem + P.sm_band); }
};
// ints[]: [0..31] reduction scratch, [32] wait flag, [33] next local item, [36] last-split
//         flag, [38] local-last flag, [40..47] b*, [48..55] decode token's index row
//         (16 bf16), [60] tensor-memory base, [64..95] per-warp counts of ordered
//         compactions (two blocks of 16)

// RoPE'd, pre-scaled query of the G heads of KV head kvh at position N - 1 -> q_s[G][128].
template <int G>
__device__ __noinline__ void rope_query(const DecodeParams& P, int b, int kvh, int N,
                                        float* q_s) {
  const int t = threadIdx.x;
  if (t < kD) {
    const int i = t & 63;
    float sn, cs;
    rope_sincosf((double)(N - 1), P.L.theta[i], &sn, &cs);
    const float scale = kLog2e * 0.08838834764831845f;   // log2(e) / sqrt(128)
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const uint16_t* q = P.q_pre + ((int64_t)b * P.L.Hq + kvh * G + h) * kD;
      const float qa = bf1(q[i]), qb = bf1(q[i + 64]);
      const float r = (t < 64) ? (qa * cs - qb * sn) : (qa * sn + qb * cs);
      q_s[h * kD + t] = r * scale;
    }
  }
}

// q_idx[h][j] = log2(e) W_qidx[h]^T q_pre[b][h] for the G heads of kvh (scores in log2 units:
// 2^(y - y_max) = exp(s - s_max), and the bins, linear over [min, max], are the same);
// fixed summation order.
template <int G>
__device__ __forceinline__ void index_query(const DecodeParams& P, int b, int kvh, float* qidx,
                                            float* tmp) {
  constexpr int NO = G * kR;
  constexpr int NPART = kFThreads / NO;
  constexpr int DPP = kD / NPART;
  const int t = threadIdx.x;
  const int o = t % NO, part = t / NO;
  const int h = kvh * G + o / kR, j = o % kR;
  const uint16_t* q = P.q_pre + ((int64_t)b * P.L.Hq + h) * kD + part * DPP;
  const float* w = P.w_qidx + ((int64_t)h * kD + part * DPP) * kR + j;
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < DPP; ++i) acc = fmaf(bf1(q[i]), __ldg(w + i * kR), acc);
  __syncthreads();
  tmp[part * NO + o] = acc;
  __syncthreads();
  if (t < NO) {
    float s = tmp[t];
    for (int pp = 1; pp < NPART; ++pp) s += tmp[pp * NO + t];
    qidx[t] = s * kLog2e;
  }
  __syncthreads();
}

// Every thread gets the number of set flags among the CTA's threads before its own (in
// thread order) and the block total, for an ordered compaction of one block of kFThreads
// items. wc: two arrays of 16 ints used alternately (par = block parity), so one barrier
// per block suffices.
__device__ __forceinline__ void block_flag_prefix(bool flag, int wc_off, int par, int& before,
                                                  int& total);
__device__ __forceinline__ void block_flag_prefix_impl(bool flag, int* w, int& before,
                                                       int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t bal = __ballot_sync(0xffffffffu, flag);
  if (lane == 0) w[warp] = __popc(bal);
  __syncthreads();
  const int v = lane < 16 ? w[lane] : 0;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 16; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const int upto = __shfl_sync(0xffffffffu, incl, warp);      // warps 0..warp
  const int mine = __shfl_sync(0xffffffffu, v, warp);
  total = __shfl_sync(0xffffffffu, incl, 15);
  before = upto - mine + __popc(bal & ((1u << lane) - 1u));
}

// G scores of one 32-byte index row (channel pairs in packed f32x2 multiply-adds, even and
// odd channel sums added at the end). Phases S and H call this same routine, so a recomputed
// score is bit-identical to the first one.
template <int G>
__device__ __forceinline__ void score_row(const float2 (&qi)[G][kR / 2], const unsigned char* row,
                                          float (&s)[G]) {
  const uint4 a = *reinterpret_cast<const uint4*>(row);
  const uint4 c2 = *reinterpret_cast<const uint4*>(row + 16);
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, c2.x, c2.y, c2.z, c2.w};
  float2 x[kR / 2];
#pragma unroll
  for (int jj = 0; jj < kR / 2; ++jj) x[jj] = make_float2(bf_lo(w[jj]), bf_hi(w[jj]));
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float2 a2 = __fmul2_rn(qi[h][0], x[0]);
#pragma unroll
    for (int jj = 1; jj < kR / 2; ++jj) a2 = __ffma2_rn(qi[h][jj], x[jj], a2);
    s[h] = a2.x + a2.y;
  }
}

__device__ __forceinline__ int bin_of(float s, float lo, float inv) {
  return min(kBins - 1, (int)((s - lo) * inv));
}

// ------------------------------------------------------------------------------ kernel
template <int G>
struct DecodeCta {
  const DecodeParams& P;
  Smem<G> sm;
  int C, NC, P_ret;
  bool abort_ = false;

  __device__ explicit DecodeCta(const DecodeParams& p) : P(p), sm(p) {}

  __device__ __forceinline__ int group_of(int k) const { return upper_index(sm.cbase(), P.n_groups, k); }
  __device__ __forceinline__ int nch(int g) const { return sm.cbase()[g + 1] - sm.cbase()[g]; }
  __device__ __forceinline__ int gN(int g) const { return sm.N()[g / P.L.n_ret]; }

  __device__ __forceinline__ void trace(int ev) {
#ifdef RTP_TRACE
    if (threadIdx.x == 0 && P.trace) {
      unsigned long long t;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
      P.trace[(int64_t)blockIdx.x * kTraceEvents + ev] = t;
    }
#else
    (void)ev;
#endif
  }
  __device__ __forceinline__ void trace_count(int ev) {
#ifdef RTP_TRACE
    if (threadIdx.x == 0 && P.trace) P.trace[(int64_t)blockIdx.x * kTraceEvents + ev] += 1;
#else
    (void)ev;
#endif
  }

  // the decode token (position N - 1) of sequence b, KV head kvh into the caches
  __device__ __forceinline__ void append_new(int b, int kvh, int N, uint16_t* idx_patch) {
    const int64_t o = ((int64_t)b * P.L.Hkv + kvh) * kD;
    append_token(P.L, P.cache, P.k_new + o, P.v_new + o, P.w_kidx, b, kvh, (int64_t)(N - 1),
                 sm.tmp(), idx_patch);
  }

  // arrival on a counter after this CTA's writes
  __device__ __forceinline__ void arrive(uint32_t* ctr) {
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      atomicAdd(ctr, 1u);
    }
  }

  // Waits until *ctr >= target: thread 0 polls with acquire loads while the CTA waits at a
  // barrier. false on timeout / abort.
  __device__ __forceinline__ bool wait_for(const uint32_t* ctr, uint32_t target) {
    const long long t0 = clock64();
    volatile uint32_t* abort_flag = P.misc + 1;
    while (true) {
      if (threadIdx.x == 0) {
        int f = 0;
        if (ld_acquire(ctr) >= target) {
          f = 1;
          __threadfence();
        } else if (*abort_flag) {
          f = 2;
        } else if (clock64() - t0 > P.spin_limit) {
          set_status(P.status, -5);
          *abort_flag = 1u;
          __threadfence();
          f = 2;
        }
        sm.ints()[32] = f;
      }
      __syncthreads();
      const int f = sm.ints()[32];
      __syncthreads();
      if (f == 1) return true;
      if (f == 2) return false;
      if (threadIdx.x == 0) __nanosleep(32);
    }
  }

  // ------------------------------------------------------------ plan (every CTA identical)
  __device__ __forceinline__ void plan() {
    const int t = threadIdx.x;
    int sumN = 0, sumL = 0;
    for (int b = t; b < P.L.B; b += kFThreads) {
      const int n = seq_len_checked(P, b);
      sm.N()[b] = n;
      sumN += n;
      sumL += min(n, P.L.ring);
    }
    const long long Tr = (long long)block_sum_int(sumN, sm.ints()) * P.L.n_ret;
    const long long loc_rows = (long long)block_sum_int(sumL, sm.ints()) * P.L.n_loc;
    // CTAs [0, P_ret) take the chunks, the others start on local items at once; the split
    // follows the bytes of each side (index read twice as a proxy for index and gather)
    C = 1024;
    P_ret = 0;
    if (Tr > 0) {
      const double ret_b = 64.0 * (double)Tr, loc_b = 512.0 * (double)loc_rows;
      const int pr = (int)((double)P.P * ret_b / (ret_b + loc_b) + 0.5);
      P_ret = max(1, min(P.P, pr));
      // chunk size: the fewest steps (chunks per CTA) whose chunks fit the score slot, at
      // most kMaxSteps; C >= C_min keeps the chunks per group within the workspace arrays
      long long steps = (Tr + (long long)P_ret * P.C_cap - 1) / ((long long)P_ret * P.C_cap);
      steps = max(1LL, min(steps, (long long)kMaxSteps));
      long long c = P.C_min;
      while (true) {
        const long long den = steps * P_ret - P.n_groups;
        if (den < 1) {
          if (P_ret < P.P) ++P_ret; else ++steps;
          continue;
        }
        c = (Tr + den - 1) / den;
        c = max(c, (long long)P.C_min);
        c = (c + 63) / 64 * 64;
        if ((c > P.C_cap && steps < kMaxSteps) || c > kMaxChunk) { ++steps; continue; }
        break;
      }
      C = (int)c;
    }
    for (int g = t; g < P.n_groups; g += kFThreads) sm.cbase()[g] = (gN(g) + C - 1) / C;
    __syncthreads();
    NC = block_scan_excl(sm.cbase(), P.n_groups, sm.ints());
    if (t == 0) sm.cbase()[P.n_groups] = NC;
    if (blockIdx.x == 0 && t == 0) P.misc[2] = (uint32_t)C;
    // invalid sequences: zero their outputs once (CTA 0) and record the status
    if (blockIdx.x == 0) {
      for (int b = 0; b < P.L.B; ++b) {
        if (sm.N()[b] != 0) continue;
        for (int o = t; o < P.L.Hq * kD; o += kFThreads) P.out[(int64_t)b * P.L.Hq * kD + o] = 0;
        for (int o = t; o < P.L.Hq; o += kFThreads) P.sel_counts[(int64_t)b * P.L.Hq + o] = 0;
        if (t == 0) set_status(P.status, -6);
      }
    }
    __syncthreads();
  }

  // ------------------------------------------------------------ index streaming
  // The chunk's index rows (32 B each, contiguous) stream through a ring of kSStages stages
  // of kSRows rows in the staging region with cp.async (seven stages, 112 KB, in flight);
  // thread t takes row t of each stage and calls fn(nl, ok, y[G]) with its G scores (nl: row
  // within the chunk; ok: the row exists). Every thread calls fn for every stage.
  static constexpr int kSRows = 512, kSStages = 8;
  __device__ __forceinline__ void stream_issue(unsigned char* stage, const unsigned char* src,
                                               int st, int nst, int len) {
    if (st < nst) {
      unsigned char* dst = stage + (st % kSStages) * (kSRows * 32);
      const int rows = min(kSRows, len - st * kSRows);
      for (int piece = threadIdx.x; piece < rows * 2; piece += kFThreads)
        cp_async16(dst + piece * 16, src + ((int64_t)st * kSRows * 32) + piece * 16);
    }
    cp_async_commit();
  }
  template <class Fn>
  __device__ __forceinline__ void stream_chunk(int g, int j, bool patch, Fn& fn) {
    const int b = g / P.L.n_ret, r = g % P.L.n_ret, kvh = P.L.ret_kv[r];
    const int N = gN(g);
    const int n0 = j * C, n1 = min(N, n0 + C), len = n1 - n0;
    const unsigned char* src = (const unsigned char*)(
        P.cache.idx + ((int64_t)r * P.L.T_total + P.cache.seq_off[b] + n0) * kR);
    const int nst = (len + kSRows - 1) / kSRows;
    unsigned char* stage = sm.stage();
    __syncthreads();                       // the staging region may still be in use
#pragma unroll
    for (int st = 0; st < kSStages - 1; ++st) stream_issue(stage, src, st, nst, len);
    index_query<G>(P, b, kvh, sm.qidx(), reinterpret_cast<float*>(sm.tmp()));
    // The chunk holding the decode token writes it while the first stages are in flight; a
    // copy of its index row may still be stale, so the stage holding it is patched below.
    uint16_t* idx_patch = reinterpret_cast<uint16_t*>(sm.ints() + 48);   // 16 bf16
    if (patch) append_new(b, kvh, N, idx_patch);
    float2 qi[G][kR / 2];                    // index query, channel pairs (2j, 2j + 1)
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int jj = 0; jj < kR / 2; ++jj)
        qi[h][jj] = make_float2(sm.qidx()[h * kR + 2 * jj], sm.qidx()[h * kR + 2 * jj + 1]);
#pragma unroll 1
    for (int st = 0; st < nst; ++st) {
      stream_issue(stage, src, st + kSStages - 1, nst, len);
      cp_async_wait<kSStages - 1>();
      __syncthreads();
      const int rows = min(kSRows, len - st * kSRows);
      unsigned char* buf = stage + (st % kSStages) * (kSRows * 32);
      if (patch && st == nst - 1) {        // the last row of the chunk is the decode token
        if (threadIdx.x < kR / 2)
          reinterpret_cast<uint32_t*>(buf + (rows - 1) * 32)[threadIdx.x] =
              reinterpret_cast<const uint32_t*>(idx_patch)[threadIdx.x];
        __syncthreads();
      }
      const int i = threadIdx.x;
      float y[G];
#pragma unroll
      for (int h = 0; h < G; ++h) y[h] = -INFINITY;
      if (i < rows) score_row<G>(qi, buf + i * 32, y);
      fn(st * kSRows + i, i < rows, y);
      __syncthreads();                     // before the stage is refilled
    }
    cp_async_wait<0>();
  }

  // Per-row work of phase S. Per head: min and max; the sum of 2^(y - rf) against a
  // per-thread reference rf (R below, moved up only when a score exceeds it by 64, so the
  // terms never overflow); and the mass 2^(y - R) of the row in its band (shared word of
  // this lane position). R is the maximum of the chunk's first stage, found when that stage
  // is scored (every thread takes part). When the chunk's scores are kept, each stage's G
  // scores go to G tensor-memory columns of the thread's lane (a warp-wide store).
  struct SStats {
    float mn[G], mx[G], rf[G], ls[G], R[G], over[G];
    int tail[G];
    int band_off;                  // byte offsets into rtp_smem: [G][kBandN][32] band words,
    int red_off;                   // [16][G] reduction scratch
    uint32_t tbase;                // tensor-memory base
    bool use_slot;
    __device__ __forceinline__ SStats(uint32_t tb, bool u, int bw, int r)
        : band_off(bw), red_off(r), tbase(tb), use_slot(u) {
#pragma unroll
      for (int k = 0; k < G; ++k) {
        mn[k] = INFINITY; mx[k] = -INFINITY; rf[k] = INFINITY; ls[k] = 0.f; R[k] = 0.f;
        over[k] = 0.f; tail[k] = 0;
      }
    }
    __device__ __forceinline__ void operator()(int nl, bool ok, const float (&y)[G]) {
      if (nl < kSRows) {                     // first stage: R = its maximum per head
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
        float* red = smem_at<float>(red_off);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float v = ok ? y[h] : -INFINITY;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
          if (lane == 0) red[warp * G + h] = v;
        }
        __syncthreads();
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float v = red[h];
          for (int w = 1; w < kFThreads / 32; ++w) v = fmaxf(v, red[w * G + h]);
          R[h] = v;
          rf[h] = v;
        }
        __syncthreads();
      }
      if (use_slot) Tmem<G>::st(tmem_addr(tbase, (nl / kSRows) * G), y);   // whole warp
      if (!ok) return;
      uint32_t* band = smem_at<uint32_t>(band_off) + (threadIdx.x & 31);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        mn[h] = fminf(mn[h], y[h]);
        mx[h] = fmaxf(mx[h], y[h]);
        const float t = R[h] - y[h];
        const float e = exp2f(-t);
        // band: kk = floor(t) in [-8, 30] (round-down add of 1.5 * 2^23), i = kk + 4
        const float tc = fminf(fmaxf(t, -8.f), 30.f);
        const int kk = __float_as_int(__fadd_rd(tc, 12582912.f)) - 0x4B400000;
        if (kk < -4) {
          over[h] += e;
        } else if (kk >= kBandN - 4) {
          ++tail[h];
        } else {                             // e * 2^(kk + 19) lies in (2^18, 2^19]
          const uint32_t q = (uint32_t)__float2uint_ru(e * __int_as_float((kk + 19 + 127) << 23));
          atomicAdd(band + (h * kBandN + kk + 4) * 32, q);
        }
        if (rf[h] == R[h] && t >= -64.f) {
          ls[h] += e;
        } else {                             // a score 64 above R (rare)
          const float d = y[h] - rf[h];
          if (d > 64.f) {
            ls[h] = ls[h] * exp2f(-d) + 1.f;
            rf[h] = y[h];
          } else {
            ls[h] += exp2f(d);
          }
        }
      }
    }
  };

  // Per-row work of phase H: a row whose score reaches ycut for some head is binned; heads
  // whose bin reaches the cutoff add its fixed-point mass to the shared histogram (two 32-bit
  // words per bin, exact), and the row becomes a candidate, written in row order.
  struct HEmit {
    float lo[G], hi[G], inv[G], ycut[G];
    int bch[G];
    int hist_off;                  // byte offsets into rtp_smem: histogram words (lo, hi),
    int wc_off;                    // per-warp counts of the ordered compaction
    uint32_t* cpos;
    uint2* cbin;
    int n0, run, par;
    __device__ __forceinline__ void operator()(int nl, bool ok, const float (&y)[G]) {
      bool pass = false;
#pragma unroll
      for (int h = 0; h < G; ++h) pass |= y[h] >= ycut[h];
      bool cand = false;
      uint32_t bw0 = 0, bw1 = 0;
      uint32_t* hlo = smem_at<uint32_t>(hist_off);
      uint32_t* hhi = hlo + G * kHistStride;
      if (ok && pass) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const int b = inv[h] > 0.f ? bin_of(y[h], lo[h], inv[h]) : 0;
          if (h < 4) bw0 |= (uint32_t)b << (8 * h); else bw1 |= (uint32_t)b << (8 * (h - 4));
          if (b >= bch[h]) {
            cand = true;
            const float ex = y[h] - hi[h];
            if (ex > -42.f) {                // below 2^-41 the fixed-point mass rounds to 0
              const unsigned long long q = __float2ull_rn(exp2f(ex) * kMassScale);
              const int bi = h * kHistStride + b;
              const uint32_t ql = (uint32_t)q, qh = (uint32_t)(q >> 32);
              const uint32_t old = atomicAdd(&hlo[bi], ql);
              const uint32_t up = qh + ((old + ql < old) ? 1u : 0u);
              if (up) atomicAdd(&hhi[bi], up);
            }
          }
        }
      }
      int before, total;
      block_flag_prefix(cand, wc_off, par, before, total);
      if (cand) {
        cpos[run + before] = (uint32_t)(n0 + nl);
        cbin[run + before] = make_uint2(bw0, bw1);
      }
      run += total;
      par ^= 1;
    }
  };

  // Rows of the attention loop: the gather list (position << 8 | head mask) or a contiguous
  // range of ring rows.
  struct ListRows {
    const uint32_t* list;
    const uint16_t* kb;
    const uint16_t* vb;
    __device__ __forceinline__ void operator()(int i, const uint16_t*& kp, const uint16_t*& vp,
                                               uint32_t& mk) const {
      const uint32_t w = list[i];
      kp = kb + (int64_t)(w >> 8) * kD;
      vp = vb + (int64_t)(w >> 8) * kD;
      mk = w & 0xffu;
    }
  };
  struct RangeRows {
    const uint16_t* kb;
    const uint16_t* vb;
    __device__ __forceinline__ void operator()(int i, const uint16_t*& kp, const uint16_t*& vp,
                                               uint32_t& mk) const {
      kp = kb + (int64_t)i * kD;
      vp = vb + (int64_t)i * kD;
      mk = 0xffu;
    }
  };

  // ------------------------------------------------------------ phase S
  // Per head: min, max, and the sum of 2^(y - r) against a per-thread reference r (the first
  // score, moved up only when a score exceeds it by 64, so 2^(y - r) never overflows and the
  // common step is one exponential and one add).
  __device__ __forceinline__ void phase_score(int k, bool use_slot) {
    const int g = group_of(k), j = k - sm.cbase()[g];
    const int N = gN(g);
    const bool patch = P.k_new && min(N, (j + 1) * C) == N;
    float* bnd = sm.band();                  // [G][kBandN][32]
    for (int i = threadIdx.x; i < G * kBandN * 32; i += kFThreads) bnd[i] = 0.f;
    SStats sst((uint32_t)sm.ints()[60], use_slot, P.sm_band, P.sm_tmp);
    trace(kEvS0);
    stream_chunk(g, j, patch, sst);             // begins with a barrier (bands zeroed)
    if (use_slot) tmem_wait_st();
    trace(kEvS1);
    float (&mn)[G] = sst.mn;
    float (&mx)[G] = sst.mx;
    float (&rf)[G] = sst.rf;
    float (&ls)[G] = sst.ls;
    // chunk statistics per head: min, max, sum 2^(y - max); warp shuffles, then a fixed-order
    // pass over the warps
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float* red = reinterpret_cast<float*>(sm.tmp());         // [4][G][16]
#pragma unroll
    for (int h = 0; h < G; ++h) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        mn[h] = fminf(mn[h], __shfl_xor_sync(0xffffffffu, mn[h], o));
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], o));
        const float r2 = __shfl_xor_sync(0xffffffffu, rf[h], o);
        const float l2 = __shfl_xor_sync(0xffffffffu, ls[h], o);
        const float rr = fmaxf(rf[h], r2);
        ls[h] = (rr == -INFINITY) ? 0.f : ls[h] * exp2f(rf[h] - rr) + l2 * exp2f(r2 - rr);
        rf[h] = rr;
      }
      if (lane == 0) {
        red[(0 * G + h) * 16 + warp] = mn[h];
        red[(1 * G + h) * 16 + warp] = mx[h];
        red[(2 * G + h) * 16 + warp] = rf[h];
        red[(3 * G + h) * 16 + warp] = ls[h];
      }
    }
    __syncthreads();
    if (threadIdx.x < G) {
      const int h = threadIdx.x;
      float a = INFINITY, z = -INFINITY;
      for (int w = 0; w < kFThreads / 32; ++w) {
        a = fminf(a, red[(0 * G + h) * 16 + w]);
        z = fmaxf(z, red[(1 * G + h) * 16 + w]);
      }
      double l = 0.0;                        // references never exceed the chunk max
      for (int w = 0; w < kFThreads / 32; ++w) {
        const float rw = red[(2 * G + h) * 16 + w];
        if (rw != -INFINITY) l += (double)red[(3 * G + h) * 16 + w] * (double)exp2f(rw - z);
      }
      P.cstat[((int64_t)g * P.max_nch + j) * G + h] = make_float4(a, z, (float)l, 0.f);
    }
    // the chunk's bands: the warps' words (summed in 64 bits and rounded up to float), the
    // over masses and tail counts reduced from the threads, and R
    __syncthreads();
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float ov = sst.over[h];
      int tc = sst.tail[h];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        ov += __shfl_xor_sync(0xffffffffu, ov, o);
        tc += __shfl_xor_sync(0xffffffffu, tc, o);
      }
      if (lane == 0) {
        red[(0 * G + h) * 16 + warp] = ov;
        reinterpret_cast<int*>(red)[(1 * G + h) * 16 + warp] = tc;
      }
    }
    __syncthreads();
    float* gb = P.bands + ((int64_t)g * P.max_nch + j) * G * kBandRec;
    const uint32_t* bnd_u = reinterpret_cast<const uint32_t*>(bnd);
    for (int i = threadIdx.x; i < G * kBandRec; i += kFThreads) {
      const int h = i / kBandRec, k = i % kBandRec;
      float v = 0.f;
      if (k < kBandN) {
        unsigned long long sum = 0;
        for (int l = 0; l < 32; ++l) sum += bnd_u[(h * kBandN + k) * 32 + l];
        v = __fmul_ru(__ull2float_ru(sum), __int_as_float((127 - (k - 4 + 19)) << 23));
      } else if (k == kBandOver) {
        for (int w = 0; w < kFThreads / 32; ++w) v += red[(0 * G + h) * 16 + w];
        v = __fmul_ru(v, 1.001f);               // bounds the rounding of the float sum
      } else if (k == kBandTail) {
        int c = 0;
        for (int w = 0; w < kFThreads / 32; ++w) c += reinterpret_cast<const int*>(red)[(1 * G + h) * 16 + w];
        v = (float)c * exp2f(-(float)(kBandN - 4));    // each at most 2^-(kBandN - 4)
      } else if (k == kBandR) {
        v = sst.R[h];
      }
      gb[i] = v;
    }
    arrive(P.bar + (int64_t)g * 4 + 0);
  }

  // A tighter cutoff from the chunks' mass bands. A band of chunk c holds tokens whose
  // scores lie in an interval (y_low, y_high]; for an edge e the tokens below e are within the
  // bands with y_low < e, so U(e) = sum of those bands' masses (relative to hi) bounds the
  // mass below e from above (a small margin on y_low covers the rounding of the band index).
  // C_b >= T - U(e_b), so every b with T - U(e_b) >= p T satisfies b <= b*; the largest such
  // b is the cutoff when it exceeds the first bound. U is built per head as a scatter of the
  // band masses onto their first bin (shared atomics) and a prefix sum (one warp per head).
  __device__ __forceinline__ void band_cutoff(int g, int nc, int step, HEmit& em) {
    uint32_t* dU = reinterpret_cast<uint32_t*>(sm.hist());  // [G][257], units of T 2^-27
    for (int i = threadIdx.x; i < G * 257; i += kFThreads) dU[i] = 0u;
    __syncthreads();
    if (!P.select_all) {
      const float* gb = P.bands + (int64_t)g * P.max_nch * G * kBandRec;
      const int tot = nc * G * kBandRec;
      for (int i = threadIdx.x; i < tot; i += kFThreads) {
        const int k = i % kBandRec, h = (i / kBandRec) % G;
        if (k >= kBandR) continue;
        const float v = __ldcg(gb + i);
        if (!(v > 0.f)) continue;
        const float Rc = __ldcg(gb + (i - k) + kBandR);
        float hi = 0.f, lo = 0.f, inv = 0.f;
#pragma unroll
        for (int hh = 0; hh < G; ++hh)
          if (hh == h) { hi = em.hi[hh]; lo = em.lo[hh]; inv = em.inv[hh]; }
        if (!(inv > 0.f)) continue;
        const double T = sm.tcache()[step * G + h];
        // the band's mass relative to the group max, in units of T 2^-27, rounded up (all
        // bands together stay far below 2^32 units: their mass is at most a few T)
        const double mu = (double)v * exp2((double)Rc - (double)hi) / T * 134217728.0;
        const uint32_t q = mu >= 4.0e9 ? 4000000000u : (uint32_t)ceil(mu);
        int b0 = 0;
        if (k != kBandTail) {
          const float ylow = (k == kBandOver ? Rc + 4.f : Rc + 3.f - (float)k) - 0.01f;
          const float x = (ylow - lo) * inv;
          b0 = x < 0.f ? 0 : min(256, (int)x + 1);
        }
        if (q) atomicAdd(dU + h * 257 + b0, q);
      }
    }
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (warp < G && !P.select_all) {
      const int h = warp;
      float inv = 0.f;
#pragma unroll
      for (int hh = 0; hh < G; ++hh) if (hh == h) inv = em.inv[hh];
      if (inv > 0.f) {
        // lane l holds bins 8l .. 8l + 7: inclusive prefix of dU (64-bit sums)
        unsigned long long v[8], run = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) { run += dU[h * 257 + lane * 8 + e]; v[e] = run; }
        unsigned long long incl = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned long long y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const unsigned long long base = incl - run;
        // U(e_b) / T = prefix 2^-27 (each part rounded up); b is certified when
        // 1 - 1.001 U / T >= p
        int best = -1;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const double u = (double)(base + v[e]) * (1.0 / 134217728.0) * 1.001;
          if (1.0 - u >= P.p) best = lane * 8 + e;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) best = max(best, __shfl_xor_sync(0xffffffffu, best, o));
        if (lane == 0) sm.ints()[40 + h] = best;
      } else if (lane == 0) {
        sm.ints()[40 + h] = -1;
      }
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < G; ++h)
      if (!P.select_all) em.bch[h] = max(em.bch[h], sm.ints()[40 + h]);
    __syncthreads();                       // the scratch is rewritten next
  }

  // ------------------------------------------------------------ phase H
  // Group range and total mass from the chunk statistics (double, fixed order: every CTA
  // gets the same values); the cutoff: with T the group's total mass, every token below
  // bin(c), c = hi + log2((1 - p) T' / N), T' = T (1 - 1e-3), has mass below (1 - p) T' / N,
  // so together they hold less than (1 - p) of the total, C_bin(c) > p T, and b* can not fall
  // under the cutoff bin (the 1e-3 absorbs the rounding of T, the log and the bin edges).
  // A token is binned only when a score reaches half a bin below the cutoff bin's edge (so
  // every token whose bin reaches the cutoff is binned, and the others cost one compare).
  // Masses are 2^(y - max) in 2^-40 fixed point, summed with two 32-bit shared atomics per
  // (token, head): the low-word add returns the old value and its carry goes to the high word.
  __device__ __forceinline__ void phase_hist(int k, int step, bool from_slot) {
    const int g = group_of(k), j = k - sm.cbase()[g];
    const int N = gN(g), n0 = j * C, len = min(N, n0 + C) - n0;
    const int nc = nch(g);
    trace(kEvH0);
    if (!wait_for(P.bar + (int64_t)g * 4 + 0, (uint32_t)nc)) { abort_ = true; return; }
    trace(kEvHw);
    // group statistics: thread t folds chunks t / G, t / G + kFThreads / G, ... of head t % G
    double* part = sm.tmp();                                 // [kFThreads]
    float* st3 = sm.res();                                   // [G][3] lo, hi, inv
    {
      const int t = threadIdx.x, h = t % G;
      float a = INFINITY, z = -INFINITY;
      for (int c = t / G; c < nc; c += kFThreads / G) {
        const float4 v = __ldcg(P.cstat + ((int64_t)g * P.max_nch + c) * G + h);
        a = fminf(a, v.x);
        z = fmaxf(z, v.y);
      }
#pragma unroll
      for (int o = G; o < 32; o <<= 1) {
        a = fminf(a, __shfl_xor_sync(0xffffffffu, a, o));
        z = fmaxf(z, __shfl_xor_sync(0xffffffffu, z, o));
      }
      float* pf = reinterpret_cast<float*>(part);
      if ((t & 31) < G) {
        pf[(t >> 5) * G + h] = a;
        pf[512 + (t >> 5) * G + h] = z;
      }
      __syncthreads();
      if (t < G) {
        float lo = INFINITY, hi = -INFINITY;
        for (int w = 0; w < kFThreads / 32; ++w) {
          lo = fminf(lo, pf[w * G + t]);
          hi = fmaxf(hi, pf[512 + w * G + t]);
        }
        st3[t * 3 + 0] = lo;
        st3[t * 3 + 1] = hi;
        st3[t * 3 + 2] = (hi > lo && !P.select_all) ? (float)kBins / (hi - lo) : 0.f;
      }
      __syncthreads();
      const float hih = st3[h * 3 + 1];
      double acc = 0.0;
      for (int c = t / G; c < nc; c += kFThreads / G) {
        const float4 v = __ldcg(P.cstat + ((int64_t)g * P.max_nch + c) * G + h);
        acc += (double)v.z * (double)exp2f(v.y - hih);
      }
      __syncthreads();
      part[t] = acc;
      __syncthreads();
      if (t < G) {
        double v = 0.0;
        for (int i = t; i < kFThreads; i += G) v += part[i];
        sm.tcache()[step * G + t] = v;
      }
      __syncthreads();
    }
    trace(kEvHs);
    uint32_t* hlo = sm.hist();
    uint32_t* hhi = hlo + G * kHistStride;
    HEmit em;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      em.lo[h] = st3[h * 3 + 0];
      em.hi[h] = st3[h * 3 + 1];
      em.inv[h] = st3[h * 3 + 2];
      em.bch[h] = 0;
      if (P.p < 1.0 && em.inv[h] > 0.f) {
        const double T = sm.tcache()[step * G + h];
        const float arg = (float)((1.0 - P.p) * T * (1.0 - 1e-3) / (double)N);
        const float c = em.hi[h] + log2f(arg);
        em.bch[h] = c > em.lo[h] ? bin_of(c, em.lo[h], em.inv[h]) : 0;
      }
    }
    const int bch_first = em.bch[0];
    band_cutoff(g, nc, step, em);
#ifdef RTP_TRACE
    if (threadIdx.x == 0 && P.trace) {
      P.trace[(int64_t)blockIdx.x * kTraceEvents + kEvBch0] = (unsigned long long)bch_first;
      P.trace[(int64_t)blockIdx.x * kTraceEvents + kEvBand0] = (unsigned long long)em.bch[0];
    }
#endif
    (void)bch_first;
#pragma unroll
    for (int h = 0; h < G; ++h)
      em.ycut[h] = em.bch[h] > 0 ? em.lo[h] + ((float)em.bch[h] - 0.5f) / em.inv[h] : -INFINITY;
    em.hist_off = P.sm_hist;
    em.cpos = P.cpos + (int64_t)g * P.cand_stride + n0;
    em.cbin = P.cbin + (int64_t)g * P.cand_stride + n0;
    em.wc_off = P.sm_int + 64 * 4;          // [2][16]
    em.n0 = n0;
    em.run = 0;
    em.par = 0;
    for (int i = threadIdx.x; i < 2 * G * kHistStride; i += kFThreads) hlo[i] = 0u;
    __syncthreads();
    if (from_slot) {
      const uint32_t tb = (uint32_t)sm.ints()[60];
#pragma unroll 1
      for (int i0 = 0; i0 < len; i0 += kFThreads) {
        const int nl = i0 + threadIdx.x;
        float y[G];
        Tmem<G>::ld(tmem_addr(tb, (i0 / kSRows) * G), y);     // whole warp
        tmem_wait_ld();
        if (nl >= len) {
#pragma unroll
          for (int h = 0; h < G; ++h) y[h] = -INFINITY;
        }
        em(nl, nl < len, y);
        if (i0 == 0) trace(kEvHb);
      }
    } else {
      stream_chunk(g, j, false, em);
    }
    __syncthreads();
    trace(kEvH1);
    unsigned long long* gh = P.hist + (int64_t)g * G * kBins;
    for (int i = threadIdx.x; i < G * kBins; i += kFThreads) {
      const int hh = i / kBins, b = i % kBins;
      const unsigned long long v =
          ((unsigned long long)hhi[hh * kHistStride + b] << 32) | hlo[hh * kHistStride + b];
      if (v) atomicAdd(gh + i, v);
    }
    if (threadIdx.x == 0) P.ccnt[(int64_t)g * P.max_nch + j] = (uint32_t)em.run;
#ifdef RTP_TRACE
    if (threadIdx.x == 0 && P.trace) P.trace[(int64_t)blockIdx.x * kTraceEvents + kEvNCand] += (unsigned long long)em.run;
#endif
    arrive(P.bar + (int64_t)g * 4 + 1);
  }

  __device__ __forceinline__ void merge(const float* parts, int n, float* dst, uint16_t* out_rows,
                                        int buf_bytes) {
    merge_partials<G>(parts, n, dst, out_rows, reinterpret_cast<float*>(sm.stage()), buf_bytes,
                      kFThreads);
  }

  // ------------------------------------------------------------ phase W
  // Split j of group g: candidates [e0, e1) of the group's list (chunk after chunk), loaded
  // in batches of kListCap; a candidate is kept when a head's bin reaches its b*, with the
  // mask of those heads, in candidate order. The list and the chunk prefix sit at the end of
  // the free region (the score slot is dead by now); the tiles use its start. The rotated
  // query is formed before the wait.
  static constexpr int kEPer = kListCap / kFThreads;        // entries per thread per batch
  __device__ __forceinline__ void phase_attend(int k, int step) {
    const int g = group_of(k), j = k - sm.cbase()[g];
    const int b = g / P.L.n_ret, r = g % P.L.n_ret, kvh = P.L.ret_kv[r];
    const int N = gN(g);
    const int S = nch(g);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    rope_query<G>(P, b, kvh, N, sm.q());
    if (!wait_for(P.bar + (int64_t)g * 4 + 1, (uint32_t)S)) { abort_ = true; return; }
    trace(kEvW0);
    const int pref_bytes = ((S + 1) * 4 + 15) / 16 * 16;
    int* pref = reinterpret_cast<int*>(sm.stage() + P.free_bytes - pref_bytes);
    uint32_t* list = reinterpret_cast<uint32_t*>(reinterpret_cast<unsigned char*>(pref) - kListCap * 4);
    // one round trip: the group histogram (warp h: head h) and the chunks' candidate counts
    unsigned long long hv[8];
    if (warp < G && !P.select_all) {
      const unsigned long long* gh = P.hist + ((int64_t)g * G + warp) * kBins + lane * 8;
#pragma unroll
      for (int e = 0; e < 8; ++e) hv[e] = __ldcg(gh + e);
    }
    for (int c = threadIdx.x; c < S; c += kFThreads)
      pref[c] = (int)__ldcg(P.ccnt + (int64_t)g * P.max_nch + c);
    // b* per head: the highest bin whose mass from the top reaches p T
    if (warp < G) {
      int best = 0;
      if (!P.select_all) {
        unsigned long long lt = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) lt += hv[e];
        unsigned long long x = lt;            // inclusive suffix sum over lanes
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned long long y = __shfl_down_sync(0xffffffffu, x, o);
          if (lane + o < 32) x += y;
        }
        const double thr = P.p * sm.tcache()[step * G + warp] * (double)kMassScale;
        best = -1;
        unsigned long long cum = x - lt;
#pragma unroll
        for (int e = 7; e >= 0; --e) {
          cum += hv[e];
          if (best < 0 && (double)cum >= thr) best = lane * 8 + e;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) best = max(best, __shfl_xor_sync(0xffffffffu, best, o));
        best = max(best, 0);
      }
      if (lane == 0) sm.ints()[40 + warp] = best;
    }
    __syncthreads();
    int bs[G];
#pragma unroll
    for (int h = 0; h < G; ++h) bs[h] = sm.ints()[40 + h];
    if (j == 0 && threadIdx.x < G) P.bstar[(int64_t)g * G + threadIdx.x] = bs[threadIdx.x];
    const int U = block_scan_excl(pref, S, sm.ints());
    const int nsplit = min(min(S, kTeam), max(1, (U + kSplitRows - 1) / kSplitRows));
    if (j >= nsplit) return;
    const int e0 = (int)(((long long)U * j) / nsplit), e1 = (int)(((long long)U * (j + 1)) / nsplit);
    const int64_t rowbase = (int64_t)r * P.L.T_total + P.cache.seq_off[b];
    const uint16_t* kb = P.cache.k_ret + rowbase * kD;
    const uint16_t* vb = P.cache.v_ret + rowbase * kD;
    const uint32_t* gpos = P.cpos + (int64_t)g * P.cand_stride;
    const uint2* gbin = P.cbin + (int64_t)g * P.cand_stride;
    const int nwa = min(kFThreads / 32, (P.free_bytes - pref_bytes - kListCap * 4) / kTileBytes);
    int hc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) hc[h] = 0;
    WarpAttn W;
    attn_begin<G>(W, sm.qbuf(), sm.q(), kFThreads);
    trace(kEvW1);
    const int wc_off = P.sm_int + 64 * 4;
    int par = 0;
#pragma unroll 1
    for (int b0 = e0; b0 < e1; b0 += kListCap) {
      const int b1 = min(e1, b0 + kListCap);
      // all of this thread's entries of the batch in flight at once
      uint32_t pos[kEPer];
      uint2 bw[kEPer];
#pragma unroll
      for (int u = 0; u < kEPer; ++u) {
        const int e = b0 + u * kFThreads + threadIdx.x;
        pos[u] = 0;
        bw[u] = make_uint2(0, 0);
        if (e < b1) {
          const int c = upper_index(pref, S, e);
          const int64_t o = (int64_t)c * C + (e - pref[c]);
          pos[u] = __ldcg(gpos + o);
          bw[u] = __ldcg(gbin + o);
        }
      }
      __syncthreads();                    // the previous batch's list is no longer read
      int nb = 0;                         // kept entries of this batch (every thread)
      const int nu = (b1 - b0 + kFThreads - 1) / kFThreads;   // uniform over the CTA
#pragma unroll
      for (int u = 0; u < kEPer; ++u) {
        if (u < nu) {
          const int e = b0 + u * kFThreads + threadIdx.x;
          uint32_t mask = 0;
          if (e < b1) {
#pragma unroll
            for (int h = 0; h < G; ++h) {
              const int bb = (int)(((h < 4 ? bw[u].x : bw[u].y) >> (8 * (h & 3))) & 0xffu);
              if (bb >= bs[h]) { mask |= 1u << h; hc[h]++; }
            }
          }
          int before, total;
          block_flag_prefix(mask != 0, wc_off, par, before, total);
          par ^= 1;
          if (mask) list[nb + before] = (pos[u] << 8) | mask;
          nb += total;
        }
      }
      __syncthreads();
      trace(kEvWl);
      const ListRows rows{list, kb, vb};
      attn_tiles<G>(W, nb, rows, sm.stage(), nwa, false);
    }
    attn_end<G>(W, nwa, sm.res(), reinterpret_cast<float*>(sm.stage()), kFThreads);
    trace(kEvW2);
    // per-head counts of this split
    int* red = reinterpret_cast<int*>(sm.tmp());              // [16][G]
#pragma unroll
    for (int h = 0; h < G; ++h) {
      int v = hc[h];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) red[warp * G + h] = v;
    }
    __syncthreads();
    if (threadIdx.x < G) {
      int v = 0;
      for (int w = 0; w < kFThreads / 32; ++w) v += red[w * G + threadIdx.x];
      if (v) atomicAdd(P.hcnt + (int64_t)g * G + threadIdx.x, v);
    }
    // partial -> workspace; the last split merges the group's partials
    const int stride = G * (kD + 2);
    float* mine = P.part + (int64_t)k * stride;
    for (int o = threadIdx.x; o < stride; o += kFThreads) mine[o] = sm.res()[o];
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      sm.ints()[36] = atomicAdd(P.team_arr + sm.cbase()[g], 1u) == (uint32_t)(nsplit - 1);
    }
    __syncthreads();
    if (!sm.ints()[36]) return;
    __threadfence();
    merge(P.part + (int64_t)sm.cbase()[g] * stride, nsplit, nullptr,
          P.out + ((int64_t)b * P.L.Hq + kvh * G) * kD, P.free_bytes);
    if (threadIdx.x < G)
      P.sel_counts[(int64_t)b * P.L.Hq + kvh * G + threadIdx.x] =
          __ldcg(P.hcnt + (int64_t)g * G + threadIdx.x);
    trace(kEvW3);
    __syncthreads();
  }

  // ------------------------------------------------------------ local items
  // Attention over one slice of RL ring rows of a local head; the tile copies are issued
  // before the query is loaded. The partials of a head merge by the last arrival.
  __device__ __forceinline__ void local_item(int li) {
    const int lg = li / P.PL, piece = li % P.PL;
    const int b = lg / P.L.n_loc, x = lg % P.L.n_loc, kvh = P.L.loc_kv[x];
    const int N = sm.N()[b];
    if (N == 0) return;                             // invalid sequence: outputs zeroed in plan
    trace(kEvLoc0);
    const int nrows_all = min(N, P.L.ring);
    const int r0 = piece * P.RL;
    const int nrows = max(0, min(nrows_all - r0, P.RL));
    if (P.k_new) {
      const int64_t rr = (N - 1) < P.L.sinks ? (N - 1) : P.L.sinks + (N - 1 - P.L.sinks) % P.L.window;
      if (rr >= r0 && rr < r0 + nrows) append_new(b, kvh, N, nullptr);
    }
    const int64_t ring0 = ((int64_t)x * P.L.B + b) * P.L.ring + r0;
    const int nwa = min(kFThreads / 32, P.free_bytes / kTileBytes);
    const uint16_t* kb = P.cache.k_loc + ring0 * kD;
    const uint16_t* vb = P.cache.v_loc + ring0 * kD;
    const RangeRows rowfn{kb, vb};
    attn_first_copy(nrows, rowfn, sm.stage(), nwa);
    rope_query<G>(P, b, kvh, N, sm.q());
    __syncthreads();
    WarpAttn W;
    attn_begin<G>(W, sm.qbuf(), sm.q(), kFThreads);
    attn_tiles<G>(W, nrows, rowfn, sm.stage(), nwa, true);
    attn_end<G>(W, nwa, sm.res(), reinterpret_cast<float*>(sm.stage()), kFThreads);
    const int stride = G * (kD + 2);
    float* mine = P.lpart + (int64_t)li * stride;
    for (int o = threadIdx.x; o < stride; o += kFThreads) mine[o] = sm.res()[o];
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      sm.ints()[38] = atomicAdd(P.loc_arr + lg, 1u) == (uint32_t)(P.PL - 1);
    }
    __syncthreads();
    if (sm.ints()[38]) {
      __threadfence();
      merge(P.lpart + (int64_t)lg * P.PL * stride, P.PL, nullptr,
            P.out + ((int64_t)b * P.L.Hq + kvh * G) * kD, P.free_bytes);
      if (threadIdx.x < G) P.sel_counts[(int64_t)b * P.L.Hq + kvh * G + threadIdx.x] = nrows_all;
    }
    __syncthreads();
    trace(kEvLoc1);
  }

  // local items from the global queue until it is empty (thread 0 takes the next index while
  // the current item runs, so the queue costs one atomic round trip in total)
  __device__ __forceinline__ void local_items() {
    trace(kEvDrain);
    if (threadIdx.x == 0) sm.ints()[33] = (int)atomicAdd(P.misc + 0, 1u);
    __syncthreads();
    int li = sm.ints()[33];
    while (li < P.n_loc_items) {
      __syncthreads();
      unsigned int next = 0;
      if (threadIdx.x == 0) next = atomicAdd(P.misc + 0, 1u);
      trace_count(kEvNLocDrain);
      local_item(li);
      if (threadIdx.x == 0) sm.ints()[33] = (int)next;
      __syncthreads();
      li = sm.ints()[33];
    }
  }

  // Chunks k_t = blockIdx.x + t P_ret of a chunk CTA, in group order. Phase S runs for every
  // chunk in turn; the chunks of a group get their phase H once the CTA has scored the first
  // chunk of the next group (or at the end), so the wait for the group's other chunks
  // overlaps that scoring. Phase H of every chunk but the last recomputes its scores; the
  // last chunk keeps them in the shared-memory slot when it fits. Then phase W of every
  // chunk, then local items until the queue is empty. CTAs [P_ret, P) only run local items.
  __device__ void run() {
    trace(kEvStart);
    plan();
    trace(kEvPlan);
    const int i = blockIdx.x;
    const int m = (i < P_ret && i < NC) ? (NC - i + P_ret - 1) / P_ret : 0;
    bool last_in_slot = false;
    if (m > 0) {
      const int kl = i + (m - 1) * P_ret, gl = group_of(kl), jl = kl - sm.cbase()[gl];
      last_in_slot = min(gN(gl), (jl + 1) * C) - jl * C <= P.C_cap;
    }
    int pstart = 0;
    for (int t = 0; t < m; ++t) {
      const int k = i + t * P_ret;
      phase_score(k, t == m - 1 && last_in_slot);
      if (pstart < t && group_of(i + pstart * P_ret) != group_of(k)) {
        for (int s = pstart; s < t; ++s) {
          phase_hist(i + s * P_ret, s, false);
          if (abort_) return;
        }
        pstart = t;
      }
    }
    for (int s = pstart; s < m; ++s) {
      phase_hist(i + s * P_ret, s, s == m - 1 && last_in_slot);
      if (abort_) return;
    }
    for (int t = 0; t < m; ++t) {
      phase_attend(i + t * P_ret, t);
      if (abort_) return;
    }
    local_items();
    trace(kEvEnd);
  }
};

// The CTA's tensor memory is allocated by warp 0 before anything else and freed by warp 0
// after every thread has left run() (run returns on every path, aborts included).
template <int G>
__global__ void __launch_bounds__(kFThreads, 1) decode_kernel(const __grid_constant__ DecodeParams P) {
  int* tw = reinterpret_cast<int*>(rtp_smem + P.sm_int) + 60;
  if ((threadIdx.x >> 5) == 0) tmem_alloc(smem_u32(tw));
  tmem_fence_before_sync();
  __syncthreads();
  tmem_fence_after_sync();
  DecodeCta<G> cta(P);
  cta.run();
  tmem_fence_before_sync();
  __syncthreads();
  tmem_fence_after_sync();
  if ((threadIdx.x >> 5) == 0) tmem_dealloc((uint32_t)*tw);
}

// ------------------------------------------------------------------------------ sel_idx
// Debug output: ascending positions each query head attended to. One CTA per (b, h): the
// selected candidates of the head are marked in a shared-memory bitmap window of kEmitBits
// positions, which is then read in order.
constexpr int kEmitBits = 1 << 18;
template <int G>
__global__ void __launch_bounds__(kThreads) emit_sel_kernel(DecodeParams P, int32_t* sel_idx,
                                                            int64_t sel_stride) {
  __shared__ uint32_t bm[kEmitBits / 32];
  __shared__ int wsum[kThreads / 32];
  const int b = blockIdx.x / P.L.Hq, h = blockIdx.x % P.L.Hq;
  const int kvh = h / G, jh = h % G;
  const int N = seq_len_checked(P, b);
  int32_t* dst = sel_idx + ((int64_t)b * P.L.Hq + h) * sel_stride;
  if (N == 0) return;
  const int slot = P.L.slot[kvh];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  if (slot < 0) {
    const int s1 = min(N, P.L.sinks);
    const int w0 = max(P.L.sinks, N - P.L.window);
    const int cnt = s1 + max(0, N - w0);
    for (int k = t; k < cnt; k += kThreads) dst[k] = k < s1 ? k : w0 + (k - s1);
    return;
  }
  const int g = b * P.L.n_ret + slot;
  const int C = (int)__ldcg(P.misc + 2);
  const int nchg = (N + C - 1) / C;
  const int bst = __ldcg(P.bstar + (int64_t)g * G + jh);
  const uint32_t* gpos = P.cpos + (int64_t)g * P.cand_stride;
  const uint2* gbin = P.cbin + (int64_t)g * P.cand_stride;
  int base = 0;
  constexpr int kWords = kEmitBits / 32, kPer = kWords / kThreads;
  for (int w0 = 0; w0 < N; w0 += kEmitBits) {
    for (int i = t; i < kWords; i += kThreads) bm[i] = 0u;
    __syncthreads();
    for (int c = 0; c < nchg; ++c) {
      const int cnt = (int)__ldcg(P.ccnt + (int64_t)g * P.max_nch + c);
      for (int e = t; e < cnt; e += kThreads) {
        const int64_t o = (int64_t)c * C + e;
        const uint2 bw = __ldcg(gbin + o);
        const int bb = (int)(((jh < 4 ? bw.x : bw.y) >> (8 * (jh & 3))) & 0xffu);
        const int pos = (int)__ldcg(gpos + o) - w0;
        if (bb >= bst && pos >= 0 && pos < kEmitBits) atomicOr(&bm[pos >> 5], 1u << (pos & 31));
      }
    }
    __syncthreads();
    int cnt = 0;
#pragma unroll 1
    for (int q = 0; q < kPer; ++q) cnt += __popc(bm[t * kPer + q]);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int before = 0, total = 0;
    for (int w = 0; w < kThreads / 32; ++w) { before += w < warp ? wsum[w] : 0; total += wsum[w]; }
    int o = base + before + incl - cnt;
#pragma unroll 1
    for (int q = 0; q < kPer; ++q) {
      uint32_t word = bm[t * kPer + q];
      while (word) {
        const int bit = __ffs(word) - 1;
        word &= word - 1;
        dst[o++] = w0 + (t * kPer + q) * 32 + bit;
      }
    }
    base += total;
    __syncthreads();
  }
}

}  // namespace rtp
