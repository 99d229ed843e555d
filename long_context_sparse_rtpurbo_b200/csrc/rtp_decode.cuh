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
  int64_t cand_stride;   // list entries per group (>= max_seq_len)
  // shared-memory layout (byte offsets into the dynamic buffer)
  int sm_stage, sm_q, sm_qbuf, sm_qidx, sm_hist, sm_res, sm_tmp, sm_int, sm_N, sm_cbase,
      sm_tcache, sm_lcache, free_bytes;
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
  float2* grange;              // [n_groups][G]  group (min score, 256 / (max - min)), debug output
  uint32_t* sellist;           // [n_groups][cand_stride] selected rows of recomputed chunks
  float* part;                 // [NC_max][G][130]
  float* tpart;                // [NC_max][G][130]
  float* lpart;                // [n_loc_items][G][130]
  unsigned long long* trace;   // [P][kTraceEvents] %globaltimer stamps (tracing builds only)
};

// Phase-boundary timestamps, recorded only when built with -DRTP_TRACE.
// Each event keeps its last occurrence; kEvNLocWait / kEvNLocDrain count local items.
enum TraceEvent { kEvStart, kEvPlan, kEvS0, kEvS1, kEvH0, kEvHw, kEvH1, kEvW0, kEvW1, kEvW2,
                  kEvW3, kEvLoc0, kEvLoc1, kEvDrain, kEvEnd, kEvNLocWait, kEvNLocDrain,
                  kEvHs, kEvWl, kTraceEvents = 32 };

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
  __device__ float2* lcache() const { return (float2*)(rtp_smem + P.sm_lcache); }
};
// ints[]: [0..31] reduction scratch, [32] wait flag, [33] next local item, [36] last-split
//         flag, [38] local-last flag, [40..47] b*, [48..55] decode token's index row
//         (16 bf16), [60] tensor-memory base, [64..95] per-warp counts of ordered
//         compactions (two blocks of 16), [96..127] tensor-memory column of each chunk

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
        if (c > P.C_cap && steps < kMaxSteps) { ++steps; continue; }
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

  // Per-row work of phase S. Per head: min, max, and the sum of 2^(y - rf) against a
  // per-thread reference rf (the first score, moved up only when a score exceeds it by 64, so
  // the terms never overflow and the common step is one exponential and one add). When the
  // chunk's scores are kept, each stage's G scores go to G tensor-memory columns of the
  // thread's lane (a warp-wide store).
  struct SStats {
    float mn[G], mx[G], rf[G], ls[G];
    uint32_t tbase;                // tensor-memory base
    int col0;                      // first column of this chunk (-1: scores not kept)
    __device__ __forceinline__ SStats(uint32_t tb, int c) : tbase(tb), col0(c) {
#pragma unroll
      for (int k = 0; k < G; ++k) { mn[k] = INFINITY; mx[k] = -INFINITY; rf[k] = -INFINITY; ls[k] = 0.f; }
    }
    __device__ __forceinline__ void operator()(int nl, bool ok, const float (&y)[G]) {
      if (col0 >= 0) Tmem<G>::st(tmem_addr(tbase, col0 + (nl / kSRows) * G), y);   // whole warp
      if (!ok) return;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        mn[h] = fminf(mn[h], y[h]);
        mx[h] = fmaxf(mx[h], y[h]);
        const float d = y[h] - rf[h];
        if (d > 64.f) {
          ls[h] = ls[h] * exp2f(-d) + 1.f;
          rf[h] = y[h];
        } else {
          ls[h] += exp2f(d);
        }
      }
    }
  };

  // Per-row work of phase H: for each head whose score reaches ycut (half a bin below the
  // cutoff bin's edge), the bin; when it reaches the cutoff, the row's fixed-point mass goes
  // to the shared histogram (two 32-bit words per bin, exact).
  struct HHist {
    float lo[G], hi[G], inv[G], ycut[G];
    int bch[G];
    int hist_off;                  // byte offset of the histogram words in rtp_smem
    __device__ __forceinline__ void operator()(int nl, bool ok, const float (&y)[G]) {
      (void)nl;
      if (!ok) return;
      uint32_t* hlo = smem_at<uint32_t>(hist_off);
      uint32_t* hhi = hlo + G * kHistStride;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        if (y[h] >= ycut[h]) {
          const int b = inv[h] > 0.f ? bin_of(y[h], lo[h], inv[h]) : 0;
          const float ex = y[h] - hi[h];
          if (b >= bch[h] && ex > -42.f) {   // below 2^-41 the fixed-point mass rounds to 0
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
  };

  // Per-row work of phase W when the scores are recomputed: the head mask of the row (heads
  // whose bin reaches b*) and the ordered compaction of the selected rows into a list in
  // global memory.
  struct WSel {
    float lo[G], inv[G];
    int bs[G];
    int hc[G];
    uint32_t* out;                 // the chunk's list (global)
    int n0, nb, par, wc_off;
    __device__ __forceinline__ void operator()(int nl, bool ok, const float (&y)[G]) {
      uint32_t mask = 0;
      if (ok) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const int b = inv[h] > 0.f ? bin_of(y[h], lo[h], inv[h]) : 0;
          if (b >= bs[h]) { mask |= 1u << h; hc[h]++; }
        }
      }
      int before, total;
      block_flag_prefix(mask != 0, wc_off, par, before, total);
      par ^= 1;
      if (mask) out[nb + before] = ((uint32_t)(n0 + nl) << 8) | mask;
      nb += total;
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
  // tcol: first tensor-memory column of the chunk's scores, -1 when they are not kept.
  __device__ __forceinline__ void phase_score(int k, int tcol) {
    const int g = group_of(k), j = k - sm.cbase()[g];
    const int N = gN(g);
    const bool patch = P.k_new && min(N, (j + 1) * C) == N;
    SStats sst((uint32_t)sm.ints()[60], tcol);
    trace(kEvS0);
    stream_chunk(g, j, patch, sst);
    if (tcol >= 0) tmem_wait_st();
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
    arrive(P.bar + (int64_t)g * 4 + 0);
  }

  // ------------------------------------------------------------ phase H
  // Group range and total mass from the chunk statistics (double, fixed order: every CTA
  // gets the same values); the cutoff: with T the group's total mass, every token below
  // bin(c), c = hi + log2((1 - p) T' / N), T' = T (1 - 1e-3), has mass below (1 - p) T' / N,
  // so together they hold less than (1 - p) of the total, C_bin(c) > p T, and b* can not fall
  // under the cutoff bin (the 1e-3 absorbs the rounding of T, the log and the bin edges).
  // Rows whose bin reaches the cutoff add their masses (2^(y - max) in 2^-40 fixed point) to
  // the group's histogram. The range (lo, 256 / (hi - lo)) and T are kept for phase W.
  __device__ __forceinline__ void phase_hist(int k, int step, int tcol) {
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
        const float inv = (hi > lo && !P.select_all) ? (float)kBins / (hi - lo) : 0.f;
        st3[t * 3 + 0] = lo;
        st3[t * 3 + 1] = hi;
        st3[t * 3 + 2] = inv;
        sm.lcache()[step * G + t] = make_float2(lo, inv);
        if (j == 0) P.grange[(int64_t)g * G + t] = make_float2(lo, inv);
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
    HHist hh;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      hh.lo[h] = st3[h * 3 + 0];
      hh.hi[h] = st3[h * 3 + 1];
      hh.inv[h] = st3[h * 3 + 2];
      hh.bch[h] = 0;
      if (P.p < 1.0 && hh.inv[h] > 0.f) {
        const double T = sm.tcache()[step * G + h];
        const float arg = (float)((1.0 - P.p) * T * (1.0 - 1e-3) / (double)N);
        const float c = hh.hi[h] + log2f(arg);
        hh.bch[h] = c > hh.lo[h] ? bin_of(c, hh.lo[h], hh.inv[h]) : 0;
      }
      hh.ycut[h] = hh.bch[h] > 0 ? hh.lo[h] + ((float)hh.bch[h] - 0.5f) / hh.inv[h] : -INFINITY;
    }
    hh.hist_off = P.sm_hist;
    uint32_t* hlo = sm.hist();
    uint32_t* hhi = hlo + G * kHistStride;
    for (int i = threadIdx.x; i < 2 * G * kHistStride; i += kFThreads) hlo[i] = 0u;
    __syncthreads();
    if (tcol >= 0) {
      const uint32_t tb = (uint32_t)sm.ints()[60];
#pragma unroll 1
      for (int i0 = 0; i0 < len; i0 += kFThreads) {
        const int nl = i0 + threadIdx.x;
        float y[G];
        Tmem<G>::ld(tmem_addr(tb, tcol + (i0 / kSRows) * G), y);     // whole warp
        tmem_wait_ld();
        hh(nl, nl < len, y);
      }
    } else {
      stream_chunk(g, j, false, hh);
    }
    __syncthreads();
    trace(kEvH1);
    unsigned long long* gh = P.hist + (int64_t)g * G * kBins;
    for (int i = threadIdx.x; i < G * kBins; i += kFThreads) {
      const int hd = i / kBins, b = i % kBins;
      const unsigned long long v =
          ((unsigned long long)hhi[hd * kHistStride + b] << 32) | hlo[hd * kHistStride + b];
      if (v) atomicAdd(gh + i, v);
    }
    arrive(P.bar + (int64_t)g * 4 + 1);
  }

  __device__ __forceinline__ void merge(const float* parts, int n, float* dst, uint16_t* out_rows,
                                        int buf_bytes) {
    merge_partials<G>(parts, n, dst, out_rows, reinterpret_cast<float*>(sm.stage()), buf_bytes,
                      kFThreads);
  }

  // ------------------------------------------------------------ phase W
  // The chunk's own rows with bin >= b* for some head (from its kept scores, or recomputed
  // from the index rows), with the mask of those heads, in row order; their K/V rows are
  // gathered once for all G heads. Kept scores: the list is built in shared memory at the
  // end of the staging region and handed to the attention loop whenever it fills up.
  // Recomputed scores: the list is written to global memory first (the index ring and the
  // tiles share the staging region), then read back in batches. The rotated query is formed
  // before the wait. Partials merge in teams of kTeam by the last arrivals.
  __device__ __forceinline__ void phase_attend(int k, int step, int tcol) {
    const int g = group_of(k), j = k - sm.cbase()[g];
    const int b = g / P.L.n_ret, r = g % P.L.n_ret, kvh = P.L.ret_kv[r];
    const int N = gN(g), n0 = j * C, len = min(N, n0 + C) - n0;
    const int S = nch(g);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    rope_query<G>(P, b, kvh, N, sm.q());
    if (!wait_for(P.bar + (int64_t)g * 4 + 1, (uint32_t)S)) { abort_ = true; return; }
    trace(kEvW0);
    // b* per head (warp h: head h): the highest bin whose mass from the top reaches p T
    if (warp < G) {
      int best = 0;
      if (!P.select_all) {
        const unsigned long long* gh = P.hist + ((int64_t)g * G + warp) * kBins + lane * 8;
        unsigned long long hv[8], lt = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) { hv[e] = __ldcg(gh + e); lt += hv[e]; }
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
    WSel ws;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      ws.bs[h] = sm.ints()[40 + h];
      const float2 li = sm.lcache()[step * G + h];
      ws.lo[h] = li.x;
      ws.inv[h] = li.y;
      ws.hc[h] = 0;
    }
    if (j == 0 && threadIdx.x < G) P.bstar[(int64_t)g * G + threadIdx.x] = ws.bs[threadIdx.x];
    ws.n0 = n0;
    ws.nb = 0;
    ws.par = 0;
    ws.wc_off = P.sm_int + 64 * 4;
    const int64_t rowbase = (int64_t)r * P.L.T_total + P.cache.seq_off[b];
    const uint16_t* kb = P.cache.k_ret + rowbase * kD;
    const uint16_t* vb = P.cache.v_ret + rowbase * kD;
    uint32_t* list = reinterpret_cast<uint32_t*>(sm.stage() + P.free_bytes - kListCap * 4);
    const int nwa = min(kFThreads / 32, (P.free_bytes - kListCap * 4) / kTileBytes);
    const ListRows rows{list, kb, vb};
    WarpAttn W;
    if (tcol >= 0) {
      attn_begin<G>(W, sm.qbuf(), sm.q(), kFThreads);
      trace(kEvW1);
      const uint32_t tb = (uint32_t)sm.ints()[60];
#pragma unroll 1
      for (int i0 = 0; i0 < len; i0 += kFThreads) {
        if (ws.nb > kListCap - kFThreads) {   // the list is full: attend to it first
          __syncthreads();
          attn_tiles<G>(W, ws.nb, rows, sm.stage(), nwa, false);
          __syncthreads();
          ws.nb = 0;
        }
        const int nl = i0 + threadIdx.x;
        float y[G];
        Tmem<G>::ld(tmem_addr(tb, tcol + (i0 / kSRows) * G), y);     // whole warp
        tmem_wait_ld();
        uint32_t mask = 0;
        if (nl < len) {
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const int bb = ws.inv[h] > 0.f ? bin_of(y[h], ws.lo[h], ws.inv[h]) : 0;
            if (bb >= ws.bs[h]) { mask |= 1u << h; ws.hc[h]++; }
          }
        }
        int before, total;
        block_flag_prefix(mask != 0, ws.wc_off, ws.par, before, total);
        ws.par ^= 1;
        if (mask) list[ws.nb + before] = ((uint32_t)(n0 + nl) << 8) | mask;
        ws.nb += total;
      }
      __syncthreads();
      trace(kEvWl);
      attn_tiles<G>(W, ws.nb, rows, sm.stage(), nwa, false);
    } else {
      uint32_t* gl = P.sellist + (int64_t)g * P.cand_stride + n0;
      ws.out = gl;
      stream_chunk(g, j, false, ws);
      __syncthreads();
      attn_begin<G>(W, sm.qbuf(), sm.q(), kFThreads);
      trace(kEvWl);
      const int total = ws.nb;
#pragma unroll 1
      for (int b0 = 0; b0 < total; b0 += kListCap) {
        const int nb = min(kListCap, total - b0);
        __syncthreads();
        for (int i = threadIdx.x; i < nb; i += kFThreads) list[i] = __ldcg(gl + b0 + i);
        __syncthreads();
        attn_tiles<G>(W, nb, rows, sm.stage(), nwa, false);
      }
    }
    attn_end<G>(W, nwa, sm.res(), reinterpret_cast<float*>(sm.stage()), kFThreads);
    trace(kEvW2);
    // per-head counts of this chunk
    int* red = reinterpret_cast<int*>(sm.tmp());              // [16][G]
#pragma unroll
    for (int h = 0; h < G; ++h) {
      int v = ws.hc[h];
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
    // partial -> workspace; team / group merge by the last arrivals
    const int stride = G * (kD + 2);
    float* mine = P.part + (int64_t)k * stride;
    for (int o = threadIdx.x; o < stride; o += kFThreads) mine[o] = sm.res()[o];
    const int team = j / kTeam, nteams = (S + kTeam - 1) / kTeam;
    const int tcount = min(kTeam, S - team * kTeam);
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      sm.ints()[36] = atomicAdd(P.team_arr + sm.cbase()[g] + team, 1u) == (uint32_t)(tcount - 1);
    }
    __syncthreads();
    if (!sm.ints()[36]) return;
    __threadfence();
    uint16_t* orow = P.out + ((int64_t)b * P.L.Hq + kvh * G) * kD;
    const float* tparts = P.part + (int64_t)(sm.cbase()[g] + team * kTeam) * stride;
    if (nteams == 1) {
      merge(tparts, tcount, nullptr, orow, P.free_bytes);
    } else {
      merge(tparts, tcount, P.tpart + (int64_t)(sm.cbase()[g] + team) * stride, nullptr, P.free_bytes);
      __syncthreads();
      if (threadIdx.x == 0) {
        __threadfence();
        sm.ints()[37] = atomicAdd(P.bar + (int64_t)g * 4 + 2, 1u) == (uint32_t)(nteams - 1);
      }
      __syncthreads();
      if (!sm.ints()[37]) return;
      __threadfence();
      merge(P.tpart + (int64_t)sm.cbase()[g] * stride, nteams, nullptr, orow, P.free_bytes);
    }
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
  // overlaps that scoring. The scores of the first chunks are kept in tensor memory as long
  // as its columns last (kTmemColsPerThread / G stages of kSRows rows per thread); phases H
  // and W of later chunks recompute them from the index rows. Then phase W of every chunk,
  // then local items until the queue is empty. CTAs [P_ret, P) only run local items.
  __device__ void run() {
    trace(kEvStart);
    plan();
    trace(kEvPlan);
    const int i = blockIdx.x;
    const int m = (i < P_ret && i < NC) ? (NC - i + P_ret - 1) / P_ret : 0;
    int* tcols = sm.ints() + 96;                              // [kMaxSteps]
    if (threadIdx.x == 0) {
      int col = 0;
      for (int t = 0; t < m; ++t) {
        const int k = i + t * P_ret, g = group_of(k), j = k - sm.cbase()[g];
        const int len = min(gN(g), (j + 1) * C) - j * C;
        const int need = (len + kSRows - 1) / kSRows * G;
        if (col + need <= kTmemColsPerThread) { tcols[t] = col; col += need; } else { tcols[t] = -1; }
      }
    }
    __syncthreads();
    int pstart = 0;
    for (int t = 0; t < m; ++t) {
      const int k = i + t * P_ret;
      phase_score(k, tcols[t]);
      if (pstart < t && group_of(i + pstart * P_ret) != group_of(k)) {
        for (int s = pstart; s < t; ++s) {
          phase_hist(i + s * P_ret, s, tcols[s]);
          if (abort_) return;
        }
        pstart = t;
      }
    }
    for (int s = pstart; s < m; ++s) {
      phase_hist(i + s * P_ret, s, tcols[s]);
      if (abort_) return;
    }
    for (int t = 0; t < m; ++t) {
      phase_attend(i + t * P_ret, t, tcols[t]);
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
// Debug output: ascending positions each query head attended to. One CTA of kFThreads threads
// per (b, h): a retrieval head's scores are recomputed with the decode kernel's own routines
// (the same index query, the same per-row arithmetic, so the same bits), binned with the
// group's range and compared with its b*; the selected positions are compacted in order.
template <int G>
__global__ void __launch_bounds__(kFThreads) emit_sel_kernel(DecodeParams P, int32_t* sel_idx,
                                                             int64_t sel_stride) {
  __shared__ float qidx[G * kR];
  __shared__ float tmp[kFThreads];
  __shared__ int wc[32];
  const int b = blockIdx.x / P.L.Hq, h = blockIdx.x % P.L.Hq;
  const int kvh = h / G, jh = h % G;
  const int N = seq_len_checked(P, b);
  int32_t* dst = sel_idx + ((int64_t)b * P.L.Hq + h) * sel_stride;
  if (N == 0) return;
  const int slot = P.L.slot[kvh];
  const int t = threadIdx.x;
  if (slot < 0) {
    const int s1 = min(N, P.L.sinks);
    const int w0 = max(P.L.sinks, N - P.L.window);
    const int cnt = s1 + max(0, N - w0);
    for (int k = t; k < cnt; k += kFThreads) dst[k] = k < s1 ? k : w0 + (k - s1);
    return;
  }
  const int g = b * P.L.n_ret + slot;
  const int bst = __ldcg(P.bstar + (int64_t)g * G + jh);
  const float2 li = __ldcg(P.grange + (int64_t)g * G + jh);
  index_query<G>(P, b, kvh, qidx, tmp);
  float2 qi[G][kR / 2];
#pragma unroll
  for (int hh = 0; hh < G; ++hh)
#pragma unroll
    for (int jj = 0; jj < kR / 2; ++jj)
      qi[hh][jj] = make_float2(qidx[hh * kR + 2 * jj], qidx[hh * kR + 2 * jj + 1]);
  const unsigned char* src = (const unsigned char*)(
      P.cache.idx + ((int64_t)slot * P.L.T_total + P.cache.seq_off[b]) * kR);
  int base = 0, par = 0;
#pragma unroll 1
  for (int i0 = 0; i0 < N; i0 += kFThreads) {
    const int n = i0 + t;
    bool keep = false;
    if (n < N) {
      float y[G];
      score_row<G>(qi, src + (int64_t)n * 32, y);
      const int bb = li.y > 0.f ? bin_of(y[jh], li.x, li.y) : 0;
      keep = bb >= bst;
    }
    int before, total;
    block_flag_prefix_impl(keep, wc + par * 16, before, total);
    par ^= 1;
    if (keep) dst[base + before] = n;
    base += total;
  }
}

}  // namespace rtp
