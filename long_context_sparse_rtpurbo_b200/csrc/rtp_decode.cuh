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
//   S  the chunk's index rows are streamed once from HBM, each warp through its own slots of
//      a ring (no block barrier per stage), and scored on the tensor cores, 32 rows per warp
//      tile, in log2 units (the index query carries log2(e)); per-chunk (min, max,
//      sum 2^(y - max)) per head. The scores stay in tensor memory as long as its columns
//      last; later chunks of the CTA recompute them from the index rows when needed.
//   H  from the group's (min, max, total mass): the 256 linear bins and a cutoff bin under
//      which no token can be selected (their total mass is below (1 - p) of the total). A
//      score reaches a bin exactly when it reaches the bin's lower edge, found once per head
//      by bisection over the floats, so the test per score is one compare; the scores at or
//      above the cutoff are compacted per warp and added (fixed-point masses) to the group's
//      histogram (exact integer sums). Phase H of a group runs after phase S of the CTA's
//      next group, which hides the wait for the other chunks.
//   W  b* per head from the group's histogram; each chunk selects its rows with a score at
//      or above the edge of b* for some head (per-warp compaction, batches of 8 stages),
//      gathers their K/V rows once for all G heads (tensor-core tiles, a head that did not
//      select a row masks it) and writes a partial softmax state; the last chunk to finish
//      merges all partials of the group into the output rows and the selected counts.
// Local items (a slice of one local head's ring) come from a global queue; the chunk CTAs
// drain it when their chunks are done.
// Every wait is bounded (clock64 limit): on expiry the kernel records RTP_ETIMEOUT, raises
// an abort flag that ends every other wait, and returns.
#pragma once

#include "rtp_append.cuh"
#include "rtp_attend.cuh"
#include "rtp_score.cuh"
#include "rtp_tmem.cuh"

namespace rtp {

constexpr int kFThreads = 512;          // threads of the decode kernel
constexpr int kWarps = kFThreads / 32;
constexpr int kHeadPad = 8;             // words between the heads' rows of shared buffers
constexpr int kHistStride = 256 + kHeadPad;
constexpr int kMaxSteps = 32;           // chunks per CTA, upper bound
constexpr int kSRows = kWarps * kWRows; // index rows per stage (one 32-row tile per warp)
constexpr int kSStages = 8;             // ring depth (stages in flight: kSStages - 1)
constexpr int kSlotBytes = kWRows * 32; // one warp's slot of a stage
constexpr int kStageBytes = kSRows * 32;
constexpr int kWBatch = 16;             // stages per selection batch of phase W
constexpr int kHistPad = 4;             // u64 words per bin of the global histogram: one
                                        // 32-byte sector per bin spreads the CTAs' atomic
                                        // adds over more L2 lines
constexpr int kWListCap = kWBatch * kWRows;           // list entries per warp and batch
constexpr int kHQueueMax = 32 * 9;      // per-warp candidate queue of phase H (entries)
constexpr int kIntsWords = 256;         // words of the shared ints[] array
// tail of the staging region (bytes back from its end): phase W's lists and row-mask bytes,
// phase H's candidate queues (different phases, so they may overlap)
constexpr int kTailList = kWarps * kWListCap * 4;
constexpr int kTailRm = kTailList + kWarps * kWRows * 8;
constexpr int kTailHq = kWarps * kHQueueMax * 8;
constexpr int kTailMax = kTailHq > kTailRm ? kTailHq : kTailRm;

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
  int select_all;    // p >= 1 (top-p mode)
  double p;
  long long topk;    // > 0: fixed-budget top-k (count threshold) instead of top-p
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
  uint32_t* bar;               // [n_groups][4]  S arrivals, H arrivals, W arrivals     (zeroed)
  uint32_t* loc_arr;           // [n_lgroups]    local item arrivals                (zeroed)
  uint32_t* misc;              // [0] local queue head, [1] abort, [2] chunk size     (zeroed)
  unsigned long long* hist;    // [n_groups][G][256][kHistPad] fixed-point bin masses (word 0;
                               //   zeroed by the group's first chunk in phase S)
  int32_t* hcnt;               // [n_groups][G]  selected tokens per head (zeroed likewise)
  int32_t* bstar;              // [n_groups][G]  threshold bins (debug output)
  float4* cstat;               // [n_groups][max_nch][G]  chunk (min, max, sum 2^(y - max))
  float2* grange;              // [n_groups][G]  group (min score, 256 / (max - min)), debug output
  uint32_t* sellist;           // [n_groups][cand_stride] selected rows of recomputed chunks
  unsigned char* part;         // [NC_max] partials (Part<G>::kBytes each)
  unsigned char* lpart;        // [n_loc_items] partials
  unsigned long long* trace;   // [P][kTraceEvents] %globaltimer stamps (tracing builds only)
};

// Phase-boundary timestamps, recorded only when built with -DRTP_TRACE.
// Each event keeps its last occurrence; kEvNLocWait / kEvNLocDrain count local items.
enum TraceEvent { kEvStart, kEvPlan, kEvS0, kEvS1, kEvH0, kEvHw, kEvH1, kEvW0, kEvW1, kEvW2,
                  kEvW3, kEvLoc0, kEvLoc1, kEvDrain, kEvEnd, kEvNLocWait, kEvNLocDrain,
                  kEvHs, kEvWl, kEvWb, kEvWh, kTraceEvents = 32 };

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
  __device__ float4* lcache() const { return (float4*)(rtp_smem + P.sm_lcache); }
};
// ints[]: [0..31] reduction scratch, [32] wait flag, [33] next local item, [36] last-split
//         flag, [38] local-last flag, [40..47] b*, [48..55] decode token's index row
//         (16 bf16), [60] tensor-memory base, [96..127] tensor-memory column of each chunk,
//         [128..144] prefix of the per-warp list counts, [160..167] selected rows per head,
//         [176..183] (float) per-head score edge of the cutoff / threshold bin,
//         [192..223] (float4) per-head lo, 256 / (hi - lo), hi
constexpr int kIntPre = 128, kIntCnt = 160, kIntEdge = 176, kIntHp = 192;

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
// items. w: one of two arrays of 16 ints used alternately, so one barrier per block suffices.
__device__ __forceinline__ void block_flag_prefix(bool flag, int* w, int& before, int& total) {
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

__device__ __forceinline__ int bin_of(float s, float lo, float inv) {
  return min(kBins - 1, (int)((s - lo) * inv));
}

// Lower edge of bin b as a score: the smallest float y in [lo, hi] with bin_of(y) >= b
// (-inf for b <= 0). bin_of is non-decreasing in y (a rounded subtraction, a rounded product
// with inv > 0, truncation), so for every score y in [lo, hi]: bin_of(y) >= b <=> y >= edge.
// Warp-collective search over the order-preserving integer images of the floats in
// (lo, hi]: the lanes test 32 candidates per round, first the 32 floats around the rounded
// guess lo + b / inv, then 32-way splits of the remaining interval (a, z] with
// bin_of(a) < b <= bin_of(z), until it holds one float. Every lane returns the edge.
__device__ __forceinline__ float bin_edge_warp(int b, float lo, float hi, float inv) {
  if (b <= 0) return -INFINITY;
  if (!(inv > 0.f) || bin_of(hi, lo, inv) < b) return INFINITY;
  const int lane = threadIdx.x & 31;
  uint32_t a = f2ord(lo), z = f2ord(hi);                      // bin_of(lo) = 0 < b
  const uint32_t g = f2ord(fminf(fmaxf(lo + (float)b / inv, lo), hi));
  uint32_t base = g > a + 16u ? g - 16u : a + 1u, step = 1u;
#pragma unroll 1
  for (int round = 0; round < 16 && z - a > 1u; ++round) {
    const uint64_t c64 = (uint64_t)base + (uint64_t)step * (uint32_t)lane;
    const uint32_t c = c64 >= (uint64_t)z ? z : (c64 <= (uint64_t)a ? a + 1u : (uint32_t)c64);
    const bool up = bin_of(ord2f(c), lo, inv) >= b;
    const uint32_t bal = __ballot_sync(0xffffffffu, up);   // a suffix of the lanes
    if (bal) z = min(z, __shfl_sync(0xffffffffu, c, __ffs(bal) - 1));
    if (~bal) a = max(a, __shfl_sync(0xffffffffu, c, 31 - __clz(~bal)));
    step = max(1u, (z - a) / 32u);
    base = a + step;
  }
  return ord2f(z);
}

__device__ __forceinline__ float ex2_approx(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
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
    // follows the bytes of each side (index read twice as a proxy for index and gather), but
    // the chunk CTAs are at least as many as hold the retrieval rows at one tensor-memory
    // capacity each: a CTA's chunks run their phases one after another (and wait on the other
    // CTAs' chunks of the same groups), while local items are taken from a queue by whichever
    // CTA is free, so the retrieval chain is the one to keep short
    C = 1024;
    P_ret = 0;
    if (Tr > 0) {
      const double ret_b = 64.0 * (double)Tr, loc_b = 512.0 * (double)loc_rows;
      const int pr = (int)((double)P.P * ret_b / (ret_b + loc_b) + 0.5);
      const long long pcap = (Tr + P.C_cap - 1) / P.C_cap;
      P_ret = max(1, min(P.P, max(pr, (int)min(pcap, (long long)P.P))));
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

  // ------------------------------------------------------------ chunks and streaming
  // Chunk j of a group with nc chunks is the set of its 32-row tiles j, j + nc, j + 2 nc, ...
  // (of the group's ceil(N / 32) tiles): interleaved, so a run of selected tokens is spread
  // over many chunks (and CTAs). In local stage st, warp w takes the chunk's tile 16 st + w.
  __device__ __forceinline__ static int chunk_tiles(int N, int nc, int j) {
    return ((N + kWRows - 1) / kWRows - j + nc - 1) / nc;
  }
  __device__ __forceinline__ static int chunk_stages(int N, int nc, int j) {
    return (chunk_tiles(N, nc, j) + kWarps - 1) / kWarps;
  }
  // first group row of the tile of warp w in local stage st (N when the warp has none)
  __device__ __forceinline__ static int tile_row(int N, int nc, int j, int ntl, int st, int w) {
    const int i = st * kWarps + w;
    return i < ntl ? (j + i * nc) * kWRows : N;
  }

  // The chunk's index rows stream through a ring of kSStages stages; warp w copies its tile
  // of each stage itself into its 1 KB slot (cp.async, two 16-byte pieces per lane, the
  // halves of rows 4..7 mod 8 swapped; rows past the group end are zeroed) and scores it on
  // the tensor cores, so a stage needs no block barrier. fn(st, rb, c, T) gets the warp's tile
  // scores (rb: group row of the tile's row 0, N when the warp has no tile this stage; rows
  // at or past N score 0 and are masked by the callers).
  __device__ __forceinline__ void slot_issue(uint32_t ring, const unsigned char* src, int st,
                                             int nst, int N, int nc, int j, int ntl, bool last) {
    if (st < nst) {
      const int lane = threadIdx.x & 31;
      const int rb = tile_row(N, nc, j, ntl, st, threadIdx.x >> 5);
      const uint32_t slot = ring + (st % kSStages) * kStageBytes;
      const uint64_t pol = l2_evict_first();
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int p = lane + 32 * u, r = p >> 1, hh = p & 1;
        if (rb + r < N) {
          const unsigned char* g = src + (int64_t)(rb + r) * 32 + hh * 16;
          if (last) cp_async16_s_ef(slot + idx_half_off(r, hh), g, pol);
          else      cp_async16_s(slot + idx_half_off(r, hh), g);
        }
        else {    // zero rows: a stale inf or NaN times a zero query column would poison the
                  // other half-tile's scores
          st_shared_zero16(slot + idx_half_off(r, hh));
        }
      }
    }
    cp_async_commit();
  }
  // last: this is the launch's last read of these rows (L2 evict-first); chunks whose scores
  // are recomputed later keep the default policy on their earlier reads
  template <class Fn>
  __device__ __forceinline__ void stream_chunk(int g, int j, bool patch, bool last, Fn& fn) {
    const int b = g / P.L.n_ret, r = g % P.L.n_ret, kvh = P.L.ret_kv[r];
    const int N = gN(g), nc = nch(g);
    const int ntl = chunk_tiles(N, nc, j), nst = chunk_stages(N, nc, j);
    const unsigned char* src = (const unsigned char*)(
        P.cache.idx + ((int64_t)r * P.L.T_total + P.cache.seq_off[b]) * kR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t ring = smem_u32(sm.stage()) + warp * kSlotBytes;
    __syncthreads();                       // the staging region may still be in use
#pragma unroll
    for (int st = 0; st < kSStages - 1; ++st) slot_issue(ring, src, st, nst, N, nc, j, ntl, last);
    index_query<G>(P, b, kvh, sm.qidx(), reinterpret_cast<float*>(sm.tmp()));
    // The chunk holding the decode token writes it while the first stages are in flight; a
    // copy of its index row may be stale, so the warp holding it patches its slot.
    uint16_t* idx_patch = reinterpret_cast<uint16_t*>(sm.ints() + 48);   // 16 bf16
    if (patch) {
      append_new(b, kvh, N, idx_patch);
      __syncthreads();
    }
    ScoreTile<G> T;
    T.init(sm.qidx());
    const int prow = patch ? N - 1 : -1;
#pragma unroll 1
    for (int st = 0; st < nst; ++st) {
      slot_issue(ring, src, st + kSStages - 1, nst, N, nc, j, ntl, last);
      cp_async_wait<kSStages - 1>();
      __syncwarp();
      const uint32_t slot = ring + (st % kSStages) * kStageBytes;
      const int rb = tile_row(N, nc, j, ntl, st, warp);
      if (prow >= rb && prow < rb + kWRows) {
        const int rr = prow - rb;
        if (lane < 8)
          st_shared_u32(slot + idx_half_off(rr, lane >> 2) + (lane & 3) * 4,
                        reinterpret_cast<const uint32_t*>(idx_patch)[lane]);
        __syncwarp();
      }
      float c[ScoreTile<G>::V];
      T.score(slot, c);
      fn(st, rb, c, T);
      __syncwarp();                        // the slot is refilled by the next issue
    }
    cp_async_wait<0>();
  }

  static constexpr int V = ScoreTile<G>::V;

  // Per-tile work of phase S: the scores go to V tensor-memory columns of the lane (when the
  // chunk's scores are kept); per slot (one head per slot): min, max, and the sum of
  // 2^(y - rf) against a per-lane reference rf (the first score, moved up only when a score
  // exceeds it by 64, so the terms never overflow).
  struct SStats {
    float mn[2], mx[2], rf[2], ls[2];
    uint32_t taddr;                // tensor-memory address of the chunk's first column
    bool keep;
    int N;                         // group rows (rows at or past N are not the group's)
    __device__ __forceinline__ SStats(uint32_t ta, bool k, int n) : taddr(ta), keep(k), N(n) {
#pragma unroll
      for (int e = 0; e < 2; ++e) { mn[e] = INFINITY; mx[e] = -INFINITY; rf[e] = -INFINITY; ls[e] = 0.f; }
    }
    // (min, max, rf, ls) of slot e combined with another state
    __device__ __forceinline__ void combine(int e, float mn2, float mx2, float r2, float l2) {
      mn[e] = fminf(mn[e], mn2);
      mx[e] = fmaxf(mx[e], mx2);
      const float rr = fmaxf(rf[e], r2);
      ls[e] = (rr == -INFINITY) ? 0.f : ls[e] * exp2f(rf[e] - rr) + l2 * exp2f(r2 - rr);
      rf[e] = rr;
    }
    __device__ __forceinline__ void merge_slots() { combine(0, mn[1], mx[1], rf[1], ls[1]); }
    __device__ __forceinline__ void merge_lanes(int o) {
#pragma unroll
      for (int e = 0; e < 2; ++e)
        combine(e, __shfl_xor_sync(0xffffffffu, mn[e], o), __shfl_xor_sync(0xffffffffu, mx[e], o),
                __shfl_xor_sync(0xffffffffu, rf[e], o), __shfl_xor_sync(0xffffffffu, ls[e], o));
    }
    __device__ __forceinline__ void operator()(int st, int rb, const float (&c)[V],
                                               const ScoreTile<G>& T) {
      if (keep) {                          // warp-collective: converged first
        __syncwarp();
        Tmem<V>::st(taddr + st * V, c);
      }
#pragma unroll
      for (int v = 0; v < V; ++v) {
        const int e = v & 1;
        if (T.ok[e] && rb + T.row[v] < N) {
          const float y = c[v];
          mn[e] = fminf(mn[e], y);
          mx[e] = fmaxf(mx[e], y);
          const float d = y - rf[e];
          if (d > 64.f) {
            ls[e] = ls[e] * ex2_approx(-d) + 1.f;
            rf[e] = y;
          } else {
            ls[e] += ex2_approx(d);
          }
        }
      }
    }
  };

  // Per-tile work of phase H: scores at or above their head's cutoff edge are compacted into
  // the warp's queue (score, head); every 32 queued entries are binned and their fixed-point
  // masses added to the shared histogram (two 32-bit words per bin, exact).
  struct HComp {
    float thr[2];                  // per slot: cutoff edge (+inf for a padding column)
    int hd[2];
    int N, qn, qoff, hp_off, hist_off;
    bool count_only;               // top-k: each score adds 1 (counts, not masses)
    __device__ __forceinline__ void add(float y, int h) const {
      const float4 p = smem_at<float4>(hp_off)[h];           // lo, inv, hi
      const int b = p.y > 0.f ? bin_of(y, p.x, p.y) : 0;
      const float ex = y - p.z;
      if (count_only || ex > -42.f) {       // below 2^-41 the fixed-point mass rounds to 0
        const unsigned long long q =
            count_only ? 1ull : __float2ull_rn(exp2f(ex) * kMassScale);
        uint32_t* hlo = smem_at<uint32_t>(hist_off);
        uint32_t* hhi = hlo + G * kHistStride;
        const int bi = h * kHistStride + b;
        const uint32_t ql = (uint32_t)q, qh = (uint32_t)(q >> 32);
        const uint32_t old = atomicAdd(&hlo[bi], ql);
        const uint32_t up = qh + ((old + ql < old) ? 1u : 0u);
        if (up) atomicAdd(&hhi[bi], up);
      }
    }
    __device__ __forceinline__ void operator()(int st, int rb, const float (&c)[V],
                                               const ScoreTile<G>& T) {
      (void)st;
      const int lane = threadIdx.x & 31;
      const uint32_t lt = (1u << lane) - 1u;
      float2* q = smem_at<float2>(qoff);
#pragma unroll
      for (int v = 0; v < V; ++v) {
        const int e = v & 1;
        const bool cand = rb + T.row[v] < N && c[v] >= thr[e];
        const uint32_t bal = __ballot_sync(0xffffffffu, cand);
        if (cand) q[qn + __popc(bal & lt)] = make_float2(c[v], __int_as_float(hd[e]));
        qn += __popc(bal);
      }
      __syncwarp();
      while (qn >= 32) {
        qn -= 32;
        const float2 x = q[qn + lane];
        add(x.x, __float_as_int(x.y));
        __syncwarp();                       // the entries are overwritten by the next tile
      }
    }
    __device__ __forceinline__ void finish() {
      const int lane = threadIdx.x & 31;
      if (lane < qn) {
        const float2 x = smem_at<float2>(qoff)[lane];
        add(x.x, __float_as_int(x.y));
      }
      qn = 0;
    }
  };

  // Selection of one tile in phase W: each (lane, value) writes its (row, head) byte, then
  // lane r forms row r's head mask. hc: selected scores per slot.
  __device__ __forceinline__ static uint32_t tile_select(const float (&c)[V], int rb, int N,
                                                         const float (&ts)[2],
                                                         const ScoreTile<G>& T, int rm_off,
                                                         int (&hc)[2]) {
    unsigned char* rm = smem_at<unsigned char>(rm_off);
#pragma unroll
    for (int v = 0; v < V; ++v) {
      const int e = v & 1;
      if (T.ok[e]) {
        const bool s = rb + T.row[v] < N && c[v] >= ts[e];
        hc[e] += s;
        rm[T.row[v] * 8 + T.head[e]] = s;
      }
    }
    __syncwarp();
    const uint2 x = smem_at<uint2>(rm_off)[threadIdx.x & 31];
    uint32_t mask = 0;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const uint32_t w = h < 4 ? x.x : x.y;
      mask |= ((w >> ((h & 3) * 8)) & 1u) << h;
    }
    __syncwarp();                           // the bytes are rewritten by the next tile
    return mask;
  }

  // Per-tile work of phase W when the scores are recomputed: the selected rows of the warp
  // go, in row order, to the group's list in global memory: the warp's q-th entry to the
  // slot of the q-th row of its own tiles (row 32 * tile(q / 32) + q % 32), so the chunks'
  // and warps' regions never overlap.
  struct WSel {
    float ts[2];
    int hc[2];
    int N, nc, j, ntl, rm_off, nw;
    uint32_t* gl;                  // the group's list (global)
    __device__ __forceinline__ void operator()(int st, int rb, const float (&c)[V],
                                               const ScoreTile<G>& T) {
      (void)st;
      const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
      const uint32_t mask = tile_select(c, rb, N, ts, T, rm_off, hc);
      const uint32_t bal = __ballot_sync(0xffffffffu, mask != 0);
      if (mask) {
        const int q = nw + __popc(bal & ((1u << lane) - 1u));
        gl[tile_row(N, nc, j, ntl, q / kWRows, warp) + q % kWRows] = ((uint32_t)(rb + lane) << 8) | mask;
      }
      nw += __popc(bal);
    }
  };

  // Rows of the attention loop: the concatenation of the warps' lists (entry i of the
  // concatenation is entry q = i - pre[w] of the warp w with pre[w] <= i < pre[w + 1]; it
  // sits at w * stride + q of `list`, or, in the group's global list of a recomputed chunk,
  // at the slot WSel gave it), or a contiguous range of ring rows.
  struct WarpListRows {
    const uint32_t* list;
    const uint16_t* kb;
    const uint16_t* vb;
    int pre_off;                   // byte offset of pre[17] in rtp_smem
    int stride;                    // > 0: fixed per-warp stride; 0: WSel slots
    int N, nc, j, ntl;
    int64_t cap;                   // entries the list holds
    int* status;
    __device__ __forceinline__ void operator()(int i, const uint16_t*& kp, const uint16_t*& vp,
                                               uint32_t& mk) const {
      const int* pre = smem_at<int>(pre_off);
      const int w = upper_index(pre, kWarps, i);
      const int q = i - pre[w];
      const int at = stride > 0 ? w * stride + q : tile_row(N, nc, j, ntl, q / kWRows, w) + q % kWRows;
      if (!RTP_CHECK(at >= 0 && at < cap, status)) { kp = kb; vp = vb; mk = 0u; return; }
      const uint32_t e = list[at];
      if (!RTP_CHECK((int)(e >> 8) < N, status)) { kp = kb; vp = vb; mk = 0u; return; }
      kp = kb + (int64_t)(e >> 8) * kD;
      vp = vb + (int64_t)(e >> 8) * kD;
      mk = e & 0xffu;
    }
  };
  struct RangeRows {
    const uint16_t* kb;
    const uint16_t* vb;
    int n;                         // rows in range
    int* status;
    __device__ __forceinline__ void operator()(int i, const uint16_t*& kp, const uint16_t*& vp,
                                               uint32_t& mk) const {
      if (!RTP_CHECK(i >= 0 && i < n, status)) { kp = kb; vp = vb; mk = 0u; return; }
      kp = kb + (int64_t)i * kD;
      vp = vb + (int64_t)i * kD;
      mk = 0xffu;
    }
  };

  __device__ __forceinline__ int tail(int bytes_back) const { return P.sm_stage + P.free_bytes - bytes_back; }
  __device__ __forceinline__ uint32_t chunk_taddr(int tcol) const {
    return tmem_addr((uint32_t)sm.ints()[60], tcol);
  }

  // Per-warp list counts -> prefix pre[0..16] in ints[kIntPre...] (block-wide; ends with a
  // barrier). Returns the total.
  __device__ __forceinline__ int list_prefix(int nw) {
    int* pre = sm.ints() + kIntPre;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncthreads();
    if (lane == 0) pre[1 + warp] = nw;
    __syncthreads();
    if (threadIdx.x == 0) {
      pre[0] = 0;
      for (int w = 0; w < kWarps; ++w) pre[1 + w] += pre[w];
    }
    __syncthreads();
    return pre[kWarps];
  }

  // ------------------------------------------------------------ phase S
  // tcol: first tensor-memory column of the chunk's scores, -1 when they are not kept.
  __device__ __forceinline__ void phase_score(int k, int tcol) {
    const int g = group_of(k), j = k - sm.cbase()[g];
    const int N = gN(g);
    const bool patch = P.k_new && ((N - 1) / kWRows) % nch(g) == j;   // holds row N - 1
    SStats sst(tcol >= 0 ? chunk_taddr(tcol) : 0u, tcol >= 0, N);
    trace(kEvS0);
    stream_chunk(g, j, patch, tcol >= 0, sst);
    if (tcol >= 0) {
      __syncwarp();
      tmem_wait_st();
    }
    trace(kEvS1);
    // chunk statistics per head: lanes of one tig hold the same heads (reduce over gid),
    // then a fixed-order pass over (warp, tig, slot)
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) sst.merge_lanes(o);
    // complete the warp's stats of each head in one lane: G = 1: both slots of tig 0;
    // G = 2: tig 0 and 1; G = 4: tig t and t + 2 (G = 8: every (tig, slot) is one head)
    {
      const int tig = lane & 3;
      if (G < 8) {
#pragma unroll
        for (int e = 0; e < 2; ++e)
          if (2 * tig + e >= 2 * G) { sst.mn[e] = INFINITY; sst.mx[e] = -INFINITY; sst.rf[e] = -INFINITY; sst.ls[e] = 0.f; }
      }
      if (G == 1) sst.merge_slots();
      if (G == 2) sst.merge_lanes(1);
      if (G == 4) sst.merge_lanes(2);
    }
    float4* red = reinterpret_cast<float4*>(sm.tmp());       // [16 warps][8 heads]
    if (lane < 4) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int n = 2 * lane + e;
        const bool own = G == 8 ? true : (G == 4 ? n < 4 : (G == 2 ? n < 2 : n == 0));
        if (own) red[warp * 8 + n] = make_float4(sst.mn[e], sst.mx[e], sst.rf[e], sst.ls[e]);
      }
    }
    __syncthreads();
    if (warp < G) {                        // warp h: lanes over the warps, fixed shuffle tree
      const float4 x = lane < kWarps ? red[lane * 8 + warp] : make_float4(INFINITY, -INFINITY, -INFINITY, 0.f);
      float a = x.x, z = x.y;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        a = fminf(a, __shfl_xor_sync(0xffffffffu, a, o));
        z = fmaxf(z, __shfl_xor_sync(0xffffffffu, z, o));
      }
      double l = x.z != -INFINITY ? (double)x.w * (double)exp2f(x.z - z) : 0.0;   // rf <= max
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
      if (lane == 0) P.cstat[((int64_t)g * P.max_nch + j) * G + warp] = make_float4(a, z, (float)l, 0.f);
    }
    if (j == 0) {   // the group's histogram and counts, before any chunk of it reaches phase H
      unsigned long long* gh = P.hist + (int64_t)g * G * kBins * kHistPad;
      for (int i = threadIdx.x; i < G * kBins * kHistPad; i += kFThreads) gh[i] = 0ull;
      if (threadIdx.x < G) P.hcnt[(int64_t)g * G + threadIdx.x] = 0;
    }
    arrive(P.bar + (int64_t)g * 4 + 0);
  }

  // ------------------------------------------------------------ phase H
  // Group range and total mass from the chunk statistics (double, fixed order: every CTA
  // gets the same values); the cutoff: with T the group's total mass, every token below
  // bin(c), c = hi + log2((1 - p) T' / N), T' = T (1 - 1e-3), has mass below (1 - p) T' / N,
  // so together they hold less than (1 - p) of the total, C_bin(c) > p T, and b* can not fall
  // under the cutoff bin (the 1e-3 absorbs the rounding of T, the log and the bin edges).
  // Scores in bins at or above the cutoff add their masses (2^(y - max) in 2^-40 fixed point)
  // to the group's histogram. The range (lo, 256 / (hi - lo), hi) and T are kept for phase W.
  __device__ __forceinline__ void phase_hist(int k, int step, int tcol) {
    const int g = group_of(k), j = k - sm.cbase()[g];
    const int N = gN(g);
    const int nc = nch(g);
    trace(kEvH0);
    if (!wait_for(P.bar + (int64_t)g * 4 + 0, (uint32_t)nc)) { abort_ = true; return; }
    trace(kEvHw);
    // group statistics in one pass: thread t folds chunks t / G, t / G + kFThreads / G, ... of
    // head t % G into (min, max, mass relative to its running max); lanes of one head, then
    // the warps, combine in a fixed order (every CTA gets the same values)
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    {
      const int t = threadIdx.x, h = t % G;
      float a = INFINITY, z = -INFINITY;
      double m = 0.0;                      // sum 2^(y - z) over the folded chunks
      for (int c = t / G; c < nc; c += kFThreads / G) {
        const float4 v = __ldcg(P.cstat + ((int64_t)g * P.max_nch + c) * G + h);
        a = fminf(a, v.x);
        if (v.y > z) {
          m = (z == -INFINITY ? 0.0 : m * (double)exp2f(z - v.y)) + (double)v.z;
          z = v.y;
        } else {
          m += (double)v.z * (double)exp2f(v.y - z);
        }
      }
#pragma unroll
      for (int o = G; o < 32; o <<= 1) {
        const float a2 = __shfl_xor_sync(0xffffffffu, a, o);
        const float z2 = __shfl_xor_sync(0xffffffffu, z, o);
        const double m2 = __shfl_xor_sync(0xffffffffu, m, o);
        const float zz = fmaxf(z, z2);
        m = zz == -INFINITY ? 0.0
                            : m * (double)exp2f(z - zz) + m2 * (double)exp2f(z2 - zz);
        a = fminf(a, a2);
        z = zz;
      }
      double* pd = sm.tmp();                                 // [16 warps][G] (a, z, m)
      if (lane < G) {
        pd[(warp * G + h) * 3 + 0] = (double)a;
        pd[(warp * G + h) * 3 + 1] = (double)z;
        pd[(warp * G + h) * 3 + 2] = m;
      }
      __syncthreads();
    }
    if (warp < G) {                        // warp h: lanes over the warps, fixed shuffle trees
      const double* pd = sm.tmp();
      const int h = warp;
      float a = INFINITY, z = -INFINITY;
      double m = 0.0;
      if (lane < kWarps) {
        a = (float)pd[(lane * G + h) * 3 + 0];
        z = (float)pd[(lane * G + h) * 3 + 1];
        m = pd[(lane * G + h) * 3 + 2];
      }
      float lo = a, hi = z;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
      }
      double T = z != -INFINITY ? m * (double)exp2f(z - hi) : 0.0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) T += __shfl_xor_sync(0xffffffffu, T, o);
      const float inv = (hi > lo && !P.select_all) ? (float)kBins / (hi - lo) : 0.f;
      // cutoff bin, its score edge; per-head parameters of the binning (top-k counts every
      // token: no cutoff)
      int bch = 0;
      if (P.topk == 0 && P.p < 1.0 && inv > 0.f) {
        const float arg = (float)((1.0 - P.p) * T * (1.0 - 1e-3) / (double)N);
        const float c = hi + log2f(arg);
        bch = c > lo ? bin_of(c, lo, inv) : 0;
      }
      const float e = bin_edge_warp(bch, lo, hi, inv);
      if (lane == 0) {
        sm.lcache()[step * G + h] = make_float4(lo, inv, hi, 0.f);
        if (j == 0) P.grange[(int64_t)g * G + h] = make_float2(lo, inv);
        sm.tcache()[step * G + h] = T;
        reinterpret_cast<float4*>(sm.ints() + kIntHp)[h] = make_float4(lo, inv, hi, 0.f);
        reinterpret_cast<float*>(sm.ints())[kIntEdge + h] = e;
      }
    }
    uint32_t* hlo = sm.hist();
    uint32_t* hhi = hlo + G * kHistStride;
    for (int i = threadIdx.x; i < 2 * G * kHistStride; i += kFThreads) hlo[i] = 0u;
    __syncthreads();
    trace(kEvHs);
    HComp hc;
    {
      const int tig = threadIdx.x & 3;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int n = 2 * tig + e;
        const bool ok = G == 8 ? true : n < 2 * G;
        hc.hd[e] = G == 8 ? n : n % G;
        hc.thr[e] = ok ? reinterpret_cast<const float*>(sm.ints())[kIntEdge + hc.hd[e]] : INFINITY;
      }
    }
    hc.N = N;
    hc.qn = 0;
    hc.qoff = tail(kTailHq) + warp * kHQueueMax * 8;
    hc.hp_off = P.sm_int + kIntHp * 4;
    hc.hist_off = P.sm_hist;
    hc.count_only = P.topk > 0;
    if (tcol >= 0) {
      ScoreTile<G> T;                      // lane layout only (no query needed)
      T.init(sm.qidx());
      const uint32_t ta = chunk_taddr(tcol);
      const int ntl = chunk_tiles(N, nc, j), nst = chunk_stages(N, nc, j);
#pragma unroll 1
      for (int st = 0; st < nst; ++st) {
        float c[V];
        __syncwarp();                      // tcgen05.ld is warp-collective
        Tmem<V>::ld(ta + st * V, c);
        tmem_wait_ld();
        hc(st, tile_row(N, nc, j, ntl, st, warp), c, T);
      }
    } else {
      stream_chunk(g, j, false, false, hc);
    }
    hc.finish();
    __syncthreads();
    trace(kEvH1);
    unsigned long long* gh = P.hist + (int64_t)g * G * kBins * kHistPad;
    for (int i = threadIdx.x; i < G * kBins; i += kFThreads) {
      const int hd = i / kBins, b = i % kBins;
      const unsigned long long v =
          ((unsigned long long)hhi[hd * kHistStride + b] << 32) | hlo[hd * kHistStride + b];
      if (v) atomicAdd(gh + (int64_t)i * kHistPad, v);
    }
    arrive(P.bar + (int64_t)g * 4 + 1);
  }

  // ------------------------------------------------------------ phase W
  // b* per head from the group's histogram and the score edge of b*; the chunk's rows with a
  // score at or above the edge for some head (from the kept scores, or recomputed from the
  // index rows), with the mask of those heads; their K/V rows are gathered once for all G
  // heads. Kept scores: per-warp lists in shared memory, attended every kWBatch stages.
  // Recomputed scores: per-warp regions of the chunk's list in global memory (the index
  // ring and the tiles share the staging region), attended after the pass. The rotated query
  // is formed before the wait. The partials of the group are merged by the last arrival.
  __device__ __forceinline__ void phase_attend(int k, int step, int tcol) {
    const int g = group_of(k), j = k - sm.cbase()[g];
    const int b = g / P.L.n_ret, r = g % P.L.n_ret, kvh = P.L.ret_kv[r];
    const int N = gN(g);
    const int S = nch(g);
    const int ntl = chunk_tiles(N, S, j), nst = chunk_stages(N, S, j);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    rope_query<G>(P, b, kvh, N, sm.q());
    __syncthreads();
    WarpAttn W;
    attn_begin<G>(W, sm.qbuf(), sm.q(), kFThreads);
    ScoreTile<G> T;
    T.init(sm.qidx());                     // lane layout; its query part is not used here
    if (!wait_for(P.bar + (int64_t)g * 4 + 1, (uint32_t)S)) { abort_ = true; return; }
    trace(kEvW0);
    // b* per head (warp h: head h): the highest bin whose mass from the top reaches p T (top-k:
    // whose count from the top reaches k)
    if (warp < G) {
      int best = 0;
      if (!P.select_all) {
        const unsigned long long* gh =
            P.hist + (((int64_t)g * G + warp) * kBins + lane * 8) * kHistPad;
        unsigned long long hv[8], lt = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) { hv[e] = __ldcg(gh + e * kHistPad); lt += hv[e]; }
        unsigned long long x = lt;            // inclusive suffix sum over lanes
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned long long y = __shfl_down_sync(0xffffffffu, x, o);
          if (lane + o < 32) x += y;
        }
        const double thr = P.topk > 0 ? (double)P.topk
                                      : P.p * sm.tcache()[step * G + warp] * (double)kMassScale;
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
      trace(kEvWh);
      const float4 li = sm.lcache()[step * G + warp];
      const float e = bin_edge_warp(best, li.x, li.z, li.y);
      if (lane == 0) {
        sm.ints()[40 + warp] = best;
        reinterpret_cast<float*>(sm.ints())[kIntEdge + warp] = e;
        sm.ints()[kIntCnt + warp] = 0;
      }
    }
    __syncthreads();
    trace(kEvWb);
    if (j == 0 && threadIdx.x < G) P.bstar[(int64_t)g * G + threadIdx.x] = sm.ints()[40 + threadIdx.x];
    float ts[2];
    int hc[2] = {0, 0};
#pragma unroll
    for (int e = 0; e < 2; ++e)
      ts[e] = T.ok[e] ? reinterpret_cast<const float*>(sm.ints())[kIntEdge + T.head[e]] : INFINITY;
    const int64_t rowbase = (int64_t)r * P.L.T_total + P.cache.seq_off[b];
    const uint16_t* kb = P.cache.k_ret + rowbase * kD;
    const uint16_t* vb = P.cache.v_ret + rowbase * kD;
    const int rm_off = tail(kTailRm) + warp * kWRows * 8;
    const int nwa = min(kFThreads / 32, (P.free_bytes - kTailRm) / kTileBytes);
    if (tcol >= 0) {
      uint32_t* list = smem_at<uint32_t>(tail(kTailList));
      uint32_t* wl = list + warp * kWListCap;
      const WarpListRows rows{list, kb, vb, P.sm_int + kIntPre * 4, kWListCap, N, S, j, ntl,
                              (int64_t)kWarps * kWListCap, P.status};
      trace(kEvW1);
      const uint32_t ta = chunk_taddr(tcol);
#pragma unroll 1
      for (int s0 = 0; s0 < nst; s0 += kWBatch) {
        int nw = 0;
        const int s1 = min(nst, s0 + kWBatch);
#pragma unroll 1
        for (int st = s0; st < s1; ++st) {
          float c[V];
          __syncwarp();                    // tcgen05.ld is warp-collective
          Tmem<V>::ld(ta + st * V, c);
          tmem_wait_ld();
          const int rb = tile_row(N, S, j, ntl, st, warp);
          const uint32_t mask = tile_select(c, rb, N, ts, T, rm_off, hc);
          const uint32_t bal = __ballot_sync(0xffffffffu, mask != 0);
          if (mask) wl[nw + __popc(bal & ((1u << lane) - 1u))] = ((uint32_t)(rb + lane) << 8) | mask;
          nw += __popc(bal);
        }
        const int total = list_prefix(nw);
        trace(kEvWl);
        attn_tiles<G>(W, total, rows, sm.stage(), nwa, false);
        __syncthreads();                   // the lists are rewritten by the next batch
      }
    } else {
      uint32_t* gl = P.sellist + (int64_t)g * P.cand_stride;
      WSel wsel;
      wsel.ts[0] = ts[0]; wsel.ts[1] = ts[1];
      wsel.hc[0] = 0; wsel.hc[1] = 0;
      wsel.N = N; wsel.nc = S; wsel.j = j; wsel.ntl = ntl;
      wsel.rm_off = rm_off;
      wsel.nw = 0;
      wsel.gl = gl;
      stream_chunk(g, j, false, true, wsel);
      hc[0] = wsel.hc[0]; hc[1] = wsel.hc[1];
      __threadfence_block();
      const int total = list_prefix(wsel.nw);
      trace(kEvWl);
      const WarpListRows rows{gl, kb, vb, P.sm_int + kIntPre * 4, 0, N, S, j, ntl,
                              P.cand_stride, P.status};
      attn_tiles<G>(W, total, rows, sm.stage(), nwa, false);
    }
    attn_end<G>(W, nwa, sm.res(), reinterpret_cast<float*>(sm.stage()), kFThreads);
    trace(kEvW2);
    // per-head counts of this chunk
#pragma unroll
    for (int e = 0; e < 2; ++e)
      if (T.ok[e] && hc[e]) atomicAdd(sm.ints() + kIntCnt + T.head[e], hc[e]);
    __syncthreads();
    if (threadIdx.x < G) {
      const int v = sm.ints()[kIntCnt + threadIdx.x];
      if (v) atomicAdd(P.hcnt + (int64_t)g * G + threadIdx.x, v);
    }
    // partial -> workspace; the last chunk of the group to finish merges all of them
    write_partial<G, kFThreads>(sm.res(), P.part + (int64_t)k * Part<G>::kBytes);
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      sm.ints()[36] = atomicAdd(P.bar + (int64_t)g * 4 + 2, 1u) == (uint32_t)(S - 1);
    }
    __syncthreads();
    if (!sm.ints()[36]) return;
    __threadfence();
    merge(P.part + (int64_t)sm.cbase()[g] * Part<G>::kBytes, S,
          P.out + ((int64_t)b * P.L.Hq + kvh * G) * kD);
    if (threadIdx.x < G)
      P.sel_counts[(int64_t)b * P.L.Hq + kvh * G + threadIdx.x] =
          __ldcg(P.hcnt + (int64_t)g * G + threadIdx.x);
    trace(kEvW3);
    __syncthreads();
  }

  __device__ __forceinline__ void merge(const unsigned char* parts, int n, uint16_t* out_rows) {
    merge_all<G, kFThreads>(parts, n, out_rows, sm.stage(), P.free_bytes, sm.res());
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
    const RangeRows rowfn{kb, vb, nrows, P.status};
    attn_first_copy(nrows, rowfn, sm.stage(), nwa);
    rope_query<G>(P, b, kvh, N, sm.q());
    __syncthreads();
    WarpAttn W;
    attn_begin<G>(W, sm.qbuf(), sm.q(), kFThreads);
    attn_tiles<G>(W, nrows, rowfn, sm.stage(), nwa, true);
    attn_end<G>(W, nwa, sm.res(), reinterpret_cast<float*>(sm.stage()), kFThreads);
    write_partial<G, kFThreads>(sm.res(), P.lpart + (int64_t)li * Part<G>::kBytes);
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      sm.ints()[38] = atomicAdd(P.loc_arr + lg, 1u) == (uint32_t)(P.PL - 1);
    }
    __syncthreads();
    if (sm.ints()[38]) {
      __threadfence();
      merge(P.lpart + (int64_t)lg * P.PL * Part<G>::kBytes, P.PL,
            P.out + ((int64_t)b * P.L.Hq + kvh * G) * kD);
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
        const int need = chunk_stages(gN(g), nch(g), j) * V;
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
// (the same index query, the same tensor-core tile, so the same bits), binned with the
// group's range and compared with its b* (through bin_of, not the score edge the decode
// kernel compares with, so a test of the two sets also checks the edge); the selected
// positions are compacted in order.
template <int G>
__global__ void __launch_bounds__(kFThreads) emit_sel_kernel(DecodeParams P, int32_t* sel_idx,
                                                             int64_t sel_stride) {
  __shared__ float qidx[G * kR];
  __shared__ float tmp[kFThreads];
  __shared__ int wc[32];
  __shared__ __align__(16) unsigned char rows_s[kWarps][kSlotBytes];
  __shared__ unsigned char keep_s[kWarps][kWRows];
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
    for (int k = t; k < cnt; k += kFThreads)
      if (RTP_CHECK(k < sel_stride, P.status)) dst[k] = k < s1 ? k : w0 + (k - s1);
    return;
  }
  const int g = b * P.L.n_ret + slot;
  const int bst = __ldcg(P.bstar + (int64_t)g * G + jh);
  const float2 li = __ldcg(P.grange + (int64_t)g * G + jh);
  index_query<G>(P, b, kvh, qidx, tmp);
  ScoreTile<G> T;
  T.init(qidx);
  const unsigned char* src = (const unsigned char*)(
      P.cache.idx + ((int64_t)slot * P.L.T_total + P.cache.seq_off[b]) * kR);
  const uint32_t sa = smem_u32(rows_s[warp]);
  int base = 0, par = 0;
#pragma unroll 1
  for (int i0 = 0; i0 < N; i0 += kSRows) {
    const int rb = i0 + warp * kWRows;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int p = lane + 32 * u, r = p >> 1, hh = p & 1;
      *reinterpret_cast<uint4*>(rows_s[warp] + idx_half_off(r, hh)) =
          rb + r < N ? __ldg(reinterpret_cast<const uint4*>(src + (int64_t)(rb + r) * 32 + hh * 16))
                     : make_uint4(0u, 0u, 0u, 0u);
    }
    __syncwarp();
    float c[ScoreTile<G>::V];
    T.score(sa, c);
#pragma unroll
    for (int v = 0; v < ScoreTile<G>::V; ++v) {
      const int e = v & 1;
      if (T.ok[e] && T.head[e] == jh) {
        const int bb = li.y > 0.f ? bin_of(c[v], li.x, li.y) : 0;
        keep_s[warp][T.row[v]] = (rb + T.row[v] < N) && bb >= bst;
      }
    }
    __syncwarp();
    const bool keep = keep_s[warp][lane] != 0;
    int before, total;
    block_flag_prefix(keep, wc + par * 16, before, total);
    par ^= 1;
    if (keep && RTP_CHECK(base + before < sel_stride, P.status)) dst[base + before] = rb + lane;
    base += total;
    __syncwarp();                          // rows_s / keep_s are rewritten next round
  }
}

}  // namespace rtp
