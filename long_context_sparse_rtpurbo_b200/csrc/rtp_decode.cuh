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
// its N tokens are cut into chunks of C tokens; chunk k runs on CTA k mod P (so a CTA holds
// at most a few chunks, in group order). Per group the chunks pass three phases, separated by
// arrival counters in global memory (two device-wide dependencies):
//   S  the chunk's index rows are streamed once from HBM; G scores per row; per-chunk
//      (min, max, sum exp(s - max)) per head. The CTA's last chunk keeps its scores in
//      shared memory; the scores of earlier chunks are recomputed from the index rows, which
//      are still in L2, when their phase H comes.
//   H  from the group's (min, max, total mass): the 256 linear bins and a cutoff bin under
//      which no token can be selected (their total mass is below (1 - p) of the total); per
//      bin fixed-point masses of the tokens at or above the cutoff go to the group's
//      histogram (exact 64-bit sums), and these tokens are emitted as candidates with their
//      bins. Phase H of a group runs after phase S of the CTA's next group, which hides the
//      wait for the other chunks.
//   W  b* per head from the group's histogram; the group's candidates are split evenly over
//      the chunks' CTAs; each keeps the candidates with bin >= b* for some head, gathers
//      their K/V rows once for all G heads (tensor-core tiles, a head that did not select a
//      row masks it) and writes a partial softmax state; partials merge in teams of 32, the
//      last team writes the output rows and the selected counts.
// Local items (a slice of one local head's ring) come from a global queue; a CTA runs them
// while it waits for a group's arrivals, and drains the queue at the end.
// Every wait is bounded (clock64 limit): on expiry the kernel records RTP_ETIMEOUT, raises
// an abort flag that ends every other wait, and returns.
#pragma once

#include "rtp_append.cuh"
#include "rtp_attend.cuh"

namespace rtp {

constexpr int kFThreads = 512;          // threads of the decode kernel
constexpr int kTeam = 32;               // partials merged per team
constexpr int kHeadPad = 8;             // words between the heads' rows of shared buffers
constexpr int kHistStride = 256 + kHeadPad;
constexpr int kSplitRows = 64;          // fewest candidates per gather split
constexpr int kStageBytes = 72 * 1024;  // staging region (index ring, tiles, merge scratch)
constexpr int kChainWarps = kStageBytes / kTileBytes;   // tile warps while the slot is live
constexpr int kMaxSteps = 32;           // chunks per CTA, upper bound
constexpr int kListCap = 4096;          // gather entries staged per batch

struct DecodeParams {
  LayerShape L;
  int P;             // CTAs of the launch
  int C_min;         // smallest chunk (tokens), bounds the chunks per group
  int C_cap;         // chunk tokens whose scores fit the shared-memory score slot
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
  int sm_stage, sm_slot, sm_q, sm_qbuf, sm_qidx, sm_hist, sm_res, sm_tmp, sm_int, sm_N, sm_cbase,
      sm_tcache, free_bytes;
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
  float4* cstat;               // [n_groups][max_nch][G]  chunk (min, max, sum exp(s - max))
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
                  kTraceEvents = 32 };

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

__device__ __forceinline__ int block_max_int(int v, int* scratch /*>= 32 ints*/) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  int s = scratch[0];
  for (int w = 1; w < kFThreads / 32; ++w) s = max(s, scratch[w]);
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
// The score slot follows the staging region, so once the slot is dead (phase W and the final
// local items) the two form one free region of free_bytes.
extern __shared__ __align__(16) unsigned char rtp_smem[];

template <int G> struct Smem {
  const DecodeParams& P;
  __device__ explicit Smem(const DecodeParams& p) : P(p) {}
  __device__ unsigned char* stage() const { return rtp_smem + P.sm_stage; }
  __device__ float* slot() const { return (float*)(rtp_smem + P.sm_slot); }
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
};
// ints[]: [0..31] reduction scratch, [32] wait flag, [33] local item claimed, [34] local
//         queue empty, [35] candidate counter, [36] team-last flag, [37] group-last flag,
//         [38] local-last flag, [40..47] b*, [48..55] decode token's index row (16 bf16)

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

// q_idx[h][j] = W_qidx[h]^T q_pre[b][h] for the G heads of kvh; fixed summation order.
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
    qidx[t] = s;
  }
  __syncthreads();
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
  int C, NC;

  __device__ explicit DecodeCta(const DecodeParams& p) : P(p), sm(p) {}

  __device__ __forceinline__ int group_of(int k) const { return upper_index(sm.cbase(), P.n_groups, k); }
  __device__ __forceinline__ int nch(int g) const { return sm.cbase()[g + 1] - sm.cbase()[g]; }
  __device__ __forceinline__ int gN(int g) const { return sm.N()[g / P.L.n_ret]; }
  __device__ __forceinline__ int64_t slot_hs() const { return (int64_t)P.C_cap + kHeadPad; }

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
  // barrier; while the target is not reached the CTA runs local items from the queue (with
  // the staging region only when the score slot is live). false on timeout / abort.
  __device__ bool wait_for(const uint32_t* ctr, uint32_t target, bool slot_live) {
    const long long t0 = clock64();
    volatile uint32_t* abort_flag = P.misc + 1;
    while (true) {
      if (threadIdx.x == 0) {
        int f = 0;
        if (ld_acquire(ctr) >= target) {
          f = 1;
        } else if (*abort_flag) {
          f = 2;
        } else if (clock64() - t0 > P.spin_limit) {
          set_status(P.status, -5);
          *abort_flag = 1u;
          __threadfence();
          f = 2;
        } else if (!sm.ints()[34]) {
          const uint32_t li = atomicAdd(P.misc + 0, 1u);
          if (li < (uint32_t)P.n_loc_items) { sm.ints()[33] = (int)li; f = 3; }
          else sm.ints()[34] = 1;
        }
        if (f == 1) __threadfence();
        sm.ints()[32] = f;
      }
      __syncthreads();
      const int f = sm.ints()[32];
      __syncthreads();
      if (f == 1) return true;
      if (f == 2) return false;
      if (f == 3) {
        trace_count(kEvNLocWait);
        local_item(sm.ints()[33], slot_live);
        continue;
      }
      if (threadIdx.x == 0) __nanosleep(64);
    }
  }

  // ------------------------------------------------------------ plan (every CTA identical)
  __device__ void plan() {
    const int t = threadIdx.x;
    if (t == 0) { sm.ints()[34] = P.n_loc_items == 0; }
    for (int b = t; b < P.L.B; b += kFThreads) sm.N()[b] = seq_len_checked(P, b);
    __syncthreads();
    int sumN = 0;
    for (int b = t; b < P.L.B; b += kFThreads) sumN += sm.N()[b];
    const long long Tr = (long long)block_sum_int(sumN, sm.ints()) * P.L.n_ret;
    // chunk size: the fewest steps (chunks per CTA) whose chunks fit the score slot, at most
    // kMaxSteps; C >= C_min keeps the chunks per group within the workspace arrays
    C = 1024;
    if (Tr > 0) {
      long long steps = max(1LL, (Tr + (long long)P.P * P.C_cap - 1) / ((long long)P.P * P.C_cap));
      steps = min(steps, (long long)kMaxSteps);
      long long c = P.C_min;
      while (true) {
        const long long den = steps * P.P - P.n_groups;
        if (den < 1) { ++steps; continue; }
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
  // of kSRows rows in the staging region with cp.async; thread t takes row t of each stage
  // and calls fn(nl, s[G]) with its G scores (nl: row within the chunk).
  static constexpr int kSRows = 512, kSStages = 4;
  template <class Fn>
  __device__ __forceinline__ void stream_chunk(int g, int j, bool patch, Fn fn) {
    const int b = g / P.L.n_ret, r = g % P.L.n_ret, kvh = P.L.ret_kv[r];
    const int N = gN(g);
    const int n0 = j * C, n1 = min(N, n0 + C);
    const unsigned char* src = (const unsigned char*)(
        P.cache.idx + ((int64_t)r * P.L.T_total + P.cache.seq_off[b] + n0) * kR);
    const int nst = (n1 - n0 + kSRows - 1) / kSRows;
    auto issue = [&](int st) {
      if (st < nst) {
        unsigned char* dst = sm.stage() + (st % kSStages) * (kSRows * 32);
        const int rows = min(kSRows, n1 - n0 - st * kSRows);
        for (int piece = threadIdx.x; piece < rows * 2; piece += kFThreads)
          cp_async16(dst + piece * 16, src + ((int64_t)st * kSRows * 32) + piece * 16);
      }
      cp_async_commit();
    };
    __syncthreads();                       // the staging region may still be in use
#pragma unroll
    for (int st = 0; st < kSStages - 1; ++st) issue(st);
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
      issue(st + kSStages - 1);
      cp_async_wait<kSStages - 1>();
      __syncthreads();
      const int rows = min(kSRows, n1 - n0 - st * kSRows);
      unsigned char* buf = sm.stage() + (st % kSStages) * (kSRows * 32);
      if (patch && st == nst - 1) {        // the last row of the chunk is the decode token
        if (threadIdx.x < kR / 2)
          reinterpret_cast<uint32_t*>(buf + (rows - 1) * 32)[threadIdx.x] =
              reinterpret_cast<const uint32_t*>(idx_patch)[threadIdx.x];
        __syncthreads();
      }
      const int i = threadIdx.x;
      float s[G];
      if (i < rows) score_row<G>(qi, buf + i * 32, s);
      fn(st * kSRows + i, i < rows, s);
      __syncthreads();                     // before the slot is refilled
    }
    cp_async_wait<0>();
  }

  // ------------------------------------------------------------ phase S
  __device__ __noinline__ void phase_score(int k, bool use_slot) {
    const int g = group_of(k), j = k - sm.cbase()[g];
    const int N = gN(g);
    const bool patch = P.k_new && min(N, (j + 1) * C) == N;
    float mn[G], mx[G], ls[G];
#pragma unroll
    for (int h = 0; h < G; ++h) { mn[h] = INFINITY; mx[h] = -INFINITY; ls[h] = 0.f; }
    float* slot = sm.slot();
    const int64_t hs = slot_hs();
    trace(kEvS0);
    stream_chunk(g, j, patch, [&](int nl, bool ok, const float (&s)[G]) {
      if (!ok) return;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        if (use_slot) slot[h * hs + nl] = s[h];
        mn[h] = fminf(mn[h], s[h]);
        // running sum of exp(s - max) relative to this thread's running max
        if (s[h] > mx[h]) {
          ls[h] = ls[h] * exp2f((mx[h] - s[h]) * kLog2e) + 1.f;
          mx[h] = s[h];
        } else {
          ls[h] += exp2f((s[h] - mx[h]) * kLog2e);
        }
      }
    });
    trace(kEvS1);
    // chunk statistics per head: warp shuffles, then a fixed-order pass over the warps
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float* red = reinterpret_cast<float*>(sm.tmp());         // [3][G][16]
#pragma unroll
    for (int h = 0; h < G; ++h) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, mx[h], o);
        const float l2 = __shfl_xor_sync(0xffffffffu, ls[h], o);
        mn[h] = fminf(mn[h], __shfl_xor_sync(0xffffffffu, mn[h], o));
        const float mm = fmaxf(mx[h], m2);
        ls[h] = (mm == -INFINITY) ? 0.f
                                  : ls[h] * exp2f((mx[h] - mm) * kLog2e) + l2 * exp2f((m2 - mm) * kLog2e);
        mx[h] = mm;
      }
      if (lane == 0) {
        red[(0 * G + h) * 16 + warp] = mn[h];
        red[(1 * G + h) * 16 + warp] = mx[h];
        red[(2 * G + h) * 16 + warp] = ls[h];
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
      double l = 0.0;
      for (int w = 0; w < kFThreads / 32; ++w) {
        const float mw = red[(1 * G + h) * 16 + w];
        if (mw != -INFINITY) l += (double)red[(2 * G + h) * 16 + w] * (double)exp2f((mw - z) * kLog2e);
      }
      P.cstat[((int64_t)g * P.max_nch + j) * G + h] = make_float4(a, z, (float)l, 0.f);
    }
    arrive(P.bar + (int64_t)g * 4 + 0);
  }

  // ------------------------------------------------------------ phase H
  // Group range and total mass from the chunk statistics (double, fixed order: every CTA
  // gets the same values); the cutoff: with T the group's total mass, every token below
  // bin(c), c = hi + ln((1 - p) T' / N), T' = T (1 - 1e-3), has mass below (1 - p) T' / N, so
  // together they hold less than (1 - p) of the total, C_bin(c) > p T, and b* can not fall
  // under the cutoff bin (the 1e-3 absorbs the rounding of T, the log and the bin edges).
  // Masses are exp(s - max) in 2^-40 fixed point, summed with two 32-bit shared atomics per
  // (token, head): the low-word add returns the old value and its carry goes to the high word.
  __device__ __noinline__ void phase_hist(int k, int step, bool from_slot) {
    const int g = group_of(k), j = k - sm.cbase()[g];
    const int N = gN(g), n0 = j * C, len = min(N, n0 + C) - n0;
    const int nc = nch(g);
    trace(kEvH0);
    // the slot may hold the CTA's last chunk while an earlier chunk waits here
    if (!wait_for(P.bar + (int64_t)g * 4 + 0, (uint32_t)nc, true)) { abort_ = true; return; }
    trace(kEvHw);
    // group statistics: thread t folds chunks t / G, t / G + kFThreads / G, ... of head t % G
    double* part = sm.tmp();                                 // [kFThreads]
    float* st3 = reinterpret_cast<float*>(sm.res());         // [G][3] lo, hi, inv
    {
      const int t = threadIdx.x, h = t % G;
      float a = INFINITY, z = -INFINITY;
      for (int c = t / G; c < nc; c += kFThreads / G) {
        const float4 v = __ldcg(P.cstat + ((int64_t)g * P.max_nch + c) * G + h);
        a = fminf(a, v.x);
        z = fmaxf(z, v.y);
      }
      // reduce over the threads of head h (lanes t, t + G, ...) inside each warp, then warps
#pragma unroll
      for (int o = G; o < 32; o <<= 1) {
        a = fminf(a, __shfl_xor_sync(0xffffffffu, a, o));
        z = fmaxf(z, __shfl_xor_sync(0xffffffffu, z, o));
      }
      int* ri = sm.ints();
      __syncthreads();
      if ((t & 31) < G) {
        reinterpret_cast<float*>(part)[(t >> 5) * G + h] = a;
        reinterpret_cast<float*>(part)[512 + (t >> 5) * G + h] = z;
      }
      __syncthreads();
      if (t < G) {
        float lo = INFINITY, hi = -INFINITY;
        for (int w = 0; w < kFThreads / 32; ++w) {
          lo = fminf(lo, reinterpret_cast<float*>(part)[w * G + t]);
          hi = fmaxf(hi, reinterpret_cast<float*>(part)[512 + w * G + t]);
        }
        st3[t * 3 + 0] = lo;
        st3[t * 3 + 1] = hi;
        st3[t * 3 + 2] = (hi > lo && !P.select_all) ? (float)kBins / (hi - lo) : 0.f;
      }
      (void)ri;
      __syncthreads();
      const float hih = st3[h * 3 + 1];
      double acc = 0.0;
      for (int c = t / G; c < nc; c += kFThreads / G) {
        const float4 v = __ldcg(P.cstat + ((int64_t)g * P.max_nch + c) * G + h);
        acc += (double)v.z * (double)exp2f((v.y - hih) * kLog2e);
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
    uint32_t* hlo = sm.hist();
    uint32_t* hhi = hlo + G * kHistStride;
    for (int i = threadIdx.x; i < 2 * G * kHistStride; i += kFThreads) hlo[i] = 0u;
    float lo[G], hi[G], inv[G];
    int bch[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      lo[h] = st3[h * 3 + 0];
      hi[h] = st3[h * 3 + 1];
      inv[h] = st3[h * 3 + 2];
      bch[h] = 0;
      if (P.p < 1.0 && inv[h] > 0.f) {
        const double T = sm.tcache()[step * G + h];
        const float arg = (float)((1.0 - P.p) * T * (1.0 - 1e-3) / (double)N);
        const float c = hi[h] + logf(arg);
        bch[h] = c > lo[h] ? bin_of(c, lo[h], inv[h]) : 0;
      }
    }
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t* cpos = P.cpos + (int64_t)g * P.cand_stride + n0;
    uint2* cbin = P.cbin + (int64_t)g * P.cand_stride + n0;
    int run = 0;                             // candidates written so far (every thread)
    int* wc = sm.ints();                     // per-warp counts of the current block
    // candidates of one block of kFThreads tokens, written in token order
    auto emit = [&](int nl, bool ok, const float (&s)[G]) {
      bool cand = false;
      uint32_t bw0 = 0, bw1 = 0;
      if (ok) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const int b = inv[h] > 0.f ? bin_of(s[h], lo[h], inv[h]) : 0;
          if (h < 4) bw0 |= (uint32_t)b << (8 * h); else bw1 |= (uint32_t)b << (8 * (h - 4));
          if (b >= bch[h]) {
            cand = true;
            const float ex = (s[h] - hi[h]) * kLog2e;
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
      const uint32_t bal = __ballot_sync(0xffffffffu, cand);
      if (lane == 0) wc[warp] = __popc(bal);
      __syncthreads();
      int before = 0, total = 0;
#pragma unroll
      for (int w = 0; w < kFThreads / 32; ++w) {
        const int x = wc[w];
        before += w < warp ? x : 0;
        total += x;
      }
      if (cand) {
        const int o = run + before + __popc(bal & ((1u << lane) - 1u));
        cpos[o] = (uint32_t)(n0 + nl);
        cbin[o] = make_uint2(bw0, bw1);
      }
      run += total;
      __syncthreads();                       // wc is rewritten by the next block
    };
    if (from_slot) {
      const float* slot = sm.slot();
      const int64_t hs = slot_hs();
#pragma unroll 1
      for (int i0 = 0; i0 < len; i0 += kFThreads) {
        const int nl = i0 + threadIdx.x;
        float s[G];
#pragma unroll
        for (int h = 0; h < G; ++h) s[h] = nl < len ? slot[h * hs + nl] : 0.f;
        emit(nl, nl < len, s);
      }
    } else {
      stream_chunk(g, j, false, emit);
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
    if (threadIdx.x == 0) P.ccnt[(int64_t)g * P.max_nch + j] = (uint32_t)run;
    arrive(P.bar + (int64_t)g * 4 + 1);
  }

  // b* of the G heads of group g into sm.ints()[40 + h]; warp h handles head h.
  __device__ void find_bstar(int g, int step) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (warp < G) {
      const int h = warp;
      if (P.select_all) {
        if (lane == 0) sm.ints()[40 + h] = 0;
      } else {
        const unsigned long long* gh = P.hist + ((int64_t)g * G + h) * kBins;
        unsigned long long v[8], lt = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) { v[e] = __ldcg(gh + lane * 8 + e); lt += v[e]; }
        unsigned long long x = lt;            // inclusive suffix sum over lanes
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned long long y = __shfl_down_sync(0xffffffffu, x, o);
          if (lane + o < 32) x += y;
        }
        const double thr = P.p * sm.tcache()[step * G + h] * (double)kMassScale;
        int best = -1;
        unsigned long long cum = x - lt;
#pragma unroll
        for (int e = 7; e >= 0; --e) {
          cum += v[e];
          if (best < 0 && (double)cum >= thr) best = lane * 8 + e;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) best = max(best, __shfl_xor_sync(0xffffffffu, best, o));
        if (lane == 0) sm.ints()[40 + h] = best < 0 ? 0 : best;
      }
    }
    __syncthreads();
  }

  __device__ __noinline__ void merge(const float* parts, int n, float* dst, uint16_t* out_rows,
                                     bool slot_live) {
    merge_partials<G>(parts, n, dst, out_rows, reinterpret_cast<float*>(sm.stage()),
                      slot_live ? kStageBytes : P.free_bytes, kFThreads);
  }

  // ------------------------------------------------------------ phase W
  // Split j of group g: candidates [e0, e1) of the group's list (chunk after chunk), in
  // batches of kListCap; a candidate is kept when a head's bin reaches its b*, with the mask
  // of those heads. The list and the chunk prefix sit at the end of the free region (the
  // score slot is dead by now); the tiles use its start.
  __device__ __noinline__ void phase_attend(int k, int step) {
    const int g = group_of(k), j = k - sm.cbase()[g];
    const int b = g / P.L.n_ret, r = g % P.L.n_ret, kvh = P.L.ret_kv[r];
    const int N = gN(g);
    const int S = nch(g);
    if (!wait_for(P.bar + (int64_t)g * 4 + 1, (uint32_t)S, false)) { abort_ = true; return; }
    trace(kEvW0);
    find_bstar(g, step);
    int bs[G];
#pragma unroll
    for (int h = 0; h < G; ++h) bs[h] = sm.ints()[40 + h];
    if (j == 0 && threadIdx.x < G) P.bstar[(int64_t)g * G + threadIdx.x] = bs[threadIdx.x];
    const int pref_bytes = ((S + 1) * 4 + 15) / 16 * 16;
    int* pref = reinterpret_cast<int*>(sm.stage() + P.free_bytes - pref_bytes);
    uint32_t* list = reinterpret_cast<uint32_t*>(reinterpret_cast<unsigned char*>(pref) - kListCap * 4);
    for (int c = threadIdx.x; c < S; c += kFThreads)
      pref[c] = (int)__ldcg(P.ccnt + (int64_t)g * P.max_nch + c);
    __syncthreads();
    const int U = block_scan_excl(pref, S, sm.ints());
    const int nsplit = min(S, max(1, (U + kSplitRows - 1) / kSplitRows));
    if (j >= nsplit) return;
    rope_query<G>(P, b, kvh, N, sm.q());
    const int e0 = (int)(((long long)U * j) / nsplit), e1 = (int)(((long long)U * (j + 1)) / nsplit);
    const int64_t rowbase = (int64_t)r * P.L.T_total + P.cache.seq_off[b];
    const uint16_t* kb = P.cache.k_ret + rowbase * kD;
    const uint16_t* vb = P.cache.v_ret + rowbase * kD;
    const uint32_t* gpos = P.cpos + (int64_t)g * P.cand_stride;
    const uint2* gbin = P.cbin + (int64_t)g * P.cand_stride;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwa = min(kFThreads / 32, (P.free_bytes - pref_bytes - kListCap * 4) / kTileBytes);
    int hc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) hc[h] = 0;
    __syncthreads();                      // sm.q() complete
    WarpAttn W;
    attn_begin<G>(W, sm.qbuf(), sm.q(), kFThreads);
    trace(kEvW1);
#pragma unroll 1
    for (int b0 = e0; b0 < e1; b0 += kListCap) {
      const int b1 = min(e1, b0 + kListCap);
      int nb = 0;                         // kept entries of this batch (every thread)
      int* wc = sm.ints();
      __syncthreads();                    // the previous batch's list is no longer read
      for (int x0 = b0; x0 < b1; x0 += kFThreads) {
        const int e = x0 + threadIdx.x;
        uint32_t mask = 0, pos = 0;
        if (e < b1) {
          const int c = upper_index(pref, S, e);
          const int64_t o = (int64_t)c * C + (e - pref[c]);
          pos = __ldcg(gpos + o);
          const uint2 bw = __ldcg(gbin + o);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const int bb = (int)(((h < 4 ? bw.x : bw.y) >> (8 * (h & 3))) & 0xffu);
            if (bb >= bs[h]) { mask |= 1u << h; hc[h]++; }
          }
        }
        // kept entries in candidate order
        const uint32_t bal = __ballot_sync(0xffffffffu, mask != 0);
        if (lane == 0) wc[warp] = __popc(bal);
        __syncthreads();
        int before = 0, total = 0;
#pragma unroll
        for (int w = 0; w < kFThreads / 32; ++w) {
          const int x = wc[w];
          before += w < warp ? x : 0;
          total += x;
        }
        if (mask) list[nb + before + __popc(bal & ((1u << lane) - 1u))] = (pos << 8) | mask;
        nb += total;
        __syncthreads();
      }
      attn_tiles<G>(W, nb, [&](int i, const uint16_t*& kp, const uint16_t*& vp, uint32_t& mk) {
        const uint32_t w = list[i];
        kp = kb + (int64_t)(w >> 8) * kD;
        vp = vb + (int64_t)(w >> 8) * kD;
        mk = w & 0xffu;
      }, sm.stage(), nwa);
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
    // partial -> workspace; team / group merge by the last arrivals
    const int stride = G * (kD + 2);
    float* mine = P.part + (int64_t)k * stride;
    for (int o = threadIdx.x; o < stride; o += kFThreads) mine[o] = sm.res()[o];
    const int team = j / kTeam, nteams = (nsplit + kTeam - 1) / kTeam;
    const int tcount = min(kTeam, nsplit - team * kTeam);
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
      merge(tparts, tcount, nullptr, orow, false);
    } else {
      merge(tparts, tcount, P.tpart + (int64_t)(sm.cbase()[g] + team) * stride, nullptr, false);
      __syncthreads();
      if (threadIdx.x == 0) {
        __threadfence();
        sm.ints()[37] = atomicAdd(P.bar + (int64_t)g * 4 + 2, 1u) == (uint32_t)(nteams - 1);
      }
      __syncthreads();
      if (!sm.ints()[37]) return;
      __threadfence();
      merge(P.tpart + (int64_t)sm.cbase()[g] * stride, nteams, nullptr, orow, false);
    }
    if (threadIdx.x < G)
      P.sel_counts[(int64_t)b * P.L.Hq + kvh * G + threadIdx.x] =
          __ldcg(P.hcnt + (int64_t)g * G + threadIdx.x);
    trace(kEvW3);
    __syncthreads();
  }

  // ------------------------------------------------------------ local items
  // Attention over one slice of RL ring rows of a local head; the partials of a head merge
  // by the last arrival. slot_live: the score slot holds scores (staging region only).
  __device__ __noinline__ void local_item(int li, bool slot_live) {
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
    rope_query<G>(P, b, kvh, N, sm.q());
    __syncthreads();
    const int64_t ring0 = ((int64_t)x * P.L.B + b) * P.L.ring + r0;
    const int nwa = slot_live ? kChainWarps : min(kFThreads / 32, P.free_bytes / kTileBytes);
    const uint16_t* kb = P.cache.k_loc + ring0 * kD;
    const uint16_t* vb = P.cache.v_loc + ring0 * kD;
    WarpAttn W;
    attn_begin<G>(W, sm.qbuf(), sm.q(), kFThreads);
    attn_tiles<G>(W, nrows, [&](int i, const uint16_t*& kp, const uint16_t*& vp, uint32_t& mk) {
      kp = kb + (int64_t)i * kD;
      vp = vb + (int64_t)i * kD;
      mk = 0xffu;
    }, sm.stage(), nwa);
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
            P.out + ((int64_t)b * P.L.Hq + kvh * G) * kD, slot_live);
      if (threadIdx.x < G) P.sel_counts[(int64_t)b * P.L.Hq + kvh * G + threadIdx.x] = nrows_all;
    }
    __syncthreads();
    trace(kEvLoc1);
  }

  bool abort_ = false;

  // Chunks k_t = blockIdx.x + t P of this CTA, in group order. Phase S runs for every chunk
  // in turn; the chunks of a group get their phase H once the CTA has scored the first chunk
  // of the next group (or at the end), so the wait for the group's other chunks overlaps
  // that scoring. Phase H of every chunk but the last recomputes its scores; the last chunk
  // keeps them in the shared-memory slot when it fits. Then phase W of every chunk, then the
  // remaining local items.
  __device__ void run() {
    trace(kEvStart);
    plan();
    trace(kEvPlan);
    const int i = blockIdx.x;
    const int m = i < NC ? (NC - i + P.P - 1) / P.P : 0;
    bool last_in_slot = false;
    if (m > 0) {
      const int kl = i + (m - 1) * P.P, gl = group_of(kl);
      last_in_slot = min(gN(gl), (kl - sm.cbase()[gl] + 1) * C) - (kl - sm.cbase()[gl]) * C <= P.C_cap;
    }
    int pstart = 0;
    for (int t = 0; t < m; ++t) {
      const int k = i + t * P.P;
      phase_score(k, t == m - 1 && last_in_slot);
      if (pstart < t && group_of(i + pstart * P.P) != group_of(k)) {
        for (int s = pstart; s < t; ++s) {
          phase_hist(i + s * P.P, s, false);
          if (abort_) return;
        }
        pstart = t;
      }
    }
    for (int s = pstart; s < m; ++s) {
      phase_hist(i + s * P.P, s, s == m - 1 && last_in_slot);
      if (abort_) return;
    }
    for (int t = 0; t < m; ++t) {
      phase_attend(i + t * P.P, t);
      if (abort_) return;
    }
    // remaining local items
    trace(kEvDrain);
    while (true) {
      if (threadIdx.x == 0) {
        int li = -1;
        if (!sm.ints()[34]) {
          const uint32_t x = atomicAdd(P.misc + 0, 1u);
          if (x < (uint32_t)P.n_loc_items) li = (int)x; else sm.ints()[34] = 1;
        }
        sm.ints()[33] = li;
      }
      __syncthreads();
      const int li = sm.ints()[33];
      __syncthreads();
      if (li < 0) break;
      trace_count(kEvNLocDrain);
      local_item(li, false);
    }
    trace(kEvEnd);
  }
};

template <int G>
__global__ void __launch_bounds__(kFThreads, 1) decode_kernel(const __grid_constant__ DecodeParams P) {
  DecodeCta<G> cta(P);
  cta.run();
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
