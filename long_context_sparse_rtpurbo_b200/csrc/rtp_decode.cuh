// Decode step of one layer in one persistent kernel: index scoring, the 256-bin top-p
// threshold, selection, and exact softmax attention over the selected rows (retrieval heads)
// or over the sinks + window (local heads).
//
// "Full Attention Strikes Back" (paper text) §3.2: eq. (4) s(m,n) = (W^Q q^pre)^T (W^K k^pre),
// eq. (5) O = sum over S of softmax(q^T k / sqrt(d)) v with S = Top-P(s, p); local heads use
// attention sinks plus a sliding window. MCISLAB DeepRead notes on RTPurbo, "Method": top-p
// is found sort-free with a 256-bin histogram per head, fused with the scoring.
//
// Work split. A retrieval group is one (sequence, retrieval KV head) with its G query heads;
// its N tokens are cut into chunks of C tokens. CTAs [0, P_ret) run the retrieval chunks
// (chunk k on CTA k mod P_ret, in waves that fit the shared-memory score buffers); the other
// CTAs start on the local heads at once, P_ret following the byte share of the two sides.
// Per group the chunks pass four phases, separated by arrival counters in global memory:
//   S  scores of the G heads for the chunk's tokens (kept in shared memory when every CTA
//      owns at most one chunk, else in the workspace); group min / max by integer atomics.
//   H  the chunk's 256-bin mass histogram exp(s - max) per head, added to the group's
//      histogram in 2^-40 fixed point (exact and order independent).
//   T  b* per head from the group histogram; tokens whose bin >= b* for any head are
//      compacted in ascending order into entries (n << 8 | head mask); counts.
//   W  the group's entries are split evenly over its chunks' CTAs; each gathers its rows
//      once for all G heads (a head that did not select a row skips it) and writes a
//      partial softmax state; partials merge in teams of 32, the last team writes out.
// Local items (a slice of one local head's ring) come from a global queue; retrieval CTAs
// join when their chunks are done, so a local item never delays the retrieval chain.
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

struct DecodeParams {
  LayerShape L;
  int P;             // CTAs of the launch
  int C_min;         // smallest chunk (tokens), bounds the chunk count
  int C_cap;         // chunk tokens whose scores fit the shared-memory score buffer
  int max_nch;       // chunks per group upper bound (shared array size)
  int NC_max;        // chunks per launch upper bound (workspace arrays)
  int n_groups;      // B * n_ret
  int n_lgroups;     // B * n_loc
  int PL;            // local items per local group
  int RL;            // ring rows per local item
  int n_loc_items;
  int select_all;    // p >= 1
  double p;
  long long spin_limit;
  int64_t maxN_pad;
  // shared-memory layout (byte offsets into the dynamic buffer)
  int sm_scores, sm_stage, sm_res, sm_qret, sm_qloc, sm_qidx, sm_tmp, sm_hist, sm_N, sm_cbase,
      sm_pref, sm_int;
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
  uint32_t* lohi;              // [n_groups][2][G]   ~ord(min), ord(max)        (zeroed)
  int32_t* hcnt;               // [n_groups][G]      selected tokens per head    (zeroed)
  uint32_t* bar;               // [n_groups][4]      phase arrivals, teams done  (zeroed)
  uint32_t* team_arr;          // [NC_max]           team arrivals              (zeroed)
  uint32_t* loc_arr;           // [n_lgroups]        local item arrivals        (zeroed)
  uint32_t* misc;              // [0] local queue head, [1] abort, [2] chunk size (zeroed)
  unsigned long long* hist;    // [n_groups][G][256]                            (zeroed)
  float* scores;               // [n_groups][G][maxN_pad] (when chunks do not fit on chip)
  uint32_t* ent;               // [n_groups][maxN_pad]
  uint32_t* ccnt;              // [n_groups][max_nch]
  float2* cstat;               // [n_groups][max_nch][G] chunk (max score, sum exp(s - max))
  float* part;                 // [NC_max][G][130]
  float* tpart;                // [NC_max][G][130]
  float* lpart;                // [n_loc_items][G][130]
  unsigned long long* trace;   // [P][kTraceEvents] %globaltimer stamps (tracing builds only)
};

// Phase-boundary timestamps, recorded only when built with -DRTP_TRACE.
enum TraceEvent { kEvStart, kEvPlan, kEvScore, kEvWait1, kEvHist, kEvWait2, kEvSelect, kEvWait3,
                  kEvAttend, kEvLocal, kEvEnd, kEvS0, kEvS1, kEvH0, kEvH1, kEvH2, kEvT0, kEvT1,
                  kEvW0, kEvW1, kEvW2, kTraceEvents = 32 };

// ------------------------------------------------------------------------------ helpers
__device__ __forceinline__ int seq_len_checked(const DecodeParams& P, int b) {
  // three independent loads, one round trip
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

// stage: index-row staging (phase S), K/V row staging and merge scratch (attention).
// Dynamic shared memory of the decode kernel; its regions sit at the offsets in DecodeParams.
extern __shared__ __align__(16) unsigned char rtp_smem[];

// Region pointers, formed on each use from the kernel parameters (constant bank) rather than
// held in registers across the phases.
template <int G> struct Smem {
  const DecodeParams& P;
  __device__ explicit Smem(const DecodeParams& p) : P(p) {}
  __device__ float* scores() const { return (float*)(rtp_smem + P.sm_scores); }
  __device__ unsigned char* stage() const { return rtp_smem + P.sm_stage; }
  __device__ float* res() const { return (float*)(rtp_smem + P.sm_res); }
  __device__ float* qret() const { return (float*)(rtp_smem + P.sm_qret); }
  __device__ float* qloc() const { return (float*)(rtp_smem + P.sm_qloc); }
  __device__ float* qidx() const { return (float*)(rtp_smem + P.sm_qidx); }
  __device__ float* tmp() const { return (float*)(rtp_smem + P.sm_tmp); }
  __device__ unsigned long long* hist() const { return (unsigned long long*)(rtp_smem + P.sm_hist); }
  __device__ int* N() const { return (int*)(rtp_smem + P.sm_N); }
  __device__ int* cbase() const { return (int*)(rtp_smem + P.sm_cbase); }
  __device__ int* pref() const { return (int*)(rtp_smem + P.sm_pref); }
  __device__ int* ints() const { return (int*)(rtp_smem + P.sm_int); }
};
// ints[]: [0..31] reduction scratch, [32] wait flag, [33] next local item, [34] group of the
//         total in tmp, [40..47] b*, [48..50] last-arrival flags, [56..63] decode token's
//         index row (phase S of the last chunk)

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

template <int G>
__device__ __forceinline__ void load_range(const DecodeParams& P, int g, float* lo, float* hi,
                                           float* inv) {
#pragma unroll
  for (int h = 0; h < G; ++h) {
    lo[h] = ord2f(~__ldcg(P.lohi + ((int64_t)g * 2 + 0) * G + h));
    hi[h] = ord2f(__ldcg(P.lohi + ((int64_t)g * 2 + 1) * G + h));
    inv[h] = (hi[h] > lo[h] && !P.select_all) ? (float)kBins / (hi[h] - lo[h]) : 0.f;
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
  int C, NC, smem_mode, P_ret;

  __device__ explicit DecodeCta(const DecodeParams& p) : P(p), sm(p) {}

  __device__ __forceinline__ int group_of(int k) const { return upper_index(sm.cbase(), P.n_groups, k); }
  __device__ __forceinline__ int nch(int g) const { return sm.cbase()[g + 1] - sm.cbase()[g]; }
  __device__ __forceinline__ int gN(int g) const { return sm.N()[g / P.L.n_ret]; }

  __device__ __forceinline__ float* score_ptr(int g, int j) const {
    return smem_mode ? sm.scores() : P.scores + (int64_t)g * G * P.maxN_pad + (int64_t)j * C;
  }
  __device__ __forceinline__ int64_t score_hstride() const {
    return smem_mode ? (int64_t)P.C_cap + kHeadPad : P.maxN_pad;
  }

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

  // the decode token (position N - 1) of sequence b, KV head kvh into the caches
  __device__ __forceinline__ void append_new(int b, int kvh, int N, uint16_t* idx_patch) {
    const int64_t o = ((int64_t)b * P.L.Hkv + kvh) * kD;
    append_token(P.L, P.cache, P.k_new + o, P.v_new + o, P.w_kidx, b, kvh, (int64_t)(N - 1),
                 reinterpret_cast<double*>(sm.tmp()), idx_patch);
    if (threadIdx.x == 0) sm.ints()[34] = -1;  // sm.tmp() no longer holds a group total
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
  __device__ bool wait_for(const uint32_t* ctr, uint32_t target) {
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
        }
        if (f == 1) __threadfence();
        sm.ints()[32] = f;
      }
      __syncthreads();
      const int f = sm.ints()[32];
      __syncthreads();
      if (f == 1) return true;
      if (f == 2) return false;
      if (threadIdx.x == 0) __nanosleep(100);
    }
  }

  // ------------------------------------------------------------ plan (every CTA identical)
  __device__ void plan() {
    const int t = threadIdx.x;
    if (t == 0) sm.ints()[34] = -1;           // no group total in sm.tmp() yet
    for (int b = t; b < P.L.B; b += kFThreads) sm.N()[b] = seq_len_checked(P, b);
    __syncthreads();
    int sumN = 0, sumL = 0, maxN = 0;
    for (int b = t; b < P.L.B; b += kFThreads) {
      sumN += sm.N()[b];
      sumL += min(sm.N()[b], P.L.ring);
      maxN = max(maxN, sm.N()[b]);
    }
    const long long Tr = (long long)block_sum_int(sumN, sm.ints()) * P.L.n_ret;
    const long long loc_rows = (long long)block_sum_int(sumL, sm.ints()) * P.L.n_loc;
    maxN = block_max_int(maxN, sm.ints());
    // CTAs [0, P_ret) run the retrieval chain, the others start on local items at once; the
    // split follows the bytes of each side (index read twice as a proxy for index + gather).
    P_ret = 0;
    C = 1024;
    smem_mode = 1;
    if (Tr > 0) {
      const double ret_b = 64.0 * (double)Tr, loc_b = 512.0 * (double)loc_rows;
      int pr = (int)((double)P.P * ret_b / (ret_b + loc_b) + 0.5);
      pr = max(1, min(P.P, pr));
      const long long one_wave = (Tr + P.C_cap - 1) / P.C_cap + P.n_groups;   // chunks at C_cap
      pr = max(pr, (int)min((long long)P.P, one_wave));
      const int need = (maxN + P.C_cap - 1) / P.C_cap;          // a group within one wave
      if (need > P.P) {
        smem_mode = 0;                                          // scores spill to the workspace
        pr = P.P;
        long long c = (Tr + 2LL * P.P - 1) / (2LL * P.P);
        c = max(c, (long long)P.C_min);
        C = (int)((c + 255) / 256 * 256);
      } else {
        pr = max(pr, need);
        long long c = (pr > P.n_groups) ? (Tr + (pr - P.n_groups) - 1) / (pr - P.n_groups)
                                        : (Tr + pr - 1) / pr;
        c = max(c, (long long)P.C_min);
        c = max(c, (long long)((maxN + pr - 1) / pr));
        c = (c + 255) / 256 * 256;
        C = (int)min(c, (long long)P.C_cap);                   // C_cap: more than one wave
      }
      P_ret = pr;
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

  // ------------------------------------------------------------ phase S
  // The chunk's index rows (32 B each, contiguous) stream through a ring of kSStages stages
  // of kSRows rows in shared memory with cp.async; the projected query is formed while the
  // first stages are in flight.
  static constexpr int kSRows = 512, kSStages = 4;
  __device__ void phase_score(int k) {
    const int g = group_of(k), j = k - sm.cbase()[g];
    const int b = g / P.L.n_ret, r = g % P.L.n_ret, kvh = P.L.ret_kv[r];
    const int N = gN(g);
    const int n0 = j * C, n1 = min(N, n0 + C);
    const unsigned char* src =
        (const unsigned char*)(P.cache.idx + ((int64_t)r * P.L.T_total + P.cache.seq_off[b] + n0) * kR);
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
    __syncthreads();                       // the stage buffer may still be read by a merge
#pragma unroll
    for (int st = 0; st < kSStages - 1; ++st) issue(st);
    index_query<G>(P, b, kvh, sm.qidx(), sm.tmp());
    // The chunk holding the decode token writes it while the first stages are in flight; a
    // copy of its index row may still be stale, so the stage holding it is patched below.
    const bool patch = P.k_new && n1 == N;
    uint16_t* idx_patch = reinterpret_cast<uint16_t*>(sm.ints() + 56);   // 16 bf16
    if (patch) append_new(b, kvh, N, idx_patch);
    trace(kEvS0);
    float2 qi[G][kR / 2];                    // index query, channel pairs (2j, 2j + 1)
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int jj = 0; jj < kR / 2; ++jj)
        qi[h][jj] = make_float2(sm.qidx()[h * kR + 2 * jj], sm.qidx()[h * kR + 2 * jj + 1]);
    float mn[G], mx[G];
#pragma unroll
    for (int h = 0; h < G; ++h) { mn[h] = INFINITY; mx[h] = -INFINITY; }
    float* sc = score_ptr(g, j);
    const int64_t hs = score_hstride();
#pragma unroll 1
    for (int st = 0; st < nst; ++st) {
      issue(st + kSStages - 1);
      cp_async_wait<kSStages - 1>();
      __syncthreads();
      const int rows = min(kSRows, n1 - n0 - st * kSRows);
      const unsigned char* buf = sm.stage() + (st % kSStages) * (kSRows * 32);
      if (patch && st == nst - 1) {        // the last row of the chunk is the decode token
        if (threadIdx.x < kR / 2)
          reinterpret_cast<uint32_t*>(const_cast<unsigned char*>(buf) + (rows - 1) * 32)[threadIdx.x] =
              reinterpret_cast<const uint32_t*>(idx_patch)[threadIdx.x];
        __syncthreads();
      }
#pragma unroll 1
      for (int i = threadIdx.x; i < rows; i += kFThreads) {
        const uint4 a = *reinterpret_cast<const uint4*>(buf + i * 32);
        const uint4 c2 = *reinterpret_cast<const uint4*>(buf + i * 32 + 16);
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, c2.x, c2.y, c2.z, c2.w};
        float2 x[kR / 2];                      // channel pairs: even and odd sums, then added
#pragma unroll
        for (int jj = 0; jj < kR / 2; ++jj) x[jj] = make_float2(bf_lo(w[jj]), bf_hi(w[jj]));
        const int nl = st * kSRows + i;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float2 a2 = __fmul2_rn(qi[h][0], x[0]);
#pragma unroll
          for (int jj = 1; jj < kR / 2; ++jj) a2 = __ffma2_rn(qi[h][jj], x[jj], a2);
          const float acc = a2.x + a2.y;
          sc[h * hs + nl] = acc;
          mn[h] = fminf(mn[h], acc);
          mx[h] = fmaxf(mx[h], acc);
        }
      }
      __syncthreads();                     // before the slot is refilled
    }
    cp_async_wait<0>();
    trace(kEvS1);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float* red = sm.tmp();                    // [2][G][16], then [G][16]
    if (threadIdx.x == 0) sm.ints()[34] = -1; // sm.tmp() no longer holds a group total
    __syncthreads();
#pragma unroll
    for (int h = 0; h < G; ++h) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        mn[h] = fminf(mn[h], __shfl_xor_sync(0xffffffffu, mn[h], o));
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], o));
      }
      if (lane == 0) { red[(0 * G + h) * 16 + warp] = mn[h]; red[(1 * G + h) * 16 + warp] = mx[h]; }
    }
    __syncthreads();
    float cmax[G];                          // the chunk's max per head (every thread)
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float z = red[(1 * G + h) * 16];
      for (int w = 1; w < kFThreads / 32; ++w) z = fmaxf(z, red[(1 * G + h) * 16 + w]);
      cmax[h] = z;
    }
    if (threadIdx.x < G) {
      const int h = threadIdx.x;
      float a = red[(0 * G + h) * 16];
      for (int w = 1; w < kFThreads / 32; ++w) a = fminf(a, red[(0 * G + h) * 16 + w]);
      atomicMax(P.lohi + ((int64_t)g * 2 + 0) * G + h, ~f2ord(a));
      atomicMax(P.lohi + ((int64_t)g * 2 + 1) * G + h, f2ord(cmax[h]));
    }
    // the chunk's total mass relative to its max: sum exp(s - cmax) over the shared scores
    float ls[G];
#pragma unroll
    for (int h = 0; h < G; ++h) ls[h] = 0.f;
#pragma unroll 4
    for (int i = threadIdx.x; i < n1 - n0; i += kFThreads)
#pragma unroll
      for (int h = 0; h < G; ++h) ls[h] += exp2f((sc[h * hs + i] - cmax[h]) * kLog2e);
    __syncthreads();
#pragma unroll
    for (int h = 0; h < G; ++h) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ls[h] += __shfl_xor_sync(0xffffffffu, ls[h], o);
      if (lane == 0) red[h * 16 + warp] = ls[h];
    }
    __syncthreads();
    if (threadIdx.x < G) {
      const int h = threadIdx.x;
      double l = 0.0;                       // fixed order
      for (int w = 0; w < kFThreads / 32; ++w) l += (double)red[h * 16 + w];
      P.cstat[((int64_t)g * P.max_nch + j) * G + h] = make_float2(cmax[h], (float)l);
    }
    arrive(P.bar + (int64_t)g * 4 + 0);
    // the RoPE'd query of phase W (scores-in-shared-memory schedule), formed off the critical
    // path: after this chunk has arrived, while the other chunks of the group finish
    if (smem_mode) rope_query<G>(P, b, kvh, N, sm.qret());
  }

  // Total mass T_h = sum over the group's chunks of L_c exp(hi_c - hi), for the G heads,
  // from the chunk statistics of phase S (double, fixed order: every CTA gets the same value)
  // -> sm.tot[h] (as a double in units of the head's max-score token).
  __device__ void group_total(int g, const float* hi, double* tot) {
    if (sm.ints()[34] == g) return;          // still in sm.tmp() from this group's phase H
    const int n = nch(g);
    double* part = reinterpret_cast<double*>(sm.stage());      // [kFThreads]
    const int t = threadIdx.x;
    const int h = t % G;
    double acc = 0.0;
    for (int c = t / G; c < n; c += kFThreads / G) {
      const float2 st = __ldcg(P.cstat + ((int64_t)g * P.max_nch + c) * G + h);
      acc += (double)st.y * (double)exp2f((st.x - hi[h]) * kLog2e);
    }
    __syncthreads();
    part[t] = acc;
    __syncthreads();
    if (t < G) {
      double v = 0.0;
      for (int i = t; i < kFThreads; i += G) v += part[i];
      tot[t] = v;
    }
    if (t == 0) sm.ints()[34] = g;
    __syncthreads();
  }

  // ------------------------------------------------------------ phase H
  // Masses are exp(s - max) in 2^-40 fixed point. Only bins at or above a cutoff bin get
  // per-bin sums: with T the group's total mass (from phase S), every token below bin(c),
  // c = hi + ln((1 - p) T' / N) and T' = T (1 - 1e-3), has mass below (1 - p) T' / N, so
  // together they hold less than (1 - p) of the total, C_bin(c) > p T and b* can not fall
  // under the cutoff bin (the 1e-3 absorbs the rounding of T, the log and the bin edges). The per-bin sums use two 32-bit shared atomics per token: the low-word add
  // returns the old value and its carry goes to the high word (exact). Lanes take interleaved
  // (token, head) elements and the heads' rows are padded, so a warp's atomics spread over
  // the banks.
  __device__ void phase_hist(int k) {
    const int g = group_of(k), j = k - sm.cbase()[g];
    const int N = gN(g);
    const int n0 = j * C, n1 = min(N, n0 + C);
    uint32_t* hlo = reinterpret_cast<uint32_t*>(sm.hist());
    uint32_t* hhi = hlo + G * kHistStride;
    for (int i = threadIdx.x; i < 2 * G * kHistStride; i += kFThreads) hlo[i] = 0u;
    float lo[G], hi[G], inv[G];
    load_range<G>(P, g, lo, hi, inv);
    double* tot = reinterpret_cast<double*>(sm.tmp());          // [G]
    group_total(g, hi, tot);
    trace(kEvH0);
    const int h = threadIdx.x % G;          // G divides kFThreads: the thread's head is fixed
    float loh = 0.f, hih = 0.f, invh = 0.f;
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
      if (hh == h) { loh = lo[hh]; hih = hi[hh]; invh = inv[hh]; }
    int bch = 0;
    if (P.p < 1.0 && invh > 0.f) {
      const float arg = (float)((1.0 - P.p) * tot[h] * (1.0 - 1e-3) / (double)N);
      const float c = hih + logf(arg);
      bch = c > loh ? bin_of(c, loh, invh) : 0;
    }
    const float* sc = score_ptr(g, j);
    const int64_t hs = score_hstride();
    const int len = n1 - n0;
#pragma unroll 4
    for (int e = threadIdx.x; e < len * G; e += kFThreads) {
      const int nl = e / G;
      const float sv = sc[h * hs + nl];
      const int b = bin_of(sv, loh, invh);
      if (b >= bch) {
        const float ex = (sv - hih) * kLog2e;
        if (ex > -42.f) {                     // below 2^-41 the fixed-point mass rounds to 0
          const unsigned long long q = __float2ull_rn(exp2f(ex) * kMassScale);
          const int bi = h * kHistStride + b;
          const uint32_t ql = (uint32_t)q, qh = (uint32_t)(q >> 32);
          const uint32_t old = atomicAdd(&hlo[bi], ql);
          const uint32_t up = qh + ((old + ql < old) ? 1u : 0u);
          if (up) atomicAdd(&hhi[bi], up);
        }
      }
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
    trace(kEvH2);
    arrive(P.bar + (int64_t)g * 4 + 1);
  }

  // b* of the G heads of group g into sm.ints()[40 + h]; warp h handles head h.
  __device__ void find_bstar(int g, const float* hi) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    double* tot = reinterpret_cast<double*>(sm.tmp());
    if (!P.select_all) group_total(g, hi, tot);
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
        const double thr = P.p * tot[h] * (double)kMassScale;
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

  // ------------------------------------------------------------ phase T
  // Tiles of kFThreads * kTRun tokens; in a tile each thread owns a run of consecutive
  // tokens: masks in registers, one block-wide scan of the per-thread counts, then each
  // thread writes its run's entries. The run length is odd, so the 32 lanes of a warp, which
  // read scores one run apart, hit 32 different banks.
  static constexpr int kTRun = 32;
  __device__ void phase_select(int k) {
    const int g = group_of(k), j = k - sm.cbase()[g];
    const int N = gN(g);
    const int n0 = j * C, n1 = min(N, n0 + C);
    float lo[G], hi[G], inv[G];
    load_range<G>(P, g, lo, hi, inv);
    find_bstar(g, hi);
    trace(kEvT0);
    int bs[G];
#pragma unroll
    for (int h = 0; h < G; ++h) bs[h] = sm.ints()[40 + h];
    const float* sc = score_ptr(g, j);
    const int64_t hs = score_hstride();
    uint32_t* ent = P.ent + (int64_t)g * P.maxN_pad + n0;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int hc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) hc[h] = 0;
    int base = 0;
    uint8_t* mk = sm.stage();                  // per-token head masks of the current tile
#pragma unroll 1
    for (int tb = 0; tb < n1 - n0; tb += kFThreads * kTRun) {
      const int len = min(kFThreads * kTRun, n1 - n0 - tb);
      const int per = ((len + kFThreads - 1) / kFThreads) | 1;
      const int t0 = threadIdx.x * per, t1 = min(len, t0 + per);
      int cnt = 0;
#pragma unroll 1
      for (int nl = t0; nl < t1; ++nl) {
        uint32_t mask = 0;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float sv = sc[h * hs + tb + nl];
          if (bin_of(sv, lo[h], inv[h]) >= bs[h]) { mask |= 1u << h; hc[h]++; }
        }
        mk[nl] = (uint8_t)mask;
        cnt += mask != 0;
      }
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      __syncthreads();
      if (lane == 31) sm.ints()[warp] = incl;
      __syncthreads();
      int before = 0, total = 0;
      for (int w = 0; w < kFThreads / 32; ++w) {
        const int x = sm.ints()[w];
        before += (w < warp) ? x : 0;
        total += x;
      }
      int pos = base + before + incl - cnt;
#pragma unroll 1
      for (int nl = t0; nl < t1; ++nl) {
        const uint32_t mask = mk[nl];
        if (mask) ent[pos++] = ((uint32_t)(n0 + tb + nl) << 8) | mask;
      }
      base += total;
      __syncthreads();                       // mk is rewritten by the next tile
    }
    trace(kEvT1);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      int v = hc[h];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      hc[h] = v;
    }
    __syncthreads();
    if (lane == 0) {
#pragma unroll
      for (int h = 0; h < G; ++h) reinterpret_cast<int*>(sm.tmp())[warp * G + h] = hc[h];
    if (threadIdx.x == 0) sm.ints()[34] = -1; // sm.tmp() no longer holds a group total
    }
    __syncthreads();
    if (threadIdx.x < G) {
      int v = 0;
      for (int w = 0; w < kFThreads / 32; ++w) v += reinterpret_cast<int*>(sm.tmp())[w * G + threadIdx.x];
      if (v) atomicAdd(P.hcnt + (int64_t)g * G + threadIdx.x, v);
    }
    if (threadIdx.x == 0) P.ccnt[(int64_t)g * P.max_nch + j] = (uint32_t)base;
    arrive(P.bar + (int64_t)g * 4 + 2);
  }

  // Attention over cnt rows; result in sm.res(). Gather mode (ent != nullptr): row i is entry
  // e0 + i of the group's compacted list (chunk-local runs located through sm.pref() over nch
  // chunks of Cc tokens); contiguous mode: row i is row r0 + i of kb / vb. One instance of
  // the attention loop serves both, which keeps the kernel's code small.
  struct Rows {
    const uint16_t* kb; const uint16_t* vb;   // row 0 of the sequence (gather) or of the range
    const uint32_t* ent; const int* pref; int e0, nch, Cc;
    const uint32_t* sent;                     // the rows' entries staged in shared memory
  };
  __device__ __noinline__ void attend_list(const float* q_s, int cnt, const Rows R) {
    const int hl = threadIdx.x & 15;
    float2 q[G][4];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        q[h][e] = make_float2(q_s[h * kD + hl * 8 + 2 * e], q_s[h * kD + hl * 8 + 2 * e + 1]);
    AttnState<G> st;
    st.init();
    attend_rows<G>(st, q, cnt, [&](int i, const uint16_t*& kp, const uint16_t*& vp, uint32_t& mask) {
      int64_t n = i;
      mask = 0xffu;
      if (R.sent) {
        const uint32_t w = R.sent[i];
        n = w >> 8;
        mask = w & 0xffu;
      } else if (R.ent) {
        const int e = R.e0 + i;
        const int c = upper_index(R.pref, R.nch, e);
        const uint32_t w = __ldcg(R.ent + (int64_t)c * R.Cc + (e - R.pref[c]));
        n = w >> 8;
        mask = w & 0xffu;
      }
      kp = R.kb + n * kD;
      vp = R.vb + n * kD;
    }, sm.stage(), kFThreads);
    attend_merge<G>(st, reinterpret_cast<float*>(sm.stage()), sm.res(), kFThreads);
  }

  __device__ __noinline__ void merge(const float* parts, int n, float* dst, uint16_t* out_rows) {
    // the score buffer is free whenever partials are merged
    merge_partials<G>(parts, n, dst, out_rows, sm.scores(), 4 * G * P.C_cap, kFThreads);
  }

  // ------------------------------------------------------------ phase W
  __device__ void phase_attend(int k) {
    const int g = group_of(k), j = k - sm.cbase()[g];
    const int b = g / P.L.n_ret, r = g % P.L.n_ret, kvh = P.L.ret_kv[r];
    const int N = gN(g);
    const int S = nch(g);
    for (int c = threadIdx.x; c < S; c += kFThreads)
      sm.pref()[c] = (int)__ldcg(P.ccnt + (int64_t)g * P.max_nch + c);
    __syncthreads();
    const int U = block_scan_excl(sm.pref(), S, sm.ints());
    if (threadIdx.x == 0) sm.pref()[S] = U;
    if (!smem_mode) rope_query<G>(P, b, kvh, N, sm.qret());   // else formed in phase S
    __syncthreads();
    const int e0 = (int)(((long long)U * j) / S), e1 = (int)(((long long)U * (j + 1)) / S);
    const int64_t rowbase = (int64_t)r * P.L.T_total + P.cache.seq_off[b];
    const uint32_t* gent = P.ent + (int64_t)g * P.maxN_pad;
    Rows rows{P.cache.k_ret + rowbase * kD, P.cache.v_ret + rowbase * kD, gent, sm.pref(), e0, S, C,
              nullptr};
    // this split's entries in one batch of loads, into the (now free) score buffer
    uint32_t* es = reinterpret_cast<uint32_t*>(sm.scores());
    if (e1 - e0 <= P.C_cap * G) {
      for (int i = threadIdx.x; i < e1 - e0; i += kFThreads) {
        const int e = e0 + i;
        const int c = upper_index(sm.pref(), S, e);
        es[i] = __ldcg(gent + (int64_t)c * C + (e - sm.pref()[c]));
      }
      __syncthreads();
      rows.sent = es;
    }
    trace(kEvW0);
    attend_list(sm.qret(), e1 - e0, rows);
    trace(kEvW1);
    // partial -> workspace; team / group merge by the last arrivals
    const int stride = G * (kD + 2);
    float* mine = P.part + (int64_t)k * stride;
    for (int o = threadIdx.x; o < stride; o += kFThreads) mine[o] = sm.res()[o];
    const int team = j / kTeam, nteams = (S + kTeam - 1) / kTeam;
    const int tcount = min(kTeam, S - team * kTeam);
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      sm.ints()[48] = atomicAdd(P.team_arr + sm.cbase()[g] + team, 1u) == (uint32_t)(tcount - 1);
    }
    __syncthreads();
    trace(kEvW2);
    if (!sm.ints()[48]) return;
    __threadfence();
    uint16_t* orow = P.out + ((int64_t)b * P.L.Hq + kvh * G) * kD;
    const float* tparts = P.part + (int64_t)(sm.cbase()[g] + team * kTeam) * stride;
    if (nteams == 1) {
      merge(tparts, tcount, nullptr, orow);
    } else {
      merge(tparts, tcount, P.tpart + (int64_t)(sm.cbase()[g] + team) * stride, nullptr);
      __syncthreads();
      if (threadIdx.x == 0) {
        __threadfence();
        sm.ints()[49] = atomicAdd(P.bar + (int64_t)g * 4 + 3, 1u) == (uint32_t)(nteams - 1);
      }
      __syncthreads();
      if (!sm.ints()[49]) return;
      __threadfence();
      merge(P.tpart + (int64_t)sm.cbase()[g] * stride, nteams, nullptr, orow);
    }
    if (threadIdx.x < G)
      P.sel_counts[(int64_t)b * P.L.Hq + kvh * G + threadIdx.x] =
          __ldcg(P.hcnt + (int64_t)g * G + threadIdx.x);
    __syncthreads();
  }

  // ------------------------------------------------------------ local items
  // Runs local items from the global queue until it is empty. Thread 0 takes the next index
  // while the current item runs, so the queue costs one atomic round trip in total.
  __device__ void local_items() {
    if (threadIdx.x == 0) sm.ints()[33] = (int)atomicAdd(P.misc + 0, 1u);
    __syncthreads();
    int li = sm.ints()[33];
    while (li < P.n_loc_items) {
      __syncthreads();
      unsigned int next = 0;
      if (threadIdx.x == 0) next = atomicAdd(P.misc + 0, 1u);
      local_item(li);
      if (threadIdx.x == 0) sm.ints()[33] = (int)next;
      __syncthreads();
      li = sm.ints()[33];
    }
  }

  __device__ void local_item(int li) {
    const int lg = li / P.PL, piece = li % P.PL;
    const int b = lg / P.L.n_loc, x = lg % P.L.n_loc, kvh = P.L.loc_kv[x];
    const int N = sm.N()[b];
    if (N == 0) return;                             // invalid sequence: outputs zeroed in plan
    const int nrows_all = min(N, P.L.ring);
    const int r0 = piece * P.RL;
    const int nrows = max(0, min(nrows_all - r0, P.RL));
    if (P.k_new) {
      const int64_t rr = (N - 1) < P.L.sinks ? (N - 1) : P.L.sinks + (N - 1 - P.L.sinks) % P.L.window;
      if (rr >= r0 && rr < r0 + nrows) append_new(b, kvh, N, nullptr);
    }
    rope_query<G>(P, b, kvh, N, sm.qloc());
    __syncthreads();
    const int64_t ring0 = ((int64_t)x * P.L.B + b) * P.L.ring + r0;
    Rows rows{P.cache.k_loc + ring0 * kD, P.cache.v_loc + ring0 * kD, nullptr, nullptr, 0, 0, 0,
              nullptr};
    attend_list(sm.qloc(), nrows, rows);
    const int stride = G * (kD + 2);
    float* mine = P.lpart + (int64_t)li * stride;
    for (int o = threadIdx.x; o < stride; o += kFThreads) mine[o] = sm.res()[o];
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      sm.ints()[50] = atomicAdd(P.loc_arr + lg, 1u) == (uint32_t)(P.PL - 1);
    }
    __syncthreads();
    if (sm.ints()[50]) {
      __threadfence();
      merge(P.lpart + (int64_t)lg * P.PL * stride, P.PL, nullptr,
            P.out + ((int64_t)b * P.L.Hq + kvh * G) * kD);
      if (threadIdx.x < G) P.sel_counts[(int64_t)b * P.L.Hq + kvh * G + threadIdx.x] = nrows_all;
    }
    __syncthreads();
  }

  __device__ void run() {
    trace(kEvStart);
    plan();
    trace(kEvPlan);
    bool ok = true;
    if ((int)blockIdx.x < P_ret) {
      if (smem_mode) {
        // waves: chunk k runs on CTA k mod P_ret in wave k / P_ret, start to finish. A group
        // never has two chunks on one CTA, and a wait only depends on chunks of the same or
        // the next wave held by other CTAs, which finish their current chunk first.
        for (int k = blockIdx.x; ok && k < NC; k += P_ret) {
          const int g = group_of(k);
          phase_score(k);
          trace(kEvScore);
          ok = wait_for(P.bar + (int64_t)g * 4 + 0, (uint32_t)nch(g));
          trace(kEvWait1);
          if (!ok) break;
          phase_hist(k);
          trace(kEvHist);
          ok = wait_for(P.bar + (int64_t)g * 4 + 1, (uint32_t)nch(g));
          trace(kEvWait2);
          if (!ok) break;
          phase_select(k);
          trace(kEvSelect);
          ok = wait_for(P.bar + (int64_t)g * 4 + 2, (uint32_t)nch(g));
          trace(kEvWait3);
          if (!ok) break;
          phase_attend(k);
          trace(kEvAttend);
        }
      } else {
        // scores in the workspace: phase-major over this CTA's chunks, so no wait ever
        // depends on a later phase
        for (int k = blockIdx.x; k < NC; k += P_ret) phase_score(k);
        for (int k = blockIdx.x; ok && k < NC; k += P_ret) {
          const int g = group_of(k);
          ok = wait_for(P.bar + (int64_t)g * 4 + 0, (uint32_t)nch(g));
          if (ok) phase_hist(k);
        }
        for (int k = blockIdx.x; ok && k < NC; k += P_ret) {
          const int g = group_of(k);
          ok = wait_for(P.bar + (int64_t)g * 4 + 1, (uint32_t)nch(g));
          if (ok) phase_select(k);
        }
        for (int k = blockIdx.x; ok && k < NC; k += P_ret) {
          const int g = group_of(k);
          ok = wait_for(P.bar + (int64_t)g * 4 + 2, (uint32_t)nch(g));
          if (ok) phase_attend(k);
        }
      }
    }
    if (!ok) return;
    local_items();
    trace(kEvLocal);
    trace(kEvEnd);
  }
};

template <int G>
__global__ void __launch_bounds__(kFThreads, 1) decode_kernel(const __grid_constant__ DecodeParams P) {
  DecodeCta<G> cta(P);
  cta.run();
}

// ------------------------------------------------------------------------------ sel_idx
// Debug output: ascending positions each query head attended to. One CTA per (b, h).
template <int G>
__global__ void __launch_bounds__(kThreads) emit_sel_kernel(DecodeParams P, int32_t* sel_idx,
                                                            int64_t sel_stride) {
  const int b = blockIdx.x / P.L.Hq, h = blockIdx.x % P.L.Hq;
  const int kvh = h / G, jh = h % G;
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
  const int g = b * P.L.n_ret + slot;
  const int C = (int)__ldcg(P.misc + 2);
  const int nchg = (N + C - 1) / C;
  const uint32_t* ent = P.ent + (int64_t)g * P.maxN_pad;
  int base = 0;
  for (int c = 0; c < nchg; ++c) {
    const int cnt = (int)__ldcg(P.ccnt + (int64_t)g * P.max_nch + c);
    for (int k0 = 0; k0 < cnt; k0 += kThreads) {
      const int k = k0 + threadIdx.x;
      uint32_t w = 0;
      bool keep = false;
      if (k < cnt) { w = __ldcg(ent + (int64_t)c * C + k); keep = (w >> jh) & 1u; }
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
