// C ABI of librtp: argument checks, host-side planning of grids and workspace, launches.
// The declarations and their contracts are in include/rtp.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <atomic>
#include <mutex>

#include "../../include/rtp.h"
#include "rtp_attr_cache.h"
#include "rtp_decode.cuh"
#include "rtp_prefill.cuh"

using namespace rtp;

namespace {

thread_local int32_t g_launches = 0;

constexpr int kPlanCTAs = 160;      // upper bound on decode CTAs (one per SM; B200 has 148)
constexpr long long kSpinLimitDefault = 2000000000LL;   // ~1 s of SM clock per device wait

// Test hooks (see include/rtp.h): the device-wait limit of later launches, and an error code
// the next entry-point call returns before enqueueing anything.
std::atomic<long long> g_spin_limit{kSpinLimitDefault};
std::atomic<int> g_fail_next{0};

int take_injected() { return g_fail_next.exchange(0); }

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
// 16-byte aligned (or null): the kernels move bf16 rows in 16-byte pieces
inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
inline int align16(int x) { return (x + 15) & ~15; }

struct Plan {
  LayerShape L;
  int C_min, max_nch, NC_max, n_groups, n_lgroups, n_loc_items;
  int64_t cand_stride;
  size_t off_ctrl, ctrl_bytes;
  size_t off_bar, off_locarr, off_misc, off_hist, off_hcnt;
  size_t off_bstar, off_cstat, off_grange, off_sellist, off_part, off_lpart,
      off_trace, total;
};

int check_desc(const rtp_layer_desc* d, LayerShape& L) {
  if (!d || !d->slot_of_kv) return RTP_EINVAL;
  if (d->B < 1 || d->B > 4096 || d->Hkv < 1 || d->Hkv > kMaxHkv || d->Hq < 1) return RTP_ESHAPE;
  if (d->Hq % d->Hkv != 0) return RTP_ESHAPE;
  const int G = d->Hq / d->Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return RTP_ESHAPE;
  if (d->head_dim != kD || d->idx_dim != kR) return RTP_ESHAPE;
  if (d->sinks < 0 || d->window < 1 || d->max_seq_len < 1) return RTP_EINVAL;
  if (d->max_seq_len > (int64_t(1) << 24)) return RTP_ESHAPE;     // gather entries pack n in 24 bits
  if (!(d->rope_base > 0.0)) return RTP_EINVAL;
  memset(&L, 0, sizeof(L));
  L.B = d->B; L.Hq = d->Hq; L.Hkv = d->Hkv; L.G = G;
  L.sinks = d->sinks; L.window = d->window; L.ring = d->sinks + d->window;
  L.maxN = d->max_seq_len; L.rope_base = d->rope_base;
  for (int i = 0; i < kD / 2; ++i) L.theta[i] = std::pow(d->rope_base, -2.0 * i / (double)kD);
  bool seen_r[kMaxHkv] = {false}, seen_l[kMaxHkv] = {false};
  int nr = 0, nl = 0;
  for (int g = 0; g < d->Hkv; ++g) {
    const int s = d->slot_of_kv[g];
    if (s >= 0) {
      if (s >= d->Hkv || seen_r[s]) return RTP_EINVAL;
      seen_r[s] = true; L.ret_kv[s] = (int16_t)g; ++nr;
    } else {
      const int x = -1 - s;
      if (x >= d->Hkv || seen_l[x]) return RTP_EINVAL;
      seen_l[x] = true; L.loc_kv[x] = (int16_t)g; ++nl;
    }
    L.slot[g] = (int16_t)s;
  }
  for (int s = 0; s < nr; ++s) if (!seen_r[s]) return RTP_EINVAL;   // slots must be dense
  for (int x = 0; x < nl; ++x) if (!seen_l[x]) return RTP_EINVAL;
  L.n_ret = nr; L.n_loc = nl;
  return RTP_OK;
}

int make_plan(const rtp_layer_desc* d, Plan& pl) {
  const int rc = check_desc(d, pl.L);
  if (rc != RTP_OK) return rc;
  const LayerShape& L = pl.L;
  const int G = L.G;
  const int64_t maxN = L.maxN;
  pl.n_groups = L.B * L.n_ret;
  pl.n_lgroups = L.B * L.n_loc;
  if (pl.n_groups > 8 * kFThreads) return RTP_ESHAPE;
  // chunks: at least C_min tokens, so a launch has at most kMaxSteps chunks per CTA and a
  // group at most 4096 chunks (the shared-memory prefix of phase W)
  int64_t cmin = (int64_t(pl.n_groups) * maxN + int64_t(kMaxSteps) * kPlanCTAs - 1) /
                 (int64_t(kMaxSteps) * kPlanCTAs);
  cmin = std::max<int64_t>(cmin, 64);
  cmin = std::max<int64_t>(cmin, (maxN + 4095) / 4096);
  cmin = (cmin + 63) / 64 * 64;
  pl.C_min = (int)cmin;
  pl.max_nch = (int)((maxN + cmin - 1) / cmin);
  pl.NC_max = (int)std::min<int64_t>(int64_t(pl.n_groups) * pl.max_nch,
                                     int64_t(kMaxSteps) * kPlanCTAs + pl.n_groups);
  pl.NC_max = std::max(pl.NC_max, 1);
  pl.cand_stride = (maxN + 63) / 64 * 64;
  // local items: at least 64 ring rows each (the split itself depends on the SM count and
  // is made at launch, see local_split)
  const int64_t loc_rows = std::min<int64_t>(maxN, L.ring);
  pl.n_loc_items = (int)(int64_t(pl.n_lgroups) * ((loc_rows + 63) / 64));
  const size_t part_bytes = size_t((8 * G + 15) / 16 * 16 + 2 * G * kD);   // Part<G>::kBytes
  size_t o = 256;                                   // [0, 256): status word
  pl.off_ctrl = o;
  pl.off_bar = o;    o = align256(o + sizeof(uint32_t) * pl.n_groups * 4);
  pl.off_locarr = o; o = align256(o + sizeof(uint32_t) * std::max(pl.n_lgroups, 1));
  pl.off_misc = o;   o = align256(o + sizeof(uint32_t) * 16);
  pl.ctrl_bytes = o - pl.off_ctrl;
  pl.off_hist = o;   o = align256(o + sizeof(unsigned long long) * pl.n_groups * G * kBins * kHistPad);
  pl.off_hcnt = o;   o = align256(o + sizeof(int32_t) * pl.n_groups * G);
  pl.off_bstar = o;  o = align256(o + sizeof(int32_t) * pl.n_groups * G);
  pl.off_cstat = o;  o = align256(o + 16 * size_t(pl.n_groups) * pl.max_nch * G);
  pl.off_grange = o; o = align256(o + 8 * size_t(pl.n_groups) * G);
  pl.off_sellist = o; o = align256(o + sizeof(uint32_t) * size_t(pl.n_groups) * pl.cand_stride);
  pl.off_part = o;   o = align256(o + part_bytes * pl.NC_max);
  pl.off_lpart = o;  o = align256(o + part_bytes * std::max(pl.n_loc_items, 1));
#ifdef RTP_TRACE
  pl.off_trace = o;  o = align256(o + sizeof(unsigned long long) * kPlanCTAs * kTraceEvents);
#else
  pl.off_trace = 0;
#endif
  pl.total = o;
  return RTP_OK;
}

template <class T>
T* at(void* ws, size_t off) { return reinterpret_cast<T*>(static_cast<char*>(ws) + off); }

struct DevInfo {
  int dev = 0, sms = 0, smem_optin = 0;
};

int dev_info(DevInfo& di) {
  static thread_local int cached_dev = -1;
  static thread_local DevInfo cached;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return RTP_ECUDA;
  if (dev != cached_dev) {
    DevInfo x;
    x.dev = dev;
    if (cudaDeviceGetAttribute(&x.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&x.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess)
      return RTP_ECUDA;
    cached = x;
    cached_dev = dev;
  }
  di = cached;
  return RTP_OK;
}

// Ring rows per local item (RL, a multiple of the 16-row tile, at least 64) and items per
// local group (PL): about as many items as CTAs (an item's fixed costs, the query, the merge
// of the warps and of the items, are paid per item, its rows stream at the tile loop's
// rate), but at least 256 rows each; a layer without retrieval heads has only local items,
// so they are cut to about one per CTA.
void local_split(const LayerShape& L, int n_lgroups, int n_ret, int P, int& PL, int& RL) {
  const int64_t rows = std::min<int64_t>(L.maxN, L.ring);
  int64_t pl = n_lgroups > 0 ? (P + n_lgroups - 1) / n_lgroups : 1;
  pl = std::min<int64_t>(pl, (rows + 255) / 256);
  if (n_ret == 0 && n_lgroups > 0) pl = std::max<int64_t>(pl, P / n_lgroups);
  pl = std::max<int64_t>(pl, 1);
  int64_t rl = (rows + pl - 1) / pl;
  rl = std::max<int64_t>(64, (rl + 15) / 16 * 16);
  RL = (int)rl;
  PL = (int)((rows + rl - 1) / rl);
}

// Shared-memory layout of the decode kernel: the staging region (index ring, tiles, merge
// buffers; at its end the per-warp lists and row masks of phase W and the candidate queues of
// phase H), then the small arrays. The kept scores of a CTA's chunks live in tensor memory
// (C_cap rows per CTA). Returns the bytes, or -1 when the staging region would be too small
// for the index ring and the tails.
int smem_layout(DecodeParams& P, const Plan& pl, int smem_optin) {
  const int G = P.L.G;
  int small = 0;
  small += align16(4 * G * kD);                         // q
  small += kQBytes;                                     // query buffer (bf16 hi / lo)
  small += align16(4 * G * kR);                         // qidx
  small += align16(8 * G * kHistStride);                // hist (two 32-bit words per bin)
  small += align16(4 * G * (kD + 2));                   // res
  small += align16(8 * kFThreads);                      // tmp
  small += align16(4 * kIntsWords);                     // ints
  small += align16(4 * P.L.B);                          // N
  small += align16(4 * (pl.n_groups + 1));              // cbase
  small += align16(8 * kMaxSteps * G);                  // tcache
  small += align16(16 * kMaxSteps * G);                 // lcache
  const int budget = smem_optin - 1024;
  const int stage = (budget - small) / 1024 * 1024;
  if (stage < kStageBytes * kSStages + kTailMax) return -1;   // ring + phase H/W tails
  P.C_cap = kTmemColsPerThread / (G == 8 ? 8 : 4) * kSRows;
  int o = 0;
  P.sm_stage = o; o += stage;
  P.free_bytes = o;
  P.sm_q = o;     o += align16(4 * G * kD);
  P.sm_qbuf = o;  o += kQBytes;
  P.sm_qidx = o;  o += align16(4 * G * kR);
  P.sm_hist = o;  o += align16(8 * G * kHistStride);
  P.sm_res = o;   o += align16(4 * G * (kD + 2));
  P.sm_tmp = o;   o += align16(8 * kFThreads);
  P.sm_int = o;   o += align16(4 * kIntsWords);
  P.sm_N = o;     o += align16(4 * P.L.B);
  P.sm_cbase = o; o += align16(4 * (pl.n_groups + 1));
  P.sm_tcache = o; o += align16(8 * kMaxSteps * G);
  P.sm_lcache = o; o += align16(16 * kMaxSteps * G);
  return o;
}

// The shared-memory opt-in of decode_kernel<G> is a per-device function attribute: set it
// once per (device, instance) (rtp_attr_cache.h).
AttrCache<4, 64> g_attr;
AttrCache<1, 64> g_attr_pf;     // prefill_kernel

template <int G>
int ensure_smem_attr(int dev, int smem) {
  constexpr int gi = G == 1 ? 0 : (G == 2 ? 1 : (G == 4 ? 2 : 3));
  const int rc = g_attr.ensure(gi, dev, smem, [](int, int bytes) {
    // the current device is `dev` (the caller's cudaGetDevice)
    return cudaFuncSetAttribute(decode_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                bytes) == cudaSuccess ? 0 : 1;
  });
  return rc == 0 ? RTP_OK : RTP_ECUDA;
}

template <int G>
int launch_decode(DecodeParams& P, const Plan& pl, const DevInfo& di, cudaStream_t st,
                  int32_t* sel_idx, int64_t sel_stride) {
  const int smem = smem_layout(P, pl, di.smem_optin);
  if (smem < 0) return RTP_ESHAPE;
  if (ensure_smem_attr<G>(di.dev, smem) != RTP_OK) return RTP_ECUDA;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_kernel<G>, kFThreads, smem) !=
          cudaSuccess || per_sm < 1)
    return RTP_ECUDA;
  P.P = std::min(di.sms, kPlanCTAs);
  if (pl.n_groups >= kMaxSteps * P.P) return RTP_ESHAPE;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(P.P);
  cfg.blockDim = dim3(kFThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, decode_kernel<G>, P) != cudaSuccess) return RTP_ECUDA;
  int n = 1;
  if (sel_idx) {
    emit_sel_kernel<G><<<P.L.B * P.L.Hq, kFThreads, 0, st>>>(P, sel_idx, sel_stride);
    ++n;
  }
  g_launches += n;
  return cudaGetLastError() == cudaSuccess ? RTP_OK : RTP_ECUDA;
}

// rtp_decode_step, optionally appending the decode token in the same launch (k_new != null)
int decode_impl(const rtp_layer_desc* desc, const rtp_cache* cache, const uint16_t* q_pre,
                const float* w_qidx, const int32_t* seq_lens, double p, uint16_t* out,
                int32_t* sel_counts, int32_t* sel_idx, int64_t sel_stride, void* ws,
                size_t ws_bytes, rtp_stream_t stream, const uint16_t* k_new,
                const uint16_t* v_new, const float* w_kidx, int64_t topk = 0);

}  // namespace

extern "C" {

const char* rtp_status_str(int status) {
  switch (status) {
    case RTP_OK: return "ok";
    case RTP_EINVAL: return "invalid argument (null pointer or scalar out of range)";
    case RTP_ESHAPE: return "unsupported or inconsistent shape";
    case RTP_EWORKSPACE: return "workspace missing or too small";
    case RTP_ECUDA: return "CUDA launch or API call failed";
    case RTP_ETIMEOUT: return "device-side wait timed out";
    case RTP_EDEVICE: return "device found bad data (sequence length or position outside capacity)";
    case RTP_ECHECK: return "bounds check failed on the device (RTP_CHECKS build)";
    default: return "unknown status";
  }
}

int rtp_build_slot_map(const uint8_t* ret_mask_host, int32_t Hkv, int32_t* slot_of_kv_host,
                       int32_t* n_ret, int32_t* n_loc) {
  if (!ret_mask_host || !slot_of_kv_host) return RTP_EINVAL;
  if (Hkv < 1 || Hkv > kMaxHkv) return RTP_ESHAPE;
  int r = 0, l = 0;
  for (int g = 0; g < Hkv; ++g) slot_of_kv_host[g] = ret_mask_host[g] ? r++ : -1 - (l++);
  if (n_ret) *n_ret = r;
  if (n_loc) *n_loc = l;
  return RTP_OK;
}

size_t rtp_workspace_bytes(const rtp_layer_desc* desc) {
  Plan pl;
  if (make_plan(desc, pl) != RTP_OK) return 0;
  return pl.total;
}

int rtp_workspace_init(void* ws, size_t ws_bytes, rtp_stream_t stream) {
  if (!ws || ws_bytes < 256) return RTP_EWORKSPACE;
  return cudaMemsetAsync(ws, 0, 256, (cudaStream_t)stream) == cudaSuccess ? RTP_OK : RTP_ECUDA;
}

int rtp_append_kv(const rtp_layer_desc* desc, const rtp_cache* cache, const uint16_t* k_pre,
                  const uint16_t* v, const float* w_kidx, const int32_t* start_pos,
                  const int32_t* n_new_b, int32_t n_new, void* ws, rtp_stream_t stream) {
  g_launches = 0;
  if (const int inj = take_injected()) return inj;
  LayerShape L;
  const int rc = check_desc(desc, L);
  if (rc != RTP_OK) return rc;
  if (!cache || !k_pre || !v || !start_pos || !cache->seq_off || !cache->seq_cap)
    return RTP_EINVAL;
  if (n_new < 0) return RTP_EINVAL;
  if (n_new == 0) return RTP_OK;
  if (L.n_ret > 0 && (!cache->k_ret || !cache->v_ret || !cache->idx || !w_kidx)) return RTP_EINVAL;
  if (L.n_loc > 0 && (!cache->k_loc || !cache->v_loc)) return RTP_EINVAL;
  if (!al16(k_pre) || !al16(v) || !al16(cache->k_ret) || !al16(cache->v_ret) ||
      !al16(cache->idx) || !al16(cache->k_loc) || !al16(cache->v_loc))
    return RTP_EINVAL;
  if (cache->T_total < 1 && L.n_ret > 0) return RTP_ESHAPE;
  L.T_total = cache->T_total;
  CachePtrs C{cache->k_ret, cache->v_ret, cache->idx, cache->k_loc, cache->v_loc, cache->seq_off,
              cache->seq_cap};
  const dim3 grid((n_new + kAppendTok - 1) / kAppendTok, L.B, L.Hkv);
  if (grid.x > 0x7fffffffu || L.B > 65535) return RTP_ESHAPE;
  append_kernel<<<grid, 128, 0, (cudaStream_t)stream>>>(
      L, C, k_pre, v, w_kidx, start_pos, n_new_b, n_new, ws ? static_cast<int*>(ws) : nullptr);
  g_launches = 1;
  return cudaGetLastError() == cudaSuccess ? RTP_OK : RTP_ECUDA;
}

int rtp_decode_step(const rtp_layer_desc* desc, const rtp_cache* cache, const uint16_t* q_pre,
                    const float* w_qidx, const int32_t* seq_lens, double p, uint16_t* out,
                    int32_t* sel_counts, int32_t* sel_idx, int64_t sel_stride, void* ws,
                    size_t ws_bytes, rtp_stream_t stream) {
  return decode_impl(desc, cache, q_pre, w_qidx, seq_lens, p, out, sel_counts, sel_idx,
                     sel_stride, ws, ws_bytes, stream, nullptr, nullptr, nullptr);
}

int rtp_decode_step_append(const rtp_layer_desc* desc, const rtp_cache* cache,
                           const uint16_t* k_new, const uint16_t* v_new, const float* w_kidx,
                           const uint16_t* q_pre, const float* w_qidx, const int32_t* seq_lens,
                           double p, uint16_t* out, int32_t* sel_counts, int32_t* sel_idx,
                           int64_t sel_stride, void* ws, size_t ws_bytes, rtp_stream_t stream) {
  if (!k_new || !v_new || !desc || !desc->slot_of_kv) return RTP_EINVAL;
  bool any_ret = false;
  for (int g = 0; g < desc->Hkv; ++g) any_ret = any_ret || desc->slot_of_kv[g] >= 0;
  if (any_ret && !w_kidx) return RTP_EINVAL;
  return decode_impl(desc, cache, q_pre, w_qidx, seq_lens, p, out, sel_counts, sel_idx,
                     sel_stride, ws, ws_bytes, stream, k_new, v_new, w_kidx);
}

int rtp_decode_step_topk(const rtp_layer_desc* desc, const rtp_cache* cache,
                         const uint16_t* q_pre, const float* w_qidx, const int32_t* seq_lens,
                         int64_t k, uint16_t* out, int32_t* sel_counts, int32_t* sel_idx,
                         int64_t sel_stride, void* ws, size_t ws_bytes, rtp_stream_t stream) {
  if (k < 1) {
    g_launches = 0;
    if (const int inj = take_injected()) return inj;
    return RTP_EINVAL;
  }
  return decode_impl(desc, cache, q_pre, w_qidx, seq_lens, 0.5, out, sel_counts, sel_idx,
                     sel_stride, ws, ws_bytes, stream, nullptr, nullptr, nullptr, k);
}

}  // extern "C"

namespace {

int decode_impl(const rtp_layer_desc* desc, const rtp_cache* cache, const uint16_t* q_pre,
                const float* w_qidx, const int32_t* seq_lens, double p, uint16_t* out,
                int32_t* sel_counts, int32_t* sel_idx, int64_t sel_stride, void* ws,
                size_t ws_bytes, rtp_stream_t stream, const uint16_t* k_new,
                const uint16_t* v_new, const float* w_kidx, int64_t topk) {
  g_launches = 0;
  if (const int inj = take_injected()) return inj;
  Plan pl;
  const int rc = make_plan(desc, pl);
  if (rc != RTP_OK) return rc;
  const LayerShape& L = pl.L;
  if (!cache || !q_pre || !seq_lens || !out || !sel_counts || !cache->seq_off || !cache->seq_cap)
    return RTP_EINVAL;
  if (!(p > 0.0) || p != p) return RTP_EINVAL;
  if (L.n_ret > 0 && (!cache->k_ret || !cache->v_ret || !cache->idx || !w_qidx)) return RTP_EINVAL;
  if (L.n_loc > 0 && (!cache->k_loc || !cache->v_loc)) return RTP_EINVAL;
  if (L.n_ret > 0 && cache->T_total < 1) return RTP_ESHAPE;
  if (sel_idx && sel_stride < L.maxN) return RTP_EINVAL;
  if (!al16(q_pre) || !al16(out) || !al16(k_new) || !al16(v_new) || !al16(cache->k_ret) ||
      !al16(cache->v_ret) || !al16(cache->idx) || !al16(cache->k_loc) || !al16(cache->v_loc))
    return RTP_EINVAL;
  if (!ws || ws_bytes < pl.total) return RTP_EWORKSPACE;
  if ((reinterpret_cast<uintptr_t>(ws) & 255) != 0) return RTP_EWORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  DevInfo di;
  if (dev_info(di) != RTP_OK) return RTP_ECUDA;
  DecodeParams P;
  memset(&P, 0, sizeof(P));
  P.L = L;
  P.L.T_total = cache->T_total;
  P.C_min = pl.C_min; P.max_nch = pl.max_nch; P.NC_max = pl.NC_max;
  P.n_groups = pl.n_groups; P.n_lgroups = pl.n_lgroups;
  local_split(L, pl.n_lgroups, L.n_ret, std::min(di.sms, kPlanCTAs), P.PL, P.RL);
  P.n_loc_items = pl.n_lgroups * P.PL;          // <= pl.n_loc_items (RL >= 64)
  P.select_all = (topk == 0 && p >= 1.0) ? 1 : 0;
  P.p = p;
  P.topk = topk;
  P.spin_limit = g_spin_limit.load();
  P.cand_stride = pl.cand_stride;
  P.q_pre = q_pre; P.w_qidx = w_qidx; P.seq_lens = seq_lens;
  P.k_new = k_new; P.v_new = v_new; P.w_kidx = w_kidx;
  P.cache = CachePtrs{cache->k_ret, cache->v_ret, cache->idx, cache->k_loc, cache->v_loc,
                      cache->seq_off, cache->seq_cap};
  P.out = out; P.sel_counts = sel_counts;
  P.status = at<int>(ws, 0);
  P.bar = at<uint32_t>(ws, pl.off_bar);
  P.loc_arr = at<uint32_t>(ws, pl.off_locarr);
  P.misc = at<uint32_t>(ws, pl.off_misc);
  P.hist = at<unsigned long long>(ws, pl.off_hist);
  P.hcnt = at<int32_t>(ws, pl.off_hcnt);
  P.bstar = at<int32_t>(ws, pl.off_bstar);
  P.cstat = at<float4>(ws, pl.off_cstat);
  P.grange = at<float2>(ws, pl.off_grange);
  P.sellist = at<uint32_t>(ws, pl.off_sellist);
  P.part = at<unsigned char>(ws, pl.off_part);
  P.lpart = at<unsigned char>(ws, pl.off_lpart);
  P.trace = pl.off_trace ? at<unsigned long long>(ws, pl.off_trace) : nullptr;
  if (cudaMemsetAsync(at<char>(ws, pl.off_ctrl), 0, pl.ctrl_bytes, st) != cudaSuccess)
    return RTP_ECUDA;
  int r;
  switch (L.G) {
    case 1: r = launch_decode<1>(P, pl, di, st, sel_idx, sel_stride); break;
    case 2: r = launch_decode<2>(P, pl, di, st, sel_idx, sel_stride); break;
    case 4: r = launch_decode<4>(P, pl, di, st, sel_idx, sel_stride); break;
    default: r = launch_decode<8>(P, pl, di, st, sel_idx, sel_stride); break;
  }
  return r;
}

}  // namespace

extern "C" {

// Scratch of rtp_decode_step_static: one fixed buffer per device that loads the library,
// held until the process exits. Host code only ever uses its device address, obtained with
// cudaGetSymbolAddress on each device (the symbol itself is a host-side stand-in).
static __device__ __align__(256) unsigned char g_static_scratch[RTP_STATIC_SCRATCH_BYTES];

namespace {
std::mutex g_static_mu;
void* g_static_ptr[64] = {nullptr};

// Device address of g_static_scratch on the current device; the first call on a device looks
// it up and clears the status word (not capturable: it uses synchronous runtime calls).
int static_scratch(void** ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return RTP_ECUDA;
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (!g_static_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return RTP_ECUDA;
    if (cudaMemset(p, 0, 256) != cudaSuccess) return RTP_ECUDA;
    g_static_ptr[dev] = p;
  }
  *ptr = g_static_ptr[dev];
  return RTP_OK;
}
}  // namespace

int rtp_decode_step_static(const rtp_layer_desc* desc, const rtp_cache* cache,
                           const uint16_t* q_pre, const float* w_qidx, const int32_t* seq_lens,
                           double p, uint16_t* out, int32_t* sel_counts, rtp_stream_t stream) {
  g_launches = 0;
  if (const int inj = take_injected()) return inj;
  const size_t need = rtp_workspace_bytes(desc);
  if (need == 0) {
    Plan pl;
    return make_plan(desc, pl);              // the description's own error code
  }
  if (need > (size_t)RTP_STATIC_SCRATCH_BYTES) return RTP_EWORKSPACE;
  void* ws = nullptr;
  const int rc = static_scratch(&ws);
  if (rc != RTP_OK) return rc;
  // the status word is not reported by this entry point; clear what an earlier call left
  if (cudaMemsetAsync(ws, 0, 256, (cudaStream_t)stream) != cudaSuccess) return RTP_ECUDA;
  return rtp_decode_step(desc, cache, q_pre, w_qidx, seq_lens, p, out, sel_counts, nullptr, 0,
                         ws, (size_t)RTP_STATIC_SCRATCH_BYTES, stream);
}

// prefill workspace: the status word (256 bytes), then the rotated keys [B][Hkv][n_max][128]
size_t rtp_prefill_workspace_bytes(const rtp_layer_desc* desc, int32_t n_max) {
  LayerShape L;
  if (check_desc(desc, L) != RTP_OK || n_max < 1 || n_max > desc->max_seq_len) return 0;
  return 256 + align256((size_t)L.B * L.Hkv * (size_t)n_max * kD * sizeof(uint16_t));
}

int rtp_prefill(const rtp_layer_desc* desc, const uint16_t* q_pre, const uint16_t* k_pre,
                const uint16_t* v, const int32_t* n_b, int32_t n_max, uint16_t* out, void* ws,
                size_t ws_bytes, rtp_stream_t stream) {
  g_launches = 0;
  if (const int inj = take_injected()) return inj;
  LayerShape L;
  const int rc = check_desc(desc, L);
  if (rc != RTP_OK) return rc;
  if (!q_pre || !k_pre || !v || !n_b || !out || n_max < 0) return RTP_EINVAL;
  if (!al16(q_pre) || !al16(k_pre) || !al16(v) || !al16(out)) return RTP_EINVAL;
  if (n_max > desc->max_seq_len) return RTP_ESHAPE;
  if (n_max == 0) return RTP_OK;
  if (!ws || ws_bytes < rtp_prefill_workspace_bytes(desc, n_max)) return RTP_EWORKSPACE;
  if ((reinterpret_cast<uintptr_t>(ws) & 255) != 0) return RTP_EWORKSPACE;
  DevInfo di;
  if (dev_info(di) != RTP_OK) return RTP_ECUDA;
  const int rc2 = g_attr_pf.ensure(0, di.dev, kPfSmem, [](int, int bytes) {
    return cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                bytes) == cudaSuccess ? 0 : 1;
  });
  if (rc2 != 0) return RTP_ECUDA;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemsetAsync(ws, 0, 256, st) != cudaSuccess) return RTP_ECUDA;
  uint16_t* k_rope = at<uint16_t>(ws, 256);
  const dim3 g1((n_max + kAppendTok - 1) / kAppendTok, L.B, L.Hkv);
  prefill_rope_keys<<<g1, 128, 0, st>>>(L, k_pre, n_b, n_max, k_rope);
  PrefillParams PP;
  memset(&PP, 0, sizeof(PP));
  PP.L = L;
  PP.q_pre = q_pre; PP.k_rope = k_rope; PP.v = v; PP.n_b = n_b; PP.out = out;
  PP.status = static_cast<int*>(ws);
  PP.spin_limit = g_spin_limit.load();
  PP.n_max = n_max;
  const dim3 g2((n_max + kPfQ - 1) / kPfQ, L.Hq, L.B);
  prefill_kernel<<<g2, kPfThreads, kPfSmem, st>>>(PP);
  g_launches = 2;
  return cudaGetLastError() == cudaSuccess ? RTP_OK : RTP_ECUDA;
}

int rtp_read_device_status(void* ws, rtp_stream_t stream) {
  if (!ws) return RTP_EWORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaStreamSynchronize(st) != cudaSuccess) return RTP_ECUDA;
  int v = 0;
  if (cudaMemcpy(&v, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return RTP_ECUDA;
  if (cudaMemset(ws, 0, sizeof(int)) != cudaSuccess) return RTP_ECUDA;
  return v;
}

int32_t rtp_last_launch_count(void) { return g_launches; }

int rtp_debug_set_wait_limit(int64_t cycles) {
  if (cycles < 0) return RTP_EINVAL;
  g_spin_limit.store(cycles == 0 ? kSpinLimitDefault : (long long)cycles);
  return RTP_OK;
}

int rtp_debug_fail_next_call(int status) {
  if (status > 0 || status < RTP_EDEVICE) return RTP_EINVAL;
  g_fail_next.store(status);
  return RTP_OK;
}

}  // extern "C"
