// C ABI of librtp: argument checks, host-side planning of grids and workspace, launches.
// The declarations and their contracts are in include/rtp.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>

#include "../../include/rtp.h"
#include "rtp_decode.cuh"

using namespace rtp;

namespace {

thread_local int32_t g_launches = 0;

constexpr int kPlanSMs = 148;       // B200 SM count used to size the score chunks
constexpr int kLocRows = 128;       // ring rows per local attention item
constexpr int kMaxChunks = 1024;

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct Plan {
  LayerShape L;
  int C, MC, S, PL, n_groups, n_ret_items, n_loc_items;
  size_t off_ctrl, ctrl_bytes;
  size_t off_lohi, off_hcnt, off_arr_ret, off_arr_loc, off_hist;
  size_t off_scores, off_ent, off_ccnt, off_part_ret, off_part_loc, total;
};

int check_desc(const rtp_layer_desc* d, LayerShape& L) {
  if (!d || !d->slot_of_kv) return RTP_EINVAL;
  if (d->B < 1 || d->Hkv < 1 || d->Hkv > kMaxHkv || d->Hq < 1) return RTP_ESHAPE;
  if (d->Hq % d->Hkv != 0) return RTP_ESHAPE;
  const int G = d->Hq / d->Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return RTP_ESHAPE;
  if (d->head_dim != kD || d->idx_dim != kR) return RTP_ESHAPE;
  if (d->sinks < 0 || d->window < 1 || d->max_seq_len < 1) return RTP_EINVAL;
  if (d->max_seq_len > (int64_t(1) << 24)) return RTP_ESHAPE;     // entries pack n in 24 bits
  if (!(d->rope_base > 0.0)) return RTP_EINVAL;
  memset(&L, 0, sizeof(L));
  L.B = d->B; L.Hq = d->Hq; L.Hkv = d->Hkv; L.G = G;
  L.sinks = d->sinks; L.window = d->window; L.ring = d->sinks + d->window;
  L.maxN = d->max_seq_len; L.rope_base = d->rope_base;
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
  // score chunks: about two per SM over all groups, 1K..64K tokens, <= kMaxChunks per group
  int64_t C = (int64_t(pl.n_groups) * maxN + 2 * kPlanSMs - 1) / (2 * kPlanSMs);
  C = std::max<int64_t>(C, 1024);
  C = std::max<int64_t>(C, (maxN + kMaxChunks - 1) / kMaxChunks);
  C = std::min<int64_t>(C, 65536);
  C = (C + 255) / 256 * 256;
  pl.C = (int)C;
  pl.MC = (int)((maxN + C - 1) / C);
  if (pl.MC > kMaxChunks) return RTP_ESHAPE;
  pl.S = (int)std::min<int64_t>(32, std::max<int64_t>(1, maxN / 2048));
  const int64_t loc_rows = std::min<int64_t>(maxN, L.ring);
  pl.PL = (int)((loc_rows + kLocRows - 1) / kLocRows);
  pl.n_ret_items = pl.n_groups * pl.S;
  pl.n_loc_items = L.B * L.n_loc * pl.PL;
  size_t o = 256;                                   // [0, 256): status word
  pl.off_ctrl = o;
  pl.off_lohi = o; o = align256(o + sizeof(uint32_t) * pl.n_groups * 2 * G);
  pl.off_hcnt = o; o = align256(o + sizeof(int32_t) * pl.n_groups * G);
  pl.off_arr_ret = o; o = align256(o + sizeof(uint32_t) * pl.n_groups);
  pl.off_arr_loc = o; o = align256(o + sizeof(uint32_t) * L.B * L.n_loc);
  pl.off_hist = o; o = align256(o + sizeof(unsigned long long) * pl.n_groups * G * kBins);
  pl.ctrl_bytes = o - pl.off_ctrl;
  const int64_t stride = int64_t(pl.MC) * pl.C;
  pl.off_scores = o; o = align256(o + sizeof(float) * pl.n_groups * G * stride);
  pl.off_ent = o; o = align256(o + sizeof(uint32_t) * pl.n_groups * stride);
  pl.off_ccnt = o; o = align256(o + sizeof(uint32_t) * pl.n_groups * pl.MC);
  pl.off_part_ret = o; o = align256(o + sizeof(float) * pl.n_ret_items * G * (kD + 2));
  pl.off_part_loc = o; o = align256(o + sizeof(float) * pl.n_loc_items * G * (kD + 2));
  pl.total = o;
  return RTP_OK;
}

template <class T>
T* at(void* ws, size_t off) { return reinterpret_cast<T*>(static_cast<char*>(ws) + off); }

template <int G>
int launch_decode(DecodeParams& P, const Plan& pl, cudaStream_t st, int32_t* sel_idx,
                  int64_t sel_stride) {
  int n = 0;
  if (pl.n_groups > 0) {
    const dim3 grid(pl.MC, pl.n_groups);
    score_kernel<G><<<grid, kThreads, 0, st>>>(P); ++n;
    if (!P.select_all) { hist_kernel<G><<<grid, kThreads, 0, st>>>(P); ++n; }
    select_kernel<G><<<grid, kThreads, 0, st>>>(P); ++n;
  }
  const int items = pl.n_ret_items + pl.n_loc_items;
  if (items > 0) {
    const size_t dyn = sizeof(float) * (16 * G * kD + G * (kD + 2));
    static bool attr_set = false;     // per template instance
    if (!attr_set) {
      if (cudaFuncSetAttribute(attend_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)dyn) != cudaSuccess)
        return RTP_ECUDA;
      attr_set = true;
    }
    attend_kernel<G><<<items, kThreads, dyn, st>>>(P); ++n;
  }
  if (sel_idx) {
    emit_sel_kernel<G><<<P.L.B * P.L.Hq, kThreads, 0, st>>>(P, sel_idx, sel_stride); ++n;
  }
  g_launches += n;
  return cudaGetLastError() == cudaSuccess ? RTP_OK : RTP_ECUDA;
}

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
  LayerShape L;
  const int rc = check_desc(desc, L);
  if (rc != RTP_OK) return rc;
  if (!cache || !k_pre || !v || !start_pos || !cache->seq_off || !cache->seq_cap)
    return RTP_EINVAL;
  if (n_new < 0) return RTP_EINVAL;
  if (n_new == 0) return RTP_OK;
  if (L.n_ret > 0 && (!cache->k_ret || !cache->v_ret || !cache->idx || !w_kidx)) return RTP_EINVAL;
  if (L.n_loc > 0 && (!cache->k_loc || !cache->v_loc)) return RTP_EINVAL;
  if (cache->T_total < 1 && L.n_ret > 0) return RTP_ESHAPE;
  L.T_total = cache->T_total;
  CachePtrs C{cache->k_ret, cache->v_ret, cache->idx, cache->k_loc, cache->v_loc, cache->seq_off,
              cache->seq_cap};
  const dim3 grid((n_new + kAppendTok - 1) / kAppendTok, L.B);
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
  g_launches = 0;
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
  if (!ws || ws_bytes < pl.total) return RTP_EWORKSPACE;
  if ((reinterpret_cast<uintptr_t>(ws) & 255) != 0) return RTP_EWORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  DecodeParams P;
  memset(&P, 0, sizeof(P));
  P.L = L;
  P.L.T_total = cache->T_total;
  P.C = pl.C; P.MC = pl.MC; P.S = pl.S; P.RL = kLocRows; P.PL = pl.PL;
  P.n_groups = pl.n_groups; P.n_ret_items = pl.n_ret_items; P.n_loc_items = pl.n_loc_items;
  P.select_all = p >= 1.0 ? 1 : 0;
  P.p = p;
  P.q_pre = q_pre; P.w_qidx = w_qidx; P.seq_lens = seq_lens;
  P.cache = CachePtrs{cache->k_ret, cache->v_ret, cache->idx, cache->k_loc, cache->v_loc,
                      cache->seq_off, cache->seq_cap};
  P.out = out; P.sel_counts = sel_counts;
  P.status = at<int>(ws, 0);
  P.lohi = at<uint32_t>(ws, pl.off_lohi);
  P.hcnt = at<int32_t>(ws, pl.off_hcnt);
  P.arrive_ret = at<uint32_t>(ws, pl.off_arr_ret);
  P.arrive_loc = at<uint32_t>(ws, pl.off_arr_loc);
  P.hist = at<unsigned long long>(ws, pl.off_hist);
  P.scores = at<float>(ws, pl.off_scores);
  P.ent = at<uint32_t>(ws, pl.off_ent);
  P.chunk_cnt = at<uint32_t>(ws, pl.off_ccnt);
  P.part_ret = at<float>(ws, pl.off_part_ret);
  P.part_loc = at<float>(ws, pl.off_part_loc);
  if (cudaMemsetAsync(at<char>(ws, pl.off_ctrl), 0, pl.ctrl_bytes, st) != cudaSuccess)
    return RTP_ECUDA;
  int r;
  switch (L.G) {
    case 1: r = launch_decode<1>(P, pl, st, sel_idx, sel_stride); break;
    case 2: r = launch_decode<2>(P, pl, st, sel_idx, sel_stride); break;
    case 4: r = launch_decode<4>(P, pl, st, sel_idx, sel_stride); break;
    default: r = launch_decode<8>(P, pl, st, sel_idx, sel_stride); break;
  }
  return r;
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

}  // extern "C"
