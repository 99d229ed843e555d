/*
 * rtp.h -- C ABI of the RTPurbo per-layer decode-step and prefill attention library
 * (librtp.so, sm_100a).
 *
 * What the library computes (sources named by page and section):
 *   "Full Attention Strikes Back: Transferring Full Attention into Sparse within Hundred
 *   Training Steps" (paper text), §3.2: local heads attend over attention sinks plus a sliding
 *   window; retrieval heads score every cached token with the low-rank pre-RoPE index
 *   score of eq. (4), s(m,n) = (W^Q q^pre_m)^T (W^K k^pre_n) with r = 16, keep the token set
 *   S = Top-P(s, p) of eq. (5), and run exact softmax attention over S with the full-dimension
 *   RoPE'd q and k of eq. (1). MCISLAB DeepRead notes on RTPurbo, "Method": p = 0.9, and the
 *   selection is sort-free through a 256-bin, 1 KB-per-head histogram fused with scoring.
 *
 * Conventions for every entry point:
 *   - Pointers are DEVICE pointers unless marked "host". bf16 tensors are passed as their
 *     16-bit patterns (uint16_t). All layouts are dense, row-major, innermost index last.
 *   - The caller owns every buffer. The library never allocates or frees memory, never
 *     synchronises the device and never copies between host and device, except where an
 *     entry point says so (rtp_read_device_status).
 *   - Work is enqueued on the caller's CUDA stream (a cudaStream_t passed as rtp_stream_t;
 *     NULL is the legacy default stream).
 *   - Return values: RTP_OK or a negative RTP_E* code. On a host-side error nothing is
 *     enqueued. Errors found on the device (a sequence length outside its capacity) skip the
 *     offending sequence and set a sticky status word in the workspace; read it with
 *     rtp_read_device_status.
 *   - head_dim must be 128 and idx_dim 16; G = Hq / Hkv must be 1, 2, 4 or 8. Query head h
 *     reads KV head h / G.
 *   - The bf16 row arrays (the caches k_ret, v_ret, idx, k_loc, v_loc; q_pre, k_pre, v,
 *     k_new, v_new and out) are read and written in 16-byte pieces: their device pointers must
 *     be 16-byte aligned (RTP_EINVAL otherwise, before anything is enqueued).
 *
 * Also: the causal prefill of a prompt (rtp_prefill, same paper §3.2: dense for retrieval heads,
 * sinks + window for local heads) on the fifth-generation tensor cores.
 */
#ifndef RTP_H
#define RTP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* rtp_stream_t;   /* same type as cudaStream_t */

enum {
  RTP_OK = 0,
  RTP_EINVAL = -1,      /* a null or misaligned pointer, or a scalar out of range */
  RTP_ESHAPE = -2,      /* inconsistent or unsupported shape */
  RTP_EWORKSPACE = -3,  /* workspace missing or smaller than rtp_workspace_bytes() */
  RTP_ECUDA = -4,       /* a CUDA launch or API call failed */
  RTP_ETIMEOUT = -5,    /* a device-side wait gave up (status word only) */
  RTP_EDEVICE = -6,     /* the device found bad data, e.g. seq_lens[b] > seq_cap[b] */
  RTP_ECHECK = -7       /* builds with -DRTP_CHECKS only: a gathered row, ring row, list slot or
                           debug-list index fell outside its buffer (status word only; the access
                           was redirected to a valid row that contributes nothing) */
};

/* Per-layer description. Host struct; the library reads it during the call only. */
typedef struct {
  int32_t B;              /* sequences in the batch, >= 1 */
  int32_t Hq;             /* query heads */
  int32_t Hkv;            /* KV heads; Hq % Hkv == 0 */
  int32_t head_dim;       /* 128 */
  int32_t idx_dim;        /* 16, the index projection rank r */
  int32_t sinks;          /* attention-sink tokens of the local heads, >= 0 */
  int32_t window;         /* sliding-window tokens of the local heads, >= 1 (current included) */
  int32_t pad0;
  double rope_base;       /* RoPE base; theta_i = base^(-2i/d) on channel pairs (i, i + d/2) */
  int64_t max_seq_len;    /* upper bound on every seq_lens[b] and start_pos[b] + n_new; sizes
                             grids and the workspace */
  const int32_t* slot_of_kv; /* host [Hkv]: slot >= 0 is the KV head's row block in the
                                retrieval caches; slot < 0 marks a local head whose ring is
                                block (-1 - slot) of the local caches. See rtp_build_slot_map. */
} rtp_layer_desc;

/* The caches of one layer. */
typedef struct {
  uint16_t* k_ret;        /* bf16 [n_ret][T_total][128]: RoPE'd keys of retrieval KV heads */
  uint16_t* v_ret;        /* bf16 [n_ret][T_total][128]: values of retrieval KV heads */
  uint16_t* idx;          /* bf16 [n_ret][T_total][16]: index keys W_kidx^T k_pre */
  uint16_t* k_loc;        /* bf16 [n_loc][B][sinks + window][128]: RoPE'd key ring */
  uint16_t* v_loc;        /* bf16 [n_loc][B][sinks + window][128]: value ring */
  const int64_t* seq_off; /* [B]: first row of sequence b inside T_total */
  const int32_t* seq_cap; /* [B]: rows reserved for sequence b (positions 0..cap-1) */
  int64_t T_total;        /* host: rows per retrieval slot, >= seq_off[b] + seq_cap[b] */
} rtp_cache;
/* Ring layout of a local KV head: position n < sinks lives in row n; position n >= sinks in
 * row sinks + (n - sinks) % window. After appending position N-1, rows 0..min(N, sinks +
 * window)-1 hold exactly the positions a local head attends to. */

/* Static string for a status code. */
const char* rtp_status_str(int status);

/* Builds slot_of_kv (host [Hkv]) from a host retrieval mask (nonzero = retrieval KV head):
 * retrieval heads get slots 0, 1, ... in head order, local heads -1, -2, ... in head order.
 * n_ret / n_loc (host, nullable) receive the counts. */
int rtp_build_slot_map(const uint8_t* ret_mask_host, int32_t Hkv, int32_t* slot_of_kv_host,
                       int32_t* n_ret, int32_t* n_loc);

/* Bytes of workspace rtp_decode_step needs for this description (0 on a bad description). */
size_t rtp_workspace_bytes(const rtp_layer_desc* desc);

/* Clears the workspace's sticky status word. Call once after allocating a workspace. */
int rtp_workspace_init(void* ws, size_t ws_bytes, rtp_stream_t stream);

/*
 * Append step (paper §2.2 eq. (1), §3.2 eq. (4)): writes n_new tokens per sequence at
 * positions start_pos[b] .. start_pos[b] + n_b - 1, where n_b = n_new_b ? n_new_b[b] : n_new.
 *   k_pre, v : bf16 [B][n_new][Hkv][128], pre-RoPE keys and values (rows j >= n_b unused).
 *   w_kidx   : fp32 [Hkv][128][16]; rows of local heads are not read.
 *   start_pos: [B]; n_new_b: [B] or NULL.
 * Retrieval KV heads: k_ret row = bf16(R(pos) k_pre), v_ret row = v, idx row =
 * bf16(W_kidx^T k_pre); RoPE angles and the projection are evaluated in double precision.
 * Local KV heads: the same RoPE'd key and v go to the ring row of pos; tokens that a later
 * token of the same call overwrites are skipped. A token at pos >= seq_cap[b] is not written
 * and sets RTP_EDEVICE in ws's status word (ws may be NULL: then it is only skipped).
 * Usable as a bulk fill (n_new large) and as the decode-step append (n_new = 1).
 */
int rtp_append_kv(const rtp_layer_desc* desc, const rtp_cache* cache, const uint16_t* k_pre,
                  const uint16_t* v, const float* w_kidx, const int32_t* start_pos,
                  const int32_t* n_new_b, int32_t n_new, void* ws, rtp_stream_t stream);

/*
 * Decode step of one layer (paper §3.2 eq. (4)-(5)) at position m = seq_lens[b] - 1, after
 * the current token was appended.
 *   q_pre     : bf16 [B][Hq][128], pre-RoPE queries; the library rotates them by R(m).
 *   w_qidx    : fp32 [Hq][128][16]; rows of local query heads are not read.
 *   seq_lens  : [B], 1 <= seq_lens[b] <= seq_cap[b], and <= max_seq_len.
 *   p         : top-p mass in (0, 1]; p >= 1 selects every token.
 *   out       : bf16 [B][Hq][128] attention output.
 *   sel_counts: [B][Hq]; retrieval heads: |S|; local heads: tokens attended.
 *   sel_idx   : [B][Hq][sel_stride] or NULL; when given, receives the ascending positions a
 *               head attended to (sel_stride >= max_seq_len). Debug / parity output; it costs
 *               extra launches.
 *   ws        : workspace of at least rtp_workspace_bytes(desc) bytes, 256-byte aligned,
 *               initialised once with rtp_workspace_init. Calls that share a workspace
 *               must be stream-ordered.
 * Selection (per retrieval query head): scores s_n of all n < N; lo/hi = min/max s; bin(s) =
 * min(255, floor(256 (s - lo) / (hi - lo))); mass M_b = sum over bin b of exp(s - hi); b* =
 * highest bin whose cumulative mass from the top reaches p of the total; S = tokens with
 * bin >= b*. All tokens are kept when p >= 1 or hi == lo.
 */
int rtp_decode_step(const rtp_layer_desc* desc, const rtp_cache* cache, const uint16_t* q_pre,
                    const float* w_qidx, const int32_t* seq_lens, double p, uint16_t* out,
                    int32_t* sel_counts, int32_t* sel_idx, int64_t sel_stride, void* ws,
                    size_t ws_bytes, rtp_stream_t stream);

/*
 * rtp_append_kv of the decode token (n_new = 1 at position seq_lens[b] - 1) and rtp_decode_step
 * in one launch, with identical results: the caches end up holding the token exactly as
 * rtp_append_kv writes it, and the outputs equal those of the two calls in sequence.
 *   k_new, v_new: bf16 [B][Hkv][128], the decode token's pre-RoPE key and value.
 *   w_kidx      : fp32 [Hkv][128][16] (may be NULL when the layer has no retrieval head).
 * Other arguments as rtp_decode_step. Inside the launch, the CTA whose chunk holds the new
 * row of a retrieval group, and the local item whose ring slice holds it, write the token
 * before reading those rows; every other reader comes after a device-wide arrival. The pages
 * describe the two steps separately; one launch saves the second launch of every layer.
 * Errors as rtp_decode_step; RTP_EINVAL when k_new or v_new is NULL, or w_kidx is NULL in a
 * layer with retrieval heads. An invalid seq_lens[b] skips the sequence (nothing is written).
 */
int rtp_decode_step_append(const rtp_layer_desc* desc, const rtp_cache* cache,
                           const uint16_t* k_new, const uint16_t* v_new, const float* w_kidx,
                           const uint16_t* q_pre, const float* w_qidx, const int32_t* seq_lens,
                           double p, uint16_t* out, int32_t* sel_counts, int32_t* sel_idx,
                           int64_t sel_stride, void* ws, size_t ws_bytes, rtp_stream_t stream);

/*
 * Decode step with a fixed-budget top-k selector in place of top-p (the budget the paper's
 * Table 1 compares top-p against; the same 256-bin histogram, with a count threshold):
 * b* = highest bin whose token count from the top reaches k; S = tokens with bin >= b*, so S
 * holds the k highest scores plus, at most, other tokens of bin b*. All tokens are kept when
 * k >= N or hi == lo. Local heads as in rtp_decode_step.
 *   k: >= 1 (RTP_EINVAL otherwise). Other arguments and errors as rtp_decode_step.
 */
int rtp_decode_step_topk(const rtp_layer_desc* desc, const rtp_cache* cache,
                         const uint16_t* q_pre, const float* w_qidx, const int32_t* seq_lens,
                         int64_t k, uint16_t* out, int32_t* sel_counts, int32_t* sel_idx,
                         int64_t sel_stride, void* ws, size_t ws_bytes, rtp_stream_t stream);

/*
 * Causal prefill of one layer over a prompt at positions 0 .. n_b[b] - 1 (paper §3.2:
 * retrieval heads attend densely in prefill, local heads to the attention sinks plus the
 * sliding window in prefill as in decode). Query row m of head h attends to the positions
 * j <= m (retrieval KV head of h) or to j < sinks and m - window < j <= m (local KV head);
 * keys are R(j) k_pre rounded to bf16 as rtp_append_kv stores them, q = R(m) q_pre in
 * single precision, weights softmax(q . k / sqrt(128)), out = sum of weights times v.
 *   q_pre : bf16 [B][n_max][Hq][128], pre-RoPE queries.
 *   k_pre, v : bf16 [B][n_max][Hkv][128], pre-RoPE keys and values (the same buffers an
 *           rtp_append_kv of the prompt takes; this call does not write the cache).
 *   n_b   : device int32 [B], prompt lengths; clamped to [0, n_max] on the device.
 *   out   : bf16 [B][n_max][Hq][128]; rows m >= n_b[b] are not written.
 *   ws    : at least rtp_prefill_workspace_bytes(desc, n_max) bytes, 256-byte aligned: a
 *           status word (cleared by each call; rtp_read_device_status reads it) and the rotated
 *           keys. A decode workspace reused here needs rtp_workspace_init before the next
 *           decode step.
 * S = Q K^T and P V run on the tensor cores (tcgen05) with fp32 accumulation; the query and
 * the probabilities enter as two bf16 terms each (value and rounded remainder), so the result
 * carries fp32-level error before the bf16 output rounding. A device wait for the tensor cores
 * that runs out (rtp_debug_set_wait_limit) records RTP_ETIMEOUT in the status word and leaves
 * the rows of that CTA unwritten.
 * n_max == 0 does nothing. Errors: RTP_EINVAL (null pointer, n_max < 0), RTP_ESHAPE (bad
 * description, n_max > max_seq_len), RTP_EWORKSPACE, RTP_ECUDA. Two launches (and a 256-byte
 * memset of the status word).
 */
size_t rtp_prefill_workspace_bytes(const rtp_layer_desc* desc, int32_t n_max);
int rtp_prefill(const rtp_layer_desc* desc, const uint16_t* q_pre, const uint16_t* k_pre,
                const uint16_t* v, const int32_t* n_b, int32_t n_max, uint16_t* out, void* ws,
                size_t ws_bytes, rtp_stream_t stream);

/* Size of the library-owned scratch of rtp_decode_step_static (bytes). */
#define RTP_STATIC_SCRATCH_BYTES (16u << 20)

/*
 * rtp_decode_step without a caller-provided workspace, for callers that cannot allocate
 * device memory: an engine whose memory planner has already handed out the whole device
 * pool, code running inside a CUDA-graph replay or a callback where cudaMalloc is not
 * allowed, or a host that links the library without a device allocator of its own. The
 * paper has no counterpart; this is a convenience of the C ABI only.
 *   Same arguments and results as rtp_decode_step, minus sel_idx and the workspace.
 *   Scratch: a fixed RTP_STATIC_SCRATCH_BYTES (16 MiB) buffer inside the library, one per
 *   device, held until the process exits. A description whose rtp_workspace_bytes() exceeds
 *   it returns RTP_EWORKSPACE and launches nothing.
 *   Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *   The first call on a device looks up the buffer's device address (cudaGetSymbolAddress)
 *   and clears its status word with synchronous runtime calls: make that first call before
 *   any stream capture on that device.
 *   All calls on a device share the buffer and it keeps the last call's contents; the call
 *   clears the parts that must start at zero, the status word included. Calls whose work
 *   overlaps on the GPU (different streams, or host threads without ordering) race on it:
 *   order them on one stream.
 *   Device-side status is not reported: neither RTP_EDEVICE (an invalid sequence still
 *   yields zero outputs and counts) nor RTP_ETIMEOUT (a device wait that ran out leaves the
 *   outputs of that call undefined) reaches the caller.
 */
int rtp_decode_step_static(const rtp_layer_desc* desc, const rtp_cache* cache,
                           const uint16_t* q_pre, const float* w_qidx, const int32_t* seq_lens,
                           double p, uint16_t* out, int32_t* sel_counts, rtp_stream_t stream);

/* Synchronises `stream`, returns the workspace's sticky device status (RTP_OK, RTP_EDEVICE or
 * RTP_ETIMEOUT) and clears it. Host-blocking; not for the hot loop. */
int rtp_read_device_status(void* ws, rtp_stream_t stream);

/* Number of kernel launches the last rtp_decode_step / rtp_append_kv call on this thread
 * enqueued (for launch accounting). */
int32_t rtp_last_launch_count(void);

/*
 * Test hooks for the failure paths. The pages describe no failure handling; these exist so
 * the error paths can be exercised without faulting a GPU.
 *   rtp_debug_set_wait_limit: the limit, in SM clock cycles, of every device-side wait of
 *     later decode and prefill launches (0 restores the default of about one second; negative values are
 *     RTP_EINVAL). A wait that runs out records RTP_ETIMEOUT in the workspace status word and
 *     raises an abort flag that ends the launch's other waits; the outputs of that call are
 *     undefined and its workspace must be re-initialised with rtp_workspace_init. Process-wide.
 *   rtp_debug_fail_next_call: the next call of rtp_append_kv, rtp_decode_step,
 *     rtp_decode_step_append, rtp_decode_step_topk, rtp_decode_step_static or rtp_prefill (on
 *     any thread) returns `status` (one
 *     of the negative RTP_E* codes; 0 cancels) before checking its arguments, and enqueues
 *     nothing. Process-wide, consumed by that one call.
 */
int rtp_debug_set_wait_limit(int64_t cycles);
int rtp_debug_fail_next_call(int status);

#ifdef __cplusplus
}
#endif

#endif /* RTP_H */
