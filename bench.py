"""Decode-step benchmark of the RTPurbo sparse attention path on B200.

One step = one decode step of every layer of the workload: per layer, the append of the
current token and the decode step, for the whole batch, in one launch (rtp_decode_step_append;
--separate-append: rtp_append_kv with n_new = 1, then rtp_decode_step), replayed from a CUDA
graph. Metric: decode layer-steps/s (a layer-step is one layer over the whole batch), plus the
achieved HBM bandwidth of the algorithmic bytes the step must move.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 4] [--extra 2,3,5]
                  [--impl ours|reference]

The headline line is the 1M-token workload (4); the 32K (2), 128K x 4 (3) and ragged B = 64
(5, at p = 0.8, 0.9 and 0.95) workloads are measured in the same run and reported under
"extra", each with its own roofline and ms_per_step (--extra "" skips them).
With N > 1 (torchrun), every rank runs an independent replica of the workload on its GPU
(no data-path collective); value = layer-steps of all ranks / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode layer-steps/s"
L2_BYTES = 126 * 2 ** 20


# --------------------------------------------------------------------------- helpers (CPU-testable)
def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (identity at world size 1)."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(units_per_rank_step: float, steps: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: units of all ranks over the slowest rank's time."""
    return units_per_rank_step * steps * world / (max_ms / 1e3)


def algorithmic_bytes(w, unions, include_append=True) -> float:
    """Bytes one layer-step must move (caches bf16), summed over the workload's layers.

    Retrieval KV head: the 32-B index row of every cached token plus the 512-B K/V row of every
    token in the union of its query heads' selected sets; local KV head: 512 B per attended
    row; q in and out, 512 B per query head; the append writes 512 B (+32 B index) per KV head;
    W_qidx 8 KB per retrieval query head (and W_kidx 8 KB per retrieval KV head, append).
    ``unions[l][(b, g)]`` = union size of retrieval KV head g of sequence b in layer l.
    """
    ring = w.sinks + w.window
    total = 0.0
    for l in range(w.layers):
        for b in range(w.B):
            N = int(w.seq_lens[b])
            for g in range(w.Hkv):
                if w.ret_mask[l, g]:
                    total += 32 * N + 512 * unions[l][(b, g)]
                    if include_append:
                        total += 512 + 32
                else:
                    total += 512 * min(N, ring)
                    if include_append:
                        total += 512
            total += w.Hq * 512
        n_ret_kv = int(w.ret_mask[l].sum())
        total += 8192 * n_ret_kv * w.G
        if include_append:
            total += 8192 * n_ret_kv
    return total


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.p = None

    def __enter__(self):
        try:
            self.p = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.p = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.p is not None:
            time.sleep(0.25)
            self.p.terminate()
            try:
                self.out, _ = self.p.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.p.kill()

    def summary(self):
        rows = []
        for line in (self.out or "").splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 7:
                continue
            try:
                rows.append((float(f[0]), float(f[1]), f[3:7]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v == "Active"})
        return {"sm_mhz": float(np.median([r[0] for r in rows])), "sm_max_mhz": rows[0][1],
                "reasons": reasons, "samples": len(rows)}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# --------------------------------------------------------------------------- CPU oracle arm
def prepare_oracle_layers(w, layers):
    """Host float64 inputs of whole layer-steps (generation is not part of the timing)."""
    from synth import gen
    out = []
    for l in layers:
        q = gen.bf16_bits_to_f32(w.q_pre_bits(l)).astype(np.float64)
        kp = {(b, g): gen.bf16_bits_to_f32(w.kpre_bits(l, b, g, 0, int(w.seq_lens[b]))).astype(np.float64)
              for b in range(w.B) for g in range(w.Hkv)}
        vv = {(b, g): gen.bf16_bits_to_f32(w.v_bits(l, b, g, 0, int(w.seq_lens[b]))).astype(np.float64)
              for b in range(w.B) for g in range(w.Hkv)}
        out.append((l, q, kp, vv))
    return out


def oracle_layer_steps(w, prepared, budget_s: float, max_steps=None):
    """Times the oracle on whole layer-steps (all heads of all sequences of a layer), cycling
    through the prepared layers until ``budget_s`` seconds are spent (at least one step).
    Returns (layer-steps done, seconds)."""
    from oracle import rtp_oracle as O
    done, spent = 0, 0.0
    while True:
        l, q, kp, vv = prepared[done % len(prepared)]
        t0 = time.perf_counter()
        O.decode_layer(q, w.w_qidx(l), w.w_kidx(l), lambda b, g: kp[(b, g)],
                       lambda b, g: vv[(b, g)], w.ret_mask[l], w.seq_lens, w.p, w.sinks, w.window,
                       w.rope_base)
        spent += time.perf_counter() - t0
        done += 1
        if spent >= budget_s or (max_steps is not None and done >= max_steps):
            return done, spent


def _layer_inputs_f64(w, l, pairs):
    from synth import gen
    q = gen.bf16_bits_to_f32(w.q_pre_bits(l)).astype(np.float64)
    kp = {(b, g): gen.bf16_bits_to_f32(w.kpre_bits(l, b, g, 0, int(w.seq_lens[b]))).astype(np.float64)
          for b, g in pairs}
    vv = {(b, g): gen.bf16_bits_to_f32(w.v_bits(l, b, g, 0, int(w.seq_lens[b]))).astype(np.float64)
          for b, g in pairs}
    return q, kp, vv


def oracle_full_step(w):
    """Times the oracle on one whole step: every layer, every head of every sequence (the
    inputs of each layer generated untimed, layer by layer). Returns (layer-steps, seconds)."""
    from oracle import rtp_oracle as O
    spent = 0.0
    for l in range(w.layers):
        q, kp, vv = _layer_inputs_f64(w, l, [(b, g) for b in range(w.B) for g in range(w.Hkv)])
        t0 = time.perf_counter()
        O.decode_layer(q, w.w_qidx(l), w.w_kidx(l), lambda b, g: kp[(b, g)],
                       lambda b, g: vv[(b, g)], w.ret_mask[l], w.seq_lens, w.p, w.sinks, w.window,
                       w.rope_base)
        spent += time.perf_counter() - t0
        del q, kp, vv
    return w.layers, spent


class OracleGroupSample:
    """Bounded oracle sample for long contexts: the G query heads of one retrieval KV head and
    of one local KV head of sequence 0 (inputs generated once, untimed); a step is scaled from
    their times by the workload's mix of retrieval and local (sequence, KV head) pairs over
    all layers."""

    def __init__(self, w):
        self.w = w
        self.l = next(i for i in range(w.layers) if w.ret_mask[i].any() and not w.ret_mask[i].all())
        self.g_r = int(np.nonzero(w.ret_mask[self.l])[0][0])
        self.g_l = int(np.nonzero(~w.ret_mask[self.l])[0][0])
        self.inputs = {g: _layer_inputs_f64(w, self.l, [(0, g)]) for g in (self.g_r, self.g_l)}
        self.n_ret = int(w.ret_mask.sum()) * w.B
        self.n_loc = int((~w.ret_mask).sum()) * w.B

    def time_groups(self):
        from oracle import rtp_oracle as O
        w, t = self.w, {}
        for g, (q, kp, vv) in self.inputs.items():
            heads = [(0, g * w.G + i) for i in range(w.G)]
            t0 = time.perf_counter()
            O.decode_layer(q, w.w_qidx(self.l), w.w_kidx(self.l), lambda b, gg: kp[(b, gg)],
                           lambda b, gg: vv[(b, gg)], w.ret_mask[self.l], w.seq_lens, w.p,
                           w.sinks, w.window, w.rope_base, heads=heads)
            t[g] = time.perf_counter() - t0
        return t

    def step_seconds(self, t):
        """Seconds of one whole step (all layers) scaled from the two group times."""
        return self.n_ret * t[self.g_r] + self.n_loc * t[self.g_l]

    def describe(self, t):
        w = self.w
        return (f"{w.name}: the {w.G} query heads of retrieval KV head {self.g_r} and of local KV "
                f"head {self.g_l} of layer {self.l}, sequence 0 ({t[self.g_r]:.2f} s, "
                f"{t[self.g_l]:.3f} s of float64 NumPy); a {w.layers}-layer step scaled as "
                f"{self.n_ret} retrieval + {self.n_loc} local (sequence, KV head) pairs")


def oracle_group_sample(w):
    """One timing of OracleGroupSample. Returns (layer-steps/s, seconds spent, description)."""
    smp = OracleGroupSample(w)
    t = smp.time_groups()
    return w.layers / smp.step_seconds(t), sum(t.values()), smp.describe(t)


def oracle_retained_mass(w, p=None, k=None):
    """Retained mass of the selected sets, from the oracle, for every retrieval query head of
    the workload's first layer with two or more retrieval KV heads, sequence 0: the top-p sets
    (p), or the fixed-budget top-k sets (k). Two shares: of the dense softmax weights over all
    cached tokens (full attention; DeepRead "Key Results", "Full Attention Strikes Back"
    §2.3), and of the index-space mass exp(s - max s) the selector works on."""
    from oracle import rtp_oracle as O
    from synth import gen
    layer = next((l for l in range(w.layers) if w.ret_mask[l].sum() >= 2),
                 next(l for l in range(w.layers) if w.ret_mask[l].any()))
    N = int(w.seq_lens[0])
    qb = w.q_pre_bits(layer)
    masses, imass, sizes = [], [], []
    for g in np.nonzero(w.ret_mask[layer])[0]:
        kp = gen.bf16_bits_to_f32(w.kpre_bits(layer, 0, int(g), 0, N)).astype(np.float64)
        kidx = O.index_keys(kp, w.w_kidx(layer)[g])
        for h in range(g * w.G, (g + 1) * w.G):
            q = gen.bf16_bits_to_f32(qb[0, h]).astype(np.float64)
            s = O.index_scores(O.index_query(q, w.w_qidx(layer)[h]), kidx)
            sel = O.topk_histogram(s, k) if k else O.topp_histogram(s, p)
            pos = np.nonzero(sel.mask)[0]
            masses.append(O.full_attention_mass(q, kp, pos, w.rope_base))
            e = np.exp(s - s.max())
            imass.append(float(e[pos].sum() / e.sum()))
            sizes.append(len(pos))
    return {"mean": float(np.mean(masses)), "min": float(np.min(masses)),
            "max": float(np.max(masses)),
            "index_mass": {"mean": float(np.mean(imass)), "min": float(np.min(imass)),
                           "max": float(np.max(imass))},
            "tokens_mean": float(np.mean(sizes)),
            "tokens_total": int(np.sum(sizes)), "heads": len(masses),
            "sample": f"every retrieval query head of layer {layer}, sequence 0, of {w.name} "
                      f"({'top-k k=%d' % k if k else 'top-p p=%g' % p}), float64 oracle"}


def sample_layers(w):
    """A retrieval-head layer and a local-only (or the next) layer: the two kinds of layer-step."""
    ret = [l for l in range(w.layers) if w.ret_mask[l].any()]
    loc = [l for l in range(w.layers) if not w.ret_mask[l].any()]
    pick = ret[:1] + (loc[:1] if loc else [l for l in range(w.layers) if l not in ret[:1]][:1])
    return pick or [0]


def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def run_reference(args, w):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    steps_s = []
    if int(w.seq_lens.max()) > 65536:
        # long contexts: per step, the scaled per-head-group sample (a whole layer-step at 1M
        # is minutes of float64 work and tens of GB of float64 inputs)
        smp = OracleGroupSample(w)
        for i in range(args.warmup + args.steps):
            t = smp.time_groups()
            if i >= args.warmup:
                steps_s.append(smp.step_seconds(t) / w.layers)
        sample = "per step, " + smp.describe(t)
    else:
        prepared = prepare_oracle_layers(w, sample_layers(w))
        for i in range(args.warmup + args.steps):
            n, s = oracle_layer_steps(w, prepared[i % len(prepared):] + prepared[:i % len(prepared)],
                                      0.0, max_steps=1)
            if i >= args.warmup:
                steps_s.append(s / n)
        sample = (f"one whole layer-step (all heads, all sequences) of {w.name} per step, "
                  f"alternating layers {[p[0] for p in prepared]} (one with retrieval heads, one "
                  f"without)")
    v = 1.0 / float(np.mean(steps_s))
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "layer-steps/s",
            "n_gpus": 0, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": float(np.mean(steps_s)) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, None),
            "cpu_baseline": {"value": v, "unit": "layer-steps/s", "cores": cpu_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "layer-steps/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(w, flush):
    return {"workload": w.name, "layers": w.layers, "B": int(w.B), "Hq": w.Hq, "Hkv": w.Hkv,
            "head_dim": 128, "idx_dim": 16, "seq_len": int(w.seq_lens.max()),
            "tokens": int(w.seq_lens.sum()), "retrieval_kv_heads": int(w.ret_mask.sum()),
            "p": w.p, "sinks": w.sinks, "window": w.window, "l2": flush,
            "parallelism": "replicas"}


# --------------------------------------------------------------------------- GPU arm
def _bits_to_dev(bits, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)


# The device sources the decode kernel is compiled from: a recorded ncu traffic figure holds
# while their hash is the one recorded beside it.
DECODE_KERNEL_SOURCES = ("rtp_common.cuh", "rtp_append.cuh", "rtp_attend.cuh", "rtp_score.cuh",
                         "rtp_tmem.cuh", "rtp_decode.cuh")


def _traffic(kernel: str, workload: str):
    """DRAM bytes per launch of ``kernel`` on ``workload`` from a committed ncu summary, if it
    was taken on the current kernel source (the sha256 of its device sources recorded beside
    it); else None."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    src = os.path.join(ROOT, "long_context_sparse_rtpurbo_b200", "csrc")
    h = hashlib.sha256()
    for name in DECODE_KERNEL_SOURCES:
        with open(os.path.join(src, name), "rb") as f:
            h.update(f.read())
    e = d.get(f"{kernel}/{workload}")
    if not e or e.get("source_sha256") != h.hexdigest():
        return None
    return e


class GpuWorkload:
    """Every layer of a workload on one GPU: caches filled by the counter-stream fill kernel
    up to position N - 1, the decode token's k / v and the query packed per layer (the step's
    input), outputs per layer. measure(p) times one step per CUDA-graph replay."""

    def __init__(self, w, dev, fused):
        import torch
        from long_context_sparse_rtpurbo_b200.layer import DecodeLayer
        from synth.gpu import LayerFiller
        self.w, self.dev, self.fused = w, dev, fused
        N = np.asarray(w.seq_lens, np.int64)
        self.N = N
        B, Hq, Hkv, Lyr = w.B, w.Hq, w.Hkv, w.layers
        nq, nk = B * Hq * 128, B * Hkv * 128
        per_layer_in = nq + 2 * nk
        self.inp = torch.empty(Lyr * per_layer_in, dtype=torch.bfloat16, device=dev)
        self.out_all = torch.empty((Lyr, B, Hq, 128), dtype=torch.bfloat16, device=dev)
        self.cnt_all = torch.empty((Lyr, B, Hq), dtype=torch.int32, device=dev)
        self.layers = []
        t_fill = time.perf_counter()
        chunk = max(1024, min(16384, (1 << 27) // max(1, B * Hkv * 128 * 2)))
        for l in range(Lyr):
            lay = DecodeLayer(B, Hq, Hkv, w.sinks, w.window, int(N.max()), w.ret_mask[l], N, dev,
                              w.rope_base)
            wq = torch.from_numpy(np.array(w.w_qidx(l))).to(dev)
            wk = torch.from_numpy(np.array(w.w_kidx(l))).to(dev)
            filler = LayerFiller(w, l, dev)
            top = int(N.max()) - 1
            for t0 in range(0, top, chunk):
                n = min(chunk, top - t0)
                nv = np.clip(N - 1 - t0, 0, n).astype(np.int32)
                k, v = filler.fill(np.full(B, t0), n, nv)
                lay.append(k, v, wk, torch.full((B,), t0, dtype=torch.int32, device=dev),
                           torch.from_numpy(nv).to(dev))
            base = l * per_layer_in
            q = self.inp[base:base + nq].view(B, Hq, 128)
            knew = self.inp[base + nq:base + nq + nk].view(B, 1, Hkv, 128)
            vnew = self.inp[base + nq + nk:base + per_layer_in].view(B, 1, Hkv, 128)
            q.copy_(_bits_to_dev(w.q_pre_bits(l), dev))
            kk, vv = filler.fill(N - 1, 1)
            knew.copy_(kk)
            vnew.copy_(vv)
            self.layers.append(dict(lay=lay, q=q, wq=wq, wk=wk, knew=knew, vnew=vnew,
                                    start=torch.tensor(N - 1, dtype=torch.int32, device=dev),
                                    seq=torch.tensor(N, dtype=torch.int32, device=dev),
                                    out=self.out_all[l], cnt=self.cnt_all[l]))
            del filler
        torch.cuda.synchronize()
        self.setup_s = time.perf_counter() - t_fill

    def step(self, p, with_append=True, launches=None, topk=0):
        from long_context_sparse_rtpurbo_b200 import rtp
        w = self.w
        B, Hkv = w.B, w.Hkv
        for L in self.layers:
            if topk:                           # fixed-budget top-k: append, then decode
                if with_append:
                    L["lay"].append(L["knew"], L["vnew"], L["wk"], L["start"])
                    if launches is not None:
                        launches[0] += rtp.rtp_last_launch_count()
                L["lay"].decode_topk(L["q"], L["wq"], L["seq"], topk, L["out"], L["cnt"])
                if launches is not None:
                    launches[0] += rtp.rtp_last_launch_count()
                continue
            if with_append and self.fused:     # append + decode in one launch
                L["lay"].decode_append(L["knew"].view(B, Hkv, 128), L["vnew"].view(B, Hkv, 128),
                                       L["wk"], L["q"], L["wq"], L["seq"], p, L["out"], L["cnt"])
                if launches is not None:
                    launches[0] += rtp.rtp_last_launch_count()
                continue
            if with_append:
                L["lay"].append(L["knew"], L["vnew"], L["wk"], L["start"])
                if launches is not None:
                    launches[0] += rtp.rtp_last_launch_count()
            L["lay"].decode(L["q"], L["wq"], L["seq"], p, L["out"], L["cnt"])
            if launches is not None:
                launches[0] += rtp.rtp_last_launch_count()

    def selections(self, p, topk=0):
        """Union sizes of the selected sets per retrieval (sequence, KV head) and the
        per-head counts (untimed, through sel_idx), for the algorithmic byte count."""
        import torch
        w, N, dev = self.w, self.N, self.dev
        B, Hq, Hkv = w.B, w.Hq, w.Hkv
        unions, conc, diff, allc = [], [], [], []
        for l, L in enumerate(self.layers):
            u = {}
            if w.ret_mask[l].any():
                sel = torch.full((B, Hq, int(N.max())), -1, dtype=torch.int32, device=dev)
                cnt = torch.empty((B, Hq), dtype=torch.int32, device=dev)
                out = torch.empty((B, Hq, 128), dtype=torch.bfloat16, device=dev)
                if topk:
                    L["lay"].decode_topk(L["q"], L["wq"], L["seq"], topk, out, cnt, sel)
                else:
                    L["lay"].decode(L["q"], L["wq"], L["seq"], p, out, cnt, sel)
                c = cnt.cpu().numpy()
                for b in range(B):
                    for g in range(Hkv):
                        if not w.ret_mask[l, g]:
                            continue
                        hs = range(g * w.G, (g + 1) * w.G)
                        parts = [sel[b, h, :int(c[b, h])] for h in hs]
                        u[(b, g)] = int(torch.unique(torch.cat(parts)).numel())
                        for h in hs:
                            kind = w.group_layout(l, b, g).targets[h % w.G][0]
                            (conc if kind == "conc" else diff).append(int(c[b, h]))
                            allc.append(int(c[b, h]))
                del sel
            unions.append(u)
            st = L["lay"].status()
            if st != 0:
                raise RuntimeError(f"device status {st} in layer {l}")
        return unions, conc, diff, allc

    def measure(self, p, args, world, e2e=False, topk=0):
        import torch
        import torch.distributed as dist
        w, dev = self.w, self.dev
        fused = self.fused and not topk        # the top-k entry point has no fused append
        Lyr = w.layers
        launches = [0]
        self.step(p, launches=launches, topk=topk)   # eager (attributes set outside capture)
        per_step_launches = launches[0]
        unions, conc, diff, allc = self.selections(p, topk)
        step_bytes = algorithmic_bytes(w, unions, include_append=True)
        dec_bytes = algorithmic_bytes(w, unions, include_append=False)
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self.step(p, topk=topk)
            g_full = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_full, stream=side):
                self.step(p, topk=topk)
            g_dec = torch.cuda.CUDAGraph()                  # the decode kernel alone
            with torch.cuda.graph(g_dec, stream=side):
                self.step(p, with_append=fused, topk=topk)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()

        def barrier():
            if world > 1:
                dist.barrier()

        def timed(fn, k):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            barrier()
            torch.cuda.synchronize()
            e0.record()
            for _ in range(k):
                fn()
            e1.record()
            torch.cuda.synchronize()
            barrier()
            return e0.elapsed_time(e1)

        for _ in range(args.warmup):
            g_full.replay()
        torch.cuda.synchronize()
        local = dev.index if dev.index is not None else 0
        with ClockSampler(local) as clk:
            t_end = time.perf_counter() + args.preroll      # untimed pre-roll under load
            while time.perf_counter() < t_end:
                g_full.replay()
                torch.cuda.synchronize()
            torch.cuda.nvtx.range_push("rtp_timed")
            ms = timed(g_full.replay, args.steps)
            torch.cuda.nvtx.range_pop()
            dec_ms = timed(g_dec.replay, args.steps)
        clocks = clk.summary()
        ms_step = max_over_ranks(ms / args.steps, world, dev)
        dec_step = max_over_ranks(dec_ms / args.steps, world, dev)
        res = {}
        if e2e:
            # H2D of the step's inputs from pinned memory, the step, D2H of the outputs
            inp_host = self.inp.cpu().pin_memory()
            out_host = torch.empty(self.out_all.shape, dtype=self.out_all.dtype).pin_memory()
            cnt_host = torch.empty(self.cnt_all.shape, dtype=self.cnt_all.dtype).pin_memory()

            def e2e_step():
                self.inp.copy_(inp_host, non_blocking=True)
                g_full.replay()
                out_host.copy_(self.out_all, non_blocking=True)
                cnt_host.copy_(self.cnt_all, non_blocking=True)

            for _ in range(max(3, args.warmup)):
                e2e_step()
            e2e_ms = max_over_ranks(timed(e2e_step, args.steps) / args.steps, world, dev)
            h2d = self.inp.numel() * self.inp.element_size()
            d2h = (self.out_all.numel() * self.out_all.element_size() +
                   self.cnt_all.numel() * self.cnt_all.element_size())
            res["e2e"] = {"value": aggregate(Lyr, 1, world, e2e_ms), "unit": "layer-steps/s",
                          "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                          "ms_per_step": e2e_ms}
        del g_full, g_dec
        peak, peak_kind = load_peaks()
        kern_bytes = step_bytes if fused else dec_bytes   # the fused kernel also appends
        achieved = kern_bytes / (dec_step * 1e-3) / 1e9
        tr = _traffic("rtp_decode_step", w.name)
        N = self.N
        attended = float(sum(allc)) + sum(min(int(n), w.sinks + w.window) * w.G
                                          for l in range(Lyr) for n in N
                                          for g in range(w.Hkv) if not w.ret_mask[l, g])
        scored = float(sum(int(n) * w.G for l in range(Lyr) for n in N
                           for g in range(w.Hkv) if w.ret_mask[l, g]))
        res.update({
            "value": aggregate(Lyr, 1, world, ms_step), "unit": "layer-steps/s",
            "ms_per_step": ms_step, "p": None if topk else p, "topk": topk or None,
            "config": workload_config(w, "inputs larger than L2 (%.2f GB read per step vs "
                                         "126 MB L2)" % (step_bytes / 1e9)),
            "achieved_step_gbs": step_bytes / (ms_step * 1e-3) / 1e9,
            "step_bytes": step_bytes,
            "token_heads_per_s": {"attended": attended * world / (ms_step * 1e-3),
                                  "scored": scored * world / (ms_step * 1e-3)},
            "roofline": {"kernel": "rtp_decode_step", "bound": "hbm", "achieved": achieved,
                         "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                         "peak_kind": peak_kind + " hbm_gbs (copy bandwidth, burst)",
                         "traffic": None if tr is None else tr["dram_bytes_per_launch"],
                         "bytes_per_launch": kern_bytes / Lyr,
                         "launch_us": dec_step * 1e3 / Lyr, "fused_append": fused,
                         "frac_of_nominal_8tbs": achieved / 8000.0},
            "gpu_launches": per_step_launches * args.steps,
            "clocks": clocks,
            "selected_tokens": {"concentrated_mean": float(np.mean(conc)) if conc else None,
                                "diffuse_mean": float(np.mean(diff)) if diff else None,
                                "min": int(min(allc)) if allc else None,
                                "max": int(max(allc)) if allc else None,
                                "union_mean": float(np.mean([x for u in unions for x in u.values()]))
                                if allc else None},
            "setup_s": self.setup_s,
        })
        return res

    def close(self):
        import torch
        del self.layers, self.inp, self.out_all, self.cnt_all
        torch.cuda.empty_cache()


def load_tensor_peak():
    """Dense bf16 tensor-core peak (TFLOP/s): the sustained cuBLAS figure (a prefill step runs
    for a fraction of a second under the power cap)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["bf16_tflops_sustained"]), "measured bf16_tflops_sustained"
    return 1400.0, "fallback (sustained)"


def prefill_flops(w, n):
    """Algorithmic FLOPs of the attention of a prefill of n tokens over every layer: 4 * 128
    per (query head, row m, attended key), attended = m + 1 for a retrieval head and
    min(m + 1, sinks + window) for a local one."""
    m = np.arange(n, dtype=np.float64)
    dense = float((m + 1).sum())
    local = float(np.minimum(m + 1, w.sinks + w.window).sum())
    per = [(dense if w.ret_mask[l, g] else local) * w.G for l in range(w.layers)
           for g in range(w.Hkv)]
    return 4.0 * 128 * float(sum(per)) * w.B


class PrefillWorkload:
    """A causal prefill of an n-token prompt through every layer of a workload's head layout:
    per layer rtp_append_kv of the prompt into that layer's caches, then rtp_prefill (the
    RoPE'd-key pre-pass and the attention). One prompt (the layer-0 streams: q_pre from the
    prompt-query streams at scale 2, k_pre and v from the fill kernel) feeds every layer."""

    def __init__(self, w, n, dev):
        import torch
        from long_context_sparse_rtpurbo_b200 import rtp
        from long_context_sparse_rtpurbo_b200.layer import DecodeLayer
        from synth.gpu import LayerFiller
        self.w, self.n, self.dev = w, n, dev
        t0 = time.perf_counter()
        B, Hq, Hkv = w.B, w.Hq, w.Hkv
        qb = np.zeros((B, n, Hq, 128), np.uint16)
        for b in range(B):
            for h in range(Hq):
                qb[b, :, h] = w.prompt_q_bits(0, b, h, 0, n, 2.0)
        self.q = _bits_to_dev(qb, dev)
        del qb
        self.k, self.v = LayerFiller(w, 0, dev).fill(np.zeros(B, np.int64), n)
        self.out = torch.empty((B, n, Hq, 128), dtype=torch.bfloat16, device=dev)
        self.nb = torch.full((B,), n, dtype=torch.int32, device=dev)
        self.start = torch.zeros(B, dtype=torch.int32, device=dev)
        caps = np.full(B, n, np.int64)
        self.layers = []
        for l in range(w.layers):
            lay = DecodeLayer(B, Hq, Hkv, w.sinks, w.window, n, w.ret_mask[l], caps, dev,
                              w.rope_base)
            wk = torch.from_numpy(np.array(w.w_kidx(l), np.float32)).to(dev)
            self.layers.append((lay, wk))
        need = rtp.rtp_prefill_workspace_bytes(self.layers[0][0].desc, n)
        self.ws = torch.empty(need, dtype=torch.uint8, device=dev)
        torch.cuda.synchronize()
        self.setup_s = time.perf_counter() - t0

    def step(self, attention_only=False):
        from long_context_sparse_rtpurbo_b200 import rtp
        for lay, wk in self.layers:
            if not attention_only:
                rtp.rtp_append_kv(lay.desc, lay.cache, self.k, self.v, wk, self.start, self.nb,
                                  self.n, lay.ws)
            rtp.rtp_prefill(lay.desc, self.q, self.k, self.v, self.nb, self.n, self.out,
                            self.ws, self.ws.numel())

    def measure(self, args, world):
        import torch
        from long_context_sparse_rtpurbo_b200 import rtp
        w, n, dev = self.w, self.n, self.dev
        self.step()
        per_step_launches = 0
        for lay, wk in self.layers:
            rtp.rtp_append_kv(lay.desc, lay.cache, self.k, self.v, wk, self.start, self.nb, n,
                              lay.ws)
            per_step_launches += rtp.rtp_last_launch_count()
            rtp.rtp_prefill(lay.desc, self.q, self.k, self.v, self.nb, n, self.out, self.ws,
                            self.ws.numel())
            per_step_launches += rtp.rtp_last_launch_count()
        torch.cuda.synchronize()
        assert rtp.rtp_read_device_status(self.ws) == 0

        def timed(fn, k):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            if world > 1:
                torch.distributed.barrier()
            torch.cuda.synchronize()
            e0.record()
            for _ in range(k):
                fn()
            e1.record()
            torch.cuda.synchronize()
            if world > 1:
                torch.distributed.barrier()
            return e0.elapsed_time(e1)

        for _ in range(max(3, args.warmup)):
            self.step()
        steps = max(1, args.prefill_steps)
        local = dev.index if dev.index is not None else 0
        with ClockSampler(local) as clk:
            ms = timed(self.step, steps) / steps
            attn_ms = timed(lambda: self.step(True), steps) / steps
        ms = max_over_ranks(ms, world, dev)
        attn_ms = max_over_ranks(attn_ms, world, dev)
        flops = prefill_flops(w, n)
        peak, peak_kind = load_tensor_peak()
        achieved = flops / (attn_ms * 1e-3) / 1e12
        tokens = float(n * w.B)
        return {
            "metric": "prefill tokens/s", "value": tokens * world / (ms * 1e-3),
            "unit": "tokens/s", "ms_per_step": ms, "higher_is_better": True,
            "config": {"workload": f"qwen3-8b-prefill-{n // 1024}k-b{w.B}", "layers": w.layers,
                       "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "head_dim": 128, "prompt": n,
                       "sinks": w.sinks, "window": w.window,
                       "retrieval_pairs": int(w.ret_mask[:w.layers].sum()),
                       "step": "per layer: rtp_append_kv of the prompt, then rtp_prefill",
                       "flush": "inputs larger than L2 (%.0f MB of q / k / v / out per layer)"
                                % ((self.q.numel() + self.k.numel() + self.v.numel() +
                                    self.out.numel()) * 2 / 1e6)},
            "attention_ms_per_step": attn_ms,
            "roofline": {"kernel": "rtp_prefill", "bound": "tensor", "achieved": achieved,
                         "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                         "peak_kind": peak_kind, "traffic": None,
                         "flops_per_step": flops,
                         "note": "algorithmic FLOPs (4 * 128 per attended query-key pair) over "
                                 "the time of rtp_prefill (RoPE'd-key pre-pass + attention); "
                                 "the kernel issues twice as many tensor-core FLOPs (query and "
                                 "probabilities as two bf16 terms each)"},
            "gpu_launches": per_step_launches * steps,
            "clocks": clk.summary(),
            "setup_s": self.setup_s,
        }

    def close(self):
        import torch
        del self.layers, self.q, self.k, self.v, self.out, self.ws
        torch.cuda.empty_cache()


def oracle_prefill_sample(w, n, n_sample=2048):
    """The CPU oracle on a bounded sample of the prefill: prefill_head of one retrieval and
    one local query head over the first n_sample prompt tokens, scaled to a whole n-token,
    36-layer step by the algorithmic FLOPs of each head kind."""
    from oracle import rtp_oracle as O
    from synth import gen
    l_ret = int(np.nonzero(w.ret_mask.any(axis=1))[0][0])
    g_ret = int(np.nonzero(w.ret_mask[l_ret])[0][0])
    g_loc = int(np.nonzero(~w.ret_mask[l_ret])[0][0])
    f64 = lambda bits: gen.bf16_bits_to_f32(bits).astype(np.float64)
    spent = {}
    for kind, g in (("retrieval", g_ret), ("local", g_loc)):
        q = f64(w.prompt_q_bits(0, 0, g * w.G, 0, n_sample, 2.0))
        k = f64(w.kpre_bits(0, 0, g, 0, n_sample))
        v = f64(w.v_bits(0, 0, g, 0, n_sample))
        t0 = time.perf_counter()
        O.prefill_head(q, k, v, kind == "local", w.sinks, w.window, w.rope_base)
        spent[kind] = time.perf_counter() - t0
    m_s = np.arange(n_sample, dtype=np.float64)
    m_f = np.arange(n, dtype=np.float64)
    cap = w.sinks + w.window
    scale = {"retrieval": (m_f + 1).sum() / (m_s + 1).sum(),
             "local": np.minimum(m_f + 1, cap).sum() / np.minimum(m_s + 1, cap).sum()}
    n_ret = int(w.ret_mask[:w.layers].sum()) * w.G * w.B
    n_loc = int((~w.ret_mask[:w.layers]).sum()) * w.G * w.B
    step_s = (n_ret * spent["retrieval"] * scale["retrieval"] +
              n_loc * spent["local"] * scale["local"])
    return {"value": float(n * w.B / step_s), "unit": "tokens/s", "cores": cpu_threads(),
            "kind": "oracle",
            "sample": f"prefill_head of one retrieval and one local query head over the first "
                      f"{n_sample} prompt tokens ({spent['retrieval'] + spent['local']:.2f} s of "
                      f"float64 NumPy), scaled to {n_ret} retrieval + {n_loc} local query heads "
                      f"of a {n}-token, {w.layers}-layer step by each kind's algorithmic FLOPs"}


def _cpu_baseline(w, budget_s):
    """The oracle on the host cores: whole layer-steps (alternating a layer with retrieval
    heads and one without) up to budget_s seconds, or, for contexts beyond 64K tokens, the
    scaled per-head-group sample."""
    if int(w.seq_lens.max()) > 65536:
        v, spent, desc = oracle_group_sample(w)
        return {"value": v, "unit": "layer-steps/s", "cores": cpu_threads(), "kind": "oracle",
                "sample": desc}
    prepared = prepare_oracle_layers(w, sample_layers(w))
    n_done, spent = oracle_layer_steps(w, prepared, budget_s)
    return {"value": n_done / spent, "unit": "layer-steps/s", "cores": cpu_threads(),
            "kind": "oracle",
            "sample": f"{n_done} whole layer-steps of {w.name} (all heads, alternating layers "
                      f"{[p[0] for p in prepared]}: one with retrieval heads, one without), "
                      f"{spent:.1f} s of float64 NumPy"}


def run_ours(args, w):
    import datetime
    import torch
    import torch.distributed as dist
    from synth import workloads

    rank, world, local = dist_env()
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    fused = not args.separate_append

    gw = GpuWorkload(w, dev, fused)
    m = gw.measure(w.p, args, world, e2e=not args.no_e2e)
    gw.close()
    del gw
    if args.no_e2e:
        m["e2e"] = {"value": float("nan"), "unit": "layer-steps/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0, "ms_per_step": float("nan")}
    line = {"metric": METRIC, "value": m.pop("value"), "unit": m.pop("unit"), "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": m.pop("ms_per_step"),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic"}
    line.update(m)
    extra = {}
    for spec in [x for x in (args.extra or "").split(",") if x.strip()]:
        wi = int(spec)
        if wi == args.workload:
            continue
        we = workloads.workload(wi)
        if args.layers:
            we.layers = min(we.layers, args.layers)
        ps = [0.8, 0.9, 0.95] if wi == 5 else [we.p]
        gw = GpuWorkload(we, dev, fused)
        for p in ps:
            me = gw.measure(p, args, world)
            key = we.name if len(ps) == 1 else f"{we.name}@p={p}"
            extra[key] = me
        if wi == 2 and args.topk > 0:          # the fixed-budget top-k variant at 32K
            extra[f"{we.name}@topk={args.topk}"] = gw.measure(we.p, args, world, topk=args.topk)
        gw.close()
        del gw
    if args.prefill > 0:                       # the causal prefill of a prompt (f1)
        wp = workloads.workload(2)
        if args.layers:
            wp.layers = min(wp.layers, args.layers)
        pw = PrefillWorkload(wp, args.prefill, dev)
        me = pw.measure(args, world)
        pw.close()
        del pw
        if rank == 0 and world == 1 and not args.no_cpu:
            me["cpu_baseline"] = oracle_prefill_sample(wp, args.prefill)
        extra[me["config"]["workload"]] = me
    if extra:
        line["extra"] = extra
    if rank == 0 and world == 1 and not args.no_cpu:
        line["cpu_baseline"] = _cpu_baseline(w, args.cpu_budget)
        for key, me in extra.items():
            if me["config"]["workload"] != "qwen3-8b-32k-b1":
                continue
            we = workloads.workload(2)
            if args.layers:
                we.layers = min(we.layers, args.layers)
            if me.get("topk"):                  # the budget-vs-mass comparison of the pages
                me["retained_full_attention_mass"] = oracle_retained_mass(we, k=me["topk"])
                continue
            me["retained_full_attention_mass"] = oracle_retained_mass(we, p=me["p"])
            n, spent = oracle_full_step(we)      # one whole 36-layer step
            me["cpu_baseline"] = {"value": n / spent, "unit": "layer-steps/s",
                                  "cores": cpu_threads(), "kind": "oracle",
                                  "sample": f"one whole step of {we.name}: all {n} layers, "
                                            f"every head, {spent:.1f} s of float64 NumPy"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=4)
    ap.add_argument("--extra", default="2,3,5",
                    help="workloads measured in the same run and reported under 'extra'")
    ap.add_argument("--topk", type=int, default=2048,
                    help="k of the fixed-budget top-k variant measured on the 32K workload "
                         "(0: skip)")
    ap.add_argument("--prefill", type=int, default=32768,
                    help="prompt length of the prefill measured under 'extra' (0: skip)")
    ap.add_argument("--prefill-steps", type=int, default=3,
                    help="timed 36-layer prefill steps")
    ap.add_argument("--p", type=float, default=None)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--layers", type=int, default=0, help="run only the first N layers")
    ap.add_argument("--preroll", type=float, default=0.6, help="untimed seconds before timing")
    ap.add_argument("--separate-append", action="store_true",
                    help="append with rtp_append_kv and decode with rtp_decode_step (two launches "
                         "per layer) instead of rtp_decode_step_append")
    args = ap.parse_args(argv)
    from synth import workloads
    w = workloads.workload(args.workload, args.p)
    if args.layers:
        w.layers = min(w.layers, args.layers)
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    main()
