"""Decode-step benchmark of the RTPurbo sparse attention path on B200.

One step = one decode step of every layer of the workload: per layer, the append of the
current token and the decode step, for the whole batch, in one launch (rtp_decode_step_append;
--separate-append: rtp_append_kv with n_new = 1, then rtp_decode_step), replayed from a CUDA
graph. Metric: decode layer-steps/s (a layer-step is one layer over the whole batch), plus the
achieved HBM bandwidth of the algorithmic bytes the step must move.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 2] [--impl ours|reference]

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
    prepared = prepare_oracle_layers(w, sample_layers(w))
    steps_s = []
    for i in range(args.warmup + args.steps):
        n, s = oracle_layer_steps(w, prepared[i % len(prepared):] + prepared[:i % len(prepared)],
                                  0.0, max_steps=1)
        if i >= args.warmup:
            steps_s.append(s / n)
    v = 1.0 / float(np.mean(steps_s))
    sample = (f"one whole layer-step (all heads, all sequences) of {w.name} per step, alternating "
              f"layers {[p[0] for p in prepared]} (one with retrieval heads, one without)")
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


def _traffic(kernel: str):
    """DRAM bytes per launch of ``kernel`` from a committed ncu summary, if it was taken on the
    current source (its sha256 recorded beside it); else None."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    src = os.path.join(ROOT, "long_context_sparse_rtpurbo_b200", "csrc")
    h = hashlib.sha256()
    for name in sorted(os.listdir(src)):
        with open(os.path.join(src, name), "rb") as f:
            h.update(f.read())
    e = d.get(kernel)
    if not e or e.get("source_sha256") != h.hexdigest():
        return None
    return e


def run_ours(args, w):
    import datetime
    import torch
    import torch.distributed as dist
    from long_context_sparse_rtpurbo_b200 import rtp
    from long_context_sparse_rtpurbo_b200.layer import DecodeLayer
    from synth.gpu import LayerFiller

    rank, world, local = dist_env()
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    N = np.asarray(w.seq_lens, np.int64)
    B, Hq, Hkv, Lyr = w.B, w.Hq, w.Hkv, w.layers
    # packed per-step inputs (q of all layers, current-token k/v) and outputs
    nq, nk = B * Hq * 128, B * Hkv * 128
    per_layer_in = nq + 2 * nk
    inp = torch.empty(Lyr * per_layer_in, dtype=torch.bfloat16, device=dev)
    out_all = torch.empty((Lyr, B, Hq, 128), dtype=torch.bfloat16, device=dev)
    cnt_all = torch.empty((Lyr, B, Hq), dtype=torch.int32, device=dev)
    layers = []
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
        q = inp[base:base + nq].view(B, Hq, 128)
        knew = inp[base + nq:base + nq + nk].view(B, 1, Hkv, 128)
        vnew = inp[base + nq + nk:base + per_layer_in].view(B, 1, Hkv, 128)
        q.copy_(_bits_to_dev(w.q_pre_bits(l), dev))
        kk, vv = filler.fill(N - 1, 1)
        knew.copy_(kk)
        vnew.copy_(vv)
        layers.append(dict(lay=lay, q=q, wq=wq, wk=wk, knew=knew, vnew=vnew,
                           start=torch.tensor(N - 1, dtype=torch.int32, device=dev),
                           seq=torch.tensor(N, dtype=torch.int32, device=dev),
                           out=out_all[l], cnt=cnt_all[l]))
        del filler
    torch.cuda.synchronize()
    t_fill = time.perf_counter() - t_fill

    launches = {"n": 0}

    fused = not args.separate_append

    def step(with_append=True, count=False):
        for L in layers:
            if with_append and fused:          # append + decode in one launch
                L["lay"].decode_append(L["knew"].view(B, Hkv, 128), L["vnew"].view(B, Hkv, 128),
                                       L["wk"], L["q"], L["wq"], L["seq"], w.p, L["out"],
                                       L["cnt"])
                if count:
                    launches["n"] += rtp.rtp_last_launch_count()
                continue
            if with_append:
                L["lay"].append(L["knew"], L["vnew"], L["wk"], L["start"])
                if count:
                    launches["n"] += rtp.rtp_last_launch_count()
            L["lay"].decode(L["q"], L["wq"], L["seq"], w.p, L["out"], L["cnt"])
            if count:
                launches["n"] += rtp.rtp_last_launch_count()

    # one eager step (sets kernel attributes outside capture), then the unions of the
    # selected sets (untimed, with sel_idx) for the algorithmic byte count
    step(count=True)
    per_step_launches = launches["n"]
    unions, conc, diff, allc = [], [], [], []
    for l, L in enumerate(layers):
        u = {}
        if w.ret_mask[l].any():
            sel = torch.full((B, Hq, int(N.max())), -1, dtype=torch.int32, device=dev)
            cnt = torch.empty((B, Hq), dtype=torch.int32, device=dev)
            out = torch.empty((B, Hq, 128), dtype=torch.bfloat16, device=dev)
            L["lay"].decode(L["q"], L["wq"], L["seq"], w.p, out, cnt, sel)
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
    step_bytes = algorithmic_bytes(w, unions, include_append=True)
    dec_bytes = algorithmic_bytes(w, unions, include_append=False)

    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
        g_full = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_full, stream=side):
            step()
        g_dec = torch.cuda.CUDAGraph()                      # the decode kernel alone
        with torch.cuda.graph(g_dec, stream=side):
            step(with_append=fused)
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
    with ClockSampler(local) as clk:
        t_end = time.perf_counter() + args.preroll          # untimed pre-roll under load
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

    # end to end: H2D of the step's inputs from pinned memory, the step, D2H of the outputs
    inp_host = inp.cpu().pin_memory()
    out_host = torch.empty(out_all.shape, dtype=out_all.dtype).pin_memory()
    cnt_host = torch.empty(cnt_all.shape, dtype=cnt_all.dtype).pin_memory()

    def e2e_step():
        inp.copy_(inp_host, non_blocking=True)
        g_full.replay()
        out_host.copy_(out_all, non_blocking=True)
        cnt_host.copy_(cnt_all, non_blocking=True)

    if args.no_e2e:
        e2e_ms = float("nan")
    else:
        for _ in range(max(3, args.warmup)):
            e2e_step()
        e2e_ms = max_over_ranks(timed(e2e_step, args.steps) / args.steps, world, dev)
    h2d = inp.numel() * inp.element_size()
    d2h = out_all.numel() * out_all.element_size() + cnt_all.numel() * cnt_all.element_size()

    value = aggregate(Lyr, 1, world, ms_step)
    peak, peak_kind = load_peaks()
    kern_bytes = step_bytes if fused else dec_bytes       # the fused kernel also appends
    achieved = kern_bytes / (dec_step * 1e-3) / 1e9
    tr = _traffic("rtp_decode_step")
    attended = float(sum(allc)) + sum(min(int(n), w.sinks + w.window) * w.G
                                      for l in range(Lyr) for n in N
                                      for g in range(Hkv) if not w.ret_mask[l, g])
    scored = float(sum(int(n) * w.G for l in range(Lyr) for n in N
                       for g in range(Hkv) if w.ret_mask[l, g]))
    line = {
        "metric": METRIC, "value": value, "unit": "layer-steps/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": workload_config(w, "inputs larger than L2 (%.2f GB read per step vs 126 MB L2)"
                                  % (step_bytes / 1e9)),
        "achieved_step_gbs": step_bytes / (ms_step * 1e-3) / 1e9 * 1.0,
        "step_bytes": step_bytes,
        "token_heads_per_s": {"attended": attended * world / (ms_step * 1e-3),
                              "scored": scored * world / (ms_step * 1e-3)},
        "roofline": {"kernel": "rtp_decode_step", "bound": "hbm", "achieved": achieved,
                     "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_kind": peak_kind + " hbm_gbs (copy bandwidth)",
                     "traffic": None if tr is None else tr["dram_bytes_per_launch"],
                     "bytes_per_launch": kern_bytes / Lyr, "launch_us": dec_step * 1e3 / Lyr,
                     "fused_append": fused, "frac_of_nominal_8tbs": achieved / 8000.0},
        "e2e": {"value": aggregate(Lyr, 1, world, e2e_ms), "unit": "layer-steps/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": per_step_launches * args.steps,
        "clocks": clocks,
        "selected_tokens": {"concentrated_mean": float(np.mean(conc)) if conc else None,
                            "diffuse_mean": float(np.mean(diff)) if diff else None,
                            "min": int(min(allc)) if allc else None,
                            "max": int(max(allc)) if allc else None,
                            "union_mean": float(np.mean([x for u in unions for x in u.values()]))
                            if allc else None},
        "setup_s": t_fill,
    }
    if rank == 0 and world == 1 and not args.no_cpu:
        del layers
        torch.cuda.empty_cache()
        prepared = prepare_oracle_layers(w, sample_layers(w))
        n_done, spent = oracle_layer_steps(w, prepared, args.cpu_budget)
        line["cpu_baseline"] = {"value": n_done / spent, "unit": "layer-steps/s",
                                "cores": cpu_threads(), "kind": "oracle",
                                "sample": f"{n_done} whole layer-steps of {w.name} (all heads, "
                                          f"alternating layers {[p[0] for p in prepared]}: one "
                                          f"with retrieval heads, one without), {spent:.1f} s of "
                                          f"float64 NumPy"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        del g_full, g_dec
        dist.barrier()
        dist.destroy_process_group()


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=2)
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
