"""Host logic of bench.py: max-over-ranks timing with two gloo ranks on CPU, whole-job
aggregation, and the algorithmic byte count of a layer-step."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp

import bench
from synth import workloads


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    r, w, lr = bench.dist_env()
    ms = bench.max_over_ranks(1.5 + rank, w)           # rank 1 is the slow one
    q.put((r, w, lr, ms, bench.aggregate(36, 10, w, ms)))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r, (rank, world, lr, ms, v) in enumerate(out):
        assert (rank, world, lr) == (r, 2, r)
        assert ms == 2.5                               # every rank sees the slowest rank's time
        assert abs(v - 36 * 10 * 2 / 2.5e-3) < 1e-6    # units of all ranks / max time


def test_aggregate_single_rank():
    assert bench.max_over_ranks(3.0, 1) == 3.0
    assert bench.aggregate(36, 1, 1, 1.0) == 36000.0


def test_algorithmic_bytes_closed_form():
    w = workloads.workload(1)                          # 1 layer, KV head 0 retrieval, 1 local
    N = int(w.seq_lens[0])
    unions = [{(0, 0): 100}]
    got = bench.algorithmic_bytes(w, unions, include_append=False)
    ring = w.sinks + w.window
    want = (32 * N + 512 * 100) + 512 * min(N, ring) + w.Hq * 512 + 8192 * w.G
    assert got == want
    full = bench.algorithmic_bytes(w, unions, include_append=True)
    assert full - got == (512 + 32) + 512 + 8192


def test_prefill_flops_counts_attended_pairs():
    """The prefill roofline's FLOPs: 4 * 128 per attended (query head, row, key), counted here
    pair by pair from the oracle's position sets on a tiny layout."""
    import dataclasses
    import numpy as np
    from oracle import rtp_oracle as O
    w = dataclasses.replace(workloads.workload(1), sinks=3, window=7)     # 1 retrieval, 1 local
    n = 40
    pairs = 0
    for g in range(w.Hkv):
        for m in range(n):
            att = m + 1 if w.ret_mask[0, g] else O.local_positions(m + 1, w.sinks, w.window).size
            pairs += att * w.G
    assert bench.prefill_flops(w, n) == 4 * 128 * pairs * w.B
    assert np.isclose(bench.prefill_flops(workloads.workload(2), 32768) / 1e12, 79.96, atol=0.01)


def test_reference_arm_line_fields(capsys, monkeypatch):
    """--impl reference prints one JSON line with the oracle as the CPU baseline."""
    import json
    monkeypatch.setenv("RANK", "0")
    bench.main(["--impl", "reference", "--workload", "1", "--steps", "1", "--warmup", "0"])
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "layer-steps/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
