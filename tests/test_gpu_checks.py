"""The bounds-checked debug build (librtp_checks.so, compiled with -DRTP_CHECKS: every
gathered row, ring row, list slot and debug-list index is checked before it is touched) on the
parity cases, in a child process that loads it through RTP_LIBRARY_PATH: no check fires and
the results meet the oracle. And repeated runs of the release build select the same sets and
write the same outputs, bit for bit. Needs a B200."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from synth import workloads

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "long_context_sparse_rtpurbo_b200", "librtp_checks.so")

CHILD = r"""
import dataclasses, sys
import numpy as np, torch
sys.path.insert(0, ROOT)
sys.path.insert(0, ROOT + "/tests")
from long_context_sparse_rtpurbo_b200 import _lib, rtp
assert _lib.LIB_PATH.endswith("librtp_checks.so"), _lib.LIB_PATH
import parity as P
from synth import workloads

def small(**kw):
    w = workloads.workload(1)
    a = dict(B=1, Hq=8, Hkv=2, sinks=4, window=256, ret_mask=np.array([[True, False]]))
    a.update(kw)
    return dataclasses.replace(w, **a)

P.run_layer_parity(workload_index=1, layer=0, p=0.9)                          # top-p, lists
P.run_layer_parity(w=small(B=6, seq_lens=np.array([1, 3, 259, 260, 261, 5000]),
                           kind="needle"), layer=0)                           # ragged, edges
P.run_layer_parity(w=small(seq_lens=np.array([4096])), layer=0, k=64)         # top-k
w = workloads.workload(4)                                                     # recompute path
layer = next(l for l in range(w.layers) if w.ret_mask[l].sum() == 4)
ret = [g for g in range(w.Hkv) if w.ret_mask[layer, g]]
P.run_layer_parity(w=w, layer=layer, source="gpu",
                   heads=[(0, ret[-1] * w.G), (0, ret[0] * w.G)])
w = small(seq_lens=np.array([4096]), window=64)                               # prefill
n = 300
lay = P.make_layer(w, 0, "cuda", seq_lens=[n], caps=[n])
wk = torch.from_numpy(np.array(w.w_kidx(0), np.float32)).to("cuda")
qb, kb, vb = P.prefill_inputs(w, 0, n, 2.0)
out = P.prefill(lay, qb, kb, vb, [n], wk, "cuda")
assert rtp.rtp_read_device_status(lay.pf_ws) == 0
P.check_prefill(w, 0, [n], qb, kb, vb, out)
print("checks build: all cases clean")
"""


def test_bounds_checked_build_on_parity_cases():
    assert os.path.exists(LIB), "librtp_checks.so is built by __graft_entry__.build()"
    env = dict(os.environ, RTP_LIBRARY_PATH=LIB)
    r = subprocess.run([sys.executable, "-c", CHILD.replace("ROOT", repr(ROOT))], env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "all cases clean" in r.stdout


def test_repeated_decodes_are_bit_identical():
    """Two decodes of the same 32K Qwen3-8B-shaped layer select the same ascending sets and
    write the same outputs and counts (the histogram sums are exact integers, so the order in
    which CTAs add them does not matter)."""
    import parity as P
    w = workloads.workload(2)
    layer = next(l for l in range(w.layers) if w.ret_mask[l].sum() >= 2)
    q, wq, wk = P.layer_inputs(w, layer, "cuda")
    lay = P.make_layer(w, layer, "cuda")
    P.fill_layer(w, layer, lay, wk, w.seq_lens, source="gpu", device="cuda")
    runs = [P.decode(lay, q, wq, w.seq_lens, w.p, "cuda", with_sel=True) for _ in range(3)]
    assert lay.status() == 0
    for out, cnt, sel in runs[1:]:
        assert torch.equal(out.view(torch.int16), runs[0][0].view(torch.int16))
        assert torch.equal(cnt, runs[0][1])
        assert torch.equal(sel, runs[0][2])
