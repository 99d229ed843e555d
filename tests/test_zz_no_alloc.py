"""The allocation-free decode entry point (rtp_decode_step_static) against rtp_decode_step.

rtp_decode_step_static serves callers that cannot allocate device memory (an engine whose
planner already owns the device pool, work issued where cudaMalloc is not allowed): it runs the
same decode on a fixed scratch buffer inside the library. It runs the same kernel on the same
inputs as the workspace entry point, so two calls in a row through the C ABI must reproduce
its outputs and counts bit for bit; a layer too large for the fixed buffer must be refused
without a launch. This file is collected last on purpose; it also passes alone in a fresh
process.
"""
import numpy as np
import pytest
import torch

from long_context_sparse_rtpurbo_b200 import _lib, rtp
from synth import workloads

pytestmark = pytest.mark.gpu


def test_static_scratch_matches_workspace_entry_point():
    import parity
    w = workloads.workload(1)
    q, wq, wk = parity.layer_inputs(w, 0, "cuda")
    lay = parity.make_layer(w, 0, "cuda")
    assert lay.ws_bytes <= _lib.RTP_STATIC_SCRATCH_BYTES
    parity.fill_layer(w, 0, lay, wk, w.seq_lens, device="cuda")
    sl = torch.as_tensor(np.asarray(w.seq_lens, np.int32), device="cuda")
    ref = torch.zeros((w.B, w.Hq, 128), dtype=torch.bfloat16, device="cuda")
    ref_cnt = torch.zeros((w.B, w.Hq), dtype=torch.int32, device="cuda")
    lay.decode(q, wq, sl, w.p, ref, ref_cnt)
    torch.cuda.synchronize()
    for _ in range(2):                                 # two calls in a row share the scratch
        out = torch.full((w.B, w.Hq, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        cnt = torch.full((w.B, w.Hq), -1, dtype=torch.int32, device="cuda")
        rtp.rtp_decode_step_static(lay.desc, lay.cache, q, wq, sl, w.p, out, cnt)
        torch.cuda.synchronize()
        assert torch.isfinite(out.float()).all()
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
        assert torch.equal(cnt, ref_cnt)


def test_static_scratch_rejects_layers_beyond_its_size():
    w = workloads.workload(1)
    big = rtp.LayerDesc(64, 32, 8, 4, 2048, 1 << 20, rtp.rtp_build_slot_map([1] * 8)[0])
    assert rtp.rtp_workspace_bytes(big) > _lib.RTP_STATIC_SCRATCH_BYTES
    dummy = torch.zeros(1, device="cuda")
    cache = rtp.make_cache(dummy, dummy, dummy, dummy, dummy, dummy, dummy, 1 << 20)
    with pytest.raises(rtp.RtpError) as e:
        rtp.rtp_decode_step_static(big, cache, dummy, dummy, dummy, 0.9, dummy, dummy)
    assert e.value.code == _lib.RTP_EWORKSPACE
