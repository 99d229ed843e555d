"""GPU parity of the causal prefill (rtp_prefill) against the CPU oracle, through the C ABI."""
import dataclasses

import numpy as np
import pytest
import torch

from oracle import rtp_oracle as O
from synth import workloads

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _parity():
    import parity
    return parity


def _small(G=4, Hkv=2, B=1, sinks=4, window=64, ret=(True, False)):
    w = workloads.workload(1)
    return dataclasses.replace(w, B=B, Hq=G * Hkv, Hkv=Hkv, sinks=sinks, window=window,
                               seq_lens=np.full(B, 4096), ret_mask=np.array([list(ret)], bool))


def _wk(w, layer):
    return torch.from_numpy(np.array(w.w_kidx(layer), np.float32)).to(DEV)


def _run(w, n_b, n_max, q_scale=1.0, rows=None, heads=None):
    P = _parity()
    n_b = np.asarray(n_b, np.int64)
    caps = np.maximum(n_b, 1)
    lay = P.make_layer(w, 0, DEV, seq_lens=caps, caps=caps)
    qb, kb, vb = P.prefill_inputs(w, 0, n_max, q_scale)
    out = P.prefill(lay, qb, kb, vb, n_b, _wk(w, 0), DEV)
    assert lay.status() == 0
    return P.check_prefill(w, 0, n_b, qb, kb, vb, out, rows=rows, heads=heads), lay, out


@pytest.mark.parametrize("q_scale", [1.0, 4.0])
def test_prefill_small_all_rows(q_scale):
    """Every row of a ragged two-sequence prompt (several 64-row tiles and a ragged tail),
    one retrieval and one local KV head; q_scale 4 makes the rows peaked."""
    w = _small(B=2)
    rep, _, _ = _run(w, [300, 173], 300, q_scale)
    assert rep["rows"] == (300 + 173) * w.Hq


@pytest.mark.parametrize("G", [1, 2, 8])
def test_prefill_group_sizes(G):
    w = _small(G=G)
    _run(w, [257], 257, 2.0)


def test_prefill_edges():
    """Prompt lengths 0, 1, below the sinks, at the ring's edge and one tile plus one; a
    window longer than every prompt (local heads then attend densely) in a second call."""
    w = _small(B=6)
    _run(w, [0, 1, 3, 68, 69, 65], 69, 2.0)
    w2 = _small(B=2, window=4096)
    _run(w2, [200, 129], 200, 2.0)


def test_prefill_no_sinks_and_all_local():
    w = _small(sinks=0, window=37, ret=(False, False))
    _run(w, [250], 250, 3.0)


def test_prefill_fills_the_cache_for_decode():
    """DecodeLayer.prefill appends the prompt: a decode step at N = n_b + 1 after it equals
    the decode oracle (the usual decode parity rule)."""
    P = _parity()
    n_b = np.array([500, 333])
    seq = n_b + 1
    w = dataclasses.replace(_small(B=2, window=64), seq_lens=seq)
    lay = P.make_layer(w, 0, DEV, seq_lens=seq, caps=seq)
    q, wq, wk = P.layer_inputs(w, 0, DEV)
    qb, kb, vb = P.prefill_inputs(w, 0, 500)
    P.prefill(lay, qb, kb, vb, n_b, wk, DEV)
    kn = np.stack([w.kpre_bits(0, b, g, n_b[b], n_b[b] + 1)[0] for b in range(w.B)
                   for g in range(w.Hkv)]).reshape(w.B, w.Hkv, 128)
    vn = np.stack([w.v_bits(0, b, g, n_b[b], n_b[b] + 1)[0] for b in range(w.B)
                   for g in range(w.Hkv)]).reshape(w.B, w.Hkv, 128)
    sl = torch.as_tensor(seq.astype(np.int32), device=DEV)
    out = torch.zeros((w.B, w.Hq, 128), dtype=torch.bfloat16, device=DEV)
    cnt = torch.zeros((w.B, w.Hq), dtype=torch.int32, device=DEV)
    lay.decode_append(P.bits_to_torch(kn, DEV), P.bits_to_torch(vn, DEV), wk, q, wq, sl, w.p,
                      out, cnt)
    torch.cuda.synchronize()
    assert lay.status() == 0
    P.check_outputs(w, 0, seq, w.p, out, cnt)


def test_prefill_qwen_layer_32k_sampled_rows():
    """A 32K prompt on the Qwen3-8B layer shape (32 query heads, 8 KV heads, a layer with
    retrieval heads), the configuration the bench times; rows sampled at tile and window
    edges and at random, for every head."""
    w0 = workloads.workload(2)
    layer = int(np.nonzero(w0.ret_mask.any(axis=1))[0][0])
    w = dataclasses.replace(w0, B=1)
    n = 32768
    rng = np.random.default_rng(5)
    rows = np.concatenate([[0, 1, 3, 4, 63, 64, 2051, 2052, 2053, 4095, n - 65, n - 1],
                           rng.integers(0, n, 6)])
    P = _parity()
    caps = np.array([n])
    lay = P.make_layer(w, layer, DEV, seq_lens=caps, caps=caps)
    qb, kb, vb = P.prefill_inputs(w, layer, n, 2.0)
    out = P.prefill(lay, qb, kb, vb, [n], _wk(w, layer), DEV)
    rep = P.check_prefill(w, layer, [n], qb, kb, vb, out, rows=rows)
    assert rep["rows"] == np.unique(rows).size * w.Hq


def test_prefill_argument_errors():
    from long_context_sparse_rtpurbo_b200 import rtp
    from long_context_sparse_rtpurbo_b200._lib import RTP_EINVAL, RTP_ESHAPE, RTP_EWORKSPACE
    w = _small()
    lay = _parity().make_layer(w, 0, DEV, seq_lens=[64], caps=[64])
    q = torch.zeros((1, 64, w.Hq, 128), dtype=torch.bfloat16, device=DEV)
    kv = torch.zeros((1, 64, w.Hkv, 128), dtype=torch.bfloat16, device=DEV)
    nb = torch.full((1,), 64, dtype=torch.int32, device=DEV)
    out = torch.zeros_like(q)
    need = rtp.rtp_prefill_workspace_bytes(lay.desc, 64)
    assert need == 256 + 64 * w.Hkv * 256
    ws = torch.zeros(need, dtype=torch.uint8, device=DEV)
    for args, code in (((lay.desc, q, kv, kv, nb, -1, out, ws), RTP_EINVAL),
                       ((lay.desc, q, kv, kv, nb, 65, out, ws), RTP_ESHAPE),
                       ((lay.desc, None, kv, kv, nb, 64, out, ws), RTP_EINVAL),
                       ((lay.desc, q, kv, kv, nb, 64, out, ws[:need - 256]), RTP_EWORKSPACE)):
        with pytest.raises(rtp.RtpError) as e:
            rtp.rtp_prefill(*args)
        assert e.value.code == code
    assert rtp.rtp_prefill(lay.desc, q, kv, kv, nb, 0, out, None) == 0   # nothing to do


def test_prefill_wait_timeout_then_recovery():
    """With the device-wait limit at one SM cycle the prefill's first wait for its MMAs runs
    out: the call returns, the status word holds RTP_ETIMEOUT and the rows stay unwritten;
    with the default limit the same prompt then meets parity."""
    from long_context_sparse_rtpurbo_b200 import rtp
    from long_context_sparse_rtpurbo_b200._lib import RTP_ETIMEOUT
    P = _parity()
    w = _small(B=1)
    n = 200
    lay = P.make_layer(w, 0, DEV, seq_lens=[n], caps=[n])
    qb, kb, vb = P.prefill_inputs(w, 0, n, 2.0)
    try:
        rtp.rtp_debug_set_wait_limit(1)
        out = P.prefill(lay, qb, kb, vb, [n], _wk(w, 0), DEV)
        st = rtp.rtp_read_device_status(lay.pf_ws)
    finally:
        rtp.rtp_debug_set_wait_limit(0)
    assert st == RTP_ETIMEOUT
    assert bool((out.float() == -7.0).all())
    out = P.prefill(lay, qb, kb, vb, [n], _wk(w, 0), DEV)
    assert rtp.rtp_read_device_status(lay.pf_ws) == 0
    P.check_prefill(w, 0, [n], qb, kb, vb, out)
