"""GPU parity of the CUDA path against the CPU oracle, through the C ABI (needs a B200)."""
import dataclasses

import numpy as np
import pytest
import torch

from oracle import rtp_oracle as O
from synth import gen, workloads

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _parity():
    import parity
    return parity


def test_gpu_fill_matches_numpy_stream():
    from synth.gpu import LayerFiller
    w = workloads.workload(1)
    f = LayerFiller(w, 0, DEV)
    k, v = f.fill(np.array([37]), 300)
    k = k.view(torch.int16).cpu().numpy().view(np.uint16)
    v = v.view(torch.int16).cpu().numpy().view(np.uint16)
    for g in range(w.Hkv):
        np.testing.assert_array_equal(k[0, :, g], w.kpre_bits(0, 0, g, 37, 337))
        np.testing.assert_array_equal(v[0, :, g], w.v_bits(0, 0, g, 37, 337))
    c = w.group_layout(0, 0, 0).clusters[0]                    # a planted run
    k, _ = f.fill(np.array([c.start - 3]), c.length + 6)
    k = k.view(torch.int16).cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(k[0, :, 0], w.kpre_bits(0, 0, 0, c.start - 3, c.start + c.length + 3))


def test_append_matches_oracle_rows():
    P = _parity()
    w = workloads.workload(1)
    q, wq, wk = P.layer_inputs(w, 0, DEV)
    N = int(w.seq_lens[0])
    lay = P.make_layer(w, 0, DEV)
    P.fill_layer(w, 0, lay, wk, [N], chunk=1000, device=DEV)   # ragged chunks
    torch.cuda.synchronize()
    assert lay.status() == 0
    kp = P.bits_to_f64(w.kpre_bits(0, 0, 0, 0, N))
    vv = P.bits_to_f64(w.v_bits(0, 0, 0, 0, N))
    k_ref, v_ref, i_ref = O.append_rows(kp, vv, w.w_kidx(0)[0], np.arange(N), w.rope_base)
    k_gpu = lay.k_ret[0, :N].double().cpu().numpy()
    i_gpu = lay.idx[0, :N].double().cpu().numpy()
    v_gpu = lay.v_ret[0, :N].double().cpu().numpy()
    np.testing.assert_array_equal(v_gpu, v_ref)
    # RoPE and the projection run in double on both sides: equal bf16 except, at most, values
    # within one bf16 spacing of a rounding tie
    for got, ref in ((k_gpu, k_ref), (i_gpu, i_ref)):
        mism = got != ref
        assert mism.mean() < 1e-5, mism.sum()
        if mism.any():
            ulp = np.ldexp(1.0, np.frexp(ref[mism])[1] - 8)
            assert np.all(np.abs(got[mism] - ref[mism]) <= ulp)
    # local ring of KV head 1: row n < sinks -> n; else sinks + (n - sinks) % window
    kp1 = P.bits_to_f64(w.kpre_bits(0, 0, 1, 0, N))
    pos = O.local_positions(N, w.sinks, w.window)
    rows = np.where(pos < w.sinks, pos, w.sinks + (pos - w.sinks) % w.window)
    k_ref1 = O.bf16_round(O.rope_rotate(kp1[pos], pos, w.rope_base))
    got1 = lay.k_loc[0, 0].double().cpu().numpy()[rows]
    assert (got1 != k_ref1).mean() < 1e-5


@pytest.mark.parametrize("p", [0.9, 0.5, 0.99, 0.999, 0.999995, 1.0])
def test_tiny_layer_parity(p):
    rep = _parity().run_layer_parity(workload_index=1, layer=0, p=p)
    assert rep["max_abs"] <= 1e-2


def _small(G=4, Hkv=2, B=1, seq=(4096,), sinks=4, window=256, ret=(True, False), kind="mix",
           lam=(1.65, 2.05)):
    w = workloads.workload(1)
    return dataclasses.replace(w, B=B, Hq=G * Hkv, Hkv=Hkv, seq_lens=np.array(seq),
                               sinks=sinks, window=window,
                               ret_mask=np.array([list(ret)], bool), kind=kind,
                               lam_conc=lam[0], lam_diff=lam[1])


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_group_sizes(G):
    w = _small(G=G, seq=(3000,))
    _parity().run_layer_parity(w=w, layer=0)


def test_ragged_batch_and_edge_lengths():
    """N = 1, N < sinks, N around sinks + window, ragged lengths in one batch."""
    w = _small(B=6, Hkv=2, seq=(1, 3, 259, 260, 261, 5000), kind="needle")
    _parity().run_layer_parity(w=w, layer=0)


def test_dense_reduction_on_gpu():
    """p = 1 and window >= N: every head attends every token."""
    w = _small(seq=(2000,), window=4096)
    rep = _parity().run_layer_parity(w=w, layer=0, p=1.0)
    for e in rep["heads"]:
        assert e["count"] == 2000


def test_all_retrieval_and_all_local_layers():
    _parity().run_layer_parity(w=_small(ret=(True, True), seq=(5000,)), layer=0)
    _parity().run_layer_parity(w=_small(ret=(False, False), seq=(5000,)), layer=0)


def test_device_status_on_bad_seq_len():
    """seq_lens[b] above seq_cap[b]: the sequence is skipped, the status word says so."""
    P = _parity()
    w = _small(B=2, seq=(500, 800))
    q, wq, wk = P.layer_inputs(w, 0, DEV)
    lay = P.make_layer(w, 0, DEV, seq_lens=[500, 800], caps=[500, 800])
    P.fill_layer(w, 0, lay, wk, [500, 800], device=DEV)
    out, cnt, _ = P.decode(lay, q, wq, [501, 800], 0.9, DEV, with_sel=False)
    assert lay.status() == -6
    assert np.all(cnt[0].cpu().numpy() == 0)
    assert np.all(cnt[1].cpu().numpy() > 0)
    assert lay.status() == 0                                        # read clears it


def test_qwen_layer_32k_parity():
    """One full Qwen3-8B-shaped layer at N = 32768 (every head), caches from the GPU fill."""
    w = workloads.workload(2)
    layer = int(np.nonzero(w.ret_mask.sum(1) >= 2)[0][0])
    rep = _parity().run_layer_parity(w=w, layer=layer, source="gpu")
    kind = lambda h: w.group_layout(layer, 0, h // w.G).targets[h % w.G][0]
    conc = [e["n_gpu"] for e in rep["heads"] if e["retrieval"] and kind(e["h"]) == "conc"]
    diff = [e["n_gpu"] for e in rep["heads"] if e["retrieval"] and kind(e["h"]) == "diff"]
    assert conc and diff and np.mean(diff) > 2.5 * np.mean(conc)


@pytest.mark.parametrize("G,N", [(8, 600_000), (4, 700_000)])
def test_two_wave_schedule(G, N):
    """Two retrieval groups with more rows than one chunk per CTA holds at the tensor-memory
    score capacity (16384 rows per CTA for G <= 4, 8192 for G = 8; 1.2-1.4M rows over at most
    148 CTAs): CTAs take two chunks, and a group's phases wait on chunks of both waves."""
    w = _small(G=G, Hkv=2, seq=(N,), window=2048, ret=(True, True))
    heads = [(0, 0), (0, G - 1), (0, G), (0, 2 * G - 1)]
    rep = _parity().run_layer_parity(w=w, layer=0, source="gpu", heads=heads)
    assert all(e["retrieval"] and e["count"] > 0 for e in rep["heads"])


@pytest.mark.parametrize("k", [1, 64, 2048, 4096, 5000])
def test_topk_tiny_layer_parity(k):
    """The fixed-budget top-k selector (count threshold on the same histogram), N = 4096:
    k = 1, small, mid, k = N and k > N (every token)."""
    rep = _parity().run_layer_parity(workload_index=1, layer=0, k=k)
    for e in rep["heads"]:
        if e["retrieval"]:
            assert e["count"] >= min(k, 4096)


@pytest.mark.parametrize("G", [1, 8])
def test_topk_group_sizes(G):
    _parity().run_layer_parity(w=_small(G=G, seq=(3000,)), layer=0, k=300)


def test_topk_qwen_layer_32k():
    """A full Qwen3-8B-shaped layer at N = 32768 with k = 2048 (every head)."""
    w = workloads.workload(2)
    layer = int(np.nonzero(w.ret_mask.sum(1) >= 2)[0][0])
    rep = _parity().run_layer_parity(w=w, layer=layer, source="gpu", k=2048)
    assert all(e["count"] >= 2048 for e in rep["heads"] if e["retrieval"])


# Full benchmark sizes, in the launch configuration the bench times (one layer of the 36, all
# caches filled on the GPU); the oracle checks sampled heads one by one.
def _layer_with(w, n_ret):
    return int(np.nonzero(w.ret_mask.sum(1) == n_ret)[0][0])


def _kv(w, layer, retrieval):
    return [int(g) for g in np.nonzero(w.ret_mask[layer] == retrieval)[0]]


def test_full_size_128k_b4_layer():
    """128K x 4 (Qwen3-8B shape), a layer with three retrieval KV heads: twelve groups whose
    chunks need two waves; every query head of two groups (the last sequence's last group,
    the first sequence's first group) and one local head."""
    w = workloads.workload(3)
    layer = _layer_with(w, 3)
    ret, loc = _kv(w, layer, True), _kv(w, layer, False)
    heads = [(3, ret[-1] * w.G + i) for i in range(w.G)] + \
            [(0, ret[0] * w.G + i) for i in range(w.G)] + [(2, loc[0] * w.G)]
    rep = _parity().run_layer_parity(w=w, layer=layer, source="gpu", heads=heads)
    assert all(e["count"] > 0 for e in rep["heads"])


def test_full_size_1m_layer():
    """1M tokens (B = 1), a layer with two retrieval KV heads (chunks in two waves): every
    query head of the second group."""
    w = workloads.workload(4)
    layer = _layer_with(w, 2)
    g = _kv(w, layer, True)[-1]
    heads = [(0, g * w.G + i) for i in range(w.G)]
    rep = _parity().run_layer_parity(w=w, layer=layer, source="gpu", heads=heads)
    assert all(e["retrieval"] and e["count"] > 0 for e in rep["heads"])


def test_recomputed_scores_1m_four_groups():
    """1M tokens, a layer with four retrieval KV heads: 4M index rows over at most 148 CTAs
    is more than the 16384 rows whose scores one CTA's tensor memory holds, so the CTAs' later
    chunks recompute their scores from the index rows in phases H and W (the recompute path
    and its global per-warp lists). Every query head of the last group (whose chunks come
    last on each CTA) and one head of the first."""
    w = workloads.workload(4)
    layer = _layer_with(w, 4)
    ret = _kv(w, layer, True)
    assert len(ret) == 4 and w.G == 4
    assert 4 * int(w.seq_lens[0]) > 148 * 16384
    heads = [(0, ret[-1] * w.G + i) for i in range(w.G)] + [(0, ret[0] * w.G)]
    rep = _parity().run_layer_parity(w=w, layer=layer, source="gpu", heads=heads)
    assert all(e["retrieval"] and e["count"] > 0 for e in rep["heads"])


@pytest.mark.parametrize("p", [0.8, 0.95])
def test_full_size_ragged_b64_other_p(p):
    """The ragged batch of 64 sequences at the other two top-p values the workload draws
    from: the retrieval heads of three sequences (first, middle, last)."""
    w = workloads.workload(5)
    layer = _layer_with(w, 1)
    ret = _kv(w, layer, True)
    heads = [(b, ret[0] * w.G + i) for b in (0, 31, 63) for i in (0, w.G - 1)]
    rep = _parity().run_layer_parity(w=w, layer=layer, p=p, source="gpu", heads=heads)
    assert all(e["count"] > 0 for e in rep["heads"])


def test_wait_timeout_then_recovery():
    """A device-side wait that runs out: with the wait limit at one SM cycle, a fused
    decode + append (the CTA holding the decode token appends it before it arrives, so the
    group's other CTAs reach their wait first) returns through RTP_ETIMEOUT in the status
    word, without hanging; after rtp_workspace_init and with the default limit, the same
    layer (the token appended again, the same rows) decodes with parity."""
    from long_context_sparse_rtpurbo_b200 import rtp
    from long_context_sparse_rtpurbo_b200._lib import RTP_ETIMEOUT
    P = _parity()
    w = _small(G=4, Hkv=2, seq=(300_000,), window=2048, ret=(True, False))
    seq = np.asarray(w.seq_lens, np.int64)
    q, wq, wk = P.layer_inputs(w, 0, DEV)
    kb, vb = _token_bits(w, 0, seq)
    k_new, v_new = P.bits_to_torch(kb, DEV), P.bits_to_torch(vb, DEV)
    sl = torch.as_tensor(seq.astype(np.int32), device=DEV)
    lay = P.make_layer(w, 0, DEV)
    P.fill_layer(w, 0, lay, wk, seq - 1, source="gpu", device=DEV)
    out = torch.zeros((w.B, w.Hq, 128), dtype=torch.bfloat16, device=DEV)
    cnt = torch.zeros((w.B, w.Hq), dtype=torch.int32, device=DEV)
    try:
        rtp.rtp_debug_set_wait_limit(1)
        lay.decode_append(k_new, v_new, wk, q, wq, sl, w.p, out, cnt)
        st = lay.status()
    finally:
        rtp.rtp_debug_set_wait_limit(0)
    assert st == RTP_ETIMEOUT
    rtp.rtp_workspace_init(lay.ws)
    lay.append(k_new.view(w.B, 1, w.Hkv, 128), v_new.view(w.B, 1, w.Hkv, 128), wk,
               torch.as_tensor((seq - 1).astype(np.int32), device=DEV))
    out, cnt, sel = P.decode(lay, q, wq, seq, w.p, DEV, with_sel=True)
    assert lay.status() == 0
    heads = [(0, i) for i in range(w.G)] + [(0, w.G)]
    P.check_outputs(w, 0, seq, w.p, out, cnt, sel, heads)


def _token_bits(w, layer, seq_lens):
    """The decode token (position N_b - 1) of every sequence and KV head: bf16 [B][Hkv][128]."""
    kb = np.zeros((w.B, w.Hkv, 128), np.uint16)
    vb = np.zeros_like(kb)
    for b in range(w.B):
        n = int(seq_lens[b])
        for g in range(w.Hkv):
            kb[b, g] = w.kpre_bits(layer, b, g, n - 1, n)[0]
            vb[b, g] = w.v_bits(layer, b, g, n - 1, n)[0]
    return kb, vb


@pytest.mark.parametrize("case", ["mix", "ragged", "waves", "local", "local_ragged"])
def test_fused_append_equals_two_calls(case):
    """rtp_decode_step_append equals rtp_append_kv (n_new = 1) followed by rtp_decode_step:
    identical caches, counts and outputs, bit for bit (the same arithmetic runs in both)."""
    P = _parity()
    if case == "mix":
        w = _small(G=4, Hkv=2, seq=(5000,))
    elif case == "ragged":      # N = 1, N < sinks, N around the ring's wrap, a long one
        w = _small(B=6, Hkv=2, seq=(1, 3, 259, 260, 261, 5000), kind="needle")
    elif case == "waves":       # two groups in two waves
        w = _small(G=8, Hkv=2, seq=(600_000,), window=2048, ret=(True, True))
    elif case == "local":       # no retrieval head: only local items
        w = _small(G=4, Hkv=2, seq=(5000,), ret=(False, False))
    else:                       # only local heads, ragged lengths
        w = _small(B=6, Hkv=2, seq=(1, 3, 259, 260, 261, 5000), kind="needle", ret=(False, False))
    seq = np.asarray(w.seq_lens, np.int64)
    q, wq, wk = P.layer_inputs(w, 0, DEV)
    kb, vb = _token_bits(w, 0, seq)
    k_new, v_new = P.bits_to_torch(kb, DEV), P.bits_to_torch(vb, DEV)
    sl = torch.as_tensor(seq.astype(np.int32), device=DEV)
    res = []
    for fused in (False, True):
        lay = P.make_layer(w, 0, DEV)
        for t in (lay.k_ret, lay.v_ret, lay.idx, lay.k_loc, lay.v_loc):
            t.zero_()                      # rows no token reaches compare equal too
        P.fill_layer(w, 0, lay, wk, seq - 1, source="gpu", device=DEV)
        out = torch.zeros((w.B, w.Hq, 128), dtype=torch.bfloat16, device=DEV)
        cnt = torch.zeros((w.B, w.Hq), dtype=torch.int32, device=DEV)
        if fused:
            lay.decode_append(k_new, v_new, wk, q, wq, sl, w.p, out, cnt)
        else:
            lay.append(k_new.view(w.B, 1, w.Hkv, 128), v_new.view(w.B, 1, w.Hkv, 128), wk,
                       torch.as_tensor((seq - 1).astype(np.int32), device=DEV))
            lay.decode(q, wq, sl, w.p, out, cnt)
        torch.cuda.synchronize()
        assert lay.status() == 0
        res.append([t.clone() for t in (out.view(torch.int16), cnt, lay.k_ret.view(torch.int16),
                                         lay.v_ret.view(torch.int16), lay.idx.view(torch.int16),
                                         lay.k_loc.view(torch.int16), lay.v_loc.view(torch.int16))])
        del lay
    for a, b in zip(*res):
        assert torch.equal(a, b)
