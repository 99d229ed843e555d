"""Parity harness: runs the CUDA path through the C ABI and the CPU oracle on the same seeded
inputs and compares them under the rules below. Used by the GPU tests and by smoke().

Rules (selection: Top-P through the 256-bin histogram; outputs: bf16 against float64):
* a retrieval head's GPU set equals the oracle set except for tokens whose oracle score lies
  within one bin width of the oracle's threshold-bin edge; the oracle mass of the GPU set is
  >= p - 1e-6 of the total;
* outputs are compared on the GPU's own set, in the bf16 output format (the float64 oracle
  output rounded to bf16, nearest-even): max-abs <= 1e-2 and mean-abs <= 1e-3;
* sel_counts equals the size of the set; a local head attends min(N, sinks + window) tokens.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import rtp_oracle as O
from synth import gen, workloads
from long_context_sparse_rtpurbo_b200.layer import DecodeLayer

MAX_ABS = 1e-2
MEAN_ABS = 1e-3
MASS_SLACK = 1e-6


def bits_to_f64(bits) -> np.ndarray:
    return gen.bf16_bits_to_f32(bits).astype(np.float64)


def bits_to_torch(bits: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def layer_inputs(w, layer, device):
    """q_pre (bf16, device), W_qidx / W_kidx (fp32, device) of one layer."""
    q = bits_to_torch(w.q_pre_bits(layer), device)
    wq = torch.from_numpy(np.array(w.w_qidx(layer), np.float32)).to(device)
    wk = torch.from_numpy(np.array(w.w_kidx(layer), np.float32)).to(device)
    return q, wq, wk


def fill_layer(w, layer, lay: DecodeLayer, wk: torch.Tensor, upto, source="numpy", chunk=4096,
               device="cuda"):
    """Appends positions 0..upto[b]-1 of every sequence, in chunks, from the counter streams
    (NumPy on the host, or the GPU fill kernel)."""
    upto = np.asarray(upto, np.int64)
    filler = None
    if source == "gpu":
        from synth.gpu import LayerFiller
        filler = LayerFiller(w, layer, device)
    top = int(upto.max())
    for t0 in range(0, top, chunk):
        n = min(chunk, top - t0)
        nv = np.clip(upto - t0, 0, n).astype(np.int32)
        if filler is not None:
            k, v = filler.fill(np.full(w.B, t0), n, nv)
        else:
            kb = np.zeros((w.B, n, w.Hkv, 128), np.uint16)
            vb = np.zeros_like(kb)
            for b in range(w.B):
                if nv[b] == 0:
                    continue
                for g in range(w.Hkv):
                    kb[b, :nv[b], g] = w.kpre_bits(layer, b, g, t0, t0 + int(nv[b]))
                    vb[b, :nv[b], g] = w.v_bits(layer, b, g, t0, t0 + int(nv[b]))
            k, v = bits_to_torch(kb, device), bits_to_torch(vb, device)
        lay.append(k, v, wk, torch.full((w.B,), t0, dtype=torch.int32, device=device),
                   torch.from_numpy(nv).to(device))


def make_layer(w, layer, device="cuda", seq_lens=None, caps=None):
    seq_lens = np.asarray(w.seq_lens if seq_lens is None else seq_lens, np.int64)
    caps = seq_lens if caps is None else np.asarray(caps, np.int64)
    return DecodeLayer(w.B, w.Hq, w.Hkv, w.sinks, w.window, int(caps.max()), w.ret_mask[layer],
                       caps, device, w.rope_base)


def decode(lay: DecodeLayer, q, wq, seq_lens, p, device="cuda", with_sel=True, k=None):
    B, Hq = lay.B, lay.Hq
    out = torch.zeros((B, Hq, 128), dtype=torch.bfloat16, device=device)
    cnt = torch.zeros((B, Hq), dtype=torch.int32, device=device)
    stride = int(lay.desc.c.max_seq_len)
    sel = torch.full((B, Hq, stride), -1, dtype=torch.int32, device=device) if with_sel else None
    sl = torch.as_tensor(np.asarray(seq_lens, np.int32), device=device)
    if k is not None:
        lay.decode_topk(q, wq, sl, k, out, cnt, sel)
    else:
        lay.decode(q, wq, sl, p, out, cnt, sel)
    torch.cuda.synchronize()
    return out, cnt, sel


def check_selection(s, p, gpu_set: np.ndarray) -> dict:
    """Selection rule check for one retrieval head (oracle scores ``s``)."""
    sel = O.topp_histogram(s, p)
    ref = np.nonzero(sel.mask)[0]
    diff = np.setxor1d(ref, gpu_set)
    w = np.exp(s - s.max())
    mass = w[gpu_set].sum() / w.sum()
    ok_mass = mass >= p - MASS_SLACK if p < 1 else len(gpu_set) == len(s)
    if sel.select_all:
        near = np.zeros(len(diff), bool)
    else:
        near = np.abs(s[diff] - sel.edge()) <= sel.width
    return dict(n_ref=len(ref), n_gpu=len(gpu_set), n_diff=len(diff), n_far=int((~near).sum()),
                mass=float(mass), ok=bool(ok_mass and near.all()), bstar=sel.bstar)


def check_selection_topk(s, k, gpu_set: np.ndarray) -> dict:
    """Selection rule check for one retrieval head under the fixed-budget top-k selector:
    the same one-bin-width rule, and at least min(k, N) tokens."""
    sel = O.topk_histogram(s, k)
    ref = np.nonzero(sel.mask)[0]
    diff = np.setxor1d(ref, gpu_set)
    if sel.select_all:
        near = np.zeros(len(diff), bool)
    else:
        near = np.abs(s[diff] - sel.edge()) <= sel.width
    ok_count = len(gpu_set) >= min(int(k), len(s))
    return dict(n_ref=len(ref), n_gpu=len(gpu_set), n_diff=len(diff), n_far=int((~near).sum()),
                ok=bool(ok_count and near.all()), bstar=sel.bstar)


def run_layer_parity(workload_index=1, layer=0, p=None, check_sets=True, heads=None,
                     source="numpy", device="cuda", w=None, seq_lens=None, k=None) -> dict:
    """Builds one layer, appends all tokens, decodes once (top-p, or top-k when k is given)
    and compares with the oracle. Returns a report; raises AssertionError on a parity
    failure."""
    w = w if w is not None else workloads.workload(workload_index)
    p = w.p if p is None else p
    seq_lens = np.asarray(w.seq_lens if seq_lens is None else seq_lens, np.int64)
    q, wq, wk = layer_inputs(w, layer, device)
    lay = make_layer(w, layer, device, seq_lens)
    fill_layer(w, layer, lay, wk, seq_lens, source=source, device=device)
    out, cnt, sel = decode(lay, q, wq, seq_lens, p, device, with_sel=check_sets, k=k)
    st = lay.status()
    assert st == 0, f"device status {st}"
    report = check_outputs(w, layer, seq_lens, p, out, cnt, sel, heads, k=k)
    report["layer"] = lay
    return report


def check_outputs(w, layer, seq_lens, p, out, cnt, sel=None, heads=None, k=None) -> dict:
    """Compares one decode's outputs (device tensors) with the oracle under the rules above,
    for the (b, h) pairs in ``heads`` (every head when None). Raises AssertionError."""
    seq_lens = np.asarray(seq_lens, np.int64)
    out = out.float().cpu().numpy()
    cnt = cnt.cpu().numpy()
    sel = sel.cpu().numpy() if sel is not None else None
    qb = w.q_pre_bits(layer)
    wq_h, wk_h = w.w_qidx(layer), w.w_kidx(layer)
    pairs = heads if heads is not None else [(b, h) for b in range(w.B) for h in range(w.Hq)]
    report = dict(heads=[], max_abs=0.0, mean_abs=0.0, sel_far=0)
    cache = {}
    for (b, h) in pairs:
        g = h // w.G
        N = int(seq_lens[b])
        if (b, g) not in cache:
            cache[(b, g)] = (bits_to_f64(w.kpre_bits(layer, b, g, 0, N)),
                             bits_to_f64(w.v_bits(layer, b, g, 0, N)))
        kp, vv = cache[(b, g)]
        qpre = bits_to_f64(qb[b, h])
        entry = dict(b=b, h=h, retrieval=bool(w.ret_mask[layer, g]), count=int(cnt[b, h]))
        if w.ret_mask[layer, g]:
            kidx = O.index_keys(kp, wk_h[g])
            s = O.index_scores(O.index_query(qpre, wq_h[h]), kidx)
            if sel is not None:
                gset = sel[b, h, :cnt[b, h]].astype(np.int64)
                assert np.all(np.diff(gset) > 0), "sel_idx not ascending"
                assert gset.size == 0 or (gset[0] >= 0 and gset[-1] < N)
            else:
                gset = np.nonzero((O.topp_histogram(s, p) if k is None
                                   else O.topk_histogram(s, k)).mask)[0]
            chk = check_selection(s, p, gset) if k is None else check_selection_topk(s, k, gset)
            entry.update(chk)
            assert chk["ok"], f"selection parity failed at (b={b}, h={h}): {chk}"
            assert cnt[b, h] == len(gset)
            K = O.bf16_round(O.rope_rotate(kp[gset], gset, w.rope_base))
            ref = O.attend(O.rope_rotate(qpre, N - 1, w.rope_base), K, vv[gset])
        else:
            r = O.local_head(qpre, kp, vv, w.sinks, w.window, w.rope_base)
            ref = r.out
            assert cnt[b, h] == r.count, (cnt[b, h], r.count)
            if sel is not None:
                assert np.array_equal(sel[b, h, :r.count], r.sel)
        err = np.abs(out[b, h] - O.bf16_round(ref))      # both sides in the bf16 output format
        entry.update(max_abs=float(err.max()), mean_abs=float(err.mean()))
        report["max_abs"] = max(report["max_abs"], entry["max_abs"])
        report["mean_abs"] = max(report["mean_abs"], entry["mean_abs"])
        assert entry["max_abs"] <= MAX_ABS and entry["mean_abs"] <= MEAN_ABS, entry
        report["heads"].append(entry)
    return report


# ------------------------------------------------------------------------------ prefill
def prefill_inputs(w, layer, n_max, q_scale=1.0):
    """bf16 bits of a prompt at positions 0..n_max-1 of every sequence: q_pre
    [B][n_max][Hq][128] from the prompt-query streams, k_pre and v [B][n_max][Hkv][128] from
    the same streams the decode workloads use."""
    qb = np.zeros((w.B, n_max, w.Hq, 128), np.uint16)
    kb = np.zeros((w.B, n_max, w.Hkv, 128), np.uint16)
    vb = np.zeros_like(kb)
    for b in range(w.B):
        for h in range(w.Hq):
            qb[b, :, h] = w.prompt_q_bits(layer, b, h, 0, n_max, q_scale)
        for g in range(w.Hkv):
            kb[b, :, g] = w.kpre_bits(layer, b, g, 0, n_max)
            vb[b, :, g] = w.v_bits(layer, b, g, 0, n_max)
    return qb, kb, vb


def prefill(lay: DecodeLayer, qb, kb, vb, n_b, wk, device="cuda", sentinel=-7.0):
    """rtp_prefill through the layer (append of the prompt, then the prefill attention); out
    is pre-filled with ``sentinel`` so rows the call must not write can be checked."""
    B, n_max = qb.shape[0], qb.shape[1]
    q, k, v = (bits_to_torch(x, device) for x in (qb, kb, vb))
    out = torch.full((B, n_max, lay.Hq, 128), sentinel, dtype=torch.bfloat16, device=device)
    nb = torch.as_tensor(np.asarray(n_b, np.int32), device=device)
    lay.prefill(q, k, v, wk, nb, out)
    torch.cuda.synchronize()
    return out


def check_prefill(w, layer, n_b, qb, kb, vb, out, rows=None, heads=None,
                  sentinel=-7.0) -> dict:
    """Compares prefill outputs (device tensor [B][n_max][Hq][128]) with the oracle: every row
    m < n_b[b] (oracle prefill_head) or the sampled ``rows`` (the row's own oracle: dense
    attention over positions 0..m for a retrieval head, the sinks + window head with N = m + 1
    for a local one), in the bf16 output format under the decode rule (max-abs <= 1e-2,
    mean-abs <= 1e-3 per head); rows m >= n_b[b] must still hold the sentinel."""
    out = out.float().cpu().numpy()
    pairs = heads if heads is not None else [(b, h) for b in range(w.B) for h in range(w.Hq)]
    report = dict(max_abs=0.0, mean_abs=0.0, rows=0)
    krot = {}                # (b, g) -> the stored keys bf16(R(j) k_j) of a retrieval head
    for (b, h) in pairs:
        g = h // w.G
        N = int(n_b[b])
        local = not bool(w.ret_mask[layer, g])
        assert np.all(out[b, N:, h] == sentinel), f"rows >= n_b written at (b={b}, h={h})"
        if N == 0:
            continue
        q = bits_to_f64(qb[b, :N, h])
        k = bits_to_f64(kb[b, :N, g])
        v = bits_to_f64(vb[b, :N, g])
        if rows is None:
            ms = np.arange(N)
            ref = O.prefill_head(q, k, v, local, w.sinks, w.window, w.rope_base)
        else:
            ms = np.unique(np.clip(np.asarray(rows, np.int64), 0, N - 1))
            ref = np.zeros((ms.size, 128))
            for i, m in enumerate(ms):
                if local:
                    ref[i] = O.local_head(q[m], k[:m + 1], v[:m + 1], w.sinks, w.window,
                                          w.rope_base).out
                else:
                    if (b, g) not in krot:
                        krot[(b, g)] = O.bf16_round(O.rope_rotate(k, np.arange(N), w.rope_base))
                    K = krot[(b, g)][:m + 1]
                    ref[i] = O.attend(O.rope_rotate(q[m], m, w.rope_base), K, v[:m + 1])
        err = np.abs(out[b, ms, h] - O.bf16_round(ref))
        mx, mn = float(err.max()), float(err.mean())
        report["max_abs"] = max(report["max_abs"], mx)
        report["mean_abs"] = max(report["mean_abs"], mn)
        report["rows"] += int(ms.size)
        assert mx <= MAX_ABS and mn <= MEAN_ABS, dict(b=b, h=h, local=local, max_abs=mx,
                                                      mean_abs=mn)
    return report
