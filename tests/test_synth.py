"""The seeded input generator: determinism, distribution and planted structure (CPU)."""
import numpy as np
import torch

from synth import gen, workloads


def test_mix64_known_values():
    """splitmix64 with state 0: the first outputs of the published generator."""
    state = 0
    outs = []
    for _ in range(3):
        state = (state + 0x9E3779B97F4A7C15) & ((1 << 64) - 1)
        outs.append(int(gen.mix64(np.uint64(state))))
    assert outs == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_stream_is_counter_addressable_and_deterministic():
    key = gen.stream_key(3, gen.T_KPRE, 5, 1, 2)
    a = gen.normal_f32(key, np.arange(1000))
    b = gen.normal_f32(key, np.arange(500, 1000))
    np.testing.assert_array_equal(a[500:], b)
    assert gen.stream_key(3, gen.T_KPRE, 5, 1, 2) != gen.stream_key(3, gen.T_KPRE, 5, 1, 3)


def test_normal_moments():
    x = gen.normal_f32(gen.stream_key(0, 1), np.arange(1 << 20)).astype(np.float64)
    assert abs(x.mean()) < 5e-3
    assert abs(x.var() - 1.0) < 5e-3
    assert np.abs(x).max() < 3.47


def test_bf16_bits_match_torch():
    x = gen.normal_f32(gen.stream_key(1, 2), np.arange(100000)) * np.float32(7.3)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(gen.f32_to_bf16_bits(x), ref)


def test_planted_shift_moves_projection():
    w = workloads.workload(1)
    lay = w.group_layout(0, 0, 0)
    c = lay.clusters[0]
    W = w.w_kidx(0)[0].astype(np.float64)
    np.testing.assert_allclose(W.T @ c.delta.astype(np.float64),
                               c.strength * np.sqrt(c.u @ W.T @ W @ c.u) * c.u, atol=1e-4)
    rows = gen.bf16_bits_to_f32(w.kpre_bits(0, 0, 0, c.start, c.start + c.length))
    base = gen.bf16_bits_to_f32(gen.token_rows_bits(gen.stream_key(w.seed, gen.T_KPRE, 0, 0, 0),
                                                    c.start, c.start + c.length, 128))
    shift = (rows.astype(np.float64) - base) @ W
    np.testing.assert_allclose(shift.mean(0), W.T @ c.delta, atol=0.05)


def test_query_projection_hits_target():
    w = workloads.workload(2)
    layer = int(np.nonzero(w.ret_mask.any(1))[0][0])
    qb = w.q_pre_bits(layer)
    for h in range(w.Hq):
        tgt = w.q_target(layer, 0, h)
        if tgt is None:
            continue
        q = gen.bf16_bits_to_f32(qb[0, h]).astype(np.float64)
        got = q @ w.w_qidx(layer)[h].astype(np.float64)
        assert np.linalg.norm(got - tgt) < 0.05 * np.linalg.norm(tgt)


def test_workload_shapes():
    for i in range(1, 6):
        w = workloads.workload(i)
        assert w.Hq % w.Hkv == 0
        if i > 1:
            assert w.ret_mask.sum() == 43 and w.ret_mask.shape == (36, 8)
    w5 = workloads.workload(5)
    assert w5.seq_lens.min() >= 8192 and w5.seq_lens.max() <= 65536 and len(w5.seq_lens) == 64


def test_topk_vs_topp_budget_on_the_32k_workload():
    """The comparison the pages draw between a fixed top-k budget and top-p (oracle only, one
    32K layer with two retrieval groups, every query head): with k equal to the mean top-p
    budget, the concentrated heads keep more than p of their mass and at least one diffuse
    head keeps less; giving every head at least p needs k = the largest top-p set, which
    spends more tokens in total than top-p does."""
    from oracle import rtp_oracle as O
    w = workloads.workload(2)
    layer = int(np.nonzero(w.ret_mask.sum(1) >= 2)[0][0])
    N = int(w.seq_lens[0])
    qb = w.q_pre_bits(layer)
    rows = []
    for g in np.nonzero(w.ret_mask[layer])[0]:
        kp = gen.bf16_bits_to_f32(w.kpre_bits(layer, 0, int(g), 0, N)).astype(np.float64)
        kidx = O.index_keys(kp, w.w_kidx(layer)[g])
        for h in range(g * w.G, (g + 1) * w.G):
            q = gen.bf16_bits_to_f32(qb[0, h]).astype(np.float64)
            s = O.index_scores(O.index_query(q, w.w_qidx(layer)[h]), kidx)
            kind = w.group_layout(layer, 0, int(g)).targets[h % w.G][0]
            rows.append((kind, s, int(O.topp_histogram(s, w.p).mask.sum())))
    mean_budget = int(round(np.mean([r[2] for r in rows])))
    mass = lambda s, m: float(np.exp(s - s.max())[m].sum() / np.exp(s - s.max()).sum())
    conc = [mass(s, O.topk_exact(s, mean_budget)) for kind, s, _ in rows if kind == "conc"]
    diff = [mass(s, O.topk_exact(s, mean_budget)) for kind, s, _ in rows if kind == "diff"]
    assert conc and diff
    assert min(conc) > w.p and min(diff) < w.p
    k_all = max(r[2] for r in rows)
    assert len(rows) * k_all > sum(r[2] for r in rows)


def test_cluster_prefilter_keeps_the_top_p_set_on_the_32k_workload():
    """The centroid pre-filter of RTPurboV2 (oracle only, K = 128 clusters of one retrieval KV
    head's index keys at 32K, cluster-level top-p at p = 0.9): a concentrated head hits a small
    share of the tokens yet keeps almost all of its token-level top-p set; a diffuse head hits
    more and still keeps most of it. The numbers are reported in the design notes."""
    from oracle import rtp_oracle as O
    w = workloads.workload(2)
    layer = next(l for l in range(w.layers) if w.ret_mask[l].sum() >= 1)
    g = int(np.nonzero(w.ret_mask[layer])[0][0])
    N = int(w.seq_lens[0])
    kp = gen.bf16_bits_to_f32(w.kpre_bits(layer, 0, g, 0, N)).astype(np.float64)
    kidx = O.index_keys(kp, w.w_kidx(layer)[g])
    mu, assign = O.kmeans_index_keys(kidx, 128, iters=10)
    qb = w.q_pre_bits(layer)
    seen = set()
    for h in range(g * w.G, (g + 1) * w.G):
        q_idx = O.index_query(gen.bf16_bits_to_f32(qb[0, h]).astype(np.float64),
                              w.w_qidx(layer)[h])
        v1 = O.topp_histogram(O.index_scores(q_idx, kidx), w.p).mask
        hit = O.cluster_select(q_idx, mu, assign, w.p)
        recall = v1[hit].sum() / v1.sum()
        kind = w.group_layout(layer, 0, g).targets[h % w.G][0]
        seen.add(kind)
        if kind == "conc":
            assert hit.mean() < 0.1 and recall > 0.95, (hit.mean(), recall)
        else:
            assert hit.mean() < 0.5 and recall > 0.85, (hit.mean(), recall)
    assert seen == {"conc", "diff"}
