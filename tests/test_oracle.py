"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a library routine, exact
rational arithmetic, a closed form, an invariant of the definition, or brute force.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import rtp_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- bf16 rounding
def _bf16_exact(x: float) -> float:
    """Round-to-nearest-even to 8 significant bits with exact rationals."""
    if x == 0 or not math.isfinite(x):
        return x
    f = Fraction(x)
    sign = -1 if f < 0 else 1
    a = abs(f)
    e = 0
    while a >= 2:
        a /= 2
        e += 1
    while a < 1:
        a *= 2
        e -= 1
    e = max(e, -126)                       # subnormal spacing 2^-133
    q = Fraction(2) ** (e - 7)
    n = abs(f) / q
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * float(fl * q)


def test_bf16_round_matches_torch_on_float32_inputs():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
                        rng.standard_normal(1000) * 1e-39]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.bf16_round(x.astype(np.float64)), ref)


def test_bf16_round_matches_exact_rationals_on_float64_inputs():
    rng = np.random.default_rng(1)
    xs = list(rng.standard_normal(3000) * 10.0 ** rng.integers(-12, 12, 3000))
    # exact ties: odd multiples of half a bf16 spacing
    for k in range(1, 200, 2):
        xs.append(1.0 + k * 2.0 ** -8)
        xs.append(-(3.0 + k * 2.0 ** -7))
    xs += [2.0 ** -130 * 1.37, -(2.0 ** -128) * 1.5]     # bf16 subnormal range
    got = O.bf16_round(np.array(xs))
    for x, g in zip(xs, got):
        assert g == _bf16_exact(float(x)), x


# ----------------------------------------------------------------------------- RoPE, eq. (1)-(2)
def test_rope_theta_decreasing_and_endpoints():
    th = O.rope_theta(128, 1e6)
    assert th[0] == 1.0
    assert np.all(np.diff(th) < 0)
    assert math.isclose(th[-1], 1e6 ** (-126 / 128), rel_tol=1e-15)


def test_rope_matches_complex_rotation():
    """Each pair (i, i+64) is the complex number x_i + j x_{i+64} times exp(j m theta_i)."""
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 128))
    pos = np.array([0, 1, 17, 4095, 1048575])
    th = 1e6 ** (-np.arange(64) * 2.0 / 128)
    z = (x[:, :64] + 1j * x[:, 64:]) * np.exp(1j * pos[:, None] * th[None, :])
    ref = np.concatenate([z.real, z.imag], axis=1)
    np.testing.assert_allclose(O.rope_rotate(x, pos), ref, rtol=0, atol=1e-12)


def test_rope_identity_and_orthogonality():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((7, 128))
    np.testing.assert_array_equal(O.rope_rotate(x, np.zeros(7)), x)
    y = O.rope_rotate(x, np.arange(7) * 1000 + 5)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)


def test_rope_score_depends_only_on_offset_eq2():
    """Eq. (2): q_m^T k_n = sum_i [a_i cos(theta_i D) + b_i sin(theta_i D)], D = m - n."""
    rng = np.random.default_rng(4)
    q, k = rng.standard_normal(128), rng.standard_normal(128)
    th = O.rope_theta(128, 1e6)
    qa, qb, ka, kb = q[:64], q[64:], k[:64], k[64:]
    a = qa * ka + qb * kb
    b = qa * kb - qb * ka
    for m, n in [(10, 3), (5000, 4999), (1_000_000, 123), (77, 77)]:
        got = O.rope_rotate(q, m) @ O.rope_rotate(k, n)
        closed = np.sum(a * np.cos(th * (m - n)) + b * np.sin(th * (m - n)))
        assert abs(got - closed) < 1e-9 * np.linalg.norm(q) * np.linalg.norm(k)
        for c in (1, 1000, 65536):
            sh = O.rope_rotate(q, m + c) @ O.rope_rotate(k, n + c)
            assert abs(sh - got) < 1e-9 * np.linalg.norm(q) * np.linalg.norm(k)


# ----------------------------------------------------------------------------- eq. (4)
def test_index_keys_selector_weight_reduces_to_columns():
    """With W^K = [I_16; 0] the projection of a bf16 key is its first 16 channels, exactly."""
    rng = np.random.default_rng(5)
    k = O.bf16_round(rng.standard_normal((50, 128)))
    W = np.zeros((128, 16))
    W[:16, :16] = np.eye(16)
    np.testing.assert_array_equal(O.index_keys(k, W), k[:, :16])
    # a permuting selector catches a transposed operand
    W2 = np.zeros((128, 16))
    perm = rng.permutation(128)[:16]
    W2[perm, np.arange(16)] = 1.0
    np.testing.assert_array_equal(O.index_keys(k, W2), k[:, perm])


def test_index_scores_match_torch_and_bilinear_form():
    """s = (W^Q q)^T (W^K k) equals q^T (W^Q^T W^K) k before rounding and torch's matmul."""
    rng = np.random.default_rng(6)
    q = rng.standard_normal(128)
    k = rng.standard_normal((40, 128))
    Wq = rng.standard_normal((128, 16)) / 11.3
    Wk = rng.standard_normal((128, 16)) / 11.3
    s = O.index_scores(O.index_query(q, Wq), k @ Wk)
    bil = k @ (Wk @ Wq.T) @ q
    np.testing.assert_allclose(s, bil, rtol=1e-12, atol=1e-12)
    tq = torch.from_numpy(q) @ torch.from_numpy(Wq)
    tk = torch.from_numpy(k) @ torch.from_numpy(Wk)
    np.testing.assert_allclose(s, (tk @ tq).numpy(), rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------- eq. (5): Top-P
def test_topp_hand_worked_example():
    """Scores {0, 0, ln2, ln8}: masses {1/8, 1/8, 1/4, 1}, T = 3/2; bins 0, 0, 85, 255
    (256 ln2/ln8 = 85.33). p=0.9 -> C_0 = 1.5 >= 1.35 is the first bin from the top that
    reaches pT, so b* = 0 (all); p=0.8 -> C_85 = 1.25 >= 1.2 -> {2, 3}; p=0.6 -> C_255 = 1 ->
    {3}."""
    s = np.array([0.0, 0.0, math.log(2.0), math.log(8.0)])
    sel = O.topp_histogram(s, 0.9)
    assert list(sel.bins) == [0, 0, 85, 255]
    np.testing.assert_allclose(sel.T, 1.5, rtol=1e-15)
    assert sel.bstar == 0 and sel.mask.all()
    sel = O.topp_histogram(s, 0.8)
    assert sel.bstar == 85 and list(np.nonzero(sel.mask)[0]) == [2, 3]
    sel = O.topp_histogram(s, 0.6)
    assert sel.bstar == 255 and list(np.nonzero(sel.mask)[0]) == [3]
    assert list(np.nonzero(O.topp_exact(s, 0.8))[0]) == [2, 3]
    assert list(np.nonzero(O.topp_exact(s, 0.6))[0]) == [3]


def _brute_minimal_set(s, p):
    """Minimal-cardinality subsets with mass >= p * total, by enumeration."""
    w = np.exp(s - s.max())
    T = w.sum()
    N = len(s)
    for k in range(1, N + 1):
        best = None
        for comb in itertools.combinations(range(N), k):
            m = w[list(comb)].sum()
            if m >= p * T and (best is None or m > best[0]):
                best = (m, comb)
        if best is not None:
            return k, best[0]
    return N, T


@pytest.mark.parametrize("seed", range(12))
def test_topp_exact_is_minimal_set_by_enumeration(seed):
    rng = np.random.default_rng(100 + seed)
    N = int(rng.integers(1, 13))
    s = rng.standard_normal(N) * rng.uniform(0.1, 4.0)
    p = float(rng.uniform(0.3, 0.99))
    k, best_mass = _brute_minimal_set(s, p)
    ex = O.topp_exact(s, p)
    assert ex.sum() == k
    w = np.exp(s - s.max())
    assert math.isclose(w[ex].sum(), best_mass, rel_tol=1e-12)


@pytest.mark.parametrize("seed", range(40))
def test_topp_histogram_invariants(seed):
    """S_exact is a subset of S; extra tokens all sit in bin b*; mass(S) >= p; bins above b*
    hold less than p of the mass (b* is maximal); exact top-p agrees with a full sort."""
    rng = np.random.default_rng(200 + seed)
    N = int(rng.integers(2, 5000 if seed % 4 == 0 else 64))
    s = rng.standard_normal(N) * rng.uniform(0.2, 6.0)
    if seed % 5 == 1:                                     # a planted run
        s[: max(1, N // 20)] += rng.uniform(2, 8)
    if seed % 7 == 2:                                     # heavy ties
        s = np.round(s)
    p = float(rng.choice([0.5, 0.8, 0.9, 0.95, 0.99]))
    sel = O.topp_histogram(s, p)
    ex = O.topp_exact(s, p)
    w = np.exp(s - s.max())
    T = w.sum()
    assert np.all(sel.mask[ex])
    extra = sel.mask & ~ex
    if not sel.select_all:
        assert np.all(sel.bins[extra] == sel.bstar)
        above = w[sel.bins > sel.bstar].sum()
        assert above < p * T * (1 + 1e-12)
    assert w[sel.mask].sum() >= p * T * (1 - 1e-12)
    # the exact set is a prefix of the order by (score desc, index asc)
    order = np.lexsort((np.arange(N), -s))
    k = int(ex.sum())
    assert set(order[:k]) == set(np.nonzero(ex)[0])
    assert w[order[: k - 1]].sum() < p * T * (1 + 1e-12) or k == 1


def test_topp_special_cases():
    s = np.full(10, 3.25)
    assert O.topp_histogram(s, 0.9).mask.all()            # all scores equal -> all
    rng = np.random.default_rng(7)
    s = rng.standard_normal(100)
    assert O.topp_histogram(s, 1.0).mask.all()            # p >= 1 -> all
    assert O.topp_exact(s, 1.0).all()
    s = np.zeros(100)
    s[37] = 100.0                                          # one dominant token -> its bin only
    sel = O.topp_histogram(s, 0.9)
    assert sel.bstar == 255 and list(np.nonzero(sel.mask)[0]) == [37]
    sel = O.topp_histogram(np.array([1.5]), 0.9)           # N = 1
    assert sel.mask.all()
    with pytest.raises(ValueError):
        O.topp_histogram(np.array([]), 0.9)


def test_topk_hand_worked_example():
    """Scores {0, 1, 2, 3}: bins 0, 85, 170, 255 (256 / 3 = 85.33); counts from the top 1, 2,
    3, 4, so k = 1 -> b* = 255 {3}; k = 2 -> 170 {2, 3}; k = 3 -> 85 {1, 2, 3}. Scores
    {0, 10, 10.01, 10.02}: the three high scores share bin 255 (256 * 10 / 10.02 = 255.49),
    so k = 2 keeps all three (the extra token sits in the threshold bin)."""
    s = np.array([0.0, 1.0, 2.0, 3.0])
    for k, bstar, want in ((1, 255, [3]), (2, 170, [2, 3]), (3, 85, [1, 2, 3])):
        sel = O.topk_histogram(s, k)
        assert list(sel.bins) == [0, 85, 170, 255]
        assert sel.bstar == bstar and list(np.nonzero(sel.mask)[0]) == want
        assert list(np.nonzero(O.topk_exact(s, k))[0]) == want
    s = np.array([0.0, 10.0, 10.01, 10.02])
    sel = O.topk_histogram(s, 2)
    assert sel.bstar == 255 and list(np.nonzero(sel.mask)[0]) == [1, 2, 3]
    assert list(np.nonzero(O.topk_exact(s, 2))[0]) == [2, 3]


@pytest.mark.parametrize("seed", range(12))
def test_topk_contains_a_top_k_set_by_enumeration(seed):
    """Every k-subset whose scores are all >= the scores outside it is a valid top-k; the
    histogram set contains one of them and its other tokens lie in bin b*."""
    rng = np.random.default_rng(300 + seed)
    N = int(rng.integers(2, 11))
    s = rng.standard_normal(N) * rng.uniform(0.1, 4.0)
    if seed % 3 == 0:
        s = np.round(s, 1)                                  # ties
    k = int(rng.integers(1, N))
    sel = O.topk_histogram(s, k)
    valid = [set(c) for c in itertools.combinations(range(N), k)
             if min(s[list(c)]) >= max(np.delete(s, list(c)), default=-np.inf)]
    got = set(np.nonzero(sel.mask)[0])
    assert valid and any(c <= got for c in valid)
    c = next(c for c in valid if c <= got)
    assert all(sel.bins[n] == sel.bstar for n in got - c)
    assert set(np.nonzero(O.topk_exact(s, k))[0]) in valid


@pytest.mark.parametrize("seed", range(30))
def test_topk_histogram_invariants(seed):
    """|S| >= k; bins above b* hold fewer than k tokens (b* maximal); b* is the bin of the
    k-th highest score; the sorted top-k is a subset and the extras sit in bin b*."""
    rng = np.random.default_rng(400 + seed)
    N = int(rng.integers(2, 5000 if seed % 3 == 0 else 80))
    s = rng.standard_normal(N) * rng.uniform(0.2, 6.0)
    if seed % 5 == 1:
        s[: max(1, N // 20)] += rng.uniform(2, 8)
    if seed % 7 == 2:
        s = np.round(s)
    k = int(rng.integers(1, N + 1))
    sel = O.topk_histogram(s, k)
    ex = O.topk_exact(s, k)
    assert sel.mask.sum() >= k
    assert np.all(sel.mask[ex])
    if not sel.select_all:
        assert (sel.bins > sel.bstar).sum() < k
        kth = np.sort(s)[::-1][k - 1]
        assert sel.bstar == O.score_bins(np.array([kth]), sel.lo, sel.hi)[0]
        assert np.all(sel.bins[sel.mask & ~ex] == sel.bstar)


def test_topk_special_cases():
    rng = np.random.default_rng(9)
    s = rng.standard_normal(50)
    assert O.topk_histogram(s, 50).mask.all()              # k = N -> all
    assert O.topk_histogram(s, 80).mask.all()              # k > N -> all
    assert O.topk_histogram(np.full(10, 1.5), 3).mask.all()   # all scores equal -> all
    assert O.topk_histogram(np.array([2.0]), 1).mask.all()     # N = 1
    with pytest.raises(ValueError):
        O.topk_histogram(s, 0)
    with pytest.raises(ValueError):
        O.topk_histogram(np.array([]), 1)


def test_bins_linear_over_min_max():
    s = np.linspace(-3.0, 5.0, 257)                        # exactly on the 256 bin edges
    b = O.score_bins(s, -3.0, 5.0)
    assert b[0] == 0 and b[-1] == 255
    assert np.all(b[:-1] == np.arange(256))


# ----------------------------------------------------------------------------- attention
def _rope_complex(x, pos, base=1e6):
    th = base ** (-np.arange(64) * 2.0 / 128)
    z = (x[..., :64] + 1j * x[..., 64:]) * np.exp(1j * np.asarray(pos)[..., None] * th)
    return np.concatenate([z.real, z.imag], axis=-1)


def test_attend_matches_torch_sdpa():
    rng = np.random.default_rng(8)
    q = rng.standard_normal(128)
    K = rng.standard_normal((300, 128))
    V = rng.standard_normal((300, 128))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None, None, :], torch.from_numpy(K)[None, None],
        torch.from_numpy(V)[None, None])[0, 0, 0].numpy()
    np.testing.assert_allclose(O.attend(q, K, V), ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(O.attend(q, K[3:4], V[3:4]), V[3])


def test_layer_reduces_to_dense_attention():
    """p = 1 (retrieval) and window >= N (local) make the layer dense softmax attention over all
    N RoPE'd, bf16-stored keys; compared with torch SDPA and a complex-number RoPE."""
    rng = np.random.default_rng(9)
    B, Hq, Hkv, N = 2, 4, 2, 300
    q_pre = O.bf16_round(rng.standard_normal((B, Hq, 128)))
    kp = O.bf16_round(rng.standard_normal((B, Hkv, N, 128)))
    vv = O.bf16_round(rng.standard_normal((B, Hkv, N, 128)))
    wq = rng.standard_normal((Hq, 128, 16)) / 11.3
    wk = rng.standard_normal((Hkv, 128, 16)) / 11.3
    res = O.decode_layer(q_pre, wq, wk, lambda b, g: kp[b, g], lambda b, g: vv[b, g],
                         np.array([True, False]), [N, N], 1.0, sinks=4, window=N)
    for b in range(B):
        for h in range(Hq):
            g = h // 2
            K = O.bf16_round(_rope_complex(kp[b, g], np.arange(N)))
            q = _rope_complex(q_pre[b, h], N - 1)
            ref = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(q)[None, None, None], torch.from_numpy(K)[None, None],
                torch.from_numpy(vv[b, g])[None, None])[0, 0, 0].numpy()
            np.testing.assert_allclose(res[(b, h)].out, ref, rtol=1e-10, atol=1e-12)
            assert res[(b, h)].count == N


def test_local_positions_bruteforce():
    for N in range(1, 40):
        for sinks in range(0, 6):
            for window in range(1, 12):
                ref = [n for n in range(N) if n < sinks or n >= N - window]
                got = O.local_positions(N, sinks, window)
                assert list(got) == ref, (N, sinks, window)


def test_single_token_cache():
    """N = 1: the only token is selected and the output is its value row."""
    rng = np.random.default_rng(10)
    kp = O.bf16_round(rng.standard_normal((1, 128)))
    vv = O.bf16_round(rng.standard_normal((1, 128)))
    r = O.retrieval_head(rng.standard_normal(128), rng.standard_normal((128, 16)), kp, vv,
                         rng.standard_normal((128, 16)), 0.9)
    assert r.count == 1
    np.testing.assert_array_equal(r.out, vv[0])
    r = O.local_head(rng.standard_normal(128), kp, vv, 4, 256)
    np.testing.assert_array_equal(r.out, vv[0])


def test_page_constants():
    """Constants the pages fix: r = 16, p = 0.9, 256 bins of fp32 mass = 1 KB per head."""
    with open(os.path.join(GOLDEN, "page_constants.json")) as f:
        c = json.load(f)
    assert c["idx_dim"] == O.IDX_DIM
    assert c["n_bins"] == O.N_BINS
    assert c["hist_bytes_per_head"] == O.N_BINS * 4
    assert c["top_p"] == 0.9


def _bf_rope(x, m, base=1e6):
    """R(m) x with plain floats: channel pairs (i, i + 64), angle m * base^(-2i/128)."""
    out = [0.0] * 128
    for i in range(64):
        ang = m * base ** (-2.0 * i / 128)
        c, s = math.cos(ang), math.sin(ang)
        out[i] = x[i] * c - x[i + 64] * s
        out[i + 64] = x[i] * s + x[i + 64] * c
    return out


def _bf_head(q, kp, vv, wq, wk, p, retrieval, sinks, window):
    """One query head from the definitions, with loops: scores, the 256-bin rule, softmax."""
    N = len(kp)
    bf = lambda vals: [float(x) for x in O.bf16_round(np.array(vals))]
    if retrieval:
        qi = [sum(q[d] * wq[d][j] for d in range(128)) for j in range(16)]
        ki = [bf([sum(kp[n][d] * wk[d][j] for d in range(128)) for j in range(16)])
              for n in range(N)]
        s = [sum(qi[j] * ki[n][j] for j in range(16)) for n in range(N)]
        lo, hi = min(s), max(s)
        if p >= 1.0 or hi == lo:
            sel = list(range(N))
        else:
            bins = [min(255, math.floor((x - lo) * 256 / (hi - lo))) for x in s]
            mass = [0.0] * 256
            for n in range(N):
                mass[bins[n]] += math.exp(s[n] - hi)
            suffix, acc = [0.0] * 256, 0.0
            for b in range(255, -1, -1):
                acc += mass[b]
                suffix[b] = acc
            bstar = max(b for b in range(256) if suffix[b] >= p * suffix[0])
            sel = [n for n in range(N) if bins[n] >= bstar]
    else:
        sel = sorted(set(range(min(sinks, N))) | set(range(max(0, N - window), N)))
    qr = _bf_rope(q, N - 1)
    z = []
    for n in sel:
        k = bf(_bf_rope(kp[n], n))
        z.append(sum(qr[d] * k[d] for d in range(128)) / math.sqrt(128))
    zmax = max(z)
    w = [math.exp(x - zmax) for x in z]
    out = [sum(w[i] * vv[n][d] for i, n in enumerate(sel)) / sum(w) for d in range(128)]
    return out, sel


@pytest.mark.parametrize("seed", range(4))
def test_decode_layer_bruteforce_tiny(seed):
    """The whole layer (two retrieval KV heads and one local, G = 2, two sequences, N <= 64)
    against a loop-by-loop evaluation of the definitions: query head h reads KV head h // G,
    selected keys are rotated by their own positions, the query by N - 1."""
    rng = np.random.default_rng(100 + seed)
    B, Hkv, G, sinks, window = 2, 3, 2, 2, 5
    Hq = Hkv * G
    ret = [True, False, True]
    lens = [int(rng.choice([1, 3, 8, 33, 64])), int(rng.choice([2, 6, 19, 64]))]
    p = [0.5, 0.9, 0.99, 1.0][seed]
    r16 = lambda a: O.bf16_round(a)
    q = r16(rng.standard_normal((B, Hq, 128)) * 1.5)
    wq = rng.standard_normal((Hq, 128, 16)) / np.sqrt(128)
    wk = rng.standard_normal((Hkv, 128, 16)) / np.sqrt(128)
    kp = {(b, g): r16(rng.standard_normal((lens[b], 128))) for b in range(B) for g in range(Hkv)}
    vv = {(b, g): r16(rng.standard_normal((lens[b], 128))) for b in range(B) for g in range(Hkv)}
    res = O.decode_layer(q, wq, wk, lambda b, g: kp[(b, g)], lambda b, g: vv[(b, g)],
                         np.array(ret), np.array(lens), p, sinks, window)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            out, sel = _bf_head(q[b, h].tolist(), kp[(b, g)].tolist(), vv[(b, g)].tolist(),
                                wq[h].tolist(), wk[g].tolist(), p, ret[g], sinks, window)
            r = res[(b, h)]
            assert r.count == len(sel)
            assert list(r.sel) == sel
            np.testing.assert_allclose(r.out, out, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- retained mass
def _mass_case(seed, N):
    rng = np.random.default_rng(300 + seed)
    q = O.bf16_round(rng.standard_normal(128) * 2.0)
    kp = O.bf16_round(rng.standard_normal((N, 128)))
    return rng, q, kp


def test_full_attention_mass_of_every_position_is_one():
    _, q, kp = _mass_case(0, 500)
    assert abs(O.full_attention_mass(q, kp, np.arange(500)) - 1.0) < 1e-14
    assert O.full_attention_mass(q, kp, np.array([], np.int64)) == 0.0


def test_full_attention_mass_matches_torch_softmax_weights():
    """The dense attention weights from torch's softmax over the complex-RoPE'd, bf16-stored
    keys, summed over the subset (and its complement summing to the rest)."""
    rng, q, kp = _mass_case(1, 700)
    N = 700
    K = O.bf16_round(_rope_complex(kp, np.arange(N)))
    qr = _rope_complex(q, N - 1)
    wts = torch.softmax(torch.from_numpy(K) @ torch.from_numpy(qr) / math.sqrt(128), dim=0).numpy()
    sub = np.sort(rng.choice(N, size=90, replace=False))
    rest = np.setdiff1d(np.arange(N), sub)
    got = O.full_attention_mass(q, kp, sub)
    assert abs(got - wts[sub].sum()) < 1e-12
    assert abs(got + O.full_attention_mass(q, kp, rest) - 1.0) < 1e-12


@pytest.mark.parametrize("N", [1, 5, 33, 64])
def test_full_attention_mass_bruteforce_tiny(N):
    """Loop-by-loop evaluation of the definition: keys rotated by their own positions and
    stored in bf16, the query rotated by N - 1, weights exp(q.k / sqrt(128)) normalised over
    all N tokens, summed over the subset."""
    rng, q, kp = _mass_case(2 + N, N)
    sub = sorted(set(int(x) for x in rng.integers(0, N, size=max(1, N // 3))))
    qr = _bf_rope(q.tolist(), N - 1)
    z = []
    for n in range(N):
        k = [float(x) for x in O.bf16_round(np.array(_bf_rope(kp[n].tolist(), n)))]
        z.append(sum(qr[d] * k[d] for d in range(128)) / math.sqrt(128))
    zmax = max(z)
    w = [math.exp(x - zmax) for x in z]
    ref = sum(w[n] for n in sub) / sum(w)
    assert abs(O.full_attention_mass(q, kp, np.array(sub)) - ref) < 1e-12


# ----------------------------------------------------------------------------- prefill (f1)
def test_prefill_retrieval_matches_torch_causal_sdpa():
    """Dense causal prefill against torch SDPA (is_causal) on the same RoPE'd inputs."""
    rng = np.random.default_rng(11)
    n = 48
    q = rng.standard_normal((n, 128))
    k = rng.standard_normal((n, 128))
    v = rng.standard_normal((n, 128))
    got = O.prefill_head(q, k, v, False, 4, 16)
    pos = np.arange(n)
    Q = torch.from_numpy(_rope_complex(q, pos))
    K = torch.from_numpy(O.bf16_round(_rope_complex(k, pos)))
    ref = torch.nn.functional.scaled_dot_product_attention(
        Q[None, None], K[None, None], torch.from_numpy(v)[None, None], is_causal=True)[0, 0]
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-10, atol=1e-12)


def test_prefill_local_matches_sdpa_with_a_position_mask():
    """Sinks + window prefill against torch SDPA with a boolean mask built row by row from
    the pinned decode-time position sets (query m sees local_positions(m + 1))."""
    rng = np.random.default_rng(12)
    n, sinks, window = 40, 3, 7
    q = rng.standard_normal((n, 128))
    k = rng.standard_normal((n, 128))
    v = rng.standard_normal((n, 128))
    got = O.prefill_head(q, k, v, True, sinks, window)
    mask = np.zeros((n, n), bool)
    for m in range(n):
        mask[m, O.local_positions(m + 1, sinks, window)] = True
    pos = np.arange(n)
    Q = torch.from_numpy(_rope_complex(q, pos))
    K = torch.from_numpy(O.bf16_round(_rope_complex(k, pos)))
    ref = torch.nn.functional.scaled_dot_product_attention(
        Q[None, None], K[None, None], torch.from_numpy(v)[None, None],
        attn_mask=torch.from_numpy(mask)[None, None])[0, 0]
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("local", [False, True])
def test_prefill_rows_equal_the_decode_step(local):
    """Row m of a prefill equals the decode-step attention with N = m + 1 (dense attention
    for a retrieval head at p = 1, the sinks + window head for a local one): two oracle
    paths for the same quantity."""
    rng = np.random.default_rng(13 + int(local))
    n, sinks, window = 30, 2, 5
    q = rng.standard_normal((n, 128))
    k = rng.standard_normal((n, 128))
    v = rng.standard_normal((n, 128))
    got = O.prefill_head(q, k, v, local, sinks, window)
    for m in range(n):
        if local:
            ref = O.local_head(q[m], k[: m + 1], v[: m + 1], sinks, window).out
        else:
            pos = np.arange(m + 1)
            ref = O.attend(O.rope_rotate(q[m], m), O.bf16_round(O.rope_rotate(k[: m + 1], pos)),
                           v[: m + 1])
        np.testing.assert_allclose(got[m], ref, rtol=1e-10, atol=1e-12)


# ------------------------------------------------------------- centroid pre-filter (f3)
def _blobs(rng, n_blobs, per, r=16, spread=0.05):
    centres = rng.standard_normal((n_blobs, r)) * 3.0
    x = np.concatenate([c + spread * rng.standard_normal((per, r)) for c in centres])
    return x[rng.permutation(x.shape[0])]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_kmeans_matches_sklearn_lloyd_from_the_same_start(seed):
    """The k-means of the index keys against scikit-learn's Lloyd k-means started from the same
    centroids (positions floor(i N / K)), run to convergence: the same clusters and centroids."""
    from sklearn.cluster import KMeans
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((300, 16))
    K = 12
    mu, assign = O.kmeans_index_keys(x, K, iters=300)
    init = x[(np.arange(K) * 300) // K]
    km = KMeans(n_clusters=K, init=init, n_init=1, algorithm="lloyd", max_iter=300, tol=0.0)
    km.fit(x)
    assert np.array_equal(assign, km.labels_)
    np.testing.assert_allclose(mu, km.cluster_centers_, rtol=1e-10, atol=1e-12)


def test_kmeans_fixed_point_and_separated_blobs():
    """At convergence every key sits in its nearest centroid's cluster and every centroid is
    the mean of its keys. Runs of consecutive tokens drawn around separated centres (one run
    per initial position floor(i N / K)) come out as exactly the runs."""
    rng = np.random.default_rng(4)
    x = _blobs(rng, 8, 40)
    mu, assign = O.kmeans_index_keys(x, 8, iters=100)
    d = ((x[:, None, :] - mu[None]) ** 2).sum(axis=2)
    assert np.array_equal(d.argmin(axis=1), assign)
    for k in range(8):
        np.testing.assert_allclose(mu[k], x[assign == k].mean(axis=0), rtol=0, atol=1e-12)
    centres = rng.standard_normal((8, 16)) * 3.0
    runs = np.concatenate([c + 0.05 * rng.standard_normal((40, 16)) for c in centres])
    mu, assign = O.kmeans_index_keys(runs, 8, iters=100)
    assert np.array_equal(assign, np.arange(320) // 40)
    np.testing.assert_allclose(mu, runs.reshape(8, 40, 16).mean(axis=1), rtol=0, atol=1e-12)


def test_kmeans_clamps_k_and_keeps_empty_centroids():
    x = np.arange(5 * 16, dtype=np.float64).reshape(5, 16)
    mu, assign = O.kmeans_index_keys(x, 128, iters=5)
    assert mu.shape == (5, 16) and np.array_equal(assign, np.arange(5))
    # duplicated keys: the second initial centroid equals the first, loses every tie and keeps
    # its position as an empty cluster
    y = np.zeros((4, 16))
    y[2:] = 1.0
    mu, assign = O.kmeans_index_keys(y, 2, iters=5)      # starts at rows 0 and 2
    assert np.array_equal(assign, [0, 0, 1, 1])
    z = np.zeros((4, 16))
    mu, assign = O.kmeans_index_keys(z, 2, iters=5)      # both starts at 0: ties to cluster 0
    assert np.array_equal(assign, [0, 0, 0, 0]) and np.array_equal(mu, np.zeros((2, 16)))


def test_cluster_select_with_one_token_per_cluster_is_exact_top_p():
    """K = N (every token its own cluster, the centroid its key): the estimated masses are the
    token masses exp(s - max s), so the hit set is the exact sorted top-p set."""
    rng = np.random.default_rng(5)
    for _ in range(20):
        n = int(rng.integers(1, 60))
        kidx = rng.standard_normal((n, 16))
        q = rng.standard_normal(16) * rng.uniform(0.2, 3.0)
        p = float(rng.uniform(0.05, 0.999))
        got = O.cluster_select(q, kidx, np.arange(n), p)
        assert np.array_equal(got, O.topp_exact(O.index_scores(q, kidx), p))


def test_cluster_select_hand_worked_case():
    """Two clusters: 3 tokens at centroid score 0 and 1 token at centroid score ln 2. Masses
    3 * exp(-ln 2) = 1.5 and 1: the three-token cluster leads; p = 0.6 of 2.5 = 1.5 is reached
    by it alone, p = 0.61 needs both."""
    cent = np.array([[0.0] * 16, [math.log(2.0)] + [0.0] * 15])
    q = np.array([1.0] + [0.0] * 15)
    assign = np.array([0, 0, 1, 0])
    c, mass = O.cluster_mass(q, cent, assign)
    np.testing.assert_allclose(c, [0.0, math.log(2.0)])
    np.testing.assert_allclose(mass, [1.5, 1.0])
    assert np.array_equal(O.cluster_select(q, cent, assign, 0.6), [True, True, False, True])
    assert O.cluster_select(q, cent, assign, 0.61).all()


def test_clustered_head_at_p1_is_dense_attention():
    """p = 1 hits every cluster: the head's output is dense attention over all N tokens."""
    rng = np.random.default_rng(6)
    N = 200
    k_pre = O.bf16_round(rng.standard_normal((N, 128)))
    v = O.bf16_round(rng.standard_normal((N, 128)))
    q_pre = O.bf16_round(rng.standard_normal(128))
    wq = rng.standard_normal((128, 16)) / np.sqrt(128)
    wk = rng.standard_normal((128, 16)) / np.sqrt(128)
    mu, assign = O.kmeans_index_keys(O.index_keys(k_pre, wk), 16, iters=20)
    r = O.clustered_head(q_pre, wq, k_pre, v, wk, mu, assign, 1.0)
    pos = np.arange(N)
    ref = O.attend(O.rope_rotate(q_pre, N - 1), O.bf16_round(O.rope_rotate(k_pre, pos)), v)
    assert r.count == N
    np.testing.assert_allclose(r.out, ref, rtol=1e-12, atol=1e-12)
    # p < 1: the attended set is a union of whole clusters
    r2 = O.clustered_head(q_pre, wq, k_pre, v, wk, mu, assign, 0.5)
    hit = set(assign[r2.sel].tolist())
    assert set(np.nonzero(np.isin(assign, list(hit)))[0].tolist()) == set(r2.sel.tolist())
