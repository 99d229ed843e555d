"""Plain float64 CPU oracle of RTPurbo's per-layer decode-step attention.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` import this module. The CUDA library never calls it and shares no code with it.

Sources, named by page and section:

* [P] "Full Attention Strikes Back: Transferring Full Attention into Sparse within Hundred
  Training Steps" (paper text, Chinese translation): §2.2 eq. (1) RoPE and eq. (2) the
  relative-offset form of a RoPE score; §3.2 eq. (4) the low-rank pre-RoPE index score and
  eq. (5) exact softmax attention over S = Top-P(s, p); §3.2 local heads use attention sinks
  plus a sliding window in prefill and decode.
* [DR] MCISLAB DeepRead notes "2605-RTPurbo", section "Method": top-p with p = 0.9 on a
  16-dim projection; hardware kernels: sort-free top-p through a 256-bin histogram (1 KB per
  head) that fuses scoring and selection.
* [GS] gist.science explainer of the same paper, "Dynamische Top-p-Auswahl": the selector
  accumulates attention mass in the low-dimensional space until the cumulative share p.
* [V2] RTPurboV2 article, finding 3 ("adaptive clustering on high-quality features"): the N
  tokens of a retrieval head are grouped into K semantic clusters in the low-rank space (K = 128
  in the article), the query is first matched against the K centroids, and the full attention
  runs only inside the hit clusters; the architecture summary pairs this clustering index with
  the dynamic top-p of V1.

Readings where the pages are silent (each is repeated where it is used):

* R1 mass temperature: the mass of a token is softmax(s) with scale 1 (eq. (4) has none).
* R2 one W_kidx per KV head (one index row serves its whole query group), one W_qidx per
  query head; the index key is stored as bf16.
* R3 retrieval heads are marked per KV head and get no forced sinks or window.
* R4 the 256 bins are linear over the exact per-head [min, max] of the scores and hold the
  mass sum(exp(s - max)) of their tokens.
* R5 b* is the highest bin whose cumulative mass from the top reaches p of the total; the
  whole bin b* is kept, so the set is a superset of the exact sorted top-p set. p >= 1, or
  all scores equal, selects every token.
* R7 RoPE pairs channel i with channel i + d/2 (rotate-half) and theta_i = base^(-2i/d),
  angles in float64.
* R8 the window is the last ``window`` positions (the current token included) and the sinks
  are positions 0..sinks-1, without duplicates.
* R9 the attention scale is 1/sqrt(d_h).

The pages print no worked example of a whole layer that can be reproduced without trained
weights, so no published number pins the composition; it is pinned instead by a brute-force
evaluation of the definitions on tiny inputs (N <= 64), and each part by its own tests, in
``tests/test_oracle.py``.
"""
from __future__ import annotations

import dataclasses

import numpy as np

HEAD_DIM = 128
IDX_DIM = 16
N_BINS = 256
BF16_MAX = float.fromhex("0x1.fep127")


# --------------------------------------------------------------------------- storage rounding
def bf16_round(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value (ties to even); returns float64.

    Caches are bf16 ([P] is silent on storage; R2 for the index key). bfloat16 keeps
    8 significant bits and the float32 exponent range, with subnormal spacing 2^-133.
    """
    x = np.asarray(x, dtype=np.float64)
    out = x.copy()
    fin = np.isfinite(x) & (x != 0)
    xv = x[fin]
    _, e = np.frexp(xv)                                  # |x| in [2^(e-1), 2^e)
    q = np.ldexp(1.0, np.maximum(e, -125) - 8)           # spacing of bf16 values near x
    r = np.rint(xv / q) * q                              # rint: ties to even
    r = np.where(np.abs(r) > BF16_MAX, np.copysign(np.inf, xv), r)
    out[fin] = r
    return out


# --------------------------------------------------------------------------- eq. (1): RoPE
def rope_theta(head_dim: int = HEAD_DIM, base: float = 1e6) -> np.ndarray:
    """theta_i = base^(-2i/d), i = 0..d/2-1, decreasing in i ([P] §2.2 eq. (1); R7)."""
    i = np.arange(head_dim // 2, dtype=np.float64)
    return base ** (-2.0 * i / head_dim)


def rope_rotate(x, pos, base: float = 1e6) -> np.ndarray:
    """R(pos) x: a 2x2 rotation by pos*theta_i on each channel pair (i, i + d/2).

    [P] §2.2 eq. (1): R_i(m) = [[cos m theta_i, -sin m theta_i], [sin m theta_i, cos m theta_i]],
    q_m = R(m) q, k_n = R(n) k. Pairing is rotate-half (R7). ``pos`` broadcasts against the
    leading axes of ``x``.
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    h = d // 2
    ang = np.asarray(pos, dtype=np.float64)[..., None] * rope_theta(d, base)
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., :h], x[..., h:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


# --------------------------------------------------------------------------- eq. (4): index scores
def index_keys(k_pre, w_kidx) -> np.ndarray:
    """Stored index keys bf16(W^K k^pre) of the cached tokens ([P] §3.2 eq. (4); R2).

    ``k_pre`` [N][d] (pre-RoPE keys), ``w_kidx`` [d][r]: the projection acts on pre-RoPE
    features; the r = 16 result is stored in bf16.
    """
    return bf16_round(np.asarray(k_pre, np.float64) @ np.asarray(w_kidx, np.float64))


def index_query(q_pre, w_qidx) -> np.ndarray:
    """W^Q q^pre of the current query ([P] §3.2 eq. (4)); kept in float64."""
    return np.asarray(q_pre, np.float64) @ np.asarray(w_qidx, np.float64)


def index_scores(q_idx, kidx) -> np.ndarray:
    """s(m, n) = (W^Q q^pre_m)^T (W^K k^pre_n) for every cached n ([P] §3.2 eq. (4))."""
    return np.asarray(kidx, np.float64) @ np.asarray(q_idx, np.float64)


# --------------------------------------------------------------------------- eq. (5): Top-P
@dataclasses.dataclass
class Selection:
    mask: np.ndarray          # bool [N]: token n is in S
    bstar: int                # threshold bin (0 when everything is selected)
    lo: float                 # min score
    hi: float                 # max score
    bins: np.ndarray          # int [N] bin of each token (zeros when everything is selected)
    M: np.ndarray             # float64 [256] mass per bin
    C: np.ndarray             # float64 [256] mass of bins >= b
    T: float                  # total mass
    select_all: bool

    @property
    def width(self) -> float:
        return (self.hi - self.lo) / N_BINS

    def edge(self) -> float:
        """Lower edge of bin b*: lo + b* (hi - lo) / 256."""
        return self.lo + self.bstar * self.width


def score_bins(s, lo: float, hi: float) -> np.ndarray:
    """bin(s) = min(255, floor(256 (s - lo) / (hi - lo))): 256 linear bins over [lo, hi] (R4)."""
    s = np.asarray(s, np.float64)
    return np.minimum(N_BINS - 1, np.floor((s - lo) * N_BINS / (hi - lo))).astype(np.int64)


def topp_histogram(s, p: float) -> Selection:
    """Top-P(s, p) through the 256-bin mass histogram ([P] §3.2 eq. (5); [DR] "Method";
    [GS] "Dynamische Top-p-Auswahl"; readings R1, R4, R5).

    mass_n = exp(s_n - max s); M_b = sum of the masses of bin b; C_b = sum_{b' >= b} M_b';
    T = C_0; b* = max{b : C_b >= p T}; S = {n : bin(s_n) >= b*}.
    """
    s = np.asarray(s, np.float64)
    N = s.shape[0]
    if N < 1:
        raise ValueError("Top-P needs at least one token")
    lo, hi = float(s.min()), float(s.max())
    if p >= 1.0 or hi == lo:
        mass = np.exp(s - hi)
        M = np.zeros(N_BINS)
        M[0] = mass.sum()
        C = np.full(N_BINS, 0.0)
        C[0] = M[0]
        return Selection(np.ones(N, bool), 0, lo, hi, np.zeros(N, np.int64), M, C,
                         float(M[0]), True)
    bins = score_bins(s, lo, hi)
    mass = np.exp(s - hi)
    M = np.bincount(bins, weights=mass, minlength=N_BINS)
    C = np.cumsum(M[::-1])[::-1]
    T = float(C[0])
    bstar = int(np.nonzero(C >= p * T)[0].max())
    return Selection(bins >= bstar, bstar, lo, hi, bins, M, C, T, False)


def topp_exact(s, p: float) -> np.ndarray:
    """Exact Top-P: the smallest prefix of the tokens sorted by score (descending; equal
    scores by lower index first) whose mass exp(s - max) reaches p of the total
    ([P] §3.2 eq. (5); [GS] "Dynamische Top-p-Auswahl"). Returns a bool mask."""
    s = np.asarray(s, np.float64)
    N = s.shape[0]
    if p >= 1.0:
        return np.ones(N, bool)
    order = np.lexsort((np.arange(N), -s))
    cum = np.cumsum(np.exp(s[order] - s.max()))
    k = int(np.searchsorted(cum, p * cum[-1], side="left")) + 1
    mask = np.zeros(N, bool)
    mask[order[:min(k, N)]] = True
    return mask


# --------------------------------------------------------------------------- fixed top-k variant
def topk_histogram(s, k: int) -> Selection:
    """Fixed-budget top-k through the same 256-bin histogram, with a count threshold in place
    of the mass threshold: the top-k selector the pages compare Top-P against ([P] Table 1,
    top-k budgets vs top-p; [DR] "Method": the 256-bin threshold).

    count_b = number of tokens in bin b; K_b = sum_{b' >= b} count_b'; b* = max{b : K_b >= k};
    S = {n : bin(s_n) >= b*}. k >= N, or all-equal scores, selects every token. The fields M
    and C of the result hold the counts and their suffix sums; T = N.

    b* is the bin of the k-th highest score: the k highest scores all have bins >= it, and if
    k tokens had bins above it the k-th highest score would too. So S holds the exact top-k
    plus, at most, tokens of that one bin.
    """
    s = np.asarray(s, np.float64)
    N = s.shape[0]
    if N < 1:
        raise ValueError("top-k needs at least one token")
    if k < 1:
        raise ValueError("top-k needs k >= 1")
    lo, hi = float(s.min()), float(s.max())
    if k >= N or hi == lo:
        cnt = np.zeros(N_BINS)
        cnt[0] = N
        return Selection(np.ones(N, bool), 0, lo, hi, np.zeros(N, np.int64), cnt, cnt.copy(),
                         float(N), True)
    bins = score_bins(s, lo, hi)
    cnt = np.bincount(bins, minlength=N_BINS).astype(np.float64)
    C = np.cumsum(cnt[::-1])[::-1]
    bstar = int(np.nonzero(C >= k)[0].max())
    return Selection(bins >= bstar, bstar, lo, hi, bins, cnt, C, float(N), False)


def topk_exact(s, k: int) -> np.ndarray:
    """The k highest scores (equal scores by lower index first), by sort. Returns a bool mask."""
    s = np.asarray(s, np.float64)
    order = np.lexsort((np.arange(s.shape[0]), -s))
    mask = np.zeros(s.shape[0], bool)
    mask[order[:min(int(k), s.shape[0])]] = True
    return mask


# --------------------------------------------------------------------------- eq. (5): attention
def attend(q, K, V, scale: float | None = None) -> np.ndarray:
    """sum_n softmax_n(q^T k_n / sqrt(d)) v_n over the rows given ([P] §3.2 eq. (5); R9)."""
    q = np.asarray(q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    if scale is None:
        scale = 1.0 / np.sqrt(q.shape[-1])
    z = (K @ q) * scale
    w = np.exp(z - z.max())
    return (w @ V) / w.sum()


def local_positions(N: int, sinks: int, window: int) -> np.ndarray:
    """Positions a local head attends to at decode with N cached tokens (current included):
    the sinks {0..sinks-1} and the last ``window`` positions, without duplicates
    ([P] §3.2, local heads: sliding window with attention sinks; R8)."""
    a = np.arange(min(sinks, N))
    b = np.arange(max(sinks, N - window), N)
    return np.concatenate([a, b]).astype(np.int64)


# --------------------------------------------------------------------------- one head, one layer
@dataclasses.dataclass
class HeadResult:
    out: np.ndarray            # float64 [d]
    count: int                 # |S| (retrieval) or |L| (local)
    sel: np.ndarray | None     # ascending selected positions (retrieval)
    selection: Selection | None
    scores: np.ndarray | None


def retrieval_head(q_pre, w_qidx_h, k_pre, v, w_kidx_g, p: float, base: float = 1e6) -> HeadResult:
    """One retrieval query head at decode position m = N - 1 ([P] §3.2 eq. (4)-(5)).

    k_pre, v: [N][d] pre-RoPE keys and values of the head's KV head (bf16 values as float64).
    """
    k_pre = np.asarray(k_pre, np.float64)
    N = k_pre.shape[0]
    kidx = index_keys(k_pre, w_kidx_g)
    s = index_scores(index_query(q_pre, w_qidx_h), kidx)
    sel = topp_histogram(s, p)
    idx = np.nonzero(sel.mask)[0]
    K = bf16_round(rope_rotate(k_pre[idx], idx, base))
    q = rope_rotate(q_pre, N - 1, base)
    out = attend(q, K, np.asarray(v, np.float64)[idx])
    return HeadResult(out, int(idx.size), idx, sel, s)


def local_head(q_pre, k_pre, v, sinks: int, window: int, base: float = 1e6) -> HeadResult:
    """One local query head: attention over the sinks plus the window ([P] §3.2; R8)."""
    k_pre = np.asarray(k_pre, np.float64)
    N = k_pre.shape[0]
    pos = local_positions(N, sinks, window)
    K = bf16_round(rope_rotate(k_pre[pos], pos, base))
    q = rope_rotate(q_pre, N - 1, base)
    out = attend(q, K, np.asarray(v, np.float64)[pos])
    return HeadResult(out, int(pos.size), pos, None, None)


def full_attention_mass(q_pre, k_pre, sel_positions, base: float = 1e6) -> float:
    """Retained mass of a selected set: the share of the dense attention weights
    softmax(q^T k_n / sqrt(d)) over all N cached tokens (RoPE'd, bf16-stored keys; query at
    position N - 1) that falls on ``sel_positions``. [DR] "Key Results" reports this share
    (above 0.93 at 89.2 % sparsity) for the sets the selector keeps; [P] §2.3 compares top-k
    and top-p sets by the same quantity."""
    k_pre = np.asarray(k_pre, np.float64)
    N = k_pre.shape[0]
    K = bf16_round(rope_rotate(k_pre, np.arange(N), base))
    q = rope_rotate(q_pre, N - 1, base)
    z = (K @ q) / np.sqrt(q.shape[-1])
    w = np.exp(z - z.max())
    return float(w[np.asarray(sel_positions, np.int64)].sum() / w.sum())


def decode_layer(q_pre, w_qidx, w_kidx, k_pre, v, ret_mask, seq_lens, p: float, sinks: int,
                 window: int, base: float = 1e6, heads=None):
    """Whole decode layer over a batch ([P] §3.2): retrieval query heads use eq. (4)-(5),
    local query heads use sinks + window. Query head h reads KV head h // G (GQA).

    q_pre [B][Hq][d]; w_qidx [Hq][d][r]; w_kidx [Hkv][d][r]; k_pre, v: callables
    (b, g) -> [N_b][d] arrays; ret_mask [Hkv] bool; ``heads`` optionally restricts the
    (b, h) pairs computed. Returns {(b, h): HeadResult}.
    """
    B, Hq, _ = np.asarray(q_pre).shape
    Hkv = len(ret_mask)
    G = Hq // Hkv
    res = {}
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hq)]
    for b, h in pairs:
        g = h // G
        N = int(seq_lens[b])
        kp = np.asarray(k_pre(b, g), np.float64)[:N]
        vv = np.asarray(v(b, g), np.float64)[:N]
        if ret_mask[g]:
            res[(b, h)] = retrieval_head(q_pre[b][h], w_qidx[h], kp, vv, w_kidx[g], p, base)
        else:
            res[(b, h)] = local_head(q_pre[b][h], kp, vv, sinks, window, base)
    return res


# --------------------------------------------------------------------------- prefill (f1)
def prefill_head(q_pre, k_pre, v, local: bool, sinks: int, window: int,
                 base: float = 1e6) -> np.ndarray:
    """Causal prefill of one query head over a prompt of n tokens at positions 0..n-1
    ([P] §3.2: retrieval heads use dense attention in prefill, local heads attention sinks
    plus a sliding window in prefill and decode). Query m attends to the positions n <= m
    (retrieval) or to local_positions(m + 1, sinks, window) (local); keys are stored RoPE'd in
    bf16 (as the append writes them), q = R(m) q_pre, scale 1 / sqrt(d).

    q_pre, k_pre, v: [n][d] (bf16 values as float64). Returns float64 [n][d].
    """
    q_pre = np.asarray(q_pre, np.float64)
    k_pre = np.asarray(k_pre, np.float64)
    v = np.asarray(v, np.float64)
    n, d = q_pre.shape
    pos = np.arange(n)
    K = bf16_round(rope_rotate(k_pre, pos, base))
    Q = rope_rotate(q_pre, pos, base)
    z = (Q @ K.T) / np.sqrt(d)
    m_idx, n_idx = np.meshgrid(pos, pos, indexing="ij")
    allowed = n_idx <= m_idx
    if local:
        allowed &= (n_idx < sinks) | (n_idx > m_idx - window)
    z = np.where(allowed, z, -np.inf)
    w = np.exp(z - z.max(axis=1, keepdims=True))
    return (w @ v) / w.sum(axis=1, keepdims=True)


# ----------------------------------------------------------- [V2] centroid pre-filter (f3)
def kmeans_index_keys(kidx, K: int = 128, iters: int = 10):
    """Lloyd's k-means of one retrieval KV head's stored index keys ([V2] finding 3: the tokens
    grouped into K clusters in the 16-dim low-rank space, K = 128 in the article).

    Readings: (R-f3a) the initial centroids are the keys at positions floor(i N / K), i < K
    (deterministic, spread over the sequence); K > N is clamped to N. (R-f3b) an iteration
    assigns every key to its nearest centroid in squared Euclidean distance (ties to the lower
    cluster id), then moves every non-empty cluster's centroid to the mean of its keys (an empty
    cluster keeps its centroid); at most `iters` iterations, fewer when an assignment repeats.

    kidx: [N][r] (bf16 values as float64). Returns (centroids [K][r] float64, assign [N] int64).
    """
    x = np.asarray(kidx, np.float64)
    N = x.shape[0]
    K = min(K, N)
    mu = x[(np.arange(K) * N) // K].copy()
    assign = None
    for _ in range(iters):
        d = ((x[:, None, :] - mu[None, :, :]) ** 2).sum(axis=2)     # [N][K]
        new = d.argmin(axis=1)                                        # first minimum: lower id
        if assign is not None and np.array_equal(new, assign):
            break
        assign = new
        for k in range(K):
            members = assign == k
            if members.any():
                mu[k] = x[members].mean(axis=0)
    return mu, assign


def cluster_mass(q_idx, centroids, assign):
    """Coarse match ([V2] finding 3, step 1): centroid scores c_k = q_idx . mu_k and the
    estimated mass of each cluster, |C_k| exp(c_k - max c) (R-f3c: a cluster's members stand at
    their centroid's score, with the token mass of R1). Returns (c [K], mass [K])."""
    c = np.asarray(centroids, np.float64) @ np.asarray(q_idx, np.float64)
    counts = np.bincount(np.asarray(assign), minlength=c.shape[0]).astype(np.float64)
    return c, counts * np.exp(c - c.max())


def cluster_select(q_idx, centroids, assign, p: float) -> np.ndarray:
    """The hit clusters ([V2] finding 3 with the dynamic top-p of V1; R-f3d): clusters in
    descending estimated mass (ties to the lower id), the smallest prefix whose mass reaches p
    of the total; p >= 1 hits every non-empty cluster. Returns the bool mask of hit tokens."""
    _, mass = cluster_mass(q_idx, centroids, assign)
    K = mass.shape[0]
    if p >= 1.0:
        hit = mass > 0
    else:
        order = np.lexsort((np.arange(K), -mass))
        cum = np.cumsum(mass[order])
        n = int(np.searchsorted(cum, p * cum[-1], side="left")) + 1
        hit = np.zeros(K, bool)
        hit[order[:min(n, K)]] = True
    return hit[np.asarray(assign)]


def clustered_head(q_pre, w_qidx_h, k_pre, v, w_kidx_g, centroids, assign, p: float,
                   base: float = 1e6) -> HeadResult:
    """A retrieval query head at m = N - 1 through the centroid pre-filter ([V2] finding 3,
    step 2; R-f3e): exact softmax attention (R9) over every token of the hit clusters."""
    k_pre = np.asarray(k_pre, np.float64)
    N = k_pre.shape[0]
    mask = cluster_select(index_query(q_pre, w_qidx_h), centroids, assign, p)
    idx = np.nonzero(mask)[0]
    K = bf16_round(rope_rotate(k_pre[idx], idx, base))
    out = attend(rope_rotate(q_pre, N - 1, base), K, np.asarray(v, np.float64)[idx])
    s = index_scores(index_query(q_pre, w_qidx_h), index_keys(k_pre, w_kidx_g))
    return HeadResult(out, int(idx.size), idx, None, s)


def append_rows(k_pre, v, w_kidx_g, positions, base: float = 1e6):
    """Rows the append step stores for one KV head: bf16(R(n) k_pre_n), v_n and the index key
    bf16(W^K k_pre_n) ([P] §2.2 eq. (1), §3.2 eq. (4); R2, R7)."""
    k_pre = np.asarray(k_pre, np.float64)
    k = bf16_round(rope_rotate(k_pre, np.asarray(positions), base))
    kidx = None if w_kidx_g is None else index_keys(k_pre, w_kidx_g)
    return k, np.asarray(v, np.float64), kidx
