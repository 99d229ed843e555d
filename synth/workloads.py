"""The five synthetic decode workloads and their planted structure.

Shapes follow the Qwen3-8B attention layout (36 layers, 32 query heads, 8 KV heads, head
dim 128) with a 16-dim index projection, 4 attention sinks and a 2048-token window
(256 in the tiny case). Nothing here computes a step of the method; the module only
decides *what* the inputs are:

* retrieval mask: a seeded choice of 43 of the 288 (layer, KV head) pairs (about 15%
  retrieval heads, the ratio of the paper's head split); the tiny case marks KV head 0;
* W_qidx, W_kidx: float32, entries ~ N(0, 1/128) from the counter stream;
* k_pre, v: bf16 rows ~ N(0, 1) from the counter stream;
* planted clusters in the retrieval KV heads: runs of consecutive tokens whose pre-RoPE
  key is shifted by the minimum-norm vector ``delta = W_k (W_k^T W_k)^{-1} (alpha u)``, which
  moves the 16-dim projection ``W_k^T k_pre`` by ``alpha u`` (u a unit 16-vector); ``alpha`` is
  set from a strength in background standard deviations, ``alpha / sqrt(u^T W_k^T W_k u)``;
* queries: for a retrieval query head the target projection is ``lam * u_hat / sigma`` (``u_hat``
  the head's cluster direction, or the normalised weighted sum of several for a diffuse head;
  ``sigma = sqrt(u_hat^T W_k^T W_k u_hat)`` the background standard deviation of the index
  key along it, so lam is a temperature in background units for every head);
  ``q_pre = z + W_q (W_q^T W_q)^{-1} (target - W_q^T z)`` with ``z`` from the counter stream, so the
  projected query equals the target before bf16 storage rounding. ``lam`` is the one
  temperature knob, fixed per workload so that concentrated heads keep a few hundred tokens
  and diffuse heads a few thousand at 32K, the spread the paper's notes report between a
  single-needle and a multi-key task.
"""
from __future__ import annotations

import dataclasses
from functools import lru_cache

import numpy as np

from . import gen

HEAD_DIM = 128
IDX_DIM = 16


@dataclasses.dataclass
class Cluster:
    start: int
    length: int
    u: np.ndarray            # float64 [16], unit
    strength: float          # in background standard deviations
    delta: np.ndarray        # float32 [128], added to k_pre rows of the run


@dataclasses.dataclass
class GroupLayout:
    clusters: list           # list[Cluster]
    targets: list            # per query head of the group: (kind, [cluster ids], weights)


@dataclasses.dataclass
class Workload:
    name: str
    index: int               # 1-based workload number
    layers: int
    B: int
    Hq: int
    Hkv: int
    seq_lens: np.ndarray     # int64 [B]
    sinks: int
    window: int
    p: float
    lam_conc: float
    lam_diff: float
    head_dim: int = HEAD_DIM
    idx_dim: int = IDX_DIM
    rope_base: float = 1e6
    seed: int = 0
    ret_mask: np.ndarray = None   # bool [layers][Hkv]
    kind: str = "mix"             # "needle" | "mix" | "mix_depth" | "diffuse16"

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def retrieval_kv(self, layer: int):
        return [g for g in range(self.Hkv) if self.ret_mask[layer, g]]

    def local_kv(self, layer: int):
        return [g for g in range(self.Hkv) if not self.ret_mask[layer, g]]

    # ----------------------------------------------------------- weights
    def w_kidx(self, layer: int) -> np.ndarray:
        """float32 [Hkv][128][16]."""
        return _weights(self.seed, gen.T_WKIDX, layer, self.Hkv, self.head_dim, self.idx_dim)

    def w_qidx(self, layer: int) -> np.ndarray:
        """float32 [Hq][128][16]."""
        return _weights(self.seed, gen.T_WQIDX, layer, self.Hq, self.head_dim, self.idx_dim)

    # ----------------------------------------------------------- structure
    def group_layout(self, layer: int, b: int, kvh: int) -> GroupLayout:
        return _group_layout(self, layer, b, kvh)

    def shifts(self, layer: int, b: int, kvh: int):
        """(start, length, delta) of the planted runs of one KV head (empty for local heads)."""
        if not self.ret_mask[layer, kvh]:
            return []
        return [(c.start, c.length, c.delta) for c in self.group_layout(layer, b, kvh).clusters]

    # ----------------------------------------------------------- rows
    def kpre_bits(self, layer: int, b: int, kvh: int, t0: int, t1: int) -> np.ndarray:
        key = gen.stream_key(self.seed, gen.T_KPRE, layer, b, kvh)
        return gen.token_rows_bits(key, t0, t1, self.head_dim, self.shifts(layer, b, kvh))

    def v_bits(self, layer: int, b: int, kvh: int, t0: int, t1: int) -> np.ndarray:
        key = gen.stream_key(self.seed, gen.T_V, layer, b, kvh)
        return gen.token_rows_bits(key, t0, t1, self.head_dim)

    def prompt_q_bits(self, layer: int, b: int, h: int, t0: int, t1: int,
                      scale: float = 1.0) -> np.ndarray:
        """bf16 bits [t1 - t0][128] of the pre-RoPE queries of query head h at prompt
        positions t0..t1-1 (prefill inputs): rows of their own counter stream, each value
        times ``scale`` (one float32 multiplication) before rounding; scale sets how peaked
        the prompt's attention rows are."""
        key = gen.stream_key(self.seed, gen.T_QPROMPT, layer, b, h)
        c = np.arange(t0 * self.head_dim, t1 * self.head_dim, dtype=np.uint64)
        x = gen.normal_f32(key, c.reshape(t1 - t0, self.head_dim)) * np.float32(scale)
        return gen.f32_to_bf16_bits(x)

    def q_target(self, layer: int, b: int, h: int):
        """Target 16-dim projected query of a retrieval query head (float64), else None."""
        kvh = h // self.G
        if not self.ret_mask[layer, kvh]:
            return None
        lay = self.group_layout(layer, b, kvh)
        kind, ids, wts = lay.targets[h % self.G]
        d = np.zeros(self.idx_dim)
        for i, w in zip(ids, wts):
            d += w * lay.clusters[i].u
        d /= np.linalg.norm(d)
        lam = self.lam_conc if kind == "conc" else self.lam_diff
        # in units of the background score standard deviation along d: sqrt(d^T W_k^T W_k d)
        W = self.w_kidx(layer)[kvh].astype(np.float64)
        return lam / np.sqrt(d @ (W.T @ W) @ d) * d

    def q_pre_bits(self, layer: int) -> np.ndarray:
        """bf16 bits [B][Hq][128] of the pre-RoPE queries of one layer."""
        out = np.zeros((self.B, self.Hq, self.head_dim), dtype=np.uint16)
        wq = self.w_qidx(layer).astype(np.float64)
        for b in range(self.B):
            for h in range(self.Hq):
                key = gen.stream_key(self.seed, gen.T_QPRE, layer, b, h)
                z = gen.normal_f32(key, np.arange(self.head_dim)).astype(np.float64)
                tgt = self.q_target(layer, b, h)
                if tgt is not None:
                    W = wq[h]                                   # [128][16]
                    corr = W @ np.linalg.solve(W.T @ W, tgt - W.T @ z)
                    z = z + corr
                out[b, h] = gen.f32_to_bf16_bits(z.astype(np.float32))
        return out


@lru_cache(maxsize=256)
def _weights_cached(seed, tensor, layer, heads, d, r):
    out = np.empty((heads, d, r), dtype=np.float32)
    scale = np.float32(1.0 / np.sqrt(d))
    for h in range(heads):
        key = gen.stream_key(seed, tensor, layer, 0, h)
        out[h] = (gen.normal_f32(key, np.arange(d * r)) * scale).reshape(d, r)
    out.setflags(write=False)
    return out


def _weights(seed, tensor, layer, heads, d, r):
    return _weights_cached(seed, tensor, layer, heads, d, r)


def _place(rng, lengths, n_tokens):
    """Non-overlapping runs with the given lengths at uniform random depths in [0, n_tokens)."""
    lengths = list(lengths)
    total = sum(lengths)
    if total > n_tokens:
        raise ValueError("clusters do not fit")
    order = rng.permutation(len(lengths))
    cuts = np.sort(rng.integers(0, n_tokens - total + 1, size=len(lengths)))
    starts = [0] * len(lengths)
    acc = 0
    for rank, i in enumerate(order):
        starts[i] = int(cuts[rank]) + acc
        acc += lengths[i]
    return starts


def _unit(rng, r):
    u = rng.standard_normal(r)
    return u / np.linalg.norm(u)


def _split(total, parts):
    base = total // parts
    return [base + (1 if i < total % parts else 0) for i in range(parts)]


_LAYOUT_CACHE: dict = {}


def _group_layout(w: Workload, layer: int, b: int, kvh: int) -> GroupLayout:
    ck = (w.seed, w.kind, w.G, int(w.seq_lens[b]), layer, b, kvh)
    if ck in _LAYOUT_CACHE:
        return _LAYOUT_CACHE[ck]
    rng = np.random.default_rng([w.seed, 7, layer, b, kvh])
    N = int(w.seq_lens[b])
    G = w.G
    specs = []     # (length, strength)
    targets = []
    if w.kind == "needle":
        specs = [(32, 4.0)]
        targets = [("conc", [0], [1.0]) for _ in range(G)]
    elif w.kind == "mix":
        specs = [(400, 4.0)] + [(n, 4.0) for n in _split(2500, 8)]
        for j in range(G):
            if j % 2 == 0:
                targets.append(("conc", [0], [1.0]))
            else:
                targets.append(("diff", list(range(1, 9)), [1.0] * 8))
    elif w.kind == "mix_depth":
        for j in range(G):
            s = float(rng.uniform(2.0, 5.0))
            first = len(specs)
            if j % 2 == 0:
                specs.append((400, s))
                targets.append(("conc", [first], [1.0]))
            else:
                specs.extend((n, s) for n in _split(2500, 8))
                targets.append(("diff", list(range(first, first + 8)), [1.0] * 8))
    elif w.kind == "diffuse16":
        specs = [(int(rng.integers(64, 1025)), 4.0) for _ in range(16)]
        for j in range(G):
            targets.append(("diff", list(range(16)), list(rng.uniform(0.5, 1.5, size=16))))
    else:
        raise ValueError(w.kind)
    avail = max(N - 1, 0)
    total = sum(n for n, _ in specs)
    if total > avail:                      # short sequence: shrink the runs to fit
        specs = [(int(n * avail // total), s) for n, s in specs]
    starts = _place(rng, [n for n, _ in specs], max(avail, 1))
    W = w.w_kidx(layer)[kvh].astype(np.float64)          # [128][16]
    WtW = W.T @ W
    clusters = []
    for (n, s), st in zip(specs, starts):
        u = _unit(rng, w.idx_dim)
        alpha = s * np.sqrt(u @ WtW @ u)
        delta = (W @ np.linalg.solve(WtW, alpha * u)).astype(np.float32)
        clusters.append(Cluster(start=int(st), length=int(n), u=u, strength=s, delta=delta))
    lay = GroupLayout(clusters=clusters, targets=targets)
    _LAYOUT_CACHE[ck] = lay
    return lay


def _ret_mask_qwen(seed: int, layers: int = 36, hkv: int = 8, n_ret: int = 43) -> np.ndarray:
    rng = np.random.default_rng([seed, 11])
    pick = rng.choice(layers * hkv, size=n_ret, replace=False)
    m = np.zeros((layers, hkv), dtype=bool)
    m.reshape(-1)[pick] = True
    return m


# Query temperatures (lam) per workload; see the module docstring.
# (concentrated, diffuse). At 32K with 4-sigma clusters (1, 2, 5) they keep about 420 and 2500
# tokens per head on average at p = 0.9. Longer contexts need a sharper query for the same
# sparsity: at 128K (3) about 1.5-3K tokens per head (about 95% sparse), at 1M (4) several
# thousand per head (about 98.5% sparse), in line with the sparsity the paper's notes report
# growing with context length (89.2% at 64K, above 97% at 512K).
LAM = {
    1: (1.67, 1.97),
    2: (1.67, 1.97),
    3: (2.45, 2.65),
    4: (3.3, 3.3),
    5: (1.67, 1.97),
}


def workload(index: int, p: float | None = None) -> Workload:
    """Workload 1..5; ``p`` overrides the top-p mass (workload 5 runs at 0.8, 0.9, 0.95)."""
    seed = index - 1
    lc, ld = LAM[index]
    if index == 1:
        m = np.zeros((1, 2), dtype=bool)
        m[0, 0] = True
        return Workload("tiny-1layer-4k", 1, 1, 1, 4, 2, np.array([4096]), 4, 256,
                        0.9 if p is None else p, lc, ld, seed=seed, ret_mask=m, kind="needle")
    m = _ret_mask_qwen(seed)
    if index == 2:
        return Workload("qwen3-8b-32k-b1", 2, 36, 1, 32, 8, np.array([32768]), 4, 2048,
                        0.9 if p is None else p, lc, ld, seed=seed, ret_mask=m, kind="mix")
    if index == 3:
        return Workload("qwen3-8b-128k-b4", 3, 36, 4, 32, 8, np.full(4, 131072), 4, 2048,
                        0.9 if p is None else p, lc, ld, seed=seed, ret_mask=m, kind="mix_depth")
    if index == 4:
        return Workload("qwen3-8b-1m-b1", 4, 36, 1, 32, 8, np.array([1 << 20]), 4, 2048,
                        0.9 if p is None else p, lc, ld, seed=seed, ret_mask=m, kind="diffuse16")
    if index == 5:
        rng = np.random.default_rng([seed, 13])
        lens = rng.integers(8192, 65537, size=64)
        return Workload("qwen3-8b-ragged-b64", 5, 36, 64, 32, 8, lens, 4, 2048,
                        0.9 if p is None else p, lc, ld, seed=seed, ret_mask=m, kind="mix")
    raise ValueError(index)
