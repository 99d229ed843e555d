"""The prefill kernel's arithmetic, modelled on the CPU, against the float64 oracle: why the
query and the probabilities enter the tensor cores as two bf16 terms each.

The model follows the kernel's steps in NumPy: the rotated, scaled query in float32 split
into bf16 terms, logits accumulated in float32 over 64-key tiles, the softmax reference moved
only when a tile's maximum exceeds it by 2^8, probabilities split into bf16 terms, the output
and the row sum accumulated in float32, the result rounded to bf16. With both splits the
outputs meet the parity rule (max-abs 1e-2, mean-abs 1e-3 in the bf16 format) at every query
scale the GPU tests use; with one bf16 term each the same inputs break it at scale 4."""
import numpy as np
import pytest

from oracle import rtp_oracle as O

LOG2E = np.float32(1.4426950408889634)


def _bf(x):
    return O.bf16_round(np.asarray(x, np.float64)).astype(np.float32)


def _model(q_pre, k_pre, v, split_q, split_p, tile=64, slack=8.0):
    n = q_pre.shape[0]
    pos = np.arange(n)
    K = O.bf16_round(O.rope_rotate(k_pre, pos)).astype(np.float32)
    V = v.astype(np.float32)
    q = (O.rope_rotate(q_pre, pos).astype(np.float32) * (LOG2E / np.float32(np.sqrt(128.0))))
    q_hi = _bf(q)
    q_lo = _bf(q - q_hi) if split_q else np.zeros_like(q)
    out = np.zeros((n, 128), np.float32)
    for m in range(n):
        m_ref, l_run = -np.inf, np.float32(0.0)
        o = np.zeros(128, np.float32)
        for k0 in range(0, m + 1, tile):
            keys = np.arange(k0, min(k0 + tile, m + 1))
            s = ((K[keys].astype(np.float64) @ q_hi[m].astype(np.float64)).astype(np.float32) +
                 (K[keys].astype(np.float64) @ q_lo[m].astype(np.float64)).astype(np.float32))
            mx = float(s.max())
            if mx > m_ref + slack:
                alpha = np.float32(np.exp2(m_ref - mx)) if np.isfinite(m_ref) else np.float32(0)
                o *= alpha
                l_run *= alpha
                m_ref = mx
            p = np.exp2(s - np.float32(m_ref)).astype(np.float32)
            l_run += p.sum(dtype=np.float32)
            p_hi = _bf(p)
            p_lo = _bf(p - p_hi) if split_p else np.zeros_like(p)
            o += ((p_hi.astype(np.float64) @ V[keys]).astype(np.float32) +
                  (p_lo.astype(np.float64) @ V[keys]).astype(np.float32))
        out[m] = o / l_run
    return O.bf16_round(out.astype(np.float64))


def _case(scale, seed=0, n=160):
    rng = np.random.default_rng(seed)
    q = O.bf16_round(rng.standard_normal((n, 128)) * scale)
    k = O.bf16_round(rng.standard_normal((n, 128)))
    v = O.bf16_round(rng.standard_normal((n, 128)))
    ref = O.bf16_round(O.prefill_head(q, k, v, False, 4, 64))
    return q, k, v, ref


@pytest.mark.parametrize("scale", [1.0, 2.0, 4.0])
def test_two_term_model_meets_the_parity_rule(scale):
    q, k, v, ref = _case(scale)
    err = np.abs(_model(q, k, v, True, True) - ref)
    assert err.max() <= 1e-2 and err.mean() <= 1e-3, (err.max(), err.mean())


def test_one_term_model_breaks_the_rule_at_scale_4():
    q, k, v, ref = _case(4.0)
    err = np.abs(_model(q, k, v, False, False) - ref)
    assert err.max() > 1e-2 or err.mean() > 1e-3, (err.max(), err.mean())
