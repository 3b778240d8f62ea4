"""Sampled (temperature > 0) verification of a drafted block, float64 reference
(test infrastructure, like the rest of oracle/; nothing here is called by the
library or the benchmark's timed path).

Sources (page title, section):
  [P1] "DFlash — 블록 확산 드래프터로 6배 빨라지는 투기적 디코딩", §1: the verify
       step keeps the drafts that pass and, from the first one that does not,
       samples from the target's distribution, so that the output follows the
       distribution of the target decoding on its own (lossless); the scheme is
       the standard speculative decoding of Leviathan et al. (2023) named there.
  [P2] "한 번에 초안을 생성하는 DFlash ..." (results): the speed-up holds with
       sampling at temperature 1, not only for greedy decoding.

The sampled drafter draws its tokens with gumbel_draft: the Gumbel-max rule over
the counter-based uniforms of oracle.philox (the CUDA side generates the same
stream from the same published generator).

Reading (the pages name the scheme but print no formula): the standard
speculative-sampling rule, position by position over the block. Draft d_i was
drawn from the drafter's distribution q_i (the block drafter predicts every
mask position in one pass, so q_i does not depend on d_1..d_{i-1}); the target
distribution p_{i-1} at the previous position scores it. d_i is accepted when
u_i < p_{i-1}(d_i) / q_i(d_i); at the first rejection the correction token is
drawn from the residual max(0, p_{i-1} - q_i), normalised; when every draft
passes, the bonus token is drawn from p_{B-1}. Random numbers are inputs:
u_accept[i-1] for the test at draft i, u_final for the one final draw
(inverse-CDF over the vocabulary in index order).
"""
from __future__ import annotations

from typing import Sequence, Tuple

import numpy as np

from .philox import draft_uniforms


def softmax_t(logits, temperature: float) -> np.ndarray:
    """Row-wise softmax of logits / temperature in float64 (temperature > 0)."""
    z = np.asarray(logits, dtype=np.float64) / float(temperature)
    z = z - z.max(axis=-1, keepdims=True)
    e = np.exp(z)
    return e / e.sum(axis=-1, keepdims=True)


def sample_index(probs, u: float) -> int:
    """Inverse-CDF draw: the smallest index v with sum_{w<=v} probs[w] > u * sum(probs)."""
    p = np.asarray(probs, dtype=np.float64)
    c = np.cumsum(p)
    v = int(np.searchsorted(c, u * c[-1], side="right"))
    return min(v, len(p) - 1)


def sampled_verify(p, q, draft: Sequence[int], u_accept: Sequence[float], u_final: float) -> Tuple[int, int]:
    """Speculative-sampling verification of one block.

    p [B, V]: target probabilities at block positions 0..B-1 (row j is the
    distribution of the token at position j+1); q [B-1, V]: the drafter's
    distribution that draft i was drawn from (row i-1); draft [B-1]: d_1..d_{B-1};
    u_accept [B-1], u_final: uniforms in [0, 1).
    Returns (a, next): the number of accepted drafts and the token that follows
    them (the correction drawn from the residual, or the bonus token)."""
    p = np.asarray(p, dtype=np.float64)
    q = np.asarray(q, dtype=np.float64)
    B = len(p)
    for i in range(1, B):
        d = int(draft[i - 1])
        pi, qi = p[i - 1, d], q[i - 1, d]
        # accept with probability min(1, p/q): u < p/q, written without a division
        if u_accept[i - 1] * qi < pi:
            continue
        resid = np.maximum(p[i - 1] - q[i - 1], 0.0)
        if resid.sum() <= 0.0:   # only when p == q at this row, where rejection has probability 0
            resid = p[i - 1]
        return i - 1, sample_index(resid, u_final)
    return B - 1, sample_index(p[B - 1], u_final)


def gumbel_sample(logits, temperature: float, u) -> np.ndarray:
    """Draws one token per row from softmax(logits / temperature) by the Gumbel-max
    rule: argmax_v (logits_v / temperature - log(-log u_v)), u [rows, V] uniforms
    in (0, 1). The form a fused LM-head epilogue can evaluate tile by tile."""
    z = np.asarray(logits, dtype=np.float64) / float(temperature)
    g = -np.log(-np.log(np.asarray(u, dtype=np.float64)))
    return np.argmax(z + g, axis=-1)


def gumbel_draft(logits, temperature: float, seed: int, b: int) -> np.ndarray:
    """The sampled drafter's tokens for request b: row i-1 of logits [B-1, V] holds
    the drafter's logits at block position i, and d_i is their Gumbel-max draw
    with the Philox draft-noise uniforms of (seed, b, i) (oracle.philox)."""
    logits = np.asarray(logits, dtype=np.float64)
    Bm1, V = logits.shape
    u = np.stack([draft_uniforms(seed, b, i, V) for i in range(1, Bm1 + 1)]) if Bm1 else np.zeros((0, V))
    return gumbel_sample(logits, temperature, u)


def gumbel_scores(logits, temperature: float, seed: int, b: int) -> np.ndarray:
    """The perturbed scores logits / T - log(-log u) that gumbel_draft maximises."""
    logits = np.asarray(logits, dtype=np.float64)
    Bm1, V = logits.shape
    u = np.stack([draft_uniforms(seed, b, i, V) for i in range(1, Bm1 + 1)])
    return logits / float(temperature) - np.log(-np.log(u))
