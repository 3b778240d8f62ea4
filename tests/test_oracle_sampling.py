"""Pins for oracle/sampling.py (sampled verification), checked against what the
mathematics fixes rather than against the code's own formula:

* the distribution of the first emitted token equals the target's p_0 exactly
  (up to the quadrature step) for any drafter distribution q, computed by
  integrating over the draft and both uniforms on a fine midpoint grid;
* special cases: q == p accepts everything; a draft the target gives
  probability 0 is always rejected; at vanishing temperature the rule reduces
  to the greedy verify of oracle.dflash;
* the whole speculative loop over a small Markov-chain target emits sequences
  with the target's own joint distribution (seeded Monte Carlo, total-variation
  bound);
* Gumbel-max draws follow softmax(logits / T) (seeded Monte Carlo) and reduce
  to the argmax at vanishing temperature."""
import itertools

import numpy as np
import pytest

from oracle import dflash as O
from oracle import sampling as S


def first_token_marginal(p, q, n_grid=4000):
    """P(first emitted token = v) for B = 2 (one draft d ~ q[0]), integrating the
    acceptance uniform and the resampling uniform over midpoint grids."""
    V = p.shape[1]
    us = (np.arange(n_grid) + 0.5) / n_grid
    out = np.zeros(V)
    for d in range(V):
        if q[0, d] == 0:
            continue
        for ua in us[:: n_grid // 400]:   # 400 acceptance points (the test is a threshold in u)
            # the resampling draw only matters on rejection; integrate it on the full grid
            a, _ = S.sampled_verify(p, q, [d], [ua], 0.5)
            w = q[0, d] / 400
            if a == 1:
                out[d] += w
            else:
                counts = np.bincount([S.sampled_verify(p, q, [d], [ua], uf)[1] for uf in us[::40]], minlength=V)
                out += w * counts / counts.sum()
    return out


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_first_token_follows_the_target_distribution(seed):
    rng = np.random.default_rng(seed)
    V = 5
    p = S.softmax_t(rng.normal(size=(2, V)) * 2, 1.0)
    q = S.softmax_t(rng.normal(size=(1, V)) * 2, 1.0)
    m = first_token_marginal(p, q)
    np.testing.assert_allclose(m, p[0], atol=4e-3)
    # and the drafter's own distribution is far from it (the check has teeth)
    assert np.abs(q[0] - p[0]).max() > 0.05


def test_equal_distributions_accept_every_draft():
    rng = np.random.default_rng(3)
    p = S.softmax_t(rng.normal(size=(5, 7)), 0.7)
    q = p[:4]
    for trial in range(50):
        d = [S.sample_index(q[i], rng.random()) for i in range(4)]
        a, nxt = S.sampled_verify(p, q, d, rng.random(4) * 0.999999, rng.random())
        assert a == 4
        assert 0 <= nxt < 7


def test_draft_with_zero_target_probability_is_rejected():
    p = np.array([[0.0, 0.5, 0.5], [0.2, 0.3, 0.5]])
    q = np.array([[1.0, 0.0, 0.0]])
    for u in np.linspace(0, 0.999, 50):
        a, nxt = S.sampled_verify(p, q, [0], [u], 0.3)
        assert a == 0 and nxt in (1, 2)
    # the correction comes from max(0, p - q) normalised = p here (q has no mass where p has)
    assert S.sampled_verify(p, q, [0], [0.5], 0.25)[1] == 1
    assert S.sampled_verify(p, q, [0], [0.5], 0.75)[1] == 2


@pytest.mark.parametrize("seed", range(6))
def test_vanishing_temperature_reduces_to_greedy_verify(seed):
    rng = np.random.default_rng(10 + seed)
    B, V = 6, 11
    logits = rng.normal(size=(B, V))
    g = logits.argmax(-1)
    d = [int(g[i - 1]) if rng.random() < 0.7 else int(rng.integers(V)) for i in range(1, B)]
    p = S.softmax_t(logits, 1e-4)
    q = np.zeros((B - 1, V))
    q[np.arange(B - 1), d] = 1.0   # a greedy drafter: all mass on its draft
    got = S.sampled_verify(p, q, d, rng.random(B - 1) * 0.999, rng.random())
    assert got == O.verify(logits, d)


def test_speculative_loop_matches_the_target_joint_distribution():
    """A Markov-chain 'target' p(next | prev) over V tokens and a block drafter
    with its own per-position distributions; the first L emitted tokens of the
    speculative loop must follow the chain's joint law."""
    rng = np.random.default_rng(7)
    V, B, L, N = 3, 3, 3, 40000
    T = S.softmax_t(rng.normal(size=(V, V)) * 1.5, 1.0)          # T[prev] = p(. | prev)
    Q = S.softmax_t(rng.normal(size=(B - 1, V, V)) * 1.5, 1.0)   # Q[i][anchor]: drafter at mask i
    start = 1
    counts = {}
    for _ in range(N):
        out, anchor = [], start
        while len(out) < L:
            d = [S.sample_index(Q[i][anchor], rng.random()) for i in range(B - 1)]
            blk = [anchor] + d
            p = np.stack([T[blk[j]] for j in range(B)])
            q = np.stack([Q[i][anchor] for i in range(B - 1)])
            a, nxt = S.sampled_verify(p, q, d, rng.random(B - 1), rng.random())
            out += d[:a] + [nxt]
            anchor = nxt
        key = tuple(out[:L])
        counts[key] = counts.get(key, 0) + 1
    tv = 0.0
    for seq in itertools.product(range(V), repeat=L):
        prob, prev = 1.0, start
        for t in seq:
            prob *= T[prev, t]
            prev = t
        tv += abs(counts.get(seq, 0) / N - prob)
    assert tv / 2 < 0.02


def test_gumbel_max_draws_follow_the_softmax():
    rng = np.random.default_rng(5)
    logits = np.array([[0.3, -1.0, 1.2, 0.0]])
    T, N = 0.8, 60000
    u = rng.random(size=(N, 4))
    draws = S.gumbel_sample(np.repeat(logits, N, 0), T, u)
    freq = np.bincount(draws, minlength=4) / N
    np.testing.assert_allclose(freq, S.softmax_t(logits, T)[0], atol=8e-3)
    # vanishing temperature: the argmax
    assert (S.gumbel_sample(np.repeat(logits, 100, 0), 1e-6, rng.random(size=(100, 4))) == 2).all()


def test_gumbel_draft_uses_the_philox_stream_and_follows_softmax():
    """gumbel_draft is the Gumbel-max rule over the Philox draft uniforms: its
    token at position i maximises the perturbed scores, and over many requests
    (independent streams) the draws follow softmax(logits / T)."""
    from oracle import philox as X
    rng = np.random.default_rng(5)
    logits = rng.normal(size=(3, 6))
    d = S.gumbel_draft(logits, 0.8, seed=99, b=2)
    for i in range(1, 4):
        u = X.draft_uniforms(99, 2, i, 6)
        assert d[i - 1] == int(np.argmax(logits[i - 1] / 0.8 - np.log(-np.log(u))))
    draws = np.array([S.gumbel_draft(logits[:1], 0.8, seed=7, b=b)[0] for b in range(20000)])
    freq = np.bincount(draws, minlength=6) / draws.size
    np.testing.assert_allclose(freq, S.softmax_t(logits[:1], 0.8)[0], atol=0.012)
