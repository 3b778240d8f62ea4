"""Pins for oracle/policy.py (dynamic block-size scheduling), against what the
mathematics fixes rather than the code's own formulas:

* acceptance counts: hand-worked cases of the definition (a cycle that accepted
  a drafts tested positions 1..a+1, within the block);
* expected tokens: the closed form of the geometric sum for a constant
  acceptance rate, and brute-force enumeration of every accept/reject pattern
  of the drafts for position-dependent rates;
* the estimator converges to the rates of a simulated acceptance process;
* the choice: free verification (cost independent of B) picks the largest
  block, drafts that are never accepted pick the smallest, and under a cost that
  grows with bs * B the chosen block never grows with the concurrency."""
import itertools

import numpy as np

from oracle import policy as Pol


def test_acceptance_counts_hand_worked():
    # B = 4: a = 0 tested position 1 (rejected); a = 2 tested 1..3, accepted 1..2;
    # a = 3 (all accepted) tested 1..3, accepted 1..3
    t, a = Pol.acceptance_counts([0, 2, 3], B=4, n_pos=6)
    np.testing.assert_array_equal(t, [0, 3, 2, 2, 0, 0])
    np.testing.assert_array_equal(a, [0, 2, 2, 1, 0, 0])
    t, a = Pol.acceptance_counts([0, 0], B=1, n_pos=3)   # B = 1 drafts nothing
    assert t.sum() == 0 and a.sum() == 0


def _policy_with_alpha(alpha, n_pos=17):
    """A policy whose estimates equal alpha exactly: (A + 1) / (T + 2) = alpha."""
    p = Pol.BlockPolicy([1, 2, 4, 8, 16], decay=1.0, n_pos=n_pos)
    T = np.full(n_pos, 1e6)
    p.T = T
    p.A = np.asarray(alpha) * (T + 2.0) - 1.0
    np.testing.assert_allclose(p.alpha(), alpha, rtol=1e-12)
    return p


def test_expected_tokens_constant_rate_closed_form():
    for al in (0.3, 0.62, 0.9):
        p = _policy_with_alpha(np.full(17, al))
        for B in (1, 2, 5, 16):
            closed = 1.0 + al * (1 - al ** (B - 1)) / (1 - al)
            assert abs(p.expected_tokens(B) - closed) < 1e-9


def test_expected_tokens_by_enumeration():
    rng = np.random.default_rng(0)
    alpha = rng.uniform(0.2, 0.95, size=17)
    p = _policy_with_alpha(alpha)
    for B in (1, 2, 3, 6):
        e = 0.0
        for pattern in itertools.product([0, 1], repeat=B - 1):
            prob = np.prod([alpha[i + 1] if x else 1 - alpha[i + 1] for i, x in enumerate(pattern)])
            a = next((i for i, x in enumerate(pattern) if not x), B - 1)   # leading accepts
            e += prob * (a + 1)
        assert abs(p.expected_tokens(B) - e) < 1e-9


def test_estimator_converges_to_the_simulated_rates():
    rng = np.random.default_rng(1)
    true = np.concatenate([[0.0], np.linspace(0.9, 0.5, 15)])
    p = Pol.BlockPolicy([4, 8, 16], decay=1.0, n_pos=16)
    for _ in range(400):
        acc = []
        for _ in range(32):
            a = 0
            while a < 15 and rng.random() < true[a + 1]:
                a += 1
            acc.append(a)
        p.observe(*Pol.acceptance_counts(acc, 16, 16))
    np.testing.assert_allclose(p.alpha()[1:9], true[1:9], atol=0.02)


def test_choice_limits_and_monotonicity():
    good = _policy_with_alpha(np.full(17, 0.8))
    assert good.choose([1.0] * 5) == 16                 # verification costs the same at any B
    bad = Pol.BlockPolicy([1, 2, 4, 8, 16], decay=1.0, n_pos=17)
    bad.observe(*Pol.acceptance_counts([0] * 10000, 16, 17))
    assert bad.choose_linear(1, 1.0, 0.01) == 1          # drafts never accepted: no drafting
    chosen = [good.choose_linear(bs, 1.0, 0.01) for bs in (1, 2, 4, 8, 16, 32, 64, 128)]
    assert all(x >= y for x, y in zip(chosen, chosen[1:])) and chosen[0] == 16 and chosen[-1] < 16
