"""Pins for the oracle's greedy verify: hand-worked golden cases, exhaustive
enumeration of small cases against the lossless characterisation, and the
planted-prefix inputs the benchmark uses."""
import itertools

import numpy as np
import pytest
import torch

from oracle import dflash as O
from block_diffusion_speculative_cycle_b200 import synth
from tests.golden_io import verify_cases


@pytest.mark.parametrize("case", verify_cases(), ids=lambda c: c[0])
def test_golden_cases(case):
    name, z, d, a, nxt = case
    assert O.verify(z, d) == (a, nxt)


def test_exhaustive_small_cases_are_lossless():
    # Characterisation: the committed tokens d_1..d_a, next must be exactly the target's
    # own greedy tokens g_0..g_a, and a must be maximal (a = B-1 or d_{a+1} != g_a).
    V = 3
    vals = [0.0, 1.0, 1.0]  # ties on purpose
    rows = sorted(set(itertools.permutations(vals)))
    for B in (1, 2, 3):
        for zr in itertools.product(rows, repeat=B):
            z = np.array(zr, dtype=np.float32)
            g = [min(i for i in range(V) if z[j, i] == z[j].max()) for j in range(B)]
            for d in itertools.product(range(V), repeat=B - 1):
                a, nxt = O.verify(z, d)
                committed = list(d[:a]) + [nxt]
                assert committed == g[:a + 1]
                assert a == B - 1 or d[a] != g[a]


@pytest.mark.parametrize("bs,B,V,mean", [(1, 16, 1000, 6.5), (32, 16, 257, 6.0), (8, 10, 300, 3.25), (4, 1, 50, 1.0)])
def test_planted_prefix_is_recovered(bs, B, V, mean):
    g = torch.Generator().manual_seed(bs * B)
    draft = torch.randint(0, V, (bs, B - 1), generator=g, dtype=torch.int32)
    z, planted = synth.planted_logits(draft, V, 2.0, mean, seed=bs + B, dtype=torch.bfloat16)
    a, nxt = O.verify_batch(O.f64(z), draft.numpy())
    np.testing.assert_array_equal(a, planted.numpy())
    for r in range(bs):
        assert nxt[r] == O.greedy_argmax(O.f64(z[r, a[r]]))


def test_planted_prefix_distribution_mean():
    draft = torch.zeros((4000, 15), dtype=torch.int32)
    draft[:, ::2] = 1
    _, planted = synth.planted_logits(draft, 8, 2.0, 6.5, seed=3, dtype=torch.float32)
    # geometric mean 6.5, clipped at 15: E[min(G,15)] = sum_{k=1..15} (1-p)^k
    p = 1 / 7.5
    expect = sum((1 - p) ** k for k in range(1, 16))
    assert abs(float(planted.float().mean()) - expect) < 0.25
