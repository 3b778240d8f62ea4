"""The library's block-size policy (host C++) and its device acceptance counts
against oracle/policy.py.

The policy's arithmetic is the same double-precision sequence as the oracle's,
so expected tokens agree bit for bit and the choices are identical on random
histories and costs; the device counts are integer atomics, compared exactly."""
import numpy as np
import pytest
import torch

from block_diffusion_speculative_cycle_b200 import BlockPolicy, dflash_acceptance_count
from oracle import policy as Pol


@pytest.mark.parametrize("seed", range(4))
def test_policy_matches_the_oracle_on_random_histories(seed):
    rng = np.random.default_rng(seed)
    n_pos, cands, decay = 17, [2, 4, 8, 10, 16], float(rng.uniform(0.5, 1.0))
    lib, ref = BlockPolicy(cands, decay, n_pos), Pol.BlockPolicy(cands, decay, n_pos)
    for _ in range(20):
        B = int(rng.choice(cands))
        acc = rng.integers(0, B, size=int(rng.integers(1, 40)))
        t, a = Pol.acceptance_counts(acc, B, n_pos)
        lib.observe(t, a)
        ref.observe(t, a)
        for Bq in range(1, n_pos + 1):
            assert lib.expected_tokens(Bq) == ref.expected_tokens(Bq)
        costs = rng.uniform(0.5, 3.0, size=len(cands))
        assert lib.choose(list(costs)) == ref.choose(costs)
        bs = int(rng.integers(1, 64))
        assert lib.choose_linear(bs, 1.0, 0.01) == ref.choose_linear(bs, 1.0, 0.01)
    lib.close()


def test_policy_rejects_bad_arguments():
    with pytest.raises(Exception):
        BlockPolicy([0, 4], 0.9, 17)          # block size 0
    with pytest.raises(Exception):
        BlockPolicy([4, 32], 0.9, 17)         # beyond n_pos
    p = BlockPolicy([4, 8], 0.9, 17)
    with pytest.raises(Exception):
        p.choose([1.0])                       # one cost per candidate
    with pytest.raises(Exception):
        p.choose([1.0, 0.0])                  # costs must be positive
    assert p.expected_tokens(99) == -1.0
    p.close()


@pytest.mark.gpu
@pytest.mark.parametrize("bs,B", [(1, 16), (32, 16), (7, 10), (5, 1), (300, 8)])
def test_device_acceptance_counts_match_the_oracle(bs, B):
    rng = np.random.default_rng(bs + B)
    n_pos = 17
    counts = torch.zeros(2 * n_pos, dtype=torch.int64, device="cuda")
    want_t, want_a = np.zeros(n_pos, np.int64), np.zeros(n_pos, np.int64)
    for _ in range(3):   # counts accumulate across calls
        acc = rng.integers(0, B, size=bs).astype(np.int32)
        dflash_acceptance_count(torch.from_numpy(acc).cuda(), B, counts)
        t, a = Pol.acceptance_counts(acc, B, n_pos)
        want_t += t
        want_a += a
    got = counts.cpu().numpy()
    np.testing.assert_array_equal(got[:n_pos], want_t)
    np.testing.assert_array_equal(got[n_pos:], want_a)
