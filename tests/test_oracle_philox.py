"""Pins for oracle/philox.py, the counter-based generator the sampled drafter's
Gumbel noise comes from: the published known-answer vectors of Philox4x32-10,
and properties of the uniform mapping that hold by construction of the
definition (range, exactness in float32, independence of the counter words)."""
import os

import numpy as np

from oracle import philox as X

HERE = os.path.dirname(os.path.abspath(__file__))


def kat_vectors():
    rows = []
    with open(os.path.join(HERE, "golden", "philox4x32_10_kat.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                w = [int(t, 16) for t in line.split()]
                rows.append((w[0:4], w[4:6], w[6:10]))
    return rows


def test_known_answer_vectors():
    rows = kat_vectors()
    assert len(rows) == 3
    for ctr, key, want in rows:
        got = [int(x) for x in X.philox4x32_10(ctr, key)]
        assert got == want


def test_vectorised_counters_match_scalar_calls():
    ctr = (np.arange(5), np.full(5, 7), np.arange(5) * 3, np.zeros(5))
    many = X.philox4x32_10(ctr, (11, 12))
    for j in range(5):
        one = X.philox4x32_10((j, 7, 3 * j, 0), (11, 12))
        np.testing.assert_array_equal(many[:, j], one)


def test_uniforms_lie_strictly_inside_the_unit_interval_and_are_float32_exact():
    u = X.word_to_uniform(np.array([0, 511, 512, 0xFFFFFFFF], dtype=np.uint64))
    assert u[0] == 0.5 / 2 ** 23 and u[3] == 1 - 0.5 / 2 ** 23
    assert u[0] == u[1] and u[2] == 1.5 / 2 ** 23   # the low 9 bits are dropped
    assert np.all((u > 0) & (u < 1))
    np.testing.assert_array_equal(u.astype(np.float32).astype(np.float64), u)


def test_draft_uniforms_follow_the_word_layout_and_look_uniform():
    V = 1000
    u = X.draft_uniforms(0x1234_5678_9ABC, b=3, i=5, V=V)
    # entry v is word (v mod 128) div 32 of the block at counter (v div 128, v mod 32, i, b)
    for v in (0, 1, 31, 32, 127, 128, 999):
        w = X.philox4x32_10((v // 128, v % 32, 5, 3), (0x5678_9ABC, 0x1234))
        assert u[v] == X.word_to_uniform(w[(v % 128) // 32])
    # different positions and requests give different streams
    assert not np.array_equal(u, X.draft_uniforms(0x1234_5678_9ABC, b=3, i=4, V=V))
    assert not np.array_equal(u, X.draft_uniforms(0x1234_5678_9ABC, b=2, i=5, V=V))
    # moments of U(0, 1) within 5 standard errors on 100k draws
    big = np.concatenate([X.draft_uniforms(7, b, 1, 10000) for b in range(10)])
    se = np.sqrt(1 / 12 / big.size)
    assert abs(big.mean() - 0.5) < 5 * se
    assert abs(big.var() - 1 / 12) < 5 * np.sqrt(1 / 180 / big.size)
