"""Pins for the oracle's building blocks: closed forms, invariants and library
routines that the oracle does not use itself."""
import numpy as np
import pytest
import torch

from oracle import dflash as O


def rng(seed=0):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- RMSNorm

def test_rms_norm_unit_rms_and_scale_invariance():
    x = rng().normal(size=(5, 64)) * 3.0
    y = O.rms_norm(x, np.ones(64), 0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-13)
    np.testing.assert_allclose(O.rms_norm(7.5 * x, np.ones(64), 0.0), y, rtol=1e-13)
    g = rng(1).normal(size=64)
    np.testing.assert_allclose(O.rms_norm(x, g, 0.0), y * g, rtol=1e-13)


def test_rms_norm_matches_torch_library():
    x = rng(2).normal(size=(7, 96))
    g = rng(3).normal(size=96)
    ref = torch.nn.functional.rms_norm(torch.tensor(x), (96,), torch.tensor(g), eps=1e-6).numpy()
    np.testing.assert_allclose(O.rms_norm(x, g, 1e-6), ref, rtol=1e-12, atol=1e-12)


def test_rms_norm_eps_closed_form():
    # a constant row c: rms = |c|, so y = c / sqrt(c^2 + eps)
    x = np.full((1, 8), 0.01)
    np.testing.assert_allclose(O.rms_norm(x, np.ones(8), 1e-4), 0.01 / np.sqrt(1e-4 + 1e-4), rtol=1e-14)


# ---------------------------------------------------------------- SiLU

def test_silu_matches_torch_and_limits():
    x = np.linspace(-30, 30, 601)
    np.testing.assert_allclose(O.silu(x), torch.nn.functional.silu(torch.tensor(x)).numpy(), rtol=1e-13, atol=1e-300)
    assert O.silu(np.array([0.0]))[0] == 0.0
    np.testing.assert_allclose(O.silu(np.array([40.0])), 40.0, rtol=1e-15)
    assert abs(O.silu(np.array([-40.0]))[0]) < 1e-15


# ---------------------------------------------------------------- RoPE

def test_rope_position_zero_is_identity():
    x = rng(4).normal(size=(3, 2, 16))
    np.testing.assert_array_equal(O.apply_rope(x, [0, 0, 0], 1e4), x)


def test_rope_matches_complex_rotation():
    # pair (i, i+d/2) as the complex number x_i + j x_{i+d/2}, multiplied by e^{j pos w_i},
    # w_i = theta^(-2i/d): an independent formulation of the rotation
    d, theta = 16, 500.0
    x = rng(5).normal(size=(4, 3, d))
    pos = [0, 3, 17, 1000]
    w = np.array([theta ** (-2.0 * i / d) for i in range(d // 2)])
    z = x[..., : d // 2] + 1j * x[..., d // 2:]
    rot = np.exp(1j * np.outer(pos, w))[:, None, :]
    zr = z * rot
    np.testing.assert_allclose(O.apply_rope(x, pos, theta), np.concatenate([zr.real, zr.imag], -1),
                               rtol=1e-12, atol=1e-12)


def test_rope_first_pair_closed_form():
    # i = 0 has frequency 1 for any theta: the first pair turns by exactly pos radians
    x = np.zeros((1, 1, 8)); x[0, 0, 0] = 1.0
    y = O.apply_rope(x, [2], 1e6)
    np.testing.assert_allclose([y[0, 0, 0], y[0, 0, 4]], [np.cos(2.0), np.sin(2.0)], rtol=1e-15)


def test_rope_preserves_norm_and_relative_position():
    d = 32
    q = rng(6).normal(size=(1, 1, d))
    k = rng(7).normal(size=(1, 1, d))
    for p in (0, 5, 123):
        np.testing.assert_allclose(np.linalg.norm(O.apply_rope(q, [p], 1e4)), np.linalg.norm(q), rtol=1e-13)
    dots = [float(np.sum(O.apply_rope(q, [a], 1e4) * O.apply_rope(k, [b], 1e4)))
            for a, b in ((10, 3), (107, 100), (7, 0))]
    np.testing.assert_allclose(dots, dots[0], rtol=1e-10)


# ---------------------------------------------------------------- attention

def _sdpa(q, k, v):
    # library routine: q [B, nq, d], k/v [T, nkv, d]; GQA by repeating kv heads
    g = q.shape[1] // k.shape[1]
    Q = torch.tensor(q).permute(1, 0, 2)[None]
    K = torch.tensor(k).repeat_interleave(g, dim=1).permute(1, 0, 2)[None]
    V = torch.tensor(v).repeat_interleave(g, dim=1).permute(1, 0, 2)[None]
    o = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=False)
    return o[0].permute(1, 0, 2).numpy()


@pytest.mark.parametrize("T,Bq,nq,nkv,d", [(1, 1, 2, 1, 8), (5, 4, 4, 2, 16), (69, 16, 8, 2, 32), (3, 2, 4, 4, 8)])
def test_block_attention_matches_sdpa(T, Bq, nq, nkv, d):
    r = rng(T * 7 + Bq)
    q, k, v = r.normal(size=(Bq, nq, d)), r.normal(size=(T, nkv, d)), r.normal(size=(T, nkv, d))
    np.testing.assert_allclose(O.block_attention(q, k, v), _sdpa(q, k, v), rtol=1e-12, atol=1e-12)


def test_attention_equal_scores_give_mean_and_dominant_key_selects():
    d = 8
    v = rng(8).normal(size=(6, 1, d))
    q = np.zeros((2, 1, d))
    k = rng(9).normal(size=(6, 1, d))
    np.testing.assert_allclose(O.block_attention(q, k, v)[:, 0], np.tile(v[:, 0].mean(0), (2, 1)), rtol=1e-14)
    k2 = np.zeros((6, 1, d)); k2[4, 0, 0] = 1e3
    q2 = np.zeros((1, 1, d)); q2[0, 0, 0] = 1.0
    np.testing.assert_allclose(O.block_attention(q2, k2, v)[0, 0], v[4, 0], rtol=1e-12)


def test_attention_context_permutation_invariant():
    r = rng(10)
    q, k, v = r.normal(size=(4, 4, 16)), r.normal(size=(20, 2, 16)), r.normal(size=(20, 2, 16))
    perm = r.permutation(20)
    np.testing.assert_allclose(O.block_attention(q, k[perm], v[perm]), O.block_attention(q, k, v), rtol=1e-12)


def test_gqa_with_group_one_equals_per_head_attention():
    r = rng(11)
    q, k, v = r.normal(size=(3, 2, 8)), r.normal(size=(5, 2, 8)), r.normal(size=(5, 2, 8))
    o = O.block_attention(q, k, v)
    for h in range(2):
        np.testing.assert_allclose(o[:, h:h + 1], O.block_attention(q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1]),
                                   rtol=1e-14)


# ---------------------------------------------------------------- argmax

def test_greedy_argmax_brute_force_and_ties():
    r = rng(12)
    for _ in range(200):
        z = r.integers(-3, 4, size=r.integers(1, 9)).astype(np.float32)
        best = max(range(len(z)), key=lambda i: (z[i], -i))
        assert O.greedy_argmax(z) == best
    assert O.greedy_argmax(np.array([1.0, 3.0, 3.0, 2.0])) == 1
    assert O.greedy_argmax(np.array([np.nan, -np.inf, np.nan])) == 1
    assert O.greedy_argmax(np.array([np.nan, np.nan])) == 0
    assert O.greedy_argmax(np.array([-0.0, 0.0])) == 0
    assert O.greedy_argmax(np.array([np.nan, 2.0, np.inf, np.inf])) == 2
