"""Pins for the oracle's injection and block drafter.

The decoder-layer arithmetic is pinned against the `transformers` Llama layer
(a library implementation written independently of the oracle), driven the way
the DFlash pages describe the drafter: the injected context K/V sit in the
layer's cache and the block attends to them and to itself with no mask."""
import numpy as np
import pytest
import torch

from oracle import dflash as O
from block_diffusion_speculative_cycle_b200 import synth
from tests import hf_pin

SMALL = synth.TINY.replace(hidden=64, intermediate=96, n_q_heads=4, n_kv_heads=2, head_dim=16, vocab=50,
                           n_feat_layers=3, target_hidden=32, rope_theta=1e4, dtype="f32", n_layers=2)


def small_weights(cfg=SMALL, seed=0):
    w = synth.make_drafter_weights(cfg, seed=seed, std=0.2)
    # non-trivial gains so a dropped gain fails
    g = torch.Generator().manual_seed(seed + 100)
    for lw in w["layers"]:
        lw["attn_norm"] = 1.0 + 0.3 * torch.randn(cfg.hidden, generator=g)
        lw["mlp_norm"] = 1.0 + 0.3 * torch.randn(cfg.hidden, generator=g)
    w["final_norm"] = 1.0 + 0.3 * torch.randn(cfg.hidden, generator=g)
    return w


def library_inject(cfg, layers, rot, c, start):
    """K/V of context rows through the library's own k_proj / v_proj / RoPE."""
    from transformers.models.llama import modeling_llama as ml
    n = c.shape[0]
    x = torch.tensor(c)[None]
    pos = torch.arange(start, start + n)[None]
    cos, sin = rot(x, pos)
    out = []
    for layer in layers:
        k = layer.self_attn.k_proj(x).view(1, n, cfg.n_kv_heads, cfg.head_dim).transpose(1, 2)
        v = layer.self_attn.v_proj(x).view(1, n, cfg.n_kv_heads, cfg.head_dim).transpose(1, 2)
        _, k = ml.apply_rotary_pos_emb(k, k, cos, sin)
        out.append((k, v))
    return out


def library_draft(cfg, weights, layers, rot, kv_ctx, anchor, P, B):
    from transformers.cache_utils import DynamicCache
    cache = DynamicCache()
    for l, (k, v) in enumerate(kv_ctx):
        cache.update(k, v, l)
    emb = torch.tensor(O.f64(weights["embed"]))
    ids = [anchor] + [cfg.mask_token_id] * (B - 1)
    x = emb[ids][None]
    pos = torch.arange(P, P + B)[None]
    cos, sin = rot(x, pos)
    hidden = []
    with torch.no_grad():
        for layer in layers:
            out = layer(x, attention_mask=None, position_ids=pos, past_key_values=cache, use_cache=True,
                        position_embeddings=(cos, sin))
            x = out[0] if isinstance(out, tuple) else out
            hidden.append(x[0].numpy().copy())
    y = torch.nn.functional.rms_norm(x[0], (cfg.hidden,), torch.tensor(O.f64(weights["final_norm"])), cfg.rms_eps)
    logits = y[1:] @ torch.tensor(O.f64(weights["lm_head"])).T
    return hidden, y.numpy(), logits.numpy()


@pytest.mark.parametrize("P,B", [(0, 1), (0, 4), (1, 2), (5, 4), (23, 3)])
def test_inject_and_draft_match_library_layers(P, B):
    cfg = SMALL
    w = small_weights(cfg, seed=P + B)
    feats = O.f64(synth.make_features(cfg, P, seed=7)) if P else np.zeros((0, cfg.feat_dim))
    c, kv = O.inject(cfg, w, feats, 0)
    _, layers, rot = hf_pin.decoder_layers(cfg, w)
    with torch.no_grad():
        lib_kv = library_inject(cfg, layers, rot, c, 0) if P else [
            (torch.zeros(1, cfg.n_kv_heads, 0, cfg.head_dim, dtype=torch.float64),) * 2 for _ in layers]
    for (k, v), (lk, lv) in zip(kv, lib_kv):
        np.testing.assert_allclose(k, lk[0].transpose(0, 1).numpy(), rtol=1e-5, atol=1e-6)
        np.testing.assert_allclose(v, lv[0].transpose(0, 1).numpy(), rtol=1e-12, atol=1e-12)
    cache = O.Cache(cfg)
    cache.write(0, kv)
    res = O.draft_block(cfg, w, anchor=3, cache=cache, B=B)
    hidden, y, logits = library_draft(cfg, w, layers, rot, lib_kv, 3, P, B)
    for a, b in zip(res["hidden"][:-1], hidden):
        np.testing.assert_allclose(a, b, rtol=1e-5, atol=1e-5)
    np.testing.assert_allclose(res["hidden"][-1], y, rtol=1e-5, atol=1e-5)
    np.testing.assert_allclose(res["logits"], logits, rtol=1e-5, atol=1e-5)


def test_fusion_projection_is_library_linear():
    cfg = SMALL
    w = small_weights(cfg)
    f = O.f64(synth.make_features(cfg, 6))
    ref = torch.nn.functional.linear(torch.tensor(f), torch.tensor(O.f64(w["fc"]))).numpy()
    c, _ = O.inject(cfg, w, f, 0)
    np.testing.assert_allclose(c, ref, rtol=1e-12, atol=1e-12)


def test_inject_linear_and_chunkable():
    cfg = SMALL
    w = small_weights(cfg)
    f1 = O.f64(synth.make_features(cfg, 8, seed=1))
    f2 = O.f64(synth.make_features(cfg, 8, seed=2))
    _, a = O.inject(cfg, w, f1, 4)
    _, b = O.inject(cfg, w, f2, 4)
    _, s = O.inject(cfg, w, f1 + f2, 4)
    for (ka, va), (kb, vb), (ks, vs) in zip(a, b, s):
        np.testing.assert_allclose(ks, ka + kb, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(vs, va + vb, rtol=1e-10, atol=1e-12)
    # inject 5 rows then 3 rows == inject 8 rows at once
    whole = O.Cache(cfg); whole.write(0, O.inject(cfg, w, f1, 0)[1])
    parts = O.Cache(cfg); parts.write(0, O.inject(cfg, w, f1[:5], 0)[1]); parts.write(5, O.inject(cfg, w, f1[5:], 5)[1])
    for l in range(cfg.n_layers):
        np.testing.assert_allclose(parts.k[l], whole.k[l], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(parts.v[l], whole.v[l], rtol=1e-12, atol=1e-14)


def test_block_attention_is_non_causal():
    cfg = SMALL
    w = small_weights(cfg)
    x = np.random.default_rng(0).normal(size=(4, cfg.hidden))
    pos = np.arange(10, 14)
    kc = np.random.default_rng(1).normal(size=(10, cfg.n_kv_heads, cfg.head_dim))
    vc = np.random.default_rng(2).normal(size=(10, cfg.n_kv_heads, cfg.head_dim))
    y0 = O.drafter_layer(cfg, w["layers"][0], x, pos, kc, vc)
    x2 = x.copy(); x2[3] += 1.0
    y1 = O.drafter_layer(cfg, w["layers"][0], x2, pos, kc, vc)
    # the last block row changes the outputs of every earlier row
    assert np.all(np.abs(y1[:3] - y0[:3]).max(axis=1) > 1e-6)


def test_context_permutation_invariance_of_draft():
    cfg = SMALL
    w = small_weights(cfg)
    feats = O.f64(synth.make_features(cfg, 12, seed=3))
    _, kv = O.inject(cfg, w, feats, 0)
    c0 = O.Cache(cfg); c0.write(0, kv)
    perm = np.random.default_rng(5).permutation(12)
    c1 = O.Cache.from_arrays(cfg, [k[perm] for k, _ in kv], [v[perm] for _, v in kv])
    r0 = O.draft_block(cfg, w, 7, c0, 4)
    r1 = O.draft_block(cfg, w, 7, c1, 4)
    np.testing.assert_allclose(r0["logits"], r1["logits"], rtol=1e-10, atol=1e-12)


def test_zero_layer_drafter_closed_form():
    # no layers: every masked row predicts argmax(RMSNorm(E[mask]) · W_lm)
    cfg = SMALL.replace(n_layers=0)
    w = small_weights(cfg)
    res = O.draft_block(cfg, w, 5, O.Cache(cfg), 4)
    e = O.f64(w["embed"])[cfg.mask_token_id]
    y = e / np.sqrt(np.mean(e * e) + cfg.rms_eps) * O.f64(w["final_norm"])
    t = int(np.argmax(O.f64(w["lm_head"]) @ y))
    assert list(res["draft"]) == [t, t, t]


def test_attention_to_context_depends_on_relative_position_only():
    # shifting context and block together by 40 positions leaves the pass unchanged (RoPE)
    cfg = SMALL
    w = small_weights(cfg)
    feats = O.f64(synth.make_features(cfg, 9, seed=4))
    c0 = O.Cache(cfg); c0.write(0, O.inject(cfg, w, feats, 0)[1])
    shifted = O.inject(cfg, w, feats, 40)[1]
    r0 = O.draft_block(cfg, w, 2, c0, 3)
    x = O.f64(w["embed"])[[2, cfg.mask_token_id, cfg.mask_token_id]]
    for l, lw in enumerate(w["layers"]):
        x = O.drafter_layer(cfg, lw, x, np.arange(49, 52), shifted[l][0], shifted[l][1])
    np.testing.assert_allclose(x, r0["hidden"][cfg.n_layers - 1], rtol=1e-9, atol=1e-10)


# --------------------------------------------------------------------------- sliding window

def _window_case(seed=0, P=40, B=4):
    from block_diffusion_speculative_cycle_b200 import synth
    cfg = synth.TINY
    w = synth.make_drafter_weights(cfg, seed=seed, share_embed_lm_head=True)
    feats = synth.make_features(cfg, P, seed=seed + 1)
    cache = O.Cache(cfg)
    cache.write(0, O.inject(cfg, w, feats, 0)[1])
    return cfg, w, cache, feats


def test_window_wider_than_the_context_is_no_window():
    cfg, w, cache, _ = _window_case()
    full = O.draft_block(cfg, w, 5, cache, 4)
    for W in (40, 41, 1000):
        win = O.draft_block(cfg, w, 5, cache, 4, window=W)
        for a, b in zip(full["hidden"], win["hidden"]):
            np.testing.assert_array_equal(a, b)


def test_window_ignores_exactly_the_rows_before_it():
    """Changing context rows older than the window leaves the pass unchanged; changing
    the oldest row inside it does not."""
    cfg, w, cache, feats = _window_case()
    W, P = 16, 40
    base = O.draft_block(cfg, w, 5, cache, 4, window=W)
    old = O.Cache(cfg)
    f2 = feats.clone()
    f2[: P - W] = -f2[: P - W] * 3.0
    old.write(0, O.inject(cfg, w, f2, 0)[1])
    same = O.draft_block(cfg, w, 5, old, 4, window=W)
    for a, b in zip(base["hidden"], same["hidden"]):
        np.testing.assert_array_equal(a, b)
    inside = O.Cache(cfg)
    f3 = feats.clone()
    f3[P - W] = -f3[P - W] * 3.0
    inside.write(0, O.inject(cfg, w, f3, 0)[1])
    moved = O.draft_block(cfg, w, 5, inside, 4, window=W)
    assert np.abs(moved["hidden"][-1] - base["hidden"][-1]).max() > 1e-6


def test_window_equals_a_cache_holding_only_its_rows():
    """The window's rows keep their absolute positions: attending to the last W rows
    of a long context is attending to a cache that holds only them, at the same P
    (checked through the decoder library pin below: block_attention over the window
    equals scaled_dot_product_attention over those keys)."""
    import torch
    cfg, w, cache, _ = _window_case()
    W, P = 10, 40
    win = O.draft_block(cfg, w, 7, cache, 4, window=W)
    only = O.Cache.from_arrays(cfg, [k[P - W:P] for k in cache.k], [v[P - W:P] for v in cache.v])
    ref = O.draft_block(cfg, w, 7, only, 4, ctx_len=P)   # positions P.., keys: the W kept rows
    for a, b in zip(win["hidden"], ref["hidden"]):
        np.testing.assert_array_equal(a, b)
    # the first layer's attention of the windowed pass against SDPA on those keys
    lw = w["layers"][0]
    x = O.f64(w["embed"])[[7] + [cfg.mask_token_id] * 3]
    h = O.rms_norm(x, lw["attn_norm"], cfg.rms_eps)
    pos = np.arange(P, P + 4)
    q = O.apply_rope(O.linear(h, lw["wq"]).reshape(4, cfg.n_q_heads, cfg.head_dim), pos, cfg.rope_theta)
    k = O.apply_rope(O.linear(h, lw["wk"]).reshape(4, cfg.n_kv_heads, cfg.head_dim), pos, cfg.rope_theta)
    v = O.linear(h, lw["wv"]).reshape(4, cfg.n_kv_heads, cfg.head_dim)
    keys = np.concatenate([cache.k[0][P - W:P], k]); vals = np.concatenate([cache.v[0][P - W:P], v])
    o = O.block_attention(q, keys, vals)
    g = cfg.n_q_heads // cfg.n_kv_heads
    tq = torch.from_numpy(q).permute(1, 0, 2)[None]
    tk = torch.from_numpy(keys).permute(1, 0, 2).repeat_interleave(g, 0)[None]
    tv = torch.from_numpy(vals).permute(1, 0, 2).repeat_interleave(g, 0)[None]
    ref_o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)[0].permute(1, 0, 2).numpy()
    np.testing.assert_allclose(o, ref_o, rtol=1e-10, atol=1e-12)
