"""The lossless invariant ("DFlash — 블록 확산 드래프터로 6배 빨라지는 투기적 디코딩" §1):
speculative greedy decoding must emit exactly the target's own greedy tokens,
whatever the drafter proposes. Also pins the tiny target against the
`transformers` causal Llama model."""
import numpy as np
import pytest
import torch

from oracle import dflash as O
from oracle import target as T
from block_diffusion_speculative_cycle_b200 import synth
from tests import hf_pin
from tests.tiny_setup import TARGET_CFG, tiny_pair


def test_tiny_target_matches_library_causal_lm():
    tw, _ = tiny_pair()
    tgt = T.TinyTarget(TARGET_CFG, tw, n_feat=3, max_len=64)
    toks = synth.make_tokens(TARGET_CFG, 20, seed=9).tolist()
    logits, feats = tgt.forward(toks, 0, tgt.new_cache())
    m = hf_pin.causal_lm(TARGET_CFG, tw)
    with torch.no_grad():
        out = m(torch.tensor([toks]), output_hidden_states=True)
    np.testing.assert_allclose(logits, out.logits[0].numpy(), rtol=1e-5, atol=1e-5)
    # the library lists the embedding output first, then each layer's output
    # (the last one after the final norm); taps 0 and 1 are plain layer outputs
    H = TARGET_CFG.hidden
    np.testing.assert_allclose(feats[:, :H], out.hidden_states[1][0].numpy(), rtol=1e-5, atol=1e-5)
    np.testing.assert_allclose(feats[:, H:2 * H], out.hidden_states[2][0].numpy(), rtol=1e-5, atol=1e-5)
    assert T.tapped_layers(4, 3) == [0, 1, 3]
    assert T.tapped_layers(36, 5) == [0, 8, 17, 26, 35]


def test_block_forward_equals_token_by_token():
    tw, _ = tiny_pair()
    tgt = T.TinyTarget(TARGET_CFG, tw, n_feat=3, max_len=64)
    toks = synth.make_tokens(TARGET_CFG, 12, seed=4).tolist()
    c1 = tgt.new_cache()
    l1, f1 = tgt.forward(toks, 0, c1)
    c2 = tgt.new_cache()
    l2, f2 = tgt.forward(toks[:5], 0, c2)
    l3, f3 = tgt.forward(toks[5:], 5, c2)
    np.testing.assert_array_equal(l1, np.concatenate([l2, l3]))
    np.testing.assert_array_equal(f1, np.concatenate([f2, f3]))


def _run(seed, n_new, B, cheat_p=None):
    tw, dw = tiny_pair(seed)
    tgt = T.TinyTarget(TARGET_CFG, tw, n_feat=3, max_len=64 + n_new + B + 1)
    prompt = synth.make_tokens(TARGET_CFG, 64, seed=50 + seed).tolist()
    ref = T.greedy_decode(tgt, prompt, n_new)
    drafter = T.OracleDrafter(synth.TINY, dw)
    draft_fn = drafter.draft
    if cheat_p is not None:
        rng = np.random.default_rng(seed)

        def draft_fn(anchor, P, B_):
            d = list(drafter.draft(anchor, P, B_))
            for i in range(1, B_):
                k = P + i - len(prompt)
                if k < len(ref) and rng.random() < cheat_p:
                    d[i - 1] = ref[k]
            return d
    stats = {}
    out = T.spec_generate(tgt, prompt, n_new, B, drafter.inject, draft_fn, O.verify, stats)
    return out, ref, stats["accepted"]


@pytest.mark.parametrize("seed", [0, 1])
def test_spec_decode_is_lossless(seed):
    out, ref, acc = _run(seed, 256, 4)
    assert out == ref


def test_spec_decode_lossless_at_every_acceptance_length():
    out, ref, acc = _run(2, 256, 4, cheat_p=0.75)
    assert out == ref
    assert set(acc) == {0, 1, 2, 3}
