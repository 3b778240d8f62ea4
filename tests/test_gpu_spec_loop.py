"""The speculative loop entirely on the device (target forward, draft, verify,
commit and injection all in the library; nothing read back inside a cycle).

Lossless: its output equals the GPU target's own greedy decode (one token per
forward) token for token, and that equals the oracle target's greedy decode
(float64 NumPy). The target's block forward and its one-row forward give the
same logits bits (same split plan and per-row arithmetic), so the first
equality is exact by construction, whatever the drafter proposes. A variant
plants the reference continuation into the drafts with probability 0.75 (a
test-side hook between drafting and the target's forward), so that every
acceptance length 0..B-1 occurs."""
import numpy as np
import pytest
import torch

from block_diffusion_speculative_cycle_b200 import synth
from block_diffusion_speculative_cycle_b200.loop import GpuTarget, SpecDecoder, greedy_decode_gpu
from oracle import target as T
from tests.gpu_harness import PagedCache, make_drafter, to_dev
from tests.tiny_setup import TARGET_CFG, tiny_pair

pytestmark = pytest.mark.gpu

P0, N_TOK, PAGE = 64, 256, 64
CHECK = 4   # cycles between the host's progress checks (the loop may overshoot by that many blocks)


def setup(seed, bs, B, window=0):
    tw, dw = tiny_pair(seed)
    taps = T.tapped_layers(TARGET_CFG.n_layers, synth.TINY.n_feat_layers)
    cap = 2 * P0 + N_TOK + (2 * CHECK + 4) * B
    target = GpuTarget(TARGET_CFG, to_dev(tw), bs, max_rows=max(P0, B), capacity=cap, taps=taps, page_size=PAGE)
    pages = (cap + PAGE - 1) // PAGE
    table = torch.arange(bs * pages, dtype=torch.int32).reshape(bs, pages)
    drafter, _ = make_drafter(synth.TINY, dw, max_block=B, max_batch=bs, max_inject_rows=bs * max(P0, B),
                              page_size=PAGE, window=window)
    cache = PagedCache(synth.TINY, table, bs * pages, PAGE)
    dec = SpecDecoder(target, drafter, cache.k, cache.v, cache.table, bs * pages, cap - 2 * B, B, N_TOK + B)
    prompts = torch.stack([synth.make_tokens(TARGET_CFG, P0, seed=60 + seed * 10 + r) for r in range(bs)])
    return tw, target, drafter, dec, prompts


def planting_hook(ref_dev, p, seed):
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)

    def hook(dec):
        B = dec.B
        i = torch.arange(1, B, device="cuda", dtype=torch.int64)[None, :]
        idx = dec.ctx_len[:, None].to(torch.int64) + i - P0           # output index of position P + i
        ok = idx < ref_dev.shape[1]
        plant = (torch.rand(idx.shape, generator=gen, device="cuda") < p) & ok
        ref = torch.gather(ref_dev, 1, idx.clamp(max=ref_dev.shape[1] - 1))
        dec.draft[:, :B - 1] = torch.where(plant, ref, dec.draft[:, :B - 1].to(torch.int64)).to(torch.int32)
    return hook


@pytest.mark.parametrize("bs,B,seed,window", [(1, 4, 0, 0), (3, 8, 1, 0), (2, 16, 2, 48)])
def test_device_loop_is_lossless(bs, B, seed, window):
    tw, target, drafter, dec, prompts = setup(seed, bs, B, window)
    prompts_dev = prompts.cuda()
    ref_gpu = greedy_decode_gpu(target, prompts_dev, N_TOK)
    torch.cuda.synchronize()
    # the oracle target's own greedy decode agrees with the GPU target's
    for r in range(bs):
        tgt = T.TinyTarget(TARGET_CFG, tw, n_feat=3, max_len=P0 + N_TOK + 1)
        want = T.greedy_decode(tgt, prompts[r].tolist(), N_TOK)
        assert ref_gpu[r].cpu().tolist() == want, f"request {r}: GPU target vs oracle target"
    # plain speculative decoding
    dec.prefill(prompts_dev)
    out = dec.generate(N_TOK, check_every=CHECK)
    target.ctx.check()
    drafter.check()
    assert torch.equal(out, ref_gpu)
    target.close()
    drafter.close()


@pytest.mark.parametrize("B", [4, 8])
def test_device_loop_lossless_at_every_acceptance_length(B):
    bs = 2
    tw, target, drafter, dec, prompts = setup(3, bs, B)
    prompts_dev = prompts.cuda()
    ref_gpu = greedy_decode_gpu(target, prompts_dev, N_TOK)
    dec.prefill(prompts_dev)
    accepted = []

    def hook(d, h=planting_hook(ref_gpu.to(torch.int64), 0.75, 7)):
        h(d)

    orig_cycle = dec.cycle

    def cycle(hook_=None, stream=None):
        orig_cycle(hook, stream)
        accepted.append(dec.acc.clone())
    dec.cycle = cycle
    out = dec.generate(N_TOK, check_every=CHECK)
    target.ctx.check()
    drafter.check()
    assert torch.equal(out, ref_gpu)
    acc = torch.stack(accepted).cpu().numpy()
    assert set(np.unique(acc).tolist()) == set(range(B))   # every acceptance length 0..B-1
    target.close()
    drafter.close()
