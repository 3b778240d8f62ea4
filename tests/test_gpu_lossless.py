"""The lossless invariant with the CUDA path in the loop.

Speculative greedy decoding whose inject, draft and verify steps are the
library's (features from the oracle's tiny causal target, block logits of that
target checked by the GPU verify kernel) must reproduce the target's own greedy
decode token for token, whatever the drafter proposes. A second variant
overwrites drafts with the target's continuation at random, so that every
acceptance length 0..B-1 occurs and both the commit and the re-injection of a
full block are exercised. The drafter runs in fp32 (CUDA-core path) and in bf16
(tensor-core path, fp16 attention) over the same target."""
import numpy as np
import pytest
import torch

from block_diffusion_speculative_cycle_b200 import synth, verify as gpu_verify
from oracle import target as T
from tests.gpu_harness import PagedCache, make_drafter
from tests.tiny_setup import TARGET_CFG, tiny_pair

pytestmark = pytest.mark.gpu

PAGE = 64


class GpuDrafter:
    """The library's drafter for one request, wired for oracle.target.spec_generate."""

    def __init__(self, cfg, weights_cpu, max_len, B, max_inject, cache_dtype=None, window=0):
        self.cfg = cfg
        pages = (max_len + B + PAGE - 1) // PAGE
        table = torch.arange(pages, dtype=torch.int32)[None]
        self.d, _ = make_drafter(cfg, weights_cpu, max_block=B, max_batch=1, max_inject_rows=max_inject,
                                 page_size=PAGE, cache_dtype=cache_dtype, window=window)
        self.cache = PagedCache(cfg, table, pages, PAGE, dtype=cache_dtype)
        self.num_pages = pages

    def inject(self, feats, start):
        f = torch.as_tensor(np.asarray(feats, dtype=np.float32)).to(self.cfg.torch_dtype)
        n = f.shape[0]
        f = f.reshape(1, n, -1).cuda()
        n_new = torch.tensor([n], dtype=torch.int32, device="cuda")
        st = torch.tensor([start], dtype=torch.int32, device="cuda")
        self.d.inject(f, 1, n, n_new, st, self.cache.k, self.cache.v, self.cache.table, self.num_pages)

    def draft(self, anchor, P, B):
        out = torch.zeros((1, max(B - 1, 1)), dtype=torch.int32, device="cuda")
        self.d.draft(torch.tensor([anchor], dtype=torch.int32, device="cuda"),
                     torch.tensor([P], dtype=torch.int32, device="cuda"), 1, B, self.cache.k, self.cache.v,
                     self.cache.table, self.num_pages, P, out)
        self.d.check()
        return out.cpu()[0, :B - 1].tolist()


def gpu_verify_fn(z, d):
    logits = torch.as_tensor(np.asarray(z, dtype=np.float32))[None].cuda()
    draft = torch.as_tensor(np.asarray(d, dtype=np.int32)).reshape(1, -1).cuda()
    acc, nxt = gpu_verify(logits, draft)
    return int(acc.item()), int(nxt.item())


def run(dtype, seed, n_new, B, cheat_p=None, window=0):
    """dtype: "f32", "bf16" (bf16 KV cache) or "bf16-f16cache" (fp16 KV cache, tcgen05 attention)."""
    cache_dtype = torch.float16 if dtype == "bf16-f16cache" else None
    dtype = "bf16" if cache_dtype is not None else dtype
    tw, dw = tiny_pair(seed)
    dcfg = synth.TINY if dtype == "f32" else synth.TINY.replace(dtype="bf16")
    if dtype != "f32":
        dw = {k: (v if k == "layers" else v.to(torch.bfloat16) if v.dim() == 2 else v) for k, v in dw.items()}
        dw["layers"] = [{k: (v.to(torch.bfloat16) if v.dim() == 2 else v) for k, v in lw.items()}
                        for lw in dw["layers"]]
    prompt = synth.make_tokens(TARGET_CFG, 64, seed=50 + seed).tolist()
    tgt = T.TinyTarget(TARGET_CFG, tw, n_feat=3, max_len=64 + n_new + B + 1)
    ref = T.greedy_decode(tgt, prompt, n_new)
    drafter = GpuDrafter(dcfg, dw, 64 + n_new + B + 1, B, max_inject=64, cache_dtype=cache_dtype, window=window)
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
    tgt2 = T.TinyTarget(TARGET_CFG, tw, n_feat=3, max_len=64 + n_new + B + 1)
    out = T.spec_generate(tgt2, prompt, n_new, B, drafter.inject, draft_fn, gpu_verify_fn, stats)
    drafter.d.close()
    return out, ref, stats["accepted"]


@pytest.mark.parametrize("dtype", ["f32", "bf16", "bf16-f16cache"])
def test_gpu_spec_decode_is_lossless(dtype):
    out, ref, _ = run(dtype, 0, 96, 4)
    assert out == ref


@pytest.mark.parametrize("dtype", ["f32", "bf16", "bf16-f16cache"])
def test_gpu_spec_decode_lossless_at_every_acceptance_length(dtype):
    out, ref, acc = run(dtype, 2, 128, 4, cheat_p=0.75)
    assert out == ref
    assert set(acc) == {0, 1, 2, 3}


@pytest.mark.parametrize("dtype", ["f32", "bf16-f16cache"])
def test_gpu_spec_decode_with_a_sliding_window_drafter_is_lossless(dtype):
    """A drafter that sees only the last 48 context positions proposes differently,
    but the output is still the target's own greedy decode."""
    out, ref, acc = run(dtype, 3, 128, 4, cheat_p=0.5, window=48)
    assert out == ref
    assert len(set(acc)) > 1
