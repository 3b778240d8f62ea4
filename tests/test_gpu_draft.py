"""dflash_inject_ctx + dflash_draft_block against the oracle on seeded inputs.

Bars: hidden states within max-abs-rel 1e-4 (fp32 drafter) / 2e-2 (bf16
drafter) per layer and for the final normed rows; draft tokens identical
wherever the oracle's top-2 logit gap exceeds 1e-2."""
import numpy as np
import pytest
import torch

from block_diffusion_speculative_cycle_b200 import synth
from oracle import dflash as O
from tests.gpu_harness import PagedCache, make_drafter, max_abs_rel, top2_gap

pytestmark = pytest.mark.gpu

SMALL_BF16 = synth.DrafterConfig(name="small-bf16", hidden=512, n_layers=2, n_q_heads=4, n_kv_heads=2,
                                 head_dim=128, intermediate=1024, vocab=2048, n_feat_layers=3,
                                 target_hidden=256, rope_theta=1e4, dtype="bf16")
TOL = {"f32": 1e-4, "bf16": 2e-2}


def run_case(cfg, ctx_lens, B, seed=0, chunks=1, max_new_pad=0, anchors=None, share=True, cache_dtype=None):
    bs = len(ctx_lens)
    ctx = torch.tensor(ctx_lens, dtype=torch.int32)
    w = synth.make_drafter_weights(cfg, seed=seed, share_embed_lm_head=share)
    page = 64
    table, num_pages = synth.make_page_table(ctx, page, extra_tokens=B, seed=seed + 1)
    max_new = max(max(ctx_lens), 1) + max_new_pad
    feats = synth.make_features(cfg, bs * max_new, seed=seed + 2).reshape(bs, max_new, cfg.feat_dim)
    if anchors is None:
        anchors = synth.make_tokens(cfg, bs, seed=seed + 3)
    drafter, _ = make_drafter(cfg, w, max_block=B, max_batch=bs, max_inject_rows=bs * max_new, page_size=page,
                              cache_dtype=cache_dtype)
    cache = PagedCache(cfg, table, num_pages, page, dtype=cache_dtype)

    # GPU: inject (optionally in several chunks), then one draft pass
    dev = "cuda"
    bounds = np.linspace(0, max(ctx_lens), chunks + 1).astype(int)
    for c0, c1 in zip(bounds[:-1], bounds[1:]):
        n_new = torch.tensor([max(0, min(P, c1) - c0) for P in ctx_lens], dtype=torch.int32, device=dev)
        start = torch.full((bs,), int(c0), dtype=torch.int32, device=dev)
        f = feats[:, c0:c1 + max_new_pad].contiguous().to(dev)
        drafter.inject(f, bs, f.shape[1], n_new, start, cache.k, cache.v, cache.table, num_pages)
    draft = torch.zeros((bs, B - 1), dtype=torch.int32, device=dev)
    hidden = torch.zeros((cfg.n_layers + 1, bs, B, cfg.hidden), dtype=torch.float32, device=dev)
    drafter.draft(anchors.to(dev), ctx.to(dev), bs, B, cache.k, cache.v, cache.table, num_pages, max(ctx_lens),
                  draft, hidden)
    drafter.check()
    torch.cuda.synchronize()
    draft, hidden = draft.cpu().numpy(), hidden.cpu().numpy()

    # oracle, request by request, from the same CPU inputs
    tol = TOL[cfg.dtype]
    for r in range(bs):
        P = ctx_lens[r]
        oc = O.Cache(cfg)
        if P:
            oc.write(0, O.inject(cfg, w, feats[r, :P], 0)[1])
        ref = O.draft_block(cfg, w, int(anchors[r]), oc, B)
        for l in range(cfg.n_layers + 1):
            err = max_abs_rel(hidden[l, r], ref["hidden"][l])
            assert err <= tol, f"request {r} layer {l}: max-abs-rel {err:.3g} > {tol}"
        if B > 1:
            gap = top2_gap(ref["logits"])
            sure = gap > 1e-2
            np.testing.assert_array_equal(draft[r][sure], ref["draft"][sure])
    return draft


@pytest.mark.parametrize("B", [1, 4])
def test_tiny_fp32(B):
    run_case(synth.TINY, [64], B)


def test_tiny_fp32_ragged_batch_chunked_inject():
    run_case(synth.TINY, [0, 5, 64, 131], 4, seed=3, chunks=3)


@pytest.mark.parametrize("ctx_lens,B", [([200], 16), ([0, 77, 300], 10), ([1], 2), ([64, 64], 1)])
def test_small_bf16(ctx_lens, B):
    run_case(SMALL_BF16, ctx_lens, B, seed=len(ctx_lens) + B)


@pytest.mark.parametrize("ctx_lens,B", [([200], 16), ([0, 77, 300], 10)])
def test_small_bf16_fp16_cache(ctx_lens, B):
    """bf16 drafter with an fp16 KV cache: injection writes fp16 pages and the
    attention kernel reads them without conversion."""
    run_case(SMALL_BF16, ctx_lens, B, seed=len(ctx_lens) + B + 7, cache_dtype=torch.float16)


def test_small_bf16_chunked_inject_and_padding_rows():
    run_case(SMALL_BF16, [130, 257], 16, seed=11, chunks=4, max_new_pad=3)


def test_small_bf16_untied_head_and_many_requests():
    lens = list(np.random.default_rng(0).integers(0, 400, size=12))
    run_case(SMALL_BF16, [int(x) for x in lens], 16, seed=5, share=False)


def test_small_bf16_fp16_cache_long_contexts():
    """Contexts of 1000-4000 keys over 16 requests: each attention CTA streams a
    dozen key tiles or more through its ring (wrap-around, lazy rescaling of the
    running maximum), on the fp16 cache the tcgen05 attention kernel reads."""
    lens = [int(x) for x in np.random.default_rng(7).integers(1000, 4001, size=16)]
    run_case(SMALL_BF16, lens, 16, seed=9, cache_dtype=torch.float16)


@pytest.mark.parametrize("plan", ["host", "device"])
def test_attention_split_plans_on_a_ragged_batch(plan, monkeypatch):
    """Both split plans of the tcgen05 attention on one ragged batch (an empty
    context, one key, a page boundary, a few thousand keys): the host's plan for
    the longest request (cluster merge), and the split size the device picks from
    the actual context lengths (global merge; CTAs past a request's keys exit)."""
    monkeypatch.setenv("DFLASH_ATTN_PLAN", plan)
    lens = [0, 1, 64, 3000, 777, 2048, 130, 1500]
    run_case(SMALL_BF16, lens, 16, seed=12, cache_dtype=torch.float16)


@pytest.mark.parametrize("cfg,cache_dtype,plan",
                         [(synth.TINY, None, "host"), (SMALL_BF16, None, "host"), (SMALL_BF16, torch.float16, "host"),
                          (SMALL_BF16, torch.float16, "device")],
                         ids=["fp32-simt", "bf16-mma", "fp16-tcgen05", "fp16-tcgen05-device-plan"])
@pytest.mark.parametrize("window", [128, 100])
def test_sliding_window_matches_the_oracle_with_released_pages(cfg, cache_dtype, plan, window, monkeypatch):
    """Sliding-window drafting: each request's block sees its last `window` context
    positions. After injection the page-table slots wholly below every window are
    set to -1 (pages released): the pass must not read them, flag nothing, and
    match the oracle's windowed pass."""
    monkeypatch.setenv("DFLASH_ATTN_PLAN", plan)
    ctx_lens, B, page = [300, 50, 700, 129], 16, 64
    bs = len(ctx_lens)
    ctx = torch.tensor(ctx_lens, dtype=torch.int32)
    w = synth.make_drafter_weights(cfg, seed=8, share_embed_lm_head=False)
    table, num_pages = synth.make_page_table(ctx, page, extra_tokens=B, seed=9)
    max_new = max(ctx_lens)
    feats = synth.make_features(cfg, bs * max_new, seed=10).reshape(bs, max_new, cfg.feat_dim)
    anchors = synth.make_tokens(cfg, bs, seed=11)
    drafter, _ = make_drafter(cfg, w, max_block=B, max_batch=bs, max_inject_rows=bs * max_new, page_size=page,
                              cache_dtype=cache_dtype, window=window)
    cache = PagedCache(cfg, table, num_pages, page, dtype=cache_dtype)
    n_new = torch.tensor(ctx_lens, dtype=torch.int32, device="cuda")
    start = torch.zeros(bs, dtype=torch.int32, device="cuda")
    drafter.inject(feats.cuda(), bs, max_new, n_new, start, cache.k, cache.v, cache.table, num_pages)
    drafter.check()
    released = table.clone()
    for r, P in enumerate(ctx_lens):
        lo = O.window_start(P, window)
        released[r, : lo // page] = -1
    assert int((released < 0).sum()) > int((table < 0).sum())   # some pages are gone
    draft = torch.zeros((bs, B - 1), dtype=torch.int32, device="cuda")
    hidden = torch.zeros((cfg.n_layers + 1, bs, B, cfg.hidden), dtype=torch.float32, device="cuda")
    drafter.draft(anchors.cuda(), ctx.cuda(), bs, B, cache.k, cache.v, released.cuda(), num_pages, max(ctx_lens),
                  draft, hidden)
    drafter.check()   # no page outside the windows was touched
    draft, hidden = draft.cpu().numpy(), hidden.cpu().numpy()
    tol = TOL[cfg.dtype]
    moved = 0.0
    for r, P in enumerate(ctx_lens):
        oc = O.Cache(cfg)
        oc.write(0, O.inject(cfg, w, feats[r, :P], 0)[1])
        ref = O.draft_block(cfg, w, int(anchors[r]), oc, B, window=window)
        for l in range(cfg.n_layers + 1):
            err = max_abs_rel(hidden[l, r], ref["hidden"][l])
            assert err <= tol, f"request {r} layer {l}: max-abs-rel {err:.3g}"
        sure = top2_gap(ref["logits"]) > 1e-2
        np.testing.assert_array_equal(draft[r][sure], ref["draft"][sure])
        if P > window:
            full = O.draft_block(cfg, w, int(anchors[r]), oc, B)
            moved = max(moved, max_abs_rel(full["hidden"][-1], ref["hidden"][-1]))
    assert moved > 2 * tol   # the window changes the pass well beyond the bar (the check has teeth)
    drafter.close()
