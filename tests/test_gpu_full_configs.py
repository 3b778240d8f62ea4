"""Parity at the benchmark workloads' full sizes, in the launch configuration the
benchmark uses (bf16, paged cache, one draft pass over the whole batch).

The drafter cache holds seeded random K/V (std 3, about the scale injection
produces with N(0, 0.02) weights and N(0, 1) features), held once as bf16 and
once as fp16 (the same values: both attention kernels are checked); the oracle
reads the same CPU tensors. Each test checks a sample of requests against the oracle:
every layer's residual stream and the final normed rows within max-abs-rel
2e-2, and the draft tokens wherever the oracle's top-2 logit gap exceeds 1e-2.
Injection is checked separately: 16 rows injected past the context, read back
from the cache pages and compared with the oracle's K (with RoPE) and V."""
import numpy as np
import pytest
import torch

from block_diffusion_speculative_cycle_b200 import synth
from oracle import dflash as O
from tests.gpu_harness import PagedCache, gather_cpu_cache, make_drafter, max_abs_rel, top2_gap

pytestmark = pytest.mark.gpu

TOL = 2e-2
_WEIGHTS = {}


def weights_for(cfg):
    """(CPU weights in the model dtype, the same values widened once to float64
    for the oracle, which then reads them without converting per request)."""
    if cfg.name not in _WEIGHTS:
        _WEIGHTS.clear()
        w = synth.make_drafter_weights(cfg, seed=0)
        w64 = {k: (O.f64(v) if torch.is_tensor(v) else v) for k, v in w.items() if k != "layers"}
        w64["layers"] = [{k: O.f64(v) for k, v in lw.items()} for lw in w["layers"]]
        _WEIGHTS[cfg.name] = (w, w64)
    return _WEIGHTS[cfg.name]


def _both_types(t: torch.Tensor) -> torch.Tensor:
    """Cache values exactly representable in bf16 and in fp16: bf16 values whose
    magnitude is below fp16's normal range are set to zero (bf16's 8-bit
    significand fits in fp16's 11 bits everywhere else), so one oracle pass
    serves a bf16 and an fp16 cache."""
    t = t.to(torch.bfloat16)
    return torch.where(t.float().abs() < 2.0 ** -14, torch.zeros_like(t), t)


def run_workload(name, sample, B=None, inject_rows=16, cache_dtypes=(None, torch.float16)):
    """sample: requests checked layer by layer and for injection; every request
    is checked for its final normed rows and draft tokens. The GPU runs once per
    KV-cache element type in cache_dtypes (None: the model's bf16, read by the
    mma.sync attention kernel; fp16: read by the tcgen05 attention kernel); the
    cache holds the same values in both, so the oracle runs once."""
    w = synth.WORKLOADS[name]
    cfg = w.cfg
    B = B or w.block
    bs = w.batch
    weights, w64 = weights_for(cfg)
    ctx = synth.make_ctx_lens(w)
    table, num_pages = synth.make_page_table(ctx, w.page_size, extra_tokens=max(B, inject_rows), seed=11)
    pools = synth.make_kv_cache(cfg, num_pages, w.page_size, seed=12, std=3.0)
    pools = [{k: _both_types(t) for k, t in lay.items()} for lay in pools]
    anchors = synth.make_tokens(cfg, bs, seed=13)
    feats = synth.make_features(cfg, bs * inject_rows, seed=14).reshape(bs, inject_rows, cfg.feat_dim)
    n_new = torch.full((bs,), inject_rows, dtype=torch.int32)
    dev = "cuda"
    runs = []
    for cache_dtype in cache_dtypes:
        drafter, _ = make_drafter(cfg, weights, max_block=B, max_batch=bs, max_inject_rows=bs * inject_rows,
                                  page_size=w.page_size, cache_dtype=cache_dtype)
        cache = PagedCache(cfg, table, num_pages, w.page_size, init=pools, dtype=cache_dtype)
        draft = torch.zeros((bs, B - 1), dtype=torch.int32, device=dev)
        hidden = torch.zeros((cfg.n_layers + 1, bs, B, cfg.hidden), dtype=torch.float32, device=dev)
        drafter.draft(anchors.to(dev), ctx.to(dev), bs, B, cache.k, cache.v, cache.table, num_pages,
                      int(ctx.max()), draft, hidden)
        # injection of inject_rows rows per request at positions P .. P+inject_rows-1
        drafter.inject(feats.to(dev), bs, inject_rows, n_new.to(dev), ctx.to(dev), cache.k, cache.v, cache.table,
                       num_pages)
        drafter.check()
        torch.cuda.synchronize()
        runs.append((str(cache_dtype or "model"), draft.cpu().numpy(), hidden.cpu().numpy(), cache))
        drafter.close()

    for r in range(bs):
        P = int(ctx[r])
        oc = gather_cpu_cache(cfg, pools, table, r, P, w.page_size)
        ref = O.draft_block(cfg, w64, int(anchors[r]), oc, B)
        sure = top2_gap(ref["logits"]) > 1e-2 if B > 1 else None
        kv = O.inject(cfg, w64, feats[r], P)[1] if r in sample else None
        for tag, draft, hidden, cache in runs:
            layers = range(cfg.n_layers + 1) if r in sample else [cfg.n_layers]
            for l in layers:
                err = max_abs_rel(hidden[l, r], ref["hidden"][l])
                assert err <= TOL, f"{name} ({tag} cache) request {r} layer {l}: max-abs-rel {err:.3g}"
            if B > 1:
                np.testing.assert_array_equal(draft[r][sure], ref["draft"][sure],
                                              err_msg=f"{name} ({tag} cache) request {r}")
                assert sure.mean() > 0.5
            if kv is None:
                continue
            # injected rows, read back from the pages
            pos = np.arange(P, P + inject_rows)
            pages = table[r].numpy()[pos // w.page_size]
            slots = pos % w.page_size
            for l in (0, cfg.n_layers - 1):
                kg = cache.k[l][torch.as_tensor(pages)].float().cpu().numpy()[np.arange(inject_rows), :, slots, :]
                vg = cache.v[l][torch.as_tensor(pages)].float().cpu().numpy()[np.arange(inject_rows), :, slots, :]
                assert max_abs_rel(kg, kv[l][0]) <= TOL, f"{name} ({tag} cache) request {r} layer {l}: injected K"
                assert max_abs_rel(vg, kv[l][1]) <= TOL, f"{name} ({tag} cache) request {r} layer {l}: injected V"


def test_qwen3_8b_shaped_bs1_ctx2048_block16():
    run_workload("qwen8b_b16", sample=[0])


def test_llama31_8b_shaped_bs1_ctx4096_block10():
    run_workload("llama8b_b10", sample=[0])


def test_qwen3_8b_shaped_serving_bs32_ragged_paged():
    run_workload("qwen8b_b16_serve_bs32", sample=[0, 17, 31])


def test_qwen3_8b_shaped_serving_bs1():
    run_workload("qwen8b_b16_serve_bs1", sample=[0])


def test_qwen3_8b_shaped_serving_bs4():
    run_workload("qwen8b_b16_serve_bs4", sample=[1, 3])


def test_qwen3_8b_shaped_serving_bs8():
    run_workload("qwen8b_b16_serve_bs8", sample=[0, 6])


def test_qwen3_8b_shaped_serving_bs16():
    run_workload("qwen8b_b16_serve_bs16", sample=[2, 15])


def test_coder30b_shaped_bs1_ctx32768_block16():
    run_workload("coder30b_b16_bs1", sample=[0])


def test_coder30b_shaped_bs1_ctx32768_block8():
    run_workload("coder30b_b8_bs1", sample=[0])


def test_coder30b_shaped_bs8_ctx32768_block16():
    run_workload("coder30b_b16_bs8", sample=[5])
