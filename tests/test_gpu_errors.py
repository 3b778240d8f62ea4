"""Device-detected input errors are flagged, not faulted.

Out-of-range token ids, page ids, cache positions and context lengths reach
the kernels only through device memory, so the host cannot check them. Each
kernel tests every such index before it touches memory, skips (or clamps) the
element and sets a bit in the context's status word; dflash_get_error reads
and clears it (DFLASH_ERR_DEVICE). These tests plant one bad value at a time
and check that the call completes, the status is reported once, and a clean
call afterwards reports nothing. Host-detectable argument errors are refused
before any launch (DFLASH_ERR_ARG)."""
import pytest
import torch

from block_diffusion_speculative_cycle_b200 import DFlashError, synth
from tests.gpu_harness import PagedCache, make_drafter

pytestmark = pytest.mark.gpu

ERR_ARG, ERR_TIMEOUT, ERR_DEVICE = 1, 4, 5

SMALL_BF16 = synth.DrafterConfig(name="small-bf16", hidden=512, n_layers=2, n_q_heads=4, n_kv_heads=2,
                                 head_dim=128, intermediate=1024, vocab=2048, n_feat_layers=3,
                                 target_hidden=256, rope_theta=1e4, dtype="bf16")


def setup(cfg, ctx_len=128, B=4):
    w = synth.make_drafter_weights(cfg, seed=0)
    ctx = torch.tensor([ctx_len], dtype=torch.int32)
    table, num_pages = synth.make_page_table(ctx, 64, extra_tokens=B, seed=1)
    drafter, _ = make_drafter(cfg, w, max_block=B, max_batch=1, max_inject_rows=ctx_len, page_size=64)
    cache = PagedCache(cfg, table, num_pages, 64)
    feats = synth.make_features(cfg, ctx_len, seed=2).reshape(1, ctx_len, cfg.feat_dim).cuda()
    n_new = torch.tensor([ctx_len], dtype=torch.int32, device="cuda")
    start = torch.zeros(1, dtype=torch.int32, device="cuda")
    drafter.inject(feats, 1, ctx_len, n_new, start, cache.k, cache.v, cache.table, num_pages)
    drafter.check()
    return drafter, cache, num_pages, ctx


def draft(drafter, cache, num_pages, anchor, ctx, B, table=None, max_ctx=None):
    out = torch.zeros((1, B - 1), dtype=torch.int32, device="cuda")
    drafter.draft(anchor.cuda(), ctx.cuda(), 1, B, cache.k, cache.v, cache.table if table is None else table,
                  num_pages, int(ctx.max()) if max_ctx is None else max_ctx, out)
    torch.cuda.synchronize()
    return out


def expect_device_error(drafter):
    with pytest.raises(DFlashError) as e:
        drafter.check()
    assert e.value.status == ERR_DEVICE
    drafter.check()   # reading the status cleared it


@pytest.mark.parametrize("cfg", [synth.TINY, SMALL_BF16], ids=["fp32", "bf16"])
def test_bad_anchor_token_is_flagged(cfg):
    drafter, cache, num_pages, ctx = setup(cfg)
    draft(drafter, cache, num_pages, torch.tensor([cfg.vocab + 7], dtype=torch.int32), ctx, 4)
    expect_device_error(drafter)
    draft(drafter, cache, num_pages, torch.tensor([3], dtype=torch.int32), ctx, 4)
    drafter.check()
    drafter.close()


@pytest.mark.parametrize("cfg", [synth.TINY, SMALL_BF16], ids=["fp32", "bf16"])
def test_bad_page_id_is_flagged(cfg):
    drafter, cache, num_pages, ctx = setup(cfg)
    bad = cache.table.clone()
    bad[0, 1] = num_pages + 3          # the second context page points outside the pool
    draft(drafter, cache, num_pages, torch.tensor([3], dtype=torch.int32), ctx, 4, table=bad)
    expect_device_error(drafter)
    drafter.close()


@pytest.mark.parametrize("cfg", [synth.TINY, SMALL_BF16], ids=["fp32", "bf16"])
def test_context_length_beyond_max_ctx_is_flagged(cfg):
    drafter, cache, num_pages, ctx = setup(cfg)
    draft(drafter, cache, num_pages, torch.tensor([3], dtype=torch.int32), torch.tensor([ctx.item() + 50],
          dtype=torch.int32), 4, max_ctx=int(ctx.item()))
    expect_device_error(drafter)
    drafter.close()


def test_injection_past_the_page_table_is_flagged():
    cfg = SMALL_BF16
    drafter, cache, num_pages, ctx = setup(cfg)
    feats = synth.make_features(cfg, 8, seed=5).reshape(1, 8, cfg.feat_dim).cuda()
    n_new = torch.tensor([8], dtype=torch.int32, device="cuda")
    start = torch.tensor([cache.table.shape[1] * 64 - 4], dtype=torch.int32, device="cuda")   # 4 rows run off
    drafter.inject(feats, 1, 8, n_new, start, cache.k, cache.v, cache.table, num_pages)
    torch.cuda.synchronize()
    expect_device_error(drafter)
    drafter.close()


def test_host_argument_errors_launch_nothing():
    cfg = SMALL_BF16
    drafter, cache, num_pages, ctx = setup(cfg)
    with pytest.raises(DFlashError) as e:
        draft(drafter, cache, num_pages, torch.tensor([3], dtype=torch.int32), ctx, 9)   # B > max_block
    assert e.value.status == ERR_ARG
    drafter.check()
    drafter.close()


def test_a_device_wait_that_runs_out_reports_timeout_and_a_fresh_context_works(monkeypatch):
    """Failure injection without a fault: with DFLASH_TEST_STALL_NS set when the
    context is created, every tensor-core GEMM epilogue also waits on a barrier
    that nothing arrives at, bounded by 1 ms. Injection and the draft pass must
    come back, each report DFLASH_ERR_TIMEOUT once, and a context created
    afterwards without the hook must match the oracle again."""
    from tests.test_gpu_draft import run_case
    cfg, ctx_len, B = SMALL_BF16, 128, 4
    monkeypatch.setenv("DFLASH_TEST_STALL_NS", "1000000")
    w = synth.make_drafter_weights(cfg, seed=0)
    ctx = torch.tensor([ctx_len], dtype=torch.int32)
    table, num_pages = synth.make_page_table(ctx, 64, extra_tokens=B, seed=1)
    drafter, _ = make_drafter(cfg, w, max_block=B, max_batch=1, max_inject_rows=ctx_len, page_size=64)
    monkeypatch.delenv("DFLASH_TEST_STALL_NS")
    cache = PagedCache(cfg, table, num_pages, 64)
    feats = synth.make_features(cfg, ctx_len, seed=2).reshape(1, ctx_len, cfg.feat_dim).cuda()
    n_new = torch.tensor([ctx_len], dtype=torch.int32, device="cuda")
    start = torch.zeros(1, dtype=torch.int32, device="cuda")
    for step in ("inject", "draft"):
        if step == "inject":
            drafter.inject(feats, 1, ctx_len, n_new, start, cache.k, cache.v, cache.table, num_pages)
        else:
            draft(drafter, cache, num_pages, torch.tensor([3], dtype=torch.int32), ctx, B)
        with pytest.raises(DFlashError) as e:
            drafter.check()
        assert e.value.status == ERR_TIMEOUT, step
        drafter.check()   # reported once
    drafter.close()
    run_case(cfg, [200], 16, seed=21)
