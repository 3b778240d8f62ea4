"""Sampled (temperature > 0) drafting and verify against the oracle.

* dflash_draft_block_sample: the stored drafter logits match the oracle's within
  the drafter's bars (1e-4 fp32, 2e-2 bf16, max-abs-rel); the drawn tokens equal
  the oracle's Gumbel-max draws over the same Philox uniforms wherever the top-2
  gap of the oracle's perturbed scores exceeds 1e-2 (the same rule as for greedy
  tokens: the decision is taken on scores that differ by rounding).
* dflash_verify_sampled: the accepted length equals oracle.sampling.sampled_verify
  on the same logits and uniforms wherever no acceptance test is within rounding
  of its threshold (|u q(d) - p(d)| > 1e-5 of the larger); the next token equals
  the oracle's where the draw's target u * total lies clear of every running-sum
  boundary by more than the fp32 summation error (2e-6 + 1.5e-7 sqrt(V) of the
  total), and otherwise is a valid inverse-CDF index within that tolerance; and
  over many requests with one drafted token the first emitted token follows the
  target's distribution (the lossless property of speculative sampling)."""
import numpy as np
import pytest
import torch

from block_diffusion_speculative_cycle_b200 import synth, verify_sampled
from oracle import dflash as O
from oracle import sampling as S
from tests.gpu_harness import PagedCache, make_drafter, max_abs_rel, top2_gap
from tests.test_gpu_draft import SMALL_BF16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg,ctx_lens,B,T,tol", [(synth.TINY, [64], 4, 1.0, 1e-4),
                                                  (SMALL_BF16, [200, 0, 77], 16, 0.7, 2e-2),
                                                  (SMALL_BF16, [130], 10, 1.5, 2e-2)])
def test_sampled_draft_matches_the_oracle(cfg, ctx_lens, B, T, tol):
    bs = len(ctx_lens)
    seed = 0x5EED_0000_1234 + B
    ctx = torch.tensor(ctx_lens, dtype=torch.int32)
    w = synth.make_drafter_weights(cfg, seed=3, share_embed_lm_head=True)
    table, num_pages = synth.make_page_table(ctx, 64, extra_tokens=B, seed=4)
    max_new = max(max(ctx_lens), 1)
    feats = synth.make_features(cfg, bs * max_new, seed=5).reshape(bs, max_new, cfg.feat_dim)
    anchors = synth.make_tokens(cfg, bs, seed=6)
    drafter, _ = make_drafter(cfg, w, max_block=B, max_batch=bs, max_inject_rows=bs * max_new, page_size=64)
    cache = PagedCache(cfg, table, num_pages, 64)
    n_new = torch.tensor(ctx_lens, dtype=torch.int32, device="cuda")
    start = torch.zeros(bs, dtype=torch.int32, device="cuda")
    drafter.inject(feats.cuda(), bs, max_new, n_new, start, cache.k, cache.v, cache.table, num_pages)
    draft = torch.zeros((bs, B - 1), dtype=torch.int32, device="cuda")
    ylog = torch.zeros((bs, B - 1, cfg.vocab), dtype=torch.float32, device="cuda")
    drafter.draft_sample(anchors.cuda(), ctx.cuda(), bs, B, cache.k, cache.v, cache.table, num_pages, max(ctx_lens),
                         T, seed, draft, ylog)
    drafter.check()
    draft, ylog = draft.cpu().numpy(), ylog.cpu().numpy()
    checked = 0
    for r in range(bs):
        P = ctx_lens[r]
        oc = O.Cache(cfg)
        if P:
            oc.write(0, O.inject(cfg, w, feats[r, :P], 0)[1])
        ref = O.draft_block(cfg, w, int(anchors[r]), oc, B)
        assert max_abs_rel(ylog[r], ref["logits"]) <= tol
        want = S.gumbel_draft(ref["logits"], T, seed, r)
        sure = top2_gap(S.gumbel_scores(ref["logits"], T, seed, r)) > 1e-2
        np.testing.assert_array_equal(draft[r][sure], want[sure])
        checked += int(sure.sum())
    assert checked >= 0.8 * bs * (B - 1)
    drafter.close()


def _oracle(z, y, d, ua, uf, T):
    """oracle (a, next), whether every acceptance test is clear of its threshold,
    and the running sums (index order) and target of the final draw."""
    p = S.softmax_t(z, T)
    q = S.softmax_t(y, T) if len(y) else np.zeros((0, z.shape[1]))
    a, nxt = S.sampled_verify(p, q, d, ua, uf)
    clear = True
    for i in range(1, min(a + 2, len(z))):
        lhs, rhs = ua[i - 1] * q[i - 1, d[i - 1]], p[i - 1, d[i - 1]]
        if abs(lhs - rhs) <= 1e-5 * max(lhs, rhs):
            clear = False
    w = np.maximum(p[a] - q[a], 0.0) if a < len(z) - 1 else p[a]
    if w.sum() <= 0:
        w = p[a]
    c = np.cumsum(w)
    return a, nxt, clear, c, uf * c[-1]


def draw_tol(V):
    """Fraction of the total within which fp32 running sums of V positive terms (each
    from a fast exponential) may place a boundary: about sqrt(V) roundings of 2^-24
    plus the exponentials' relative error. The draw is compared exactly when its
    target lies farther than this from every boundary, and otherwise checked to be
    a valid inverse-CDF index within it."""
    return 2e-6 + 1.5e-7 * np.sqrt(V)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("bs,B,V,T", [(6, 16, 151936, 1.0), (5, 10, 20000, 0.6), (4, 1, 9000, 1.3),
                                      (32, 4, 8192, 1.0)])
def test_sampled_verify_matches_the_oracle(dtype, bs, B, V, T):
    rng = np.random.default_rng(bs * 1000 + B)
    z = (rng.normal(size=(bs, B, V)) * 2.0).astype(np.float32)
    z = torch.from_numpy(z).to(dtype).float().numpy()          # the values the kernel reads
    # drafter logits near the target's (high acceptance), drafts drawn from q
    y = (z[:, :B - 1] + rng.normal(size=(bs, B - 1, V)) * 0.7).astype(np.float32)
    d = np.zeros((bs, max(B - 1, 0)), dtype=np.int32)
    for r in range(bs):
        for i in range(B - 1):
            d[r, i] = rng.choice(V, p=S.softmax_t(y[r, i], T))
    ua = rng.random((bs, max(B - 1, 1))).astype(np.float32)
    uf = rng.random(bs).astype(np.float32)
    acc, nxt = verify_sampled(torch.from_numpy(z).to(dtype).cuda(), torch.from_numpy(y).cuda() if B > 1 else None,
                              torch.from_numpy(d).cuda() if B > 1 else None, T, torch.from_numpy(ua).cuda(),
                              torch.from_numpy(uf).cuda())
    torch.cuda.synchronize()
    acc, nxt = acc.cpu().numpy(), nxt.cpu().numpy()
    n_clear = n_exact_draws = 0
    for r in range(bs):
        a, n, clear, c, target = _oracle(z[r].astype(np.float64), y[r].astype(np.float64), d[r],
                                         ua[r].astype(np.float64), float(uf[r]), T)
        assert 0 <= acc[r] <= B - 1 and 0 <= nxt[r] < V
        if not clear:
            continue
        n_clear += 1
        assert int(acc[r]) == a, f"request {r}: accepted {acc[r]} vs {a}"
        tol = draw_tol(V) * c[-1]
        if np.min(np.abs(c - target)) > tol:
            n_exact_draws += 1
            assert int(nxt[r]) == n, f"request {r}: next {nxt[r]} vs {n}"
        else:
            v = int(nxt[r])
            lo = c[v - 1] if v > 0 else 0.0
            assert lo - tol <= target <= c[v] + tol and c[v] > lo, f"request {r}: {v} is not a valid draw"
    assert n_clear >= bs - 1
    if V <= 20000:
        assert n_exact_draws >= 1
    if B > 2:
        assert len(set(acc.tolist())) > 1   # the cases exercise more than one acceptance length


def test_sampled_verify_first_token_follows_the_target():
    """Many requests share p_0, q_1 and draw d_1 ~ q_1 and fresh uniforms: the first
    emitted token (d_1 if accepted, else the residual draw) follows p_0."""
    n, V, T = 40000, 6, 1.0
    rng = np.random.default_rng(11)
    z0 = rng.normal(size=(2, V)) * 1.5
    y0 = rng.normal(size=(1, V)) * 1.5
    p0, q1 = S.softmax_t(z0, T)[0], S.softmax_t(y0, T)[0]
    z = np.broadcast_to(z0, (n, 2, V)).astype(np.float32).copy()
    y = np.broadcast_to(y0, (n, 1, V)).astype(np.float32).copy()
    d = rng.choice(V, size=(n, 1), p=q1).astype(np.int32)
    acc, nxt = verify_sampled(torch.from_numpy(z).cuda(), torch.from_numpy(y).cuda(), torch.from_numpy(d).cuda(), T,
                              torch.from_numpy(rng.random((n, 1)).astype(np.float32)).cuda(),
                              torch.from_numpy(rng.random(n).astype(np.float32)).cuda())
    acc, nxt = acc.cpu().numpy(), nxt.cpu().numpy()
    first = np.where(acc == 1, d[:, 0], nxt)
    freq = np.bincount(first, minlength=V) / n
    se = np.sqrt(p0 * (1 - p0) / n)
    assert np.all(np.abs(freq - p0) < 5 * se + 1e-4), (freq, p0)
    assert np.abs(q1 - p0).max() > 0.05   # the drafter's distribution differs (the check has teeth)
