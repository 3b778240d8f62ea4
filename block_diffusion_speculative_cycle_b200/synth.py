"""Seeded synthetic inputs for the DFlash draft cycle.

This module only draws random numbers and lays them out; it holds none of the
cycle's arithmetic (no projection, norm, attention, argmax or verify step).
Both the CUDA path and the CPU oracle are fed from what it returns, so the two
sides always see identical inputs.

Workload shapes follow the drafter families named on the DFlash pages
("DFlash — 블록 확산 드래프터로 6배 빨라지는 투기적 디코딩", §2 block sizes and
§3.1 drafter sizes; "DFlash – 플래시 추측적 디코딩을 위한 블록 확산" §2.2 and §4):
Qwen3-8B-like and LLaMA-3.1-8B-like 5-layer drafters, a Qwen3-Coder-30B-A3B-like
8-layer drafter, and a tiny fp32 drafter for exhaustive checks.

Value distributions (stand-ins for trained checkpoints and datasets, which are
not available): linear and embedding weights N(0, 0.02) rounded to the model
dtype, RMSNorm gains 1, target features N(0, 1), token ids uniform over
[0, V-1) (id V-1 is the mask token), target block logits N(0, sigma) with a
planted agreement prefix whose length is geometric.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field
from typing import Dict, List, Optional

import torch


@dataclass(frozen=True)
class DrafterConfig:
    """Shape of one drafter plus the target features it consumes."""
    name: str
    hidden: int
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    intermediate: int
    vocab: int
    n_feat_layers: int
    target_hidden: int
    rope_theta: float
    rms_eps: float = 1e-6
    dtype: str = "bf16"          # "bf16" or "f32": storage type of weights / features
    target_layers: int = 0       # depth of the target the features come from

    @property
    def mask_token_id(self) -> int:
        return self.vocab - 1

    @property
    def feat_dim(self) -> int:
        return self.n_feat_layers * self.target_hidden

    @property
    def q_dim(self) -> int:
        return self.n_q_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def replace(self, **kw) -> "DrafterConfig":
        return dataclasses.replace(self, **kw)


@dataclass(frozen=True)
class Workload:
    """One draft-cycle workload: a drafter plus batch / context / block sizes."""
    name: str
    cfg: DrafterConfig
    block: int                   # B: anchor + B-1 masks
    batch: int = 1
    ctx_len: int = 64            # P when all requests share one length
    ctx_range: Optional[tuple] = None   # (lo, hi) inclusive: per-request P ~ U{lo..hi}
    page_size: int = 64
    logit_sigma: float = 1.0
    accept_mean: float = 6.5     # mean of the planted geometric agreement prefix
    seed: int = 0


TINY = DrafterConfig(name="tiny", hidden=256, n_layers=2, n_q_heads=4, n_kv_heads=2, head_dim=64,
                     intermediate=768, vocab=1024, n_feat_layers=3, target_hidden=256,
                     rope_theta=1e4, dtype="f32", target_layers=4)
QWEN3_8B = DrafterConfig(name="qwen3-8b-drafter", hidden=4096, n_layers=5, n_q_heads=32, n_kv_heads=8,
                         head_dim=128, intermediate=12288, vocab=151936, n_feat_layers=5,
                         target_hidden=4096, rope_theta=1e6, dtype="bf16", target_layers=36)
LLAMA31_8B = DrafterConfig(name="llama3.1-8b-drafter", hidden=4096, n_layers=5, n_q_heads=32, n_kv_heads=8,
                           head_dim=128, intermediate=14336, vocab=128256, n_feat_layers=5,
                           target_hidden=4096, rope_theta=5e5, dtype="bf16", target_layers=32)
CODER_30B = DrafterConfig(name="qwen3-coder-30b-a3b-drafter", hidden=2048, n_layers=8, n_q_heads=32,
                          n_kv_heads=4, head_dim=128, intermediate=6144, vocab=151936, n_feat_layers=6,
                          target_hidden=2048, rope_theta=1e6, dtype="bf16", target_layers=48)

WORKLOADS: Dict[str, Workload] = {
    "tiny_b4": Workload("tiny_b4", TINY, block=4, batch=1, ctx_len=64, logit_sigma=1.0, accept_mean=1.5),
    "qwen8b_b16": Workload("qwen8b_b16", QWEN3_8B, block=16, batch=1, ctx_len=2048, logit_sigma=2.0,
                           accept_mean=6.5),
    "llama8b_b10": Workload("llama8b_b10", LLAMA31_8B, block=10, batch=1, ctx_len=4096, logit_sigma=2.0,
                            accept_mean=3.25),
    "coder30b_b16_bs1": Workload("coder30b_b16_bs1", CODER_30B, block=16, batch=1, ctx_len=32768,
                                 logit_sigma=2.0, accept_mean=6.5),
    "coder30b_b16_bs8": Workload("coder30b_b16_bs8", CODER_30B, block=16, batch=8, ctx_len=32768,
                                 logit_sigma=2.0, accept_mean=6.5),
    "coder30b_b8_bs1": Workload("coder30b_b8_bs1", CODER_30B, block=8, batch=1, ctx_len=32768,
                                logit_sigma=2.0, accept_mean=6.5),
}
# Kernel-profiling case: one Qwen3-8B-shaped layer and a 16384-row LM head, so that
# every GEMM call site keeps its real shape (the gate/up weights alone exceed L2)
# while the device footprint stays under 1 GB.
WORKLOADS["qwen8b_b16_l1_v16k"] = Workload("qwen8b_b16_l1_v16k", QWEN3_8B.replace(n_layers=1, vocab=16384), block=16,
                                           batch=1, ctx_len=2048, logit_sigma=2.0, accept_mean=6.5)
for _bs in (1, 4, 8, 16, 32):
    WORKLOADS[f"qwen8b_b16_serve_bs{_bs}"] = Workload(
        f"qwen8b_b16_serve_bs{_bs}", QWEN3_8B, block=16, batch=_bs, ctx_range=(512, 8192),
        page_size=64, logit_sigma=2.0, accept_mean=6.0)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _normal(g, shape, std, dtype):
    return (torch.randn(shape, generator=g, dtype=torch.float32) * std).to(dtype)


def make_drafter_weights(cfg: DrafterConfig, seed: int = 0, std: float = 0.02,
                         share_embed_lm_head: bool = False,
                         embed: Optional[torch.Tensor] = None) -> Dict[str, object]:
    """Random drafter weights (CPU tensors in the model dtype; norm gains fp32 ones).

    Layout: every linear weight is [out_features, in_features] row-major.
    `embed` lets a caller pass the (target-owned) embedding to share."""
    g = _gen(seed)
    dt = cfg.torch_dtype
    H = cfg.hidden
    w: Dict[str, object] = {}
    w["fc"] = _normal(g, (H, cfg.feat_dim), std, dt)
    w["embed"] = embed if embed is not None else _normal(g, (cfg.vocab, H), std, dt)
    w["lm_head"] = w["embed"] if share_embed_lm_head else _normal(g, (cfg.vocab, H), std, dt)
    w["final_norm"] = torch.ones(H, dtype=torch.float32)
    layers = []
    for _ in range(cfg.n_layers):
        layers.append({
            "attn_norm": torch.ones(H, dtype=torch.float32),
            "wq": _normal(g, (cfg.q_dim, H), std, dt),
            "wk": _normal(g, (cfg.kv_dim, H), std, dt),
            "wv": _normal(g, (cfg.kv_dim, H), std, dt),
            "wo": _normal(g, (H, cfg.q_dim), std, dt),
            "mlp_norm": torch.ones(H, dtype=torch.float32),
            "wgate": _normal(g, (cfg.intermediate, H), std, dt),
            "wup": _normal(g, (cfg.intermediate, H), std, dt),
            "wdown": _normal(g, (H, cfg.intermediate), std, dt),
        })
    w["layers"] = layers
    return w


def make_features(cfg: DrafterConfig, n_rows: int, seed: int = 1) -> torch.Tensor:
    """Target hidden features, already concatenated over the n_f tapped layers:
    [n_rows, n_f * H_t], N(0, 1) in the model dtype."""
    g = _gen(seed)
    return torch.randn((n_rows, cfg.feat_dim), generator=g, dtype=torch.float32).to(cfg.torch_dtype)


def make_tokens(cfg: DrafterConfig, n: int, seed: int = 2) -> torch.Tensor:
    """Token ids uniform over [0, V-1) (the mask id V-1 is never drawn)."""
    g = _gen(seed)
    return torch.randint(0, cfg.vocab - 1, (n,), generator=g, dtype=torch.int32)


def make_ctx_lens(w: Workload, seed: int = 3) -> torch.Tensor:
    """Per-request context lengths P_r: fixed, or uniform over w.ctx_range."""
    if w.ctx_range is None:
        return torch.full((w.batch,), w.ctx_len, dtype=torch.int32)
    g = _gen(seed)
    lo, hi = w.ctx_range
    return torch.randint(lo, hi + 1, (w.batch,), generator=g, dtype=torch.int32)


def make_page_table(ctx_lens: torch.Tensor, page_size: int, extra_tokens: int, seed: int = 4,
                    shuffle: bool = True):
    """A ragged paged layout: request r owns ceil((P_r+extra)/page) pages drawn
    without replacement from one pool (shuffled so pages are not contiguous).

    Returns (page_table [bs, max_pages] int32, num_pages). Unused slots hold -1."""
    need = [(int(p) + extra_tokens + page_size - 1) // page_size for p in ctx_lens.tolist()]
    total = sum(need)
    max_pages = max(need) if need else 0
    g = _gen(seed)
    perm = torch.randperm(total, generator=g) if shuffle else torch.arange(total)
    table = torch.full((len(need), max(max_pages, 1)), -1, dtype=torch.int32)
    o = 0
    for r, n in enumerate(need):
        table[r, :n] = perm[o:o + n].to(torch.int32)
        o += n
    return table, total


def make_kv_cache(cfg: DrafterConfig, num_pages: int, page_size: int, seed: int = 5,
                  std: float = 1.0) -> List[Dict[str, torch.Tensor]]:
    """Random K/V page pools per layer, layout [num_pages, n_kv, page_size, head_dim]
    in the model dtype (used where a test wants a cache without running injection)."""
    g = _gen(seed)
    out = []
    for _ in range(cfg.n_layers):
        k = _normal(g, (num_pages, cfg.n_kv_heads, page_size, cfg.head_dim), std, cfg.torch_dtype)
        v = _normal(g, (num_pages, cfg.n_kv_heads, page_size, cfg.head_dim), std, cfg.torch_dtype)
        out.append({"k": k, "v": v})
    return out


def planted_logits(draft: torch.Tensor, vocab: int, sigma: float, accept_mean: float,
                   seed: int = 6, dtype: torch.dtype = torch.bfloat16,
                   accepted: Optional[torch.Tensor] = None):
    """Target block logits [bs, B, V] with a planted agreement prefix.

    draft: [bs, B-1] draft tokens. For each request a planted length a is drawn
    Geometric on {0, 1, ...} with mean accept_mean (clipped at B-1), unless given.
    Rows j < a get logit(draft[j]) = row max + 1 (so the target's top token is the
    draft's), row a (if a < B-1) gets logit(draft[a]) = row min - 1 (a certain
    mismatch). Values are set after rounding to `dtype`, so the planted entries are
    exactly representable. Returns (logits, planted_a)."""
    bs, Bm1 = draft.shape
    B = Bm1 + 1
    g = _gen(seed)
    z = (torch.randn((bs, B, vocab), generator=g, dtype=torch.float32) * sigma).to(dtype).float()
    if accepted is None:
        p = 1.0 / (1.0 + accept_mean)
        u = torch.rand((bs,), generator=g, dtype=torch.float64)
        # inverse CDF of the geometric law on {0,1,...}: floor(log(1-u)/log(1-p))
        a = torch.floor(torch.log1p(-u) / torch.log1p(torch.tensor(-p, dtype=torch.float64))).to(torch.int64)
        a = torch.clamp(a, 0, Bm1)
    else:
        a = accepted.to(torch.int64).clone()
    for r in range(bs):
        ar = int(a[r])
        for j in range(ar):
            row = z[r, j]
            row[int(draft[r, j])] = float(row.max()) + 1.0
        if ar < Bm1:
            row = z[r, ar]
            row[int(draft[r, ar])] = float(row.min()) - 1.0
    return z.to(dtype), a.to(torch.int32)
