"""Tiny causal target model, greedy decoding and the speculative loop (float64).

Test infrastructure (see oracle/__init__.py). This is what the lossless check
runs: speculative greedy decoding with any drafter must emit exactly the tokens
the target emits on its own ([P1] "DFlash — 블록 확산 드래프터로 6배 빨라지는
투기적 디코딩" §1: the verify result equals target-only decoding, "lossless").

The target is a pre-norm causal decoder built from the same pieces as the
drafter layer. It processes every row through one function, `step`, whether
the row comes from the prompt, from greedy decoding or from a verify block, so
a block forward gives bit-identical logits to token-by-token decoding.

Features for the drafter are the residual-stream outputs of a fixed, uniformly
spaced set of target layers, shallowest to deepest ([P2]; [P3] §2.2 context
feature extraction), concatenated in that order.
"""
from __future__ import annotations

from typing import Callable, Dict, List, Sequence, Tuple

import numpy as np

from .dflash import apply_rope, f64, greedy_argmax, linear, rms_norm, silu, softmax_rows


def tapped_layers(n_layers: int, n_feat: int) -> List[int]:
    """Uniformly spaced layer indices floor(i * (L-1) / (n_f-1)), i = 0..n_f-1."""
    if n_feat == 1:
        return [n_layers - 1]
    return [(i * (n_layers - 1)) // (n_feat - 1) for i in range(n_feat)]


class TinyTarget:
    """Causal decoder: E[token] -> L x (RMSNorm, GQA attention with RoPE, residual;
    RMSNorm, SwiGLU, residual) -> RMSNorm -> logits = y · Eᵀ (tied head)."""

    def __init__(self, cfg, weights: Dict, n_feat: int, max_len: int = 4096):
        self.cfg = cfg
        self.n_layers = len(weights["layers"])
        self.embed = f64(weights["embed"])
        self.lm_head = f64(weights["lm_head"])
        self.final_norm = f64(weights["final_norm"])
        self.layers = [{k: f64(v) for k, v in lw.items()} for lw in weights["layers"]]
        self.taps = tapped_layers(self.n_layers, n_feat)
        self.max_len = max_len

    def new_cache(self) -> Dict:
        c = self.cfg
        shape = (self.max_len, c.n_kv_heads, c.head_dim)
        return {"k": [np.zeros(shape) for _ in range(self.n_layers)],
                "v": [np.zeros(shape) for _ in range(self.n_layers)], "len": 0}

    def step(self, token: int, pos: int, cache: Dict) -> Tuple[np.ndarray, np.ndarray]:
        """Process one token at position pos (attending to positions 0..pos).
        Returns (logits [V], features [n_f * H])."""
        c = self.cfg
        assert pos == cache["len"], "rows must be processed in position order"
        x = self.embed[int(token)][None, :]
        feats = []
        for l, lw in enumerate(self.layers):
            h = rms_norm(x, lw["attn_norm"], c.rms_eps)
            q = apply_rope(linear(h, lw["wq"]).reshape(1, c.n_q_heads, c.head_dim), [pos], c.rope_theta)
            k = apply_rope(linear(h, lw["wk"]).reshape(1, c.n_kv_heads, c.head_dim), [pos], c.rope_theta)
            v = linear(h, lw["wv"]).reshape(1, c.n_kv_heads, c.head_dim)
            cache["k"][l][pos] = k[0]
            cache["v"][l][pos] = v[0]
            keys = cache["k"][l][:pos + 1]
            vals = cache["v"][l][:pos + 1]
            g = c.n_q_heads // c.n_kv_heads
            o = np.empty((c.n_q_heads, c.head_dim))
            for j in range(c.n_q_heads):
                p = softmax_rows(q[0, j][None, :] @ keys[:, j // g, :].T / np.sqrt(c.head_dim))
                o[j] = (p @ vals[:, j // g, :])[0]
            x = x + linear(o.reshape(1, -1), lw["wo"])
            h = rms_norm(x, lw["mlp_norm"], c.rms_eps)
            x = x + linear(silu(linear(h, lw["wgate"])) * linear(h, lw["wup"]), lw["wdown"])
            if l in self.taps:
                feats.append(x[0])
        cache["len"] = pos + 1
        y = rms_norm(x, self.final_norm, c.rms_eps)
        logits = linear(y, self.lm_head)[0]
        return logits, np.concatenate(feats)

    def forward(self, tokens: Sequence[int], start: int, cache: Dict) -> Tuple[np.ndarray, np.ndarray]:
        """Causal forward of tokens at positions start.. (row by row through step)."""
        out = [self.step(t, start + i, cache) for i, t in enumerate(tokens)]
        return np.stack([o[0] for o in out]), np.stack([o[1] for o in out])

    @staticmethod
    def truncate(cache: Dict, n: int) -> None:
        cache["len"] = n


def target_token(logits_row: np.ndarray) -> int:
    """The target's greedy choice, taken on fp32-rounded logits: the verify kernel
    sees fp32 logits, so both sides decide in that precision."""
    return greedy_argmax(np.asarray(logits_row, dtype=np.float32))


def greedy_decode(target: TinyTarget, prompt: Sequence[int], n_new: int) -> List[int]:
    """Plain autoregressive greedy decoding of n_new tokens by the target alone."""
    cache = target.new_cache()
    logits, _ = target.forward(prompt, 0, cache)
    out = [target_token(logits[-1])]
    while len(out) < n_new:
        lg, _ = target.step(out[-1], len(prompt) + len(out) - 1, cache)
        out.append(target_token(lg))
    return out


def spec_generate(target: TinyTarget, prompt: Sequence[int], n_new: int, B: int,
                  inject_fn: Callable, draft_fn: Callable, verify_fn: Callable,
                  stats: Dict = None) -> List[int]:
    """Speculative greedy decoding with a block drafter ([P1] §2 cycle; [P3] §2.2).

    Loop: the target prefill gives the features of positions 0..P-1 and the
    first token (the anchor). Each cycle: draft_fn(anchor, P, B) -> d_1..d_{B-1};
    the target runs the block [anchor, d_1..d_{B-1}] at positions P..P+B-1 in one
    causal pass; verify_fn(block logits as fp32, d) -> (a, next); commit
    d_1..d_a, next; the target cache keeps positions < P+a+1; the features of
    positions P..P+a are injected at start P; P += a+1; anchor = next.

    inject_fn(feats [n, n_f*H], start) and draft_fn / verify_fn are supplied by
    the caller (the oracle's own, or the CUDA path's)."""
    cache = target.new_cache()
    logits, feats = target.forward(prompt, 0, cache)
    P = len(prompt)
    anchor = target_token(logits[-1])
    out = [anchor]
    inject_fn(feats, 0)
    accepted = []
    while len(out) < n_new:
        d = [int(t) for t in draft_fn(anchor, P, B)]
        z, fb = target.forward([anchor] + d, P, cache)
        a, nxt = verify_fn(np.asarray(z, dtype=np.float32), d)
        accepted.append(a)
        out += d[:a] + [int(nxt)]
        target.truncate(cache, P + a + 1)
        inject_fn(fb[:a + 1], P)
        P += a + 1
        anchor = int(nxt)
    if stats is not None:
        stats["accepted"] = accepted
    return out[:n_new]


class OracleDrafter:
    """The oracle drafter wired for spec_generate (one request)."""

    def __init__(self, cfg, weights: Dict):
        from .dflash import Cache
        self.cfg = cfg
        self.weights = weights
        self.cache = Cache(cfg)

    def inject(self, feats, start: int) -> None:
        from .dflash import inject
        _, kv = inject(self.cfg, self.weights, feats, start)
        self.cache.write(start, kv)

    def draft(self, anchor: int, P: int, B: int):
        from .dflash import draft_block
        assert self.cache.length == P
        return draft_block(self.cfg, self.weights, anchor, self.cache, B)["draft"]
