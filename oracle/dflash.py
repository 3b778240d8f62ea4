"""DFlash draft cycle, float64 reference (test infrastructure; see oracle/__init__.py).

Sources (page title, section):
  [P1] "DFlash — 블록 확산 드래프터로 6배 빨라지는 투기적 디코딩", §1 (verify rule),
       §2 (anchor + B-1 masks, one forward pass, KV injection), §6 (non-causal
       in-block attention), §7 (1-step masked prediction)
  [P2] "한 번에 초안을 생성하는 DFlash ..." (uniformly spaced target layers fused
       by a lightweight projection, injected into every drafter layer's K/V)
  [P3] "기술 요약: DFlash – 플래시 추측적 디코딩을 위한 블록 확산", §2.2 (context
       feature extraction, KV injection into the drafter KV cache, parallel block
       prediction), §2.3 (embedding and LM head shared with the target, frozen)

Readings where the pages are silent (each the plainest one the rest of the pages support):
  * the projection is one bias-free linear map, no norm after it;
  * each layer injects with its own Wk/Wv, without that layer's input RMSNorm;
    K gets RoPE at the context token's absolute position;
  * the cache holds only injected context; block K/V are transient;
  * context occupies positions 0..P-1, the anchor P, the masks P+1..P+B-1;
  * output at block position i (i >= 1) is the draft for that position;
  * drafter layer = pre-norm RMSNorm (gain, eps) -> GQA attention with
    rotate-half RoPE -> residual; RMSNorm -> SwiGLU MLP -> residual;
    q head j reads kv head floor(j / (n_q / n_kv)); softmax scale 1/sqrt(d);
  * argmax: lowest index among equal maxima, NaN ranks below every number;
  * a sliding window of W positions keeps the last W context positions
    (P-W .. P-1) visible to the block, with their original (absolute) RoPE.

Everything is computed in float64 from the inputs as given (bf16 inputs are
widened exactly); nothing is rounded in between.
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np


def f64(a) -> np.ndarray:
    """Widen a NumPy array or a CPU torch tensor (any float dtype) to float64."""
    if hasattr(a, "detach"):  # torch tensor: bf16 has no NumPy dtype, widen via float32
        import torch
        t = a.detach().cpu()
        if t.dtype == torch.bfloat16:
            t = t.to(torch.float32)
        a = t.numpy()
    return np.asarray(a, dtype=np.float64)


def linear(x: np.ndarray, w) -> np.ndarray:
    """y = x · Wᵀ with W stored [out, in]."""
    return x @ f64(w).T


def rms_norm(x: np.ndarray, gain, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * gain."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * f64(gain)


def silu(x: np.ndarray) -> np.ndarray:
    """silu(x) = x * sigmoid(x) = x / (1 + e^-x)."""
    return x / (1.0 + np.exp(-x))


def rope_inv_freq(head_dim: int, theta: float) -> np.ndarray:
    """Rotary frequencies theta^(-2i/d), i = 0 .. d/2-1."""
    i = np.arange(head_dim // 2, dtype=np.float64)
    return theta ** (-2.0 * i / head_dim)


def apply_rope(x: np.ndarray, pos: Sequence[int], theta: float) -> np.ndarray:
    """Rotate-half rotary embedding. x [n, heads, d]; pos [n] absolute positions.

    Pair (i, i + d/2) is rotated by angle pos * theta^(-2i/d)."""
    d = x.shape[-1]
    half = d // 2
    ang = np.outer(np.asarray(pos, dtype=np.float64), rope_inv_freq(d, theta))[:, None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def softmax_rows(s: np.ndarray) -> np.ndarray:
    s = s - np.max(s, axis=-1, keepdims=True)
    p = np.exp(s)
    return p / np.sum(p, axis=-1, keepdims=True)


def block_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """Non-causal grouped-query attention of the block queries over all keys.

    q [Bq, n_q, d]; k, v [T, n_kv, d] (context keys followed by block keys).
    Every query sees every key: no mask ([P1] §6: in-block attention is
    non-causal). Returns o [Bq, n_q, d]."""
    n_q, d = q.shape[1], q.shape[2]
    n_kv = k.shape[1]
    g = n_q // n_kv
    o = np.empty_like(q)
    for j in range(n_q):
        h = j // g
        p = softmax_rows(q[:, j, :] @ k[:, h, :].T / np.sqrt(d))
        o[:, j, :] = p @ v[:, h, :]
    return o


# --------------------------------------------------------------------------- inject

def fuse_features(feats, w_fc) -> np.ndarray:
    """Context feature c = F · W_fcᵀ: the concatenated target-layer features
    projected to the drafter width ([P2]; [P3] §2.2 context feature extraction)."""
    return linear(f64(feats), w_fc)


def inject(cfg, weights: Dict, feats, start: int) -> Tuple[np.ndarray, List[Tuple[np.ndarray, np.ndarray]]]:
    """KV injection ([P3] §2.2; [P1] §2 "Target과의 결합 — KV Injection").

    feats [n, n_f*H_t] are the fused-layer features of context positions
    start .. start+n-1. Returns (c [n, H], per layer (K [n, n_kv, d], V [n, n_kv, d])):
    K_l = RoPE(c · Wk_lᵀ) at the absolute positions, V_l = c · Wv_lᵀ."""
    c = fuse_features(feats, weights["fc"])
    n = c.shape[0]
    pos = np.arange(start, start + n)
    kv = []
    for lw in weights["layers"]:
        k = linear(c, lw["wk"]).reshape(n, cfg.n_kv_heads, cfg.head_dim)
        v = linear(c, lw["wv"]).reshape(n, cfg.n_kv_heads, cfg.head_dim)
        kv.append((apply_rope(k, pos, cfg.rope_theta), v))
    return c, kv


class Cache:
    """Drafter KV cache of one request: per layer, injected K/V of positions 0..P-1."""

    def __init__(self, cfg):
        self.cfg = cfg
        self.k = [np.zeros((0, cfg.n_kv_heads, cfg.head_dim)) for _ in range(cfg.n_layers)]
        self.v = [np.zeros((0, cfg.n_kv_heads, cfg.head_dim)) for _ in range(cfg.n_layers)]
        self.length = 0

    def write(self, start: int, kv) -> None:
        """Store injected rows at positions start.. (truncating anything after)."""
        for l, (k, v) in enumerate(kv):
            self.k[l] = np.concatenate([self.k[l][:start], k], axis=0)
            self.v[l] = np.concatenate([self.v[l][:start], v], axis=0)
        self.length = start + (len(kv[0][0]) if kv else 0)

    @staticmethod
    def from_arrays(cfg, ks, vs) -> "Cache":
        c = Cache(cfg)
        c.k = [f64(k) for k in ks]
        c.v = [f64(v) for v in vs]
        c.length = c.k[0].shape[0] if c.k else 0
        return c


# --------------------------------------------------------------------------- draft

def drafter_layer(cfg, lw: Dict, x: np.ndarray, pos: np.ndarray, k_ctx: np.ndarray,
                  v_ctx: np.ndarray) -> np.ndarray:
    """One drafter layer over the block rows x [B, H] at positions pos.

    The block's own K/V join the injected context K/V for this pass only."""
    B = x.shape[0]
    h = rms_norm(x, lw["attn_norm"], cfg.rms_eps)
    q = apply_rope(linear(h, lw["wq"]).reshape(B, cfg.n_q_heads, cfg.head_dim), pos, cfg.rope_theta)
    k = apply_rope(linear(h, lw["wk"]).reshape(B, cfg.n_kv_heads, cfg.head_dim), pos, cfg.rope_theta)
    v = linear(h, lw["wv"]).reshape(B, cfg.n_kv_heads, cfg.head_dim)
    o = block_attention(q, np.concatenate([k_ctx, k], axis=0), np.concatenate([v_ctx, v], axis=0))
    x = x + linear(o.reshape(B, cfg.q_dim), lw["wo"])
    h = rms_norm(x, lw["mlp_norm"], cfg.rms_eps)
    x = x + linear(silu(linear(h, lw["wgate"])) * linear(h, lw["wup"]), lw["wdown"])
    return x


def window_start(P: int, window: int) -> int:
    """First context position a block at P attends to: P - window for a sliding
    window of `window` positions ("DFlash 소개": the MLX backend bounds the
    drafter's KV cache by a sliding window for long contexts), 0 without one
    (window 0)."""
    return max(0, P - window) if window > 0 else 0


def draft_block(cfg, weights: Dict, anchor: int, cache: Cache, B: int,
                ctx_len: Optional[int] = None, window: int = 0) -> Dict[str, object]:
    """One non-autoregressive drafter pass ([P1] §2 cycle steps 1-3; [P3] §2.2).

    Block = the anchor (last accepted token) at position P, then B-1 mask tokens
    at P+1..P+B-1; all B-1 masked positions are predicted in this single pass
    through the shared, frozen embedding and LM head ([P3] §2.3). With a sliding
    window (window > 0) the block attends to context positions
    window_start(P, window) .. P-1 only; the block itself is always fully visible.

    Returns dict(draft [B-1] int, logits [B-1, V] float64, hidden: list of the
    residual stream after every layer [B, H] plus the final normed rows)."""
    P = cache.length if ctx_len is None else ctx_len
    lo = window_start(P, window)
    ids = [int(anchor)] + [cfg.mask_token_id] * (B - 1)
    x = f64(weights["embed"])[ids]
    pos = np.arange(P, P + B)
    hidden = []
    for l, lw in enumerate(weights["layers"]):
        x = drafter_layer(cfg, lw, x, pos, cache.k[l][lo:P], cache.v[l][lo:P])
        hidden.append(x)
    y = rms_norm(x, weights["final_norm"], cfg.rms_eps)
    hidden.append(y)
    logits = linear(y[1:], weights["lm_head"])
    draft = [greedy_argmax(row) for row in logits]
    return {"draft": np.asarray(draft, dtype=np.int64), "logits": logits, "hidden": hidden}


# --------------------------------------------------------------------------- verify

def greedy_argmax(z) -> int:
    """Index of the largest value; the lowest index among equal maxima.

    NaN ranks below every number; a row of NaN only gives 0. Comparison is in
    the precision of the values given (no rounding here)."""
    z = np.asarray(z)
    valid = ~np.isnan(z)
    if not valid.any():
        return 0
    m = z[valid].max()
    return int(np.flatnonzero(valid & (z == m))[0])


def verify(logits, draft) -> Tuple[int, int]:
    """Greedy verification of one block ([P1] §1: accept while the draft matches,
    the first mismatch is replaced by the target's own token; §2 step 4).

    logits [B, V]: the target's logits at block positions P..P+B-1 (row j scores
    the token at position P+j+1); draft [B-1]: d_1..d_{B-1}.
    g_j = argmax logits[j]; a = number of leading i >= 1 with d_i == g_{i-1};
    next = g_a (the correction, or the bonus token when all B-1 are accepted).
    The committed tokens are d_1..d_a followed by next."""
    B = len(logits)
    g = [greedy_argmax(logits[j]) for j in range(B)]
    a = 0
    while a < B - 1 and int(draft[a]) == g[a]:
        a += 1
    return a, g[a]


def verify_batch(logits, draft) -> Tuple[np.ndarray, np.ndarray]:
    """verify() for every request of a batch: logits [bs, B, V], draft [bs, B-1]."""
    res = [verify(logits[r], draft[r]) for r in range(len(logits))]
    return (np.asarray([a for a, _ in res], dtype=np.int64),
            np.asarray([n for _, n in res], dtype=np.int64))
