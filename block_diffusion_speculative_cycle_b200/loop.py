"""Speculative decoding entirely on the device: a causal target (the library's
dflash_target_forward), the block drafter, greedy verify and the device-side
commit, shaped like the pages' spec_generate(target, draft, input_ids,
num_speculative_tokens, temperature, max_new_tokens) ("DFlash 소개", usage;
"DFlash — 블록 확산 드래프터로 6배 빨라지는 투기적 디코딩" §1-2 for the cycle).

Every cycle is enqueued without reading anything back: the anchor, context
length, injection rows and start position, and the output, live in device
tensors that dflash_spec_commit updates, so cycles can be graph-captured and the
host only checks progress between batches of cycles. This module only orders
library calls; the arithmetic runs in the library's kernels.
"""
from __future__ import annotations

from typing import Callable, Optional, Sequence

import torch

from ._binding import (Drafter, dflash_spec_commit, dflash_target_forward, dflash_verify,
                       dflash_verify_workspace_size)


class GpuTarget:
    """A causal target of the drafter's layer type on the device (fp32), with its
    own paged KV cache (identity page table) of `capacity` positions per request."""

    def __init__(self, cfg, weights_dev, bs: int, max_rows: int, capacity: int, taps: Sequence[int],
                 page_size: int = 64):
        self.cfg, self.bs, self.taps = cfg, bs, list(taps)
        # the target context: the drafter-layer machinery with the target's weights (fc unused)
        self.ctx = Drafter(cfg, weights_dev, max_block=max_rows, max_batch=bs, max_inject_rows=1, page_size=page_size)
        pages = (capacity + page_size - 1) // page_size
        dev = weights_dev["embed"].device
        self.table = torch.arange(bs * pages, dtype=torch.int32, device=dev).reshape(bs, pages)
        self.num_pages = bs * pages
        shape = (self.num_pages, cfg.n_kv_heads, page_size, cfg.head_dim)
        self.kc = [torch.zeros(shape, dtype=torch.float32, device=dev) for _ in range(cfg.n_layers)]
        self.vc = [torch.zeros(shape, dtype=torch.float32, device=dev) for _ in range(cfg.n_layers)]
        self.max_ctx = capacity - max_rows   # every forward passes the same bound (same split plan)

    def forward(self, tokens, anchor, draft, n, pos0, logits, feats, stream=None):
        """feats None: no tapped features are written."""
        taps = self.taps if feats is not None else []
        dflash_target_forward(self.ctx.handle, tokens, anchor, draft, self.bs, n, pos0, self.kc, self.vc, self.table,
                              self.num_pages, self.max_ctx, taps, logits, feats, stream)

    def close(self):
        self.ctx.close()


class SpecDecoder:
    """Greedy speculative decoding of `bs` requests with block size B.

    drafter: a Drafter whose cache pools / page table are given (k_cache, v_cache,
    table, num_pages, max_ctx); target: a GpuTarget with taps matching the
    drafter's feature layers."""

    def __init__(self, target: GpuTarget, drafter: Drafter, d_kc, d_vc, d_table, d_num_pages: int, d_max_ctx: int,
                 B: int, max_out: int):
        self.t, self.d = target, drafter
        self.dkc, self.dvc, self.dtable, self.dnum, self.dmax = d_kc, d_vc, d_table, d_num_pages, d_max_ctx
        self.B, self.bs, self.max_out = B, target.bs, max_out
        dev = d_table.device
        i32 = dict(dtype=torch.int32, device=dev)
        bs, V, F = self.bs, target.cfg.vocab, len(target.taps) * target.cfg.hidden
        self.anchor = torch.zeros(bs, **i32)
        self.ctx_len = torch.zeros(bs, **i32)
        self.n_new = torch.zeros(bs, **i32)
        self.start = torch.zeros(bs, **i32)
        self.out = torch.zeros((bs, max_out), **i32)
        self.out_len = torch.zeros(bs, **i32)
        self.draft = torch.zeros((bs, max(B - 1, 1)), **i32)
        self.acc = torch.zeros(bs, **i32)
        self.nxt = torch.zeros(bs, **i32)
        self.logits = torch.zeros((bs, B, V), dtype=torch.float32, device=dev)
        self.feats = torch.zeros((bs, B, F), dtype=torch.float32, device=dev)
        self.ws = torch.zeros(dflash_verify_workspace_size(bs, B), dtype=torch.uint8, device=dev)

    def prefill(self, prompt: torch.Tensor, stream=None):
        """prompt [bs, P0] int32 (device): the target's prefill gives the first token
        (the anchor) and the features of positions 0..P0-1, injected into the drafter."""
        bs, P0 = prompt.shape
        dev = prompt.device
        V, F = self.t.cfg.vocab, len(self.t.taps) * self.t.cfg.hidden
        logits = torch.zeros((bs, P0, V), dtype=torch.float32, device=dev)
        feats = torch.zeros((bs, P0, F), dtype=torch.float32, device=dev)
        zero = torch.zeros(bs, dtype=torch.int32, device=dev)
        self.t.forward(prompt, None, None, P0, zero, logits, feats, stream)
        # the anchor: greedy choice on the last prompt row (verify with a one-row block)
        last = logits[:, P0 - 1:P0, :].contiguous()
        ws = torch.zeros(dflash_verify_workspace_size(bs, 1), dtype=torch.uint8, device=dev)
        dflash_verify(last, self.draft, self.acc, self.anchor, ws, stream)
        n_all = torch.full((bs,), P0, dtype=torch.int32, device=dev)
        self.d.inject(feats, bs, P0, n_all, zero, self.dkc, self.dvc, self.dtable, self.dnum, stream)
        self.ctx_len.fill_(P0)
        self.out[:, 0] = self.anchor
        self.out_len.fill_(1)

    def cycle(self, hook: Optional[Callable] = None, stream=None):
        """Enqueue one cycle (no host synchronisation): draft at the current context
        length, the target's block forward [anchor, d_1..d_{B-1}], greedy verify,
        device-side commit, injection of the committed rows' features. `hook(self)`,
        if given, runs after drafting (tests use it to plant drafts)."""
        B, bs = self.B, self.bs
        self.d.draft(self.anchor, self.ctx_len, bs, B, self.dkc, self.dvc, self.dtable, self.dnum, self.dmax,
                     self.draft, None, stream)
        if hook is not None:
            hook(self)
        self.t.forward(None, self.anchor, self.draft, B, self.ctx_len, self.logits, self.feats, stream)
        dflash_verify(self.logits, self.draft, self.acc, self.nxt, self.ws, stream)
        dflash_spec_commit(bs, B, self.draft, self.acc, self.nxt, self.out, self.out_len, self.anchor, self.ctx_len,
                           self.n_new, self.start, stream)
        self.d.inject(self.feats, bs, B, self.n_new, self.start, self.dkc, self.dvc, self.dtable, self.dnum, stream)

    def generate(self, n_tokens: int, check_every: int = 16, hook: Optional[Callable] = None):
        """Run cycles until every request has n_tokens tokens (the host reads the
        output lengths once per `check_every` cycles)."""
        while True:
            for _ in range(check_every):
                self.cycle(hook)
            if int(self.out_len.min().item()) >= n_tokens:
                return self.out[:, :n_tokens]


def greedy_decode_gpu(target: GpuTarget, prompt: torch.Tensor, n_tokens: int) -> torch.Tensor:
    """The target's own greedy decoding on the device, one token per forward (the
    reference the speculative loop must reproduce)."""
    bs, P0 = prompt.shape
    dev = prompt.device
    V = target.cfg.vocab
    logits = torch.zeros((bs, P0, V), dtype=torch.float32, device=dev)
    zero = torch.zeros(bs, dtype=torch.int32, device=dev)
    target.forward(prompt, None, None, P0, zero, logits, None, None)
    tok = torch.zeros(bs, dtype=torch.int32, device=dev)
    acc = torch.zeros(bs, dtype=torch.int32, device=dev)
    dummy = torch.zeros((bs, 1), dtype=torch.int32, device=dev)
    ws = torch.zeros(dflash_verify_workspace_size(bs, 1), dtype=torch.uint8, device=dev)
    dflash_verify(logits[:, P0 - 1:P0, :].contiguous(), dummy, acc, tok, ws)
    out = torch.zeros((bs, n_tokens), dtype=torch.int32, device=dev)
    out[:, 0] = tok
    step_logits = torch.zeros((bs, 1, V), dtype=torch.float32, device=dev)
    pos = torch.full((bs,), P0, dtype=torch.int32, device=dev)
    for k in range(1, n_tokens):
        target.forward(None, out[:, k - 1].contiguous(), None, 1, pos, step_logits, None, None)
        dflash_verify(step_logits, dummy, acc, tok, ws)
        out[:, k] = tok
        pos += 1
    return out
