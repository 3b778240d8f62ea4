"""Shared set-up for the GPU parity tests: the same seeded CPU inputs go to the
CUDA path (moved to the device) and to the oracle (widened to float64). No
value read back from the GPU is ever fed to the oracle."""
from __future__ import annotations

import numpy as np
import torch

from block_diffusion_speculative_cycle_b200 import Drafter, synth
from oracle import dflash as O


def to_dev(weights, dev="cuda"):
    out = {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in weights.items() if k != "layers"}
    out["layers"] = [{k: v.to(dev) for k, v in lw.items()} for lw in weights["layers"]]
    return out


def max_abs_rel(gpu: np.ndarray, ref: np.ndarray) -> float:
    """max_i |gpu - ref| / max_i |ref| over one tensor."""
    denom = float(np.max(np.abs(ref)))
    return float(np.max(np.abs(gpu - ref))) / (denom if denom > 0 else 1.0)


def top2_gap(logits: np.ndarray) -> np.ndarray:
    s = np.sort(logits, axis=-1)
    return s[..., -1] - s[..., -2]


class PagedCache:
    """Device page pools [num_pages, n_kv, page, d] per layer plus a page table."""

    def __init__(self, cfg, page_table: torch.Tensor, num_pages: int, page_size: int, dev="cuda", init=None,
                 dtype=None):
        self.cfg = cfg
        self.page_size = page_size
        self.num_pages = num_pages
        self.table_cpu = page_table
        self.table = page_table.to(dev)
        shape = (num_pages, cfg.n_kv_heads, page_size, cfg.head_dim)
        dt = dtype or cfg.torch_dtype
        if init is None:
            self.k = [torch.zeros(shape, dtype=dt, device=dev) for _ in range(cfg.n_layers)]
            self.v = [torch.zeros(shape, dtype=dt, device=dev) for _ in range(cfg.n_layers)]
        else:
            self.k = [lay["k"].to(device=dev, dtype=dt) for lay in init]
            self.v = [lay["v"].to(device=dev, dtype=dt) for lay in init]

    @property
    def max_pages(self):
        return self.table.shape[1]


def slots_of(pos: np.ndarray, page_size: int) -> np.ndarray:
    return (pos % page_size).astype(np.int64)


def gather_cpu_cache(cfg, pools_cpu, table_cpu: torch.Tensor, r: int, P: int, page_size: int):
    """Oracle view of request r's first P positions from CPU page pools (synth input)."""
    ks, vs = [], []
    pos = np.arange(P)
    pages = torch.as_tensor(table_cpu[r].numpy()[pos // page_size].astype(np.int64))
    slots = torch.as_tensor(slots_of(pos, page_size))
    for lay in pools_cpu:
        # gather this request's rows first, then widen only those
        k = O.f64(lay["k"][pages, :, slots, :])   # [P, n_kv, d]
        v = O.f64(lay["v"][pages, :, slots, :])
        ks.append(k)
        vs.append(v)
    return O.Cache.from_arrays(cfg, ks, vs)


def make_drafter(cfg, weights_cpu, max_block, max_batch=1, max_inject_rows=64, page_size=64, cache_dtype=None,
                 window=0):
    wd = to_dev(weights_cpu)
    return Drafter(cfg, wd, max_block=max_block, max_batch=max_batch, max_inject_rows=max_inject_rows,
                   page_size=page_size, cache_dtype=cache_dtype, window=window), wd
