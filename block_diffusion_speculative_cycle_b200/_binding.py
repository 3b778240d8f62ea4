"""ctypes binding of include/dflash.h (same entry-point names), plus `Drafter`,
a small convenience owner of one context.

Tensors are torch CUDA tensors; their data pointers and the current CUDA
stream are passed straight to the C ABI. Nothing here computes any part of
the cycle.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, List, Optional, Sequence

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libdflash.so")

DFLASH_F32 = 0
DFLASH_BF16 = 1
DFLASH_F16 = 2

_STATUS = {0: "DFLASH_OK", 1: "DFLASH_ERR_ARG", 2: "DFLASH_ERR_CUDA", 3: "DFLASH_ERR_OOM",
           4: "DFLASH_ERR_TIMEOUT", 5: "DFLASH_ERR_DEVICE", 6: "DFLASH_ERR_UNSUPPORTED"}

EXPORTS = ["dflash_create", "dflash_destroy", "dflash_inject_ctx", "dflash_draft_block", "dflash_draft_block_sample",
           "dflash_verify_sampled_workspace_size", "dflash_verify_sampled",
           "dflash_verify_workspace_size", "dflash_verify", "dflash_verify_noalloc", "dflash_profile_enable", "dflash_profile_read",
           "dflash_profile_gemm_chain", "dflash_get_error", "dflash_status_string", "dflash_acceptance_count",
           "dflash_block_policy_create", "dflash_block_policy_destroy", "dflash_block_policy_observe",
           "dflash_block_policy_expected_tokens", "dflash_block_policy_choose", "dflash_block_policy_choose_linear",
           "dflash_target_forward", "dflash_spec_commit"]


class DFlashError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_STATUS.get(status, status)}")


class dflash_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "hidden", "n_layers", "n_q_heads", "n_kv_heads", "head_dim", "intermediate", "vocab", "n_feat_layers",
        "target_hidden", "mask_token_id", "max_block", "max_batch", "max_inject_rows", "page_size")] + [
        ("rope_theta", ctypes.c_float), ("rms_eps", ctypes.c_float), ("dtype", ctypes.c_int),
        ("cache_dtype", ctypes.c_int), ("window", ctypes.c_int)]


_P = ctypes.c_void_p
_PP = ctypes.POINTER(ctypes.c_void_p)


class dflash_profile_entry(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int), ("total_ms", ctypes.c_double),
                ("bytes", ctypes.c_double), ("flops", ctypes.c_double)]


class dflash_weights(ctypes.Structure):
    _fields_ = [("fc", _P), ("embed", _P), ("lm_head", _P), ("final_norm", _P), ("attn_norm", _PP), ("wq", _PP),
                ("wk", _PP), ("wv", _PP), ("wo", _PP), ("mlp_norm", _PP), ("wgate", _PP), ("wup", _PP),
                ("wdown", _PP)]


_lib = None


def load_library(path: Optional[str] = None):
    """Load libdflash.so (built in-tree by build.py). Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise ImportError(f"libdflash.so not found at {path}; build it with "
                          "`python -m block_diffusion_speculative_cycle_b200.build`")
    lib = ctypes.CDLL(path)
    c_int, c_size = ctypes.c_int, ctypes.c_size_t
    lib.dflash_create.argtypes = [ctypes.POINTER(dflash_config), ctypes.POINTER(dflash_weights), ctypes.POINTER(_P)]
    lib.dflash_create.restype = c_int
    lib.dflash_destroy.argtypes = [_P]
    lib.dflash_destroy.restype = None
    lib.dflash_inject_ctx.argtypes = [_P, _P, c_int, c_int, _P, _P, _PP, _PP, _P, c_int, c_int, _P]
    lib.dflash_inject_ctx.restype = c_int
    lib.dflash_draft_block.argtypes = [_P, _P, _P, c_int, c_int, _PP, _PP, _P, c_int, c_int, c_int, _P, _P, _P]
    lib.dflash_draft_block.restype = c_int
    lib.dflash_draft_block_sample.argtypes = [_P, _P, _P, c_int, c_int, _PP, _PP, _P, c_int, c_int, c_int,
                                              ctypes.c_float, ctypes.c_ulonglong, _P, _P, _P, _P]
    lib.dflash_draft_block_sample.restype = c_int
    lib.dflash_verify_sampled_workspace_size.argtypes = [c_int, c_int, c_int]
    lib.dflash_verify_sampled_workspace_size.restype = c_size
    lib.dflash_verify_sampled.argtypes = [_P, c_int, _P, _P, c_int, c_int, c_int, ctypes.c_float, _P, _P, _P, _P, _P,
                                          c_size, _P]
    lib.dflash_verify_sampled.restype = c_int
    lib.dflash_verify_workspace_size.argtypes = [c_int, c_int]
    lib.dflash_verify_workspace_size.restype = c_size
    lib.dflash_verify.argtypes = [_P, c_int, _P, c_int, c_int, c_int, _P, _P, _P, c_size, _P]
    lib.dflash_verify.restype = c_int
    lib.dflash_verify_noalloc.argtypes = [_P, c_int, _P, c_int, c_int, c_int, _P, _P, _P]
    lib.dflash_verify_noalloc.restype = c_int
    lib.dflash_profile_enable.argtypes = [_P, c_int]
    lib.dflash_profile_enable.restype = c_int
    lib.dflash_profile_read.argtypes = [_P, ctypes.POINTER(dflash_profile_entry), c_int]
    lib.dflash_profile_read.restype = c_int
    lib.dflash_profile_gemm_chain.argtypes = [_P, _P, c_int, c_int, _P, _P, _PP, _PP, _P, c_int, c_int, _P, c_int, _P]
    lib.dflash_profile_gemm_chain.restype = c_int
    c_dbl, c_u64p = ctypes.c_double, ctypes.POINTER(ctypes.c_ulonglong)
    lib.dflash_acceptance_count.argtypes = [_P, c_int, c_int, _P, c_int, _P]
    lib.dflash_acceptance_count.restype = c_int
    lib.dflash_block_policy_create.argtypes = [ctypes.POINTER(c_int), c_int, c_dbl, c_int, ctypes.POINTER(_P)]
    lib.dflash_block_policy_create.restype = c_int
    lib.dflash_block_policy_destroy.argtypes = [_P]
    lib.dflash_block_policy_destroy.restype = None
    lib.dflash_block_policy_observe.argtypes = [_P, c_u64p, c_u64p, c_int]
    lib.dflash_block_policy_observe.restype = c_int
    lib.dflash_block_policy_expected_tokens.argtypes = [_P, c_int]
    lib.dflash_block_policy_expected_tokens.restype = c_dbl
    lib.dflash_block_policy_choose.argtypes = [_P, ctypes.POINTER(c_dbl), c_int]
    lib.dflash_block_policy_choose.restype = c_int
    lib.dflash_block_policy_choose_linear.argtypes = [_P, c_int, c_dbl, c_dbl]
    lib.dflash_block_policy_choose_linear.restype = c_int
    lib.dflash_target_forward.argtypes = [_P, _P, _P, _P, c_int, c_int, _P, _PP, _PP, _P, c_int, c_int, c_int,
                                          ctypes.POINTER(c_int), c_int, _P, _P, _P]
    lib.dflash_target_forward.restype = c_int
    lib.dflash_spec_commit.argtypes = [c_int, c_int, _P, _P, _P, _P, c_int, _P, _P, _P, _P, _P, _P]
    lib.dflash_spec_commit.restype = c_int
    lib.dflash_get_error.argtypes = [_P, _P]
    lib.dflash_get_error.restype = c_int
    lib.dflash_status_string.argtypes = [c_int]
    lib.dflash_status_string.restype = ctypes.c_char_p
    _lib = lib
    return lib


def exported_symbols(path: Optional[str] = None) -> List[str]:
    """Names of the C-ABI entry points the library exports (resolved with dlsym)."""
    lib = ctypes.CDLL(path or LIB_PATH)
    found = []
    for name in EXPORTS:
        try:
            getattr(lib, name)
            found.append(name)
        except AttributeError:
            pass
    return found


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr_array(tensors: Sequence) -> ctypes.Array:
    arr = (ctypes.c_void_p * max(1, len(tensors)))()
    for i, t in enumerate(tensors):
        arr[i] = t.data_ptr()
    return arr


def _check(status: int, where: str):
    if status != 0:
        raise DFlashError(status, where)


def dflash_status_string(status: int) -> str:
    return load_library().dflash_status_string(status).decode()


def dflash_create(cfg: dflash_config, weights: dflash_weights) -> int:
    lib = load_library()
    h = _P()
    _check(lib.dflash_create(ctypes.byref(cfg), ctypes.byref(weights), ctypes.byref(h)), "dflash_create")
    return h.value


def dflash_destroy(handle: int) -> None:
    load_library().dflash_destroy(handle)


def dflash_inject_ctx(handle, feats, bs, max_new, n_new, start_pos, k_cache, v_cache, page_table,
                      num_pages, stream=None) -> None:
    lib = load_library()
    _check(lib.dflash_inject_ctx(handle, _ptr(feats), bs, max_new, _ptr(n_new), _ptr(start_pos),
                                 _ptr_array(k_cache), _ptr_array(v_cache), _ptr(page_table),
                                 page_table.shape[1], num_pages, _stream(stream)), "dflash_inject_ctx")


def dflash_draft_block(handle, anchor, ctx_len, bs, B, k_cache, v_cache, page_table, num_pages, max_ctx, draft,
                       hidden_out=None, stream=None) -> None:
    lib = load_library()
    _check(lib.dflash_draft_block(handle, _ptr(anchor), _ptr(ctx_len), bs, B, _ptr_array(k_cache),
                                  _ptr_array(v_cache), _ptr(page_table), page_table.shape[1], num_pages, max_ctx,
                                  _ptr(draft), _ptr(hidden_out), _stream(stream)), "dflash_draft_block")


def dflash_draft_block_sample(handle, anchor, ctx_len, bs, B, k_cache, v_cache, page_table, num_pages, max_ctx,
                              temperature, seed, draft, draft_logits, hidden_out=None, stream=None) -> None:
    lib = load_library()
    _check(lib.dflash_draft_block_sample(handle, _ptr(anchor), _ptr(ctx_len), bs, B, _ptr_array(k_cache),
                                         _ptr_array(v_cache), _ptr(page_table), page_table.shape[1], num_pages,
                                         max_ctx, float(temperature), int(seed), _ptr(draft), _ptr(draft_logits),
                                         _ptr(hidden_out), _stream(stream)), "dflash_draft_block_sample")


def dflash_verify_sampled_workspace_size(bs: int, B: int, V: int) -> int:
    return int(load_library().dflash_verify_sampled_workspace_size(bs, B, V))


def dflash_verify_sampled(logits, draft_logits, draft, temperature, u_accept, u_final, accepted, next_token,
                          workspace, stream=None) -> None:
    import torch
    lib = load_library()
    bs, B, V = logits.shape
    dt = DFLASH_BF16 if logits.dtype == torch.bfloat16 else DFLASH_F32
    _check(lib.dflash_verify_sampled(_ptr(logits), dt, _ptr(draft_logits), _ptr(draft), bs, B, V, float(temperature),
                                     _ptr(u_accept), _ptr(u_final), _ptr(accepted), _ptr(next_token),
                                     _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)),
           "dflash_verify_sampled")


def verify_sampled(logits, draft_logits, draft, temperature, u_accept, u_final, workspace=None, stream=None):
    """Allocate outputs (and scratch unless given) and run dflash_verify_sampled; returns (accepted, next_token)."""
    import torch
    bs, B, V = logits.shape
    dev = logits.device
    acc = torch.empty(bs, dtype=torch.int32, device=dev)
    nxt = torch.empty(bs, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = torch.zeros(dflash_verify_sampled_workspace_size(bs, B, V), dtype=torch.uint8, device=dev)
    dflash_verify_sampled(logits, draft_logits, draft, temperature, u_accept, u_final, acc, nxt, workspace, stream)
    return acc, nxt


def dflash_verify_workspace_size(bs: int, B: int) -> int:
    return int(load_library().dflash_verify_workspace_size(bs, B))


def dflash_verify(logits, draft, accepted, next_token, workspace, stream=None) -> None:
    import torch
    lib = load_library()
    bs, B, V = logits.shape
    dt = DFLASH_BF16 if logits.dtype == torch.bfloat16 else DFLASH_F32
    _check(lib.dflash_verify(_ptr(logits), dt, _ptr(draft), bs, B, V, _ptr(accepted), _ptr(next_token),
                             _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)),
           "dflash_verify")


def dflash_profile_enable(handle, enable: bool) -> None:
    _check(load_library().dflash_profile_enable(handle, 1 if enable else 0), "dflash_profile_enable")


def dflash_profile_read(handle) -> List[dict]:
    """Aggregated per-kernel timings since the last read: list of dicts
    (name, launches, total_ms, bytes, flops)."""
    arr = (dflash_profile_entry * 32)()
    n = load_library().dflash_profile_read(handle, arr, 32)
    if n < 0:
        raise DFlashError(-n, "dflash_profile_read")
    return [{"name": arr[i].name.decode(), "launches": arr[i].launches, "total_ms": arr[i].total_ms,
             "bytes": arr[i].bytes, "flops": arr[i].flops} for i in range(n)]


def dflash_profile_gemm_chain(handle, feats, bs, max_new, n_new, start_pos, k_cache, v_cache, page_table,
                              num_pages, ctx_len, B, stream=None) -> None:
    lib = load_library()
    _check(lib.dflash_profile_gemm_chain(handle, _ptr(feats), bs, max_new, _ptr(n_new), _ptr(start_pos),
                                         _ptr_array(k_cache), _ptr_array(v_cache), _ptr(page_table),
                                         page_table.shape[1], num_pages, _ptr(ctx_len), B, _stream(stream)),
           "dflash_profile_gemm_chain")


def dflash_acceptance_count(accepted, B, counts, stream=None) -> None:
    """counts: device uint64 (int64) tensor [2 * n_pos]: tested, then accepted per position."""
    n_pos = counts.numel() // 2
    _check(load_library().dflash_acceptance_count(_ptr(accepted), accepted.numel(), B, _ptr(counts), n_pos,
                                                  _stream(stream)), "dflash_acceptance_count")


class BlockPolicy:
    """The library's block-size policy (host-side C++ object)."""

    def __init__(self, candidates, decay: float, n_pos: int):
        lib = load_library()
        arr = (ctypes.c_int * len(candidates))(*[int(b) for b in candidates])
        h = _P()
        _check(lib.dflash_block_policy_create(arr, len(candidates), float(decay), n_pos, ctypes.byref(h)),
               "dflash_block_policy_create")
        self.handle, self.n_pos = h.value, n_pos
        self.candidates = sorted(int(b) for b in candidates)

    def close(self):
        if getattr(self, "handle", None):
            load_library().dflash_block_policy_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def observe(self, tested, accepted) -> None:
        t = (ctypes.c_ulonglong * self.n_pos)(*[int(x) for x in tested])
        a = (ctypes.c_ulonglong * self.n_pos)(*[int(x) for x in accepted])
        _check(load_library().dflash_block_policy_observe(self.handle, t, a, self.n_pos),
               "dflash_block_policy_observe")

    def expected_tokens(self, B: int) -> float:
        return float(load_library().dflash_block_policy_expected_tokens(self.handle, B))

    def choose(self, costs) -> int:
        c = (ctypes.c_double * len(costs))(*[float(x) for x in costs])
        r = load_library().dflash_block_policy_choose(self.handle, c, len(costs))
        if r < 0:
            raise DFlashError(-r, "dflash_block_policy_choose")
        return r

    def choose_linear(self, bs: int, c0: float, c1: float) -> int:
        r = load_library().dflash_block_policy_choose_linear(self.handle, bs, float(c0), float(c1))
        if r < 0:
            raise DFlashError(-r, "dflash_block_policy_choose_linear")
        return r


def dflash_target_forward(handle, tokens, anchor, draft, bs, n, pos0, k_cache, v_cache, page_table, num_pages,
                          max_ctx, taps, logits, feats, stream=None) -> None:
    lib = load_library()
    tp = (ctypes.c_int * max(1, len(taps)))(*[int(t) for t in taps])
    _check(lib.dflash_target_forward(handle, _ptr(tokens), _ptr(anchor), _ptr(draft), bs, n, _ptr(pos0),
                                     _ptr_array(k_cache), _ptr_array(v_cache), _ptr(page_table), page_table.shape[1],
                                     num_pages, max_ctx, tp, len(taps), _ptr(logits), _ptr(feats), _stream(stream)),
           "dflash_target_forward")


def dflash_spec_commit(bs, B, draft, accepted, next_token, out_tokens, out_len, anchor, ctx_len, n_new, start_pos,
                       stream=None) -> None:
    _check(load_library().dflash_spec_commit(bs, B, _ptr(draft), _ptr(accepted), _ptr(next_token), _ptr(out_tokens),
                                              out_tokens.shape[1], _ptr(out_len), _ptr(anchor), _ptr(ctx_len),
                                              _ptr(n_new), _ptr(start_pos), _stream(stream)), "dflash_spec_commit")


def dflash_get_error(handle, stream=None) -> int:
    return int(load_library().dflash_get_error(handle, _stream(stream)))


def verify(logits, draft, workspace=None, stream=None):
    """Allocate outputs (and scratch unless given) and run dflash_verify; returns (accepted, next_token)."""
    import torch
    bs, B, _ = logits.shape
    dev = logits.device
    acc = torch.empty(bs, dtype=torch.int32, device=dev)
    nxt = torch.empty(bs, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = torch.zeros(dflash_verify_workspace_size(bs, B), dtype=torch.uint8, device=dev)
    if draft is None or draft.numel() == 0:
        draft = torch.zeros((bs, max(B - 1, 1)), dtype=torch.int32, device=dev)
    dflash_verify(logits, draft, acc, nxt, workspace, stream)
    return acc, nxt


class Drafter:
    """Owns one dflash context for a set of device weights (kept referenced).

    cfg: a synth.DrafterConfig-like object (hidden, n_layers, ..., dtype "bf16"/"f32").
    weights: dict with fc, embed, lm_head, final_norm and per-layer dicts (see synth)."""

    def __init__(self, cfg, weights: Dict, max_block: int, max_batch: int = 1, max_inject_rows: int = 64,
                 page_size: int = 64, cache_dtype=None, window: int = 0):
        import torch
        self.cfg = cfg
        self.weights = weights
        c = dflash_config()
        c.hidden, c.n_layers, c.n_q_heads, c.n_kv_heads = cfg.hidden, cfg.n_layers, cfg.n_q_heads, cfg.n_kv_heads
        c.head_dim, c.intermediate, c.vocab = cfg.head_dim, cfg.intermediate, cfg.vocab
        c.n_feat_layers, c.target_hidden, c.mask_token_id = cfg.n_feat_layers, cfg.target_hidden, cfg.mask_token_id
        c.max_block, c.max_batch, c.max_inject_rows, c.page_size = max_block, max_batch, max_inject_rows, page_size
        c.rope_theta, c.rms_eps = cfg.rope_theta, cfg.rms_eps
        c.dtype = DFLASH_BF16 if cfg.dtype == "bf16" else DFLASH_F32
        # KV cache element type: the model dtype unless fp16 is asked for (bf16 drafters)
        c.cache_dtype = DFLASH_F16 if cache_dtype == torch.float16 else c.dtype
        c.window = window
        self.cache_dtype = torch.float16 if cache_dtype == torch.float16 else cfg.torch_dtype
        self.config = c
        L = weights["layers"]
        self._arrays = {k: _ptr_array([lw[k] for lw in L]) for k in
                        ("attn_norm", "wq", "wk", "wv", "wo", "mlp_norm", "wgate", "wup", "wdown")}
        w = dflash_weights()
        w.fc, w.embed, w.lm_head = weights["fc"].data_ptr(), weights["embed"].data_ptr(), weights["lm_head"].data_ptr()
        w.final_norm = weights["final_norm"].data_ptr()
        for k, arr in self._arrays.items():
            setattr(w, k, ctypes.cast(arr, _PP))
        self.handle = dflash_create(c, w)
        self.page_size = page_size

    def close(self):
        if getattr(self, "handle", None):
            dflash_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def inject(self, feats, bs, max_new, n_new, start_pos, k_cache, v_cache, page_table, num_pages, stream=None):
        dflash_inject_ctx(self.handle, feats, bs, max_new, n_new, start_pos, k_cache, v_cache, page_table,
                          num_pages, stream)

    def draft(self, anchor, ctx_len, bs, B, k_cache, v_cache, page_table, num_pages, max_ctx, draft,
              hidden_out=None, stream=None):
        dflash_draft_block(self.handle, anchor, ctx_len, bs, B, k_cache, v_cache, page_table, num_pages, max_ctx,
                           draft, hidden_out, stream)

    def draft_sample(self, anchor, ctx_len, bs, B, k_cache, v_cache, page_table, num_pages, max_ctx, temperature, seed,
                     draft, draft_logits, hidden_out=None, stream=None):
        dflash_draft_block_sample(self.handle, anchor, ctx_len, bs, B, k_cache, v_cache, page_table, num_pages,
                                  max_ctx, temperature, seed, draft, draft_logits, hidden_out, stream)

    def check(self, stream=None):
        st = dflash_get_error(self.handle, stream)
        if st != 0:
            raise DFlashError(st, "device status")
