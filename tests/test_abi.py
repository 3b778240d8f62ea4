"""Host-side checks of the C ABI that need no GPU: the library builds, loads and
exports every entry point include/dflash.h declares, and the binding declares
the same names."""
import ctypes
import os
import re

import pytest

from block_diffusion_speculative_cycle_b200 import _binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_entry_points():
    src = open(os.path.join(ROOT, "include", "dflash.h"), encoding="utf-8").read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dflash_[a-z_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib_path():
    return build.build()


def test_header_declares_the_cycle_calls():
    names = declared_entry_points()
    for n in ("dflash_inject_ctx", "dflash_draft_block", "dflash_verify", "dflash_create", "dflash_destroy"):
        assert n in names


def test_library_exports_every_declared_symbol(lib_path):
    exported = _binding.exported_symbols(lib_path)
    missing = [n for n in declared_entry_points() if n not in exported]
    assert not missing, missing
    assert sorted(_binding.EXPORTS) == declared_entry_points()


def test_status_strings_and_workspace_size(lib_path):
    lib = _binding.load_library(lib_path)
    assert lib.dflash_status_string(0) == b"ok"
    assert lib.dflash_status_string(5).startswith(b"out-of-range")
    assert lib.dflash_verify_workspace_size(0, 4) == 0
    assert lib.dflash_verify_workspace_size(3, 16) >= 3 * 16 * 8 + 3 * 4


def test_create_rejects_bad_config_without_touching_the_gpu(lib_path):
    import ctypes
    lib = _binding.load_library(lib_path)
    cfg = _binding.dflash_config()
    w = _binding.dflash_weights()
    h = ctypes.c_void_p()
    assert lib.dflash_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h)) == 1   # DFLASH_ERR_ARG
    assert lib.dflash_create(None, None, ctypes.byref(h)) == 1
    assert lib.dflash_verify(None, 0, None, 1, 4, 10, None, None, None, 0, None) == 1


def test_drafter_config_marshalling(monkeypatch):
    """The Drafter wrapper fills dflash_config field by field (no GPU: the C call is stubbed)."""
    import torch
    from block_diffusion_speculative_cycle_b200 import synth
    seen = {}
    monkeypatch.setattr(_binding, "dflash_create", lambda c, w: seen.setdefault("c", c) and 0)
    cfg = synth.TINY
    _binding.Drafter(cfg, synth.make_drafter_weights(cfg, seed=0), max_block=4, max_batch=2, max_inject_rows=8)
    c = seen.pop("c")
    assert (c.hidden, c.n_layers, c.max_block, c.max_batch, c.max_inject_rows) == (cfg.hidden, cfg.n_layers, 4, 2, 8)
    assert c.dtype == _binding.DFLASH_F32 and c.cache_dtype == _binding.DFLASH_F32
    cfg16 = cfg.replace(dtype="bf16")
    d = _binding.Drafter(cfg16, synth.make_drafter_weights(cfg16, seed=0), max_block=4, cache_dtype=torch.float16)
    c = seen.pop("c")
    assert c.dtype == _binding.DFLASH_BF16 and c.cache_dtype == _binding.DFLASH_F16
    assert d.cache_dtype == torch.float16


def _valid_config():
    """A supported bf16 drafter shape (the checks below each break one field)."""
    c = _binding.dflash_config()
    c.hidden, c.n_layers, c.n_q_heads, c.n_kv_heads, c.head_dim = 512, 2, 4, 2, 128
    c.intermediate, c.vocab, c.n_feat_layers, c.target_hidden, c.mask_token_id = 1024, 2048, 3, 256, 2047
    c.max_block, c.max_batch, c.max_inject_rows, c.page_size = 16, 2, 64, 64
    c.rope_theta, c.rms_eps, c.dtype, c.cache_dtype = 1e4, 1e-6, _binding.DFLASH_BF16, _binding.DFLASH_BF16
    return c


def _fake_weights():
    import ctypes
    w = _binding.dflash_weights()
    arr = (ctypes.c_void_p * 2)(16, 16)
    w.fc = w.embed = w.lm_head = w.final_norm = 16   # never dereferenced: every case below fails first
    for k in ("attn_norm", "wq", "wk", "wv", "wo", "mlp_norm", "wgate", "wup", "wdown"):
        setattr(w, k, ctypes.cast(arr, _binding._PP))
    return w, arr


@pytest.mark.parametrize("field,value,status", [
    ("mask_token_id", 2048, 1),            # outside the vocabulary
    ("n_kv_heads", 3, 1),                  # n_q not a multiple of n_kv
    ("dtype", 7, 1),                       # unknown weight type
    ("head_dim", 96, 6),                   # only 64 and 128
    ("hidden", 576, 6),                    # not a multiple of the 128-row weight tile
    ("vocab", 2000, 6),
    ("max_block", 70, 6),                  # g * B > 128 query rows per head group
])
def test_create_validates_each_field_on_the_host(lib_path, field, value, status):
    import ctypes
    lib = _binding.load_library(lib_path)
    c = _valid_config()
    setattr(c, field, value)
    if field == "vocab":
        c.mask_token_id = value - 1
    w, _keep = _fake_weights()
    h = ctypes.c_void_p()
    assert lib.dflash_create(ctypes.byref(c), ctypes.byref(w), ctypes.byref(h)) == status
    assert not h.value


def test_fp16_cache_needs_a_bf16_drafter(lib_path):
    import ctypes
    lib = _binding.load_library(lib_path)
    c = _valid_config()
    c.dtype, c.cache_dtype = _binding.DFLASH_F32, _binding.DFLASH_F16
    w, _keep = _fake_weights()
    h = ctypes.c_void_p()
    assert lib.dflash_create(ctypes.byref(c), ctypes.byref(w), ctypes.byref(h)) == 1


def test_cycle_calls_reject_a_null_context(lib_path):
    lib = _binding.load_library(lib_path)
    assert lib.dflash_inject_ctx(None, None, 1, 1, None, None, None, None, None, 1, 1, None) == 1
    assert lib.dflash_draft_block(None, None, None, 1, 4, None, None, None, 1, 1, 0, None, None, None) == 1
    assert lib.dflash_get_error(None, None) == 1


def test_loop_sampling_and_policy_calls_check_their_arguments_on_the_host(lib_path):
    """The device-loop, sampled and acceptance-count calls refuse bad arguments with
    DFLASH_ERR_ARG (1) before any launch, so these run without a GPU. Pointers that
    are only checked for null are fake addresses, never dereferenced."""
    lib = _binding.load_library(lib_path)
    fake = ctypes.c_void_p(0x1000)
    # a null context
    taps = (ctypes.c_int * 1)(0)
    assert lib.dflash_target_forward(None, fake, None, None, 1, 1, fake, None, None, fake, 1, 1, 0, taps, 0, fake,
                                     None, None) == 1
    assert lib.dflash_draft_block_sample(None, fake, fake, 1, 4, None, None, fake, 1, 1, 0, ctypes.c_float(1.0), 7,
                                         fake, fake, None, None) == 1
    # the commit: empty batch, or drafts missing for B > 1
    args = [fake, fake, fake, fake, 8, fake, fake, fake, fake, fake, None]
    assert lib.dflash_spec_commit(0, 4, *args) == 1
    assert lib.dflash_spec_commit(1, 4, None, *args[1:]) == 1
    # sampled verify: temperature, empty batch, misaligned workspace
    ws_bytes = lib.dflash_verify_sampled_workspace_size(2, 4, 1000)
    assert ws_bytes > 0
    good_ws = ctypes.c_void_p(0x100000)

    def vs(bs, temp, ws):
        return lib.dflash_verify_sampled(fake, _binding.DFLASH_F32, fake, fake, bs, 4, 1000, ctypes.c_float(temp), fake,
                                         fake, fake, fake, ws, ws_bytes, None)

    assert vs(2, 0.0, good_ws) == 1
    assert vs(2, float("inf"), good_ws) == 1
    assert vs(0, 1.0, good_ws) == 1
    assert vs(2, 1.0, ctypes.c_void_p(0x100010)) == 1
    # acceptance counts: null arrays, a block past the count array; B = 1 tests nothing
    assert lib.dflash_acceptance_count(None, 2, 4, fake, 16, None) == 1
    assert lib.dflash_acceptance_count(fake, 2, 17, fake, 16, None) == 1
    assert lib.dflash_acceptance_count(fake, 2, 1, fake, 16, None) == 0
