"""B200 (sm_100a) DFlash draft cycle: Python binding of libdflash.so.

The binding only marshals arguments: every step of inject, draft and verify
runs in the library's CUDA kernels. Importing this package does not load the
library; the first call does, and it raises if the library is missing (there
is no CPU fallback).
"""
from ._binding import (  # noqa: F401
    DFLASH_BF16, DFLASH_F16, DFLASH_F32, DFlashError, Drafter, dflash_create, dflash_destroy, dflash_draft_block,
    dflash_get_error, dflash_inject_ctx, dflash_profile_enable, dflash_profile_gemm_chain, dflash_profile_read,
    dflash_status_string, dflash_verify, dflash_verify_workspace_size,
    dflash_draft_block_sample, dflash_verify_sampled, dflash_verify_sampled_workspace_size,
    BlockPolicy, dflash_acceptance_count, dflash_spec_commit, dflash_target_forward, exported_symbols, load_library,
    verify, verify_sampled,
)
