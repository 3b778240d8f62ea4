"""dflash_verify_noalloc: the verify entry point for callers that cannot
allocate device memory (a custom-operator interface that only hands over input
and output buffers, or a serving loop whose memory pool already owns the GPU's
free memory, where cudaMalloc can fail and synchronises the device). Its
scratch is a fixed array inside the library, so this test checks, through the
C ABI, that two calls in a row give exactly what the allocating dflash_verify
gives on the same inputs and what the oracle's verify gives (accepted length
equal to the planted one), including B = 1 with no draft array, and that sizes
beyond the fixed scratch are refused. Kept in a file pytest collects last."""
import ctypes

import numpy as np
import pytest
import torch

from block_diffusion_speculative_cycle_b200 import _binding, dflash_verify_workspace_size, load_library, synth
from oracle import dflash as O

pytestmark = pytest.mark.gpu


def _ptr(t):
    return t.data_ptr() if t is not None else None


def _noalloc(lib, logits, draft, acc, nxt):
    dt = _binding.DFLASH_BF16 if logits.dtype == torch.bfloat16 else _binding.DFLASH_F32
    bs, B, V = logits.shape
    return lib.dflash_verify_noalloc(logits.data_ptr(), dt, _ptr(draft), bs, B, V, acc.data_ptr(),
                                     nxt.data_ptr(), torch.cuda.current_stream().cuda_stream)


def _allocating(lib, logits, draft, acc, nxt):
    dt = _binding.DFLASH_BF16 if logits.dtype == torch.bfloat16 else _binding.DFLASH_F32
    bs, B, V = logits.shape
    ws = torch.zeros(dflash_verify_workspace_size(bs, B), dtype=torch.uint8, device="cuda")
    return lib.dflash_verify(logits.data_ptr(), dt, _ptr(draft), bs, B, V, acc.data_ptr(), nxt.data_ptr(),
                             ws.data_ptr(), ws.numel(), torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("dtype,bs,B,V", [(torch.bfloat16, 8, 16, 151936), (torch.float32, 3, 10, 1000),
                                          (torch.bfloat16, 4, 1, 8200)])
def test_noalloc_verify_matches_dflash_verify_and_the_oracle_twice_in_a_row(dtype, bs, B, V):
    """Two calls in a row (the second finds the shared scratch as the first left
    it): both give dflash_verify's result and the oracle's, bit for bit, and the
    planted acceptance lengths. B = 1 passes no draft array at all."""
    lib = load_library()
    for call in range(2):
        g = torch.Generator().manual_seed(1000 * call + bs)
        d_cpu = torch.randint(0, V, (bs, max(B - 1, 1)), generator=g, dtype=torch.int32)
        z_cpu, planted = synth.planted_logits(d_cpu[:, :B - 1], V, 2.0, 4.0, seed=call + V, dtype=dtype)
        ora_a, ora_n = O.verify_batch(O.f64(z_cpu), d_cpu[:, :B - 1].numpy())
        z = z_cpu.cuda()
        d = d_cpu.cuda() if B > 1 else None
        ref_a = torch.full((bs,), -1, dtype=torch.int32, device="cuda")
        ref_n = torch.full((bs,), -1, dtype=torch.int32, device="cuda")
        got_a = torch.full((bs,), -2, dtype=torch.int32, device="cuda")
        got_n = torch.full((bs,), -2, dtype=torch.int32, device="cuda")
        assert _allocating(lib, z, d, ref_a, ref_n) == 0
        assert _noalloc(lib, z, d, got_a, got_n) == 0
        torch.cuda.synchronize()
        np.testing.assert_array_equal(got_a.cpu().numpy(), ref_a.cpu().numpy())
        np.testing.assert_array_equal(got_n.cpu().numpy(), ref_n.cpu().numpy())
        np.testing.assert_array_equal(got_a.cpu().numpy(), ora_a)
        np.testing.assert_array_equal(got_n.cpu().numpy(), ora_n)
        np.testing.assert_array_equal(got_a.cpu().numpy(), planted.numpy())


def test_noalloc_verify_refuses_sizes_beyond_its_scratch():
    lib = load_library()
    t = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    # bs * B above the fixed capacity: refused on the host, nothing launched
    assert lib.dflash_verify_noalloc(t.data_ptr(), 1, t.data_ptr(), 257, 16, 10, t.data_ptr(), t.data_ptr(),
                                     stream) == 1
    assert lib.dflash_verify_noalloc(t.data_ptr(), 1, t.data_ptr(), 1025, 1, 10, t.data_ptr(), t.data_ptr(),
                                     stream) == 1
