"""dflash_verify against the oracle's verify: bit-exact accepted lengths and
next tokens on the same logits."""
import numpy as np
import pytest
import torch

from block_diffusion_speculative_cycle_b200 import dflash_verify_workspace_size, synth, verify
from oracle import dflash as O
from tests.golden_io import verify_cases

pytestmark = pytest.mark.gpu


def _check(z_cpu, d_cpu, ws=None):
    acc, nxt = verify(z_cpu.cuda(), d_cpu.cuda() if d_cpu.numel() else None, workspace=ws)
    torch.cuda.synchronize()
    ra, rn = O.verify_batch(O.f64(z_cpu), d_cpu.numpy())
    np.testing.assert_array_equal(acc.cpu().numpy(), ra)
    np.testing.assert_array_equal(nxt.cpu().numpy(), rn)
    return acc.cpu().numpy()


@pytest.mark.parametrize("case", verify_cases(), ids=lambda c: c[0])
def test_golden_cases(case):
    name, z, d, a, nxt = case
    zt = torch.from_numpy(z)[None].contiguous()
    dt = torch.from_numpy(d.astype(np.int32))[None].contiguous()
    acc, n = verify(zt.cuda(), dt.cuda() if dt.numel() else None)
    assert (int(acc[0]), int(n[0])) == (a, nxt)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("bs,B,V,mean", [(1, 16, 151936, 6.5), (4, 10, 128256, 3.25), (32, 16, 151936, 6.0),
                                         (3, 4, 1000, 1.5), (2, 1, 8193, 1.0), (5, 7, 16385, 2.0)])
def test_planted_prefixes(dtype, bs, B, V, mean):
    g = torch.Generator().manual_seed(bs * 100 + B)
    d = torch.randint(0, V, (bs, B - 1), generator=g, dtype=torch.int32)
    z, planted = synth.planted_logits(d, V, 2.0, mean, seed=bs + B + V, dtype=dtype)
    acc = _check(z, d)
    np.testing.assert_array_equal(acc, planted.numpy())


def test_ties_nan_and_signed_zero_rows():
    V = 9000
    z = torch.zeros((2, 3, V), dtype=torch.float32)
    z[0, 0, 7] = 5.0; z[0, 0, 8500] = 5.0            # tie across chunks -> 7
    z[0, 1, :] = float("nan"); z[0, 1, 4000] = -float("inf")
    z[0, 2, :] = -0.0; z[0, 2, 3] = 0.0              # all zeros -> 0
    z[1] = float("nan")                               # all NaN rows -> 0
    d = torch.tensor([[7, 4000], [0, 0]], dtype=torch.int32)
    acc = _check(z, d)
    assert list(acc) == [2, 2]


def test_workspace_is_left_clean_for_the_next_call():
    bs, B, V = 8, 16, 4096
    ws = torch.zeros(dflash_verify_workspace_size(bs, B), dtype=torch.uint8, device="cuda")
    for seed in range(3):
        g = torch.Generator().manual_seed(seed)
        d = torch.randint(0, V, (bs, B - 1), generator=g, dtype=torch.int32)
        z, planted = synth.planted_logits(d, V, 1.0, 5.0, seed=seed, dtype=torch.bfloat16)
        np.testing.assert_array_equal(_check(z, d, ws), planted.numpy())
    torch.cuda.synchronize()
    assert int(ws.count_nonzero()) == 0
