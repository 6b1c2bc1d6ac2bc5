"""The permute (step 4) on its own, bitwise: xr[pos[t, j]] = x[tb + t] for every
kept slot, nothing else written.  Rows of 1 KiB to 64 KiB (bf16 and fp32; the
kernel copies them in 16-byte vectors, one token per CTA at these sizes), with
dropped slots and tokens that keep none, over a token range that does not start
at 0.
"""
import numpy as np
import pytest
import torch

from combine_moe_route_12_b200 import moe

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("H,dtype", [(512, "bf16"), (1024, "bf16"), (2048, "bf16"), (7168, "bf16"),
                                     (16384, "bf16"), (512, "f32"), (4096, "f32"), (16384, "f32")])
def test_permute_rows_bitwise(H, dtype):
    T, k, tb, tc = 600, 8, 88, 512
    rng = np.random.default_rng(H + (1 if dtype == "f32" else 0))
    # pos: a permutation of the kept slots onto receive rows; ~1/5 of the slots dropped,
    # and every slot of tokens 0..15 of the range
    keep = rng.random((tc, k)) > 0.2
    keep[:16] = False
    n = int(keep.sum())
    pos = np.full((tc, k), -1, np.int32)
    pos[keep] = rng.permutation(n).astype(np.int32)
    cfg = moe.make_config(T, H, 16, k, 64, 2, -1, dtype)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    x = torch.randn(T, H, device="cuda").to(tdt)
    xr = torch.full((n + 4, H), float("nan"), device="cuda", dtype=tdt)
    moe.moe_permute(cfg, x, torch.from_numpy(pos).cuda(), tb, tc, xr)
    torch.cuda.synchronize()
    tt, jj = np.nonzero(keep)
    want = x[torch.from_numpy(tb + tt).cuda()]
    got = xr[torch.from_numpy(pos[tt, jj].astype(np.int64)).cuda()]
    assert torch.equal(got.view(torch.int16 if dtype == "bf16" else torch.int32),
                       want.view(torch.int16 if dtype == "bf16" else torch.int32))
    assert torch.isnan(xr[n:]).all()   # rows past the kept ones untouched
