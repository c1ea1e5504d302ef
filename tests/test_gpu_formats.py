"""Device rounding routines against the oracle, over every fp32 bit pattern."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt", ["e2m1", "e4m3"])
def test_device_rounding_exhaustive(kvq, fmt):
    dev_fn = kvq.round_e2m1 if fmt == "e2m1" else kvq.round_e4m3
    ref_fn = oracle.e2m1_encode if fmt == "e2m1" else oracle.e4m3_encode
    chunk = 1 << 28
    bad = 0
    for start in range(0, 1 << 32, chunk):
        bits = (torch.arange(start, start + chunk, dtype=torch.int64, device="cuda") - (1 << 31)).to(torch.int32)
        bits = bits ^ torch.tensor(-(1 << 31), dtype=torch.int32, device="cuda")   # back to start..start+chunk
        x = bits.view(torch.float32)
        got = dev_fn(x).cpu().numpy()
        xh = x.cpu().numpy()
        want = ref_fn(xh)
        ok = (got == want) | np.isnan(xh)
        if not ok.all():
            i = np.flatnonzero(~ok)[0]
            pytest.fail(f"{fmt}: input bits 0x{xh.view(np.uint32)[i]:08x} ({xh[i]!r}) device {got[i]} oracle {want[i]}")
        bad += (~ok).sum()
    assert bad == 0
