"""Device rounding routines against the oracle, over every fp32 bit pattern.

kvq_round_e2m1 converts through the routine every quantiser of the library
uses (eight values per call, in pairs: even positions through the
low-nibble operand, odd ones through the high-nibble operand).  Each chunk is
converted twice, the second time shifted by one element, so that every bit
pattern goes through both operand positions."""
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
        if fmt == "e2m1":
            shifted = dev_fn(torch.cat([torch.zeros(1, dtype=x.dtype, device=x.device), x]))[1:].cpu().numpy()
            ok &= (shifted == want) | np.isnan(xh)
        if not ok.all():
            i = np.flatnonzero(~ok)[0]
            pytest.fail(f"{fmt}: input bits 0x{xh.view(np.uint32)[i]:08x} ({xh[i]!r}) device {got[i]} oracle {want[i]}")
        bad += (~ok).sum()
    assert bad == 0
