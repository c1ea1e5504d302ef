"""Pins of the oracle's NVFP4 formats (E2M1 elements, E4M3 block scales)."""
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle
from conftest import ROOT, read_golden


def test_e2m1_grid_matches_golden():
    rows = read_golden("e2m1_grid.txt")
    assert len(rows) == 16
    for code, val in rows:
        got = oracle.e2m1_value(int(code))
        assert got == float(val)
        assert np.signbit(got) == val.startswith("-")


def test_e2m1_largest_is_six_and_grid_is_symmetric():
    vals = oracle.e2m1_value(np.arange(16))
    assert vals.max() == 6.0 and vals.min() == -6.0
    np.testing.assert_array_equal(vals[8:], -vals[:8])


def test_e4m3_grid_properties():
    vals = oracle.e4m3_value(np.arange(256))
    finite = vals[~np.isnan(vals)]
    assert np.isnan(vals[0x7F]) and np.isnan(vals[0xFF])
    assert finite.max() == 448.0                      # E4M3FN largest finite
    assert vals[1] == 2.0 ** -9                        # smallest subnormal
    assert vals[8] == 2.0 ** -6                        # smallest normal
    pos = vals[:0x7F]
    assert np.all(np.diff(pos) > 0)                    # codes ordered by value


def test_e4m3_encode_matches_torch_float8_cast():
    # library routine: torch's fp32 -> float8_e4m3fn cast rounds to nearest even;
    # compared inside the finite range, on every grid value, every midpoint and
    # random values.
    grid = oracle.e4m3_value(np.arange(0x7F))
    mids = (grid[:-1] + grid[1:]) / 2
    rng = np.random.default_rng(7)
    rand = np.exp(rng.uniform(np.log(2.0 ** -12), np.log(440.0), 200_000))
    x = np.concatenate([grid, mids, rand, -rand]).astype(np.float32)
    x = x[np.abs(x) < 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode(x)
    np.testing.assert_array_equal(got, ref)


def test_e4m3_encode_saturates():
    x = np.array([448.0, 455.9, 456.0, 1e6, np.inf], np.float32)
    assert np.all(oracle.e4m3_encode(x) == 0x7E)


def test_e2m1_encode_ties_and_saturation():
    x = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.5, 1e30, -0.0, -0.1, -5.0], np.float32)
    want = np.array([0, 2, 2, 4, 4, 6, 6, 7, 7, 8, 8, 14], np.uint8)
    np.testing.assert_array_equal(oracle.e2m1_encode(x), want)


def test_exhaustive_rounding_against_brute_force(tmp_path):
    """All 2^32 fp32 inputs: oracle rounding == independent nearest-value search."""
    exe = tmp_path / "brute"
    src = os.path.join(ROOT, "tests", "c", "brute_formats.c")
    subprocess.run(["gcc", "-O2", "-fopenmp", "-o", str(exe), src, "-ldl", "-lm"], check=True)
    out = subprocess.run([str(exe), oracle.build()], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "e2m1_mismatch 0" in out.stdout and "e4m3_mismatch 0" in out.stdout


def test_round_bf16_matches_torch_cast():
    # the oracle's bf16 rounding (keys of the mixed cache) against torch's
    # round-to-nearest-even cast, on random values and on exact ties
    import torch
    rng = np.random.default_rng(11)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 100000),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, -1.00390625, 3.0e38, 1e-40], np.float32)])
    # exact ties: the lower 16 bits are 0x8000, with an even and an odd kept part
    ties = (np.arange(1000, dtype=np.uint32) << 16 | 0x3F800000 | 0x8000).view(np.float32)
    x = np.concatenate([x, ties])
    want = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(oracle.round_bf16(x).view(np.uint32), want.view(np.uint32))
