"""Register and local-memory budget of the hot kernels, from ptxas's resource report.

The decode is issue-bound at two 9-warp CTAs per SM: it must fit in 96
registers (16 K registers per SM sub-partition over its 5 warps, in units of
8) with no local-memory spill, or every page pays for spill traffic.  The
append, both prefills and the KLT key append must not spill either.  The
report is what `nvcc -Xptxas -v` prints; this test compiles the sources with
the library's own flags and reads it.
"""
import concurrent.futures
import importlib.util
import os
import re
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_spec = importlib.util.spec_from_file_location("kvq_build", os.path.join(ROOT, "bit_attention_decode_b200", "build.py"))
_build = importlib.util.module_from_spec(_spec)
_spec.loader.exec_module(_build)

SOURCES = ["kvq_decode_tc.cu", "kvq_quant.cu", "kvq_prefill_tc.cu", "kvq_prefill_fp4.cu", "kvq_klt.cu"]


def _nvcc():
    return _build.NVCC if os.path.exists(_build.NVCC) else shutil.which("nvcc")


def _report(src, out_dir):
    r = subprocess.run([_nvcc(), *_build.FLAGS, "-Xptxas", "-v", "-c", os.path.join(_build.CSRC, src),
                        "-o", os.path.join(out_dir, src + ".o")], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    entries, cur = {}, None
    for line in (r.stdout + r.stderr).splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            cur = m.group(1)
            entries[cur] = {}
            continue
        if cur is None:
            continue
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m:
            entries[cur]["spill"] = int(m.group(1)) + int(m.group(2))
        m = re.search(r"Used (\d+) registers", line)
        if m:
            entries[cur]["regs"] = int(m.group(1))
    return entries


@pytest.fixture(scope="module")
def resources():
    if _nvcc() is None:
        pytest.skip("nvcc not available")
    with tempfile.TemporaryDirectory() as d:
        with concurrent.futures.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
            reports = list(ex.map(lambda s: _report(s, d), SOURCES))
    out = {}
    for rep in reports:
        out.update(rep)
    return out


def _select(resources, *parts):
    hits = {k: v for k, v in resources.items() if all(p in k for p in parts)}
    assert hits, f"no entry matching {parts}"
    return hits


def test_decode_fits_two_ctas_per_sm_without_spills(resources):
    # packed-key instantiations: decode_tc_kernel<TQ, TO, false>
    for name, r in _select(resources, "decode_tc_kernel", "Lb0E").items():
        assert r["spill"] == 0, (name, r)
        assert r["regs"] <= 96, (name, r)


@pytest.mark.parametrize("kernel", ["append_kernel", "prefill_tc", "prefill_fp4", "klt_append_keys_kernel"])
def test_hot_kernels_do_not_spill(resources, kernel):
    for name, r in _select(resources, kernel).items():
        assert r["spill"] == 0, (name, r)
