"""The bounds-checked build of the library (librq_bounds.so, compiled with
-DRQ_BOUNDS_CHECK).  In that build every kernel tests each index it computes
at run time -- the tile's rows and scale bytes against the call's arrays, the
stage offsets against shared memory, the heads, query rows, records, tail
tokens and page-table entries of the finishing step, the encoders'
destination and source rows -- before the access, raises a status bit
(decode: workspace bit 128; encoders and reconstruction: encoder bit 8) when
a test fails and skips the access.  Nothing traps.

Every entry point runs on tiny and edge shapes (tests/bounds_workload.py) in
a subprocess with the bounds-checked library and again with the normal one:
every status word must be 0, and the results of the two builds must agree
(codes and scales bit for bit; decode and reconstruction outputs too, since
the checks change no arithmetic).
"""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def _run(lib, out):
    env = dict(os.environ, RQ_LIBRARY=lib)
    r = subprocess.run([sys.executable, os.path.join(HERE, "bounds_workload.py"), out], env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    return torch.load(out)


def _same(a, b, path):
    if isinstance(a, (tuple, list)):
        assert len(a) == len(b), path
        for i, (x, y) in enumerate(zip(a, b)):
            _same(x, y, f"{path}[{i}]")
        return
    assert a.shape == b.shape and a.dtype == b.dtype, path
    assert torch.equal(a.view(torch.uint8) if a.dtype != torch.float32 else a,
                       b.view(torch.uint8) if b.dtype != torch.float32 else b) or \
        torch.allclose(a, b, rtol=0, atol=0, equal_nan=True), path


def test_bounds_checked_build_is_clean_and_matches(tmp_path):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kv_cache_residual_rq_b200 import build
    lib_b = build.build(bounds=True)
    lib_n = build.build()
    got = _run(lib_b, str(tmp_path / "bounds.pt"))
    want = _run(lib_n, str(tmp_path / "normal.pt"))
    assert got["lib"].endswith("librq_bounds.so") and want["lib"].endswith("librq.so")
    assert len(got["status"]) > 60
    bad = {k: v for k, v in got["status"].items() if v}
    assert not bad, f"status words raised in the bounds-checked build: {bad}"
    assert not any(want["status"].values())
    assert got["res"].keys() == want["res"].keys()
    for k in want["res"]:
        _same(got["res"][k], want["res"][k], k)
