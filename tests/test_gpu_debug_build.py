"""The bounds-checked debug build (libsegquant_debug.so, SQ_DEBUG_BOUNDS): every
plain global store of every kernel tests its index against its buffer's
logical extent first, and records SQ_ERR_DEVICE_BOUNDS for one it skips.

A child process loads the debug build (SQ_LIBRARY) and runs the parity,
fuzz, split-tail, W4A8, single-scale, FP8 and host-pipeline suites with it:
every case must give the oracle's results and leave the error word clear
(tests/conftest.py checks the word after each GPU test under the debug
build), and the bounds probe must be caught.  The full-size configurations
are left to the release build (the debug build computes the same results,
only slower to compile)."""
import os
import re
import subprocess
import sys

import pytest

from w8a8_gemm_b200 import binding as B
from w8a8_gemm_b200 import build as sqbuild

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


def test_release_build_has_no_checks_and_refuses_the_probe():
    import torch
    assert not B.sq_debug_bounds_checks()
    buf = torch.zeros(9, dtype=torch.int32, device="cuda")
    with pytest.raises(B.SegQuantError) as e:
        B.sq_debug_bounds_probe(buf, 8)
    assert e.value.code == B.SQ_ERR_UNSUPPORTED
    assert int(buf.sum()) == 0


def test_suites_pass_under_the_debug_build():
    lib = sqbuild.build(debug=True)
    env = dict(os.environ, SQ_LIBRARY=lib)
    files = ["debug_build_cases.py", "test_gpu_parity.py", "test_gpu_fuzz.py",
             "test_gpu_split_tail.py", "test_gpu_w4.py", "test_gpu_single_scale.py",
             "test_gpu_fp8.py", "test_gpu_host.py", "test_gpu_quantize_plan.py"]
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
           "-k", "not full_size and not ffn_workload",
           *[os.path.join(HERE, f) for f in files]]
    r = subprocess.run(cmd, env=env, cwd=os.path.dirname(HERE), capture_output=True, text=True,
                       timeout=1200)
    tail = (r.stdout + r.stderr)[-3000:]
    assert r.returncode == 0, tail
    m = re.search(r"(\d+) passed", r.stdout)
    assert m and " failed" not in r.stdout and " skipped" not in r.stdout, tail
    assert int(m.group(1)) >= 80, tail   # the suites above, not a stray subset
