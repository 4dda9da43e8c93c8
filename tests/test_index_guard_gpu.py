"""The index-guard debug build on the GPU.

libdeltalog_guard.so is the library compiled with DL_INDEX_GUARD: every
shared-memory write of the kernels (stores and cp.async destinations) checks
that it lies inside the block's shared memory and is aligned, and a write
that fails is skipped and reported in bit 1 of the fault word. This test
runs the parity suites of the merge kernels (warp-MMA and tcgen05), the
read (both forms), the pool step and the int8 base in a child process with that library
loaded; every case must still match the fp64 oracle, and after each one the
guard must report nothing.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SUITES = ["test_parity_gpu.py", "test_merge_tc_gpu.py", "test_pool_gpu.py", "test_i8_gpu.py", "test_fused_read_gpu.py"]


def test_parity_suites_pass_under_the_index_guard():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gated_delta_rule_104_b200 import build

    lib = build.build(guard=True)
    env = dict(os.environ, DELTALOG_LIBRARY=lib, DL_EXPECT_INDEX_GUARD="1")
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
           *[os.path.join(HERE, s) for s in SUITES]]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1500)
    assert r.returncode == 0, (r.stdout + r.stderr)[-4000:]
    assert " passed" in r.stdout
