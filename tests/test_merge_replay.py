"""CPU replay of the addresses of the warp-MMA merge, the replay-prep kernel
and the fused append-read kernel (no GPU).

tests/replay/merge_replay.cpp walks the loops of merge.cu (the compact pool
walk included), of replay_prep and of append_read_fused in deferred_read.cu
(ReplayPrep from prep.cuh) with the layout functions the kernels themselves
use (merge_layout.h, prep_layout.h, fused_layout.h), for
every instantiation and a grid of log fills, and checks every shared-memory
access for bounds and alignment, that the regions do not overlap and fit the
shared memory the launch requests, and that the swizzles are one-to-one. A
region believed a few bytes shorter than the kernels use (past any row
padding they never touch) must make it fail; the first case is the class of
overrun once found by hand: the pool walk's fifth word beyond a 16-byte
reserve.
"""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "replay", "merge_replay.cpp")
CSRC = os.path.join(ROOT, "gated_delta_rule_104_b200", "csrc")


@pytest.fixture(scope="module")
def replay(tmp_path_factory):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ not available")
    exe = str(tmp_path_factory.mktemp("replay") / "merge_replay")
    subprocess.run([gxx, "-std=c++17", "-O2", "-Wall", "-Werror", f"-I{CSRC}", "-o", exe, SRC], check=True)
    return exe


def run(exe, *args):
    return subprocess.run([exe, *args], capture_output=True, text=True, timeout=300)


def test_every_access_in_bounds_and_aligned(replay):
    r = run(replay)
    assert r.returncode == 0, r.stdout[-3000:]
    assert r.stdout.strip().endswith("cases, 0 failures")


# (region, bytes): 4 bytes past the end of what the kernels touch; the strided
# float arrays carry row padding they never read (sx, sxw, sv: 4 floats; ff: 8)
PLANTS = [("xw", 16), ("tile", 4), ("kh", 4), ("ff", 36), ("fa", 4), ("gn", 4), ("sq", 4), ("sx", 20),
          ("sb", 4), ("sv", 20), ("sxw", 20), ("scl", 4), ("wsc", 4),
          ("w0.sk", 4), ("w0.sa", 4), ("w0.as", 4), ("w0.beta", 4), ("w0.d", 4), ("w0.cn", 4), ("w0.s", 4),
          ("w3.xrow", 4)]


@pytest.mark.parametrize("region,nbytes", PLANTS)
def test_a_planted_overrun_is_caught(replay, region, nbytes):
    r = run(replay, "prep" if "." in region else "merge", "shrink", region, str(nbytes))
    assert r.returncode == 1, r.stdout[-2000:]
    assert "out of region" in r.stdout


# the fused kernel: the last float of a slot (w's last row), the last 16 bytes
# of a base buffer, a prep warp's X rows, and a base one row short per head
FUSED_PLANTS = [("slot3", 4), ("ring7.2", 4), ("w5.xrow", 4), ("w0.sk", 4), ("unit", 0)]


@pytest.mark.parametrize("region,nbytes", FUSED_PLANTS)
def test_a_planted_overrun_in_the_fused_read_is_caught(replay, region, nbytes):
    r = run(replay, "fused", "shrink", region, str(nbytes))
    assert r.returncode == 1, r.stdout[-2000:]
    assert "out of region" in r.stdout
