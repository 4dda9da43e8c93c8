"""CPU replay of the tensor-core merge kernel's addresses (no GPU).

tests/replay/merge_tc_replay.cpp walks the loops of merge_tc.cu with the
same layout functions the kernel uses (merge_tc_layout.h) and checks every
shared-memory, tensor-memory and global access for bounds and alignment,
that the swizzled operand layouts are one-to-one and are the layouts the
tensor-core descriptors read, and that the layout fits the shared memory the
launch requests. A planted overrun (a region believed 4 bytes shorter than
the kernel uses) must make it fail: the class of error that a 16-byte
reserve holding a fifth 4-byte word is.
"""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "replay", "merge_tc_replay.cpp")
CSRC = os.path.join(ROOT, "gated_delta_rule_104_b200", "csrc")


@pytest.fixture(scope="module")
def replay(tmp_path_factory):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ not available")
    exe = str(tmp_path_factory.mktemp("replay") / "merge_tc_replay")
    subprocess.run([gxx, "-std=c++17", "-O1", "-Wall", "-Werror", f"-I{CSRC}", "-o", exe, SRC], check=True)
    return exe


def run(exe, *args):
    return subprocess.run([exe, *args], capture_output=True, text=True, timeout=120)


def test_every_access_in_bounds_and_aligned(replay):
    r = run(replay)
    assert r.returncode == 0, r.stdout[-3000:]
    assert "384 cases, 0 failures" in r.stdout


@pytest.mark.parametrize("region", ["sc", "kh", "ff", "raw_k", "raw_v", "raw_q", "red", "qf", "gam", "tile", "scl"])
def test_a_planted_four_byte_overrun_is_caught(replay, region):
    r = run(replay, "shrink", region, "4")
    assert r.returncode == 1, r.stdout[-2000:]
    assert "out of region" in r.stdout
