import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload checks")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle

    oracle.build()
    return oracle


@pytest.fixture(autouse=True)
def _index_guard_clean(request):
    """Under DL_EXPECT_INDEX_GUARD=1 (the child run of test_index_guard_gpu.py,
    with the index-guard library loaded): after each GPU test, no kernel may
    have skipped an out-of-bounds shared-memory write (bit 1 of the fault
    word)."""
    yield
    if os.environ.get("DL_EXPECT_INDEX_GUARD") != "1" or request.node.get_closest_marker("gpu") is None:
        return
    import gated_delta_rule_104_b200 as g

    assert g.dl_index_guard_build(), "the index-guard library is not the one loaded"
    flags = g.dl_device_faults(clear=True)
    assert not (flags & 2), "index guard: " + g.load().dl_last_error().decode()
