import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs an NVIDIA B200 (sm_100a) GPU")


@pytest.fixture(scope="session")
def cuda_lib():
    """libhstu_attn.so, rebuilt first if any source is newer than it."""
    from hstu_pointwise_attention_jagged_b200 import build, binding
    build.build()
    return binding.load_library()


@pytest.fixture(scope="session")
def orc():
    import oracle
    return oracle.default()


def pytest_terminal_summary(terminalreporter):
    """One line per GPU parity comparison: global rel_l2, max_abs, and the worst user and row."""
    try:
        from gpu_util import PARITY_LOG
    except Exception:
        return
    if not PARITY_LOG:
        return
    tr = terminalreporter
    tr.section("parity (rel_l2 global / worst user / worst row, max_abs)")
    for r in PARITY_LOG:
        tr.write_line("%-40s rel %.2e  user %d %.2e  row %d %.2e  max_abs %.1e  (%d rows)" % (
            r["what"][:40], r["rel_l2"], r["worst_user"], r["worst_user_rel_l2"], r["worst_row"],
            r["worst_row_rel_l2"], r["max_abs"], r["rows"]))
