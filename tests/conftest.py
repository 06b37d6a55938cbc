import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HERE = os.path.dirname(os.path.abspath(__file__))
for p in (ROOT, HERE):
    if p not in sys.path:
        sys.path.insert(0, p)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def lib():
    """The CUDA library through its Python binding; fails loudly if it is not built."""
    import hadamard_butterfly_rotation_b200 as hbr
    return hbr


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Report every rounding-boundary exclusion the code parity checks made: codes (and whole
    groups, for scales near a binary16 midpoint) whose oracle decision lies within 1e-5 of a
    rounding boundary are not compared; this lists how many, per check."""
    try:
        from parity import EXCLUSIONS
    except Exception:
        return
    if not EXCLUSIONS:
        return
    tr = terminalreporter
    tr.section("rounding-boundary exclusions (codes / groups not compared)")
    tot_c = tot_g = all_c = all_g = 0
    for test, what, c, g, nc, ng in EXCLUSIONS:
        tr.write_line(f"{test} [{what}]: {c} of {nc} codes, {g} of {ng} groups")
        tot_c, tot_g, all_c, all_g = tot_c + c, tot_g + g, all_c + nc, all_g + ng
    tr.write_line(f"total: {tot_c} of {all_c} codes ({tot_c / max(all_c, 1):.2e}), "
                  f"{tot_g} of {all_g} groups ({tot_g / max(all_g, 1):.2e}) excluded in {len(EXCLUSIONS)} checks")
