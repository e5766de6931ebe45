import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size parity cases")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle

    oracle.build()
    return oracle


def pytest_terminal_summary(terminalreporter):
    """Totals of the parity checks run in this session: how many O elements
    were judged by the half-ulp term of the bound and how many lse rows fell
    under the relative-error floor (see tests/helpers.py)."""
    try:
        import helpers
    except Exception:
        return
    s = helpers.STATS
    if not s["compares"]:
        return
    terminalreporter.write_line(
        f"parity totals: {s['compares']} compares, {s['o_elems']} O elements (max err {s['o_max_err']:.3e}); "
        f"{s['o_widened']} judged by the half-ulp term (max err {s['o_widened_max_err']:.3e}, "
        f"max excess over TOL_O {s['o_widened_max_excess']:.3e}); {s['lse_rows']} lse rows "
        f"(max rel {s['lse_max_rel']:.3e}), {s['lse_floor_rows']} under the floor "
        f"(max abs err {s['lse_floor_max_abs']:.3e})")
