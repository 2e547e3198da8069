import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size cases (minutes of oracle time)")


@pytest.fixture(scope="session")
def orc():
    import oracle
    return oracle.get()


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Measured errors of every GPU parity comparison of the session (gpu_helpers.MARGINS)."""
    mod = sys.modules.get("gpu_helpers")
    rows = getattr(mod, "MARGINS", None) if mod else None
    if not rows:
        return
    tr = terminalreporter
    tr.section("parity margins (measured error against the fp64 oracle; 'of bound' = error / allowed)")
    tr.write_line(f"{'case':<58} {'dtype':<9} {'rows':>9} {'max|dout|':>11} {'of bound':>9} {'max|dlse|':>11} {'of bound':>9}")
    worst = {}
    for tag, dt, n, e, r, le, lr in rows:
        tr.write_line(f"{tag[:58]:<58} {dt:<9} {n:>9} {e:>11.3e} {r:>9.3f} {le:>11.3e} {lr:>9.3f}")
        w = worst.setdefault(dt, [0.0, 0.0])
        w[0], w[1] = max(w[0], r), max(w[1], lr)
    for dt, (r, lr) in sorted(worst.items()):
        tr.write_line(f"worst {dt}: out at {r:.3f} of its bound, lse at {lr:.3f} of its bound")
