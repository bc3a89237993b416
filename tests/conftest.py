import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: CPU test that takes more than a few seconds")


@pytest.fixture(scope="session")
def root():
    return ROOT


def pytest_terminal_summary(terminalreporter):
    """Parity errors of every GPU-vs-oracle comparison that ran (worst per label)."""
    mod = sys.modules.get("tests.parity_helpers")
    rec = getattr(mod, "RECORD", None) if mod else None
    near = getattr(mod, "NEAR_TIES", None) if mod else None
    if near:
        tot = {}
        for what, rows, n in near:
            a, b = tot.get(what, (0, 0))
            tot[what] = (a + rows, b + n)
        tr = terminalreporter
        tr.section("selection near-ties (oracle relative score gap < 1e-5; left out of element-wise checks)")
        tr.write_line(f"{'selection comparison':60s} {'rows':>8s} {'near-tie':>9s}")
        for what, (rows, n) in sorted(tot.items()):
            tr.write_line(f"{what[:60]:60s} {rows:8d} {n:9d}")
        tr.write_line(f"{'total':60s} {sum(r for r, _ in tot.values()):8d} {sum(n for _, n in tot.values()):9d}")
    if not rec:
        return
    worst = {}
    for what, dtype, max_abs, rel in rec:
        key = (what, dtype)
        a, r = worst.get(key, (0.0, 0.0))
        worst[key] = (max(a, max_abs), max(r, rel))
    tr = terminalreporter
    tr.section("parity against the oracle (worst per comparison)")
    tr.write_line(f"{'comparison':60s} {'dtype':5s} {'max_abs':>10s} {'rel_l2':>10s}")
    for (what, dtype), (a, r) in sorted(worst.items()):
        tr.write_line(f"{what[:60]:60s} {dtype:5s} {a:10.3e} {r:10.3e}")
