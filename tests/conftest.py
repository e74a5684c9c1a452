import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle
    oracle.build()
    return oracle


def _margins_summary(tr):
    """Observed parity margins of the o comparisons against the oracle: per
    test, the largest |o_gpu - o_ref| and how many elements with |o_ref| < 2.56
    (where bf16 output rounding stays under 1e-2) exceed the literal 1e-2."""
    from tests.helpers import MARGINS
    if not MARGINS:
        return
    per = {}
    for test, _what, mx, over, small in MARGINS:
        m = per.setdefault(test, [0.0, 0, 0, 0])
        m[0] = max(m[0], mx)
        m[1] += over
        m[2] += small
        m[3] += 1
    tr.section("parity margins of o against the oracle")
    tr.write_line(f"{'max |do|':>10} {'>1e-2 @|o|<2.56':>16} {'of':>10} {'checks':>7}  test")
    for test, (mx, over, small, n) in sorted(per.items()):
        tr.write_line(f"{mx:10.3e} {over:16d} {small:10d} {n:7d}  {test}")
    tot_over = sum(v[1] for v in per.values())
    tot_small = sum(v[2] for v in per.values())
    tr.write_line(f"overall: max |do| {max(v[0] for v in per.values()):.3e}; elements with |o_ref| < 2.56 over "
                  f"the literal 1e-2: {tot_over} of {tot_small}")


def _ulp_summary(tr):
    """Projection outputs against the oracle, counted in bf16 steps."""
    import sys
    mod = sys.modules.get("tests.test_gpu_qkv")
    counts = getattr(mod, "ULP_COUNTS", None) if mod else None
    if not counts:
        return
    tr.section("projection outputs against the oracle, in bf16 steps")
    agg = {}
    for what, n, e0, e1, e2, mx in counts:
        a = agg.setdefault(what, [0, 0, 0, 0, 0])
        a[0] += n
        a[1] += e0
        a[2] += e1
        a[3] += e2
        a[4] = max(a[4], mx)
    for what, (n, e0, e1, e2, mx) in sorted(agg.items()):
        tr.write_line(f"{what:>8}: {n} values, identical {e0 / n:.5f}, one step {e1 / n:.5f}, "
                      f"more {e2 / n:.5f} (max {mx} steps)")


def pytest_terminal_summary(terminalreporter):
    _margins_summary(terminalreporter)
    _ulp_summary(terminalreporter)
