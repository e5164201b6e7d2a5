import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: CPU test that takes more than a few seconds")


@pytest.fixture(scope="session")
def ref_oracle():
    import oracle
    return oracle.default()


def pytest_terminal_summary(terminalreporter):
    """One line per test module: outputs compared against the oracle, how many fall outside
    the pass rule (one BF16 ulp + 1e-3) and how many outside the strict 2^-8 |ref| + 1e-3 form
    (reported, not enforced)."""
    from tolerance import RECORD
    if not RECORD:
        return
    agg = {}
    for mod, n, fail, strict in RECORD:
        a = agg.setdefault(mod, [0, 0, 0, 0])
        a[0] += 1
        a[1] += n
        a[2] += fail
        a[3] += strict
    terminalreporter.write_sep("-", "parity against the oracle")
    for mod, (calls, n, fail, strict) in sorted(agg.items()):
        terminalreporter.write_line(f"{mod}: {calls} comparisons, {n} outputs, {fail} outside 1 ulp + 1e-3, "
                                    f"{strict} outside 2^-8 |ref| + 1e-3 ({100.0 * strict / max(n, 1):.4f} %)")
