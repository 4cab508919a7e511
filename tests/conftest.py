import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture
def golden_dir():
    return GOLDEN


def pytest_terminal_summary(terminalreporter):
    """Achieved output errors of the GPU parity tests (max-abs, RMS-relative) per test,
    the worst comparison of each; also written as JSON to $SLR_ERRORS_JSON when set."""
    mod = sys.modules.get("gpu_common")
    if mod is None or not getattr(mod, "ERRORS", None):
        return
    worst = {}
    for test, what, ma, rr in mod.ERRORS:
        w = worst.setdefault(test, [what, ma, rr, 0])
        w[1], w[2], w[3] = max(w[1], ma), max(w[2], rr), w[3] + 1
    terminalreporter.section("achieved output errors (tolerances: max-abs 2e-2, rms-rel 5e-3)")
    for test, (what, ma, rr, n) in sorted(worst.items()):
        terminalreporter.write_line(f"{test}: max-abs {ma:.2e}  rms-rel {rr:.2e}  ({n} comparisons)")
    path = os.environ.get("SLR_ERRORS_JSON")
    if path:
        import json
        with open(path, "w") as f:
            json.dump({t: {"max_abs": v[1], "rms_rel": v[2], "comparisons": v[3]} for t, v in worst.items()}, f,
                      indent=1)
