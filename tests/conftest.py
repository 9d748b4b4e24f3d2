import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU case")


def pytest_terminal_summary(terminalreporter):
    """Worst error / gate ratio per compared quantity of the parity tests that ran; also
    written as JSON to $MAO_GATE_REPORT when that variable names a file."""
    from tests import gates
    worst = gates.summary()
    if not worst:
        return
    tr = terminalreporter
    tr.write_line("parity gates (worst error / gate per quantity):")
    for q, (r, e, g, label) in sorted(worst.items()):
        tr.write_line(f"  {q:28s} {e:10.3e} / {g:10.3e} = {r:6.3f}   ({label})")
    path = os.environ.get("MAO_GATE_REPORT")
    if path:
        import json
        with open(path, "w") as f:
            json.dump({"worst": {q: {"ratio": r, "error": e, "gate": g, "case": label}
                                 for q, (r, e, g, label) in worst.items()},
                       "records": gates.RECORDS}, f)
