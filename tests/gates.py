"""Records every (error, gate) comparison a parity test makes, so that a run can
print how close each quantity came to its gate (and the assertion message of a
failure names both numbers)."""

from __future__ import annotations

import numpy as np

RECORDS = []  # (label, quantity, error, gate)


def rel(a, b) -> float:
    """Relative Frobenius error ||a - b|| / ||b||."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def max_over_rms(a, b) -> float:
    """Largest elementwise error, in units of the reference's root mean square."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    rms = float(np.sqrt(np.mean(b * b))) if b.size else 0.0
    return float(np.max(np.abs(a - b)) / max(rms, 1e-300)) if b.size else 0.0


def check(label: str, quantity: str, err: float, gate: float) -> None:
    RECORDS.append((label, quantity, float(err), float(gate)))
    assert err < gate, f"{label} {quantity}: error {err:.3e} >= gate {gate:.3e}"


def summary():
    """Per quantity: the worst error / gate ratio seen, with its error and gate."""
    worst = {}
    for label, q, e, g in RECORDS:
        r = e / g if g > 0 else float("inf")
        if q not in worst or r > worst[q][0]:
            worst[q] = (r, e, g, label)
    return worst
