"""Record of every floating-point parity comparison made in a test session: what was compared, the
measured max |gpu - ref| and relative L2 error, and the bounds they were held to.  The session's
terminal summary prints it (tests/conftest.py), so the size of the real errors is on record next to
the tolerances."""
from __future__ import annotations

RESULTS: list[tuple[str, float, float, float, float]] = []


def record(what: str, max_abs: float, rel_l2: float, bound_abs: float, bound_rel: float) -> None:
    RESULTS.append((what, float(max_abs), float(rel_l2), float(bound_abs), float(bound_rel)))
