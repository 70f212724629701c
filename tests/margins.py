"""Attention errors the GPU parity tests measured, printed at the end of the
run (conftest's terminal summary) so the margin to each tolerance is visible."""
from __future__ import annotations

MARGINS: list[tuple[str, float, float]] = []


def record(label: str, err: float, tol: float) -> None:
    MARGINS.append((label, float(err), float(tol)))


def summary_lines() -> list[str]:
    worst: dict[str, tuple[float, float]] = {}
    for label, err, tol in MARGINS:
        if label not in worst or err / tol > worst[label][0] / worst[label][1]:
            worst[label] = (err, tol)
    return [f"{label:<58s} {err:9.3e} of {tol:.0e}  ({100 * err / tol:5.1f}%)"
            for label, (err, tol) in sorted(worst.items())]
