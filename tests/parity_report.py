"""Per-output error records of the GPU parity tests, printed at the end of a
pytest run (see conftest.py), so that a passing run still shows how close
each output came to its bound."""
from __future__ import annotations

RECORDS: list[dict] = []


def record(test: str, output: str, max_abs: float, bound: str, worst_excess: float,
           max_ref: float) -> None:
    RECORDS.append(dict(test=test, output=output, max_abs=max_abs, bound=bound,
                        worst_excess=worst_excess, max_ref=max_ref))


def lines() -> list[str]:
    out = []
    for r in RECORDS:
        out.append(f"{r['test']:<44s} {r['output']:<7s} max|err| {r['max_abs']:.3e}  "
                   f"max|ref| {r['max_ref']:.3e}  bound {r['bound']:<22s} "
                   f"worst(err - bound) {r['worst_excess']:+.3e}")
    return out
