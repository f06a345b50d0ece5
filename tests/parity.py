"""Parity bar shared by the tests: bf16 attention output, converted to fp32,
against the fp64 oracle: max |err| <= 2e-2 and mean |err| <= 2e-3.

Every comparison is recorded (case name, rows compared, max / mean absolute
and max relative error); tests/conftest.py prints the records at the end of
the session, so a quiet run still shows how far each case is from the bar."""
import numpy as np

MAX_ABS = 2e-2
MEAN_ABS = 2e-3

RECORDS = []


def errors(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    d = np.abs(got - want)
    rel = d / np.maximum(np.abs(want), 1e-3)
    return {"max_abs": float(d.max()) if d.size else 0.0,
            "mean_abs": float(d.mean()) if d.size else 0.0,
            "max_rel": float(rel.max()) if rel.size else 0.0,
            "nan": int(np.isnan(got).sum())}


def within(got, want) -> bool:
    e = errors(got, want)
    return e["nan"] == 0 and e["max_abs"] <= MAX_ABS and e["mean_abs"] <= MEAN_ABS


def assert_parity(got, want, what=""):
    e = errors(got, want)
    RECORDS.append((what, int(np.asarray(want).size), e))
    assert e["nan"] == 0 and e["max_abs"] <= MAX_ABS and e["mean_abs"] <= MEAN_ABS, f"{what}: {e}"
    return e
