"""Collects the error figures of every parity check in a test session.

Each check in ``parity_util`` appends ``(test id, {figure: value})``; the
conftest attaches them to the test report (``record_property``), prints the
worst of each figure at the end of the session, and writes them all as JSON
lines to the file named by the ``FA_PARITY_REPORT`` environment variable when
it is set.  No dependencies, so that the CPU-only session can import it.
"""
from __future__ import annotations

import os

RECORDS: list = []


def current_test() -> str:
    return os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]


def record(figures: dict) -> None:
    RECORDS.append((current_test(), dict(figures)))


# Figures where larger is worse and that are worth a line in the summary.
SUMMARY_KEYS = ("o_max_below", "o_excess_above", "o_max", "o_rel_l2", "lse_max",
                "dq_max_below", "dk_max_below", "dv_max_below",
                "dq_excess_above", "dk_excess_above", "dv_excess_above",
                "dq_max", "dk_max", "dv_max", "dbias_max_below", "dbias_excess_above")


def worst() -> dict:
    """{figure: (value, test id)} over all records, for SUMMARY_KEYS."""
    out = {}
    for test, figs in RECORDS:
        for key in SUMMARY_KEYS:
            val = figs.get(key)
            if val is None:
                continue
            if key not in out or val > out[key][0]:
                out[key] = (val, test)
    return out
