import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a CUDA device (B200, sm_100a) and the built library")
    config.addinivalue_line(
        "markers", "slow: oracle work of tens of seconds or more")


def pytest_collection_modifyitems(config, items):
    # Tests needing a GPU are skipped, not failed, where none is present.
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(autouse=True)
def _parity_figures(record_property):
    """Attach the error figures of the test's parity checks to its report."""
    import parity_log
    start = len(parity_log.RECORDS)
    yield
    for i, (_, figs) in enumerate(parity_log.RECORDS[start:]):
        for key, val in figs.items():
            record_property(f"check{i}.{key}", val)


def pytest_terminal_summary(terminalreporter):
    import json
    import parity_log
    if not parity_log.RECORDS:
        return
    worst = parity_log.worst()
    terminalreporter.write_line(
        f"parity: {len(parity_log.RECORDS)} checks; worst figures (bounds: O max-abs 1e-2 "
        "and rel-L2 5e-3, dQ/dK/dV max-abs 2e-2, LSE 1e-3; '_below' = raw error where "
        "the bound applies raw, '_excess_above' = beyond the bf16 floor elsewhere):")
    for key, (val, test) in worst.items():
        terminalreporter.write_line(f"  {key} = {val:.4g}  ({test})")
    path = os.environ.get("FA_PARITY_REPORT")
    if path:
        with open(path, "w") as f:
            for test, figs in parity_log.RECORDS:
                f.write(json.dumps({"test": test, **figs}) + "\n")
