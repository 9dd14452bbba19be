import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter):
    """The measured error of every GPU parity comparison against its bound."""
    try:
        from tests.gpu_helpers import MEASURED
    except Exception:   # the GPU helpers were not imported in this session
        return
    if not MEASURED:
        return
    tr = terminalreporter
    tr.write_sep("-", "parity errors (max-abs / relative Frobenius, against their bounds)")
    for m in MEASURED:
        tr.write_line("%-60s %.2e / %.2e   (bounds %.0e / %.0e, max |ref| %.2f)" % (
            m["what"][:60], m["max_abs"], m["rel_fro"], m["atol"], m["rtol"], m["max_abs_ref"]))
    path = os.environ.get("DBSA_PARITY_LOG")
    if path:
        import json
        with open(path, "w") as f:
            json.dump(MEASURED, f, indent=1)
