import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


def read_golden(path):
    """key -> list of tokens, skipping comments; rows of tables come back under integer keys."""
    out, rows = {}, []
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            tok = line.split()
            if tok[0].lstrip("-").isdigit():
                rows.append(tok)
            else:
                out[tok[0]] = tok[1:]
    if rows:
        out["rows"] = rows
    return out


def pytest_terminal_summary(terminalreporter):
    """Code mismatches of every GPU parity comparison with the oracle (near-tie decisions and the
    trajectories that follow them), one line per comparison."""
    sup = sys.modules.get("gpu_support")
    notes = getattr(sup, "NOTES", None)
    if notes:
        terminalreporter.section("measured figures")
        for label, text in notes:
            terminalreporter.write_line(f"{label}: {text}")
    log = getattr(sup, "PARITY_LOG", None)
    if not log:
        return
    terminalreporter.section("code parity against the oracle")
    for label, st in log:
        terminalreporter.write_line(
            f"{label}: agree {st['agree']:.6f}, mismatched codes {st['mismatches']}"
            + (f", rows diverged {st['rows_diverged']}, max level diff {st['max_level_diff']}"
               if "rows_diverged" in st else "")
            + (f", E rel {st['E_rel']:.2e}" if "E_rel" in st else ""))
