import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_collection_modifyitems(config, items):
    import torch
    if torch.cuda.is_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def pytest_terminal_summary(terminalreporter):
    """Near-tie report of the parity tests: per configuration, the query rows checked, the rows
    whose GPU selection differs from the oracle's exact set (every difference inside the
    near-tie band), the swapped pairs, and the rows where the band's near-zero floor decided."""
    try:
        from tests.dsa_cases import NEAR_TIE_REPORT
    except Exception:
        return
    if not NEAR_TIE_REPORT:
        return
    terminalreporter.write_sep("-", "near-tie report (selection parity)")
    terminalreporter.write_line(f"{'configuration':<28} {'rows':>8} {'rows with swaps':>16} {'pairs':>8} "
                                f"{'floor used':>11}")
    for name, (rows, swapped_rows, pairs, floor) in sorted(NEAR_TIE_REPORT.items()):
        terminalreporter.write_line(f"{name:<28} {rows:>8} {swapped_rows:>16} {pairs:>8} {floor:>11}")
