import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workloads (minutes)")


def pytest_collection_modifyitems(config, items):
    # GPU tests cannot run without a device; CPU runs select -m "not gpu".
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


_PARITY = {}


@pytest.fixture(scope="session")
def parity_report():
    """Worst parity errors per workload, printed in the session summary."""
    return _PARITY


def pytest_terminal_summary(terminalreporter):
    if not _PARITY:
        return
    tr = terminalreporter
    tr.write_sep("-", "parity against the float64 oracle (every query token)")
    for name, r in _PARITY.items():
        tr.write_line(f"{name}: {r['tokens']} tokens, max|o-o_ref| {r['o_max']:.3e}, "
                      f"max beyond bf16 rounding {r['o_max_beyond_rounding']:.3e}, rel-L2 {r['o_rel_l2']:.3e}, "
                      f"max|lse-lse_ref| {r['lse']:.3e} (oracle {r['oracle_s']:.0f} s on {r['threads']} threads)")
