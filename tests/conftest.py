import os
import sys
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]
if str(ROOT) not in sys.path:
    sys.path.insert(0, str(ROOT))

GOLDEN = Path(__file__).resolve().parent / "golden"


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: longer CPU test")


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle
    return oracle.load()


@pytest.fixture(scope="session")
def golden_dir():
    return GOLDEN


def read_golden(name: str):
    """Data lines of a golden fixture (comment lines start with '#')."""
    rows = []
    for line in (GOLDEN / name).read_text(encoding="utf-8").splitlines():
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        rows.append(line.split())
    return rows


@pytest.fixture(scope="session")
def pa_lib():
    """The product C-ABI library (built in-tree on first use)."""
    from paged_kv_cache_444_b200 import _lib
    return _lib.load()


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU test collected but no CUDA device is visible")
    return torch.device("cuda", 0)


def pytest_terminal_summary(terminalreporter):
    """Print the full-size parity errors the GPU tests recorded."""
    try:
        from parity_helpers import PARITY_REPORT
    except Exception:
        return
    if not PARITY_REPORT:
        return
    tr = terminalreporter
    tr.section("full-size parity: max-abs error vs the fp64 oracle")
    tr.write_line(f"{'workload':<22}{'kernel':<28}{'vs oracle':>12}{'vs rounded':>12}{'tol':>9}")
    for r in PARITY_REPORT:
        tr.write_line(f"{r['workload']:<22}{r['kernel']:<28}{r['max_abs_vs_oracle']:>12.3e}"
                      f"{r['max_abs_vs_rounded_oracle']:>12.3e}{r['tolerance']:>9.0e}")
