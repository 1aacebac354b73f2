import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built library")
    config.addinivalue_line("markers", "slow: long-running parity case")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


def pytest_terminal_summary(terminalreporter):
    """How many bf16 elements needed the rounding term of the bound (more than
    the flat max-abs tolerance) over all element-wise checks of the run."""
    try:
        from helpers import ULP_ADMITTED
    except ImportError:
        return
    if not ULP_ADMITTED:
        return
    total = sum(n for _, _, n in ULP_ADMITTED)
    adm = [(w, a, n) for w, a, n in ULP_ADMITTED if a]
    terminalreporter.write_line(
        f"bf16 parity: {len(ULP_ADMITTED)} element-wise checks, {total} elements; "
        f"{sum(a for _, a, _ in adm)} above the flat 2e-2 (admitted by the half-ulp term) in {len(adm)} checks"
        + ("".join(f"; {w}: {a}/{n}" for w, a, n in adm[:8])))
