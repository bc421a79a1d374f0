import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def pytest_terminal_summary(terminalreporter):
    """How many outputs the GPU parity checks accepted as rounding-boundary cases (the
    exact value within half an I/O ulp of the GPU's, yet more than the tolerance away from
    the oracle rounded to the I/O dtype), and how many on their distance to the exact
    value alone, per I/O dtype."""
    parity = sys.modules.get("parity")
    tally = getattr(parity, "BOUNDARY_TALLY", None)
    if not tally:
        return
    per = {}
    for io, n, total, exact in tally:
        a, b, c = per.get(io, (0, 0, 0))
        per[io] = (a + n, b + total, c + exact)
    terminalreporter.write_sep("-", "parity: rounding-boundary cases accepted")
    for io, (n, total, exact) in sorted(per.items()):
        terminalreporter.write_line(f"{io}: {n} of {total} outputs compared; {exact} more further than the "
                                    f"tolerance from the rounded oracle but within it of the exact value")
