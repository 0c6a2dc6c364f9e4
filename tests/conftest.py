import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 and the built CUDA library")


def pytest_collection_modifyitems(config, items):
    # Keep the file whose tests must run last at the end of the session.
    items.sort(key=lambda it: os.path.basename(str(it.fspath)).startswith("test_zz_"))


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def pytest_terminal_summary(terminalreporter):
    # Output comparisons of the session with their margins, passing or not:
    # the error beyond the rounding of the result to its storage type and the
    # raw max-abs error (both over the reference's RMS; bound 2e-2 on the
    # first), and the relative Frobenius error (bound 5e-3).
    parity = sys.modules.get("parity")
    rows = getattr(parity, "MARGINS", None)
    if not rows:
        return
    tr = terminalreporter
    tr.section("output parity margins (largest first)")
    tr.write_line(f"{'comparison':60s} {'beyond-rounding/RMS':>20s} {'raw max-abs/RMS':>16s} "
                  f"{'rel. Frobenius':>15s} {'elements':>10s}")
    # the 40 largest, then every full-size workload
    shown = sorted(rows, key=lambda r: -r[1])[:40]
    shown += [r for r in rows if "full size" in r[0] and r not in shown]
    for what, excess, raw, frob, n in shown:
        tr.write_line(f"{what[:60]:60s} {excess:20.3e} {raw:16.3e} {frob:15.3e} {n:10d}")
    tr.write_line(f"{len(rows)} comparisons; worst beyond-rounding/RMS "
                  f"{max(r[1] for r in rows):.3e}, worst raw max-abs/RMS "
                  f"{max(r[2] for r in rows):.3e}, worst rel. Frobenius "
                  f"{max(r[3] for r in rows):.3e}")
