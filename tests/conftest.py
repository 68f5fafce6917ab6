import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


@pytest.fixture(scope="session")
def cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def pytest_terminal_summary(terminalreporter):
    """One line per forward parity case: the raw max abs error of O (all elements,
    and those with |O_ref| < 4, where the bound applies raw), the mean, the LSE."""
    try:
        from helpers import FWD_STATS, GRAD_STATS
    except Exception:
        return
    tr = terminalreporter
    if GRAD_STATS:
        tr.write_line("backward parity (relative L2 errors):")
        for name, errs in GRAD_STATS:
            tr.write_line(f"  {name}: " + ", ".join(f"{k} {v:.2e}" for k, v in errs.items()))
    if not FWD_STATS:
        return
    tr.write_line("forward parity (raw o_max | o_max where |O_ref|<4 | excess | n(|O_ref|>=4) | o_mean | lse_max):")
    for name, st in FWD_STATS:
        tr.write_line(f"  {name}: {st['o_max']:.2e} | {st['o_max_below4']:.2e} | {st['o_max_excess']:.2e} | "
                      f"{st['n_big']} | {st['o_mean']:.1e} | {st['lse_max']:.1e}")
