import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload")


@pytest.fixture(scope="session")
def has_gpu():
    import torch
    return torch.cuda.is_available()


# Errors of every GPU-vs-oracle comparison of this session: (tensor, raw
# max-abs, max-abs beyond the bf16 rounding of the output, rel-L2).  The
# summary at the end of the run prints the largest of each per tensor name.
_ERRORS = []


def record_error(name, raw, beyond_rounding, rel_l2):
    _ERRORS.append((name, float(raw), float(beyond_rounding), float(rel_l2)))


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    if not _ERRORS:
        return
    worst = {}
    for name, raw, mx, rel in _ERRORS:
        n, r, m, l = worst.get(name, (0, 0.0, 0.0, 0.0))
        worst[name] = (n + 1, max(r, raw), max(m, mx), max(l, rel))
    terminalreporter.write_line("GPU vs oracle, largest errors per tensor (comparisons, raw max-abs, "
                                "max-abs beyond bf16 output rounding, rel-L2):")
    for name in sorted(worst):
        n, r, m, l = worst[name]
        terminalreporter.write_line(f"  {name:>14s} n={n:3d} raw={r:.3e} beyond={m:.3e} relL2={l:.3e}")
