import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def gpu_available() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def cuda_device():
    if not gpu_available():
        pytest.skip("no CUDA device")
    import torch
    return torch.device("cuda:0")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """The parity record of the session: every full-size workload's comparison on its own
    line (mismatch counts, and a histogram of the mismatches' distance to their rounding or
    scale boundary), then the totals over every other comparison."""
    try:
        from oracle.parity import REPORTS, HIST_LABELS
    except Exception:
        return
    if not REPORTS:
        return
    tr = terminalreporter
    tr.write_sep("-", f"parity record ({len(REPORTS)} comparisons against the oracle)")
    rest = [r for r in REPORTS if not r.label.startswith("workload ")]
    if rest:
        total = rest[0]
        for r in rest[1:]:
            total = total.merge(r)
        exact = sum(1 for r in rest if r.mismatch_elements == 0 and r.zero_sign_forgiven == 0)
        worst = max(rest, key=lambda r: r.mismatch_elements / max(r.n, 1))
        hist = " ".join(f"{l}:{c}" for l, c in zip(HIST_LABELS, total.hist_elements) if c)
        tr.write_line(f"small shapes: {len(rest)} comparisons, {exact} bit-exact; {total.n} elements, "
                      f"{total.mismatch_elements} differ, all inside F: {total.unflagged_code_mismatch == 0 and total.unflagged_scale_mismatch == 0}; "
                      f"zero-sign forgiven {total.zero_sign_forgiven}; element distances [{hist}]; worst "
                      f"{worst.mismatch_elements}/{worst.n} ({worst.label})")
    for r in REPORTS:
        if r.label.startswith("workload "):
            tr.write_line(r.line())
