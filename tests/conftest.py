import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Report the rounding half-point cases met by the GPU parity tests and
    the largest decode-attention difference from the oracle."""
    try:
        from tests.gpu_helpers import ATTN_ERR_LOG, HALF_POINT_LOG
    except Exception:
        return
    if ATTN_ERR_LOG:
        ranked = sorted(ATTN_ERR_LOG, key=lambda x: -x[1])
        terminalreporter.write_line(
            f"GPU decode: {len(ATTN_ERR_LOG)} attention comparisons with the oracle; largest max-abs "
            f"differences (tolerance 2e-3): " + "; ".join(f"{e:.3g} {n}" for n, e in ranked[:6]))
    if not HALF_POINT_LOG:
        return
    n = sum(h for h, _ in HALF_POINT_LOG)
    codes = sum(c for _, c in HALF_POINT_LOG)
    terminalreporter.write_line(
        f"GPU parity: {codes} codes compared with the oracle in {len(HALF_POINT_LOG)} comparisons; "
        f"{n} differed, each at a rounding half-point (within 1e-6)")
