import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running check")


def pytest_collection_modifyitems(config, items):
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


def pytest_terminal_summary(terminalreporter):
    """Summary of the bf16 GEMM output checks: how far the GPU's bf16 results
    sat from the fp64 reference, in bf16 ulps."""
    try:
        from tests.gpu_util import BF16_CHECKS
    except Exception:  # pragma: no cover
        return
    if not BF16_CHECKS:
        return
    worst = max(BF16_CHECKS, key=lambda c: c[1])
    least = min(BF16_CHECKS, key=lambda c: c[2])
    n = sum(c[3] for c in BF16_CHECKS)
    terminalreporter.write_line(
        "bf16 GEMM checks: %d checks, %d elements; max %.3f ulp (%s); lowest share within 1 ulp %.6f (%s)"
        % (len(BF16_CHECKS), n, worst[1], worst[0], least[2], least[0]))
