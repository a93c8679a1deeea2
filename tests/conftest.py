import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: large-size parity case (still part of -m gpu)")
    config.addinivalue_line("markers", "expects_timeout: the test makes a device-side wait give up on purpose")


def pytest_collection_modifyitems(config, items):
    # GPU tests are skipped (not failed) when no GPU is present so that the
    # CPU suite can be run with or without the marker filter.
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


@pytest.fixture(autouse=True)
def _no_device_timeout(request):
    """After every GPU test: no kernel of the library gave up on a device-side wait."""
    yield
    if "gpu" not in request.keywords or request.node.get_closest_marker("expects_timeout"):
        return
    import torch
    if not torch.cuda.is_available():
        return
    import block_sparse_attention_cube_b200 as vsa
    vsa.device_status()


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """How many selection rows the near-tie rule excused in each comparison of the session."""
    try:
        from tests._util import NEAR_TIE_LOG
    except Exception:  # pragma: no cover
        return
    if not NEAR_TIE_LOG:
        return
    tr = terminalreporter
    tr.section("near-tie rows (GPU selection differs from the oracle's)")
    rows = sum(r for _, r, _, _ in NEAR_TIE_LOG)
    excused = sum(e for _, _, e, _ in NEAR_TIE_LOG)
    failed = sum(f for _, _, _, f in NEAR_TIE_LOG)
    tr.write_line(f"total: {excused} of {rows} rows excused as near-ties, {failed} failed, "
                  f"{len(NEAR_TIE_LOG)} comparisons")
    for label, r, e, f in NEAR_TIE_LOG:
        if e or f or "wan" in label:
            tr.write_line(f"  {label}: {e} of {r} rows excused, {f} failed")
