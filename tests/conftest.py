import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
TESTS = os.path.dirname(os.path.abspath(__file__))
if TESTS not in sys.path:
    sys.path.insert(0, TESTS)


def _apply_test_tuning():
    """PA_TEST_DECODE_TUNING="shape=paired,planner=1,..." runs this test process's decode calls under a
    scheduling alternative of the library (pa_decode_tuned); the library itself reads no environment."""
    spec = os.environ.get("PA_TEST_DECODE_TUNING", "")
    if not spec:
        return
    import paged_kv_cache_362_b200 as pa

    kw = dict(item.split("=", 1) for item in spec.split(","))
    pa.set_default_tuning(pa.tuning(**{k: (v if k == "shape" else int(v)) for k, v in kw.items()}))


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")
    _apply_test_tuning()


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
