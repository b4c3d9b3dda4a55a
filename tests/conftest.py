import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built library")


def read_golden(name):
    """Rows of a '|'-separated golden fixture, comments dropped."""
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append([field.split() for field in line.split("|")])
    return rows


@pytest.fixture(autouse=True)
def _bounds_check_record(request):
    """Under the bounds-check build (KVQ_LIBRARY=debug), every GPU test must leave the
    library's record of failed bounds checks empty."""
    yield
    if os.environ.get("KVQ_LIBRARY") != "debug" or request.node.get_closest_marker("gpu") is None:
        return
    import torch
    if not torch.cuda.is_available():
        return
    from mixed_precision_quantized_pack_b200 import kvq as K
    assert K.kvq_debug_build(), "KVQ_LIBRARY=debug but the loaded library has no bounds checks"
    rec = K.kvq_debug_take_record(K._stream())
    assert rec["failures"] == 0, f"a bounds check failed: {rec}"
