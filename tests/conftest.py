import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


# The checksum and streaming tests are collected after every other module,
# so that under -x a failure in them leaves the decoders' parity tests
# already run.
# The no-allocation entry point's tests come after those, at the very end.
RUN_LAST = ("test_gpu_xxh3.py", "test_gpu_stream.py", "test_zz_no_alloc.py")


def pytest_collection_modifyitems(config, items):
    rank = {name: i for i, name in enumerate(RUN_LAST)}
    last = [it for it in items if os.path.basename(str(it.fspath)) in rank]
    if last:
        last.sort(key=lambda it: rank[os.path.basename(str(it.fspath))])  # stable: keeps each file's own order
        items[:] = [it for it in items if it not in last] + last


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")
