import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


# Set in a child process that runs GPU tests against the library's debug
# variant (MXQ_LIBRARY=.../libmxq_debug.so): after every GPU test, no index
# check of any kernel may have failed.
EXPECT_CLEAN_CHECKS = "MXQ_EXPECT_CLEAN_CHECKS"


@pytest.fixture(autouse=True)
def _no_failed_index_check(request):
    yield
    if os.environ.get(EXPECT_CLEAN_CHECKS) and request.node.get_closest_marker("gpu"):
        import nvfp4_quantization_amax_b200 as mxq

        rec = mxq.debug_checks()
        assert rec is None, "failed index check (id, index, extent): %s" % (rec,)


def read_golden(name):
    """Rows of a golden fixture: comment lines and trailing comments dropped."""
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    return rows


@pytest.fixture(scope="session")
def facts():
    return {k: float(v) for k, v in read_golden("format_facts.txt")}
