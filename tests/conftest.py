"""pytest configuration: the ``gpu`` marker, the repository root on sys.path, and the order in
which test files run."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# Files collected after all others, in this order.  The file of the no-allocation entry point
# comes last of all, so that with -x a failure there cannot hide any other file's results.
RUN_LAST = ("test_gauge_gpu.py", "test_joint_gpu.py", "test_bench_modes_gpu.py",
            "test_wait_timeout_gpu.py", "test_zz_no_alloc.py")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_collection_modifyitems(session, config, items):
    def rank(item):
        name = os.path.basename(str(item.fspath))
        return RUN_LAST.index(name) + 1 if name in RUN_LAST else 0
    items.sort(key=rank)  # stable: the order within each group is kept
