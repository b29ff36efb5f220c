import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def built_lib():
    """The C-ABI library, built in-tree first when it is missing (host-only
    entry points of it run without a GPU)."""
    lib_path = os.path.join(ROOT, "block_sparse_local_nb_b200", "libnb_b200.so")
    if not os.path.exists(lib_path):
        from block_sparse_local_nb_b200.build import build

        build()
    from block_sparse_local_nb_b200 import binding

    return binding.lib()


@pytest.fixture(scope="session")
def golden_dir():
    return GOLDEN


def read_golden(name):
    """Yield the non-comment, non-empty lines of a golden fixture, split on whitespace."""
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line.split()


@pytest.fixture(autouse=True)
def _no_kernel_wait_timeouts(request):
    """After every GPU test: no kernel gave up on a bounded wait."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    import block_sparse_local_nb_b200 as nb

    code = nb.nb_kernel_error(clear=True)
    assert code == 0, f"a kernel recorded wait-timeout code {code:#x}"
