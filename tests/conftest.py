import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs an NVIDIA B200 (sm_100a) and the built CUDA library")


@pytest.fixture(scope="session")
def orc():
    import oracle
    return oracle.default()


# Files run in dependency order, so that with -x the first failure is the
# root cause: the oracle against its pins before anything is compared with
# it, the input generator, the library's loading and host validation, its
# resource report, the bounds on every device wait, its kernel selection,
# the benchmark's rank logic and its profile summaries, then GPU parity of
# the plain calls, of the variants, and last the allocation-free backward.
# Files not listed run after the variants; tests keep their order within a
# file.
_ORDER = ["test_oracle_pins.py", "test_oracle_mutants.py", "test_workloads.py",
          "test_library_cpu.py", "test_build_cpu.py", "test_device_safety_cpu.py",
          "test_host_geometry.py", "test_bench_multirank.py", "test_profiles_cpu.py",
          "test_parity_gpu.py", "test_variants_gpu.py"]
_LAST = "test_zz_no_alloc.py"


def _rank(item) -> float:
    name = os.path.basename(str(item.fspath))
    if name == _LAST:
        return len(_ORDER) + 1
    return _ORDER.index(name) if name in _ORDER else len(_ORDER)


def pytest_collection_modifyitems(session, config, items):
    items.sort(key=_rank)     # stable: order within a file is kept
