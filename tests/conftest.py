import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU check")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_sessionstart(session):
    # The CUDA library and the oracle are built in-tree (nvcc cross-compiles
    # sm_100a without a GPU); rebuild them if a source is newer.
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_msa_build", os.path.join(ROOT, "block_sparse_long_03_b200", "build.py"))
    lib_build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(lib_build)
    lib_build.build()
    if os.environ.get("MSA_LIBRARY") == "checked":
        lib_build.build(checked=True)
    import oracle
    oracle.build()


@pytest.fixture(autouse=True)
def _no_failed_bounds_checks(request):
    """Under the checked build (MSA_LIBRARY=checked) every GPU test must end
    with no failed device bounds check."""
    yield
    if os.environ.get("MSA_LIBRARY") == "checked" and "gpu" in request.keywords:
        from block_sparse_long_03_b200 import binding
        assert binding.lib.msa_bounds_failures() == 0, "a device bounds check failed"
