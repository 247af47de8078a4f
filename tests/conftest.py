import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def _librfx_build():
    """The package's build script, loaded by path: importing the package itself
    needs the library it builds."""
    import importlib.util
    path = os.path.join(ROOT, "block_quantized_moe_rocmfpx_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_librfx_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA B200 (sm_100a) device")
    # build the in-tree libraries if a source changed (nvcc cross-compiles sm_100a on any host)
    _librfx_build().build()
    import synth
    synth.build()
    synth.build_dev()


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)
