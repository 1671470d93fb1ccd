import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def load_build_module():
    """The package's build helper, loaded by path (importing the package
    itself requires the built library)."""
    import importlib.util
    path = os.path.join(ROOT, "video_diffusion_transformer_02_b200", "_build.py")
    spec = importlib.util.spec_from_file_location("vattn_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def pytest_sessionstart(session):
    # Build the CUDA library (cross-compiles on a CPU host) and the oracle
    # before any test imports them.
    load_build_module().build()
    import oracle
    oracle.build()


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA B200 (sm_100a) device")


def pytest_collection_modifyitems(config, items):
    # GPU tests run only where a device exists; on a CPU host they are skipped
    # (the driver selects them explicitly with -m gpu on a B200).
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device on this host")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)
