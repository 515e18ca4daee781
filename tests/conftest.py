import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _build_library():
    """Compiles libsvdq.so if it is missing or stale, before any test imports the package
    (importing the package loads the library).  The builder is loaded from its file so that
    this needs no package import."""
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_svdq_build", os.path.join(ROOT, "bit_diffusion_transformer_act_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()


_build_library()


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs an sm_100a GPU (B200) and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size CPU work (oracle on large shapes)")


@pytest.fixture(scope="session")
def cuda_lib():
    """The loaded C-ABI library bound to cuda:0; fails loudly if it is missing."""
    import torch
    if not torch.cuda.is_available():
        pytest.fail("gpu test run without a visible CUDA device")
    import bit_diffusion_transformer_act_b200 as pkg
    return pkg
