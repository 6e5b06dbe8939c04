import os
import pathlib
import re
import shutil
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running full-size case")


@pytest.fixture(scope="session")
def cuda_lib():
    """The CUDA library on a GPU; GPU tests fail loudly if it cannot load."""
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU test collected without a CUDA device")
    import newton_schulz_09_b200 as dm
    dm.load_library()
    return dm


@pytest.fixture
def scratch_dir(request) -> pathlib.Path:
    """An empty per-test folder inside the repository's git-ignored build
    folder (tests keep their files inside the working tree)."""
    name = re.sub(r"[^A-Za-z0-9_.-]+", "_", request.node.nodeid)[-120:]
    path = pathlib.Path(ROOT) / "_build" / "test_scratch" / name
    if path.exists():
        shutil.rmtree(path)
    path.mkdir(parents=True)
    return path
