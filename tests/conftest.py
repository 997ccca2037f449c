import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    # build libkvc.so if it is missing or older than its sources (nvcc
    # cross-compiles for sm_100a without a GPU)
    import importlib.util
    path = os.path.join(ROOT, "compressed_decode_attention_kvc_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_kvc_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")
