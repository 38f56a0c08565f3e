import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


@pytest.fixture(scope="session")
def cuda_dev():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


@pytest.fixture(scope="session")
def big_inputs(cuda_dev):
    """Full-size seeded inputs of a named workload: host bf16 bits + device copies.

    Keeps only the most recently requested workload alive to bound memory.
    """
    import numpy as np
    import torch

    import synth

    cache = {}

    def get(name):
        if name not in cache:
            cache.clear()
            torch.cuda.empty_cache()
            w = synth.WORKLOADS[name]
            q, k, v = synth.qkv_numpy(w)
            dev = [torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(cuda_dev) for a in (q, k, v)]
            cache[name] = (q, k, v, *dev)
        return cache[name]

    yield get
    cache.clear()
