import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: long oracle runs")


_CACHE = {}


def weights(n_layers: int, seed: int = 1234) -> np.ndarray:
    """Seeded bf16 weight blob, generated once per process."""
    key = (n_layers, seed)
    if key not in _CACHE:
        from audio_encoder_b200 import synth
        _CACHE[key] = synth.make_weights(n_layers, seed)
    return _CACHE[key]


_MODELS = {}


def oracle_model(n_layers: int, seed: int = 1234):
    import oracle
    key = (n_layers, seed)
    if key not in _MODELS:
        _MODELS[key] = oracle.Model(weights(n_layers, seed), n_layers)
    return _MODELS[key]


@pytest.fixture(scope="session")
def w4():
    return weights(4)


@pytest.fixture(scope="session")
def om4():
    return oracle_model(4)
