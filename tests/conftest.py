import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200) and the built CUDA library")
    config.addinivalue_line("markers", "slow: CPU test that takes more than a few seconds")


@pytest.fixture(scope="session")
def micro_cfg():
    import synth
    return synth.ModelConfig("micro", n_layers=2, d_model=32, n_heads=2, head_dim=16, d_ff=64, vocab=64,
                             n_updated=1, T=40, k=12, b=8, eta=0.05, dtype="f32", seed=0x5EED)
