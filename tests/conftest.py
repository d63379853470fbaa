import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def load_codebook(g: int) -> np.ndarray:
    """Global codebook written by oracle/make_codebooks.py ([256][g] fp32)."""
    return np.fromfile(os.path.join(GOLDEN, f"codebook_g{g}.f32"), dtype="<f4").reshape(256, g)


@pytest.fixture(scope="session")
def codebooks():
    return {8: load_codebook(8), 4: load_codebook(4)}
