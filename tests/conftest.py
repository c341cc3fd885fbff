import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the CUDA library")


def bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) exactly to float64."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bits(x) -> np.ndarray:
    """Round float values to bf16 (nearest-even, via torch) and return the bits."""
    import torch
    from long_context_prefill_attngate_b200.synthetic import bf16_bits
    return bf16_bits(torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16))


@pytest.fixture(scope="session")
def oracle():
    import oracle as _o
    _o.build()
    return _o
