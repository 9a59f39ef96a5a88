"""Shared set-up for the GPU parity tests: the CUDA library must be the code that runs."""

import pytest
import torch

from spacetime_attention_b200 import build as B
from spacetime_attention_b200 import ops


@pytest.fixture(scope="session")
def gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    B.build()
    ops.library()
    return torch.device("cuda:0")
