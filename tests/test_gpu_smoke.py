"""The round-trip entry point: one small decode step on cuda:0 checked
against the oracle (GPU only)."""
import os
import sys

import pytest

pytestmark = pytest.mark.gpu
sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))


def test_smoke_runs_and_matches_oracle():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA device")
    import __graft_entry__
    __graft_entry__.smoke()
