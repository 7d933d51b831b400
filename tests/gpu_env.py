"""Shared set-up for the GPU tests: build the library, one context."""
import pytest


def require_gpu():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device (run with -m 'not gpu' on a CPU box)")


def context():
    require_gpu()
    from matrix_aware_optimizers_muon_b200 import Context, build
    build.build()
    return Context(0)
