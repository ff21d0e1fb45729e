"""Shared test set-up: the ``gpu`` marker and conversions of the seeded inputs
into the plain numpy form the oracle takes."""

import os
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter):
    """The measured errors of the parity checks that ran, against their bounds."""
    try:
        from parity_util import REPORT
    except ImportError:
        return
    if not REPORT:
        return
    terminalreporter.write_line("parity measurements (value / bound):")
    for what, val, tol in REPORT:
        terminalreporter.write_line(f"  {what}: {val:.3e} / {tol:g}")


def bf16_to_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 bit patterns (no arithmetic)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def oracle_weights(w: dict) -> dict:
    """Seeded weights (torch, from ``synth.model_weights``) -> oracle input dict."""
    def lin(x):
        if isinstance(x, tuple):
            codes, scales = x
            return (codes.numpy(), scales.numpy())
        return bf16_to_bits(x)

    layers = []
    for lw in w["layers"]:
        layers.append({k: (lin(v) if k.startswith("w") else bf16_to_bits(v))
                       for k, v in lw.items()})
    return {"embed": bf16_to_bits(w["embed"]), "final_norm": bf16_to_bits(w["final_norm"]),
            "layers": layers}


def gpu_available() -> bool:
    return torch.cuda.is_available()


@pytest.fixture(scope="session")
def cuda_device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")
