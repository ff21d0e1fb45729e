"""Helpers of the GPU parity tests: tolerances, comparisons and the
teacher-forced greedy check."""

from __future__ import annotations

import numpy as np
import torch

import oracle

# Acceptance bars of the forward pass against the fp64 oracle.
BLOCK_REL_L2 = 1e-3   # per-block hidden-state relative L2: each block's own error,
                      # the block fed the oracle's input to it (fs_debug_block)
LOGIT_ABS = 2e-2      # max |delta logit|, end to end
GREEDY_STEPS = 32     # greedy ids must agree for this many steps, end to end
# Sanity bound on the hidden states of a whole end-to-end run. Rounding K and V
# to bf16 (as the cache stores them) turns fp32 rounding noise into whole-ulp
# flips, which adds about 4e-5 relative L2 per block; after 28 blocks an fp32
# forward sits near 1.1e-3. This bound only catches gross errors.
E2E_BLOCK_REL_L2 = 3e-3


# (label, measured value, bound) of every per-block and logit check of the
# session, printed in the terminal summary (tests/conftest.py).
REPORT = []


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def assert_blocks_close(gpu_hidden, ref_hidden, tol=BLOCK_REL_L2, what=""):
    """gpu_hidden, ref_hidden: [L+1, rows, H]. Returns the per-block errors."""
    errs = [rel_l2(gpu_hidden[l], ref_hidden[l]) for l in range(ref_hidden.shape[0])]
    worst = max(errs)
    REPORT.append((f"{what} per-block rel-L2", worst, tol))
    assert worst <= tol, f"{what} per-block rel-L2 {worst:.3e} > {tol} (all: {errs})"
    return errs


def assert_logits_close(gpu_logits, ref_logits, tol=LOGIT_ABS, what=""):
    d = float(np.max(np.abs(np.asarray(gpu_logits, np.float64) - ref_logits)))
    if what:
        REPORT.append((f"{what} max |dlogit|", d, tol))
    assert d <= tol, f"{what} max |dlogit| {d:.3e} > {tol}"
    return d


def top2_gap(logits) -> float:
    l = np.sort(np.asarray(logits, np.float64))
    return float(l[-1] - l[-2])


def check_greedy_step(gpu_id: int, gpu_logits, ref_logits) -> bool:
    """True if the step is unambiguous. An ambiguous step (oracle top-2 gap
    below twice the measured max |delta logit|) passes when the GPU picked
    either of the two candidates within that margin."""
    ref_id = oracle.greedy_select(ref_logits)
    margin = 2.0 * float(np.max(np.abs(np.asarray(gpu_logits, np.float64) - ref_logits)))
    if top2_gap(ref_logits) >= margin:
        assert gpu_id == ref_id, f"greedy id {gpu_id} != oracle {ref_id}"
        return True
    close = np.flatnonzero(np.asarray(ref_logits) >= np.max(ref_logits) - margin)
    assert gpu_id in close, f"greedy id {gpu_id} not within the ambiguity margin of {ref_id}"
    return False


def to_dev(a, device="cuda:0", dtype=torch.float32) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(dtype).to(device)


def oracle_tensor(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)
