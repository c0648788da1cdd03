"""Shared helpers for the GPU parity tests: tolerances, error metric, and
running the oracle on the exact values the GPU consumed."""
import os

import numpy as np
import torch

import oracle
from gdn_inputs import as_f32_numpy

# Error metric: max |gpu - ref| / max |ref| over every element compared.
# Bars: 1e-4 for float32 inputs, 2e-2 for bfloat16 inputs (float32 accumulation
# and float32 state), applied to the outputs and the final state separately.
TOL = {"f32": 1e-4, "bf16": 2e-2}

# Every error the GPU tests compute, with the test that computed it: printed in the terminal summary
# (tests/conftest.py) and, when GDN_PARITY_LOG names a file, appended to it as JSON lines.
ACHIEVED = []


def rel_err(gpu, ref) -> float:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    if ref.size == 0:
        return 0.0
    scale = np.abs(ref).max()
    assert np.isfinite(gpu).all(), "non-finite GPU values"
    e = float(np.abs(gpu - ref).max() / max(scale, 1e-30))
    test = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
    ACHIEVED.append((test, e))
    return e


def oracle_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def oracle_forward(inp, heads=None, batches=None):
    """Oracle on CPU tensors from gdn_inputs.forward_inputs, optionally restricted
    to a subset of heads / batch rows.  Returns float64 (out, S_final)."""
    def sel(t, hax):
        if t is None:
            return None
        if batches is not None:
            t = t[list(batches)]
        if heads is not None:
            t = t[:, :, list(heads)] if hax == 2 else t[:, list(heads)]
        return t

    q, k, v = sel(inp["q"], 2), sel(inp["k"], 2), sel(inp["v"], 2)
    la, be = sel(inp["log_alpha"], 2), sel(inp["beta"], 2)
    S0 = sel(inp["S0"], 1)
    S0n = None if S0 is None else as_f32_numpy(S0).astype(np.float64)
    return oracle.forward(as_f32_numpy(q), as_f32_numpy(k), as_f32_numpy(v), as_f32_numpy(la), as_f32_numpy(be),
                          S0n, nthreads=oracle_threads())


def to_device(inp, device="cuda"):
    return {k: (None if v is None else v.to(device)) for k, v in inp.items()}


def cpu_f64(t):
    return t.detach().to("cpu", torch.float64).numpy()
