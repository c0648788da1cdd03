"""gdn_forward on pinned host buffers large enough for the host pipeline (needs a B200): the
problem is cut along T into pieces whose copies in and out overlap the kernels, the state passing
between pieces on the device.  Checked against the same call on device buffers and against the
float64 oracle on sampled heads."""
import numpy as np
import pytest
import torch

import gated_delta_rule_142_b200 as gdn
import oracle
from gdn_inputs import as_f32_numpy, forward_inputs, raw_inputs
from parity_util import TOL, cpu_f64, oracle_threads, rel_err

pytestmark = pytest.mark.gpu

NAMES = ("q", "k", "v", "log_alpha", "beta")


def run(inp, chunk, host, raw=False, S0_on_device=False):
    if host:
        d = {n: inp[n].pin_memory() for n in NAMES}
    else:
        d = {n: inp[n].cuda() for n in NAMES}
    S0 = inp["S0"]
    if S0 is not None:
        S0 = S0.cuda() if (S0_on_device or not host) else S0.pin_memory()
    fn = gdn.forward_raw if raw else gdn.forward
    out, Sf = fn(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0, chunk=chunk)
    torch.cuda.synchronize()
    return out, Sf


def test_bf16_pipeline_matches_device_call_and_oracle():
    B, T, H, dim = 1, 16384, 16, 128  # 270 MB of token-major tensors: four pieces
    inp = forward_inputs(B, T, H, dim, dim, "bf16", seed=601, s0_std=0.05, alpha_mu=-3.0)
    out_h, Sf_h = run(inp, 64, host=True)
    assert not out_h.is_cuda and not Sf_h.is_cuda
    out_d, Sf_d = run(inp, 64, host=False)
    assert rel_err(cpu_f64(out_h), cpu_f64(out_d)) <= 5e-3
    assert rel_err(cpu_f64(Sf_h), cpu_f64(Sf_d)) <= 5e-3
    for h in (0, 9):
        sel = lambda t: as_f32_numpy(t[:, :, h:h + 1].contiguous())  # noqa: E731
        ro, rs = oracle.forward(*[sel(inp[n]) for n in NAMES], inp["S0"][:, h:h + 1].numpy().astype(np.float64),
                                nthreads=oracle_threads())
        assert rel_err(cpu_f64(out_h)[:, :, h:h + 1], ro) <= TOL["bf16"], h
        assert rel_err(cpu_f64(Sf_h)[:, h:h + 1], rs) <= TOL["bf16"], h


def test_f32_pipeline_with_batch_rows_is_exact():
    """Several batch rows (strided piece copies) on the CUDA-core forward: the pieces compute the
    same chunks from the same states as one call, so the results are bit-identical."""
    B, T, H, dim = 2, 4096, 8, 64  # 67 MB of token-major tensors
    inp = forward_inputs(B, T, H, dim, dim, "f32", seed=602, s0_std=0.2)
    out_h, Sf_h = run(inp, 32, host=True, S0_on_device=True)
    out_d, Sf_d = run(inp, 32, host=False)
    assert torch.equal(out_h, out_d.cpu())
    assert torch.equal(Sf_h.cpu(), Sf_d.cpu())


def test_raw_inputs_through_the_pipeline():
    B, T, H, dim = 1, 16384, 16, 128
    r = raw_inputs((B, T, H), dim, dim, "bf16", seed=603, s0_shape=(B, H, dim, dim), s0_std=0.05,
                   zero_rows=0.02)
    inp = {"q": r["q"], "k": r["k"], "v": r["v"], "log_alpha": r["x_alpha"], "beta": r["x_beta"], "S0": r["S0"]}
    out_h, Sf_h = run(inp, 64, host=True, raw=True)
    out_d, Sf_d = run(inp, 64, host=False, raw=True)
    assert rel_err(cpu_f64(out_h), cpu_f64(out_d)) <= 5e-3
    assert rel_err(cpu_f64(Sf_h), cpu_f64(Sf_d)) <= 5e-3


def test_pipeline_can_be_switched_off(monkeypatch):
    monkeypatch.setenv("GDN_HOST_PIPELINE", "0")
    B, T, H, dim = 2, 4096, 8, 64
    inp = forward_inputs(B, T, H, dim, dim, "f32", seed=604, s0_std=0.2)
    out_h, Sf_h = run(inp, 32, host=True)
    out_d, Sf_d = run(inp, 32, host=False)
    assert torch.equal(out_h, out_d.cpu()) and torch.equal(Sf_h, Sf_d.cpu())
