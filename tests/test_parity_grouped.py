"""GPU parity of the grouped-heads entry points (gdn_forward_grouped, gdn_decode_step_grouped)
against the float64 oracle's grouped forward (needs a B200).  Same bar as the forward:
max |gpu - ref| / max |ref| <= 1e-4 for float32 inputs, <= 2e-2 for bfloat16 inputs."""
import numpy as np
import pytest
import torch

import gated_delta_rule_142_b200 as gdn
import oracle
from gdn_inputs import as_f32_numpy, forward_inputs
from parity_util import TOL, cpu_f64, oracle_threads, rel_err

pytestmark = pytest.mark.gpu


def grouped(B, T, Hq, Hkv, d, dtype, seed, s0=0.1, alpha_mu=0.0):
    """q from a forward draw with Hq heads; k, v, gates, S0 from one with Hkv heads."""
    a = forward_inputs(B, T, Hq, d, d, dtype, seed=seed)
    b = forward_inputs(B, T, Hkv, d, d, dtype, seed=seed + 1, s0_std=s0, alpha_mu=alpha_mu)
    return {"q": a["q"], "k": b["k"], "v": b["v"], "log_alpha": b["log_alpha"], "beta": b["beta"], "S0": b["S0"]}


NAMES = ("q", "k", "v", "log_alpha", "beta")


def check(inp, dtype, chunk, host=False, label=""):
    dev = lambda t: None if t is None else (t.pin_memory() if host else t.cuda())  # noqa: E731
    out, Sf = gdn.forward_grouped(*[dev(inp[n]) for n in NAMES], dev(inp["S0"]), chunk=chunk)
    torch.cuda.synchronize()
    S0 = None if inp["S0"] is None else as_f32_numpy(inp["S0"]).astype(np.float64)
    ro, rS = oracle.forward_grouped(*[as_f32_numpy(inp[n]) for n in NAMES], S0, nthreads=oracle_threads())
    eo, es = rel_err(cpu_f64(out), ro), rel_err(cpu_f64(Sf), rS)
    assert eo <= TOL[dtype] and es <= TOL[dtype], (label, eo, es)


@pytest.mark.parametrize("B,T,Hq,Hkv", [(1, 300, 8, 2), (2, 130, 4, 1), (1, 64, 6, 3), (2, 257, 16, 2)])
def test_two_kernel_forward(B, T, Hq, Hkv):
    """bf16, d = 128, chunk 64: the ATMA shape (8 query / 2 key-value heads) and others.  One chain
    per key-value head (its query head hk * G), and the other query heads' outputs from that
    memory's checkpoints and U^T by the grouped-output kernel."""
    gdn.timing_start()
    try:
        check(grouped(B, T, Hq, Hkv, 128, "bf16", seed=700 + T), "bf16", 64, label="%d/%d" % (Hq, Hkv))
    finally:
        kinds = gdn.timing_stop()
    assert kinds["group_out"][1] == 1 and kinds["chain"][1] == 1, kinds


@pytest.mark.parametrize("nseg", ["3", "7"])
def test_two_kernel_forward_with_segments(monkeypatch, nseg):
    """Segments of the key-value heads' chains: transfers, prefix and entry states per memory."""
    monkeypatch.setenv("GDN_SEGMENTS", nseg)
    check(grouped(1, 1000, 8, 2, 128, "bf16", seed=711, alpha_mu=-3.0), "bf16", 64, label="segments " + nseg)
    check(grouped(2, 700, 4, 2, 128, "bf16", seed=712, alpha_mu=0.0), "bf16", 64, label="fast decay " + nseg)


def test_other_paths_recompute_per_query_head(monkeypatch):
    """With the two-kernel forward switched off (GDN_FORWARD_PATH=fused) grouped heads take the
    CUDA-core forward, where each query head recomputes its memory; same bar at d = 128."""
    monkeypatch.setenv("GDN_FORWARD_PATH", "fused")
    gdn.timing_start()
    try:
        check(grouped(1, 200, 8, 2, 128, "bf16", seed=713), "bf16", 64, label="recompute")
    finally:
        kinds = gdn.timing_stop()
    assert "group_out" not in kinds, kinds


@pytest.mark.parametrize("dtype,d,chunk", [("f32", 64, 32), ("f32", 16, 16), ("bf16", 64, 64)])
def test_cuda_core_forward(dtype, d, chunk):
    check(grouped(2, 100, 8, 2, d, dtype, seed=720 + d), dtype, chunk, label="%s d%d" % (dtype, d))


def test_host_buffers_and_empty_sequence():
    check(grouped(1, 70, 4, 2, 128, "bf16", seed=731), "bf16", 64, host=True, label="host")
    inp = grouped(1, 0, 4, 2, 128, "bf16", seed=733)
    out, Sf = gdn.forward_grouped(*[inp[n].cuda() for n in NAMES], inp["S0"].cuda(), chunk=64)
    torch.cuda.synchronize()
    assert out.shape == (1, 0, 4, 128) and torch.equal(Sf.cpu(), inp["S0"])


def test_one_group_is_the_plain_forward():
    inp = grouped(1, 150, 4, 4, 128, "bf16", seed=741)
    a = gdn.forward_grouped(*[inp[n].cuda() for n in NAMES], inp["S0"].cuda(), chunk=64)
    b = gdn.forward(*[inp[n].cuda() for n in NAMES], inp["S0"].cuda(), chunk=64)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 32)])
def test_decode_steps(dtype, d):
    steps, B, Hq, Hkv = 3, 4, 8, 2
    q = forward_inputs(steps, B, Hq, d, d, dtype, seed=750)["q"]          # [steps, B, Hq, d]
    kv = forward_inputs(steps, B, Hkv, d, d, dtype, seed=751)
    g = torch.Generator(device="cpu")
    g.manual_seed(752)
    S = torch.randn((B, Hkv, d, d), generator=g) * 0.05
    S_dev, S_ref = S.cuda(), S.numpy().astype(np.float64)
    for t in range(steps):
        x = [q[t], kv["k"][t], kv["v"][t], kv["log_alpha"][t], kv["beta"][t]]
        o = gdn.decode_step_grouped(*[a.contiguous().cuda() for a in x], S_dev)
        torch.cuda.synchronize()
        ro = oracle.decode_step_grouped(*[as_f32_numpy(a.contiguous()) for a in x], S_ref)
        assert rel_err(cpu_f64(o), ro) <= TOL[dtype], t
    assert rel_err(cpu_f64(S_dev), S_ref) <= TOL[dtype]
