"""GPU parity of gdn_decode_step against the float64 oracle (needs a B200)."""
import numpy as np
import pytest
import torch

import gated_delta_rule_142_b200 as gdn
import oracle
from gdn_inputs import WORKLOADS, as_f32_numpy, decode_inputs, workload_inputs
from parity_util import TOL, cpu_f64, oracle_threads, rel_err

pytestmark = pytest.mark.gpu


def oracle_steps(inp, steps, heads=None):
    """Oracle over `steps` consecutive tokens: a decode sequence is a forward pass
    with T = steps.  heads: optional list of flat (b*H + h) indices."""
    S = inp["S"]
    B, H, dv, dk = S.shape
    q, k, v = inp["q"][:steps], inp["k"][:steps], inp["v"][:steps]
    la, be = inp["log_alpha"][:steps], inp["beta"][:steps]
    # [steps, B, H, d] -> [1, steps, B*H, d]
    flat = lambda x: x.reshape(steps, B * H, *x.shape[3:]).unsqueeze(0)  # noqa: E731
    q, k, v, la, be = flat(q), flat(k), flat(v), flat(la), flat(be)
    S0 = S.reshape(1, B * H, dv, dk)
    if heads is not None:
        q, k, v, la, be = (x[:, :, heads] for x in (q, k, v, la, be))
        S0 = S0[:, heads]
    out, Sf = oracle.forward(as_f32_numpy(q), as_f32_numpy(k), as_f32_numpy(v), as_f32_numpy(la),
                             as_f32_numpy(be), as_f32_numpy(S0).astype(np.float64), nthreads=oracle_threads())
    return out[0], Sf[0]  # [steps, nh, dv], [nh, dv, dk]


def run_steps(inp, steps):
    dev = {k: v.cuda() for k, v in inp.items()}
    S = dev["S"].clone()
    outs = []
    for t in range(steps):
        outs.append(gdn.decode_step(dev["q"][t], dev["k"][t], dev["v"][t], dev["log_alpha"][t], dev["beta"][t], S))
    torch.cuda.synchronize()
    return torch.stack(outs), S


@pytest.mark.parametrize("dtype,dk,dv", [("f32", 16, 16), ("f32", 128, 128), ("f32", 32, 64), ("bf16", 64, 128),
                                         ("bf16", 128, 16), ("bf16", 128, 128), ("f32", 128, 32)])
def test_small_shapes(dtype, dk, dv):
    steps = 12
    inp = decode_inputs(steps, 3, 5, dk, dv, dtype, seed=40 + dk + dv, s0_std=0.3)
    outs, S = run_steps(inp, steps)
    ref_o, ref_S = oracle_steps(inp, steps)
    B, H = 3, 5
    assert rel_err(cpu_f64(outs).reshape(steps, B * H, dv), ref_o) <= TOL[dtype]
    assert rel_err(cpu_f64(S).reshape(B * H, dv, dk), ref_S) <= TOL[dtype]


def test_workload_1024_steps():
    """B=64, H=16, d=128, 1024 consecutive steps: every head for the first 16 steps,
    and 24 sampled heads over all 1024 steps (outputs and final state)."""
    w = WORKLOADS["decode_bf16_b64h16_d128_x1024"]
    inp = workload_inputs(w)
    outs, S = run_steps(inp, w.steps)
    B, H, dv, dk = inp["S"].shape
    o = cpu_f64(outs).reshape(w.steps, B * H, dv)
    # every head, first 16 steps
    ref_o, _ = oracle_steps(inp, 16)
    assert rel_err(o[:16], ref_o) <= TOL["bf16"]
    heads = sorted(set(np.random.default_rng(0).choice(B * H, 24, replace=False).tolist()) | {0, B * H - 1})
    ref_o, ref_S = oracle_steps(inp, w.steps, heads=heads)
    assert rel_err(o[:, heads], ref_o) <= TOL["bf16"]
    assert rel_err(cpu_f64(S).reshape(B * H, dv, dk)[heads], ref_S) <= TOL["bf16"]


def test_decode_matches_forward():
    """n decode steps == one forward over T = n (both against the oracle, and each other)."""
    steps, B, H, d = 40, 2, 3, 128
    inp = decode_inputs(steps, B, H, d, d, "bf16", seed=51, s0_std=0.1)
    outs, S = run_steps(inp, steps)
    dev = {k: v.cuda() for k, v in inp.items()}
    tfirst = lambda x: x.permute(1, 0, *range(2, x.dim())).contiguous()  # noqa: E731
    of, Sf = gdn.forward(tfirst(dev["q"]), tfirst(dev["k"]), tfirst(dev["v"]), tfirst(dev["log_alpha"]),
                         tfirst(dev["beta"]), dev["S"], chunk=64)
    torch.cuda.synchronize()
    assert rel_err(cpu_f64(of.transpose(0, 1)), cpu_f64(outs)) <= TOL["bf16"]
    assert rel_err(cpu_f64(Sf), cpu_f64(S)) <= TOL["bf16"]
    ref_o, ref_S = oracle_steps(inp, steps)
    assert rel_err(cpu_f64(outs).reshape(steps, B * H, d), ref_o) <= TOL["bf16"]


def test_reset_and_identity_gates():
    steps, B, H, d = 6, 2, 2, 64
    inp = decode_inputs(steps, B, H, d, d, "f32", seed=53, s0_std=0.5)
    inp["log_alpha"][2] = float("-inf")
    inp["log_alpha"][4] = 0.0
    inp["beta"][4] = 0.0
    outs, S = run_steps(inp, steps)
    ref_o, ref_S = oracle_steps(inp, steps)
    assert rel_err(cpu_f64(outs).reshape(steps, B * H, d), ref_o) <= TOL["f32"]
    assert rel_err(cpu_f64(S).reshape(B * H, d, d), ref_S) <= TOL["f32"]


def test_host_buffers_are_staged():
    steps, B, H, d = 3, 2, 2, 128
    inp = decode_inputs(steps, B, H, d, d, "bf16", seed=57, s0_std=0.2)
    ref_o, ref_S = oracle_steps(inp, steps)
    S = inp["S"].clone().pin_memory()
    outs = []
    for t in range(steps):
        # keep the pinned inputs referenced until the stream has consumed them
        args = [inp[name][t].pin_memory() for name in ("q", "k", "v", "log_alpha", "beta")]
        outs.append(gdn.decode_step(*args, S))
        torch.cuda.synchronize()
        del args
    assert rel_err(cpu_f64(torch.stack(outs)).reshape(steps, B * H, d), ref_o) <= TOL["bf16"]
    assert rel_err(cpu_f64(S).reshape(B * H, d, d), ref_S) <= TOL["bf16"]


def test_steps_replayed_from_a_cuda_graph():
    """Device-buffer decode steps can be captured in a CUDA graph (the bench times them that way);
    a replay gives the oracle's result, like the eager calls."""
    steps, B, H, d = 5, 4, 2, 128
    inp = decode_inputs(steps, B, H, d, d, "bf16", seed=59, s0_std=0.1)
    ref_o, ref_S = oracle_steps(inp, steps)
    dd = {k: v.cuda() for k, v in inp.items()}
    S = dd["S"].clone()
    outs = torch.empty((steps, B, H, d), dtype=dd["q"].dtype, device="cuda")
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        cap = torch.cuda.current_stream()
        for t in range(steps):
            gdn.decode_step(dd["q"][t], dd["k"][t], dd["v"][t], dd["log_alpha"][t], dd["beta"][t], S, out=outs[t],
                            stream=cap)
    S.copy_(dd["S"])  # capture does not run the kernels; start the replay from the initial state
    graph.replay()
    torch.cuda.synchronize()
    assert rel_err(cpu_f64(outs).reshape(steps, B * H, d), ref_o) <= TOL["bf16"]
    assert rel_err(cpu_f64(S).reshape(B * H, d, d), ref_S) <= TOL["bf16"]


@pytest.mark.parametrize("B", [128, 512])
def test_serving_batch(B):
    """Decode at serving batch sizes (128 to 512 sequences), bf16, d = 128; every head checked at
    B = 128, a sample of heads at B = 512."""
    steps, H, d = 3, 4, 128
    inp = decode_inputs(steps, B, H, d, d, "bf16", seed=61 + B, s0_std=0.05)
    outs, S = run_steps(inp, steps)
    heads = None if B == 128 else list(range(0, B * H, 37))
    ref_o, ref_S = oracle_steps(inp, steps, heads=heads)
    o = cpu_f64(outs).reshape(steps, B * H, d)
    Sn = cpu_f64(S).reshape(B * H, d, d)
    if heads is not None:
        o, Sn = o[:, heads], Sn[heads]
    assert rel_err(o, ref_o.reshape(o.shape)) <= TOL["bf16"]
    assert rel_err(Sn, ref_S.reshape(Sn.shape)) <= TOL["bf16"]
