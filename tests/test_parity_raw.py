"""GPU parity of the raw-input entry points (gdn_forward_raw, gdn_forward_varlen_raw,
gdn_decode_step_raw) against the float64 oracle's input stage + recurrence (needs a B200).

q and k arrive in any scale (row norms log-uniform in [1/20, 20] times sqrt(d), some rows zero),
the gates as logits; the kernels normalise and map them.  Same bar as the plain forward:
max |gpu - ref| / max |ref| <= 1e-4 for float32 inputs, <= 2e-2 for bfloat16 inputs."""
import numpy as np
import pytest
import torch

import gated_delta_rule_142_b200 as gdn
import oracle
from gdn_inputs import as_f32_numpy, raw_inputs
from parity_util import TOL, cpu_f64, oracle_threads, rel_err

pytestmark = pytest.mark.gpu

NAMES = ("q", "k", "v", "x_alpha", "x_beta")


def oracle_raw(inp):
    S0 = None if inp["S0"] is None else as_f32_numpy(inp["S0"]).astype(np.float64)
    return oracle.forward_raw(*[as_f32_numpy(inp[n]) for n in NAMES], S0, nthreads=oracle_threads())


def fwd_inputs(B, T, H, d, dtype, seed, s0_std=0.1, alpha_mu=0.0, zero_rows=0.03):
    return raw_inputs((B, T, H), d, d, dtype, seed, s0_shape=(B, H, d, d), s0_std=s0_std, alpha_mu=alpha_mu,
                      zero_rows=zero_rows)


def check_forward(inp, dtype, chunk, host=False, label=""):
    dev = {n: (None if inp[n] is None else (inp[n].pin_memory() if host else inp[n].cuda()))
           for n in NAMES + ("S0",)}
    out, Sf = gdn.forward_raw(dev["q"], dev["k"], dev["v"], dev["x_alpha"], dev["x_beta"], dev["S0"], chunk=chunk)
    torch.cuda.synchronize()
    ref_o, ref_S = oracle_raw(inp)
    eo, es = rel_err(cpu_f64(out), ref_o), rel_err(cpu_f64(Sf), ref_S)
    assert eo <= TOL[dtype] and es <= TOL[dtype], (label, eo, es)


@pytest.mark.parametrize("B,T,H", [(2, 300, 4), (1, 64, 3), (3, 1, 2)])
def test_two_kernel_forward(B, T, H):
    """bf16, d = 128, chunk 64: the prep kernel normalises q, k and maps the gates on its own loads."""
    check_forward(fwd_inputs(B, T, H, 128, "bf16", seed=101 + T), "bf16", 64, label="T=%d" % T)


@pytest.mark.parametrize("nseg", [3, 5])
def test_two_kernel_forward_segments(monkeypatch, nseg):
    """Long sequence cut into segments: the transfer pass reads the same folded gate record."""
    monkeypatch.setenv("GDN_SEGMENTS", str(nseg))
    check_forward(fwd_inputs(1, 1000, 2, 128, "bf16", seed=111 + nseg, alpha_mu=-4.0), "bf16", 64,
                  label="segments=%d" % nseg)


def test_large_logits_and_zero_rows():
    """Gate logits up to +-30 (alpha and beta at both ends of (0, 1)) and a tenth of the q, k rows zero."""
    inp = fwd_inputs(2, 200, 2, 128, "bf16", seed=121, zero_rows=0.1)
    inp["x_alpha"].mul_(8.0)
    inp["x_beta"].mul_(8.0)
    inp["x_alpha"].clamp_(-30, 30)
    inp["x_beta"].clamp_(-30, 30)
    check_forward(inp, "bf16", 64, label="large logits")


@pytest.mark.parametrize("dtype,d,chunk", [("f32", 64, 32), ("f32", 128, 64), ("bf16", 64, 64), ("f32", 16, 16)])
def test_input_stage_pass_then_forward(dtype, d, chunk):
    """Shapes outside the two-kernel forward run the input stage as a pass of its own, then the
    CUDA-core forward."""
    check_forward(fwd_inputs(2, 150, 3, d, dtype, seed=131 + d + chunk), dtype, chunk,
                  label="%s d%d C%d" % (dtype, d, chunk))


def test_single_kernel_fallback(monkeypatch):
    monkeypatch.setenv("GDN_FORWARD_PATH", "fused")
    check_forward(fwd_inputs(1, 200, 2, 128, "bf16", seed=141), "bf16", 64, label="fused")


def test_host_buffers():
    check_forward(fwd_inputs(1, 130, 2, 128, "bf16", seed=151), "bf16", 64, host=True, label="host")


def test_unit_rows_and_gate_logits_match_the_plain_forward():
    """On unit-norm rows with logits whose gates are given, the raw forward equals the plain one up
    to the rounding of the folded factors."""
    inp = fwd_inputs(2, 256, 4, 128, "bf16", seed=161, zero_rows=0.0)
    qn, kn, la, be = oracle.input_stage(as_f32_numpy(inp["q"]), as_f32_numpy(inp["k"]),
                                        as_f32_numpy(inp["x_alpha"]), as_f32_numpy(inp["x_beta"]))
    d = {n: inp[n].cuda() for n in NAMES}
    S0 = inp["S0"].cuda()
    out_r, S_r = gdn.forward_raw(d["q"], d["k"], d["v"], d["x_alpha"], d["x_beta"], S0, chunk=64)
    # the plain forward on the stage's results (q, k rounded to bf16 on the way)
    qb = torch.from_numpy(qn.astype(np.float32)).to(torch.bfloat16).cuda()
    kb = torch.from_numpy(kn.astype(np.float32)).to(torch.bfloat16).cuda()
    out_p, S_p = gdn.forward(qb, kb, d["v"], torch.from_numpy(la.astype(np.float32)).cuda(),
                             torch.from_numpy(be.astype(np.float32)).cuda(), S0, chunk=64)
    torch.cuda.synchronize()
    assert rel_err(cpu_f64(out_r), cpu_f64(out_p)) <= 2e-2
    assert rel_err(cpu_f64(S_r), cpu_f64(S_p)) <= 2e-2


@pytest.mark.parametrize("lengths", [[1, 63, 64, 65, 200, 0, 130], [300, 7]])
def test_varlen_packed(lengths):
    H, d = 4, 128
    T = sum(lengths)
    inp = raw_inputs((T, H), d, d, "bf16", seed=171 + T, s0_shape=(len(lengths), H, d, d), s0_std=0.1,
                     zero_rows=0.03)
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + n)
    dev = {n: inp[n].cuda() for n in NAMES + ("S0",)}
    out, Sf = gdn.forward_varlen_raw(dev["q"], dev["k"], dev["v"], dev["x_alpha"], dev["x_beta"], cu, dev["S0"],
                                     chunk=64)
    torch.cuda.synchronize()
    ref_o, ref_S = oracle.forward_varlen_raw(*[as_f32_numpy(inp[n]) for n in NAMES], cu,
                                             as_f32_numpy(inp["S0"]).astype(np.float64), oracle_threads())
    assert rel_err(cpu_f64(out), ref_o) <= TOL["bf16"]
    assert rel_err(cpu_f64(Sf), ref_S) <= TOL["bf16"]


def test_varlen_per_sequence_fallback():
    lengths, H, d = [40, 0, 77], 3, 64
    T = sum(lengths)
    inp = raw_inputs((T, H), d, d, "f32", seed=181, s0_shape=(3, H, d, d), s0_std=0.2, zero_rows=0.03)
    cu = [0, 40, 40, 117]
    dev = {n: inp[n].cuda() for n in NAMES + ("S0",)}
    out, Sf = gdn.forward_varlen_raw(dev["q"], dev["k"], dev["v"], dev["x_alpha"], dev["x_beta"], cu, dev["S0"],
                                     chunk=32)
    torch.cuda.synchronize()
    ref_o, ref_S = oracle.forward_varlen_raw(*[as_f32_numpy(inp[n]) for n in NAMES], cu,
                                             as_f32_numpy(inp["S0"]).astype(np.float64), oracle_threads())
    assert rel_err(cpu_f64(out), ref_o) <= TOL["f32"]
    assert rel_err(cpu_f64(Sf), ref_S) <= TOL["f32"]


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 32), ("f32", 128)])
def test_decode_steps(dtype, d):
    """Three raw decode steps in a row against the oracle's raw decode, state carried on both sides."""
    steps, B, H = 3, 4, 8
    inp = raw_inputs((steps, B, H), d, d, dtype, seed=191 + d, s0_shape=(B, H, d, d), s0_std=0.05,
                     zero_rows=0.05)
    S = inp["S0"].cuda()
    S_ref = as_f32_numpy(inp["S0"]).astype(np.float64)
    for t in range(steps):
        x = {n: inp[n][t].contiguous() for n in NAMES}
        out = gdn.decode_step_raw(*[x[n].cuda() for n in NAMES], S)
        torch.cuda.synchronize()
        ref = oracle.decode_step_raw(*[as_f32_numpy(x[n]) for n in NAMES], S_ref)
        assert rel_err(cpu_f64(out), ref) <= TOL[dtype], t
    assert rel_err(cpu_f64(S), S_ref) <= TOL[dtype]
