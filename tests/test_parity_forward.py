"""GPU parity of gdn_forward against the float64 oracle (needs a B200).

Every case draws seeded inputs, runs the CUDA path through the C ABI (via the
ctypes binding) and compares outputs and final state with the oracle on the
same values: max |gpu - ref| / max |ref| <= 1e-4 for float32 inputs and
<= 2e-2 for bfloat16 inputs.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_142_b200 as gdn
from gdn_inputs import WORKLOADS, forward_inputs, workload_inputs
from parity_util import TOL, cpu_f64, oracle_forward, rel_err, to_device

pytestmark = pytest.mark.gpu


def run_gpu(inp, chunk, S_final=True):
    d = to_device(inp)
    out, Sf = gdn.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], chunk=chunk,
                          output_final_state=S_final)
    torch.cuda.synchronize()
    return out, Sf


def check(inp, dtype, chunk, heads=None, label=""):
    out, Sf = run_gpu(inp, chunk)
    ref_o, ref_S = oracle_forward(inp, heads=heads)
    o = cpu_f64(out)
    S = cpu_f64(Sf)
    if heads is not None:
        o, S = o[:, :, list(heads)], S[:, list(heads)]
    eo, eS = rel_err(o, ref_o), rel_err(S, ref_S)
    assert eo <= TOL[dtype], "%s out err %.3e" % (label, eo)
    assert eS <= TOL[dtype], "%s state err %.3e" % (label, eS)
    return eo, eS


def test_workload_fp32_tiny():
    w = WORKLOADS["fwd_f32_b1h2_t64_d16_c16"]
    check(workload_inputs(w), w.dtype, w.chunk, label=w.name)


@pytest.mark.parametrize("dtype,dk,dv,chunk,T,s0", [
    ("f32", 16, 16, 16, 1, False),
    ("f32", 32, 64, 32, 100, True),
    ("f32", 128, 128, 64, 130, True),
    ("f32", 64, 16, 16, 47, True),
    ("f32", 128, 32, 64, 200, False),
    ("bf16", 128, 128, 64, 130, True),
    ("bf16", 128, 128, 64, 64, False),
    ("bf16", 128, 128, 64, 1, True),
    ("bf16", 64, 128, 32, 77, True),
    ("bf16", 16, 32, 16, 33, False),
    ("bf16", 128, 64, 64, 257, True),
])
def test_small_shapes(dtype, dk, dv, chunk, T, s0):
    inp = forward_inputs(2, T, 3, dk, dv, dtype, seed=100 + T + dk + dv, s0_std=0.5 if s0 else None)
    check(inp, dtype, chunk, label="%s dk%d dv%d C%d T%d" % (dtype, dk, dv, chunk, T))


def test_workload_train_2k_full():
    w = WORKLOADS["fwd_bf16_b8h16_t2k_d128"]
    check(workload_inputs(w), w.dtype, w.chunk, label=w.name)


def test_workload_64k_sampled_heads():
    w = WORKLOADS["fwd_bf16_b1h16_t64k_d128"]
    check(workload_inputs(w), w.dtype, w.chunk, heads=[0, 9], label=w.name)


def test_workload_256k_sampled_head_and_final_state():
    w = WORKLOADS["fwd_bf16_b1h16_t256k_d128"]
    check(workload_inputs(w), w.dtype, w.chunk, heads=[5], label=w.name)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_chunk_size_does_not_change_the_result(dtype):
    inp = forward_inputs(1, 150, 2, 64, 64, dtype, seed=7, s0_std=0.3)
    ref_o, ref_S = oracle_forward(inp)
    outs = []
    for C in (16, 32, 64):
        out, Sf = run_gpu(inp, C)
        assert rel_err(cpu_f64(out), ref_o) <= TOL[dtype]
        assert rel_err(cpu_f64(Sf), ref_S) <= TOL[dtype]
        outs.append(cpu_f64(out))
    assert rel_err(outs[0], outs[2]) <= 2 * TOL[dtype]


def test_empty_and_degenerate_sizes():
    inp = forward_inputs(2, 0, 2, 32, 32, "bf16", seed=3, s0_std=0.5)
    out, Sf = run_gpu(inp, 32)
    assert out.shape == (2, 0, 2, 32)
    assert torch.equal(Sf.cpu(), inp["S0"])
    inp["S0"] = None
    _, Sz = run_gpu(inp, 32)
    assert not Sz.cpu().any()
    inp0 = forward_inputs(0, 8, 2, 32, 32, "bf16", seed=3)
    out0, _ = run_gpu(inp0, 32)
    assert out0.numel() == 0


def test_in_place_state():
    inp = forward_inputs(2, 70, 2, 128, 128, "bf16", seed=11, s0_std=0.1)
    ref_o, ref_S = oracle_forward(inp)
    d = to_device(inp)
    S = d["S0"].clone()
    out, Sf = gdn.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S, chunk=64, S_final=S)
    torch.cuda.synchronize()
    assert Sf.data_ptr() == S.data_ptr()
    assert rel_err(cpu_f64(out), ref_o) <= TOL["bf16"]
    assert rel_err(cpu_f64(S), ref_S) <= TOL["bf16"]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_reset_gate(dtype):
    """alpha = 0 at some tokens (log_alpha = -inf) and a near-reset (-30): the past is erased."""
    inp = forward_inputs(1, 140, 2, 64, 32, dtype, seed=13, s0_std=0.5)
    inp["log_alpha"][0, 5, 0] = float("-inf")
    inp["log_alpha"][0, 63, 1] = float("-inf")
    inp["log_alpha"][0, 64, 0] = -30.0
    inp["log_alpha"][0, 100:103, :] = float("-inf")
    check(inp, dtype, 64, label="reset")


def test_identity_gates_keep_state():
    """alpha = 1, beta = 0: out = S0 q and S_final = S0 (bit-exact for the state)."""
    inp = forward_inputs(1, 96, 2, 32, 32, "f32", seed=17, s0_std=0.5)
    inp["log_alpha"].zero_()
    inp["beta"].zero_()
    out, Sf = run_gpu(inp, 32)
    assert torch.equal(Sf.cpu(), inp["S0"])
    ref = torch.einsum("bhrc,bthc->bthr", inp["S0"].double(), inp["q"].double())
    assert rel_err(cpu_f64(out), ref.numpy()) <= 1e-5


def test_split_continuation():
    """forward(T) == forward(T1) followed by forward(T - T1) from its final state."""
    inp = forward_inputs(2, 200, 2, 128, 128, "bf16", seed=19, s0_std=0.1)
    d = to_device(inp)
    o_full, S_full = gdn.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], chunk=64)
    T1 = 75
    sl = lambda x, a, b: x[:, a:b].contiguous()  # noqa: E731
    o1, S1 = gdn.forward(sl(d["q"], 0, T1), sl(d["k"], 0, T1), sl(d["v"], 0, T1), sl(d["log_alpha"], 0, T1),
                         sl(d["beta"], 0, T1), d["S0"], chunk=64)
    o2, S2 = gdn.forward(sl(d["q"], T1, 200), sl(d["k"], T1, 200), sl(d["v"], T1, 200),
                         sl(d["log_alpha"], T1, 200), sl(d["beta"], T1, 200), S1, chunk=64)
    torch.cuda.synchronize()
    ref_o, ref_S = oracle_forward(inp)
    assert rel_err(cpu_f64(torch.cat([o1, o2], 1)), ref_o) <= TOL["bf16"]
    assert rel_err(cpu_f64(S2), ref_S) <= TOL["bf16"]
    assert rel_err(cpu_f64(S2), cpu_f64(S_full)) <= TOL["bf16"]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_host_buffers_are_staged(dtype):
    """Pinned and pageable host tensors go through the library's staging path."""
    inp = forward_inputs(2, 90, 2, 64, 64, dtype, seed=23, s0_std=0.2)
    ref_o, ref_S = oracle_forward(inp)
    pinned = {k: (None if v is None else v.pin_memory()) for k, v in inp.items()}
    for src in (pinned, inp):
        out, Sf = gdn.forward(src["q"], src["k"], src["v"], src["log_alpha"], src["beta"], src["S0"], chunk=32)
        torch.cuda.synchronize()
        assert out.device.type == "cpu"
        assert rel_err(cpu_f64(out), ref_o) <= TOL[dtype]
        assert rel_err(cpu_f64(Sf), ref_S) <= TOL[dtype]


def test_simt_path_matches_on_the_tensor_core_shape(monkeypatch):
    """The float32 CUDA-core path also serves bf16 inputs; both paths meet the bar."""
    inp = forward_inputs(2, 130, 2, 128, 128, "bf16", seed=29, s0_std=0.1)
    ref_o, ref_S = oracle_forward(inp)
    monkeypatch.setenv("GDN_FORWARD_PATH", "simt")
    out, Sf = run_gpu(inp, 64)
    assert rel_err(cpu_f64(out), ref_o) <= TOL["bf16"]
    assert rel_err(cpu_f64(Sf), ref_S) <= TOL["bf16"]


def test_results_are_deterministic():
    inp = forward_inputs(2, 100, 4, 128, 128, "bf16", seed=31, s0_std=0.1)
    a = run_gpu(inp, 64)
    b = run_gpu(inp, 64)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("nseg", [2, 3, 5])
def test_segmented_long_sequence(monkeypatch, nseg):
    """Sequence cut into segments: transfer pass, float32 prefix over segments, output pass.
    A ragged last chunk and a non-zero initial state are included."""
    monkeypatch.setenv("GDN_SEGMENTS", str(nseg))
    inp = forward_inputs(1, 1000, 2, 128, 128, "bf16", seed=61 + nseg, s0_std=0.1, alpha_mu=-3.0)
    check(inp, "bf16", 64, label="segments=%d" % nseg)


def test_segmented_fast_decay(monkeypatch):
    """Segments with fast decay (alpha ~ 0.45) and resets inside segments."""
    monkeypatch.setenv("GDN_SEGMENTS", "4")
    inp = forward_inputs(2, 777, 2, 128, 128, "bf16", seed=67, s0_std=0.1)
    inp["log_alpha"][0, 300, 1] = float("-inf")
    inp["log_alpha"][1, 500:505, 0] = -30.0
    check(inp, "bf16", 64, label="segments fast decay")


def test_forward_plan_reports_scratch_and_launches(monkeypatch):
    """The planning query agrees with what the forward does.  Two-kernel path: 32.5 KB of workspace
    per chunk and two launches, plus segment scratch and two more launches for a long sequence
    with few heads.  Single-kernel path: no scratch and one launch, or segment scratch and three."""
    per_chunk, seg_unit = 32768 + 528, 3 * 16 * 128 * 128 * 4
    s, n = gdn.forward_plan(8, 2048, 16, 128, 128, 64)
    assert (s, n) == (8 * 16 * 32 * per_chunk, 2)
    s, n = gdn.forward_plan(1, 65536, 16, 128, 128, 64)
    rest = s - 16 * 1024 * per_chunk
    boundaries = rest // seg_unit  # segments - 1, then one int flag per head and boundary (256-byte rounded)
    assert n == 4 and boundaries > 0 and rest - boundaries * seg_unit == -(-16 * boundaries * 4 // 256) * 256
    assert gdn.forward_plan(1, 100, 2, 64, 64, 32) == (0, 1)  # CUDA-core path
    monkeypatch.setenv("GDN_FORWARD_PATH", "fused")
    assert gdn.forward_plan(8, 2048, 16, 128, 128, 64) == (0, 1)
    s, n = gdn.forward_plan(1, 65536, 16, 128, 128, 64)
    assert n == 3 and s > 0 and s % seg_unit == 0


@pytest.mark.parametrize("T,nseg", [(130, 1), (1000, 3)])
def test_single_kernel_path(monkeypatch, T, nseg):
    """The single-kernel tensor-core forward (used when the two-kernel workspace cannot be had)
    meets the same bar, with and without segments."""
    monkeypatch.setenv("GDN_FORWARD_PATH", "fused")
    monkeypatch.setenv("GDN_SEGMENTS", str(nseg))
    inp = forward_inputs(2, T, 2, 128, 128, "bf16", seed=73 + T, s0_std=0.1, alpha_mu=-3.0)
    check(inp, "bf16", 64, label="single kernel T=%d segments=%d" % (T, nseg))


@pytest.mark.parametrize("alpha_mu", [-1.75, -3.0])
def test_segmented_transfers_negligible_and_exact_mixed(monkeypatch, alpha_mu):
    """Segment transfers whose decay makes the entering state negligible (the product of the chunks'
    transfer bounds reaches e^-40 inside the segment: only the segment's tail is run, the identity run
    and the prefix product are skipped) next to heads whose gates barely decay (the exact transfer
    runs), in one launch: heads 0 and 2 decay, heads 1 and 3 keep alpha close to 1."""
    monkeypatch.setenv("GDN_SEGMENTS", "4")
    inp = forward_inputs(1, 64 * 40 + 17, 4, 128, 128, "bf16", seed=81, s0_std=0.1, alpha_mu=alpha_mu)
    inp["log_alpha"][:, :, 1::2] = -1e-3 * torch.rand(inp["log_alpha"][:, :, 1::2].shape,
                                                       generator=torch.Generator().manual_seed(5))
    check(inp, "bf16", 64, label="mixed transfers alpha_mu=%g" % alpha_mu)
