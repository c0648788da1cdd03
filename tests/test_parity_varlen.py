"""GPU parity of gdn_forward_varlen (packed sequences of different lengths) against the float64
oracle run on each sequence alone (needs a B200).  Same bar as the fixed-length forward:
max |gpu - ref| / max |ref| <= 1e-4 for float32 inputs, <= 2e-2 for bfloat16 inputs."""
import numpy as np
import pytest
import torch

import gated_delta_rule_142_b200 as gdn
import oracle
from gdn_inputs import as_f32_numpy, varlen_inputs
from parity_util import TOL, cpu_f64, rel_err

pytestmark = pytest.mark.gpu


def oracle_varlen(inp):
    args = [as_f32_numpy(inp[n]) for n in ("q", "k", "v", "log_alpha", "beta")]
    S0 = None if inp["S0"] is None else as_f32_numpy(inp["S0"]).astype(np.float64)
    return oracle.forward_varlen(*args, inp["cu_seqlens"], S0)


def run_gpu(inp, chunk, host=False):
    dev = {n: (None if inp[n] is None else (inp[n].pin_memory() if host else inp[n].cuda()))
           for n in ("q", "k", "v", "log_alpha", "beta", "S0")}
    out, Sf = gdn.forward_varlen(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["beta"], inp["cu_seqlens"],
                                 dev["S0"], chunk=chunk)
    torch.cuda.synchronize()
    return out, Sf


def check(inp, dtype, chunk, host=False, label=""):
    out, Sf = run_gpu(inp, chunk, host)
    ref_o, ref_S = oracle_varlen(inp)
    if ref_o.size:
        assert rel_err(cpu_f64(out), ref_o) <= TOL[dtype], label
    assert rel_err(cpu_f64(Sf), ref_S) <= TOL[dtype], label


@pytest.mark.parametrize("lengths", [[1, 63, 64, 65, 200, 0, 130], [300], [64, 64, 64], [129, 5, 77, 1, 256]])
def test_packed_tensor_core_path(lengths):
    """bf16, d = 128, chunk 64: every sequence at once on the two-kernel forward; partial chunks at
    the end of a sequence sit next to the next sequence's tokens in the packed tensor."""
    inp = varlen_inputs(lengths, 4, 128, 128, "bf16", seed=sum(lengths) + len(lengths), s0_std=0.1)
    check(inp, "bf16", 64, label=str(lengths))


def test_equal_lengths_match_the_batched_forward():
    B, T, H = 3, 150, 2
    inp = varlen_inputs([T] * B, H, 128, 128, "bf16", seed=41, s0_std=0.1)
    out_v, S_v = run_gpu(inp, 64)
    d = {n: inp[n].cuda() for n in ("q", "k", "v", "log_alpha", "beta")}
    out_b, S_b = gdn.forward(d["q"].view(B, T, H, 128), d["k"].view(B, T, H, 128), d["v"].view(B, T, H, 128),
                             d["log_alpha"].view(B, T, H), d["beta"].view(B, T, H), inp["S0"].cuda(), chunk=64)
    torch.cuda.synchronize()
    assert rel_err(cpu_f64(out_v).reshape(B, T, H, 128), cpu_f64(out_b)) <= 1e-6
    assert rel_err(cpu_f64(S_v), cpu_f64(S_b)) <= 1e-6


@pytest.mark.parametrize("dtype,d,chunk,lengths", [("f32", 64, 32, [5, 70, 0, 33]), ("bf16", 64, 64, [100, 17]),
                                                   ("f32", 128, 64, [65, 3])])
def test_per_sequence_paths(dtype, d, chunk, lengths):
    """Shapes outside the packed tensor-core path run one fixed-length launch per sequence."""
    inp = varlen_inputs(lengths, 3, d, d, dtype, seed=7 + d + chunk, s0_std=0.2)
    check(inp, dtype, chunk, label="%s d%d C%d" % (dtype, d, chunk))


def test_single_kernel_fallback(monkeypatch):
    monkeypatch.setenv("GDN_FORWARD_PATH", "fused")
    inp = varlen_inputs([130, 64, 7], 2, 128, 128, "bf16", seed=43, s0_std=0.1)
    check(inp, "bf16", 64, label="fused per sequence")


def test_host_buffers_and_empty_batch():
    inp = varlen_inputs([65, 10], 2, 128, 128, "bf16", seed=47, s0_std=0.1)
    check(inp, "bf16", 64, host=True, label="host buffers")
    empty = varlen_inputs([0, 0], 2, 128, 128, "bf16", seed=49, s0_std=0.3)
    out, Sf = run_gpu(empty, 64)
    assert out.shape == (0, 2, 128)
    assert torch.equal(Sf.cpu(), empty["S0"])


def test_rejects_bad_offsets():
    inp = varlen_inputs([10, 20], 1, 64, 64, "bf16", seed=51)
    d = {n: inp[n].cuda() for n in ("q", "k", "v", "log_alpha", "beta")}
    for cu in ([0, 20, 10], [1, 10, 30], [0, 10, 29]):
        with pytest.raises(gdn.GdnError):
            gdn.forward_varlen(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], cu, chunk=64)


@pytest.mark.parametrize("lengths,nseg,alpha_mu", [
    ([1000, 65, 0, 300, 1], "3", 0.0),      # the 16-chunk sequence cut 6 + 6 + 4, its last chunk partial
    ([768, 768, 64], "4", 0.0),             # whole-chunk sequences cut 3 + 3 + 3 + 3
    ([64 * 40 + 17, 130, 2000], "5", -1.75),  # decay that makes some transfers negligible, not all
    ([64 * 40 + 17, 130, 2000], "5", -3.0),
])
def test_long_sequences_cut_into_segments(monkeypatch, lengths, nseg, alpha_mu):
    """Sequences longer than the segment length run as segments: transfers of every segment but
    the last, a prefix over them from the sequence's S0, and outputs from each segment's entry
    state.  Shorter sequences in the same batch run whole.  GDN_SEGMENTS cuts the longest
    sequence into that many segments."""
    monkeypatch.setenv("GDN_SEGMENTS", nseg)
    inp = varlen_inputs(lengths, 3, 128, 128, "bf16", seed=sum(lengths) + int(nseg), s0_std=0.1, alpha_mu=alpha_mu)
    check(inp, "bf16", 64, label="%s cut %s" % (lengths, nseg))


def test_one_long_sequence_among_short_ones_is_cut_by_the_planner(monkeypatch):
    """Without an override the planner cuts a sequence that would outlast every other SM's work:
    one 16K-token sequence beside three short ones, 4 heads."""
    monkeypatch.delenv("GDN_SEGMENTS", raising=False)
    inp = varlen_inputs([16384 + 33, 100, 2000, 64], 4, 128, 128, "bf16", seed=91, s0_std=0.05, alpha_mu=-3.0)
    gdn.timing_start()
    try:
        check(inp, "bf16", 64, label="planner cut")
    finally:
        kinds = gdn.timing_stop()
    assert {"prep", "transfer", "prefix", "chain"} <= set(kinds), kinds
