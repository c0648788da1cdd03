"""GPU parity of gdn_forward_conv: the short causal convolution of q, k and v
(ATMA, Sec. 3: depthwise causal "Canon" convolutions in front of the memory),
then the raw forward (the input stage of the same section, and the Sec. 3.3
memory).

The float64 reference is the composition of the oracle's two parts:
oracle.causal_conv on each of q, k, v with its carried state, then
oracle.forward_raw on the results.  The call runs the three convolutions as
one launch into scratch and then the raw forward; it must also equal, bit for
bit, the two-step composition through the public calls (gdn_causal_conv on
each tensor, then gdn_forward_raw), since both round the convolution to the
input dtype at the same point.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_142_b200 as gdn
import oracle
from gdn_inputs import as_f32_numpy, raw_inputs
from parity_util import TOL, cpu_f64, oracle_threads, rel_err, to_device

pytestmark = pytest.mark.gpu


def conv_inputs(B, T, H, d, dtype, W, seed, with_state=True):
    r = raw_inputs((B, T, H), d, d, dtype, seed=seed, s0_shape=(B, H, d, d), s0_std=0.1)
    g = torch.Generator().manual_seed(seed + 7)
    w = torch.randn((3, H * d, W), generator=g) * 0.5
    w[:, :, 0] += 1.0  # a residual-like tap, as a trained short convolution tends to have
    st = torch.randn((3, B, W - 1, H * d), generator=g) if with_state else None
    if st is not None:
        st = st.to(torch.bfloat16 if dtype == "bf16" else torch.float32).float()  # the inputs it stands for
    r.update(conv_weight=w, conv_state=st)
    return r


def reference(r, B, T, H, d, W):
    ys, states = [], []
    for i, name in enumerate(("q", "k", "v")):
        x = as_f32_numpy(r[name]).reshape(B, T, H * d).astype(np.float64)
        st = None if r["conv_state"] is None else r["conv_state"][i].numpy().astype(np.float64)
        y, s_after = oracle.causal_conv(x, r["conv_weight"][i].numpy(), st)
        ys.append(y.reshape(B, T, H, d))
        states.append(s_after)
    S0 = None if r["S0"] is None else as_f32_numpy(r["S0"]).astype(np.float64)
    o, S = oracle.forward_raw(ys[0], ys[1], ys[2], as_f32_numpy(r["x_alpha"]), as_f32_numpy(r["x_beta"]), S0,
                              nthreads=oracle_threads())
    return o, S, np.stack(states)


def run_call(d_, chunk=64):
    return gdn.forward_conv(d_["q"], d_["k"], d_["v"], d_["x_alpha"], d_["x_beta"], d_["conv_weight"],
                            d_["conv_state"], d_["S0"], chunk=chunk)


@pytest.mark.parametrize("T,W,nseg,with_state", [
    (300, 4, None, True),
    (300, 4, None, False),
    (257, 3, None, True),
    (130, 2, None, True),
    (64, 1, None, False),
    (1000, 4, "3", True),
    (2048, 4, "4", True),
])
def test_matches_the_composed_oracle(monkeypatch, T, W, nseg, with_state):
    if nseg:
        monkeypatch.setenv("GDN_SEGMENTS", nseg)
    B, H, d = 2, 2, 128
    r = conv_inputs(B, T, H, d, "bf16", W, seed=500 + T + W, with_state=with_state)
    ref_o, ref_S, ref_state = reference(r, B, T, H, d, W)
    out, Sf, st = run_call(to_device(r))
    torch.cuda.synchronize()
    assert rel_err(cpu_f64(out), ref_o) <= TOL["bf16"]
    assert rel_err(cpu_f64(Sf), ref_S) <= TOL["bf16"]
    if W > 1:
        assert np.array_equal(cpu_f64(st), ref_state)  # the carried inputs are copies: exact


@pytest.mark.parametrize("T,nseg", [(300, None), (1000, "3")])
def test_bit_identical_to_conv_then_raw_forward(monkeypatch, T, nseg):
    """The one-launch convolution computes and rounds exactly as gdn_causal_conv does, so the call and
    the composition of public calls on the GPU give identical bits."""
    if nseg:
        monkeypatch.setenv("GDN_SEGMENTS", nseg)
    B, H, d, W = 1, 3, 128, 4
    r = conv_inputs(B, T, H, d, "bf16", W, seed=600 + T)
    g = to_device(r)
    out, Sf, _ = run_call(g)
    ys = []
    for i, name in enumerate(("q", "k", "v")):
        y, _ = gdn.causal_conv(g[name], g["conv_weight"][i].contiguous(), g["conv_state"][i].contiguous(),
                               want_state=False)
        ys.append(y)
    o2, S2 = gdn.forward_raw(ys[0], ys[1], ys[2], g["x_alpha"], g["x_beta"], g["S0"], chunk=64)
    torch.cuda.synchronize()
    assert torch.equal(out, o2)
    assert torch.equal(Sf, S2)


@pytest.mark.parametrize("dtype,d,chunk,tol", [("f32", 64, 32, "f32"), ("bf16", 64, 32, "bf16")])
def test_other_shapes(dtype, d, chunk, tol):
    B, T, H, W = 2, 150, 2, 4
    r = conv_inputs(B, T, H, d, dtype, W, seed=700 + d)
    ref_o, ref_S, ref_state = reference(r, B, T, H, d, W)
    out, Sf, st = run_call(to_device(r), chunk=chunk)
    torch.cuda.synchronize()
    assert rel_err(cpu_f64(out), ref_o) <= TOL[tol]
    assert rel_err(cpu_f64(Sf), ref_S) <= TOL[tol]
    assert np.array_equal(cpu_f64(st), ref_state)


def test_state_carried_across_calls_in_place():
    """A sequence cut into calls of 200, 1 and 99 tokens with the convolution state updated in place
    (and the memory state passed on) equals one call over the whole sequence."""
    B, T, H, d, W = 1, 300, 2, 128, 4
    r = conv_inputs(B, T, H, d, "bf16", W, seed=801)
    ref_o, ref_S, ref_state = reference(r, B, T, H, d, W)
    g = to_device(r)
    st = g["conv_state"].clone()
    S = g["S0"].clone()
    outs = []
    for a, b in ((0, 200), (200, 201), (201, 300)):
        sl = {n: g[n][:, a:b].contiguous() for n in ("q", "k", "v", "x_alpha", "x_beta")}
        o, S_new, _ = gdn.forward_conv(sl["q"], sl["k"], sl["v"], sl["x_alpha"], sl["x_beta"], g["conv_weight"], st,
                                       S, chunk=64, conv_state_out=st)
        S = S_new
        outs.append(o)
    torch.cuda.synchronize()
    assert rel_err(cpu_f64(torch.cat(outs, 1)), ref_o) <= TOL["bf16"]
    assert rel_err(cpu_f64(S), ref_S) <= TOL["bf16"]
    assert np.array_equal(cpu_f64(st), ref_state)


def test_empty_sequence_passes_both_states():
    B, H, d, W = 2, 2, 128, 3
    r = conv_inputs(B, 0, H, d, "bf16", W, seed=900)
    out, Sf, st = run_call(to_device(r))
    torch.cuda.synchronize()
    assert out.numel() == 0
    assert torch.equal(Sf.cpu(), r["S0"])
    assert torch.equal(st.cpu(), r["conv_state"])
