"""GPU parity of gdn_causal_conv against the float64 oracle (needs a B200): outputs and the carried
state, every width 1..4, short and multi-tile sequences, with and without history, in place."""
import numpy as np
import pytest
import torch

import gated_delta_rule_142_b200 as gdn
import oracle
from gdn_inputs import as_f32_numpy
from parity_util import cpu_f64, rel_err

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-6, "bf16": 1e-2}  # one rounding of the output to the dtype


def draw(B, T, C, W, dtype, seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    x = torch.randn((B, T, C), generator=g).to(td)
    w = torch.randn((C, W), generator=g)
    s = torch.randn((B, W - 1, C), generator=g)
    return x, w, s


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("W", [1, 2, 3, 4])
@pytest.mark.parametrize("T", [1, 5, 300])
def test_matches_oracle(dtype, W, T):
    B, C = 2, 16 * 128
    x, w, s = draw(B, T, C, W, dtype, seed=800 + 10 * W + T)
    for state in (None, s):
        y, so = gdn.causal_conv(x.cuda(), w.cuda(), None if state is None else state.cuda())
        torch.cuda.synchronize()
        ry, rs = oracle.causal_conv(as_f32_numpy(x), w.numpy(), None if state is None else state.numpy())
        assert rel_err(cpu_f64(y), ry) <= TOL[dtype]
        if W > 1:
            assert rel_err(cpu_f64(so), rs) <= 1e-7  # the state is the inputs themselves


def test_in_place_state_and_decode_steps():
    """Decode carries the state in place, one token per call; a long call in place reads a copy."""
    B, C, W = 3, 512, 4
    x, w, s = draw(B, 40, C, W, "bf16", seed=850)
    ry, rs = oracle.causal_conv(as_f32_numpy(x), w.numpy(), s.numpy())
    st = s.clone().cuda()
    wd = w.cuda()
    ys = []
    for t in range(40):
        y, _ = gdn.causal_conv(x[:, t:t + 1].contiguous().cuda(), wd, st, state_out=st)
        ys.append(y)
    torch.cuda.synchronize()
    assert rel_err(cpu_f64(torch.cat(ys, 1)), ry) <= TOL["bf16"]
    assert rel_err(cpu_f64(st), rs) <= 1e-7
    x2, _, _ = draw(B, 700, C, W, "bf16", seed=851)
    st2 = s.clone().cuda()
    y2, _ = gdn.causal_conv(x2.cuda(), wd, st2, state_out=st2)
    torch.cuda.synchronize()
    ry2, rs2 = oracle.causal_conv(as_f32_numpy(x2), w.numpy(), s.numpy())
    assert rel_err(cpu_f64(y2), ry2) <= TOL["bf16"] and rel_err(cpu_f64(st2), rs2) <= 1e-7


def test_empty_sequence_passes_the_state_through():
    x, w, s = draw(2, 0, 64, 3, "f32", seed=860)
    y, so = gdn.causal_conv(x.cuda(), w.cuda(), s.cuda())
    torch.cuda.synchronize()
    assert y.shape == (2, 0, 64) and torch.equal(so.cpu(), s)


@pytest.mark.parametrize("dtype,C", [("bf16", 100), ("f32", 66), ("bf16", 2056)])
def test_channel_counts_of_either_kernel(dtype, C):
    """Channel counts that are not a whole number of 16-byte words take the one-channel kernel; the
    others take the wide one (2056 bf16 channels: 257 words).  Tokens 130 = two 64-token tiles and a
    ragged third."""
    B, T, W = 2, 130, 4
    x, w, s = draw(B, T, C, W, dtype, seed=870 + C)
    y, so = gdn.causal_conv(x.cuda(), w.cuda(), s.cuda())
    torch.cuda.synchronize()
    ry, rs = oracle.causal_conv(as_f32_numpy(x), w.numpy(), s.numpy())
    assert rel_err(cpu_f64(y), ry) <= TOL[dtype]
    assert rel_err(cpu_f64(so), rs) <= 1e-7


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_wide_and_one_channel_kernels_give_identical_bits(dtype):
    """The same input at a 16-byte aligned address (wide kernel) and one element past it (one-channel
    kernel): both compute w0 x_t first and then the older inputs, so the outputs are bit-identical."""
    B, T, C, W = 2, 257, 1024, 4
    x, w, s = draw(B, T, C, W, dtype, seed=880)
    xa = x.cuda()
    buf = torch.empty(x.numel() + 8, dtype=x.dtype, device="cuda")
    xm = buf[1:1 + x.numel()].view(B, T, C)
    xm.copy_(xa)
    ybuf = torch.empty_like(buf)
    ym = ybuf[1:1 + x.numel()].view(B, T, C)
    assert xm.data_ptr() % 16 != 0 and ym.data_ptr() % 16 != 0
    y1, s1 = gdn.causal_conv(xa, w.cuda(), s.cuda())
    _, s2 = gdn.causal_conv(xm, w.cuda(), s.cuda(), out=ym)
    torch.cuda.synchronize()
    assert torch.equal(y1, ym)
    assert torch.equal(s1, s2)
