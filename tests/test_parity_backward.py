"""GPU parity of gdn_backward (reverse mode of the forward) against the float64 oracle's reverse
mode on the same inputs (needs a B200).  Same bar as the forward, per gradient tensor:
max |gpu - ref| / max |ref| <= 1e-4 for float32 inputs, <= 2e-2 for bfloat16 inputs."""
import numpy as np
import pytest
import torch

import gated_delta_rule_142_b200 as gdn
import oracle
from gdn_inputs import as_f32_numpy, forward_inputs
from parity_util import TOL, cpu_f64, oracle_threads, rel_err

pytestmark = pytest.mark.gpu

NAMES = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0")


def grads_in(B, T, H, dv, dk, dtype, seed, final=True):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    d_out = torch.randn((B, T, H, dv), generator=g, dtype=torch.float32).to(td)
    dSf = torch.randn((B, H, dv, dk), generator=g, dtype=torch.float32) if final else None
    return d_out, dSf


def check(inp, d_out, dSf, dtype, chunk, host=False, label=""):
    dev = lambda t: None if t is None else (t.pin_memory() if host else t.cuda())  # noqa: E731
    got = gdn.backward(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), dev(inp["log_alpha"]), dev(inp["beta"]),
                       dev(inp["S0"]), dev(d_out), dev(dSf), chunk=chunk)
    torch.cuda.synchronize()
    S0 = None if inp["S0"] is None else as_f32_numpy(inp["S0"]).astype(np.float64)
    ref = oracle.backward(*[as_f32_numpy(inp[n]) for n in ("q", "k", "v", "log_alpha", "beta")], S0,
                          as_f32_numpy(d_out).astype(np.float64),
                          None if dSf is None else dSf.numpy().astype(np.float64), nthreads=oracle_threads())
    for name, gt, rf in zip(NAMES, got, ref):
        e = rel_err(cpu_f64(gt), rf)
        assert e <= TOL[dtype], "%s %s err %.3e" % (label, name, e)
    return got


@pytest.mark.parametrize("dtype,B,T,H,dk,dv,chunk,s0", [
    ("f32", 1, 64, 2, 16, 16, 16, False),
    ("f32", 2, 100, 3, 32, 64, 32, True),
    ("f32", 1, 130, 2, 128, 128, 64, True),
    ("f32", 1, 47, 2, 64, 16, 16, True),
    ("bf16", 2, 150, 2, 128, 128, 64, True),
    ("bf16", 1, 1, 2, 128, 128, 64, True),
    ("bf16", 2, 77, 3, 64, 128, 32, False),
])
def test_backward_matches_oracle(dtype, B, T, H, dk, dv, chunk, s0):
    inp = forward_inputs(B, T, H, dk, dv, dtype, seed=300 + T + dk + dv, s0_std=0.5 if s0 else None)
    d_out, dSf = grads_in(B, T, H, dv, dk, dtype, seed=400 + T)
    check(inp, d_out, dSf, dtype, chunk, label="%s B%d T%d H%d dk%d dv%d C%d" % (dtype, B, T, H, dk, dv, chunk))


def test_backward_training_shape_sampled_heads():
    """The 2K training shape (B8 H16 d128 C64, bf16): the whole batch on the GPU, the oracle on two
    (b, h) problems cut out of it (heads and batch rows are independent)."""
    B, T, H, d = 8, 2048, 16, 128
    inp = forward_inputs(B, T, H, d, d, "bf16", seed=1, s0_std=0.02)
    d_out, dSf = grads_in(B, T, H, d, d, "bf16", seed=11)
    got = gdn.backward(*[inp[n].cuda() for n in ("q", "k", "v", "log_alpha", "beta", "S0")], d_out.cuda(),
                       dSf.cuda(), chunk=64)
    torch.cuda.synchronize()
    for (b, h) in ((0, 0), (5, 11)):
        sl = lambda t: as_f32_numpy(t[b:b + 1, :, h:h + 1].contiguous())  # noqa: E731
        ref = oracle.backward(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["log_alpha"]), sl(inp["beta"]),
                              inp["S0"][b:b + 1, h:h + 1].numpy().astype(np.float64),
                              sl(d_out).astype(np.float64), dSf[b:b + 1, h:h + 1].numpy().astype(np.float64),
                              nthreads=oracle_threads())
        for i, name in enumerate(NAMES[:5]):
            gt = cpu_f64(got[i])[b:b + 1, :, h:h + 1]
            assert rel_err(gt, ref[i]) <= TOL["bf16"], (b, h, name)
        assert rel_err(cpu_f64(got[5])[b:b + 1, h:h + 1], ref[5]) <= TOL["bf16"], (b, h, "dS0")


def test_simt_recompute_matches(monkeypatch):
    """bf16, d = 128, chunk 64 recomputes the forward on the tensor cores by default; the CUDA-core
    recompute (GDN_BWD_RECOMPUTE=simt) meets the same bar."""
    monkeypatch.setenv("GDN_BWD_RECOMPUTE", "simt")
    inp = forward_inputs(2, 150, 2, 128, 128, "bf16", seed=511, s0_std=0.5)
    d_out, dSf = grads_in(2, 150, 2, 128, 128, "bf16", seed=512)
    check(inp, d_out, dSf, "bf16", 64, label="simt recompute")


def test_chunk_size_does_not_change_the_gradients():
    inp = forward_inputs(1, 100, 2, 32, 32, "f32", seed=501, s0_std=0.3)
    d_out, dSf = grads_in(1, 100, 2, 32, 32, "f32", seed=502)
    a = gdn.backward(*[inp[n].cuda() for n in ("q", "k", "v", "log_alpha", "beta", "S0")], d_out.cuda(),
                     dSf.cuda(), chunk=16)
    b = gdn.backward(*[inp[n].cuda() for n in ("q", "k", "v", "log_alpha", "beta", "S0")], d_out.cuda(),
                     dSf.cuda(), chunk=64)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert rel_err(cpu_f64(x), cpu_f64(y)) <= 1e-5


def test_host_buffers_and_no_final_gradient():
    inp = forward_inputs(1, 70, 2, 64, 64, "f32", seed=503, s0_std=0.2)
    d_out, _ = grads_in(1, 70, 2, 64, 64, "f32", seed=504, final=False)
    check(inp, d_out, None, "f32", 32, host=True, label="host buffers")


def test_empty_sequence_passes_the_final_gradient_through():
    inp = forward_inputs(1, 0, 2, 16, 16, "f32", seed=505, s0_std=0.2)
    d_out, dSf = grads_in(1, 0, 2, 16, 16, "f32", seed=506)
    got = gdn.backward(*[inp[n].cuda() for n in ("q", "k", "v", "log_alpha", "beta", "S0")], d_out.cuda(),
                       dSf.cuda(), chunk=16)
    torch.cuda.synchronize()
    assert torch.equal(got[5].cpu(), dSf)


@pytest.mark.parametrize("B,T,H,s0,final", [(1, 64, 1, True, True), (2, 300, 3, True, False), (1, 1000, 2, False, True),
                                            (3, 128, 4, False, False)])
def test_tensor_core_backward(monkeypatch, B, T, H, s0, final):
    """bf16, d = 128, chunk 64 runs the tensor-core reverse mode (a reverse chain and a
    chunk-parallel gradient pass: two backward launches, where the CUDA-core one takes three with its
    two bf16 casts); whole chunks, ragged last chunks, with and without S0 and dS_final."""
    monkeypatch.delenv("GDN_BWD_PATH", raising=False)
    monkeypatch.delenv("GDN_BWD_RECOMPUTE", raising=False)
    inp = forward_inputs(B, T, H, 128, 128, "bf16", seed=600 + T + H, s0_std=0.5 if s0 else None)
    d_out, dSf = grads_in(B, T, H, 128, 128, "bf16", seed=700 + T, final=final)
    gdn.timing_start()
    try:
        check(inp, d_out, dSf, "bf16", 64, label="tc B%d T%d H%d" % (B, T, H))
    finally:
        kinds = gdn.timing_stop()
    assert kinds["backward"][1] == 2, kinds


def test_tensor_core_and_cuda_core_backward_agree(monkeypatch):
    """The two reverse modes on the same inputs: each meets the bar against the oracle, and they
    agree with each other within it."""
    inp = forward_inputs(2, 200, 2, 128, 128, "bf16", seed=811, s0_std=0.3)
    d_out, dSf = grads_in(2, 200, 2, 128, 128, "bf16", seed=812)
    monkeypatch.delenv("GDN_BWD_PATH", raising=False)
    a = check(inp, d_out, dSf, "bf16", 64, label="tensor cores")
    monkeypatch.setenv("GDN_BWD_PATH", "simt")
    gdn.timing_start()
    try:
        b = check(inp, d_out, dSf, "bf16", 64, label="cuda cores")
    finally:
        kinds = gdn.timing_stop()
    assert kinds["backward"][1] == 3, kinds
    for x, y in zip(a, b):
        assert rel_err(cpu_f64(x), cpu_f64(y)) <= TOL["bf16"]


@pytest.mark.parametrize("final,s0", [(True, True), (False, False)])
def test_tensor_core_backward_segments_negligible_and_exact(monkeypatch, final, s0):
    """A long sequence cut into segments (four here): the reverse chain's transfers, their prefix from
    dS_final, then every segment's walk at once.  Heads 0 and 2 decay fast, so the chunks past the head
    of a segment reach its start scaled by at most e^-40: the zero run walks the head alone and the
    identity run is skipped; heads 1 and 3 keep alpha close to 1, so both runs walk the whole segment
    and the prefix multiplies by the exact transfer.  Ragged last chunk, with and without S0 and
    dS_final; still two backward launches (the transfers are timed as transfer launches)."""
    monkeypatch.setenv("GDN_SEGMENTS", "4")
    monkeypatch.delenv("GDN_BWD_PATH", raising=False)
    monkeypatch.delenv("GDN_BWD_RECOMPUTE", raising=False)
    B, T, H = 1, 64 * 24 + 17, 4
    inp = forward_inputs(B, T, H, 128, 128, "bf16", seed=91, s0_std=0.3 if s0 else None)
    inp["log_alpha"][:, :, 1::2] = -1e-3 * torch.rand(inp["log_alpha"][:, :, 1::2].shape,
                                                       generator=torch.Generator().manual_seed(6))
    d_out, dSf = grads_in(B, T, H, 128, 128, "bf16", seed=92, final=final)
    gdn.timing_start()
    try:
        check(inp, d_out, dSf, "bf16", 64, label="segments final=%s" % final)
    finally:
        kinds = gdn.timing_stop()
    assert kinds["backward"][1] == 2, kinds
    assert kinds["transfer"][1] == 2, kinds  # the recompute's forward transfers and the reverse ones


def test_tensor_core_backward_segments_match_one_walk(monkeypatch):
    """The segmented reverse chain gives the gradients of the single walk (GDN_SEGMENTS=1) to within
    the bf16 bar, both against the oracle."""
    monkeypatch.delenv("GDN_BWD_PATH", raising=False)
    B, T, H = 1, 64 * 20, 2
    inp = forward_inputs(B, T, H, 128, 128, "bf16", seed=93, s0_std=0.1, alpha_mu=-3.0)
    d_out, dSf = grads_in(B, T, H, 128, 128, "bf16", seed=94)
    monkeypatch.setenv("GDN_SEGMENTS", "5")
    a = check(inp, d_out, dSf, "bf16", 64, label="five segments")
    monkeypatch.setenv("GDN_SEGMENTS", "1")
    b = check(inp, d_out, dSf, "bf16", 64, label="one walk")
    for x, y in zip(a, b):
        assert rel_err(cpu_f64(x), cpu_f64(y)) <= TOL["bf16"]


def test_tensor_core_backward_many_segments(monkeypatch):
    """Sixteen segments over 4,000 tokens (63 chunks, ragged last chunk): head 0 decays fast (every reverse
    transfer negligible within a short head of its segment), head 1 keeps alpha close to 1 (every transfer
    exact, the prefix chaining fifteen products)."""
    monkeypatch.setenv("GDN_SEGMENTS", "16")
    monkeypatch.delenv("GDN_BWD_PATH", raising=False)
    monkeypatch.delenv("GDN_BWD_RECOMPUTE", raising=False)
    B, T, H = 1, 4000, 2
    inp = forward_inputs(B, T, H, 128, 128, "bf16", seed=95, s0_std=0.2)
    inp["log_alpha"][:, :, 1] = -1e-3 * torch.rand(inp["log_alpha"][:, :, 1].shape,
                                                    generator=torch.Generator().manual_seed(7))
    d_out, dSf = grads_in(B, T, H, 128, 128, "bf16", seed=96)
    check(inp, d_out, dSf, "bf16", 64, label="sixteen segments")


def test_tensor_core_backward_segments_two_batch_rows(monkeypatch):
    """Segments with two batch rows (the transfer slots, prefix chains and entry adjoints of every
    (b, h)), a ragged last chunk, S0 and dS_final given."""
    monkeypatch.setenv("GDN_SEGMENTS", "5")
    monkeypatch.delenv("GDN_BWD_PATH", raising=False)
    monkeypatch.delenv("GDN_BWD_RECOMPUTE", raising=False)
    B, T, H = 2, 1500, 2
    inp = forward_inputs(B, T, H, 128, 128, "bf16", seed=97, s0_std=0.3, alpha_mu=-4.0)
    d_out, dSf = grads_in(B, T, H, 128, 128, "bf16", seed=98)
    check(inp, d_out, dSf, "bf16", 64, label="segments, two batch rows")
