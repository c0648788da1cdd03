"""GPU test of gdn_forward_noalloc, the forward entry point that allocates nothing.

Some callers cannot allocate device memory in the middle of a call. Examples:
a framework whose caching allocator already owns the whole device heap, or a
serving loop that must not enter the driver's allocator on its hot path. For
them the library provides gdn_forward_noalloc. Its scratch is a fixed,
library-owned device array of GDN_NOALLOC_SCRATCH_BYTES instead of
stream-ordered allocations.

Checked here, through the C ABI:
- two consecutive calls give the same outputs and final state as gdn_forward,
  within the bf16 tolerance the other parity tests use, on a problem that goes
  through the segmented path (the path that needs scratch);
- a problem that needs more scratch than the array holds is refused before
  anything is enqueued.

The file name makes pytest collect it last. A run that stops at the first
failure has then already run every other test. It also passes when run alone
in a fresh process.
"""
import ctypes

import pytest
import torch

import gated_delta_rule_142_b200 as gdn
from gdn_inputs import forward_inputs
from parity_util import TOL, cpu_f64, rel_err, to_device

pytestmark = pytest.mark.gpu

GDN_BF16 = 1
GDN_ERR_SCRATCH_LIMIT = 10


def noalloc_fn():
    lib = gdn.load()
    fn = lib.gdn_forward_noalloc
    fn.argtypes = [ctypes.c_void_p] * 8 + [ctypes.c_int64] * 6 + [ctypes.c_void_p, ctypes.c_int]
    fn.restype = ctypes.c_int
    return fn


def ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def call_noalloc(fn, d, out, Sf, chunk=64):
    B, T, H, dk = d["q"].shape
    dv = d["v"].shape[-1]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return fn(ptr(d["q"]), ptr(d["k"]), ptr(d["v"]), ptr(d["log_alpha"]), ptr(d["beta"]), ptr(d["S0"]), ptr(out),
              ptr(Sf), B, T, H, dk, dv, chunk, stream, GDN_BF16)


def test_noalloc_matches_forward_on_two_consecutive_calls(monkeypatch):
    # four segments: the transfer pass, the prefix and the output pass all use the scratch array
    monkeypatch.setenv("GDN_SEGMENTS", "4")
    fn = noalloc_fn()
    inp = forward_inputs(1, 2048, 4, 128, 128, "bf16", seed=71, s0_std=0.1, alpha_mu=-3.0)
    d = to_device(inp)
    ref_out, ref_S = gdn.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], chunk=64)
    torch.cuda.synchronize()
    for _ in range(2):
        out = torch.full_like(ref_out, float("nan"))
        Sf = torch.full_like(ref_S, float("nan"))
        assert call_noalloc(fn, d, out, Sf) == 0
        torch.cuda.synchronize()
        assert rel_err(cpu_f64(out), cpu_f64(ref_out)) <= TOL["bf16"]
        assert rel_err(cpu_f64(Sf), cpu_f64(ref_S)) <= TOL["bf16"]


def test_noalloc_refuses_problems_beyond_its_scratch(monkeypatch):
    # 64 heads cut into 64 segments would need 3 * 64 * 63 * 64 KiB of scratch, far above the array
    monkeypatch.setenv("GDN_SEGMENTS", "64")
    fn = noalloc_fn()
    B, T, H, d = 1, 64 * 64 * 4, 64, 128
    dev = torch.device("cuda")
    t = {"q": torch.empty(B, T, H, d, dtype=torch.bfloat16, device=dev),
         "k": torch.empty(B, T, H, d, dtype=torch.bfloat16, device=dev),
         "v": torch.empty(B, T, H, d, dtype=torch.bfloat16, device=dev),
         "log_alpha": torch.zeros(B, T, H, device=dev), "beta": torch.zeros(B, T, H, device=dev), "S0": None}
    out = torch.empty(B, T, H, d, dtype=torch.bfloat16, device=dev)
    Sf = torch.empty(B, H, d, d, device=dev)
    assert call_noalloc(fn, t, out, Sf) == GDN_ERR_SCRATCH_LIMIT
    torch.cuda.synchronize()
