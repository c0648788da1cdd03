"""GPU test of gdn_forward_noalloc, the forward entry point that allocates nothing.

Some callers cannot allocate device memory in the middle of a call. Examples:
a framework whose caching allocator already owns the whole device heap, or a
serving loop that must not enter the driver's allocator on its hot path. For
them the library provides gdn_forward_noalloc. Its scratch is a fixed,
library-owned device array of GDN_NOALLOC_SCRATCH_BYTES (32 MiB) instead of
stream-ordered allocations.

Checked here, through the C ABI, against the float64 oracle (not against
gdn_forward, so that an error the two entry points shared would still show):
- the two-kernel path (its per-chunk workspace and the segment scratch in the
  array): two checked calls on the same problem, with a call on an unrelated
  problem (another seed, another segment count) between them, so that the
  second checked call starts from array contents it did not write itself;
- the single-kernel path that problems whose per-chunk workspace exceeds the
  array take, with its segment transfers, prefix and entry states in the
  array;
- a long sequence whose planned segment scratch exceeds the array runs with
  fewer segments instead, and a segment count forced beyond the array is
  refused before anything is enqueued.

The file name makes pytest collect it last. A run that stops at the first
failure has then already run every other test. It also passes when run alone
in a fresh process.
"""
import ctypes

import pytest
import torch

import gated_delta_rule_142_b200 as gdn
from gdn_inputs import forward_inputs
from parity_util import TOL, cpu_f64, oracle_forward, rel_err, to_device

pytestmark = pytest.mark.gpu

GDN_BF16 = 1
GDN_ERR_SCRATCH_LIMIT = 10
SCRATCH_BYTES = 32 << 20


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


def run_noalloc(fn, d):
    B, T, H, _ = d["q"].shape
    out = torch.full((B, T, H, d["v"].shape[-1]), float("nan"), dtype=d["q"].dtype, device="cuda")
    Sf = torch.full((B, H, d["v"].shape[-1], d["q"].shape[-1]), float("nan"), device="cuda")
    assert call_noalloc(fn, d, out, Sf) == 0
    torch.cuda.synchronize()
    return out, Sf


def check_against_oracle(inp, out, Sf, heads=None):
    ref_o, ref_S = oracle_forward(inp, heads=heads)
    o, S = cpu_f64(out), cpu_f64(Sf)
    if heads is not None:
        o, S = o[:, :, list(heads)], S[:, list(heads)]
    assert rel_err(o, ref_o) <= TOL["bf16"]
    assert rel_err(S, ref_S) <= TOL["bf16"]


def test_noalloc_two_kernel_path_with_unrelated_call_between(monkeypatch):
    fn = noalloc_fn()
    inp = forward_inputs(1, 2048, 4, 128, 128, "bf16", seed=71, s0_std=0.1, alpha_mu=-3.0)
    other = forward_inputs(2, 1500, 3, 128, 128, "bf16", seed=72, s0_std=0.3)
    d, d_other = to_device(inp), to_device(other)
    # four segments: the per-chunk workspace, the transfers, the prefix and the entry states all sit in
    # the array (about 4.2 MB of workspace and 2.3 MB of segment scratch)
    monkeypatch.setenv("GDN_SEGMENTS", "4")
    out, Sf = run_noalloc(fn, d)
    check_against_oracle(inp, out, Sf)
    # an unrelated problem with another segment count overwrites the array with its own data
    monkeypatch.setenv("GDN_SEGMENTS", "3")
    o2, S2 = run_noalloc(fn, d_other)
    check_against_oracle(other, o2, S2)
    monkeypatch.setenv("GDN_SEGMENTS", "4")
    out, Sf = run_noalloc(fn, d)
    check_against_oracle(inp, out, Sf)


def test_noalloc_single_kernel_path_when_the_workspace_does_not_fit(monkeypatch):
    # 4 heads x 512 chunks of 32.5 KB workspace = 68 MB > 32 MiB: the single-kernel forward runs, with
    # its 4-segment transfers, prefix and entry states (2.4 MB) in the array
    B, T, H = 1, 32768, 4
    assert H * (T // 64) * (32768 + 528) > SCRATCH_BYTES
    monkeypatch.setenv("GDN_SEGMENTS", "4")
    fn = noalloc_fn()
    inp = forward_inputs(B, T, H, 128, 128, "bf16", seed=74, s0_std=0.05, alpha_mu=-3.0)
    d = to_device(inp)
    out, Sf = run_noalloc(fn, d)
    check_against_oracle(inp, out, Sf, heads=[0, 3])


def test_noalloc_lowers_the_segment_count_to_fit(monkeypatch):
    # 8 heads over 256K tokens: the planner's segment scratch (about 37 segments, 57 MB) exceeds the
    # array, so the call runs with the most segments that fit (22) instead of being refused
    monkeypatch.delenv("GDN_SEGMENTS", raising=False)
    fn = noalloc_fn()
    inp = forward_inputs(1, 262144, 8, 128, 128, "bf16", seed=75, alpha_mu=-3.0)
    d = to_device(inp)
    out, Sf = run_noalloc(fn, d)
    check_against_oracle(inp, out, Sf, heads=[6])


def test_noalloc_refuses_a_forced_segment_count_beyond_its_scratch(monkeypatch):
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
