"""Failure detection without a GPU fault (needs a B200).

Device side: every wait in the kernels is bounded; a wait that gives up sets a device error word
that gdn_device_status reports as GDN_ERR_DEVICE_TIMEOUT.  The self-test kernel's bounded wait on an
mbarrier phase that nothing completes gives up by design: the status is reported once, cleared, and
the context stays usable.  Host side: GDN_TEST_FAIL_ALLOC=1 makes every scratch allocation fail; the
forwards fall back to paths without scratch where one exists and otherwise return GDN_ERR_ALLOC."""
import numpy as np
import pytest
import torch

import gated_delta_rule_142_b200 as gdn
import oracle
from gdn_inputs import as_f32_numpy, forward_inputs, varlen_inputs
from parity_util import TOL, cpu_f64, oracle_threads, rel_err

pytestmark = pytest.mark.gpu

GDN_OK, GDN_ERR_ALLOC, GDN_ERR_DEVICE_TIMEOUT = 0, 5, 7
NAMES = ("q", "k", "v", "log_alpha", "beta")


def forward_matches(inp, chunk=64):
    out, Sf = gdn.forward(*[inp[n].cuda() for n in NAMES], inp["S0"].cuda(), chunk=chunk)
    torch.cuda.synchronize()
    ro, rS = oracle.forward(*[as_f32_numpy(inp[n]) for n in NAMES], as_f32_numpy(inp["S0"]).astype(np.float64),
                            nthreads=oracle_threads())
    assert rel_err(cpu_f64(out), ro) <= TOL["bf16"] and rel_err(cpu_f64(Sf), rS) <= TOL["bf16"]


def test_status_is_clean_after_normal_work():
    forward_matches(forward_inputs(2, 130, 4, 128, 128, "bf16", seed=901, s0_std=0.1))
    assert gdn.device_status() == GDN_OK


def test_a_wait_that_gives_up_is_reported_once_and_the_context_survives():
    gdn.device_status()  # clear anything earlier
    gdn.selftest_device_timeout()
    assert gdn.device_status() == GDN_ERR_DEVICE_TIMEOUT
    assert gdn.device_status() == GDN_OK
    forward_matches(forward_inputs(1, 200, 2, 128, 128, "bf16", seed=902, s0_std=0.1))
    assert gdn.device_status() == GDN_OK


def test_allocation_failure_falls_back_or_reports(monkeypatch):
    monkeypatch.setenv("GDN_TEST_FAIL_ALLOC", "1")
    # the two-kernel forward cannot get its workspace: the single-kernel forward (no scratch) runs
    forward_matches(forward_inputs(2, 130, 4, 128, 128, "bf16", seed=903, s0_std=0.1))
    # packed prefill falls back to one single-kernel launch per sequence
    inp = varlen_inputs([70, 5, 130], 2, 128, 128, "bf16", seed=904, s0_std=0.1)
    out, Sf = gdn.forward_varlen(*[inp[n].cuda() for n in NAMES], inp["cu_seqlens"], inp["S0"].cuda(), chunk=64)
    torch.cuda.synchronize()
    ro, rS = oracle.forward_varlen(*[as_f32_numpy(inp[n]) for n in NAMES], inp["cu_seqlens"],
                                   as_f32_numpy(inp["S0"]).astype(np.float64))
    assert rel_err(cpu_f64(out), ro) <= TOL["bf16"] and rel_err(cpu_f64(Sf), rS) <= TOL["bf16"]
    # host buffers need staging copies; the backward needs its checkpoints: both report GDN_ERR_ALLOC
    host = forward_inputs(1, 64, 2, 64, 64, "f32", seed=905, s0_std=0.1)
    with pytest.raises(gdn.GdnError) as e:
        gdn.forward(*[host[n].pin_memory() for n in NAMES], host["S0"].pin_memory(), chunk=32)
    assert e.value.status == GDN_ERR_ALLOC
    d = {n: host[n].cuda() for n in NAMES}
    with pytest.raises(gdn.GdnError) as e:
        gdn.backward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], host["S0"].cuda(),
                     torch.ones_like(d["v"]), None, chunk=32)
    assert e.value.status == GDN_ERR_ALLOC
    monkeypatch.delenv("GDN_TEST_FAIL_ALLOC")
    forward_matches(forward_inputs(2, 130, 4, 128, 128, "bf16", seed=906, s0_std=0.1))
