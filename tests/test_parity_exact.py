"""Bit-exact GPU parity on inputs whose exact result every path represents.

ATMA, Sec. 3.3 (gated-delta memory equation).  With orthonormal keys
k_t = s_t e_{i_t} (s_t = +-1, every key index used at most once), alpha = 1
and beta_t in {1/4, 1/2, 3/4, 1}, the update touches one column of the state:

    S_t[:, i_t] = (1 - beta_t) S_{t-1}[:, i_t] + beta_t s_t v_t,  other columns unchanged,

and with one-hot queries q_t = r_t e_{j_t} the output is o_t = r_t S_t[:, j_t].
With S0 and v on the 1/16 grid inside [-2, 2], every intermediate of the
chunkwise algorithm is a dyadic rational of at most 8 significant bits:
  * K K^T is the identity, so A = 0 and T = (I + A)^{-1} = I exactly;
  * the decays are e^0 = 1;
  * W = diag(beta) K, Ut = diag(beta) V, and U = Ut - W S^T = beta (v - s S0[:, i])
    on the 1/64 grid with |numerator| <= 256;
  * the state and the outputs on the 1/64 grid within [-3.5, 3.5].
All of these are exact in bfloat16, and their products and sums are exact in
float32.  So the bfloat16 tensor-core path (bf16 operands, float32
accumulation), its segmented form, the single-kernel form, the CUDA-core path
and decode must reproduce the float64 oracle bit for bit: the outputs equal
the oracle's values (which this test first checks are representable in the
output dtype) and the final state equals them in float32.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_142_b200 as gdn
from parity_util import oracle_forward, to_device


def dyadic_inputs(B, T, H, dk, dv, dtype, seed):
    assert T <= dk, "every key index is used at most once"
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    td = {"f32": torch.float32, "bf16": torch.bfloat16}[dtype]
    k = torch.zeros(B, T, H, dk)
    q = torch.zeros(B, T, H, dk)
    for b in range(B):
        for h in range(H):
            perm = torch.randperm(dk, generator=g)[:T]
            sk = torch.randint(0, 2, (T,), generator=g) * 2 - 1
            jq = torch.randint(0, dk, (T,), generator=g)
            sq = torch.randint(0, 2, (T,), generator=g) * 2 - 1
            k[b, torch.arange(T), h, perm] = sk.float()
            q[b, torch.arange(T), h, jq] = sq.float()
    v = torch.randint(-32, 33, (B, T, H, dv), generator=g).float() / 16
    beta = torch.randint(1, 5, (B, T, H), generator=g).float() / 4
    S0 = torch.randint(-32, 33, (B, H, dv, dk), generator=g).float() / 16
    return {"q": q.to(td), "k": k.to(td), "v": v.to(td), "log_alpha": torch.zeros(B, T, H), "beta": beta,
            "S0": S0}


def exact_reference(inp, td):
    ref_o, ref_S = oracle_forward(inp)
    o = torch.from_numpy(ref_o)
    # the construction keeps every value representable: rounding to the output dtype changes nothing
    assert torch.equal(o.to(td).double(), o), "oracle outputs not representable in the output dtype"
    assert torch.equal(torch.from_numpy(ref_S).float().double(), torch.from_numpy(ref_S))
    return o.to(td), torch.from_numpy(ref_S).float()


@pytest.mark.gpu
@pytest.mark.parametrize("path,dtype,d,chunk,T,env", [
    ("tensor cores, two kernels", "bf16", 128, 64, 128, {}),
    ("tensor cores, two kernels, ragged tail", "bf16", 128, 64, 100, {}),
    ("tensor cores, segments", "bf16", 128, 64, 128, {"GDN_SEGMENTS": "2"}),
    ("tensor cores, one kernel", "bf16", 128, 64, 128, {"GDN_FORWARD_PATH": "fused"}),
    ("tensor cores, one kernel, segments", "bf16", 128, 64, 128,
     {"GDN_FORWARD_PATH": "fused", "GDN_SEGMENTS": "2"}),
    ("CUDA cores, bf16 inputs", "bf16", 128, 64, 128, {"GDN_FORWARD_PATH": "simt"}),
    ("CUDA cores, float32", "f32", 32, 16, 32, {}),
    ("CUDA cores, float32, d64", "f32", 64, 32, 64, {}),
])
def test_dyadic_orthonormal_keys_bit_exact(monkeypatch, path, dtype, d, chunk, T, env):
    for key, val in env.items():
        monkeypatch.setenv(key, val)
    td = {"f32": torch.float32, "bf16": torch.bfloat16}[dtype]
    inp = dyadic_inputs(2, T, 3, d, d, dtype, seed=900 + T + d)
    ref_o, ref_S = exact_reference(inp, td)
    g = to_device(inp)
    out, Sf = gdn.forward(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], g["S0"], chunk=chunk)
    torch.cuda.synchronize()
    mism_o = int((out.cpu() != ref_o).sum())
    mism_S = int((Sf.cpu() != ref_S).sum())
    assert mism_o == 0 and mism_S == 0, "%s: %d output and %d state elements differ" % (path, mism_o, mism_S)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_dyadic_orthonormal_keys_decode_bit_exact(dtype):
    td = {"f32": torch.float32, "bf16": torch.bfloat16}[dtype]
    T, d = 40, 128
    inp = dyadic_inputs(2, T, 3, d, d, dtype, seed=950)
    ref_o, ref_S = exact_reference(inp, td)
    g = to_device(inp)
    S = g["S0"].clone()
    outs = []
    for t in range(T):
        step = [g[n][:, t].contiguous() for n in ("q", "k", "v", "log_alpha", "beta")]
        outs.append(gdn.decode_step(*step, S))
    torch.cuda.synchronize()
    o = torch.stack(outs, 1).cpu()
    assert int((o != ref_o).sum()) == 0
    assert int((S.cpu() != ref_S).sum()) == 0


def test_dyadic_construction_on_cpu_is_what_the_docstring_says():
    """The construction itself, checked without a GPU: the oracle's state follows the column
    recurrence in the docstring exactly."""
    inp = dyadic_inputs(1, 16, 1, 16, 16, "f32", seed=3)
    ref_o, ref_S = oracle_forward(inp)
    S = inp["S0"][0, 0].double().numpy().copy()
    for t in range(16):
        kt = inp["k"][0, t, 0].double().numpy()
        i = int(np.argmax(np.abs(kt)))
        s = kt[i]
        bt = float(inp["beta"][0, t, 0])
        S[:, i] = (1 - bt) * S[:, i] + bt * s * inp["v"][0, t, 0].double().numpy()
        qt = inp["q"][0, t, 0].double().numpy()
        j = int(np.argmax(np.abs(qt)))
        assert np.array_equal(ref_o[0, t, 0], qt[j] * S[:, j])
    assert np.array_equal(ref_S[0, 0], S)

