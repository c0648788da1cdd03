"""Seeded synthetic inputs for the gated delta rule.

This module is shared by the tests, the benchmark and the smoke check.  It
only draws random numbers and shapes them into the input distributions of
the named workloads; it contains none of the recurrence's arithmetic, and it
imports neither the CUDA library nor the oracle.

Draw order for a forward workload (one ``torch.Generator('cpu')`` seeded with
``seed``, all draws float32): q, k, v, x_beta, x_alpha, S0.
  * q, k ~ N(0, 1), each row L2-normalised in float32, then cast to the
    workload dtype (the cast values are what both sides consume);
  * v ~ N(0, 1), cast to the workload dtype;
  * beta = sigmoid(x_beta), x_beta ~ N(0, 1)                   (float32)
  * log_alpha = -softplus(x_alpha), x_alpha ~ N(alpha_mu, 1)     (float32)
  * S0 ~ N(0, s0_std) (float32, standard deviation s0_std) or absent.
The decode workload draws, per step in step order, q, k, v, x_beta, x_alpha
the same way (stacked over steps), after the initial state S.

Raw inputs (for the entry points that run the input stage themselves) draw
q, k, v, x_beta, x_alpha, a row scale for q and one for k, then S0:
  * q, k ~ N(0, 1) times a per-row scale log-uniform in [1/20, 20], with a
    fraction ``zero_rows`` of the rows set to zero; cast to the dtype;
  * v ~ N(0, 1); x_beta ~ N(0, 2); x_alpha ~ N(alpha_mu, 2) (float32 logits).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str                 # "forward" or "decode"
    dtype: str                # "f32" or "bf16" (q, k, v, out)
    B: int
    H: int
    dk: int
    dv: int
    T: int = 0                # forward length
    chunk: int = 64
    steps: int = 0            # decode steps
    s0_std: Optional[float] = None
    alpha_mu: float = 0.0
    seed: int = 0
    describe: str = field(default="", compare=False)


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("fwd_f32_b1h2_t64_d16_c16", "forward", "f32", B=1, H=2, dk=16, dv=16, T=64, chunk=16,
                 seed=0, describe="fp32, B=1 H=2 T=64 dk=dv=16 chunk=16, S0=0"),
        Workload("fwd_bf16_b8h16_t2k_d128", "forward", "bf16", B=8, H=16, dk=128, dv=128, T=2048, chunk=64,
                 s0_std=0.02, seed=1, describe="bf16 in / fp32 state, B=8 H=16 T=2048 d=128 chunk=64, S0~N(0,0.02)"),
        Workload("fwd_bf16_b1h16_t64k_d128", "forward", "bf16", B=1, H=16, dk=128, dv=128, T=65536, chunk=64,
                 alpha_mu=-3.0, seed=2, describe="bf16, B=1 H=16 T=65536 d=128 chunk=64, slow decay"),
        Workload("fwd_bf16_b1h16_t256k_d128", "forward", "bf16", B=1, H=16, dk=128, dv=128, T=262144, chunk=64,
                 alpha_mu=-3.0, seed=3, describe="bf16, B=1 H=16 T=262144 d=128 chunk=64, slow decay, S_T"),
        Workload("decode_bf16_b64h16_d128_x1024", "decode", "bf16", B=64, H=16, dk=128, dv=128, steps=1024,
                 s0_std=0.02, seed=4, describe="decode, B=64 H=16 d=128, 1024 steps, S~N(0,0.02)"),
        Workload("decode_bf16_b256h16_d128_x256", "decode", "bf16", B=256, H=16, dk=128, dv=128, steps=256,
                 s0_std=0.02, seed=5, describe="decode, B=256 H=16 d=128 (state 268 MB, twice L2), 256 steps"),
    ]
}


def torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def _unit_rows(g: torch.Generator, shape, dtype: torch.dtype) -> torch.Tensor:
    x = torch.randn(shape, generator=g, dtype=torch.float32)
    x.div_(x.norm(dim=-1, keepdim=True).clamp_min(1e-30))
    return x.to(dtype)


def forward_inputs(B: int, T: int, H: int, dk: int, dv: int, dtype: str = "bf16", seed: int = 0,
                   s0_std: Optional[float] = None, alpha_mu: float = 0.0) -> Dict[str, torch.Tensor]:
    """CPU tensors: q, k [B,T,H,dk], v [B,T,H,dv] (dtype), log_alpha, beta [B,T,H] fp32,
    S0 [B,H,dv,dk] fp32 or None."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    td = torch_dtype(dtype)
    q = _unit_rows(g, (B, T, H, dk), td)
    k = _unit_rows(g, (B, T, H, dk), td)
    v = torch.randn((B, T, H, dv), generator=g, dtype=torch.float32).to(td)
    beta = torch.sigmoid(torch.randn((B, T, H), generator=g, dtype=torch.float32))
    log_alpha = -torch.nn.functional.softplus(
        torch.randn((B, T, H), generator=g, dtype=torch.float32) + alpha_mu)
    S0 = None
    if s0_std is not None:
        S0 = torch.randn((B, H, dv, dk), generator=g, dtype=torch.float32) * s0_std
    return {"q": q, "k": k, "v": v, "log_alpha": log_alpha, "beta": beta, "S0": S0}


def decode_inputs(steps: int, B: int, H: int, dk: int, dv: int, dtype: str = "bf16", seed: int = 0,
                  s0_std: float = 0.02, alpha_mu: float = 0.0) -> Dict[str, torch.Tensor]:
    """CPU tensors: S [B,H,dv,dk] fp32; q, k [steps,B,H,dk], v [steps,B,H,dv] (dtype);
    log_alpha, beta [steps,B,H] fp32."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    td = torch_dtype(dtype)
    S = torch.randn((B, H, dv, dk), generator=g, dtype=torch.float32) * s0_std
    q = _unit_rows(g, (steps, B, H, dk), td)
    k = _unit_rows(g, (steps, B, H, dk), td)
    v = torch.randn((steps, B, H, dv), generator=g, dtype=torch.float32).to(td)
    beta = torch.sigmoid(torch.randn((steps, B, H), generator=g, dtype=torch.float32))
    log_alpha = -torch.nn.functional.softplus(
        torch.randn((steps, B, H), generator=g, dtype=torch.float32) + alpha_mu)
    return {"S": S, "q": q, "k": k, "v": v, "log_alpha": log_alpha, "beta": beta}


def varlen_inputs(lengths, H: int, dk: int, dv: int, dtype: str = "bf16", seed: int = 0,
                  s0_std: Optional[float] = None, alpha_mu: float = 0.0) -> Dict[str, object]:
    """Packed sequences of the given lengths: CPU tensors q, k [T,H,dk], v [T,H,dv] (dtype),
    log_alpha, beta [T,H] fp32 (drawn as one forward_inputs sequence of T = sum(lengths)
    tokens), S0 [N,H,dv,dk] fp32 or None, and cu_seqlens, a list of N + 1 offsets."""
    lengths = [int(x) for x in lengths]
    T = sum(lengths)
    d = forward_inputs(1, T, H, dk, dv, dtype, seed, None, alpha_mu)
    out: Dict[str, object] = {n: d[n][0] for n in ("q", "k", "v", "log_alpha", "beta")}
    out["S0"] = None
    if s0_std is not None:
        g = torch.Generator(device="cpu")
        g.manual_seed(seed + 1)
        out["S0"] = torch.randn((len(lengths), H, dv, dk), generator=g, dtype=torch.float32) * s0_std
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + n)
    out["cu_seqlens"] = cu
    return out


def raw_inputs(shape, dk: int, dv: int, dtype: str = "bf16", seed: int = 0, s0_shape=None,
               s0_std: Optional[float] = None, alpha_mu: float = 0.0, zero_rows: float = 0.0) -> Dict[str, object]:
    """CPU tensors for the raw-input entry points, `shape` the (token, head) grid ([B,T,H],
    [T,H] or [B,H]): q, k [*shape, dk] and v [*shape, dv] (dtype, q and k not normalised),
    x_alpha, x_beta [*shape] float32 gate logits, S0 of `s0_shape` (N(0, s0_std)) or None."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    td = torch_dtype(dtype)
    shape = tuple(int(x) for x in shape)
    q = torch.randn(shape + (dk,), generator=g, dtype=torch.float32)
    k = torch.randn(shape + (dk,), generator=g, dtype=torch.float32)
    v = torch.randn(shape + (dv,), generator=g, dtype=torch.float32).to(td)
    x_beta = torch.randn(shape, generator=g, dtype=torch.float32) * 2.0
    x_alpha = torch.randn(shape, generator=g, dtype=torch.float32) * 2.0 + alpha_mu
    for x in (q, k):
        u = torch.rand(shape + (1,), generator=g, dtype=torch.float32)
        x.mul_(torch.exp((u * 2.0 - 1.0) * 2.9957323))  # 20 ** (2u - 1)
        if zero_rows > 0:
            x.mul_((torch.rand(shape + (1,), generator=g, dtype=torch.float32) >= zero_rows).to(torch.float32))
    S0 = None
    if s0_std is not None and s0_shape is not None:
        S0 = torch.randn(tuple(s0_shape), generator=g, dtype=torch.float32) * s0_std
    return {"q": q.to(td), "k": k.to(td), "v": v, "x_alpha": x_alpha, "x_beta": x_beta, "S0": S0}


def length_mix(n: int, lo: int, hi: int, seed: int = 0):
    """n sequence lengths drawn log-uniformly from [lo, hi] (a prefill batch of mixed requests)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    u = torch.rand((n,), generator=g, dtype=torch.float64)
    return [int(round(lo * (hi / lo) ** float(x))) for x in u]


def workload_inputs(w: Workload, steps: Optional[int] = None) -> Dict[str, torch.Tensor]:
    if w.kind == "forward":
        return forward_inputs(w.B, w.T, w.H, w.dk, w.dv, w.dtype, w.seed, w.s0_std, w.alpha_mu)
    return decode_inputs(steps or w.steps, w.B, w.H, w.dk, w.dv, w.dtype, w.seed, w.s0_std or 0.02, w.alpha_mu)


def as_f32_numpy(t: Optional[torch.Tensor]):
    """Exact float32 numpy view of an fp32 or bf16 tensor (None passes through)."""
    if t is None:
        return None
    return t.detach().to("cpu", torch.float32).contiguous().numpy()
