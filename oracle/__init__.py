"""float64 CPU oracle for the gated delta rule -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never does, and
this package imports nothing from the product.  It wraps ``gdn_oracle.c``
(plain C, double precision, OpenMP over (batch, head)) through ctypes.

What is computed follows "ATMA: Long-Context Language Modeling via Polar
Attention and Gated-Delta Compression Memory", Sec. 3.3 (the gated-delta
memory equation), with gamma_t renamed alpha_t, M renamed S and r renamed o:

    S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   o_t = S_t q_t.

Array conventions (numpy, C-contiguous):
    q, k [B, T, H, dk] and v [B, T, H, dv] as float32 (bf16 inputs are passed
    as their exact float32 values); log_alpha, beta [B, T, H] float32;
    S0 / S_final [B, H, dv, dk] float64; out [B, T, H, dv] float64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "gdn_oracle.c")
LIBRARY = os.path.join(_HERE, "libgdn_oracle.so")

_i64 = ctypes.c_int64
_ptr = ctypes.c_void_p


def build(src: str = SOURCE, out: str = LIBRARY, force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math: IEEE double throughout)."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    tmp = out + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall", "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    os.replace(tmp, out)
    return out


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(_ptr)


class Oracle:
    """ctypes view of one compiled oracle library (the real one, or a test mutant)."""

    def __init__(self, path: str):
        self.path = path
        self.lib = ctypes.CDLL(path)
        L = self.lib
        L.gdn_oracle_forward.argtypes = [_ptr] * 8 + [_i64] * 5 + [ctypes.c_int]
        L.gdn_oracle_forward_chunked.argtypes = [_ptr] * 8 + [_i64] * 6 + [ctypes.c_int]
        L.gdn_oracle_decode_step.argtypes = [_ptr] * 7 + [_i64] * 4 + [ctypes.c_int]
        L.gdn_oracle_segment_transfer.argtypes = [_ptr] * 6 + [_i64] * 4
        L.gdn_oracle_dense_product.argtypes = [_ptr] * 8 + [_i64] * 3
        L.gdn_oracle_input_stage.argtypes = [_ptr] * 8 + [_i64] * 2
        L.gdn_oracle_forward_raw.argtypes = [_ptr] * 8 + [_i64] * 5 + [ctypes.c_int]
        L.gdn_oracle_decode_step_raw.argtypes = [_ptr] * 7 + [_i64] * 4 + [ctypes.c_int]
        L.gdn_oracle_backward.argtypes = [_ptr] * 14 + [_i64] * 5 + [ctypes.c_int]
        L.gdn_oracle_forward_grouped.argtypes = [_ptr] * 8 + [_i64] * 6 + [ctypes.c_int]
        L.gdn_oracle_backward_chunked.argtypes = [_ptr] * 14 + [_i64] * 6
        for f in ("gdn_oracle_forward", "gdn_oracle_forward_chunked", "gdn_oracle_decode_step",
                  "gdn_oracle_segment_transfer", "gdn_oracle_dense_product", "gdn_oracle_input_stage",
                  "gdn_oracle_forward_raw", "gdn_oracle_decode_step_raw", "gdn_oracle_backward",
                  "gdn_oracle_forward_grouped", "gdn_oracle_backward_chunked"):
            getattr(L, f).restype = ctypes.c_int

    # -- the definition: token-by-token recurrence ---------------------------------
    def forward(self, q, k, v, log_alpha, beta, S0=None, nthreads: int = 0, want_out: bool = True,
                raw: bool = False):
        """Sequential recurrence.  Returns (out [B,T,H,dv] float64 or None, S_final float64).
        raw=True: q, k in any scale and log_alpha, beta holding the gate logits x_alpha, x_beta;
        the input stage (see input_stage) runs first, in float64."""
        q, k, v, la, be = _f32(q), _f32(k), _f32(v), _f32(log_alpha), _f32(beta)
        B, T, H, dk = q.shape
        dv = v.shape[-1]
        _check_shapes(q, k, v, la, be, B, T, H, dk, dv)
        S0 = None if S0 is None else _f64(S0)
        if S0 is not None:
            assert S0.shape == (B, H, dv, dk)
        out = np.empty((B, T, H, dv), np.float64) if want_out else None
        Sf = np.empty((B, H, dv, dk), np.float64)
        fn = self.lib.gdn_oracle_forward_raw if raw else self.lib.gdn_oracle_forward
        rc = fn(_p(q), _p(k), _p(v), _p(la), _p(be), _p(S0), _p(out), _p(Sf), B, T, H, dk, dv, nthreads)
        if rc != 0:
            raise RuntimeError("gdn_oracle_forward failed (%d)" % rc)
        return out, Sf

    def input_stage(self, q, k, x_alpha, x_beta):
        """Unit-norm q, k (x / sqrt(|x|^2 + 1e-12) over the last axis), log alpha = -softplus(x_alpha),
        beta = sigmoid(x_beta), all float64, shapes as given."""
        q, k, xa, xb = _f32(q), _f32(k), _f32(x_alpha), _f32(x_beta)
        d = q.shape[-1]
        rows = q.size // d
        assert k.shape == q.shape and xa.size == rows and xb.size == rows
        qn, kn = np.empty(q.shape, np.float64), np.empty(k.shape, np.float64)
        la, be = np.empty(xa.shape, np.float64), np.empty(xb.shape, np.float64)
        rc = self.lib.gdn_oracle_input_stage(_p(q), _p(k), _p(xa), _p(xb), _p(qn), _p(kn), _p(la), _p(be), rows, d)
        if rc != 0:
            raise RuntimeError("gdn_oracle_input_stage failed (%d)" % rc)
        return qn, kn, la, be

    def decode_step(self, q, k, v, log_alpha, beta, S, nthreads: int = 0, raw: bool = False):
        """One token for every (b, h); S [B,H,dv,dk] float64 is updated in place.
        q, k [B,H,dk]; v [B,H,dv]; gates [B,H].  Returns out [B,H,dv] float64.
        raw=True: the input stage first, as in forward()."""
        q, k, v, la, be = _f32(q), _f32(k), _f32(v), _f32(log_alpha), _f32(beta)
        B, H, dk = q.shape
        dv = v.shape[-1]
        assert S.dtype == np.float64 and S.flags.c_contiguous and S.shape == (B, H, dv, dk)
        assert k.shape == (B, H, dk) and v.shape == (B, H, dv) and la.shape == (B, H) and be.shape == (B, H)
        out = np.empty((B, H, dv), np.float64)
        fn = self.lib.gdn_oracle_decode_step_raw if raw else self.lib.gdn_oracle_decode_step
        rc = fn(_p(q), _p(k), _p(v), _p(la), _p(be), _p(S), _p(out), B, H, dk, dv, nthreads)
        if rc != 0:
            raise RuntimeError("gdn_oracle_decode_step failed (%d)" % rc)
        return out

    def backward(self, q, k, v, log_alpha, beta, S0, d_out, dS_final=None, nthreads: int = 0):
        """Reverse mode of the recurrence for the loss L with dL/dout = d_out [B,T,H,dv] and
        dL/dS_final = dS_final [B,H,dv,dk] (None = 0).  Returns float64
        (dq, dk, dv, dlog_alpha, dbeta, dS0) in the layouts of the inputs."""
        q, k, v, la, be = _f32(q), _f32(k), _f32(v), _f32(log_alpha), _f32(beta)
        B, T, H, dk = q.shape
        dv = v.shape[-1]
        _check_shapes(q, k, v, la, be, B, T, H, dk, dv)
        S0 = None if S0 is None else _f64(S0)
        d_out = _f64(d_out)
        assert d_out.shape == (B, T, H, dv)
        dS_final = None if dS_final is None else _f64(dS_final)
        gq, gk = np.empty((B, T, H, dk)), np.empty((B, T, H, dk))
        gv = np.empty((B, T, H, dv))
        gla, gbe = np.empty((B, T, H)), np.empty((B, T, H))
        gS0 = np.empty((B, H, dv, dk))
        rc = self.lib.gdn_oracle_backward(_p(q), _p(k), _p(v), _p(la), _p(be), _p(S0), _p(d_out), _p(dS_final),
                                          _p(gq), _p(gk), _p(gv), _p(gla), _p(gbe), _p(gS0), B, T, H, dk, dv,
                                          nthreads)
        if rc != 0:
            raise RuntimeError("gdn_oracle_backward failed (%d)" % rc)
        return gq, gk, gv, gla, gbe, gS0

    def backward_chunked(self, q, k, v, log_alpha, beta, S0, d_out, dS_final=None, chunk: int = 64):
        """The reverse mode in chunkwise form (the adjoint of each line of the chunk algebra), float64;
        same arguments and results as backward()."""
        q, k, v, la, be = _f32(q), _f32(k), _f32(v), _f32(log_alpha), _f32(beta)
        B, T, H, dk = q.shape
        dv = v.shape[-1]
        _check_shapes(q, k, v, la, be, B, T, H, dk, dv)
        S0 = None if S0 is None else _f64(S0)
        d_out = _f64(d_out)
        dS_final = None if dS_final is None else _f64(dS_final)
        gq, gk = np.empty((B, T, H, dk)), np.empty((B, T, H, dk))
        gv = np.empty((B, T, H, dv))
        gla, gbe = np.empty((B, T, H)), np.empty((B, T, H))
        gS0 = np.empty((B, H, dv, dk))
        rc = self.lib.gdn_oracle_backward_chunked(_p(q), _p(k), _p(v), _p(la), _p(be), _p(S0), _p(d_out),
                                                  _p(dS_final), _p(gq), _p(gk), _p(gv), _p(gla), _p(gbe), _p(gS0),
                                                  B, T, H, dk, dv, chunk)
        if rc != 0:
            raise RuntimeError("gdn_oracle_backward_chunked failed (%d)" % rc)
        return gq, gk, gv, gla, gbe, gS0

    def forward_grouped(self, q, k, v, log_alpha, beta, S0=None, nthreads: int = 0):
        """Grouped heads: q [B,T,Hq,dk]; k [B,T,Hkv,dk], v [B,T,Hkv,dv], gates [B,T,Hkv];
        S0 [B,Hkv,dv,dk].  Query head h reads the memory of key-value head h // (Hq // Hkv).
        Returns (out [B,T,Hq,dv], S_final [B,Hkv,dv,dk]) float64."""
        q, k, v, la, be = _f32(q), _f32(k), _f32(v), _f32(log_alpha), _f32(beta)
        B, T, Hq, dk = q.shape
        Hkv, dv = k.shape[2], v.shape[-1]
        assert k.shape == (B, T, Hkv, dk) and v.shape == (B, T, Hkv, dv)
        assert la.shape == (B, T, Hkv) and be.shape == (B, T, Hkv) and Hq % Hkv == 0
        S0 = None if S0 is None else _f64(S0)
        out = np.empty((B, T, Hq, dv), np.float64)
        Sf = np.empty((B, Hkv, dv, dk), np.float64)
        rc = self.lib.gdn_oracle_forward_grouped(_p(q), _p(k), _p(v), _p(la), _p(be), _p(S0), _p(out), _p(Sf),
                                                 B, T, Hq, Hkv, dk, dv, nthreads)
        if rc != 0:
            raise RuntimeError("gdn_oracle_forward_grouped failed (%d)" % rc)
        return out, Sf

    # -- test-only alternative forms ----------------------------------------------
    def forward_chunked(self, q, k, v, log_alpha, beta, S0=None, chunk: int = 64, nthreads: int = 0):
        """Chunkwise (UT-transform) form of the same recurrence, float64."""
        q, k, v, la, be = _f32(q), _f32(k), _f32(v), _f32(log_alpha), _f32(beta)
        B, T, H, dk = q.shape
        dv = v.shape[-1]
        _check_shapes(q, k, v, la, be, B, T, H, dk, dv)
        S0 = None if S0 is None else _f64(S0)
        out = np.empty((B, T, H, dv), np.float64)
        Sf = np.empty((B, H, dv, dk), np.float64)
        rc = self.lib.gdn_oracle_forward_chunked(_p(q), _p(k), _p(v), _p(la), _p(be), _p(S0), _p(out),
                                                 _p(Sf), B, T, H, dk, dv, chunk, nthreads)
        if rc != 0:
            raise RuntimeError("gdn_oracle_forward_chunked failed (%d)" % rc)
        return out, Sf

    def segment_transfer(self, k, v, log_alpha, beta, chunk: int = 64):
        """Affine transfer (M [dk,dk], Bseg [dv,dk]) of one head's run of tokens: k [T,dk], v [T,dv]."""
        k, v, la, be = _f32(k), _f32(v), _f32(log_alpha), _f32(beta)
        T, dk = k.shape
        dv = v.shape[1]
        M = np.empty((dk, dk), np.float64)
        Bs = np.empty((dv, dk), np.float64)
        rc = self.lib.gdn_oracle_segment_transfer(_p(k), _p(v), _p(la), _p(be), _p(M), _p(Bs), T, dk, dv, chunk)
        if rc != 0:
            raise RuntimeError("gdn_oracle_segment_transfer failed (%d)" % rc)
        return M, Bs

    def dense_product(self, q, k, v, log_alpha, beta, S0=None):
        """Brute-force product form for one head, T <= 16: q,k [T,dk], v [T,dv], S0 [dv,dk]."""
        q, k, v, la, be = _f32(q), _f32(k), _f32(v), _f32(log_alpha), _f32(beta)
        T, dk = q.shape
        dv = v.shape[1]
        S0 = None if S0 is None else _f64(S0)
        out = np.empty((T, dv), np.float64)
        Sf = np.empty((dv, dk), np.float64)
        rc = self.lib.gdn_oracle_dense_product(_p(q), _p(k), _p(v), _p(la), _p(be), _p(S0), _p(out), _p(Sf),
                                               T, dk, dv)
        if rc != 0:
            raise RuntimeError("gdn_oracle_dense_product failed (%d)" % rc)
        return out, Sf


def _check_shapes(q, k, v, la, be, B, T, H, dk, dv):
    assert k.shape == (B, T, H, dk), (k.shape, (B, T, H, dk))
    assert v.shape == (B, T, H, dv)
    assert la.shape == (B, T, H) and be.shape == (B, T, H)


_default: Optional[Oracle] = None


def get() -> Oracle:
    """The oracle built from the committed source (compiled on first use)."""
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def forward(*args, **kw):
    return get().forward(*args, **kw)


def decode_step(*args, **kw):
    return get().decode_step(*args, **kw)


def input_stage(*args, **kw):
    return get().input_stage(*args, **kw)


def forward_raw(q, k, v, x_alpha, x_beta, S0=None, nthreads: int = 0):
    """The input stage, then the recurrence (float64 throughout)."""
    return get().forward(q, k, v, x_alpha, x_beta, S0, nthreads=nthreads, raw=True)


def decode_step_raw(q, k, v, x_alpha, x_beta, S, nthreads: int = 0):
    return get().decode_step(q, k, v, x_alpha, x_beta, S, nthreads=nthreads, raw=True)


def forward_varlen_raw(q, k, v, x_alpha, x_beta, cu_seqlens, S0=None, nthreads: int = 0):
    """forward_varlen with the input stage first."""
    return forward_varlen(q, k, v, x_alpha, x_beta, cu_seqlens, S0, nthreads, raw=True)


def forward_varlen(q, k, v, log_alpha, beta, cu_seqlens, S0=None, nthreads: int = 0, raw: bool = False):
    """Packed sequences: the recurrence run on each sequence i (tokens cu_seqlens[i] ..
    cu_seqlens[i+1]-1) from its own initial state S0[i] (zero when S0 is None), with no state
    passed from one sequence to the next.  q, k [T,H,dk], v [T,H,dv], gates [T,H],
    S0 [N,H,dv,dk].  Returns (out [T,H,dv] float64, S_final [N,H,dv,dk] float64)."""
    o = get()
    T, H, dk = q.shape
    dv = v.shape[-1]
    cu = [int(x) for x in cu_seqlens]
    N = len(cu) - 1
    out = np.zeros((T, H, dv), np.float64)
    Sf = np.zeros((N, H, dv, dk), np.float64)
    for i in range(N):
        a, b = cu[i], cu[i + 1]
        s0 = None if S0 is None else np.asarray(S0[i:i + 1], np.float64)
        if b == a:
            if s0 is not None:
                Sf[i] = s0[0]
            continue
        oi, si = o.forward(q[None, a:b], k[None, a:b], v[None, a:b], log_alpha[None, a:b], beta[None, a:b], s0,
                           nthreads=nthreads, raw=raw)
        out[a:b] = oi[0]
        Sf[i] = si[0]
    return out, Sf


def causal_conv(x, weight, state=None):
    """Depthwise causal convolution, float64 (the short convolution of ATMA Sec. 3 in its plain
    reading): y_t[c] = sum_{j<W} weight[c, j] x_{t-j}[c] over x [B,T,C], the W-1 inputs before
    t = 0 taken from state [B,W-1,C] (oldest first) or zero.  Returns (y, state after: the last
    W-1 inputs)."""
    x = np.asarray(x, np.float64)
    w = np.asarray(weight, np.float64)
    B, T, C = x.shape
    W = w.shape[1]
    hist = np.zeros((B, W - 1, C)) if state is None else np.asarray(state, np.float64)
    xx = np.concatenate([hist, x], axis=1)          # token t of x is xx[:, t + W - 1]
    y = np.zeros((B, T, C))
    for j in range(W):
        y += w[:, j] * xx[:, W - 1 - j: W - 1 - j + T]
    return y, xx[:, T:T + W - 1].copy()


def forward_grouped(*args, **kw):
    return get().forward_grouped(*args, **kw)


def decode_step_grouped(q, k, v, log_alpha, beta, S, nthreads: int = 0):
    """Grouped-heads decode step: the forward over one token.  q [B,Hq,dk], k [B,Hkv,dk],
    v [B,Hkv,dv], gates [B,Hkv]; S [B,Hkv,dv,dk] float64 updated in place.  Returns out [B,Hq,dv]."""
    o, Sf = get().forward_grouped(q[:, None], k[:, None], v[:, None], log_alpha[:, None], beta[:, None], S,
                                  nthreads=nthreads)
    S[...] = Sf
    return o[:, 0]


def backward(*args, **kw):
    return get().backward(*args, **kw)


def forward_chunked(*args, **kw):
    return get().forward_chunked(*args, **kw)
