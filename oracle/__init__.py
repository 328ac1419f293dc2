"""FP64 CPU oracle for the gated delta-net scan -- TEST INFRASTRUCTURE.

Only `tests/`, `__graft_entry__.smoke()` and the CPU-baseline leg of
`bench.py` may import this package.  The CUDA library never imports, links
or calls it, and it shares no code with the library: the one thing both
sides use is the seeded input generator (`gated_delta_rule_72_b200.inputs`),
which holds none of the method's arithmetic.

`scan()` runs the plain sequential recurrence of `gdn_oracle.c` in double
precision.  Every input is widened to float64 exactly as given (bf16 and
fp32 values are exactly representable), so the oracle sees the same numbers
as the GPU.  See `gdn_oracle.c` for the definition and the cited passages.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.gdn_oracle_scan.argtypes = [ctypes.c_int] * 6 + [dp] * 6 + [dp] * 2 + [dp] * 3 + [ctypes.c_int]
        lib.gdn_oracle_scan.restype = ctypes.c_int
        _lib = lib
    return _lib


MODES = {"causal": 0, "reverse": 1, "bidir": 2}


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu")
        x = x.double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def scan(q, k, v, alpha, beta, mode="causal", state_in=None, state_in_bwd=None,
         erase=None, write=None, threads=None):
    """Run the recurrence for every (b,h) sequence in float64.

    q,k: [B,T,H,dk]; v: [B,T,H,dv]; alpha, beta: [B,T,H];
    state_in: [B,H,dk,dv] initial causal state (None = zero);
    state_in_bwd: initial reverse state R_{T+1} (None = zero).
    erase / write: optional separate erase and write coefficients (test hook);
    by default both are beta.
    Returns (o [B,T,H,dv], state_out [B,H,dk,dv] or None, state_bwd_out or None)
    as float64 numpy arrays.  state_out is the causal state after token T;
    state_bwd_out the reverse state after token 1.
    """
    lib = _load()
    q, k, v, alpha = _f64(q), _f64(k), _f64(v), _f64(alpha)
    beta = _f64(beta)
    erase = beta if erase is None else _f64(erase)
    write = beta if write is None else _f64(write)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == (B, T, H, dk) and v.shape == (B, T, H, dv)
    assert alpha.shape == (B, T, H) and erase.shape == (B, T, H) and write.shape == (B, T, H)
    m = MODES[mode]
    s0 = _f64(state_in)
    s0b = _f64(state_in_bwd)
    for s in (s0, s0b):
        assert s is None or s.shape == (B, H, dk, dv)
    o = np.zeros((B, T, H, dv), np.float64)
    sf = np.zeros((B, H, dk, dv), np.float64) if m in (0, 2) else None
    sb = np.zeros((B, H, dk, dv), np.float64) if m in (1, 2) else None
    if threads is None:
        threads = os.cpu_count() or 1
    rc = lib.gdn_oracle_scan(B, T, H, dk, dv, m, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                             _ptr(erase), _ptr(write), _ptr(s0), _ptr(s0b), _ptr(o),
                             _ptr(sf), _ptr(sb), int(threads))
    if rc != 0:
        raise RuntimeError("gdn_oracle_scan failed (%d)" % rc)
    return o, sf, sb


def readout_gate(o, z, gamma=None, eps=1e-6):
    """Readout epilogue of the linear branch, in float64: per (b, t, h) row of
    d_v values, the RMS-normalised readout scaled per channel by gamma and by
    the sigmoid of the content-dependent gate z:

        y = o / sqrt(mean(o ** 2) + eps) * gamma * 1 / (1 + exp(-z))

    Source: AI summary of "Video DeltaNet: A Video-Native Hybrid Attention for
    Livestream Video Generation", "Key Contributions" 1 (each branch has its
    own content-dependent sigmoid gate; the linear branch's readout is RMS
    normalised).  The page fixes neither the axis nor the order; the reading
    taken here: the norm runs over the head's d_v channels of one token, and
    the gate multiplies the normalised readout.  gamma None = ones.
    o, z: [B, T, H, dv]; gamma: [dv].  Returns float64 [B, T, H, dv]."""
    o = _f64(o)
    z = _f64(z)
    assert o.shape == z.shape
    dv = o.shape[-1]
    g = np.ones(dv) if gamma is None else _f64(gamma)
    assert g.shape == (dv,)
    y = np.empty_like(o)
    flat_o, flat_z, flat_y = o.reshape(-1, dv), z.reshape(-1, dv), y.reshape(-1, dv)
    for r in range(flat_o.shape[0]):
        row = flat_o[r]
        inv = 1.0 / np.sqrt(np.mean(row * row) + eps)
        for j in range(dv):
            flat_y[r, j] = row[j] * inv * g[j] / (1.0 + np.exp(-flat_z[r, j]))
    return y
