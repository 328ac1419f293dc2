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


def vda_scan(q, k, v, alpha_f, beta, U, mode="causal", state_in=None, state_in_bwd=None):
    """Frame-wise delta operator (VDA), in float64.  The sequence is split
    into frames of U consecutive tokens (T = F * U).  For frame f with keys
    K_f (U x dk), values V_f (U x dv), per-token write strengths beta and a
    per-frame decay alpha_f:

        A_f = K_f^T diag(beta) K_f,   B_f = K_f^T diag(beta) V_f
        S_f = (I + A_f)^{-1} (alpha_f S_{f-1} + B_f)

    the minimiser of ||S - alpha_f S_{f-1}||^2 + sum_u beta_u ||S^T k_u - v_u||^2:
    the state that stays close to the decayed memory while fitting every
    key-value pair of the frame at once.  Causal readout: o_u = S_f^T q_u for
    the tokens u of frame f.  Reverse (strict): R_f = (I + A_f)^{-1}
    (alpha_f R_{f+1} + B_f) from R_{F+1} = state_in_bwd, read as
    o_u = R_{f+1}^T q_u (the frames after f only); bidir adds the two.

    Source: AI summary of "Video DeltaNet: A Video-Native Hybrid Attention for
    Livestream Video Generation", "Key Contributions" 2 (the closed form
    S_t = (S_bar_t + B_t)(I + A_t)^{-1}, written there for a state that maps
    keys to values, i.e. the transpose of the layout here) and "Methodology in
    Plain English" (the least-squares objective in words).  The pages leave
    S_bar, A and B undefined; the reading here (S_bar = decayed previous state,
    A and B the frame's beta-weighted key Gram and key-value products) is the
    one that objective gives.  np.linalg.solve is the library step.

    q, k: [B, T, H, dk]; v: [B, T, H, dv]; alpha_f: [B, F, H]; beta: [B, T, H].
    Returns (o [B, T, H, dv], S_F or None, R_1 or None), float64."""
    q, k, v, alpha_f, beta = (_f64(x) for x in (q, k, v, alpha_f, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert U >= 1 and T % U == 0
    F = T // U
    assert alpha_f.shape == (B, F, H) and beta.shape == (B, T, H)
    s0, r0 = _f64(state_in), _f64(state_in_bwd)
    o = np.zeros((B, T, H, dv))
    sf = np.zeros((B, H, dk, dv)) if mode in ("causal", "bidir") else None
    sb = np.zeros((B, H, dk, dv)) if mode in ("reverse", "bidir") else None
    eye = np.eye(dk)
    for b in range(B):
        for h in range(H):
            def frame(f):
                t = slice(f * U, (f + 1) * U)
                K, V, be = k[b, t, h], v[b, t, h], beta[b, t, h]
                return t, K.T @ (be[:, None] * K), K.T @ (be[:, None] * V)
            if mode in ("causal", "bidir"):
                S = np.zeros((dk, dv)) if s0 is None else s0[b, h].copy()
                for f in range(F):
                    t, A, Bm = frame(f)
                    S = np.linalg.solve(eye + A, alpha_f[b, f, h] * S + Bm)
                    o[b, t, h] += q[b, t, h] @ S
                sf[b, h] = S
            if mode in ("reverse", "bidir"):
                R = np.zeros((dk, dv)) if r0 is None else r0[b, h].copy()
                for f in range(F - 1, -1, -1):
                    t, A, Bm = frame(f)
                    o[b, t, h] += q[b, t, h] @ R
                    R = np.linalg.solve(eye + A, alpha_f[b, f, h] * R + Bm)
                sb[b, h] = R
    return o, sf, sb
