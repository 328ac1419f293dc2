"""Torch-facing wrappers over the C-ABI (device memory and streams only).

`scan_causal`, `scan_bidir` and `step` take CUDA tensors, allocate the output
(and the workspace unless one is passed), and call the library on the
current torch stream.  No arithmetic of the scan happens here.
"""
from __future__ import annotations

import torch

from . import _lib

_DT = {torch.float32: _lib.GDN_F32, torch.bfloat16: _lib.GDN_BF16}


def _ptr(t):
    return None if t is None else t.data_ptr()


def _check(t, name, dtype=None, shape=None):
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor (the library has no CPU path)" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))


def _dims(q, k, v, alpha, beta):
    if q.dtype not in _DT:
        raise ValueError("q must be float32 or bfloat16")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    _check(q, "q")
    _check(k, "k", q.dtype, (B, T, H, dk))
    _check(v, "v", q.dtype, (B, T, H, dv))
    _check(alpha, "alpha", torch.float32, (B, T, H))
    _check(beta, "beta", torch.float32, (B, T, H))
    return B, T, H, dk, dv, _DT[q.dtype]


def workspace_size(B, T, H, dk, dv, dtype=torch.bfloat16, bidir=False,
                   out_dtype=torch.float32) -> int:
    return int(_lib.gdn_workspace_size(B, T, H, dk, dv, _DT[dtype], _DT[out_dtype],
                                       int(bool(bidir))))


def _out(B, T, H, dv, device, out, out_dtype):
    if out is None:
        return torch.empty((B, T, H, dv), dtype=out_dtype, device=device), _DT[out_dtype]
    if out.dtype not in _DT:
        raise ValueError("out must be float32 or bfloat16")
    _check(out, "out", None, (B, T, H, dv))
    return out, _DT[out.dtype]


def _workspace(nbytes, device, workspace):
    if nbytes == 0:
        return None, 0
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
    elif workspace.numel() * workspace.element_size() < nbytes:
        raise ValueError("workspace too small: %d < %d bytes" % (workspace.numel(), nbytes))
    return workspace, workspace.numel() * workspace.element_size()


def _raise(fn, st):
    if st != 0:
        raise _lib.GDNError(fn, st)


def scan_causal(q, k, v, alpha, beta, state=None, *, return_state=True, out=None,
                out_dtype=torch.float32, state_out=None, workspace=None):
    """Causal scan.  Returns (o, final_state) (final_state None if not asked).
    o is fp32 unless out_dtype (or the dtype of `out`) is bfloat16."""
    B, T, H, dk, dv, dt = _dims(q, k, v, alpha, beta)
    if state is not None:
        _check(state, "state", torch.float32, (B, H, dk, dv))
    o, odt = _out(B, T, H, dv, q.device, out, out_dtype)
    if return_state and state_out is None:
        state_out = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    ws, nbytes = _workspace(workspace_size(B, T, H, dk, dv, q.dtype, False, o.dtype), q.device,
                            workspace)
    stream = torch.cuda.current_stream(q.device).cuda_stream
    st = _lib.gdn_scan_causal(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(state),
                              _ptr(state_out), _ptr(o), B, T, H, dk, dv, dt, odt, _ptr(ws), nbytes,
                              stream)
    _raise("gdn_scan_causal", st)
    return o, state_out


def scan_bidir(q, k, v, alpha, beta, *, out=None, out_dtype=torch.float32, workspace=None,
               state=None, state_bwd=None, return_states=False):
    """Bidirectional scan (causal + strict reverse readouts, summed in fp32).

    state / state_bwd: initial states ([B,H,dk,dv] fp32) of the causal scan
    (S_0) and of the reverse scan (R_{T+1}); None = zero.  Returns o, or with
    return_states=True (o, S_T, R_1)."""
    B, T, H, dk, dv, dt = _dims(q, k, v, alpha, beta)
    for t, name in ((state, "state"), (state_bwd, "state_bwd")):
        if t is not None:
            _check(t, name, torch.float32, (B, H, dk, dv))
    o, odt = _out(B, T, H, dv, q.device, out, out_dtype)
    ws, nbytes = _workspace(workspace_size(B, T, H, dk, dv, q.dtype, True, o.dtype), q.device,
                            workspace)
    stream = torch.cuda.current_stream(q.device).cuda_stream
    if state is None and state_bwd is None and not return_states:
        st = _lib.gdn_scan_bidir(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(o),
                                 B, T, H, dk, dv, dt, odt, _ptr(ws), nbytes, stream)
        _raise("gdn_scan_bidir", st)
        return o
    s_out = s_out_b = None
    if return_states:
        s_out = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
        s_out_b = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    st = _lib.gdn_scan_bidir_states(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(state),
                                    _ptr(state_bwd), _ptr(s_out), _ptr(s_out_b), _ptr(o), B, T, H, dk,
                                    dv, dt, odt, _ptr(ws), nbytes, stream)
    _raise("gdn_scan_bidir_states", st)
    return (o, s_out, s_out_b) if return_states else o


def step(q, k, v, alpha, beta, state, *, out=None, out_dtype=torch.float32, workspace=None):
    """One streaming call; `state` ([B,H,dk,dv] fp32) is updated in place."""
    B, T, H, dk, dv, dt = _dims(q, k, v, alpha, beta)
    _check(state, "state", torch.float32, (B, H, dk, dv))
    o, odt = _out(B, T, H, dv, q.device, out, out_dtype)
    ws, nbytes = _workspace(workspace_size(B, T, H, dk, dv, q.dtype, False, o.dtype), q.device,
                            workspace)
    stream = torch.cuda.current_stream(q.device).cuda_stream
    st = _lib.gdn_step(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(state), _ptr(o),
                       B, T, H, dk, dv, dt, odt, _ptr(ws), nbytes, stream)
    _raise("gdn_step", st)
    return o


def readout_gate(o, z, gamma=None, eps=1e-6, *, out=None, out_dtype=None):
    """Readout epilogue: y = o / sqrt(mean(o^2 over d_v) + eps) * gamma * sigmoid(z),
    per (b, t, h).  o, z: [B,T,H,dv] (fp32 or bf16); gamma: [dv] fp32 or None.
    y is `out` (may be o or z itself, same dtype) or a new tensor of
    out_dtype (default: o's dtype)."""
    _check(o, "o")
    if o.dtype not in _DT:
        raise ValueError("o must be float32 or bfloat16")
    B, T, H, dv = o.shape
    _check(z, "z", None, (B, T, H, dv))
    if z.dtype not in _DT:
        raise ValueError("z must be float32 or bfloat16")
    if gamma is not None:
        _check(gamma, "gamma", torch.float32, (dv,))
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=out_dtype or o.dtype, device=o.device)
    else:
        _check(out, "out", None, (B, T, H, dv))
    if out.dtype not in _DT:
        raise ValueError("out must be float32 or bfloat16")
    stream = torch.cuda.current_stream(o.device).cuda_stream
    st = _lib.gdn_readout_gate(_ptr(o), _DT[o.dtype], _ptr(z), _DT[z.dtype], _ptr(gamma), float(eps),
                               _ptr(out), _DT[out.dtype], B, T, H, dv, stream)
    _raise("gdn_readout_gate", st)
    return out


def vda_scan(q, k, v, alpha_frame, beta, U, *, bidir=False, state=None, state_bwd=None, return_states=False,
             out=None, out_dtype=torch.float32, workspace=None):
    """Frame-wise delta operator over frames of U tokens (T = F * U):
    S_f = (I + K^T diag(beta) K)^{-1} (alpha_f S_{f-1} + K^T diag(beta) V), read by
    every token of frame f (bidir: plus the reverse scan, read strictly).
    alpha_frame: [B, F, H] fp32; beta: [B, T, H] fp32.  Returns o, or with
    return_states (o, S_F, R_1) (R_1 None unless bidir)."""
    if q.dtype not in _DT:
        raise ValueError("q must be float32 or bfloat16")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if U < 1 or T % U != 0:
        raise ValueError("T (%d) must be a multiple of the frame length U (%d)" % (T, U))
    F = T // U
    _check(q, "q")
    _check(k, "k", q.dtype, (B, T, H, dk))
    _check(v, "v", q.dtype, (B, T, H, dv))
    _check(alpha_frame, "alpha_frame", torch.float32, (B, F, H))
    _check(beta, "beta", torch.float32, (B, T, H))
    for t, name in ((state, "state"), (state_bwd, "state_bwd")):
        if t is not None:
            _check(t, name, torch.float32, (B, H, dk, dv))
    o, odt = _out(B, T, H, dv, q.device, out, out_dtype)
    s_out = s_out_b = None
    if return_states:
        s_out = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
        if bidir:
            s_out_b = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    ws, nbytes = _workspace(int(_lib.gdn_vda_workspace_size(B, F, U, H, dk, dv, int(bool(bidir)))), q.device,
                            workspace)
    stream = torch.cuda.current_stream(q.device).cuda_stream
    st = _lib.gdn_vda_scan(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha_frame), _ptr(beta), _ptr(state),
                           _ptr(state_bwd), _ptr(s_out), _ptr(s_out_b), _ptr(o), B, F, U, H, dk, dv,
                           int(bool(bidir)), _DT[q.dtype], odt, _ptr(ws), nbytes, stream)
    _raise("gdn_vda_scan", st)
    return (o, s_out, s_out_b) if return_states else o
