"""Helpers for the GPU parity tests: the error metric, tolerances and an
oracle call on selected heads."""
import numpy as np
import torch

import oracle

# max|gpu - oracle| / rms(oracle): fp32 inputs 1e-4, bf16 inputs 2e-2
TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def rel_err(x, ref) -> float:
    x = x.detach().double().cpu().numpy() if hasattr(x, "detach") else np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    rms = np.sqrt(np.mean(ref ** 2))
    if rms == 0:
        return float(np.max(np.abs(x)))
    return float(np.max(np.abs(x - ref)) / rms)


def rel_err_bf16_out(x, ref) -> float:
    """The error metric for a bf16 OUTPUT: rounding the exact result to bf16
    alone moves an element by up to 2^-8 of its magnitude, so that much is
    taken off each element's error before max / rms."""
    x = x.detach().double().cpu().numpy() if hasattr(x, "detach") else np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = np.sqrt(np.mean(ref ** 2))
    excess = np.abs(x - ref) - np.ldexp(np.abs(ref), -8)
    return float(max(np.max(excess), 0.0) / rms)


def oracle_heads(inp, heads=None, mode="causal", state_in=None, t_slice=None, state_in_bwd=None,
                 with_bwd=False):
    """Oracle on a subset of heads (all if None); inputs are the CPU copies of
    exactly the tensors the GPU used.  Returns numpy (o, state_out), or with
    with_bwd (o, state_out, reverse state_out)."""
    def pick(t, axis_h):
        t = t.detach().cpu()
        if t_slice is not None and axis_h == 2:
            t = t[:, t_slice]
        if heads is not None:
            t = t[:, :, heads] if axis_h == 2 else t[:, heads]
        return t
    q, k, v = (pick(inp[n], 2) for n in ("q", "k", "v"))
    a, b = pick(inp["alpha"], 2), pick(inp["beta"], 2)
    s0 = None if state_in is None else pick(state_in, 1)
    r0 = None if state_in_bwd is None else pick(state_in_bwd, 1)
    o, sf, sb = oracle.scan(q, k, v, a, b, mode=mode, state_in=s0, state_in_bwd=r0)
    return (o, sf, sb) if with_bwd else (o, sf)


def to_dev(inp, device="cuda"):
    return {n: t.to(device) for n, t in inp.items()}
