"""Full-size workloads, in the launch configuration the benchmark times,
checked against the FP64 oracle on sampled heads (every output of those
heads), plus size-independent properties on all heads."""
import numpy as np
import pytest
import torch

import gated_delta_rule_72_b200 as gdn
from gated_delta_rule_72_b200 import inputs
from tests.gpu_util import TOL, oracle_heads, rel_err, to_dev

pytestmark = pytest.mark.gpu


def _check_heads(o_gpu, inp, heads, mode="causal", s_gpu=None):
    o_ref, s_ref = oracle_heads(inp, heads=heads, mode=mode)
    tol = TOL[inp["q"].dtype]
    err = rel_err(o_gpu[:, :, heads], o_ref)
    print("parity max|o - o_oracle| / rms(o_oracle) = %.3e (heads %s)" % (err, heads))
    assert np.isfinite(err) and err <= tol, err
    if s_gpu is not None:
        serr = rel_err(s_gpu[:, heads], s_ref)
        print("parity max|S - S_oracle| / rms(S_oracle) = %.3e" % serr)
        assert serr <= tol, serr
    return err


def test_stream480_causal():
    """B=1, H=12, T=32,760, d=128, bf16."""
    inp = inputs.workload_inputs("stream480")
    d = to_dev(inp)
    o, s = gdn.scan_causal(d["q"], d["k"], d["v"], d["alpha"], d["beta"])
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()
    _check_heads(o.cpu(), inp, [0, 7, 11], s_gpu=s.cpu())


def test_skewed_causal():
    """B=4, H=32, T=16,384, d=128, bf16, log alpha ~ U[-2,0], beta ~ U[0.9,1]."""
    inp = inputs.workload_inputs("skewed")
    d = to_dev(inp)
    o, s = gdn.scan_causal(d["q"], d["k"], d["v"], d["alpha"], d["beta"])
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()
    _check_heads(o.cpu(), inp, [0, 31], s_gpu=s.cpu())


def test_bidir720():
    """B=1, H=20, T=75,600, d=128, bf16, bidirectional."""
    inp = inputs.workload_inputs("bidir720")
    d = to_dev(inp)
    o = gdn.scan_bidir(d["q"], d["k"], d["v"], d["alpha"], d["beta"])
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()
    _check_heads(o.cpu(), inp, [0, 3, 19], mode="bidir")


def test_rollout_168_steps():
    """168 gdn_step calls of 1,560 tokens (H=16, d=128, bf16, state carried)
    equal one 262,080-token causal scan: the oracle on sampled heads, and the
    GPU single call on every head."""
    w = inputs.WORKLOADS["rollout"]
    inp = inputs.workload_inputs(w)
    d = to_dev(inp)
    state = torch.zeros(w.B, w.H, w.dk, w.dv, device="cuda")
    o = torch.empty(w.B, w.total_T, w.H, w.dv, dtype=torch.float32, device="cuda")
    nb = gdn.workspace_size(w.B, w.T, w.H, w.dk, w.dv, torch.bfloat16)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    for i in range(w.calls):
        sl = slice(i * w.T, (i + 1) * w.T)
        part = {n: t[:, sl].contiguous() for n, t in d.items()}
        o[:, sl] = gdn.step(part["q"], part["k"], part["v"], part["alpha"], part["beta"], state,
                            workspace=ws)
    o_one, s_one = gdn.scan_causal(d["q"], d["k"], d["v"], d["alpha"], d["beta"])
    torch.cuda.synchronize()
    tol = TOL[torch.bfloat16]
    assert rel_err(o, o_one.float().cpu().numpy()) <= tol
    assert rel_err(state, s_one.cpu().numpy()) <= tol
    _check_heads(o.cpu(), inp, [0, 5, 15], s_gpu=state.cpu())


def test_no_device_wait_gave_up():
    """Every bounded device-side wait (TMA arrival, tensor-core completion) in
    the kernels run so far completed in time."""
    assert gdn.gdn_device_timeouts() == 0
