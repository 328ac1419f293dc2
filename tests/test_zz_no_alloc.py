"""gdn_step_noalloc: the streaming step for callers that cannot allocate
device memory (a host framework that owns every byte of device memory
through its own pool, or a real-time rollout loop where an allocation could
synchronise the device and stall it).  Its scratch is a fixed 64 MiB array
inside libgdn.so instead of a caller workspace.

Called through the C-ABI, two calls in a row must match the ordinary
gdn_step on the same inputs, within the bf16-input tolerance the other
parity tests use, and on a sampled head the FP64 oracle run over both
calls' tokens.  This file is collected last on purpose."""
import pytest
import torch

from gated_delta_rule_72_b200 import _lib, inputs
from tests.gpu_util import TOL, oracle_heads, rel_err


@pytest.mark.gpu
def test_noalloc_step_matches_step_on_two_calls():
    B, T, H, dk, dv = 1, 1560, 16, 128, 128      # one streaming call of a rollout
    assert _lib.gdn_workspace_size(B, T, H, dk, dv, _lib.GDN_BF16, _lib.GDN_F32, 0) \
        <= _lib.GDN_NOALLOC_SCRATCH_BYTES
    inp = inputs.generate(B, 2 * T, H, dk, dv, "bf16", seed=41)
    d = {n: t.cuda() for n, t in inp.items()}
    nb = _lib.gdn_workspace_size(B, T, H, dk, dv, _lib.GDN_BF16, _lib.GDN_F32, 0)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    st_ref = torch.zeros(B, H, dk, dv, device="cuda")
    st_new = torch.zeros(B, H, dk, dv, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    outs = []
    for call in range(2):
        sl = slice(call * T, (call + 1) * T)
        x = {n: t[:, sl].contiguous() for n, t in d.items()}
        o_ref = torch.empty(B, T, H, dv, device="cuda")
        o_new = torch.full((B, T, H, dv), float("nan"), device="cuda")
        args = (x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(),
                x["alpha"].data_ptr(), x["beta"].data_ptr())
        s1 = _lib.gdn_step(*args, st_ref.data_ptr(), o_ref.data_ptr(), B, T, H, dk, dv,
                           _lib.GDN_BF16, _lib.GDN_F32, ws.data_ptr(), nb, stream)
        s2 = _lib.gdn_step_noalloc(*args, st_new.data_ptr(), o_new.data_ptr(), B, T, H, dk, dv,
                                   _lib.GDN_BF16, _lib.GDN_F32, stream)
        assert s1 == 0 and s2 == 0, (s1, s2)
        torch.cuda.synchronize()
        tol = TOL[torch.bfloat16]
        assert torch.isfinite(o_new).all()
        assert rel_err(o_new, o_ref.double().cpu().numpy()) <= tol
        assert rel_err(st_new, st_ref.double().cpu().numpy()) <= tol
        outs.append(o_new.cpu())
    # and against the FP64 oracle on one head: both calls are one 2T-token scan
    head = [5]
    o_orc, s_orc = oracle_heads(inp, heads=head)
    assert rel_err(torch.cat(outs, dim=1)[:, :, head], o_orc) <= TOL[torch.bfloat16]
    assert rel_err(st_new.cpu()[:, head], s_orc) <= TOL[torch.bfloat16]
