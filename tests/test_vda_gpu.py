"""GPU parity of the frame-wise delta operator (gdn_vda_scan) against the
FP64 oracle (oracle.vda_scan): causal and bidirectional, with initial and
final states, fp32 and bf16 inputs, frame lengths that are not multiples of
the kernels' token blocks.  Tolerance as for the token scans:
max|gpu - oracle| / rms(oracle) <= 1e-4 (fp32 inputs), 2e-2 (bf16 inputs)."""
import pytest
import torch

import gated_delta_rule_72_b200 as gdn
import oracle
from gated_delta_rule_72_b200 import inputs
from tests.gpu_util import TOL, rel_err, rel_err_bf16_out, to_dev

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def _frame_inputs(B, F, U, H, dk, dv, dtype, seed):
    inp = inputs.generate(B, F * U, H, dk, dv, dtype, seed=seed)
    inp["alpha_frame"] = inp["alpha"][:, ::U].contiguous()    # one decay per frame
    return inp


def _state(B, H, dk, dv, seed):
    g = torch.Generator("cpu").manual_seed(seed)
    return (0.3 * torch.randn(B, H, dk, dv, generator=g)).float()


@pytest.mark.parametrize("bidir", [False, True])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64), (64, 128)])
@pytest.mark.parametrize("F,U", [(3, 40), (2, 130), (5, 1)])
def test_vda_parity(bidir, dtype, dk, dv, F, U):
    B, H = 2, 3
    inp = _frame_inputs(B, F, U, H, dk, dv, dtype, seed=4000 + F * U + dk + dv)
    s0, r0 = _state(B, H, dk, dv, F + U), _state(B, H, dk, dv, F + U + 1)
    d = to_dev(inp)
    o, sf, sb = gdn.vda_scan(d["q"], d["k"], d["v"], d["alpha_frame"], d["beta"], U, bidir=bidir,
                             state=s0.cuda(), state_bwd=r0.cuda() if bidir else None, return_states=True)
    torch.cuda.synchronize()
    o_ref, sf_ref, sb_ref = oracle.vda_scan(inp["q"], inp["k"], inp["v"], inp["alpha_frame"], inp["beta"], U,
                                            mode="bidir" if bidir else "causal", state_in=s0,
                                            state_in_bwd=r0 if bidir else None)
    tol = TOL[DT[dtype]]
    assert rel_err(o, o_ref) <= tol
    assert rel_err(sf, sf_ref) <= tol
    if bidir:
        assert rel_err(sb, sb_ref) <= tol


def test_vda_bf16_output_and_zero_frames():
    B, F, U, H, dk, dv = 1, 4, 50, 2, 128, 128
    inp = _frame_inputs(B, F, U, H, dk, dv, "bf16", seed=4100)
    d = to_dev(inp)
    o16 = gdn.vda_scan(d["q"], d["k"], d["v"], d["alpha_frame"], d["beta"], U, bidir=True,
                       out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    o_ref, _, _ = oracle.vda_scan(inp["q"], inp["k"], inp["v"], inp["alpha_frame"], inp["beta"], U, mode="bidir")
    assert rel_err_bf16_out(o16, o_ref) <= TOL[torch.bfloat16]
    # no frames: the states pass through
    s0 = _state(B, H, dk, dv, 9).cuda()
    e = {n: t[:, :0].contiguous() for n, t in d.items()}
    _, sf, _ = gdn.vda_scan(e["q"], e["k"], e["v"], e["alpha_frame"], e["beta"], U, state=s0, return_states=True)
    torch.cuda.synchronize()
    assert torch.equal(sf, s0)


def test_vda_frames_equal_token_scan_for_one_token_frames():
    """U = 1 on the GPU: the frame operator equals the token scan with
    beta' = beta / (1 + beta |k|^2) (unit keys: beta / (1 + beta)), both run by
    the library (token path and chunked path as the call length decides)."""
    B, T, H, dk, dv = 1, 150, 2, 128, 128
    inp = inputs.generate(B, T, H, dk, dv, "f32", seed=4200)
    d = to_dev(inp)
    kk = (d["k"].double() ** 2).sum(-1)
    b2 = (d["beta"] / (1 + d["beta"].double() * kk)).float().contiguous()
    o1, s1, _ = gdn.vda_scan(d["q"], d["k"], d["v"], d["alpha"], d["beta"], 1, return_states=True)
    o2, s2 = gdn.scan_causal(d["q"], d["k"], d["v"], d["alpha"], b2)
    torch.cuda.synchronize()
    assert rel_err(o1, o2.double().cpu().numpy()) <= 1e-4
    assert rel_err(s1, s2.double().cpu().numpy()) <= 1e-4


def test_vda480_full_frame_length():
    """The benchmarked frame-wise workload as timed (B=1, H=12, 21 frames of
    1,560 tokens, d = 128, bf16, bidirectional): two sampled heads against the
    oracle, every output of those heads."""
    w = inputs.WORKLOADS["vda480"]
    inp = inputs.workload_inputs(w)
    af = inputs.frame_alpha(inp["alpha"], w.frame)
    d = to_dev(inp)
    o = gdn.vda_scan(d["q"], d["k"], d["v"], af.cuda(), d["beta"], w.frame, bidir=True)
    torch.cuda.synchronize()
    assert torch.isfinite(o).all()
    heads = [2, 9]
    sel = lambda t: t[:, :, heads].contiguous()
    o_ref, _, _ = oracle.vda_scan(sel(inp["q"]), sel(inp["k"]), sel(inp["v"]), sel(af), sel(inp["beta"]), w.frame,
                                  mode="bidir")
    err = rel_err(o.cpu()[:, :, heads], o_ref)
    print("vda480 parity max|o - o_oracle| / rms(o_oracle) = %.3e" % err)
    assert err <= TOL[torch.bfloat16]
