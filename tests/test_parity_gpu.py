"""GPU parity: the CUDA library against the FP64 oracle, element by element,
on the same seeded inputs.  Tolerance (max|gpu - oracle| / rms(oracle)):
1e-4 for fp32 inputs, 2e-2 for bf16 inputs; the final state is held to the
same bar against rms of the oracle's state."""
import numpy as np
import pytest
import torch

import gated_delta_rule_72_b200 as gdn
from gated_delta_rule_72_b200 import inputs
from tests.gpu_util import TOL, oracle_heads, rel_err, rel_err_bf16_out, to_dev

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def _state(B, H, dk, dv, seed):
    g = torch.Generator("cpu").manual_seed(seed)
    return (0.3 * torch.randn(B, H, dk, dv, generator=g)).float()


def test_tiny_workload():
    """B=1, H=2, T=256, d=64, fp32, chunk 64, seed 0."""
    w = inputs.WORKLOADS["tiny"]
    inp = inputs.workload_inputs(w)
    d = to_dev(inp)
    o, s = gdn.scan_causal(d["q"], d["k"], d["v"], d["alpha"], d["beta"])
    torch.cuda.synchronize()
    o_ref, s_ref = oracle_heads(inp)
    assert rel_err(o, o_ref) <= 1e-4
    assert rel_err(s, s_ref) <= 1e-4


SHAPES = [(64, 64), (128, 128), (64, 128), (128, 64)]


def _kernel_family(names):
    """'token', 'tc' or 'simt': which path the kernels recorded belong to."""
    fams = {"token" if n == "token_step" else n.split("_")[0] for n in names}
    assert len(fams) == 1, names
    return fams.pop()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", SHAPES)
@pytest.mark.parametrize("T", [1, 63, 64, 65, 127, 200])
def test_causal_shapes(dtype, dk, dv, T):
    """Causal scans with state in and out; bf16 inputs run on the tensor
    cores for either key width (d_k = 64 padded to 128 with zero columns),
    fp32 inputs on the CUDA cores (short calls may take the token path)."""
    B, H = 2, 3
    inp = inputs.generate(B, T, H, dk, dv, dtype, seed=1000 + T + dk + dv)
    s0 = _state(B, H, dk, dv, seed=T)
    d = to_dev(inp)
    gdn.gdn_set_kernel_timing(1)
    gdn.gdn_read_kernel_timing()
    try:
        o, s = gdn.scan_causal(d["q"], d["k"], d["v"], d["alpha"], d["beta"], s0.cuda())
        torch.cuda.synchronize()
        fam = _kernel_family(gdn.gdn_read_kernel_timing())
    finally:
        gdn.gdn_set_kernel_timing(0)
    assert fam in ("token", "tc" if dtype == "bf16" else "simt"), fam
    if T > 64:
        assert fam == ("tc" if dtype == "bf16" else "simt"), fam
    o_ref, s_ref = oracle_heads(inp, state_in=s0)
    tol = TOL[DT[dtype]]
    assert rel_err(o, o_ref) <= tol
    assert rel_err(s, s_ref) <= tol


@pytest.mark.parametrize("path", ["token", "chunked"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", SHAPES)
@pytest.mark.parametrize("T", [1, 2, 17, 63, 64])
def test_short_calls_both_paths(path, dtype, dk, dv, T):
    """Calls of at most 64 tokens: the token-by-token kernel (default) and the
    chunked path (short-call threshold 0) both match the oracle, state in and
    out, bf16 output included."""
    B, H = 2, 3
    inp = inputs.generate(B, T, H, dk, dv, dtype, seed=3000 + T + dk + dv)
    s0 = _state(B, H, dk, dv, seed=T + 7)
    d = to_dev(inp)
    prev = gdn.gdn_set_short_call_tokens(64 if path == "token" else 0)
    gdn.gdn_set_kernel_timing(1)
    gdn.gdn_read_kernel_timing()
    try:
        o, s = gdn.scan_causal(d["q"], d["k"], d["v"], d["alpha"], d["beta"], s0.cuda())
        o16, _ = gdn.scan_causal(d["q"], d["k"], d["v"], d["alpha"], d["beta"], s0.cuda(),
                                 out_dtype=torch.bfloat16)
        names = set(gdn.gdn_read_kernel_timing())
    finally:
        gdn.gdn_set_kernel_timing(0)
        gdn.gdn_set_short_call_tokens(prev)
    assert (names == {"token_step"}) == (path == "token"), names
    o_ref, s_ref = oracle_heads(inp, state_in=s0)
    tol = TOL[DT[dtype]]
    assert rel_err(o, o_ref) <= tol
    assert rel_err(s, s_ref) <= tol
    assert rel_err_bf16_out(o16, o_ref) <= TOL[torch.bfloat16]


def test_short_call_threshold_switches_path():
    """A 65-token call takes the chunked path whatever the threshold (it is
    clamped to 64); a 64-token call takes the token path by default."""
    inp = inputs.generate(1, 65, 2, 128, 128, "bf16", seed=5)
    d = to_dev(inp)
    gdn.gdn_set_kernel_timing(1)
    gdn.gdn_read_kernel_timing()
    try:
        prev = gdn.gdn_set_short_call_tokens(1000)
        gdn.scan_causal(d["q"], d["k"], d["v"], d["alpha"], d["beta"])
        gdn.scan_causal(d["q"][:, :64].contiguous(), d["k"][:, :64].contiguous(), d["v"][:, :64].contiguous(),
                        d["alpha"][:, :64].contiguous(), d["beta"][:, :64].contiguous())
        names = set(gdn.gdn_read_kernel_timing())
    finally:
        gdn.gdn_set_kernel_timing(0)
        gdn.gdn_set_short_call_tokens(prev)
    assert "token_step" in names
    assert names - {"token_step"}, names


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (128, 64), (64, 128)])
@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 130, 257])
def test_bidir_shapes(dtype, dk, dv, T):
    """Bidirectional scans: bf16 inputs on the tensor cores for both key
    widths, fp32 inputs on the CUDA cores."""
    B, H = 1, 3
    inp = inputs.generate(B, T, H, dk, dv, dtype, seed=2000 + T + dk)
    d = to_dev(inp)
    gdn.gdn_set_kernel_timing(1)
    gdn.gdn_read_kernel_timing()
    try:
        o = gdn.scan_bidir(d["q"], d["k"], d["v"], d["alpha"], d["beta"])
        torch.cuda.synchronize()
        fam = _kernel_family(gdn.gdn_read_kernel_timing())
    finally:
        gdn.gdn_set_kernel_timing(0)
    assert fam == ("tc" if dtype == "bf16" else "simt"), fam
    o_ref, _ = oracle_heads(inp, mode="bidir")
    assert rel_err(o, o_ref) <= TOL[DT[dtype]]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (128, 64)])
@pytest.mark.parametrize("T", [1, 64, 130])
def test_bidir_initial_states(dtype, dk, dv, T):
    """Bidirectional with a causal initial state S_0 and a reverse initial
    state R_{T+1}: o and both final states (S_T, R_1) against the oracle."""
    B, H = 1, 3
    inp = inputs.generate(B, T, H, dk, dv, dtype, seed=2500 + T + dk + dv)
    s0, r0 = _state(B, H, dk, dv, seed=T + 1), _state(B, H, dk, dv, seed=T + 2)
    d = to_dev(inp)
    o, sf, sb = gdn.scan_bidir(d["q"], d["k"], d["v"], d["alpha"], d["beta"], state=s0.cuda(),
                               state_bwd=r0.cuda(), return_states=True)
    torch.cuda.synchronize()
    o_ref, sf_ref, sb_ref = oracle_heads(inp, mode="bidir", state_in=s0, state_in_bwd=r0, with_bwd=True)
    tol = TOL[DT[dtype]]
    assert rel_err(o, o_ref) <= tol
    assert rel_err(sf, sf_ref) <= tol
    assert rel_err(sb, sb_ref) <= tol


@pytest.mark.parametrize("H", [3, 40])
def test_bidir_states_in_place(H):
    """Output states updated in place (each direction's buffer holds its
    initial state, then its final one), on the fused launch (H = 3) and the
    two-launch path with 64-column slices (H = 40); T = 0 passes the states
    through."""
    B, T, dk, dv = 1, 130, 128, 128
    inp = inputs.generate(B, T, H, dk, dv, "bf16", seed=2600 + H)
    s0, r0 = _state(B, H, dk, dv, seed=H), _state(B, H, dk, dv, seed=H + 50)
    d = to_dev(inp)
    sf, sb = s0.cuda(), r0.cuda()
    B_, T_, H_, dk_, dv_ = B, T, H, dk, dv
    o = torch.empty(B, T, H, dv, device="cuda")
    ws = torch.empty(gdn.workspace_size(B, T, H, dk, dv, torch.bfloat16, bidir=True), dtype=torch.uint8,
                     device="cuda")
    st = gdn.gdn_scan_bidir_states(d["q"].data_ptr(), d["k"].data_ptr(), d["v"].data_ptr(),
                                   d["alpha"].data_ptr(), d["beta"].data_ptr(), sf.data_ptr(), sb.data_ptr(),
                                   sf.data_ptr(), sb.data_ptr(), o.data_ptr(), B_, T_, H_, dk_, dv_, 1, 0,
                                   ws.data_ptr(), ws.numel(), torch.cuda.current_stream().cuda_stream)
    assert st == 0
    torch.cuda.synchronize()
    o_ref, sf_ref, sb_ref = oracle_heads(inp, mode="bidir", state_in=s0, state_in_bwd=r0, with_bwd=True)
    assert rel_err(o, o_ref) <= TOL[torch.bfloat16]
    assert rel_err(sf, sf_ref) <= TOL[torch.bfloat16]
    assert rel_err(sb, sb_ref) <= TOL[torch.bfloat16]
    e = {n: t[:, :0].contiguous() for n, t in d.items()}
    o0, sf0, sb0 = gdn.scan_bidir(e["q"], e["k"], e["v"], e["alpha"], e["beta"], state=sf, state_bwd=sb,
                                  return_states=True)
    torch.cuda.synchronize()
    assert torch.equal(sf0, sf) and torch.equal(sb0, sb)


@pytest.mark.parametrize("gates", ["default", "skewed"])
def test_streaming_splits_match_one_call(gates):
    """gdn_step over arbitrary call boundaries (lengths 1, 63, 64, 65, ...)
    equals one causal scan, and both equal the oracle."""
    B, T, H, dk, dv = 1, 600, 2, 128, 128
    inp = inputs.generate(B, T, H, dk, dv, "bf16", seed=77, gates=gates)
    d = to_dev(inp)
    o_one, s_one = gdn.scan_causal(d["q"], d["k"], d["v"], d["alpha"], d["beta"])
    cuts = [0, 1, 64, 127, 191, 192, 257, 300, 365, 429, 430, 599, 600]
    state = torch.zeros(B, H, dk, dv, device="cuda")
    outs = []
    for a, b in zip(cuts, cuts[1:]):
        sl = {n: t[:, a:b].contiguous() for n, t in d.items()}
        outs.append(gdn.step(sl["q"], sl["k"], sl["v"], sl["alpha"], sl["beta"], state))
    o_split = torch.cat(outs, dim=1)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle_heads(inp)
    tol = TOL[torch.bfloat16]
    assert rel_err(o_split, o_ref) <= tol
    assert rel_err(state, s_ref) <= tol
    assert rel_err(o_one, o_ref) <= tol
    # the two GPU evaluations differ only by chunk boundaries
    assert rel_err(o_split.float(), o_one.float().cpu().double().numpy()) <= tol


def test_identity_gates_keep_state():
    """alpha = 1, beta = 0: every token is an identity step, o_t = S_0^T q_t."""
    B, T, H, dk, dv = 1, 100, 2, 64, 64
    inp = inputs.generate(B, T, H, dk, dv, "f32", seed=5)
    inp["alpha"] = torch.ones_like(inp["alpha"])
    inp["beta"] = torch.zeros_like(inp["beta"])
    s0 = _state(B, H, dk, dv, 9)
    d = to_dev(inp)
    o, s = gdn.scan_causal(d["q"], d["k"], d["v"], d["alpha"], d["beta"], s0.cuda())
    torch.cuda.synchronize()
    want = torch.einsum("bthi,bhij->bthj", inp["q"].double(), s0.double())
    assert rel_err(o, want.numpy()) <= 1e-5
    assert torch.equal(s.cpu(), s0)


def test_empty_sequence_passes_state():
    B, H, dk, dv = 2, 3, 128, 64
    s0 = _state(B, H, dk, dv, 3).cuda()
    e = torch.empty(B, 0, H, dk, device="cuda")
    ev = torch.empty(B, 0, H, dv, device="cuda")
    g = torch.empty(B, 0, H, device="cuda")
    o, s = gdn.scan_causal(e, e, ev, g, g, s0)
    torch.cuda.synchronize()
    assert o.shape == (B, 0, H, dv)
    assert torch.equal(s, s0)
    o, s = gdn.scan_causal(e, e, ev, g, g, None)
    assert torch.count_nonzero(s) == 0
    o = gdn.scan_bidir(e, e, ev, g, g)
    assert o.shape == (B, 0, H, dv)


def test_in_place_state_update():
    B, T, H, dk, dv = 1, 130, 2, 64, 128
    inp = inputs.generate(B, T, H, dk, dv, "f32", seed=11)
    s0 = _state(B, H, dk, dv, 4)
    d = to_dev(inp)
    st = s0.cuda().clone()
    o = gdn.step(d["q"], d["k"], d["v"], d["alpha"], d["beta"], st)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle_heads(inp, state_in=s0)
    assert rel_err(o, o_ref) <= 1e-4
    assert rel_err(st, s_ref) <= 1e-4


@pytest.mark.parametrize("mode", ["causal", "bidir"])
def test_bf16_output(mode):
    """o_dt = bf16: the fp32 result rounded once; held to the bf16 bar after
    allowing the rounding of the output itself (2^-8 relative per element)."""
    B, T, H, dk, dv = 1, 333, 2, 128, 128
    inp = inputs.generate(B, T, H, dk, dv, "bf16", seed=31)
    d = to_dev(inp)
    if mode == "causal":
        o, _ = gdn.scan_causal(d["q"], d["k"], d["v"], d["alpha"], d["beta"],
                               out_dtype=torch.bfloat16)
        o32, _ = gdn.scan_causal(d["q"], d["k"], d["v"], d["alpha"], d["beta"])
    else:
        o = gdn.scan_bidir(d["q"], d["k"], d["v"], d["alpha"], d["beta"], out_dtype=torch.bfloat16)
        o32 = gdn.scan_bidir(d["q"], d["k"], d["v"], d["alpha"], d["beta"])
    torch.cuda.synchronize()
    assert o.dtype == torch.bfloat16
    o_ref, _ = oracle_heads(inp, mode=mode)
    assert rel_err_bf16_out(o, o_ref) <= 2e-2
    # the bf16 output is the fp32 output rounded once (round to nearest even)
    assert torch.equal(o, o32.to(torch.bfloat16))


def test_workspace_is_reusable_and_contents_do_not_matter():
    B, T, H, dk, dv = 1, 200, 2, 128, 128
    inp = inputs.generate(B, T, H, dk, dv, "bf16", seed=12)
    d = to_dev(inp)
    nb = gdn.workspace_size(B, T, H, dk, dv, torch.bfloat16, bidir=True)
    ws = torch.full((nb,), 0x7F, dtype=torch.uint8, device="cuda")  # garbage (NaN-ish floats)
    o1 = gdn.scan_bidir(d["q"], d["k"], d["v"], d["alpha"], d["beta"], workspace=ws)
    o2 = gdn.scan_bidir(d["q"], d["k"], d["v"], d["alpha"], d["beta"], workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    o_ref, _ = oracle_heads(inp, mode="bidir")
    assert rel_err(o1, o_ref) <= 2e-2


@pytest.mark.parametrize("mode", ["causal", "bidir"])
def test_strong_forgetting_gates(mode):
    """A stretch of tokens with alpha = e^-8: a 16-token block of it decays by
    e^-128, beyond where the masks' decay factors can be split into per-block
    factors, so those chunks take the one-exponential-per-entry path."""
    B, H, T, d = 1, 3, 300, 128
    inp = inputs.generate(B, T, H, d, d, "bf16", seed=4242)
    a = inp["alpha"].clone()
    a[:, 100:150] = float(np.exp(-8.0))
    a[:, 200:203] = float(np.exp(-40.0))
    inp["alpha"] = a
    dev = to_dev(inp)
    if mode == "causal":
        o, s = gdn.scan_causal(dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"])
    else:
        o = gdn.scan_bidir(dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"])
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()
    o_ref, s_ref = oracle_heads(inp, mode=mode)
    assert rel_err(o, o_ref) <= TOL[torch.bfloat16]
    if mode == "causal":
        assert rel_err(s, s_ref) <= TOL[torch.bfloat16]


@pytest.mark.parametrize("mode,o_dtype", [("causal", torch.float32), ("bidir", torch.float32),
                                          ("causal", torch.bfloat16), ("bidir", torch.bfloat16)])
def test_many_heads_take_wide_slices(mode, o_dtype):
    """Enough heads that the chain uses 64-column state slices (B*H*d_v/32 >
    the SM count), with a ragged last chunk, a state in, and both output
    dtypes."""
    B, H, T, d = 2, 40, 200, 128
    inp = inputs.generate(B, T, H, d, d, "bf16", seed=777)
    dev = to_dev(inp)
    if mode == "causal":
        s0 = _state(B, H, d, d, seed=5)
        o, s = gdn.scan_causal(dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], s0.cuda(),
                               out_dtype=o_dtype)
        o_ref, s_ref = oracle_heads(inp, state_in=s0)
    else:
        o = gdn.scan_bidir(dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], out_dtype=o_dtype)
        o_ref, _ = oracle_heads(inp, mode="bidir")
    torch.cuda.synchronize()
    if o_dtype == torch.float32:
        assert rel_err(o, o_ref) <= TOL[torch.bfloat16]
    else:
        assert rel_err_bf16_out(o, o_ref) <= TOL[torch.bfloat16]
    if mode == "causal":
        assert rel_err(s, s_ref) <= TOL[torch.bfloat16]


def test_rollout_replays_in_a_cuda_graph():
    """A rollout of gdn_step calls (chunked and token-by-token ones) captured in
    one CUDA graph replays to the same bits as the eager calls."""
    B, H, dk, dv = 1, 4, 128, 128
    lens = [200, 40, 1, 130, 64, 65]
    T = sum(lens)
    inp = inputs.generate(B, T, H, dk, dv, "bf16", seed=91)
    d = to_dev(inp)
    cuts = np.concatenate([[0], np.cumsum(lens)])
    ws = torch.empty(gdn.workspace_size(B, max(lens), H, dk, dv, torch.bfloat16), dtype=torch.uint8,
                     device="cuda")

    def rollout(state, o):
        state.zero_()
        for a, b in zip(cuts, cuts[1:]):
            sl = {n: t[:, a:b] for n, t in d.items()}
            gdn.step(sl["q"], sl["k"], sl["v"], sl["alpha"], sl["beta"], state, out=o[:, a:b], workspace=ws)

    s_e = torch.empty(B, H, dk, dv, device="cuda")
    o_e = torch.empty(B, T, H, dv, device="cuda")
    rollout(s_e, o_e)                      # eager (also the warm-up before capture)
    torch.cuda.synchronize()
    s_g = torch.empty_like(s_e)
    o_g = torch.full_like(o_e, float("nan"))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        rollout(s_g, o_g)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(o_g, o_e)
    assert torch.equal(s_g, s_e)
    o_ref, s_ref = oracle_heads(inp)
    assert rel_err(o_g, o_ref) <= TOL[torch.bfloat16]
    assert rel_err(s_g, s_ref) <= TOL[torch.bfloat16]



DTS = {"f32": torch.float32, "bf16": torch.bfloat16}


@pytest.mark.parametrize("dv", [64, 128])
@pytest.mark.parametrize("o_dt,z_dt,y_dt", [("f32", "f32", "f32"), ("f32", "bf16", "bf16"),
                                            ("bf16", "f32", "f32"), ("bf16", "bf16", "bf16")])
@pytest.mark.parametrize("eps,with_gamma", [(1e-6, False), (0.1, True)])
def test_readout_gate(dv, o_dt, z_dt, y_dt, eps, with_gamma):
    """Readout epilogue against the oracle, ragged row count (B*T*H = 222)."""
    from oracle import readout_gate as ref_readout
    B, T, H = 2, 37, 3
    g = torch.Generator("cpu").manual_seed(dv + len(o_dt + z_dt + y_dt))
    o = (torch.randn(B, T, H, dv, generator=g) * torch.rand(B, T, H, 1, generator=g) * 3).to(DTS[o_dt])
    z = (2 * torch.randn(B, T, H, dv, generator=g)).to(DTS[z_dt])
    gamma = (0.5 + torch.rand(dv, generator=g)) if with_gamma else None
    y = gdn.readout_gate(o.cuda(), z.cuda(), None if gamma is None else gamma.cuda(), eps,
                         out_dtype=DTS[y_dt])
    torch.cuda.synchronize()
    want = ref_readout(o, z, gamma, eps)
    if y_dt == "f32":
        assert rel_err(y, want) <= 1e-4
    else:
        assert rel_err_bf16_out(y, want) <= 1e-4


def test_readout_in_place_after_a_scan():
    """The linear branch end to end: causal scan, then the readout written
    over the scan's fp32 output in place; against oracle scan + readout."""
    from oracle import readout_gate as ref_readout
    B, T, H, dk, dv = 1, 300, 4, 128, 128
    inp = inputs.generate(B, T, H, dk, dv, "bf16", seed=123)
    d = to_dev(inp)
    o, _ = gdn.scan_causal(d["q"], d["k"], d["v"], d["alpha"], d["beta"])
    g = torch.Generator("cpu").manual_seed(5)
    z = torch.randn(B, T, H, dv, generator=g)
    gamma = 0.5 + torch.rand(dv, generator=g)
    y = gdn.readout_gate(o, z.cuda(), gamma.cuda(), 1e-6, out=o)
    torch.cuda.synchronize()
    assert y.data_ptr() == o.data_ptr()
    o_ref, _ = oracle_heads(inp)
    want = ref_readout(o_ref, z, gamma, 1e-6)
    assert rel_err(y, want) <= TOL[torch.bfloat16]
