"""Sequence-parallel chains (tensor-core path, bf16 inputs, d_k = 128): each
chunk walk cut into G segments, every segment after the first started from a
zero state where the bound on the skipped state maps reaches 2^-30 (or from
the true initial state if the walk back reaches the start).  Every segment
count must meet the same oracle tolerance, with state in and out, in both
directions, for gates that forget fast, slowly or not at all."""
import numpy as np
import pytest
import torch

import gated_delta_rule_72_b200 as gdn
from gated_delta_rule_72_b200 import inputs
from tests.gpu_util import TOL, oracle_heads, rel_err, to_dev

pytestmark = pytest.mark.gpu

TOL16 = TOL[torch.bfloat16]


def _state(B, H, dk, dv, seed):
    g = torch.Generator("cpu").manual_seed(seed)
    return (0.3 * torch.randn(B, H, dk, dv, generator=g)).float()


class _Segments:
    def __init__(self, g):
        self.g = g

    def __enter__(self):
        self.prev = gdn.gdn_set_chain_segments(self.g)

    def __exit__(self, *exc):
        gdn.gdn_set_chain_segments(self.prev)


def _causal(inp, s0, G):
    d = to_dev(inp)
    with _Segments(G):
        o, s = gdn.scan_causal(d["q"], d["k"], d["v"], d["alpha"], d["beta"], s0.cuda())
    torch.cuda.synchronize()
    return o.cpu(), s.cpu()


@pytest.mark.parametrize("dv", [128, 64])
@pytest.mark.parametrize("G", [1, 2, 3, 7])
def test_segments_match_oracle(dv, G):
    """T = 48 chunks + 17 tokens, state in: every segment count within the
    bf16 tolerance of the oracle, output and final state."""
    B, H, T = 1, 3, 64 * 48 + 17
    inp = inputs.generate(B, T, H, 128, dv, "bf16", seed=4100 + G + dv)
    s0 = _state(B, H, 128, dv, seed=G)
    o, s = _causal(inp, s0, G)
    o_ref, s_ref = oracle_heads(inp, state_in=s0)
    assert rel_err(o, o_ref) <= TOL16
    assert rel_err(s, s_ref) <= TOL16


def test_segments_without_decay_walk_back_to_the_start():
    """alpha = 1: the bound never falls, so every segment walks back to the
    first chunk and starts from the initial state (exact, no approximation)."""
    B, H, T = 1, 2, 64 * 24 + 9
    inp = inputs.generate(B, T, H, 128, 128, "bf16", seed=4200)
    inp["alpha"] = torch.ones_like(inp["alpha"])
    inp["beta"] = 0.5 * inp["beta"]
    s0 = _state(B, H, 128, 128, seed=3)
    o, s = _causal(inp, s0, 4)
    o_ref, s_ref = oracle_heads(inp, state_in=s0)
    assert rel_err(o, o_ref) <= TOL16
    assert rel_err(s, s_ref) <= TOL16


def test_segments_with_longer_keys():
    """Keys of norm 1.5: beta |k|^2 exceeds 2 on some tokens, so the bound's
    key term max(1, |1 - beta |k|^2|) is active; parity still holds."""
    B, H, T = 1, 2, 64 * 32 + 40
    inp = inputs.generate(B, T, H, 128, 128, "bf16", seed=4300)
    inp["k"] = (inp["k"].float() * 1.5).to(torch.bfloat16)
    s0 = _state(B, H, 128, 128, seed=4)
    o, s = _causal(inp, s0, 5)
    o_ref, s_ref = oracle_heads(inp, state_in=s0)
    assert rel_err(o, o_ref) <= TOL16
    assert rel_err(s, s_ref) <= TOL16


@pytest.mark.parametrize("gates", ["default", "skewed"])
def test_segments_bidirectional_with_states(gates):
    """Both directions cut into 3 segments, initial states in both
    directions: output and both final states against the oracle."""
    B, H, T = 1, 2, 64 * 30 + 5
    inp = inputs.generate(B, T, H, 128, 128, "bf16", seed=4400, gates=gates)
    s0, r0 = _state(B, H, 128, 128, seed=5), _state(B, H, 128, 128, seed=6)
    d = to_dev(inp)
    with _Segments(3):
        o, sf, sb = gdn.scan_bidir(d["q"], d["k"], d["v"], d["alpha"], d["beta"], state=s0.cuda(),
                                   state_bwd=r0.cuda(), return_states=True)
    torch.cuda.synchronize()
    o_ref, sf_ref, sb_ref = oracle_heads(inp, mode="bidir", state_in=s0, state_in_bwd=r0, with_bwd=True)
    assert rel_err(o, o_ref) <= TOL16
    assert rel_err(sf, sf_ref) <= TOL16
    assert rel_err(sb, sb_ref) <= TOL16


def test_many_heads_prep_then_chain():
    """120 chains leave too few SMs for a fused launch: prep, then the chain
    launch, with two segments per chain; sampled heads against the oracle."""
    B, H, T = 2, 60, 64 * 20 + 3
    inp = inputs.generate(B, T, H, 128, 128, "bf16", seed=4500)
    s0 = _state(B, H, 128, 128, seed=7)
    gdn.gdn_set_kernel_timing(1)
    gdn.gdn_read_kernel_timing()
    try:
        o, s = _causal(inp, s0, 2)
        names = set(gdn.gdn_read_kernel_timing())
    finally:
        gdn.gdn_set_kernel_timing(0)
    assert {"tc_prep", "tc_chain"} <= names, names
    heads = [0, 37, 59]
    o_ref, s_ref = oracle_heads(inp, heads=heads, state_in=s0)
    assert rel_err(o[:, :, heads], o_ref) <= TOL16
    assert rel_err(s[:, heads], s_ref) <= TOL16


def test_segment_counts_agree_with_each_other():
    """The same inputs with 1 and 6 segments: the outputs differ only by
    rounding (the dropped state is below 2^-30 of its size)."""
    B, H, T = 1, 2, 64 * 60
    inp = inputs.generate(B, T, H, 128, 128, "bf16", seed=4600)
    s0 = _state(B, H, 128, 128, seed=8)
    o1, s1 = _causal(inp, s0, 1)
    o6, s6 = _causal(inp, s0, 6)
    ref = o1.double().numpy()
    assert np.isfinite(ref).all()
    assert rel_err(o6, ref) <= 1e-2
    assert rel_err(s6, s1.double().numpy()) <= 1e-2
