"""Pins for the FP64 oracle (CPU only).

Each test checks the oracle against something other than itself: a closed
form, an invariant of the recurrence, brute force written in a different
association, a hand-derived worked example, or an identity that links two
modes of the oracle.  Together they are chosen so that a plausible slip in
the oracle (a dropped term, a flipped sign, a readout taken before instead of
after the write, alpha applied to the write, a transposed state) fails at
least one of them.  dk != dv in most cases, so a transposed state cannot pass.
"""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def _rand(rng, B, T, H, dk, dv, unit_keys=True):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    if unit_keys:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    a = rng.uniform(0.3, 1.0, (B, T, H))
    b = rng.uniform(0.0, 1.0, (B, T, H))
    return q, k, v, a, b


# --------------------------------------------------------------------------
# worked examples (hand derivations, tests/golden/worked_examples.json)
# --------------------------------------------------------------------------
def _golden():
    with open(GOLDEN) as f:
        return json.load(f)["examples"]


@pytest.mark.parametrize("ex", _golden(), ids=lambda e: e["name"])
def test_worked_examples(ex):
    T = len(ex["alpha"])
    sh = lambda key, d: np.array(ex[key], np.float64).reshape(1, T, 1, d)
    q, k, v = sh("q", ex["dk"]), sh("k", ex["dk"]), sh("v", ex["dv"])
    a = np.array(ex["alpha"]).reshape(1, T, 1)
    b = np.array(ex["beta"]).reshape(1, T, 1)
    o, s, _ = oracle.scan(q, k, v, a, b, "causal")
    np.testing.assert_array_equal(o[0, :, 0], np.array(ex["o_causal"]))
    np.testing.assert_array_equal(s[0, 0], np.array(ex["state_causal"]))
    if "o_reverse" in ex:
        o_r, _, _ = oracle.scan(q, k, v, a, b, "reverse")
        np.testing.assert_array_equal(o_r[0, :, 0], np.array(ex["o_reverse"]))
        o_b, _, _ = oracle.scan(q, k, v, a, b, "bidir")
        np.testing.assert_array_equal(o_b[0, :, 0], np.array(ex["o_bidir"]))


# --------------------------------------------------------------------------
# closed forms: erase switched off (e = 0, w = beta or 1)
# --------------------------------------------------------------------------
def _decay(a):
    """D[t, s] = prod_{s < m <= t} a_m for s <= t, else 0 (one sequence)."""
    c = np.cumsum(np.log(a))
    D = np.exp(c[:, None] - c[None, :])
    return np.tril(D)


def test_plain_linear_attention():
    """e=0, w=1, alpha=1: o_t = sum_{s<=t} (q_t . k_s) v_s."""
    rng = np.random.default_rng(1)
    q, k, v, a, b = _rand(rng, 2, 37, 3, 5, 7, unit_keys=False)
    ones, zeros = np.ones_like(a), np.zeros_like(a)
    o, _, _ = oracle.scan(q, k, v, ones, b, erase=zeros, write=ones)
    for bb in range(2):
        for h in range(3):
            A = np.tril(q[bb, :, h] @ k[bb, :, h].T)
            np.testing.assert_allclose(o[bb, :, h], A @ v[bb, :, h], rtol=1e-12, atol=1e-12)


def test_gated_decay_sum():
    """e=0, w=1: o_t = sum_{s<=t} (prod_{s<m<=t} alpha_m) (q_t . k_s) v_s."""
    rng = np.random.default_rng(2)
    q, k, v, a, b = _rand(rng, 1, 41, 2, 6, 4, unit_keys=False)
    ones, zeros = np.ones_like(a), np.zeros_like(a)
    o, _, _ = oracle.scan(q, k, v, a, b, erase=zeros, write=ones)
    for h in range(2):
        A = (q[0, :, h] @ k[0, :, h].T) * _decay(a[0, :, h])
        np.testing.assert_allclose(o[0, :, h], A @ v[0, :, h], rtol=1e-11, atol=1e-12)


def test_gated_decay_sum_with_write_coefficient():
    """e=0, w=beta: the write is scaled by beta_s and never by alpha_s."""
    rng = np.random.default_rng(3)
    q, k, v, a, b = _rand(rng, 1, 23, 1, 3, 5, unit_keys=False)
    o, _, _ = oracle.scan(q, k, v, a, b, erase=np.zeros_like(a), write=b)
    A = (q[0, :, 0] @ k[0, :, 0].T) * _decay(a[0, :, 0]) * b[0, None, :, 0]
    np.testing.assert_allclose(o[0, :, 0], A @ v[0, :, 0], rtol=1e-11, atol=1e-12)


def test_beta_zero_pins_state_in():
    """Literal beta = 0 (no erase, no write): o_t = (prod_{m<=t} alpha_m) S_0^T q_t
    and the final state is (prod alpha) S_0."""
    rng = np.random.default_rng(4)
    q, k, v, a, _ = _rand(rng, 2, 19, 2, 4, 6)
    S0 = rng.standard_normal((2, 2, 4, 6))
    b = np.zeros_like(a)
    o, s, _ = oracle.scan(q, k, v, a, b, state_in=S0)
    cp = np.cumprod(a, axis=1)
    want = cp[..., None] * np.einsum("bthi,bhij->bthj", q, S0)
    np.testing.assert_allclose(o, want, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(s, cp[:, -1, :, None, None] * S0, rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# the delta-rule erase
# --------------------------------------------------------------------------
def test_full_erase_retrieves_last_value():
    """beta = 1 and a unit key: S_t^T k_t = v_t exactly, whatever S_{t-1}
    and alpha_t are.  Reading with q_t = k_t returns v_t."""
    rng = np.random.default_rng(5)
    q, k, v, a, b = _rand(rng, 1, 30, 3, 8, 5)
    o, _, _ = oracle.scan(k, k, v, a, np.ones_like(b))
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-12)


def test_partial_erase_identity():
    """Unit key: S_t^T k_t = alpha_t (1 - beta_t) S_{t-1}^T k_t + beta_t v_t."""
    rng = np.random.default_rng(6)
    q, k, v, a, b = _rand(rng, 1, 25, 2, 6, 3)
    _, S_prev, _ = oracle.scan(q[:, :-1], k[:, :-1], v[:, :-1], a[:, :-1], b[:, :-1])
    qq = q.copy()
    qq[:, -1] = k[:, -1]  # read the last token with its own key
    o, _, _ = oracle.scan(qq, k, v, a, b)
    t = -1
    for h in range(2):
        kt = k[0, t, h]
        want = a[0, t, h] * (1 - b[0, t, h]) * (S_prev[0, h].T @ kt) + b[0, t, h] * v[0, t, h]
        np.testing.assert_allclose(o[0, t, h], want, rtol=1e-12, atol=1e-12)


def test_projection_pythagoras_and_monotone_norm():
    """beta = 1, unit keys: (I - k k^T) is an orthogonal projection and k v^T
    is orthogonal to its range, so
    ||S_t||_F^2 = alpha_t^2 (||S_{t-1}||^2 - ||S_{t-1}^T k_t||^2) + ||v_t||^2;
    with v = 0 the state norm never increases."""
    rng = np.random.default_rng(7)
    B, T, H, dk, dv = 1, 12, 1, 5, 4
    q, k, v, a, b = _rand(rng, B, T, H, dk, dv)
    S0 = rng.standard_normal((B, H, dk, dv))
    ones = np.ones_like(b)
    prev = S0[0, 0]
    for t in range(1, T + 1):
        _, S, _ = oracle.scan(q[:, :t], k[:, :t], v[:, :t], a[:, :t], ones[:, :t], state_in=S0)
        kt, vt, at = k[0, t - 1, 0], v[0, t - 1, 0], a[0, t - 1, 0]
        want = at ** 2 * (np.sum(prev ** 2) - np.sum((prev.T @ kt) ** 2)) + np.sum(vt ** 2)
        np.testing.assert_allclose(np.sum(S[0, 0] ** 2), want, rtol=1e-12)
        prev = S[0, 0]
    # v = 0, alpha = 1: non-increasing Frobenius norm
    zv = np.zeros_like(v)
    norms = []
    for t in range(0, T + 1):
        _, S, _ = oracle.scan(q[:, :t], k[:, :t], zv[:, :t], np.ones_like(a[:, :t]),
                              ones[:, :t], state_in=S0)
        norms.append(np.linalg.norm(S))
    assert all(n1 <= n0 + 1e-12 for n0, n1 in zip(norms, norms[1:]))
    assert norms[-1] < norms[0]


def test_scalar_geometric_closed_form():
    """d_k = d_v = 1 with constant coefficients: S_t = c^t S_0 + w (1 - c^t)/(1 - c)
    where c = alpha (1 - beta k^2) and w = beta k v."""
    T = 50
    al, be, kk, vv, qq, s0 = 0.9, 0.3, 0.8, -1.7, 1.3, 2.5
    full = lambda x: np.full((1, T, 1, 1), x)
    o, s, _ = oracle.scan(full(qq), full(kk), full(vv), np.full((1, T, 1), al),
                          np.full((1, T, 1), be), state_in=np.full((1, 1, 1, 1), s0))
    c, w = al * (1 - be * kk * kk), be * kk * vv
    t = np.arange(1, T + 1)
    St = c ** t * s0 + w * (1 - c ** t) / (1 - c)
    np.testing.assert_allclose(o[0, :, 0, 0], qq * St, rtol=1e-12)
    np.testing.assert_allclose(s[0, 0, 0, 0], St[-1], rtol=1e-12)


def test_dense_transition_products():
    """Tiny sizes: S_T = (M_T ... M_1) S_0 + sum_s (M_T ... M_{s+1}) beta_s k_s v_s^T
    with M_t = alpha_t (I - beta_t k_t k_t^T), keys not normalised."""
    rng = np.random.default_rng(8)
    T, dk, dv = 7, 4, 3
    q, k, v, a, b = _rand(rng, 1, T, 1, dk, dv, unit_keys=False)
    S0 = rng.standard_normal((1, 1, dk, dv))
    M = [a[0, t, 0] * (np.eye(dk) - b[0, t, 0] * np.outer(k[0, t, 0], k[0, t, 0])) for t in range(T)]

    def prod(lo, hi):  # M_hi ... M_lo (0-based, inclusive), identity if empty
        P = np.eye(dk)
        for t in range(lo, hi + 1):
            P = M[t] @ P
        return P

    for t in range(T):
        S = prod(0, t) @ S0[0, 0]
        for s in range(t + 1):
            S = S + prod(s + 1, t) @ (b[0, s, 0] * np.outer(k[0, s, 0], v[0, s, 0]))
        o, _, _ = oracle.scan(q[:, :t + 1], k[:, :t + 1], v[:, :t + 1], a[:, :t + 1],
                              b[:, :t + 1], state_in=S0)
        np.testing.assert_allclose(o[0, t, 0], S.T @ q[0, t, 0], rtol=1e-11, atol=1e-12)


# --------------------------------------------------------------------------
# bidirectional: disjoint regions, each token counted once
# --------------------------------------------------------------------------
def test_bidir_linear_attention_counts_each_token_once():
    """e=0, w=1, alpha=1: causal covers s <= t, the reverse strict scan s > t,
    so the sum is full (non-causal) linear attention."""
    rng = np.random.default_rng(9)
    q, k, v, a, b = _rand(rng, 1, 33, 2, 5, 6, unit_keys=False)
    ones, zeros = np.ones_like(a), np.zeros_like(a)
    o, _, _ = oracle.scan(q, k, v, ones, b, mode="bidir", erase=zeros, write=ones)
    for h in range(2):
        np.testing.assert_allclose(o[0, :, h], (q[0, :, h] @ k[0, :, h].T) @ v[0, :, h],
                                   rtol=1e-11, atol=1e-11)
    o_r, _, _ = oracle.scan(q, k, v, ones, b, mode="reverse", erase=zeros, write=ones)
    np.testing.assert_array_equal(o_r[0, -1], 0.0)  # the last token sees nothing after it


def test_reverse_gated_decay_sum():
    """e=0, w=1: reverse strict readout o_t = sum_{s>t} (prod_{t<m<s} alpha_m)(q_t.k_s) v_s."""
    rng = np.random.default_rng(10)
    q, k, v, a, b = _rand(rng, 1, 29, 1, 4, 3, unit_keys=False)
    o, _, _ = oracle.scan(q, k, v, a, b, mode="reverse", erase=np.zeros_like(a),
                          write=np.ones_like(a))
    T = 29
    la = np.log(a[0, :, 0])
    D = np.zeros((T, T))
    for t in range(T):
        for s in range(t + 1, T):
            D[t, s] = np.exp(la[t + 1:s].sum())
    A = (q[0, :, 0] @ k[0, :, 0].T) * D
    np.testing.assert_allclose(o[0, :, 0], A @ v[0, :, 0], rtol=1e-11, atol=1e-12)


def test_reverse_equals_causal_on_reversed_suffix():
    """The reverse readout at t equals q_t read against the final state of a
    causal run over the time-reversed suffix x_T .. x_{t+1} (full delta rule)."""
    rng = np.random.default_rng(11)
    T = 13
    q, k, v, a, b = _rand(rng, 1, T, 2, 5, 3)
    o_r, _, R1 = oracle.scan(q, k, v, a, b, mode="reverse")
    rev = lambda x: x[:, ::-1]
    for t in range(T):
        suf = slice(t + 1, T)
        if t + 1 < T:
            _, S, _ = oracle.scan(rev(q[:, suf]), rev(k[:, suf]), rev(v[:, suf]),
                                  rev(a[:, suf]), rev(b[:, suf]))
            want = np.einsum("hij,hi->hj", S[0], q[0, t])
        else:
            want = np.zeros((2, 3))
        np.testing.assert_allclose(o_r[0, t], want, rtol=1e-12, atol=1e-13)
    _, S_all, _ = oracle.scan(rev(q), rev(k), rev(v), rev(a), rev(b))
    np.testing.assert_allclose(R1, S_all, rtol=1e-12, atol=1e-13)


def test_bidir_with_initial_states_in_both_directions():
    """Bidirectional with a causal initial state S_0 and a reverse initial
    state R_{T+1}: the reverse readout at t is q_t read against a causal run
    over the time-reversed suffix x_T .. x_{t+1} started from R_{T+1}; the
    causal half is the causal scan from S_0; the two add up; the final reverse
    state R_1 is the causal state of the whole reversed sequence from R_{T+1}."""
    rng = np.random.default_rng(14)
    T, H, dk, dv = 9, 2, 4, 3
    q, k, v, a, b = _rand(rng, 1, T, H, dk, dv)
    S0 = rng.normal(size=(1, H, dk, dv))
    R0 = rng.normal(size=(1, H, dk, dv))
    o, sf, sb = oracle.scan(q, k, v, a, b, mode="bidir", state_in=S0, state_in_bwd=R0)
    o_c, s_c, _ = oracle.scan(q, k, v, a, b, state_in=S0)
    rev = lambda x: x[:, ::-1]
    for t in range(T):
        suf = slice(t + 1, T)
        if t + 1 < T:
            _, S, _ = oracle.scan(rev(q[:, suf]), rev(k[:, suf]), rev(v[:, suf]),
                                  rev(a[:, suf]), rev(b[:, suf]), state_in=R0)
        else:
            S = R0
        want = o_c[0, t] + np.einsum("hij,hi->hj", S[0], q[0, t])
        np.testing.assert_allclose(o[0, t], want, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(sf, s_c, rtol=1e-12, atol=1e-13)
    _, S_all, _ = oracle.scan(rev(q), rev(k), rev(v), rev(a), rev(b), state_in=R0)
    np.testing.assert_allclose(sb, S_all, rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# streaming: state in / state out
# --------------------------------------------------------------------------
@pytest.mark.parametrize("split", [0, 1, 17, 63, 64, 65, 99, 100])
def test_split_calls_equal_one_call(split):
    rng = np.random.default_rng(12)
    q, k, v, a, b = _rand(rng, 2, 100, 2, 6, 5)
    o, s, _ = oracle.scan(q, k, v, a, b)
    part = lambda x, sl: x[:, sl]
    s1 = slice(0, split)
    s2 = slice(split, 100)
    o1, st, _ = oracle.scan(part(q, s1), part(k, s1), part(v, s1), part(a, s1), part(b, s1))
    o2, st2, _ = oracle.scan(part(q, s2), part(k, s2), part(v, s2), part(a, s2), part(b, s2),
                             state_in=st)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=1), o, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(st2, s, rtol=1e-12, atol=1e-13)


def test_empty_sequence_passes_state_through():
    rng = np.random.default_rng(13)
    S0 = rng.standard_normal((1, 3, 4, 2))
    e = np.zeros((1, 0, 3, 4))
    o, s, _ = oracle.scan(e, e, np.zeros((1, 0, 3, 2)), np.zeros((1, 0, 3)), np.zeros((1, 0, 3)),
                          state_in=S0)
    assert o.shape == (1, 0, 3, 2)
    np.testing.assert_array_equal(s, S0)


def test_threads_do_not_change_results():
    rng = np.random.default_rng(14)
    q, k, v, a, b = _rand(rng, 3, 40, 5, 8, 8)
    o1, s1, _ = oracle.scan(q, k, v, a, b, mode="bidir", threads=1)
    o2, s2, _ = oracle.scan(q, k, v, a, b, mode="bidir", threads=7)
    np.testing.assert_array_equal(o1, o2)


# --------------------------------------------------------------------------
# readout epilogue: RMS norm over d_v, per-channel gain, sigmoid gate
# --------------------------------------------------------------------------
def test_readout_worked_example():
    """o = (3, 4): mean of squares 12.5; gate z = (0, ln 3) gives sigmoid
    (1/2, 3/4); gain (2, 1): both outputs equal 3 / sqrt(12.5)."""
    o = np.array([3.0, 4.0]).reshape(1, 1, 1, 2)
    z = np.array([0.0, np.log(3.0)]).reshape(1, 1, 1, 2)
    y = oracle.readout_gate(o, z, gamma=np.array([2.0, 1.0]), eps=0.0)
    np.testing.assert_allclose(y.ravel(), [3 / np.sqrt(12.5)] * 2, rtol=1e-15)


def test_readout_normalises_and_gates():
    rng = np.random.default_rng(21)
    o = rng.normal(size=(2, 5, 3, 8)) * rng.uniform(0.1, 10, size=(2, 5, 3, 1))
    open_gate = np.full(o.shape, 40.0)         # sigmoid(40) = 1 in float64
    y = oracle.readout_gate(o, open_gate, eps=0.0)
    np.testing.assert_allclose(np.mean(y * y, axis=-1), 1.0, rtol=1e-14)     # unit RMS per row
    np.testing.assert_allclose(oracle.readout_gate(7.5 * o, open_gate, eps=0.0), y, rtol=1e-14)
    np.testing.assert_allclose(oracle.readout_gate(o, np.zeros(o.shape), eps=0.0), 0.5 * y, rtol=1e-14)
    g = rng.uniform(0.5, 2.0, size=8)
    np.testing.assert_allclose(oracle.readout_gate(o, open_gate, gamma=g, eps=0.0), y * g, rtol=1e-14)
    # eps adds to the mean of squares: a row of zeros stays zero, a constant row c gives c / sqrt(c^2 + eps)
    row = np.full((1, 1, 1, 8), 0.3)
    np.testing.assert_allclose(oracle.readout_gate(row, np.full(row.shape, 40.0), eps=0.01),
                               0.3 / np.sqrt(0.09 + 0.01), rtol=1e-14)


# --------------------------------------------------------------------------
# frame-wise delta operator (VDA)
# --------------------------------------------------------------------------
def _vda_inputs(rng, B, F, U, H, dk, dv, unit=True):
    q = rng.normal(size=(B, F * U, H, dk))
    k = rng.normal(size=(B, F * U, H, dk))
    if unit:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.normal(size=(B, F * U, H, dv))
    a = rng.uniform(0.5, 1.0, size=(B, F, H))
    b = rng.uniform(0.0, 1.0, size=(B, F * U, H))
    return q, k, v, a, b


@pytest.mark.parametrize("unit", [True, False])
def test_vda_one_token_frames_are_the_delta_rule(unit):
    """U = 1: (I + b k k^T)^{-1} = I - c k k^T with c = b / (1 + b |k|^2), so a
    frame step is the gated delta rule with erase = write = c (Sherman-Morrison);
    checked against the token recurrence of the C oracle, causal and bidir."""
    rng = np.random.default_rng(31)
    q, k, v, a, b = _vda_inputs(rng, 2, 11, 1, 2, 5, 3, unit=unit)
    c = b / (1.0 + b * np.sum(k * k, axis=-1))
    S0 = rng.normal(size=(2, 2, 5, 3))
    R0 = rng.normal(size=(2, 2, 5, 3))
    for mode in ("causal", "bidir"):
        o, sf, sb = oracle.vda_scan(q, k, v, a, b, 1, mode=mode, state_in=S0, state_in_bwd=R0)
        o2, sf2, sb2 = oracle.scan(q, k, v, a, b, mode=mode, state_in=S0, state_in_bwd=R0, erase=c, write=c)
        np.testing.assert_allclose(o, o2, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(sf, sf2, rtol=1e-10, atol=1e-12)
        if mode == "bidir":
            np.testing.assert_allclose(sb, sb2, rtol=1e-10, atol=1e-12)


def test_vda_orthonormal_frame_is_a_token_scan():
    """A frame whose U keys are orthonormal: the key directions decouple, so
    the frame step equals the token-level delta rule over the frame's tokens
    with erase = write = b_u / (1 + b_u), the frame's decay applied at its
    first token only (and 1 at the others); the readout is that of the frame's
    final state."""
    rng = np.random.default_rng(32)
    B, F, U, H, dk, dv = 1, 4, 3, 1, 6, 2
    q, k, v, a, b = _vda_inputs(rng, B, F, U, H, dk, dv)
    for f in range(F):   # orthonormal keys within each frame
        Qm, _ = np.linalg.qr(rng.normal(size=(dk, U)))
        k[0, f * U:(f + 1) * U, 0] = Qm.T
    c = b / (1.0 + b)
    a_tok = np.ones((B, F * U, H))
    a_tok[:, ::U] = a
    S0 = rng.normal(size=(B, H, dk, dv))
    o, sf, _ = oracle.vda_scan(q, k, v, a, b, U, state_in=S0)
    _, S_tok, _ = oracle.scan(q, k, v, a_tok, b, state_in=S0, erase=c, write=c)
    np.testing.assert_allclose(sf, S_tok, rtol=1e-10, atol=1e-12)
    # readout per frame: every token of frame f reads the state after the frame
    S = S0[0, 0]
    for f in range(F):
        t = slice(f * U, (f + 1) * U)
        _, S_f, _ = oracle.scan(q[:, :(f + 1) * U], k[:, :(f + 1) * U], v[:, :(f + 1) * U],
                                a_tok[:, :(f + 1) * U], b[:, :(f + 1) * U], state_in=S0,
                                erase=c[:, :(f + 1) * U], write=c[:, :(f + 1) * U])
        np.testing.assert_allclose(o[0, t, 0], q[0, t, 0] @ S_f[0, 0], rtol=1e-10, atol=1e-12)


def test_vda_inherited_state_is_not_amplified():
    """With zero values (B_f = 0) a frame step maps S to alpha (I + A)^{-1} S,
    whose spectral norm is at most alpha: ||S_f||_2 <= alpha_f ||S_{f-1}||_2,
    whatever the keys (non-unit keys with large write strengths included)."""
    rng = np.random.default_rng(33)
    B, F, U, H, dk, dv = 1, 6, 40, 1, 8, 8
    q, k, v, a, b = _vda_inputs(rng, B, F, U, H, dk, dv, unit=False)
    k *= 3.0
    v[:] = 0.0
    S = rng.normal(size=(B, H, dk, dv))
    for f in range(F):
        sl = slice(f * U, (f + 1) * U)
        _, S_next, _ = oracle.vda_scan(q[:, sl], k[:, sl], v[:, sl], a[:, f:f + 1], b[:, sl], U, state_in=S)
        assert np.linalg.norm(S_next[0, 0], 2) <= a[0, f, 0] * np.linalg.norm(S[0, 0], 2) * (1 + 1e-12)
        S = S_next


def test_vda_reverse_is_causal_on_reversed_frames():
    """The reverse readout of frame f is the causal state of the frames after
    f taken in reverse order (from R_{F+1}); R_1 is that of all frames."""
    rng = np.random.default_rng(34)
    B, F, U, H, dk, dv = 1, 5, 4, 2, 5, 3
    q, k, v, a, b = _vda_inputs(rng, B, F, U, H, dk, dv)
    R0 = rng.normal(size=(B, H, dk, dv))
    o, _, R1 = oracle.vda_scan(q, k, v, a, b, U, mode="reverse", state_in_bwd=R0)

    def rev_frames(x, per_frame=False):   # reverse the frame order, keep token order inside a frame
        if per_frame:
            return x[:, ::-1]
        n = x.shape[1] // U
        return np.concatenate([x[:, f * U:(f + 1) * U] for f in range(n - 1, -1, -1)], axis=1)

    for f in range(F):
        t = slice(f * U, (f + 1) * U)
        if f + 1 < F:
            suf = slice((f + 1) * U, F * U)
            _, S, _ = oracle.vda_scan(rev_frames(q[:, suf]), rev_frames(k[:, suf]), rev_frames(v[:, suf]),
                                      rev_frames(a[:, f + 1:], True), rev_frames(b[:, suf]), U, state_in=R0)
        else:
            S = R0
        np.testing.assert_allclose(o[0, t], np.einsum("thi,hij->thj", q[0, t], S[0]), rtol=1e-10, atol=1e-12)
    _, S_all, _ = oracle.vda_scan(rev_frames(q), rev_frames(k), rev_frames(v), rev_frames(a, True),
                                  rev_frames(b), U, state_in=R0)
    np.testing.assert_allclose(R1, S_all, rtol=1e-10, atol=1e-12)
