"""The pins must catch plausible slips in the oracle (CPU only).

Each case compiles a copy of the oracle's C source with one planted mistake
into a temporary directory, swaps it in for the real library, and checks that
at least one pin of `test_oracle_pins.py` fails.  The real oracle is put
back afterwards.
"""
import ctypes
import inspect
import json
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "gdn_oracle.c")

WRITE_LINE = "row[j] = a * (row[j] - e * ki * p[j]) + w * ki * v[j];"
CAUSAL_BODY = """            transition(S, p, J->k + tok * dk, J->v + tok * dv, J->alpha[tok],
                       J->erase[tok], J->write[tok], dk, dv);
            readout(S, J->q + tok * dk, dk, dv, J->o + tok * dv, 0);"""
REVERSE_BODY = """            readout(S, J->q + tok * dk, dk, dv, J->o + tok * dv, acc);
            transition(S, p, J->k + tok * dk, J->v + tok * dv, J->alpha[tok],
                       J->erase[tok], J->write[tok], dk, dv);"""

MUTATIONS = {
    "erase_dropped": (WRITE_LINE, "row[j] = a * (row[j]) + w * ki * v[j];"),
    "erase_sign_flipped": (WRITE_LINE, "row[j] = a * (row[j] + e * ki * p[j]) + w * ki * v[j];"),
    "alpha_on_write": (WRITE_LINE, "row[j] = a * (row[j] - e * ki * p[j] + w * ki * v[j]);"),
    "alpha_dropped": (WRITE_LINE, "row[j] = (row[j] - e * ki * p[j]) + w * ki * v[j];"),
    "write_dropped": (WRITE_LINE, "row[j] = a * (row[j] - e * ki * p[j]);"),
    "erase_uses_alpha_twice": (WRITE_LINE, "row[j] = a * (row[j] - a * e * ki * p[j]) + w * ki * v[j];"),
    "causal_readout_before_write": (CAUSAL_BODY, """            readout(S, J->q + tok * dk, dk, dv, J->o + tok * dv, 0);
            transition(S, p, J->k + tok * dk, J->v + tok * dv, J->alpha[tok],
                       J->erase[tok], J->write[tok], dk, dv);"""),
    "reverse_readout_after_write": (REVERSE_BODY, """            transition(S, p, J->k + tok * dk, J->v + tok * dv, J->alpha[tok],
                       J->erase[tok], J->write[tok], dk, dv);
            readout(S, J->q + tok * dk, dk, dv, J->o + tok * dv, acc);"""),
    "readout_transposed_state": ("acc += S[(size_t)i * dv + j] * q[i];",
                                 "acc += S[(size_t)j * dk + i] * q[i];"),
    "erase_projects_query": ("for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * k[i];\n        p[j] = acc;",
                             "for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * k[0];\n        p[j] = acc;"),
    "state_in_ignored": ("if (J->s_fwd0) memcpy(S, J->s_fwd0", "if (0) memcpy(S, J->s_fwd0"),
    "bidir_overwrites_causal": ("const int acc = (J->mode == 2);", "const int acc = 0;"),
}


def _pin_functions():
    out = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        if name == "test_worked_examples":
            for ex in pins._golden():
                out.append((name + "[" + ex["name"] + "]", lambda ex=ex: pins.test_worked_examples(ex)))
        elif name == "test_split_calls_equal_one_call":
            out.append((name, lambda: pins.test_split_calls_equal_one_call(17)))
        elif name == "test_vda_one_token_frames_are_the_delta_rule":
            for unit in (True, False):
                out.append((name + "[%s]" % unit, lambda unit=unit: pins.test_vda_one_token_frames_are_the_delta_rule(unit)))
        else:
            out.append((name, fn))
    return out


@pytest.mark.parametrize("mutation", sorted(MUTATIONS))
def test_planted_mistake_is_caught(mutation, tmp_path):
    old, new = MUTATIONS[mutation]
    src = open(SRC).read()
    assert src.count(old) >= 1, "mutation anchor not found: %s" % mutation
    mutated = src.replace(old, new)
    c_path = tmp_path / "mut.c"
    so_path = tmp_path / "libmut.so"
    c_path.write_text(mutated)
    subprocess.check_call(["gcc", "-O1", "-std=c99", "-fPIC", "-shared", "-pthread",
                           str(c_path), "-o", str(so_path)])
    real = oracle._load()
    lib = ctypes.CDLL(str(so_path))
    lib.gdn_oracle_scan.argtypes = real.gdn_oracle_scan.argtypes
    lib.gdn_oracle_scan.restype = ctypes.c_int
    failed = []
    oracle._lib = lib
    try:
        for name, fn in _pin_functions():
            try:
                fn()
            except AssertionError:
                failed.append(name)
    finally:
        oracle._lib = real
    assert failed, "no pin caught the planted mistake %r" % mutation


# --------------------------------------------------------------------------
# The numpy oracles (frame-wise operator, readout epilogue): a mutated copy of
# the function's source replaces it while the pins run.
# --------------------------------------------------------------------------
NUMPY_MUTATIONS = {
    # frame-wise operator
    "vda_beta_dropped_in_gram": ("vda_scan", "K.T @ (be[:, None] * K)", "K.T @ K"),
    "vda_beta_dropped_in_write": ("vda_scan", "K.T @ (be[:, None] * V)", "K.T @ V"),
    "vda_plain_additive_write": ("vda_scan", "S = np.linalg.solve(eye + A, alpha_f[b, f, h] * S + Bm)",
                                 "S = alpha_f[b, f, h] * (S - A @ S) + Bm"),
    "vda_decay_after_solve": ("vda_scan", "S = np.linalg.solve(eye + A, alpha_f[b, f, h] * S + Bm)",
                              "S = alpha_f[b, f, h] * np.linalg.solve(eye + A, S) + Bm"),
    "vda_readout_before_write": ("vda_scan", """                    S = np.linalg.solve(eye + A, alpha_f[b, f, h] * S + Bm)
                    o[b, t, h] += q[b, t, h] @ S""", """                    o[b, t, h] += q[b, t, h] @ S
                    S = np.linalg.solve(eye + A, alpha_f[b, f, h] * S + Bm)"""),
    "vda_reverse_not_strict": ("vda_scan", """                    o[b, t, h] += q[b, t, h] @ R
                    R = np.linalg.solve(eye + A, alpha_f[b, f, h] * R + Bm)""", """                    R = np.linalg.solve(eye + A, alpha_f[b, f, h] * R + Bm)
                    o[b, t, h] += q[b, t, h] @ R"""),
    "vda_state_in_ignored": ("vda_scan", "S = np.zeros((dk, dv)) if s0 is None else s0[b, h].copy()",
                             "S = np.zeros((dk, dv))"),
    # readout epilogue
    "readout_no_norm": ("readout_gate", "inv = 1.0 / np.sqrt(np.mean(row * row) + eps)", "inv = 1.0"),
    "readout_sum_not_mean": ("readout_gate", "np.mean(row * row)", "np.sum(row * row)"),
    "readout_gate_inverted": ("readout_gate", "(1.0 + np.exp(-flat_z[r, j]))", "(1.0 + np.exp(flat_z[r, j]))"),
    "readout_gain_dropped": ("readout_gate", "row[j] * inv * g[j]", "row[j] * inv"),
    "readout_eps_outside": ("readout_gate", "np.sqrt(np.mean(row * row) + eps)", "(np.sqrt(np.mean(row * row)) + eps)"),
}


@pytest.mark.parametrize("mutation", sorted(NUMPY_MUTATIONS))
def test_planted_mistake_in_numpy_oracle_is_caught(mutation):
    fname, old, new = NUMPY_MUTATIONS[mutation]
    real = getattr(oracle, fname)
    src = inspect.getsource(real)
    assert src.count(old) >= 1, "mutation anchor not found: %s" % mutation
    ns = {}
    exec(compile(src.replace(old, new), "<mutated %s>" % fname, "exec"), oracle.__dict__, ns)
    failed = []
    setattr(oracle, fname, ns[fname])
    try:
        for name, fn in _pin_functions():
            try:
                fn()
            except AssertionError:
                failed.append(name)
    finally:
        setattr(oracle, fname, real)
    assert failed, "no pin caught the planted mistake %r" % mutation
