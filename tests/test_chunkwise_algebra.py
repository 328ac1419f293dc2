"""The chunkwise evaluation order the kernels use equals the sequential
recurrence (FP64, CPU only).  See tests/chunkwise_np.py for the algebra."""
import numpy as np
import pytest

import oracle
from tests import chunkwise_np as cw


def _inputs(rng, B, T, H, dk, dv, gates="default"):
    q = rng.standard_normal((B, T, H, dk))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    if gates == "skewed":      # fast forgetting: log alpha in [-2, 0]
        a = np.exp(-2.0 * rng.uniform(size=(B, T, H)))
        b = rng.uniform(0.9, 1.0, (B, T, H))
    else:
        a = np.exp(-np.logaddexp(0, rng.standard_normal((B, T, H))) * 0.05)
        b = 1 / (1 + np.exp(-rng.standard_normal((B, T, H))))
    return q, k, v, a, b


@pytest.mark.parametrize("C", [4, 16, 64])
@pytest.mark.parametrize("T", [1, 5, 64, 65, 130])
@pytest.mark.parametrize("mode", ["causal", "reverse", "bidir"])
def test_chunkwise_matches_sequential(C, T, mode):
    rng = np.random.default_rng(100 + C + T)
    B, H, dk, dv = 1, 2, 8, 6
    q, k, v, a, b = _inputs(rng, B, T, H, dk, dv)
    S0 = rng.standard_normal((B, H, dk, dv))
    R0 = rng.standard_normal((B, H, dk, dv))
    o, sf, sb = oracle.scan(q, k, v, a, b, mode, state_in=S0, state_in_bwd=R0)
    o2, sf2, sb2 = cw.scan(q, k, v, a, b, mode, state_in=S0, state_in_bwd=R0, C=C)
    np.testing.assert_allclose(o2, o, rtol=1e-10, atol=1e-10)
    if sf is not None:
        np.testing.assert_allclose(sf2, sf, rtol=1e-10, atol=1e-10)
    if sb is not None:
        np.testing.assert_allclose(sb2, sb, rtol=1e-10, atol=1e-10)


def test_chunkwise_skewed_gates_long_decay():
    """log alpha in [-2,0] drives within-chunk cumulative log-gates to about
    -64; the chunk algebra only ever forms exp of non-positive differences."""
    rng = np.random.default_rng(7)
    q, k, v, a, b = _inputs(rng, 1, 200, 1, 16, 16, gates="skewed")
    o, sf, _ = oracle.scan(q, k, v, a, b)
    o2, sf2, _ = cw.scan(q, k, v, a, b, C=64)
    np.testing.assert_allclose(o2, o, rtol=1e-9, atol=1e-10)
    np.testing.assert_allclose(sf2, sf, rtol=1e-9, atol=1e-10)
