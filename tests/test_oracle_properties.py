"""Randomised properties of the fp64 oracle (no GPU), drawn by hypothesis over
small shapes, decays in [0, 1] (0 and 1 included) and block lengths:

- the three forms agree (recurrent, parallel, chunkwise: the page "Retentive
  Networks -- Microsoft ...", section "Il meccanismo", names them equivalent);
- the chunkwise result does not depend on the block length;
- the state after consecutive runs folds from the runs' own states:
  S = gamma^len S + D, the identity the state-only call and the state fold use;
- the backward's gradients are linear in the upstream gradients.
"""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle

shapes = st.tuples(st.integers(1, 2), st.integers(1, 3), st.integers(1, 24), st.integers(1, 5), st.integers(1, 5))
gammas = st.lists(st.sampled_from([0.0, 0.25, 0.5, 0.9, 0.99, 1.0]), min_size=3, max_size=3)


def _inputs(shape, seed):
    B, H, L, dk, dv = shape
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, H, L, dk)), rng.standard_normal((B, H, L, dk)),
            rng.standard_normal((B, H, L, dv)), rng.standard_normal((B, H, dk, dv)))


@settings(max_examples=60, deadline=None)
@given(shapes, gammas, st.integers(1, 30), st.integers(0, 2 ** 31 - 1))
def test_forms_agree_and_chunk_invariance(shape, gam, C, seed):
    q, k, v, s0 = _inputs(shape, seed)
    g = np.array(gam[:shape[1]])
    y_r, s_r = oracle.recurrent(q, k, v, g, s0)
    y_c, s_c = oracle.chunkwise(q, k, v, g, C, s0)
    y_p, _ = oracle.parallel(q, k, v, g, s0)
    scale = max(1.0, np.abs(y_r).max())
    assert np.abs(y_c - y_r).max() <= 1e-10 * scale and np.abs(y_p - y_r).max() <= 1e-10 * scale
    assert np.abs(s_c - s_r).max() <= 1e-10 * max(1.0, np.abs(s_r).max())


@settings(max_examples=60, deadline=None)
@given(shapes, gammas, st.lists(st.integers(0, 9), min_size=1, max_size=4), st.integers(0, 2 ** 31 - 1))
def test_state_folds_from_run_states(shape, gam, lens, seed):
    B, H, _, dk, dv = shape
    L = sum(lens)
    q, k, v, s0 = _inputs((B, H, L, dk, dv), seed)
    g = np.array(gam[:H])
    _, s_ref = oracle.recurrent(q, k, v, g, s0)
    s = s0.copy()
    t = 0
    for n in lens:
        _, d = oracle.recurrent(q[:, :, t:t + n], k[:, :, t:t + n], v[:, :, t:t + n], g)  # the run from zero
        s = (g[None, :, None, None] ** n) * s + d
        t += n
    assert np.abs(s - s_ref).max() <= 1e-10 * max(1.0, np.abs(s_ref).max())


@settings(max_examples=30, deadline=None)
@given(st.tuples(st.integers(1, 2), st.integers(1, 2), st.integers(1, 10), st.integers(1, 4), st.integers(1, 4)),
       gammas, st.integers(0, 2 ** 31 - 1))
def test_backward_is_linear_in_upstream_gradients(shape, gam, seed):
    B, H, L, dk, dv = shape
    q, k, v, s0 = _inputs(shape, seed)
    rng = np.random.default_rng(seed + 1)
    dy1, dy2 = rng.standard_normal((2, B, H, L, dv))
    ds1, ds2 = rng.standard_normal((2, B, H, dk, dv))
    g = np.array(gam[:H])
    a = oracle.backward(q, k, v, g, dy1, s0, ds1)
    b = oracle.backward(q, k, v, g, dy2, s0, ds2)
    c = oracle.backward(q, k, v, g, 2.0 * dy1 - dy2, s0, 2.0 * ds1 - ds2)
    for x, y, z in zip(a, b, c):
        assert np.allclose(z, 2.0 * x - y, rtol=1e-10, atol=1e-10)
