"""Pins for the fp64 oracle: it is checked against things other than itself.

* hand-worked examples (tests/golden/, each with its citation);
* exact rational brute force on tiny inputs (fractions.Fraction, no rounding);
* closed forms: gamma = 1 is causal linear attention with no denominator
  (author responses on paperhub.cn, reply comparing Eq. (1) with RFA-Gate),
  computed with a running prefix sum; gamma = 0 keeps only the diagonal term;
* invariants the pages state or imply: the three forms agree (page
  "Retentive Networks -- Microsoft ...", section "Il meccanismo": three
  mathematically equivalent formulations), the result does not depend on the
  block length C, a sequence split at any point with the state carried
  reproduces the full call, and the map is linear in v and in the state.

``test_planted_mistakes_are_caught`` rebuilds the oracle with one plausible
mistake at a time and checks that these pins catch every one.
"""
from fractions import Fraction
import math
import os
import re
import shutil
import tempfile

import numpy as np
import pytest

import oracle
from tests import golden_io

RTOL = 1e-12


def rel_err(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    den = max(np.max(np.abs(b)), 1e-300)
    return float(np.max(np.abs(a - b)) / den)


def _tiny(B, H, L, dk, dv, seed, ints=False):
    rng = np.random.default_rng(seed)
    if ints:
        f = lambda *s: rng.integers(-3, 4, size=s).astype(np.float64)  # noqa: E731
    else:
        f = lambda *s: rng.standard_normal(s)  # noqa: E731
    return f(B, H, L, dk), f(B, H, L, dk), f(B, H, L, dv)


def _golden_inputs(inp, key):
    return inp[key][None, None]  # [1,1,L,d]


# ----------------------------------------------------------------- pin bodies
# Each pin takes the loaded oracle library so the planted-mistake test can run
# the same bodies against a mutated build.

def pin_three_token(lib):
    inp, cases = golden_io.load("three_token_example.txt")
    q, k, v = (_golden_inputs(inp, c) for c in "qkv")
    for g, exp in cases:
        gam = np.array([g])
        outs = [oracle.recurrent(q, k, v, gam, lib=lib), oracle.parallel(q, k, v, gam, lib=lib)]
        outs += [oracle.chunkwise(q, k, v, gam, C, lib=lib) for C in (1, 2, 3, 4)]
        for y, s in outs:
            assert np.array_equal(y[0, 0], exp["y"]), (g, y[0, 0], exp["y"])
            assert np.array_equal(s[0, 0], exp["S"]), (g, s[0, 0], exp["S"])


def pin_one_token_with_state(lib):
    inp, cases = golden_io.load("one_token_with_state.txt")
    q, k, v = (_golden_inputs(inp, c) for c in "qkv")
    s_in = inp["S_in"][None, None]
    for g, exp in cases:
        gam = np.array([g])
        for y, s in (oracle.recurrent(q, k, v, gam, s_in, lib=lib),
                     oracle.parallel(q, k, v, gam, s_in, lib=lib),
                     oracle.chunkwise(q, k, v, gam, 1, s_in, lib=lib)):
            assert np.array_equal(y[0, 0], exp["y"])
            assert np.array_equal(s[0, 0], exp["S"])


def pin_multihead_gamma_indexing(lib):
    inp, cases = golden_io.load("three_token_example.txt")
    q, k, v = (np.repeat(_golden_inputs(inp, c), 3, axis=1) for c in "qkv")
    gam = np.array([g for g, _ in cases])
    for y, s in (oracle.recurrent(q, k, v, gam, lib=lib), oracle.chunkwise(q, k, v, gam, 2, lib=lib)):
        for h, (_, exp) in enumerate(cases):
            assert np.array_equal(y[0, h], exp["y"])
            assert np.array_equal(s[0, h], exp["S"])


def _exact_bruteforce(q, k, v, g, s_in):
    """y_n = sum_{m<=n} g^(n-m) (q_n.k_m) v_m + g^(n+1) q_n S_in in exact rationals."""
    L, dk = q.shape
    dv = v.shape[1]
    F = lambda x: Fraction(float(x))  # noqa: E731  (inputs are small integers)
    y = [[Fraction(0)] * dv for _ in range(L)]
    for n in range(L):
        for m in range(n + 1):
            s = sum(F(q[n, i]) * F(k[m, i]) for i in range(dk)) * g ** (n - m)
            for j in range(dv):
                y[n][j] += s * F(v[m, j])
        for j in range(dv):
            y[n][j] += g ** (n + 1) * sum(F(q[n, i]) * F(s_in[i, j]) for i in range(dk))
    S = [[g ** L * F(s_in[i, j]) + sum(g ** (L - 1 - m) * F(k[m, i]) * F(v[m, j]) for m in range(L))
          for j in range(dv)] for i in range(dk)]
    return np.array([[float(x) for x in r] for r in y]), np.array([[float(x) for x in r] for r in S])


def pin_exact_rational(lib):
    for seed, (L, dk, dv), g in ((0, (7, 3, 2), Fraction(3, 4)), (1, (5, 2, 4), Fraction(1, 2)),
                                 (2, (6, 4, 3), Fraction(7, 8)), (3, (4, 3, 3), Fraction(0))):
        q, k, v = _tiny(1, 1, L, dk, dv, seed, ints=True)
        rng = np.random.default_rng(100 + seed)
        s_in = rng.integers(-2, 3, size=(1, 1, dk, dv)).astype(np.float64)
        y_ex, s_ex = _exact_bruteforce(q[0, 0], k[0, 0], v[0, 0], g, s_in[0, 0])
        gam = np.array([float(g)])
        for y, s in (oracle.recurrent(q, k, v, gam, s_in, lib=lib),
                     oracle.parallel(q, k, v, gam, s_in, lib=lib),
                     oracle.chunkwise(q, k, v, gam, 3, s_in, lib=lib)):
            assert rel_err(y[0, 0], y_ex) <= RTOL
            assert rel_err(s[0, 0], s_ex) <= RTOL


def pin_gamma_one_is_unnormalised_linear_attention(lib):
    q, k, v = _tiny(2, 3, 19, 5, 4, 7)
    gam = np.ones(3)
    # prefix sum of outer products, then a plain product: no denominator
    prefix = np.cumsum(np.einsum("bhld,bhle->bhlde", k, v), axis=2)
    y_ref = np.einsum("bhld,bhlde->bhle", q, prefix)
    for y, s in (oracle.recurrent(q, k, v, gam, lib=lib), oracle.parallel(q, k, v, gam, lib=lib),
                 oracle.chunkwise(q, k, v, gam, 4, lib=lib)):
        assert rel_err(y, y_ref) <= RTOL
        assert rel_err(s, prefix[:, :, -1]) <= RTOL


def pin_gamma_zero_is_diagonal(lib):
    q, k, v = _tiny(1, 2, 11, 3, 5, 8)
    gam = np.zeros(2)
    y_ref = np.einsum("bhl,bhle->bhle", np.einsum("bhld,bhld->bhl", q, k), v)
    s_ref = np.einsum("bhd,bhe->bhde", k[:, :, -1], v[:, :, -1])
    for y, s in (oracle.recurrent(q, k, v, gam, lib=lib), oracle.parallel(q, k, v, gam, lib=lib),
                 oracle.chunkwise(q, k, v, gam, 3, lib=lib)):
        assert rel_err(y, y_ref) <= RTOL
        assert rel_err(s, s_ref) <= RTOL


def pin_forms_agree(lib):
    for seed, L in enumerate((1, 2, 3, 5, 17, 64)):
        q, k, v = _tiny(1, 3, L, 4, 6, 20 + seed)
        gam = np.array([0.5, 0.9, 1.0])
        s_in = np.random.default_rng(seed).standard_normal((1, 3, 4, 6))
        y_r, s_r = oracle.recurrent(q, k, v, gam, s_in, lib=lib)
        y_p, s_p = oracle.parallel(q, k, v, gam, s_in, lib=lib)
        assert rel_err(y_p, y_r) <= RTOL and rel_err(s_p, s_r) <= RTOL
        for C in (1, 2, 3, 16, L, L + 5):
            y_c, s_c = oracle.chunkwise(q, k, v, gam, C, s_in, lib=lib)
            assert rel_err(y_c, y_r) <= RTOL and rel_err(s_c, s_r) <= RTOL


def pin_split_call(lib):
    q, k, v = _tiny(2, 2, 40, 3, 5, 31)
    gam = np.array([0.8, 0.97])
    y_full, s_full = oracle.recurrent(q, k, v, gam, lib=lib)
    for cut in (1, 13, 39):
        y1, s1 = oracle.chunkwise(q[:, :, :cut], k[:, :, :cut], v[:, :, :cut], gam, 8, lib=lib)
        y2, s2 = oracle.chunkwise(q[:, :, cut:], k[:, :, cut:], v[:, :, cut:], gam, 8, s1, lib=lib)
        assert rel_err(np.concatenate([y1, y2], axis=2), y_full) <= RTOL
        assert rel_err(s2, s_full) <= RTOL


def pin_linearity(lib):
    q, k, v1 = _tiny(1, 2, 9, 3, 4, 41)
    _, _, v2 = _tiny(1, 2, 9, 3, 4, 42)
    gam = np.array([0.7, 0.95])
    rng = np.random.default_rng(5)
    s1, s2 = rng.standard_normal((2, 1, 2, 3, 4))
    a, b = 1.75, -0.5
    y1, t1 = oracle.recurrent(q, k, v1, gam, s1, lib=lib)
    y2, t2 = oracle.recurrent(q, k, v2, gam, s2, lib=lib)
    y3, t3 = oracle.recurrent(q, k, a * v1 + b * v2, gam, a * s1 + b * s2, lib=lib)
    assert rel_err(y3, a * y1 + b * y2) <= 1e-11
    assert rel_err(t3, a * t1 + b * t2) <= 1e-11
    y4, _ = oracle.recurrent(3.0 * q, k, v1, gam, s1, lib=lib)
    assert rel_err(y4, 3.0 * y1) <= RTOL


def pin_groupnorm_golden(lib):
    inp, cases = golden_io.load("groupnorm_rows.txt")
    y = inp["y"][None, None]  # [1, 1, 2 tokens, dv 4]
    for eps, exp in cases:
        out = oracle.groupnorm(y, eps=eps, lib=lib)
        assert np.allclose(out[0, 0], exp["out"], rtol=0, atol=1e-9), (eps, out[0, 0])


def pin_groupnorm_invariants(lib):
    rng = np.random.default_rng(5)
    y = rng.standard_normal((2, 3, 5, 8)) * 3.0 + 1.5
    z = oracle.groupnorm(y, eps=0.0, lib=lib)
    # every (b, h, n) group: zero mean, unit mean square
    assert np.allclose(z.mean(-1), 0.0, atol=1e-12)
    assert np.allclose((z * z).mean(-1), 1.0, atol=1e-12)
    # invariant to a positive scale and a shift of the group
    assert np.allclose(oracle.groupnorm(2.5 * y - 7.0, eps=0.0, lib=lib), z, atol=1e-12)
    # eps only shrinks: the mean square is var / (var + eps) < 1
    ze = oracle.groupnorm(y, eps=0.5, lib=lib)
    assert np.all((ze * ze).mean(-1) < 1.0) and np.allclose(ze.mean(-1), 0.0, atol=1e-12)


def pin_groupnorm_heads(lib):
    rng = np.random.default_rng(6)
    y = rng.standard_normal((1, 2, 4, 6))
    base = oracle.groupnorm(y, lib=lib)
    y2 = y.copy()
    y2[0, 1] *= 3.0
    y2[0, 1, :, 0] += 1.0
    assert np.array_equal(oracle.groupnorm(y2, lib=lib)[0, 0], base[0, 0])  # head 0 untouched
    # per-head affine: head h uses weight[h*dv:(h+1)*dv], bias likewise
    w = np.concatenate([np.full(6, 1.0), np.full(6, 2.0)])
    b = np.concatenate([np.zeros(6), np.full(6, 0.25)])
    out = oracle.groupnorm(y, weight=w, bias=b, lib=lib)
    assert np.allclose(out[0, 0], base[0, 0], atol=1e-12)
    assert np.allclose(out[0, 1], 2.0 * base[0, 1] + 0.25, atol=1e-12)


def pin_backward_central_differences(lib):
    # L = sum(dy * y) is linear in each of q, k, v, so a central difference in
    # one entry is exact up to rounding
    rng = np.random.default_rng(9)
    B, H, L, dk, dv = 1, 2, 6, 3, 4
    q, k, v = (rng.standard_normal((B, H, L, d)) for d in (dk, dk, dv))
    dy = rng.standard_normal((B, H, L, dv))
    gam = np.array([0.8, 0.95])
    dq, dkk, dvv = oracle.parallel_backward(q, k, v, gam, dy, lib=lib)

    def loss(q_, k_, v_):
        return float(np.sum(dy * oracle.recurrent(q_, k_, v_, gam, lib=lib)[0]))

    eps = 0.5
    for arr, grad, which in ((q, dq, 0), (k, dkk, 1), (v, dvv, 2)):
        for idx in ((0, 0, 0, 0), (0, 1, 3, 1), (0, 1, 5, 2), (0, 0, 2, arr.shape[-1] - 1)):
            plus, minus = [x.copy() for x in (q, k, v)], [x.copy() for x in (q, k, v)]
            plus[which][idx] += eps
            minus[which][idx] -= eps
            fd = (loss(*plus) - loss(*minus)) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-9 * max(1.0, abs(fd)), (which, idx, fd, grad[idx])


def pin_backward_gamma_zero(lib):
    # gamma = 0 keeps only m = n: dq_n = (dy_n . v_n) k_n, dk_n = (dy_n . v_n) q_n, dv_n = (q_n . k_n) dy_n
    rng = np.random.default_rng(10)
    q, k = rng.standard_normal((2, 1, 2, 5, 3))
    v, dy = rng.standard_normal((2, 1, 2, 5, 4))
    dq, dkk, dvv = oracle.parallel_backward(q, k, v, np.zeros(2), dy, lib=lib)
    dyv = np.einsum("bhnj,bhnj->bhn", dy, v)[..., None]
    qk = np.einsum("bhni,bhni->bhn", q, k)[..., None]
    assert np.allclose(dq, dyv * k) and np.allclose(dkk, dyv * q) and np.allclose(dvv, qk * dy)


def pin_state_backward_central_differences(lib):
    # L = sum(dy * y) + sum(dS_out * S_out) is linear in each of q, k, v and
    # state_in separately, so a central difference in one entry is exact up to
    # rounding.  The forward is the pinned recurrence.
    rng = np.random.default_rng(11)
    B, H, L, dk, dv = 1, 2, 5, 3, 4
    q, k, v = (rng.standard_normal((B, H, L, d)) for d in (dk, dk, dv))
    s0 = rng.standard_normal((B, H, dk, dv))
    dy = rng.standard_normal((B, H, L, dv))
    dso = rng.standard_normal((B, H, dk, dv))
    gam = np.array([0.7, 0.9])
    grads = oracle.backward(q, k, v, gam, dy, s0, dso, lib=lib)

    def loss(q_, k_, v_, s_):
        y, so = oracle.recurrent(q_, k_, v_, gam, s_, lib=lib)
        return float(np.sum(dy * y) + np.sum(dso * so))

    eps = 0.5
    for which, idxs in ((0, ((0, 0, 0, 0), (0, 1, 4, 2))), (1, ((0, 0, 4, 1), (0, 1, 2, 0), (0, 1, 0, 2))),
                        (2, ((0, 0, 4, 3), (0, 1, 1, 0), (0, 0, 0, 2))), (3, ((0, 0, 0, 0), (0, 1, 2, 3)))):
        for idx in idxs:
            plus, minus = [x.copy() for x in (q, k, v, s0)], [x.copy() for x in (q, k, v, s0)]
            plus[which][idx] += eps
            minus[which][idx] -= eps
            fd = (loss(*plus) - loss(*minus)) / (2 * eps)
            g = grads[which][idx]
            assert abs(fd - g) <= 1e-9 * max(1.0, abs(fd)), (which, idx, fd, g)


def pin_state_backward_closed_forms(lib):
    rng = np.random.default_rng(12)
    q, k = rng.standard_normal((2, 1, 1, 4, 3))
    v, dy = rng.standard_normal((2, 1, 1, 4, 2))
    s0, dso = rng.standard_normal((2, 1, 1, 3, 2))
    # gamma = 1: plain sums; S_out = S0 + sum_m k_m^T v_m and y_n gains q_n S0
    dq, dkk, dvv, ds0 = oracle.backward(q, k, v, np.ones(1), dy, s0, dso, lib=lib)
    bq, bk, bv = oracle.parallel_backward(q, k, v, np.ones(1), dy, lib=lib)
    assert np.allclose(ds0[0, 0], dso[0, 0] + q[0, 0].T @ dy[0, 0])
    assert np.allclose(dq[0, 0], bq[0, 0] + dy[0, 0] @ s0[0, 0].T)
    assert np.allclose(dkk[0, 0], bk[0, 0] + v[0, 0] @ dso[0, 0].T)
    assert np.allclose(dvv[0, 0], bv[0, 0] + k[0, 0] @ dso[0, 0])
    # gamma = 0: S0 never reaches y or S_out; only the last token reaches S_out
    dq, dkk, dvv, ds0 = oracle.backward(q, k, v, np.zeros(1), dy, s0, dso, lib=lib)
    bq, bk, bv = oracle.parallel_backward(q, k, v, np.zeros(1), dy, lib=lib)
    assert np.array_equal(ds0, np.zeros_like(ds0)) and np.allclose(dq, bq)
    assert np.allclose(dkk[0, 0, :3], bk[0, 0, :3]) and np.allclose(dvv[0, 0, :3], bv[0, 0, :3])
    assert np.allclose(dkk[0, 0, 3], bk[0, 0, 3] + dso[0, 0] @ v[0, 0, 3])
    assert np.allclose(dvv[0, 0, 3], bv[0, 0, 3] + k[0, 0, 3] @ dso[0, 0])
    # no state given: the same as the backward without state, dS0 from dy alone
    dq, dkk, dvv, ds0 = oracle.backward(q, k, v, np.full(1, 0.5), dy, lib=lib)
    bq, bk, bv = oracle.parallel_backward(q, k, v, np.full(1, 0.5), dy, lib=lib)
    assert np.array_equal(dq, bq) and np.array_equal(dkk, bk) and np.array_equal(dvv, bv)
    w = 0.5 ** np.arange(1, 5)
    assert np.allclose(ds0[0, 0], (q[0, 0] * w[:, None]).T @ dy[0, 0])


def pin_gate_closed_forms(lib):
    ln3 = math.log(3.0)
    z = np.array([2.0, -3.0, 5.0, 7.0, 0.5])
    g = np.array([0.0, ln3, -ln3, 40.0, -1.5])
    sig = oracle.gate(z, g, "sigmoid", lib=lib)
    assert np.allclose(sig[:3], z[:3] * np.array([0.5, 0.75, 0.25]), rtol=1e-14, atol=0)
    sw = oracle.gate(z, g, "swish", lib=lib)
    assert np.allclose(sw[:3], z[:3] * np.array([0.0, 0.75 * ln3, -0.25 * ln3]), rtol=1e-14, atol=0)
    assert abs(sw[3] - 40.0 * 7.0) < 1e-12  # swish(x) -> x for large x
    assert np.array_equal(oracle.gate(z, g, "none", lib=lib), g * z)
    # sigmoid(x) + sigmoid(-x) = 1 and swish(x) - swish(-x) = x, elementwise
    ones = np.ones_like(z)
    assert np.allclose(oracle.gate(ones, g, "sigmoid", lib=lib) + oracle.gate(ones, -g, "sigmoid", lib=lib), 1.0)
    assert np.allclose(oracle.gate(ones, g, "swish", lib=lib) - oracle.gate(ones, -g, "swish", lib=lib), g)


ALL_PINS = [pin_three_token, pin_one_token_with_state, pin_multihead_gamma_indexing,
            pin_exact_rational, pin_gamma_one_is_unnormalised_linear_attention,
            pin_gamma_zero_is_diagonal, pin_forms_agree, pin_split_call, pin_linearity,
            pin_groupnorm_golden, pin_groupnorm_invariants, pin_groupnorm_heads,
            pin_backward_central_differences, pin_backward_gamma_zero,
            pin_state_backward_central_differences, pin_state_backward_closed_forms, pin_gate_closed_forms]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(oracle.load())


def test_state_shape_is_dk_by_dv():
    q, k, v = _tiny(2, 3, 5, 4, 7, 9)
    y, s = oracle.recurrent(q, k, v, np.full(3, 0.9))
    assert y.shape == (2, 3, 5, 7) and s.shape == (2, 3, 4, 7)


def test_empty_sequence_passes_state_through():
    q, k, v = _tiny(1, 2, 0, 3, 4, 1)
    s_in = np.random.default_rng(0).standard_normal((1, 2, 3, 4))
    for y, s in (oracle.recurrent(q, k, v, np.full(2, 0.5), s_in),
                 oracle.chunkwise(q, k, v, np.full(2, 0.5), 4, s_in)):
        assert y.shape == (1, 2, 0, 4) and np.array_equal(s, s_in)


def test_rejects_bad_gamma_and_chunk():
    q, k, v = _tiny(1, 1, 3, 2, 2, 0)
    for g in (-0.1, 1.5, float("nan")):
        with pytest.raises(ValueError):
            oracle.recurrent(q, k, v, np.array([g]))
    with pytest.raises(ValueError):
        oracle.chunkwise(q, k, v, np.array([0.5]), 0)


def test_threads_do_not_change_results():
    q, k, v = _tiny(3, 4, 12, 3, 5, 77)
    gam = np.linspace(0.5, 1.0, 4)
    y1, s1 = oracle.recurrent(q, k, v, gam, nthreads=1)
    y8, s8 = oracle.recurrent(q, k, v, gam, nthreads=8)
    assert np.array_equal(y1, y8) and np.array_equal(s1, s8)


# Plausible mistakes, each a one-token change to the oracle source.  Every one
# must make at least one pin fail.
MUTATIONS = [
    ("recurrent drops the decay", "S[(size_t)i * dv + j] = g * S[(size_t)i * dv + j] + kn[i] * vn[j];",
     "S[(size_t)i * dv + j] = S[(size_t)i * dv + j] + kn[i] * vn[j];"),
    ("recurrent uses q for k", "+ kn[i] * vn[j];", "+ qn[i] * vn[j];"),
    ("recurrent reads the wrong state index", "acc += qn[i] * S[(size_t)i * dv + j];",
     "acc += qn[i] * S[(size_t)i * dv + (dv - 1 - j)];"),
    ("parallel drops the diagonal", "for (int m = 0; m <= n; ++m)", "for (int m = 0; m < n; ++m)"),
    ("parallel inverts the decay exponent", "s *= gpow(g, n - m);", "s *= gpow(g, m);"),
    ("parallel state term off by one", "gpow(g, (long)n + 1)", "gpow(g, (long)n)"),
    ("chunkwise cross term off by one", "gpow(g, (long)i + 1)", "gpow(g, (long)i)"),
    ("chunkwise state decay off by one", "gpow(g, (long)l - 1 - j)", "gpow(g, (long)l - j)"),
    ("chunkwise carries undecayed state", "double acc = gl * S[", "double acc = S["),
    ("chunkwise drops the diagonal", "for (int j = 0; j <= i; ++j)", "for (int j = 0; j < i; ++j)"),
    ("0^0 taken as 0", "if (n == 0) return 1.0;", "if (n == 0) return g;"),
    ("wrong head's gamma", "J->gamma[h]", "J->gamma[(h + 1) % J->H]"),
    ("state_out not written", "if (s_out) memcpy(s_out, S,", "if (0) memcpy(s_out, S,"),
    ("groupnorm unbiased variance", "var /= dv;", "var /= (dv - 1);"),
    ("groupnorm drops eps", "sqrt(var + eps)", "sqrt(var)"),
    ("groupnorm wrong head's weight", "w[(size_t)h * dv + c]", "w[(size_t)((h + 1) % H) * dv + c]"),
    ("groupnorm mean off by one element", "mean /= dv;", "mean /= (dv + 1);"),
    ("backward dq uses q for k", "+= w * dyv * k[ok + (size_t)m * dk + i];", "+= w * dyv * q[ok + (size_t)m * dk + i];"),
    ("backward dk from the wrong row", "dkk[ok + (size_t)m * dk + i] += w * dyv * q[ok + (size_t)n * dk + i];",
     "dkk[ok + (size_t)m * dk + i] += w * dyv * q[ok + (size_t)m * dk + i];"),
    ("backward dv drops the decay", "dvv[ov + (size_t)m * dv + j] += w * qk", "dvv[ov + (size_t)m * dv + j] += qk"),
    ("state backward dq decay off by one", "const double wq = gpow(g, (long)n + 1)", "const double wq = gpow(g, (long)n)"),
    ("state backward dk decay off by one", "ws = gpow(g, (long)L - 1 - n)", "ws = gpow(g, (long)L - n)"),
    ("state backward dk uses dy for v", "+= ws * v[ov + (size_t)n * dv + j] * d;", "+= ws * dy[ov + (size_t)n * dv + j] * d;"),
    ("state backward dq reads S0 untransposed", "* s0[os + (size_t)i * dv + j];", "* s0[os + (size_t)(dk - 1 - i) * dv + j];"),
    ("dS0 drops gamma^L", "gL * dsout[", "dsout["),
    ("dS0 sum decay off by one", "acc += gpow(g, (long)n + 1) * q[", "acc += gpow(g, (long)n) * q["),
    ("gate sigmoid of -x", "1.0 / (1.0 + exp(-x))", "1.0 / (1.0 + exp(x))"),
    ("swish drops the x factor", "act == 1 ? x * s : s", "act == 1 ? s : s"),
    ("gate multiplies the wrong element", "out[i] = a * z[i];", "out[i] = a * z[n - 1 - i];"),
    ("backward misses the diagonal", "                for (int m = 0; m <= n; ++m) {\n                    const double w = gpow(g, n - m);",
     "                for (int m = 0; m < n; ++m) {\n                    const double w = gpow(g, n - m);"),
]


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistakes_are_caught(name, old, new):
    src = open(oracle._SRC).read()
    assert old in src, f"mutation anchor missing: {old}"
    tmp = tempfile.mkdtemp(prefix="oracle_mut_")
    try:
        msrc = os.path.join(tmp, "m.c")
        with open(msrc, "w") as f:
            f.write(src.replace(old, new))
        lib = oracle.load(oracle.build(msrc, os.path.join(tmp, "libm.so")))
        caught = []
        for pin in ALL_PINS:
            try:
                pin(lib)
            except AssertionError:
                caught.append(pin.__name__)
        assert caught, f"no pin catches the planted mistake: {name}"
    finally:
        shutil.rmtree(tmp, ignore_errors=True)


def test_mutation_anchors_are_unique():
    src = open(oracle._SRC).read()
    for name, old, _ in MUTATIONS:
        if name in ("0^0 taken as 0", "state_out not written"):
            continue
        assert len(re.findall(re.escape(old), src)) >= 1
