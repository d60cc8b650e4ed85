"""Pins for the oracle's layer gradients (oracle/backward.py): central finite
differences of the double-precision forward oracle, closed forms and an
invariant of the softmax. CPU only."""

import numpy as np
import pytest

from shifted_window_attention_sw_b200.inputs import make_layer_inputs

CASES = [
    # (shape, heads, window, shift): shifted with padding on two axes, unshifted, partial shift
    ((1, 3, 5, 6, 16), 2, (2, 3, 3), (1, 1, 1)),
    ((2, 2, 6, 6, 16), 2, (2, 3, 3), (0, 0, 0)),
    ((1, 4, 5, 7, 8), 1, (2, 4, 4), (1, 0, 2)),
]
NAMES = ("x", "Wqkv", "bqkv", "Wproj", "bproj", "table")


def _inputs(shape, heads, window, seed):
    return make_layer_inputs(shape, heads, window, "f32", "sensitivity", seed=seed).as_f64()


def _dy(shape, seed):
    return np.random.default_rng(seed).normal(size=shape)


@pytest.fixture(scope="module")
def bwd(oracle_mod):
    from oracle import backward

    return backward


@pytest.mark.parametrize("shape,heads,window,shift", CASES)
def test_g1_recomputed_forward_matches_oracle(oracle_mod, bwd, shape, heads, window, shift):
    # the gradient is taken of the same function the forward oracle computes
    a = _inputs(shape, heads, window, 11)
    ref = oracle_mod.forward(a["x"], window, shift, a["Wqkv"], a["bqkv"], a["Wproj"], a["bproj"], a["table"], heads)
    got = bwd.forward(a["x"], window, shift, a["Wqkv"], a["bqkv"], a["Wproj"], a["bproj"], a["table"], heads)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("shape,heads,window,shift", CASES)
def test_g2_finite_differences(oracle_mod, bwd, shape, heads, window, shift):
    # L = sum(dy * forward); central differences of the C++ forward oracle at sampled
    # coordinates of every argument (truncation error O(h^2) ~ 1e-10 relative)
    a = _inputs(shape, heads, window, 12)
    dy = _dy(shape, 13)
    grads = dict(zip(NAMES, bwd.backward(a["x"], window, shift, a["Wqkv"], a["bqkv"], a["Wproj"], a["bproj"],
                                         a["table"], heads, dy)))

    def loss(args):
        out = oracle_mod.forward(args["x"], window, shift, args["Wqkv"], args["bqkv"], args["Wproj"],
                                 args["bproj"], args["table"], heads, nthreads=1)
        return float((out * dy).sum())

    rng = np.random.default_rng(14)
    for name in NAMES:
        flat = a[name].reshape(-1)
        picks = rng.choice(flat.size, size=min(8, flat.size), replace=False)
        for p in picks:
            h = 1e-5 * max(1.0, abs(flat[p]))
            plus = {k: v.copy() for k, v in a.items()}
            minus = {k: v.copy() for k, v in a.items()}
            plus[name].reshape(-1)[p] += h
            minus[name].reshape(-1)[p] -= h
            fd = (loss(plus) - loss(minus)) / (2 * h)
            an = grads[name].reshape(-1)[p]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (name, p, fd, an)


def test_g3_projection_bias_gradient(oracle_mod, bwd):
    # y = O Wproj + bproj on every real token: dbproj is the sum of dy over the tokens
    # (padding slots are not outputs and add nothing)
    shape, heads, window, shift = (1, 3, 5, 6, 16), 2, (2, 3, 3), (1, 1, 1)
    a = _inputs(shape, heads, window, 15)
    dy = _dy(shape, 16)
    _, _, _, _, dbproj, _ = bwd.backward(a["x"], window, shift, a["Wqkv"], a["bqkv"], a["Wproj"], a["bproj"],
                                         a["table"], heads, dy)
    np.testing.assert_allclose(dbproj, dy.reshape(-1, shape[-1]).sum(axis=0), rtol=0, atol=1e-12)


def test_g3b_key_bias_gradient_is_zero(oracle_mod, bwd):
    # bk adds q_i . bk / sqrt(d) to every score of query row i, the same for all of the
    # row's keys (padded keys included: their k is bk), which the softmax ignores
    shape, heads, window, shift = (1, 3, 5, 6, 16), 2, (2, 3, 3), (1, 1, 1)
    a = _inputs(shape, heads, window, 23)
    dy = _dy(shape, 24)
    C = shape[-1]
    dbqkv = bwd.backward(a["x"], window, shift, a["Wqkv"], a["bqkv"], a["Wproj"], a["bproj"], a["table"],
                         heads, dy)[2]
    np.testing.assert_allclose(dbqkv[C:2 * C], 0.0, atol=1e-12)
    assert np.abs(dbqkv[:C]).max() > 1e-3 and np.abs(dbqkv[2 * C:]).max() > 1e-3


def test_g4_table_gradient_sums_to_zero(oracle_mod, bwd):
    # adding a constant to every table entry of a head adds it to every score of that head,
    # which the softmax ignores: each head's table gradient sums to zero
    shape, heads, window, shift = (1, 3, 5, 6, 16), 2, (2, 3, 3), (1, 1, 1)
    a = _inputs(shape, heads, window, 17)
    dy = _dy(shape, 18)
    dtable = bwd.backward(a["x"], window, shift, a["Wqkv"], a["bqkv"], a["Wproj"], a["bproj"], a["table"],
                          heads, dy)[5]
    assert np.abs(dtable).max() > 1e-3
    np.testing.assert_allclose(dtable.sum(axis=0), 0.0, atol=1e-12)


def test_g5_identity_window_closed_form(oracle_mod, bwd):
    # window (1,1,1): out = (x Wv + bv) Wproj + bproj, so dx = dy Wproj^T Wv^T,
    # dWv = x^T (dy Wproj^T), and q, k and the table get no gradient
    shape, heads = (2, 3, 4, 5, 16), 2
    a = _inputs(shape, heads, (1, 1, 1), 19)
    dy = _dy(shape, 20)
    C = shape[-1]
    dx, dWqkv, dbqkv, dWproj, dbproj, dtable = bwd.backward(a["x"], (1, 1, 1), (0, 0, 0), a["Wqkv"], a["bqkv"],
                                                           a["Wproj"], a["bproj"], a["table"], heads, dy)
    X = a["x"].reshape(-1, C)
    G = dy.reshape(-1, C)
    Wv = a["Wqkv"][:, 2 * C:]
    np.testing.assert_allclose(dx.reshape(-1, C), G @ a["Wproj"].T @ Wv.T, rtol=0, atol=1e-11)
    np.testing.assert_allclose(dWqkv[:, 2 * C:], X.T @ (G @ a["Wproj"].T), rtol=0, atol=1e-10)
    np.testing.assert_allclose(dWqkv[:, :2 * C], 0.0, atol=1e-12)
    np.testing.assert_allclose(dbqkv[:2 * C], 0.0, atol=1e-12)
    V = X @ Wv + a["bqkv"][2 * C:]
    np.testing.assert_allclose(dWproj, V.T @ G, rtol=0, atol=1e-10)
    np.testing.assert_allclose(dtable, 0.0, atol=1e-12)
