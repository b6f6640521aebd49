"""Pins of the oracle's sliding-window causal softmax attention.

The window mixer of the hybrid loops ("LT2: Linear-Time Looped Transformers",
§2: a sliding-window block of window w turns, over T loops, into a receptive
field of size T w; Appendix C: the windowed variants attend to the w - 1
previous tokens and the token itself).  Each pin compares the oracle with a
different construction: full causal attention as masked matrices when the
window covers the sequence, w = 1, equal scores (the window's mean), the
window's edge by perturbation, invariance to a shift of all keys' scores, the
T w receptive field of T stacked windows, and packed sequences.
"""
import numpy as np
import pytest

import oracle


def _softmax_rows(s):
    s = s - s.max(axis=-1, keepdims=True)
    e = np.exp(s)
    return e / e.sum(axis=-1, keepdims=True)


def _rand(rng, L, H, d, dv):
    return (rng.standard_normal((L, H, d)), rng.standard_normal((L, H, d)),
            rng.standard_normal((L, H, dv)))


@pytest.mark.parametrize("seed", [0, 1])
def test_window_covering_the_sequence_is_causal_attention(seed):
    rng = np.random.default_rng(500 + seed)
    L, H, d, dv = 23, 2, 8, 5
    q, k, v = _rand(rng, L, H, d, dv)
    o = oracle.swa_fwd(q, k, v, window=L + 3, scale=0.4)
    for h in range(H):
        s = 0.4 * q[:, h] @ k[:, h].T
        s[np.triu_indices(L, 1)] = -np.inf
        np.testing.assert_allclose(o[:, h], _softmax_rows(s) @ v[:, h], rtol=1e-12, atol=1e-13)


def test_window_of_one_returns_the_value():
    rng = np.random.default_rng(510)
    q, k, v = _rand(rng, 9, 2, 4, 3)
    np.testing.assert_array_equal(oracle.swa_fwd(q, k, v, window=1), v)


def test_equal_scores_average_the_window():
    """Zero keys: every score is 0, so o_t is the mean of v over [t - w + 1, t]."""
    rng = np.random.default_rng(520)
    L, w = 17, 5
    _, _, v = _rand(rng, L, 1, 4, 3)
    q = rng.standard_normal((L, 1, 4))
    o = oracle.swa_fwd(q, np.zeros((L, 1, 4)), v, window=w)
    for t in range(L):
        np.testing.assert_allclose(o[t, 0], v[max(0, t - w + 1):t + 1, 0].mean(axis=0), rtol=1e-13)


def test_window_edge_by_perturbation():
    """Changing key/value t - w (just outside the window) leaves o_t as it is;
    changing t - w + 1 (the oldest key inside) moves it."""
    rng = np.random.default_rng(530)
    L, w, t = 30, 7, 25
    q, k, v = _rand(rng, L, 1, 6, 4)
    base = oracle.swa_fwd(q, k, v, window=w)
    for j, moves in ((t - w, False), (t - w + 1, True)):
        k2, v2 = k.copy(), v.copy()
        k2[j] += 3.0
        v2[j] += 3.0
        o2 = oracle.swa_fwd(q, k2, v2, window=w)
        assert (np.abs(o2[t] - base[t]).max() > 1e-6) == moves, j


def test_shift_of_all_scores_changes_nothing():
    """Adding the same vector c to every key adds q_t . c to all of query t's
    scores, which the softmax removes."""
    rng = np.random.default_rng(540)
    q, k, v = _rand(rng, 20, 2, 5, 3)
    c = 2.0 * rng.standard_normal(5)
    np.testing.assert_allclose(oracle.swa_fwd(q, k + c, v, window=6), oracle.swa_fwd(q, k, v, window=6),
                               rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("T", [1, 2, 3])
def test_stacked_windows_reach_T_windows_back(T):
    """T loops of h <- h + SWA(h) (q = k = v = h, a small score scale so that
    every weight stays well above zero): position t depends on positions back
    to t - T (w - 1) and on none before, the T w receptive field of §2
    (T (w - 1) + 1 positions including t itself)."""
    rng = np.random.default_rng(550 + T)
    L, w, t = 40, 4, 35
    h0 = rng.standard_normal((L, 1, 3))

    def run(h):
        for _ in range(T):
            h = h + oracle.swa_fwd(h, h, h, window=w, scale=0.05)
        return h

    base = run(h0)
    edge = t - T * (w - 1)
    for j, moves in ((edge - 1, False), (edge, True)):
        h2 = h0.copy()
        h2[j] += 1.0
        assert (np.abs(run(h2)[t] - base[t]).max() > 1e-6) == moves, j


def test_packed_sequences_do_not_see_each_other():
    rng = np.random.default_rng(560)
    q, k, v = _rand(rng, 25, 2, 4, 3)
    cu = np.array([0, 10, 10, 25], dtype=np.int32)
    o = oracle.swa_fwd(q, k, v, window=6, cu_seqlens=cu)
    np.testing.assert_array_equal(o[:10], oracle.swa_fwd(q[:10], k[:10], v[:10], window=6))
    np.testing.assert_array_equal(o[10:], oracle.swa_fwd(q[10:], k[10:], v[10:], window=6))
