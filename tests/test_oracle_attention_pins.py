"""Pins for the oracle of sliding-window attention with RoPE and grouped KV
heads (``oracle.swa_attention``, ``oracle.rope``): closed forms and
invariants fixed by the definitions (explainer page: attention inside a
recent local window, RoPE positions, 16 query / 2 key-value heads), not by
the oracle's own code.  Planted mistakes are caught."""
import math

import numpy as np
import pytest

import oracle

RNG = np.random.default_rng(77)


def _qkv(T, Hq, Hkv, d, rng=RNG):
    return (rng.standard_normal((T, Hq, d)), rng.standard_normal((T, Hkv, d)), rng.standard_normal((T, Hkv, d)))


def test_window_of_one_returns_the_own_value():
    q, k, v = _qkv(9, 4, 2, 8)
    o = oracle.swa_attention(q, k, v, window=1)
    np.testing.assert_allclose(o, np.repeat(v, 2, axis=1), rtol=0, atol=1e-15)


def test_zero_scale_averages_the_window_and_restarts_per_sequence():
    """Uniform weights: o_t = mean of v over s in (t - W, t] of t's sequence."""
    q, k, v = _qkv(20, 2, 1, 4)
    cu = np.array([0, 7, 7, 20])
    for W in (1, 3, 5, 100):
        o = oracle.swa_attention(q, k, v, cu, window=W, scale=0.0)
        for t in range(20):
            bos = 0 if t < 7 else 7
            ref = v[max(bos, t - W + 1):t + 1, 0].mean(axis=0)
            np.testing.assert_allclose(o[t, 0], ref, rtol=1e-13, atol=1e-15)


def test_sharp_query_picks_its_key_through_the_right_kv_head():
    """Orthonormal keys and a query along key j scaled up: the softmax
    concentrates on j, and query head h must read kv head h // (Hq/Hkv)."""
    T, Hq, Hkv, d = 6, 4, 2, 8
    basis = np.eye(d)
    k = np.zeros((T, Hkv, d))
    for t in range(T):
        k[t, 0] = basis[t]
        k[t, 1] = basis[(t + 3) % d]
    v = RNG.standard_normal((T, Hkv, d))
    q = np.zeros((T, Hq, d))
    t, j = 5, 2
    for h in range(Hq):
        q[t, h] = 200.0 * k[j, h // 2]
    o = oracle.swa_attention(q, k, v, window=T, scale=1.0)
    for h in range(Hq):
        np.testing.assert_allclose(o[t, h], v[j, h // 2], rtol=0, atol=1e-12)


def test_full_window_is_causal_softmax():
    """With the window covering the sequence, a future key never matters."""
    q, k, v = _qkv(12, 2, 2, 4)
    o1 = oracle.swa_attention(q, k, v, window=100)
    k2, v2 = k.copy(), v.copy()
    k2[8:] = RNG.standard_normal(k2[8:].shape)
    v2[8:] = RNG.standard_normal(v2[8:].shape)
    o2 = oracle.swa_attention(q, k2, v2, window=100)
    np.testing.assert_array_equal(o1[:8], o2[:8])
    assert np.max(np.abs(o1[8:] - o2[8:])) > 1e-3


def test_rope_closed_forms():
    x = RNG.standard_normal((5, 3, 16))
    np.testing.assert_array_equal(oracle.rope(x, np.zeros(5, dtype=np.int64)), x)      # position 0
    pos = np.arange(5) * 37
    y = oracle.rope(x, pos)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-14)
    # d = 2: theta_0 = 1, a plain rotation by the position
    x2 = np.array([[[1.0, 0.0]]])
    for p in (0, 1, 3):
        np.testing.assert_allclose(oracle.rope(x2, np.array([p]))[0, 0], [math.cos(p), math.sin(p)], atol=1e-15)


def test_rope_scores_depend_on_relative_position_only():
    q = RNG.standard_normal((1, 1, 32))
    k = RNG.standard_normal((1, 1, 32))
    for m, n, shift in ((5, 2, 11), (0, 9, 100), (40, 40, 3)):
        a = np.sum(oracle.rope(q, np.array([m])) * oracle.rope(k, np.array([n])))
        b = np.sum(oracle.rope(q, np.array([m + shift])) * oracle.rope(k, np.array([n + shift])))
        assert a == pytest.approx(b, rel=1e-11, abs=1e-12)


def test_positions_restart_per_sequence():
    np.testing.assert_array_equal(oracle.rope_positions(np.array([0, 3, 3, 5]), 5, offset=10),
                                  [10, 11, 12, 10, 11])


def _wrong_head_map(q, k, v, **kw):
    # query head h reading kv head h % Hkv instead of h // (Hq / Hkv)
    Hq, Hkv = q.shape[1], k.shape[1]
    idx = [h % Hkv for h in range(Hq)]
    return np.stack([oracle.swa_attention(q[:, h:h + 1], k[:, idx[h]:idx[h] + 1], v[:, idx[h]:idx[h] + 1], **kw)[:, 0]
                     for h in range(Hq)], axis=1)


def test_mistakes_are_caught():
    T, Hq, Hkv, d = 6, 4, 2, 8
    basis = np.eye(d)
    k = np.zeros((T, Hkv, d))
    for t in range(T):
        k[t, 0] = basis[t]
        k[t, 1] = basis[(t + 3) % d]
    v = RNG.standard_normal((T, Hkv, d))
    q = np.zeros((T, Hq, d))
    for h in range(Hq):
        q[5, h] = 200.0 * k[2, h // 2]
    o = _wrong_head_map(q, k, v, window=T, scale=1.0)
    with pytest.raises(AssertionError):
        for h in range(Hq):
            np.testing.assert_allclose(o[5, h], v[2, h // 2], rtol=0, atol=1e-12)
