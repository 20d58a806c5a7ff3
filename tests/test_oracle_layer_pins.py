"""Pins for the oracle of the layer steps around the recurrence
(``oracle.preprocess``, ``oracle.output_gate``): closed forms, special cases
and invariants fixed by the definitions (explainer page, "Step 2: Process
tokens with Hybrid Blocks": a 1-D convolution of window 4 and an output gate
per Gated DeltaNet layer), not by the oracle's own code.  A broken variant of
each definition is planted here, on the CPU, to show that a pin catches it.
"""
import math

import numpy as np
import pytest

import oracle

RNG = np.random.default_rng(2024)


def _case(lens, H=2, d=8, rng=RNG, state=True):
    T = int(sum(lens))
    xq, xk, xv = (rng.standard_normal((T, H, d)) for _ in range(3))
    w = rng.standard_normal((3, H, d, 4))
    a, b = rng.standard_normal((T, H)) * 3, rng.standard_normal((T, H)) * 3
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    st = rng.standard_normal((len(lens), 3, 3, H, d)) if state else None
    return xq, xk, xv, w, a, b, cu, st


def _taps(H, d, tap):
    w = np.zeros((3, H, d, 4))
    w[..., tap] = 1.0
    return w


def test_identity_tap_passes_inputs_through():
    xq, xk, xv, _, a, b, cu, st = _case([7, 5])
    q, k, v, g, beta, _ = oracle.preprocess(xq, xk, xv, _taps(2, 8, 3), a, b, cu, st, eps=0.0)
    np.testing.assert_array_equal(v, xv)
    np.testing.assert_allclose(q, xq / np.linalg.norm(xq, axis=-1, keepdims=True), rtol=1e-14, atol=0)
    np.testing.assert_allclose(k, xk / np.linalg.norm(xk, axis=-1, keepdims=True), rtol=1e-14, atol=0)


def test_oldest_tap_is_a_three_token_delay_restarting_per_sequence():
    lens = [6, 2, 9]
    xq, xk, xv, _, a, b, cu, st = _case(lens)
    _, _, v, _, _, _ = oracle.preprocess(xq, xk, xv, _taps(2, 8, 0), a, b, cu, st)
    for n, L in enumerate(lens):
        bos = int(cu[n])
        for i in range(L):
            ref = xv[bos + i - 3] if i >= 3 else st[n, i, 2]
            np.testing.assert_array_equal(v[bos + i], ref)
    _, _, v0, _, _, _ = oracle.preprocess(xq, xk, xv, _taps(2, 8, 0), a, b, cu, None)
    assert np.all(v0[int(cu[1]):int(cu[1]) + 2] == 0.0)   # a 2-token sequence sees only the zero state


def test_impulse_response_is_the_taps_in_time_order():
    """A single nonzero input at position p gives y[p + 3 - i] = w[i] (tap 3
    is the current token): pins the tap order and the causality."""
    H, d, T, p = 1, 4, 12, 5
    w = RNG.standard_normal((3, H, d, 4))
    x = np.zeros((T, H, d))
    x[p] = 1.0
    a = b = np.zeros((T, H))
    _, _, v, _, _, _ = oracle.preprocess(x, x, x, w, a, b)
    for t in range(T):
        # x[p] is multiplied by tap 3 - (t - p) at output t
        ref = w[2, :, :, 3 - (t - p)] if 0 <= t - p <= 3 else np.zeros((H, d))
        np.testing.assert_array_equal(v[t], ref, err_msg="t=%d" % t)


def test_carried_conv_state_makes_splitting_exact():
    for cut in (1, 2, 3, 7):
        xq, xk, xv, w, a, b, _, st = _case([11], state=True)
        whole = oracle.preprocess(xq, xk, xv, w, a, b, None, st, activation=oracle.ACT_SILU)
        first = oracle.preprocess(xq[:cut], xk[:cut], xv[:cut], w, a[:cut], b[:cut], None, st,
                                  activation=oracle.ACT_SILU)
        second = oracle.preprocess(xq[cut:], xk[cut:], xv[cut:], w, a[cut:], b[cut:], None, first[5],
                                   activation=oracle.ACT_SILU)
        for i in range(5):
            np.testing.assert_allclose(np.concatenate([first[i], second[i]]), whole[i], rtol=1e-13, atol=1e-15)
        np.testing.assert_array_equal(second[5], whole[5])


def test_state_out_of_short_sequences_shifts_the_old_state():
    xq, xk, xv, w, a, b, cu, st = _case([1, 0, 2])
    _, _, _, _, _, so = oracle.preprocess(xq, xk, xv, w, a, b, cu, st)
    x = np.stack([xq, xk, xv], axis=0)
    np.testing.assert_array_equal(so[0, :2], st[0, 1:])
    np.testing.assert_array_equal(so[0, 2], x[:, 0])
    np.testing.assert_array_equal(so[1], st[1])          # empty sequence: state passes through
    np.testing.assert_array_equal(so[2, 0], st[2, 2])
    np.testing.assert_array_equal(so[2, 1:], np.moveaxis(x[:, 1:3], 1, 0))


def test_l2_norm_gives_unit_rows_parallel_to_the_conv_output():
    xq, xk, xv, w, a, b, cu, st = _case([9])
    q, k, v, _, _, _ = oracle.preprocess(xq, xk, xv, w, a, b, cu, st, eps=0.0)
    np.testing.assert_allclose(np.linalg.norm(q, axis=-1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(np.linalg.norm(k, axis=-1), 1.0, rtol=1e-14)
    # direction: q is a positive multiple of the unnormalised conv output (the
    # same conv with identity normalisation is v's path, so use tensor 2 weights)
    w2 = w.copy()
    w2[2] = w[0]
    st2 = st.copy()
    st2[:, :, 2] = st[:, :, 0]
    _, _, vq, _, _, _ = oracle.preprocess(xq, xk, xq, w2, a, b, cu, st2)
    cos = np.sum(q * vq, axis=-1) / np.linalg.norm(vq, axis=-1)
    np.testing.assert_allclose(cos, 1.0, rtol=1e-13)


def test_gates_closed_forms():
    assert oracle.sigmoid(np.array([0.0]))[0] == 0.5
    assert oracle.log_sigmoid(np.array([0.0]))[0] == pytest.approx(-math.log(2.0), rel=1e-15)
    a = np.linspace(-30, 30, 61)
    np.testing.assert_allclose(np.exp(oracle.log_sigmoid(a)), oracle.sigmoid(a), rtol=1e-14)
    np.testing.assert_allclose(oracle.sigmoid(a) + oracle.sigmoid(-a), 1.0, rtol=1e-15)
    big = oracle.log_sigmoid(np.array([-800.0, 800.0]))
    assert big[0] == -800.0 and big[1] == 0.0            # no overflow, exact limits
    T, H, d = 4, 1, 2
    z = np.zeros((T, H, d))
    _, _, _, g, beta, _ = oracle.preprocess(z, z, z, np.zeros((3, H, d, 4)), np.full((T, H), 3.0),
                                            np.full((T, H), -1.0))
    np.testing.assert_allclose(g, math.log(1.0 / (1.0 + math.exp(-3.0))), rtol=1e-14)
    np.testing.assert_allclose(beta, 1.0 / (1.0 + math.e), rtol=1e-14)


def test_silu_values():
    T, H, d = 3, 1, 4
    x = np.array([0.0, 1.0, -1.0, 40.0]).reshape(1, 1, 4).repeat(T, 0)
    _, _, v, _, _, _ = oracle.preprocess(x, x, x, _taps(H, d, 3), np.zeros((T, H)), np.zeros((T, H)),
                                         activation=oracle.ACT_SILU)
    ref = np.array([0.0, 1.0 / (1.0 + math.exp(-1.0)), -1.0 / (1.0 + math.e), 40.0 / (1.0 + math.exp(-40.0))])
    np.testing.assert_allclose(v[1, 0], ref, rtol=1e-15)


def test_output_gate_closed_forms():
    o = RNG.standard_normal((5, 2, 8))
    np.testing.assert_array_equal(oracle.output_gate(o, np.full_like(o, 800.0)), o)      # sigmoid -> 1
    np.testing.assert_array_equal(oracle.output_gate(o, np.zeros_like(o)), o / 2)
    np.testing.assert_allclose(oracle.output_gate(o, np.ones_like(o), gate=oracle.GATE_SILU),
                               o / (1.0 + math.exp(-1.0)), rtol=1e-15)
    c = np.full((1, 1, 8), -3.0)                         # constant row: RMS norm gives its sign
    np.testing.assert_allclose(oracle.output_gate(c, np.full_like(c, 800.0), np.ones(8), eps=0.0), -1.0,
                               rtol=1e-15)
    w = RNG.uniform(0.5, 2.0, 8)
    y1 = oracle.output_gate(o, o, w, eps=0.0)
    y2 = oracle.output_gate(7.5 * o, o, w, eps=0.0)       # the norm removes the scale of o
    np.testing.assert_allclose(y1, y2, rtol=1e-13)
    rms = np.sqrt(np.mean((oracle.output_gate(o, np.full_like(o, 800.0), np.ones(8), eps=0.0)) ** 2, axis=-1))
    np.testing.assert_allclose(rms, 1.0, rtol=1e-14)


# ---------------------------------------------------------------- planted mistakes

def _reversed_taps(xq, xk, xv, w, *args, **kw):
    return oracle.preprocess(xq, xk, xv, w[..., ::-1], *args, **kw)


def _no_restart(xq, xk, xv, w, a, b, cu=None, st=None, **kw):
    return oracle.preprocess(xq, xk, xv, w, a, b, None, None if st is None else st[:1], **kw)


def test_mistakes_are_caught():
    with pytest.raises(AssertionError):
        H, d, T, p = 1, 4, 12, 5
        w = RNG.standard_normal((3, H, d, 4))
        x = np.zeros((T, H, d))
        x[p] = 1.0
        _, _, v, _, _, _ = _reversed_taps(x, x, x, w, np.zeros((T, H)), np.zeros((T, H)))
        np.testing.assert_array_equal(v[p], w[2, :, :, 3])
    with pytest.raises(AssertionError):
        lens = [6, 2, 9]
        xq, xk, xv, _, a, b, cu, st = _case(lens)
        _, _, v, _, _, _ = _no_restart(xq, xk, xv, _taps(2, 8, 0), a, b, cu, st)
        np.testing.assert_array_equal(v[int(cu[1])], st[1, 0, 2])
