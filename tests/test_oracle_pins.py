"""Pins for the fp64 oracle: facts fixed by the mathematics of the gated delta
rule, not by the oracle's own code.

Each ``pin_*`` takes a prefill callable ``fn(q, k, v, g, beta, state_in=None,
cu_seqlens=None) -> (out [T,H,dv], state [N,H,dv,dk])`` so that the same pins
can be run against deliberately broken variants (see ``test_mutants_caught``):
every plausible mistake -- a dropped decay, read-out before the write, the
erase on the wrong side, a transposed state, a lost beta -- must fail at least
one pin.

The recurrence (InfiniteVL explainer page, "Gated DeltaNet" concept box;
standard gated delta rule):  u = beta (v - alpha S k);  S <- alpha S + u k^T;
o = S q.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(12345)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _rand_case(T, H, dk, dv, rng, alpha=None, beta=None, state=True):
    q = _unit(rng.standard_normal((T, H, dk)))
    k = _unit(rng.standard_normal((T, H, dk)))
    v = rng.standard_normal((T, H, dv))
    g = np.log(rng.uniform(0.7, 1.0, (T, H))) if alpha is None else np.full((T, H), math.log(alpha) if alpha > 0 else -np.inf)
    b = rng.uniform(0.0, 1.0, (T, H)) if beta is None else np.full((T, H), float(beta))
    s0 = rng.standard_normal((1, H, dv, dk)) if state else None
    return q, k, v, g, b, s0


# ---------------------------------------------------------------- pins

def pin_worked_example(fn):
    """Hand-derived three-token example (tests/golden/worked_example_d2.txt)."""
    rec = {}
    with open(os.path.join(GOLDEN, "worked_example_d2.txt")) as f:
        for line in f:
            if line.startswith("#") or ":" not in line:
                continue
            name, vals = line.split(":", 1)
            rec[name.strip()] = np.array([float(x) for x in vals.split()])
    T = 3
    q = rec["q"].reshape(T, 1, 2)
    k = rec["k"].reshape(T, 1, 2)
    v = rec["v"].reshape(T, 1, 2)
    g = np.log(rec["alpha"]).reshape(T, 1)
    b = rec["beta"].reshape(T, 1)
    out, st = fn(q, k, v, g, b)
    np.testing.assert_allclose(out.reshape(-1), rec["out"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(st.reshape(-1), rec["state"], rtol=0, atol=1e-12)


def pin_no_write_no_decay(fn):
    """beta = 0, alpha = 1: the state never changes and o_t = S0 q_t."""
    q, k, v, g, b, s0 = _rand_case(9, 2, 5, 3, np.random.default_rng(1), alpha=1.0, beta=0.0)
    out, st = fn(q, k, v, g, b, s0)
    np.testing.assert_allclose(st, s0, rtol=0, atol=1e-12)
    ref = np.einsum("hij,thj->thi", s0[0], q)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def pin_pure_decay(fn):
    """beta = 0, any alpha: S_t = (prod_{s<=t} alpha_s) S0 (closed form)."""
    rng = np.random.default_rng(2)
    q, k, v, g, b, s0 = _rand_case(7, 2, 4, 6, rng, beta=0.0)
    out, st = fn(q, k, v, g, b, s0)
    cum = np.exp(np.cumsum(g, axis=0))                       # [T, H]
    np.testing.assert_allclose(st[0], cum[-1][:, None, None] * s0[0], rtol=1e-12, atol=1e-14)
    ref = cum[:, :, None] * np.einsum("hij,thj->thi", s0[0], q)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-14)


def pin_exact_write(fn):
    """beta = 1, |k| = 1: the write is exact, S_t k_t = v_t, whatever alpha and
    the previous state.  Checked after every token by reading out with q = k."""
    rng = np.random.default_rng(3)
    q, k, v, g, b, s0 = _rand_case(11, 2, 6, 4, rng, beta=1.0)
    q = k.copy()                                            # read along the key just written
    out, _ = fn(q, k, v, g, b, s0)
    np.testing.assert_allclose(out, v, rtol=0, atol=1e-12)


def pin_one_token_zero_state(fn):
    """Zero state, one token: o = beta (k . q) v."""
    rng = np.random.default_rng(4)
    q, k, v, g, b, _ = _rand_case(1, 3, 5, 7, rng)
    out, st = fn(q, k, v, g, b)
    ref = b[0][:, None] * np.sum(k[0] * q[0], axis=-1)[:, None] * v[0]
    np.testing.assert_allclose(out[0], ref, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(st[0], b[0][:, None, None] * v[0][:, :, None] * k[0][:, None, :], rtol=1e-13, atol=1e-15)


def pin_reset(fn):
    """alpha = 0 (g = -inf): the old state is forgotten, S_t = beta v k^T."""
    rng = np.random.default_rng(5)
    q, k, v, g, b, s0 = _rand_case(4, 2, 5, 3, rng)
    g[-1] = -np.inf
    out, st = fn(q, k, v, g, b, s0)
    ref = b[-1][:, None, None] * v[-1][:, :, None] * k[-1][:, None, :]
    np.testing.assert_allclose(st[0], ref, rtol=1e-13, atol=1e-15)


def pin_orthonormal_memory(fn):
    """alpha = 1, beta = 1, orthonormal keys, zero state: the textbook
    associative memory S = sum_i v_i k_i^T, so S k_j = v_j for every j."""
    rng = np.random.default_rng(6)
    dk, dv, T = 6, 4, 5
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Qm[:, :T].T.reshape(T, 1, dk)
    v = rng.standard_normal((T, 1, dv))
    q = np.zeros((T, 1, dk))
    out, st = fn(q, k, v, np.zeros((T, 1)), np.ones((T, 1)))
    np.testing.assert_allclose(st[0, 0], np.einsum("ti,tj->ij", v[:, 0], k[:, 0]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(st[0, 0] @ k[:, 0].T, v[:, 0].T, rtol=0, atol=1e-12)


def pin_gradient_step(fn):
    """The delta rule is one gradient step of size beta on the online
    regression loss L(X) = 1/2 |X k - v|^2 taken from X = alpha S (torch
    autograd, fp64)."""
    rng = np.random.default_rng(7)
    q, k, v, g, b, s0 = _rand_case(1, 1, 5, 3, rng)
    _, st = fn(q, k, v, g, b, s0)
    X = torch.tensor(math.exp(g[0, 0]) * s0[0, 0], dtype=torch.float64, requires_grad=True)
    kt = torch.tensor(k[0, 0]); vt = torch.tensor(v[0, 0])
    loss = 0.5 * torch.sum((X @ kt - vt) ** 2)
    loss.backward()
    ref = (X - b[0, 0] * X.grad).detach().numpy()
    np.testing.assert_allclose(st[0, 0], ref, rtol=1e-13, atol=1e-14)


def pin_contraction(fn):
    """|k| = 1, beta in [0,1], alpha <= 1: |S_t|_2 <= alpha |S_{t-1}|_2 + beta |v_t|
    (the erase I - beta k k^T has spectral norm 1)."""
    rng = np.random.default_rng(8)
    q, k, v, g, b, s0 = _rand_case(30, 1, 6, 5, rng)
    S = s0
    for t in range(30):
        _, S2 = fn(q[t:t + 1], k[t:t + 1], v[t:t + 1], g[t:t + 1], b[t:t + 1], S)
        lhs = np.linalg.norm(S2[0, 0], 2)
        rhs = math.exp(g[t, 0]) * np.linalg.norm(S[0, 0], 2) + b[t, 0] * np.linalg.norm(v[t, 0])
        assert lhs <= rhs * (1 + 1e-12)
        S = S2


def pin_split(fn):
    """Running a sequence in two pieces with the state carried gives the same
    outputs and final state as one run."""
    rng = np.random.default_rng(9)
    q, k, v, g, b, s0 = _rand_case(23, 2, 5, 4, rng)
    out, st = fn(q, k, v, g, b, s0)
    o1, s1 = fn(q[:10], k[:10], v[:10], g[:10], b[:10], s0)
    o2, s2 = fn(q[10:], k[10:], v[10:], g[10:], b[10:], s1)
    np.testing.assert_allclose(np.concatenate([o1, o2]), out, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(s2, st, rtol=1e-12, atol=1e-13)


def pin_packing(fn):
    """Sequences packed with cu_seqlens are independent: the same as separate
    runs, each from its own initial state (empty sequences allowed)."""
    rng = np.random.default_rng(10)
    lens = [5, 0, 1, 9]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T = cu[-1]
    q, k, v, g, b, _ = _rand_case(T, 2, 4, 3, rng)
    s0 = rng.standard_normal((len(lens), 2, 3, 4))
    out, st = fn(q, k, v, g, b, s0, cu)
    for n in range(len(lens)):
        a, e = cu[n], cu[n + 1]
        o_n, s_n = fn(q[a:e], k[a:e], v[a:e], g[a:e], b[a:e], s0[n:n + 1])
        np.testing.assert_allclose(out[a:e], o_n, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(st[n], s_n[0], rtol=1e-13, atol=1e-14)


def chunked_form(q, k, v, g, beta, s0, C):
    """Independent derivation (numpy, fp64): the WY/UT chunkwise form.

    Unrolling the recurrence inside a chunk with start state S0 and
    G = cumsum(g), gamma = exp(G), Gam_ri = exp(G_r - G_i):
      (I + A) U = diag(beta) V - diag(beta gamma) K S0^T,
      A = strict_lower(diag(beta) (K K^T o Gam)),
      O = diag(gamma) Q S0^T + tril(Q K^T o Gam) U,
      S_C = gamma_C S0 + U^T diag(exp(G_C - G)) K.
    """
    T, H, dk = q.shape
    dv = v.shape[2]
    out = np.zeros((T, H, dv))
    S = np.zeros((H, dv, dk)) if s0 is None else s0[0].copy()
    for h in range(H):
        Sh = S[h]
        for s in range(0, T, C):
            e = min(T, s + C)
            K, Q, V = k[s:e, h], q[s:e, h], v[s:e, h]
            bb = beta[s:e, h]
            G = np.cumsum(g[s:e, h])
            Gam = np.tril(np.exp(G[:, None] - G[None, :]))
            A = np.tril(bb[:, None] * (K @ K.T) * Gam, -1)
            rhs = bb[:, None] * V - (bb * np.exp(G))[:, None] * (K @ Sh.T)
            U = np.linalg.solve(np.eye(e - s) + A, rhs)
            out[s:e, h] = np.exp(G)[:, None] * (Q @ Sh.T) + ((Q @ K.T) * Gam) @ U
            Sh = np.exp(G[-1]) * Sh + (np.exp(G[-1] - G)[:, None] * U).T @ K
        S[h] = Sh
    return out, S[None]


def pin_chunked_form(fn):
    """Sequential and chunkwise forms agree for every chunk size 1..T."""
    rng = np.random.default_rng(11)
    q, k, v, g, b, s0 = _rand_case(13, 2, 5, 4, rng)
    out, st = fn(q, k, v, g, b, s0)
    for C in range(1, 14):
        oc, sc = chunked_form(q, k, v, g, b, s0, C)
        np.testing.assert_allclose(oc, out, rtol=1e-10, atol=1e-11)
        np.testing.assert_allclose(sc, st, rtol=1e-10, atol=1e-11)


PINS = [pin_worked_example, pin_no_write_no_decay, pin_pure_decay,
        pin_exact_write, pin_one_token_zero_state, pin_reset,
        pin_orthonormal_memory, pin_gradient_step, pin_contraction, pin_split,
        pin_packing, pin_chunked_form]


def _oracle_fn(q, k, v, g, beta, state_in=None, cu_seqlens=None):
    return oracle.prefill(q, k, v, g, beta, state_in, cu_seqlens, nthreads=2)


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(_oracle_fn)


def test_decode_matches_one_token_prefill():
    rng = np.random.default_rng(13)
    B, H, dk, dv = 3, 2, 5, 4
    q = _unit(rng.standard_normal((B, H, dk)))
    k = _unit(rng.standard_normal((B, H, dk)))
    v = rng.standard_normal((B, H, dv))
    g = np.log(rng.uniform(0.5, 1, (B, H)))
    b = rng.uniform(0, 1, (B, H))
    s = rng.standard_normal((B, H, dv, dk))
    o, s2 = oracle.decode_step(q, k, v, g, b, s)
    cu = np.arange(B + 1)
    o_p, s_p = oracle.prefill(q, k, v, g, b, s, cu)
    np.testing.assert_array_equal(o, o_p)
    np.testing.assert_array_equal(s2, s_p)


# ------------------------------------------------ planted mistakes (CPU only)

def _mutant(kind):
    """A small pure-Python prefill with one plausible mistake planted."""
    def fn(q, k, v, g, beta, state_in=None, cu_seqlens=None):
        T, H, dk = q.shape
        dv = v.shape[2]
        cu = [0, T] if cu_seqlens is None else list(cu_seqlens)
        N = len(cu) - 1
        out = np.zeros((T, H, dv))
        st = np.zeros((N, H, dv, dk))
        for n in range(N):
            for h in range(H):
                S = np.zeros((dv, dk)) if state_in is None else np.array(state_in[n, h], dtype=float)
                for t in range(cu[n], cu[n + 1]):
                    a = math.exp(g[t, h]); bt = beta[t, h]
                    kt, vt, qt = k[t, h], v[t, h], q[t, h]
                    o_early = S @ qt
                    if kind == "residual_without_decay":
                        u = bt * (vt - S @ kt)
                    elif kind == "no_beta_on_residual":
                        u = vt - a * (S @ kt)
                    else:
                        u = bt * (vt - a * (S @ kt))
                    if kind == "decay_after_write":
                        S = a * (S + np.outer(u, kt))
                    elif kind == "erase_on_wrong_side":
                        # (I - beta k k^T) applied from the left: only
                        # type-checks when dk == dv
                        S = a * (np.eye(dk) - bt * np.outer(kt, kt)) @ S + bt * np.outer(vt, kt)
                    else:
                        S = a * S + np.outer(u, kt)
                    if kind == "readout_before_write":
                        o = o_early
                    elif kind == "transposed_readout":
                        o = S.T @ qt          # only type-checks when dk == dv
                    else:
                        o = S @ qt
                    out[t, h] = o
                st[n, h] = S
        return out, st
    return fn


MUTANTS = ["readout_before_write", "residual_without_decay", "no_beta_on_residual",
           "decay_after_write", "erase_on_wrong_side", "transposed_readout"]


def test_clean_python_variant_passes_pins():
    """The unmutated pure-Python loop passes every pin (guards the harness)."""
    for pin in PINS:
        pin(_mutant("none"))


@pytest.mark.parametrize("kind", MUTANTS)
def test_mutants_caught(kind):
    fn = _mutant(kind)
    failed = []
    for pin in PINS:
        try:
            pin(fn)
        except (AssertionError, ValueError):   # wrong value, or wrong shape
            failed.append(pin.__name__)
    assert failed, "planted mistake %r passed every pin" % kind


def test_square_pins_catch_wrong_side_erase():
    """With d_k = d_v the erase on the wrong side type-checks; the exact-write
    pin still rejects it."""
    rng = np.random.default_rng(14)
    q, k, v, g, b, s0 = _rand_case(6, 1, 4, 4, rng, beta=1.0)
    good = _mutant("none")(k, k, v, g, b, s0)[0]
    bad = _mutant("erase_on_wrong_side")(k, k, v, g, b, s0)[0]
    np.testing.assert_allclose(good, v, atol=1e-12)
    assert np.max(np.abs(bad - v)) > 1e-3


def test_oracle_threads_do_not_change_results():
    rng = np.random.default_rng(15)
    q, k, v, g, b, s0 = _rand_case(40, 4, 8, 8, rng)
    s0 = np.repeat(s0, 1, axis=0)
    o1, s1 = oracle.prefill(q, k, v, g, b, s0, nthreads=1)
    o4, s4 = oracle.prefill(q, k, v, g, b, s0, nthreads=4)
    np.testing.assert_array_equal(o1, o4)
    np.testing.assert_array_equal(s1, s4)
