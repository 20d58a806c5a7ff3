"""fp64 CPU oracle of the steps around the Gated DeltaNet recurrence inside
one layer -- TEST INFRASTRUCTURE ONLY (same rules as the rest of ``oracle``).

The explainer page (InfiniteVL, "Step 2: Process tokens with Hybrid Blocks")
states that every Gated DeltaNet layer has 16 heads, a 1-D convolution of
window 4 and an output gate.  It fixes nothing else, so the plainest readings
are taken:

* pre-processing (``preprocess``): a causal depthwise convolution of window 4
  over each of the q, k and v channels, restarted at every sequence start
  (tokens before the start are the carried convolution state, else zero),
  followed by an optional activation (none or SiLU); q and k are then
  L2-normalised per (token, head) as x / sqrt(sum x^2 + eps); the gates are
  beta = sigmoid(b) and g = log(alpha) with alpha = sigmoid(a), i.e.
  g = -softplus(-a) (the tiny workload's alpha = sigmoid(.) parametrisation).
* output gate (``output_gate``): y = n(o) * act(z) per (token, head), where
  n is the identity or an RMS norm over d_v with a per-channel weight
  (o / sqrt(mean o^2 + eps) * w), and act is sigmoid or SiLU.

Everything is plain numpy in float64, one sequence and one tap at a time.
"""
from __future__ import annotations

from typing import Optional, Tuple

import numpy as np

ACT_NONE, ACT_SILU = 0, 1
GATE_SIGMOID, GATE_SILU = 0, 1


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def sigmoid(x):
    x = _f64(x)
    out = np.empty_like(x)
    pos = x >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-x[pos]))
    e = np.exp(x[~pos])
    out[~pos] = e / (1.0 + e)
    return out


def log_sigmoid(x):
    """log(sigmoid(x)) = -softplus(-x), evaluated without overflow."""
    x = _f64(x)
    return np.minimum(x, 0.0) - np.log1p(np.exp(-np.abs(x)))


def _act(y, activation: int):
    if activation == ACT_NONE:
        return y
    if activation == ACT_SILU:
        return y * sigmoid(y)
    raise ValueError("unknown activation %r" % activation)


def preprocess(xq, xk, xv, conv_w, a, b, cu_seqlens=None, conv_state=None,
               activation: int = ACT_NONE, eps: float = 1e-6
               ) -> Tuple[np.ndarray, np.ndarray, np.ndarray, np.ndarray, np.ndarray, np.ndarray]:
    """xq, xk: [T, H, dk]; xv: [T, H, dv] (dk == dv = d); conv_w: [3, H, d, 4]
    (tensor q/k/v, head, channel, tap; tap 3 multiplies the current token,
    tap i the token 3 - i positions back); a, b: [T, H] logits;
    cu_seqlens: [N+1] or None (one sequence); conv_state: [N, 3, 3, H, d]
    or None (zeros): slot j holds the raw input at position (start - 3 + j).

    Returns (q, k, v, g, beta, conv_state_out) with conv_state_out holding
    the raw inputs at positions (end - 3 + j) of every sequence.
    """
    x = np.stack([_f64(xq), _f64(xk), _f64(xv)])          # [3, T, H, d]
    w = _f64(conv_w)
    _, T, H, d = x.shape
    if w.shape != (3, H, d, 4):
        raise ValueError("conv_w must be [3, H, d, 4]")
    cu = np.array([0, T], dtype=np.int64) if cu_seqlens is None else np.asarray(cu_seqlens, dtype=np.int64)
    N = cu.shape[0] - 1
    st = np.zeros((N, 3, 3, H, d)) if conv_state is None else _f64(conv_state)
    if st.shape != (N, 3, 3, H, d):
        raise ValueError("conv_state must be [N, 3, 3, H, d]")
    y = np.zeros_like(x)
    st_out = np.zeros((N, 3, 3, H, d))
    for n in range(N):
        bos, eos = int(cu[n]), int(cu[n + 1])

        def raw(p):   # [3, H, d] raw inputs at absolute position p (p >= bos - 3)
            return x[:, p] if p >= bos else st[n, p - bos + 3]

        for t in range(bos, eos):
            acc = np.zeros((3, H, d))
            for i in range(4):
                acc += w[..., i] * raw(t - 3 + i)
            y[:, t] = acc
        for j in range(3):
            st_out[n, j] = raw(eos - 3 + j)
    y = _act(y, activation)
    q, k, v = y[0], y[1], y[2]
    q = q / np.sqrt(np.sum(q * q, axis=-1, keepdims=True) + eps)
    k = k / np.sqrt(np.sum(k * k, axis=-1, keepdims=True) + eps)
    a = _f64(a)
    b = _f64(b)
    return q, k, v, log_sigmoid(a), sigmoid(b), st_out


def output_gate(o, z, norm_w=None, gate: int = GATE_SIGMOID, eps: float = 1e-6) -> np.ndarray:
    """o, z: [T, H, dv]; norm_w: [dv] or None.  y = n(o) * act(z)."""
    o = _f64(o)
    z = _f64(z)
    if norm_w is not None:
        ms = np.mean(o * o, axis=-1, keepdims=True)
        o = o / np.sqrt(ms + eps) * _f64(norm_w)
    if gate == GATE_SIGMOID:
        gz = sigmoid(z)
    elif gate == GATE_SILU:
        gz = z * sigmoid(z)
    else:
        raise ValueError("unknown gate %r" % gate)
    return o * gz
