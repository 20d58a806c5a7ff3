"""fp64 CPU oracle of the hybrid block's other token mixer, causal
sliding-window attention with rotary positions and grouped KV heads --
TEST INFRASTRUCTURE ONLY (same rules as the rest of ``oracle``).

The explainer page (InfiniteVL, "Step 2: Process tokens with Hybrid Blocks",
and the "Sliding Window Attention" concept box) describes the layer as
attention restricted to a recent local window of tokens (e.g. 8K), with RoPE
positions and grouped-query attention (16 query heads, 2 key-value heads).
The plainest readings taken:

* query token t of a sequence attends to the keys s of the same sequence with
  t - window < s <= t (causal, window counted in tokens, itself included);
* scores are (q_t . k_s) * scale, scale = 1/sqrt(d) unless given; softmax
  over the window;
* query head h reads key/value head h // (Hq / Hkv);
* RoPE is the rotate-half form: for i < d/2, with theta_i = base^(-2i/d) and
  angle a = p * theta_i, (x_i, x_{i+d/2}) -> (x_i cos a - x_{i+d/2} sin a,
  x_{i+d/2} cos a + x_i sin a); p is the token's position inside its
  sequence plus a caller-given offset; base 10000 unless given.

Plain numpy float64, one sequence and one head at a time.
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def positions(cu_seqlens, T: int, offset: int = 0) -> np.ndarray:
    """Position of every token inside its sequence, plus offset."""
    cu = np.array([0, T], dtype=np.int64) if cu_seqlens is None else np.asarray(cu_seqlens, dtype=np.int64)
    pos = np.zeros(T, dtype=np.int64)
    for n in range(cu.shape[0] - 1):
        b, e = int(cu[n]), int(cu[n + 1])
        pos[b:e] = np.arange(e - b) + offset
    return pos


def rope(x, pos, base: float = 10000.0) -> np.ndarray:
    """Rotate-half RoPE of x [T, H, d] at integer positions pos [T]."""
    x = _f64(x)
    d = x.shape[-1]
    half = d // 2
    theta = base ** (-2.0 * np.arange(half) / d)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * theta[None, :]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def swa_attention(q, k, v, cu_seqlens=None, window: int = 8192, scale: Optional[float] = None,
                  rows=None) -> np.ndarray:
    """q [T, Hq, d]; k, v [T, Hkv, d] (already rotated).  Returns o [T, Hq, d]
    (only the listed query rows are filled when ``rows`` is given)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    grp = Hq // Hkv
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    cu = np.array([0, T], dtype=np.int64) if cu_seqlens is None else np.asarray(cu_seqlens, dtype=np.int64)
    bos = np.zeros(T, dtype=np.int64)
    for n in range(cu.shape[0] - 1):
        bos[int(cu[n]):int(cu[n + 1])] = cu[n]
    out = np.zeros_like(q)
    ts = range(T) if rows is None else rows
    for t in ts:
        lo = max(int(bos[t]), t - window + 1)
        for h in range(Hq):
            kk = k[lo:t + 1, h // grp]
            vv = v[lo:t + 1, h // grp]
            s = kk @ q[t, h] * sc
            p = np.exp(s - s.max())
            out[t, h] = (p / p.sum()) @ vv
    return out
