"""fp64 CPU oracle of the Gated DeltaNet recurrence -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  The product path (``linear_attention_vlm_b200``)
never imports it and shares no code with it.

The arithmetic lives in ``gdn_oracle.c`` (plain C, fp64, one token at a time;
see the comment at its top for the recurrence and where the pages describe
it).  This module only compiles that file with gcc and marshals numpy arrays.

Every function here is pinned by the CPU tests in ``tests/test_oracle_pins.py``
(closed forms, invariants, a hand-derived worked example, the delta rule as a
gradient step, and an independent chunked-form derivation).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle_gdn.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``gdn_oracle.c`` into ``liboracle_gdn.so`` next to it."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp%d" % os.getpid()
    # -O2 without -ffast-math: the compiler may not reassociate fp64 sums.
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread", _SRC,
           "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        lib.gdn_oracle_prefill.argtypes = [
            dp, dp, dp, dp, dp, dp, dp, dp, ctypes.POINTER(ctypes.c_int64),
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int]
        lib.gdn_oracle_prefill.restype = ctypes.c_int
        lib.gdn_oracle_decode.argtypes = [
            dp, dp, dp, dp, dp, dp, dp, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int]
        lib.gdn_oracle_decode.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def prefill(q, k, v, g, beta, state_in=None, cu_seqlens=None,
            nthreads: Optional[int] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Sequential fp64 Gated DeltaNet over a packed batch.

    q, k: [T, H, dk]; v: [T, H, dv]; g (= log alpha), beta: [T, H];
    state_in: [N, H, dv, dk] or None (zeros); cu_seqlens: [N+1] or None
    (one sequence of length T).  Returns (out [T, H, dv], state [N, H, dv, dk]).
    """
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    T, H, dk = q.shape
    dv = v.shape[2]
    if cu_seqlens is None:
        cu = np.array([0, T], dtype=np.int64)
    else:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    N = cu.shape[0] - 1
    if k.shape != (T, H, dk) or v.shape != (T, H, dv):
        raise ValueError("q/k/v shapes disagree")
    if g.shape != (T, H) or beta.shape != (T, H):
        raise ValueError("g/beta must be [T, H]")
    if cu[-1] != T:
        raise ValueError("cu_seqlens[-1] must equal T")
    s_in = None if state_in is None else _f64(state_in)
    if s_in is not None and s_in.shape != (N, H, dv, dk):
        raise ValueError("state_in must be [N, H, dv, dk]")
    out = np.zeros((T, H, dv), dtype=np.float64)
    s_out = np.zeros((N, H, dv, dk), dtype=np.float64)
    rc = _load().gdn_oracle_prefill(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(s_in),
        _ptr(out), _ptr(s_out),
        cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), N, H, dk, dv,
        nthreads or default_threads())
    if rc != 0:
        raise RuntimeError("gdn_oracle_prefill failed (%d)" % rc)
    return out, s_out


def decode_step(q, k, v, g, beta, state) -> Tuple[np.ndarray, np.ndarray]:
    """One token per sequence.  q, k [B, H, dk]; v [B, H, dv]; g, beta [B, H];
    state [B, H, dv, dk].  Returns (out [B, H, dv], new state)."""
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    B, H, dk = q.shape
    dv = v.shape[2]
    s = _f64(state).copy()
    if s.shape != (B, H, dv, dk):
        raise ValueError("state must be [B, H, dv, dk]")
    out = np.zeros((B, H, dv), dtype=np.float64)
    rc = _load().gdn_oracle_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                   _ptr(beta), _ptr(s), _ptr(out), B, H, dk,
                                   dv)
    if rc != 0:
        raise RuntimeError("gdn_oracle_decode failed (%d)" % rc)
    return out, s


# Steps around the recurrence inside one layer (plain numpy, fp64).
from .layer_ops import (ACT_NONE, ACT_SILU, GATE_SIGMOID, GATE_SILU,  # noqa: E402,F401
                        log_sigmoid, output_gate, preprocess, sigmoid)

# The hybrid block's other token mixer (plain numpy, fp64).
from .attention import positions as rope_positions  # noqa: E402,F401
from .attention import rope, swa_attention  # noqa: E402,F401
