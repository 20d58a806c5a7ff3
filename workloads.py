"""Seeded synthetic inputs for the Gated DeltaNet hot path.

This module holds no arithmetic of the method: it only draws random numbers,
applies the input recipe (per-token L2 normalisation of q and k, beta =
sigmoid, g = log alpha), rounds to the storage precision and packs the
result.  Both the CUDA path's tests/benchmark and the oracle's callers use it.

Workloads (sizes follow the InfiniteVL pages: 16 GDN heads per layer, 8K
training context for stages I-II, 32K for long-sequence SFT, 256K prefill;
head dimension is not stated on the pages and is fixed here at 128, or 64 for
the tiny case):

  tiny_fp32          B=1, H=2,  T=256,    d=64,  fp32, alpha = sigmoid(N(3,1))
  prefill_bf16       B=1, H=16, T=8192,   d=128, bf16, g = -0.05 softplus(N(0,1))
  long_prefill_bf16  B=1, H=16, T=262144, d=128, bf16 (run as 64 x 4096 segments)
  decode_bf16        B=64 sequences, H=16, d=128, 1024 one-token steps,
                     fp32 state ~ N(0, 0.02^2)
  varlen_bf16        8 sequences, lengths uniform in [1024, 32768], packed
                     with cu_seqlens, per-sequence state ~ N(0, 0.02^2)

Random streams: one numpy PCG64 stream per (tensor, head, 4096-token block)
(or per (tensor, step) for decode), keyed by SeedSequence(seed, spawn_key).
Any subset of heads can therefore be drawn on its own and equals the same
heads of the full draw; the oracle side uses that to sample heads of the
full-size workloads.
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import os
from typing import Dict, Optional, Sequence

import numpy as np
import torch

BLOCK = 4096

# stream ids per tensor
_Q, _K, _V, _G, _B, _S, _LEN = 1, 2, 3, 4, 5, 6, 7


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    H: int
    dk: int
    dv: int
    chunk: int
    dtype: torch.dtype           # storage dtype of q, k, v, out
    alpha_dist: str              # "sigmoid3" or "logsoftplus"
    T: int = 0                   # tokens per sequence (uniform workloads)
    num_seqs: int = 1
    state_std: float = 0.0       # 0 => zero initial state
    varlen: Optional[tuple] = None   # (N, lo, hi) for packed varlen
    segments: int = 1            # long prefill: run as this many segments
    steps: int = 0               # decode: number of one-token steps


WORKLOADS: Dict[str, Workload] = {
    "tiny_fp32": Workload("tiny_fp32", H=2, dk=64, dv=64, chunk=64,
                          dtype=torch.float32, alpha_dist="sigmoid3", T=256),
    "prefill_bf16": Workload("prefill_bf16", H=16, dk=128, dv=128, chunk=64,
                             dtype=torch.bfloat16, alpha_dist="logsoftplus",
                             T=8192),
    "long_prefill_bf16": Workload("long_prefill_bf16", H=16, dk=128, dv=128,
                                  chunk=64, dtype=torch.bfloat16,
                                  alpha_dist="logsoftplus", T=262144,
                                  segments=64),
    "decode_bf16": Workload("decode_bf16", H=16, dk=128, dv=128, chunk=64,
                            dtype=torch.bfloat16, alpha_dist="logsoftplus",
                            num_seqs=64, state_std=0.02, steps=1024),
    "varlen_bf16": Workload("varlen_bf16", H=16, dk=128, dv=128, chunk=64,
                            dtype=torch.bfloat16, alpha_dist="logsoftplus",
                            num_seqs=8, state_std=0.02,
                            varlen=(8, 1024, 32768)),
}


def _rng(seed: int, *key: int) -> np.random.Generator:
    ss = np.random.SeedSequence(entropy=seed, spawn_key=tuple(int(x) for x in key))
    return np.random.Generator(np.random.PCG64(ss))


def _round(x: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    """Round float64/float32 numpy data to the storage dtype (RNE)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(dtype)


def _unit_rows(x: np.ndarray) -> np.ndarray:
    x = x.astype(np.float64)
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _softplus(x: np.ndarray) -> np.ndarray:
    return np.logaddexp(0.0, x)


def gate_from_normal(x: np.ndarray, alpha_dist: str) -> np.ndarray:
    """g = log alpha from a standard-normal draw x, computed in fp64."""
    x = x.astype(np.float64)
    if alpha_dist == "sigmoid3":          # alpha = sigmoid(N(3, 1))
        return -_softplus(-(x + 3.0))
    if alpha_dist == "logsoftplus":       # log alpha = -0.05 softplus(N(0, 1))
        return -0.05 * _softplus(x)
    raise ValueError(alpha_dist)


def seqlens(w: Workload, seed: int = 0) -> np.ndarray:
    """Per-sequence lengths of a workload."""
    if w.varlen is not None:
        n, lo, hi = w.varlen
        return _rng(seed, _LEN).integers(lo, hi, size=n, endpoint=True).astype(np.int64)
    return np.full(w.num_seqs, w.T, dtype=np.int64)


def _workers() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def _token_tensor(seed: int, tid: int, T: int, heads: Sequence[int], d: int,
                  unit: bool, dtype: torch.dtype) -> torch.Tensor:
    out = torch.empty((T, len(heads), d), dtype=dtype)

    def fill(job):
        j, h, b0 = job
        n = min(BLOCK, T - b0)
        x = _rng(seed, tid, h, b0 // BLOCK).standard_normal((n, d), dtype=np.float32)
        if unit:
            x = _unit_rows(x)
        out[b0:b0 + n, j, :] = _round(x, dtype)

    # every (head, block) has its own stream and its own slice of `out`, so
    # the blocks are drawn on a thread pool; the result does not depend on it
    jobs = [(j, h, b0) for j, h in enumerate(heads) for b0 in range(0, T, BLOCK)]
    if len(jobs) > 8:
        with concurrent.futures.ThreadPoolExecutor(_workers()) as ex:
            list(ex.map(fill, jobs))
    else:
        for job in jobs:
            fill(job)
    return out


def _scalar_tensor(seed: int, tid: int, T: int, heads: Sequence[int],
                   kind: str, alpha_dist: str) -> torch.Tensor:
    out = np.empty((T, len(heads)), dtype=np.float32)
    for j, h in enumerate(heads):
        for b0 in range(0, T, BLOCK):
            n = min(BLOCK, T - b0)
            x = _rng(seed, tid, h, b0 // BLOCK).standard_normal(n, dtype=np.float32)
            if kind == "beta":
                y = 1.0 / (1.0 + np.exp(-x.astype(np.float64)))
            else:
                y = gate_from_normal(x, alpha_dist)
            out[b0:b0 + n, j] = y.astype(np.float32)
    return torch.from_numpy(out)


def prefill_inputs(w: Workload, seed: int = 0,
                   heads: Optional[Sequence[int]] = None) -> Dict[str, torch.Tensor]:
    """Packed prefill inputs on the CPU, in storage precision.

    Returns q, k [T, Hs, dk]; v [T, Hs, dv] (w.dtype); g, beta [T, Hs] fp32;
    state_in [N, Hs, dv, dk] fp32 or None; cu_seqlens int32 [N+1].  ``heads``
    selects a subset (Hs of them), identical to those heads of the full draw.
    """
    heads = list(range(w.H)) if heads is None else list(heads)
    lens = seqlens(w, seed)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    T = int(cu[-1])
    q = _token_tensor(seed, _Q, T, heads, w.dk, True, w.dtype)
    k = _token_tensor(seed, _K, T, heads, w.dk, True, w.dtype)
    v = _token_tensor(seed, _V, T, heads, w.dv, False, w.dtype)
    g = _scalar_tensor(seed, _G, T, heads, "gate", w.alpha_dist)
    beta = _scalar_tensor(seed, _B, T, heads, "beta", w.alpha_dist)
    state = None
    if w.state_std > 0:
        N = len(lens)
        st = np.empty((N, len(heads), w.dv, w.dk), dtype=np.float32)
        for j, h in enumerate(heads):
            st[:, j] = _rng(seed, _S, h).standard_normal((N, w.dv, w.dk), dtype=np.float32) * np.float32(w.state_std)
        state = torch.from_numpy(st)
    return dict(q=q, k=k, v=v, g=g, beta=beta, state_in=state,
                cu_seqlens=torch.from_numpy(cu.astype(np.int32)))


def decode_state(w: Workload, seed: int = 0,
                 heads: Optional[Sequence[int]] = None) -> torch.Tensor:
    """Initial decode state [B, Hs, dv, dk] fp32 ~ N(0, state_std^2)."""
    heads = list(range(w.H)) if heads is None else list(heads)
    st = np.empty((w.num_seqs, len(heads), w.dv, w.dk), dtype=np.float32)
    for j, h in enumerate(heads):
        st[:, j] = _rng(seed, _S, h).standard_normal((w.num_seqs, w.dv, w.dk), dtype=np.float32) * np.float32(w.state_std)
    return torch.from_numpy(st)


def decode_tokens(w: Workload, step: int, seed: int = 0,
                  heads: Optional[Sequence[int]] = None) -> Dict[str, torch.Tensor]:
    """Inputs of decode step ``step``: q, k [B, Hs, dk], v [B, Hs, dv] in
    w.dtype; g, beta [B, Hs] fp32."""
    heads = list(range(w.H)) if heads is None else list(heads)
    B = w.num_seqs
    q = np.empty((B, len(heads), w.dk), dtype=np.float64)
    k = np.empty((B, len(heads), w.dk), dtype=np.float64)
    v = np.empty((B, len(heads), w.dv), dtype=np.float32)
    g = np.empty((B, len(heads)), dtype=np.float32)
    beta = np.empty((B, len(heads)), dtype=np.float32)
    for j, h in enumerate(heads):
        r = _rng(seed, 100, step, h)
        q[:, j] = _unit_rows(r.standard_normal((B, w.dk), dtype=np.float32))
        k[:, j] = _unit_rows(r.standard_normal((B, w.dk), dtype=np.float32))
        v[:, j] = r.standard_normal((B, w.dv), dtype=np.float32)
        g[:, j] = gate_from_normal(r.standard_normal(B, dtype=np.float32), w.alpha_dist)
        beta[:, j] = 1.0 / (1.0 + np.exp(-r.standard_normal(B, dtype=np.float32).astype(np.float64)))
    return dict(q=_round(q, w.dtype), k=_round(k, w.dtype), v=_round(v, w.dtype),
                g=torch.from_numpy(g), beta=torch.from_numpy(beta))


def random_prefill(T_list: Sequence[int], H: int, dk: int, dv: int,
                   dtype: torch.dtype, seed: int, alpha_dist: str = "logsoftplus",
                   state_std: float = 0.0) -> Dict[str, torch.Tensor]:
    """Small packed case with arbitrary per-sequence lengths (zeros allowed),
    drawn from one stream; used for ragged and edge-case parity tests."""
    r = _rng(seed, 900)
    cu = np.concatenate([[0], np.cumsum(np.asarray(T_list, dtype=np.int64))])
    T = int(cu[-1])
    q = _unit_rows(r.standard_normal((T, H, dk), dtype=np.float32)) if T else np.zeros((0, H, dk))
    k = _unit_rows(r.standard_normal((T, H, dk), dtype=np.float32)) if T else np.zeros((0, H, dk))
    v = r.standard_normal((T, H, dv), dtype=np.float32)
    g = gate_from_normal(r.standard_normal((T, H), dtype=np.float32), alpha_dist).astype(np.float32)
    beta = (1.0 / (1.0 + np.exp(-r.standard_normal((T, H), dtype=np.float32).astype(np.float64)))).astype(np.float32)
    N = len(T_list)
    state = None
    if state_std > 0:
        state = torch.from_numpy(r.standard_normal((N, H, dv, dk), dtype=np.float32) * np.float32(state_std))
    return dict(q=_round(q, dtype), k=_round(k, dtype), v=_round(v, dtype),
                g=torch.from_numpy(g), beta=torch.from_numpy(beta), state_in=state,
                cu_seqlens=torch.from_numpy(cu.astype(np.int32)))


def layer_inputs(T: int, H: int, d: int, dtype: torch.dtype = torch.bfloat16, seed: int = 0,
                 num_seqs: int = 1, state: bool = False) -> Dict[str, torch.Tensor]:
    """Raw inputs of the layer steps around the recurrence (pre-processing
    and output gate), on the CPU: projections x_q, x_k, x_v ~ N(0, 1) and gate
    input z ~ N(0, 4) in the storage dtype; convolution taps ~ N(0, 0.5^2),
    gate logits a ~ N(3, 1) (alpha = sigmoid(a), mean g near -0.05, like the
    tiny workload) and b ~ N(0, 1) (beta = sigmoid(b), like the prefill
    workload) in fp32; the RMS-norm weight ~ U[0.5, 1.5]; optionally a
    convolution state ~ N(0, 1) per sequence."""
    rng = _rng(seed, 7)
    out = {
        "xq": _round(rng.standard_normal((T, H, d), dtype=np.float32), dtype),
        "xk": _round(rng.standard_normal((T, H, d), dtype=np.float32), dtype),
        "xv": _round(rng.standard_normal((T, H, d), dtype=np.float32), dtype),
        "z": _round(2.0 * rng.standard_normal((T, H, d), dtype=np.float32), dtype),
        "conv_w": torch.from_numpy((0.5 * rng.standard_normal((3, H, d, 4))).astype(np.float32)),
        "a": torch.from_numpy((3.0 + rng.standard_normal((T, H))).astype(np.float32)),
        "b": torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)),
        "norm_w": torch.from_numpy(rng.uniform(0.5, 1.5, d).astype(np.float32)),
    }
    if state:
        out["conv_state"] = _round(rng.standard_normal((num_seqs, 3, 3, H, d), dtype=np.float32), dtype)
    return out


# sliding-window attention layer of the hybrid block: 16 query heads, 2
# key/value heads, window 8K tokens (InfiniteVL explainer page, "Step 2");
# head dimension 128 as for the linear layers
SWA_HQ, SWA_HKV, SWA_D, SWA_WINDOW = 16, 2, 128, 8192


def attention_inputs(T: int, Hq: int = SWA_HQ, Hkv: int = SWA_HKV, d: int = SWA_D,
                     dtype: torch.dtype = torch.bfloat16, seed: int = 0,
                     q_scale: float = 1.0) -> Dict[str, torch.Tensor]:
    """Inputs of the sliding-window attention layer, on the CPU: q ~
    N(0, q_scale^2), k, v ~ N(0, 1), [T, H, d] in the storage dtype (scores
    q.k / sqrt(d) then have standard deviation q_scale)."""
    rng = _rng(seed, 8)
    return {
        "q": _round(q_scale * rng.standard_normal((T, Hq, d), dtype=np.float32), dtype),
        "k": _round(rng.standard_normal((T, Hkv, d), dtype=np.float32), dtype),
        "v": _round(rng.standard_normal((T, Hkv, d), dtype=np.float32), dtype),
    }
