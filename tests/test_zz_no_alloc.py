"""gdn_prefill_noalloc: the prefill for callers that cannot allocate device
memory (a serving loop that reserves all device memory at start-up, or a
host that cannot pass a workspace pointer).  It runs the same kernels with
the library's fixed scratch array instead of a caller-owned workspace, so it
must agree with gdn_prefill -- here on two calls in a row with different
shapes, so the second call starts from the first call's leftover scratch.

This file is collected last on purpose: a run that stops at the first
failure has run every other test before it.
"""
import numpy as np
import pytest
import torch

import workloads as W
import linear_attention_vlm_b200 as gdn
from linear_attention_vlm_b200 import gdn as binding

pytestmark = pytest.mark.gpu

TOL = 2e-2   # the bf16 bar used by every parity test


def _rel(x, ref):
    x = x.detach().double().cpu().numpy()
    ref = ref.detach().double().cpu().numpy()
    return float(np.max(np.abs(x - ref)) / max(np.max(np.abs(ref)), 1e-30))


def _one_call(dev, lens, H, state_std, seed):
    x = W.random_prefill(lens, H=H, dk=128, dv=128, dtype=torch.bfloat16, seed=seed,
                         state_std=state_std)
    d = {k: (v.to(dev) if v is not None else None) for k, v in x.items()}
    cu = d["cu_seqlens"] if len(lens) > 1 else None
    ref_o, ref_s = gdn.gdn_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state_in"], cu)
    got_o, got_s = gdn.gdn_prefill_noalloc(d["q"], d["k"], d["v"], d["g"], d["beta"],
                                           d["state_in"], cu)
    torch.cuda.synchronize()
    return _rel(got_o, ref_o), _rel(got_s, ref_s)


def test_noalloc_matches_prefill_on_two_calls(cuda_device):
    e1 = _one_call(cuda_device, [100, 37, 0, 64], 2, 0.02, seed=21)
    e2 = _one_call(cuda_device, [600], 16, 0.0, seed=22)
    for eo, es in (e1, e2):
        assert eo <= TOL and es <= TOL, (e1, e2)
    # the kernels' status word lives in the scratch, out of the caller's
    # sight; the accessor reads it: every wait of the two calls completed
    assert gdn.gdn_noalloc_read_status() == 0


def _largest_fitting_tokens(H):
    """Longest single sequence of H heads whose workspace fits the scratch."""
    best = 0
    for T in range(256, 262145, 256):
        if gdn.gdn_prefill_workspace_size(1, T, H, 128, 128) <= binding.NOALLOC_SCRATCH_BYTES:
            best = T
    return best


def test_noalloc_near_the_scratch_limit(cuda_device):
    # one long sequence of 16 heads, as long as the scratch allows: few
    # sequences of many chunks take the sequence-parallel chunk ranges, so
    # the range transitions and start states sit near the end of the array
    H = 16
    T = _largest_fitting_tokens(H)
    need = gdn.gdn_prefill_workspace_size(1, T, H, 128, 128)
    assert T >= 1024 and binding.NOALLOC_SCRATCH_BYTES // 2 < need <= binding.NOALLOC_SCRATCH_BYTES
    eo, es = _one_call(cuda_device, [T], H, 0.02, seed=23)
    assert eo <= TOL and es <= TOL, (T, eo, es)
    assert gdn.gdn_noalloc_read_status() == 0


def test_noalloc_rejects_requests_beyond_the_scratch(cuda_device):
    # 16 heads x 16384 tokens needs far more than the 16 MiB scratch; the
    # request is refused on the host before any kernel is enqueued
    T, H = 16384, 16
    assert gdn.gdn_prefill_workspace_size(1, T, H, 128, 128) > binding.NOALLOC_SCRATCH_BYTES
    q = torch.zeros(T, H, 128, dtype=torch.bfloat16, device=cuda_device)
    s = torch.zeros(T, H, dtype=torch.float32, device=cuda_device)
    with pytest.raises(gdn.GdnError) as ei:
        gdn.gdn_prefill_noalloc(q, q, q, s, s)
    assert ei.value.status == binding.GDN_ERR_WORKSPACE
