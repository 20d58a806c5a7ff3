"""The device status word (include/gdn.h, gdn_read_status) and the bounded
waits behind it.

Every wait inside the tensor-core kernels is bounded; a wait that gives up
records a code in the status word and the kernel returns with its outputs
invalid but the GPU usable.  The bound is shortened through the library's
test hook (gdn_set_wait_limit) so that the waits really give up -- no broken
kernel and no unbounded wait is involved: with a bound of 0 the first wait on
a copy or MMA still in flight gives up, while the waits that drain a
kernel's work before it exits keep their 2 s bound.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads as W
import linear_attention_vlm_b200 as gdn
from linear_attention_vlm_b200 import gdn as binding

pytestmark = pytest.mark.gpu


def test_prefill_leaves_a_clear_status_word():
    x = W.random_prefill([300, 77], H=2, dk=128, dv=128, dtype=torch.bfloat16, seed=9)
    d = {k: v.cuda() for k, v in x.items() if v is not None}
    n = gdn.gdn_prefill_workspace_size(2, 377, 2, 128, 128)
    ws = torch.full((n,), 0xAB, dtype=torch.uint8, device="cuda")   # garbage before the call
    gdn.gdn_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], None, d["cu_seqlens"], workspace=ws)
    assert gdn.gdn_read_status(ws[:4].view(torch.int32)) == 0


def test_nonzero_word_reads_as_timeout():
    word = torch.tensor([73], dtype=torch.int32, device="cuda")
    assert gdn.gdn_read_status(word) == 73
    code = ctypes.c_int32(0)
    st = gdn.library().gdn_read_status(ctypes.c_void_p(word.data_ptr()), None, ctypes.byref(code))
    assert st == binding.GDN_ERR_TIMEOUT and code.value == 73


def _rel(x, ref):
    x = x.detach().double().cpu().numpy()
    return float(np.max(np.abs(x - ref)) / max(np.max(np.abs(ref)), 1e-30))


@pytest.mark.parametrize("lens,packed", [([2048], False), ([300, 77], True)], ids=["ranges", "packed"])
def test_expired_waits_are_reported_and_the_device_recovers(lens, packed):
    """A wait bound of 0: the prefill's kernels give up at their first wait
    on work in flight, leave a kernel code in the status word and exit with
    nothing in flight; a normal call on the same device then matches the
    oracle and leaves the word clear."""
    x = W.random_prefill(lens, H=2, dk=128, dv=128, dtype=torch.bfloat16, seed=41, state_std=0.02)
    d = {k: v.cuda() for k, v in x.items() if v is not None}
    N, T = len(lens), sum(lens)
    cu = d["cu_seqlens"] if packed else None
    ws = torch.empty(max(gdn.gdn_prefill_workspace_size(N, T, 2, 128, 128), 16), dtype=torch.uint8, device="cuda")
    word = ws[:4].view(torch.int32)
    gdn.gdn_set_wait_limit(0)
    try:
        gdn.gdn_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state_in"], cu, num_seqs=N, workspace=ws)
        code = gdn.gdn_read_status(word)
    finally:
        gdn.gdn_set_wait_limit(gdn.WAIT_LIMIT_DEFAULT)
    assert 50 <= code < 80, code            # the prefill kernels' codes
    out, st = gdn.gdn_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state_in"], cu, num_seqs=N,
                              workspace=ws)
    assert gdn.gdn_read_status(word) == 0
    f64 = lambda t: t.detach().to("cpu", torch.float64).numpy()
    ro, rs = oracle.prefill(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["g"]), f64(x["beta"]),
                            f64(x["state_in"]), x["cu_seqlens"].numpy().astype(np.int64))
    assert _rel(out, ro) <= 2e-2 and _rel(st, rs) <= 2e-2
