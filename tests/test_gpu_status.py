"""The device status word (include/gdn.h, gdn_read_status): clear after
normal tensor-core calls, and read back as GDN_ERR_TIMEOUT with its code when
it holds one.  A timed-out wait is never provoked on the GPU: the nonzero word
is written from the host."""
import ctypes

import pytest
import torch

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
