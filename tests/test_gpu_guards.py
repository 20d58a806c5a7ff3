"""Out-of-bounds write checks for every kernel's outputs and scratch.

No memory checker is available on the GPU machines, so every buffer a kernel
writes -- outputs, final states and the prefill workspace -- is placed
between two 4 KiB guard regions filled with a sentinel byte.  After the call
the guards must be intact (no write outside the buffer) and the outputs
finite.  The cases are the ragged ones, where tail handling decides the
bounds: lengths 1, 63, 65, 200, packed batches with empty sequences, one
long sequence cut into sequence-parallel chunk ranges, and a packed
(varlen) batch.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
import linear_attention_vlm_b200 as gdn

pytestmark = pytest.mark.gpu

GUARD = 4096
SENTINEL = 0xA5


class Guarded:
    """A device buffer of `shape`/`dtype` with GUARD sentinel bytes on both
    sides; `t` is the buffer (16-byte aligned), `intact()` checks the guards."""

    def __init__(self, shape, dtype, dev):
        n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
        self.raw = torch.full((GUARD + n + GUARD,), SENTINEL, dtype=torch.uint8, device=dev)
        self.t = self.raw[GUARD:GUARD + n].view(dtype).view(shape) if n else \
            torch.empty(shape, dtype=dtype, device=dev)
        self.n = n

    def intact(self):
        torch.cuda.synchronize()
        head = self.raw[:GUARD]
        tail = self.raw[GUARD + self.n:]
        return bool(torch.all(head == SENTINEL)) and bool(torch.all(tail == SENTINEL))


def np64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def rel_err(x, ref):
    scale = np.max(np.abs(ref)) if ref.size else 0.0
    return float(np.max(np.abs(x - ref)) / (scale if scale > 0 else 1.0)) if ref.size else 0.0


PREFILL_CASES = [
    ([1], 3, 128, torch.bfloat16, True),
    ([63], 3, 128, torch.bfloat16, True),
    ([65], 3, 128, torch.bfloat16, True),
    ([200], 3, 128, torch.bfloat16, True),
    ([0, 1, 130, 0, 64, 77], 3, 128, torch.bfloat16, True),
    ([4000], 2, 128, torch.bfloat16, False),          # sequence-parallel chunk ranges
    ([2048, 2048], 3, 128, torch.bfloat16, False),    # ranges over two sequences
    ([3000, 17, 1500, 0, 64], 4, 128, torch.bfloat16, True),   # packed (varlen)
    ([1], 2, 64, torch.float32, True),
    ([0, 1, 130, 0, 64, 77], 2, 64, torch.float32, True),
    ([200], 2, 128, torch.float32, True),
]


@pytest.mark.parametrize("lens,H,d,dtype,packed", PREFILL_CASES,
                         ids=lambda x: None if not isinstance(x, list) else "L" + "-".join(map(str, x)))
def test_prefill_writes_stay_in_bounds(cuda_device, lens, H, d, dtype, packed):
    inp = W.random_prefill(lens, H=H, dk=d, dv=d, dtype=dtype, seed=sum(lens) + H, state_std=0.02)
    t = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    N, T = len(lens), sum(lens)
    out = Guarded((T, H, d), dtype, cuda_device)
    st = Guarded((N, H, d, d), torch.float32, cuda_device)
    need = gdn.gdn_prefill_workspace_size(N, T, H, d, d, dtype=dtype)
    ws = Guarded((max(need, 16),), torch.uint8, cuda_device)
    cu = t["cu_seqlens"] if packed else None
    gdn.gdn_prefill(t["q"], t["k"], t["v"], t["g"], t["beta"], t["state_in"], cu,
                    num_seqs=None if packed else N, out=out.t, state_out=st.t, workspace=ws.t)
    assert out.intact(), "write outside out"
    assert st.intact(), "write outside state_out"
    assert ws.intact(), "write outside the workspace"
    o, s = np64(out.t), np64(st.t)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(s))
    ro, rs = oracle.prefill(np64(inp["q"]), np64(inp["k"]), np64(inp["v"]), np64(inp["g"]),
                            np64(inp["beta"]), np64(inp["state_in"]),
                            inp["cu_seqlens"].numpy().astype(np.int64))
    tol = 2e-2 if dtype == torch.bfloat16 else 1e-4
    assert rel_err(o, ro) <= tol and rel_err(s, rs) <= tol


@pytest.mark.parametrize("d,dtype", [(128, torch.bfloat16), (64, torch.float32)], ids=["bf16", "f32"])
def test_decode_writes_stay_in_bounds(cuda_device, d, dtype):
    B, H = 7, 3
    x = W.random_prefill([1] * B, H=H, dk=d, dv=d, dtype=dtype, seed=5, state_std=0.02)
    q, k, v = (x[n].reshape(B, H, d).to(cuda_device) for n in ("q", "k", "v"))
    g, b = x["g"].reshape(B, H).to(cuda_device), x["beta"].reshape(B, H).to(cuda_device)
    s_in = x["state_in"].to(cuda_device)
    out = Guarded((B, H, d), dtype, cuda_device)
    s_out = Guarded((B, H, d, d), torch.float32, cuda_device)
    gdn.gdn_decode_step(q, k, v, g, b, s_in, s_out.t, out=out.t)
    assert out.intact() and s_out.intact()
    assert torch.isfinite(out.t).all() and torch.isfinite(s_out.t).all()


@pytest.mark.parametrize("T,cu", [(300, [0, 170, 300]), (129, None), (1, None)])
def test_attention_writes_stay_in_bounds(cuda_device, T, cu):
    A = W.attention_inputs(T, Hq=4, Hkv=2, d=128, seed=6)
    cus = None if cu is None else torch.tensor(cu, dtype=torch.int32, device=cuda_device)
    qr = Guarded((T, 4, 128), torch.bfloat16, cuda_device)
    gdn.gdn_rope(A["q"].to(cuda_device), cus, out=qr.t)
    o = Guarded((T, 4, 128), torch.bfloat16, cuda_device)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    gdn.gdn_swa_attention(qr.t, A["k"].to(cuda_device), A["v"].to(cuda_device), cus, window=100,
                          out=o.t, status=status)
    assert qr.intact() and o.intact()
    assert torch.isfinite(o.t.float()).all()
    assert gdn.gdn_read_status(status) == 0


@pytest.mark.parametrize("rows", [1, 33, 1000])
def test_output_gate_writes_stay_in_bounds(cuda_device, rows):
    L = W.layer_inputs(rows, 1, 128, torch.bfloat16, seed=7)
    y = Guarded((rows, 1, 128), torch.bfloat16, cuda_device)
    gdn.gdn_output_gate(L["xv"].to(cuda_device), L["z"].to(cuda_device), L["norm_w"].to(cuda_device), out=y.t)
    assert y.intact() and torch.isfinite(y.t.float()).all()
