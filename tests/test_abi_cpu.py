"""The C ABI without a GPU: the library loads, exports every function the
header declares, sizes workspaces, and rejects bad arguments on the host
before anything is enqueued."""
import ctypes

import pytest

import linear_attention_vlm_b200 as gdn
from linear_attention_vlm_b200 import gdn as binding


@pytest.fixture(scope="module")
def lib():
    return gdn.library()


def test_exports_every_declared_symbol(lib):
    names = gdn.declared_symbols()
    assert {"gdn_prefill", "gdn_decode_step", "gdn_prefill_workspace_size",
            "gdn_status_string", "gdn_last_cuda_error"} <= set(names)
    for n in names:
        assert hasattr(lib, n), "libgdn.so does not export %s" % n


def test_status_strings(lib):
    for code in (0, 1, 2, 3, 4, 5):
        assert gdn.status_string(code).startswith("GDN_")
    assert "unknown" in gdn.status_string(99)
    assert binding._load().gdn_last_cuda_error() == b""


def test_workspace_size_is_host_arithmetic():
    import torch
    # rejected configurations report 0
    assert gdn.gdn_prefill_workspace_size(1, 8192, 16, 96, 96) == 0
    assert gdn.gdn_prefill_workspace_size(1, 8192, 16, 128, 128, chunk=32) == 0
    assert gdn.gdn_prefill_workspace_size(0, 8192, 16, 128, 128) == 0
    # supported ones are finite and grow with the token count
    a = gdn.gdn_prefill_workspace_size(1, 8192, 16, 128, 128, dtype=torch.bfloat16)
    b = gdn.gdn_prefill_workspace_size(1, 16384, 16, 128, 128, dtype=torch.bfloat16)
    assert 0 <= a <= b < (1 << 40)


def _prefill_raw(lib, **kw):
    args = dict(q=16, k=16, v=16, g=16, beta=16, state_in=None, out=16, state_out=None,
                cu=None, N=1, T=64, H=2, dk=64, dv=64, chunk=64, dtype=0, ws=None, wsb=0,
                stream=None)
    args.update(kw)
    return lib.gdn_prefill(args["q"], args["k"], args["v"], args["g"], args["beta"],
                           args["state_in"], args["out"], args["state_out"], args["cu"],
                           args["N"], args["T"], args["H"], args["dk"], args["dv"],
                           args["chunk"], args["dtype"], args["ws"], args["wsb"], args["stream"])


def test_prefill_rejects_bad_arguments(lib):
    assert _prefill_raw(lib, q=None) == binding.GDN_ERR_INVALID_ARG
    assert _prefill_raw(lib, q=17) == binding.GDN_ERR_INVALID_ARG          # misaligned
    assert _prefill_raw(lib, N=0) == binding.GDN_ERR_INVALID_ARG
    assert _prefill_raw(lib, T=-1) == binding.GDN_ERR_INVALID_ARG
    assert _prefill_raw(lib, dtype=7) == binding.GDN_ERR_INVALID_ARG
    assert _prefill_raw(lib, N=3, T=64) == binding.GDN_ERR_INVALID_ARG      # T % N != 0 without cu
    assert _prefill_raw(lib, dk=96, dv=96) == binding.GDN_ERR_UNSUPPORTED
    assert _prefill_raw(lib, dk=128, dv=64) == binding.GDN_ERR_UNSUPPORTED
    assert _prefill_raw(lib, chunk=32) == binding.GDN_ERR_UNSUPPORTED
    # partial overlap of state_in and state_out
    assert _prefill_raw(lib, state_in=4096, state_out=4096 + 64) == binding.GDN_ERR_INVALID_ARG


def test_decode_rejects_bad_arguments(lib):
    def call(**kw):
        a = dict(q=16, k=16, v=16, g=16, beta=16, si=4096, so=4096, out=16, B=1, H=1, dk=64,
                 dv=64, dtype=1)
        a.update(kw)
        return lib.gdn_decode_step(a["q"], a["k"], a["v"], a["g"], a["beta"], a["si"], a["so"],
                                   a["out"], a["B"], a["H"], a["dk"], a["dv"], a["dtype"], None)
    assert call(B=0) == binding.GDN_OK                                      # no-op
    assert call(q=None) == binding.GDN_ERR_INVALID_ARG
    assert call(out=8) == binding.GDN_ERR_INVALID_ARG
    assert call(B=-1) == binding.GDN_ERR_INVALID_ARG
    assert call(dk=32, dv=32) == binding.GDN_ERR_UNSUPPORTED
    assert call(dtype=3) == binding.GDN_ERR_INVALID_ARG
    assert call(si=4096, so=4096 + 16) == binding.GDN_ERR_INVALID_ARG       # partial overlap


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(64, 2, 64)
    s = torch.zeros(64, 2)
    with pytest.raises(ValueError):
        gdn.gdn_prefill(x, x, x, s, s)
    with pytest.raises(ValueError):
        gdn.gdn_decode_step(x[:1], x[:1], x[:1], s[:1], s[:1], torch.zeros(1, 2, 64, 64))


def _pre_raw(lib, **kw):
    base = 1 << 20
    args = dict(xq=base, xk=2 * base, xv=3 * base, w=4 * base, a=5 * base, b=6 * base, csi=None,
                q=7 * base, k=8 * base, v=9 * base, g=10 * base, beta=11 * base, cso=None, cu=None,
                N=1, T=64, H=2, d=64, act=0, eps=1e-6, dtype=1, stream=None)
    args.update(kw)
    return lib.gdn_preprocess(args["xq"], args["xk"], args["xv"], args["w"], args["a"], args["b"],
                              args["csi"], args["q"], args["k"], args["v"], args["g"], args["beta"],
                              args["cso"], args["cu"], args["N"], args["T"], args["H"], args["d"],
                              args["act"], ctypes.c_float(args["eps"]), args["dtype"], args["stream"])


def test_preprocess_rejects_bad_arguments(lib):
    inv, uns = binding.GDN_ERR_INVALID_ARG, binding.GDN_ERR_UNSUPPORTED
    assert _pre_raw(lib, xq=None) == inv
    assert _pre_raw(lib, g=(11 << 20) + 4) == inv                 # misaligned
    assert _pre_raw(lib, d=96) == uns
    assert _pre_raw(lib, act=2) == inv
    assert _pre_raw(lib, eps=-1.0) == inv
    assert _pre_raw(lib, N=3, T=64) == inv                        # uniform split must be exact
    assert _pre_raw(lib, q=1 << 20) == inv                        # output over an input
    assert _pre_raw(lib, cso=(5 << 20) + 64) == inv               # state over an input
    assert _pre_raw(lib, T=0) == binding.GDN_OK                   # nothing to do, nothing enqueued


def test_output_gate_rejects_bad_arguments(lib):
    inv = binding.GDN_ERR_INVALID_ARG
    f = lambda o=1 << 20, z=2 << 20, w=None, y=3 << 20, rows=10, dv=64, gate=0, eps=1e-6, dt=1: \
        lib.gdn_output_gate(o, z, w, y, rows, dv, gate, ctypes.c_float(eps), dt, None)
    assert f(o=None) == inv
    assert f(gate=5) == inv
    assert f(dv=32) == binding.GDN_ERR_UNSUPPORTED
    assert f(y=(2 << 20) + 16) == inv                            # y over z
    assert f(rows=0) == binding.GDN_OK


def test_session_create_rejects_bad_arguments(lib):
    bufs = binding._SessionBuffers(*([1 << 20] * 18), 1 << 30)
    h = ctypes.c_void_p()
    f = lambda **kw: lib.gdn_session_create(kw.get("B", 1), kw.get("H", 2), kw.get("d", 64), kw.get("seg", 64),
                                            kw.get("dtype", 1), kw.get("act", 0), kw.get("gate", 0),
                                            ctypes.c_float(kw.get("eps", 1e-6)), ctypes.byref(kw.get("bufs", bufs)),
                                            ctypes.byref(h))
    assert f(d=96) == binding.GDN_ERR_UNSUPPORTED
    assert f(B=0) == binding.GDN_ERR_INVALID_ARG
    assert f(gate=3) == binding.GDN_ERR_INVALID_ARG
    bad = binding._SessionBuffers(*([1 << 20] * 17 + [0]), 0)            # no workspace (bf16, d = 128 needs one)
    assert f(bufs=bad, d=128) == binding.GDN_ERR_WORKSPACE
    bad = binding._SessionBuffers(*([0] + [1 << 20] * 17), 1 << 30)        # a missing buffer
    assert f(bufs=bad) == binding.GDN_ERR_INVALID_ARG
    assert h.value is None


def test_rope_rejects_bad_arguments(lib):
    inv, uns = binding.GDN_ERR_INVALID_ARG, binding.GDN_ERR_UNSUPPORTED
    f = lambda x=1 << 20, out=2 << 20, cu=None, N=1, T=64, H=2, d=64, off=0, base=10000.0, dt=1: \
        lib.gdn_rope(x, out, cu, N, T, H, d, off, ctypes.c_float(base), dt, None)
    assert f(x=None) == inv
    assert f(out=(2 << 20) + 8) == inv                            # misaligned
    assert f(d=12) == uns
    assert f(d=264) == uns
    assert f(base=1.0) == inv
    assert f(off=-1) == inv
    assert f(dt=4) == inv
    assert f(N=3, T=64) == inv                                    # uniform split must be exact
    assert f(out=(1 << 20) + 64) == inv                           # partial overlap (in place is fine)
    assert f(T=0) == binding.GDN_OK


def test_swa_attention_rejects_bad_arguments(lib):
    inv, uns = binding.GDN_ERR_INVALID_ARG, binding.GDN_ERR_UNSUPPORTED
    base = 1 << 24

    def f(q=base, k=2 * base, v=3 * base, o=4 * base, cu=None, N=1, T=256, Hq=4, Hkv=2, d=128, win=64,
          scale=0.0, dt=1, status=None):
        return lib.gdn_swa_attention(q, k, v, o, cu, N, T, Hq, Hkv, d, win, ctypes.c_float(scale), dt, status, None)
    assert f(q=None) == inv
    assert f(o=4 * base + 8) == inv                               # misaligned
    assert f(d=64) == uns
    assert f(dt=0) == uns                                         # fp32 attention is not built
    assert f(dt=3) == inv
    assert f(Hq=3, Hkv=2) == inv
    assert f(win=0) == inv
    assert f(scale=-1.0) == inv
    assert f(N=3, T=256) == inv
    assert f(o=base + 4096) == inv                                # output over q
    assert f(status=4 * base + 2) == inv
    assert f(T=0) == binding.GDN_OK


def test_read_status_rejects_bad_words(lib):
    code = ctypes.c_int32(7)
    assert lib.gdn_read_status(None, None, ctypes.byref(code)) == binding.GDN_ERR_INVALID_ARG
    assert code.value == 0                                        # cleared before anything else
    assert lib.gdn_read_status(4098, None, None) == binding.GDN_ERR_INVALID_ARG   # not 4-byte aligned


def test_attention_bindings_refuse_bad_tensors():
    import torch
    q = torch.zeros(16, 4, 128, dtype=torch.bfloat16)
    kv = torch.zeros(16, 2, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        gdn.gdn_rope(q)                                   # CPU tensor
    with pytest.raises(ValueError):
        gdn.gdn_swa_attention(q, kv, kv)                  # CPU tensors
    with pytest.raises(ValueError):
        gdn.gdn_read_status(torch.zeros(1, dtype=torch.int32))
