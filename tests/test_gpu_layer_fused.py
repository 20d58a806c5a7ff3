"""Parity of gdn_layer_prefill (the layer's pre-processing, recurrence and
output gate in one call; fused into the prefill kernels on the tensor-core
path) with the fp64 oracle composed step by step: preprocess -> prefill ->
output_gate (explainer page, "Step 2: Process tokens with Hybrid Blocks"; the
recurrence of its "Gated DeltaNet" box).

The oracle chain rounds q, k, v and o to the storage dtype between the steps,
as the three separate calls store them.  Bars as elsewhere: bf16 2e-2, fp32
1e-4 relative to the max-norm; the convolution state is data movement and
must match bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import linear_attention_vlm_b200 as gdn

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}
EPS = 1e-6


def rel_err(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    if ref.size == 0:
        return 0.0
    scale = np.max(np.abs(ref))
    return float(np.max(np.abs(x - ref)) / (scale if scale > 0 else 1.0))


def np64(t):
    return None if t is None else t.detach().to("cpu", torch.float64).numpy()


def stored(x, dtype):
    """fp64 values rounded to the storage dtype (round to nearest even)."""
    return torch.from_numpy(np.ascontiguousarray(x)).to(dtype).to(torch.float64).numpy()


def layer_inputs(lens, H, d, dtype, seed, conv_state=True, state=True, norm=True):
    """Raw projections x ~ N(0, 1), conv taps ~ N(0, 0.5^2), a ~ N(3, 1)
    (alpha = sigmoid(a) near 0.95), b ~ N(0, 1), z ~ N(0, 1), norm weights
    1 + N(0, 0.1^2), recurrent state N(0, 0.02^2)."""
    rng = np.random.default_rng(seed)
    T, N = int(sum(lens)), len(lens)
    f = lambda *s: rng.standard_normal(s).astype(np.float32)
    inp = {
        "xq": torch.from_numpy(f(T, H, d)).to(dtype),
        "xk": torch.from_numpy(f(T, H, d)).to(dtype),
        "xv": torch.from_numpy(f(T, H, d)).to(dtype),
        "z": torch.from_numpy(f(T, H, d)).to(dtype),
        "w": torch.from_numpy(0.5 * f(3, H, d, 4)),
        "a": torch.from_numpy(3.0 + f(T, H)),
        "b": torch.from_numpy(f(T, H)),
        "cs": torch.from_numpy(f(N, 3, 3, H, d)).to(dtype) if conv_state else None,
        "state": torch.from_numpy(0.02 * f(N, H, d, d)) if state else None,
        "norm_w": torch.from_numpy(1.0 + 0.1 * f(d)) if norm else None,
        "cu": torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32),
    }
    return inp


def oracle_layer(inp, act, gate, dtype):
    cu = inp["cu"].numpy().astype(np.int64)
    q, k, v, g, beta, cs_out = oracle.preprocess(np64(inp["xq"]), np64(inp["xk"]), np64(inp["xv"]),
                                                 np64(inp["w"]), np64(inp["a"]), np64(inp["b"]), cu,
                                                 np64(inp["cs"]), activation=act, eps=EPS)
    o, st = oracle.prefill(stored(q, dtype), stored(k, dtype), stored(v, dtype), g, beta, np64(inp["state"]), cu)
    y = oracle.output_gate(stored(o, dtype), np64(inp["z"]), np64(inp["norm_w"]), gate=gate, eps=EPS)
    return y, st, cs_out


def run_layer(inp, dev, act, gate, packed=True, in_place=False):
    t = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    N = t["cu"].numel() - 1
    kw = dict(activation=act, gate=gate, eps=EPS)
    if in_place:
        kw.update(state_out=t["state"], conv_state_out=t["cs"])
    y, st, cs = gdn.gdn_layer_prefill(t["xq"], t["xk"], t["xv"], t["w"], t["a"], t["b"], t["z"], t["cs"],
                                      t["state"], t["norm_w"], t["cu"] if packed else None,
                                      num_seqs=None if packed else N, **kw)
    torch.cuda.synchronize()
    return y, st, cs


def check(inp, dev, act, gate, dtype, packed=True, in_place=False):
    y, st, cs = run_layer(inp, dev, act, gate, packed, in_place)
    ry, rst, rcs = oracle_layer(inp, act, gate, dtype)
    ey, es = rel_err(np64(y), ry), rel_err(np64(st), rst)
    assert ey <= TOL[dtype], "y err %.3g" % ey
    assert es <= TOL[dtype], "state err %.3g" % es
    assert torch.equal(cs.cpu(), torch.from_numpy(rcs).to(dtype))
    assert np.all(np.isfinite(np64(y)))
    return y, st, cs


@pytest.mark.parametrize("act,gate,norm", [(gdn.ACT_SILU, gdn.GATE_SILU, True),
                                           (gdn.ACT_NONE, gdn.GATE_SIGMOID, False)],
                         ids=["silu-silu-rms", "none-sigmoid-plain"])
@pytest.mark.parametrize("lens", [[200, 0, 130, 1, 64, 3], [65], [1, 2, 3]],
                         ids=lambda l: "lens" + "-".join(map(str, l)))
def test_layer_packed_tc(cuda_device, act, gate, norm, lens):
    inp = layer_inputs(lens, 2, 128, torch.bfloat16, seed=sum(lens) + act, norm=norm)
    check(inp, cuda_device, act, gate, torch.bfloat16)


def test_layer_without_states(cuda_device):
    inp = layer_inputs([130, 64, 7], 3, 128, torch.bfloat16, seed=5, conv_state=False, state=False)
    check(inp, cuda_device, gdn.ACT_SILU, gdn.GATE_SIGMOID, torch.bfloat16)


def test_layer_sequence_parallel_ranges(cuda_device):
    """One long unpacked sequence: the transition ranges, the combine and the
    output ranges all read the k, v, g and beta the prep kernel writes."""
    T, H = 4096, 2
    assert gdn.gdn_prefill_kernel_count(1, T, H, 128, 128) == 4
    inp = layer_inputs([T], H, 128, torch.bfloat16, seed=11)
    check(inp, cuda_device, gdn.ACT_SILU, gdn.GATE_SILU, torch.bfloat16, packed=False)


def test_layer_uniform_batch_in_place(cuda_device):
    inp = layer_inputs([192, 192, 192], 4, 128, torch.bfloat16, seed=12)
    ref = {k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    dev_inp = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    y, st, cs = run_layer(dev_inp, cuda_device, gdn.ACT_SILU, gdn.GATE_SILU, packed=False, in_place=True)
    assert st.data_ptr() == dev_inp["state"].data_ptr() and cs.data_ptr() == dev_inp["cs"].data_ptr()
    ry, rst, rcs = oracle_layer(ref, gdn.ACT_SILU, gdn.GATE_SILU, torch.bfloat16)
    assert rel_err(np64(y), ry) <= 2e-2 and rel_err(np64(st), rst) <= 2e-2
    assert torch.equal(cs.cpu(), torch.from_numpy(rcs).to(torch.bfloat16))


@pytest.mark.parametrize("dtype,d", [(torch.float32, 64), (torch.float32, 128), (torch.bfloat16, 64)],
                         ids=["f32-64", "f32-128", "bf16-64"])
def test_layer_composed_path(cuda_device, dtype, d):
    inp = layer_inputs([70, 0, 5, 129], 2, d, dtype, seed=13 + d)
    check(inp, cuda_device, gdn.ACT_SILU, gdn.GATE_SILU, dtype)


def test_layer_matches_three_calls(cuda_device):
    """The fused call and the three separate calls compute the same thing;
    they differ only in the order of two sums (the L2 and RMS norms)."""
    inp = layer_inputs([300, 77, 64], 2, 128, torch.bfloat16, seed=14)
    t = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    y, st, cs = run_layer(t, cuda_device, gdn.ACT_SILU, gdn.GATE_SILU)
    q, k, v, g, beta, cs2 = gdn.gdn_preprocess(t["xq"], t["xk"], t["xv"], t["w"], t["a"], t["b"], t["cs"], t["cu"],
                                               activation=gdn.ACT_SILU, eps=EPS)
    o, st2 = gdn.gdn_prefill(q, k, v, g, beta, t["state"], t["cu"])
    y2 = gdn.gdn_output_gate(o, t["z"], t["norm_w"], gate=gdn.GATE_SILU, eps=EPS)
    torch.cuda.synchronize()
    assert torch.equal(cs, cs2)
    assert rel_err(np64(y), np64(y2)) <= 1e-2
    assert rel_err(np64(st), np64(st2)) <= 1e-2


def test_layer_carried_over_two_calls(cuda_device):
    """Both states carried in place through two calls equal one call over the
    whole sequence (the second call's first chunk takes its halo rows from the
    convolution state)."""
    H, T1, T2 = 2, 100, 157
    inp = layer_inputs([T1 + T2], H, 128, torch.bfloat16, seed=15)
    ry, rst, rcs = oracle_layer(inp, gdn.ACT_SILU, gdn.GATE_SIGMOID, torch.bfloat16)
    t = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    st, cs = t["state"].clone(), t["cs"].clone()
    ys = []
    for sl in (slice(0, T1), slice(T1, T1 + T2)):
        y, _, _ = gdn.gdn_layer_prefill(t["xq"][sl], t["xk"][sl], t["xv"][sl], t["w"], t["a"][sl], t["b"][sl],
                                        t["z"][sl], cs, st, t["norm_w"], activation=gdn.ACT_SILU,
                                        gate=gdn.GATE_SIGMOID, eps=EPS, state_out=st, conv_state_out=cs)
        ys.append(np64(y))
    torch.cuda.synchronize()
    assert rel_err(np.concatenate(ys), ry) <= 2e-2
    assert rel_err(np64(st), rst) <= 2e-2
    assert torch.equal(cs.cpu(), torch.from_numpy(rcs).to(torch.bfloat16))


def test_layer_guard_regions(cuda_device):
    """y and the workspace sit between 4 KiB sentinel regions that must come
    back untouched."""
    lens = [200, 0, 130, 1, 63, 65]
    H, d = 2, 128
    inp = layer_inputs(lens, H, d, torch.bfloat16, seed=16)
    t = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    T, N = sum(lens), len(lens)
    G = 4096
    ny = T * H * d * 2
    nws = gdn.gdn_layer_prefill_workspace_size(N, T, H, d)
    buf = torch.full((G + ny + G + nws + G,), 0xA5, dtype=torch.uint8, device=cuda_device)
    y = buf[G:G + ny].view(torch.bfloat16).view(T, H, d)
    ws = buf[2 * G + ny:2 * G + ny + nws]
    gdn.gdn_layer_prefill(t["xq"], t["xk"], t["xv"], t["w"], t["a"], t["b"], t["z"], t["cs"], t["state"],
                          t["norm_w"], t["cu"], activation=gdn.ACT_SILU, gate=gdn.GATE_SILU, eps=EPS, y=y,
                          workspace=ws)
    torch.cuda.synchronize()
    for lo, hi in ((0, G), (G + ny, 2 * G + ny), (2 * G + ny + nws, buf.numel())):
        assert bool((buf[lo:hi] == 0xA5).all()), (lo, hi)
    ry, _, _ = oracle_layer(inp, gdn.ACT_SILU, gdn.GATE_SILU, torch.bfloat16)
    assert rel_err(np64(y), ry) <= 2e-2
    assert gdn.gdn_read_status(ws[:4].view(torch.int32)) == 0
