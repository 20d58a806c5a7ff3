"""Parity of the layer steps around the recurrence (gdn_preprocess,
gdn_output_gate, through the C ABI) with the fp64 oracle.

Bars (max |x - ref| / max |ref| per tensor): fp32 1e-4, bf16 2e-2, as for the
recurrence; the convolution state is moved, not computed, so it must match
bit for bit.  g and beta are fp32 outputs in both modes (1e-5).
"""
import numpy as np
import pytest
import torch

import oracle
import linear_attention_vlm_b200 as gdn

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def rel_err(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    scale = np.max(np.abs(ref)) if ref.size else 0.0
    return float(np.max(np.abs(x - ref)) / (scale if scale > 0 else 1.0)) if ref.size else 0.0


def np64(t):
    return None if t is None else t.detach().to("cpu", torch.float64).numpy()


def raw_inputs(lens, H, d, dtype, seed, state=True):
    """Synthetic raw projections: x ~ N(0, 1), conv taps ~ N(0, 0.5^2),
    a ~ N(3, 1) (alpha = sigmoid(a) near 0.95), b ~ N(0, 1)."""
    rng = np.random.default_rng(seed)
    T, N = int(sum(lens)), len(lens)
    x = [torch.from_numpy(rng.standard_normal((T, H, d)).astype(np.float32)).to(dtype) for _ in range(3)]
    w = torch.from_numpy((0.5 * rng.standard_normal((3, H, d, 4))).astype(np.float32))
    a = torch.from_numpy((3.0 + rng.standard_normal((T, H))).astype(np.float32))
    b = torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32))
    cs = torch.from_numpy(rng.standard_normal((N, 3, 3, H, d)).astype(np.float32)).to(dtype) if state else None
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    return x, w, a, b, cs, cu


def run_pre(x, w, a, b, cs, cu, dev, act, uniform_n=None):
    t = lambda y: None if y is None else y.to(dev)
    return gdn.gdn_preprocess(t(x[0]), t(x[1]), t(x[2]), t(w), t(a), t(b), t(cs),
                              None if uniform_n else t(cu), num_seqs=uniform_n, activation=act)


def check_pre(x, w, a, b, cs, cu, dev, act, dtype, uniform_n=None):
    got = run_pre(x, w, a, b, cs, cu, dev, act, uniform_n)
    torch.cuda.synchronize()
    ref = oracle.preprocess(np64(x[0]), np64(x[1]), np64(x[2]), np64(w), np64(a), np64(b),
                            cu.numpy().astype(np.int64), np64(cs), activation=act)
    for i, name in enumerate(("q", "k", "v")):
        e = rel_err(np64(got[i]), ref[i])
        assert e <= TOL[dtype], "%s err %.3g" % (name, e)
    assert rel_err(np64(got[3]), ref[3]) <= 1e-5
    assert rel_err(np64(got[4]), ref[4]) <= 1e-5
    # the state is data movement: bit for bit (the oracle's values are the
    # stored inputs widened to fp64, so narrowing them back is exact)
    assert torch.equal(got[5].cpu(), torch.from_numpy(ref[5]).to(dtype))
    return got


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("act", [gdn.ACT_NONE, gdn.ACT_SILU], ids=["none", "silu"])
@pytest.mark.parametrize("lens", [[1], [3], [64], [65], [0, 2, 130, 0, 71, 5], [200, 1]],
                         ids=lambda l: "lens" + "-".join(map(str, l)))
def test_preprocess_ragged(cuda_device, dtype, d, act, lens):
    x, w, a, b, cs, cu = raw_inputs(lens, 3, d, dtype, seed=sum(lens) + d + act)
    check_pre(x, w, a, b, cs, cu, cuda_device, act, dtype)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_preprocess_zero_state_and_uniform(cuda_device, dtype):
    x, w, a, b, _, cu = raw_inputs([96, 96, 96], 2, 128, dtype, seed=3, state=False)
    got = check_pre(x, w, a, b, None, cu, cuda_device, gdn.ACT_SILU, dtype)
    uni = run_pre(x, w, a, b, None, cu, cuda_device, gdn.ACT_SILU, uniform_n=3)
    torch.cuda.synchronize()
    for i in range(6):
        assert torch.equal(got[i], uni[i])


def test_preprocess_segmented_equals_whole(cuda_device):
    """Carrying the convolution state across segments gives the one-call
    result bit for bit (every token's sum is formed in the same order)."""
    x, w, a, b, cs, cu = raw_inputs([300], 2, 128, torch.bfloat16, seed=11)
    whole = run_pre(x, w, a, b, cs, cu, cuda_device, gdn.ACT_SILU)
    st = cs.to(cuda_device)
    parts = []
    for s0, s1 in ((0, 1), (1, 3), (3, 70), (70, 300)):
        seg = [xx[s0:s1] for xx in x]
        cu_s = torch.tensor([0, s1 - s0], dtype=torch.int32)
        out = gdn.gdn_preprocess(*(y.to(cuda_device) for y in seg), w.to(cuda_device), a[s0:s1].to(cuda_device),
                                 b[s0:s1].to(cuda_device), st, cu_s.to(cuda_device), activation=gdn.ACT_SILU,
                                 conv_state_out=st)                      # in place
        parts.append(out)
    torch.cuda.synchronize()
    for i in range(5):
        assert torch.equal(torch.cat([p[i] for p in parts]), whole[i]), i
    assert torch.equal(st, whole[5])


def test_preprocess_decode_tokens(cuda_device):
    """One token per sequence (the per-step use in decoding) with the state
    carried over 6 steps, against the oracle step by step."""
    B, H, d = 5, 4, 128
    x, w, a, b, cs, cu = raw_inputs([1] * B, H, d, torch.bfloat16, seed=21)
    st_dev = cs.to(cuda_device)
    st_ref = np64(cs)
    rng = np.random.default_rng(22)
    for step in range(6):
        xs = [torch.from_numpy(rng.standard_normal((B, H, d)).astype(np.float32)).to(torch.bfloat16) for _ in range(3)]
        got = gdn.gdn_preprocess(*(y.to(cuda_device) for y in xs), w.to(cuda_device), a.to(cuda_device),
                                 b.to(cuda_device), st_dev, cu.to(cuda_device), conv_state_out=st_dev)
        torch.cuda.synchronize()
        ref = oracle.preprocess(*(np64(y) for y in xs), np64(w), np64(a), np64(b), cu.numpy().astype(np.int64),
                                st_ref)
        st_ref = ref[5]
        for i in range(3):
            assert rel_err(np64(got[i]), ref[i]) <= 2e-2, (step, i)
        assert torch.equal(st_dev.cpu(), torch.from_numpy(st_ref).to(torch.bfloat16))


def test_preprocess_full_size(cuda_device):
    """The prefill workload's shape: 8192 tokens x 16 heads x 128."""
    x, w, a, b, cs, cu = raw_inputs([8192], 16, 128, torch.bfloat16, seed=5, state=False)
    check_pre(x, w, a, b, None, cu, cuda_device, gdn.ACT_NONE, torch.bfloat16)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("dv", [64, 128])
@pytest.mark.parametrize("norm", [False, True], ids=["plain", "rmsnorm"])
@pytest.mark.parametrize("gate", [gdn.GATE_SIGMOID, gdn.GATE_SILU], ids=["sigmoid", "silu"])
def test_output_gate(cuda_device, dtype, dv, norm, gate):
    rng = np.random.default_rng(dv + 2 * norm + gate)
    T, H = 77, 3
    o = torch.from_numpy(rng.standard_normal((T, H, dv)).astype(np.float32)).to(dtype)
    z = torch.from_numpy((2 * rng.standard_normal((T, H, dv))).astype(np.float32)).to(dtype)
    w = torch.from_numpy(rng.uniform(0.5, 1.5, dv).astype(np.float32)) if norm else None
    y = gdn.gdn_output_gate(o.to(cuda_device), z.to(cuda_device), None if w is None else w.to(cuda_device),
                            gate=gate)
    torch.cuda.synchronize()
    ref = oracle.output_gate(np64(o), np64(z), None if w is None else np64(w), gate=gate)
    assert rel_err(np64(y), ref) <= TOL[dtype]
    od = o.to(cuda_device)
    y2 = gdn.gdn_output_gate(od, z.to(cuda_device), None if w is None else w.to(cuda_device), gate=gate, out=od)
    torch.cuda.synchronize()
    assert y2.data_ptr() == od.data_ptr() and torch.equal(y2, y)   # in place
