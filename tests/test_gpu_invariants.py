"""The method's own invariants, checked on the CUDA path through the C ABI.

Each case puts the recurrence (explainer page, "Gated DeltaNet" box: a gate
on the old memory, an erase along the key, a write of the value, a read with
the query) at a point where its result has a closed form, and compares the
kernels with that closed form as well as with the fp64 oracle:

* beta = 0 (nothing written): the state only decays, S_T = exp(sum g) S_0,
  and every read-out is o_t = exp(G_t) S_0 q_t;
* beta = 1 with unit keys and q = k: the write is exact, so the read-out
  along the key returns the value, o_t = S_t k_t = v_t (up to the rounding of
  the unit keys to the storage precision);
* alpha = 1 over four carried-state calls of 1024 tokens: no write is ever
  forgotten, so a state-carry error at a call boundary or a chunk range
  boundary cannot fade before the end;
* gates at the edge of the kernels' documented domain (the sum of g over a
  64-token chunk at -79).

Error metric as everywhere: max |x - ref| / max |ref|.  Bars: bf16 2e-2,
fp32 1e-4.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
import linear_attention_vlm_b200 as gdn

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def rel_err(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    scale = np.max(np.abs(ref))
    return float(np.max(np.abs(x - ref)) / (scale if scale > 0 else 1.0))


def np64(t):
    return None if t is None else t.detach().to("cpu", torch.float64).numpy()


def dev_inputs(inp, dev):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def run(inp, dev, cu=True):
    t = dev_inputs(inp, dev)
    out, st = gdn.gdn_prefill(t["q"], t["k"], t["v"], t["g"], t["beta"], t.get("state_in"),
                              t["cu_seqlens"] if cu else None,
                              num_seqs=None if cu else t["cu_seqlens"].numel() - 1)
    torch.cuda.synchronize()
    return np64(out), np64(st)


def oracle_run(inp):
    return oracle.prefill(np64(inp["q"]), np64(inp["k"]), np64(inp["v"]), np64(inp["g"]),
                          np64(inp["beta"]), np64(inp.get("state_in")),
                          inp["cu_seqlens"].numpy().astype(np.int64))


# (lengths, H, d, dtype, unpacked): the tensor-core path with one chunk range
# per sequence (packed), with sequence-parallel chunk ranges (one long
# unpacked sequence), and the fp32 path
CASES = [([200, 0, 130], 2, 128, torch.bfloat16, False),
         ([4096], 2, 128, torch.bfloat16, True),
         ([200, 77], 2, 64, torch.float32, False)]
IDS = ["tc-packed", "tc-ranges", "f32"]


@pytest.mark.parametrize("lens,H,d,dtype,unpacked", CASES, ids=IDS)
def test_beta_zero_only_decays(cuda_device, lens, H, d, dtype, unpacked):
    inp = W.random_prefill(lens, H=H, dk=d, dv=d, dtype=dtype, seed=31, state_std=0.5)
    inp["beta"].zero_()
    # milder gates, so that the decay over 4096 tokens (exp(sum g)) stays
    # inside the fp32 range the kernels keep the state in
    inp["g"].mul_(0.1)
    out, st = run(inp, cuda_device, cu=not unpacked)
    cu = inp["cu_seqlens"].numpy()
    g = np64(inp["g"])
    s0 = np64(inp["state_in"])
    q = np64(inp["q"])
    ref_o = np.zeros_like(out)
    ref_s = np.zeros_like(st)
    for n in range(len(lens)):
        a, b = cu[n], cu[n + 1]
        G = np.cumsum(g[a:b], axis=0)                            # [L, H]
        for h in range(H):
            ref_o[a:b, h] = np.exp(G[:, h])[:, None] * (q[a:b, h] @ s0[n, h].T)
            ref_s[n, h] = np.exp(G[-1, h] if b > a else 0.0) * s0[n, h]
    assert rel_err(st, ref_s) <= TOL[dtype]
    assert rel_err(out, ref_o) <= TOL[dtype]
    ro, rs = oracle_run(inp)
    assert rel_err(out, ro) <= TOL[dtype] and rel_err(st, rs) <= TOL[dtype]


@pytest.mark.parametrize("lens,H,d,dtype,unpacked", CASES, ids=IDS)
def test_beta_zero_alpha_one_keeps_state(cuda_device, lens, H, d, dtype, unpacked):
    inp = W.random_prefill(lens, H=H, dk=d, dv=d, dtype=dtype, seed=32, state_std=0.5)
    inp["beta"].zero_()
    inp["g"].zero_()
    out, st = run(inp, cuda_device, cu=not unpacked)
    s0 = np64(inp["state_in"])
    # nothing is written and nothing decays: the state comes back unchanged
    # (to the rounding of the start states the chunk ranges hand on)
    assert rel_err(st, s0) <= 1e-5
    cu = inp["cu_seqlens"].numpy()
    q = np64(inp["q"])
    ref_o = np.zeros_like(out)
    for n in range(len(lens)):
        for h in range(H):
            ref_o[cu[n]:cu[n + 1], h] = q[cu[n]:cu[n + 1], h] @ s0[n, h].T
    assert rel_err(out, ref_o) <= TOL[dtype]


@pytest.mark.parametrize("lens,H,d,dtype,unpacked", CASES, ids=IDS)
def test_beta_one_unit_keys_exact_write(cuda_device, lens, H, d, dtype, unpacked):
    inp = W.random_prefill(lens, H=H, dk=d, dv=d, dtype=dtype, seed=33, state_std=0.02)
    inp["beta"].fill_(1.0)
    inp["q"] = inp["k"].clone()          # read along the key just written
    out, st = run(inp, cuda_device, cu=not unpacked)
    # o_t = S_t k_t = v_t + (1 - |k_t|^2)(alpha_t S_{t-1} k_t - v_t): the keys
    # are unit vectors rounded to the storage precision
    k = np64(inp["k"])
    dev_norm = np.max(np.abs(np.sum(k * k, axis=-1) - 1.0)) if k.size else 0.0
    assert rel_err(out, np64(inp["v"])) <= TOL[dtype] + 4 * dev_norm
    ro, rs = oracle_run(inp)
    assert rel_err(out, ro) <= TOL[dtype] and rel_err(st, rs) <= TOL[dtype]


def test_alpha_one_carried_over_four_calls(cuda_device):
    """No decay: four calls of 1024 tokens with the state carried in place
    through state_in / state_out equal one oracle run over 4096 tokens."""
    H, T, calls = 4, 1024, 4
    inp = W.random_prefill([T * calls], H=H, dk=128, dv=128, dtype=torch.bfloat16, seed=34,
                           state_std=0.02)
    inp["g"].zero_()
    t = dev_inputs(inp, cuda_device)
    assert gdn.gdn_prefill_kernel_count(1, T, H, 128, 128, packed=False) == 4   # chunk ranges
    st = t["state_in"].clone()
    outs = []
    for c in range(calls):
        sl = slice(c * T, (c + 1) * T)
        o, st = gdn.gdn_prefill(t["q"][sl], t["k"][sl], t["v"][sl], t["g"][sl], t["beta"][sl], st, None,
                                state_out=st)
        outs.append(np64(o))
    torch.cuda.synchronize()
    ro, rs = oracle_run(inp)
    assert rel_err(np64(st), rs) <= 2e-2
    for c in range(calls):
        assert rel_err(outs[c], ro[c * T:(c + 1) * T]) <= 2e-2, c


@pytest.mark.parametrize("d,dtype", [(128, torch.bfloat16), (64, torch.float32)], ids=["tc", "f32"])
def test_gate_at_domain_edge(cuda_device, d, dtype):
    """Inside one chunk the gates add up to -79 (the kernels require the sum
    over any 64 consecutive tokens to stay above -80), so the chunkwise form
    meets exp(+-79); mild gates elsewhere."""
    T, H = 448, 2
    inp = W.random_prefill([T], H=H, dk=d, dv=d, dtype=dtype, seed=35, state_std=0.02)
    inp["g"][128:192] = -79.0 / 64.0      # the third chunk: cumulative gate -79 at its end
    inp["g"][300:364, 1] = -79.0 / 64.0   # a window straddling two chunks, one head
    ro, rs = oracle_run(inp)
    out, st = run(inp, cuda_device)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(st))
    assert rel_err(out, ro) <= TOL[dtype] and rel_err(st, rs) <= TOL[dtype]
