"""The streaming session (gdn_session_*, through the C ABI): a layer step
-- pre-processing, the recurrence with a carried state, the output gate --
replayed as a CUDA graph per token count, against the fp64 oracle composed
step by step with its states carried, and against the same steps launched
without a graph (bit for bit)."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
import linear_attention_vlm_b200 as gdn

pytestmark = pytest.mark.gpu


def rel_err(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(x - ref)) / max(np.max(np.abs(ref)), 1e-30))


def np64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def _steps(B, H, d, seg, seed):
    """Full segment, full segment, partial segment, then decode tokens."""
    out = []
    for i, n in enumerate([seg, seg, seg // 3 + 1, 1, 1, 1]):
        L = W.layer_inputs(B * n, H, d, torch.bfloat16, seed=seed + i)
        out.append((n, L))
    return out


def test_session_matches_the_oracle_step_by_step(cuda_device):
    B, H, d, seg = 2, 4, 128, 150
    P = W.layer_inputs(1, H, d, torch.float32, seed=99)
    sess = gdn.GdnSession(B, H, d, seg, P["conv_w"].to(cuda_device), P["norm_w"].to(cuda_device),
                          activation=gdn.ACT_SILU, gate=gdn.GATE_SIGMOID)
    st = np.zeros((B, H, d, d))
    cs = np.zeros((B, 3, 3, H, d))
    for n, L in _steps(B, H, d, seg, seed=10):
        x = {k: v.to(cuda_device) for k, v in L.items()}
        if n == 1:
            for dst, src in ((sess.xq, x["xq"]), (sess.xk, x["xk"]), (sess.xv, x["xv"]), (sess.a, x["a"]),
                             (sess.b, x["b"]), (sess.z, x["z"])):
                dst[:B].copy_(src)
            y = sess.decode()
        else:
            y = sess.feed(x["xq"], x["xk"], x["xv"], x["a"], x["b"], x["z"])
        torch.cuda.synchronize()
        cu = np.arange(B + 1, dtype=np.int64) * n
        q, k, v, g, beta, cs = oracle.preprocess(np64(L["xq"]), np64(L["xk"]), np64(L["xv"]), np64(P["conv_w"]),
                                                 np64(L["a"]), np64(L["b"]), cu, cs, activation=oracle.ACT_SILU)
        if n == 1:
            o, st = oracle.decode_step(q, k, v, g, beta, st)
        else:
            o, st = oracle.prefill(q, k, v, g, beta, st, cu)
        ref = oracle.output_gate(o, np64(L["z"]), np64(P["norm_w"]))
        assert rel_err(np64(y), ref) <= 2e-2, n
    assert rel_err(np64(sess.state), st) <= 2e-2
    assert torch.equal(sess.conv_state.cpu(), torch.from_numpy(cs).to(torch.bfloat16))
    assert sess.graph_count() == 3          # full segment, partial segment, decode step
    sess.close()


def test_graph_replay_equals_eager_launches(cuda_device):
    B, H, d, seg = 1, 16, 128, 274           # the pages' ~274 tokens per frame, 16 heads
    P = W.layer_inputs(1, H, d, torch.float32, seed=7)
    mk = lambda: gdn.GdnSession(B, H, d, seg, P["conv_w"].to(cuda_device), P["norm_w"].to(cuda_device),
                                activation=gdn.ACT_SILU)
    sg, se = mk(), mk()
    for n, L in _steps(B, H, d, seg, seed=30):
        x = {k: v.to(cuda_device) for k, v in L.items()}
        yg = sg.feed(x["xq"], x["xk"], x["xv"], x["a"], x["b"], x["z"]).clone()
        ye = se.feed(x["xq"], x["xk"], x["xv"], x["a"], x["b"], x["z"], eager=True).clone()
        torch.cuda.synchronize()
        assert torch.equal(yg, ye), n
    assert torch.equal(sg.state, se.state) and torch.equal(sg.conv_state, se.conv_state)
    assert sg.graph_count() == 3 and se.graph_count() == 0
