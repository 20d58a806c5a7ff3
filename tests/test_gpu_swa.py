"""Parity of the sliding-window attention layer (gdn_rope,
gdn_swa_attention, through the C ABI) with the fp64 oracle.

Bars (bf16 keeps 8 significant bits: rounding is off by at most 2^-8
relative, one ulp is at most 2^-7 relative).  RoPE: fp32 |x - ref| <= 1e-5
(the angle is reduced in double, the sine and cosine are fp32); bf16 within
one ulp, 2^-7 |ref|, which leaves the fp32 arithmetic before the rounding a
margin.  Attention (bf16 in and out): |o - ref| <= 2^-8 |ref| + 2^-8 max|v|
per element: the first term is the rounding of o, the second bounds the
rounding of the probabilities (each off by at most 2^-8 relative) in a
weighted mean of values no larger than max|v|; the rms error must also stay
below 2^-8 of the rms output.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import linear_attention_vlm_b200 as gdn

pytestmark = pytest.mark.gpu

DEV = "cuda"


def np64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def cu_of(lens):
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)


def check_attn(got, ref, v, rows=None):
    got = np64(got)
    if rows is not None:
        got, ref = got[rows], ref[rows]
    vmax = float(np.max(np.abs(np64(v))))
    err = np.abs(got - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -8 * vmax
    worst = float(np.max(err - bound))
    assert worst <= 0.0, "max excess %.3g (max err %.3g)" % (worst, float(np.max(err)))
    # and the typical error is far below the bound
    assert float(np.sqrt(np.mean(err ** 2))) <= 2.0 ** -8 * max(1.0, float(np.sqrt(np.mean(ref ** 2))))


def run_attn(x, lens, window, uniform_n=None, scale=None):
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    cu = None if uniform_n else torch.tensor(cu_of(lens), dtype=torch.int32, device=DEV)
    o = gdn.gdn_swa_attention(x["q"].to(DEV), x["k"].to(DEV), x["v"].to(DEV), cu, num_seqs=uniform_n,
                              window=window, scale=scale, status=status)
    assert gdn.gdn_read_status(status) == 0   # no wait inside the kernel gave up
    return o


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("offset", [0, 123457])
def test_rope_matches_oracle(dtype, d, offset):
    lens = [1, 200, 0, 57, 1000]
    T, H = sum(lens), 3
    x = workloads.attention_inputs(T, Hq=H, Hkv=1, d=d, dtype=dtype, seed=d + offset)["q"]
    cu = cu_of(lens)
    got = gdn.gdn_rope(x.to(DEV), torch.tensor(cu, dtype=torch.int32, device=DEV), offset=offset)
    torch.cuda.synchronize()
    ref = oracle.rope(np64(x), oracle.rope_positions(cu, T, offset))
    err = np.abs(np64(got) - ref)
    if dtype == torch.float32:
        assert float(err.max()) <= 1e-5
    else:
        assert np.all(err <= 2.0 ** -7 * np.abs(ref) + 1e-6)


def test_rope_in_place_and_uniform():
    T, H, d = 512, 2, 128
    x = workloads.attention_inputs(T, Hq=H, Hkv=1, d=d, dtype=torch.bfloat16, seed=3)["q"]
    xd = x.to(DEV)
    a = gdn.gdn_rope(xd, num_seqs=4, base=500000.0)
    gdn.gdn_rope(xd, num_seqs=4, base=500000.0, out=xd)
    torch.cuda.synchronize()
    assert torch.equal(a, xd)
    ref = oracle.rope(np64(x), oracle.rope_positions(cu_of([128] * 4), T), base=500000.0)
    assert np.all(np.abs(np64(a) - ref) <= 2.0 ** -7 * np.abs(ref) + 1e-6)


@pytest.mark.parametrize("window", [1, 7, 64, 130, 300, 8192])
def test_attention_ragged_sequences(window):
    # sequences shorter and longer than a 128-token tile, an empty one, tiles
    # that straddle sequence starts
    lens = [1, 127, 0, 128, 129, 300, 45, 500]
    T = sum(lens)
    x = workloads.attention_inputs(T, Hq=4, Hkv=2, d=128, seed=window)
    o = run_attn(x, lens, window)
    ref = oracle.swa_attention(np64(x["q"]), np64(x["k"]), np64(x["v"]), cu_of(lens), window=window)
    check_attn(o, ref, x["v"])


@pytest.mark.parametrize("q_scale", [4.0, 12.0])
def test_attention_sharp_scores(q_scale):
    # score spread large enough that the running maximum moves by more than
    # the rescale threshold between key blocks
    lens = [700, 333]
    T = sum(lens)
    x = workloads.attention_inputs(T, Hq=2, Hkv=1, d=128, seed=11, q_scale=q_scale)
    # keys grow along the sequence, so later blocks raise the maximum
    ramp = torch.linspace(0.5, 3.0, T).view(T, 1, 1)
    x["k"] = (x["k"].float() * ramp).to(torch.bfloat16)
    o = run_attn(x, lens, 600)
    ref = oracle.swa_attention(np64(x["q"]), np64(x["k"]), np64(x["v"]), cu_of(lens), window=600)
    check_attn(o, ref, x["v"])


def test_attention_uniform_split_groups_and_scale():
    T, N = 1024, 4
    x = workloads.attention_inputs(T, Hq=8, Hkv=1, d=128, seed=5)
    o = run_attn(x, [T // N] * N, 100, uniform_n=N, scale=0.05)
    ref = oracle.swa_attention(np64(x["q"]), np64(x["k"]), np64(x["v"]), cu_of([T // N] * N), window=100, scale=0.05)
    check_attn(o, ref, x["v"])


def test_rope_then_attention_layer():
    lens = [384, 257]
    T = sum(lens)
    x = workloads.attention_inputs(T, Hq=4, Hkv=2, d=128, seed=21)
    cu = torch.tensor(cu_of(lens), dtype=torch.int32, device=DEV)
    q = gdn.gdn_rope(x["q"].to(DEV), cu, offset=10)
    k = gdn.gdn_rope(x["k"].to(DEV), cu, offset=10)
    o = gdn.gdn_swa_attention(q, k, x["v"].to(DEV), cu, window=200)
    torch.cuda.synchronize()
    pos = oracle.rope_positions(cu_of(lens), T, 10)
    # the oracle attends over the rotated values the kernels stored (bf16)
    qr, kr = oracle.rope(np64(x["q"]), pos), oracle.rope(np64(x["k"]), pos)
    assert np.all(np.abs(np64(q) - qr) <= 2.0 ** -7 * np.abs(qr) + 1e-6)
    ref = oracle.swa_attention(np64(q), np64(k), np64(x["v"]), cu_of(lens), window=200)
    check_attn(o, ref, x["v"])


def test_attention_full_size_sampled_rows():
    # the benchmark's layer: 32768 tokens, 16/2 heads, window 8192; rows at
    # tile edges, around the window length and at the end
    T = 32768
    x = workloads.attention_inputs(T, seed=0)
    o = run_attn(x, [T], workloads.SWA_WINDOW)
    rows = [0, 1, 127, 128, 4095, 8190, 8191, 8192, 8193, 12345, 16383, 16384, 30000, 32766, 32767]
    ref = oracle.swa_attention(np64(x["q"]), np64(x["k"]), np64(x["v"]), None, window=workloads.SWA_WINDOW,
                               rows=rows)
    check_attn(o, ref, x["v"], rows=rows)


def test_attention_packed_long_sequences_sampled_rows():
    # three packed sequences (32768 tokens in all), window 8192: rows on both
    # sides of each sequence start, at the window length and at the ends
    lens = [5000, 20000, 7768]
    T = sum(lens)
    x = workloads.attention_inputs(T, seed=3)
    o = run_attn(x, lens, workloads.SWA_WINDOW)
    rows = [0, 4999, 5000, 5001, 5127, 5128, 13191, 13192, 13193, 24999, 25000, 25001, 25100, 32767]
    ref = oracle.swa_attention(np64(x["q"]), np64(x["k"]), np64(x["v"]), cu_of(lens), window=workloads.SWA_WINDOW,
                               rows=rows)
    check_attn(o, ref, x["v"], rows=rows)


def test_attention_without_grouping():
    lens = [260, 3]
    T = sum(lens)
    x = workloads.attention_inputs(T, Hq=3, Hkv=3, d=128, seed=8)
    o = run_attn(x, lens, 130)
    ref = oracle.swa_attention(np64(x["q"]), np64(x["k"]), np64(x["v"]), cu_of(lens), window=130)
    check_attn(o, ref, x["v"])
