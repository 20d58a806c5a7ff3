#!/usr/bin/env python
"""Benchmark of the Gated DeltaNet hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

One step = one gdn_prefill call over the bf16 prefill workload (1 sequence,
16 heads, 8192 tokens, d_k = d_v = 128, chunk 64, zero initial state) with
its inputs resident in HBM.  The L2 (126 MB) is flushed before every step by
writing a 512 MiB buffer; only the prefill launches are inside the CUDA-event
intervals.  The same run times every other workload of the method, one JSON
object each:

  long_prefill   262144 tokens x 16 heads, one call and 64 carried-state
                 calls of 4096 tokens (inputs of 3.2 GB: larger than L2)
  varlen         8 packed sequences of 1024..32768 tokens with their own
                 initial states (inputs larger than L2)
  decode         64 sequences x 16 heads, 1024 one-token steps captured in
                 one CUDA graph; the state ping-pongs between two buffers
                 (128 MiB, larger than L2) so every step streams it from HBM;
                 decode_inplace is the same graph updating one 64 MiB state
  e2e            the prefill through the public API with pinned host buffers
                 (inputs copied in and out, result read back, all timed)

plus the layer steps around the recurrence, the streaming session and the
sliding-window attention layer of the hybrid block.

Multi-GPU (torchrun): every rank runs its own replica of the workload (the
units are independent sequences; there is no data-path collective); the
reported time is the max over ranks and ``value`` counts the tokens of all
ranks ("scaling": "weak").

``--impl reference`` times the fp64 CPU oracle (the only other implementation
of the method) on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 512 << 20

PREFILL = W.WORKLOADS["prefill_bf16"]
ALL_LEGS = ("prefill", "long_prefill", "varlen", "decode", "e2e", "layer", "streaming", "swa")
DECODE = W.WORKLOADS["decode_bf16"]


def peaks():
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ algorithmic work

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per call or
# launch, measured by ncu and recorded in profiles/dram_traffic.txt together
# with a hash of the kernel's sources at the time of the capture: its .cu file
# and the headers whose device code it uses (the decode kernel takes only the
# dtype conversions from gdn_internal.h).  A figure whose sources have changed
# since is not reported (traffic: null).
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.txt")
_CSRC = os.path.join("linear_attention_vlm_b200", "csrc")
KERNEL_SOURCES = {
    "prefill": [os.path.join(_CSRC, f) for f in ("prefill_tc.cu", "prefill_tc.h", "sm100.cuh", "gdn_internal.h")],
    "swa": [os.path.join(_CSRC, f) for f in ("swa.cu", "sm100.cuh", "gdn_internal.h")],
    "decode": [os.path.join(_CSRC, "decode.cu")],
    "layer": [os.path.join(_CSRC, f) for f in ("layer_ops.cu", "gdn_internal.h")],
}


def source_hash(kind):
    """First 16 hex digits of the SHA-256 of a kernel family's sources."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kind]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic(key, kind):
    """Recorded DRAM bytes for `key`, or None if absent or stale."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    want = source_hash(kind)
    with open(TRAFFIC_FILE) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 3 and not line.startswith("#") and parts[0] == key:
                return float(parts[2]) if parts[1] == want else None
    return None


def prefill_bytes(T, H, dk, dv, num_seqs, with_state_in, elem=2):
    """Bytes the prefill must move at minimum: q, k, v, g, beta in; out and
    the final state out (and the initial state in, when given)."""
    per_tok_head = (2 * dk + dv) * elem + 2 * 4 + dv * elem
    state = num_seqs * H * dv * dk * 4
    return T * H * per_tok_head + state * (2 if with_state_in else 1)


def prefill_flops(T, H, d, C=64):
    """Algorithmic flops per token-head of the chunkwise form (triangles
    counted once): intra-chunk 5 C d, state 6 d^2, solve C^2 / 3."""
    return T * H * (5 * C * d + 6 * d * d + C * C / 3.0)


def swa_attention_flops(T, Hq, d, window):
    """2 d multiply-adds for q.k and 2 d for p v per (query, visible key,
    head); one sequence of T tokens."""
    w = min(window, T)
    pairs = w * (w + 1) // 2 + (T - w) * w
    return 4 * d * Hq * pairs


def decode_bytes(B, H, dk, dv, elem=2):
    return B * H * (2 * dv * dk * 4 + (2 * dk + dv) * elem + 8 + dv * elem)


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi sampling during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.idx)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            p = [x.strip() for x in ln.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                mx.append(float(p[2]))
            except ValueError:
                continue
            for n, val in zip(names, p[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ distributed

def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    if world != n_gpus:
        print("warning: --gpus %d but WORLD_SIZE %d" % (n_gpus, world), file=sys.stderr)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world, device=None):
    """Max of a per-rank scalar over all ranks (the slowest rank's time)."""
    if world == 1:
        return x
    import torch.distributed as dist
    if device is None:
        device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(units_per_rank, world, ms_max):
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's time (independent replicas, weak scaling)."""
    return units_per_rank * world / (ms_max * 1e-3)


# ------------------------------------------------------------------ native arm

def run_native(args):
    import linear_attention_vlm_b200 as gdn

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    pk, pk_kind = peaks()
    hbm = pk["hbm_gbs"]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    launches = {}   # leg -> kernel launches inside its timed region
    legs = set(args.legs.split(",")) if args.legs else set(ALL_LEGS)
    want = lambda leg: leg in legs

    def hbm_roofline(kernel, nbytes, ms, traffic=None, **extra):
        gbs = nbytes / (ms * 1e-3) / 1e9
        r = {"kernel": kernel, "bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
             "frac": gbs / hbm, "traffic": traffic, "peak_source": pk_kind, "algorithmic_bytes": nbytes}
        r.update(extra)
        return r

    # ---- prefill inputs (seed per rank: independent replicas)
    w = PREFILL
    host = W.prefill_inputs(w, seed=rank)
    T, H, dk, dv = w.T, w.H, w.dk, w.dv
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in host.items()}
    out = torch.empty((T, H, dv), dtype=w.dtype, device=dev)
    st_out = torch.empty((1, H, dv, dk), dtype=torch.float32, device=dev)
    ws_bytes = gdn.gdn_prefill_workspace_size(1, T, H, dk, dv, w.chunk, w.dtype)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    launches_per_prefill = gdn.gdn_prefill_kernel_count(1, T, H, dk, dv, w.chunk, w.dtype, packed=False)

    def prefill_once():
        gdn.gdn_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], None, None, out=out,
                        state_out=st_out, workspace=ws)

    # ---- long prefill: 262144 tokens, one call and 64 carried-state segments
    lw = W.WORKLOADS["long_prefill_bf16"]
    if not want("long_prefill"):
        lw = dataclasses.replace(lw, T=lw.segments * 64)   # a token-sized stand-in, never timed
    lx = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v)
          for k, v in W.prefill_inputs(lw, seed=rank).items()}
    LT = lw.T
    l_out = torch.empty((LT, H, dv), dtype=lw.dtype, device=dev)
    l_st = torch.empty((1, H, dv, dk), dtype=torch.float32, device=dev)
    l_ws = torch.empty(max(gdn.gdn_prefill_workspace_size(1, LT, H, dk, dv), 16), dtype=torch.uint8, device=dev)
    seg = LT // lw.segments
    s_ws = torch.empty(max(gdn.gdn_prefill_workspace_size(1, seg, H, dk, dv), 16), dtype=torch.uint8, device=dev)
    l_launch_whole = gdn.gdn_prefill_kernel_count(1, LT, H, dk, dv, packed=False)
    l_launch_seg = gdn.gdn_prefill_kernel_count(1, seg, H, dk, dv, packed=False) * lw.segments

    def long_whole_once():
        gdn.gdn_prefill(lx["q"], lx["k"], lx["v"], lx["g"], lx["beta"], None, None, out=l_out,
                        state_out=l_st, workspace=l_ws)

    def long_segmented_once():
        l_st.zero_()
        for s0 in range(0, LT, seg):
            sl = slice(s0, s0 + seg)
            gdn.gdn_prefill(lx["q"][sl], lx["k"][sl], lx["v"][sl], lx["g"][sl], lx["beta"][sl], l_st, None,
                            out=l_out[sl], state_out=l_st, workspace=s_ws)

    # ---- varlen: 8 packed sequences, per-sequence initial states
    vw = W.WORKLOADS["varlen_bf16"]
    if not want("varlen"):
        vw = dataclasses.replace(vw, varlen=(2, 64, 64))
    vx = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v)
          for k, v in W.prefill_inputs(vw, seed=rank).items()}
    VT = int(vx["q"].shape[0])
    VN = vx["cu_seqlens"].numel() - 1
    v_out = torch.empty((VT, H, dv), dtype=vw.dtype, device=dev)
    v_st = torch.empty((VN, H, dv, dk), dtype=torch.float32, device=dev)
    v_ws = torch.empty(max(gdn.gdn_prefill_workspace_size(VN, VT, H, dk, dv), 16), dtype=torch.uint8, device=dev)
    v_launch = gdn.gdn_prefill_kernel_count(VN, VT, H, dk, dv, packed=True)

    def varlen_once():
        gdn.gdn_prefill(vx["q"], vx["k"], vx["v"], vx["g"], vx["beta"], vx["state_in"], vx["cu_seqlens"],
                        out=v_out, state_out=v_st, workspace=v_ws)

    # ---- decode: 1024 one-token steps of 64 sequences x 16 heads in one CUDA graph
    dw = DECODE
    nsteps = dw.steps if want("decode") else 2
    steps_host = [W.decode_tokens(dw, i, seed=rank) for i in range(nsteps)]
    tok = {k: torch.stack([x[k] for x in steps_host]).to(dev) for k in ("q", "k", "v", "g", "beta")}
    del steps_host
    S0 = W.decode_state(dw, seed=rank).to(dev)
    S_a, S_b = S0.clone(), torch.empty_like(S0)
    dout = torch.empty((nsteps, dw.num_seqs, dw.H, dw.dv), dtype=dw.dtype, device=dev)

    def decode_steps(pingpong):
        for i in range(nsteps):
            src = S_a if (not pingpong or i % 2 == 0) else S_b
            dst = S_a if not pingpong else (S_b if i % 2 == 0 else S_a)
            gdn.gdn_decode_step(tok["q"][i], tok["k"][i], tok["v"][i], tok["g"][i], tok["beta"][i], src, dst,
                                out=dout[i])

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream(dev)
        s.wait_stream(stream)
        with torch.cuda.stream(s):
            fn()   # warm-up outside the capture (one-time set-up of the kernels)
        stream.wait_stream(s)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            fn()
        torch.cuda.synchronize()
        return g

    graph_pp = capture(lambda: decode_steps(True))
    graph_ip = capture(lambda: decode_steps(False))

    # ---- layer steps around the recurrence, on the prefill shapes
    lay = {k: v.to(dev) for k, v in W.layer_inputs(T, H, dk, w.dtype, seed=rank).items()}
    gate_out = torch.empty_like(lay["z"])

    def preprocess_once():
        gdn.gdn_preprocess(lay["xq"], lay["xk"], lay["xv"], lay["conv_w"], lay["a"], lay["b"], None, None,
                           activation=gdn.ACT_SILU, want_state=False)

    def gate_once():
        gdn.gdn_output_gate(out, lay["z"], lay["norm_w"], gate=gdn.GATE_SIGMOID, out=gate_out)

    # the whole token mixer of one layer: one fused call, and the three calls
    lay_state = torch.zeros((1, H, dv, dk), dtype=torch.float32, device=dev)
    lay_ws = torch.empty(gdn.gdn_layer_prefill_workspace_size(1, T, H, dk, w.dtype), dtype=torch.uint8, device=dev)

    def layer_fused_once():
        gdn.gdn_layer_prefill(lay["xq"], lay["xk"], lay["xv"], lay["conv_w"], lay["a"], lay["b"], lay["z"], None, None,
                              lay["norm_w"], activation=gdn.ACT_SILU, gate=gdn.GATE_SIGMOID, y=gate_out,
                              state_out=lay_state, workspace=lay_ws, want_conv_state=False)

    def layer_unfused_once():
        q_, k_, v_, g_, b_, _ = gdn.gdn_preprocess(lay["xq"], lay["xk"], lay["xv"], lay["conv_w"], lay["a"], lay["b"],
                                                   None, None, activation=gdn.ACT_SILU, want_state=False)
        gdn.gdn_prefill(q_, k_, v_, g_, b_, None, out=out, state_out=lay_state, workspace=ws)
        gdn.gdn_output_gate(out, lay["z"], lay["norm_w"], gate=gdn.GATE_SIGMOID, out=gate_out)

    # ---- streaming session: one GDN layer step per video frame (~274 tokens per
    # frame in the pages' streaming measurement), state carried, graph replay
    FRAME = 274
    P = W.layer_inputs(FRAME, H, dk, w.dtype, seed=rank)
    sess = gdn.GdnSession(1, H, dk, FRAME, P["conv_w"].to(dev), P["norm_w"].to(dev), dtype=w.dtype,
                          activation=gdn.ACT_SILU)
    for name in ("xq", "xk", "xv", "a", "b", "z"):
        getattr(sess, name)[:FRAME].copy_(P[name].to(dev))
    # a frame: the fused layer call's kernels + the convolution-state update
    frame_launches = gdn.gdn_prefill_kernel_count(1, FRAME, H, dk, dv, w.chunk, w.dtype) + 1
    decode_launches = 2 + 1 + 1

    # ---- sliding-window attention layer of the hybrid block: RoPE on q and k,
    # then causal attention over an 8K window with 16 query / 2 key-value heads
    SWA_T = 32768 if want("swa") else 256
    ax = {k: v.to(dev) for k, v in W.attention_inputs(SWA_T, seed=rank).items()}
    swa_q, swa_k = torch.empty_like(ax["q"]), torch.empty_like(ax["k"])
    swa_o = torch.empty_like(ax["q"])

    def swa_attn_once():
        gdn.gdn_swa_attention(swa_q, swa_k, ax["v"], window=W.SWA_WINDOW, out=swa_o)

    def swa_layer_once():
        gdn.gdn_rope(ax["q"], out=swa_q)
        gdn.gdn_rope(ax["k"], out=swa_k)
        swa_attn_once()

    # ---- e2e buffers (pinned host, fresh device copies each step)
    pin = {k: v.pin_memory() for k, v in host.items() if isinstance(v, torch.Tensor) and k != "cu_seqlens"}
    out_h = torch.empty((T, H, dv), dtype=w.dtype).pin_memory()
    st_h = torch.empty((1, H, dv, dk), dtype=torch.float32).pin_memory()
    dbuf = {k: torch.empty_like(v, device=dev) for k, v in pin.items()}
    h2d = sum(v.numel() * v.element_size() for v in pin.values())
    d2h = out_h.numel() * out_h.element_size() + st_h.numel() * st_h.element_size()

    def e2e_once():
        for k, v in pin.items():
            dbuf[k].copy_(v, non_blocking=True)
        o, s = gdn.gdn_prefill(dbuf["q"], dbuf["k"], dbuf["v"], dbuf["g"], dbuf["beta"], None,
                               None, out=out, state_out=st_out, workspace=ws)
        out_h.copy_(o, non_blocking=True)
        st_h.copy_(s, non_blocking=True)

    # ---- warm-up
    for i in range(args.warmup):
        if want("prefill"):
            prefill_once()
        if want("long_prefill"):
            long_whole_once()
            long_segmented_once()
        if want("varlen"):
            varlen_once()
        if want("decode"):
            graph_pp.replay()
            graph_ip.replay()
        if want("e2e"):
            e2e_once()
        if want("layer"):
            preprocess_once()
            gate_once()
            layer_fused_once()
            layer_unfused_once()
        if want("streaming"):
            sess.prefill(FRAME)
            sess.prefill(FRAME, eager=True)
            sess.decode()
        if want("swa"):
            swa_layer_once()
    torch.cuda.synchronize()

    def timed(fn, steps, do_flush=True, reduce="mean"):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        barrier(world)
        torch.cuda.synchronize()
        for i in range(steps):
            if do_flush:
                flush.zero_()
            evs[i][0].record(stream)
            fn(i)
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        barrier(world)
        ms = [a.elapsed_time(b) for a, b in evs]
        return statistics.median(ms) if reduce == "median" else sum(ms) / len(ms)

    K = args.steps
    KL = max(3, min(K, 10))          # repeats of the long legs (milliseconds each)
    KG = max(20, min(K, 20))         # graph replays of the 1024 decode steps (median)
    ms = {}
    nan = float("nan")
    with ClockSampler(local) as clk:
        t_wall0 = time.time()
        if want("prefill"):
            ms["prefill"] = timed(lambda i: prefill_once(), K)
            launches["prefill"] = K * launches_per_prefill
        if want("long_prefill"):
            ms["long"] = timed(lambda i: long_whole_once(), KL, do_flush=False)
            launches["long"] = KL * l_launch_whole
            ms["long_seg"] = timed(lambda i: long_segmented_once(), KL, do_flush=False)
            launches["long_seg"] = KL * l_launch_seg
        if want("varlen"):
            ms["varlen"] = timed(lambda i: varlen_once(), KL, do_flush=False)
            launches["varlen"] = KL * v_launch
        if want("decode"):
            ms["dec_pp"] = timed(lambda i: graph_pp.replay(), KG, do_flush=False, reduce="median")
            ms["dec_ip"] = timed(lambda i: graph_ip.replay(), KG, do_flush=False, reduce="median")
            launches["decode"] = 2 * KG * nsteps
        if want("e2e"):
            KE = max(3, K // 10)
            ms["e2e"] = timed(lambda i: e2e_once(), KE, do_flush=False)
            launches["e2e"] = KE * launches_per_prefill
        if want("layer"):
            ms["pre"] = timed(lambda i: preprocess_once(), K)
            ms["gate"] = timed(lambda i: gate_once(), K)
            ms["layer_fused"] = timed(lambda i: layer_fused_once(), K)
            ms["layer_unfused"] = timed(lambda i: layer_unfused_once(), K)
            launches["layer"] = 2 * K + K + K * launches_per_prefill + K * (2 + launches_per_prefill)
        if want("streaming"):
            ms["frame_graph"] = timed(lambda i: sess.prefill(FRAME), K)
            ms["frame_eager"] = timed(lambda i: sess.prefill(FRAME, eager=True), K)
            ms["dec_graph"] = timed(lambda i: sess.decode(), K)
            launches["session"] = 2 * K * frame_launches + K * decode_launches
        if want("swa"):
            ms["swa_attn"] = timed(lambda i: swa_attn_once(), K)
            ms["swa_layer"] = timed(lambda i: swa_layer_once(), K)
            launches["swa"] = K + 3 * K
        wall = time.time() - t_wall0
    keys = ("prefill", "long", "long_seg", "varlen", "dec_pp", "dec_ip", "e2e", "pre", "gate",
            "frame_graph", "frame_eager", "dec_graph", "swa_attn", "swa_layer", "layer_fused", "layer_unfused")
    (ms_prefill, ms_long, ms_long_seg, ms_varlen, ms_dec_pp, ms_dec_ip, ms_e2e, ms_pre, ms_gate,
     ms_frame_graph, ms_frame_eager, ms_dec_graph, ms_swa_attn, ms_swa_layer, ms_layer_fused, ms_layer_unfused) = (
        max_over_ranks(ms.get(k, nan), world) for k in keys)
    swa_flops = swa_attention_flops(SWA_T, W.SWA_HQ, W.SWA_D, W.SWA_WINDOW)
    swa_tf = swa_flops / (ms_swa_attn * 1e-3) / 1e12
    el = 2 if w.dtype == torch.bfloat16 else 4
    pre_bytes = 6 * T * H * dk * el + 4 * T * H * 4 + 3 * H * dk * 16    # x in, q/k/v out, a/b in, g/beta out, taps
    gate_bytes = 3 * T * H * dv * el + dv * 4                             # o, z in, y out, norm weight

    value = aggregate_throughput(T, world, ms_prefill)
    pbytes = prefill_bytes(T, H, dk, dv, 1, with_state_in=False)
    pflops = prefill_flops(T, H, dk)
    lbytes = prefill_bytes(LT, H, dk, dv, 1, with_state_in=False)
    lseg_bytes = (prefill_bytes(seg, H, dk, dv, 1, with_state_in=True)) * lw.segments
    vbytes = prefill_bytes(VT, H, dk, dv, VN, with_state_in=True)
    dbytes = decode_bytes(dw.num_seqs, dw.H, dw.dk, dw.dv) * nsteps
    tensor_frac = lambda flops, ms: (flops / (ms * 1e-3) / 1e12) / pk["bf16_tflops"]
    prefill_kernel = "gdn_prefill (all %d launches of one call)"
    line = {
        "metric": "GDN prefill tokens/s and decode tokens/s on 1 B200; % of TC / HBM roofline",
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": ms_prefill,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; q,k L2-normalised N(0,1), v N(0,1), beta=sigmoid(N(0,1)), "
                "log alpha=-0.05 softplus(N(0,1)))",
        "config": {"workload": "prefill_bf16: B=1, H=16, T=8192, d_k=d_v=128, chunk=64, "
                               "zero initial state, fp32 state",
                   "global_batch": world, "seq_len": T, "heads": H, "head_dim": dk,
                   "parallelism": "replicas x%d (independent sequences)" % world,
                   "l2": "flushed before every step (512 MiB write)"},
        "roofline": hbm_roofline(prefill_kernel % launches_per_prefill, pbytes, ms_prefill,
                                 traffic=measured_traffic("prefill_bf16_call", "prefill"),
                                 traffic_note="ncu dram bytes of one call's launches, each from a cold L2",
                                 algorithmic_flops=pflops, tensor_frac=tensor_frac(pflops, ms_prefill)),
        "long_prefill": {
            "metric": "prefill tokens/s, 262144 tokens x 16 heads in one call",
            "value": aggregate_throughput(LT, world, ms_long), "unit": "tokens/s", "ms_per_step": ms_long,
            "roofline": hbm_roofline(prefill_kernel % l_launch_whole, lbytes, ms_long,
                                     traffic=measured_traffic("long_prefill_call", "prefill"),
                                     algorithmic_flops=prefill_flops(LT, H, dk),
                                     tensor_frac=tensor_frac(prefill_flops(LT, H, dk), ms_long)),
            "segmented": {"metric": "the same tokens as 64 calls of 4096 with the state carried",
                          "value": aggregate_throughput(LT, world, ms_long_seg), "unit": "tokens/s",
                          "ms_per_step": ms_long_seg,
                          "roofline": hbm_roofline("gdn_prefill x %d calls" % lw.segments, lseg_bytes,
                                                   ms_long_seg)},
            "l2": "not flushed: the inputs (3.2 GB) exceed the L2"},
        "varlen": {
            "metric": "packed prefill tokens/s, %d sequences (lengths uniform in [1024, 32768], %d tokens) x 16 "
                      "heads, per-sequence initial states" % (VN, VT),
            "value": aggregate_throughput(VT, world, ms_varlen), "unit": "tokens/s", "ms_per_step": ms_varlen,
            "roofline": hbm_roofline(prefill_kernel % v_launch, vbytes, ms_varlen,
                                     traffic=measured_traffic("varlen_call", "prefill"),
                                     algorithmic_flops=prefill_flops(VT, H, dk),
                                     tensor_frac=tensor_frac(prefill_flops(VT, H, dk), ms_varlen)),
            "l2": "not flushed: the inputs (%.0f MB) exceed the L2" % (VT * H * (2 * dk + dv) * 2 / 1e6)},
        "decode": {
            "metric": "decode tokens/s: 1024 one-token steps of 64 sequences x 16 heads in one CUDA graph, "
                      "state ping-ponged between two buffers (128 MiB, larger than the L2)",
            "value": aggregate_throughput(dw.num_seqs * nsteps, world, ms_dec_pp), "unit": "tokens/s",
            "ms_per_graph": ms_dec_pp, "us_per_step": 1e3 * ms_dec_pp / nsteps,
            "roofline": hbm_roofline("gdn_decode_kernel (per step)", dbytes // nsteps, ms_dec_pp / nsteps,
                                     traffic=measured_traffic("decode_pingpong_step", "decode")),
            "timing": "median of %d graph replays" % KG},
        "decode_inplace": {
            "metric": "the same 1024 steps updating one 64 MiB state in place",
            "value": aggregate_throughput(dw.num_seqs * nsteps, world, ms_dec_ip), "unit": "tokens/s",
            "ms_per_graph": ms_dec_ip, "us_per_step": 1e3 * ms_dec_ip / nsteps,
            "roofline": hbm_roofline("gdn_decode_kernel (per step)", dbytes // nsteps, ms_dec_ip / nsteps,
                                     traffic=measured_traffic("decode_inplace_step", "decode"),
                                     note="part of the state can stay in the 126 MB L2 between steps")},
        "preprocess": {"metric": "pre-processing tokens/s (conv4 + SiLU + q/k L2 norm + gates), prefill shapes",
                       "value": aggregate_throughput(T, world, ms_pre), "unit": "tokens/s", "ms_per_step": ms_pre,
                       "roofline": hbm_roofline("gdn_preprocess_kernel", pre_bytes, ms_pre,
                                                traffic=measured_traffic("preprocess_prefill_shapes", "layer"))},
        "output_gate": {"metric": "output gate tokens/s (RMS norm + sigmoid gate), prefill shapes",
                        "value": aggregate_throughput(T, world, ms_gate), "unit": "tokens/s", "ms_per_step": ms_gate,
                        "roofline": hbm_roofline("gdn_output_gate_kernel", gate_bytes, ms_gate,
                                                 traffic=measured_traffic("output_gate_prefill_shapes", "layer"))},
        "layer": {"metric": "GDN layer token mixer tokens/s at the prefill shapes: raw projections -> "
                            "pre-processing -> recurrence -> output gate",
                  "value": aggregate_throughput(T, world, ms_layer_fused), "unit": "tokens/s",
                  "ms_per_step": ms_layer_fused, "kernels": launches_per_prefill,
                  "unfused": {"metric": "the same as gdn_preprocess + gdn_prefill + gdn_output_gate",
                              "value": aggregate_throughput(T, world, ms_layer_unfused), "unit": "tokens/s",
                              "ms_per_step": ms_layer_unfused, "kernels": 2 + launches_per_prefill},
                  "l2": "flushed before every step"},
        "streaming": {"metric": "GDN layer frames/s: pre-processing + recurrence with carried state + "
                                "output gate per %d-token frame x %d heads, CUDA-graph replay" % (FRAME, H),
                      "value": 1e3 / ms_frame_graph * world, "unit": "frames/s",
                      "ms_per_frame_graph": ms_frame_graph, "ms_per_frame_eager": ms_frame_eager,
                      "kernels_per_frame": frame_launches,
                      "decode_step_ms_graph": ms_dec_graph, "kernels_per_decode_step": decode_launches,
                      "l2": "flushed before every frame"},
        "swa": {"metric": "sliding-window attention layer tokens/s (RoPE on q and k + attention), "
                          "T=%d, window %d, %d query / %d key-value heads, d %d, bf16"
                          % (SWA_T, W.SWA_WINDOW, W.SWA_HQ, W.SWA_HKV, W.SWA_D),
                "value": aggregate_throughput(SWA_T, world, ms_swa_layer), "unit": "tokens/s",
                "ms_per_step": ms_swa_layer, "attention_ms": ms_swa_attn,
                "roofline": {"kernel": "swa_fwd_pair_kernel", "bound": "tensor", "achieved": swa_tf,
                             "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": swa_tf / pk["bf16_tflops"],
                             "traffic": measured_traffic("swa_T32768_W8192", "swa"),
                             "peak_source": pk_kind, "algorithmic_flops": swa_flops},
                "l2": "flushed before every step"},
        "e2e": {"value": aggregate_throughput(T, world, ms_e2e), "unit": "tokens/s",
                "ms_per_step": ms_e2e, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": sum(launches.values()),
        "gpu_launches_by_leg": launches,
        "clocks": clk.summary(),
        "timed_wall_s": wall,
    }
    leg_keys = {"long_prefill": "long_prefill", "varlen": "varlen", "decode": "decode",
                "decode_inplace": "decode", "preprocess": "layer", "output_gate": "layer", "layer": "layer",
                "streaming": "streaming", "swa": "swa", "e2e": "e2e"}
    for key, leg in leg_keys.items():
        if not want(leg):
            line.pop(key, None)
    if not want("prefill"):
        line["value"] = None
        line["ms_per_step"] = None
        line["roofline"] = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and want("prefill"):
        line["cpu_baseline"] = cpu_baseline()
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph_pp, graph_ip
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------------------ oracle arm

def _oracle_sample(tokens, seed=0):
    w = W.Workload(**{**PREFILL.__dict__, "T": tokens})
    x = W.prefill_inputs(w, seed=seed)
    f = lambda t: t.to(torch.float64).numpy()
    return (f(x["q"]), f(x["k"]), f(x["v"]), f(x["g"]), f(x["beta"]))


def cpu_baseline(tokens=8192, target_s=10.0):
    """The oracle, as it stands, on the prefill workload (all 16 heads),
    repeated until about target_s seconds of host time have been spent."""
    import oracle
    q, k, v, g, b = _oracle_sample(tokens)
    n = oracle.default_threads()
    reps, total = 0, 0.0
    while total < target_s and reps < 1000:
        t0 = time.perf_counter()
        oracle.prefill(q, k, v, g, b, None, None, nthreads=n)
        total += time.perf_counter() - t0
        reps += 1
    return {"value": reps * tokens / total, "unit": "tokens/s", "cores": min(n, PREFILL.H),
            "host_cores": os.cpu_count(), "kind": "oracle",
            "sample": "full prefill_bf16 workload (%d tokens x 16 heads) run %d times, %.1f s; "
                      "threads over the 16 (sequence, head) units" % (tokens, reps, total)}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    tokens = 256
    q, k, v, g, b = _oracle_sample(tokens)
    n = oracle.default_threads()
    for _ in range(args.warmup):
        oracle.prefill(q, k, v, g, b, None, None, nthreads=n)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.prefill(q, k, v, g, b, None, None, nthreads=n)
        times.append(time.perf_counter() - t0)
    ms = 1e3 * sum(times) / len(times)
    value = tokens / (ms * 1e-3)
    sample = "first %d tokens of the prefill_bf16 workload, all 16 heads, per step" % tokens
    line = {
        "impl": "reference",
        "metric": "GDN prefill tokens/s and decode tokens/s on 1 B200; % of TC / HBM roofline",
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "prefill_bf16: B=1, H=16, T=8192, d_k=d_v=128, chunk=64 "
                               "(bounded sample per step)", "seq_len": tokens},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": min(n, PREFILL.H),
                         "host_cores": os.cpu_count(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--legs", default="",
                    help="comma-separated subset of %s (default: all); for profiling one workload" % (ALL_LEGS,))
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_native(args)


if __name__ == "__main__":
    main()
