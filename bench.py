#!/usr/bin/env python
"""Benchmark of the hybrid compressed attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline (one JSON line on rank 0): the 128K-context hybrid decode step
(batch 32; one CSA layer m=4 top-k=512 indexer 8x64, then one HCA layer
m'=128; 64 heads, KV dim 512, window 128), in us/step.  Sub-objects report
the 64K CSA prefill (tokens/s of compression + index/top-k + attention; the
projections are timed separately), the 1M-context decode (fp8 indexer keys)
and the 8K HCA prefill.  Each carries the roofline of its dominant kernel.

Multi-GPU (torchrun): every rank runs its own replica of the headline
workload (no data-path collective); the reported time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_compressed_hca_b200 import binding as hb  # noqa: E402
from long_context_compressed_hca_b200 import synth, workloads  # noqa: E402
from long_context_compressed_hca_b200.layer import CacheHandle, LayerHandle, TokenInputs  # noqa: E402

METRIC = "CSA/HCA attn prefill tokens/s & decode µs/step at 128K-1M ctx; % of roofline"
L2_FLUSH_BYTES = 256 << 20


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d["bf16_tflops_sustained"],
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = [r.split(", ") for r in out.strip().splitlines() if r.count(",") >= 8]
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------------------------- helpers
def dev_normal(shape, seed, stream, dtype=torch.float32, std=1.0):
    return synth.normal_on("cuda", shape, seed, stream, std=std, dtype=dtype)


def time_steps(step, K, flush_buf, stream, profile=False, replayed=False):
    """K device-timed steps (CUDA events on `stream`), L2 flushed before each.
    With profile=True the library's per-kernel events are sampled after every
    step (this pass is for the per-kernel breakdown, not for the step time)."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    l0 = hb.launch_count()
    with torch.cuda.stream(stream):
        for i in range(K):
            flush_buf.fill_(i & 0xFF)
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
            if profile and replayed:
                hb.profile_sample()        # a replayed graph re-records the same events
    torch.cuda.synchronize()
    if profile and not replayed:
        hb.profile_sample()
    launches = hb.launch_count() - l0
    kern = {}
    if profile:
        kern = {k: {"launches": v[0], "ms": v[1]} for k, v in hb.profile_collect().items()}
    ms = [a.elapsed_time(b) for a, b in evs]
    return ms, launches, kern


def profiled(fn):
    """Run fn with the library's per-kernel event profiling switched on."""
    hb.profile_enable(True)
    hb.profile_collect()
    try:
        return fn()
    finally:
        hb.profile_enable(False)


def dist_max(x: float) -> float:
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
        t = torch.tensor([x], device=dev, dtype=torch.float64)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        return float(t.item())
    return x


def barrier():
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.barrier()


# --------------------------------------------------------------------------- decode
# The HCA layer of a decode step runs on a side stream next to the CSA layer's
# ingest -> indexer -> top-k -> attention chain, the step's critical path.  Per
# workload: the CTA budgets of the CSA and HCA attention calls (0 = every SM) and
# whether the HCA stream has the higher priority.  Measured in alternating runs on
# one box (us per step):
#   128K batch 32: every SM, equal priority 122; HCA first 118; HCA 32 CTAs (one
#                  split per query) + HCA first 112.5; HCA 32 CTAs at equal priority 120
#   1M batch 4:    every SM 148 (HCA: 32 splits through the fp32 workspace + combine);
#                  HCA 32 CTAs (8 splits, cluster merge) at equal priority 128, HCA first
#                  145; CSA 32 CTAs as well (8 splits instead of 9 + combine) 124, 16: 131
LAYER_CTAS = {workloads.HYBRID_DECODE_128K.name: (0, 32, True),
              workloads.HYBRID_DECODE_1M.name: (32, 32, False)}


def packed(tensors):
    """Copies of `tensors` in one device buffer (each at a 256-byte aligned
    offset): the buffer and the views, so that a step's inputs or outputs move
    between host and device in one copy."""
    offs, tot = [], 0
    for t in tensors:
        offs.append(tot)
        tot += (t.numel() * t.element_size() + 255) // 256 * 256
    flat = torch.empty(tot, dtype=torch.uint8, device="cuda")
    views = []
    for t, o in zip(tensors, offs):
        v = flat[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
        v.copy_(t)
        views.append(v)
    return flat, views


class DecodeBench:
    """One decode step per sequence over synthetic caches: CSA layer + HCA layer."""

    def __init__(self, wl, seed_shift=0, side_ctas=None, side_high=None, kv_mixed=False, idx_key_dtype=None):
        self.wl = wl
        self.kv_mixed = kv_mixed
        self.idx_key_dtype = idx_key_dtype or wl.idx_key_dtype
        B, pos = wl.B, wl.pos
        seed = wl.seed + seed_shift
        main_ctas, ctas, high = LAYER_CTAS.get(wl.name, (0, 0, False))
        self.main_ctas = main_ctas
        self.side_ctas = ctas if side_ctas is None else side_ctas
        self.side_high = high if side_high is None else side_high
        self.layers, self.caches, self.x, self.outs, self.ws = [], [], [], [], []
        for li, L in enumerate(wl.layers):
            W = synth.layer_weights(L, 64, 64, seed, torch.bfloat16, layer_id=li)   # decode reads sink/biases only
            lh = LayerHandle(L, W, 64, 64, torch.bfloat16, B, idx_key_dtype=self.idx_key_dtype,
                             max_ctas=self.side_ctas if li > 0 else self.main_ctas, kv_mixed=kv_mixed)
            lcm = 32
            cap = ((pos // L.m + 8 + lcm - 1) // lcm) * lcm
            ch = CacheHandle(L, B, cap, torch.bfloat16, idx_key_dtype=self.idx_key_dtype, kv_mixed=kv_mixed)
            s = 1000 * (li + 1)
            if kv_mixed:
                # mixed-precision records of N(0,1) rows
                for buf, sid in ((ch.kv_comp, 1), (ch.win, 2)):
                    rows = buf.shape[0] * buf.shape[1]
                    hb.kv_quant_mixed(dev_normal((rows, L.c), seed, s + sid, torch.bfloat16), hb.HCA_BF16, rows,
                                      L.c, L.rd, buf)
            else:
                ch.kv_comp.copy_(dev_normal(ch.kv_comp.shape, seed, s + 1, torch.bfloat16))
                ch.win.copy_(dev_normal(ch.win.shape, seed, s + 2, torch.bfloat16))
            ch.state_kv.copy_(dev_normal(ch.state_kv.shape, seed, s + 3))
            ch.state_score.copy_(dev_normal(ch.state_score.shape, seed, s + 4))
            if L.kind == "csa":
                kf = dev_normal(ch.key_I.shape, seed, s + 5)
                if self.idx_key_dtype == "fp8":
                    kb, ks = synth.fp8_rows(kf)
                    ch.key_I.copy_(kb)
                    ch.key_I_scale.copy_(ks)
                elif self.idx_key_dtype == "fp4":
                    # rotated FP4 keys (carried in bf16), as the compressor stores them
                    rows = kf.shape[0] * kf.shape[1]
                    hb.fp4_rotate_quant(kf.contiguous(), hb.HCA_F32, rows, kf.shape[2], ch.key_I)
                else:
                    ch.key_I.copy_(kf.to(torch.bfloat16))
                ch.stateI_kv.copy_(dev_normal(ch.stateI_kv.shape, seed, s + 6))
                ch.stateI_score.copy_(dev_normal(ch.stateI_score.shape, seed, s + 7))
            x = dict(q=dev_normal((B, L.n_h, L.c), seed, s + 10, torch.bfloat16),
                     kv=dev_normal((B, L.c), seed, s + 11, torch.bfloat16),
                     comp=dev_normal((B, (4 if L.kind == "csa" else 2) * L.c), seed, s + 12))
            if L.kind == "csa":
                x.update(qI=dev_normal((B, L.n_hI, L.c_I), seed, s + 13, torch.bfloat16),
                         wI=dev_normal((B, L.n_hI), seed, s + 14, std=L.c_I ** -0.5 * L.n_hI ** -0.5),
                         compI=dev_normal((B, 4 * L.c_I), seed, s + 15))
            self.x.append(x)
            o = torch.empty(B, L.n_h, L.c, dtype=torch.bfloat16, device="cuda")
            # sized for the 128 consecutive positions the step sweep visits
            ws = torch.empty(max(hb.decode_workspace_size(lh.struct, pos + 128), 256), dtype=torch.uint8,
                             device="cuda")
            self.layers.append(lh)
            self.caches.append(ch)
            self.outs.append(o)
            self.ws.append(ws)
        # pinned host copies for the end-to-end measurement
        self.in_flat, self.inputs, self.out_flat, self.outs = self.buffer_set()
        self.host_in = self.in_flat.cpu().pin_memory()
        self.host_out = torch.empty(self.out_flat.shape, dtype=torch.uint8).pin_memory()

    def buffer_set(self):
        """A set of per-step device inputs and outputs: every layer's token
        inputs packed in one buffer and its outputs in another.  Returns
        (input buffer, TokenInputs per layer, output buffer, output per layer)."""
        names = [[k for k, v in x.items() if v is not None] for x in self.x]
        in_flat, views = packed([x[k] for x, ks in zip(self.x, names) for k in ks])
        ins, at = [], 0
        for ks in names:
            ins.append(TokenInputs(**dict(zip(ks, views[at:at + len(ks)]))))
            at += len(ks)
        out_flat, outs = packed(self.outs)
        return in_flat, ins, out_flat, outs

    def step(self, pos=None, bufs=None):
        """CSA layer on the current stream, HCA layer on a side stream (the two
        layers of the step are independent), joined before returning.  `pos`
        overrides the workload's token position, `bufs` the input/output set."""
        pos = self.wl.pos if pos is None else pos
        inputs, outs = bufs if bufs is not None else (self.inputs, self.outs)
        cur = torch.cuda.current_stream()
        if not hasattr(self, "side"):
            lo, hi = torch.cuda.Stream.priority_range()
            self.side = torch.cuda.Stream(priority=hi if self.side_high else lo)
            self.fork, self.join = torch.cuda.Event(), torch.cuda.Event()
        self.fork.record(cur)
        self.side.wait_event(self.fork)
        for i, (lh, ch, ti, o, ws) in enumerate(zip(self.layers, self.caches, inputs, outs, self.ws)):
            st = cur if i == 0 else self.side
            with torch.cuda.stream(st):
                hb.hybrid_decode_step(lh.struct, ti.struct, ch.struct, pos, o, ws)
        self.join.record(self.side)
        cur.wait_event(self.join)

    def e2e_bytes(self):
        return self.host_in.numel(), self.host_out.numel()

    def algorithmic_bytes(self):
        """Bytes each kernel of the step must move (the HBM roofline's
        numerators), per launch, and their sum for the whole step."""
        wl, B, pos = self.wl, self.wl.B, self.wl.pos
        per = {}
        for L in wl.layers:
            V = (pos + 1) // L.m
            nw = min(L.w, pos + 1)
            qo = 2 * B * L.n_h * L.c * 2
            row = hb.kv_mixed_row_bytes(L.c, L.rd) if self.kv_mixed else L.c * 2   # bytes per KV row
            if L.kind == "csa":
                kb = 1 if self.idx_key_dtype == "fp8" else 2
                per["index_scores"] = B * V * (L.c_I * kb + (4 if kb == 1 else 0)) + B * L.n_hI * (L.c_I * 2 + 4)
                per["topk"] = B * V * 4 + B * L.k * 4          # scores in, indices out
                per["attend_csa"] = B * (min(L.k, V) + nw) * row + qo
            else:
                per["attend_hca"] = B * (V + nw) * row + qo
        # the step's total counts the method's own streams (keys, rows, q/o), not the scores
        # the selection reads back
        return sum(v for k, v in per.items() if k != "topk"), per


def capture_graph(fn, stream):
    """Capture fn's launches (all on `stream`) into a CUDA graph; returns replay()."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        fn()                       # warm the host-side caches outside capture
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=stream):
        fn()
    torch.cuda.synchronize()
    return g


def time_step_sweep(b, K, W, flush, stream):
    """The emitting step (both compressors close a block: pos+1 a multiple of
    128) and the mean over 128 consecutive steps pos..pos+127 (32 CSA entries
    and one HCA entry emitted), each step its own captured graph."""
    wl = b.wl
    pe = ((wl.pos + 1 + 127) // 128) * 128 - 1
    ge = capture_graph(lambda: b.step(pe), stream)
    for _ in range(W):
        ge.replay()
    ems, _, _ = time_steps(ge.replay, K, flush, stream)
    graphs = [capture_graph(lambda p=p: b.step(p), stream) for p in range(wl.pos, wl.pos + 128)]

    def seq():
        for g in graphs:
            g.replay()
    seq()
    torch.cuda.synchronize()
    reps = max(2, min(K, 5))
    sms, _, _ = time_steps(seq, reps, flush, stream)
    del graphs, ge
    return dict(emit_pos=pe, emit_us=round(statistics.mean(ems) * 1e3, 2),
                mean_128_us=round(statistics.mean(sms) / 128 * 1e3, 2), mean_128_reps=reps)


def time_e2e_pipelined(b, K, W, stream):
    """End to end through the public API: every step copies its inputs from
    pinned host memory to the device, runs the decode step and copies its
    outputs back.  Two device buffer sets and three streams let the copies of
    neighbouring steps overlap the step, as a serving loop would; returns the
    device time per step over K steps."""
    sets = [(b.in_flat, b.inputs, b.out_flat, b.outs), b.buffer_set()]
    graphs = [capture_graph(lambda bs=bs: b.step(bufs=(bs[1], bs[3])), stream) for bs in sets]
    hout = [b.host_out, torch.empty_like(b.host_out).pin_memory()]
    s_in, s_c, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    e_in, e_done, e_out = ([torch.cuda.Event() for _ in sets] for _ in range(3))

    def one(i):
        k = i % 2
        in_flat, _, out_flat, _ = sets[k]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(e_done[k])          # this set's previous step has read its inputs
            in_flat.copy_(b.host_in, non_blocking=True)
            e_in[k].record(s_in)
        with torch.cuda.stream(s_c):
            s_c.wait_event(e_in[k])
            if i >= 2:
                s_c.wait_event(e_out[k])            # and its outputs are back on the host
            graphs[k].replay()
            e_done[k].record(s_c)
        with torch.cuda.stream(s_out):
            s_out.wait_event(e_done[k])
            hout[k].copy_(out_flat, non_blocking=True)
            e_out[k].record(s_out)

    for i in range(W):
        one(i)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    for i in range(W, W + K):
        one(i)
    t1.record(s_out)
    torch.cuda.synchronize()
    del graphs
    return t0.elapsed_time(t1) / K


def run_decode(wl, K, W, flush, stream, e2e=True, sweep=False, **variant):
    b = DecodeBench(wl, **variant)
    for _ in range(W):
        b.step()
    torch.cuda.synchronize()
    # the decode step's launches replayed as one CUDA graph
    l0 = hb.launch_count()
    graph = capture_graph(b.step, stream)
    per_step_launches = (hb.launch_count() - l0) // 2
    for _ in range(W):
        graph.replay()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ms, _, _ = time_steps(graph.replay, K, flush, stream)
    launches = per_step_launches * K
    barrier()
    torch.cuda.synchronize()
    # per-kernel times: a second graph captured with the library's event
    # profiling on, replayed K times
    def prof_pass():
        hb.profile_enable(True)
        pg = torch.cuda.CUDAGraph()
        with torch.cuda.graph(pg, stream=stream):
            b.step()
        torch.cuda.synchronize()
        return time_steps(pg.replay, K, flush, stream, profile=True, replayed=True)[2]
    kern = profiled(prof_pass)
    res = dict(bench=b, ms=ms, launches=launches, kern=kern, graph=True, side_ctas=b.side_ctas,
               side_high=b.side_high, main_ctas=b.main_ctas)
    if e2e:
        res["e2e_ms"] = [time_e2e_pipelined(b, K, W, stream)]
    del graph
    if sweep:
        res["sweep"] = time_step_sweep(b, K, W, flush, stream)
    return res


# --------------------------------------------------------------------------- prefill
class PrefillBench:
    def __init__(self, wl):
        self.wl = wl
        L = wl.layers[0]
        big = synth.layer_weights_on("cuda", L, wl.d, wl.d_c, wl.seed, torch.bfloat16)
        self.lh = LayerHandle(L, big, wl.d, wl.d_c, torch.bfloat16, wl.B)
        self.H = dev_normal((wl.B, wl.n, wl.d), wl.seed, synth.STREAMS["H"], torch.bfloat16)
        self.o = torch.empty(wl.B, wl.n, L.n_h, L.c, dtype=torch.bfloat16, device="cuda")
        self.ws = torch.empty(hb.layer_workspace_size(self.lh.struct, wl.n), dtype=torch.uint8, device="cuda")

    def step(self):
        hb.hybrid_layer_forward(self.lh.struct, self.H, self.wl.n, None, self.o, self.ws)


ATTN_PATH = ("compress_prefill", "compress_state", "index_scores", "topk", "attend")


def prefill_flops(wl):
    """Algorithmic FLOPs of the attention path (indexer + attention) and the
    compression bytes, per prefill."""
    L = wl.layers[0]
    n, B = wl.n, wl.B
    att = idx = 0
    for t in range(n):
        V = (t + 1) // L.m
        nc = min(L.k, V) if L.kind == "csa" else V
        att += (nc + min(L.w, t + 1)) * L.n_h * L.c * 4
        if L.kind == "csa":
            idx += V * L.n_hI * L.c_I * 2
    return B * att, B * idx


def run_prefill(wl, K, W, flush, stream):
    b = PrefillBench(wl)
    for _ in range(W):
        b.step()
    torch.cuda.synchronize()
    ms, launches, kern = profiled(lambda: time_steps(b.step, K, flush, stream, profile=True))
    path_ms = sum(v["ms"] for k, v in kern.items() if k.startswith(ATTN_PATH)) / K
    glue_ms = sum(v["ms"] for k, v in kern.items() if k.startswith(("gemm", "row_op", "ring"))) / K
    att_flops, idx_flops = prefill_flops(wl)
    del b
    torch.cuda.empty_cache()
    return dict(ms=ms, launches=launches, kern=kern, path_ms=path_ms, glue_ms=glue_ms,
                att_flops=att_flops, idx_flops=idx_flops)


# --------------------------------------------------------------------------- output projection
def run_oproj(T, K, W, flush, stream):
    """Grouped output projection of T tokens at the CSA layer's widths
    (64 heads x 512, g = 8 groups, d_g = 1024, d = 4096): 2*T*(n_h*c*d_g + g*d_g*d) FLOP."""
    n_h, c, g, d_g, d = 64, 512, 8, 1024, 4096
    gw = n_h * c // g
    o = dev_normal((T, n_h, c), 7, 1, torch.bfloat16)
    wo_a = dev_normal((g, d_g, gw), 7, 2, torch.bfloat16, std=gw ** -0.5)
    wo_b = dev_normal((d, g * d_g), 7, 3, torch.bfloat16, std=(g * d_g) ** -0.5)
    out = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    desc = hb.oproj_desc(T, n_h, c, g, d_g, d, hb.HCA_BF16, hb.HCA_BF16)
    ws = torch.empty(hb.output_projection_workspace_size(desc), dtype=torch.uint8, device="cuda")

    def step():
        hb.output_projection(desc, o, wo_a, wo_b, out, ws)
    for _ in range(W):
        step()
    torch.cuda.synchronize()
    ms, _, _ = time_steps(step, K, flush, stream)
    flops = 2.0 * T * (n_h * c * d_g + g * d_g * d)
    del o, wo_a, wo_b, out, ws
    torch.cuda.empty_cache()
    return statistics.mean(ms), flops


def run_chained(wl, K, W, flush, stream):
    """The two layers of the 128K decode step chained through hidden states
    (d_model 4096, query compression 1024): CSA decode inputs from h0 -> CSA
    step -> grouped output projection (8 groups of 1024) -> HCA decode inputs ->
    HCA step, on one stream (each stage needs the previous one's output).
    Returns (ms per chained step, per-kernel profile)."""
    d, d_c, g, d_g = 4096, 1024, 8, 1024
    b = DecodeBench(wl)                      # caches and step inputs at the workload's position
    B, pos = wl.B, wl.pos
    Ls = wl.layers
    lhs, xs, wss = [], [], []
    for li, L in enumerate(Ls):
        Wt = synth.layer_weights_on("cuda", L, d, d_c, wl.seed, torch.bfloat16, layer_id=li)
        lh = LayerHandle(L, Wt, d, d_c, torch.bfloat16, B)   # sequential: every SM for each attention
        lhs.append(lh)
        xs.append(TokenInputs.empty(L, B, torch.bfloat16))
        wss.append(torch.empty(max(hb.decode_inputs_workspace_size(lh.struct), 256), dtype=torch.uint8,
                               device="cuda"))
    gw = Ls[0].n_h * Ls[0].c // g
    wo_a = dev_normal((g, d_g, gw), wl.seed, 21, torch.bfloat16, std=gw ** -0.5)
    wo_b = dev_normal((d, g * d_g), wl.seed, 22, torch.bfloat16, std=(g * d_g) ** -0.5)
    od = hb.oproj_desc(B, Ls[0].n_h, Ls[0].c, g, d_g, d, hb.HCA_BF16, hb.HCA_BF16)
    wso = torch.empty(max(hb.output_projection_workspace_size(od), 256), dtype=torch.uint8, device="cuda")
    h0 = dev_normal((B, d), wl.seed, 23, torch.bfloat16)
    h1 = torch.empty(B, d, dtype=torch.bfloat16, device="cuda")

    def step():
        hb.hybrid_decode_inputs(lhs[0].struct, h0, pos, xs[0].struct, wss[0])
        hb.hybrid_decode_step(lhs[0].struct, xs[0].struct, b.caches[0].struct, pos, b.outs[0], b.ws[0])
        hb.output_projection(od, b.outs[0], wo_a, wo_b, h1, wso)
        hb.hybrid_decode_inputs(lhs[1].struct, h1, pos, xs[1].struct, wss[1])
        hb.hybrid_decode_step(lhs[1].struct, xs[1].struct, b.caches[1].struct, pos, b.outs[1], b.ws[1])

    for _ in range(W):
        step()
    torch.cuda.synchronize()
    graph = capture_graph(step, stream)
    for _ in range(W):
        graph.replay()
    torch.cuda.synchronize()
    ms, _, _ = time_steps(graph.replay, K, flush, stream)

    def prof_pass():
        hb.profile_enable(True)
        pg = torch.cuda.CUDAGraph()
        with torch.cuda.graph(pg, stream=stream):
            step()
        torch.cuda.synchronize()
        return time_steps(pg.replay, K, flush, stream, profile=True, replayed=True)[2]
    kern = profiled(prof_pass)
    del graph, b, lhs, xs, wss
    torch.cuda.empty_cache()
    return statistics.mean(ms), kern


# --------------------------------------------------------------------------- oracle arm
class OracleStep:
    """The C++ oracle's inputs for one decode step of a DecodeBench (every
    sequence, both layers), copied to the host in the bytes the GPU stores
    (bf16 bits, e4m3 codes and scales); time(n_seq) runs the oracle's decode of
    the first n_seq sequences of both layers and returns the seconds."""

    def __init__(self, bench: DecodeBench):
        import numpy as np
        from oracle import hca_oracle as O
        from oracle import hca_oracle_c as OC
        self.OC = OC
        wl, pos = bench.wl, bench.wl.pos
        self.layers = []
        bits = lambda t: t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
        for li, L in enumerate(wl.layers):
            ch, ti = bench.caches[li], bench.inputs[li]
            d = dict(L=L, q=ti.t["q"].double().cpu().numpy(), win=bits(ch.win), comp=bits(ch.kv_comp),
                     order=np.array([p % L.w for p in O.window_positions(pos, L.w)], dtype=np.int32),
                     sink=bench.layers[li].t["sink"].double().cpu().numpy())
            if L.kind == "csa":
                if bench.idx_key_dtype == "fp8":
                    d["KI"], d["KI_scale"] = ch.key_I.cpu().numpy(), ch.key_I_scale.cpu().numpy()
                else:
                    d["KI"], d["KI_scale"] = bits(ch.key_I), None
                d["qI"] = ti.t["qI"].double().cpu().numpy()
                d["wI"] = ti.t["wI"].double().cpu().numpy()
            self.layers.append(d)
        self.pos = pos

    def time(self, n_seq, threads):
        self.OC.num_threads(threads)
        t0 = time.perf_counter()
        for d in self.layers:
            L = d["L"]
            csa = L.kind == "csa"
            self.OC.decode_batch(L.kind, d["q"][:n_seq], d["win"], d["order"], d["comp"], L.m, d["sink"], L.rd,
                                 self.pos, k=L.k if csa else 0, qI=d["qI"][:n_seq] if csa else None,
                                 w=d["wI"][:n_seq] if csa else None, KI=d.get("KI"), KI_scale=d.get("KI_scale"))
        return time.perf_counter() - t0


def oracle_baseline(bench: DecodeBench, reps: int, warmup: int):
    """The C++ oracle (double precision, -O3, OpenMP over the sequences) on the
    step: every sequence on all host cores, and a bounded sample on one core
    scaled to the step.  Returns (us per step on all cores, per reps, the
    one-core figure, the one-core sample size, cores)."""
    os_ = OracleStep(bench)
    B = bench.wl.B
    cores = os_.OC.num_threads(os.cpu_count() or 1)
    for _ in range(warmup):
        os_.time(B, cores)
    all_us = [os_.time(B, cores) * 1e6 for _ in range(reps)]
    n1 = min(B, 4)
    one_us = os_.time(n1, 1) * B / n1 * 1e6
    os_.OC.num_threads(cores)
    return all_us, one_us, n1, cores


# --------------------------------------------------------------------------- main
# DRAM bytes (read + write) per launch of the decode kernels at the 128K batch-32 workload,
# from single ncu captures (profiles/*_b32.md); None where no capture covers the kernel as it is.
TRAFFIC_128K = {"index_scores": 134_291_200 + 4_877_056, "topk": 4_248_576, "attend_csa": 23_249_920 + 1_536,
                "attend_hca": 39_943_680 + 11_008}   # at the bench's budget of 32 CTAs


def roofline_hbm(bytes_per_launch, ms_per_launch, peaks, traffic=None):
    ach = bytes_per_launch / (ms_per_launch * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm"], "unit": "GB/s",
            "frac": round(ach / peaks["hbm"], 4), "traffic": traffic,
            "peak_source": f"{peaks['src']} (hbm_gbs copy test)"}


def roofline_tensor(flops_per_launch, ms_per_launch, peaks, traffic=None):
    """Against the dense bf16 peak measured as a burst (the kernels are timed
    alone within a layer of tens of ms); the sustained-peak fraction beside it."""
    ach = flops_per_launch / (ms_per_launch * 1e-3) / 1e12
    return {"bound": "tensor", "achieved": round(ach, 1), "peak": peaks["bf16"], "unit": "TFLOP/s",
            "frac": round(ach / peaks["bf16"], 4), "traffic": traffic,
            "peak_source": f"{peaks['src']} dense bf16 (cuBLAS burst)",
            "frac_of_sustained": round(ach / peaks["bf16_sus"], 4), "peak_sustained": peaks["bf16_sus"]}


# DRAM bytes per query token of the CSA prefill attention kernel (64 heads x 512):
# read + write counters of one ncu capture of the 16384-token layer (2.157 GB:
# q read once, o written once, the compressed entries served from L2), which
# scale with the token count; the traffic of longer launches is this times
# their tokens.
CSA_PREFILL_ATTN_DRAM_PER_TOKEN = 2157e6 / 16384
# DRAM bytes of the HCA prefill attention launch (batch 2 x 8192 tokens, 16
# heads x 128): read + write counters of one ncu capture of that very launch
# (71.4 MB + 20.7 MB; most of o is still in L2 when the kernel ends).
HCA_PREFILL_ATTN_DRAM = 92.1e6


def kern_ms(kern, prefix, K):
    tot = sum(v["ms"] for k, v in kern.items() if k.startswith(prefix))
    n = sum(v["launches"] for k, v in kern.items() if k.startswith(prefix))
    return tot / max(n, 1), n / K


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--only-headline", action="store_true")
    args = ap.parse_args()
    assert args.warmup >= 3, "at least 3 warm-up steps"

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    hb.lib()
    peaks = measured_peaks()
    wl = workloads.HYBRID_DECODE_128K

    if args.impl == "reference":
        # the oracle, as it stands, on the headline's config: each step is a
        # bounded sample (n sequences of the 32), scaled to the whole step
        if rank != 0:
            if world > 1:
                torch.distributed.destroy_process_group()
            return
        b = DecodeBench(wl)
        times, one_us, n1, cores = oracle_baseline(b, args.steps, args.warmup)
        v = statistics.mean(times)
        line = {"metric": METRIC, "value": round(v, 1), "unit": "us/step", "impl": "reference",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": v / 1e3,
                "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic",
                "config": {"workload": wl.name, "global_batch": wl.B, "seq_len": wl.pos,
                           "parallelism": "single process (CPU oracle)"},
                "cpu_baseline": {"value": round(v, 1), "unit": "us/step", "cores": cores, "kind": "oracle",
                                 "sample": f"all {wl.B} sequences of each step (CSA+HCA layer), C++ oracle, "
                                           f"double precision, OpenMP over the sequences",
                                 "single_core_us_per_step": round(one_us, 1),
                                 "single_core_sample": f"{n1} of {wl.B} sequences, scaled x{wl.B / n1:g}"},
                "e2e": {"value": round(v, 1), "unit": "us/step", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return

    stream = torch.cuda.Stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    clocks = ClockSampler(local if world > 1 else torch.cuda.current_device())
    clocks.start()
    head = run_decode(wl, args.steps, args.warmup, flush, stream, sweep=not args.only_headline)
    clk = clocks.stop()
    step_ms = statistics.mean(head["ms"])
    step_ms_max = dist_max(step_ms)
    e2e_ms = dist_max(statistics.mean(head["e2e_ms"]))
    tot_bytes, per_bytes = head["bench"].algorithmic_bytes()
    kern = head["kern"]
    # dominant kernel of the step (largest share of device time) and its roofline
    roof = None
    if kern:
        dom = max(kern.items(), key=lambda kv: kv[1]["ms"])[0]
        per_launch_ms = kern[dom]["ms"] / kern[dom]["launches"]
        key = next((k for k in per_bytes if dom.startswith(k) or k in dom), None)
        if key is not None:
            roof = roofline_hbm(per_bytes[key], per_launch_ms, peaks,
                                traffic=TRAFFIC_128K.get(key) if wl is workloads.HYBRID_DECODE_128K else None)
            roof["algorithmic_bytes_per_launch"] = per_bytes[key]
        else:
            roof = {"bound": "hbm", "achieved": None, "peak": peaks["hbm"], "unit": "GB/s", "frac": None,
                    "traffic": None}
        roof["kernel"] = dom
        roof["share_of_step"] = round(kern[dom]["ms"] / sum(v["ms"] for v in kern.values()), 3)
    step_roof = roofline_hbm(tot_bytes, step_ms, peaks)
    hi, ho = head["bench"].e2e_bytes()

    extras = {}
    if "sweep" in head:
        extras["decode_steps"] = dict(steady_us=round(step_ms * 1e3, 2), steady_pos=wl.pos, **head["sweep"])
    if rank == 0 and world == 1:
        # the C++ CPU oracle on the same step: every sequence on all host cores,
        # and a 4-sequence sample on one core
        all_us, one_us, n1, cores = oracle_baseline(head["bench"], 2, 1)
        extras["cpu_baseline"] = {"value": round(statistics.mean(all_us), 1), "unit": "us/step",
                                  "cores": cores, "kind": "oracle",
                                  "sample": f"all {wl.B} sequences of one step (CSA+HCA), C++ oracle, double "
                                            f"precision, OpenMP over the sequences",
                                  "single_core_us_per_step": round(one_us, 1),
                                  "single_core_sample": f"{n1} of {wl.B} sequences, scaled x{wl.B / n1:g}"}
    del head["bench"]
    torch.cuda.empty_cache()

    if world == 1 and not args.only_headline:
        # 1M-context decode
        d1 = run_decode(workloads.HYBRID_DECODE_1M, args.steps, args.warmup, flush, stream, e2e=False)
        tb, _ = d1["bench"].algorithmic_bytes()
        m1 = statistics.mean(d1["ms"])
        extras["decode_1m"] = {"workload": workloads.HYBRID_DECODE_1M.name, "us_per_step": round(m1 * 1e3, 2),
                               "launch": f"attention budgets: CSA {d1['main_ctas'] or 'all'} CTAs, HCA "
                                         f"{d1['side_ctas'] or 'all'} CTAs on a side stream of "
                                         f"{'high' if d1['side_high'] else 'equal'} priority",
                               "roofline_step": roofline_hbm(tb, m1, peaks),
                               "kernels": {k: round(v["ms"] / args.steps * 1e3, 2) for k, v in d1["kern"].items()}}
        del d1
        torch.cuda.empty_cache()
        # the 128K step with the pages' storage formats: mixed-precision KV rows
        # (f2: e4m3 + block scales, RoPE dims bf16) and the FP4 indexer path
        # (f4: rotated FP4 keys carried in bf16, bf16 scores)
        for key, variant in (("decode_128k_mixed_kv", dict(kv_mixed=True)),
                             ("decode_128k_fp4_indexer", dict(idx_key_dtype="fp4"))):
            dv = run_decode(wl, args.steps, args.warmup, flush, stream, e2e=False, **variant)
            tb, pb = dv["bench"].algorithmic_bytes()
            mv = statistics.mean(dv["ms"])
            extras[key] = {"workload": wl.name + ("_kvmixed" if "kv_mixed" in variant else "_fp4idx"),
                           "us_per_step": round(mv * 1e3, 2), "algorithmic_bytes_per_step": tb,
                           "attention_row_bytes": hb.kv_mixed_row_bytes(512, 64) if "kv_mixed" in variant else 1024,
                           "roofline_step": roofline_hbm(tb, mv, peaks),
                           "kernels": {k: round(v["ms"] / args.steps * 1e3, 2) for k, v in dv["kern"].items()}}
            del dv
            torch.cuda.empty_cache()
        # prefill workloads (fewer steps: each is a whole layer)
        for key, pwl in (("prefill_64k", workloads.CSA_PREFILL), ("prefill_128k", workloads.CSA_PREFILL_128K),
                         ("hca_prefill", workloads.HCA_PREFILL)):
            kp = max(3, min(args.steps, 5))
            r = run_prefill(pwl, kp, 3, flush, stream)
            att_ms, _ = kern_ms(r["kern"], "attend", kp)
            toks = pwl.B * pwl.n
            extras[key] = {
                "workload": pwl.name,
                "tokens_per_s": round(toks / (r["path_ms"] * 1e-3), 1),
                "path_ms": round(r["path_ms"], 3),
                "projections_ms": round(r["glue_ms"], 3),
                "layer_ms": round(statistics.mean(r["ms"]), 3),
                "roofline_attention": roofline_tensor(
                    r["att_flops"], att_ms, peaks,
                    traffic=round(CSA_PREFILL_ATTN_DRAM_PER_TOKEN * toks) if r["idx_flops"] else
                    (round(HCA_PREFILL_ATTN_DRAM) if pwl is workloads.HCA_PREFILL else None)),
                "kernels_ms": {k: round(v["ms"] / kp, 3) for k, v in r["kern"].items()},
            }
            if r["idx_flops"]:
                sc_ms, _ = kern_ms(r["kern"], "index_scores", kp)
                extras[key]["roofline_index"] = roofline_tensor(r["idx_flops"], sc_ms, peaks)

    if world == 1 and not args.only_headline:
        cms, ckern = run_chained(wl, max(3, min(args.steps, 20)), 3, flush, stream)
        extras["decode_128k_chained"] = {
            "workload": wl.name + "_chained_d4096",
            "us_per_step": round(cms * 1e3, 2),
            "chain": "CSA decode inputs from hidden states -> CSA step -> grouped output projection "
                     "(8 x 1024 -> 4096) -> HCA decode inputs -> HCA step, one stream",
            "kernels": {k: round(v["ms"] / max(3, min(args.steps, 20)) * 1e3, 2) for k, v in ckern.items()}}
        oms, ofl = run_oproj(65536, max(3, min(args.steps, 5)), 3, flush, stream)
        extras["output_projection_64k"] = {
            "workload": "grouped output projection, 65536 tokens, 64x512 -> 8x1024 -> 4096, bf16",
            "ms": round(oms, 3), "roofline": roofline_tensor(ofl, oms, peaks)}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(step_ms_max * 1e3, 2), "unit": "us/step",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms_max, 5),
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": wl.name, "global_batch": wl.B * world, "seq_len": wl.pos,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "layers_per_step": "CSA(m=4,k=512,idx 8x64) + HCA(m'=128)",
                       "l2": "flushed before every timed step (256 MiB write)",
                       "launch": "decode step replayed as one CUDA graph; CSA layer on the main stream, HCA layer "
                                 f"on a {'high-priority ' if head['side_high'] else ''}side stream "
                                 f"(attention budget {head['side_ctas'] or 'all'} CTAs)"},
            "roofline": roof,
            "roofline_step": step_roof,
            "e2e": {"value": round(e2e_ms * 1e3, 2), "unit": "us/step", "h2d_bytes_per_step": hi,
                    "host_io": "pinned host buffers; copies of neighbouring steps overlap the step",
                    "d2h_bytes_per_step": ho},
            "gpu_launches": head["launches"],
            "clocks": clk,
            "kernels_us_per_step": {k: round(v["ms"] / args.steps * 1e3, 2) for k, v in kern.items()},
            "throughput_tokens_per_s": round(wl.B * world / (step_ms_max * 1e-3), 1),
        }
        line.update(extras)
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
