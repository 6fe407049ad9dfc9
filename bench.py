#!/usr/bin/env python
"""Benchmark of the KATA forward hot path on B200.

One step = one pass of every hot-path operation over one batch of synthetic
input resident in HBM:
  1. kata_fwd_quadratic  -- flash-style O(T^2) forward (tcgen05 / TMEM),
  2. kata_fwd_chunked    -- exact O(T) chunked-state forward (state build,
                            associative scan, readout), returning the final
                            state,
  3. kata_decode_step    -- one recurrent decode token per sequence, continuing
                            from that final state.
Tokens per step = B*T (the batch's tokens; the decode token is not counted).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (launched with torchrun): the (batch, head) pairs are independent,
so each rank runs its own batch with no collective on the data path (weak
scaling); the step time is the max over ranks and `value` counts all ranks'
tokens.  `--impl reference` times the fp64 CPU oracle on the host cores on a
bounded sample of the same workload (rank 0 only).

Timing: CUDA events on the launching stream around each step, after W
warm-up steps; L2 is flushed (a 512 MiB write) between timed steps, outside
the events.  The step is captured once as a CUDA graph and replayed (the
same calls and buffers, without the host launch path between the kernels);
the per-path times come from the same calls launched one by one with events
between them.  Clocks are sampled with nvidia-smi during the timed steps.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "KATA-Mg fwd tokens/sec at T=2k and 131k (1 B200); % of roofline"
UNIT = "tokens/s"

# DRAM bytes (read + write) of one flash_fwd_kernel launch at B8 H16 T2048,
# from the ncu capture summarised in profiles/flash_fwd_kernel_ctx2k.md (the
# traffic recapture).  It is reported only while the kernel's sources are the
# ones that capture ran.
FLASH_TRAFFIC_BYTES = 50576640 + 6089984
FLASH_TRAFFIC_SOURCES = ("kernelized_feature_map_b200/csrc/flash_sm100.cu", "kernelized_feature_map_b200/csrc/sm100.cuh",
                         "kernelized_feature_map_b200/csrc/kata_trace.cuh", "kernelized_feature_map_b200/csrc/kata_common.cuh")
FLASH_TRAFFIC_SHA256 = "7f2726d66afacd6130957ecff278be8d9136251b02fe3e367a30c61ce87e8e25"


def flash_traffic(workload):
    """Measured per-launch DRAM traffic of the flash kernel, or None when the
    workload or the kernel sources differ from those of the capture."""
    import hashlib
    if workload != "layer340m_ctx2k":
        return None
    h = hashlib.sha256()
    for rel in FLASH_TRAFFIC_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as fh:
            h.update(fh.read())
    return FLASH_TRAFFIC_BYTES if h.hexdigest() == FLASH_TRAFFIC_SHA256 else None


def launches_per_step(B, H, T, p, dv, C):
    """Kernels one step launches: flash 1, decode 1, and the chunked call's
    readout plus, when the sequence spans several super-chunks (it then needs
    a workspace), the state build and the scan."""
    import kernelized_feature_map_b200 as K
    import torch
    chunked = 3 if K.kata_fwd_chunked_workspace_size(B, H, T, p, dv, C, torch.bfloat16) > 0 else 1
    return 2 + chunked


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in PEAKS_FALLBACK if k in d}, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


# ---------------------------------------------------------------------------
# algorithmic work per launch: flops per causal pair, bytes per token-head
# ---------------------------------------------------------------------------
def flash_flops(BH, T, p, dv):
    """Causal-useful tensor flops: 2 (p + dv) per (query, key<=query) pair."""
    return BH * T * (T + 1) * (p + dv)


def chunked_bytes(BH, T, p, dv, elem=2):
    """q, k, v read and o written once: (2p + 2dv) elements per token-head."""
    return BH * T * (2 * p + 2 * dv) * elem


def chunked_bwd_bytes(BH, T, p, dv, elem=2):
    """The chunked backward's HBM work: q, k, v, o, dO and D read once, dq,
    dk, dv written once: (4p + 4dv) elements and 4 bytes per token-head."""
    return BH * T * ((4 * p + 4 * dv) * elem + 4)


def decode_bytes(BH, p, dv, elem=2):
    """State S (P x dv fp32) and z (P fp32) read and written; q,k,v read, o written."""
    P = p * p
    return BH * (2 * (P * dv + P) * 4 + (2 * p + 2 * dv) * elem)


# ---------------------------------------------------------------------------
# ranks: independent batches, max-over-ranks timing
# ---------------------------------------------------------------------------
def rank_config(cfg, rank):
    """Each rank draws its own batch of the same shape (weak scaling): the seed
    is offset by the rank; shapes are unchanged."""
    return dict(cfg, seed=cfg["seed"] + 1000 * rank)


def reduce_max(values, world, device="cpu"):
    """Element-wise max of a list of floats over all ranks (identity at world 1)."""
    if world <= 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def aggregate_value(tokens_per_rank, world, step_ms):
    """Whole-job tokens/s: every rank's tokens over the slowest rank's step time."""
    return tokens_per_rank * world / (step_ms * 1e-3)


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------
class ClockSampler:
    QUERY = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []          # (host time, line)
        self.window = None       # (t_start, t_end) of the timed region

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.QUERY,
                                          "--format=csv,noheader,nounits", "-lms", "25"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def wait_first_sample(self, timeout=5.0):
        t0 = time.time()
        while self.proc and not self.lines and time.time() - t0 < timeout:
            time.sleep(0.01)

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, window=None):
        """Median SM clock, max clock and throttle reasons over `window`
        (host times; default: the whole timed region)."""
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        window = window or self.window
        lo, hi = window if window else (0.0, float("inf"))
        for ts, line in self.lines:
            # a sample describes the interval before it was printed
            if ts < lo or ts > hi + 0.1:
                continue
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_ours(args, rank, world, local_rank):
    import torch
    import kernelized_feature_map_b200 as K
    from kernelized_feature_map_b200 import _abi

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg = workloads.CONFIGS[args.workload]
    B, H, T, p, dv, C = cfg["B"], cfg["H"], cfg["T"], cfg["p"], cfg["dv"], cfg["C"]
    BH = B * H
    # each rank draws its own batch (weak scaling: per-GPU work fixed)
    cfg_r = rank_config(cfg, rank)
    qn, kn, vn = workloads.make_inputs(cfg_r)
    dq, dk, dvv, dS, dz = workloads.decode_inputs(B, H, p, dv, seed=cfg["seed"] + 7 + 1000 * rank)
    bf = torch.bfloat16

    def pinned(x, dt=bf):
        return torch.from_numpy(x).to(dt).pin_memory()

    hq, hk, hv = pinned(qn), pinned(kn), pinned(vn)
    hdq, hdk, hdv = pinned(dq), pinned(dk), pinned(dvv)
    q, k, v = hq.to(dev), hk.to(dev), hv.to(dev)
    qd, kd, vd = hdq.to(dev), hdk.to(dev), hdv.to(dev)
    o_quad = torch.empty((B, H, T, dv), dtype=bf, device=dev)
    o_chunk = torch.empty_like(o_quad)
    o_dec = torch.empty((B, H, dv), dtype=bf, device=dev)
    S = torch.empty((B, H, p * p, dv), dtype=torch.float32, device=dev)
    z = torch.empty((B, H, p * p), dtype=torch.float32, device=dev)
    ws = torch.empty(max(256, K.kata_fwd_chunked_workspace_size(B, H, T, p, dv, C, bf)), dtype=torch.uint8,
                     device=dev)
    flush = L2Flush(torch, dev)
    stream = torch.cuda.current_stream(dev)

    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    def step(times=None):
        e = [ev() for _ in range(4)] if times is not None else None
        if e: e[0].record(stream)
        K.kata_fwd_quadratic(q, k, v, o=o_quad)
        if e: e[1].record(stream)
        K.kata_fwd_chunked(q, k, v, C=C, o=o_chunk, workspace=ws, S_out=S, z_out=z, return_state=True)
        if e: e[2].record(stream)
        K.kata_decode_step(qd, kd, vd, S, z, o=o_dec)
        if e: e[3].record(stream)
        if times is not None:
            times.append(e)

    for _ in range(args.warmup):
        step()
        flush()
    torch.cuda.synchronize()
    if K.kata_get_status() != 0:
        raise RuntimeError("kernel reported a wait timeout during warm-up")

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    # the step captured once as a CUDA graph (the same three calls, the same
    # buffers): replaying it launches the step's kernels without the host
    # launch path between them
    graph = None
    if args.graph:
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step()
        stream.wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        torch.cuda.synchronize()
        for _ in range(args.warmup):
            graph.replay()
            flush()
        torch.cuda.synchronize()

    recs, grecs = [], []
    windows = {}
    clk = ClockSampler(local_rank)
    clk.__enter__()
    try:  # the clock record covers every timed part below
        clk.wait_first_sample()
        barrier()
        torch.cuda.synchronize()
        t_start = time.time()
        # per-path times: the calls launched one by one, events between them
        for _ in range(args.steps):
            step(recs)
            flush()
        # the step as a whole: graph replays
        if graph is not None:
            for _ in range(args.steps):
                a, b = ev(), ev()
                a.record(stream)
                graph.replay()
                b.record(stream)
                flush()
                grecs.append((a, b))
        torch.cuda.synchronize()
        windows["step"] = (t_start, time.time())
        barrier()
        per = np.array([[r[0].elapsed_time(r[1]), r[1].elapsed_time(r[2]), r[2].elapsed_time(r[3])] for r in recs])
        eager_step_ms = float(per.sum(axis=1).mean())
        step_ms = float(np.mean([a.elapsed_time(b) for a, b in grecs])) if grecs else eager_step_ms
        path_ms = per.mean(axis=0)
        if graph is not None:
            del graph

        # end to end through the public API with host buffers.  Every step copies
        # its inputs host -> device from pinned memory, runs the three calls and
        # copies its three outputs device -> host.  Steps are pipelined over three
        # streams with two sets of device buffers: the H2D copy of step i, the
        # compute of step i-1 and the D2H copy of step i-2 overlap (PCIe is full
        # duplex and the copy engines run beside the SMs).  The L2 is flushed on
        # the compute stream before every step.
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hdq, hdk, hdv))
        d2h = sum(t.numel() * t.element_size() for t in (o_quad, o_chunk, o_dec))
        sets = []
        for _b in range(2):
            sets.append(dict(
                q=torch.empty_like(q), k=torch.empty_like(k), v=torch.empty_like(v),
                qd=torch.empty_like(qd), kd=torch.empty_like(kd), vd=torch.empty_like(vd),
                oq=torch.empty_like(o_quad), oc=torch.empty_like(o_chunk), od=torch.empty_like(o_dec),
                S=torch.empty_like(S), z=torch.empty_like(z), ws=torch.empty_like(ws),
                hoq=torch.empty(o_quad.shape, dtype=bf).pin_memory(), hoc=torch.empty(o_chunk.shape, dtype=bf).pin_memory(),
                hod=torch.empty(o_dec.shape, dtype=bf).pin_memory()))
        s_h2d, s_cmp, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_cmp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_run(nsteps):
            for i in range(nsteps):
                bi = i % 2
                st_ = sets[bi]
                with torch.cuda.stream(s_h2d):
                    if i >= 2:
                        s_h2d.wait_event(ev_cmp[bi])  # step i-2 has finished reading this set's inputs
                    for dst, src in ((st_["q"], hq), (st_["k"], hk), (st_["v"], hv), (st_["qd"], hdq), (st_["kd"], hdk),
                                     (st_["vd"], hdv)):
                        dst.copy_(src, non_blocking=True)
                    ev_in[bi].record(s_h2d)
                with torch.cuda.stream(s_cmp):
                    s_cmp.wait_event(ev_in[bi])
                    if i >= 2:
                        s_cmp.wait_event(ev_out[bi])  # step i-2's outputs have been copied out
                    flush()
                    K.kata_fwd_quadratic(st_["q"], st_["k"], st_["v"], o=st_["oq"])
                    K.kata_fwd_chunked(st_["q"], st_["k"], st_["v"], C=C, o=st_["oc"], workspace=st_["ws"],
                                       S_out=st_["S"], z_out=st_["z"], return_state=True)
                    K.kata_decode_step(st_["qd"], st_["kd"], st_["vd"], st_["S"], st_["z"], o=st_["od"])
                    ev_cmp[bi].record(s_cmp)
                with torch.cuda.stream(s_d2h):
                    s_d2h.wait_event(ev_cmp[bi])
                    st_["hoq"].copy_(st_["oq"], non_blocking=True)
                    st_["hoc"].copy_(st_["oc"], non_blocking=True)
                    st_["hod"].copy_(st_["od"], non_blocking=True)
                    ev_out[bi].record(s_d2h)

        e2e_run(4)
        torch.cuda.synchronize()
        n_e2e = min(40, max(8, args.steps // 2))
        e_start, e_end = ev(), ev()
        e_start.record(s_h2d)
        s_cmp.wait_stream(s_h2d)
        s_d2h.wait_stream(s_h2d)
        e2e_run(n_e2e)
        s_d2h.wait_stream(s_cmp)
        s_d2h.wait_stream(s_h2d)
        e_end.record(s_d2h)
        torch.cuda.synchronize()
        e2e_ms = e_start.elapsed_time(e_end) / n_e2e

        # long context: chunked (and quadratic) at T = 131072, and the decode
        # step at the serving batch; each timed inside the clock record
        long = None
        if args.long and world == 1:
            t0 = time.time()
            long = run_long(args, K, torch, dev, stream, flush)
            windows["long_ctx"] = (t0, time.time())
            t0 = time.time()
            long["decode_b64"] = run_decode_b64(args, K, torch, dev, stream, flush)
            windows["decode_b64"] = (t0, time.time())
            if args.sweep:
                long["sweep"], long["recall"] = run_sweep(args, K, torch, dev, stream, flush)
                t0 = time.time()
                long["mg"] = run_mg(args, K, torch, dev, stream, flush)
                windows["mg"] = (t0, time.time())
                t0 = time.time()
                long["first_order"] = run_first_order(args, K, torch, dev, stream, flush)
                windows["first_order"] = (t0, time.time())
                t0 = time.time()
                long["train"] = run_train(args, K, torch, dev, stream, flush)
                windows["train"] = (t0, time.time())
        t_end = time.time()
        time.sleep(0.15)
        clk.window = (windows["step"][0], windows.get("decode_b64", windows["step"])[1])
        status = K.kata_get_status()
        return dict(step_ms=step_ms, eager_step_ms=eager_step_ms, graph=bool(args.graph), path_ms=path_ms.tolist(),
                    e2e_ms=e2e_ms, h2d=h2d, d2h=d2h, clocks=clk.summary(),
                    clocks_by_part={name: clk.summary(w) for name, w in windows.items()},
                    timed_s=t_end - windows["step"][0], long=long, status=status, tokens=B * T, BH=BH, T=T, p=p, dv=dv,
                    C=C)
    finally:
        clk.__exit__()


def run_decode_b64(args, K, torch, dev, stream, flush):
    """The decode step alone at the batched-serving size (B=64, H=16, state [256 x 64] fp32)."""
    c = workloads.DECODE
    q, k, v, S, z = workloads.decode_inputs(c["B"], c["H"], c["p"], c["dv"], seed=c["seed"], dtype=c["dtype"])
    bf = torch.bfloat16
    qd, kd, vd = (torch.from_numpy(x).to(dev, bf) for x in (q, k, v))
    Sd, zd = torch.from_numpy(S).to(dev), torch.from_numpy(z).to(dev)
    o = torch.empty((c["B"], c["H"], c["dv"]), dtype=bf, device=dev)
    ms = []
    for i in range(5 + args.long_steps * 4):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        K.kata_decode_step(qd, kd, vd, Sd, zd, o=o)
        b.record(stream)
        torch.cuda.synchronize()
        if i >= 5:
            ms.append(a.elapsed_time(b))
    return dict(ms=float(np.mean(ms)), B=c["B"], H=c["H"], p=c["p"], dv=c["dv"])


def run_long(args, K, torch, dev, stream, flush):
    cfg = workloads.CONFIGS["long_ctx131k"]
    B, H, T, p, dv = cfg["B"], cfg["H"], cfg["T"], cfg["p"], cfg["dv"]
    qn, kn, vn = workloads.make_inputs(cfg)
    bf = torch.bfloat16
    q = torch.from_numpy(qn).to(dev, bf)
    k = torch.from_numpy(kn).to(dev, bf)
    v = torch.from_numpy(vn).to(dev, bf)
    o = torch.empty((B, H, T, dv), dtype=bf, device=dev)
    out = {}
    for C in (64, 128):
        ws = torch.empty(max(256, K.kata_fwd_chunked_workspace_size(B, H, T, p, dv, C, bf)), dtype=torch.uint8,
                         device=dev)
        ms = []
        for i in range(3 + args.long_steps):
            flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            K.kata_fwd_chunked(q, k, v, C=C, o=o, workspace=ws)
            b.record(stream)
            torch.cuda.synchronize()
            if i >= 3:
                ms.append(a.elapsed_time(b))
        out["chunked_C%d_ms" % C] = float(np.mean(ms))
    # sequential inter-chunk baseline: one CTA per (b,h) walks all chunks
    out["sequential_C64_ms"] = _time_call(lambda: K.kata_fwd_chunked_sequential(q, k, v, C=64, o=o), flush, stream,
                                          3, 1)
    ms = []
    for i in range(2 + max(1, args.long_steps // 4)):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        K.kata_fwd_quadratic(q, k, v, o=o)
        b.record(stream)
        torch.cuda.synchronize()
        if i >= 2:
            ms.append(a.elapsed_time(b))
    out["quadratic_ms"] = float(np.mean(ms))
    out.update(B=B, H=H, T=T, p=p, dv=dv)
    return out


class L2Flush:
    """Empties the 126 MB L2 between timed calls: a 512 MiB write evicts
    whatever the last call left, then a 256 MiB read replaces the written
    (dirty) lines with clean ones, so that the next timed kernel neither
    finds its data in L2 nor pays for writing the flush buffer back to HBM
    (for the decode step, ~126 MB of write-back against its 136 MB of state
    traffic).  Runs outside the timed events."""

    def __init__(self, torch, dev):
        self.w = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)
        self.r = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device=dev)
        self.acc = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.fill_(1)
        self.acc.copy_(self.r.sum())


def _time_call(fn, flush, stream, reps, warm):
    import torch
    ms = []
    for i in range(warm + reps):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        if i >= warm:
            ms.append(a.elapsed_time(b))
    return float(np.mean(ms))


def run_sweep(args, K, torch, dev, stream, flush):
    """Throughput grid B x T (H=16, p=16, dv=64, bf16) for both paths, and the
    recall-shaped p=32 workload.  Sweep inputs are drawn on the device from a
    seeded generator (q, k L2-normalised N(0,1), v N(0,1)): the times do not
    depend on the values, and the largest point would take minutes to draw on
    the host."""
    bf = torch.bfloat16
    H, p, dv, C = 16, 16, 64, 64
    gen = torch.Generator(device=dev)
    grid = []
    for B in (1, 4, 16):
        for T in (1024, 4096, 16384, 65536, 131072):
            gen.manual_seed(1000 * B + T % 997)
            q = torch.randn((B, H, T, p), generator=gen, device=dev)
            k = torch.randn((B, H, T, p), generator=gen, device=dev)
            q = (q / q.norm(dim=-1, keepdim=True)).to(bf)
            k = (k / k.norm(dim=-1, keepdim=True)).to(bf)
            v = torch.randn((B, H, T, dv), generator=gen, device=dev).to(bf)
            o = torch.empty((B, H, T, dv), dtype=bf, device=dev)
            need = K.kata_fwd_chunked_workspace_size(B, H, T, p, dv, C, bf)
            ws = torch.empty(max(256, need), dtype=torch.uint8, device=dev)
            c_ms = _time_call(lambda: K.kata_fwd_chunked(q, k, v, C=C, o=o, workspace=ws), flush, stream, 3, 2)
            heavy = B * T * T > 4 * 131072 * 131072
            q_ms = _time_call(lambda: K.kata_fwd_quadratic(q, k, v, o=o), flush, stream, 1 if heavy else 3, 1)
            grid.append(dict(B=B, T=T, chunked_ms=c_ms, quadratic_ms=q_ms))
            del q, k, v, o, ws
    torch.cuda.empty_cache()
    cfg = workloads.CONFIGS["recall_p32"]
    B, H, T, p, dv = cfg["B"], cfg["H"], cfg["T"], cfg["p"], cfg["dv"]
    qn, kn, vn = workloads.make_inputs(cfg)
    q, k, v = (torch.from_numpy(x).to(dev, bf) for x in (qn, kn, vn))
    o = torch.empty((B, H, T, dv), dtype=bf, device=dev)
    ws = torch.empty(max(256, K.kata_fwd_chunked_workspace_size(B, H, T, p, dv, cfg["C"], bf)), dtype=torch.uint8,
                     device=dev)
    recall = dict(B=B, H=H, T=T, p=p, dv=dv,
                  chunked_ms=_time_call(lambda: K.kata_fwd_chunked(q, k, v, C=cfg["C"], o=o, workspace=ws), flush,
                                        stream, 3, 1),
                  quadratic_ms=_time_call(lambda: K.kata_fwd_quadratic(q, k, v, o=o), flush, stream, 3, 1))
    return grid, recall


def run_first_order(args, K, torch, dev, stream, flush):
    """First-order attention (psi(u) = u, d=16, dv=64, H=16, bf16): the
    chunked form with the associative scan against the matched sequential
    baseline (one CTA per sequence) over a batch x length grid, the pages'
    Figure 3 comparison.  Inputs are drawn on the device: q, k nonnegative
    unit vectors (|N(0,1)| normalised), v N(0,1)."""
    bf = torch.bfloat16
    H, d, dv, C = 16, 16, 64, 64
    gen = torch.Generator(device=dev)
    grid = []
    for B in (1, 4, 16):
        for T in (2048, 8192, 32768, 131072):
            gen.manual_seed(2000 * B + T % 991)
            q = torch.randn((B, H, T, d), generator=gen, device=dev).abs()
            k = torch.randn((B, H, T, d), generator=gen, device=dev).abs()
            q = (q / q.norm(dim=-1, keepdim=True)).to(bf)
            k = (k / k.norm(dim=-1, keepdim=True)).to(bf)
            v = torch.randn((B, H, T, dv), generator=gen, device=dev).to(bf)
            o = torch.empty((B, H, T, dv), dtype=bf, device=dev)
            ws = torch.empty(max(256, K.kata_fwd_linear_chunked_workspace_size(B, H, T, d, dv, C)),
                             dtype=torch.uint8, device=dev)
            s_ms = _time_call(lambda: K.kata_fwd_linear_chunked(q, k, v, C=C, o=o, workspace=ws), flush, stream, 3, 1)
            q_ms = _time_call(lambda: K.kata_fwd_linear_chunked_sequential(q, k, v, C=C, o=o), flush, stream, 3, 1)
            grid.append(dict(B=B, H=H, T=T, d=d, dv=dv, scan_ms=s_ms, sequential_ms=q_ms))
            del q, k, v, o, ws
    torch.cuda.empty_cache()
    return grid


def run_mg(args, K, torch, dev, stream, flush):
    """KATA-Mg forward (several PSD factors per head) on the workloads of
    workloads.MG_CONFIGS: the 340M model's d = 64 heads in 2 or 4 groups at
    T = 2048, in the [B,T,H,d] layout of the pages' attention call."""
    bf = torch.bfloat16
    out = {}
    for name, cfg in sorted(workloads.MG_CONFIGS.items()):
        B, H, T, d, g, dv = cfg["B"], cfg["H"], cfg["T"], cfg["d"], cfg["groups"], cfg["dv"]
        qn, kn, vn = workloads.normal_qkv(B, H, T, d, dv, seed=cfg["seed"], dtype=cfg["dtype"])
        q, k, v = (torch.from_numpy(np.ascontiguousarray(x.transpose(0, 2, 1, 3))).to(dev, bf) for x in (qn, kn, vn))
        o = torch.empty_like(v)
        ms = _time_call(lambda: K.kata_fwd_mg_quadratic(q, k, v, g, layout=cfg["layout"], o=o), flush, stream, 10, 3)
        out[name] = dict(B=B, H=H, T=T, d=d, groups=g, dv=dv, layout=cfg["layout"], ms=ms)
        # the chunked (O(T)) KATA-Mg path on the same inputs
        ws = torch.empty(max(256, K.kata_fwd_mg_chunked_workspace_size(B, H, T, d, g, dv, 64)), dtype=torch.uint8,
                         device=dev)
        ms_c = _time_call(lambda: K.kata_fwd_mg_chunked(q, k, v, g, C=64, layout=cfg["layout"], o=o, workspace=ws),
                          flush, stream, 10, 3)
        out["chunked_" + name] = dict(B=B, H=H, T=T, d=d, groups=g, dv=dv, layout=cfg["layout"], ms=ms_c,
                                      chunked=True)
        # KATA-Sigma-g (summed factors) on the same inputs: g^2 score blocks
        ms_sg = _time_call(lambda: K.kata_fwd_sg_quadratic(q, k, v, g, layout=cfg["layout"], o=o), flush, stream, 10,
                           3)
        out["sg" + name[2:]] = dict(B=B, H=H, T=T, d=d, groups=g, dv=dv, layout=cfg["layout"], ms=ms_sg, summed=True)
        del q, k, v, o
    # the chunked path at the long context (B = 1, H = 16, T = 131072), where
    # the flash-style path costs seconds; device-drawn inputs
    gen_l = torch.Generator(device=dev)
    for g in (2, 4):
        B, H, T, d, dv = 1, 16, 131072, 64, 64
        gen_l.manual_seed(500 + g)
        q = torch.randn((B, T, H, d), generator=gen_l, device=dev)
        k = torch.randn((B, T, H, d), generator=gen_l, device=dev)
        q = (q / q.norm(dim=-1, keepdim=True)).to(bf)
        k = (k / k.norm(dim=-1, keepdim=True)).to(bf)
        v = torch.randn((B, T, H, dv), generator=gen_l, device=dev).to(bf)
        o = torch.empty_like(v)
        ws = torch.empty(max(256, K.kata_fwd_mg_chunked_workspace_size(B, H, T, d, g, dv, 64)), dtype=torch.uint8,
                         device=dev)
        ms_c = _time_call(lambda: K.kata_fwd_mg_chunked(q, k, v, g, C=64, layout="bthd", o=o, workspace=ws), flush,
                          stream, 5, 2)
        out["chunked_mg%d_ctx131k" % g] = dict(B=B, H=H, T=T, d=d, groups=g, dv=dv, layout="bthd", ms=ms_c,
                                               chunked=True)
        del q, k, v, o, ws
    # KATA-Sigma-g on the chunked path (groups of 16: d = 64 in 4 groups),
    # [B,H,T,d], at T = 2048 (B = 8) and T = 131072 (B = 1)
    for B, T in ((8, 2048), (1, 131072)):
        H, d, g, dv = 16, 64, 4, 64
        gen_l.manual_seed(600 + B)
        q = torch.randn((B, H, T, d), generator=gen_l, device=dev)
        k = torch.randn((B, H, T, d), generator=gen_l, device=dev)
        q = (q / q.norm(dim=-1, keepdim=True)).to(bf)
        k = (k / k.norm(dim=-1, keepdim=True)).to(bf)
        v = torch.randn((B, H, T, dv), generator=gen_l, device=dev).to(bf)
        o = torch.empty_like(v)
        ws = torch.empty(max(256, K.kata_fwd_sg_chunked_workspace_size(B, H, T, d, g, dv, 64)), dtype=torch.uint8,
                         device=dev)
        ms_c = _time_call(lambda: K.kata_fwd_sg_chunked(q, k, v, g, C=64, o=o, workspace=ws), flush, stream, 5, 2)
        out["chunked_sg%d_ctx%s" % (g, "2k" if T == 2048 else "131k")] = dict(
            B=B, H=H, T=T, d=d, groups=g, dv=dv, layout="bhtd", ms=ms_c, chunked=True, summed=True)
        del q, k, v, o, ws
    # decode step on the concatenated per-group state (B = 64, as for the
    # single-factor decode line): HBM-bound, the state is read and written once
    gen = torch.Generator(device=dev)
    gen.manual_seed(77)
    for g in (2, 4):
        B, H, d, dv = 64, 16, 64, 64
        P = g * (d // g) ** 2
        q = torch.randn((B, H, d), generator=gen, device=dev).to(bf)
        k = torch.randn((B, H, d), generator=gen, device=dev).to(bf)
        v = torch.randn((B, H, dv), generator=gen, device=dev).to(bf)
        S = torch.randn((B, H, P, dv), generator=gen, device=dev)
        z = torch.rand((B, H, P), generator=gen, device=dev) + 0.5
        o = torch.empty((B, H, dv), dtype=bf, device=dev)
        ms = _time_call(lambda: K.kata_decode_step_mg(q, k, v, S, z, g, o=o), flush, stream, 20, 3)
        out["decode_mg%d_b64" % g] = dict(B=B, H=H, d=d, groups=g, dv=dv, P=P, ms=ms)
        # KATA-Sigma-g: the summed feature's state has the single factor's
        # (d/g)^2 rows
        Ps = (d // g) ** 2
        Ss, zs = S[:, :, :Ps].contiguous(), z[:, :, :Ps].contiguous()
        ms = _time_call(lambda: K.kata_decode_step_sg(q, k, v, Ss, zs, g, o=o), flush, stream, 20, 3)
        out["decode_sg%d_b64" % g] = dict(B=B, H=H, d=d, groups=g, dv=dv, P=Ps, ms=ms, summed=True)
        del q, k, v, S, z, o, Ss, zs
    return out


def run_train(args, K, torch, dev, stream, flush):
    """Training step of the flash path on the bench workload's shape (B8 H16
    T2048 p16 dv64, bf16): the forward that saves the denominators, then the
    backward pass for an upstream gradient; device-drawn inputs."""
    bf = torch.bfloat16
    B, H, T, p, dv = 8, 16, 2048, 16, 64
    gen = torch.Generator(device=dev)
    gen.manual_seed(99)
    q = torch.randn((B, H, T, p), generator=gen, device=dev)
    k = torch.randn((B, H, T, p), generator=gen, device=dev)
    q = (q / q.norm(dim=-1, keepdim=True)).to(bf)
    k = (k / k.norm(dim=-1, keepdim=True)).to(bf)
    v = torch.randn((B, H, T, dv), generator=gen, device=dev).to(bf)
    dO = torch.randn((B, H, T, dv), generator=gen, device=dev).to(bf)
    o, D = K.kata_fwd_quadratic_train(q, k, v)
    ws = torch.empty(max(256, int(K.lib().kata_bwd_quadratic_workspace_size(B, H, T, p, dv, 1))), dtype=torch.uint8,
                     device=dev)
    fwd_ms = _time_call(lambda: K.kata_fwd_quadratic_train(q, k, v, o=o, D=D), flush, stream, 10, 3)
    bwd_ms = _time_call(lambda: K.kata_bwd_quadratic(q, k, v, o, D, dO, workspace=ws), flush, stream, 10, 3)

    def step():
        K.kata_fwd_quadratic_train(q, k, v, o=o, D=D)
        K.kata_bwd_quadratic(q, k, v, o, D, dO, workspace=ws)
    step_ms = _time_call(step, flush, stream, 10, 3)
    out = dict(B=B, H=H, T=T, p=p, dv=dv, fwd_ms=fwd_ms, bwd_ms=bwd_ms, step_ms=step_ms)
    # the O(T) chunked training path on the same inputs, and alone at the
    # long context (B1 H16 T131072, where the O(T^2) backward takes seconds)
    chunked = {}
    for (Bc, Tc) in ((B, T), (1, 131072)):
        if (Bc, Tc) != (B, T):
            gen.manual_seed(98)
            q = torch.randn((Bc, H, Tc, p), generator=gen, device=dev)
            k = torch.randn((Bc, H, Tc, p), generator=gen, device=dev)
            q = (q / q.norm(dim=-1, keepdim=True)).to(bf)
            k = (k / k.norm(dim=-1, keepdim=True)).to(bf)
            v = torch.randn((Bc, H, Tc, dv), generator=gen, device=dev).to(bf)
            dO = torch.randn((Bc, H, Tc, dv), generator=gen, device=dev).to(bf)
        oc = torch.empty_like(v)
        Dc = torch.empty((Bc, H, Tc), dtype=torch.float32, device=dev)
        wsf = torch.empty(max(256, K.kata_fwd_chunked_workspace_size(Bc, H, Tc, p, dv, 64, bf)), dtype=torch.uint8,
                          device=dev)
        wsb = torch.empty(max(256, int(K.lib().kata_bwd_chunked_workspace_size(Bc, H, Tc, p, dv, 1))),
                          dtype=torch.uint8, device=dev)
        c_fwd = _time_call(lambda: K.kata_fwd_chunked_train(q, k, v, o=oc, D=Dc, workspace=wsf), flush, stream, 5, 2)
        c_bwd = _time_call(lambda: K.kata_bwd_chunked(q, k, v, oc, Dc, dO, workspace=wsb), flush, stream, 5, 2)
        chunked["B%d_T%d" % (Bc, Tc)] = dict(B=Bc, H=H, T=Tc, fwd_ms=c_fwd, bwd_ms=c_bwd, step_ms=c_fwd + c_bwd)
        del oc, Dc, wsf, wsb
    out["chunked"] = chunked
    return out


# ---------------------------------------------------------------------------
# reference arm: the fp64 CPU oracle on the host cores
# ---------------------------------------------------------------------------
def time_oracle(cfg, budget_s=15.0):
    """Oracle (psi recurrence, all host threads) on whole (b,h) sequences of the
    workload until about budget_s of CPU time; returns tokens/s and the sample."""
    import oracle
    B, H, T, p, dv = cfg["B"], cfg["H"], cfg["T"], cfg["p"], cfg["dv"]
    threads = oracle.default_threads()
    q, k, v = workloads.make_inputs(dict(cfg, B=1))
    # probe one head to size the sample
    t0 = time.perf_counter()
    oracle.recurrent(q[:, :1], k[:, :1], v[:, :1], nthreads=1)
    one = max(time.perf_counter() - t0, 1e-3)
    n_heads = int(max(1, min(B * H, budget_s / one * threads * 0.8)))
    n_heads = max(threads, (n_heads // threads) * threads) if n_heads >= threads else n_heads
    reps = (n_heads + H - 1) // H
    qs = np.concatenate([q] * reps, axis=0).reshape(-1, 1, T, p)[:n_heads]
    ks = np.concatenate([k] * reps, axis=0).reshape(-1, 1, T, p)[:n_heads]
    vs = np.concatenate([v] * reps, axis=0).reshape(-1, 1, T, dv)[:n_heads]
    t0 = time.perf_counter()
    oracle.recurrent(qs, ks, vs, nthreads=0)
    dt = time.perf_counter() - t0
    tokens = n_heads * T / H  # token-heads -> tokens of an H-head batch
    return dict(value=tokens / dt, cores=threads, seconds=dt,
                sample="oracle psi recurrence (fp64) over %d whole (b,h) sequences of T=%d" % (n_heads, T))


def run_reference(args, rank, world):
    if rank != 0:
        return
    cfg = workloads.CONFIGS[args.workload]
    vals = []
    for _ in range(args.warmup):
        time_oracle(cfg, budget_s=2.0)
    for _ in range(args.steps):
        vals.append(time_oracle(cfg, budget_s=args.ref_budget))
    value = float(np.mean([x["value"] for x in vals]))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": float(np.mean([x["seconds"] for x in vals]) * 1e3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(cfg, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": vals[0]["cores"], "kind": "oracle",
                         "sample": vals[0]["sample"]},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# --case: one call of the library a few times on device-drawn inputs, for
# profilers (ncu wants a short program that launches the kernel of interest a
# known number of times); nothing is timed or printed but the call's status
# ---------------------------------------------------------------------------
def run_case(args):
    import torch
    import kernelized_feature_map_b200 as K

    dev = torch.device("cuda")
    gen = torch.Generator(device=dev)
    gen.manual_seed(args.seed)
    bf = torch.bfloat16

    def unit(shape):
        x = torch.randn(shape, generator=gen, device=dev)
        return (x / x.norm(dim=-1, keepdim=True)).to(bf)

    B, H, T, d, dv, g = args.B, args.H, args.T, args.d, args.dv, args.groups
    if args.case == "decode":
        p = d // g
        q, k = unit((B, H, d)), unit((B, H, d))
        v = torch.randn((B, H, dv), generator=gen, device=dev).to(bf)
        S = torch.zeros((B, H, g * p * p, dv), dtype=torch.float32, device=dev)
        z = torch.zeros((B, H, g * p * p), dtype=torch.float32, device=dev)
        call = lambda: K.kata_decode_step_mg(q, k, v, S, z, g)  # noqa: E731
    else:
        lead = (B, T, H) if args.layout == "bthd" else (B, H, T)
        q, k = unit(lead + (d,)), unit(lead + (d,))
        v = torch.randn(lead + (dv,), generator=gen, device=dev).to(bf)
        o = torch.empty_like(v)
        if args.case == "mg":
            call = lambda: K.kata_fwd_mg_quadratic(q, k, v, g, layout=args.layout, o=o)  # noqa: E731
        elif args.case == "mg_chunked":
            ws = torch.empty(max(256, K.kata_fwd_mg_chunked_workspace_size(B, H, T, d, g, dv, args.C, bf)),
                             dtype=torch.uint8, device=dev)
            call = lambda: K.kata_fwd_mg_chunked(q, k, v, g, C=args.C, layout=args.layout, o=o,  # noqa: E731
                                                 workspace=ws)
        elif args.layout != "bhtd":
            raise SystemExit("--layout bthd is for --case mg")
        elif args.case == "quadratic":
            call = lambda: K.kata_fwd_quadratic(q, k, v, o=o)  # noqa: E731
        elif args.case == "sg_chunked":
            ws = torch.empty(max(256, K.kata_fwd_sg_chunked_workspace_size(B, H, T, d, g, dv, args.C)),
                             dtype=torch.uint8, device=dev)
            call = lambda: K.kata_fwd_sg_chunked(q, k, v, g, C=args.C, o=o, workspace=ws)  # noqa: E731
        elif args.case == "chunked_train":
            dO = torch.randn(v.shape, generator=gen, device=dev).to(bf)
            D = torch.empty((B, H, T), dtype=torch.float32, device=dev)
            wsf = torch.empty(max(256, K.kata_fwd_chunked_workspace_size(B, H, T, d, dv, args.C, bf)),
                              dtype=torch.uint8, device=dev)
            wsb = torch.empty(max(256, int(K.lib().kata_bwd_chunked_workspace_size(B, H, T, d, dv, 1))),
                              dtype=torch.uint8, device=dev)

            def call():
                K.kata_fwd_chunked_train(q, k, v, C=args.C, o=o, D=D, workspace=wsf)
                K.kata_bwd_chunked(q, k, v, o, D, dO, workspace=wsb)
        elif args.case == "linear":
            q, k = q.abs(), k.abs()  # nonnegative unit vectors: sign-definite denominators
            ws = torch.empty(max(256, K.kata_fwd_linear_chunked_workspace_size(B, H, T, d, dv, args.C)),
                             dtype=torch.uint8, device=dev)
            call = lambda: K.kata_fwd_linear_chunked(q, k, v, C=args.C, o=o, workspace=ws)  # noqa: E731
        elif args.case == "linear_sequential":
            q, k = q.abs(), k.abs()
            call = lambda: K.kata_fwd_linear_chunked_sequential(q, k, v, C=args.C, o=o)  # noqa: E731
        elif args.case == "train":
            dO = torch.randn(v.shape, generator=gen, device=dev).to(bf)
            D = torch.empty((B, H, T), dtype=torch.float32, device=dev)

            def call():
                K.kata_fwd_quadratic_train(q, k, v, o=o, D=D)
                K.kata_bwd_quadratic(q, k, v, o, D, dO)
        else:
            ws = torch.empty(max(256, K.kata_fwd_chunked_workspace_size(B, H, T, d, dv, args.C, bf)),
                             dtype=torch.uint8, device=dev)
            call = lambda: K.kata_fwd_chunked(q, k, v, C=args.C, o=o, workspace=ws)  # noqa: E731
    for _ in range(args.reps):
        call()
    torch.cuda.synchronize()
    status = K.kata_get_status()
    print("%s reps=%d status=%d (%s)" % (args.case, args.reps, status, K.status_string(status)))
    return 0 if status == 0 else 1


def config_dict(cfg, world):
    return {"workload": "%s: B=%d H=%d T=%d p=%d dv=%d C=%d bf16" % (
        "340M-layer shape" if cfg["T"] == 2048 else cfg.get("kind", ""), cfg["B"], cfg["H"], cfg["T"], cfg["p"],
        cfg["dv"], cfg["C"]),
        "B": cfg["B"], "H": cfg["H"], "T": cfg["T"], "p": cfg["p"], "dv": cfg["dv"], "C": cfg["C"],
        "step": "kata_fwd_quadratic + kata_fwd_chunked(final state) + kata_decode_step",
        "launch": "step timed as a CUDA graph replay of the three calls; per-path times launched one by one",
        "l2": "flushed between timed steps outside the timed events: a 512 MiB write, then a 256 MiB read so "
              "that the lines left in L2 are clean",
        "parallelism": "independent (b,h) batches per rank, no collective" if world > 1 else "1 GPU"}


def main():
    ap = argparse.ArgumentParser(description="KATA forward hot-path benchmark")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="layer340m_ctx2k", choices=sorted(workloads.CONFIGS))
    ap.add_argument("--long", type=int, default=1, help="also time the T=131072 workload (1 GPU)")
    ap.add_argument("--long-steps", type=int, default=8)
    ap.add_argument("--sweep", type=int, default=1, help="also time the B x T grid and the p=32 recall workload")
    ap.add_argument("--cpu-baseline", type=int, default=1)
    ap.add_argument("--graph", type=int, default=1, help="time the step as a CUDA graph replay (per-path times stay eager)")
    ap.add_argument("--ref-budget", type=float, default=15.0, help="seconds of oracle work per reference step")
    pc = ap.add_argument_group("--case: launch one call a few times on device-drawn inputs (for profilers)")
    pc.add_argument("--case", choices=["quadratic", "chunked", "mg", "mg_chunked", "decode", "train", "linear",
                                       "linear_sequential", "sg_chunked", "chunked_train"])
    pc.add_argument("--B", type=int, default=8)
    pc.add_argument("--H", type=int, default=16)
    pc.add_argument("--T", type=int, default=2048)
    pc.add_argument("--d", type=int, default=16, help="q/k width (p for the single-factor paths)")
    pc.add_argument("--dv", type=int, default=64)
    pc.add_argument("--groups", type=int, default=1)
    pc.add_argument("--layout", choices=["bhtd", "bthd"], default="bhtd")
    pc.add_argument("--C", type=int, default=64)
    pc.add_argument("--reps", type=int, default=3)
    pc.add_argument("--seed", type=int, default=0)
    args = ap.parse_args()
    if args.case:
        sys.exit(run_case(args))
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        if args.impl == "ours":
            torch.cuda.set_device(local_rank)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local_rank))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=600))

    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
            return
        res = run_ours(args, rank, world, local_rank)
        step_ms = res["step_ms"]
        e2e_ms = res["e2e_ms"]
        step_ms, e2e_ms = reduce_max([step_ms, e2e_ms], world, device="cuda")
        if rank != 0:
            return
        report(args, res, step_ms, e2e_ms, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


def roofline_points(res, peaks, cfg):
    """Each path of the metric on its own: tokens/s and the fraction of its
    binding roofline at T = 2048 (the step's batch, eager per-path times) and
    at T = 131072 (chunked C = 64 and 128, and quadratic), plus the decode
    step at B = 64; each with the clocks sampled while it was timed."""
    hb, tf = peaks["hbm_gbs"], peaks["bf16_tflops"]
    cl = res.get("clocks_by_part", {})
    BH, T, p, dv = res["BH"], res["T"], res["p"], res["dv"]
    tok = res["tokens"]
    quad_ms, chunk_ms, _ = res["path_ms"]

    def hbm_point(path, workload, ms, tokens, nbytes, clocks, **kw):
        gbs = nbytes / (ms * 1e-3) / 1e9
        return dict(path=path, workload=workload, ms=ms, tokens_per_s=tokens / (ms * 1e-3), bound="hbm",
                    achieved=gbs, peak=hb, unit="GB/s", frac=gbs / hb, clocks=clocks, **kw)

    def tensor_point(path, workload, ms, tokens, flops, clocks, **kw):
        tfs = flops / (ms * 1e-3) / 1e12
        return dict(path=path, workload=workload, ms=ms, tokens_per_s=tokens / (ms * 1e-3), bound="tensor",
                    achieved=tfs, peak=tf, unit="TFLOP/s", frac=tfs / tf, clocks=clocks, **kw)

    w2k = "B=%d H=%d T=%d p=%d dv=%d bf16" % (BH // cfg["H"], cfg["H"], T, p, dv)
    pts = [tensor_point("quadratic", w2k, quad_ms, tok, flash_flops(BH, T, p, dv), cl.get("step"), T=T),
           hbm_point("chunked", w2k, chunk_ms, tok, chunked_bytes(BH, T, p, dv), cl.get("step"), T=T, C=res["C"])]
    lg = res.get("long")
    if lg:
        lbh, ltok = lg["B"] * lg["H"], lg["B"] * lg["T"]
        wl = "B=%d H=%d T=%d p=%d dv=%d bf16" % (lg["B"], lg["H"], lg["T"], lg["p"], lg["dv"])
        for C in (64, 128):
            pts.append(hbm_point("chunked", wl, lg["chunked_C%d_ms" % C], ltok,
                                 chunked_bytes(lbh, lg["T"], lg["p"], lg["dv"]), cl.get("long_ctx"), T=lg["T"], C=C))
        pts.append(tensor_point("quadratic", wl, lg["quadratic_ms"], ltok, flash_flops(lbh, lg["T"], lg["p"], lg["dv"]),
                                cl.get("long_ctx"), T=lg["T"]))
        dc = lg["decode_b64"]
        pts.append(hbm_point("decode", "decode step B=%d H=%d state [%d x %d] fp32" % (dc["B"], dc["H"], dc["p"] ** 2,
                                                                                     dc["dv"]),
                             dc["ms"], dc["B"], decode_bytes(dc["B"] * dc["H"], dc["p"], dc["dv"]),
                             cl.get("decode_b64")))
        # KATA-Mg itself (the metric's name): flash-style at T = 2048 and the
        # chunked path at T = 2048 and 131072, d = 64 in 2 or 4 groups
        for name, m in sorted(lg.get("mg", {}).items()):
            if "P" in m or (m.get("summed") and not m.get("chunked")):
                continue
            if m.get("summed"):
                wl = "KATA-Sigma-g B=%d H=%d T=%d d=%d groups=%d dv=%d bf16" % (m["B"], m["H"], m["T"], m["d"],
                                                                               m["groups"], m["dv"])
                pts.append(hbm_point("sg_chunked", wl, m["ms"], m["B"] * m["T"],
                                     m["B"] * m["H"] * m["T"] * (2 * m["d"] + 2 * m["dv"]) * 2, cl.get("mg"),
                                     T=m["T"], groups=m["groups"]))
                continue
            wl = "KATA-Mg B=%d H=%d T=%d d=%d groups=%d dv=%d bf16 [%s]" % (m["B"], m["H"], m["T"], m["d"],
                                                                          m["groups"], m["dv"], m["layout"])
            if m.get("chunked"):
                pts.append(hbm_point("mg_chunked", wl, m["ms"], m["B"] * m["T"],
                                     m["B"] * m["H"] * m["T"] * (2 * m["d"] + 2 * m["dv"]) * 2, cl.get("mg"),
                                     T=m["T"], groups=m["groups"]))
            else:
                pts.append(tensor_point("mg_quadratic", wl, m["ms"], m["B"] * m["T"],
                                        flash_flops(m["B"] * m["H"], m["T"], m["d"], m["dv"]), cl.get("mg"),
                                        T=m["T"], groups=m["groups"]))
        # the training backward passes: the flash path (tensor, 2(3p+2dv)
        # flops per causal pair) and the chunked path (HBM, 8p + 8dv + 4
        # bytes per token-head)
        tr = lg.get("train")
        if tr:
            wt = "backward B=%d H=%d T=%d p=%d dv=%d bf16" % (tr["B"], tr["H"], tr["T"], tr["p"], tr["dv"])
            pairs = tr["B"] * tr["H"] * tr["T"] * (tr["T"] + 1) / 2
            pts.append(tensor_point("bwd_quadratic", wt, tr["bwd_ms"], tr["B"] * tr["T"],
                                    pairs * 2 * (3 * tr["p"] + 2 * tr["dv"]), cl.get("train"), T=tr["T"]))
            for c in tr.get("chunked", {}).values():
                wc = "backward B=%d H=%d T=%d p=%d dv=%d bf16" % (c["B"], c["H"], c["T"], tr["p"], tr["dv"])
                pts.append(hbm_point("bwd_chunked", wc, c["bwd_ms"], c["B"] * c["T"],
                                     chunked_bwd_bytes(c["B"] * c["H"], c["T"], tr["p"], tr["dv"]), cl.get("train"),
                                     T=c["T"]))
        # first-order attention at B1 H16 T131072: both forms
        for g in lg.get("first_order", []):
            if g["B"] != 1 or g["T"] != 131072:
                continue
            wl = "first-order psi(u)=u B=%d H=%d T=%d d=%d dv=%d bf16" % (g["B"], g["H"], g["T"], g["d"], g["dv"])
            nbytes = g["B"] * g["H"] * g["T"] * (2 * g["d"] + 2 * g["dv"]) * 2
            pts.append(hbm_point("first_order_scan", wl, g["scan_ms"], g["B"] * g["T"], nbytes,
                                 cl.get("first_order"), T=g["T"]))
            pts.append(hbm_point("first_order_sequential", wl, g["sequential_ms"], g["B"] * g["T"], nbytes,
                                 cl.get("first_order"), T=g["T"]))
    return pts


def report(args, res, step_ms, e2e_ms, world):
    peaks, peak_src = load_peaks()
    cfg = workloads.CONFIGS[args.workload]
    BH, T, p, dv = res["BH"], res["T"], res["p"], res["dv"]
    tokens_all = res["tokens"] * world
    value = aggregate_value(res["tokens"], world, step_ms)
    quad_ms, chunk_ms, dec_ms = res["path_ms"]
    fl = flash_flops(BH, T, p, dv)
    achieved = fl / (quad_ms * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "ms_per_step_eager": res["eager_step_ms"],
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config_dict(cfg, world),
        "paths": {
            "quadratic": {"ms": quad_ms, "tokens_per_s": res["tokens"] / (quad_ms * 1e-3)},
            "chunked": {"ms": chunk_ms, "tokens_per_s": res["tokens"] / (chunk_ms * 1e-3),
                        "hbm_frac": chunked_bytes(BH, T, p, dv) / (chunk_ms * 1e-3) / 1e9 / peaks["hbm_gbs"]},
            "decode": {"ms": dec_ms, "tokens_per_s": (BH / cfg["H"]) / (dec_ms * 1e-3),
                       "hbm_frac": decode_bytes(BH, p, dv) / (dec_ms * 1e-3) / 1e9 / peaks["hbm_gbs"]},
        },
        "roofline": {"kernel": "flash_fwd_kernel (kata_fwd_quadratic)", "bound": "tensor", "achieved": achieved,
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                     "traffic": flash_traffic(args.workload), "peak_source": peak_src + " (bf16 burst)",
                     "algorithmic": "%.4g causal-useful flops per launch" % fl},
        "e2e": {"value": tokens_all / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": res["h2d"],
                "d2h_bytes_per_step": res["d2h"]},
        "gpu_launches": launches_per_step(BH // cfg["H"], cfg["H"], T, p, dv, cfg["C"]) * args.steps,
        "clocks": res["clocks"],
        "timed_region_s": res["timed_s"],
        "kernel_status": res["status"],
    }
    if res["long"]:
        lg = res["long"]
        lb = chunked_bytes(lg["B"] * lg["H"], lg["T"], lg["p"], lg["dv"])
        ltok = lg["B"] * lg["T"]
        lf = flash_flops(lg["B"] * lg["H"], lg["T"], lg["p"], lg["dv"])
        line["long_ctx"] = {
            "workload": "B=%d H=%d T=%d p=%d dv=%d bf16" % (lg["B"], lg["H"], lg["T"], lg["p"], lg["dv"]),
            "chunked_C64": {"ms": lg["chunked_C64_ms"], "tokens_per_s": ltok / (lg["chunked_C64_ms"] * 1e-3),
                            "hbm_frac": lb / (lg["chunked_C64_ms"] * 1e-3) / 1e9 / peaks["hbm_gbs"]},
            "chunked_C128": {"ms": lg["chunked_C128_ms"], "tokens_per_s": ltok / (lg["chunked_C128_ms"] * 1e-3),
                             "hbm_frac": lb / (lg["chunked_C128_ms"] * 1e-3) / 1e9 / peaks["hbm_gbs"]},
            "quadratic": {"ms": lg["quadratic_ms"], "tokens_per_s": ltok / (lg["quadratic_ms"] * 1e-3),
                          "tensor_frac": lf / (lg["quadratic_ms"] * 1e-3) / 1e12 / peaks["bf16_tflops"]},
            "sequential_C64": {"ms": lg["sequential_C64_ms"],
                               "tokens_per_s": ltok / (lg["sequential_C64_ms"] * 1e-3),
                               "scan_speedup": lg["sequential_C64_ms"] / lg["chunked_C64_ms"]},
        }
        dc = lg["decode_b64"]
        db = decode_bytes(dc["B"] * dc["H"], dc["p"], dc["dv"])
        line["decode_b64"] = {
            "workload": "decode step B=%d H=%d state [%d x %d] fp32" % (dc["B"], dc["H"], dc["p"] ** 2, dc["dv"]),
            "ms": dc["ms"], "tokens_per_s": dc["B"] / (dc["ms"] * 1e-3),
            "hbm_gbs": db / (dc["ms"] * 1e-3) / 1e9, "hbm_frac": db / (dc["ms"] * 1e-3) / 1e9 / peaks["hbm_gbs"]}
        if "sweep" in lg:
            hb = peaks["hbm_gbs"]
            tf = peaks["bf16_tflops"]
            line["sweep"] = [
                {"B": g["B"], "T": g["T"], "chunked_ms": g["chunked_ms"], "quadratic_ms": g["quadratic_ms"],
                 "chunked_tokens_per_s": g["B"] * g["T"] / (g["chunked_ms"] * 1e-3),
                 "quadratic_tokens_per_s": g["B"] * g["T"] / (g["quadratic_ms"] * 1e-3),
                 "chunked_hbm_frac": chunked_bytes(g["B"] * 16, g["T"], 16, 64) / (g["chunked_ms"] * 1e-3) / 1e9 / hb,
                 "quadratic_tensor_frac": flash_flops(g["B"] * 16, g["T"], 16, 64) / (g["quadratic_ms"] * 1e-3) / 1e12
                 / tf} for g in lg["sweep"]]
            rc = lg["recall"]
            rtok = rc["B"] * rc["T"]
            line["recall_p32"] = {
                "workload": "recall-shaped keys B=%d H=%d T=%d p=%d dv=%d bf16" % (rc["B"], rc["H"], rc["T"], rc["p"],
                                                                                 rc["dv"]),
                "chunked": {"ms": rc["chunked_ms"], "tokens_per_s": rtok / (rc["chunked_ms"] * 1e-3)},
                "quadratic": {"ms": rc["quadratic_ms"], "tokens_per_s": rtok / (rc["quadratic_ms"] * 1e-3),
                              "tensor_frac": flash_flops(rc["B"] * rc["H"], rc["T"], rc["p"], rc["dv"])
                              / (rc["quadratic_ms"] * 1e-3) / 1e12 / tf}}
        if "mg" in lg:
            line["mg"] = {}
            for name, m in lg["mg"].items():
                if "P" in m:  # decode step
                    mb = 2 * m["B"] * m["H"] * (m["P"] * m["dv"] + m["P"]) * 4
                    line["mg"][name] = {
                        "workload": "%s decode step B=%d H=%d d=%d groups=%d state [%d x %d] fp32" % (
                            "KATA-Sigma-g" if m.get("summed") else "KATA-Mg", m["B"], m["H"], m["d"], m["groups"],
                            m["P"], m["dv"]),
                        "ms": m["ms"], "tokens_per_s": m["B"] / (m["ms"] * 1e-3),
                        "hbm_frac": mb / (m["ms"] * 1e-3) / 1e9 / peaks["hbm_gbs"]}
                elif m.get("chunked"):
                    # chunked KATA-Mg: HBM fraction by q, k, v read and o
                    # written once (2d + 2dv bf16 values per token-head)
                    cb = m["B"] * m["H"] * m["T"] * (2 * m["d"] + 2 * m["dv"]) * 2
                    line["mg"][name] = {
                        "workload": "%s chunked B=%d H=%d T=%d d=%d groups=%d dv=%d bf16 [%s]" % (
                            "KATA-Sigma-g" if m.get("summed") else "KATA-Mg", m["B"], m["H"], m["T"], m["d"],
                            m["groups"], m["dv"], m["layout"]),
                        "ms": m["ms"], "tokens_per_s": m["B"] * m["T"] / (m["ms"] * 1e-3),
                        "hbm_frac": cb / (m["ms"] * 1e-3) / 1e9 / peaks["hbm_gbs"]}
                else:
                    # score flops: d per pair for KATA-Mg, g*d for KATA-Sigma-g
                    # (every query group against every key group)
                    summed = m.get("summed", False)
                    width = m["groups"] * m["d"] if summed else m["d"]
                    line["mg"][name] = {
                        "workload": "%s B=%d H=%d T=%d d=%d groups=%d dv=%d bf16 [%s]" % (
                            "KATA-Sigma-g" if summed else "KATA-Mg", m["B"], m["H"], m["T"], m["d"], m["groups"],
                            m["dv"], m["layout"]),
                        "ms": m["ms"], "tokens_per_s": m["B"] * m["T"] / (m["ms"] * 1e-3),
                        "tensor_frac": flash_flops(m["B"] * m["H"], m["T"], width, m["dv"]) / (m["ms"] * 1e-3)
                        / 1e12 / peaks["bf16_tflops"]}
        if "first_order" in lg:
            hb = peaks["hbm_gbs"]
            pts = []
            for g in lg["first_order"]:
                nbytes = g["B"] * g["H"] * g["T"] * (2 * g["d"] + 2 * g["dv"]) * 2
                pts.append({"B": g["B"], "T": g["T"], "scan_ms": g["scan_ms"], "sequential_ms": g["sequential_ms"],
                            "scan_tokens_per_s": g["B"] * g["T"] / (g["scan_ms"] * 1e-3),
                            "sequential_tokens_per_s": g["B"] * g["T"] / (g["sequential_ms"] * 1e-3),
                            "scan_speedup": g["sequential_ms"] / g["scan_ms"],
                            "scan_hbm_frac": nbytes / (g["scan_ms"] * 1e-3) / 1e9 / hb})
            sp = np.array([x["scan_speedup"] for x in pts])
            line["first_order"] = {
                "workload": "first-order attention psi(u)=u, H=16 d=16 dv=64 bf16, chunked with the associative scan "
                            "vs the sequential baseline, B x T grid",
                "grid": pts, "scan_speedup_mean": float(sp.mean()),
                "scan_speedup_geomean": float(np.exp(np.log(sp).mean()))}
        if "train" in lg:
            tr = lg["train"]
            pairs = tr["B"] * tr["H"] * tr["T"] * (tr["T"] + 1) / 2
            bwd_flops = pairs * 2 * (3 * tr["p"] + 2 * tr["dv"])
            line["train"] = {
                "workload": "training step of the flash path B=%d H=%d T=%d p=%d dv=%d bf16 (forward saving D, then "
                            "backward)" % (tr["B"], tr["H"], tr["T"], tr["p"], tr["dv"]),
                "step_ms": tr["step_ms"], "tokens_per_s": tr["B"] * tr["T"] / (tr["step_ms"] * 1e-3),
                "fwd_ms": tr["fwd_ms"], "bwd_ms": tr["bwd_ms"],
                "bwd_tensor_frac": bwd_flops / (tr["bwd_ms"] * 1e-3) / 1e12 / peaks["bf16_tflops"],
                "bwd_algorithmic": "2(3p+2dv) flops per causal pair: S, dP, dV, dQ, dK"}
            line["train"]["chunked"] = {
                name: {"workload": "training step of the O(T) chunked path B=%d H=%d T=%d p=%d dv=%d bf16 (forward "
                                   "saving D, then the chunked backward)" % (c["B"], c["H"], c["T"], tr["p"], tr["dv"]),
                       "fwd_ms": c["fwd_ms"], "bwd_ms": c["bwd_ms"], "step_ms": c["step_ms"],
                       "tokens_per_s": c["B"] * c["T"] / (c["step_ms"] * 1e-3),
                       "bwd_hbm_frac": chunked_bwd_bytes(c["B"] * c["H"], c["T"], tr["p"], tr["dv"])
                       / (c["bwd_ms"] * 1e-3) / 1e9 / peaks["hbm_gbs"],
                       "bwd_algorithmic": "q, k, v, o, dO, D read and dq, dk, dv written once: 8p + 8dv + 4 bytes "
                                          "per token-head"}
                for name, c in tr.get("chunked", {}).items()}
    line["roofline"]["points"] = roofline_points(res, peaks, cfg)
    if args.cpu_baseline and world == 1:
        cb = time_oracle(cfg)
        line["cpu_baseline"] = {"value": cb["value"], "unit": UNIT, "cores": cb["cores"], "kind": "oracle",
                                "sample": cb["sample"]}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
