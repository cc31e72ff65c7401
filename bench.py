#!/usr/bin/env python3
"""Throughput of the ARL2 hybrid-attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl arl2|reference]
                    [--config 1|2|4] [--no-graphs]

One step = one frame of one hybrid layer: 4 query-only denoising passes and
one clean commit (intra softmax + inter read-out on every pass, the state
write on the commit), 1560 tokens per frame, 12 heads x 128.  The default
workload is the single-layer bf16 stream (batch 1); its inputs cycle through a
pool of 20 (Q, K, V) triples, 288 MB, larger than the 126 MB L2, with a reuse
distance of 20 passes.  Rank 0 prints one JSON line.

Under torchrun each rank runs independent streams of its own (weak scaling,
replicas only: the path has no exchange step); the job's value is the frames
of all ranks divided by the slowest rank's device time.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from hybrid_linear_attention_arl2_b200 import workloads as W  # noqa: E402

TOKENS_PER_STEP = None  # set from the config


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", default="arl2", choices=["arl2", "reference"])
    ap.add_argument("--config", type=int, default=1, choices=[1, 2, 3, 4],
                    help="1, 2, 4: one hybrid layer; 3: the 30-layer attention stack (its own JSON line)")
    ap.add_argument("--no-graphs", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--block", action="store_true",
                    help="the hybrid attention block (QKV and output projections, gates from the tokens) on the "
                         "single-layer shape (its own JSON line)")
    ap.add_argument("--token", action="store_true",
                    help="the single-layer shape with token-level access (the ablated rule; its own JSON line)")
    ap.add_argument("--profile-small", action="store_true",
                    help="a few steps, no extras: for ncu captures of the kernels")
    ap.add_argument("--profile-kv", type=int, default=0, metavar="F",
                    help="one KV-cache softmax layer: F frames committed into its cache, then three query "
                         "passes over F + 1 frames of keys, timed with CUDA events (its own JSON line; an ncu "
                         "capture of the third query skips F + 2 attention launches)")
    return ap.parse_args()


def state_launches(cfg: W.Config) -> int:
    """Kernels of one commit's state write: one cluster launch when the frame's
    chunks fit one cluster (at most 16 chunks of 128 tokens), else three."""
    return 1 if -(-cfg.tokens // 128) <= 16 else 3


# ------------------------------------------------------------------ flop / byte accounting
def frame_flops(cfg: W.Config) -> dict:
    """Algorithmic flops of one frame of one hybrid layer (all streams)."""
    B, H, d, L, P = cfg.batch, cfg.heads, cfg.head_dim, cfg.tokens, cfg.passes
    intra = 4.0 * L * L * d * H * B            # QK^T and PV, per pass
    readout = 2.0 * L * d * d * H * B          # Q (phi_q S), per pass
    maps = 2 * 2.0 * L * d * d * H * B         # K phi_k and V phi_v, commit
    ks = 2.0 * L * d * d * H * B               # K' S, commit
    delta = 2.0 * L * d * d * H * B            # K'^T R, commit
    prep = 2.0 * d * d * d * H * B             # phi_q S_N, commit
    return {"attn_per_pass": intra + readout, "frame": P * (intra + readout) + maps + ks + delta + prep}


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """SM clock, power and clock-event reasons sampled every millisecond by NVML while
    the timed region runs (read-only queries; no setting of the GPU is changed).
    Falls back to `nvidia-smi -lms 50` when NVML cannot be loaded."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.thread = None
        self.stop_flag = threading.Event()
        self.samples: list[tuple[float, float, float, tuple]] = []  # (sm, sm_max, watts, reasons)
        self.source = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self._nvml_index(pynvml))
            self.source = "nvml 1 ms"
            bits = {"hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}
            smax = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))

            def poll():
                while not self.stop_flag.is_set():
                    try:
                        sm = float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                        w = pynvml.nvmlDeviceGetPowerUsage(h) / 1e3
                        r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    except pynvml.NVMLError:
                        break
                    self.samples.append((sm, smax, w, tuple(n for n, b in bits.items() if r & b)))
                    self.stop_flag.wait(0.001)
            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            return
        except Exception:  # NVML missing or refused: nvidia-smi below
            pass
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.source = "nvidia-smi 50 ms"
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _nvml_index(self, pynvml) -> int:
        # CUDA_VISIBLE_DEVICES renumbers devices for CUDA but not for NVML
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            ids = [v.strip() for v in vis.split(",") if v.strip()]
            if self.dev < len(ids) and ids[self.dev].isdigit():
                return int(ids[self.dev])
        return self.dev

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.strip().split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, smax, w = float(parts[1]), float(parts[2]), float(parts[3])
            except ValueError:
                continue
            self.samples.append((sm, smax, w, tuple(n for n, v in zip(self.REASONS, parts[5:9])
                                                    if v.lower() == "active")))

    def stop(self) -> dict:
        self.stop_flag.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        if self.source is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock source"]}
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "source": self.source}
        sm = [s[0] for s in self.samples]
        reasons = sorted({r for s in self.samples for r in s[3]})
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(s[1] for s in self.samples),
                "sm_mhz_min": min(sm), "reasons": reasons, "samples": len(sm),
                "power_w_max": max(s[2] for s in self.samples), "source": self.source}


# ------------------------------------------------------------------ device workload
class DeviceStream:
    """Device-resident inputs of one stream set (pool of triples, gates, phi)."""

    def __init__(self, cfg: W.Config, seed_offset: int, device):
        import torch
        self.cfg = cfg
        wl = W.Workload(cfg, seed=cfg.seed + 100 * seed_offset)
        self.wl = wl
        to = lambda x: torch.from_numpy(x).to(torch.bfloat16).to(device)
        self.phi = tuple(to(p) for p in wl.phi(0))
        self.pool = []
        for i in range(cfg.pool):
            per = [wl.pool_entry(b, i) for b in range(cfg.batch)]
            self.pool.append(tuple(to(np.stack([t[j] for t in per])) for j in range(3)))
        self.device = device

    def gates(self, frame: int):
        return self.wl.alpha(0, frame), self.wl.beta(0, frame)

    def triple(self, frame: int, pas: int):
        return self.pool[self.wl.pool_index(0, frame, pas)]


def run_kv_profile(args) -> dict:
    """A KV-cache softmax layer of the stack's shape holding `F` clean frames:
    F commits fill its cache, then three query passes attend over the F + 1
    frames of keys (cache and current frame); the last two are timed."""
    import torch
    from hybrid_linear_attention_arl2_b200 import arl2
    cfg = W.CONFIGS[3]
    F = args.profile_kv
    torch.cuda.set_device(0)
    device = torch.device("cuda", 0)
    arl2.load_library()
    ds = DeviceStream(cfg, 0, device)
    B, H, L, d = cfg.batch, cfg.heads, cfg.tokens, cfg.head_dim
    stream = torch.cuda.Stream(device)
    O = torch.empty((B, L, H, d), dtype=torch.bfloat16, device=device)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    with torch.cuda.stream(stream):
        kv = arl2.KVLayer(B, H, d, L, arl2.ARL2_BF16, max_frames=F + 1, stream=stream)
        for f in range(F):
            arl2.arl2_kv_commit(kv.handle, *ds.triple(f, cfg.queries), O, stream)
        for p in range(3):
            if p > 0:
                ev[p - 1].record(stream)
            arl2.arl2_kv_query(kv.handle, *ds.triple(F, p), O, stream)
        ev[2].record(stream)
        stream.synchronize()
        if kv.last_error():
            raise RuntimeError(f"device error in the KV-layer run: {arl2.STATUS.get(kv.last_error())}")
        kv.close()
    ms = [ev[0].elapsed_time(ev[1]), ev[1].elapsed_time(ev[2])]
    kv_len = (F + 1) * L
    fl = 4.0 * L * kv_len * d * H * B
    return {"frames": F, "kv_len": kv_len, "ms": ms, "tflops": fl / (min(ms) / 1e3) / 1e12}


def whole_job_rate(ms: float, steps: int, world: int, dist=None, device="cpu"):
    """Frames/s of the whole job: every rank ran `steps` frames; the time is the
    slowest rank's device time (max over ranks).  Returns (frames/s, max ms)."""
    import torch
    ms_max = float(ms)
    if dist is not None and world > 1:
        t = torch.tensor([ms_max], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_max = float(t.item())
    return steps * world / (ms_max / 1e3), ms_max


def run_arl2(args, rank: int, world: int):
    import torch
    from hybrid_linear_attention_arl2_b200 import arl2

    cfg = W.CONFIGS[args.config]
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)

    arl2.load_library()
    ds = DeviceStream(cfg, rank, device)
    stream = torch.cuda.Stream(device)
    B, H, L, d = cfg.batch, cfg.heads, cfg.tokens, cfg.head_dim
    flops = frame_flops(cfg)

    with torch.cuda.stream(stream):
        layer = arl2.HybridLayer(B, H, d, L, arl2.ARL2_BF16, *ds.phi, corr_scale=cfg.corr_scale, stream=stream)
        O = torch.empty((B, L, H, d), dtype=torch.bfloat16, device=device)
        # frames per graph: the pool phase (20 passes = 4 frames) and the
        # state ping-pong (2 frames) both return to their start after it
        period = 20
        # every frame's gates staged on the device before any timing: before
        # each graph replay two copies move the next `period` frames' gates
        # into the slots the graph reads (rows padded to 16 bytes)
        na, nb = -(-B * H // 4) * 4, B * H * L
        n_frames = args.warmup + args.steps + 2 * period
        ga_all = torch.zeros((n_frames, na), dtype=torch.float32, device=device)
        gb_all = torch.empty((n_frames, nb), dtype=torch.float32, device=device)
        for f in range(n_frames):
            a, b = ds.gates(f)
            ga_all[f, :B * H].copy_(torch.from_numpy(a).reshape(-1))
            gb_all[f].copy_(torch.from_numpy(b).reshape(-1))
        gate_a = torch.empty((period, na), dtype=torch.float32, device=device)
        gate_b = torch.empty((period, nb), dtype=torch.float32, device=device)

        def load_gates(frame, n):
            """Gates of frames frame .. frame + n - 1 into slots 0 .. n - 1."""
            gate_a[:n].copy_(ga_all[frame:frame + n], non_blocking=True)
            gate_b[:n].copy_(gb_all[frame:frame + n], non_blocking=True)

        def frame_calls(frame, slot, ev=None):
            """One frame; `ev` = (start, end) events around its query launches."""
            for p in range(cfg.passes):
                q, k, v = ds.triple(frame, p)
                if p < cfg.queries:
                    if ev is not None and p == 0:
                        ev[0].record(stream)
                    arl2.arl2_frame_query(layer.handle, q, k, v, O, stream)
                    if ev is not None and p == cfg.queries - 1:
                        ev[1].record(stream)
                else:
                    arl2.arl2_frame_commit(layer.handle, q, k, v, gate_a[slot, :B * H], gate_b[slot], O, stream)

        # warm-up (eager): also exercises every kernel once before any capture
        for f in range(args.warmup):
            load_gates(f, 1)
            frame_calls(f, 0)
        stream.synchronize()
        err = layer.last_error()
        if err:
            raise RuntimeError(f"device error during warm-up: {arl2.STATUS.get(err)}")

        use_graphs = not args.no_graphs
        base = args.warmup
        n_rep, n_tail = divmod(args.steps, period) if use_graphs else (0, args.steps)
        if n_rep:
            # Two graphs of the same `period` frames: `graph` carries no event
            # nodes (an event node between two attention launches orders them
            # fully, so they could not overlap set-up and tail); `graph_ev`
            # adds external events (event-record nodes) before the first frame's
            # first query launch and after its last, and runs as the last
            # replay of the timed region: the span of its back-to-back query
            # launches on the launching stream, divided by their number, is the
            # attention kernel's average launch duration.
            graph, graph_ev = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
            ev_q = [(torch.cuda.Event(enable_timing=True, external=True),
                     torch.cuda.Event(enable_timing=True, external=True))]
            stream.synchronize()
            for g, evs in ((graph, None), (graph_ev, ev_q)):
                with torch.cuda.graph(g, stream=stream):
                    for i in range(period):
                        frame_calls(base + i, i, evs[0] if evs and i == 0 else None)
            # one untimed replay of each (its upload and first run)
            for g in (graph, graph_ev):
                load_gates(base, period)
                g.replay()
            stream.synchronize()
            err = layer.last_error()
            if err:
                raise RuntimeError(f"device error in the graph warm-up: {arl2.STATUS.get(err)}")

        clocks = ClockSampler(local)
        if dist is not None:
            dist.barrier()
        stream.synchronize()
        torch.cuda.synchronize()
        clocks.start()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        f = base
        tail_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(max(n_tail, 1))]
        t0.record(stream)
        for r in range(n_rep):
            load_gates(f, period)
            (graph_ev if r == n_rep - 1 else graph).replay()
            f += period
        for j in range(n_tail):  # eager frames: exactly `steps` frames in all
            load_gates(f, 1)
            frame_calls(f, 0, tail_ev[j])
            f += 1
        t1.record(stream)
        steps_done = n_rep * period + n_tail
        t1.synchronize()
        clk = clocks.stop()
        ms = t0.elapsed_time(t1)
        err = layer.last_error()
        if err:
            raise RuntimeError(f"device error in the timed region: {arl2.STATUS.get(err)}")

        # dominant-kernel duration: the query launches timed in the timed
        # region (the evented replay's first frame, else the eager frames)
        attn_ev = ev_q if n_rep else tail_ev[:n_tail]
        attn_avg_ms = float(np.mean([a.elapsed_time(b) for a, b in attn_ev])) / cfg.queries

    value, ms_max = whole_job_rate(ms, steps_done, world, dist, device)
    ms_per_step = ms_max / steps_done

    result = {
        "value": value, "ms_per_step": ms_per_step, "steps": steps_done, "clocks": clk,
        "attn_avg_ms": attn_avg_ms, "flops": flops, "launches_per_step": cfg.queries + 1 + state_launches(cfg),
        "timing": ((f"CUDA graphs of {period} frames, {n_rep} replays" + (" + " if n_tail else "") if n_rep else "")
                   + (f"{n_tail} eager frame" + ("s" if n_tail != 1 else "") if n_tail else "")),
        "attn_basis": (f"CUDA events before the first and after the last of one frame's {cfg.queries} back-to-back "
                       "query launches" + (" (last graph replay)" if n_rep else " (every eager frame)")
                       + f", span / {cfg.queries}"),
    }
    if args.config == 2 and not args.profile_small:
        result["flatness"] = long_stream_flatness(cfg, ds, device, rank)
    # end-to-end through the public API with host buffers
    if not args.no_e2e:
        result["e2e"] = run_e2e(args, cfg, ds, layer, device, stream, dist, world)
    layer.close()
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return result


def run_e2e(args, cfg, ds, layer, device, stream, dist, world):
    """Same metric through the C-ABI calls with host buffers: every step copies its
    five passes' Q, K, V and its gates from pinned host memory and reads the five
    outputs back.  Copies in (Q, K and V each on its own stream), compute and
    copies out run on separate streams with two buffer sets, so a pass's inputs
    cross PCIe while the previous pass computes and its output goes back (PCIe
    is full duplex)."""
    import torch
    from hybrid_linear_attention_arl2_b200 import arl2
    B, H, L, d = cfg.batch, cfg.heads, cfg.tokens, cfg.head_dim
    steps = max(4, min(args.steps // 4, 40))
    nbuf = 2
    host_pool = [tuple(t.cpu().pin_memory() for t in trip) for trip in ds.pool]
    outs_host = [torch.empty((B, L, H, d), dtype=torch.bfloat16).pin_memory() for _ in range(cfg.passes)]
    dq = [[torch.empty((B, L, H, d), dtype=torch.bfloat16, device=device) for _ in range(3)] for _ in range(nbuf)]
    O = [torch.empty((B, L, H, d), dtype=torch.bfloat16, device=device) for _ in range(nbuf)]
    ga = [torch.empty((B, H), dtype=torch.float32, device=device) for _ in range(nbuf)]
    gb = [torch.empty((B, H, L), dtype=torch.float32, device=device) for _ in range(nbuf)]
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    s_cp = [s_in] + [torch.cuda.Stream(device) for _ in range(2)]  # Q, K, V copies on their own streams
    loaded = [torch.cuda.Event() for _ in range(nbuf)]
    part = [[torch.cuda.Event() for _ in range(2)] for _ in range(nbuf)]
    computed = [torch.cuda.Event() for _ in range(nbuf)]
    drained = [torch.cuda.Event() for _ in range(nbuf)]
    gates = {}
    h2d = d2h = 0
    f0 = 1000
    for f in range(f0, f0 + steps):
        a, b = ds.gates(f)
        gates[f] = (torch.from_numpy(a).pin_memory(), torch.from_numpy(b).pin_memory())
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    stream.wait_event(e0)
    s_out.wait_event(e0)
    for sc in s_cp[1:]:
        sc.wait_event(e0)
    i = 0
    for f in range(f0, f0 + steps):
        for p in range(cfg.passes):
            k = i % nbuf
            trip = host_pool[ds.wl.pool_index(0, f, p)]
            if i >= nbuf:
                for sc in s_cp:
                    sc.wait_event(computed[k])  # buffer set k is free once pass i - nbuf has computed
            for j, (dst, src) in enumerate(zip(dq[k], trip)):
                with torch.cuda.stream(s_cp[j]):
                    dst.copy_(src, non_blocking=True)
                h2d += src.numel() * 2
            for j in (1, 2):
                part[k][j - 1].record(s_cp[j])
                s_in.wait_event(part[k][j - 1])
            with torch.cuda.stream(s_in):
                if p >= cfg.queries:
                    a, b = gates[f]
                    ga[k].copy_(a, non_blocking=True)
                    gb[k].copy_(b, non_blocking=True)
                    h2d += a.numel() * 4 + b.numel() * 4
            loaded[k].record(s_in)
            stream.wait_event(loaded[k])
            if i >= nbuf:
                stream.wait_event(drained[k])  # output k has been read back
            if p < cfg.queries:
                arl2.arl2_frame_query(layer.handle, dq[k][0], dq[k][1], dq[k][2], O[k], stream)
            else:
                arl2.arl2_frame_commit(layer.handle, dq[k][0], dq[k][1], dq[k][2], ga[k], gb[k], O[k], stream)
            computed[k].record(stream)
            s_out.wait_event(computed[k])
            with torch.cuda.stream(s_out):
                outs_host[p].copy_(O[k], non_blocking=True)
                d2h += O[k].numel() * 2
            drained[k].record(s_out)
            i += 1
    e1.record(s_out)  # after the last read-back, which follows every copy and kernel
    e1.synchronize()
    value, _ = whole_job_rate(e0.elapsed_time(e1), steps, world, dist, device)
    return {"value": value, "unit": "frames/s",
            "h2d_bytes_per_step": h2d // steps, "d2h_bytes_per_step": d2h // steps}


# ------------------------------------------------------------------ long stream
def long_stream_flatness(cfg, ds, device, rank) -> dict:
    """Per-frame latency and device memory against the frame index over the
    whole long stream (231 frames), with fresh state: both must stay flat
    (the state is a fixed 128 x 128 per head; nothing grows with the frame)."""
    import torch
    from hybrid_linear_attention_arl2_b200 import arl2
    B, H, L, d = cfg.batch, cfg.heads, cfg.tokens, cfg.head_dim
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        layer = arl2.HybridLayer(B, H, d, L, arl2.ARL2_BF16, *ds.phi, corr_scale=cfg.corr_scale, stream=stream)
        O = torch.empty((B, L, H, d), dtype=torch.bfloat16, device=device)
        ga = torch.empty((cfg.frames, B, H), dtype=torch.float32, device=device)
        gb = torch.empty((cfg.frames, B, H, L), dtype=torch.float32, device=device)
        for f in range(cfg.frames):
            a, b = ds.gates(f)
            ga[f].copy_(torch.from_numpy(a))
            gb[f].copy_(torch.from_numpy(b))
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(cfg.frames)]
        mem = []
        torch.cuda.synchronize()
        for f in range(cfg.frames):
            ev[f][0].record(stream)
            for p in range(cfg.passes):
                q, k, v = ds.triple(f, p)
                if p < cfg.queries:
                    arl2.arl2_frame_query(layer.handle, q, k, v, O, stream)
                else:
                    arl2.arl2_frame_commit(layer.handle, q, k, v, ga[f], gb[f], O, stream)
            ev[f][1].record(stream)
            mem.append(torch.cuda.memory_allocated(device))
        stream.synchronize()
        err = layer.last_error()
        handle_bytes = arl2.arl2_state_device_bytes(layer.handle)
        layer.close()
    if err:
        raise RuntimeError(f"device error in the long stream: {arl2.STATUS.get(err)}")
    ms = np.array([a.elapsed_time(b) for a, b in ev])
    k = max(1, cfg.frames // 10)
    slope = float(np.polyfit(np.arange(cfg.frames), ms, 1)[0])
    return {"frames": cfg.frames, "timing": "eager launches, CUDA events per frame",
            "ms_first_tenth": float(ms[:k].mean()), "ms_last_tenth": float(ms[-k:].mean()),
            "ms_median": float(np.median(ms)), "ms_slope_per_frame": slope,
            "torch_allocated_bytes_min": int(min(mem)), "torch_allocated_bytes_max": int(max(mem)),
            "handle_device_bytes": int(handle_bytes)}


# ------------------------------------------------------------------ attention block
def run_block(args, rank: int, world: int) -> dict:
    """The hybrid attention block on the single-layer shape (B=1, H=12, d=128,
    L=1560, hidden 1536): per pass X -> Q, K, V (tcgen05 GEMM) -> hybrid layer -> O W_o;
    the commit also forms its gates from X.  Inputs cycle through 40 seeded
    token matrices (192 MB > L2); each CUDA graph holds eight frames, the pool's
    whole cycle, so that every replay reads all 40."""
    import dataclasses
    import torch
    from hybrid_linear_attention_arl2_b200 import arl2
    cfg = dataclasses.replace(W.CONFIGS[1], pool=40)
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    arl2.load_library()
    wl = W.Workload(cfg, seed=cfg.seed + 100 * rank)
    to = lambda x: torch.from_numpy(x).to(torch.bfloat16).to(device)
    weights = [to(w) for w in wl.block_weights(0)]
    phi = [to(p) for p in wl.phi(0)]
    B, H, L, d = cfg.batch, cfg.heads, cfg.tokens, cfg.head_dim
    # pool entry i is the tokens of pass i % 5 of frame i // 5
    xs = [to(wl.block_input(0, i // cfg.passes, i % cfg.passes)) for i in range(cfg.pool)]
    stream = torch.cuda.Stream(device)
    period = cfg.pool // cfg.passes  # frames per graph: one pass over the pool
    with torch.cuda.stream(stream):
        blk = arl2.HybridBlock(B, H, L, *weights, *phi, corr_scale=cfg.corr_scale, stream=stream)
        Y = torch.empty_like(xs[0])

        def frame(f):
            for p in range(cfg.passes):
                x = xs[wl.pool_index(0, f, p)]
                if p < cfg.queries:
                    arl2.arl2_block_query(blk.handle, x, Y, stream)
                else:
                    arl2.arl2_block_commit(blk.handle, x, Y, stream)

        for f in range(args.warmup):
            frame(f)
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for f in range(period):
                frame(f)
        graph.replay()  # untimed: the graph's upload and first run
        stream.synchronize()
        n_rep, n_tail = divmod(args.steps, period)
        clocks = ClockSampler(local)
        torch.cuda.synchronize()
        clocks.start()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(n_rep):
            graph.replay()
        for f in range(n_tail):  # eager frames: exactly `steps` frames in all
            frame(f)
        steps = n_rep * period + n_tail
        t1.record(stream)
        t1.synchronize()
        clk = clocks.stop()
        err = blk.last_error()
        ms = t0.elapsed_time(t1)
        del graph
        blk.close()
    if err:
        raise RuntimeError(f"device error in the block run: {arl2.STATUS.get(err)}")
    D = H * d
    proj = 4 * 2.0 * B * L * D * D
    fl = frame_flops(cfg)
    frame_fl = cfg.passes * proj + fl["frame"] + 2.0 * B * L * D * 2 * H
    value, ms_max = whole_job_rate(ms, steps, world, None, device)
    return {"frames": steps, "ms": ms_max, "value": value, "clocks": clk, "flops_per_frame": frame_fl,
            "projection_flops_per_frame": cfg.passes * proj}


# ------------------------------------------------------------------ token-level access
def run_token(args, rank: int, world: int) -> dict:
    """The single-layer shape (B=1, H=12, d=128, L=1560) with token-level
    access: per frame four token-level queries and one token-level commit,
    c = 1, per-token decays and write strengths from the seeded generators
    (eight frames' worth on the device, cycled).  Inputs cycle through the
    20-triple pool of the frame-level run (288 MB > L2).  Eager launches; the
    first call allocates the handle's scratch, so it runs in the warm-up."""
    import torch
    from hybrid_linear_attention_arl2_b200 import arl2
    cfg = W.CONFIGS[1]
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    arl2.load_library()
    ds = DeviceStream(cfg, rank, device)
    wl = ds.wl
    gates = [(torch.from_numpy(wl.alpha_tok(0, f)).to(device), torch.from_numpy(wl.beta(0, f)).to(device))
             for f in range(8)]
    B, H, L, d = cfg.batch, cfg.heads, cfg.tokens, cfg.head_dim
    frames = max(1, min(args.steps, 40))
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        layer = arl2.HybridLayer(B, H, d, L, arl2.ARL2_BF16, *ds.phi, corr_scale=1.0, stream=stream)
        O = torch.empty_like(ds.pool[0][0])

        def frame(f):
            a, b = gates[f % len(gates)]
            for p in range(cfg.passes):
                q, k, v = ds.triple(f, p)
                if p < cfg.queries:
                    arl2.arl2_token_query(layer.handle, q, k, v, a, b, O, stream)
                else:
                    arl2.arl2_token_commit(layer.handle, q, k, v, a, b, O, stream)

        for f in range(max(3, args.warmup)):
            frame(f)
        stream.synchronize()
        clocks = ClockSampler(local)
        clocks.start()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for f in range(frames):
            frame(f)
        t1.record(stream)
        t1.synchronize()
        clk = clocks.stop()
        err = layer.last_error()
        ms = t0.elapsed_time(t1)
        layer.close()
    if err:
        raise RuntimeError(f"device error in the token-level run: {arl2.STATUS.get(err)}")
    value, ms_max = whole_job_rate(ms, frames, world, None, device)
    return {"frames": frames, "ms": ms_max, "value": value, "clocks": clk}


# ------------------------------------------------------------------ attention stack
def run_stack(args, rank: int, world: int) -> dict:
    """The 30-layer attention stack: layers [0, 22) hybrid, [22, 30) softmax over a
    KV cache that grows by one clean frame per frame.  A frame is 4 query passes
    and 1 commit, each pass running every layer in index order.  The timed run
    starts from fresh handles (empty states and caches) and covers `frames`
    frames; CUDA events around each pass's hybrid and softmax blocks give the
    per-layer-type split."""
    import torch
    from hybrid_linear_attention_arl2_b200 import arl2
    cfg = W.CONFIGS[3]
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    arl2.load_library()
    ds = DeviceStream(cfg, rank, device)
    wl = ds.wl
    B, H, L, d = cfg.batch, cfg.heads, cfg.tokens, cfg.head_dim
    F = max(1, min(args.steps, cfg.frames))
    nh, nl = cfg.hybrid_layers, cfg.layers
    to = lambda x: torch.from_numpy(x).to(torch.bfloat16).to(device)
    phis = [tuple(to(p) for p in wl.phi(l)) for l in range(nh)]
    # every gate of the run on the device before timing
    ga = torch.empty((F, nh, B, H), dtype=torch.float32, device=device)
    gb = torch.empty((F, nh, B, H, L), dtype=torch.float32, device=device)
    for f in range(F):
        for l in range(nh):
            ga[f, l].copy_(torch.from_numpy(wl.alpha(l, f)))
            gb[f, l].copy_(torch.from_numpy(wl.beta(l, f)))
    stream = torch.cuda.Stream(device)
    O = torch.empty((B, L, H, d), dtype=torch.bfloat16, device=device)

    def make_layers():
        hyb = [arl2.HybridLayer(B, H, d, L, arl2.ARL2_BF16, *phis[l], corr_scale=cfg.corr_scale, stream=stream)
               for l in range(nh)]
        kv = [arl2.KVLayer(B, H, d, L, arl2.ARL2_BF16, max_frames=F, stream=stream) for _ in range(nh, nl)]
        return hyb, kv

    def frame(f, hyb, kv, ev=None):
        for p in range(cfg.passes):
            if ev is not None:
                ev[p][0].record(stream)
            for l in range(nl):
                q, k, v = ds.pool[wl.pool_index(l, f, p)]
                if l < nh:
                    if p < cfg.queries:
                        arl2.arl2_frame_query(hyb[l].handle, q, k, v, O, stream)
                    else:
                        arl2.arl2_frame_commit(hyb[l].handle, q, k, v, ga[f, l], gb[f, l], O, stream)
                else:
                    if l == nh and ev is not None:
                        ev[p][1].record(stream)
                    fn = arl2.arl2_kv_query if p < cfg.queries else arl2.arl2_kv_commit
                    fn(kv[l - nh].handle, q, k, v, O, stream)
            if ev is not None:
                ev[p][2].record(stream)

    with torch.cuda.stream(stream):
        hyb, kv = make_layers()  # warm-up on throwaway handles: first-call set-up of every kernel
        for f in range(min(args.warmup, F)):
            frame(f, hyb, kv)
        stream.synchronize()
        for x in hyb + kv:
            x.close()
        hyb, kv = make_layers()
        stream.synchronize()
        evs = [[tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(cfg.passes)]
               for _ in range(F)]
        clocks = ClockSampler(local)
        torch.cuda.synchronize()
        clocks.start()
        for f in range(F):
            frame(f, hyb, kv, evs[f])
        stream.synchronize()
        clk = clocks.stop()
        err = [x.last_error() for x in hyb + kv]
        if any(err):
            raise RuntimeError(f"device error in the stack run: {[arl2.STATUS.get(e) for e in err if e]}")
        t_h = sum(e[0].elapsed_time(e[1]) for fe in evs for e in fe)
        t_k = sum(e[1].elapsed_time(e[2]) for fe in evs for e in fe)
        total = evs[0][0][0].elapsed_time(evs[-1][-1][2])
        for x in hyb + kv:
            x.close()
    fl = frame_flops(cfg)
    hyb_flops = fl["frame"] * nh * F
    kv_flops = sum(4.0 * L * (f + 1) * L * d * H * B * cfg.passes * (nl - nh) for f in range(F))
    return {"frames": F, "ms_total": total, "ms_hybrid": t_h, "ms_kv": t_k, "clocks": clk,
            "hybrid_tflops": hyb_flops / (t_h / 1e3) / 1e12, "kv_tflops": kv_flops / (t_k / 1e3) / 1e12,
            "stack_tflops": (hyb_flops + kv_flops) / (total / 1e3) / 1e12, "flops": hyb_flops + kv_flops,
            "launches": F * cfg.passes * (nh + (nl - nh)) + F * nh * state_launches(cfg)}


# ------------------------------------------------------------------ CPU oracle baseline
def cpu_oracle_rate(cfg: W.Config, budget_s: float = 12.0, sample_note=True):
    """The oracle as it stands, timed on this host's cores: frames/s of one
    hybrid layer on a bounded sample (whole frames, 4 queries + 1 commit)."""
    from oracle import arl2_oracle as o
    wl = W.Workload(cfg)
    phi = wl.phi(0)
    S = np.zeros((cfg.batch, cfg.heads, cfg.head_dim, cfg.head_dim))
    frames = 0
    t0 = time.perf_counter()
    while True:
        for p in range(cfg.passes):
            Q, K, V = wl.qkv(0, frames, p)
            if p < cfg.queries:
                o.frame_query(S, Q, K, V, phi)
            else:
                _, S = o.frame_commit(S, Q, K, V, phi, wl.alpha(0, frames), wl.beta(0, frames), cfg.c)
        frames += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    cores = len(os.sched_getaffinity(0))
    return {"value": frames / dt, "unit": "frames/s", "cores": cores, "kind": "oracle",
            "sample": f"{frames} whole frames (4 query passes + 1 commit each) of one {cfg.name} layer, "
                      f"numpy float64, {dt:.1f} s"}


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one attn_pair_kernel
# launch on the single-hybrid-layer-bf16 workload, from one ncu capture of
# `bench.py --profile-small --no-graphs`; reported only while the kernel sources
# hash to the value below (None: not captured yet).  The hash is that of the
# sources after the debug build's index checks were added and unused helpers
# left the header: the checks compile away in the release build, whose
# attention kernel compiles to the same bytes as the captured sources' (cubins
# compared from the same path, without line tables).
ATTN_TRAFFIC = {"bytes": 14858496 + 0, "sources_sha256": "e9affde710f04be4c5a6055f7795bd22b26f637b7bca31df702cc3b70b4c7cf8",
                "workload": "single-hybrid-layer-bf16",
                "capture": "profiles/attn_pair_kernel_single-hybrid-layer-bf16.md"}
ATTN_SOURCES = ("hybrid_linear_attention_arl2_b200/csrc/attn_pair.cu",
                "hybrid_linear_attention_arl2_b200/csrc/sm100.cuh",
                "hybrid_linear_attention_arl2_b200/csrc/params.h")


def attn_sources_sha256() -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in ATTN_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def attn_traffic(workload: str):
    """DRAM bytes of one attention launch, for the captured workload only."""
    if ATTN_TRAFFIC["bytes"] is None or ATTN_TRAFFIC["sources_sha256"] != attn_sources_sha256():
        return None
    return ATTN_TRAFFIC["bytes"] if workload == ATTN_TRAFFIC["workload"] else None


def peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except (OSError, ValueError):
        return None


def peak_pair(pk):
    """(burst, sustained) dense bf16 TFLOP/s and their source.  The burst figure
    is the headline denominator: the kernels are timed in regions of a few
    milliseconds at the clocks sampled alongside; the sustained figure (a
    seconds-long loop under the power cap) is reported as a second ratio."""
    if pk:
        return pk["bf16_tflops"], pk["bf16_tflops_sustained"], "of measured"
    return 1590.0, 1400.0, "of fallback"


def main():
    args = _args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    cfg = W.CONFIGS[args.config]
    if args.profile_small:
        args.steps, args.warmup = 4, 3
        args.no_e2e = args.no_cpu_baseline = True
    metric = "frames/s per hybrid layer (1560-token frames, 4 query passes + 1 commit)"
    config = {"workload": cfg.name, "batch": cfg.batch, "heads": cfg.heads, "head_dim": cfg.head_dim,
              "tokens_per_frame": cfg.tokens, "passes_per_frame": cfg.passes,
              "corr_scale": "1/L" if cfg.corr_scale < 0 else cfg.corr_scale,
              "l2": f"inputs cycle through a {cfg.pool}-triple pool "
                    f"({cfg.pool * 3 * cfg.tokens * cfg.heads * cfg.head_dim * 2 * cfg.batch / 1e6:.0f} MB > 126 MB L2)",
              "parallelism": f"replicas x{world}"}

    if args.impl == "reference":
        if rank != 0:
            return
        budget = 3.0
        steps = []
        cb = None
        for s in range(args.warmup + args.steps):
            cb = cpu_oracle_rate(cfg, budget_s=budget / max(1, args.steps))
            steps.append(cb["value"])
        value = float(np.mean(steps[args.warmup:])) if args.steps else float(np.mean(steps))
        line = {"impl": "reference", "metric": metric, "value": value, "unit": "frames/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 / value,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": config,
                "cpu_baseline": {"value": value, "unit": "frames/s", "cores": cb["cores"], "kind": "oracle",
                                 "sample": cb["sample"]},
                "e2e": {"value": value, "unit": "frames/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    if args.profile_kv and args.impl != "reference":
        res = run_kv_profile(args)
        peak_burst, peak_sus, src = peak_pair(peaks())
        print(json.dumps({"metric": "KV-cache softmax layer query pass (TFLOP/s)", "value": res["tflops"],
                          "unit": "TFLOP/s", "n_gpus": 1, "higher_is_better": True, "dtype": "bf16",
                          "data": "synthetic",
                          "config": {"workload": "kv-cache-softmax-layer-bf16", "cache_frames": res["frames"],
                                     "kv_len": res["kv_len"], "tokens_per_frame": 1560, "heads": 12,
                                     "head_dim": 128},
                          "ms": res["ms"], "frac_of_burst_peak": res["tflops"] / peak_burst,
                          "peak_basis": f"burst bf16 {src}"}), flush=True)
        return
    if args.token and args.impl != "reference":
        res = run_token(args, rank, world)
        if rank != 0:
            return
        line = {
            "metric": "frames/s per hybrid layer with token-level access (1560-token frames, 4 query passes + "
                      "1 commit)",
            "value": res["value"], "unit": "frames/s", "n_gpus": world, "steps": res["frames"],
            "warmup": max(3, args.warmup), "ms_per_step": res["ms"] / res["frames"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16 inputs, f32 scan", "data": "synthetic",
            "config": {"workload": "single-hybrid-layer-token-level-bf16", "batch": 1, "heads": 12,
                       "head_dim": 128, "tokens_per_frame": 1560, "passes_per_frame": 5, "corr_scale": 1.0,
                       "gates": "per-token decay sigmoid(N(4, 0.5)), beta sigmoid(N(0, 1))",
                       "l2": "inputs cycle through a 20-triple pool (288 MB > 126 MB L2)",
                       "timing": "eager launches, CUDA events around all timed frames"},
            "tokens_per_s": res["value"] * 1560, "clocks": res["clocks"],
        }
        print(json.dumps(line), flush=True)
        return
    if args.block and args.impl != "reference":
        res = run_block(args, rank, world)
        if rank != 0:
            return
        peak_burst, peak_sus, src = peak_pair(peaks())
        tf = res["flops_per_frame"] * res["value"] / 1e12
        line = {
            "metric": "frames/s per hybrid attention block (1560-token frames, hidden 1536, QKV/out projections "
                      "+ hybrid layer, 4 query passes + 1 commit)",
            "value": res["value"], "unit": "frames/s", "n_gpus": world, "steps": res["frames"],
            "warmup": args.warmup, "ms_per_step": res["ms"] / res["frames"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic, random-init weights",
            "config": {"workload": "hybrid-attention-block-bf16", "batch": 1, "heads": 12, "head_dim": 128,
                       "hidden": 1536, "tokens_per_frame": 1560, "passes_per_frame": 5,
                       "l2": "tokens cycle through 40 seeded 1560 x 1536 matrices (192 MB > 126 MB L2)",
                       "projections": "tcgen05 GEMMs of this library (bf16, fp32 accumulate)"},
            "tflops": tf, "pct_bf16_peak": {"value": 100.0 * tf / peak_burst, "basis": f"burst bf16 {src}",
                                            "sustained_basis": 100.0 * tf / peak_sus},
            "clocks": res["clocks"],
        }
        print(json.dumps(line), flush=True)
        return
    if args.config == 3:
        if args.impl == "reference":
            pass  # falls through to the oracle arm below with the single-layer metric
        else:
            res = run_stack(args, rank, world)
            if rank != 0:
                return
            peak_burst, peak_sus, src = peak_pair(peaks())
            line = {
                "metric": "stack frames/s (30 attention layers: 22 hybrid + 8 KV-cache softmax, 1560-token frames)",
                "value": res["frames"] * world / (res["ms_total"] / 1e3), "unit": "frames/s", "n_gpus": world,
                "steps": res["frames"], "warmup": args.warmup, "ms_per_step": res["ms_total"] / res["frames"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic",
                "config": {"workload": cfg.name, "layers": cfg.layers, "hybrid_layers": cfg.hybrid_layers,
                           "frames": res["frames"], "tokens_per_frame": cfg.tokens, "heads": cfg.heads,
                           "head_dim": cfg.head_dim, "passes_per_frame": cfg.passes,
                           "l2": "inputs cycle through a 20-triple pool (288 MB); KV caches up to 4.8 GB",
                           "timing": "eager launches, CUDA events per pass and layer type"},
                "split_ms": {"hybrid": res["ms_hybrid"], "kv_softmax": res["ms_kv"]},
                "tflops": {"stack": res["stack_tflops"], "hybrid_layers": res["hybrid_tflops"],
                           "kv_softmax_layers": res["kv_tflops"]},
                "pct_bf16_peak": {"value": 100.0 * res["stack_tflops"] / peak_burst,
                                  "basis": f"burst bf16 {src}",
                                  "sustained_basis": 100.0 * res["stack_tflops"] / peak_sus},
                "roofline": {"bound": "tensor", "kernel": "attn_pair_kernel (KV-cache softmax layers)",
                             "achieved": res["kv_tflops"], "peak": peak_burst, "unit": "TFLOP/s",
                             "frac": res["kv_tflops"] / peak_burst, "traffic": None,
                             "peak_basis": f"bf16_tflops (burst) {src}",
                             "frac_vs_sustained": res["kv_tflops"] / peak_sus},
                "clocks": res["clocks"], "gpu_launches": res["launches"],
            }
            print(json.dumps(line), flush=True)
            return
    res = run_arl2(args, rank, world)
    if rank != 0:
        return
    pk = peaks()
    fl = res["flops"]
    frame_tflops = fl["frame"] * res["value"] / max(1, world) / 1e12  # per GPU
    attn_tflops = fl["attn_per_pass"] / (res["attn_avg_ms"] / 1e3) / 1e12
    peak_burst, peak_sus, src = peak_pair(pk)
    line = {
        "metric": metric, "value": res["value"], "unit": "frames/s", "n_gpus": world, "steps": res["steps"],
        "warmup": args.warmup, "ms_per_step": res["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(config, timing=res["timing"]),
        "tokens_per_s": res["value"] * cfg.tokens * cfg.batch,
        "pct_bf16_peak": {"value": 100.0 * frame_tflops / peak_burst, "basis": f"burst bf16 {src}",
                          "sustained_basis": 100.0 * frame_tflops / peak_sus},
        "roofline": {"bound": "tensor", "kernel": "attn_pair_kernel", "achieved": attn_tflops, "peak": peak_burst,
                     "unit": "TFLOP/s", "frac": attn_tflops / peak_burst, "traffic": attn_traffic(cfg.name),
                     "peak_basis": f"bf16_tflops (burst) {src}",
                     "frac_vs_sustained": attn_tflops / peak_sus, "duration_basis": res["attn_basis"]},
        "clocks": res["clocks"],
        "gpu_launches": res["launches_per_step"] * res["steps"],
    }
    if "e2e" in res:
        line["e2e"] = res["e2e"]
    if "flatness" in res:
        line["flatness"] = res["flatness"]
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_oracle_rate(cfg, budget_s=12.0)
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
