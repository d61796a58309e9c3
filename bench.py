#!/usr/bin/env python
"""Benchmark of the routed int4 MoE FFN hot path on B200.

Default workload (one "step"): single-layer decode of 1 token through a MoE
layer with 256 experts, top-8, hidden 2048, expert width 512 -- route, the
weight-streaming expert FFN, combine.  Steps rotate over 40 resident layers
(40 x 256 experts x 3 int4 matrices = 18.1 GB in HBM, each layer with its own
activations and fresh router logits), so the 14.2 MB a step streams is never
L2-resident from an earlier step (inputs larger than L2, no flush needed).

Prints one JSON line (see the design doc for every key).  Multi-GPU: one process
per GPU (torchrun), each rank an independent replica of the workload (the
path has no exchange step), barrier + max-over-ranks timing.

--impl reference times the CPU oracle (plain C, single thread) on the same
workload: each step is one token through one layer, rotating over a small
pool of sampled token-layers.
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

E, TOPK, H, F = 256, 8, 2048, 512
LAYERS = 40
EXPERT_BYTES = 1769472  # packed int4 gate/up + down of one expert (36 B per 64 weights)
METRIC = "routed-expert tokens/s + HBM GB/s (decode), TFLOP/s (prefill) vs roofline"
WORKLOAD = ("single-layer decode: 256 experts, top-8, hidden 2048, expert width 512, 1 token per step; "
            "steps rotate over 40 resident int4 layers (18.1 GB) with fresh router logits per layer")
NV_WORKLOAD = ("NVFP4 single-layer decode: 256 experts, top-8, hidden 2048, expert width 512, 1 token per step; "
               "E2M1 weights with E4M3 scales per 16 channels and fp32 per-matrix globals, x and h quantised "
               "per token/row in the kernel; steps rotate over 40 resident NVFP4 layers (18.1 GB)")
DTYPE_W4 = "int4 weights (f16 scale/min), bf16 activations, fp32 accumulate"
# dram__bytes_read.sum + dram__bytes_write.sum of one decode launch at 1 token,
# from the ncu captures summarised in profiles/ (taken on the current kernels;
# set to None whenever the kernel changes)
DECODE_TRAFFIC = {"w4": 14242560, "nvfp4": 14289152}
DTYPE_NV = "nvfp4 weights and activations (e2m1 + e4m3/16 + fp32 global), fp32 accumulate"
# the same for the prefill FFN kernels: both launches of one layer at the bench's
# token count (the bench's first layer), from profiles/prefill_*.md
PREFILL_TRAFFIC = {"w4": 316057344, "nvfp4": 136497408}


# ---------------------------------------------------------------------------- helpers
def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            p = [v.strip() for v in ln.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                mx = max(mx, float(p[2]))
            except ValueError:
                continue
            for n, v in zip(names, p[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def dist_max(v: float) -> float:
    """Max of a per-rank value over all ranks (the slowest rank's time)."""
    import torch
    import torch.distributed as dist
    if not dist.is_initialized():
        return v
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: int, world: int, max_ms: float) -> float:
    """Whole-job throughput of independent replicas: every rank's units over
    the slowest rank's time (weak scaling; no data-path exchange)."""
    return units_per_rank * world / (max_ms / 1e3)


def dist_barrier():
    import torch.distributed as dist
    if dist.is_initialized():
        dist.barrier()


# ---------------------------------------------------------------------------- workload
def build_layers(L, seed, log, fmt="w4"):
    """Resident layers of packed experts (int4, or NVFP4 with fmt="nvfp4"),
    generated, quantised and packed on the GPU."""
    import torch
    import synth
    import quantized_moe_route_b200 as moe
    if fmt == "nvfp4":
        return build_layers_nvfp4(L, seed, log)
    gu_b, d_b = moe.moe_w4_packed_bytes(2 * F, H), moe.moe_w4_packed_bytes(H, F)
    chunk = 32
    tmp = torch.empty((chunk, 2 * F, H), dtype=torch.float32, device="cuda")
    codes = torch.empty((chunk * 2 * F, H), dtype=torch.uint8, device="cuda")
    sc = torch.empty((chunk * 2 * F, H // 64), dtype=torch.int16, device="cuda")
    mn = torch.empty_like(sc)
    layers = []
    t0 = time.time()
    for l in range(L):
        gu = torch.empty(E * gu_b, dtype=torch.uint8, device="cuda")
        dn = torch.empty(E * d_b, dtype=torch.uint8, device="cuda")
        for proj, buf, nb, (N, K), kind in ((synth.PROJ_GATE_UP, gu, gu_b, (2 * F, H), moe.MOE_W4_GATE_UP),
                                             (synth.PROJ_DOWN, dn, d_b, (H, F), moe.MOE_W4_PLAIN)):
            G = K // 64
            for e0 in range(0, E, chunk):
                w = tmp.view(-1)[: chunk * N * K].view(chunk, N, K)
                synth.cuda_expert_weights(w, seed, l, e0, proj)
                c = codes.view(-1)[: chunk * N * K].view(chunk * N, K)
                s = sc.view(-1)[: chunk * N * G].view(chunk * N, G)
                m = mn.view(-1)[: chunk * N * G].view(chunk * N, G)
                moe.moe_quantize_w4(w.view(chunk * N, K), c, s, m)
                for i in range(chunk):
                    e = e0 + i
                    moe.moe_pack_w4(c[i * N:(i + 1) * N], s[i * N:(i + 1) * N], m[i * N:(i + 1) * N], kind,
                                    buf[e * nb:(e + 1) * nb])
        layers.append((gu, dn, moe.make_layer(E, H, F, gu, dn)))
    torch.cuda.synchronize()
    del tmp, codes, sc, mn
    log(f"built {L} layers in {time.time() - t0:.1f}s")
    return layers


def build_layers_nvfp4(L, seed, log):
    import torch
    import synth
    import quantized_moe_route_b200 as moe
    gu_b, d_b = moe.moe_nvfp4_packed_bytes(2 * F, H), moe.moe_nvfp4_packed_bytes(H, F)
    chunk = 32
    tmp = torch.empty((chunk, 2 * F, H), dtype=torch.float32, device="cuda")
    codes = torch.empty((2 * F, H), dtype=torch.uint8, device="cuda")
    sf = torch.empty((2 * F, H // 16), dtype=torch.uint8, device="cuda")
    layers = []
    t0 = time.time()
    for l in range(L):
        gu = torch.empty(E * gu_b, dtype=torch.uint8, device="cuda")
        dn = torch.empty(E * d_b, dtype=torch.uint8, device="cuda")
        g_gu = torch.empty(E, dtype=torch.float32, device="cuda")
        g_d = torch.empty(E, dtype=torch.float32, device="cuda")
        for proj, buf, nb, (N, K), kind, gl in ((synth.PROJ_GATE_UP, gu, gu_b, (2 * F, H), moe.MOE_W4_GATE_UP, g_gu),
                                                 (synth.PROJ_DOWN, dn, d_b, (H, F), moe.MOE_W4_PLAIN, g_d)):
            c = codes.view(-1)[: N * K].view(N, K)
            s = sf.view(-1)[: N * K // 16].view(N, K // 16)
            for e0 in range(0, E, chunk):
                w = tmp.view(-1)[: chunk * N * K].view(chunk, N, K)
                synth.cuda_expert_weights(w, seed, l, e0, proj)
                for i in range(chunk):
                    e = e0 + i
                    moe.moe_nvfp4_global(w[i], gl[e:e + 1])
                    moe.moe_quantize_nvfp4(w[i], gl[e:e + 1], c, s)
                    moe.moe_pack_nvfp4(c, s, kind, buf[e * nb:(e + 1) * nb])
        layers.append((gu, dn, moe.make_nvfp4_layer(E, H, F, gu, dn, g_gu, g_d), g_gu, g_d))
    torch.cuda.synchronize()
    del tmp, codes, sf
    log(f"built {L} NVFP4 layers in {time.time() - t0:.1f}s")
    return layers


def layer_inputs(seed, l, T):
    import synth
    x = synth.activations_bf16(seed, l, T, H)
    logits = synth.router_logits(seed, l, T, E)
    return x, logits


def pipelined_e2e(torch, dev, stream, run_step, host_in, T, H, E, K, W, nl):
    """End-to-end time (ms) of K stream-ordered steps through the C ABI
    with host buffers.  Every step copies its inputs (x then the logits, one
    pinned buffer per layer) host -> device and its result y device -> host.
    The copies run on two copy streams beside the neighbouring steps' kernels;
    device inputs and outputs are double-buffered, and the kernels stay in
    order on `stream`.  Returns the H2D bytes per step too."""
    xb = T * H * 2
    nbytes = host_in[0].numel()
    dxl = [torch.empty(nbytes, dtype=torch.uint8, device=dev) for _ in range(2)]
    dx = [b[:xb].view(torch.int16).view(T, H) for b in dxl]
    dl = [b[xb:].view(torch.float32).view(T, E) for b in dxl]
    dy = [torch.empty((T, H), dtype=torch.int16, device=dev) for _ in range(2)]
    hy = [torch.empty((T, H), dtype=torch.int16).pin_memory() for _ in range(2)]
    cs, ds = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_k = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def steps(n, first):
        cs.wait_stream(stream)
        ds.wait_stream(stream)
        for i in range(n):
            l, b = (first + i) % nl, i % 2
            if i >= 2:
                cs.wait_event(ev_k[b])  # the step that read this input buffer is done
            with torch.cuda.stream(cs):
                dxl[b].copy_(host_in[l], non_blocking=True)
                ev_in[b].record(cs)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])  # this output buffer's last result has been read
            with torch.cuda.stream(stream):
                run_step(l, dx[b], dl[b], dy[b])
            ev_k[b].record(stream)
            ds.wait_event(ev_k[b])
            with torch.cuda.stream(ds):
                hy[b].copy_(dy[b], non_blocking=True)
                ev_out[b].record(ds)
        stream.wait_stream(cs)
        stream.wait_stream(ds)

    steps(2, 0)
    torch.cuda.synchronize()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    steps(K, W)
    a1.record(stream)
    a1.synchronize()
    return a0.elapsed_time(a1), nbytes


def pinned_inputs(torch, x_list, lg_list):
    """One pinned host buffer per layer: the bf16 activations, then the fp32 logits."""
    out = []
    for x, lg in zip(x_list, lg_list):
        xb = np.ascontiguousarray(x).view(np.uint8).reshape(-1)
        lb = np.ascontiguousarray(lg, dtype=np.float32).view(np.uint8).reshape(-1)
        buf = torch.empty(xb.size + lb.size, dtype=torch.uint8).pin_memory()
        buf[:xb.size].copy_(torch.from_numpy(xb))
        buf[xb.size:].copy_(torch.from_numpy(lb))
        out.append(buf)
    return out


def run_gpu(args, log):
    global LAYERS
    LAYERS = args.layers
    import torch
    import quantized_moe_route_b200 as moe
    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    T = args.tokens
    seed = 1000 + rank
    fmt = "nvfp4" if args.workload == "nvfp4-decode" else "w4"
    layers = build_layers(LAYERS, seed, log, fmt)
    decode_layer = moe.moe_decode_layer_nvfp4 if fmt == "nvfp4" else moe.moe_decode_layer_w4a16
    k = TOPK
    # per-layer device inputs (activations and router logits of every layer)
    xs, ls, uniq = [], [], []
    for l in range(LAYERS):
        x, lg = layer_inputs(seed, l, T)
        xs.append(torch.from_numpy(x.view(np.int16)).to(dev))
        ls.append(torch.from_numpy(lg).to(dev))
        uniq.append(len(set(np.argsort(-lg, axis=1, kind="stable")[:, :k].ravel().tolist())))
    y = torch.empty((T, H), dtype=torch.int16, device=dev)
    ws = torch.zeros(moe.moe_decode_layer_workspace_bytes(T, k, H, F), dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def step(l, ev=None):
        # one launch: route + weight-streaming expert FFN + combine
        if ev is not None:
            ev[0].record(stream)
        decode_layer(layers[l][2], xs[l], ls[l], k, y, ws, stream=stream)
        if ev is not None:
            ev[1].record(stream)

    def capture(fn, steps, first, events=None):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(steps):
                if events is None:
                    fn((first + i) % LAYERS)
                else:
                    fn((first + i) % LAYERS, events[i])
        return g

    def run_steps(fn, K, first):
        """Exactly K steps: full graphs of G steps plus one remainder graph."""
        G = min(K, args.graph_steps)
        graphs = []
        if K // G:
            graphs.append((capture(fn, G, first), K // G))
        if K % G:
            graphs.append((capture(fn, K % G, first + (K // G) * G), 1))
        return graphs

    def replay(graphs):
        with torch.cuda.stream(stream):  # a graph replays on the current stream
            for g, n in graphs:
                for _ in range(n):
                    g.replay()

    K, W = args.steps, args.warmup
    for l in range(min(W, LAYERS)):  # eager first touches, untimed
        step(l)
    torch.cuda.synchronize()
    g_warm = run_steps(step, W, 0)
    g_main = run_steps(step, K, W)
    replay(g_warm)
    torch.cuda.synchronize()

    dist_barrier()
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        dist_barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        replay(g_main)
        e1.record(stream)
        e1.synchronize()
        torch.cuda.synchronize()
        dist_barrier()
    ms = dist_max(e0.elapsed_time(e1))
    tokens = K * T * world
    value = job_throughput(K * T, world, ms)

    # Each step is exactly one launch of the decode kernel, so the timed
    # region over K is that kernel's average launch duration (back to back,
    # PDL overlap included).  For reference, a second pass brackets every
    # launch with its own events (which serialises the launches).
    P = min(K, args.graph_steps)
    evs = [(torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True))
           for _ in range(P)]
    g_prof = capture(step, P, W, evs)
    with torch.cuda.stream(stream):
        g_prof.replay()
    torch.cuda.synchronize()
    isolated_ms = sum(a.elapsed_time(b) for a, b in evs) / P
    dur_ms = ms / K
    # streamed expert bytes + activations + logits in, y out (timed steps)
    alg_bytes = sum(uniq[(W + i) % LAYERS] * EXPERT_BYTES + T * H * 2 + T * E * 4 + T * H * 2
                    for i in range(K)) / K
    peak, peak_kind = peaks()
    achieved = alg_bytes / (dur_ms / 1e3) / 1e9

    # end to end through the C ABI with host buffers: every step copies its
    # inputs (x and the logits, one pinned buffer) host -> device and its
    # result y device -> host.  The copies run on two copy streams and
    # overlap the neighbouring steps' kernels (double-buffered device inputs
    # and outputs); the kernels stay in order on the decode stream.
    xl_bytes = T * H * 2 + T * E * 4
    hxl = []
    for l in range(LAYERS):
        x, lg = layer_inputs(seed, l, T)
        buf = torch.empty(xl_bytes, dtype=torch.uint8).pin_memory()
        buf[:T * H * 2].copy_(torch.from_numpy(x.view(np.uint8).reshape(-1)))
        buf[T * H * 2:].copy_(torch.from_numpy(lg.view(np.uint8).reshape(-1)))
        hxl.append(buf)
    hy = [torch.empty((T, H), dtype=torch.int16).pin_memory() for _ in range(2)]
    dxl = [torch.empty(xl_bytes, dtype=torch.uint8, device=dev) for _ in range(2)]
    dx = [b[:T * H * 2].view(torch.int16).view(T, H) for b in dxl]
    dl = [b[T * H * 2:].view(torch.float32).view(T, E) for b in dxl]
    dy = [torch.empty((T, H), dtype=torch.int16, device=dev) for _ in range(2)]
    cs, ds = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_k = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_steps(n, first):
        cs.wait_stream(stream)
        ds.wait_stream(stream)
        for i in range(n):
            l, b = (first + i) % LAYERS, i % 2
            if i >= 2:
                cs.wait_event(ev_k[b])  # the kernel that read this input buffer is done
            with torch.cuda.stream(cs):
                dxl[b].copy_(hxl[l], non_blocking=True)
                ev_in[b].record(cs)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])  # this output buffer's last result has been read
            decode_layer(layers[l][2], dx[b], dl[b], k, dy[b], ws, stream=stream)
            ev_k[b].record(stream)
            ds.wait_event(ev_k[b])
            with torch.cuda.stream(ds):
                hy[b].copy_(dy[b], non_blocking=True)
                ev_out[b].record(ds)
        stream.wait_stream(cs)
        stream.wait_stream(ds)

    def capture_e2e(n, first):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            e2e_steps(n, first)
        return g

    with torch.cuda.stream(stream):
        e2e_steps(3, 0)
    stream.synchronize()
    Ge = min(K, args.graph_steps)
    g_e2e = []
    if K // Ge:
        g_e2e.append((capture_e2e(Ge, W), K // Ge))
    if K % Ge:
        g_e2e.append((capture_e2e(K % Ge, W + (K // Ge) * Ge), 1))
    replay(g_e2e)
    torch.cuda.synchronize()
    dist_barrier()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    replay(g_e2e)
    a1.record(stream)
    a1.synchronize()
    e2e_ms = dist_max(a0.elapsed_time(a1))
    e2e_value = tokens / (e2e_ms / 1e3)

    out = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": DTYPE_NV if fmt == "nvfp4" else DTYPE_W4, "data": "synthetic",
        "config": {"workload": NV_WORKLOAD if fmt == "nvfp4" else WORKLOAD, "experts": E, "top_k": k, "hidden": H,
                   "expert_width": F, "tokens_per_step": T, "resident_layers": LAYERS, "seed": 1000,
                   "l2": f"inputs larger than L2 ({LAYERS}-layer rotation, {LAYERS * E * EXPERT_BYTES / 1e9:.1f} GB)",
                   "parallelism": f"replicas x{world}",
                   "launch": f"one kernel per step (route + FFN + combine), CUDA graphs of "
                             f"{min(K, args.graph_steps)} steps, programmatic dependent launch"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak,
                     "traffic": DECODE_TRAFFIC.get(fmt) if T == 1 else None,
                     "traffic_source": ("ncu capture, one launch at 1 token: profiles/decode_kernel_"
                                        + ("nvfp4_" if fmt == "nvfp4" else "") + "single_layer_T1.md")
                     if T == 1 else "not captured at this batch size",
                     "kernel": f"moe::decode_kernel<{'nvfp4' if fmt == 'nvfp4' else 'int4'}, fused>",
                     "peak_kind": peak_kind, "alg_bytes_per_launch": alg_bytes,
                     "avg_launch_us": dur_ms * 1e3, "isolated_launch_us": isolated_ms * 1e3},
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": xl_bytes,
                "d2h_bytes_per_step": T * H * 2,
                "overlap": "each step's copies run on copy streams beside the neighbouring steps' kernels"},
        "gpu_launches": K,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(seed, T, budget_s=args.cpu_seconds, log=log, fmt=fmt)
    del g_main, g_warm, g_prof, g_e2e
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return out if rank == 0 else None


PREFILL_WORKLOAD = ("grouped prefill: 2048 tokens x top-8 = 16,384 routed rows over 256 experts "
                    "(router logits N(0,1) + Zipf(1.1) expert bias), hidden 2048, expert width 512; "
                    "route, permute, tcgen05 grouped FFN, combine; 4 resident layers rotated")


def run_gpu_prefill(args, log):
    import torch
    import synth
    import quantized_moe_route_b200 as moe
    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    T, k, nl = args.tokens, TOPK, args.layers
    seed = 3000 + rank
    layers = build_layers(nl, seed, log)
    bias = synth.zipf_bias(seed, E)
    xs, ls = [], []
    for l in range(nl):
        xs.append(torch.from_numpy(synth.activations_bf16(seed, l, T, H).view(np.int16)).to(dev))
        ls.append(torch.from_numpy((synth.router_logits(seed, l, T, E) + bias[None, :]).astype(np.float32)).to(dev))
    R = T * k
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    sorted_rows = torch.empty(R, dtype=torch.int32, device=dev)
    inv = torch.empty(R, dtype=torch.int32, device=dev)
    pws = torch.empty(moe.moe_permute_workspace_bytes(T, k, E), dtype=torch.uint8, device=dev)
    x_perm = torch.empty((R, H), dtype=torch.int16, device=dev)
    y_perm = torch.empty((R, H), dtype=torch.int16, device=dev)
    fws = torch.empty(moe.moe_prefill_workspace_bytes(R, F), dtype=torch.uint8, device=dev)
    y = torch.empty((T, H), dtype=torch.int16, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def step(l, ev=None, xin=None, lin=None, yout=None):
        moe.moe_route(ls[l] if lin is None else lin, k, idx, w, stream=stream)
        moe.moe_permute(idx, E, counts, offsets, sorted_rows, inv, pws, x=xs[l] if xin is None else xin,
                        x_perm=x_perm, stream=stream)
        if ev is not None:
            ev[0].record(stream)
        moe.moe_ffn_grouped_prefill(layers[l][2], x_perm, offsets, y_perm, fws, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        moe.moe_unpermute_combine(y_perm, w, y if yout is None else yout, inv=inv, stream=stream)

    K, W = args.steps, args.warmup
    with torch.cuda.stream(stream):
        for i in range(W):
            step(i % nl)
    torch.cuda.synchronize()
    dist_barrier()
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        dist_barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for i in range(K):
                step((W + i) % nl)
            e1.record(stream)
        e1.synchronize()
        torch.cuda.synchronize()
        dist_barrier()
    ms = dist_max(e0.elapsed_time(e1))
    tokens = K * T * world
    value = job_throughput(K * T, world, ms)

    # kernel-duration pass: events around the two grouped-GEMM launches
    P = min(K, 50)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(P)]
    with torch.cuda.stream(stream):
        for i in range(P):
            step((W + i) % nl, evs[i])
    torch.cuda.synchronize()
    dur_ms = sum(a.elapsed_time(b) for a, b in evs) / P
    flops = R * 6.0 * H * F
    achieved = flops / (dur_ms / 1e3) / 1e12
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peak, peak_kind = float(json.load(f)["bf16_tflops_sustained"]), "measured (sustained bf16)"
    except Exception:
        peak, peak_kind = 1400.0, "fallback (sustained bf16)"

    # end to end: each step copies x and the logits (one pinned buffer) in and
    # y out, on copy streams beside the neighbouring steps' kernels
    import synth as _s
    host_in = pinned_inputs(torch, [_s.activations_bf16(seed, l, T, H) for l in range(nl)],
                            [_s.router_logits(seed, l, T, E) + bias[None, :] for l in range(nl)])
    e2e_ms, h2d_bytes = pipelined_e2e(torch, dev, stream,
                                      lambda l, xin, lin, yout: step(l, xin=xin, lin=lin, yout=yout),
                                      host_in, T, H, E, K, W, nl)
    e2e_ms = dist_max(e2e_ms)

    out = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int4 weights (f16 scale/min), bf16 activations, fp32 accumulate", "data": "synthetic",
        "config": {"workload": PREFILL_WORKLOAD, "experts": E, "top_k": k, "hidden": H, "expert_width": F,
                   "tokens_per_step": T, "routed_rows": R, "resident_layers": nl,
                   "l2": "inputs larger than L2 (453 MB of experts per layer, 67 MB permuted rows)",
                   "parallelism": f"replicas x{world}", "launch": "stream-ordered, PDL into the FFN kernels"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": PREFILL_TRAFFIC["w4"],
                     "traffic_source": "ncu capture of the gate/up and down launches of one layer (2048 tokens): "
                                       "profiles/prefill_kernel_grouped_2048tok.md",
                     "kernel": "moe::prefill_kernel (gate/up + down launches)", "peak_kind": peak_kind,
                     "alg_flop_per_launch_pair": flops, "avg_pair_us": dur_ms * 1e3},
        "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d_bytes,
                "d2h_bytes_per_step": T * H * 2,
                "overlap": "each step's copies run on copy streams beside the neighbouring steps' kernels"},
        "gpu_launches": 8 * K,  # route, histogram, scan, scatter, gather, gate/up, down, combine
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline_prefill(seed, bias, budget_s=args.cpu_seconds, log=log)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return out if rank == 0 else None


NVP_WORKLOAD = ("NVFP4 grouped prefill: 512 tokens x top-8 = 4,096 routed rows over 256 experts (router logits "
                "N(0,1) + Zipf(1.1) expert bias), hidden 2048, expert width 512; route, permute, per-row NVFP4 "
                "quantisation of the grouped rows, block-scaled tcgen05 grouped FFN, combine; 8 resident layers rotated")


def run_gpu_prefill_nvfp4(args, log):
    """Config 5's prefill leg: HBM-bound (the touched experts' 4.5-bit weights
    dominate the bytes; the FP4 tensor cores need a few microseconds)."""
    import torch
    import synth
    import quantized_moe_route_b200 as moe
    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    T, k, nl = args.tokens, TOPK, args.layers
    seed = 4000 + rank
    layers = build_layers(nl, seed, log, "nvfp4")
    bias = synth.zipf_bias(seed, E)
    xs, ls, uniq = [], [], []
    for l in range(nl):
        xs.append(torch.from_numpy(synth.activations_bf16(seed, l, T, H).view(np.int16)).to(dev))
        lg = (synth.router_logits(seed, l, T, E) + bias[None, :]).astype(np.float32)
        ls.append(torch.from_numpy(lg).to(dev))
        uniq.append(len(set(np.argsort(-lg, axis=1, kind="stable")[:, :k].ravel().tolist())))
    R = T * k
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    sorted_rows = torch.empty(R, dtype=torch.int32, device=dev)
    inv = torch.empty(R, dtype=torch.int32, device=dev)
    pws = torch.empty(moe.moe_permute_workspace_bytes(T, k, E), dtype=torch.uint8, device=dev)
    xc = torch.empty((R, H // 2), dtype=torch.uint8, device=dev)
    xsf = torch.empty((R, H // 16), dtype=torch.uint8, device=dev)
    xg = torch.empty(R, dtype=torch.float32, device=dev)
    y_perm = torch.empty((R, H), dtype=torch.int16, device=dev)
    fws = torch.empty(moe.moe_prefill_nvfp4_workspace_bytes(R, F), dtype=torch.uint8, device=dev)
    y = torch.empty((T, H), dtype=torch.int16, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def step(l, ev=None, xin=None, lin=None, yout=None):
        moe.moe_route(ls[l] if lin is None else lin, k, idx, w, stream=stream)
        moe.moe_permute(idx, E, counts, offsets, sorted_rows, inv, pws, stream=stream)
        moe.moe_quantize_nvfp4_rows(xs[l] if xin is None else xin, xc, xsf, xg, src_rows=sorted_rows, src_div=k,
                                    rows=R, stream=stream)
        if ev is not None:
            ev[0].record(stream)
        moe.moe_ffn_grouped_prefill_nvfp4(layers[l][2], xc, xsf, xg, offsets, y_perm, fws, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        moe.moe_unpermute_combine(y_perm, w, y if yout is None else yout, inv=inv, stream=stream)

    K, W = args.steps, args.warmup
    with torch.cuda.stream(stream):
        for i in range(W):
            step(i % nl)
    torch.cuda.synchronize()
    dist_barrier()
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        dist_barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for i in range(K):
                step((W + i) % nl)
            e1.record(stream)
        e1.synchronize()
        torch.cuda.synchronize()
        dist_barrier()
    ms = dist_max(e0.elapsed_time(e1))
    tokens = K * T * world
    value = job_throughput(K * T, world, ms)

    # kernel-duration pass: events around the grouped FFN call (gate/up, h
    # quantisation, down: three launches)
    P = min(K, 50)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(P)]
    with torch.cuda.stream(stream):
        for i in range(P):
            step((W + i) % nl, evs[i])
    torch.cuda.synchronize()
    dur_ms = sum(a.elapsed_time(b) for a, b in evs) / P
    # algorithmic bytes of the call: touched experts' packed weights, the
    # quantised rows in, h out (fp32) and back in, its codes out and in, y_perm out
    act = R * (H // 2 + H // 16 + 4)
    hq = R * (F // 2 + F // 16 + 4)
    alg_bytes = sum(uniq[(W + i) % nl] * EXPERT_BYTES for i in range(P)) / P + act + 2 * R * F * 4 + 2 * hq + R * H * 2
    peak, peak_kind = peaks()
    achieved = alg_bytes / (dur_ms / 1e3) / 1e9
    flops = R * 6.0 * H * F

    # end to end: each step copies x and the logits (one pinned buffer) in and
    # y out, on copy streams beside the neighbouring steps' kernels
    import synth as _s
    host_in = pinned_inputs(torch, [_s.activations_bf16(seed, l, T, H) for l in range(nl)],
                            [_s.router_logits(seed, l, T, E) + bias[None, :] for l in range(nl)])
    e2e_ms, h2d_bytes = pipelined_e2e(torch, dev, stream,
                                      lambda l, xin, lin, yout: step(l, xin=xin, lin=lin, yout=yout),
                                      host_in, T, H, E, K, W, nl)
    e2e_ms = dist_max(e2e_ms)

    out = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": DTYPE_NV, "data": "synthetic",
        "config": {"workload": NVP_WORKLOAD, "experts": E, "top_k": k, "hidden": H, "expert_width": F,
                   "tokens_per_step": T, "routed_rows": R, "resident_layers": nl,
                   "l2": f"inputs larger than L2 ({nl} layers x 453 MB of experts rotated)",
                   "parallelism": f"replicas x{world}", "launch": "stream-ordered, PDL into the FFN kernels"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": PREFILL_TRAFFIC["nvfp4"],
                     "traffic_source": "ncu capture of the gate/up and down launches of one layer (512 tokens; "
                                       "the h quantise launch between them is not included): "
                                       "profiles/prefill_nvfp4_kernel_grouped_512tok.md",
                     "kernel": "moe::prefill_nvfp4_kernel (gate/up + h quantise + down launches)",
                     "peak_kind": peak_kind, "alg_bytes_per_call": alg_bytes, "avg_call_us": dur_ms * 1e3,
                     "tflops": flops / (dur_ms / 1e3) / 1e12},
        "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d_bytes,
                "d2h_bytes_per_step": T * H * 2,
                "overlap": "each step's copies run on copy streams beside the neighbouring steps' kernels"},
        "gpu_launches": 9 * K,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline_prefill_nvfp4(seed, bias, T, budget_s=args.cpu_seconds, log=log)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return out if rank == 0 else None


def cpu_baseline_prefill_nvfp4(seed, bias, T, budget_s, log):
    """The oracle on sampled tokens of the NVFP4 prefill batch (tokens/s)."""
    import oracle
    import synth
    import torch
    x = synth.activations_bf16(seed, 0, T, H)
    lg = (synth.router_logits(seed, 0, T, E) + bias[None, :]).astype(np.float32)
    idx, _ = oracle.route(lg, TOPK)
    toks = list(range(0, T, 61))[:6]
    experts = {}
    for e in sorted(set(idx[toks].ravel().tolist())):
        wg = torch.empty((1, 2 * F, H), device="cuda")
        wd = torch.empty((1, H, F), device="cuda")
        synth.cuda_expert_weights(wg, seed, 0, e, synth.PROJ_GATE_UP)
        synth.cuda_expert_weights(wd, seed, 0, e, synth.PROJ_DOWN)
        experts[e] = (oracle_quantize(wg[0].cpu().numpy(), "nvfp4"), oracle_quantize(wd[0].cpu().numpy(), "nvfp4"))
    t0 = time.time()
    n = 0
    while True:
        t = toks[n % len(toks)]
        oracle_forward(x[t:t + 1], lg[t:t + 1], experts, "nvfp4")
        n += 1
        if time.time() - t0 >= budget_s:
            break
    dt = time.time() - t0
    return {"value": n / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} tokens of the {T}-token NVFP4 prefill batch ({len(toks)} distinct, all 8 experts each), "
                      f"{dt:.1f}s"}


def cpu_baseline_prefill(seed, bias, budget_s, log):
    """The oracle on sampled tokens of the prefill workload (rows per second
    scaled to tokens/s); weights of the sampled tokens' experts only."""
    import oracle
    import synth
    T = 2048
    x = synth.activations_bf16(seed, 0, T, H)
    lg = (synth.router_logits(seed, 0, T, E) + bias[None, :]).astype(np.float32)
    idx, _ = oracle.route(lg, TOPK)
    toks = list(range(0, T, 97))[:8]
    need = sorted(set(idx[toks].ravel().tolist()))
    import torch
    experts = {}
    for e in need:
        wg = torch.empty((1, 2 * F, H), device="cuda")
        wd = torch.empty((1, H, F), device="cuda")
        synth.cuda_expert_weights(wg, seed, 0, e, synth.PROJ_GATE_UP)
        synth.cuda_expert_weights(wd, seed, 0, e, synth.PROJ_DOWN)
        experts[e] = (oracle.quantize_w4(wg[0].cpu().numpy()), oracle.quantize_w4(wd[0].cpu().numpy()))
    t0 = time.time()
    n = 0
    while True:
        t = toks[n % len(toks)]
        oracle.moe_forward_w4(x[t:t + 1], lg[t:t + 1], TOPK, experts)
        n += 1
        if time.time() - t0 >= budget_s:
            break
    dt = time.time() - t0
    return {"value": n / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} tokens of the 2048-token prefill batch (8 distinct, all 8 experts each), {dt:.1f}s"}


# ---------------------------------------------------------------------------- CPU oracle
def oracle_quantize(w, fmt):
    import oracle
    if fmt == "nvfp4":
        G = oracle.nvfp4_global(w)
        return (*oracle.nvfp4_quantize(w, G), G)
    return oracle.quantize_w4(w)


def oracle_forward(x, lg, experts, fmt):
    """One layer through the oracle: route, expert FFN per row, combine."""
    import oracle
    if fmt != "nvfp4":
        return oracle.moe_forward_w4(x, lg, TOPK, experts)[3]
    idx, w = oracle.route(lg, TOPK)
    ys = []
    for t in range(x.shape[0]):
        Y = np.stack([oracle.expert_ffn_nvfp4(x[t], *experts[int(e)]) for e in idx[t]])
        ys.append(oracle.combine(Y, w[t:t + 1])[0])
    return np.stack(ys)


def oracle_pool(seed, T, n, log, use_gpu_generator, fmt="w4"):
    """n sampled token-layers: canonical weights of their routed experts, built
    with the seeded generator and the oracle's own quantiser."""
    import oracle
    import synth
    pool = []
    t0 = time.time()
    for l in range(n):
        x, lg = layer_inputs(seed, l, T)
        idx, _ = oracle.route(lg, TOPK)
        experts = {}
        for e in sorted(set(idx.ravel().tolist())):
            if use_gpu_generator:
                import torch
                wg = torch.empty((1, 2 * F, H), device="cuda")
                wd = torch.empty((1, H, F), device="cuda")
                synth.cuda_expert_weights(wg, seed, l, e, synth.PROJ_GATE_UP)
                synth.cuda_expert_weights(wd, seed, l, e, synth.PROJ_DOWN)
                a, b = wg[0].cpu().numpy(), wd[0].cpu().numpy()
            else:
                a = synth.expert_weights(seed, l, e, synth.PROJ_GATE_UP, 2 * F, H)
                b = synth.expert_weights(seed, l, e, synth.PROJ_DOWN, H, F)
            experts[e] = (oracle_quantize(a, fmt), oracle_quantize(b, fmt))
        pool.append((x, lg, experts))
    log(f"oracle pool of {n} token-layers built in {time.time() - t0:.1f}s")
    return pool


def cpu_baseline(seed, T, budget_s, log, fmt="w4"):
    pool = oracle_pool(seed, T, 4, log, use_gpu_generator=True, fmt=fmt)
    t0 = time.time()
    n = 0
    while True:
        x, lg, experts = pool[n % len(pool)]
        oracle_forward(x, lg, experts, fmt)
        n += 1
        if time.time() - t0 >= budget_s:
            break
    dt = time.time() - t0
    return {"value": n * T / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} token-layer steps (T={T}) over a pool of {len(pool)} sampled layers, {dt:.1f}s"}


def run_reference(args, log):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    import oracle
    T = args.tokens
    pool = oracle_pool(1000, T, 4, log, use_gpu_generator=False)
    for i in range(args.warmup):
        x, lg, ex = pool[i % len(pool)]
        oracle.moe_forward_w4(x, lg, TOPK, ex)
    t0 = time.time()
    for i in range(args.steps):
        x, lg, ex = pool[i % len(pool)]
        oracle.moe_forward_w4(x, lg, TOPK, ex)
    dt = time.time() - t0
    value = args.steps * T / dt
    sample = f"{args.steps} token-layer steps (T={T}) rotating over {len(pool)} sampled layers"
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int4 weights (f16 scale/min), bf16 activations, fp32 accumulate", "data": "synthetic",
        "config": {"workload": WORKLOAD, "experts": E, "top_k": TOPK, "hidden": H, "expert_width": F,
                   "tokens_per_step": T, "parallelism": "single CPU thread (oracle)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100000, help="timed steps")
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="decode", choices=["decode", "prefill", "nvfp4-decode", "nvfp4-prefill"])
    ap.add_argument("--tokens", type=int, default=None, help="tokens per step (decode 1, prefill 2048)")
    ap.add_argument("--layers", type=int, default=LAYERS,
                    help="resident layers the steps rotate over (40 = 18.1 GB, larger than L2)")
    ap.add_argument("--graph-steps", type=int, default=400, help="steps captured per CUDA graph")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--quiet", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.tokens is None:
        args.tokens = {"prefill": 2048, "nvfp4-prefill": 512}.get(args.workload, 1)
    if args.workload == "prefill" and args.layers == LAYERS:
        args.layers = 4
    if args.workload == "nvfp4-prefill" and args.layers == LAYERS:
        args.layers = 8

    def log(msg):
        if not args.quiet:
            print(f"[bench] {msg}", file=sys.stderr, flush=True)

    if args.impl == "reference":
        out = run_reference(args, log)
    elif args.workload == "prefill":
        out = run_gpu_prefill(args, log)
    elif args.workload == "nvfp4-prefill":
        out = run_gpu_prefill_nvfp4(args, log)
    else:
        out = run_gpu(args, log)
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
