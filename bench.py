#!/usr/bin/env python
"""Benchmark of the routed int4 / NVFP4 MoE FFN hot path on B200.

One JSON line.  Its top level is single-layer decode: one token through one
MoE layer (256 experts, top-8, hidden 2048, expert width 512) per step,
route + weight-streaming expert FFN + combine in one launch, steps rotating
over 40 resident int4 layers (18.1 GB, so the 14.2 MB a step streams never
sits in L2 from an earlier step).  With the default --workload all, a `legs`
object adds:
  decode_stream_T1/T4/T16  40 chained layers per step (x of layer l+1 = y of
                           layer l, fresh router logits per layer), 1/4/16 tokens
  prefill_2048             2048 tokens (Zipf-skewed routing): route, permute,
                           tcgen05 grouped FFN (two launches), combine
  nvfp4_prefill_512        the NVFP4 experts on 512 Zipf-routed tokens
  nvfp4_decode_T1          single-layer decode on 40 resident NVFP4 layers
  decode_shared_T1         single-layer decode with a shared expert (weight 1)
                           beside the 8 routed ones, one launch
  decode_router_T1         single-layer decode with the router linear inside
                           the same launch (x and the bf16 router in)
  router_T1/T2048          router linear (bf16 [256][2048]) fused with routing
  quantize_clip_g64/sym128 the MSE clip-search quantisers (asymmetric g64,
                           symmetric g128) on 128 MB of fp32 weights per step
Each leg carries its own roofline (HBM GB/s, TFLOP/s or fp32 ALU ops against
the measured or derived peak), end-to-end throughput through the C ABI with
host buffers, and the CPU oracle timed on a bounded sample of the same
workload (one core and all cores).

Multi-GPU: one process per GPU (torchrun); each rank is an independent
replica of the workload (the path has no exchange step): barrier + max over
ranks of the device-timed region.

--impl reference times the CPU oracle (plain C, one thread) on the top-level
workload: each step is one token through one layer, rotating over a small
pool of sampled token-layers.
"""
from __future__ import annotations

import argparse
import hashlib
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
EXPERT_BYTES = 1769472  # packed gate/up + down of one expert (36 B per 64 weights, int4 or NVFP4)
METRIC = "routed-expert tokens/s + HBM GB/s (decode), TFLOP/s (prefill) vs roofline"
DTYPE_W4 = "int4 weights (f16 scale/min), bf16 activations, fp32 accumulate"
DTYPE_NV = "nvfp4 weights and activations (e2m1 + e4m3/16 + fp32 global), fp32 accumulate"
WORKLOAD = ("single-layer decode: 256 experts, top-8, hidden 2048, expert width 512, 1 token per step; "
            "steps rotate over 40 resident int4 layers (18.1 GB) with fresh router logits per layer")
NV_WORKLOAD = ("NVFP4 single-layer decode: 256 experts, top-8, hidden 2048, expert width 512, 1 token per step; "
               "E2M1 weights with E4M3 scales per 16 channels and fp32 per-matrix globals, x and h quantised "
               "per token/row in the kernel; steps rotate over 40 resident NVFP4 layers (18.1 GB)")
STREAM_WORKLOAD = ("40-layer decode stream: {T} token(s) per step through 40 chained int4 MoE layers (x of layer l+1 "
                   "= y of layer l), 256 experts, top-8, hidden 2048, expert width 512, fresh router logits "
                   "N(0,1) per layer; 18.1 GB resident")
PREFILL_WORKLOAD = ("grouped prefill: 2048 tokens x top-8 = 16,384 routed rows over 256 experts "
                    "(router logits N(0,1) + Zipf(1.1) expert bias), hidden 2048, expert width 512; "
                    "route, permute, tcgen05 grouped FFN, combine; 4 resident layers rotated")
NVP_WORKLOAD = ("NVFP4 grouped prefill: 512 tokens x top-8 = 4,096 routed rows over 256 experts (router logits "
                "N(0,1) + Zipf(1.1) expert bias), hidden 2048, expert width 512; route, permute, per-row NVFP4 "
                "quantisation of the grouped rows, block-scaled tcgen05 grouped FFN, combine; 8 resident layers "
                "rotated")

SHARED_WORKLOAD = ("single-layer decode with a shared expert: 256 routed experts, top-8, plus one shared expert "
                   "(weight 1) per token, hidden 2048, expert width 512, 1 token per step; steps rotate over 40 "
                   "resident int4 layers of 257 experts")
ROUTER_WORKLOAD = ("router linear + routing: x bf16 [{T}][2048] times a bf16 router [256][2048] (fp32 sums), softmax "
                   "top-8 with renormalised weights, one launch; steps rotate over 160 router matrices (168 MB)")
RDEC_WORKLOAD = ("single-layer decode with the router inside: x bf16 [{T}][2048] and a bf16 router [256][2048] in, "
                 "logits, top-8 routing, 256 int4 experts (expert width 512) and combine in one launch; steps rotate "
                 "over 40 resident layers (18.1 GB of experts, 40 router matrices)")
QUANT_WORKLOAD = ("{what}: fp32 weights N(0, 0.02) [16384][2048] (128 MB) per step, 20 clipping ratios "
                  "1.00 -> 0.81, minimum squared error per group; two input matrices alternate")

# Seeds of the synthetic inputs: weights of the int4 and NVFP4 layer sets,
# and the activations / logits of each leg (offset by the rank).
SEED_W4, SEED_NV = 1000, 4000
SEED_DECODE, SEED_STREAM, SEED_PREFILL, SEED_NVP, SEED_NVD = 1000, 2000, 3000, 4000, 5000
SEED_SHARED, SEED_ROUTER, SEED_QUANT, SEED_RDEC = 6000, 7000, 8000, 9000
PROJ_ROUTER = 2  # generator stream of a layer's router matrix (experts use 0 and 1)
# fp32 operations per weight of the clip-search quantisers, counted from the
# definition: per candidate asym g64 sub, div, rint, max, min, fma, sub, mul,
# add (9); sym g128 div, rint, add, max, min, sub, mul, sub, mul, add (10)
CLIP_OPS_PER_WEIGHT = {"clip_g64": 20 * 9, "sym128": 20 * 10}

# dram__bytes_read.sum + dram__bytes_write.sum per launch of a kernel, from an
# ncu capture, with the digest of the kernel's sources at capture time.  A
# digest that no longer matches the sources makes the bench report null.
KERNEL_SOURCES = {
    "decode": ["decode.cu", "decode_common.cuh", "decode_items.cuh", "common.cuh", "route.cuh", "nvfp4.cuh"],
    "router": ["router.cu", "route.cuh", "common.cuh"],
    "quant": ["w4_clip.cu", "common.cuh"],
    "prefill": ["prefill.cu", "tcgen05.cuh", "common.cuh"],
    "prefill_nvfp4": ["prefill_nvfp4.cu", "tcgen05.cuh", "common.cuh", "nvfp4.cuh"],
}
TRAFFIC = {
    # key -> {"bytes": DRAM read + write of the captured launch, "alg": its algorithmic bytes,
    #         "sha": digest of the kernel's sources, "how": the capture}.  A leg's traffic is
    # bytes / alg x the leg's algorithmic bytes per launch (traffic grows with the unique
    # experts a launch streams; the captures are smaller cases of the same kernel).
    "decode_w4_T1": {"bytes": 14255616, "alg": 14164992, "sha": "43e8b20b61872d94",
                     "how": "profiles/decode_kernel_single_layer_T1.md, 2 resident layers"},
    "decode_w4_shared_T1": {"bytes": 16020992, "alg": 15934464, "sha": "43e8b20b61872d94",
                            "how": "profiles/decode_kernel_single_layer_T1.md, shared expert, 2 resident layers"},
    "decode_router_T1": {"bytes": 15303168, "alg": 15213440, "sha": "43e8b20b61872d94",
                         "how": "profiles/decode_kernel_single_layer_T1.md, router inside, 2 resident layers"},
    "decode_w4_T16": {"bytes": 185648128, "alg": 182403072, "sha": "43e8b20b61872d94",
                      "how": "profiles/decode_kernel_single_layer_T1.md, stream kernel at 16 tokens, "
                             "2 resident layers"},
    "decode_w4_T4": {"bytes": 55533312, "alg": 54890496, "sha": "43e8b20b61872d94",
                     "how": "profiles/decode_kernel_single_layer_T1.md, stream kernel at 4 tokens, 2 resident layers"},
    "prefill_nvfp4_512": {"bytes": 144929536, "alg": 169852928, "sha": "6795a7bcc7dffc35",
                          "how": "profiles/prefill_nvfp4_kernel_grouped_512tok.md, the FFN call's three launches"},
    "decode_nvfp4_T1": {"bytes": 14292480, "alg": 14164992, "sha": "43e8b20b61872d94",
                        "how": "profiles/decode_kernel_nvfp4_single_layer_T1.md, 2 resident layers"},
    "prefill_w4_2048": {"bytes": 314900992, "sha": "45646a7528abf117",
                        "how": "profiles/prefill_kernel_grouped_2048tok.md, gate/up + down launch pair"},
    "router_T2048": {"bytes": 11567360, "alg": 11665408, "sha": "96de99454fcdc218",
                     "how": "profiles/router_kernels_T1_T2048.md, GEMM + routing launches"},
    "router_T1": {"bytes": 1094144, "alg": 1053760, "sha": "96de99454fcdc218",
                  "how": "profiles/router_kernels_T1_T2048.md"},
    "quant_clip_g64": {"bytes": 154823168, "sha": "c8f14825edeba35f",
                       "how": "profiles/clip_search_kernel_128MB.md"},
    "quant_sym128": {"bytes": 154248192, "sha": "c8f14825edeba35f",
                     "how": "profiles/clip_search_kernel_128MB.md"},
}


# ---------------------------------------------------------------------------- helpers
def sources_sha(kernel: str) -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "quantized_moe_route_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_of(key: str, kernel: str, alg=None):
    """(bytes per launch, source note): the captured figure, scaled to the
    leg's algorithmic bytes when both are known, if the kernel's sources still
    have the digest they had at capture time, else (None, why)."""
    rec = TRAFFIC.get(key)
    sha = sources_sha(kernel)
    if rec is None:
        return None, f"not captured for the current sources (sha {sha})"
    if rec["sha"] != sha:
        return None, f"stale: captured on sources {rec['sha']}, current {sha}"
    if alg is not None and rec.get("alg"):
        return rec["bytes"] / rec["alg"] * alg, (f"ncu capture ({rec['how']}) on sources {sha}: "
                                                 f"{rec['bytes']} B for {rec['alg']} algorithmic B, scaled")
    return rec["bytes"], f"ncu capture ({rec['how']}) on sources {sha}"


def hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def bf16_peak_sustained():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops_sustained"]), "measured (sustained bf16)"
    except Exception:
        return 1400.0, "fallback (sustained bf16)"


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


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
            time.sleep(0.15)
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


def job_throughput(units_per_rank: float, world: int, max_ms: float) -> float:
    """Whole-job throughput of independent replicas: every rank's units over
    the slowest rank's time (weak scaling; no data-path exchange)."""
    return units_per_rank * world / (max_ms / 1e3)


def dist_barrier():
    import torch.distributed as dist
    if dist.is_initialized():
        dist.barrier()


def unique_experts(logits: np.ndarray, k: int = TOPK) -> int:
    return len(set(np.argsort(-logits, axis=1, kind="stable")[:, :k].ravel().tolist()))


# ---------------------------------------------------------------------------- layers
def build_layers(L, seed, log):
    """Resident int4 layers, generated, quantised and packed on the GPU.
    Each layer holds E routed experts and, after them, a shared expert (id
    E): the routed descriptor covers the first E, the shared one all E + 1."""
    import torch
    import synth
    import quantized_moe_route_b200 as moe
    gu_b, d_b = moe.moe_w4_packed_bytes(2 * F, H), moe.moe_w4_packed_bytes(H, F)
    chunk = 32
    tmp = torch.empty((chunk, 2 * F, H), dtype=torch.float32, device="cuda")
    codes = torch.empty((chunk * 2 * F, H), dtype=torch.uint8, device="cuda")
    sc = torch.empty((chunk * 2 * F, H // 64), dtype=torch.int16, device="cuda")
    mn = torch.empty_like(sc)
    layers = []
    t0 = time.time()
    for l in range(L):
        gu = torch.empty((E + 1) * gu_b, dtype=torch.uint8, device="cuda")
        dn = torch.empty((E + 1) * d_b, dtype=torch.uint8, device="cuda")
        for proj, buf, nb, (N, K), kind in ((synth.PROJ_GATE_UP, gu, gu_b, (2 * F, H), moe.MOE_W4_GATE_UP),
                                             (synth.PROJ_DOWN, dn, d_b, (H, F), moe.MOE_W4_PLAIN)):
            G = K // 64
            for e0 in range(0, E + 1, chunk):
                n = min(chunk, E + 1 - e0)
                w = tmp.view(-1)[: n * N * K].view(n, N, K)
                synth.cuda_expert_weights(w, seed, l, e0, proj)
                c = codes.view(-1)[: n * N * K].view(n * N, K)
                s = sc.view(-1)[: n * N * G].view(n * N, G)
                m = mn.view(-1)[: n * N * G].view(n * N, G)
                moe.moe_quantize_w4(w.view(n * N, K), c, s, m)
                for i in range(n):
                    e = e0 + i
                    moe.moe_pack_w4(c[i * N:(i + 1) * N], s[i * N:(i + 1) * N], m[i * N:(i + 1) * N], kind,
                                    buf[e * nb:(e + 1) * nb])
        layers.append((gu, dn, moe.make_layer(E, H, F, gu, dn), moe.make_layer(E + 1, H, F, gu, dn)))
    torch.cuda.synchronize()
    del tmp, codes, sc, mn
    log(f"built {L} int4 layers in {time.time() - t0:.1f}s")
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


# ---------------------------------------------------------------------------- timing
class Ctx:
    """Per-process state shared by the legs: distributed setup, device,
    stream, and the resident layer sets (built once)."""

    def __init__(self, args, log):
        import torch
        self.args, self.log = args, log
        self.world, self.rank, self.local = dist_setup()
        torch.cuda.set_device(self.local)
        self.dev = torch.device("cuda", self.local)
        self.stream = torch.cuda.Stream(device=self.dev)
        self._w4, self._nv = None, None

    def w4_layers(self):
        if self._w4 is None:
            self._w4 = build_layers(self.args.layers, SEED_W4 + self.rank, self.log)
        return self._w4

    def nv_layers(self):
        if self._nv is None:
            self._nv = build_layers_nvfp4(self.args.layers, SEED_NV + self.rank, self.log)
        return self._nv

    def capture(self, fn, first, n, events=None):
        """One CUDA graph of steps first .. first + n - 1 (fn(i) enqueues step i)."""
        import torch
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream):
            for i in range(n):
                if events is None:
                    fn(first + i)
                else:
                    fn(first + i, events[i])
        return g

    def graphs(self, fn, first, K):
        """Exactly K steps as graphs of at most --graph-steps steps."""
        G = max(1, min(K, self.args.graph_steps))
        out, i = [], 0
        while i < K:
            n = min(G, K - i)
            out.append(self.capture(fn, first + i, n))
            i += n
        return out

    def replay(self, graphs):
        import torch
        with torch.cuda.stream(self.stream):
            for g in graphs:
                g.replay()

    def timed(self, fn, K, W, n_resident, eager_touch=True):
        """Device time (ms, max over ranks) of exactly K steps W .. W + K - 1,
        after every resident layer has been touched (untimed), W warm-up
        steps and one untimed replay of the timed graphs.  Returns (ms, clock
        summary)."""
        import torch
        if eager_touch:
            with torch.cuda.stream(self.stream):
                for i in range(n_resident):
                    fn(i)
        g_warm = self.graphs(fn, 0, max(W, n_resident))
        g_main = self.graphs(fn, W, K)
        self.replay(g_warm)
        self.replay(g_main)  # a graph's first replay uploads it: keep that out of the timed region
        torch.cuda.synchronize()
        dist_barrier()
        with ClockSampler(self.local) as clk:
            torch.cuda.synchronize()
            dist_barrier()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(self.stream)
            self.replay(g_main)
            e1.record(self.stream)
            e1.synchronize()
            torch.cuda.synchronize()
            dist_barrier()
        ms = dist_max(e0.elapsed_time(e1))
        del g_warm, g_main
        return ms, clk.summary()

    def e2e(self, run_step, host_in, out_shape, K, W, nl):
        """End-to-end time (ms, max over ranks) of K stream-ordered steps through
        the C ABI with host buffers: every step copies its inputs (one pinned
        buffer) host -> device and its result device -> host.  The copies run
        on two copy streams beside the neighbouring steps' kernels; device
        inputs and outputs are double-buffered and the kernels stay in order
        on the compute stream.  run_step(i, d_in, d_out) enqueues step i.
        Returns (ms, h2d bytes per step, d2h bytes per step)."""
        import torch
        dev, stream = self.dev, self.stream
        nbytes = host_in[0].numel()
        din = [torch.empty(nbytes, dtype=torch.uint8, device=dev) for _ in range(2)]
        dout = [torch.empty(out_shape, dtype=torch.int16, device=dev) for _ in range(2)]
        hout = [torch.empty(out_shape, dtype=torch.int16).pin_memory() for _ in range(2)]
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
                    din[b].copy_(host_in[l], non_blocking=True)
                    ev_in[b].record(cs)
                stream.wait_event(ev_in[b])
                if i >= 2:
                    stream.wait_event(ev_out[b])  # this output buffer's last result has been read
                with torch.cuda.stream(stream):
                    run_step(first + i, din[b], dout[b])
                ev_k[b].record(stream)
                ds.wait_event(ev_k[b])
                with torch.cuda.stream(ds):
                    hout[b].copy_(dout[b], non_blocking=True)
                    ev_out[b].record(ds)
            stream.wait_stream(cs)
            stream.wait_stream(ds)

        def capture(n, first):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                steps(n, first)
            return g

        with torch.cuda.stream(stream):
            steps(3, 0)
        stream.synchronize()
        G = max(1, min(K, self.args.graph_steps))
        gs, i = [], 0
        while i < K:
            n = min(G, K - i)
            gs.append(capture(n, W + i))
            i += n
        self.replay(gs)
        torch.cuda.synchronize()
        dist_barrier()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        self.replay(gs)
        a1.record(stream)
        a1.synchronize()
        ms = dist_max(a0.elapsed_time(a1))
        del gs
        d2h = int(np.prod(out_shape)) * 2
        return ms, nbytes, d2h


def pinned(torch, arrays):
    """One pinned host buffer holding the raw bytes of the arrays, in order."""
    parts = [np.ascontiguousarray(a).view(np.uint8).reshape(-1) for a in arrays]
    n = sum(p.size for p in parts)
    buf = torch.empty(n, dtype=torch.uint8).pin_memory()
    o = 0
    for p in parts:
        buf[o:o + p.size].copy_(torch.from_numpy(p))
        o += p.size
    return buf


def views(buf, specs):
    """Typed views of a device byte buffer: specs = [(torch dtype, shape), ...]."""
    out, o = [], 0
    for dt, shape in specs:
        n = int(np.prod(shape)) * dt.itemsize
        out.append(buf[o:o + n].view(dt).view(*shape))
        o += n
    return out


def hbm_roofline(alg_bytes, dur_ms, kernel, traffic_key, src_kernel, extra=None):
    peak, peak_kind = hbm_peak()
    achieved = alg_bytes / (dur_ms / 1e3) / 1e9
    traffic, tsrc = traffic_of(traffic_key, src_kernel, alg_bytes)
    r = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
         "traffic": traffic, "traffic_source": tsrc, "kernel": kernel, "peak_kind": peak_kind,
         "alg_bytes_per_launch": alg_bytes, "avg_launch_us": dur_ms * 1e3}
    if extra:
        r.update(extra)
    return r


# ---------------------------------------------------------------------------- legs
def leg_decode(ctx, fmt, T, shared=False):
    """Single-layer decode, T tokens per step, one fused launch per step
    (shared: each token also runs the layer's shared expert, weight 1)."""
    import torch
    import quantized_moe_route_b200 as moe
    args, k = ctx.args, TOPK
    layers = ctx.nv_layers() if fmt == "nvfp4" else ctx.w4_layers()
    nl = len(layers)
    call = (moe.moe_decode_layer_nvfp4 if fmt == "nvfp4" else
            moe.moe_decode_layer_w4a16_shared if shared else moe.moe_decode_layer_w4a16)
    desc = 3 if shared else 2
    kk = k + (1 if shared else 0)
    seed = (SEED_NVD if fmt == "nvfp4" else SEED_SHARED if shared else SEED_DECODE) + ctx.rank
    xs, ls, uniq, host = [], [], [], []
    for l in range(nl):
        x, lg = layer_inputs(seed, l, T)
        xs.append(torch.from_numpy(x.view(np.int16)).to(ctx.dev))
        ls.append(torch.from_numpy(lg).to(ctx.dev))
        uniq.append(unique_experts(lg))
        host.append(pinned(torch, [x, lg]))
    y = torch.empty((T, H), dtype=torch.int16, device=ctx.dev)
    ws = torch.zeros(moe.moe_decode_layer_workspace_bytes(T, kk, H, F), dtype=torch.uint8, device=ctx.dev)
    stream = ctx.stream

    def step(i, ev=None):
        l = i % nl
        if ev is not None:
            ev[0].record(stream)
        call(layers[l][desc], xs[l], ls[l], k, y, ws, stream=stream)
        if ev is not None:
            ev[1].record(stream)

    K, W = args.steps, args.warmup
    ms, clocks = ctx.timed(step, K, W, nl)
    value = job_throughput(K * T, ctx.world, ms)
    # each step is one launch, so the timed region over K is the kernel's
    # average launch duration (back to back, PDL overlap included); a second
    # pass brackets every launch with its own events (serialising them)
    P = min(K, args.graph_steps)
    evs = [(torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True))
           for _ in range(P)]
    g = ctx.capture(step, W, P, evs)
    ctx.replay([g])
    ctx.replay([g])
    torch.cuda.synchronize()
    isolated_ms = sum(a.elapsed_time(b) for a, b in evs) / P
    del g
    dur_ms = ms / K
    nexp = 1 if shared else 0  # the shared expert's weights, read once per step
    alg = sum((uniq[(W + i) % nl] + nexp) * EXPERT_BYTES + T * H * 2 + T * E * 4 + T * H * 2
              for i in range(K)) / K
    kname = f"moe::decode_kernel<{'nvfp4' if fmt == 'nvfp4' else 'int4'}, fused>"
    roof = hbm_roofline(alg, dur_ms, kname, f"decode_{fmt}{'_shared' if shared else ''}_T{T}", "decode",
                        {"isolated_launch_us": isolated_ms * 1e3})

    xb = T * H * 2

    def e2e_step(i, din, dout):
        l = i % nl
        x_d, l_d = views(din, [(torch.int16, (T, H)), (torch.float32, (T, E))])
        call(layers[l][desc], x_d, l_d, k, dout, ws, stream=stream)

    e2e_ms, h2d, d2h = ctx.e2e(e2e_step, host, (T, H), K, W, nl)
    assert h2d == xb + T * E * 4
    out = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ctx.world, "steps": K, "warmup": W,
        "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": DTYPE_NV if fmt == "nvfp4" else DTYPE_W4, "data": "synthetic",
        "config": {"workload": NV_WORKLOAD if fmt == "nvfp4" else SHARED_WORKLOAD if shared else WORKLOAD,
                   "experts": E, "top_k": k, "hidden": H, "shared_experts": nexp,
                   "expert_width": F, "tokens_per_step": T, "resident_layers": nl, "seed": seed - ctx.rank,
                   "l2": f"inputs larger than L2 ({nl}-layer rotation, {nl * E * EXPERT_BYTES / 1e9:.1f} GB); "
                         f"every resident layer touched before timing",
                   "parallelism": f"replicas x{ctx.world}",
                   "launch": f"one kernel per step (route + FFN + combine), CUDA graphs of "
                             f"{min(K, args.graph_steps)} steps, programmatic dependent launch"},
        "roofline": roof,
        "e2e": {"value": job_throughput(K * T, ctx.world, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "overlap": "each step's copies run on copy streams beside the neighbouring steps' kernels"},
        "gpu_launches": K,
        "clocks": clocks,
    }
    return out


def leg_stream(ctx, T):
    """40 chained layers per step: layer l reads the previous layer's y."""
    import torch
    import synth
    import quantized_moe_route_b200 as moe
    args, k = ctx.args, TOPK
    layers = ctx.w4_layers()
    nl = len(layers)
    seed = SEED_STREAM + ctx.rank
    x0 = synth.activations_bf16(seed, 0, T, H)
    lgs = np.stack([synth.router_logits(seed, l, T, E) for l in range(nl)])  # [nl][T][E]
    uniq = [unique_experts(lgs[l]) for l in range(nl)]
    d_x0 = torch.from_numpy(x0.view(np.int16)).to(ctx.dev)
    d_lg = torch.from_numpy(lgs).to(ctx.dev)
    ys = [torch.empty((T, H), dtype=torch.int16, device=ctx.dev) for _ in range(nl)]
    ws = torch.zeros(moe.moe_decode_layer_workspace_bytes(T, k, H, F), dtype=torch.uint8, device=ctx.dev)
    stream = ctx.stream

    def chain(x_in, lg, y_out):
        for l in range(nl):
            moe.moe_decode_layer_w4a16(layers[l][2], x_in if l == 0 else ys[l - 1], lg[l], k,
                                       y_out if l == nl - 1 else ys[l], ws, stream=stream)

    def step(i):
        chain(d_x0, d_lg, ys[-1])

    K, W = args.steps, args.warmup
    ms, clocks = ctx.timed(step, K, W, 1)
    value = job_throughput(K * T, ctx.world, ms)
    step_ms = ms / K
    bytes_step = sum(u * EXPERT_BYTES for u in uniq) + nl * (T * H * 2 + T * E * 4 + T * H * 2)
    roof = hbm_roofline(bytes_step / nl, step_ms / nl, "moe::decode_kernel<int4, fused>", f"decode_w4_T{T}",
                        "decode", {"alg_bytes_per_step": bytes_step, "unique_expert_bytes_per_step":
                                   sum(u * EXPERT_BYTES for u in uniq), "launches_per_step": nl})
    host = [pinned(torch, [x0, lgs])]

    def e2e_step(i, din, dout):
        x_d, l_d = views(din, [(torch.int16, (T, H)), (torch.float32, (nl, T, E))])
        chain(x_d, l_d, dout)

    e2e_ms, h2d, d2h = ctx.e2e(e2e_step, host, (T, H), K, W, 1)
    return {
        "metric": METRIC, "value": value, "unit": "tokens/s", "ms_per_step": step_ms, "steps": K, "warmup": W,
        "dtype": DTYPE_W4,
        "unique_expert_gbs": sum(u * EXPERT_BYTES for u in uniq) / (step_ms / 1e3) / 1e9,
        "config": {"workload": STREAM_WORKLOAD.format(T=T), "tokens_per_step": T, "layers_per_step": nl,
                   "unique_experts_per_layer_mean": float(np.mean(uniq)), "seed": SEED_STREAM,
                   "l2": f"inputs larger than L2 ({bytes_step / 1e6:.0f} MB of experts per step)",
                   "launch": f"{nl} kernels per step (one per layer), CUDA graphs, programmatic dependent launch"},
        "roofline": roof,
        "e2e": {"value": job_throughput(K * T, ctx.world, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "overlap": "each step's copies run on copy streams beside the neighbouring steps' kernels"},
        "gpu_launches": nl * K,
        "clocks": clocks,
    }


def _prefill_inputs(seed, T, nl, ctx):
    import torch
    import synth
    bias = synth.zipf_bias(seed, E)
    xs, ls, host, uniq = [], [], [], []
    for l in range(nl):
        x = synth.activations_bf16(seed, l, T, H)
        lg = (synth.router_logits(seed, l, T, E) + bias[None, :]).astype(np.float32)
        xs.append(torch.from_numpy(x.view(np.int16)).to(ctx.dev))
        ls.append(torch.from_numpy(lg).to(ctx.dev))
        host.append(pinned(torch, [x, lg]))
        uniq.append(unique_experts(lg))
    return xs, ls, host, uniq


def leg_prefill(ctx, T=2048, nl=4):
    import torch
    import quantized_moe_route_b200 as moe
    args, k = ctx.args, TOPK
    layers = ctx.w4_layers()[:nl]
    nl = len(layers)
    seed = SEED_PREFILL + ctx.rank
    xs, ls, host, _ = _prefill_inputs(seed, T, nl, ctx)
    R = T * k
    dev = ctx.dev
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
    stream = ctx.stream

    def run(l, x, lg, yout, ev=None):
        moe.moe_route(lg, k, idx, w, stream=stream)
        moe.moe_permute(idx, E, counts, offsets, sorted_rows, inv, pws, x=x, x_perm=x_perm, stream=stream)
        if ev is not None:
            ev[0].record(stream)
        moe.moe_ffn_grouped_prefill(layers[l][2], x_perm, offsets, y_perm, fws, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        moe.moe_unpermute_combine(y_perm, w, yout, inv=inv, stream=stream)

    def step(i, ev=None):
        l = i % nl
        run(l, xs[l], ls[l], y, ev)

    K, W = args.steps, args.warmup
    ms, clocks = ctx.timed(step, K, W, nl)
    value = job_throughput(K * T, ctx.world, ms)
    P = min(K, 50)
    evs = [(torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True))
           for _ in range(P)]
    g = ctx.capture(step, W, P, evs)
    ctx.replay([g])
    ctx.replay([g])
    torch.cuda.synchronize()
    dur_ms = sum(a.elapsed_time(b) for a, b in evs) / P
    del g
    flops = R * 6.0 * H * F
    achieved = flops / (dur_ms / 1e3) / 1e12
    peak, peak_kind = bf16_peak_sustained()
    traffic, tsrc = traffic_of("prefill_w4_2048", "prefill")

    def e2e_step(i, din, dout):
        x_d, l_d = views(din, [(torch.int16, (T, H)), (torch.float32, (T, E))])
        run(i % nl, x_d, l_d, dout)

    e2e_ms, h2d, d2h = ctx.e2e(e2e_step, host, (T, H), K, W, nl)
    return {
        "metric": METRIC, "value": value, "unit": "tokens/s", "ms_per_step": ms / K, "steps": K, "warmup": W,
        "dtype": DTYPE_W4,
        "config": {"workload": PREFILL_WORKLOAD, "tokens_per_step": T, "routed_rows": R, "resident_layers": nl,
                   "seed": SEED_PREFILL,
                   "l2": "inputs larger than L2 (up to 453 MB of experts per layer, 67 MB permuted rows)",
                   "launch": "stream-ordered, programmatic dependent launch through the chain, CUDA graphs"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic, "traffic_source": tsrc,
                     "kernel": "moe::prefill_kernel (gate/up + down launches)", "peak_kind": peak_kind,
                     "alg_flop_per_launch_pair": flops, "avg_pair_us": dur_ms * 1e3},
        "e2e": {"value": job_throughput(K * T, ctx.world, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "overlap": "each step's copies run on copy streams beside the neighbouring steps' kernels"},
        "gpu_launches": 8 * K,  # route, histogram, scan, scatter, gather, gate/up, down, combine
        "clocks": clocks,
    }


def leg_prefill_nvfp4(ctx, T=512, nl=8):
    """Config 5's prefill leg: HBM-bound (the touched experts' 4.5-bit weights
    dominate the bytes; the FP4 tensor cores need a few microseconds)."""
    import torch
    import quantized_moe_route_b200 as moe
    args, k = ctx.args, TOPK
    layers = ctx.nv_layers()[:nl]
    nl = len(layers)
    seed = SEED_NVP + ctx.rank
    xs, ls, host, uniq = _prefill_inputs(seed, T, nl, ctx)
    R = T * k
    dev = ctx.dev
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
    stream = ctx.stream

    def run(l, x, lg, yout, ev=None):
        moe.moe_route(lg, k, idx, w, stream=stream)
        moe.moe_permute(idx, E, counts, offsets, sorted_rows, inv, pws, stream=stream)
        moe.moe_quantize_nvfp4_rows(x, xc, xsf, xg, src_rows=sorted_rows, src_div=k, rows=R, stream=stream)
        if ev is not None:
            ev[0].record(stream)
        moe.moe_ffn_grouped_prefill_nvfp4(layers[l][2], xc, xsf, xg, offsets, y_perm, fws, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        moe.moe_unpermute_combine(y_perm, w, yout, inv=inv, stream=stream)

    def step(i, ev=None):
        l = i % nl
        run(l, xs[l], ls[l], y, ev)

    K, W = args.steps, args.warmup
    ms, clocks = ctx.timed(step, K, W, nl)
    value = job_throughput(K * T, ctx.world, ms)
    P = min(K, 50)
    evs = [(torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True))
           for _ in range(P)]
    g = ctx.capture(step, W, P, evs)
    ctx.replay([g])
    ctx.replay([g])
    torch.cuda.synchronize()
    dur_ms = sum(a.elapsed_time(b) for a, b in evs) / P
    del g
    # algorithmic bytes of the FFN call: touched experts' packed weights, the
    # quantised rows in, h out (fp32) and back in, its codes out and in, y_perm out
    act = R * (H // 2 + H // 16 + 4)
    hq = R * (F // 2 + F // 16 + 4)
    alg = sum(uniq[(W + i) % nl] * EXPERT_BYTES for i in range(P)) / P + act + 2 * R * F * 4 + 2 * hq + R * H * 2
    flops = R * 6.0 * H * F
    roof = hbm_roofline(alg, dur_ms, "moe::prefill_nvfp4_kernel (gate/up + h quantise + down launches)",
                        "prefill_nvfp4_512", "prefill_nvfp4",
                        {"tflops": flops / (dur_ms / 1e3) / 1e12, "alg_bytes_per_call": alg})

    def e2e_step(i, din, dout):
        x_d, l_d = views(din, [(torch.int16, (T, H)), (torch.float32, (T, E))])
        run(i % nl, x_d, l_d, dout)

    e2e_ms, h2d, d2h = ctx.e2e(e2e_step, host, (T, H), K, W, nl)
    return {
        "metric": METRIC, "value": value, "unit": "tokens/s", "ms_per_step": ms / K, "steps": K, "warmup": W,
        "dtype": DTYPE_NV,
        "config": {"workload": NVP_WORKLOAD, "tokens_per_step": T, "routed_rows": R, "resident_layers": nl,
                   "seed": SEED_NVP, "l2": f"inputs larger than L2 ({nl} layers x up to 453 MB of experts rotated)",
                   "launch": "stream-ordered, programmatic dependent launch through the chain, CUDA graphs"},
        "roofline": roof,
        "e2e": {"value": job_throughput(K * T, ctx.world, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "overlap": "each step's copies run on copy streams beside the neighbouring steps' kernels"},
        "gpu_launches": 9 * K,
        "clocks": clocks,
    }


def leg_decode_router(ctx, T):
    """Single-layer decode with the router linear in the same launch: x and
    the layer's bf16 router matrix in, y out."""
    import torch
    import synth
    import quantized_moe_route_b200 as moe
    args, k = ctx.args, TOPK
    layers = ctx.w4_layers()
    nl = len(layers)
    dev, stream = ctx.dev, ctx.stream
    seed = SEED_RDEC + ctx.rank
    tmp = torch.empty((1, E, H), dtype=torch.float32, device=dev)
    wrs, xs, host = [], [], []
    for l in range(nl):
        synth.cuda_expert_weights(tmp, seed, l, 0, PROJ_ROUTER, sigma=1.0 / np.sqrt(H))
        wrs.append(tmp[0].to(torch.bfloat16).view(torch.int16).clone())
        x = synth.activations_bf16(seed, l, T, H)
        xs.append(torch.from_numpy(x.view(np.int16)).to(dev))
        host.append(pinned(torch, [x]))
    del tmp
    y = torch.empty((T, H), dtype=torch.int16, device=dev)
    ws = torch.zeros(moe.moe_decode_layer_router_workspace_bytes(T, k, 0, E, H, F), dtype=torch.uint8, device=dev)
    # the experts each layer's call selects (for the byte count), from one untimed call per layer
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    uniq = []
    for l in range(nl):
        moe.moe_decode_layer_w4a16_router(layers[l][2], xs[l], wrs[l], k, y, ws, idx=idx, w=w, stream=stream)
        stream.synchronize()
        uniq.append(len(np.unique(idx.cpu().numpy())))

    def step(i, ev=None):
        l = i % nl
        if ev is not None:
            ev[0].record(stream)
        moe.moe_decode_layer_w4a16_router(layers[l][2], xs[l], wrs[l], k, y, ws, stream=stream)
        if ev is not None:
            ev[1].record(stream)

    K, W = args.steps, args.warmup
    ms, clocks = ctx.timed(step, K, W, nl)
    value = job_throughput(K * T, ctx.world, ms)
    dur_ms = ms / K
    alg = sum(uniq[(W + i) % nl] * EXPERT_BYTES + E * H * 2 + T * H * 2 + T * H * 2 for i in range(K)) / K
    roof = hbm_roofline(alg, dur_ms, "moe::decode_kernel<int4, fused> (router inside)", f"decode_router_T{T}",
                        "decode", {"router_bytes_per_launch": E * H * 2})

    def e2e_step(i, din, dout):
        (x_d,) = views(din, [(torch.int16, (T, H))])
        moe.moe_decode_layer_w4a16_router(layers[i % nl][2], x_d, wrs[i % nl], k, dout, ws, stream=stream)

    e2e_ms, h2d, d2h = ctx.e2e(e2e_step, host, (T, H), K, W, nl)
    return {
        "metric": METRIC, "value": value, "unit": "tokens/s", "ms_per_step": dur_ms, "steps": K, "warmup": W,
        "dtype": DTYPE_W4 + "; bf16 router, fp32 logits",
        "config": {"workload": RDEC_WORKLOAD.format(T=T), "tokens_per_step": T, "experts": E, "top_k": k,
                   "hidden": H, "expert_width": F, "resident_layers": nl, "seed": SEED_RDEC,
                   "l2": f"inputs larger than L2 ({nl}-layer rotation); every resident layer touched before timing",
                   "launch": "one kernel per step (router linear + route + FFN + combine), CUDA graphs, "
                             "programmatic dependent launch"},
        "roofline": roof,
        "e2e": {"value": job_throughput(K * T, ctx.world, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "overlap": "each step's copies run on copy streams beside the neighbouring steps' kernels"},
        "gpu_launches": K,
        "clocks": clocks,
    }


def alu_peak():
    """fp32 operations per second of the SMs' FP32 pipes: 148 SMs x 128
    lanes x one operation per clock at the maximum SM clock (an FMA counts
    as one operation, as in the per-weight counts)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            mhz = float(json.load(f)["sm_max_mhz"])
        kind = "derived: 148 SMs x 128 fp32 lanes x sm_max_mhz from MEASURED_PEAKS.json"
    except Exception:
        mhz = 1965.0
        kind = "derived: 148 SMs x 128 fp32 lanes x 1965 MHz (nominal max clock)"
    return 148 * 128 * mhz * 1e6 / 1e12, kind


def leg_router(ctx, T):
    """Router linear fused with routing (one launch per step)."""
    import torch
    import synth
    import quantized_moe_route_b200 as moe
    args, k = ctx.args, TOPK
    dev, stream = ctx.dev, ctx.stream
    nw = 160  # 168 MB of router matrices: a step's matrix is never in L2 from an earlier use
    seed = SEED_ROUTER + ctx.rank
    tmp = torch.empty((1, E, H), dtype=torch.float32, device=dev)
    wrs = []
    for l in range(nw):
        synth.cuda_expert_weights(tmp, seed, l, 0, PROJ_ROUTER, sigma=1.0 / np.sqrt(H))
        wrs.append(tmp[0].to(torch.bfloat16).view(torch.int16).clone())
    del tmp
    nx = 16 if T >= 1024 else 160
    host = []
    xs = []
    for l in range(nx):
        x = synth.activations_bf16(seed, l, T, H)
        xs.append(torch.from_numpy(x.view(np.int16)).to(dev))
        host.append(pinned(torch, [x]))
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    ws = torch.zeros(moe.moe_router_route_workspace_bytes(T, E), dtype=torch.uint8, device=dev)

    def step(i, ev=None):
        if ev is not None:
            ev[0].record(stream)
        moe.moe_router_route(xs[i % nx], wrs[i % nw], k, idx, w, ws, stream=stream)
        if ev is not None:
            ev[1].record(stream)

    K, W = args.steps, args.warmup
    ms, clocks = ctx.timed(step, K, W, max(nx, nw))
    value = job_throughput(K * T, ctx.world, ms)
    dur_ms = ms / K
    alg = T * H * 2 + E * H * 2 + T * E * 4 + T * k * 8  # x, Wr, logits, idx + w
    flops = 2.0 * T * E * H
    kname = "moe::router_gemv_kernel" if T <= 16 else "moe::router_mma_kernel + moe::route_kernel (one call)"
    roof = hbm_roofline(alg, dur_ms, kname, f"router_T{T}", "router",
                        {"tflops": flops / (dur_ms / 1e3) / 1e12,
                         "note": "HBM-bound at both sizes: at T=2048 the bytes take longer than the "
                                 "contraction at the measured bf16 peak"})

    def e2e_step(i, din, dout):
        (x_d,) = views(din, [(torch.int16, (T, H))])
        flat = dout.view(-1)
        moe.moe_router_route(x_d, wrs[i % nw], k, flat[: 2 * T * k].view(torch.int32).view(T, k),
                             flat[2 * T * k:].view(torch.float32).view(T, k), ws, stream=stream)

    e2e_ms, h2d, d2h = ctx.e2e(e2e_step, host, (T, 4 * k), K, W, nx)
    return {
        "metric": METRIC, "value": value, "unit": "tokens/s", "ms_per_step": dur_ms, "steps": K, "warmup": W,
        "dtype": "bf16 x and router weights, fp32 sums",
        "config": {"workload": ROUTER_WORKLOAD.format(T=T), "tokens_per_step": T, "experts": E, "top_k": k,
                   "hidden": H, "seed": SEED_ROUTER,
                   "l2": "inputs larger than L2 (160 router matrices rotated, "
                         f"{nx} token batches of {T * H * 2 / 1e6:.1f} MB rotated)",
                   "launch": "one kernel per step, CUDA graphs, programmatic dependent launch"},
        "roofline": roof,
        "e2e": {"value": job_throughput(K * T, ctx.world, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "overlap": "each step's copies run on copy streams beside the neighbouring steps' kernels"},
        "gpu_launches": K * (1 if T <= 16 else 2),
        "clocks": clocks,
    }


def leg_quant(ctx, what):
    """The clip-search quantisers (offline weight conversion): what =
    "clip_g64" (asymmetric group 64) or "sym128" (symmetric group 128)."""
    import torch
    import synth
    import quantized_moe_route_b200 as moe
    args = ctx.args
    dev, stream = ctx.dev, ctx.stream
    N, K = 16384, 2048
    seed = SEED_QUANT + ctx.rank
    mats, host = [], []
    tmp = torch.empty((16, 1024, K), dtype=torch.float32, device=dev)
    for j in range(2):
        synth.cuda_expert_weights(tmp, seed, j, 0, synth.PROJ_GATE_UP)
        mats.append(tmp.view(N, K).clone())
        host.append(mats[-1].cpu().view(torch.uint8).view(-1).pin_memory())
    del tmp
    codes = torch.empty((N, K), dtype=torch.uint8, device=dev)
    gs = 64 if what == "clip_g64" else 128
    scale = torch.empty((N, K // gs), dtype=torch.int16, device=dev)
    minv = torch.empty((N, K // gs), dtype=torch.int16, device=dev)

    def quant(w, c, sc, mn):
        if what == "clip_g64":
            moe.moe_quantize_w4_clip(w, c, sc, mn, stream=stream)
        else:
            moe.moe_quantize_w4_sym128(w, c, sc, stream=stream)

    def step(i, ev=None):
        if ev is not None:
            ev[0].record(stream)
        quant(mats[i % 2], codes, scale, minv)
        if ev is not None:
            ev[1].record(stream)

    Ksteps, W = min(args.steps, 50), args.warmup
    ms, clocks = ctx.timed(step, Ksteps, W, 2)
    dur_ms = ms / Ksteps
    weights = N * K
    value = job_throughput(Ksteps * weights, ctx.world, ms)
    ops = CLIP_OPS_PER_WEIGHT[what]
    peak, peak_kind = alu_peak()
    achieved = weights * ops / (dur_ms / 1e3) / 1e12
    hbm = (weights * 4 + weights + 2 * scale.numel() * (2 if what == "clip_g64" else 1)) / (dur_ms / 1e3) / 1e9
    traffic, tsrc = traffic_of(f"quant_{what}", "quant")

    def e2e_step(i, din, dout):
        (w_d,) = views(din, [(torch.float32, (N, K))])
        quant(w_d, dout.view(torch.uint8).view(N, K), scale, minv)

    e2e_ms, h2d, d2h = ctx.e2e(e2e_step, host, (N, K // 2), Ksteps, W, 2)
    return {
        "metric": "weights quantised per second vs fp32 ALU roofline", "value": value, "unit": "weights/s",
        "ms_per_step": dur_ms, "steps": Ksteps, "warmup": W,
        "dtype": "fp32 weights -> int4 codes + f16 scales (every operation correctly rounded fp32)",
        "config": {"workload": QUANT_WORKLOAD.format(
            what="asymmetric group-64 int4 (f16 scale + min)" if what == "clip_g64"
            else "symmetric group-128 int4 (f16 scale, zero point 8)"),
            "rows": N, "cols": K, "seed": SEED_QUANT,
            "l2": "inputs larger than L2 (two 128 MB matrices alternate)",
            "launch": "one kernel per step, CUDA graphs"},
        "roofline": {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "Tops/s (fp32)",
                     "frac": achieved / peak, "traffic": traffic, "traffic_source": tsrc,
                     "kernel": f"moe::clip_search_kernel<{'sym' if what == 'sym128' else 'asym'}>",
                     "peak_kind": peak_kind, "ops_per_weight": ops, "hbm_gbs": hbm,
                     "avg_launch_us": dur_ms * 1e3},
        "e2e": {"value": job_throughput(Ksteps * weights, ctx.world, e2e_ms), "unit": "weights/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "overlap": "each step's copies run on copy streams beside the neighbouring steps' kernels"},
        "gpu_launches": Ksteps,
        "clocks": clocks,
    }


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


def oracle_experts(w_seed, layer, experts, fmt):
    """Canonical weights of the given experts of one layer, drawn with the
    CPU twin of the seeded generator and quantised by the oracle."""
    import synth
    out = {}
    for e in sorted(set(int(v) for v in experts)):
        a = synth.expert_weights(w_seed, layer, e, synth.PROJ_GATE_UP, 2 * F, H)
        b = synth.expert_weights(w_seed, layer, e, synth.PROJ_DOWN, H, F)
        out[e] = (oracle_quantize(a, fmt), oracle_quantize(b, fmt))
    return out


def oracle_sample(job):
    """The sample one oracle worker evaluates: a list of zero-argument
    evaluations, and the units of the leg's metric each evaluation counts for.
    job = (kind, fmt, w_seed, in_seed, T, worker)."""
    import oracle
    import synth
    kind, fmt, w_seed, in_seed, T, wi = job
    items = []
    if kind == "router":  # single tokens of the batch against one router matrix
        l = wi % 160
        wr = synth.f32_to_bf16_bits(synth.expert_weights(w_seed, l, 0, PROJ_ROUTER, E, H, sigma=1.0 / np.sqrt(H)))
        x = synth.activations_bf16(in_seed, wi % (16 if T >= 1024 else 160), T, H)
        for j in range(4):
            t = (97 * (4 * wi + j) + 13) % T
            xt = x[t:t + 1]
            items.append(lambda xt=xt: oracle.route(oracle.router_logits(xt, wr), TOPK))
        return items, 1
    if kind.startswith("quant_"):  # 64 rows of one input matrix
        w = synth.expert_weights(in_seed, wi % 2, (64 * wi // 1024) % 16, synth.PROJ_GATE_UP, 1024, 2048)
        r0 = (64 * wi) % 1024
        rows = np.ascontiguousarray(w[r0:r0 + 64])
        fn = oracle.quantize_w4_clip if kind == "quant_clip_g64" else oracle.quantize_sym128
        return [lambda: fn(rows)], rows.size
    if kind == "router_decode":  # router linear + one layer, 2 sampled token-layers
        for j in range(2):
            l = (2 * wi + j) % LAYERS
            wr = synth.f32_to_bf16_bits(synth.expert_weights(in_seed, l, 0, PROJ_ROUTER, E, H, sigma=1.0 / np.sqrt(H)))
            x = synth.activations_bf16(in_seed, l, T, H)
            lg = oracle.router_logits(x, wr)
            idx, _ = oracle.route(lg, TOPK)
            ex = oracle_experts(w_seed, l, idx.ravel(), fmt)
            items.append(lambda x=x, wr=wr, ex=ex: oracle.moe_forward_w4(x, oracle.router_logits(x, wr), TOPK, ex))
        return items, T
    if kind == "shared":
        for j in range(2):
            l = (2 * wi + j) % LAYERS
            x, lg = layer_inputs(in_seed, l, T)
            idx, _ = oracle.route(lg, TOPK)
            ex = oracle_experts(w_seed, l, list(idx.ravel()) + [E], fmt)
            sh = ex.pop(E)
            items.append(lambda x=x, lg=lg, ex=ex, sh=sh: oracle.moe_forward_w4_shared(x, lg, TOPK, ex, sh))
        return items, T
    if kind in ("decode", "stream"):
        for j in range(2):
            l = (2 * wi + j) % LAYERS
            if kind == "stream":
                x = synth.activations_bf16(in_seed, 0, T, H)  # a layer's input in the chain has this shape
                lg = synth.router_logits(in_seed, l, T, E)
            else:
                x, lg = layer_inputs(in_seed, l, T)
            idx, _ = oracle.route(lg, TOPK)
            ex = oracle_experts(w_seed, l, idx.ravel(), fmt)
            items.append(lambda x=x, lg=lg, ex=ex: oracle_forward(x, lg, ex, fmt))
        # a decode step is one layer of T tokens; a stream step is 40 layers
        units = T if kind == "decode" else T / LAYERS
    else:  # prefill: single tokens of the Zipf-routed batch, layer 0
        bias = synth.zipf_bias(in_seed, E)
        x = synth.activations_bf16(in_seed, 0, T, H)
        lg = (synth.router_logits(in_seed, 0, T, E) + bias[None, :]).astype(np.float32)
        idx, _ = oracle.route(lg, TOPK)
        for j in range(2):
            t = (97 * (2 * wi + j) + 13) % T
            ex = oracle_experts(w_seed, 0, idx[t], fmt)
            items.append(lambda x=x[t:t + 1], lg=lg[t:t + 1], ex=ex: oracle_forward(x, lg, ex, fmt))
        units = 1
    return items, units


def oracle_worker(job_budget):
    """Evaluate one worker's sample repeatedly until the shared deadline;
    returns (units, seconds).  Runs in a spawned process (or in-process for
    the one-core figure); touches no GPU."""
    job, deadline = job_budget
    items, units = oracle_sample(job)
    n, t0 = 0, time.time()
    while True:
        items[n % len(items)]()
        n += 1
        if time.time() >= deadline and n >= 1:
            break
    return n * units, time.time() - t0


def cpu_baseline(kind, fmt, w_seed, in_seed, T, seconds, log, unit="tokens/s"):
    """The oracle, as it stands, on bounded samples of a leg's workload: one
    core, then one spawned process per host core (rows of the workload split
    over processes, each its own sample).  The value is the all-core figure."""
    import multiprocessing as mp
    t0 = time.time()
    u1, s1 = oracle_worker(((kind, fmt, w_seed, in_seed, T, 0), time.time() + seconds))
    one = u1 / s1
    n = host_cores()
    ctxp = mp.get_context("spawn")
    jobs = [((kind, fmt, w_seed, in_seed, T, i), time.time() + seconds + 6.0) for i in range(n)]
    with ctxp.Pool(n) as pool:
        res = pool.map(oracle_worker, jobs, chunksize=1)
    allc = sum(u / s for u, s in res)
    log(f"cpu baseline {kind}/{fmt}/T={T}: {one:.3g} (1 core) {allc:.3g} ({n} cores) {unit} "
        f"in {time.time() - t0:.0f}s")
    what = {"decode": f"token-layer evaluations (T={T}) over 2 sampled layers per process",
            "stream": f"layer evaluations of the 40-layer chain (T={T}, a step = 40 of them) over 2 sampled layers "
                      f"per process",
            "prefill": f"single tokens of the {T}-token Zipf-routed batch (all 8 experts each), 2 per process",
            "shared": f"token-layer evaluations (T={T}, 8 routed experts + the shared one) over 2 sampled layers "
                      f"per process",
            "router": f"single tokens of the {T}-token batch (router linear + routing), 4 per process",
            "router_decode": f"token-layer evaluations (T={T}, router linear + routing + 8 experts + combine) over "
                             f"2 sampled layers per process",
            "quant_clip_g64": "64 rows x 2048 of the input matrix (asymmetric g64 clip search) per process",
            "quant_sym128": "64 rows x 2048 of the input matrix (symmetric g128 clip search) per process"}[kind]
    return {"value": allc, "unit": unit, "cores": n, "kind": "oracle",
            "sample": f"{what}; about {seconds:.0f}s per process",
            "single_core": {"value": one, "cores": 1, "sample": f"{what.split(' per process')[0]}, "
                                                                 f"{s1:.1f}s on one core"}}


# ---------------------------------------------------------------------------- reference arm
def run_reference(args, log):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    import oracle
    T = args.tokens
    pool = []
    for l in range(4):
        x, lg = layer_inputs(SEED_DECODE, l, T)
        idx, _ = oracle.route(lg, TOPK)
        pool.append((x, lg, oracle_experts(SEED_W4, l, idx.ravel(), "w4")))
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
        "dtype": DTYPE_W4, "data": "synthetic",
        "config": {"workload": WORKLOAD, "experts": E, "top_k": TOPK, "hidden": H, "expert_width": F,
                   "tokens_per_step": T, "parallelism": "single CPU thread (oracle)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------------------- main
def run_native(args, log):
    ctx = Ctx(args, log)
    wl = args.workload
    cpu = ctx.rank == 0 and ctx.world == 1 and not args.no_cpu_baseline
    sec = args.cpu_seconds
    legs, cpu_jobs = {}, {}
    if wl in ("all", "decode"):
        top = leg_decode(ctx, "w4", args.tokens or 1)
        cpu_jobs["top"] = ("decode", "w4", SEED_W4, SEED_DECODE, args.tokens or 1)
    elif wl == "nvfp4-decode":
        top = leg_decode(ctx, "nvfp4", args.tokens or 1)
        cpu_jobs["top"] = ("decode", "nvfp4", SEED_NV, SEED_NVD, args.tokens or 1)
    elif wl == "stream":
        top = leg_stream(ctx, args.tokens or 1)
        cpu_jobs["top"] = ("stream", "w4", SEED_W4, SEED_STREAM, args.tokens or 1)
    elif wl == "prefill":
        top = leg_prefill(ctx, args.tokens or 2048)
        cpu_jobs["top"] = ("prefill", "w4", SEED_W4, SEED_PREFILL, args.tokens or 2048)
    elif wl == "nvfp4-prefill":
        top = leg_prefill_nvfp4(ctx, args.tokens or 512)
        cpu_jobs["top"] = ("prefill", "nvfp4", SEED_NV, SEED_NVP, args.tokens or 512)
    elif wl == "shared-decode":
        top = leg_decode(ctx, "w4", args.tokens or 1, shared=True)
        cpu_jobs["top"] = ("shared", "w4", SEED_W4, SEED_SHARED, args.tokens or 1)
    elif wl == "router-decode":
        top = leg_decode_router(ctx, args.tokens or 1)
        cpu_jobs["top"] = ("router_decode", "w4", SEED_W4, SEED_RDEC, args.tokens or 1)
    elif wl == "router":
        top = leg_router(ctx, args.tokens or 2048)
        cpu_jobs["top"] = ("router", "bf16", SEED_ROUTER, SEED_ROUTER, args.tokens or 2048)
    elif wl in ("quantize-clip", "quantize-sym128"):
        what = "clip_g64" if wl == "quantize-clip" else "sym128"
        top = leg_quant(ctx, what)
        cpu_jobs["top"] = ("quant_" + what, "f32", SEED_QUANT, SEED_QUANT, 0)
    else:
        raise SystemExit(f"unknown workload {wl}")
    if wl == "all":
        for T in (1, 4, 16):
            legs[f"decode_stream_T{T}"] = leg_stream(ctx, T)
            cpu_jobs[f"decode_stream_T{T}"] = ("stream", "w4", SEED_W4, SEED_STREAM, T)
        legs["prefill_2048"] = leg_prefill(ctx, 2048)
        cpu_jobs["prefill_2048"] = ("prefill", "w4", SEED_W4, SEED_PREFILL, 2048)
        legs["nvfp4_prefill_512"] = leg_prefill_nvfp4(ctx, 512)
        cpu_jobs["nvfp4_prefill_512"] = ("prefill", "nvfp4", SEED_NV, SEED_NVP, 512)
        legs["nvfp4_decode_T1"] = leg_decode(ctx, "nvfp4", 1)
        cpu_jobs["nvfp4_decode_T1"] = ("decode", "nvfp4", SEED_NV, SEED_NVD, 1)
        legs["decode_shared_T1"] = leg_decode(ctx, "w4", 1, shared=True)
        cpu_jobs["decode_shared_T1"] = ("shared", "w4", SEED_W4, SEED_SHARED, 1)
        legs["decode_router_T1"] = leg_decode_router(ctx, 1)
        cpu_jobs["decode_router_T1"] = ("router_decode", "w4", SEED_W4, SEED_RDEC, 1)
        for T in (1, 2048):
            legs[f"router_T{T}"] = leg_router(ctx, T)
            cpu_jobs[f"router_T{T}"] = ("router", "bf16", SEED_ROUTER, SEED_ROUTER, T)
        for what in ("clip_g64", "sym128"):
            legs[f"quantize_{what}"] = leg_quant(ctx, what)
            cpu_jobs[f"quantize_{what}"] = ("quant_" + what, "f32", SEED_QUANT, SEED_QUANT, 0)
    if cpu:
        for name, (kind, fmt, ws, xs, T) in cpu_jobs.items():
            cb = cpu_baseline(kind, fmt, ws, xs, T, sec, log,
                              unit="weights/s" if kind.startswith("quant_") else "tokens/s")
            (top if name == "top" else legs[name])["cpu_baseline"] = cb
    if legs:
        top["legs"] = legs
        top["gpu_launches_all_legs"] = top["gpu_launches"] + sum(v["gpu_launches"] for v in legs.values())
    if ctx.world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return top if ctx.rank == 0 else None


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200, help="timed steps of every leg")
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="all",
                    choices=["all", "decode", "stream", "prefill", "nvfp4-decode", "nvfp4-prefill", "shared-decode",
                             "router", "router-decode", "quantize-clip", "quantize-sym128"])
    ap.add_argument("--tokens", type=int, default=None,
                    help="tokens per step of a single workload (decode 1, prefill 2048, NVFP4 prefill 512)")
    ap.add_argument("--layers", type=int, default=LAYERS,
                    help="resident layers of each format (40 = 18.1 GB, larger than L2)")
    ap.add_argument("--graph-steps", type=int, default=400, help="steps captured per CUDA graph")
    ap.add_argument("--cpu-seconds", type=float, default=5.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--quiet", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    def log(msg):
        if not args.quiet:
            print(f"[bench] {msg}", file=sys.stderr, flush=True)

    if args.impl == "reference":
        if args.tokens is None:
            args.tokens = 1
        out = run_reference(args, log)
    else:
        out = run_native(args, log)
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
