#!/usr/bin/env python
"""MoE-FFN throughput of libmoeq on B200, with roofline accounting.

Default workload: the Edge0-35B-shaped MoE layer at decode (one token, top-4,
hidden 2048, 256 experts, intermediate 512, shared expert 512, int4 group-64
experts, 8-bit router and shared-expert gate, LoRA rank 16).  A step is one
pass of the whole path (router, top-K, index build, gate/up + LoRA + SwiGLU,
down + LoRA, combine) over one batch.  Consecutive steps rotate over distinct
copies of the layer resident in HBM (40 by default, about 20 GB), so no step
finds its weights in the 126 MB L2.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One JSON line is printed by rank 0.  Under torchrun (N > 1) every rank runs
its own replica (the path does not shard); value = tokens of all ranks / the
slowest rank's time.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402
from synth import workloads  # noqa: E402

METRIC = "MoE-FFN tokens/s; decode HBM GB/s and prefill TFLOP/s as % of B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
MOE_WORKLOADS = ("decode_k4", "decode_k8", "multi_tenant", "prefill", "decode_k4_g32", "multi_tenant_g32")
MIXED_WORKLOADS = ("mixed_b1", "mixed_b16")


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=MOE_WORKLOADS + MIXED_WORKLOADS, default="decode_k4")
    ap.add_argument("--copies", type=int, default=None, help="distinct layer copies rotated over (L2-cold)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the CPU-baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args(argv)


def default_steps(workload):
    return {"decode_k4": 2000, "decode_k8": 2000, "multi_tenant": 1000, "prefill": 3, "mixed_b1": 200,
            "mixed_b16": 200, "decode_k4_g32": 2000, "multi_tenant_g32": 1000}[workload]


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and throttle reasons sampled while the timed region runs.

    NVML is read every 5 ms from a thread, so that a timed region of a few tens of
    milliseconds still holds several samples; the GPU is found by its PCI address, which
    CUDA_VISIBLE_DEVICES does not renumber.  Without NVML, nvidia-smi samples every 200 ms.
    Reads only: no setting of the GPU is touched.
    """

    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_S = 0.005

    def __init__(self, cuda_index):
        self.samples = []  # (wall time, sm MHz, max sm MHz, set of active reasons)
        self.proc = None
        self.source = None
        self._halt = threading.Event()
        target = None
        try:
            import pynvml
            pynvml.nvmlInit()
            handle = self._nvml_handle(pynvml, cuda_index)
            bits = (pynvml.nvmlClocksEventReasonHwSlowdown, pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                    pynvml.nvmlClocksEventReasonSwThermalSlowdown, pynvml.nvmlClocksEventReasonSwPowerCap)
            smax = float(pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM))
            target = lambda: self._poll_nvml(pynvml, handle, bits, smax)  # noqa: E731
            self.source = "nvml every %g ms" % (1e3 * self.PERIOD_S)
        except Exception:
            try:
                self.proc = subprocess.Popen(["nvidia-smi", "-i", str(cuda_index), "--query-gpu=" + self.FIELDS,
                                              "--format=csv,noheader,nounits", "-lms", "200"],
                                             stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except OSError:
                return
            target = self._read_smi
            self.source = "nvidia-smi every 200 ms"
        self.thread = threading.Thread(target=target, daemon=True)
        self.thread.start()

    @staticmethod
    def _nvml_handle(pynvml, cuda_index):
        try:
            import torch
            pr = torch.cuda.get_device_properties(cuda_index)
            return pynvml.nvmlDeviceGetHandleByPciBusId(
                "%08X:%02X:%02X.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id))
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(cuda_index)

    def _poll_nvml(self, pynvml, handle, bits, smax):
        while not self._halt.is_set():
            try:
                sm = float(pynvml.nvmlDeviceGetClockInfo(handle, pynvml.NVML_CLOCK_SM))
                mask = pynvml.nvmlDeviceGetCurrentClocksEventReasons(handle)
            except Exception:
                return
            self.samples.append((time.time(), sm, smax, {n for n, b in zip(self.NAMES, bits) if mask & b}))
            self._halt.wait(self.PERIOD_S)

    def _read_smi(self):
        for line in self.proc.stdout:
            c = [f.strip() for f in line.split(",")]
            try:
                sm, smax = float(c[1]), float(c[2])
            except (ValueError, IndexError):
                continue
            self.samples.append((time.time(), sm, smax,
                                 {n for n, v in zip(self.NAMES, c[5:9]) if v.lower().startswith("active")}))

    def stop(self):
        self._halt.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if getattr(self, "thread", None) is not None:
            self.thread.join(timeout=5)

    def summary(self, t0, t1):
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        used = inside if inside else self.samples
        if not used:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": self.source}
        return {"sm_mhz": statistics.median(s[1] for s in used), "sm_max_mhz": max(s[2] for s in used),
                "reasons": sorted(set().union(*(s[3] for s in used))), "samples": len(inside),
                "window": "timed region" if inside else "whole run (timed region shorter than one sample)",
                "source": self.source}


# ----------------------------------------------------------------- byte / flop accounting
def expert_bytes(H, I, group=64):
    """int4 words + bf16 scale/bias of gate, up and down of one expert."""
    gu = 2 * I * (H // 2 + (H // group) * 4)
    d = H * (I // 2 + (I // group) * 4)
    return gu, d


def lora_bytes(H, I, r):
    return {"A_gu": 2 * r * H * 2, "B_gu": 2 * I * r * 2, "A_d": r * I * 2, "B_d": H * r * 2}


def router_bytes(H, E, group=64):
    return E * (H + (H // group) * 4) + (H + (H // group) * 4)


def routing_stats(idx, aid, K, n_adapters):
    """Distinct experts and distinct (expert, adapter) pairs (shared expert included)."""
    T = idx.shape[0]
    experts = set(np.unique(idx).tolist())
    if aid is None:
        a = np.zeros(T, np.int64) if n_adapters > 0 else -np.ones(T, np.int64)
    else:
        a = aid.astype(np.int64)
    pairs = {(int(e), int(a[t])) for t in range(T) for e in idx[t] if a[t] >= 0}
    spairs = {int(v) for v in np.unique(a) if v >= 0}
    return len(experts), len(pairs), len(spairs)


def step_accounting(shape, idx, aid):
    """Algorithmic bytes and flops of one layer call, per kernel unit and in total.

    Bytes: the weights a unit must touch (distinct experts, distinct expert-adapter
    pairs for LoRA) plus its activation inputs and outputs in the path's formats
    (x bf16, h bf16, per-job outputs fp32).  Flops: 2 per multiply-add the method
    defines (LoRA-A of the adapter each job uses only)."""
    H, E, K, I, Is, r, T = shape.H, shape.E, shape.K, shape.I, shape.Is, shape.rank, idx.shape[0]
    gu, d = expert_bytes(H, I, shape.group)
    sgu, sd = expert_bytes(H, Is, shape.group)
    lb = lora_bytes(H, I, r)
    slb = lora_bytes(H, Is, r)
    U, P, SP = routing_stats(idx, aid, K, shape.n_adapters)
    TK = T * K
    J = T * (K + 1)
    h_bytes = (TK * I + T * Is) * 2
    b = {
        "router": router_bytes(H, E, shape.group) + T * H * 2 + T * E * 4,
        "gate_up": U * gu + sgu + P * lb["B_gu"] + SP * slb["B_gu"] + T * H * 2 + h_bytes,
        "down": U * d + sd + P * lb["B_d"] + SP * slb["B_d"] + h_bytes + J * H * 4,
        "lora_gu": P * lb["A_gu"] + SP * slb["A_gu"] + T * H * 2,
        "lora_down": P * lb["A_d"] + SP * slb["A_d"] + h_bytes,
    }
    f = {
        "router": 2 * T * H * (E + 1),
        "gate_up": 2 * TK * 2 * H * I + 2 * T * 2 * H * Is + (2 * TK * 2 * I * r + 2 * T * 2 * Is * r if r else 0),
        "down": 2 * TK * H * I + 2 * T * H * Is + (2 * TK * H * r + 2 * T * H * r if r else 0),
        "lora_gu": 2 * TK * 2 * r * H + 2 * T * 2 * r * H if r else 0,
        "lora_down": 2 * TK * r * I + 2 * T * r * Is if r else 0,
    }
    weights = router_bytes(H, E, shape.group) + U * (gu + d) + sgu + sd + P * sum(lb.values()) + SP * sum(slb.values())
    act = 2 * T * H * 2
    b["layer"] = weights + act
    f["layer"] = sum(f.values())
    b["lora_a"] = (b["lora_gu"] + b["lora_down"]) / 2  # the CUDA-core LoRA-A kernel runs twice per call
    f["lora_a"] = (f["lora_gu"] + f["lora_down"]) / 2
    return {"kernel_bytes": b, "kernel_flops": f, "weight_bytes": weights, "act_bytes": act, "flops": f["layer"],
            "experts": U}


# library timing kind -> accounting unit
KIND_UNIT = {"router_logits": "router", "tc_router": "router", "gate_up": "gate_up", "tc_gate_up": "gate_up",
             "down": "down", "tc_down": "down", "lora_a": "lora_a", "tc_lora_gate_up": "lora_gu",
             "tc_lora_down": "lora_down", "decode_fused": "layer", "decode_chain": "layer",
             "decode_cluster": "layer"}


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of the
# dominant kernel, from one ncu capture of the kernel as it stands (the capture's
# summary is kept with the profiles).  An entry is removed whenever its kernel
# changes, so the bench reports null rather than a stale figure.
NCU_TRAFFIC = {
    # one gate/up launch over the 2048-token prompt of one layer
    ("prefill", "tc_gate_up"): 333590784 + 9545728,
    # one gate/up launch of the mixed ternary/4-bit MLP, one token
    ("mixed_b1", "mixed_gate_up"): 2014976,
}


def launch_times(kt, ms_graph):
    """Per-kind (ms per launch, launches) from the event-timed replay, less the event
    nodes' own cost: the excess of the summed event intervals over the plain graph's
    time is spread evenly over the launches (each event node adds the same gap), so
    the per-kind times add up to the plain graph's time and none exceeds a step."""
    n = sum(c for _, c in kt.values())
    if not n:
        return {}
    excess = max(0.0, sum(t for t, _ in kt.values()) - ms_graph) / n
    return {k: (max(t / c - excess, 0.0), c) for k, (t, c) in kt.items()}


def kernel_roofline(kind, dur_ms, nbytes, nflops, peaks, src, timed_s, workload=None):
    """Roofline entry of one kernel: the bound is whichever of HBM time and bf16
    tensor time is larger for its algorithmic bytes and flops; the tensor peak is
    the burst figure for a timed region under a second, else the sustained one."""
    hbm = float(peaks["hbm_gbs"])
    tpeak_key = "bf16_tflops" if timed_s < 1.0 else "bf16_tflops_sustained"
    tpk = float(peaks[tpeak_key])
    t_mem = nbytes / (hbm * 1e9)
    t_tc = nflops / (tpk * 1e12)
    sec = dur_ms * 1e-3
    gbs = nbytes / sec / 1e9
    tfs = nflops / sec / 1e12
    tensor = {"achieved": round(tfs, 2), "peak": tpk, "unit": "TFLOP/s", "frac": round(tfs / tpk, 4),
              "peak_source": "%s %s" % (src, tpeak_key)}
    if t_tc > t_mem:
        roof = {"kernel": kind, "bound": "tensor", "achieved": round(tfs, 2), "peak": tpk, "unit": "TFLOP/s",
                "frac": round(tfs / tpk, 4), "peak_source": "%s %s" % (src, tpeak_key)}
    else:
        roof = {"kernel": kind, "bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(gbs / hbm, 4), "peak_source": "%s hbm_gbs" % src, "tensor": tensor}
    tr = NCU_TRAFFIC.get((workload, kind))
    roof.update({"traffic": tr, "launch_us": round(dur_ms * 1e3, 3),
                 "bytes_per_launch": int(nbytes), "flops_per_launch": int(nflops),
                 "launch_time": "CUDA events in a graph replay, less the event nodes' overhead"})
    if tr:
        roof["traffic_source"] = "ncu capture of this kernel"
    return roof


# ----------------------------------------------------------------- distributed plumbing
def dist_setup(n_gpus):
    """One process per GPU (torchrun's RANK / LOCAL_RANK / WORLD_SIZE); NCCL on GPUs.  Without
    a GPU the ranks join a gloo group on the CPU, which is how the multi-rank plumbing is
    tested."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    cuda = torch.cuda.is_available()
    if world > 1:
        import torch.distributed as dist
        if cuda:
            torch.cuda.set_device(local)
        dist.init_process_group("nccl" if cuda else "gloo", timeout=datetime.timedelta(seconds=180))
    elif cuda:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    import torch
    if torch.cuda.is_available():
        torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, world):
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_step, steps, world, ms):
    """Whole-job throughput: the units every rank processed in `steps` steps over the
    slowest rank's time `ms` (replicas: the same work on each rank, weak scaling)."""
    return units_per_rank_step * steps * world / (ms * 1e-3)


def capture_steps(step, first, count):
    """A CUDA graph of `count` consecutive steps (step(i) enqueues on the current stream)."""
    import torch
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g, stream=side):
        for i in range(count):
            step(first + i)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    return g


def timed_replay(g, world, clocks=None):
    """Device time (ms) of one replay, bracketed by barrier + synchronize; max over ranks."""
    import torch
    g.replay()  # untimed warm-up replay
    barrier(world)
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    t0 = time.time()
    e0.record(stream)
    g.replay()
    e1.record(stream)
    e1.synchronize()
    t1 = time.time()
    barrier(world)
    return max_over_ranks(e0.elapsed_time(e1), world), t0, t1


def kernel_times(moeq, step, first, count):
    """Per-kernel device time from event nodes recorded inside one graph replay."""
    import torch
    moeq.moe_timing_enable(True)
    try:
        g = capture_steps(step, first, count)
        g.replay()
        torch.cuda.synchronize()
        kt = moeq.moe_timing_collect()
    finally:
        moeq.moe_timing_enable(False)
    del g
    return kt


# ----------------------------------------------------------------- workload construction
def build_moe_copies(shape, copies, seed, device):
    """Layer copy 0 from the host generator (the CPU baseline uses the same values);
    the other copies drawn on the device.  All packed by libmoeq's pack kernel."""
    import torch
    from int4_group_affine_b200.layer import DeviceLayer, to_device
    layers, host0 = [], None
    for c in range(copies):
        if c == 0:
            host0 = workloads.moe_weights(shape, seed=seed, layer=0)
            wd = {k: to_device(v, device) for k, v in host0.items() if k not in ("lora",) and v is not None}
            lora = [{k: to_device(v, device) for k, v in ad.items()} for ad in host0["lora"]]
        else:
            wd, lora = device_moe_weights(shape, seed, c, device)
        layers.append(DeviceLayer.from_fp32(shape, wd, lora))
        del wd
        torch.cuda.synchronize()
    return layers, host0


def device_moe_weights(shape, seed, c, device):
    import torch
    H, E, I, Is, r = shape.H, shape.E, shape.I, shape.Is, shape.rank
    kw = dict(std=shape.w_std, device=device, outlier_prob=shape.outlier_prob, outlier_factor=shape.outlier_factor)
    p = "L%d/" % c
    dims = {"router": (E, H), "sgate": (1, H), "gate": (E, I, H), "up": (E, I, H), "down": (E, H, I),
            "s_gate": (1, Is, H), "s_up": (1, Is, H), "s_down": (1, H, Is)}
    wd = {k: synth.device_normal(seed, p + k, shp, **kw) for k, shp in dims.items()}
    if shape.logit_bias_std > 0:
        wd["logit_bias"] = synth.device_normal(seed, p + "logit_bias", (E,), shape.logit_bias_std, device)
    ldims = {"gate": (E, I, H), "up": (E, I, H), "down": (E, H, I), "s_gate": (1, Is, H), "s_up": (1, Is, H),
             "s_down": (1, H, Is)}
    lora = []
    for a in range(shape.n_adapters):
        ad = {}
        for proj, (n, out, in_) in ldims.items():
            q = p + "lora%d/%s" % (a, proj)
            for nm, shp in (("A", (n, r, in_)), ("B", (n, out, r))):
                v = synth.device_normal(seed, q + "/" + nm, shp, shape.lora_std, device)
                ad[proj + "_" + nm] = v.to(torch.bfloat16).view(torch.int16).contiguous()
        lora.append(ad)
    return wd, lora


# ----------------------------------------------------------------- CPU baseline (the oracle)
def oracle_moe_layer(shape, host0):
    import oracle
    t = {}
    for name, bits in (("router", 8), ("sgate", 8), ("gate", 4), ("up", 4), ("down", 4), ("s_gate", 4),
                       ("s_up", 4), ("s_down", 4)):
        t[name + "_p"], t[name + "_s"], t[name + "_b"] = oracle.quant_affine(host0[name], bits, shape.group)
    t["logit_bias"] = host0.get("logit_bias")
    t["lora"] = host0["lora"]
    return oracle.OracleLayer(shape.H, shape.E, shape.K, shape.I, shape.Is, t, rank=shape.rank,
                              alpha=shape.alpha, group=shape.group)


def cpu_baseline_moe(shape, host0, seed, budget_s, x_inputs, aid_inputs, layers=1):
    """Oracle tokens/s on a bounded sample: whole tokens through layer copy 0, divided by
    the number of layers a step runs (a stack's prompt tokens pass through every layer)."""
    import oracle
    L = oracle_moe_layer(shape, host0)
    done, t0 = 0, time.time()
    i = 0
    while True:
        x = x_inputs[i % len(x_inputs)]
        a = None if aid_inputs is None else aid_inputs[i % len(aid_inputs)]
        tok = min(x.shape[0], 4)
        L.ffn(x[:tok], None if a is None else a[:tok])
        done += tok
        i += 1
        if time.time() - t0 >= budget_s:
            break
    el = time.time() - t0
    sample = "%d tokens of the %s layer (layer copy 0) through the fp64 oracle in %.1f s" % (done, shape.name, el)
    if layers > 1:
        sample += ", scaled to the %d-layer stack" % layers
    return {"value": done / el / layers, "unit": "tokens/s", "cores": oracle.threads(), "kind": "oracle",
            "sample": sample}


# ----------------------------------------------------------------- the timed runs
def run_moe(args, world, rank, local):
    import torch
    import int4_group_affine_b200 as moeq
    dev = torch.device("cuda", local)
    shape = workloads.MOE_SHAPES[args.workload]
    stack = args.workload == "prefill"
    copies = args.copies or (shape.layers if stack else 40)
    K, W = args.steps, args.warmup
    layers, host0 = build_moe_copies(shape, copies, args.seed + 1000 * rank, dev)
    T = shape.T
    n_inputs = 1 if stack else min(K + W, 256)
    xs_host, aids_host = [], []
    for i in range(n_inputs):
        x, aid = workloads.moe_inputs(shape, seed=args.seed + 1000 * rank, tag="bench/x%d" % i)
        xs_host.append(x)
        aids_host.append(aid)
    from int4_group_affine_b200.layer import to_device
    xs = torch.stack([to_device(x, dev) for x in xs_host])
    aids = None if aids_host[0] is None else torch.stack([to_device(a, dev) for a in aids_host])
    ws, nbytes = layers[0].workspace(T, dev)
    ys = torch.empty((2, T, shape.H), dtype=torch.int16, device=dev)
    xa = torch.empty((T, shape.H), dtype=torch.int16, device=dev)
    xb = torch.empty_like(xa)
    stream = torch.cuda.current_stream(dev)

    def step(s):
        if stack:  # one step = the whole stack of copies over the prompt
            src = xs[0]
            for l, lay in enumerate(layers):
                dst = xa if l % 2 == 0 else xb
                moeq.moe_block_forward(lay.L, src, None, T, 1e-6, dst, ws, nbytes)
                src = dst
        else:
            i = s % n_inputs
            moeq.moe_ffn_forward(layers[s % copies].L, xs[i], None if aids is None else aids[i], T, ys[s % 2],
                                 ws, nbytes)

    for s in range(W):
        step(s)
    torch.cuda.synchronize()
    g = capture_steps(step, W, K)
    clocks = ClockSampler(local)
    time.sleep(0.5)
    ms, t_wall0, t_wall1 = timed_replay(g, world)
    time.sleep(0.5)
    clocks.stop()
    del g
    ms_step = ms / K
    tokens_per_step = T  # prefill: the prompt's tokens through the whole stack per step

    # per-kernel durations: the same steps captured again with library event timing on
    kt = launch_times(kernel_times(moeq, step, W, K), ms)
    launches_per_step = sum(c for _, c in kt.values()) / K

    # routing of each timed step (for byte accounting), recomputed outside the timed region
    acc = accounting_for_steps(moeq, shape, layers, xs, xs_host, aids_host, K, W, copies, n_inputs, stack, dev)

    # end to end: pinned host input -> device, forward, device -> host result, per step
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(moeq, shape, layers, xs_host, aids_host, K, W, copies, n_inputs, stack, ws, nbytes, dev,
                      world)

    peaks, src = measured_peaks()
    hbm = float(peaks["hbm_gbs"])
    dom = max(kt.items(), key=lambda kv: kv[1][0] * kv[1][1])[0] if kt else None
    roof = None
    if dom is not None and dom in KIND_UNIT:
        unit = KIND_UNIT[dom]
        roof = kernel_roofline(dom, kt[dom][0], acc["kernel_bytes"][unit], acc["kernel_flops"][unit],
                               peaks, src, ms * 1e-3, args.workload)
    step_bytes = acc["weight_bytes"] + acc["act_bytes"]
    step_gbs = step_bytes / (ms_step * 1e-3) / 1e9
    value = job_throughput(tokens_per_step, K, world, ms)
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": round(ms_step, 6), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int4 weights, bf16 activations, fp32 accumulate", "data": "synthetic (seeded generator; no trained weights)",
        "config": {"workload": shape.name, "hidden": shape.H, "experts": shape.E, "top_k": shape.K,
                   "inter": shape.I, "shared_inter": shape.Is, "tokens": T, "group": shape.group,
                   "lora_rank": shape.rank,
                   "adapters": shape.n_adapters, "layer_copies": copies,
                   "l2": "inputs larger than L2: %d distinct layer copies (%.1f GB) rotated per step" %
                         (copies, sum(l.nbytes() for l in layers) / 1e9),
                   "parallelism": "replicas" if world > 1 else "single GPU",
                   "step": "one %s" % ("40-layer block stack pass" if stack else "MoE layer call")},
        "roofline": roof,
        "step_roofline": {"bound": "hbm", "achieved": round(step_gbs, 1), "peak": hbm, "unit": "GB/s",
                          "frac": round(step_gbs / hbm, 4), "bytes_per_step": int(step_bytes),
                          "what": "touched expert + LoRA + router bytes per step / step time"},
        "tflops": round(acc["flops"] / (ms_step * 1e-3) / 1e12, 3),
        "kernels": {k: {"ms_per_launch": round(v[0], 6), "launches": v[1]} for k, v in kt.items()},
        "gpu_launches": int(round(launches_per_step * K)),
        "clocks": clocks.summary(t_wall0, t_wall1),
    }
    if stack:
        out["config"]["unit"] = "prompt tokens through the %d-layer stack" % copies
    if e2e is not None:
        out["e2e"] = e2e
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline_moe(shape, host0, args.seed, args.cpu_seconds, xs_host, aids_host,
                                               copies if stack else 1)
    return out


def accounting_for_steps(moeq, shape, layers, xs, xs_host, aids_host, K, W, copies, n_inputs, stack, dev):
    import torch
    T, E, Kk = shape.T, shape.E, shape.K
    idx = torch.empty((T, Kk), dtype=torch.int32, device=dev)
    w = torch.empty((T, Kk), dtype=torch.float32, device=dev)
    sg = torch.empty(T, dtype=torch.float32, device=dev)
    logits = torch.empty((T, E), dtype=torch.float32, device=dev)
    tot = None
    nsteps = 1 if stack else min(K, 64)
    for s in range(nsteps):
        lay = layers[0 if stack else (W + s) % copies]
        i = 0 if stack else (W + s) % n_inputs
        moeq.moe_router_topk(xs[i], lay.L.router, lay.L.shared_gate, lay.t.get("logit_bias"), T, shape.H, E, Kk,
                             idx, w, sg, logits)
        a = step_accounting(shape, idx.cpu().numpy(), aids_host[i])
        if tot is None:
            tot = {"kernel_bytes": dict(a["kernel_bytes"]), "kernel_flops": dict(a["kernel_flops"]),
                   "weight_bytes": a["weight_bytes"], "act_bytes": a["act_bytes"], "flops": a["flops"]}
        else:
            for kk in ("kernel_bytes", "kernel_flops"):
                for k in tot[kk]:
                    tot[kk][k] += a[kk][k]
            for k in ("weight_bytes", "act_bytes", "flops"):
                tot[k] += a[k]
    for kk in ("kernel_bytes", "kernel_flops"):
        for k in tot[kk]:
            tot[kk][k] /= nsteps
    for k in ("weight_bytes", "act_bytes", "flops"):
        tot[k] /= nsteps
    if stack:  # the whole stack per step; each layer's routing approximated by copy 0's
        L = len(layers)
        for k in ("weight_bytes", "act_bytes", "flops"):
            tot[k] *= L
    return tot


def run_e2e(moeq, shape, layers, xs_host, aids_host, K, W, copies, n_inputs, stack, ws, nbytes, dev, world):
    import torch
    T, H = shape.T, shape.H
    hx = torch.from_numpy(np.stack(xs_host).view(np.int16)).pin_memory()
    ha = None if aids_host[0] is None else torch.from_numpy(np.stack(aids_host)).pin_memory()
    hy = torch.empty((T, H), dtype=torch.int16).pin_memory()
    dx = torch.empty((T, H), dtype=torch.int16, device=dev)
    da = None if ha is None else torch.empty(T, dtype=torch.int32, device=dev)
    dy = torch.empty((T, H), dtype=torch.int16, device=dev)
    xa = torch.empty_like(dx)
    xb = torch.empty_like(dx)
    stream = torch.cuda.current_stream(dev)

    # decode-sized calls go through moe_ffn_forward_host: the library moves x in and y out
    # itself (at one token the decode kernel reads and writes the pinned host buffers across
    # the bus); larger calls copy x in, run moe_ffn_forward and copy y out
    host_api = not stack and T <= 8

    def step(s):
        i = s % n_inputs
        if da is not None:
            da.copy_(ha[i], non_blocking=True)
        if host_api:
            moeq.moe_ffn_forward_host(layers[s % copies].L, hx[i], da, T, hy, ws, nbytes)
            return
        dx.copy_(hx[i], non_blocking=True)
        if stack:
            src = dx
            for l, lay in enumerate(layers):
                dst = xa if l % 2 == 0 else xb
                moeq.moe_block_forward(lay.L, src, None, T, 1e-6, dst, ws, nbytes)
                src = dst
            hy.copy_(src, non_blocking=True)
        else:
            moeq.moe_ffn_forward(layers[s % copies].L, dx, da, T, dy, ws, nbytes)
            hy.copy_(dy, non_blocking=True)

    for s in range(W):
        step(s)
    torch.cuda.synchronize()
    g = capture_steps(step, W, K)
    ms, _, _ = timed_replay(g, world)
    del g
    toks = T
    h2d = T * H * 2 + (0 if ha is None else T * 4)
    return {"value": round(job_throughput(toks, K, world, ms), 2), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": T * H * 2, "ms_per_step": round(ms / K, 6),
            "transfers": "moe_ffn_forward_host (pinned host x and y)" if host_api
            else "cudaMemcpyAsync from / to pinned host memory around the call"}


# ----------------------------------------------------------------- mixed layout
def run_mixed(args, world, rank, local):
    import torch
    import int4_group_affine_b200 as moeq
    from int4_group_affine_b200.layer import DeviceMixed, to_device
    dev = torch.device("cuda", local)
    shape = workloads.MIXED_SHAPES[args.workload]
    copies = args.copies or 4 * shape.layers  # 4 stack copies (~330 MB) so the stack cannot live in L2
    K, W = args.steps, args.warmup
    mats = []
    host0 = None
    for c in range(copies):
        if c == 0:
            host0 = workloads.mixed_weights(shape, seed=args.seed + 1000 * rank, layer=0)
            Wd = {k: to_device(v, dev) for k, v in host0.items()}
        else:
            Wd = {k: synth.device_normal(args.seed + 1000 * rank, "M%d/%s" % (c, k), shp, shape.w_std, dev)
                  for k, shp in (("gate", (shape.I, shape.H)), ("up", (shape.I, shape.H)), ("down", (shape.H, shape.I)))}
        mats.append({k: DeviceMixed.from_fp32(v, shape.rho) for k, v in Wd.items()})
        del Wd
    torch.cuda.synchronize()
    T, H, L = shape.T, shape.H, shape.layers
    x = to_device(workloads.mixed_inputs(shape, seed=args.seed + 1000 * rank), dev)
    nb = moeq.moe_mixed_mlp_workspace_bytes(H, shape.I, T)
    ws = torch.empty(nb, dtype=torch.uint8, device=dev)
    bufs = [torch.empty_like(x), torch.empty_like(x)]
    stream = torch.cuda.current_stream(dev)
    nstacks = copies // L

    def step(s):
        base = (s % nstacks) * L
        src = x
        for l in range(L):
            m = mats[base + l]
            dst = bufs[l % 2]
            moeq.moe_mixed_mlp_forward(m["gate"].T, m["up"].T, m["down"].T, src, T, 1, 1e-6, dst, ws, nb)
            src = dst

    for s in range(W):
        step(s)
    torch.cuda.synchronize()
    g = capture_steps(step, W, K)
    clocks = ClockSampler(local)
    time.sleep(0.5)
    ms, t0, t1 = timed_replay(g, world)
    time.sleep(0.5)
    clocks.stop()
    del g
    ms_step = ms / K
    kt = launch_times(kernel_times(moeq, step, W, K), ms)
    layer_bytes = sum(m.nbytes() for m in mats[0].values())
    peaks, src = measured_peaks()
    hbm = float(peaks["hbm_gbs"])
    dom = max(kt.items(), key=lambda kv: kv[1][0] * kv[1][1])[0]
    per = {"mixed_gate_up": mats[0]["gate"].nbytes() + mats[0]["up"].nbytes(),
           "mixed_down": mats[0]["down"].nbytes()}.get(dom)
    roof = None
    if per:
        dur = kt[dom][0]
        gbs = per / (dur * 1e-3) / 1e9
        tr = NCU_TRAFFIC.get((args.workload, dom))
        roof = {"kernel": dom, "bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(gbs / hbm, 4), "traffic": tr, "peak_source": "%s hbm_gbs" % src,
                "launch_us": round(dur * 1e3, 3), "bytes_per_launch": per,
                "launch_time": "CUDA events in a graph replay, less the event nodes' overhead"}
        if tr:
            roof["traffic_source"] = "ncu capture of this kernel"
    step_gbs = L * layer_bytes / (ms_step * 1e-3) / 1e9
    out = {
        "metric": METRIC, "value": round(job_throughput(T, K, world, ms), 2), "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": W, "ms_per_step": round(ms_step, 6), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "ternary/int4 weights, bf16 activations, fp32 accumulate",
        "data": "synthetic (seeded generator; no trained weights)",
        "config": {"workload": shape.name, "hidden": H, "inter": shape.I, "layers": L, "rho": shape.rho,
                   "tokens": T, "stack_copies": nstacks,
                   "l2": "inputs larger than L2: %d stack copies (%.0f MB) rotated per step" %
                         (nstacks, nstacks * L * layer_bytes / 1e6),
                   "step": "one %d-layer pre-norm residual MLP stack pass" % L},
        "roofline": roof,
        "step_roofline": {"bound": "hbm", "achieved": round(step_gbs, 1), "peak": hbm, "unit": "GB/s",
                          "frac": round(step_gbs / hbm, 4), "bytes_per_step": L * layer_bytes},
        "kernels": {k: {"ms_per_launch": round(v[0], 6), "launches": v[1]} for k, v in kt.items()},
        "gpu_launches": int(sum(c for _, c in kt.values())),
        "clocks": clocks.summary(t0, t1),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        q = {k: oracle.quant_mixed(v, shape.rho) for k, v in host0.items()}
        xh = workloads.mixed_inputs(shape, seed=args.seed)
        n, t_0 = 0, time.time()
        while time.time() - t_0 < args.cpu_seconds:
            oracle.mixed_block(q["gate"], q["up"], q["down"], H, shape.I, shape.rho, xh)
            n += 1
        el = time.time() - t_0
        out["cpu_baseline"] = {"value": n * T / (el * L), "unit": "tokens/s", "cores": oracle.threads(),
                               "kind": "oracle", "sample": "%d single-layer passes (layer 0) of %d tokens in %.1f s, "
                               "scaled to the %d-layer stack" % (n, T, el, L)}
    return out


# ----------------------------------------------------------------- reference arm (the oracle)
def run_reference(args):
    import oracle
    shape = workloads.MOE_SHAPES.get(args.workload)
    K, W = args.steps, args.warmup
    if shape is None:
        s = workloads.MIXED_SHAPES[args.workload]
        host0 = workloads.mixed_weights(s, seed=args.seed)
        q = {k: oracle.quant_mixed(v, s.rho) for k, v in host0.items()}
        xh = workloads.mixed_inputs(s, seed=args.seed)
        for _ in range(W):
            oracle.mixed_block(q["gate"], q["up"], q["down"], s.H, s.I, s.rho, xh)
        t0 = time.time()
        for _ in range(K):
            oracle.mixed_block(q["gate"], q["up"], q["down"], s.H, s.I, s.rho, xh)
        el = time.time() - t0
        value = K * s.T / (el * s.layers)
        sample = "each step: one layer (layer 0) of the %d-layer stack over %d tokens, scaled by 1/%d" % (
            s.layers, s.T, s.layers)
        name = s.name
    else:
        host0 = workloads.moe_weights(shape, seed=args.seed, layer=0)
        L = oracle_moe_layer(shape, host0)
        tok = 1 if shape.T == 1 else 2
        xs = [workloads.moe_inputs(shape, seed=args.seed, tag="bench/x%d" % i) for i in range(K + W)]
        for i in range(W):
            L.ffn(xs[i][0][:tok], None if xs[i][1] is None else xs[i][1][:tok])
        t0 = time.time()
        for i in range(W, W + K):
            L.ffn(xs[i][0][:tok], None if xs[i][1] is None else xs[i][1][:tok])
        el = time.time() - t0
        value = K * tok / el
        if shape.layers > 1:
            value /= shape.layers
        sample = "each step: %d token(s) of the %s layer through the fp64 oracle%s" % (
            tok, shape.name, " (scaled to the %d-layer stack)" % shape.layers if shape.layers > 1 else "")
        name = shape.name
    return {"metric": METRIC, "value": round(value, 4), "unit": "tokens/s", "n_gpus": 1, "steps": K, "warmup": W,
            "ms_per_step": round(el * 1e3 / K, 3), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic (seeded generator; no trained weights)", "impl": "reference",
            "config": {"workload": name},
            "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s", "cores": oracle.threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main(argv=None):
    args = parse_args(argv)
    if args.steps is None:
        args.steps = default_steps(args.workload)
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return 0
        print(json.dumps(run_reference(args)), flush=True)
        return 0
    import torch
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device for --impl ours")
    world, rank, local = dist_setup(args.gpus)
    try:
        out = run_mixed(args, world, rank, local) if args.workload in MIXED_WORKLOADS else \
            run_moe(args, world, rank, local)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
