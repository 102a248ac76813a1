"""Benchmark of the NF4 fused-expert MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl e4b|reference]
                    [--workload NAME] [--no-sweep]

One step = one pass of the whole hot path (router top-k, permutation, grouped
NF4 gate_up GEMM with SwiGLU, down GEMM, weighted combine) over one batch of
synthetic tokens, on one of R layer replicas cycled so that the bytes a cycle
touches exceed the 126 MB L2 several times (decode) -- "inputs larger than L2".
Steps are replayed from CUDA graphs (one graph per replica cycle plus
single-step graphs for the remainder) and timed with CUDA events; with
N > 1 GPUs (torchrun) every rank runs its own replicas (weak scaling, no
data-path collective) and the time is the max over ranks.

Printed: one JSON line (rank 0).  `value` is routed tokens/s (M*k per step) for
the whole job; `roofline` is the dominant kernel's achieved HBM GB/s or
TFLOP/s (algorithmic bytes/FLOPs per launch over its average CUDA-event
duration, measured live in a kernel-timing pass) against the measured peak;
`e2e` is the same metric through the public call with host buffers and the
host<->device copies inside the timed region; `cpu_baseline` is the float64
oracle on a bounded sample, on this host's cores.  `--impl reference` times the
oracle itself as the reference arm.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from quantized_moe_expert_nf4_b200 import workloads  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
METRIC = "routed tokens/s and TFLOP/s per MoE layer; fraction of HBM/bf16 roofline"

# name -> (layer configuration, tokens M[, 4-bit storage: "nf4" unless named])
WORKLOADS = {
    "olmoe_m1": ("olmoe", 1), "olmoe_m4": ("olmoe", 4), "olmoe_m8": ("olmoe", 8), "olmoe_m2048": ("olmoe", 2048),
    "qwen3_m4096": ("qwen3", 4096), "qwen3_lora_m4096": ("qwen3_lora", 4096),
    "gptoss_m1": ("gptoss", 1), "gptoss_m8192": ("gptoss", 8192), "tiny_m64": ("tiny", 64),
    "olmoe_fp4_m8": ("olmoe", 8, "fp4"), "qwen3_fp4_m4096": ("qwen3", 4096, "fp4"),
}
STORAGE = {"nf4": 0, "fp4": 1}   # e4b_quant_type


def workload(name):
    """(layer configuration name, M, storage name) of a bench workload."""
    w = WORKLOADS[name]
    return w[0], w[1], (w[2] if len(w) > 2 else "nf4")


DEFAULT_WORKLOAD = "olmoe_m1"
# Sweep rows that also carry the end-to-end measurement and a CPU-oracle sample.
E2E_SWEEP = ("qwen3_m4096", "gptoss_m8192")
# Every other workload of the table runs in the default sweep, so the JSON line
# carries the prefill rows' (M >= 4096) tensor-core fractions and the gpt-oss
# decode row beside the OLMoE ones.
DEFAULT_SWEEP = ("olmoe_m4", "olmoe_m8", "olmoe_m2048", "qwen3_m4096", "qwen3_lora_m4096", "gptoss_m1",
                 "gptoss_m8192", "olmoe_fp4_m8", "qwen3_fp4_m4096")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------------------
# Algorithmic work of one forward (counts only what the method must touch).
def expert_bytes(cfg):
    """Packed nibbles + fp32 absmax of one expert, both stacks."""
    return 3 * cfg.H * cfg.I * (0.5 + 4.0 / 64.0)


def gate_up_expert_bytes(cfg):
    return 2 * cfg.H * cfg.I * (0.5 + 4.0 / 64.0)


def step_work(cfg, M, touched):
    S = M * cfg.k
    flops = 6.0 * S * cfg.H * cfg.I + (2.0 * S * cfg.lora_r * (cfg.H + 2 * cfg.I) if cfg.lora_r else 0.0)
    nbytes = touched * expert_bytes(cfg) + 2 * M * cfg.H * 2 + 8 * S + M * cfg.E * 4
    if cfg.lora_r:
        nbytes += touched * cfg.lora_r * (cfg.H + 2 * cfg.I) * 2
    return flops, nbytes


# ---------------------------------------------------------------------------
class ClockSampler:
    """Polls NVML (SM clock, throttle reasons) from a thread during a region."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index):
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as ex:  # NVML unavailable: report it, keep measuring
            self.error = str(ex)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.samples.append((mhz, rs))
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._h is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = [s[0] for s in self.samples]
        mask = 0
        for _, r in self.samples:
            mask |= r
        reasons = sorted(n for b, n in self.REASONS.items() if mask & b and n != "gpu_idle")
        return {"sm_mhz": float(statistics.median(mhz)), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------
def cpu_cores():
    try:
        from threadpoolctl import threadpool_info
        n = max((d.get("num_threads", 1) for d in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def cpu_model():
    """The host CPU's model name (first /proc/cpuinfo entry), or the platform string."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or platform.machine()


class OracleSample:
    """A bounded sample of the workload, prepared for the float64 oracle.

    Set-up (untimed): the first `max_tokens` tokens of replica batches, their
    routing, and the oracle's own quantisation of the experts they touch.
    `step(i)` times one sample the way the oracle stands: routing weights, a
    fresh expert stack (so dequantisation is paid every step, as the GPU reads
    the packed bytes every step) and the per-token forward.
    """

    def __init__(self, cfg, M, max_tokens=8, replicas=2, storage="nf4"):
        from oracle import fp4, nf4, routing

        quant = {"nf4": nf4, "fp4": fp4}[storage]
        self.cfg, self.M, self.storage = cfg, M, storage
        self.ntok = min(M, max_tokens)
        E, H, I = cfg.E, cfg.H, cfg.I
        self.samples = []
        for rep in range(replicas):
            logits = workloads.router_logits(cfg, M, 0, rep)[: self.ntok]
            x = workloads.bf16_bits_to_f32(workloads.activations_bf16(cfg, M, 0)).astype(np.float64)[: self.ntok]
            ids = routing.topk(logits, cfg.k)
            gp = np.zeros((E, I * H), np.uint8)
            ga = np.zeros((E, 2 * I * H // 64), np.float32)
            dp = np.zeros((E, H * I // 2), np.uint8)
            da = np.zeros((E, H * I // 64), np.float32)
            for e in sorted(set(ids.reshape(-1).tolist())):
                gp[e], ga[e] = quant.quantize_expert(workloads.gate_up_expert(cfg, e))
                dp[e], da[e] = quant.quantize_expert(workloads.down_expert(cfg, e))
            self.samples.append((logits, x, ids, gp, ga, dp, da))
        self.la = self.lb = None
        if cfg.lora_r:
            self.la = workloads.bf16_bits_to_f32(workloads.lora_A(cfg)).astype(np.float64)
            self.lb = workloads.bf16_bits_to_f32(workloads.lora_B(cfg)).astype(np.float64)

    def step(self, i):
        from oracle import moe, routing

        cfg = self.cfg
        logits, x, ids, gp, ga, dp, da = self.samples[i % len(self.samples)]
        t0 = time.perf_counter()
        st = moe.ExpertStack(gp, ga, dp, da, cfg.E, cfg.H, cfg.I, self.la, self.lb, workloads.lora_scale(cfg),
                             quant=self.storage)
        w = routing.route_weights(logits, ids)
        moe.moe_forward_per_token(x, ids, w, st)
        return time.perf_counter() - t0

    def describe(self):
        return (f"{self.ntok} token(s) per step from {len(self.samples)} replica batch(es) of the {self.cfg.name}-shaped "
                f"M={self.M} workload through the float64 oracle: routing weights, dequantisation of the touched "
                f"experts, per-token SwiGLU expert MLPs and combine")


def oracle_rate(cfg, M, budget_s=12.0, max_tokens=8, storage="nf4"):
    """(routed tokens/s, description, seconds) of the oracle on a bounded sample."""
    smp = OracleSample(cfg, M, max_tokens=max_tokens, replicas=2, storage=storage)
    smp.step(0)  # warm-up
    spent, toks, i = 0.0, 0, 0
    while spent < budget_s and i < 1000:
        spent += smp.step(i)
        toks += smp.ntok * cfg.k
        i += 1
    return toks / spent, smp.describe() + f"; {i} steps timed", spent


# ---------------------------------------------------------------------------
def run_reference(args, cfg, M, rank, world):
    if rank != 0:
        return None
    cores = cpu_cores()
    smp = OracleSample(cfg, M, max_tokens=8, replicas=2, storage=workload(args.workload)[2])
    for i in range(args.warmup):
        smp.step(i)
    t_total = 0.0
    for i in range(args.steps):
        t_total += smp.step(i)
    value = smp.ntok * cfg.k * args.steps / t_total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "routed_tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "E": cfg.E, "H": cfg.H, "I": cfg.I, "k": cfg.k, "M": M,
                   "routing": cfg.routing, "weights": f"{smp.storage.upper()}/64 fp32 absmax",
                   "sample_tokens_per_step": smp.ntok},
        "cpu_baseline": {"value": value, "unit": "routed_tokens/s", "cores": cores, "cpu": cpu_model(),
                         "kind": "oracle", "sample": smp.describe()},
        "e2e": {"value": value, "unit": "routed_tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return line


# ---------------------------------------------------------------------------
class Bench:
    def __init__(self, cfg, M, device, replicas, seed_base=0, storage="nf4"):
        import torch
        from quantized_moe_expert_nf4_b200 import e4b, synthetic

        self.torch, self.e4b = torch, e4b
        self.cfg, self.M, self.device = cfg, M, device
        self.quant_type = STORAGE[storage]
        self.layers, self.xs, self.logits = [], [], []
        # replica 0: the seeded workload weights; others: seeded GPU draws of the same law
        self.layers.append(synthetic.make_device_layer(cfg, seed=seed_base, device=device, quant_type=self.quant_type))
        for r in range(1, replicas):
            self.layers.append(self._gpu_replica(seed_base * 1000 + r))
        for r in range(replicas):
            x, lg = synthetic.inputs(cfg, M, seed=seed_base, replica=r, device=device)
            self.xs.append(x)
            self.logits.append(lg)
        self.outs = [torch.empty((M, cfg.H), dtype=torch.bfloat16, device=device) for _ in range(replicas)]
        self.ws = e4b.workspace(e4b.e4b_moe_expert_forward_workspace_size(M, self.layers[0].stack, cfg.k), device)
        self.touched = [self._touched(r) for r in range(replicas)]

    def _gpu_replica(self, seed):
        torch, e4b, cfg = self.torch, self.e4b, self.cfg
        from quantized_moe_expert_nf4_b200 import synthetic

        g = torch.Generator(device=self.device)
        g.manual_seed(seed)

        def pack(N, K):
            packed = torch.empty((cfg.E, N * K // 2), dtype=torch.uint8, device=self.device)
            absmax = torch.empty((cfg.E, N * K // 64), dtype=torch.float32, device=self.device)
            for e0 in range(0, cfg.E, 8):
                e1 = min(cfg.E, e0 + 8)
                W = torch.randn((e1 - e0, N, K), generator=g, device=self.device) * cfg.weight_std
                e4b.e4b_quantize_stack(W, packed[e0:e1], absmax[e0:e1], self.quant_type)
            return packed, absmax

        gp, ga = pack(2 * cfg.I, cfg.H)
        dp, da = pack(cfg.H, cfg.I)
        la = lb = None
        if cfg.lora_r:
            la = (torch.randn((cfg.E, cfg.lora_r, cfg.H), generator=g, device=self.device) * cfg.lora_std).bfloat16()
            lb = (torch.randn((cfg.E, 2 * cfg.I, cfg.lora_r), generator=g, device=self.device) * cfg.lora_std).bfloat16()
        stack = e4b.ExpertStack(gp, ga, dp, da, cfg.E, cfg.H, cfg.I, la, lb, cfg.lora_alpha, self.quant_type)
        return synthetic.DeviceLayer(cfg, gp, ga, dp, da, la, lb, stack)

    def _touched(self, r):
        """Experts with at least one routed slot, read from the library's own routing."""
        torch, e4b, cfg, M = self.torch, self.e4b, self.cfg, self.M
        S = M * cfg.k
        ids = torch.empty(S, dtype=torch.int32, device=self.device)
        w = torch.empty(S, dtype=torch.float32, device=self.device)
        offs = torch.empty(cfg.E + 1, dtype=torch.int32, device=self.device)
        perm = torch.empty(S, dtype=torch.int32, device=self.device)
        inv = torch.empty(S, dtype=torch.int32, device=self.device)
        ws = e4b.workspace(e4b.e4b_moe_route_permute_workspace_size(M, cfg.E, cfg.k), self.device)
        e4b.e4b_moe_route_permute(self.logits[r], cfg.k, True, ids, w, offs, perm, inv, ws)
        return int((offs[1:] - offs[:-1] > 0).sum().item())

    def forward(self, r):
        cfg = self.cfg
        self.e4b.e4b_moe_expert_forward(self.xs[r], self.logits[r], cfg.k, True, self.layers[r].stack, self.outs[r],
                                        self.ws)

    def capture(self):
        torch = self.torch
        R = len(self.layers)
        s = torch.cuda.Stream(device=self.device)
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for r in range(R):     # warm the library (attributes, caches) before capture
                self.forward(r)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        self.g_cycle = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.g_cycle):
            for r in range(R):
                self.forward(r)
        self.launches_per_step = self.e4b.last_launches()
        self.path = self.e4b.last_path()
        self.g_single = []
        for r in range(R):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self.forward(r)
            self.g_single.append(g)
        torch.cuda.synchronize()

    def run_steps(self, K, start=0):
        R = len(self.layers)
        i = 0
        while i < K:
            r = (start + i) % R
            if r == 0 and K - i >= R:
                self.g_cycle.replay()
                i += R
            else:
                self.g_single[r].replay()
                i += 1

    def time_steps(self, K, dist=None):
        torch = self.torch
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        self.run_steps(K)
        b.record()
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        return a.elapsed_time(b) / 1e3

    def kernel_timing(self, K):
        """Eager pass with per-kernel CUDA events: {name: (avg ms, launches)}."""
        e4b = self.e4b
        R = len(self.layers)
        self.torch.cuda.synchronize()
        e4b.timing_enable(True)
        for i in range(K):
            self.forward(i % R)
        res = e4b.timing_read()
        e4b.timing_enable(False)
        return {n: (ms / max(c, 1), c) for n, (ms, c) in res.items()}

    def e2e(self, K):
        """Public call with host buffers, per step: H2D copy of the step's inputs
        from pinned memory, the forward, and a D2H copy of its output into pinned
        memory.  At decode sizes (M <= 8) the host's per-call work sets the pace, so
        x and the router logits travel in one copy (one pinned staging buffer per
        replica holding both, the forward reading views of one device buffer) in
        the forward's own stream, with nothing else per step; above, the copies run
        on their own streams and overlap the forwards (e2e_pipelined)."""
        if self.M > 8:
            return self.e2e_pipelined(K)
        torch, cfg, M = self.torch, self.cfg, self.M
        R = len(self.layers)
        nx, nl = M * cfg.H * 2, M * cfg.E * 4              # bytes of x (bf16) and logits (fp32); nx % 16 == 0
        hin = []
        for x, l in zip(self.xs, self.logits):
            buf = torch.empty(nx + nl, dtype=torch.uint8).pin_memory()
            buf[:nx].copy_(x.cpu().view(torch.uint8).reshape(-1))
            buf[nx:].copy_(l.cpu().view(torch.uint8).reshape(-1))
            hin.append(buf)
        ho = [torch.empty((M, cfg.H), dtype=torch.bfloat16).pin_memory() for _ in range(R)]
        din = torch.empty(nx + nl, dtype=torch.uint8, device=self.xs[0].device)
        dx = din[:nx].view(torch.bfloat16).view(M, cfg.H)
        dl = din[nx:].view(torch.float32).view(M, cfg.E)
        do = torch.empty_like(self.outs[0])
        for i in range(min(3, K)):
            din.copy_(hin[i % R], non_blocking=True)
            self.e4b.e4b_moe_expert_forward(dx, dl, cfg.k, True, self.layers[i % R].stack, do, self.ws)
            ho[i % R].copy_(do, non_blocking=True)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for i in range(K):
            r = i % R
            din.copy_(hin[r], non_blocking=True)
            self.e4b.e4b_moe_expert_forward(dx, dl, cfg.k, True, self.layers[r].stack, do, self.ws)
            ho[r].copy_(do, non_blocking=True)
        b.record()
        torch.cuda.synchronize()
        t = a.elapsed_time(b) / 1e3
        return M * cfg.k * K / t, nx + nl, M * cfg.H * 2

    def e2e_pipelined(self, K):
        """Public call with host buffers, per step: H2D copies of the step's inputs
        from pinned memory, the forward, and a D2H copy of its output into pinned
        memory -- pipelined the way a serving loop runs them: the input copies of
        step i+1 (on a copy stream, into the other of two device input buffers)
        and the output copy of step i-1 (on a second copy stream) overlap the
        forward of step i; events order every buffer reuse."""
        torch, cfg, M = self.torch, self.cfg, self.M
        R = len(self.layers)
        hx = [x.cpu().pin_memory() for x in self.xs]
        hl = [l.cpu().pin_memory() for l in self.logits]
        ho = [torch.empty((M, cfg.H), dtype=torch.bfloat16).pin_memory() for _ in range(R)]
        dx = [torch.empty_like(self.xs[0]) for _ in range(2)]
        dl = [torch.empty_like(self.logits[0]) for _ in range(2)]
        do = [torch.empty_like(self.outs[0]) for _ in range(2)]
        comp = torch.cuda.current_stream()
        h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
        ev = lambda: torch.cuda.Event()
        copied, computed, read = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        used = [False, False]

        def step(i):
            b, r = i & 1, i % R
            with torch.cuda.stream(h2d_s):
                if used[b]:
                    h2d_s.wait_event(computed[b])        # the forward of step i-2 has read dx[b], dl[b]
                dx[b].copy_(hx[r], non_blocking=True)
                dl[b].copy_(hl[r], non_blocking=True)
                copied[b].record(h2d_s)
            comp.wait_event(copied[b])
            if used[b]:
                comp.wait_event(read[b])                 # the D2H of step i-2 has read do[b]
            self.e4b.e4b_moe_expert_forward(dx[b], dl[b], cfg.k, True, self.layers[r].stack, do[b], self.ws)
            computed[b].record(comp)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(computed[b])
                ho[r].copy_(do[b], non_blocking=True)
                read[b].record(d2h_s)
            used[b] = True

        for i in range(min(3, K)):
            step(i)
        torch.cuda.synchronize()
        a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(comp)
        h2d_s.wait_event(a)                              # the first input copy starts inside the timed region
        for i in range(K):
            step(i)
        for b in range(2):
            comp.wait_event(read[b])                     # every output has reached host memory
        e.record(comp)
        torch.cuda.synchronize()
        t = a.elapsed_time(e) / 1e3
        h2d = M * cfg.H * 2 + M * cfg.E * 4
        d2h = M * cfg.H * 2
        return M * cfg.k * K / t, h2d, d2h

    def e2e_graph(self, K):
        """As e2e, with each step's H2D input copies, public forward call and D2H
        read of the result captured once per replica in a CUDA graph and replayed
        per step (the graph-capture serving the decode path is built for): the
        copies still run every step; the host no longer issues each call."""
        torch, cfg, M = self.torch, self.cfg, self.M
        R = len(self.layers)
        hx = [x.cpu().pin_memory() for x in self.xs]
        hl = [l.cpu().pin_memory() for l in self.logits]
        ho = [torch.empty((M, cfg.H), dtype=torch.bfloat16).pin_memory() for _ in range(R)]
        dx = torch.empty_like(self.xs[0])
        dl = torch.empty_like(self.logits[0])
        do = torch.empty_like(self.outs[0])
        graphs = []
        for r in range(R):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                dx.copy_(hx[r], non_blocking=True)
                dl.copy_(hl[r], non_blocking=True)
                self.e4b.e4b_moe_expert_forward(dx, dl, cfg.k, True, self.layers[r].stack, do, self.ws)
                ho[r].copy_(do, non_blocking=True)
            graphs.append(g)
        for i in range(min(3, K)):
            graphs[i % R].replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for i in range(K):
            graphs[i % R].replay()
        b.record()
        torch.cuda.synchronize()
        t = a.elapsed_time(b) / 1e3
        del graphs
        h2d = M * cfg.H * 2 + M * cfg.E * 4
        d2h = M * cfg.H * 2
        return M * cfg.k * K / t, h2d, d2h


def replicas_for(cfg, M):
    S = M * cfg.k
    touched = workloads.expected_touched(workloads.popularity(cfg), cfg.E, S)
    per_step = max(touched * expert_bytes(cfg), 1.0)
    return int(min(32, max(2, math.ceil(4 * L2_BYTES / per_step))))


# DRAM bytes (read + write) per launch from one ncu capture of the kernel as it
# is now, keyed by (layer config, M, kernel); a kernel changed since its capture
# has no entry.
MEASURED_TRAFFIC = {
    ("olmoe", 1, "decode.fused"): 28421888 + 0,
    ("olmoe", 2048, "gemm.tc.swiglu"): 218631424 + 19088128,
    ("olmoe", 2048, "gemm.tc"): 109154304 + 32880896,
}


def dominant_roofline(cfg, M, kt, touched_avg, peaks, long_region):
    name, (avg_ms, n) = max(kt.items(), key=lambda kv: kv[1][0] * kv[1][1])
    S = M * cfg.k
    if name.startswith("decode.fused"):
        # HBM-bound: the whole layer in one launch, so its algorithmic bytes are
        # the step's (both stacks of the touched experts, x, out, the router logits)
        alg = step_work(cfg, M, touched_avg)[1]
        achieved = alg / (avg_ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        return name, {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                      "traffic": MEASURED_TRAFFIC.get((cfg.name, M, name)), "kernel": name, "avg_us": avg_ms * 1e3,
                      "algorithmic_bytes_per_launch": alg, "peak_source": peaks["source"] + " hbm_gbs"}
    if name.startswith("decode.gate_up") or name.startswith("decode.down"):
        # HBM-bound: the projection's packed bytes + absmax of the touched experts
        per_expert = gate_up_expert_bytes(cfg) if "gate_up" in name else cfg.H * cfg.I * (0.5 + 4.0 / 64)
        alg = touched_avg * per_expert + (M * cfg.H * 2 if "gate_up" in name else 0)
        achieved = alg / (avg_ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        return name, {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                      "traffic": MEASURED_TRAFFIC.get((cfg.name, M, name)), "kernel": name, "avg_us": avg_ms * 1e3,
                      "algorithmic_bytes_per_launch": alg, "peak_source": peaks["source"] + " hbm_gbs"}
    # tensor-bound GEMM of the grouped path
    if "swiglu" in name:
        flops = 2.0 * S * 2 * cfg.I * cfg.H
    else:
        flops = 2.0 * S * cfg.H * cfg.I
    achieved = flops / (avg_ms * 1e-3) / 1e12
    key = "bf16_tflops_sustained" if long_region else "bf16_tflops"
    peak = peaks[key]
    return name, {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                  "traffic": MEASURED_TRAFFIC.get((cfg.name, M, name)), "kernel": name, "avg_us": avg_ms * 1e3,
                  "algorithmic_flops_per_launch": flops,
                  "peak_source": peaks["source"] + " " + key}


def reduce_over_ranks(value, dist, device, op="max"):
    """Max (or min) of a per-rank float over all ranks; identity without a process group."""
    if dist is None:
        return float(value)
    import torch

    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.MIN)
    return float(t.item())


def job_throughput(per_rank_units, steps, world, max_seconds):
    """Whole-job units/s: every rank processes `per_rank_units` per step (weak scaling)."""
    return world * per_rank_units * steps / max_seconds


def measure(args, name, rank, world, dist, peaks, primary, e2e_steps=None):
    import torch

    cfgname, M, storage = workload(name)
    cfg = workloads.CONFIGS[cfgname]
    dev = f"cuda:{torch.cuda.current_device()}"
    R = args.replicas if args.replicas > 0 else replicas_for(cfg, M)
    b = Bench(cfg, M, dev, R, seed_base=rank, storage=storage)
    b.capture()
    b.run_steps(args.warmup)
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device())
    with sampler:
        t = b.time_steps(args.steps, dist)
    t = reduce_over_ranks(t, dist, dev, "max")
    S = M * cfg.k
    value = job_throughput(S, args.steps, world, t)
    ms = 1e3 * t / args.steps
    touched_avg = float(np.mean([b.touched[i % R] for i in range(args.steps)]))
    flops, nbytes = step_work(cfg, M, touched_avg)
    t_star = max(nbytes / (peaks["hbm_gbs"] * 1e9), flops / (peaks["bf16_tflops"] * 1e12))
    step_bound = "hbm" if nbytes / (peaks["hbm_gbs"] * 1e9) >= flops / (peaks["bf16_tflops"] * 1e12) else "tensor"
    t_star_nom = max(nbytes / (NOMINAL_PEAKS["hbm_gbs"] * 1e9), flops / (NOMINAL_PEAKS["bf16_tflops"] * 1e12))
    if args.no_kernel_timing:
        kt, roof = {}, None
    else:
        kt = b.kernel_timing(min(max(args.steps, 20), 400))
        kname, roof = dominant_roofline(cfg, M, kt, touched_avg, peaks, long_region=t > 1.0)
    res = {
        "value": value, "ms_per_step": ms, "tflops": world * flops / (ms * 1e-3) / 1e12 if ms else None,
        "path": b.path, "launches_per_step": b.launches_per_step, "touched_experts_avg": touched_avg,
        "replicas": R, "roofline": roof,
        "step_roofline": {"bound": step_bound, "t_star_us": t_star * 1e6, "frac": t_star / (ms * 1e-3),
                          "algorithmic_bytes": nbytes, "algorithmic_flops": flops,
                          "peaks": {"hbm_gbs": peaks["hbm_gbs"], "bf16_tflops": peaks["bf16_tflops"],
                                    "source": peaks["source"]},
                          "nominal": {"peaks": NOMINAL_PEAKS, "source": "nominal B200 figures",
                                      "t_star_us": t_star_nom * 1e6, "frac": t_star_nom / (ms * 1e-3)}},
        "kernels_us": {k: v[0] * 1e3 for k, v in kt.items()},
        "clocks": sampler.summary(),
    }
    res["e2e"] = None
    res["e2e_graph"] = None
    if (primary or e2e_steps) and not args.no_e2e:
        K = e2e_steps or min(args.steps, 2000)
        ev, h2d, d2h = b.e2e(K)
        ev = reduce_over_ranks(ev, dist, dev, "min") * world
        res["e2e"] = {"value": ev, "unit": "routed_tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                      "how": ("per step: one H2D copy of x and the logits from one pinned buffer, the public "
                              "forward call on views of one device buffer, D2H of the output into pinned memory, "
                              "all in the forward's stream" if b.M <= 8 else
                              "per step: H2D of the inputs from pinned memory on a copy stream (double-buffered), "
                              "the public forward call, D2H of the output into pinned memory on a second copy "
                              "stream; copies of neighbouring steps overlap the forward")}
        gerr = None
        try:
            gv, h2d, d2h = b.e2e_graph(K)
        except Exception as exc:  # reported, the headline line still prints
            gv, gerr = 0.0, f"{type(exc).__name__}: {exc}"
        gv = reduce_over_ranks(gv, dist, dev, "min") * world   # every rank takes this collective
        res["e2e_graph"] = {"error": gerr} if gerr else {
            "value": gv, "unit": "routed_tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "how": "per step: one CUDA-graph replay of the H2D input copies, the public forward call and the D2H "
                   "read, captured per replica"}
    res["cfg"] = cfg
    res["M"] = M
    res["storage"] = storage
    del b
    torch.cuda.empty_cache()
    return res


# Nominal B200 figures (HBM3e 8 TB/s, dense bf16 2.25 PFLOP/s), reported beside the measured peaks.
NOMINAL_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}


def time_quantize(cfg, dev, reps=3, storage="nf4"):
    """Load-time step, timed apart from the forward: e4b_quantize_stack on the
    layer's whole gate_up stack from fp32 ([E, 2I, H]); HBM-bound (4 B read +
    0.5 + 4/64 B written per weight)."""
    import torch

    from quantized_moe_expert_nf4_b200 import e4b

    W = torch.randn((cfg.E, 2 * cfg.I, cfg.H), device=dev, dtype=torch.float32)
    n = W.numel()
    packed = torch.empty(n // 2, dtype=torch.uint8, device=dev)
    absmax = torch.empty(n // 64, dtype=torch.float32, device=dev)
    qt = STORAGE[storage]
    e4b.e4b_quantize_stack(W, packed, absmax, qt)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        e4b.e4b_quantize_stack(W, packed, absmax, qt)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    nbytes = n * (4 + 0.5 + 4.0 / 64)
    del W, packed, absmax
    torch.cuda.empty_cache()
    return {"stack": f"gate_up [{cfg.E}, {2 * cfg.I}, {cfg.H}] fp32", "storage": storage, "ms": ms,
            "bytes": nbytes, "GB_per_s": nbytes / (ms * 1e-3) / 1e9}


MXFP4_WORKLOAD = "gptoss_m8192"   # released MXFP4 experts: gpt-oss-shaped gate_up, prefill routing


def time_mxfp4(name, dev, steps=5, warmup=2):
    """The grouped GEMM straight from MXFP4 bytes (e4b_grouped_mxfp4_gemm) on the
    gate_up projection of the workload's layer shape: the routed rows of the
    workload's own routing (e4b_moe_route_permute), seeded random e2m1 codes and
    e8m0 scales around 2^0, SwiGLU epilogue, bf16 out.  Algorithmic FLOPs
    2*S*2I*H; timed apart from the forward with CUDA events on its stream."""
    import torch

    from quantized_moe_expert_nf4_b200 import e4b, synthetic

    cfgname, M, _ = workload(name)
    cfg = workloads.CONFIGS[cfgname]
    E, H, I, k = cfg.E, cfg.H, cfg.I, cfg.k
    S = M * k
    x, logits = synthetic.inputs(cfg, M, device=dev)
    ids = torch.empty((M, k), dtype=torch.int32, device=dev)
    w = torch.empty((M, k), dtype=torch.float32, device=dev)
    offs = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(S, dtype=torch.int32, device=dev)
    inv = torch.empty(S, dtype=torch.int32, device=dev)
    rws = e4b.workspace(e4b.e4b_moe_route_permute_workspace_size(M, E, k), dev)
    e4b.e4b_moe_route_permute(logits, k, True, ids, w, offs, perm, inv, rws)
    row_token = torch.div(perm, k, rounding_mode="floor").to(torch.int32)
    g = torch.Generator(device=dev)
    g.manual_seed(11)
    N, K = 2 * I, H
    blocks = torch.randint(0, 256, (E, N * K // 2), generator=g, device=dev, dtype=torch.uint8)
    scales = torch.randint(124, 131, (E, N * K // 32), generator=g, device=dev, dtype=torch.uint8)
    out = torch.empty((S, I), dtype=torch.bfloat16, device=dev)
    ws = e4b.workspace(e4b.e4b_grouped_mxfp4_gemm_workspace_size(S, N, K), dev)

    def call():
        e4b.e4b_grouped_mxfp4_gemm(x, row_token, offs, S, blocks, scales, N, K, out, e4b.E4B_EPI_SWIGLU, ws)

    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        call()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    flops = 2.0 * S * N * K
    res = {"workload": name, "projection": f"gate_up [{E}, {N}, {K}] MXFP4", "routed_rows": S, "ms": ms,
           "tflops": flops / (ms * 1e-3) / 1e12, "algorithmic_flops": flops, "path": e4b.last_path()}
    del x, logits, ids, w, offs, perm, inv, rws, row_token, blocks, scales, out, ws
    torch.cuda.empty_cache()
    return res


def repeat_forward(name, reps):
    """Profiling driver for ncu captures: the workload's layer (seed 0) and its
    first input batch, then `reps` calls of the public forward; nothing is
    timed.  Prints the path of the last call."""
    import torch

    from quantized_moe_expert_nf4_b200 import e4b, synthetic

    cfgname, M = WORKLOADS[name][:2]
    cfg = workloads.CONFIGS[cfgname]
    e4b.load_library()
    layer = synthetic.make_device_layer(cfg)
    x, logits = synthetic.inputs(cfg, M)
    out = torch.empty((M, cfg.H), dtype=torch.bfloat16, device="cuda")
    ws = e4b.workspace(e4b.e4b_moe_expert_forward_workspace_size(M, layer.stack, cfg.k))
    for _ in range(reps):
        e4b.e4b_moe_expert_forward(x, logits, cfg.k, True, layer.stack, out, ws)
    torch.cuda.synchronize()
    print("ok", e4b.last_path(), flush=True)


BACKWARD_WORKLOAD = "qwen3_lora_m4096"   # the pages' training shape: Qwen3-MoE-shaped layer with per-expert LoRA


def time_backward(name, dev, steps=10, warmup=3):
    """The layer backward (e4b_moe_expert_backward: recompute, two grouped dgrad
    products, router and adapter gradients), timed apart from the forward with
    CUDA events on its stream.  Algorithmic FLOPs: the recompute 6*S*H*I plus the
    two dgrad products 6*S*H*I (plus the adapter's terms)."""
    import torch

    from quantized_moe_expert_nf4_b200 import e4b, synthetic

    cfgname, M, _ = workload(name)
    cfg = workloads.CONFIGS[cfgname]
    layer = synthetic.make_device_layer(cfg, device=dev)
    x, logits = synthetic.inputs(cfg, M, device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(7)
    dout = torch.randn((M, cfg.H), generator=g, device=dev).bfloat16()
    dx = torch.empty((M, cfg.H), dtype=torch.float32, device=dev)
    dl = torch.empty((M, cfg.E), dtype=torch.float32, device=dev)
    dA = dB = None
    if cfg.lora_r:
        dA = torch.empty((cfg.E, cfg.lora_r, cfg.H), dtype=torch.float32, device=dev)
        dB = torch.empty((cfg.E, 2 * cfg.I, cfg.lora_r), dtype=torch.float32, device=dev)
    ws = e4b.workspace(e4b.e4b_moe_expert_backward_workspace_size(M, layer.stack, cfg.k), dev)

    def call():
        e4b.e4b_moe_expert_backward(x, logits, cfg.k, True, layer.stack, dout, dx, dl, dA, dB, ws)

    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        call()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    launches = e4b.last_launches()
    e4b.timing_enable(True)
    call()
    kt = e4b.timing_read()
    e4b.timing_enable(False)
    S = M * cfg.k
    flops = 12.0 * S * cfg.H * cfg.I
    if cfg.lora_r:
        flops += 6.0 * S * cfg.lora_r * (cfg.H + 2 * cfg.I)
    res = {"workload": name, "ms": ms, "value": S / (ms * 1e-3), "unit": "routed_tokens/s",
           "tflops": flops / (ms * 1e-3) / 1e12, "algorithmic_flops": flops, "launches": launches,
           "path": e4b.last_path(), "kernels_us": {k: v[0] * 1e3 / max(v[1], 1) for k, v in kt.items()}}
    del layer, x, logits, dout, dx, dl, dA, dB, ws
    torch.cuda.empty_cache()
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="e4b", choices=["e4b", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end host-buffer pass")
    ap.add_argument("--no-kernel-timing", action="store_true", help="skip the per-kernel event pass")
    ap.add_argument("--no-backward", action="store_true", help="skip the layer-backward timing")
    ap.add_argument("--no-mxfp4", action="store_true", help="skip the MXFP4 grouped-GEMM timing")
    ap.add_argument("--replicas", type=int, default=0, help="layer replicas (0: enough to exceed L2 4x)")
    ap.add_argument("--repeat-forward", type=int, default=0, metavar="N",
                    help="profiling driver: build the workload's layer and call the forward N times, untimed")
    args = ap.parse_args()
    if args.repeat_forward > 0:
        repeat_forward(args.workload, args.repeat_forward)
        return
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    cfgname, M, storage = workload(args.workload)
    cfg = workloads.CONFIGS[cfgname]

    if args.impl == "reference":
        run_reference(args, cfg, M, rank, world)
        return

    import torch

    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as td

        td.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device(f"cuda:{local}"))
        dist = td
    from quantized_moe_expert_nf4_b200 import build, e4b

    build.build()
    e4b.load_library()
    peaks = load_peaks()

    main_res = measure(args, args.workload, rank, world, dist, peaks, primary=True)
    sweep = []
    if not args.no_sweep and args.workload == DEFAULT_WORKLOAD:
        for name in DEFAULT_SWEEP:
            try:
                r = measure(args, name, rank, world, dist, peaks, primary=False,
                            e2e_steps=min(args.steps, 200) if name in E2E_SWEEP else None)
            except Exception as exc:  # a failing sweep row is reported, the headline line still prints
                sweep.append({"workload": name, "error": f"{type(exc).__name__}: {exc}"})
                torch.cuda.empty_cache()
                continue
            sweep.append({"workload": name, "storage": r["storage"], "value": r["value"],
                          "ms_per_step": r["ms_per_step"],
                          "tflops": r["tflops"], "path": r["path"], "touched_experts_avg": r["touched_experts_avg"],
                          "roofline_frac": r["roofline"]["frac"] if r["roofline"] else None,
                          "roofline_bound": r["roofline"]["bound"] if r["roofline"] else None,
                          "roofline_kernel": r["roofline"]["kernel"] if r["roofline"] else None,
                          "step_roofline_frac": r["step_roofline"]["frac"],
                          "clocks": r["clocks"]})
            if name in E2E_SWEEP:
                sweep[-1]["e2e"] = r["e2e"]
                sweep[-1]["e2e_graph"] = r["e2e_graph"]
                if rank == 0 and world == 1 and not args.no_cpu_baseline:
                    rc, rstorage = workloads.CONFIGS[workload(name)[0]], workload(name)[2]
                    rate, desc, spent = oracle_rate(rc, workload(name)[1], budget_s=3.0, max_tokens=2,
                                                    storage=rstorage)
                    sweep[-1]["cpu_baseline"] = {"value": rate, "unit": "routed_tokens/s", "cores": cpu_cores(),
                                                 "cpu": cpu_model(), "kind": "oracle", "sample": desc,
                                                 "seconds": spent}
    quant = None
    bwd = None
    mx = None
    if rank == 0 and world == 1:
        quant = time_quantize(cfg, f"cuda:{local}")
        quant["frac_hbm"] = quant["GB_per_s"] / peaks["hbm_gbs"]
        q4 = time_quantize(cfg, f"cuda:{local}", storage="fp4")
        quant["fp4"] = {"GB_per_s": q4["GB_per_s"], "ms": q4["ms"], "frac_hbm": q4["GB_per_s"] / peaks["hbm_gbs"]}
        if not args.no_mxfp4:
            try:
                mx = time_mxfp4(MXFP4_WORKLOAD, f"cuda:{local}")
                mx["frac_tensor"] = mx["tflops"] / peaks["bf16_tflops"]
            except Exception as exc:  # reported, the headline line still prints
                mx = {"workload": MXFP4_WORKLOAD, "error": f"{type(exc).__name__}: {exc}"}
                torch.cuda.empty_cache()
        if not args.no_backward:
            bwd = time_backward(BACKWARD_WORKLOAD, f"cuda:{local}")
            bwd["frac_tensor"] = bwd["tflops"] / peaks["bf16_tflops"]
    if rank == 0:
        cb = None
        if world == 1 and not args.no_cpu_baseline:
            rate, desc, spent = oracle_rate(cfg, M, budget_s=12.0, max_tokens=8, storage=storage)
            cb = {"value": rate, "unit": "routed_tokens/s", "cores": cpu_cores(), "cpu": cpu_model(), "kind": "oracle",
                  "sample": desc, "seconds": spent}
        line = {
            "metric": METRIC, "value": main_res["value"], "unit": "routed_tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": main_res["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": args.workload, "model": f"{cfg.name}-shaped MoE layer", "E": cfg.E, "H": cfg.H,
                       "I": cfg.I, "k": cfg.k, "M": M, "routing": cfg.routing, "weights": f"{storage.upper()}/64 fp32 absmax",
                       "replicas": main_res["replicas"],
                       "l2": f"inputs larger than L2: {main_res['replicas']} layer replicas cycled",
                       "global_batch": M * world, "parallelism": f"replicas x{world}", "timing": "CUDA graphs"},
            "tflops": main_res["tflops"], "path": main_res["path"],
            "touched_experts_avg": main_res["touched_experts_avg"],
            "roofline": main_res["roofline"], "step_roofline": main_res["step_roofline"],
            "kernels_us": main_res["kernels_us"],
            "cpu_baseline": cb, "e2e": main_res["e2e"], "e2e_graph": main_res["e2e_graph"],
            "clocks": main_res["clocks"],
            "gpu_launches": main_res["launches_per_step"] * args.steps,
            "quantize": quant,
            "backward": bwd,
            "mxfp4_gemm": mx,
            "sweep": sweep,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
