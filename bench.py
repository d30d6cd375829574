#!/usr/bin/env python
"""Benchmark of one top-k MoE FFN layer step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload (the headline): a Qwen3.6-35B-A3B-shaped MoE layer (hidden 2048,
256 experts top-8, expert inter 512, shared expert inter 512 with sigmoid
gate, FP8 e4m3 weights with fp32 128x128 block scales, bf16 activations),
decode at rows = 1.  One step = one layer forward (router + top-k, routed and
shared experts, blend) through the C ABI.  Inputs are seeded and synthetic
and resident in HBM; 16 device copies of the layer's weights (12.9 GB) are
used in rotation, so a step never finds its weights in the 126 MB L2.

Printed: one JSON line (rank 0).  `value` is achieved HBM GB/s over the
algorithmic bytes of the step (whole job: summed over ranks), with
microseconds per layer, tokens/s and the fraction of the measured copy
bandwidth beside it; a rows = 64 sub-measurement; the dominant kernel's
roofline from per-kernel CUDA events; the same metric end to end through the
public API with host buffers (`e2e`); and the CPU oracle on the host's cores
(`cpu_baseline`).  N > 1 (torchrun) runs independent replicas, one per GPU
(the layer has no exchange step): max-over-ranks time, weak scaling.

`--impl reference` times the CPU oracle (the reference arm of this build) on
the same workload and prints the same line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE layer µs & HBM GB/s (% of peak) at rows=1/64; prefill FP8 TFLOP/s (% peak)"
WORKLOAD = "Qwen3.6-35B-A3B-shaped MoE FFN layer, decode rows=1"
N_INSTANCES = 16
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
# The arithmetic each leg computes in.
DECODE_DTYPE = ("fp8e4m3 weights (fp32 block scales) x bf16 x for gate/up and x fp32 h for down, "
                "exact products, fp32 accumulate")
GROUPED_DTYPE = ("fp8e4m3 weights (fp32 block scales) x activations as two e4m3 terms (hi + lo, fp32 scale "
                 "per 128 block), fp32 accumulate")


# ----------------------------------------------------------------- helpers

def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-extras", action="store_true", help="skip the rows=64 and per-kernel legs")
    ap.add_argument("--profile", choices=["decode", "prefill", "narrow", "nvfp4"], default=None,
                    help="a small case for a profiler: a few eager layer calls on one weight copy, then exit "
                         "(decode: rows=1; prefill: 4096 biased rows; narrow: the narrow grouped GEMMs at --rows)")
    ap.add_argument("--rows", type=int, default=64, help="rows of --profile narrow")
    ap.add_argument("--calls", type=int, default=4, help="layer calls of --profile")
    ap.add_argument("--sweep", action="store_true",
                    help="time every decode workload (35B rows 1..64, 397B rows 1 and 32) and print one JSON line")
    return ap.parse_args(argv)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), float(j.get("bf16_tflops", FALLBACK_BF16_TFLOPS)), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def algorithmic_bytes(d, rows: int, n_active: int, residual: bool = False) -> dict:
    """Bytes the layer step must move (each touched weight byte once)."""
    H, I, Is, E = d.hidden, d.inter, d.shared_inter, d.n_experts
    k = d.top_k
    exp_b = 3 * I * H + 4 * ((2 * I // 128) * (H // 128) + (H // 128) * (I // 128))
    sh_b = 3 * Is * H + 4 * ((2 * Is // 128) * (H // 128) + (H // 128) * (Is // 128))
    router = 2 * E * H + 2 * H
    act = 2 * rows * H * (3 if residual else 2)
    gu = (n_active * (2 * I * H + 4 * (2 * I // 128) * (H // 128)) + 2 * Is * H
          + 4 * (2 * Is // 128) * (H // 128) + 2 * rows * H + 4 * rows * (k * I + Is))
    dn = (n_active * (I * H + 4 * (H // 128) * (I // 128)) + Is * H + 4 * (H // 128) * (Is // 128)
          + 4 * rows * (k * I + Is) + 2 * rows * H)
    rt = router + 2 * rows * H + rows * (8 * k + 4)
    total = n_active * exp_b + sh_b + router + act
    return {"total": total, "experts": n_active * exp_b + sh_b, "decode_step": total,
            "router_topk": rt, "gate_up": gu, "down_blend": dn}


def prefill_flops(d, rows: int) -> dict:
    """Algorithmic FLOPs of a prefill step (2 per multiply-add): router GEMV,
    then per token k routed experts and the shared expert (gate_up 2I x H,
    down H x I)."""
    H, I, Is, E, k = d.hidden, d.inter, d.shared_inter, d.n_experts, d.top_k
    g1 = rows * (k * 2 * (2 * I) * H + 2 * (2 * Is) * H)
    g2 = rows * (k * 2 * I * H + 2 * Is * H)
    rt = rows * (2 * E * H + 2 * H)
    return {"total": g1 + g2 + rt, "gemm_gate_up": g1, "gemm_down": g2, "router_topk": rt}


def prefill_bytes(d, rows: int, n_active: int) -> int:
    """Bytes a prefill step must move: the touched weights once, x, out."""
    return algorithmic_bytes(d, rows, n_active)["total"]


def prefill_executed_flops(d, counts) -> dict:
    """Tensor-core FLOPs the two GEMMs issue: every expert's rows padded to
    128-row tiles, and each activation as two e4m3 terms (hi and lo)."""
    H, I, Is = d.hidden, d.inter, d.shared_inter
    tiles = sum((int(c) + 127) // 128 for c in counts)
    ts = (int(sum(counts)) // d.top_k + 127) // 128
    g1 = 2 * 2 * 128 * (tiles * 2 * I * H + ts * 2 * Is * H)
    g2 = 2 * 2 * 128 * (tiles * I * H + ts * Is * H)
    return {"gemm_gate_up": g1, "gemm_down": g2}


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons for one GPU."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str | None):
        self.bus_id = bus_id
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.bus_id:
            cmd += ["-i", self.bus_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark_begin(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = [l for (t, l) in self.lines if self.t0 is None or (self.t0 - 0.05 <= t <= (self.t1 or t) + 0.15)]
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in rows:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def source_hash(paths) -> str:
    h = hashlib.sha256()
    for p in paths:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload_tag: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source (else None).  The summary names the source
    files the kernel is built from (`source_files:`, paths under the package's
    csrc/; all of csrc/ when absent) and their hash at capture time."""
    prof = os.path.join(ROOT, "profiles", f"{kernel}_{workload_tag}.md")
    if not os.path.exists(prof):
        return None
    txt = open(prof).read()
    m = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    h = re.search(r"source_sha256_16:\s*([0-9a-f]+)", txt)
    if not m or not h:
        return None
    csrc = os.path.join(ROOT, "sparse_moe_ffn_topk_b200", "csrc")
    f = re.search(r"source_files:\s*(.+)", txt)
    names = f.group(1).split() if f else os.listdir(csrc)
    srcs = sorted(os.path.join(csrc, n) for n in names)
    if not all(os.path.exists(q) for q in srcs) or h.group(1) != source_hash(srcs):
        return None
    return float(m.group(1))


# ------------------------------------------------------------- distributed

class Dist:
    def __init__(self, gpus: int):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = False
        if self.world > 1:
            import datetime

            import torch
            import torch.distributed as dist
            backend = "nccl" if torch.cuda.is_available() else "gloo"
            if backend == "nccl":
                torch.cuda.set_device(self.local)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = True

    def barrier(self):
        if self.pg:
            import torch.distributed as dist
            dist.barrier()

    def max(self, v: float) -> float:
        return reduce_max(v, self.pg)

    def close(self):
        if self.pg:
            import torch.distributed as dist
            dist.destroy_process_group()


def reduce_max(v: float, active: bool) -> float:
    """Max of a float over the ranks of the default process group (identity
    without one)."""
    if not active:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(v)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    return units_per_rank * world / max_seconds


# --------------------------------------------------------------- our arm

def make_instances(layer, n: int):
    import torch

    import sparse_moe_ffn_topk_b200 as moe  # noqa: F401
    base = {
        "router_w": torch.from_numpy(layer.router_w.view("int16")).view(torch.bfloat16),
        "shared_gate": torch.from_numpy(layer.shared_gate.view("int16")).view(torch.bfloat16),
        "expert_w8": torch.from_numpy(layer.expert_w8),
        "expert_scales": torch.from_numpy(layer.expert_scales),
        "shared_w8": torch.from_numpy(layer.shared_w8),
        "shared_scales": torch.from_numpy(layer.shared_scales),
    }
    first = {k: v.cuda() for k, v in base.items()}
    insts = [first] + [{k: v.clone() for k, v in first.items()} for _ in range(n - 1)]
    return insts


class DecodeBench:
    def __init__(self, dims, insts, xs, rows, path=None):
        import torch

        import sparse_moe_ffn_topk_b200 as moe
        self.moe, self.torch = moe, torch
        self.path = moe.MOE_PATH_AUTO if path is None else path
        self.d, self.insts, self.xs, self.rows = dims, insts, xs, rows
        self.outs = [torch.empty(rows, dims.hidden, dtype=torch.bfloat16, device="cuda") for _ in range(len(xs))]
        self.ws = moe.alloc_workspace(dims, rows)
        self.stream = torch.cuda.Stream()

    def step(self, i, events=None):
        w = self.insts[i % len(self.insts)]
        x = self.xs[i % len(self.xs)]
        out = self.outs[i % len(self.outs)]
        args = (self.d, x, w["router_w"], w["expert_w8"], w["expert_scales"], w["shared_w8"], w["shared_scales"],
                w["shared_gate"], out, self.ws)
        if events is None:
            self.moe.ffn_forward_path(*args, path=self.path, stream=self.stream)
        else:
            self.moe.ffn_forward_timed(*args, events=events, path=self.path, stream=self.stream)

    def graph(self, first: int, count: int, events=None):
        torch = self.torch
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream):
            for j in range(count):
                self.step(first + j, None if events is None else events[j])
        return g

    def run_steps(self, first: int, count: int, chunk: int = 256):
        """Graphs covering exactly `count` steps starting at `first`."""
        graphs = []
        done = 0
        while done < count:
            n = min(chunk, count - done)
            graphs.append(self.graph(first + done, n))
            done += n
        return graphs

    def time_steps(self, steps: int, warmup: int, dist: Dist, sampler: ClockSampler | None = None):
        torch = self.torch
        with torch.cuda.stream(self.stream):
            for i in range(min(warmup, 3)):
                self.step(i)                       # eager, also sets up kernel attributes
        torch.cuda.synchronize()
        wg = self.run_steps(0, max(warmup, 3))
        tg = self.run_steps(max(warmup, 3), steps)
        for g in wg:
            g.replay()
        # a graph's first replay also uploads it (about 2 us a kernel node
        # measured here); a serving loop replays the same graph many times,
        # so each timed graph is replayed once, untimed, first
        for g in tg:
            g.replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        dist.barrier()
        torch.cuda.synchronize()
        if sampler:
            sampler.mark_begin()
        with torch.cuda.stream(self.stream):
            torch.cuda.nvtx.range_push("timed")
            e0.record(self.stream)
            for g in tg:
                g.replay()
            e1.record(self.stream)
            torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        # keep the same load for >= 1 s so the clock samples see it
        t_end = time.time() + max(0.0, 1.0 - ms / 1000.0)
        while time.time() < t_end:
            for g in tg:
                g.replay()
            torch.cuda.synchronize()
        if sampler:
            sampler.mark_end()
        dist.barrier()
        torch.cuda.synchronize()
        return ms, len(tg)

    def per_kernel_us(self, steps: int, names, batch: int = 48):
        """Mean duration of each kernel of a step, from CUDA events the library
        records around its launches (programmatic dependent launch off).
        Steps are enqueued eagerly behind a GPU sleep, so that the stream is
        full before the GPU reaches them and each event interval is GPU time."""
        torch = self.torch
        nk = self.moe.kernel_launches(self.d, self.rows, self.path)
        per = []
        done = 0
        while done < steps:
            n = min(batch, steps - done)
            evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)] for _ in range(n)]
            for row in evs:
                for e in row:
                    e.record(self.stream)  # torch creates the event handle on first record
            with torch.cuda.stream(self.stream):
                torch.cuda._sleep(50_000_000)  # ~25 ms of GPU time while the host enqueues
                for j in range(n):
                    self.step(done + j, events=evs[j])
            torch.cuda.synchronize()
            per += [[row[j].elapsed_time(row[j + 1]) * 1000.0 for j in range(nk)] for row in evs]
            done += n
        return {names[j] if j < len(names) else f"k{j}": statistics.median(p[j] for p in per) for j in range(nk)}

    def routing(self, n_steps: int):
        """Distinct experts per step, from the routing this path computes."""
        torch, moe = self.torch, self.moe
        counts = []
        idx = torch.empty(self.rows, self.d.top_k, dtype=torch.int32, device="cuda")
        for i in range(n_steps):
            w = self.insts[i % len(self.insts)]
            out = self.outs[i % len(self.outs)]
            moe.ffn_forward_path(self.d, self.xs[i % len(self.xs)], w["router_w"], w["expert_w8"],
                                 w["expert_scales"], w["shared_w8"], w["shared_scales"], w["shared_gate"], out,
                                 self.ws, topk_idx=idx)
            counts.append(int(torch.unique(idx).numel()))
        return counts


class ChainBench(DecodeBench):
    """A stack of layers behind their RMSNorms: step i runs layer i mod L on
    the one residual stream r in place, r <- r + layer(bf16(rmsnorm(r) * w)),
    so every step reads the previous step's output (one launch per layer on
    the decode path, chained by programmatic dependent launch)."""

    def __init__(self, dims, insts, norm_ws, resid, rows):
        super().__init__(dims, insts, [resid], rows)
        self.norm_ws = norm_ws
        self.r = resid

    def step(self, i, events=None):
        w = self.insts[i % len(self.insts)]
        self.moe.ffn_forward_norm(self.d, self.r, self.norm_ws[i % len(self.norm_ws)], 1e-6, w["router_w"],
                                  w["expert_w8"], w["expert_scales"], w["shared_w8"], w["shared_scales"],
                                  w["shared_gate"], self.r, self.ws, stream=self.stream)


class Nvfp4Bench(DecodeBench):
    """Decode steps of a layer with NVFP4 experts (moe_ffn_forward_nvfp4):
    the router, gate/up and down + blend kernels; insts hold each weight
    copy's NVFP4 codes, block scales and tensor scales."""

    def step(self, i, events=None):
        w = self.insts[i % len(self.insts)]
        self.moe.ffn_forward_nvfp4(self.d, self.xs[i % len(self.xs)], w["router_w"], w["w4"], w["sf"], w["gs"],
                                   w["sw4"], w["ssf"], w["sgs"], w["shared_gate"], self.outs[i % len(self.outs)],
                                   self.ws, stream=self.stream)


def nvfp4_instances(d, n: int, seed: int):
    """n copies of a layer's weights with NVFP4 experts, drawn on the GPU (the
    timing does not depend on the values): codes uniform, block scales e4m3
    codes of values around the N(0, 0.02) weights' block maxima, tensor scale
    amax/(448*6); router and gate N(0, 0.02) bf16."""
    import torch

    g = torch.Generator(device="cuda").manual_seed(seed)
    E, H, I, Is = d.n_experts, d.hidden, d.inter, d.shared_inter
    gs = 0.1 / (448 * 6)  # a matrix maximum near 5 sigma

    def scales(n_):
        # a 16-element block maximum near 2.5 sigma: amax16 / (6 gs) ~ 224, spread x [0.5, 1.5]
        return (torch.rand(n_, generator=g, device="cuda") + 0.5).mul(224.0).to(torch.float8_e4m3fn).view(torch.uint8)

    insts = []
    for _ in range(n):
        insts.append({
            "router_w": (0.02 * torch.randn(E, H, generator=g, device="cuda")).to(torch.bfloat16),
            "shared_gate": (0.02 * torch.randn(H, generator=g, device="cuda")).to(torch.bfloat16),
            "w4": torch.randint(0, 256, (E, 3 * I * H // 2), generator=g, device="cuda", dtype=torch.uint8),
            "sf": scales(E * 3 * I * H // 16).view(E, -1),
            "gs": torch.full((E, 2), gs, device="cuda", dtype=torch.float32),
            "sw4": torch.randint(0, 256, (3 * Is * H // 2,), generator=g, device="cuda", dtype=torch.uint8),
            "ssf": scales(3 * Is * H // 16),
            "sgs": torch.full((2,), gs, device="cuda", dtype=torch.float32),
        })
    return insts


def nvfp4_bytes(d, rows: int, n_active: float) -> float:
    """Algorithmic bytes of an NVFP4 step: the active experts' codes, block
    scales and tensor scales, the shared expert, router, gate, x and out."""
    H, I, Is, E = d.hidden, d.inter, d.shared_inter, d.n_experts
    per = lambda i: 3 * i * H / 2 + 3 * i * H / 16 + 8
    return n_active * per(I) + per(Is) + 2 * E * H + 2 * H + 2 * rows * H * 2


class PrefillBench(DecodeBench):
    """Prefill steps of the same layer: `rows` tokens, a per-expert router
    bias, the prefill path (permute -> tcgen05 grouped GEMMs -> blend)."""

    def __init__(self, dims, inst, bias, xs, rows):
        super().__init__(dims, [inst], xs, rows)
        self.bias = bias

    def step(self, i, events=None):
        w = self.insts[0]
        x = self.xs[i % len(self.xs)]
        out = self.outs[i % len(self.outs)]
        args = (self.d, x, w["router_w"], w["expert_w8"], w["expert_scales"], w["shared_w8"], w["shared_scales"],
                w["shared_gate"], out, self.ws)
        if events is None:
            self.moe.ffn_forward_path(*args, path=self.moe.MOE_PATH_PREFILL, router_bias=self.bias,
                                      stream=self.stream)
        else:
            self.moe.ffn_forward_timed(*args, events=events, path=self.moe.MOE_PATH_PREFILL,
                                       router_bias=self.bias, stream=self.stream)

    def expert_counts(self):
        torch, moe = self.torch, self.moe
        idx = torch.empty(self.rows, self.d.top_k, dtype=torch.int32, device="cuda")
        w = self.insts[0]
        moe.ffn_forward_path(self.d, self.xs[0], w["router_w"], w["expert_w8"], w["expert_scales"],
                             w["shared_w8"], w["shared_scales"], w["shared_gate"], self.outs[0], self.ws,
                             path=moe.MOE_PATH_PREFILL, router_bias=self.bias, topk_idx=idx)
        return torch.bincount(idx.flatten().long(), minlength=self.d.n_experts).cpu().tolist()


PREFILL_KERNELS = ["router_topk", "scan", "permute", "gemm_gate_up", "gemm_down", "blend"]


def prefill_leg(args, d, inst, dist: Dist, bus, hbm_peak, bf16_peak, peak_kind):
    """The 4096-token prefill: whole-step and per-kernel times, TFLOP/s
    against the FP8 dense peak (the measured bf16 GEMM peak x 2, the nominal
    fp8:bf16 ratio of the part)."""
    import torch

    import moe_inputs as mi
    rows = 4096
    bias = torch.from_numpy(mi.make_router(d, args.seed, True)[2]).cuda()
    xs = [torch.from_numpy(mi.make_x(d, rows, seed=args.seed + 3, stream=i).view("int16")).view(torch.bfloat16)
          .cuda() for i in range(2)]
    pb = PrefillBench(d, inst, bias, xs, rows)
    counts = pb.expert_counts()
    n_active = sum(1 for c in counts if c)
    fl = prefill_flops(d, rows)
    ex = prefill_executed_flops(d, counts)
    fp8_peak = 2.0 * bf16_peak
    kp = max(10, min(50, args.steps // 40))
    sampler = ClockSampler(bus)
    sampler.start()
    ms, _ = pb.time_steps(kp, max(3, min(args.warmup, 5)), dist, sampler)
    clocks = sampler.stop()
    s = dist.max(ms / 1000.0)
    step_s = s / kp
    tflops = aggregate(kp * fl["total"], dist.world, s) / 1e12
    res = {"workload": f"Qwen3.6-35B-A3B-shaped MoE FFN layer, prefill rows={rows}, per-expert router bias N(0,1)",
           "rows": rows, "steps": kp, "us_per_layer": round(step_s * 1e6, 2),
           "tokens_per_s": round(aggregate(kp * rows, dist.world, s), 1),
           "tflops": round(tflops, 1), "fp8_peak_tflops": round(fp8_peak, 1),
           "frac_of_fp8_peak": round(tflops / dist.world / fp8_peak, 4), "dtype": GROUPED_DTYPE,
           "hbm_gb_s": round(aggregate(kp * prefill_bytes(d, rows, n_active), dist.world, s) / 1e9, 1),
           "flops_per_step": int(fl["total"]), "distinct_experts": n_active,
           "max_expert_rows": int(max(counts)), "mean_expert_rows": round(sum(counts) / len(counts), 1),
           "peak_source": f"{peak_kind} bf16 GEMM {bf16_peak} TFLOP/s (burst) x 2 (nominal fp8:bf16 ratio)",
           "clocks": clocks,
           "gpu_launches": int(pb.moe.kernel_launches(d, rows, pb.moe.MOE_PATH_PREFILL) * kp)}
    if not args.no_extras:
        per = pb.per_kernel_us(min(kp, 24), PREFILL_KERNELS, batch=8)
        res["per_kernel_us"] = {k: round(v, 2) for k, v in per.items()}
        dom = max(("gemm_gate_up", "gemm_down"), key=lambda k: per[k])
        ach = fl[dom] / (per[dom] * 1e-6) / 1e12
        exe = ex[dom] / (per[dom] * 1e-6) / 1e12
        res["roofline"] = {"kernel": dom, "bound": "tensor", "achieved": round(ach, 1), "peak": round(fp8_peak, 1),
                           "unit": "TFLOP/s", "frac": round(ach / fp8_peak, 4),
                           "traffic": profiled_traffic(dom, "qwen36_35b_prefill_rows4096"),
                           "algorithmic_flops_per_launch": int(fl[dom]),
                           "executed_tflops": round(exe, 1), "executed_frac": round(exe / fp8_peak, 4),
                           "note": "achieved counts the layer's own FLOPs; executed counts the MMAs issued "
                                   "(128-row tile padding, and two e4m3 terms per activation)"}
    del pb
    return res


def e2e_measure(dims, insts, rows: int, steps: int, dist: Dist, seed: int):
    """The same metric through the public call with host buffers
    (moe_ffn_forward_host): every step reads its x from pinned host memory and
    writes its output to pinned host memory, inside the timed region."""
    import torch

    import moe_inputs as mi
    import sparse_moe_ffn_topk_b200 as moe
    nx = 64
    xs_host = [torch.from_numpy(mi.make_x(dims, rows, seed=seed + 7, stream=i).view("int16")).view(torch.bfloat16)
               .pin_memory() for i in range(nx)]
    outs_host = [torch.empty(rows, dims.hidden, dtype=torch.bfloat16).pin_memory() for _ in range(nx)]
    ws = moe.alloc_workspace(dims, rows)
    s = torch.cuda.Stream()

    def one(i):
        w = insts[i % len(insts)]
        moe.ffn_forward_host(dims, xs_host[i % nx], w["router_w"], w["expert_w8"], w["expert_scales"],
                             w["shared_w8"], w["shared_scales"], w["shared_gate"], outs_host[i % nx], ws, stream=s)

    with torch.cuda.stream(s):
        for i in range(5):
            one(i)  # eager: sets up kernel attributes
    torch.cuda.synchronize()
    # The steps are replayed from CUDA graphs (as a serving loop would run
    # them); every step in a graph still reads its x from pinned host memory
    # and writes its output to pinned host memory.
    chunk = 250
    graphs = []
    for first in range(0, steps, chunk):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for j in range(first, min(steps, first + chunk)):
                one(j)
        graphs.append(g)
    for g in graphs:
        g.replay()  # the first replay also uploads the graph (untimed)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        e0.record(s)
        for g in graphs:
            g.replay()
        e1.record(s)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    dist.barrier()
    del graphs
    return ms, 2 * rows * dims.hidden, 2 * rows * dims.hidden


def cpu_model() -> str:
    """The host CPU's model name (/proc/cpuinfo), or the platform string."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or platform.machine()


def cpu_oracle_leg(dims, layer, rows: int, seed: int, budget_s: float = 12.0, max_steps: int = 40):
    """The CPU oracle, as it stands, on a bounded sample of the workload:
    consecutive rows=`rows` layer steps on fresh x until the time budget."""
    import moe_inputs as mi
    import oracle
    steps, t_total, used = 0, 0.0, 1
    n_active = []
    while steps < max_steps and t_total < budget_s:
        x = mi.make_x(dims, rows, seed=seed + 11, stream=steps)
        t = time.perf_counter()
        r = oracle.moe_forward(dims, x, layer.router_w, layer.expert_w8, layer.expert_scales, layer.shared_w8,
                               layer.shared_scales, layer.shared_gate, want_logits=False, nthreads=os.cpu_count())
        t_total += time.perf_counter() - t
        used = max(used, min(rows, os.cpu_count() or 1))
        n_active.append(len(set(r.idx.ravel().tolist())))
        steps += 1
    return steps, t_total, used, n_active


def run_ours(args, dist: Dist):
    import numpy as np
    import torch

    import moe_inputs as mi
    import sparse_moe_ffn_topk_b200 as moe

    torch.cuda.set_device(dist.local)
    d = mi.QWEN36_35B_A3B
    hbm_peak, bf16_peak, peak_kind = peaks()
    t0 = time.time()
    layer = mi.make_layer(d, seed=args.seed)
    gen_s = time.time() - t0
    insts = make_instances(layer, N_INSTANCES)
    props = torch.cuda.get_device_properties(dist.local)
    bus = None
    try:
        bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
    except Exception:
        pass
    names = ["decode_step"]

    def x_set(rows, n):
        return [torch.from_numpy(mi.make_x(d, rows, seed=args.seed + 1, stream=1000 * rows + i).view("int16"))
                .view(torch.bfloat16).cuda() for i in range(n)]

    # ---- headline: rows = 1
    rows = 1
    b1 = DecodeBench(d, insts, x_set(rows, 64), rows)
    u1 = b1.routing(64)
    U1 = statistics.mean(u1)
    by1 = algorithmic_bytes(d, rows, U1)
    sampler = ClockSampler(bus)
    sampler.start()
    ms, _ = b1.time_steps(args.steps, args.warmup, dist, sampler)
    clocks = sampler.stop()
    max_s = dist.max(ms / 1000.0)
    us_layer = max_s * 1e6 / args.steps
    value = aggregate(args.steps * by1["total"], dist.world, max_s) / 1e9
    print(f"[bench] rows=1: {us_layer:.2f} us/layer, {value:.1f} GB/s, U={U1:.2f}", file=sys.stderr, flush=True)
    launches = moe.kernel_launches(d, rows)

    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(max_s * 1000.0 / args.steps, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": DECODE_DTYPE, "data": "synthetic (seeded)",
        "config": {"workload": WORKLOAD, "hidden": d.hidden, "experts": d.n_experts, "top_k": d.top_k,
                   "inter": d.inter, "shared_inter": d.shared_inter, "rows": rows,
                   "l2": f"inputs larger than L2: {N_INSTANCES} rotating weight instances "
                         f"({N_INSTANCES * (d.n_experts * d.expert_bytes) / 1e9:.1f} GB)",
                   "parallelism": f"replicas x{dist.world}" if dist.world > 1 else "single GPU",
                   "timing": "CUDA events on the launching stream around CUDA-graph replays of exactly K steps; "
                             "W warm-up steps, and each timed graph replayed once untimed before (graph upload)"},
        "us_per_layer": round(us_layer, 3),
        "tokens_per_s": round(aggregate(args.steps * rows, dist.world, max_s), 1),
        "hbm_frac_of_measured": round(value / dist.world / hbm_peak, 4),
        "expert_bytes_gbs": round(aggregate(args.steps * by1["experts"], dist.world, max_s) / 1e9, 2),
        "bytes_per_step": int(by1["total"]), "distinct_experts_per_step": round(U1, 2),
        "gpu_launches": int(launches * args.steps),
        "clocks": clocks,
        "peak_source": f"{peak_kind} ({hbm_peak} GB/s copy)",
        "weights_generation_s": round(gen_s, 1),
    }

    # ---- roofline of the dominant kernel (per-kernel events, PDL off)
    if not args.no_extras:
        kp = b1.per_kernel_us(min(args.steps, 256), names)
        dom = max(kp, key=lambda k: kp[k])
        ach = by1[dom] / (kp[dom] * 1e-6) / 1e9
        result["per_kernel_us"] = {k: round(v, 3) for k, v in kp.items()}
        result["roofline"] = {"kernel": dom, "bound": "hbm", "achieved": round(ach, 1), "peak": hbm_peak,
                              "unit": "GB/s", "frac": round(ach / hbm_peak, 4),
                              "traffic": profiled_traffic(dom, "qwen36_35b_decode_rows1"),
                              "algorithmic_bytes_per_launch": int(by1[dom]),
                              "note": "per-kernel CUDA events with programmatic dependent launch off; "
                                      f"peak = {peak_kind} HBM copy bandwidth"}

        # ---- rows = 64
        r64 = 64
        b64 = DecodeBench(d, insts, x_set(r64, 16), r64)
        u64 = statistics.mean(b64.routing(16))
        by64 = algorithmic_bytes(d, r64, u64)
        k64 = max(20, args.steps // 20)
        ms64, _ = b64.time_steps(k64, min(args.warmup, 5), dist)
        s64 = dist.max(ms64 / 1000.0)
        gbs64 = aggregate(k64 * by64["total"], dist.world, s64) / 1e9
        result["rows64"] = {"us_per_layer": round(s64 * 1e6 / k64, 3), "gb_s": round(gbs64, 1),
                            "hbm_frac_of_measured": round(gbs64 / dist.world / hbm_peak, 4),
                            "tokens_per_s": round(aggregate(k64 * r64, dist.world, s64), 1),
                            "distinct_experts_per_step": round(u64, 1), "steps": k64,
                            "dtype": GROUPED_DTYPE if moe.auto_path(d, r64) != moe.MOE_PATH_DECODE else DECODE_DTYPE,
                            "kernels": {moe.MOE_PATH_DECODE: "decode", moe.MOE_PATH_PREFILL: "grouped",
                                        moe.MOE_PATH_PREFILL_NARROW: "narrow"}[moe.auto_path(d, r64)]}

    # ---- a chain of layers behind their norms (rows = 1): one launch per layer
    if not args.no_extras:
        g = torch.Generator().manual_seed(args.seed + 7)
        nws = [(1.0 + 0.1 * torch.randn(d.hidden, generator=g)).to(torch.bfloat16).cuda()
               for _ in range(N_INSTANCES)]
        r0 = torch.from_numpy(mi.make_residual(d, rows, seed=args.seed, stream=77).view("int16")).view(
            torch.bfloat16).cuda()
        cb = ChainBench(d, insts, nws, r0, rows)
        kc = args.steps
        msc, _ = cb.time_steps(kc, args.warmup, dist)
        sc = dist.max(msc / 1000.0)
        result["chain"] = {"layers": N_INSTANCES, "steps": kc, "us_per_layer": round(sc * 1e6 / kc, 3),
                           "gb_s": round(aggregate(kc * by1["total"], dist.world, sc) / 1e9, 1),
                           "hbm_frac_of_measured": round(aggregate(kc * by1["total"], dist.world, sc) / 1e9
                                                         / dist.world / hbm_peak, 4),
                           "what": "each step: r <- r + layer_l(bf16(rmsnorm(r) * w_l)) in place, l = step mod "
                                   f"{N_INSTANCES}; the norm runs inside the decode-step kernel"}
        del cb

    # ---- NVFP4 experts (the 397B-A17B checkpoint's format), decode rows = 1
    if not args.no_extras:
        d4 = mi.QWEN35_397B_A17B
        ninst = 4  # 4 x 3.7 GB of expert weights: larger than L2
        i4 = nvfp4_instances(d4, ninst, args.seed + 11)
        x4 = [torch.from_numpy(mi.make_x(d4, 1, seed=args.seed + 1, stream=4000 + i).view("int16"))
              .view(torch.bfloat16).cuda() for i in range(64)]
        nb = Nvfp4Bench(d4, i4, x4, 1)
        with torch.cuda.stream(nb.stream):
            u4 = []
            for i in range(16):  # distinct experts a step reads (routing via the same router kernel)
                idx = torch.empty(1, d4.top_k, dtype=torch.int32, device="cuda")
                tw = torch.empty(1, d4.top_k, dtype=torch.float32, device="cuda")
                tg = torch.empty(1, dtype=torch.float32, device="cuda")
                w = i4[i % ninst]
                moe.router_topk(d4, x4[i], w["router_w"], w["shared_gate"], idx, tw, tg, nb.ws, stream=nb.stream)
                u4.append(int(torch.unique(idx).numel()))
        k4 = args.steps
        ms4, _ = nb.time_steps(k4, args.warmup, dist)
        s4 = dist.max(ms4 / 1000.0)
        b4 = nvfp4_bytes(d4, 1, statistics.mean(u4))
        g4 = aggregate(k4 * b4, dist.world, s4) / 1e9
        result["nvfp4"] = {"workload": "Qwen3.5-397B-A17B-shaped MoE FFN layer with NVFP4 experts, decode rows=1",
                           "us_per_layer": round(s4 * 1e6 / k4, 3), "gb_s": round(g4, 1),
                           "hbm_frac_of_measured": round(g4 / dist.world / hbm_peak, 4),
                           "bytes_per_step": int(b4), "distinct_experts_per_step": round(statistics.mean(u4), 2),
                           "steps": k4, "kernels": ["router_topk", "nvfp4_gate_up", "nvfp4_down_blend"],
                           "dtype": "e2m1 weights (e4m3 scale per 16, fp32 per matrix) x bf16 x for gate/up and x "
                                    "fp32 h for down, exact products, fp32 accumulate (CUDA cores)",
                           "l2": f"{ninst} weight copies ({ninst * 3.7:.1f} GB of expert codes)"}
        print(f"[bench] nvfp4 397B rows=1: {s4 * 1e6 / k4:.2f} us/layer, {g4:.1f} GB/s", file=sys.stderr, flush=True)
        del nb, i4

    # ---- prefill, 4096 tokens
    result["prefill"] = prefill_leg(args, d, insts[0], dist, bus, hbm_peak, bf16_peak, peak_kind)
    p = result["prefill"]
    print(f"[bench] prefill: {p['us_per_layer']:.1f} us/layer, {p['tflops']:.1f} TFLOP/s "
          f"({100 * p['frac_of_fp8_peak']:.1f}% of fp8 peak)", file=sys.stderr, flush=True)

    # ---- end to end through the public call with host buffers
    ke = min(args.steps, 1000)
    ems, h2d, d2h = e2e_measure(d, insts, rows, ke, dist, args.seed)
    es = dist.max(ems / 1000.0)
    result["e2e"] = {"value": round(aggregate(ke * by1["total"], dist.world, es) / 1e9, 2), "unit": "GB/s",
                     "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                     "us_per_layer": round(es * 1e6 / ke, 3), "steps": ke,
                     "timing": "CUDA-graph replays of the public host-buffer call (moe_ffn_forward_host); each "
                               "step reads x from pinned host memory and writes out to pinned host memory "
                               "inside the timed region (no copy-engine transfers)"}

    # ---- the CPU oracle on this host (rank 0, N = 1 only)
    if dist.world == 1:
        steps, secs, cores, na = cpu_oracle_leg(d, layer, rows, args.seed)
        byc = algorithmic_bytes(d, rows, statistics.mean(na))
        result["cpu_baseline"] = {"value": round(steps * byc["total"] / secs / 1e9, 4), "unit": "GB/s",
                                  "cores": cores, "kind": "oracle", "cpu_model": cpu_model(),
                                  "host_threads": os.cpu_count(),
                                  "sample": f"{steps} layer steps at rows={rows} (fresh x each), "
                                            f"{secs:.1f} s, {secs / steps * 1e3:.1f} ms/layer"}
        if not args.no_extras:
            # the oracle threaded over rows, at 64 rows
            s64n, s64t, c64, na64 = cpu_oracle_leg(d, layer, 64, args.seed, budget_s=10.0, max_steps=4)
            by64c = algorithmic_bytes(d, 64, statistics.mean(na64))
            result["cpu_baseline"]["rows64"] = {
                "value": round(s64n * by64c["total"] / s64t / 1e9, 4), "unit": "GB/s", "threads": c64,
                "ms_per_layer": round(s64t / s64n * 1e3, 1),
                "tokens_per_s": round(s64n * 64 / s64t, 1),
                "sample": f"{s64n} layer steps at rows=64 (fresh x each), {s64t:.1f} s"}
    del b1
    return result


def run_reference(args, dist: Dist):
    """The CPU oracle as the reference arm, on rank 0 only."""
    import moe_inputs as mi
    if dist.rank != 0:
        return None
    d = mi.QWEN36_35B_A3B
    rows = 1
    # a bounded sample: only the experts the sampled steps route to are drawn
    import oracle
    rw, g, _ = mi.make_router(d, args.seed)
    K = max(1, args.steps)
    n = min(K, 30)
    xs = [mi.make_x(d, rows, seed=args.seed + 11, stream=i) for i in range(n)]
    need = set()
    for x in xs:
        _, idx, _, _ = oracle.router_topk(d, x, rw, g)
        need |= set(idx.ravel().tolist())
    layer = mi.make_layer(d, seed=args.seed, experts=need)
    for i in range(min(args.warmup, 1)):
        oracle.moe_forward(d, xs[0], layer.router_w, layer.expert_w8, layer.expert_scales, layer.shared_w8,
                           layer.shared_scales, layer.shared_gate, want_logits=False)
    t = time.perf_counter()
    na = []
    for x in xs:
        r = oracle.moe_forward(d, x, layer.router_w, layer.expert_w8, layer.expert_scales, layer.shared_w8,
                               layer.shared_scales, layer.shared_gate, want_logits=False)
        na.append(len(set(r.idx.ravel().tolist())))
    secs = time.perf_counter() - t
    by = algorithmic_bytes(d, rows, statistics.mean(na))
    value = n * by["total"] / secs / 1e9
    sample = f"{n} layer steps at rows={rows} (fresh x each), {secs:.1f} s, {secs / n * 1e3:.1f} ms/layer"
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": dist.world,
        "steps": n, "warmup": min(args.warmup, 1), "ms_per_step": round(secs * 1000.0 / n, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": WORKLOAD, "hidden": d.hidden, "experts": d.n_experts, "top_k": d.top_k,
                   "inter": d.inter, "shared_inter": d.shared_inter, "rows": rows,
                   "parallelism": "host CPU (oracle)"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def run_sweep(args, dist: Dist):
    """Every row count of the decode workloads (35B-A3B-shaped rows 1, 2, 8,
    16, 32, 64, with 4 and 128 to 1024 beside them; 397B-A17B-shaped rows 1
    and 32, with 4 and 256)
    on each path that takes it: the decode kernels (up to 64 rows), the
    grouped GEMMs with 128-row token tiles, and the narrow grouped GEMMs;
    each line says whether it is the path MOE_PATH_AUTO takes.  CUDA events
    over CUDA-graph replays, 16 rotating weight copies (35B) or two (397B)."""
    import torch

    import moe_inputs as mi
    import sparse_moe_ffn_topk_b200 as moe
    torch.cuda.set_device(dist.local)
    hbm_peak, _, peak_kind = peaks()
    names = {moe.MOE_PATH_DECODE: "decode", moe.MOE_PATH_PREFILL: "grouped", moe.MOE_PATH_PREFILL_NARROW: "narrow"}
    res = []
    for dims, name, rows_list, n_inst in ((mi.QWEN36_35B_A3B, "Qwen3.6-35B-A3B-shaped",
                                           [1, 2, 4, 8, 16, 32, 64, 128, 256, 512, 1024], 16),
                                          (mi.QWEN35_397B_A17B, "Qwen3.5-397B-A17B-shaped", [1, 4, 32, 256], 2)):
        insts = make_instances(mi.make_layer(dims, seed=args.seed), n_inst)
        for rows in rows_list:
            xs = [torch.from_numpy(mi.make_x(dims, rows, seed=args.seed + 1, stream=1000 * rows + i).view("int16"))
                  .view(torch.bfloat16).cuda() for i in range(16)]
            auto = moe.auto_path(dims, rows)
            paths = [moe.MOE_PATH_PREFILL, moe.MOE_PATH_PREFILL_NARROW]
            if rows <= 64:
                paths.insert(0, moe.MOE_PATH_DECODE)
            for pcode in paths:
                b = DecodeBench(dims, insts, xs, rows, path=pcode)
                u = statistics.mean(b.routing(16))
                by = algorithmic_bytes(dims, rows, u)
                k = max(50, min(args.steps, 4000 // rows))
                ms, _ = b.time_steps(k, max(3, args.warmup), dist)
                sec = dist.max(ms / 1000.0)
                gbs = aggregate(k * by["total"], dist.world, sec) / 1e9
                res.append({"workload": f"{name} rows={rows}", "path": names[pcode], "auto": pcode == auto,
                            "us_per_layer": round(sec * 1e6 / k, 3),
                            "gb_s": round(gbs, 1), "hbm_frac_of_measured": round(gbs / dist.world / hbm_peak, 4),
                            "tokens_per_s": round(aggregate(k * rows, dist.world, sec), 1),
                            "distinct_experts": round(u, 1), "bytes_per_step": int(by["total"]), "steps": k})
                print(f"[sweep] {res[-1]['workload']} {names[pcode]}{' (auto)' if pcode == auto else ''}: "
                      f"{res[-1]['us_per_layer']} us, {gbs:.0f} GB/s", file=sys.stderr, flush=True)
                del b
        del insts
        torch.cuda.empty_cache()
    return {"sweep": res, "peak_source": f"{peak_kind} ({hbm_peak} GB/s copy)", "n_gpus": dist.world}


def run_profile_case(args):
    """A few eager calls of one workload (35B-shaped layer, one weight copy):
    decode at rows = 1 on fresh x each call, the 4096-token biased prefill, or
    the narrow grouped GEMMs at --rows rows; or the 397B-shaped layer with
    NVFP4 experts at rows = 1.  Small enough for a profiler to replay every
    kernel."""
    import torch

    import moe_inputs as mi
    import sparse_moe_ffn_topk_b200 as moe
    if args.profile == "nvfp4":
        # the 397B-A17B-shaped layer with NVFP4 experts, one weight copy (3.7 GB) drawn on the GPU
        d4 = mi.QWEN35_397B_A17B
        w = nvfp4_instances(d4, 1, args.seed + 11)[0]
        ws = moe.alloc_workspace(d4, 1)
        out = torch.empty(1, d4.hidden, dtype=torch.bfloat16, device="cuda")
        for i in range(args.calls):
            x = torch.from_numpy(mi.make_x(d4, 1, seed=args.seed + 5, stream=i).view("int16")).view(torch.bfloat16).cuda()
            moe.ffn_forward_nvfp4(d4, x, w["router_w"], w["w4"], w["sf"], w["gs"], w["sw4"], w["ssf"], w["sgs"],
                                  w["shared_gate"], out, ws)
        torch.cuda.synchronize()
        st = moe.device_status(ws)
        print(json.dumps({"profile": args.profile, "calls": args.calls, "rows": 1, "device_status": st}), flush=True)
        return 0 if st == moe.MOE_OK else 1
    d = mi.QWEN36_35B_A3B
    inst = make_instances(mi.make_layer(d, seed=args.seed), 1)[0]
    if args.profile == "decode":
        rows, bias, path = 1, None, moe.MOE_PATH_AUTO
    elif args.profile == "narrow":
        rows, bias, path = args.rows, None, moe.MOE_PATH_PREFILL_NARROW
    else:
        rows, path = 4096, moe.MOE_PATH_PREFILL
        bias = torch.from_numpy(mi.make_router(d, args.seed, True)[2]).cuda()
    ws = moe.alloc_workspace(d, rows)
    out = torch.empty(rows, d.hidden, dtype=torch.bfloat16, device="cuda")
    for i in range(args.calls):
        x = torch.from_numpy(mi.make_x(d, rows, seed=args.seed + 5, stream=i).view("int16")).view(torch.bfloat16).cuda()
        moe.ffn_forward_path(d, x, inst["router_w"], inst["expert_w8"], inst["expert_scales"], inst["shared_w8"],
                             inst["shared_scales"], inst["shared_gate"], out, ws, path=path, router_bias=bias)
    torch.cuda.synchronize()
    st = moe.device_status(ws)
    print(json.dumps({"profile": args.profile, "calls": args.calls, "rows": rows, "device_status": st}), flush=True)
    return 0 if st == moe.MOE_OK else 1


def main(argv=None):
    args = parse_args(argv)
    if args.profile:
        return run_profile_case(args)
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return 0
        res = run_reference(args, Dist.__new__(Dist) if False else _NoDist(world, rank))
        print(json.dumps(res), flush=True)
        return 0
    dist = Dist(args.gpus)
    try:
        res = run_sweep(args, dist) if args.sweep else run_ours(args, dist)
        if dist.rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        dist.close()
    return 0


class _NoDist:
    def __init__(self, world, rank):
        self.world, self.rank, self.local = world, rank, 0


if __name__ == "__main__":
    sys.exit(main())
