"""Phase times of the decode step kernel, from its ``%globaltimer`` trace build.

    python -m sparse_moe_ffn_topk_b200.build --trace
    python -m sparse_moe_ffn_topk_b200.phase_trace [--rows N]

Runs the Qwen3.6-35B-A3B-shaped layer (16 weight copies, larger than L2) as a
CUDA graph of 16 decode steps a few times, then prints, for the last step of
the last replay, each phase point's time after the first CTA started (min,
median and max over the CTAs) and the down items' points, as a markdown
table.  The trace build records one timestamp per (CTA, point) from one
thread; it is the library's own kernel with those stores added, so its times
run a little above the plain build's.
"""
from __future__ import annotations

import argparse
import ctypes
import os
import sys

import numpy as np

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)

# step points (thread 0 of each CTA unless noted)
POINTS = [
    (0, "kernel start"),
    (1, "PDL wait passed"),
    (2, "x staged"),
    (3, "router rows done (this CTA's logits published)"),
    (12, "top-k started"),
    (13, "top-k done"),
    (14, "distinct-expert list done"),
    (5, "plan done"),
    (15, "this CTA's last gate/up unit counted (epilogue thread)"),
    (7, "gate/up done (warp 0)"),
    (8, "P3 entered (warp 0)"),
    (10, "down items done (all warps)"),
    (11, "output written"),
]


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--rows", type=int, default=1)
    ap.add_argument("--replays", type=int, default=4)
    args = ap.parse_args(argv)

    import torch

    sys.path.insert(0, ROOT)
    import moe_inputs as mi

    import sparse_moe_ffn_topk_b200 as moe
    from sparse_moe_ffn_topk_b200 import build

    if not os.path.exists(build.TRACE_LIB):
        raise SystemExit(f"{build.TRACE_LIB} is missing: python -m sparse_moe_ffn_topk_b200.build --trace")
    moe._lib = None
    moe.LIB_PATH = build.TRACE_LIB
    L = moe.lib()
    L.moe_debug_step_trace.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    L.moe_debug_item_trace.argtypes = [ctypes.c_void_p, ctypes.c_void_p]

    d = mi.QWEN36_35B_A3B
    layer = mi.make_layer(d, seed=0)
    base = {"router_w": torch.from_numpy(layer.router_w.view("int16")).view(torch.bfloat16).cuda(),
            "shared_gate": torch.from_numpy(layer.shared_gate.view("int16")).view(torch.bfloat16).cuda(),
            "expert_w8": torch.from_numpy(layer.expert_w8).cuda(),
            "expert_scales": torch.from_numpy(layer.expert_scales).cuda(),
            "shared_w8": torch.from_numpy(layer.shared_w8).cuda(),
            "shared_scales": torch.from_numpy(layer.shared_scales).cuda()}
    insts = [base] + [{k: v.clone() for k, v in base.items()} for _ in range(15)]
    xs = [torch.from_numpy(mi.make_x(d, args.rows, seed=1, stream=1000 * args.rows + i).view("int16"))
          .view(torch.bfloat16).cuda() for i in range(16)]
    out = torch.empty(args.rows, d.hidden, dtype=torch.bfloat16, device="cuda")
    ws = moe.alloc_workspace(d, args.rows)
    st = torch.cuda.Stream()

    def call(i):
        w = insts[i % 16]
        moe.ffn_forward_path(d, xs[i % 16], w["router_w"], w["expert_w8"], w["expert_scales"], w["shared_w8"],
                             w["shared_scales"], w["shared_gate"], out, ws, path=moe.MOE_PATH_DECODE, stream=st)

    with torch.cuda.stream(st):
        for i in range(20):
            call(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        for i in range(16):
            call(i)
    with torch.cuda.stream(st):
        for _ in range(args.replays):
            g.replay()
    torch.cuda.synchronize()
    if moe.device_status(ws) != moe.MOE_OK:
        raise SystemExit("a bounded wait ran out")

    ctas = torch.cuda.get_device_properties(0).multi_processor_count
    tb = np.zeros(256 * 16, dtype=np.uint64)
    ib = np.zeros(256 * 64 * 6, dtype=np.uint64)
    if L.moe_debug_step_trace(tb.ctypes.data, ctypes.c_void_p(st.cuda_stream)) != 0:
        raise SystemExit("reading the trace failed")
    if L.moe_debug_item_trace(ib.ctypes.data, ctypes.c_void_p(st.cuda_stream)) != 0:
        raise SystemExit("reading the trace failed")
    t = tb.reshape(256, 16)[:ctas].astype(np.int64)
    it = ib.reshape(256, 64, 6)[:ctas].astype(np.int64)
    t0 = t[:, 0][t[:, 0] > 0].min()

    def row(name, v):
        v = (v[v > 0] - t0) / 1000.0
        return f"| {name} | {v.min():.2f} | {np.median(v):.2f} | {v.max():.2f} |" if len(v) else f"| {name} | - | - | - |"

    print(f"Decode step, Qwen3.6-35B-A3B-shaped layer, rows = {args.rows}: the last step of a 16-step graph "
          f"(replay {args.replays}), microseconds after the first CTA started, over {ctas} CTAs.\n")
    print("| point | min | median | max |")
    print("|---|---|---|---|")
    for i, name in POINTS:
        print(row(name, t[:, i]))
    # down items (trace rows 48-63 in claim order): expert seen counted, weight rows seen, done
    dn = it[:, 48:64, :3]
    n = (dn[:, :, 2] > 0).sum(axis=1)
    first = dn[:, 0, :]
    last = np.array([dn[c, n[c] - 1, :] if n[c] else np.zeros(3, np.int64) for c in range(ctas)])
    print(row("first down item: its expert seen counted", first[:, 0]))
    print(row("first down item: its weight rows seen", first[:, 1]))
    print(row("first down item: done", first[:, 2]))
    print(row("last down item: its expert seen counted", last[:, 0]))
    print(row("last down item: done", last[:, 2]))
    return 0


if __name__ == "__main__":
    sys.exit(main())
